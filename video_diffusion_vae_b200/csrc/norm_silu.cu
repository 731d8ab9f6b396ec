// Standalone channel RMS-norm + affine + SiLU over channels-last activations.
//
//   y[v, c] = SiLU( x[v, c] / max(||x[v, :]||_2, eps) * sqrt(C) * gamma[c] + beta[c] )
//
// (TensorRT-LLM issue #19309 "Opt-in BF16 norm-SiLU fusion for Wan VAE
// decoding", section "Feature, motivation and proposed scope": the decoder's
// norm1/norm2/norm_out are channel normalisation + affine + SiLU, fused here
// into one pass; FastVideo Wan2.2 VAE decoder README, "Limits": fp32 norm
// statistics.)
//
// HBM-bound: one read and one write of the tensor.  A group of L lanes owns a
// voxel (L = 32 for C >= 256); each lane moves 16-byte vectors (8 bf16 / 4 fp32
// channels), so a warp's accesses to a voxel are one contiguous, fully
// coalesced run.  The sum of squares is reduced with shuffles inside the
// group.  Each lane keeps its channels' gamma/beta in registers for the whole
// grid-stride loop; two voxel groups are in flight per iteration.
#include "internal.h"
#include "ptx.cuh"

namespace wvae {

namespace {

constexpr int kNormThreads = 256;

__device__ __forceinline__ float silu_fast(float s) { return s * __frcp_rn(1.0f + __expf(-s)); }
__device__ __forceinline__ float silu_exact(float s) { return s / (1.0f + expf(-s)); }

// VEC = channels per 16-byte vector (8 for bf16, 4 for fp32); CH = vectors per lane.
template <typename T, int VEC, int CH, int UNROLL>
__global__ void __launch_bounds__(kNormThreads) norm_silu_kernel(const T* __restrict__ x, T* y,
                                                                 const float* __restrict__ gamma,
                                                                 const float* __restrict__ beta,
                                                                 long nvox, int C, int L,
                                                                 float eps) {
  const int lane = threadIdx.x & 31;
  const int sub = lane % L;                    // lane inside its voxel group
  const int groups_per_warp = 32 / L;
  const int nvec = C / VEC;                    // vectors per voxel
  const long warp_global = (static_cast<long>(blockIdx.x) * kNormThreads + threadIdx.x) >> 5;
  const long nwarps = (static_cast<long>(gridDim.x) * kNormThreads) >> 5;
  const float rootC = sqrtf(static_cast<float>(C));

  float g[CH][VEC], b[CH][VEC];
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int vi = sub + k * L;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const int c = vi * VEC + e;
      g[k][e] = (vi < nvec) ? gamma[c] : 0.0f;
      b[k][e] = (vi < nvec) ? beta[c] : 0.0f;
    }
  }

  // The loop bound is uniform across the warp (shuffles below need all lanes).
  const long step = nwarps * groups_per_warp;
  for (long wbase = warp_global * groups_per_warp; wbase < nvox; wbase += step * UNROLL) {
    const long base = wbase + lane / L;
    float v[UNROLL][CH][VEC];
    float ss[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const long vox = base + u * step;
      ss[u] = 0.0f;
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int vi = sub + k * L;
        if (vox < nvox && vi < nvec) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x + vox * C) + vi);
          if constexpr (VEC == 8) {
            v[u][k][0] = bf16lo(raw.x); v[u][k][1] = bf16hi(raw.x);
            v[u][k][2] = bf16lo(raw.y); v[u][k][3] = bf16hi(raw.y);
            v[u][k][4] = bf16lo(raw.z); v[u][k][5] = bf16hi(raw.z);
            v[u][k][6] = bf16lo(raw.w); v[u][k][7] = bf16hi(raw.w);
          } else {
            v[u][k][0] = __uint_as_float(raw.x); v[u][k][1] = __uint_as_float(raw.y);
            v[u][k][2] = __uint_as_float(raw.z); v[u][k][3] = __uint_as_float(raw.w);
          }
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) v[u][k][e] = 0.0f;
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) ss[u] = fmaf(v[u][k][e], v[u][k][e], ss[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      for (int off = L >> 1; off > 0; off >>= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const long vox = base + u * step;
      if (vox >= nvox) continue;
      const float r = rootC / fmaxf(sqrtf(ss[u]), eps);
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int vi = sub + k * L;
        if (vi >= nvec) continue;
        float o[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float s = v[u][k][e] * r * g[k][e] + b[k][e];
          o[e] = (VEC == 8) ? silu_fast(s) : silu_exact(s);
        }
        uint4 w;
        if constexpr (VEC == 8) {
          w.x = pack_bf16x2(o[0], o[1]); w.y = pack_bf16x2(o[2], o[3]);
          w.z = pack_bf16x2(o[4], o[5]); w.w = pack_bf16x2(o[6], o[7]);
        } else {
          w.x = __float_as_uint(o[0]); w.y = __float_as_uint(o[1]);
          w.z = __float_as_uint(o[2]); w.w = __float_as_uint(o[3]);
        }
        reinterpret_cast<uint4*>(y + vox * C)[vi] = w;
      }
    }
  }
}

template <typename T, int VEC>
cudaError_t launch_impl(const T* x, T* y, const float* gamma, const float* beta, long nvox, int C,
                        float eps, int num_sms, cudaStream_t stream) {
  const int nvec = C / VEC;
  int L = 1;
  while (L < nvec && L < 32) L <<= 1;
  const int ch = (nvec + L - 1) / L;
  const long groups = nvox;
  const long warps_needed = (groups * L + 31) / 32;
  long blocks = (warps_needed + (kNormThreads / 32) - 1) / (kNormThreads / 32);
  const long max_blocks = static_cast<long>(num_sms) * (2048 / kNormThreads);
  if (blocks > max_blocks) blocks = max_blocks;
  if (blocks < 1) blocks = 1;
  const int grid = static_cast<int>(blocks);
  if (ch == 1)
    norm_silu_kernel<T, VEC, 1, 2><<<grid, kNormThreads, 0, stream>>>(x, y, gamma, beta, nvox, C, L, eps);
  else if (ch == 2)
    norm_silu_kernel<T, VEC, 2, 2><<<grid, kNormThreads, 0, stream>>>(x, y, gamma, beta, nvox, C, L, eps);
  else if (ch <= 4)
    norm_silu_kernel<T, VEC, 4, 1><<<grid, kNormThreads, 0, stream>>>(x, y, gamma, beta, nvox, C, L, eps);
  else if (ch <= 8)
    norm_silu_kernel<T, VEC, 8, 1><<<grid, kNormThreads, 0, stream>>>(x, y, gamma, beta, nvox, C, L, eps);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_norm_silu_bf16(const __nv_bfloat16* x, __nv_bfloat16* y, const float* gamma,
                                  const float* beta, long nvox, int C, float eps, int num_sms,
                                  cudaStream_t stream) {
  return launch_impl<__nv_bfloat16, 8>(x, y, gamma, beta, nvox, C, eps, num_sms, stream);
}

cudaError_t launch_norm_silu_f32(const float* x, float* y, const float* gamma, const float* beta,
                                 long nvox, int C, float eps, int num_sms, cudaStream_t stream) {
  return launch_impl<float, 4>(x, y, gamma, beta, nvox, C, eps, num_sms, stream);
}

}  // namespace wvae

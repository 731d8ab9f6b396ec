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
// HBM-bound: one read and one write of the tensor, and the bf16 path also
// close to the SM's issue and SFU limits (about 12 elements per SM clock at
// full HBM rate), so SiLU costs one SFU operation (tanh form) per element.
//
// bf16 (norm_silu_ring_kernel): launched as a programmatic dependent of the
// previous kernel on the stream, so its set-up (barriers, gamma / beta)
// overlaps that kernel's tail and only the data waits for it (about 2.6 us
// of a 24 us launch on 112.5 MB).  One persistent CTA per SM.  Warp 0 streams
// contiguous chunks of whole voxels (about 64 KB: the activation is
// channels-last, so a chunk is one byte range) into a 3-stage ring of
// shared-memory stages with bulk asynchronous copies, keeping ~190 KB per SM in flight
// without holding registers; 16 consumer warps take the voxels of each chunk.
// A group of L lanes owns a voxel (L = 32 for C >= 256) and moves 16-byte
// vectors, so shared-memory reads and global writes of a voxel are contiguous
// runs.  A lane's channels never change: its gamma/beta (pre-halved for the
// tanh form of SiLU) live in registers for the whole kernel.
//
// fp32 (norm_silu_kernel, the reference path): each warp issues the loads of
// U voxel groups into registers, reduces, and writes; exact SiLU.
#include "internal.h"
#include "ptx.cuh"

namespace wvae {

namespace {

constexpr int kNormThreads = 256;

__device__ __forceinline__ float silu_exact(float s) { return s / (1.0f + expf(-s)); }

template <int VEC>
__device__ __forceinline__ void unpack(const uint4& r, float (&v)[VEC]) {
  if constexpr (VEC == 8) {
    v[0] = bf16lo(r.x); v[1] = bf16hi(r.x); v[2] = bf16lo(r.y); v[3] = bf16hi(r.y);
    v[4] = bf16lo(r.z); v[5] = bf16hi(r.z); v[6] = bf16lo(r.w); v[7] = bf16hi(r.w);
  } else {
    v[0] = __uint_as_float(r.x); v[1] = __uint_as_float(r.y);
    v[2] = __uint_as_float(r.z); v[3] = __uint_as_float(r.w);
  }
}

// VEC = channels per 16-byte vector (8 bf16 / 4 fp32); CH = vectors per lane;
// U = voxel groups in flight per warp.
template <typename T, int VEC, int CH, int U>
__global__ void __launch_bounds__(kNormThreads, (VEC == 8 && CH <= 4) ? 3 : 2) norm_silu_kernel(const T* __restrict__ x, T* y,
                                                                 const float* __restrict__ gamma,
                                                                 const float* __restrict__ beta,
                                                                 long nvox, int C, int L,
                                                                 float eps) {
  const int lane = threadIdx.x & 31;
  const int sub = lane % L;
  const int gpw = 32 / L;                      // voxel groups per warp
  const int nvec = C / VEC;
  float g[CH][VEC], b[CH][VEC];
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int vi = sub + k * L;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      g[k][e] = vi < nvec ? __ldg(gamma + vi * VEC + e) : 0.0f;
      b[k][e] = vi < nvec ? __ldg(beta + vi * VEC + e) : 0.0f;
    }
  }
  const long warp_global = (static_cast<long>(blockIdx.x) * kNormThreads + threadIdx.x) >> 5;
  const long nwarps = (static_cast<long>(gridDim.x) * kNormThreads) >> 5;
  const float rootC = sqrtf(static_cast<float>(C));
  const long step = nwarps * gpw;

  // The loop bound is uniform across the warp (the shuffles need all lanes).
  for (long wbase = warp_global * gpw; wbase < nvox; wbase += step * U) {
    const long base = wbase + lane / L;
    uint4 raw[U][CH];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long vox = base + u * step;
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int vi = sub + k * L;
        raw[u][k] = (vox < nvox && vi < nvec)
                        ? __ldcs(reinterpret_cast<const uint4*>(x + vox * C) + vi)
                        : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    float ss[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      ss[u] = 0.0f;
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        float v[VEC];
        unpack<VEC>(raw[u][k], v);
#pragma unroll
        for (int e = 0; e < VEC; ++e) ss[u] = fmaf(v[e], v[e], ss[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      for (int off = L >> 1; off > 0; off >>= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long vox = base + u * step;
      const float r = rootC / fmaxf(sqrtf(ss[u]), eps);
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int vi = sub + k * L;
        if (vox >= nvox || vi >= nvec) continue;
        float v[VEC], o[VEC];
        unpack<VEC>(raw[u][k], v);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float s = v[e] * r * g[k][e] + b[k][e];
          o[e] = silu_exact(s);
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

// ------------------------------------------------------- bf16: TMA-fed ring
constexpr int kRingStages = 3;
constexpr int kRingChunkBytes = 65536;

// CH: 16-byte vectors per lane; V: voxels a lane group carries through one
// pass (their load, reduction and output chains interleave, hiding the
// latency of each); NW: consumer warps.
template <int CH, int V, int NW>
__global__ void __launch_bounds__(32 * (NW + 1), 1)
    norm_silu_ring_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* y,
                          const float* __restrict__ gamma, const float* __restrict__ beta,
                          long nvox, int C, int L, int vpc, float eps, unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const uint32_t chunk_bytes = static_cast<uint32_t>(vpc) * C * 2;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + kRingStages * chunk_bytes);
  uint64_t* empty = full + kRingStages;
  int* abort_flag = reinterpret_cast<int*>(empty + kRingStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRingStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), NW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const long nchunks = (nvox + vpc - 1) / vpc;
  // Launched as a programmatic dependent of the previous kernel on the stream:
  // the set-up above overlaps its tail; nothing reads x or writes y before
  // that kernel has completed and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" :::);

  if (warp == 0) {
    if (lane != 0) return;
    uint32_t it = 0;
    for (long ch = blockIdx.x; ch < nchunks; ch += gridDim.x, ++it) {
      const uint32_t st = it % kRingStages, ph = (it / kRingStages) & 1u;
      if (!mbar_wait_bounded(smem_u32(&empty[st]), ph ^ 1u, abort_flag, err,
                             DEVERR_TIMEOUT_PRODUCER))
        break;
      const long v0 = ch * vpc;
      const long nv = nvox - v0 < vpc ? nvox - v0 : vpc;
      const uint32_t bytes = static_cast<uint32_t>(nv) * C * 2;
      mbar_arrive_expect_tx(smem_u32(&full[st]), bytes);
      bulk_load(smem_u32(smem_raw + st * chunk_bytes), x + v0 * C, bytes, smem_u32(&full[st]));
    }
    // Do not leave while copies issued by this thread may still be landing.
    for (uint32_t st = 0; st < static_cast<uint32_t>(kRingStages) && st < it; ++st) {
      const uint32_t last = st + ((it - 1 - st) / kRingStages) * kRingStages;
      volatile int never = 0;
      mbar_wait_bounded(smem_u32(&full[st]), (last / kRingStages) & 1u, &never, err,
                        DEVERR_TIMEOUT_DRAIN, kDrainLimitNs);
    }
    return;
  }

  const int cw = warp - 1;
  const int sub = lane % L, grp = lane / L, gpw = 32 / L;
  const int nvec = C / 8;
  // channel pairs (2e, 2e + 1) of each of the lane's vectors, pre-halved
  float2 g[CH][4], b[CH][4];
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    const int vi = sub + k * L;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      g[k][e] = vi < nvec ? make_float2(0.5f * __ldg(gamma + vi * 8 + 2 * e),
                                        0.5f * __ldg(gamma + vi * 8 + 2 * e + 1))
                          : make_float2(0.0f, 0.0f);
      b[k][e] = vi < nvec ? make_float2(0.5f * __ldg(beta + vi * 8 + 2 * e),
                                        0.5f * __ldg(beta + vi * 8 + 2 * e + 1))
                          : make_float2(0.0f, 0.0f);
    }
  }
  const float rootC = sqrtf(static_cast<float>(C));
  const float eps2 = eps * eps;
  const bool eps2_normal = eps2 >= 1.17549435e-38f;  // FLT_MIN
  uint32_t it = 0;
  for (long ch = blockIdx.x; ch < nchunks; ch += gridDim.x, ++it) {
    const uint32_t st = it % kRingStages, ph = (it / kRingStages) & 1u;
    int ok = 0;
    if (lane == 0)
      ok = mbar_wait_bounded(smem_u32(&full[st]), ph, abort_flag, err, DEVERR_TIMEOUT_EPILOGUE)
               ? 1
               : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    __syncwarp();
    const long v0 = ch * vpc;
    const int nv = nvox - v0 < vpc ? static_cast<int>(nvox - v0) : vpc;
    const uint8_t* stage = smem_raw + st * chunk_bytes;
    // A warp takes gpw * V consecutive voxels per pass: lane group grp holds
    // voxels vb + grp + j gpw, j < V.  The bound is warp-uniform (the shuffles
    // need every lane).
    for (int vb = cw * gpw * V; vb < nv; vb += NW * gpw * V) {
      float2 xp[V][CH][4];
      float ss[V];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int vl = vb + grp + j * gpw;
        const bool live = vl < nv;
        const uint4* src = reinterpret_cast<const uint4*>(stage + static_cast<size_t>(vl) * C * 2);
        float2 ssa = make_float2(0.0f, 0.0f), ssb = ssa;  // two packed chains
#pragma unroll
        for (int k = 0; k < CH; ++k) {
          const int vi = sub + k * L;
          const uint4 raw = (live && vi < nvec) ? src[vi] : make_uint4(0u, 0u, 0u, 0u);
          xp[j][k][0] = make_float2(bf16lo(raw.x), bf16hi(raw.x));
          xp[j][k][1] = make_float2(bf16lo(raw.y), bf16hi(raw.y));
          xp[j][k][2] = make_float2(bf16lo(raw.z), bf16hi(raw.z));
          xp[j][k][3] = make_float2(bf16lo(raw.w), bf16hi(raw.w));
          ssa = ffma2(xp[j][k][0], xp[j][k][0], ssa);
          ssb = ffma2(xp[j][k][1], xp[j][k][1], ssb);
          ssa = ffma2(xp[j][k][2], xp[j][k][2], ssa);
          ssb = ffma2(xp[j][k][3], xp[j][k][3], ssb);
        }
        ss[j] = (ssa.x + ssa.y) + (ssb.x + ssb.y);
      }
      for (int off = L >> 1; off > 0; off >>= 1) {
#pragma unroll
        for (int j = 0; j < V; ++j) ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], off);
      }
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int vl = vb + grp + j * gpw;
        const bool live = vl < nv;
        // sqrt(C) / max(||x||, eps) = sqrt(C) * rsqrt(max(ss, eps^2)) while eps^2 is normal
        const float r = eps2_normal ? rootC * rsqrtf(fmaxf(ss[j], eps2))
                                    : rootC / fmaxf(sqrtf(ss[j]), eps);
        const float2 r2 = make_float2(r, r);
        uint4* dst = reinterpret_cast<uint4*>(y + (v0 + vl) * C);
#pragma unroll
        for (int k = 0; k < CH; ++k) {
          const int vi = sub + k * L;
          if (!live || vi >= nvec) continue;
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 o = silu_half2(ffma2(xp[j][k][e], fmul2(r2, g[k][e]), b[k][e]));
            w4[e] = pack_bf16x2(o.x, o.y);
          }
          dst[vi] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[st]));
  }
}

template <int CH, int V, int NW>
cudaError_t launch_ring(const __nv_bfloat16* x, __nv_bfloat16* y, const float* gamma,
                        const float* beta, long nvox, int C, int L, float eps, int num_sms,
                        cudaStream_t stream, bool dependent = true) {
  int vpc = kRingChunkBytes / (C * 2);
  if (vpc < 1) vpc = 1;
  const size_t smem = static_cast<size_t>(kRingStages) * vpc * C * 2 + 2 * kRingStages * 8 + 16;
  auto kern = norm_silu_ring_kernel<CH, V, NW>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long nchunks = (nvox + vpc - 1) / vpc;
  const int grid = nchunks < num_sms ? static_cast<int>(nchunks) : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(32 * (NW + 1), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = dependent ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, x, y, gamma, beta, nvox, C, L, vpc, eps, device_error_word());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int VEC, int CH, int U>
cudaError_t launch_one(const T* x, T* y, const float* gamma, const float* beta, long nvox, int C,
                       int L, float eps, int num_sms, cudaStream_t stream) {
  auto kern = norm_silu_kernel<T, VEC, CH, U>;
  const size_t smem = 0;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kNormThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const long groups_per_block = (kNormThreads / 32) * (32 / L);
  long blocks = (nvox + groups_per_block * U - 1) / (groups_per_block * U);
  const long cap = static_cast<long>(num_sms) * per_sm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  kern<<<static_cast<int>(blocks), kNormThreads, smem, stream>>>(x, y, gamma, beta, nvox, C, L, eps);
  return cudaGetLastError();
}

template <typename T, int VEC>
cudaError_t launch_impl(const T* x, T* y, const float* gamma, const float* beta, long nvox, int C,
                        float eps, int num_sms, cudaStream_t stream) {
  const int nvec = C / VEC;
  int L = 1;
  while (L < nvec && L < 32) L <<= 1;
  const int ch = (nvec + L - 1) / L;
  // U * CH <= 4 vectors (64 bytes) in flight per lane keeps 3 blocks of 256 per SM
  if (ch == 1) return launch_one<T, VEC, 1, 4>(x, y, gamma, beta, nvox, C, L, eps, num_sms, stream);
  if (ch == 2) return launch_one<T, VEC, 2, 2>(x, y, gamma, beta, nvox, C, L, eps, num_sms, stream);
  if (ch <= 4) return launch_one<T, VEC, 4, 1>(x, y, gamma, beta, nvox, C, L, eps, num_sms, stream);
  if (ch <= 8) return launch_one<T, VEC, 8, 1>(x, y, gamma, beta, nvox, C, L, eps, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_norm_silu_bf16(const __nv_bfloat16* x, __nv_bfloat16* y, const float* gamma,
                                  const float* beta, long nvox, int C, float eps, int num_sms,
                                  cudaStream_t stream) {
  const int nvec = C / 8;
  int L = 1;
  while (L < nvec && L < 32) L <<= 1;
  const int ch = (nvec + L - 1) / L;
  if (ch == 1) return launch_ring<1, 2, 16>(x, y, gamma, beta, nvox, C, L, eps, num_sms, stream);
  if (ch == 2) return launch_ring<2, 2, 16>(x, y, gamma, beta, nvox, C, L, eps, num_sms, stream);
  if (ch <= 4) return launch_ring<4, 1, 16>(x, y, gamma, beta, nvox, C, L, eps, num_sms, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_norm_silu_f32(const float* x, float* y, const float* gamma, const float* beta,
                                 long nvox, int C, float eps, int num_sms, cudaStream_t stream) {
  return launch_impl<float, 4>(x, y, gamma, beta, nvox, C, eps, num_sms, stream);
}

}  // namespace wvae

// Layout kernels: weight prepack, latent re-layout, nearest upsample, casts.
#include "internal.h"

namespace wvae {

namespace {

__device__ __forceinline__ float load_w(const void* w, int is_f32, long i) {
  return is_f32 ? static_cast<const float*>(w)[i]
                : __bfloat162float(static_cast<const __nv_bfloat16*>(w)[i]);
}

// PyTorch [cout][cin][taps] -> bf16 [cout_pad][taps][cin_pad], zero padding.
// Row n of the packed matrix is output channel n with K = (tap, input channel)
// contiguous: the K-major operand the tensor-core kernel loads with TMA.
__global__ void prepack_bf16_kernel(const void* w, int is_f32, const float* bias, int cout,
                                    int cin, int taps, int cout_pad, int cin_pad,
                                    __nv_bfloat16* wp, float* bias_p) {
  const long total = static_cast<long>(cout_pad) * taps * cin_pad;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx % cin_pad);
    const int tap = static_cast<int>((idx / cin_pad) % taps);
    const int o = static_cast<int>(idx / (static_cast<long>(cin_pad) * taps));
    float v = 0.0f;
    if (o < cout && i < cin) v = load_w(w, is_f32, (static_cast<long>(o) * cin + i) * taps + tap);
    wp[idx] = __float2bfloat16_rn(v);
    if (idx < cout_pad) bias_p[idx] = (bias != nullptr && idx < cout) ? bias[idx] : 0.0f;
  }
}

// Nearest 2x upsample + 3x3 conv as four 2x2 "phase" convs on the low-res
// input.  Output pixel (2i+p, 2j+q) reads input rows i + r + p - 1 (r = 0, 1)
// and columns j + c + q - 1 (c = 0, 1); row tap r of phase p combines the
// 3x3 rows kh in R(p, r): R(0,0) = {0}, R(0,1) = {1,2}, R(1,0) = {0,1},
// R(1,1) = {2} (and the same for columns).  The combined weights are summed
// in fp32 and rounded once to bf16.  Packed as [cout_pad][phase*4 + r*2 + c]
// [cin_pad], phase = 2p + q.
__device__ __forceinline__ int phase_lo(int p, int r) { return (p == 0) ? (r == 0 ? 0 : 1) : (r == 0 ? 0 : 2); }
__device__ __forceinline__ int phase_hi(int p, int r) { return (p == 0) ? (r == 0 ? 0 : 2) : (r == 0 ? 1 : 2); }

__global__ void prepack_phase_bf16_kernel(const void* w, int is_f32, const float* bias, int cout,
                                          int cin, int cout_pad, int cin_pad, __nv_bfloat16* wp,
                                          float* bias_p) {
  const long total = static_cast<long>(cout_pad) * 16 * cin_pad;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx % cin_pad);
    const int tap = static_cast<int>((idx / cin_pad) % 16);
    const int o = static_cast<int>(idx / (static_cast<long>(cin_pad) * 16));
    const int phase = tap >> 2, p = phase >> 1, q = phase & 1, r = (tap >> 1) & 1, c = tap & 1;
    float v = 0.0f;
    if (o < cout && i < cin) {
      const long base = (static_cast<long>(o) * cin + i) * 9;
      for (int kh = phase_lo(p, r); kh <= phase_hi(p, r); ++kh)
        for (int kw = phase_lo(q, c); kw <= phase_hi(q, c); ++kw)
          v += load_w(w, is_f32, base + kh * 3 + kw);
    }
    wp[idx] = __float2bfloat16_rn(v);
    if (idx < cout_pad) bias_p[idx] = (bias != nullptr && idx < cout) ? bias[idx] : 0.0f;
  }
}

// PyTorch [cout][cin][taps] -> fp32 [taps][cin][cout].
__global__ void prepack_f32_kernel(const void* w, int is_f32, const float* bias, int cout, int cin,
                                   int taps, float* wp, float* bias_p) {
  const long total = static_cast<long>(cout) * taps * cin;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int o = static_cast<int>(idx % cout);
    const int i = static_cast<int>((idx / cout) % cin);
    const int tap = static_cast<int>(idx / (static_cast<long>(cout) * cin));
    wp[idx] = load_w(w, is_f32, (static_cast<long>(o) * cin + i) * taps + tap);
    if (idx < cout) bias_p[idx] = bias != nullptr ? bias[idx] : 0.0f;
  }
}

// [C][T][H][W] -> [T][H][W][Cpad]; one thread per output element.
__global__ void ncdhw_to_cl_kernel(const __nv_bfloat16* x, __nv_bfloat16* y, int C, int Cpad,
                                   long nvox) {
  const long total = nvox * Cpad;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % Cpad);
    const long v = idx / Cpad;
    y[idx] = c < C ? x[static_cast<long>(c) * nvox + v] : __float2bfloat16_rn(0.0f);
  }
}

// [T][H][W][C] -> [T][2H][2W][C] in 16-byte vectors.
__global__ void upsample2x_kernel(const uint4* x, uint4* y, int T, int H, int W, int vec_per_vox) {
  const long total = static_cast<long>(T) * 4 * H * W * vec_per_vox;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int vi = static_cast<int>(idx % vec_per_vox);
    long r = idx / vec_per_vox;
    const int w2 = static_cast<int>(r % (2 * W));
    r /= 2 * W;
    const int h2 = static_cast<int>(r % (2 * H));
    const long t = r / (2 * H);
    y[idx] = __ldg(x + ((t * H + h2 / 2) * W + w2 / 2) * vec_per_vox + vi);
  }
}

__global__ void f32_to_bf16_kernel(const float* x, __nv_bfloat16* y, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i]);
}

int grid_for(long n, int threads) {
  long g = (n + threads - 1) / threads;
  if (g > 148L * 16) g = 148L * 16;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_prepack_bf16(const void* w, int w_is_f32, const float* bias, int cout, int cin,
                                int taps, int cout_pad, int cin_pad, __nv_bfloat16* wp,
                                float* bias_p, cudaStream_t stream) {
  const long total = static_cast<long>(cout_pad) * taps * cin_pad;
  prepack_bf16_kernel<<<grid_for(total, 256), 256, 0, stream>>>(w, w_is_f32, bias, cout, cin, taps,
                                                                cout_pad, cin_pad, wp, bias_p);
  return cudaGetLastError();
}

cudaError_t launch_prepack_phase_bf16(const void* w, int w_is_f32, const float* bias, int cout,
                                      int cin, int cout_pad, int cin_pad, __nv_bfloat16* wp,
                                      float* bias_p, cudaStream_t stream) {
  const long total = static_cast<long>(cout_pad) * 16 * cin_pad;
  prepack_phase_bf16_kernel<<<grid_for(total, 256), 256, 0, stream>>>(w, w_is_f32, bias, cout, cin,
                                                                      cout_pad, cin_pad, wp, bias_p);
  return cudaGetLastError();
}

cudaError_t launch_prepack_f32(const void* w, int w_is_f32, const float* bias, int cout, int cin,
                               int taps, float* wp, float* bias_p, cudaStream_t stream) {
  const long total = static_cast<long>(cout) * taps * cin;
  prepack_f32_kernel<<<grid_for(total, 256), 256, 0, stream>>>(w, w_is_f32, bias, cout, cin, taps,
                                                               wp, bias_p);
  return cudaGetLastError();
}

cudaError_t launch_ncdhw_to_cl_pad(const __nv_bfloat16* x, __nv_bfloat16* y, int C, int Cpad,
                                   int T, int H, int W, cudaStream_t stream) {
  const long nvox = static_cast<long>(T) * H * W;
  ncdhw_to_cl_kernel<<<grid_for(nvox * Cpad, 256), 256, 0, stream>>>(x, y, C, Cpad, nvox);
  return cudaGetLastError();
}

cudaError_t launch_upsample2x(const void* x, void* y, int elem_bytes, int T, int H, int W, int C,
                              cudaStream_t stream) {
  const int vpv = C * elem_bytes / 16;
  const long total = static_cast<long>(T) * 4 * H * W * vpv;
  upsample2x_kernel<<<grid_for(total, 256), 256, 0, stream>>>(static_cast<const uint4*>(x),
                                                              static_cast<uint4*>(y), T, H, W, vpv);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* x, __nv_bfloat16* y, size_t n, cudaStream_t stream) {
  f32_to_bf16_kernel<<<grid_for(static_cast<long>(n), 256), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace wvae

// Winograd F(2x2, 3x3) form of the causal 3x3x3 conv: the transforms around
// the tensor-core products.
//
// The page-3 decoder multiplies Winograd-transformed weights and activations
// (FastVideo "Wan2.2 VAE decoder (sm_100a, sm_103a)" README, "Use": the
// weights get Winograd transforms once; "Performance and memory": the
// products are 60 % of its GPU time).  The algorithm is the minimal-filtering
// form of Lavin and Gray ("Fast Algorithms for Convolutional Neural
// Networks", CVPR 2016, section 4): for a 4 x 4 input tile d (stride 2) and a
// 3 x 3 filter g the 2 x 2 output tile is
//     Y = A^T [ (G g G^T) * (B^T d B) ] A          (* elementwise)
// with the published matrices
//     B^T = [1 0 -1 0; 0 1 1 0; 0 -1 1 0; 0 1 0 -1]
//     G   = [1 0 0; 1/2 1/2 1/2; 1/2 -1/2 1/2; 0 0 1]
//     A^T = [1 1 1 0; 0 1 -1 -1].
// Spatially only: the causal temporal taps stay direct, so with U = G g G^T
// per (o, i, kt) and V = B^T d B per (frame, tile, i) the conv is, for each
// of the 16 transform positions xi,
//     M_xi[t, tile, o] = sum_{kt, i} U_xi[o, kt, i] V_xi[t + kt - 2, tile, i],
// a causal 3-tap temporal conv over the plane V_xi: the tensor-core conv
// kernel runs it (16 planes, fp16 operands, fp32 accumulation, fp16 M), and
// the output transform adds bias and residual.  Operands are fp16 because
// the transforms of bf16 values need more mantissa than bf16 holds; fp16
// keeps the direct conv's accuracy at the same tensor-core rate.
//
// Layouts: V [16][T][tH][tW][Cin] fp16, M [16][T][tH][tW][Cout] fp16 with
// tH = ceil(H / 2), tW = ceil(W / 2); xi = 4a + b for row a and column b of
// the 4 x 4 transform; packed U [cout_pad][16 xi x 3 kt][cin_pad] fp16.
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace wvae {

namespace {

__device__ __forceinline__ float load_wt(const void* w, int is_f32, long i) {
  return is_f32 ? static_cast<const float*>(w)[i]
                : __bfloat162float(static_cast<const __nv_bfloat16*>(w)[i]);
}

// U = G g G^T for each (o, i, kt): one thread per packed element.
__global__ void wino_prepack_kernel(const void* w, int is_f32, const float* bias, int cout, int cin,
                                    int cout_pad, int cin_pad, __half* up, float* bias_zero,
                                    float* bias_p) {
  const long total = static_cast<long>(cout_pad) * 48 * cin_pad;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx % cin_pad);
    const int tap = static_cast<int>((idx / cin_pad) % 48);
    const int o = static_cast<int>(idx / (static_cast<long>(cin_pad) * 48));
    const int xi = tap / 3, kt = tap % 3, a = xi >> 2, b = xi & 3;
    float u = 0.0f;
    if (o < cout && i < cin) {
      const long base = ((static_cast<long>(o) * cin + i) * 3 + kt) * 9;
      // row a of G applied to the 3 rows of g, then column b of G^T
      float r[3];
      for (int c = 0; c < 3; ++c) {
        const float g0 = load_wt(w, is_f32, base + c), g1 = load_wt(w, is_f32, base + 3 + c),
                    g2 = load_wt(w, is_f32, base + 6 + c);
        r[c] = a == 0 ? g0 : (a == 1 ? 0.5f * (g0 + g1 + g2) : (a == 2 ? 0.5f * (g0 - g1 + g2) : g2));
      }
      u = b == 0 ? r[0] : (b == 1 ? 0.5f * (r[0] + r[1] + r[2])
                                  : (b == 2 ? 0.5f * (r[0] - r[1] + r[2]) : r[2]));
    }
    up[idx] = __float2half_rn(u);
    if (idx < cout_pad) {
      bias_zero[idx] = 0.0f;
      bias_p[idx] = (bias != nullptr && idx < cout) ? bias[idx] : 0.0f;
    }
  }
}

// V = B^T d B: one thread per (t, tile row, tile column, 4 channels); the
// patch is read a column at a time (B^T applied to its 4 rows), then B on
// the columns.
__global__ void wino_input_kernel(const __nv_bfloat16* __restrict__ x, __half* __restrict__ v,
                                  int T, int H, int W, int C, int tH, int tW) {
  const int cg = C / 4;
  const long total = static_cast<long>(T) * tH * tW * cg;
  const size_t plane = static_cast<size_t>(T) * tH * tW * C;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int c4 = static_cast<int>(idx % cg);
    long r = idx / cg;
    const int tw = static_cast<int>(r % tW);
    r /= tW;
    const int th = static_cast<int>(r % tH);
    const int t = static_cast<int>(r / tH);
    float e[4][4][4];   // (B^T d)[a][column j][channel]
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int ww = 2 * tw - 1 + j;
      float d[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int hh = 2 * th - 1 + i;
        uint2 q = make_uint2(0u, 0u);
        if (hh >= 0 && hh < H && ww >= 0 && ww < W)
          q = *reinterpret_cast<const uint2*>(x + ((static_cast<size_t>(t) * H + hh) * W + ww) * C +
                                              c4 * 4);
        d[i][0] = bf16lo(q.x); d[i][1] = bf16hi(q.x);
        d[i][2] = bf16lo(q.y); d[i][3] = bf16hi(q.y);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        e[0][j][k] = d[0][k] - d[2][k];
        e[1][j][k] = d[1][k] + d[2][k];
        e[2][j][k] = d[2][k] - d[1][k];
        e[3][j][k] = d[1][k] - d[3][k];
      }
    }
    const size_t off = ((static_cast<size_t>(t) * tH + th) * tW + tw) * C + c4 * 4;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float o[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        o[0][k] = e[a][0][k] - e[a][2][k];
        o[1][k] = e[a][1][k] + e[a][2][k];
        o[2][k] = e[a][2][k] - e[a][1][k];
        o[3][k] = e[a][1][k] - e[a][3][k];
      }
#pragma unroll
      for (int b = 0; b < 4; ++b)
        *reinterpret_cast<uint2*>(v + (4 * a + b) * plane + off) =
            make_uint2(pack_f16x2(o[b][0], o[b][1]), pack_f16x2(o[b][2], o[b][3]));
    }
  }
}

// y = A^T M A + bias (+ residual): one thread per (t, tile row, tile column, 8 channels).
__global__ void wino_output_kernel(const __half* __restrict__ m, const float* __restrict__ bias,
                                   const __nv_bfloat16* __restrict__ residual,
                                   __nv_bfloat16* __restrict__ y, int T, int H, int W, int C,
                                   int tH, int tW) {
  const int cg = C / 8;
  const long total = static_cast<long>(T) * tH * tW * cg;
  const size_t plane = static_cast<size_t>(T) * tH * tW * C;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int c8 = static_cast<int>(idx % cg);
    long r = idx / cg;
    const int tw = static_cast<int>(r % tW);
    r /= tW;
    const int th = static_cast<int>(r % tH);
    const int t = static_cast<int>(r / tH);
    const size_t off = ((static_cast<size_t>(t) * tH + th) * tW + tw) * C + c8 * 8;
    // rows: s[p][b] = (A^T M)[p][b]
    float s[2][4][8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float mv[4][8];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const uint4 q = *reinterpret_cast<const uint4*>(m + (4 * a + b) * plane + off);
        mv[a][0] = f16lo(q.x); mv[a][1] = f16hi(q.x);
        mv[a][2] = f16lo(q.y); mv[a][3] = f16hi(q.y);
        mv[a][4] = f16lo(q.z); mv[a][5] = f16hi(q.z);
        mv[a][6] = f16lo(q.w); mv[a][7] = f16hi(q.w);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        s[0][b][k] = mv[0][k] + mv[1][k] + mv[2][k];
        s[1][b][k] = mv[1][k] - mv[2][k] - mv[3][k];
      }
    }
    float bs[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) bs[k] = bias[c8 * 8 + k];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const int hh = 2 * th + p;
      if (hh >= H) continue;
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int ww = 2 * tw + q2;
        if (ww >= W) continue;
        float o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          o[k] = (q2 == 0 ? s[p][0][k] + s[p][1][k] + s[p][2][k]
                          : s[p][1][k] - s[p][2][k] - s[p][3][k]) + bs[k];
        const size_t vo = ((static_cast<size_t>(t) * H + hh) * W + ww) * C + c8 * 8;
        if (residual != nullptr) {
          const uint4 rq = *reinterpret_cast<const uint4*>(residual + vo);
          o[0] += bf16lo(rq.x); o[1] += bf16hi(rq.x); o[2] += bf16lo(rq.y); o[3] += bf16hi(rq.y);
          o[4] += bf16lo(rq.z); o[5] += bf16hi(rq.z); o[6] += bf16lo(rq.w); o[7] += bf16hi(rq.w);
        }
        uint4 w4;
        w4.x = pack_bf16x2(o[0], o[1]);
        w4.y = pack_bf16x2(o[2], o[3]);
        w4.z = pack_bf16x2(o[4], o[5]);
        w4.w = pack_bf16x2(o[6], o[7]);
        *reinterpret_cast<uint4*>(y + vo) = w4;
      }
    }
  }
}

int grid_for(long total, int threads) {
  long g = (total + threads - 1) / threads;
  if (g > 148L * 16) g = 148L * 16;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_wino_prepack(const void* w, bool is_f32, const float* bias, int cout, int cin,
                                int cout_pad, int cin_pad, __half* up, float* bias_zero,
                                float* bias_p, cudaStream_t stream) {
  const long total = static_cast<long>(cout_pad) * 48 * cin_pad;
  wino_prepack_kernel<<<grid_for(total, 256), 256, 0, stream>>>(
      w, is_f32 ? 1 : 0, bias, cout, cin, cout_pad, cin_pad, up, bias_zero, bias_p);
  return cudaGetLastError();
}

cudaError_t launch_wino_input(const __nv_bfloat16* x, __half* v, int T, int H, int W, int C,
                              cudaStream_t stream) {
  const int tH = (H + 1) / 2, tW = (W + 1) / 2;
  const long total = static_cast<long>(T) * tH * tW * (C / 4);
  wino_input_kernel<<<grid_for(total, 256), 256, 0, stream>>>(x, v, T, H, W, C, tH, tW);
  return cudaGetLastError();
}

cudaError_t launch_wino_output(const __half* m, const float* bias, const __nv_bfloat16* residual,
                               __nv_bfloat16* y, int T, int H, int W, int C, cudaStream_t stream) {
  const int tH = (H + 1) / 2, tW = (W + 1) / 2;
  const long total = static_cast<long>(T) * tH * tW * (C / 8);
  wino_output_kernel<<<grid_for(total, 128), 128, 0, stream>>>(m, bias, residual, y, T, H, W, C,
                                                               tH, tW);
  return cudaGetLastError();
}

}  // namespace wvae

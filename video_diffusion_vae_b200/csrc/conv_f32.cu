// fp32 causal conv3d on CUDA cores: the precision reference path (dtype
// WVAE_F32).  Same definition as the tensor-core kernel: zero front frames (or
// the cached frames), a zero border, fp32 accumulation.  One thread per
// (voxel, output channel); threads of a block cover consecutive output
// channels so weight reads ([tap][cin][cout] packing) are coalesced and input
// reads are broadcasts.
#include "internal.h"

namespace wvae {

namespace {

__global__ void conv_f32_kernel(const ConvF32Params p) {
  const int o = blockIdx.y * blockDim.x + threadIdx.x;
  const long vox = blockIdx.x;
  if (o >= p.cout) return;
  const int w = static_cast<int>(vox % p.W);
  const int h = static_cast<int>((vox / p.W) % p.H);
  const int t = static_cast<int>(vox / (static_cast<long>(p.W) * p.H));
  float acc = p.bias[o];
  int tap = 0;
  for (int kt = 0; kt < p.KT; ++kt)
    for (int kh = 0; kh < p.KH; ++kh)
      for (int kw = 0; kw < p.KW; ++kw, ++tap) {
        const int ts = t + kt - (p.KT - 1);
        const int hs = h + kh - (p.KH - 1) / 2;
        const int ws = w + kw - (p.KW - 1) / 2;
        if (hs < 0 || hs >= p.H || ws < 0 || ws >= p.W) continue;
        const float* src;
        if (ts >= 0)
          src = p.x + ((static_cast<long>(ts) * p.H + hs) * p.W + ws) * p.cin;
        else if (p.cache != nullptr)
          src = p.cache + ((static_cast<long>(ts + p.KT - 1) * p.H + hs) * p.W + ws) * p.cin;
        else
          continue;
        const float* wt = p.w + static_cast<long>(tap) * p.cin * p.cout + o;
        for (int i = 0; i < p.cin; ++i) acc = fmaf(wt[static_cast<long>(i) * p.cout], src[i], acc);
      }
  if (p.residual != nullptr) acc += p.residual[vox * p.cout + o];
  p.y[vox * p.cout + o] = acc;
}

}  // namespace

cudaError_t launch_conv_f32(const ConvF32Params& p, cudaStream_t stream) {
  const long nvox = static_cast<long>(p.T) * p.H * p.W;
  dim3 block(p.cout < 128 ? ((p.cout + 31) / 32) * 32 : 128);
  dim3 grid(static_cast<unsigned>(nvox), (p.cout + block.x - 1) / block.x);
  conv_f32_kernel<<<grid, block, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace wvae

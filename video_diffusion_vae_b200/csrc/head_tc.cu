// The decoder head on the sm_100a tensor cores: causal 3x3x3 conv from the
// last stage's activation (C = 64 or 128 channels, norm_out + SiLU already
// applied by the producing conv) to 12 channels, written as the 2x2
// pixel-shuffled NCDHW video: video[c, t, 2h+i, 2w+j] = out[t, h, w, 4c+2i+j].
// (FastVideo "Wan2.2 VAE decoder (sm_100a, sm_103a)" README, opening section:
// 48 latent channels and 16x16 spatial compression, so the last conv's 12
// channels are 3 video channels x 2 x 2 pixels; "Limits": bf16 operands,
// fp32 accumulation.)
//
// With 16 output channels (12 used) a tcgen05.mma of N = 16 is mostly fixed
// issue cost.  Here one MMA carries nine taps at once: N = 144 = (kt, kw, o)
// for the 3 temporal x 3 column taps x 16 channels, the 3 row taps run in K
// (the A window holds the tile's rows plus a one-row halo above and below,
// and row tap kh reads it kh rows down: whole 128-byte swizzle atoms).  A
// TMEM lane (one computed voxel of input frame f) then holds the partial
// sums P[kt][kw][o] of that frame.  Output column w needs P[.][0] from
// column w - 1, P[.][1] from w and P[.][2] from w + 1 (the neighbouring
// lanes of the same tile row: warp shuffles), and output frame t needs
// Q[2] of input frame t, Q[1] of t - 1 and Q[0] of t - 2: a CTA takes one
// spatial tile through all frames in order, and each epilogue thread carries
// the two pending sums of its voxel from frame to frame in registers.  So
// every input frame is read once per tile (3x fewer A bytes than one pass
// per temporal tap) and a tile's MMAs are 3x fewer and 3x wider than with the
// column taps alone in N.
//
// Tile: 8 rows x 16 computed columns (one M = 128 MMA), yielding 8 x 14
// output voxels (columns 0 and 15 are halo).  The weights (3 row taps x
// C/64 chunks x 144 rows x 128 B: 108 KB at C = 128) stay in shared memory
// for the whole kernel, read from the standard packed blob
// [16][27 taps][C] with 9 boxes of 16 rows per tile.  Two TMEM accumulators
// alternate between frames: the epilogue of frame f overlaps the MMAs of
// frame f + 1.  Warp 0 issues the TMA loads, warp 1 the MMAs, warps 2..5 run
// the epilogue (one TMEM lane quarter each).
#include "internal.h"
#include "ptx.cuh"

namespace wvae {

namespace {

constexpr int kRows = kHeadTileRows;                  // 8
constexpr int kCols = kHeadTileCols;                  // 16 computed columns
constexpr int kN = 144;                               // (kt, kw, o)
constexpr int kAccCols = 256;                         // TMEM columns per accumulator
constexpr int kAStages = 4;
constexpr uint32_t kABytes = (kRows + 2) * kCols * 128;   // 20480: {64 ch, 16 w, 10 h}
constexpr uint32_t kBTileBytes = kN * 128;                // 18432
constexpr uint32_t kBoxBytes = 16 * 128;                  // one (kt, kw) box of 16 rows

struct HeadSmem {
  uint8_t* b;          // [3 kh][nchunk] weight tiles of 144 rows
  uint8_t* a;          // [kAStages] A windows
  uint64_t* full;      // [kAStages]
  uint64_t* empty;     // [kAStages]
  uint64_t* bfull;     // [1]
  uint64_t* tfull;     // [2]
  uint64_t* tempty;    // [2]
  uint64_t* drain;     // [1]
  uint32_t* tmem_slot;
  int* abort_flag;
};

__device__ __forceinline__ HeadSmem head_carve(uint8_t* raw, int nchunk) {
  HeadSmem s;
  const uint32_t base = smem_u32(raw);
  uint8_t* al = raw + ((1024u - (base & 1023u)) & 1023u);
  s.b = al;
  s.a = al + 3 * nchunk * kBTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.a + kAStages * kABytes);
  s.full = bars;
  s.empty = s.full + kAStages;
  s.bfull = s.empty + kAStages;
  s.tfull = s.bfull + 1;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.drain + 1);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_slot + 1);
  return s;
}

__device__ __forceinline__ void head_tile(const HeadParams& p, int tile, int& h0, int& w0) {
  const int tw = tile % p.tiles_w, th = tile / p.tiles_w;
  h0 = th * kRows;
  w0 = tw * kHeadOutCols;
}

__device__ void head_producer(const HeadParams& p, const HeadSmem& s) {
  const int nchunk = p.cin / 64;
  // all weight tiles once: tile (kh, chunk) rows (kt, kw, o) <- packed taps (kt, kh, kw)
  const uint32_t bbar = smem_u32(s.bfull);
  mbar_arrive_expect_tx(bbar, static_cast<uint32_t>(3 * nchunk) * kBTileBytes);
  for (int kh = 0; kh < 3; ++kh)
    for (int ch = 0; ch < nchunk; ++ch) {
      const uint32_t dst = smem_u32(s.b + (kh * nchunk + ch) * kBTileBytes);
      for (int kt = 0; kt < 3; ++kt)
        for (int kw = 0; kw < 3; ++kw) {
          const int tap = (kt * 3 + kh) * 3 + kw;
          tma_load_2d(dst + (kt * 3 + kw) * kBoxBytes, &p.tmB, bbar, tap * p.cin + ch * 64, 0);
        }
    }
  const int f0 = p.has_cache ? -2 : 0;
  uint32_t ia = 0;
  bool aborted = false;
  for (int tile = blockIdx.x; tile < p.num_tiles && !aborted; tile += gridDim.x) {
    int h0, w0;
    head_tile(p, tile, h0, w0);
    for (int f = f0; f < p.T && !aborted; ++f)
      for (int ch = 0; ch < nchunk; ++ch, ++ia) {
        const uint32_t st = ia % kAStages, ph = (ia / kAStages) & 1u;
        if (!mbar_wait_bounded(smem_u32(&s.empty[st]), ph ^ 1u, s.abort_flag, p.err,
                               DEVERR_TIMEOUT_PRODUCER)) {
          aborted = true;
          break;
        }
        const uint32_t bar = smem_u32(&s.full[st]);
        mbar_arrive_expect_tx(bar, kABytes);
        const uint32_t dst = smem_u32(s.a + st * kABytes);
        if (f < 0)
          tma_load_4d(dst, &p.tmC, bar, ch * 64, w0 - 1, h0 - 1, f + 2);
        else
          tma_load_4d(dst, &p.tmA, bar, ch * 64, w0 - 1, h0 - 1, f);
      }
  }
  // Do not leave while copies issued by this thread may still be landing.
  for (uint32_t st = 0; st < static_cast<uint32_t>(kAStages) && st < ia; ++st) {
    const uint32_t last = st + ((ia - 1 - st) / kAStages) * kAStages;
    volatile int never = 0;
    mbar_wait_bounded(smem_u32(&s.full[st]), (last / kAStages) & 1u, &never, p.err,
                      DEVERR_TIMEOUT_DRAIN, kDrainLimitNs);
  }
  volatile int never = 0;
  mbar_wait_bounded(bbar, 0, &never, p.err, DEVERR_TIMEOUT_DRAIN, kDrainLimitNs);
}

template <int NCHUNK>
__device__ void head_mma(const HeadParams& p, const HeadSmem& s, uint32_t tmem_base) {
  const uint32_t idesc = umma_idesc_bf16(128, kN);
  const uint64_t adesc0 = umma_desc_sw128(smem_u32(s.a));
  const uint64_t bdesc0 = umma_desc_sw128(smem_u32(s.b));
  const uint32_t a_step = kABytes >> 4, b_step = kBTileBytes >> 4;
  const uint32_t kh_step = (kCols * 128) >> 4;   // one window row of 16 voxels
  bool ok = mbar_wait_bounded(smem_u32(s.bfull), 0, s.abort_flag, p.err, DEVERR_TIMEOUT_MMA);
  if (ok) tc_fence_after();
  const int f0 = p.has_cache ? -2 : 0;
  uint32_t ia = 0, it = 0;
  for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
    for (int f = f0; f < p.T && ok; ++f, ++it) {
      const uint32_t acc = it & 1u, aph = (it >> 1) & 1u;
      if (!mbar_wait_bounded(smem_u32(&s.tempty[acc]), aph ^ 1u, s.abort_flag, p.err,
                             DEVERR_TIMEOUT_MMA)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + acc * kAccCols;
#pragma unroll
      for (int ch = 0; ch < NCHUNK; ++ch, ++ia) {
        const uint32_t st = ia % kAStages, ph = (ia / kAStages) & 1u;
        if (!mbar_try_wait(smem_u32(&s.full[st]), ph) &&
            !mbar_wait_bounded(smem_u32(&s.full[st]), ph, s.abort_flag, p.err, DEVERR_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a_st = adesc0 + st * a_step;
#pragma unroll
        for (int kh = 0; kh < 3; ++kh) {
          const uint64_t b_t = bdesc0 + (kh * NCHUNK + ch) * b_step;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(d, a_st + kh * kh_step + 2u * k, b_t + 2u * k, idesc,
                      (ch | kh | k) != 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(&s.empty[st]));
      }
      if (!ok) break;
      umma_commit(smem_u32(&s.tfull[acc]));
    }
  }
  // Every MMA issued by this thread has finished before TMEM / smem go away.
  umma_commit(smem_u32(s.drain));
  volatile int never = 0;
  mbar_wait_bounded(smem_u32(s.drain), 0, &never, p.err, DEVERR_TIMEOUT_DRAIN, kDrainLimitNs);
}

// Q[o] = P[kw=1][o] (this column) + P[kw=0][o] of column - 1 + P[kw=2][o] of column + 1
__device__ __forceinline__ void column_sum(uint32_t taddr, float (&q)[16]) {
  uint32_t r0[16], r1[16], r2[16];
  tmem_ld16(taddr, r0);
  tmem_ld16(taddr + 16, r1);
  tmem_ld16(taddr + 32, r2);
  tmem_wait_ld();
#pragma unroll
  for (int o = 0; o < 16; ++o)
    q[o] = __uint_as_float(r1[o]) + __shfl_up_sync(0xffffffffu, __uint_as_float(r0[o]), 1) +
           __shfl_down_sync(0xffffffffu, __uint_as_float(r2[o]), 1);
}

__device__ void head_epilogue(const HeadParams& p, const HeadSmem& s, uint32_t tmem_base, int warp,
                              int lane) {
  const int q = warp & 3;                       // TMEM lane quarter of this warp
  const int idx = q * 32 + lane;                // computed voxel of the tile, row-major
  const int r = idx / kCols, c = idx % kCols;
  float bias[12];
#pragma unroll
  for (int o = 0; o < 12; ++o) bias[o] = p.bias[o];
  const int f0 = p.has_cache ? -2 : 0;
  // video rows: 2 (h - row0) + i for the rows_out rows from row0 on
  const int rows_out = p.rows_out > 0 ? p.rows_out : p.H;
  const size_t H2 = 2 * static_cast<size_t>(rows_out), W2 = 2 * static_cast<size_t>(p.W);
  uint32_t it = 0;
  for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
    int h0, w0;
    head_tile(p, tile, h0, w0);
    const int h = h0 + r, w = w0 - 1 + c;
    const bool valid = h < p.H && c >= 1 && c <= kCols - 2 && w < p.W && h >= p.row0 &&
                       h < p.row0 + rows_out;
    const int hv = h - p.row0;
    float pend_a[16], pend_b[16];     // partial sums of output frames f and f + 1
#pragma unroll
    for (int o = 0; o < 16; ++o) pend_a[o] = pend_b[o] = 0.0f;
    for (int f = f0; f < p.T; ++f, ++it) {
      const uint32_t acc = it & 1u, aph = (it >> 1) & 1u;
      int okw = 0;
      if (lane == 0)
        okw = mbar_wait_bounded(smem_u32(&s.tfull[acc]), aph, s.abort_flag, p.err,
                                DEVERR_TIMEOUT_EPILOGUE) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) return;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      float qs[16], out[16];
      column_sum(taddr + 2 * 48, qs);           // kt = 2: output frame f
#pragma unroll
      for (int o = 0; o < 16; ++o) out[o] = pend_a[o] + qs[o];
      column_sum(taddr + 1 * 48, qs);           // kt = 1: output frame f + 1
#pragma unroll
      for (int o = 0; o < 16; ++o) pend_a[o] = pend_b[o] + qs[o];
      column_sum(taddr, qs);                    // kt = 0: output frame f + 2
#pragma unroll
      for (int o = 0; o < 16; ++o) pend_b[o] = qs[o];
      tc_fence_before();
      mbar_arrive(smem_u32(&s.tempty[acc]));
      if (f >= 0 && valid) {
        // channel o = 4c' + 2i + j -> video[c', f, 2h + i, 2w + j]: pixel pairs (j = 0, 1)
#pragma unroll
        for (int cv = 0; cv < 3; ++cv)
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int o = 4 * cv + 2 * i;
            const size_t off = ((static_cast<size_t>(cv) * p.T + f) * H2 + 2 * hv + i) * W2 + 2 * w;
            *reinterpret_cast<uint32_t*>(p.video + off) =
                pack_bf16x2(out[o] + bias[o], out[o + 1] + bias[o + 1]);
          }
      }
    }
  }
}

__global__ void __launch_bounds__(kHeadThreads, 1) head_tc_kernel(const __grid_constant__ HeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  const int nchunk = p.cin / 64;
  const HeadSmem s = head_carve(smem_raw, nchunk);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(smem_u32(&s.full[i]), 1);
      mbar_init(smem_u32(&s.empty[i]), 1);
    }
    mbar_init(smem_u32(s.bfull), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s.tfull[i]), 1);
      mbar_init(smem_u32(&s.tempty[i]), 128);
    }
    mbar_init(smem_u32(s.drain), 1);
    *s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s.tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;
  if (warp == 0) {
    if (lane == 0) head_producer(p, s);
  } else if (warp == 1) {
    if (lane == 0) {
      if (nchunk == 1)
        head_mma<1>(p, s, tmem_base);
      else
        head_mma<2>(p, s, tmem_base);
    }
  } else {
    head_epilogue(p, s, tmem_base, warp, lane);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace

size_t head_tc_smem_bytes(int cin) {
  return 1024 + static_cast<size_t>(3 * (cin / 64)) * kBTileBytes +
         static_cast<size_t>(kAStages) * kABytes + 256;
}

cudaError_t launch_head_tc(const HeadParams& p, int num_sms, cudaStream_t stream) {
  const size_t smem = head_tc_smem_bytes(p.cin);
  cudaError_t e = cudaFuncSetAttribute(head_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  head_tc_kernel<<<grid, kHeadThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace wvae

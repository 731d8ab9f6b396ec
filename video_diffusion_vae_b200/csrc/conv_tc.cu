// Causal conv3d as an implicit GEMM on the sm_100a tensor cores.
//
//   out[m, n] = sum_k A[m, k] * B[n, k]
//   m: an output voxel (t, h, w);  n: an output channel;
//   k: (tap, input channel), tap = (kt, kh, kw) over the KT x KH x KW window.
//   A[m, (tap, i)] = a[t + kt - (KT-1), h + kh - (KH-1)/2, w + kw - (KW-1)/2, i]
//
// The causal front frames and the spatial border are zero (or, for t' < 0, the
// previous chunk's cached frames).  No padded copy exists: every K block is one
// TMA box load of the channels-last activation at the tap-shifted coordinates,
// and the tensor map's out-of-bounds fill supplies the zeros.  (Conv definition:
// FastVideo "Wan2.2 VAE decoder (sm_100a, sm_103a)" README, "Limits": bf16
// operands, fp32 accumulation; temporal caching: TensorRT-LLM issue #19309,
// "Feature, motivation and proposed scope".)
//
// One CTA per SM, persistent over output tiles of tile_rows x tile_cols voxels
// of one frame (128 S voxels: S MMA sub-tiles of 128 consecutive voxels in
// row-major order; the shape is chosen per layer to balance the waves) x BN
// output channels.  Warp roles:
//   warp 0      TMA producer: A box {64 ch, tile_cols w, tile_rows h, 1 t} +
//               B box {64, BN} per K block into a ring of `stages` stages;
//   warp 1      MMA issuer: per K block, 4 K steps x S sub-tiles of
//               tcgen05.mma (M=128, N=BN<=256, K=16) sharing the weight tile,
//               into TMEM (two accumulators when 2 S BN <= 512, so the
//               epilogue of tile i overlaps the main loop of tile i+1);
//   warps 2..9  epilogue, two groups of 4 warps (one warp per TMEM lane
//               quarter each): one TMEM lane = one output voxel per thread;
//               with S >= 2 the groups take alternate sub-tiles, with S = 1
//               each takes half of the channels (the two halves of the RMS
//               sum meet in shared memory).
// 512 output channels with the next layer's norm fused: a cluster of two CTAs
// splits N (each runs the S = 2, BN = 256 main loop on its half of the
// channels for the same M tiles) and the two epilogues exchange each voxel's
// partial sum of squares through distributed shared memory.
// tcgen05.mma issue runs nearly in step with execution, so every cycle the
// issuing thread spends waiting on a barrier is a tensor-pipe bubble: S
// sub-tiles per weight tile put S times more MMA work behind each wait.
// The epilogue adds bias (and residual), and may emit the raw result (fp32 or
// bf16, optionally 2x-upsampled), the next layer's SiLU(norm(.)) activation
// (the whole channel vector of the voxel is in the thread's TMEM lane, so the
// RMS statistic needs no cross-thread reduction), or the 2x2 pixel-shuffled
// NCDHW video.  An optional second K segment (the 1x1x1 shortcut of a
// channel-changing residual block) reads its own input and weights.
#include "internal.h"
#include "ptx.cuh"

namespace wvae {

namespace {

struct Smem {
  uint8_t* stages;        // stage s at stages + s * stage_bytes, 1024-aligned
  uint32_t stage_bytes;
  uint32_t a_bytes;
  uint32_t tx_bytes;      // bytes the TMA loads of one main-loop stage deliver
  uint64_t* full;         // [kMaxStages]
  uint64_t* empty;        // [kMaxStages]
  uint64_t* tfull;        // [2]
  uint64_t* tempty;       // [2]
  uint64_t* drain;        // [1]
  uint64_t* ssbar;        // [1] the two epilogue groups' partial RMS sums are written
  uint64_t* xbar;         // [2] (per tile parity) the peer CTA's partial sums have arrived
  float* ss_part;         // [2 tile parities][2 groups][128 rows]
  float* xpart;           // [2 tile parities][256]: partial sums written by the peer CTA
  uint32_t* tmem_slot;
  int* abort_flag;
  float* bias;            // [512]
  float* gamma;           // [512]
  float* beta;            // [512]
};

constexpr uint32_t kCtrlBytes = 512 + 3 * 512 * 4 + 2 * 2 * 128 * 4 + 2 * 256 * 4;

__device__ __forceinline__ Smem carve(uint8_t* raw, const ConvParams& p) {
  Smem s;
  uint32_t base = smem_u32(raw);
  uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* al = raw + pad;
  s.a_bytes = conv_tc_a_bytes(p);
  s.stage_bytes = s.a_bytes + conv_tc_b_bytes(p);
  s.tx_bytes = (p.rowhalo ? static_cast<uint32_t>(p.tile_rows + p.KH - 1) : static_cast<uint32_t>(p.tile_rows)) *
                   static_cast<uint32_t>(p.tile_cols) * 128u +
               conv_tc_b_bytes(p);
  s.stages = al;
  uint8_t* ctrl = al + p.stages * s.stage_bytes;
  s.full = reinterpret_cast<uint64_t*>(ctrl);
  s.empty = s.full + kMaxStages;
  s.tfull = s.empty + kMaxStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.ssbar = s.drain + 1;
  s.xbar = s.ssbar + 1;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.xbar + 2);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_slot + 1);
  s.bias = reinterpret_cast<float*>(ctrl + 512);
  s.gamma = s.bias + 512;
  s.beta = s.gamma + 512;
  s.ss_part = s.beta + 512;
  s.xpart = s.ss_part + 2 * 2 * 128;
  return s;
}

struct TileCoord {
  int n_tile, phase, t, th, tw;
};

// Tile order: N tile fastest, then upsample phase (the four phases of an M
// tile read the same input), then M tiles (column, row, frame).
// With nsplit = 2 the two CTAs of a cluster take the same tiles and the CTA
// rank is the N tile.
__device__ __forceinline__ TileCoord decode_tile(const ConvParams& p, int tile, int crank) {
  TileCoord c;
  int m;
  if (p.nsplit == 2) {
    c.n_tile = crank;
    m = tile;
  } else {
    c.n_tile = tile % p.n_tiles;
    m = tile / p.n_tiles;
  }
  c.phase = m % p.phases;
  m /= p.phases;
  c.tw = m % p.tiles_w;
  m /= p.tiles_w;
  c.th = m % p.tiles_h;
  c.t = m / p.tiles_h;
  return c;
}

// ------------------------------------------------------------------ producer
__device__ __forceinline__ int tile_first(const ConvParams& p) {
  return p.nsplit == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
}
__device__ __forceinline__ int tile_stride(const ConvParams& p) {
  return p.nsplit == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
}

__device__ void producer(const ConvParams& p, const Smem& s, int crank) {
  const int cchunks = p.cin_pad / kBK;
  const int kwkh = p.KH * p.KW;
  const int b_rows = p.BN > 256 ? 256 : p.BN;
  const int b_loads = p.BN > 256 ? 2 : 1;
  const uint32_t b_box_bytes = static_cast<uint32_t>(b_rows) * kBK * 2;
  uint32_t it = 0;
  bool aborted = false;
  for (int tile = tile_first(p); tile < p.num_tiles && !aborted; tile += tile_stride(p)) {
    const TileCoord tc = decode_tile(p, tile, crank);
    const int h0 = tc.th * p.tile_rows, w0 = tc.tw * p.tile_cols;
    for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
      const uint32_t st = it % p.stages;
      const uint32_t ph = (it / p.stages) & 1u;
      if (!mbar_wait_bounded(smem_u32(&s.empty[st]), ph ^ 1u, s.abort_flag, p.err,
                             DEVERR_TIMEOUT_PRODUCER)) {
        aborted = true;
        break;
      }
      const uint32_t bar = smem_u32(&s.full[st]);
      const uint32_t a_dst = smem_u32(s.stages + st * s.stage_bytes);
      const uint32_t b_dst = a_dst + s.a_bytes;
      if (p.rowhalo && kb < p.kblocks_main) {
        // (kt, kw, channel chunk): rows h0 - (KH-1)/2 .. h0 + tile_rows + KH/2 once,
        // the KH row taps' weight tiles side by side
        mbar_arrive_expect_tx(bar, s.tx_bytes);
        const int tap2 = kb / cchunks, cc = kb - tap2 * cchunks;
        const int kt = tap2 / p.KW, kw = tap2 - kt * p.KW;
        const int ts = tc.t + kt - (p.KT - 1);
        const int hs = h0 - (p.KH - 1) / 2, ws = w0 + kw - (p.KW - 1) / 2;
        if (ts < 0 && p.has_cache)
          tma_load_4d(a_dst, &p.tmC, bar, cc * kBK, ws, hs, ts + p.KT - 1);
        else
          tma_load_4d(a_dst, &p.tmA, bar, cc * kBK, ws, hs, ts);
        for (int kh = 0; kh < p.KH; ++kh) {
          const int tap = (kt * p.KH + kh) * p.KW + kw;
          tma_load_2d(b_dst + kh * static_cast<uint32_t>(p.BN) * 128u, &p.tmB, bar,
                      tap * p.cin_pad + cc * kBK, tc.n_tile * p.BN);
        }
        continue;
      }
      mbar_arrive_expect_tx(bar, s.tx_bytes);
      if (kb < p.kblocks_main) {
        const int tap = kb / cchunks, cc = kb - tap * cchunks;
        const int kt = tap / kwkh, r = tap - kt * kwkh;
        const int kh = r / p.KW, kw = r - kh * p.KW;
        const int ts = tc.t + kt - (p.KT - 1);
        // phase mode: output (2h+p', 2w+q') reads input rows h + kh + p' - 1
        const int oh = p.phases == 4 ? (tc.phase >> 1) - 1 : -(p.KH - 1) / 2;
        const int ow = p.phases == 4 ? (tc.phase & 1) - 1 : -(p.KW - 1) / 2;
        const int hs = h0 + kh + oh;
        const int ws = w0 + kw + ow;
        if (ts < 0 && p.has_cache)
          tma_load_4d(a_dst, &p.tmC, bar, cc * kBK, ws, hs, ts + p.KT - 1);
        else
          tma_load_4d(a_dst, &p.tmA, bar, cc * kBK, ws, hs, ts);
        const int kcoord = (tc.phase * 4 * (p.phases == 4) + tap) * p.cin_pad + cc * kBK;
        for (int l = 0; l < b_loads; ++l)
          tma_load_2d(b_dst + l * b_box_bytes, &p.tmB, bar, kcoord, tc.n_tile * p.BN + l * 256);
      } else {
        const int cc = kb - p.kblocks_main;
        tma_load_4d(a_dst, &p.tmA2, bar, cc * kBK, w0, h0, tc.t);
        for (int l = 0; l < b_loads; ++l)
          tma_load_2d(b_dst + l * b_box_bytes, &p.tmB2, bar, cc * kBK, tc.n_tile * p.BN + l * 256);
      }
    }
  }
  // Do not leave while copies issued by this thread may still be landing.
  const uint32_t issued = it;
  for (uint32_t st = 0; st < static_cast<uint32_t>(p.stages) && st < issued; ++st) {
    const uint32_t last = st + ((issued - 1 - st) / p.stages) * p.stages;
    const uint32_t ph = (last / p.stages) & 1u;
    volatile int never = 0;
    mbar_wait_bounded(smem_u32(&s.full[st]), ph, &never, p.err, DEVERR_TIMEOUT_DRAIN,
                      kDrainLimitNs);
  }
}

// ----------------------------------------------------------------------- MMA
__device__ __noinline__ bool mma_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned* err) {
  return mbar_wait_bounded(bar, parity, abort_flag, err, DEVERR_TIMEOUT_MMA);
}

// S sub-tiles and HALVES weight halves are compile-time so the issue loop is
// fully unrolled: the thread must hand the next MMA to the tensor core as soon
// as it can take it.  KHT > 1 (row-halo mode): each K step runs the KHT row taps, the A operand
// shifted down by one tile row (tile_cols voxels, whole 8-row swizzle atoms)
// and the B operand moved to that tap's weight tile.
template <int S, int HALVES, int KHT>
__device__ void mma_issuer(const ConvParams& p, const Smem& s, uint32_t tmem_base) {
  const int n_inst = p.BN > 256 ? 256 : p.BN;
  const uint32_t idesc = umma_idesc_bf16(kBM, n_inst);
  // Descriptors of stage 0; the start field counts 16-byte units: stage st
  // adds stage_bytes / 16, sub-tile s adds 16 KB / 16, K step k adds 32 B / 16
  // and the second weight half 32 KB / 16.
  const uint64_t adesc0 = umma_desc_sw128(smem_u32(s.stages));
  const uint64_t bdesc0 = umma_desc_sw128(smem_u32(s.stages) + s.a_bytes);
  const uint32_t stage_step = s.stage_bytes >> 4;
  const uint32_t sub_step = (static_cast<uint32_t>(kBM) * 128u) >> 4;
  const uint32_t kh_step_a = static_cast<uint32_t>(p.tile_cols) * 8u;  // tile_cols * 128 B / 16
  const uint32_t kh_step_b = static_cast<uint32_t>(p.BN) * 8u;
  const uint32_t full0 = smem_u32(&s.full[0]), empty0 = smem_u32(&s.empty[0]);
  const uint32_t bn = static_cast<uint32_t>(p.BN);
  const uint32_t acc_cols = static_cast<uint32_t>(S) * bn;
  uint32_t st = 0, ph = 0, ai = 0;
  bool aborted = false;
  for (int tile = tile_first(p); tile < p.num_tiles && !aborted; tile += tile_stride(p), ++ai) {
    const uint32_t acc = ai % p.num_acc;
    const uint32_t aph = (ai / p.num_acc) & 1u;
    if (!mbar_wait_bounded(smem_u32(&s.tempty[acc]), aph ^ 1u, s.abort_flag, p.err,
                           DEVERR_TIMEOUT_MMA)) {
      aborted = true;
      break;
    }
    tc_fence_after();
    const uint32_t d_tmem = tmem_base + acc * acc_cols;
    for (int kb = 0; kb < p.kblocks; ++kb) {
      const uint32_t bar = full0 + st * 8u;
      if (!mbar_try_wait(bar, ph) && !mma_wait_slow(bar, ph, s.abort_flag, p.err)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const uint64_t a_st = adesc0 + st * stage_step;
      const uint64_t b_st = bdesc0 + st * stage_step;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
#pragma unroll
        for (int kh = 0; kh < KHT; ++kh) {
          const uint32_t accumulate = (kb | k | kh) != 0 ? 1u : 0u;
          const uint64_t b_k = b_st + kh * kh_step_b + 2u * k;
#pragma unroll
          for (int sub = 0; sub < S; ++sub) {
            const uint64_t a_k = a_st + sub * sub_step + kh * kh_step_a + 2u * k;
            const uint32_t d_sub = d_tmem + static_cast<uint32_t>(sub) * bn;
            umma_bf16(d_sub, a_k, b_k, idesc, accumulate);
            if (HALVES == 2) umma_bf16(d_sub + 256u, a_k, b_k + 2048u, idesc, accumulate);
          }
        }
      }
      umma_commit(empty0 + st * 8u);
      if (++st == static_cast<uint32_t>(p.stages)) {
        st = 0;
        ph ^= 1u;
      }
    }
    if (aborted) break;
    umma_commit(smem_u32(&s.tfull[acc]));
  }
  // Every MMA issued by this thread has finished before TMEM/smem go away.
  umma_commit(smem_u32(s.drain));
  volatile int never = 0;
  mbar_wait_bounded(smem_u32(s.drain), 0, &never, p.err, DEVERR_TIMEOUT_DRAIN, kDrainLimitNs);
}

// ------------------------------------------------------------------ epilogue
template <int NC>
__device__ __forceinline__ void tmem_load_chunk(uint32_t taddr, float (&v)[NC]);
template <>
__device__ __forceinline__ void tmem_load_chunk<32>(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}
template <>
__device__ __forceinline__ void tmem_load_chunk<16>(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  tmem_ld16(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

template <int NC>
__device__ __forceinline__ void add_residual(const ConvEpilogue& ep, size_t off, float (&v)[NC]) {
  if (ep.residual_f32) {
    const float4* r = reinterpret_cast<const float4*>(static_cast<const float*>(ep.residual) + off);
#pragma unroll
    for (int q = 0; q < NC / 4; ++q) {
      float4 f = r[q];
      v[4 * q] += f.x;
      v[4 * q + 1] += f.y;
      v[4 * q + 2] += f.z;
      v[4 * q + 3] += f.w;
    }
  } else {
    const uint4* r =
        reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(ep.residual) + off);
#pragma unroll
    for (int q = 0; q < NC / 8; ++q) {
      uint4 u = r[q];
      v[8 * q + 0] += bf16lo(u.x);
      v[8 * q + 1] += bf16hi(u.x);
      v[8 * q + 2] += bf16lo(u.y);
      v[8 * q + 3] += bf16hi(u.y);
      v[8 * q + 4] += bf16lo(u.z);
      v[8 * q + 5] += bf16hi(u.z);
      v[8 * q + 6] += bf16lo(u.w);
      v[8 * q + 7] += bf16hi(u.w);
    }
  }
}

template <int NC>
__device__ __forceinline__ void store_bf16(__nv_bfloat16* dst, const float (&v)[NC]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < NC / 8; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = u;
  }
}

template <int NC>
__device__ __forceinline__ void store_f32(float* dst, const float (&v)[NC]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < NC / 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Loads columns [c0, c0 + NC) of this thread's accumulator lane and returns
// acc + bias (+ residual) in v.
template <int NC>
__device__ __forceinline__ void result_chunk(const ConvParams& p, const Smem& s, uint32_t taddr,
                                             int c0, int n0, bool valid, size_t vox,
                                             float (&v)[NC]) {
  tmem_load_chunk<NC>(taddr + c0, v);
#pragma unroll
  for (int j = 0; j < NC; ++j) v[j] += s.bias[n0 + c0 + j];
  if (p.ep.residual != nullptr && valid)
    add_residual<NC>(p.ep, vox * p.cout + n0 + c0, v);
}

template <int NC>
__device__ __forceinline__ void store_raw(const ConvParams& p, int c0, int n0, size_t ovox,
                                          const float (&v)[NC]) {
  const ConvEpilogue& ep = p.ep;
  if (ep.out != nullptr) {
    const size_t off = ovox * p.cout + n0 + c0;
    if (ep.out_f32)
      store_f32<NC>(static_cast<float*>(ep.out) + off, v);
    else
      store_bf16<NC>(static_cast<__nv_bfloat16*>(ep.out) + off, v);
  }
}

template <int NC>
__device__ __forceinline__ void store_act(const ConvParams& p, const Smem& s, int c0, int n0,
                                          size_t ovox, float rs, const float (&v)[NC]) {
  float a[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) {
    a[j] = silu_half(v[j] * rs * s.gamma[n0 + c0 + j] + s.beta[n0 + c0 + j]);
  }
  store_bf16<NC>(p.ep.act + ovox * p.cout + n0 + c0, a);
}

// Outputs that need no RMS statistic: the raw result and the video.
template <int NC>
__device__ __forceinline__ void emit_chunk(const ConvParams& p, int c0, int n0,
                                           const TileCoord& tc, int h, int w, size_t ovox,
                                           const float (&v)[NC]) {
  const ConvEpilogue& ep = p.ep;
  store_raw<NC>(p, c0, n0, ovox, v);
  if (ep.video != nullptr) {
    const int H2 = 2 * p.H, W2 = 2 * p.W;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int o = n0 + c0 + j;
      if (o < p.cout) {
        const int c = o >> 2, i = (o >> 1) & 1, jj = o & 1;
        const size_t idx =
            ((static_cast<size_t>(c) * p.T + tc.t) * H2 + 2 * h + i) * W2 + 2 * w + jj;
        ep.video[idx] = __float2bfloat16_rn(v[j]);
      }
    }
  }
}

template <int NC>
__device__ __forceinline__ void tmem_store_chunk(uint32_t taddr, const float (&v)[NC]) {
  uint32_t r[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) r[j] = __float_as_uint(v[j]);
  if constexpr (NC == 32)
    tmem_st32(taddr, r);
  else
    tmem_st16(taddr, r);
}

// First pass over columns [c_lo, c_hi) of this thread's lane when the next
// layer's norm is fused: h = acc + bias (+ residual) goes out raw (if asked),
// back into the lane (so the second pass reads neither the residual nor the
// bias again), and into the returned sum of squares.
template <int NC>
__device__ __forceinline__ void pass1_chunk(const ConvParams& p, const Smem& s, uint32_t taddr,
                                            int c0, int n0, bool valid, size_t vox, float& ss) {
  float v[NC];
  result_chunk<NC>(p, s, taddr, c0, n0, valid, vox, v);
#pragma unroll
  for (int j = 0; j < NC; ++j) ss = fmaf(v[j], v[j], ss);
  if (valid) store_raw<NC>(p, c0, n0, vox, v);
  tmem_store_chunk<NC>(taddr + c0, v);
}
__device__ __forceinline__ float lane_pass1(const ConvParams& p, const Smem& s, uint32_t taddr,
                                           int c_lo, int c_hi, int n0, bool valid, size_t vox) {
  float ss = 0.0f;
  int c0 = c_lo;
  for (; c0 + 32 <= c_hi; c0 += 32) pass1_chunk<32>(p, s, taddr, c0, n0, valid, vox, ss);
  if (c0 < c_hi) pass1_chunk<16>(p, s, taddr, c0, n0, valid, vox, ss);
  tmem_wait_st();
  return ss;
}

// Second pass: the next layer's activation SiLU(h r gamma + beta) from h in the lane.
__device__ __forceinline__ void lane_pass2(const ConvParams& p, const Smem& s, uint32_t taddr,
                                          int c_lo, int c_hi, int n0, bool valid, size_t vox,
                                          float rs) {
  int c0 = c_lo;
  for (; c0 + 32 <= c_hi; c0 += 32) {
    float v[32];
    tmem_load_chunk<32>(taddr + c0, v);
    if (valid) store_act<32>(p, s, c0, n0, vox, rs, v);
  }
  if (c0 < c_hi) {
    float v[16];
    tmem_load_chunk<16>(taddr + c0, v);
    if (valid) store_act<16>(p, s, c0, n0, vox, rs, v);
  }
}

// Single pass when no norm is fused: raw result and / or video.
__device__ __forceinline__ void lane_emit(const ConvParams& p, const Smem& s, uint32_t taddr,
                                          int c_lo, int c_hi, int n0, bool valid, size_t vox,
                                          const TileCoord& tc, int h, int w) {
  int c0 = c_lo;
  for (; c0 + 32 <= c_hi; c0 += 32) {
    float v[32];
    result_chunk<32>(p, s, taddr, c0, n0, valid, vox, v);
    if (valid) emit_chunk<32>(p, c0, n0, tc, h, w, vox, v);
  }
  if (c0 < c_hi) {
    float v[16];
    result_chunk<16>(p, s, taddr, c0, n0, valid, vox, v);
    if (valid) emit_chunk<16>(p, c0, n0, tc, h, w, vox, v);
  }
}

__device__ void epilogue(const ConvParams& p, const Smem& s, uint32_t tmem_base, int warp,
                         int lane, int crank) {
  const int q = warp & 3;           // TMEM lane quarter this warp may access
  const int grp = (warp - 2) >> 2;  // epilogue group 0 or 1
  const int row = q * 32 + lane;
  const float rootC = sqrtf(static_cast<float>(p.cout));
  const bool split_cols = p.S == 1;
  const int half = p.BN / 2;
  uint32_t ti = 0;
  for (int tile = tile_first(p); tile < p.num_tiles; tile += tile_stride(p), ++ti) {
    const uint32_t acc = ti % p.num_acc;
    const uint32_t aph = (ti / p.num_acc) & 1u;
    int ok = 0;
    if (lane == 0)
      ok = mbar_wait_bounded(smem_u32(&s.tfull[acc]), aph, s.abort_flag, p.err,
                             DEVERR_TIMEOUT_EPILOGUE)
               ? 1
               : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    __syncwarp();  // order the other lanes' reads after lane 0's acquire
    tc_fence_after();
    const TileCoord tc = decode_tile(p, tile, crank);
    const int n0 = tc.n_tile * p.BN;
    for (int sub = split_cols ? 0 : grp; sub < p.S; sub += split_cols ? 1 : 2) {
      const int idx = sub * kBM + row;  // voxel of the tile, row-major
      const int h = tc.th * p.tile_rows + idx / p.tile_cols;
      const int w = tc.tw * p.tile_cols + idx % p.tile_cols;
      const bool valid = h < p.H && w < p.W;
      // output voxel: (t, h, w), or (t, 2h + p', 2w + q') of the 2H x 2W output in phase mode
      const size_t vox = p.phases == 4
                             ? (static_cast<size_t>(tc.t) * 2 * p.H + 2 * h + (tc.phase >> 1)) *
                                       (2 * p.W) + 2 * w + (tc.phase & 1)
                             : (static_cast<size_t>(tc.t) * p.H + h) * p.W + w;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             acc * static_cast<uint32_t>(p.S * p.BN) +
                             static_cast<uint32_t>(sub * p.BN);
      const int c_lo = split_cols ? grp * half : 0;
      const int c_hi = split_cols ? c_lo + half : p.BN;
      if (p.ep.act == nullptr) {
        lane_emit(p, s, taddr, c_lo, c_hi, n0, valid, vox, tc, h, w);
      } else {
        float ss = lane_pass1(p, s, taddr, c_lo, c_hi, n0, valid, vox);
        if (p.nsplit == 2) {
          // the other half of the channels is in the peer CTA: swap partial sums
          const int slot = (ti & 1u) * 256 + sub * 128 + row;
          const uint32_t peer = static_cast<uint32_t>(crank ^ 1);
          st_shared_cluster_f32(mapa_shared(smem_u32(&s.xpart[slot]), peer), ss);
          mbar_arrive_cluster(mapa_shared(smem_u32(&s.xbar[ti & 1u]), peer));
          int got = 0;
          if (lane == 0)
            got = mbar_wait_cluster_bounded(smem_u32(&s.xbar[ti & 1u]), (ti >> 1) & 1u,
                                            s.abort_flag, p.err, DEVERR_TIMEOUT_EPILOGUE)
                      ? 1
                      : 0;
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) return;
          __syncwarp();
          ss += s.xpart[slot];
        } else if (split_cols) {
          // exchange the two halves' sums through shared memory (bounded wait)
          float* part = s.ss_part + (ti & 1u) * 256;
          part[grp * 128 + row] = ss;
          mbar_arrive(smem_u32(s.ssbar));
          int got = 0;
          if (lane == 0)
            got = mbar_wait_bounded(smem_u32(s.ssbar), ti & 1u, s.abort_flag, p.err,
                                    DEVERR_TIMEOUT_EPILOGUE)
                      ? 1
                      : 0;
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) return;
          __syncwarp();
          ss += part[(grp ^ 1) * 128 + row];
        }
        const float rs = rootC / fmaxf(sqrtf(ss), p.ep.eps);
        lane_pass2(p, s, taddr, c_lo, c_hi, n0, valid, vox, rs);
      }
    }
    tc_fence_before();
    mbar_arrive(smem_u32(&s.tempty[acc]));
  }
}

__global__ void __launch_bounds__(kConvThreads, 1) conv_tc_kernel(const __grid_constant__ ConvParams p) {
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve(smem_raw, p);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(smem_u32(&s.full[i]), 1);
      mbar_init(smem_u32(&s.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s.tfull[i]), 1);
      mbar_init(smem_u32(&s.tempty[i]), 256);
    }
    mbar_init(smem_u32(s.drain), 1);
    mbar_init(smem_u32(s.ssbar), 256);
    mbar_init(smem_u32(&s.xbar[0]), 256);  // 256 epilogue threads of the peer CTA
    mbar_init(smem_u32(&s.xbar[1]), 256);
    *s.abort_flag = 0;
    fence_mbar_init();
  }
  // Per-channel vectors for every output channel (a CTA may visit several
  // n-slices); the shortcut bias folds into the bias.
  for (int i = threadIdx.x; i < p.cout_pad; i += blockDim.x) {
    s.bias[i] = p.ep.bias[i] + (p.ep.bias2 != nullptr ? p.ep.bias2[i] : 0.0f);
    if (p.ep.act != nullptr && i < p.cout) {
      // halved for silu_half
      s.gamma[i] = 0.5f * p.ep.gamma[i];
      s.beta[i] = 0.5f * p.ep.beta[i];
    }
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
  // With a CTA pair, both CTAs' barriers exist before either writes to the other.
  if (p.nsplit == 2) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;
  const int crank = p.nsplit == 2 ? static_cast<int>(cluster_ctarank()) : 0;

  if (warp == 0) {
    if (lane == 0) producer(p, s, crank);
  } else if (warp == 1) {
    if (lane == 0) {
      if (p.rowhalo)
        mma_issuer<2, 1, 3>(p, s, tmem_base);
      else if (p.BN > 256)
        mma_issuer<1, 2, 1>(p, s, tmem_base);
      else if (p.S == 1)
        mma_issuer<1, 1, 1>(p, s, tmem_base);
      else if (p.S == 2)
        mma_issuer<2, 1, 1>(p, s, tmem_base);
      else
        mma_issuer<4, 1, 1>(p, s, tmem_base);
    }
  } else {
    epilogue(p, s, tmem_base, warp, lane, crank);
  }

  tc_fence_before();
  __syncthreads();
  // Neither CTA of a pair leaves while the other may still write into it.
  if (p.nsplit == 2) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace

size_t conv_tc_smem_bytes(const ConvParams& p, int stages) {
  const size_t stage = static_cast<size_t>(conv_tc_a_bytes(p)) + conv_tc_b_bytes(p);
  return 1024 + stages * stage + kCtrlBytes;
}

int conv_tc_stages_for(const ConvParams& p) {
  const size_t limit = 232448;  // 227 KB opt-in dynamic shared memory per block
  int st = kMaxStages;
  while (st > 2 && conv_tc_smem_bytes(p, st) > limit) --st;
  return st;
}

namespace {
size_t launch_smem(const ConvParams& p) {
  // Every CTA allocates all 512 TMEM columns, so exactly one may live on an SM:
  // ask for more than half of the SM's shared memory even when the ring is small.
  size_t smem = conv_tc_smem_bytes(p, p.stages);
  if (smem < 120 * 1024) smem = 120 * 1024;
  return smem;
}

cudaLaunchConfig_t launch_config(const ConvParams& p, int grid, size_t smem, cudaStream_t stream,
                                 cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kConvThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.nsplit == 2 ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
}  // namespace

int conv_tc_max_clusters(const ConvParams& p) {
  const size_t smem = launch_smem(p);
  if (cudaFuncSetAttribute(conv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_config(p, 2, smem, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, conv_tc_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_conv_tc(const ConvParams& p, int grid, cudaStream_t stream) {
  const size_t smem = launch_smem(p);
  cudaError_t e = cudaFuncSetAttribute(conv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_config(p, grid, smem, stream, attr);
  e = cudaLaunchKernelEx(&cfg, conv_tc_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace wvae

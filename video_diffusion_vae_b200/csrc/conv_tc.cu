// Causal conv3d as an implicit GEMM on the sm_100a tensor cores.
//
//   out[m, n] = sum_k A[m, k] * B[n, k]
//   m: an output voxel (t, h, w);  n: an output channel;
//   k: (tap, input channel), tap = (kt, kh, kw) over the KT x KH x KW window.
//   A[m, (tap, i)] = a[t + kt - (KT-1), h + kh - (KH-1)/2, w + kw - (KW-1)/2, i]
//
// The causal front frames and the spatial border are zero (or, for t' < 0, the
// previous chunk's cached frames).  No padded copy exists: every A load is one
// TMA box of the channels-last activation at tap-shifted coordinates, and the
// tensor map's out-of-bounds fill supplies the zeros.  (Conv definition:
// FastVideo "Wan2.2 VAE decoder (sm_100a, sm_103a)" README, "Limits": bf16
// operands, fp32 accumulation; temporal caching: TensorRT-LLM issue #19309,
// "Feature, motivation and proposed scope".)
//
// One CTA per SM, persistent over output tiles of tile_rows x tile_cols voxels
// of one frame (128 S voxels: S MMA sub-tiles of 128 consecutive voxels in
// row-major order; the shape is chosen per layer to balance the waves) x BN
// output channels.  The reduction runs in K groups (kt, column tap kw, 64
// input channels).  Warp roles:
//   warp 0      TMA producer: per group one A window {64 ch, tile_cols w,
//               tile_rows + KH - 1 h, 1 t} (the tile plus its row-tap halo)
//               into the A ring, and the KH weight tiles {64, BN} of the
//               group's row taps into the B ring;
//   warp 1      MMA issuer: per weight tile (row tap kh), 4 K steps x S
//               sub-tiles of tcgen05.mma (M=128, N=BN<=256, K=16) whose A
//               operand starts kh tile rows into the window (whole 8-row
//               swizzle atoms, so no copy), into TMEM (two accumulators when
//               2 S BN <= 512: the epilogue of tile i overlaps the main loop
//               of tile i+1);
//   warps 2..9  epilogue, two groups of 4 warps (one warp per TMEM lane
//               quarter each) taking alternate sub-tiles: one TMEM lane = one
//               output voxel per thread.
// The row-tap windows load each input row about once per (kt, kw) instead of
// once per tap, which keeps the refill of shared memory from L2 off the
// critical path.
// 512 output channels with the next layer's norm fused: a cluster of two CTAs
// splits N (each runs the S = 2, BN = 256 main loop on its half of the
// channels for the same M tiles) and the two epilogues exchange each voxel's
// partial sum of squares through distributed shared memory.
// One N tile of 128 or 256 channels per CTA (no shortcut, not Winograd): a
// cluster of two CTAs shares M = 256 MMAs (conv_tc_kernel<true>,
// tcgen05.mma.cta_group::2): each CTA keeps its own tile and A windows and
// loads half of every weight tile, rank 0 issues the MMAs and multicasts its
// commits to both CTAs, and both epilogues release the accumulator on rank
// 0's barrier.
// tcgen05.mma issue runs nearly in step with execution, so every cycle the
// issuing thread spends waiting on a barrier is a tensor-pipe bubble: S
// sub-tiles per weight tile put S times more MMA work behind each wait.
// The upsample convs on CTA pairs and the pair layers whose one accumulator is
// released after epilogue pass 1 (conv_tc_staged_kernel) write their outputs
// through shared memory: each epilogue warp stages a 32-channel chunk of its 32
// voxels in a 4 KB buffer and one lane issues TMA stores of its two 16-voxel
// row segments, where per-lane stores of voxel rows kept the load/store pipe
// busy for 70 % of the upsample convs' time (their four phases write fp32 +
// bf16 outputs four times the input's size).
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
  uint8_t* a_ring;        // A stage i at a_ring + i * a_bytes, 1024-aligned
  uint8_t* b_ring;        // B stage j at b_ring + j * b_bytes, 1024-aligned
  uint32_t stage;         // staged-store buffers (tma_out): kStageWarpBytes per epilogue warp
  uint32_t a_bytes, b_bytes;
  uint64_t* full_a;       // [kMaxStages]
  uint64_t* empty_a;      // [kMaxStages]
  uint64_t* full_b;       // [kMaxStages]
  uint64_t* empty_b;      // [kMaxStages]
  uint64_t* tfull;        // [2]
  uint64_t* tempty;       // [2]
  uint64_t* drain;        // [1]
  uint64_t* xbar;         // [2] (per tile parity) the peer CTA's partial sums have arrived
  float* xpart;           // [2 tile parities][256]: partial sums written by the peer CTA
  uint32_t* tmem_slot;
  int* abort_flag;
  float* bias;            // [512]
  float* gamma;           // [512]
  float* beta;            // [512]
};

constexpr uint32_t kCtrlBytes = 512 + 3 * 512 * 4 + 2 * 256 * 4;

__device__ __forceinline__ Smem carve(uint8_t* raw, const ConvParams& p) {
  Smem s;
  uint32_t base = smem_u32(raw);
  uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* al = raw + pad;
  s.a_bytes = conv_tc_a_bytes(p);
  s.b_bytes = conv_tc_b_bytes(p);
  s.a_ring = al;
  s.b_ring = al + p.stages_a * s.a_bytes;
  uint8_t* stage = s.b_ring + p.stages_b * s.b_bytes;  // 1024-aligned: whole 1 KB stages
  s.stage = smem_u32(stage);
  uint8_t* ctrl = stage + conv_tc_stage_bytes(p);
  s.full_a = reinterpret_cast<uint64_t*>(ctrl);
  s.empty_a = s.full_a + kMaxStages;
  s.full_b = s.empty_a + kMaxStages;
  s.empty_b = s.full_b + kMaxStages;
  s.tfull = s.empty_b + kMaxStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.xbar = s.drain + 1;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.xbar + 2);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_slot + 1);
  s.bias = reinterpret_cast<float*>(ctrl + 512);
  s.gamma = s.bias + 512;
  s.beta = s.gamma + 512;
  s.xpart = s.beta + 512;
  return s;
}

struct TileCoord {
  int n_tile, phase, t, th, tw;
};

// Tile order: N tile fastest, then upsample phase (the four phases of an M
// tile read the same input), then frame (the KT temporal taps of neighbouring
// frames read the same input frames: a frame of a large layer does not stay
// in L2 until the next frame's tiles come round), then tile column and row.
// With nsplit = 2 the two CTAs of a cluster take the same tiles and the CTA
// rank is the N tile.  With a pair, loop index t names an (N tile, phase) and
// a pair of spatial M tiles: rank r takes spatial tile 2i + r (both CTAs of a
// pair multiply by the same weights); when the count of spatial tiles is odd
// the last pair's rank 1 takes a copy of the last one so that the pair's MMAs
// stay whole, and writes nothing (tile_own).
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
  if (p.pair) {
    m = 2 * m + crank;
    if (m >= p.m_tiles) m = p.m_tiles - 1;
  }
  c.t = m % p.T;
  m /= p.T;
  c.tw = m % p.tiles_w;
  c.th = m / p.tiles_w;
  return c;
}

// ------------------------------------------------------------------ producer
// Every role walks the same sequence of loop indices: tile_first, then steps
// of tile_stride, below tile_count; the two CTAs of a cluster (nsplit = 2 or
// a pair) share each index (decode_tile).
__device__ __forceinline__ bool cluster2(const ConvParams& p) { return p.nsplit == 2 || p.pair; }
__device__ __forceinline__ int tile_first(const ConvParams& p) {
  return cluster2(p) ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
}
__device__ __forceinline__ int tile_stride(const ConvParams& p) {
  return cluster2(p) ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
}
__device__ __forceinline__ int tile_count(const ConvParams& p) {
  return p.pair ? ((p.m_tiles + 1) >> 1) * p.phases * p.n_tiles : p.num_tiles;
}
__device__ __forceinline__ bool tile_own(const ConvParams& p, int t, int crank) {
  return !p.pair || 2 * (t / (p.n_tiles * p.phases)) + crank < p.m_tiles;
}

// Waits, bounded, until every copy this thread issued into a ring has landed.
__device__ void drain_ring(const uint64_t* full, uint32_t issued, int stages, unsigned* err) {
  for (uint32_t st = 0; st < static_cast<uint32_t>(stages) && st < issued; ++st) {
    const uint32_t last = st + ((issued - 1 - st) / stages) * stages;
    volatile int never = 0;
    mbar_wait_bounded(smem_u32(&full[st]), (last / stages) & 1u, &never, err, DEVERR_TIMEOUT_DRAIN,
                      kDrainLimitNs);
  }
}

// K group = (kt, column tap kw, 64 input channels): one A window holding the
// tile's rows plus the row-tap halo goes to the A ring, then the kh_eff weight
// tiles of taps (kt, 0..kh_eff-1, kw) to the B ring, b_tiles per stage.  A
// second-segment group (1x1x1 shortcut) is one A tile without halo and one
// weight tile (alone in its B stage).
template <bool PAIR>
__device__ void producer(const ConvParams& p, const Smem& s, int crank) {
  const int cchunks = p.cin_pad / kBK;
  const uint32_t a_tx_main = conv_tc_a_rows(p) * static_cast<uint32_t>(p.tile_cols) * 128u;
  const uint32_t a_tx_sc = static_cast<uint32_t>(p.tile_rows * p.tile_cols) * 128u;
  const uint32_t tile_tx = static_cast<uint32_t>(conv_tc_b_rows(p)) * 128u;
  const int kw_stride = p.kw_eff * p.nw;  // tap = ((kt kh_eff + kh) kw_stride + kw) (+ phase)
  // With a pair each CTA loads its own A window and half of each weight tile;
  // both halves complete on rank 0's barrier, which rank 0 alone arms for the
  // bytes of both CTAs.
  const int b_row0 = PAIR ? crank * conv_tc_b_rows(p) : 0;
  const bool arms = !PAIR || crank == 0;
  const uint32_t tx_mul = PAIR ? 2u : 1u;
  auto bar_of = [&](const uint64_t* b) {
    if constexpr (PAIR)
      return mapa_shared(smem_u32(b), 0);
    else
      return smem_u32(b);
  };
  auto load4 = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0, int c1, int c2, int c3) {
    if constexpr (PAIR)
      tma_load_4d_pair(dst, m, bar, c0, c1, c2, c3);
    else
      tma_load_4d(dst, m, bar, c0, c1, c2, c3);
  };
  uint32_t ia = 0, ib = 0;
  bool aborted = false;
  for (int tile = tile_first(p); tile < tile_count(p) && !aborted; tile += tile_stride(p)) {
    const TileCoord tc = decode_tile(p, tile, crank);
    const int h0 = tc.th * p.tile_rows, w0 = tc.tw * p.out_cols;
    // output (h, w) reads input row h + oh + kh and column w + ow + kw; phase
    // mode: output (2h+p', 2w+q') reads rows h + p' - 1 + r, columns w + q' - 1 + c
    const int oh = p.phases == 4 ? (tc.phase >> 1) - 1 : -(p.KH - 1) / 2;
    const int ow = p.phases == 4 ? (tc.phase & 1) - 1 : -(p.KW - 1) / 2;
    // phase mode: phase p's 4 taps; Winograd: transform plane xi's KT temporal taps
    const int tap0 = p.phases == 4 ? tc.phase * 4 : (p.wino ? tc.phase * p.KT : 0);
    for (int g = 0; g < p.groups; ++g) {
      const bool main_seg = g < p.groups_main;
      int kt = 0, kw = 0, cc;
      if (main_seg) {
        const int tw = g / cchunks;
        cc = g - tw * cchunks;
        kt = tw / p.kw_eff;
        kw = tw - kt * p.kw_eff;
      } else {
        cc = g - p.groups_main;
      }
      const uint32_t a_tx = main_seg ? a_tx_main : a_tx_sc;
      // the A window of the group (on its own barrier, or on the B stage's)
      auto load_a = [&](uint32_t dst, uint32_t bar) {
        if (main_seg) {
          const int ts = tc.t + kt - (p.KT - 1);
          if (p.wino)
            tma_load_5d(dst, &p.tmA, bar, cc * kBK, w0, h0, ts, tc.phase);
          else if (ts < 0 && p.has_cache)
            load4(dst, &p.tmC, bar, cc * kBK, w0 + ow + kw, h0 + oh, ts + p.KT - 1);
          else
            load4(dst, &p.tmA, bar, cc * kBK, w0 + ow + kw, h0 + oh, ts);
        } else {
          load4(dst, &p.tmA2, bar, cc * kBK, w0, h0, tc.t);
        }
      };
      if (!p.combined) {
        const uint32_t st = ia % p.stages_a, ph = (ia / p.stages_a) & 1u;
        if (!mbar_wait_bounded(smem_u32(&s.empty_a[st]), ph ^ 1u, s.abort_flag, p.err,
                               DEVERR_TIMEOUT_PRODUCER)) {
          aborted = true;
          break;
        }
        const uint32_t bar = bar_of(&s.full_a[st]);
        if (arms) mbar_arrive_expect_tx(smem_u32(&s.full_a[st]), tx_mul * a_tx);
        load_a(smem_u32(s.a_ring + st * s.a_bytes), bar);
        ++ia;
      }
      const int nkh = main_seg ? p.kh_eff : 1;
      const int per_stage = main_seg ? p.b_tiles : 1;
      for (int kh0 = 0; kh0 < nkh; kh0 += per_stage, ++ib) {
        const uint32_t st = ib % p.stages_b, ph = (ib / p.stages_b) & 1u;
        if (!mbar_wait_bounded(smem_u32(&s.empty_b[st]), ph ^ 1u, s.abort_flag, p.err,
                               DEVERR_TIMEOUT_PRODUCER)) {
          aborted = true;
          break;
        }
        const uint32_t bar = bar_of(&s.full_b[st]);
        const uint32_t dst = smem_u32(s.b_ring + st * s.b_bytes);
        const uint32_t b_tx = main_seg ? s.b_bytes : tile_tx;
        if (p.combined) {
          // one stage per group: A slot st travels with B slot st on one barrier
          if (arms) mbar_arrive_expect_tx(smem_u32(&s.full_b[st]), tx_mul * (a_tx + b_tx));
          load_a(smem_u32(s.a_ring + st * s.a_bytes), bar);
        } else if (arms) {
          mbar_arrive_expect_tx(smem_u32(&s.full_b[st]), tx_mul * b_tx);
        }
        auto load_b = [&](uint32_t d, const CUtensorMap* m, int c0, int c1) {
          if constexpr (PAIR)
            tma_load_2d_pair(d, m, bar, c0, c1);
          else
            tma_load_2d(d, m, bar, c0, c1);
        };
        if (main_seg) {
          // weight tiles [row tap j][column tap u], BN rows each (BN / 2 with a pair)
          for (int j = 0; j < per_stage; ++j)
            for (int u = 0; u < p.nw; ++u) {
              const int tap = tap0 + (kt * p.kh_eff + kh0 + j) * kw_stride + kw + u;
              load_b(dst + (j * p.nw + u) * tile_tx, &p.tmB, tap * p.cin_pad + cc * kBK,
                     tc.n_tile * p.BN + b_row0);
            }
        } else {
          load_b(dst, &p.tmB2, cc * kBK, tc.n_tile * p.BN + b_row0);
        }
      }
      if (aborted) break;
    }
  }
  // Do not leave while copies issued by this thread may still be landing.  A
  // pair's rank 1 has no barriers of its own for them: rank 0 drains the
  // shared ones, and neither CTA leaves before the other (the kernel's last
  // cluster barrier).
  if (PAIR && crank != 0) return;
  drain_ring(s.full_a, ia, p.stages_a, p.err);
  drain_ring(s.full_b, ib, p.stages_b, p.err);
}

// ----------------------------------------------------------------------- MMA
__device__ __noinline__ bool mma_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned* err) {
  return mbar_wait_bounded(bar, parity, abort_flag, err, DEVERR_TIMEOUT_MMA);
}

// S sub-tiles, KHT row taps and BT weight tiles per B stage are compile-time
// so the issue loop is fully unrolled: the thread must hand the next MMA to
// the tensor core as soon as it can take it.  Per weight tile (row tap kh),
// 4 K steps x S sub-tiles of M=128 x N=BN x K=16; the A operand of row tap kh
// starts kh tile rows (kh * tile_cols voxels, whole 8-row swizzle atoms) into
// the A window.
__device__ __forceinline__ bool mma_wait(uint32_t bar, uint32_t ph, const Smem& s,
                                         const ConvParams& p) {
  return mbar_try_wait(bar, ph) || mma_wait_slow(bar, ph, s.abort_flag, p.err);
}

// COMBINED: a group's A window and weight tiles share one stage and barrier.
// PAIR: M = 256 MMAs over the CTA pair (issued by rank 0 only), commits
// multicast to the barriers of both CTAs.
template <int S, int KHT, int BT, bool COMBINED, bool PAIR>
__device__ void mma_issuer(const ConvParams& p, const Smem& s, uint32_t tmem_base) {
  static_assert(BT == 1 || BT == KHT, "a B stage holds one weight tile or the group's row taps");
  static_assert(!COMBINED || BT == KHT, "a combined stage holds all of a group's weight tiles");
  const uint32_t n_mma = static_cast<uint32_t>(p.nw * p.BN);  // N of one MMA
  const int m_mma = PAIR ? 2 * kBM : kBM;
  const uint32_t idesc = p.wino ? umma_idesc_f16(m_mma, static_cast<int>(n_mma))
                                : umma_idesc_bf16(m_mma, static_cast<int>(n_mma));
  auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    if constexpr (PAIR)
      umma_bf16_pair(d, a, b, idesc, acc);
    else
      umma_bf16(d, a, b, idesc, acc);
  };
  auto commit = [&](uint32_t bar) {
    if constexpr (PAIR)
      umma_commit_pair_both(bar);
    else
      umma_commit(bar);
  };
  // Descriptors of stage 0 of each ring; the start field counts 16-byte units.
  const uint64_t adesc0 = umma_desc_sw128(smem_u32(s.a_ring));
  const uint64_t bdesc0 = umma_desc_sw128(smem_u32(s.b_ring));
  const uint32_t a_step = s.a_bytes >> 4, b_step = s.b_bytes >> 4;
  const uint32_t sub_step = (static_cast<uint32_t>(kBM) * 128u) >> 4;
  const uint32_t kh_step = static_cast<uint32_t>(p.tile_cols) * 8u;  // tile_cols * 128 B / 16
  // one row tap's weight tiles in the B stage: nw x (BN, or BN / 2 with a pair) rows x 128 B / 16
  const uint32_t tap_step = static_cast<uint32_t>(p.nw * conv_tc_b_rows(p)) * 8u;
  const uint32_t full_a0 = smem_u32(&s.full_a[0]), empty_a0 = smem_u32(&s.empty_a[0]);
  const uint32_t full_b0 = smem_u32(&s.full_b[0]), empty_b0 = smem_u32(&s.empty_b[0]);
  const uint32_t n_stride = conv_tc_acc_stride(p);  // TMEM columns per sub-tile
  const uint32_t acc_cols = static_cast<uint32_t>(S) * n_stride;
  uint32_t sa = 0, pa = 0, sb = 0, pb = 0, ai = 0;
  bool aborted = false;
  for (int tile = tile_first(p); tile < tile_count(p) && !aborted; tile += tile_stride(p), ++ai) {
    const uint32_t acc = ai % p.num_acc;
    const uint32_t aph = (ai / p.num_acc) & 1u;
    if (!mbar_wait_bounded(smem_u32(&s.tempty[acc]), aph ^ 1u, s.abort_flag, p.err,
                           DEVERR_TIMEOUT_MMA)) {
      aborted = true;
      break;
    }
    tc_fence_after();
    const uint32_t d_tmem = tmem_base + acc * acc_cols;
    for (int g = 0; g < p.groups && !aborted; ++g) {
      if (!COMBINED && !mma_wait(full_a0 + sa * 8u, pa, s, p)) {
        aborted = true;
        break;
      }
      const uint64_t a_st = adesc0 + (COMBINED ? sb : sa) * a_step;
      const uint32_t first = g == 0 ? 0u : 1u;  // the tile's first MMA overwrites
      // MMAs of row tap kh (A rows kh.., weight tile j of the B stage)
      auto issue = [&](int kh, int j) {
        const uint64_t a_kh = a_st + kh * kh_step;
        const uint64_t b_st = bdesc0 + sb * b_step + j * tap_step;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint32_t accumulate = (k | kh) != 0 ? 1u : first;
#pragma unroll
          for (int sub = 0; sub < S; ++sub)
            mma(d_tmem + static_cast<uint32_t>(sub) * n_stride, a_kh + sub * sub_step + 2u * k,
                b_st + 2u * k, accumulate);
        }
      };
      auto release_b = [&]() {
        commit(empty_b0 + sb * 8u);
        if (++sb == static_cast<uint32_t>(p.stages_b)) {
          sb = 0;
          pb ^= 1u;
        }
      };
      if (g < p.groups_main) {
#pragma unroll
        for (int kh = 0; kh < KHT; ++kh) {
          if (kh % BT == 0) {
            if (!mma_wait(full_b0 + sb * 8u, pb, s, p)) {
              aborted = true;
              break;
            }
            tc_fence_after();
          }
          issue(kh, kh % BT);
          if (kh % BT == BT - 1) release_b();
        }
      } else {
        // second segment: one weight tile, A without halo
        if (!mma_wait(full_b0 + sb * 8u, pb, s, p)) {
          aborted = true;
        } else {
          tc_fence_after();
          issue(0, 0);
          release_b();
        }
      }
      if (aborted) break;
      if (!COMBINED) {
        commit(empty_a0 + sa * 8u);
        if (++sa == static_cast<uint32_t>(p.stages_a)) {
          sa = 0;
          pa ^= 1u;
        }
      }
    }
    if (aborted) break;
    commit(smem_u32(&s.tfull[acc]));
  }
  // Every MMA issued by this thread has finished before TMEM/smem go away.
  if constexpr (PAIR)
    umma_commit_pair_local(smem_u32(s.drain));
  else
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
  if (ep.vec32) {
    if (ep.residual_f32) {
      const float* r = static_cast<const float*>(ep.residual) + off;
#pragma unroll
      for (int q = 0; q < NC / 8; ++q) {
        uint32_t u[8];
        ld_global_v8(r + 8 * q, u);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * q + e] += __uint_as_float(u[e]);
      }
    } else {
      const __nv_bfloat16* r = static_cast<const __nv_bfloat16*>(ep.residual) + off;
#pragma unroll
      for (int q = 0; q < NC / 16; ++q) {
        uint32_t u[8];
        ld_global_v8(r + 16 * q, u);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[16 * q + 2 * e] += bf16lo(u[e]);
          v[16 * q + 2 * e + 1] += bf16hi(u[e]);
        }
      }
    }
    return;
  }
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
__device__ __forceinline__ void store_bf16(__nv_bfloat16* dst, const float (&v)[NC], bool vec32) {
  if (vec32) {
#pragma unroll
    for (int q = 0; q < NC / 16; ++q) {
      uint32_t u[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) u[e] = pack_bf16x2(v[16 * q + 2 * e], v[16 * q + 2 * e + 1]);
      st_global_v8(dst + 16 * q, u);
    }
    return;
  }
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
__device__ __forceinline__ void store_f16(__half* dst, const float (&v)[NC]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < NC / 8; ++q)
    d[q] = make_uint4(pack_f16x2(v[8 * q], v[8 * q + 1]), pack_f16x2(v[8 * q + 2], v[8 * q + 3]),
                      pack_f16x2(v[8 * q + 4], v[8 * q + 5]), pack_f16x2(v[8 * q + 6], v[8 * q + 7]));
}

template <int NC>
__device__ __forceinline__ void store_f32(float* dst, const float (&v)[NC], bool vec32) {
  if (vec32) {
#pragma unroll
    for (int q = 0; q < NC / 8; ++q) {
      uint32_t u[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) u[e] = __float_as_uint(v[8 * q + e]);
      st_global_v8(dst + 8 * q, u);
    }
    return;
  }
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < NC / 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// ---- staged stores (tma_out)
// A warp's 32 voxels (one per lane) x 32 channels go through the warp's own
// shared buffer, one row per voxel (fp32 rows of 128 B, bf16 rows of 64 B)
// with the 16-byte pieces XOR-swizzled where the tensor map's 128B / 64B
// swizzle expects them, so each 16-byte shared store of 8 lanes covers all 32
// banks once.  Lane 0 then writes the two 16-voxel halves (each inside one
// tile row) with one TMA store each.  Per-lane global stores of voxel rows
// touch 32 cache lines per warp instruction, and on the layers with large
// outputs they kept the load/store pipe busy for most of the kernel's time.
struct StoreRows {  // this lane's voxel as a box origin (lanes 0 and 16 are read)
  int ok;           // written: own tile, inside H x W and inside the row window
  int q;            // column phase (phase mode), else 0
  int w, r, r2;     // box coordinates: column, row of the [rows][W] view, and the
                    // row of the second output frame (temporal 2x copies) or -1
};

struct Stage {
  uint32_t buf;  // this warp's buffer
  int lane;
  StoreRows sr;
};

// The buffer is free once the previous chunk's bulk stores have read it.  (A
// second buffer per warp, so that this waits on the chunk before that, measured
// no faster: the wait is not what holds the epilogue up.)
__device__ __forceinline__ void stage_acquire(const Stage& st) {
  if (st.lane == 0) bulk_wait_read_all();
  __syncwarp();
}

__device__ __forceinline__ void stage_f32(const Stage& st, const float (&v)[32]) {
  const uint32_t row = st.buf + static_cast<uint32_t>(st.lane) * 128u;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    st_shared_v4(row + (static_cast<uint32_t>((j ^ st.lane) & 7) << 4), __float_as_uint(v[4 * j]),
                 __float_as_uint(v[4 * j + 1]), __float_as_uint(v[4 * j + 2]),
                 __float_as_uint(v[4 * j + 3]));
}

__device__ __forceinline__ void stage_b16(const Stage& st, const uint32_t (&u)[16]) {
  const uint32_t row = st.buf + static_cast<uint32_t>(st.lane) * 64u;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    st_shared_v4(row + (static_cast<uint32_t>((j ^ (st.lane >> 1)) & 3) << 4), u[4 * j],
                 u[4 * j + 1], u[4 * j + 2], u[4 * j + 3]);
}

// seg_bytes: bytes of 16 staged rows (2048 fp32, 1024 bf16); x: the first channel.
__device__ __forceinline__ void stage_commit(const Stage& st, const CUtensorMap* tm,
                                             uint32_t seg_bytes, int x) {
  fence_proxy_async_smem();  // this lane's shared stores before the async proxy reads them
  __syncwarp();
  const StoreRows& a = st.sr;
  const int ok1 = __shfl_sync(0xffffffffu, a.ok, 16);
  const int w1 = __shfl_sync(0xffffffffu, a.w, 16);
  const int r1 = __shfl_sync(0xffffffffu, a.r, 16);
  const int rr1 = __shfl_sync(0xffffffffu, a.r2, 16);
  if (st.lane == 0) {
    if (a.ok) {
      tma_store_4d(tm, st.buf, x, a.q, a.w, a.r);
      if (a.r2 >= 0) tma_store_4d(tm, st.buf, x, a.q, a.w, a.r2);
    }
    if (ok1) {
      tma_store_4d(tm, st.buf + seg_bytes, x, a.q, w1, r1);
      if (rr1 >= 0) tma_store_4d(tm, st.buf + seg_bytes, x, a.q, w1, rr1);
    }
    bulk_commit_group();
  }
}

// The raw result chunk (fp32 or bf16) through the buffer.
__device__ __forceinline__ void stage_raw(const ConvParams& p, Stage& st, int x,
                                          const float (&v)[32]) {
  stage_acquire(st);
  if (p.ep.out_f32) {
    stage_f32(st, v);
    stage_commit(st, &p.tmO, 2048, x);
  } else {
    uint32_t u[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) u[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
    stage_b16(st, u);
    stage_commit(st, &p.tmO, 1024, x);
  }
}

// Loads columns [c0, c0 + NC) of this thread's accumulator lane and returns
// acc + bias (+ residual) in v.
template <int NC>
__device__ __forceinline__ void result_chunk(const ConvParams& p, const Smem& s, uint32_t taddr,
                                             int c0, int n0, bool valid, size_t vox,
                                             float (&v)[NC]) {
  tmem_load_chunk<NC>(taddr + c0, v);
#pragma unroll
  for (int q = 0; q < NC / 4; ++q) {  // 128-bit shared loads of the bias
    const float4 bq = reinterpret_cast<const float4*>(s.bias + n0 + c0)[q];
    v[4 * q] += bq.x;
    v[4 * q + 1] += bq.y;
    v[4 * q + 2] += bq.z;
    v[4 * q + 3] += bq.w;
  }
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
      store_f32<NC>(static_cast<float*>(ep.out) + off, v, ep.vec32 != 0);
    else if (ep.out_f16)
      store_f16<NC>(static_cast<__half*>(ep.out) + off, v);
    else
      store_bf16<NC>(static_cast<__nv_bfloat16*>(ep.out) + off, v, ep.vec32 != 0);
  }
}

// The next layer's activation bf16 pairs: SiLU_half((v rs) gamma/2 + beta/2).
template <int NC>
__device__ __forceinline__ void act_words(const ConvParams& p, const Smem& s, int c0, int n0,
                                          float rs, const float (&v)[NC], uint32_t (&u)[NC / 2]) {
  const float2 r2 = make_float2(rs, rs);
  const float4* g4 = reinterpret_cast<const float4*>(s.gamma + n0 + c0);
  const float4* b4 = reinterpret_cast<const float4*>(s.beta + n0 + c0);
#pragma unroll
  for (int e = 0; e < NC / 2; ++e) {  // channel pair e as two lanes of a 128-bit load
    const float4 g = g4[e >> 1], b = b4[e >> 1];
    const float2 g2 = (e & 1) ? make_float2(g.z, g.w) : make_float2(g.x, g.y);
    const float2 b2 = (e & 1) ? make_float2(b.z, b.w) : make_float2(b.x, b.y);
    const float2 o = silu_half2(ffma2(fmul2(make_float2(v[2 * e], v[2 * e + 1]), r2), g2, b2));
    u[e] = pack_bf16x2(o.x, o.y);
  }
}

template <int NC>
__device__ __forceinline__ void store_act(const ConvParams& p, const Smem& s, int c0, int n0,
                                          size_t ovox, float rs, const float (&v)[NC]) {
  // packed pairs: SiLU_half((v rs) gamma/2 + beta/2)
  const float2 r2 = make_float2(rs, rs);
  const float4* g4 = reinterpret_cast<const float4*>(s.gamma + n0 + c0);
  const float4* b4 = reinterpret_cast<const float4*>(s.beta + n0 + c0);
  auto g2 = [&](int i) {  // channel pair i as two lanes of a 128-bit load
    const float4 g = g4[i >> 1];
    return (i & 1) ? make_float2(g.z, g.w) : make_float2(g.x, g.y);
  };
  auto b2 = [&](int i) {
    const float4 b = b4[i >> 1];
    return (i & 1) ? make_float2(b.z, b.w) : make_float2(b.x, b.y);
  };
  __nv_bfloat16* dst = p.ep.act + ovox * p.cout + n0 + c0;
  if (p.ep.vec32) {
#pragma unroll
    for (int q = 0; q < NC / 16; ++q) {
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = 16 * q + 2 * e;
        const float2 o =
            silu_half2(ffma2(fmul2(make_float2(v[j], v[j + 1]), r2), g2(j / 2), b2(j / 2)));
        w[e] = pack_bf16x2(o.x, o.y);
      }
      st_global_v8(dst + 16 * q, w);
    }
    return;
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < NC / 8; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 8 * q + 2 * e;
      const float2 o =
          silu_half2(ffma2(fmul2(make_float2(v[j], v[j + 1]), r2), g2(j / 2), b2(j / 2)));
      w[e] = pack_bf16x2(o.x, o.y);
    }
    d[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// The activation chunk through the buffer.
__device__ __forceinline__ void stage_act(const ConvParams& p, const Smem& s, Stage& st,
                                          int c0, int n0, float rs, const float (&v)[32]) {
  uint32_t u[16];
  act_words<32>(p, s, c0, n0, rs, v, u);
  stage_acquire(st);
  stage_b16(st, u);
  stage_commit(st, &p.tmAct, 1024, n0 + c0);
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
// No second output voxel (see the temporal 2x copies in epilogue()).
constexpr size_t kNoVox = ~static_cast<size_t>(0);

template <int NC, bool STAGED>
__device__ __forceinline__ void pass1_chunk(const ConvParams& p, const Smem& s, Stage& st,
                                            uint32_t taddr, int c0, int n0, bool valid,
                                            size_t vox, size_t vox2, float& ss, bool keep) {
  float v[NC];
  result_chunk<NC>(p, s, taddr, c0, n0, valid, vox, v);
  float2 sa = make_float2(0.0f, 0.0f), sb = sa;  // two packed chains
#pragma unroll
  for (int j = 0; j < NC; j += 4) {
    const float2 x0 = make_float2(v[j], v[j + 1]), x1 = make_float2(v[j + 2], v[j + 3]);
    sa = ffma2(x0, x0, sa);
    sb = ffma2(x1, x1, sb);
  }
  ss += (sa.x + sa.y) + (sb.x + sb.y);
  if constexpr (STAGED && NC == 32) {
    if (p.ep.out != nullptr && n0 + c0 < p.cout) stage_raw(p, st, n0 + c0, v);
    if (keep) tmem_store_chunk<NC>(taddr + c0, v);
    return;
  }
  if (valid) {
    store_raw<NC>(p, c0, n0, vox, v);
    if (vox2 != kNoVox) store_raw<NC>(p, c0, n0, vox2, v);
  }
  if (keep) tmem_store_chunk<NC>(taddr + c0, v);
}
// keep = false: h is not stored back (the caller re-reads it from the fp32
// raw output instead).
template <bool STAGED>
__device__ __forceinline__ float lane_pass1(const ConvParams& p, const Smem& s, Stage& st,
                                           uint32_t taddr, int c_lo, int c_hi, int n0,
                                           bool valid, size_t vox, size_t vox2, bool keep) {
  float ss = 0.0f;
  int c0 = c_lo;
  for (; c0 + 32 <= c_hi; c0 += 32)
    pass1_chunk<32, STAGED>(p, s, st, taddr, c0, n0, valid, vox, vox2, ss, keep);
  if (c0 < c_hi) pass1_chunk<16, STAGED>(p, s, st, taddr, c0, n0, valid, vox, vox2, ss, keep);
  if (keep) tmem_wait_st();
  return ss;
}

// Second pass reading h back from the fp32 raw output this thread wrote in
// pass 1 (the accumulator is released already).
template <bool STAGED>
__device__ __forceinline__ void lane_pass2_global(const ConvParams& p, const Smem& s,
                                                 Stage& st, int n0, bool valid, size_t vox,
                                                 size_t vox2, float rs) {
  if (!STAGED && !valid) return;
  const float* h = static_cast<const float*>(p.ep.out) + vox * p.cout + n0;
  int c0 = 0;
  for (; c0 + 32 <= p.BN; c0 += 32) {
    float v[32];
    if (!valid) {  // staged stores: the warp's lanes all take part
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.0f;
    } else if (p.ep.vec32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t u[8];
        ld_global_v8(h + c0 + 8 * q, u);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * q + e] = __uint_as_float(u[e]);
      }
    } else {
      const float4* h4 = reinterpret_cast<const float4*>(h + c0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 f = h4[q];
        v[4 * q] = f.x;
        v[4 * q + 1] = f.y;
        v[4 * q + 2] = f.z;
        v[4 * q + 3] = f.w;
      }
    }
    if constexpr (STAGED) {
      if (n0 + c0 < p.cout) stage_act(p, s, st, c0, n0, rs, v);
      continue;
    }
    store_act<32>(p, s, c0, n0, vox, rs, v);
    if (vox2 != kNoVox) store_act<32>(p, s, c0, n0, vox2, rs, v);
  }
  if (c0 < p.BN && valid) {
    float v[16];
    const float4* h4 = reinterpret_cast<const float4*>(h + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = h4[q];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
    store_act<16>(p, s, c0, n0, vox, rs, v);
    if (vox2 != kNoVox) store_act<16>(p, s, c0, n0, vox2, rs, v);
  }
}

// Second pass: the next layer's activation SiLU(h r gamma + beta) from h in the lane.
template <bool STAGED>
__device__ __forceinline__ void lane_pass2(const ConvParams& p, const Smem& s, Stage& st,
                                          uint32_t taddr, int c_lo, int c_hi, int n0, bool valid,
                                          size_t vox, size_t vox2, float rs) {
  int c0 = c_lo;
  for (; c0 + 32 <= c_hi; c0 += 32) {
    float v[32];
    tmem_load_chunk<32>(taddr + c0, v);
    if constexpr (STAGED) {
      if (n0 + c0 < p.cout) stage_act(p, s, st, c0, n0, rs, v);
    } else if (valid) {
      store_act<32>(p, s, c0, n0, vox, rs, v);
      if (vox2 != kNoVox) store_act<32>(p, s, c0, n0, vox2, rs, v);
    }
  }
  if (c0 < c_hi) {
    float v[16];
    tmem_load_chunk<16>(taddr + c0, v);
    if (valid) {
      store_act<16>(p, s, c0, n0, vox, rs, v);
      if (vox2 != kNoVox) store_act<16>(p, s, c0, n0, vox2, rs, v);
    }
  }
}

// Single pass when no norm is fused: raw result and / or video.
template <bool STAGED>
__device__ __forceinline__ void lane_emit(const ConvParams& p, const Smem& s, Stage& st,
                                          uint32_t taddr, int c_lo, int c_hi, int n0, bool valid,
                                          size_t vox, size_t vox2, const TileCoord& tc, int h,
                                          int w) {
  int c0 = c_lo;
  for (; c0 + 32 <= c_hi; c0 += 32) {
    float v[32];
    result_chunk<32>(p, s, taddr, c0, n0, valid, vox, v);
    if constexpr (STAGED) {  // no video with staged stores
      if (p.ep.out != nullptr && n0 + c0 < p.cout) stage_raw(p, st, n0 + c0, v);
    } else if (valid) {
      emit_chunk<32>(p, c0, n0, tc, h, w, vox, v);
      if (vox2 != kNoVox) store_raw<32>(p, c0, n0, vox2, v);
    }
  }
  if (c0 < c_hi) {
    float v[16];
    result_chunk<16>(p, s, taddr, c0, n0, valid, vox, v);
    if (valid) {
      emit_chunk<16>(p, c0, n0, tc, h, w, vox, v);
      if (vox2 != kNoVox) store_raw<16>(p, c0, n0, vox2, v);
    }
  }
}

// Column taps in N (nw = 3): the lane holds, for its computed column c, the
// partial sums P_u (u = 0, 1, 2: BN columns each) of column tap u over the
// input column at c.  Output column c needs P_0 from column c - 1, P_1 from
// c and P_2 from c + 1: the neighbouring lanes of the same tile row (a warp
// holds two rows of 16; the edge columns 0 and 15 are halo and not output).
template <int NB>
__device__ __noinline__ void lane_emit_taps_in_n(const ConvParams& p, const Smem& s,
                                                    uint32_t taddr, int n0, bool valid,
                                                    size_t vox, const TileCoord& tc, int h,
                                                    int w) {
  float v[NB], t[NB];
  tmem_load_chunk<NB>(taddr + NB, v);
  tmem_load_chunk<NB>(taddr, t);
#pragma unroll
  for (int j = 0; j < NB; ++j) v[j] += __shfl_up_sync(0xffffffffu, t[j], 1);
  tmem_load_chunk<NB>(taddr + 2 * NB, t);
#pragma unroll
  for (int j = 0; j < NB; ++j) v[j] += __shfl_down_sync(0xffffffffu, t[j], 1) + s.bias[n0 + j];
  if (valid) emit_chunk<NB>(p, 0, n0, tc, h, w, vox, v);
}

template <bool PAIR, bool STAGED>
__device__ void epilogue(const ConvParams& p, const Smem& s, uint32_t tmem_base, int warp,
                         int lane, int crank) {
  const int q = warp & 3;           // TMEM lane quarter this warp may access
  const int grp = (warp - 2) >> 2;  // epilogue group 0 or 1
  const int row = q * 32 + lane;
  const float rootC = sqrtf(static_cast<float>(p.cout));
  // With a fused norm and an fp32 raw output, pass 2 can read h back from that
  // output, so the accumulator is released right after pass 1 and the next
  // tile's main loop overlaps pass 2 (the host sets early_release where one
  // accumulator fills TMEM and CTAs run several tiles).
  const bool early = p.early_release != 0;
  uint32_t ti = 0;
  Stage st;
  st.buf = s.stage + static_cast<uint32_t>(warp - 2) * kStageWarpBytes;
  st.lane = lane;
  // The accumulator's release: on this CTA's barrier, or on rank 0's with a
  // pair (rank 0's MMAs write both CTAs' accumulators).
  auto release = [&](uint32_t acc) {
    tc_fence_before();
    if constexpr (PAIR)
      mbar_arrive_cluster(mapa_shared(smem_u32(&s.tempty[acc]), 0));
    else
      mbar_arrive(smem_u32(&s.tempty[acc]));
  };
  for (int tile = tile_first(p); tile < tile_count(p); tile += tile_stride(p), ++ti) {
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
    const bool own = tile_own(p, tile, crank);
    const int n0 = tc.n_tile * p.BN;
    for (int sub = grp; sub < p.S; sub += 2) {  // the groups take alternate sub-tiles
      const int idx = sub * kBM + row;  // computed voxel of the tile, row-major
      const int c = idx % p.tile_cols;
      const int h = tc.th * p.tile_rows + idx / p.tile_cols;
      const int w = tc.tw * p.out_cols + c - (p.nw > 1 ? 1 : 0);
      // phase mode with a row window (out_rows > 0): output row 2h + p' lands at row
      // 2h + p' - out_row0 of an out_rows-row output, or nowhere
      const int ho = p.phases == 4 ? 2 * h + (tc.phase >> 1) - p.out_row0 : h;
      const int Ho = p.out_rows > 0 ? p.out_rows : 2 * p.H;
      const bool valid = own && h < p.H && w < p.W && (p.nw == 1 || (c >= 1 && c <= p.tile_cols - 2)) &&
                         (p.out_rows == 0 || (ho >= 0 && ho < p.out_rows));
      // output voxel: (t, h, w), or (t, 2h + p', 2w + q') of the 2H x 2W output in phase
      // mode.  With a temporal 2x step (phase mode only) input frame t goes to output
      // frames 2t - 1 and 2t (tdup 1: frame 0 of the decode once), or 2t and 2t + 1
      // (tdup 2: a continuing chunk).
      int t0 = tc.t, t1 = -1;
      if (p.tdup == 1) {
        t0 = tc.t == 0 ? 0 : 2 * tc.t - 1;
        t1 = tc.t == 0 ? -1 : 2 * tc.t;
      } else if (p.tdup == 2) {
        t0 = 2 * tc.t;
        t1 = 2 * tc.t + 1;
      }
      auto out_vox = [&](int to) {
        if (p.wino)  // transform plane xi = phase of the products
          return ((static_cast<size_t>(tc.phase) * p.T + to) * p.H + h) * p.W + w;
        return p.phases == 4 ? (static_cast<size_t>(to) * Ho + ho) * (2 * p.W) + 2 * w + (tc.phase & 1)
                             : (static_cast<size_t>(to) * p.H + h) * p.W + w;
      };
      const size_t vox = out_vox(t0);
      const size_t vox2 = t1 < 0 ? kNoVox : out_vox(t1);
      st.sr.ok = valid ? 1 : 0;
      st.sr.q = p.phases == 4 ? (tc.phase & 1) : 0;
      st.sr.w = w;
      {
        const int hr = p.phases == 4 ? ho : h;     // row inside the output frame
        const int rows = p.phases == 4 ? Ho : p.H;  // rows per output frame
        st.sr.r = t0 * rows + hr;
        st.sr.r2 = t1 < 0 ? -1 : t1 * rows + hr;
      }
      const uint32_t n_stride = conv_tc_acc_stride(p);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             (acc * static_cast<uint32_t>(p.S) + static_cast<uint32_t>(sub)) * n_stride;
      if (p.nw > 1) {
        lane_emit_taps_in_n<16>(p, s, taddr, n0, valid, vox, tc, h, w);  // BN = 16
      } else if (p.ep.act == nullptr) {
        lane_emit<STAGED>(p, s, st, taddr, 0, p.BN, n0, valid, vox, vox2, tc, h, w);
      } else {
        float ss = lane_pass1<STAGED>(p, s, st, taddr, 0, p.BN, n0, valid, vox, vox2, !early);
        if (early) release(acc);
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
          if (!got) {
            if (STAGED && lane == 0) bulk_wait_all();
            return;
          }
          __syncwarp();
          ss += s.xpart[slot];
        }
        const float rs = rootC / fmaxf(sqrtf(ss), p.ep.eps);
        if (early) {
          if constexpr (STAGED) {
            // pass 2 reads h back from the raw output that lane 0's bulk stores wrote
            if (lane == 0) {
              bulk_wait_all();
              fence_proxy_async_global();
            }
            __syncwarp();
            asm volatile("" ::: "memory");
          }
          lane_pass2_global<STAGED>(p, s, st, n0, valid, vox, vox2, rs);
        } else {
          lane_pass2<STAGED>(p, s, st, taddr, 0, p.BN, n0, valid, vox, vox2, rs);
        }
      }
    }
    if (!early) release(acc);
  }
  // the buffers' last bulk stores complete before the CTA leaves
  if (STAGED && lane == 0) bulk_wait_all();
}

// S = 2 throughout; narrow layers (and 1-row kernels) put a group's window and
// weight tiles in one stage.
template <bool PAIR>
__device__ void run_mma(const ConvParams& p, const Smem& s, uint32_t tmem_base) {
  if (p.kh_eff == 1)
    mma_issuer<2, 1, 1, true, PAIR>(p, s, tmem_base);
  else if (p.kh_eff == 2)
    p.combined ? mma_issuer<2, 2, 2, true, PAIR>(p, s, tmem_base)
               : mma_issuer<2, 2, 1, false, PAIR>(p, s, tmem_base);
  else
    p.combined ? mma_issuer<2, 3, 3, true, PAIR>(p, s, tmem_base)
               : mma_issuer<2, 3, 1, false, PAIR>(p, s, tmem_base);
}

// PAIR (= p.pair) is a template parameter so that only the pair kernels hold
// cta_group::2 instructions: a kernel with them is launched as clusters of 2.
// STAGED (= p.tma_out) picks the epilogue's staged TMA stores.
template <bool PAIR, bool STAGED>
__device__ __forceinline__ void conv_tc_body(const ConvParams& p) {
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve(smem_raw, p);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages_a; ++i) {
      mbar_init(smem_u32(&s.full_a[i]), 1);
      mbar_init(smem_u32(&s.empty_a[i]), 1);
    }
    for (int i = 0; i < p.stages_b; ++i) {
      mbar_init(smem_u32(&s.full_b[i]), 1);
      mbar_init(smem_u32(&s.empty_b[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s.tfull[i]), 1);
      // every epilogue thread releases the accumulator (both CTAs' with a pair)
      mbar_init(smem_u32(&s.tempty[i]), PAIR ? 512 : 256);
    }
    mbar_init(smem_u32(s.drain), 1);
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
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(s.tmem_slot), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(s.tmem_slot), 512);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  tc_fence_before();
  __syncthreads();
  // With a cluster of two, both CTAs' barriers exist before either writes to the other.
  if (cluster2(p)) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *s.tmem_slot;
  const int crank = cluster2(p) ? static_cast<int>(cluster_ctarank()) : 0;

  if (warp == 0) {
    if (lane == 0) producer<PAIR>(p, s, crank);
  } else if (warp == 1) {
    // a pair's MMAs are rank 0's
    if (lane == 0 && (!PAIR || crank == 0)) run_mma<PAIR>(p, s, tmem_base);
  } else {
    epilogue<PAIR, STAGED>(p, s, tmem_base, warp, lane, crank);
  }

  tc_fence_before();
  __syncthreads();
  // Neither CTA of a cluster leaves while the other may still write into it
  // (or, with a pair, while rank 0's MMAs may still read its shared memory).
  if (cluster2(p)) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, 512);
    else
      tmem_dealloc(tmem_base, 512);
  }
}

template <bool PAIR>
__global__ void __launch_bounds__(kConvThreads, 1) conv_tc_kernel(const __grid_constant__ ConvParams p) {
  conv_tc_body<PAIR, false>(p);
}

// The pair kernel whose epilogue writes its outputs with staged TMA stores.
__global__ void __launch_bounds__(kConvThreads, 1)
    conv_tc_staged_kernel(const __grid_constant__ ConvParams p) {
  conv_tc_body<true, true>(p);
}

}  // namespace

size_t conv_tc_smem_bytes(const ConvParams& p) {
  return 1024 + static_cast<size_t>(p.stages_a) * conv_tc_a_bytes(p) +
         static_cast<size_t>(p.stages_b) * conv_tc_b_bytes(p) + conv_tc_stage_bytes(p) + kCtrlBytes;
}

void conv_tc_choose_stages(ConvParams& p) {
  // 227 KB opt-in per block
  const size_t budget = 232448 - 1024 - kCtrlBytes - conv_tc_stage_bytes(p);
  const size_t a = conv_tc_a_bytes(p), b = conv_tc_b_bytes(p);
  if (p.combined) {
    // one stage per group: equal depths
    size_t n = budget / (a + b);
    if (n > static_cast<size_t>(kMaxStages)) n = kMaxStages;
    p.stages_a = p.stages_b = static_cast<int>(n < 2 ? 2 : n);
    return;
  }
  // A pair's half weight tiles leave room for a third A window (measured:
  // ~0.5-1 % on the 256-wide pair layers); otherwise two A stages
  if (p.pair) {
    size_t nb3 = (budget - 3 * a) / b;
    if (nb3 > static_cast<size_t>(kMaxStages)) nb3 = kMaxStages;
    if (nb3 >= 4) {
      p.stages_a = 3;
      p.stages_b = static_cast<int>(nb3);
      return;
    }
  }
  // each A window serves kh_eff weight tiles: two A stages, the rest for B
  size_t nb = (budget - 2 * a) / b;
  if (nb > static_cast<size_t>(kMaxStages)) nb = kMaxStages;
  p.stages_b = static_cast<int>(nb < 2 ? 2 : nb);
  size_t na = (budget - p.stages_b * b) / a;
  if (na > 4) na = 4;
  p.stages_a = static_cast<int>(na < 2 ? 2 : na);
}

namespace {
size_t launch_smem(const ConvParams& p) {
  // Every CTA allocates all 512 TMEM columns, so exactly one may live on an SM:
  // ask for more than half of the SM's shared memory even when the ring is small.
  size_t smem = conv_tc_smem_bytes(p);
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
  attr[0].val.clusterDim.x = (p.nsplit == 2 || p.pair) ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
}  // namespace

int conv_tc_max_clusters(const ConvParams& p) {
  const size_t smem = launch_smem(p);
  auto kern = p.tma_out ? conv_tc_staged_kernel : (p.pair ? conv_tc_kernel<true> : conv_tc_kernel<false>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_config(p, 2, smem, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_conv_tc(const ConvParams& p, int grid, cudaStream_t stream) {
  const size_t smem = launch_smem(p);
  auto kern = p.tma_out ? conv_tc_staged_kernel : (p.pair ? conv_tc_kernel<true> : conv_tc_kernel<false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_config(p, grid, smem, stream, attr);
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace wvae

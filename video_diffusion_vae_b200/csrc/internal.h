// Host/device shared declarations of the library's internal launch interface.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace wvae {

// ----------------------------------------------------------- conv (tcgen05)
// A CTA tile of tile_rows x tile_cols voxels of one frame (16 x 16 or 8 x 32)
// is S = 2 MMA sub-tiles of kBM = 128 consecutive voxels in row-major order;
// their M=128 MMAs share each weight tile.  The reduction runs in K groups of
// kBK = 64 input channels of one (kt, kw) tap column.
constexpr int kTileH = 8;
constexpr int kTileW = 16;
constexpr int kBM = kTileH * kTileW;  // 128
constexpr int kBK = 64;
constexpr int kConvThreads = 320;     // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue (2 groups)
constexpr int kMaxStages = 8;

// What the epilogue does with acc + bias (+ residual), per output voxel.
struct ConvEpilogue {
  const float* bias;        // fp32 [cout_pad] (packed blob)
  const float* bias2;       // fp32 [cout_pad] shortcut bias, or null
  const void* residual;     // [T][H][W][cout] or null
  int residual_f32;         // residual dtype: 1 fp32, 0 bf16
  void* out;                // raw result [T][H][W][cout] ([T][2H][2W][cout] in phase mode), or null
  int out_f32;              // out dtype: 1 fp32, 0 bf16 (or fp16 with out_f16)
  int out_f16;              // out is fp16 (the Winograd products)
  __nv_bfloat16* act;       // SiLU(norm(result)) bf16 [T][H][W][cout], or null
  const float* gamma;       // fp32 [cout] for act
  const float* beta;        // fp32 [cout] for act
  float eps;
  __nv_bfloat16* video;     // 2x2 pixel-shuffled NCDHW [cout/4][T][2H][2W], or null
  int vec32;                // residual / out / act are 32-byte aligned: 256-bit accesses
};

struct ConvParams {
  CUtensorMap tmA;   // main input, bf16 [T][H][W][cin_pad],
                     // box {64, tile_cols, tile_rows + kh_eff - 1, 1} (the row-tap window)
  CUtensorMap tmB;   // main weights, bf16 [cout_pad][taps * cin_pad], box {64, BN}
  CUtensorMap tmC;   // cached frames, bf16 [KT-1][H][W][cin_pad], box as tmA (has_cache)
  CUtensorMap tmA2;  // shortcut input, bf16 [T][H][W][cin2_pad], box {64, tile_cols,
                     // tile_rows, 1} (cin2_pad > 0)
  CUtensorMap tmB2;  // shortcut weights, bf16 [cout_pad][cin2_pad]
  CUtensorMap tmO;   // staged stores (tma_out): the raw output viewed as [rows][W][Q][cout]
                     // (Q = 2 column phases in phase mode, else 1; rows = output frames x
                     // output rows), fp32 (128B swizzle) or bf16 (64B), box {32, 1, 16, 1}
  CUtensorMap tmAct; // staged stores: the activation output, bf16, as tmO
  int T, H, W;
  int cin_pad, cin2_pad;
  int cout, cout_pad;
  int KT, KH, KW;
  int phases;        // 4: upsample-conv phase mode (KH = KW = 2, output at (2h+p, 2w+q))
  int wino;          // 1: Winograd products: phases = 16 transform planes, fp16 operands, A
                     //    = the planes [16][T][H][W][cin] (tmA 5-D, H x W = the tile grid),
                     //    weights [cout_pad][16 x KT][cin_pad], out [16][T][H][W][cout]
  int out_row0, out_rows;  // phase mode: output row 2h + p' is written at row 2h + p' - out_row0
                           //    of an out_rows-row output, if inside it (out_rows 0: 2H rows)
  int tdup;          // phase mode: a temporal 2x step in the output frames (1: input frame
                     //    t -> 2t - 1 and 2t, frame 0 once; 2: t -> 2t and 2t + 1)
  int nsplit;        // 2: a cluster of 2 CTAs splits N (rank = N tile) and exchanges the
                     //    RMS partial sums over distributed shared memory
  int pair;          // 1: a cluster of 2 CTAs shares M = 256 MMAs (cta_group::2): rank r
                     //    takes M tile 2i + r of pair tile i and loads half of each weight
                     //    tile (BN / 2 rows); rank 0 issues the MMAs
  int has_cache;
  int BN, n_tiles;
  int S;             // MMA sub-tiles per CTA tile (2)
  int tile_rows, tile_cols;  // CTA tile, tile_rows * tile_cols = 128 S voxels of one frame
  int kh_eff, kw_eff;  // row / column taps per A window: KH, KW (2, 2 in phase mode; kw_eff
                       // = 1 when the column taps ride in N)
  int nw;            // column taps per MMA: 1, or KW (narrow layers: N = KW * BN, the
                     // epilogue adds the taps' partial sums from the neighbouring columns)
  int out_cols;      // output columns per tile: tile_cols, or tile_cols - 2 when nw = KW
  int b_tiles;       // weight tiles per B-ring stage: 1, or kh_eff (a group's row taps
                     // behind one wait, for narrow BN where one tile is little MMA work)
  int combined;      // 1 (b_tiles == kh_eff): a group's A window and weight tiles travel
                     // in one stage on one barrier (A and B rings in lockstep)
  int tiles_w, tiles_h, m_tiles, num_tiles;
  int stages_a, stages_b, num_acc;  // A-window ring, weight-tile ring, TMEM accumulators
  int tma_out;       // 1: the epilogue stages 32-channel chunks in shared memory (a buffer
                     //    per epilogue warp) and writes them with TMA stores (tmO / tmAct)
                     //    instead of per-lane stores
  int early_release; // 1: release the accumulator after epilogue pass 1 (fused norm + fp32
                     //    raw output, one accumulator, several tiles per CTA)
  int groups_main;   // K groups of the main segment: (kt, column tap, 64 input channels)
  int groups;        // + one group per 64 channels of the second segment
  ConvEpilogue ep;
  unsigned* err;
};

// A window of a main-segment K group: the tile's rows plus the row-tap halo.
__host__ __device__ inline uint32_t conv_tc_a_rows(const ConvParams& p) {
  return static_cast<uint32_t>(p.tile_rows + p.kh_eff - 1);
}
// Shared-memory bytes of one A-ring stage (1024-aligned) and one B-ring stage.
__host__ __device__ inline uint32_t conv_tc_a_bytes(const ConvParams& p) {
  return (conv_tc_a_rows(p) * static_cast<uint32_t>(p.tile_cols) * 128u + 1023u) & ~1023u;
}
// Rows of one weight tile held by a CTA: BN, or BN / 2 with a CTA pair.
__host__ __device__ inline int conv_tc_b_rows(const ConvParams& p) {
  return p.pair ? p.BN / 2 : p.BN;
}
__host__ __device__ inline uint32_t conv_tc_b_bytes(const ConvParams& p) {
  return static_cast<uint32_t>(p.b_tiles * p.nw * conv_tc_b_rows(p)) * 128u;
}
// TMEM columns per sub-tile accumulator: the MMA's N (nw BN) rounded up to 32.
__host__ __device__ inline uint32_t conv_tc_acc_stride(const ConvParams& p) {
  return (static_cast<uint32_t>(p.nw * p.BN) + 31u) & ~31u;
}
// Staged-store buffers: 4 KB per epilogue warp (32 voxels x 32 fp32 channels).
constexpr uint32_t kStageWarpBytes = 4096;
__host__ __device__ inline uint32_t conv_tc_stage_bytes(const ConvParams& p) {
  return p.tma_out ? 8u * kStageWarpBytes : 0u;
}
size_t conv_tc_smem_bytes(const ConvParams& p);
// Sets p.stages_a / p.stages_b for the layer (needs BN, tile shape, kh_eff).
void conv_tc_choose_stages(ConvParams& p);
// Clusters of 2 that fit on the device at once (nsplit = 2 launches), 0 on error.
int conv_tc_max_clusters(const ConvParams& p);
cudaError_t launch_conv_tc(const ConvParams& p, int grid, cudaStream_t stream);

// ------------------------------------------------------------ fp32 direct conv
struct ConvF32Params {
  const float* x;      // [T][H][W][cin]
  const float* cache;  // [KT-1][H][W][cin] or null
  const float* w;      // packed fp32 [taps][cin][cout]
  const float* bias;   // [cout]
  const float* residual;
  float* y;            // [T][H][W][cout]
  int T, H, W, cin, cout, KT, KH, KW;
};
cudaError_t launch_conv_f32(const ConvF32Params& p, cudaStream_t stream);

// ---------------------------------------------------------------- norm-SiLU
cudaError_t launch_norm_silu_bf16(const __nv_bfloat16* x, __nv_bfloat16* y, const float* gamma,
                                  const float* beta, long nvox, int C, float eps, int num_sms,
                                  cudaStream_t stream);
cudaError_t launch_norm_silu_f32(const float* x, float* y, const float* gamma, const float* beta,
                                 long nvox, int C, float eps, int num_sms, cudaStream_t stream);

// ------------------------------------------------------------ layout kernels
cudaError_t launch_prepack_bf16(const void* w, int w_is_f32, const float* bias, int cout, int cin,
                                int taps, int cout_pad, int cin_pad, __nv_bfloat16* wp,
                                float* bias_p, cudaStream_t stream);
// Upsample-conv weights [cout][cin][1][3][3] -> four 2x2 phase kernels, bf16
// [cout_pad][16][cin_pad] (see layout.cu).
cudaError_t launch_prepack_phase_bf16(const void* w, int w_is_f32, const float* bias, int cout,
                                      int cin, int cout_pad, int cin_pad, __nv_bfloat16* wp,
                                      float* bias_p, cudaStream_t stream);
cudaError_t launch_prepack_f32(const void* w, int w_is_f32, const float* bias, int cout, int cin,
                               int taps, float* wp, float* bias_p, cudaStream_t stream);
// NCDHW [C][T][H][W] bf16 -> channels-last [T][H][W][Cpad] bf16, zero-filled pad channels.
cudaError_t launch_ncdhw_to_cl_pad(const __nv_bfloat16* x, __nv_bfloat16* y, int C, int Cpad,
                                   int T, int H, int W, cudaStream_t stream);
// channels-last [T][H][W][C] -> [T][2H][2W][C], nearest (fp32 reference path).
cudaError_t launch_upsample2x(const void* x, void* y, int elem_bytes, int T, int H, int W, int C,
                              cudaStream_t stream);
// fp32 [n] -> bf16 [n]
cudaError_t launch_f32_to_bf16(const float* x, __nv_bfloat16* y, size_t n, cudaStream_t stream);

// ------------------------------------------------------------- head (tcgen05)
// The decoder head (causal 3x3x3 conv C -> 12, 2x2 pixel shuffle into the
// NCDHW video) with the 3 temporal x 3 column taps in N (N = 144); see
// head_tc.cu.  C = 64 or 128.
constexpr int kHeadTileRows = 8;
constexpr int kHeadTileCols = 16;   // computed columns; 14 are output
constexpr int kHeadOutCols = 14;
constexpr int kHeadThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

struct HeadParams {
  CUtensorMap tmA;   // activation bf16 [T][H][W][cin], box {64, 16, 10, 1}
  CUtensorMap tmC;   // cached frames bf16 [2][H][W][cin], same box (has_cache)
  CUtensorMap tmB;   // packed weights bf16 [16][27 * cin] (standard prepack), box {64, 16}
  const float* bias; // fp32 [16] (packed blob)
  __nv_bfloat16* video;  // [3][T][2H][2W]
  int T, H, W, cin;
  int tiles_w, tiles_h, num_tiles;
  int has_cache;     // frames -2, -1 come from tmC
  int row0, rows_out;  // video rows 2 (h - row0) + i for rows h in [row0, row0 + rows_out)
                       // (rows_out 0: all H rows, row0 0)
  unsigned* err;
};
size_t head_tc_smem_bytes(int cin);
cudaError_t launch_head_tc(const HeadParams& p, int num_sms, cudaStream_t stream);

// ---------------------------------------------------- Winograd F(2x2, 3x3)
cudaError_t launch_wino_prepack(const void* w, bool is_f32, const float* bias, int cout, int cin,
                                int cout_pad, int cin_pad, __half* up, float* bias_zero,
                                float* bias_p, cudaStream_t stream);
cudaError_t launch_wino_input(const __nv_bfloat16* x, __half* v, int T, int H, int W, int C,
                              cudaStream_t stream);
cudaError_t launch_wino_output(const __half* m, const float* bias, const __nv_bfloat16* residual,
                               __nv_bfloat16* y, int T, int H, int W, int C, cudaStream_t stream);

// Device error word (defined in api.cu).
unsigned* device_error_word();

}  // namespace wvae

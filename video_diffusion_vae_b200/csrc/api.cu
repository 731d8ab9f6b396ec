// The exported C ABI (include/wvae.h): argument validation, TMA descriptors,
// conv planning and the composition of the residual block, the upsample conv
// and the decoder trunk out of the kernels.  Nothing here allocates device
// memory: every buffer, including workspaces, belongs to the caller.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/wvae.h"
#include "internal.h"

namespace wvae {

__device__ unsigned g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  bool ok = false;
  int num_sms = 0;
  unsigned* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

wvae_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return WVAE_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    d.init = true;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return WVAE_ERR_NO_DEVICE;
    }
    void* sym = nullptr;
    if (major == 10 && minor == 0 && cudaGetSymbolAddress(&sym, g_device_error) == cudaSuccess) {
      d.err = static_cast<unsigned*>(sym);
      d.ok = true;
    }
    cudaGetLastError();
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
              cudaSuccess &&
          q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
      cudaGetLastError();
    }
  }
  if (!d.ok || g_encode == nullptr) return WVAE_ERR_NO_DEVICE;
  *out = &d;
  return WVAE_OK;
}

inline bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int round_up(int v, int m) { return (v + m - 1) / m * m; }
inline size_t round_up_sz(size_t v, size_t m) { return (v + m - 1) / m * m; }

inline wvae_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return WVAE_OK;
  cudaGetLastError();
  return WVAE_ERR_CUDA;
}

bool kernel_ok(int kt, int kh, int kw) {
  return (kt == 3 && kh == 3 && kw == 3) || (kt == 1 && kh == 3 && kw == 3) ||
         (kt == 1 && kh == 1 && kw == 1);
}

// --------------------------------------------------------- packed weights
struct PackedLayout {
  int cout_pad, cin_pad, taps;
  size_t w_bytes, bias_off, total;
};

PackedLayout packed_layout(int cout, int cin, int kt, int kh, int kw, wvae_dtype dtype) {
  PackedLayout L;
  L.taps = kt * kh * kw;
  if (dtype == WVAE_BF16) {
    L.cout_pad = round_up(cout, 16);
    L.cin_pad = round_up(cin, 64);
    L.w_bytes = static_cast<size_t>(L.cout_pad) * L.taps * L.cin_pad * 2;
  } else {
    L.cout_pad = cout;
    L.cin_pad = cin;
    L.w_bytes = static_cast<size_t>(cout) * L.taps * cin * 4;
  }
  L.bias_off = round_up_sz(L.w_bytes, 256);
  L.total = L.bias_off + static_cast<size_t>(L.cout_pad) * 4;
  return L;
}

// ------------------------------------------------------------ TMA descriptors
bool encode_act(CUtensorMap* m, const void* base, int C, int W, int H, int T, int box_w, int box_h) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(W),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(C) * 2 * W,
                           static_cast<cuuint64_t>(C) * 2 * W * H};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_w),
                       static_cast<cuuint32_t>(box_h), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// The 16 Winograd transform planes [16][T][H][W][C] fp16 (H x W: the tile grid).
bool encode_planes(CUtensorMap* m, const void* base, int C, int W, int H, int T, int box_w,
                   int box_h) {
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(W),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T), 16};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(C) * 2 * W,
                           static_cast<cuuint64_t>(C) * 2 * W * H,
                           static_cast<cuuint64_t>(C) * 2 * W * H * T};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_w),
                       static_cast<cuuint32_t>(box_h), 1, 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// An epilogue output [rows][W][Q][C] (C channels, Q column phases) for staged
// TMA stores of 32 channels x 16 voxels of one row: fp32 rows of 128 B under
// the 128B swizzle, bf16 rows of 64 B under the 64B swizzle.
bool encode_store(CUtensorMap* m, void* base, int eb, int C, int Q, int W, long rows) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(Q),
                        static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * eb, static_cast<cuuint64_t>(C) * eb * Q,
                           static_cast<cuuint64_t>(C) * eb * Q * W};
  cuuint32_t box[4] = {32, 1, 16, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return g_encode(m, eb == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  eb == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_weights(CUtensorMap* m, const void* base, int K, int N, int box_rows,
                    CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, type, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// --------------------------------------------------------- tensor-core conv
struct TcConv {
  const void* x = nullptr;   // [T][H][W][cin_pad] bf16
  int cin_pad = 0;
  const void* cache = nullptr;
  const void* packed = nullptr;
  int cout = 0, KT = 3, KH = 3, KW = 3;
  const void* x2 = nullptr;  // shortcut input [T][H][W][cin2_pad]
  int cin2_pad = 0;
  const void* packed2 = nullptr;
  int T = 0, H = 0, W = 0;
  int phases = 1;            // 4: upsample-conv phase mode (packed by prepack_upsample)
  int tdup = 0;              // phase mode: temporal 2x copies of the output (ConvParams::tdup)
  int wino = 0;              // Winograd products over the 16 transform planes (ConvParams::wino)
  int out_row0 = 0, out_rows = 0;  // phase mode: output row window (ConvParams)
  ConvEpilogue ep{};
};

wvae_status run_tc_conv(const DeviceInfo& d, TcConv a, cudaStream_t stream) {
  static_assert(sizeof(ConvParams) < 4000, "kernel parameter space");
  if (a.phases == 4) {
    a.KT = 1;
    a.KH = 2;
    a.KW = 2;
  }
  if (a.wino) {  // 16 planes x KT temporal taps, 1 x 1 spatially
    a.phases = 16;
    a.KH = 1;
    a.KW = 1;
  }
  // phase mode packs 4 phases x 4 taps along K, Winograd 16 planes x KT taps
  const PackedLayout L = a.phases == 4 ? packed_layout(a.cout, a.cin_pad, 1, 4, 4, WVAE_BF16)
                         : a.wino      ? packed_layout(a.cout, a.cin_pad, a.KT, 16, 1, WVAE_BF16)
                                       : packed_layout(a.cout, a.cin_pad, a.KT, a.KH, a.KW, WVAE_BF16);
  ConvParams p;
  std::memset(&p, 0, sizeof(p));
  p.T = a.T;
  p.H = a.H;
  p.W = a.W;
  p.cin_pad = a.cin_pad;
  p.cin2_pad = a.cin2_pad;
  p.cout = a.cout;
  p.cout_pad = L.cout_pad;
  p.KT = a.KT;
  p.KH = a.KH;
  p.KW = a.KW;
  p.phases = a.phases;
  p.tdup = a.phases == 4 ? a.tdup : 0;
  p.wino = a.wino;
  p.out_row0 = a.phases == 4 ? a.out_row0 : 0;
  p.out_rows = a.phases == 4 ? a.out_rows : 0;
  p.has_cache = a.cache != nullptr;
  // The fused norm needs every output channel of a voxel: one CTA holds them
  // all (BN = Cout) up to 256; at 512 a cluster of two CTAs splits N and swaps
  // the partial sums of squares.
  const bool need_all_channels = a.ep.act != nullptr;
  p.nsplit = 1;
  if (L.cout_pad <= 256) {
    p.BN = L.cout_pad;
  } else if (L.cout_pad == 512) {
    p.BN = 256;
    if (need_all_channels) p.nsplit = 2;
  } else {
    if (need_all_channels) return WVAE_ERR_UNSUPPORTED;
    p.BN = (L.cout_pad % 256 == 0) ? 256 : (L.cout_pad % 128 == 0 ? 128 : 16);
  }
  p.n_tiles = L.cout_pad / p.BN;
  // Sub-tiles per CTA tile: S M=128 MMAs share each weight tile (see conv_tc.cu).
  p.S = 2;
  // At 16 output channels (the head) a tcgen05.mma is mostly fixed issue
  // cost, so the three column taps ride in N (N = 48) and the epilogue adds
  // each tap's partial sum from the neighbouring column's TMEM lane.
  const bool kwn = p.BN == 16 && a.KH == 3 && a.KW == 3 && a.phases == 1 && a.cin2_pad == 0 &&
                   a.ep.act == nullptr && a.ep.residual == nullptr && p.nsplit == 1;
  p.nw = kwn ? a.KW : 1;
  // CTA pairs (M = 256 MMAs, each CTA loading half of every weight tile) for
  // the 128- and 256-wide N tiles of direct convs: half the weight bytes per
  // SM through the fill and shared memory.
  p.pair = (p.nsplit == 1 && (p.BN == 128 || p.BN == 256) && p.nw == 1 && !a.wino &&
            a.cin2_pad == 0)
               ? 1
               : 0;
  p.num_acc = 2 * p.S * static_cast<int>(conv_tc_acc_stride(p)) <= 512 ? 2 : 1;
  // Row taps share one A window (the tile plus its row halo) per (kt, kw); up
  // to 128 output channels a B stage carries all of a window's row taps.
  p.kh_eff = a.phases == 4 ? 2 : a.KH;
  p.kw_eff = a.phases == 4 ? 2 : (kwn ? 1 : a.KW);
  p.b_tiles = (p.BN <= 128 || p.kh_eff == 1) ? p.kh_eff : 1;
  p.combined = p.b_tiles == p.kh_eff ? 1 : 0;
  // Tile shape: 128 S voxels as tile_rows x tile_cols, tile_cols in {16, 32,
  // 64}; the narrowest shape among those needing the fewest waves of tiles over
  // the CTAs (or CTA pairs) that run at once.
  const int slots = p.nsplit == 2 ? d.num_sms / 2 : d.num_sms;
  const int per_m = p.phases * (p.nsplit == 2 ? 1 : p.n_tiles);
  auto waves = [&](int rows, int cols) {
    const long tiles = static_cast<long>(a.T) * ((a.H + rows - 1) / rows) * ((a.W + cols - 1) / cols) * per_m;
    return (tiles + slots - 1) / slots;
  };
  p.tile_cols = kTileW;
  p.tile_rows = kBM * p.S / kTileW;
  if (!kwn) {
    for (int cols = 2 * kTileW; cols <= 64 && kBM * p.S / cols >= kTileH; cols *= 2) {
      if (waves(kBM * p.S / cols, cols) < waves(p.tile_rows, p.tile_cols)) {
        p.tile_cols = cols;
        p.tile_rows = kBM * p.S / cols;
      }
    }
  }
  // with the column taps in N the two edge columns of a tile only feed their
  // neighbours: 16 computed columns give 14 outputs
  p.out_cols = kwn ? p.tile_cols - 2 : p.tile_cols;
  p.tiles_w = (a.W + p.out_cols - 1) / p.out_cols;
  p.tiles_h = (a.H + p.tile_rows - 1) / p.tile_rows;
  p.m_tiles = a.T * p.tiles_h * p.tiles_w;
  p.num_tiles = p.m_tiles * per_m;
  // Staged TMA stores of the raw output and the activation (see conv_tc.cu) on
  // CTA pairs, for the upsample convs, whose outputs (four phases, fp32 + bf16)
  // are large against their MMA work (the per-lane stores kept the load/store
  // pipe busy for 70 % of the kernel's time), and for the layers whose one
  // accumulator is released after epilogue pass 1 (fp32 + bf16 outputs, the
  // next tile's MMAs waiting on that pass).  Elsewhere the buffers' 32 KB of
  // shared memory (a ring stage less) cost more than they saved.
  const bool early_layer = p.num_acc == 1 && a.ep.act != nullptr && a.ep.out != nullptr &&
                           a.ep.out_f32 && p.num_tiles > slots;
  p.tma_out = (p.pair && (p.phases == 4 || early_layer) && p.nw == 1 && !a.wino &&
               a.ep.video == nullptr && !a.ep.out_f16 && p.BN % 32 == 0 && a.cout % 16 == 0 &&
               (a.ep.out != nullptr || a.ep.act != nullptr) && a16(a.ep.out) && a16(a.ep.act))
                  ? 1
                  : 0;
  conv_tc_choose_stages(p);
  if (p.tma_out && (p.combined ? p.stages_a < 3 : p.stages_b < 3)) {
    p.tma_out = 0;
    conv_tc_choose_stages(p);
  }
  p.groups_main = (a.phases == 4 ? 1 : a.KT) * p.kw_eff * (a.cin_pad / kBK);
  p.groups = p.groups_main + a.cin2_pad / kBK;
  a.ep.bias = reinterpret_cast<const float*>(static_cast<const char*>(a.packed) + L.bias_off);
  if (a.packed2 != nullptr) {
    const PackedLayout L2 = packed_layout(a.cout, a.cin2_pad, 1, 1, 1, WVAE_BF16);
    a.ep.bias2 = reinterpret_cast<const float*>(static_cast<const char*>(a.packed2) + L2.bias_off);
  }
  p.ep = a.ep;
  // 256-bit epilogue accesses need 32-byte aligned rows and bases
  auto a32 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 31u) == 0; };
  p.ep.vec32 = (a.cout % 16 == 0 && a32(a.ep.residual) && a32(a.ep.out) && a32(a.ep.act)) ? 1 : 0;
  p.err = d.err;
  const int box_rows = conv_tc_b_rows(p);  // BN <= 256, or BN / 2 with a pair
  const int a_rows = static_cast<int>(conv_tc_a_rows(p));
  if (a.wino) {
    if (!encode_planes(&p.tmA, a.x, a.cin_pad, a.W, a.H, a.T, p.tile_cols, a_rows))
      return WVAE_ERR_CUDA;
    if (!encode_weights(&p.tmB, a.packed, L.taps * a.cin_pad, L.cout_pad, box_rows,
                        CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
      return WVAE_ERR_CUDA;
  } else {
    if (!encode_act(&p.tmA, a.x, a.cin_pad, a.W, a.H, a.T, p.tile_cols, a_rows))
      return WVAE_ERR_CUDA;
    if (!encode_weights(&p.tmB, a.packed, L.taps * a.cin_pad, L.cout_pad, box_rows))
      return WVAE_ERR_CUDA;
  }
  if (p.tma_out) {
    // output frames (temporal 2x copies in phase mode) x rows per output frame
    const int t_out = p.tdup == 1 ? 2 * a.T - 1 : (p.tdup == 2 ? 2 * a.T : a.T);
    const int rows = a.phases == 4 ? (p.out_rows > 0 ? p.out_rows : 2 * a.H) : a.H;
    const int q = a.phases == 4 ? 2 : 1;
    if (a.ep.out != nullptr && !encode_store(&p.tmO, a.ep.out, a.ep.out_f32 ? 4 : 2, a.cout, q, a.W,
                                             static_cast<long>(t_out) * rows))
      return WVAE_ERR_CUDA;
    if (a.ep.act != nullptr && !encode_store(&p.tmAct, a.ep.act, 2, a.cout, q, a.W,
                                             static_cast<long>(t_out) * rows))
      return WVAE_ERR_CUDA;
  }
  if (a.cache != nullptr && !encode_act(&p.tmC, a.cache, a.cin_pad, a.W, a.H, a.KT - 1, p.tile_cols,
                                        a_rows))
    return WVAE_ERR_CUDA;
  if (a.cin2_pad > 0) {
    if (!encode_act(&p.tmA2, a.x2, a.cin2_pad, a.W, a.H, a.T, p.tile_cols, p.tile_rows)) return WVAE_ERR_CUDA;
    if (!encode_weights(&p.tmB2, a.packed2, a.cin2_pad, L.cout_pad, box_rows)) return WVAE_ERR_CUDA;
  }
  p.early_release = early_layer ? 1 : 0;
  int grid;
  if (p.nsplit == 2 || p.pair) {
    int clusters = conv_tc_max_clusters(p);
    if (clusters < 1) clusters = d.num_sms / 2;
    // a pair takes two spatial tiles of one (N tile, phase) at a time
    const int units = p.pair ? ((p.m_tiles + 1) / 2) * p.phases * p.n_tiles : p.num_tiles;
    grid = 2 * (units < clusters ? units : clusters);
  } else {
    grid = p.num_tiles < d.num_sms ? p.num_tiles : d.num_sms;
  }
  return cuda_status(launch_conv_tc(p, grid, stream));
}

size_t bytes_of(wvae_dtype dt) { return dt == WVAE_BF16 ? 2 : 4; }

bool bf16_cout_ok(int cout) { return cout > 0 && cout % 16 == 0 && (cout <= 256 || cout == 512); }

}  // namespace

unsigned* device_error_word() {
  DeviceInfo* d = nullptr;
  return device_info(&d) == WVAE_OK ? d->err : nullptr;
}

}  // namespace wvae

using namespace wvae;

extern "C" {

const char* wvae_status_string(int status) {
  switch (status) {
    case WVAE_OK: return "ok";
    case WVAE_ERR_INVALID_ARG: return "invalid argument";
    case WVAE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case WVAE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case WVAE_ERR_WORKSPACE: return "workspace or packed buffer too small";
    case WVAE_ERR_CUDA: return "CUDA error";
    case WVAE_ERR_TIMEOUT: return "a kernel wait exceeded its limit";
    case WVAE_ERR_NO_DEVICE: return "no sm_100 device is current";
    default: return "unknown status";
  }
}

int wvae_version(void) { return (1 << 16) | 0; }

wvae_status wvae_device_error(unsigned int* code, int reset) {
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  unsigned v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
  if (cudaMemcpy(&v, d->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_status(cudaGetLastError());
  if (reset) {
    const unsigned zero = 0;
    if (cudaMemcpy(d->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return cuda_status(cudaGetLastError());
  }
  if (code) *code = v;
  return v ? WVAE_ERR_TIMEOUT : WVAE_OK;
}

// ------------------------------------------------------------------ norm-SiLU
wvae_status wvae_norm_silu(const void* x, void* y, const float* gamma, const float* beta, int T,
                           int H, int W, int C, float eps, wvae_dtype dtype, wvae_stream_t stream) {
  if (!x || !y || !gamma || !beta) return WVAE_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || W < 1 || C < 1 || !(eps > 0.0f)) return WVAE_ERR_INVALID_ARG;
  if (dtype != WVAE_BF16 && dtype != WVAE_F32) return WVAE_ERR_UNSUPPORTED;
  const int vec = dtype == WVAE_BF16 ? 8 : 4;
  if (C % vec != 0 || C < 8 || C > 1024) return WVAE_ERR_UNSUPPORTED;
  if (!a16(x) || !a16(y)) return WVAE_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  const long nvox = static_cast<long>(T) * H * W;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WVAE_BF16)
    return cuda_status(launch_norm_silu_bf16(static_cast<const __nv_bfloat16*>(x),
                                             static_cast<__nv_bfloat16*>(y), gamma, beta, nvox, C,
                                             eps, d->num_sms, s));
  return cuda_status(launch_norm_silu_f32(static_cast<const float*>(x), static_cast<float*>(y),
                                          gamma, beta, nvox, C, eps, d->num_sms, s));
}

// ------------------------------------------------------------------ prepack
size_t wvae_conv_packed_bytes(int cout, int cin, int kt, int kh, int kw, wvae_dtype dtype) {
  if (cout < 1 || cin < 1 || !kernel_ok(kt, kh, kw)) return 0;
  if (dtype != WVAE_BF16 && dtype != WVAE_F32) return 0;
  return packed_layout(cout, cin, kt, kh, kw, dtype).total;
}

wvae_status wvae_prepack_conv(const void* w, wvae_dtype w_dtype, const float* bias, int cout,
                              int cin, int kt, int kh, int kw, wvae_dtype dtype, void* packed,
                              size_t packed_bytes, wvae_stream_t stream) {
  if (!w || !packed) return WVAE_ERR_INVALID_ARG;
  if (cout < 1 || cin < 1) return WVAE_ERR_INVALID_ARG;
  if (!kernel_ok(kt, kh, kw)) return WVAE_ERR_UNSUPPORTED;
  if ((w_dtype != WVAE_BF16 && w_dtype != WVAE_F32) || (dtype != WVAE_BF16 && dtype != WVAE_F32))
    return WVAE_ERR_UNSUPPORTED;
  if (!a16(packed)) return WVAE_ERR_ALIGNMENT;
  const PackedLayout L = packed_layout(cout, cin, kt, kh, kw, dtype);
  if (packed_bytes < L.total) return WVAE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* bias_p = reinterpret_cast<float*>(static_cast<char*>(packed) + L.bias_off);
  if (dtype == WVAE_BF16)
    return cuda_status(launch_prepack_bf16(w, w_dtype == WVAE_F32, bias, cout, cin, L.taps,
                                           L.cout_pad, L.cin_pad,
                                           static_cast<__nv_bfloat16*>(packed), bias_p, s));
  return cuda_status(launch_prepack_f32(w, w_dtype == WVAE_F32, bias, cout, cin, L.taps,
                                        static_cast<float*>(packed), bias_p, s));
}

// ------------------------------------------------------------- causal conv3d
size_t wvae_causal_conv3d_workspace_bytes(int T, int H, int W, int cin, int has_norm,
                                          wvae_dtype dtype) {
  if (!has_norm || T < 1 || H < 1 || W < 1 || cin < 1) return 0;
  return round_up_sz(static_cast<size_t>(T) * H * W * cin * bytes_of(dtype), 256);
}

wvae_status wvae_causal_conv3d(const void* x, const void* cache, const void* packed_w, int T,
                               int H, int W, int cin, int cout, int kt, int kh, int kw,
                               const float* norm_gamma, const float* norm_beta,
                               const void* residual, void* y, wvae_dtype dtype, void* workspace,
                               size_t ws_bytes, wvae_stream_t stream) {
  if (!x || !packed_w || !y) return WVAE_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || W < 1 || cin < 1 || cout < 1) return WVAE_ERR_INVALID_ARG;
  if ((norm_gamma == nullptr) != (norm_beta == nullptr)) return WVAE_ERR_INVALID_ARG;
  if (!kernel_ok(kt, kh, kw)) return WVAE_ERR_UNSUPPORTED;
  if (dtype != WVAE_BF16 && dtype != WVAE_F32) return WVAE_ERR_UNSUPPORTED;
  if (cache != nullptr && kt < 2) return WVAE_ERR_INVALID_ARG;
  if (x == y || (residual != nullptr && residual == y) || (cache != nullptr && cache == y))
    return WVAE_ERR_INVALID_ARG;
  if (!a16(x) || !a16(y) || !a16(packed_w) || (cache && !a16(cache)) ||
      (residual && !a16(residual)) || (workspace && !a16(workspace)))
    return WVAE_ERR_ALIGNMENT;
  if (dtype == WVAE_BF16 && (cin % 64 != 0 || !bf16_cout_ok(cout))) return WVAE_ERR_UNSUPPORTED;
  if (dtype == WVAE_F32 && (cin % 4 != 0 || cout % 4 != 0)) return WVAE_ERR_UNSUPPORTED;
  const bool has_norm = norm_gamma != nullptr;
  const size_t need = wvae_causal_conv3d_workspace_bytes(T, H, W, cin, has_norm, dtype);
  if (has_norm && (workspace == nullptr || ws_bytes < need)) return WVAE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const void* a = x;
  if (has_norm) {
    st = wvae_norm_silu(x, workspace, norm_gamma, norm_beta, T, H, W, cin, 1e-12f, dtype, stream);
    if (st != WVAE_OK) return st;
    a = workspace;
  }
  if (dtype == WVAE_F32) {
    const PackedLayout L = packed_layout(cout, cin, kt, kh, kw, WVAE_F32);
    ConvF32Params p;
    p.x = static_cast<const float*>(a);
    p.cache = static_cast<const float*>(cache);
    p.w = static_cast<const float*>(packed_w);
    p.bias = reinterpret_cast<const float*>(static_cast<const char*>(packed_w) + L.bias_off);
    p.residual = static_cast<const float*>(residual);
    p.y = static_cast<float*>(y);
    p.T = T; p.H = H; p.W = W; p.cin = cin; p.cout = cout; p.KT = kt; p.KH = kh; p.KW = kw;
    return cuda_status(launch_conv_f32(p, s));
  }
  TcConv c;
  c.x = a;
  c.cin_pad = cin;
  c.cache = cache;
  c.packed = packed_w;
  c.cout = cout;
  c.KT = kt; c.KH = kh; c.KW = kw;
  c.T = T; c.H = H; c.W = W;
  c.ep.residual = residual;
  c.ep.residual_f32 = 0;
  c.ep.out = y;
  c.ep.out_f32 = 0;
  return run_tc_conv(*d, c, s);
}

// ---------------------------------------------------- Winograd F(2x2, 3x3)
namespace {
// Packed Winograd weights: fp16 U [cout_pad][16 x 3][cin_pad], then a zero
// bias (the products take none) and the conv's bias, fp32 [cout_pad] each.
PackedLayout wino_layout(int cout, int cin) {
  PackedLayout L = packed_layout(cout, cin, 3, 16, 1, WVAE_BF16);
  L.total += static_cast<size_t>(L.cout_pad) * 4;
  return L;
}
size_t wino_planes_bytes(int T, int H, int W, int C) {
  return round_up_sz(16ull * T * ((H + 1) / 2) * ((W + 1) / 2) * C * 2, 256);
}
}  // namespace

size_t wvae_conv_winograd_packed_bytes(int cout, int cin) {
  if (cout < 1 || cin < 1) return 0;
  return wino_layout(cout, cin).total;
}

wvae_status wvae_prepack_conv_winograd(const void* w, wvae_dtype w_dtype, const float* bias,
                                       int cout, int cin, void* packed, size_t packed_bytes,
                                       wvae_stream_t stream) {
  if (!w || !packed) return WVAE_ERR_INVALID_ARG;
  if (cout < 1 || cin < 1) return WVAE_ERR_INVALID_ARG;
  if (w_dtype != WVAE_BF16 && w_dtype != WVAE_F32) return WVAE_ERR_UNSUPPORTED;
  if (!a16(packed)) return WVAE_ERR_ALIGNMENT;
  const PackedLayout L = wino_layout(cout, cin);
  if (packed_bytes < L.total) return WVAE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  float* bias_zero = reinterpret_cast<float*>(static_cast<char*>(packed) + L.bias_off);
  return cuda_status(launch_wino_prepack(w, w_dtype == WVAE_F32, bias, cout, cin, L.cout_pad,
                                         L.cin_pad, static_cast<__half*>(packed), bias_zero,
                                         bias_zero + L.cout_pad,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

size_t wvae_causal_conv3d_winograd_workspace_bytes(int T, int H, int W, int cin, int cout) {
  if (T < 1 || H < 1 || W < 1 || cin < 1 || cout < 1) return 0;
  return wino_planes_bytes(T, H, W, cin) + wino_planes_bytes(T, H, W, cout);
}

wvae_status wvae_causal_conv3d_winograd(const void* x, const void* packed_w, int T, int H, int W,
                                        int cin, int cout, const void* residual, void* y,
                                        void* workspace, size_t ws_bytes, wvae_stream_t stream) {
  if (!x || !packed_w || !y || !workspace) return WVAE_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || W < 1 || cin < 1 || cout < 1) return WVAE_ERR_INVALID_ARG;
  if (x == y || (residual != nullptr && residual == y)) return WVAE_ERR_INVALID_ARG;
  if (!a16(x) || !a16(y) || !a16(packed_w) || !a16(workspace) || (residual && !a16(residual)))
    return WVAE_ERR_ALIGNMENT;
  if (cin % 64 != 0 || !bf16_cout_ok(cout)) return WVAE_ERR_UNSUPPORTED;
  if (ws_bytes < wvae_causal_conv3d_winograd_workspace_bytes(T, H, W, cin, cout))
    return WVAE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  __half* v = static_cast<__half*>(workspace);
  __half* m = reinterpret_cast<__half*>(static_cast<char*>(workspace) +
                                        wino_planes_bytes(T, H, W, cin));
  st = cuda_status(launch_wino_input(static_cast<const __nv_bfloat16*>(x), v, T, H, W, cin, s));
  if (st != WVAE_OK) return st;
  TcConv c;
  c.x = v;
  c.cin_pad = cin;
  c.packed = packed_w;
  c.cout = cout;
  c.KT = 3;
  c.T = T;
  c.H = (H + 1) / 2;
  c.W = (W + 1) / 2;
  c.wino = 1;
  c.ep.out = m;
  c.ep.out_f16 = 1;
  st = run_tc_conv(*d, c, s);
  if (st != WVAE_OK) return st;
  const PackedLayout L = wino_layout(cout, cin);
  const float* bias = reinterpret_cast<const float*>(static_cast<const char*>(packed_w) + L.bias_off) +
                      L.cout_pad;
  return cuda_status(launch_wino_output(m, bias, static_cast<const __nv_bfloat16*>(residual),
                                        static_cast<__nv_bfloat16*>(y), T, H, W, cout, s));
}

// ------------------------------------------------------------ residual block
size_t wvae_resblock_workspace_bytes(int T, int H, int W, int cin, int cout, wvae_dtype dtype) {
  if (T < 1 || H < 1 || W < 1 || cin < 1 || cout < 1) return 0;
  const size_t nvox = static_cast<size_t>(T) * H * W;
  const size_t c1 = dtype == WVAE_F32 ? std::max(cin, cout) : cin;
  return round_up_sz(nvox * c1 * bytes_of(dtype), 256) + round_up_sz(nvox * cout * bytes_of(dtype), 256);
}

wvae_status wvae_resblock(const void* x, void* y, int T, int H, int W, int cin, int cout,
                          const float* gamma1, const float* beta1, const void* w1_packed,
                          const float* gamma2, const float* beta2, const void* w2_packed,
                          const void* wsc_packed, wvae_dtype dtype, void* workspace,
                          size_t ws_bytes, wvae_stream_t stream) {
  if (!x || !y || !gamma1 || !beta1 || !w1_packed || !gamma2 || !beta2 || !w2_packed)
    return WVAE_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || W < 1 || cin < 1 || cout < 1) return WVAE_ERR_INVALID_ARG;
  if ((cin != cout) != (wsc_packed != nullptr)) return WVAE_ERR_INVALID_ARG;
  if (x == y) return WVAE_ERR_INVALID_ARG;
  if (dtype != WVAE_BF16 && dtype != WVAE_F32) return WVAE_ERR_UNSUPPORTED;
  if (!a16(x) || !a16(y) || !a16(w1_packed) || !a16(w2_packed) || (wsc_packed && !a16(wsc_packed)) ||
      (workspace && !a16(workspace)))
    return WVAE_ERR_ALIGNMENT;
  if (dtype == WVAE_BF16 && (cin % 64 != 0 || cout % 64 != 0 || !bf16_cout_ok(cout)))
    return WVAE_ERR_UNSUPPORTED;
  if (dtype == WVAE_F32 && (cin % 4 != 0 || cout % 4 != 0)) return WVAE_ERR_UNSUPPORTED;
  const size_t need = wvae_resblock_workspace_bytes(T, H, W, cin, cout, dtype);
  if (workspace == nullptr || ws_bytes < need) return WVAE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t nvox = static_cast<size_t>(T) * H * W;
  char* a1 = static_cast<char*>(workspace);
  const size_t a1_ch = dtype == WVAE_F32 ? std::max(cin, cout) : cin;
  char* a2 = a1 + round_up_sz(nvox * a1_ch * bytes_of(dtype), 256);

  // A1 = SiLU(norm1(x))
  st = wvae_norm_silu(x, a1, gamma1, beta1, T, H, W, cin, 1e-12f, dtype, stream);
  if (st != WVAE_OK) return st;

  if (dtype == WVAE_F32) {
    // h1 = conv1(A1) -> a2 buffer, then A2 in place, then conv2 (+ shortcut).
    st = wvae_causal_conv3d(a1, nullptr, w1_packed, T, H, W, cin, cout, 3, 3, 3, nullptr, nullptr,
                            nullptr, a2, dtype, nullptr, 0, stream);
    if (st != WVAE_OK) return st;
    st = wvae_norm_silu(a2, a2, gamma2, beta2, T, H, W, cout, 1e-12f, dtype, stream);
    if (st != WVAE_OK) return st;
    const void* res = x;
    if (wsc_packed != nullptr) {
      // the shortcut goes to the a1 buffer (A1 is no longer needed; it is
      // sized for max(cin, cout) channels on this path)
      st = wvae_causal_conv3d(x, nullptr, wsc_packed, T, H, W, cin, cout, 1, 1, 1, nullptr,
                              nullptr, nullptr, a1, dtype, nullptr, 0, stream);
      if (st != WVAE_OK) return st;
      res = a1;
    }
    return wvae_causal_conv3d(a2, nullptr, w2_packed, T, H, W, cout, cout, 3, 3, 3, nullptr,
                              nullptr, res, y, dtype, nullptr, 0, stream);
  }

  // conv1 with norm2 + SiLU in its epilogue: writes A2 directly.
  TcConv c1;
  c1.x = a1;
  c1.cin_pad = cin;
  c1.packed = w1_packed;
  c1.cout = cout;
  c1.T = T; c1.H = H; c1.W = W;
  c1.ep.act = reinterpret_cast<__nv_bfloat16*>(a2);
  c1.ep.gamma = gamma2;
  c1.ep.beta = beta2;
  c1.ep.eps = 1e-12f;
  st = run_tc_conv(*d, c1, s);
  if (st != WVAE_OK) return st;

  // conv2 (+ the 1x1x1 shortcut as a second K segment, or + x) -> y.
  TcConv c2;
  c2.x = a2;
  c2.cin_pad = cout;
  c2.packed = w2_packed;
  c2.cout = cout;
  c2.T = T; c2.H = H; c2.W = W;
  if (wsc_packed != nullptr) {
    c2.x2 = x;
    c2.cin2_pad = cin;
    c2.packed2 = wsc_packed;
  } else {
    c2.ep.residual = x;
    c2.ep.residual_f32 = 0;
  }
  c2.ep.out = y;
  c2.ep.out_f32 = 0;
  return run_tc_conv(*d, c2, s);
}

// ------------------------------------------------------ upsample + 3x3 conv
size_t wvae_upsample_conv_packed_bytes(int cout, int cin, wvae_dtype dtype) {
  if (cout < 1 || cin < 1) return 0;
  if (dtype == WVAE_BF16) return packed_layout(cout, cin, 1, 4, 4, WVAE_BF16).total;
  if (dtype == WVAE_F32) return packed_layout(cout, cin, 1, 3, 3, WVAE_F32).total;
  return 0;
}

wvae_status wvae_prepack_upsample_conv(const void* w, wvae_dtype w_dtype, const float* bias,
                                       int cout, int cin, wvae_dtype dtype, void* packed,
                                       size_t packed_bytes, wvae_stream_t stream) {
  if (!w || !packed) return WVAE_ERR_INVALID_ARG;
  if (cout < 1 || cin < 1) return WVAE_ERR_INVALID_ARG;
  if ((w_dtype != WVAE_BF16 && w_dtype != WVAE_F32) || (dtype != WVAE_BF16 && dtype != WVAE_F32))
    return WVAE_ERR_UNSUPPORTED;
  if (!a16(packed)) return WVAE_ERR_ALIGNMENT;
  if (packed_bytes < wvae_upsample_conv_packed_bytes(cout, cin, dtype)) return WVAE_ERR_WORKSPACE;
  if (dtype == WVAE_F32)
    return wvae_prepack_conv(w, w_dtype, bias, cout, cin, 1, 3, 3, WVAE_F32, packed, packed_bytes,
                             stream);
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  const PackedLayout L = packed_layout(cout, cin, 1, 4, 4, WVAE_BF16);
  float* bias_p = reinterpret_cast<float*>(static_cast<char*>(packed) + L.bias_off);
  return cuda_status(launch_prepack_phase_bf16(w, w_dtype == WVAE_F32, bias, cout, cin, L.cout_pad,
                                               L.cin_pad, static_cast<__nv_bfloat16*>(packed),
                                               bias_p, reinterpret_cast<cudaStream_t>(stream)));
}

size_t wvae_upsample_conv_workspace_bytes(int T, int H, int W, int cin, wvae_dtype dtype) {
  if (T < 1 || H < 1 || W < 1 || cin < 1 || dtype != WVAE_F32) return 0;
  return round_up_sz(static_cast<size_t>(T) * 4 * H * W * cin * bytes_of(dtype), 256);
}

wvae_status wvae_upsample_conv(const void* x, void* y, int T, int H, int W, int cin, int cout,
                               const void* packed_w, wvae_dtype dtype, void* workspace,
                               size_t ws_bytes, wvae_stream_t stream) {
  if (!x || !y || !packed_w) return WVAE_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || W < 1 || cin < 1 || cout < 1) return WVAE_ERR_INVALID_ARG;
  if (x == y) return WVAE_ERR_INVALID_ARG;
  if (dtype != WVAE_BF16 && dtype != WVAE_F32) return WVAE_ERR_UNSUPPORTED;
  if (!a16(x) || !a16(y) || !a16(packed_w) || (workspace && !a16(workspace)))
    return WVAE_ERR_ALIGNMENT;
  if (dtype == WVAE_BF16 && (cin % 64 != 0 || !bf16_cout_ok(cout))) return WVAE_ERR_UNSUPPORTED;
  if (dtype == WVAE_F32 && (cin % 4 != 0 || cout % 4 != 0)) return WVAE_ERR_UNSUPPORTED;
  const size_t need = wvae_upsample_conv_workspace_bytes(T, H, W, cin, dtype);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return WVAE_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  wvae_status st = device_info(&d);
  if (st != WVAE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WVAE_BF16) {
    TcConv c;
    c.x = x;
    c.cin_pad = cin;
    c.packed = packed_w;
    c.cout = cout;
    c.T = T; c.H = H; c.W = W;
    c.phases = 4;
    c.ep.out = y;
    c.ep.out_f32 = 0;
    return run_tc_conv(*d, c, s);
  }
  st = cuda_status(launch_upsample2x(x, workspace, static_cast<int>(bytes_of(dtype)), T, H, W, cin, s));
  if (st != WVAE_OK) return st;
  return wvae_causal_conv3d(workspace, nullptr, packed_w, T, 2 * H, 2 * W, cin, cout, 1, 3, 3,
                            nullptr, nullptr, nullptr, y, dtype, nullptr, 0, stream);
}

// ------------------------------------------------------------ decoder trunk
namespace {
const int kDefaultWidths[4] = {512, 512, 256, 128};
constexpr int kZChannels = 48;
constexpr int kZPad = 64;
constexpr int kHeadOut = 12;

struct TrunkBuffers {
  size_t zcl, h, act1, act2, up;   // byte offsets
  size_t total;
};

// F, Hs, Ws: frames, rows and columns per stage.
TrunkBuffers trunk_buffers(const int* F, const int* Hs, const int* Ws, const int* C) {
  TrunkBuffers b;
  size_t off = 0;
  auto take = [&](size_t n) {
    size_t o = off;
    off += round_up_sz(n, 256);
    return o;
  };
  const size_t v0 = static_cast<size_t>(F[0]) * Hs[0] * Ws[0];
  size_t max_h = 0, max_act = 0, max_up = 0;
  for (int s = 0; s < 4; ++s) {
    const size_t vs = static_cast<size_t>(F[s]) * Hs[s] * Ws[s];
    max_h = std::max(max_h, vs * C[s] * 4);
    max_act = std::max(max_act, vs * C[s] * 2);
    if (s < 3) max_up = std::max(max_up, vs * C[s] * 2);
  }
  b.zcl = take(v0 * kZPad * 2);
  b.h = take(max_h);
  b.act1 = take(max_act);
  b.act2 = take(max_act);
  b.up = take(max_up);
  b.total = off;
  return b;
}
}  // namespace

namespace {
// Causal conv inputs whose last two frames a chunk hands to the next one:
// conv_in, the 16 res-block convs (conv1 and conv2 of 2 blocks x 4 stages),
// the head.  Offsets into the caller's cache buffer, in that order.
constexpr int kTrunkCaches = 18;

struct TrunkCaches {
  size_t off[kTrunkCaches];
  size_t bytes[kTrunkCaches];
  size_t total;
};

TrunkCaches trunk_caches(int H, int W, const int* C) {
  TrunkCaches c;
  size_t off = 0;
  int i = 0;
  auto take = [&](size_t n) {
    c.off[i] = off;
    c.bytes[i] = n;
    off += round_up_sz(n, 256);
    ++i;
  };
  take(2ull * H * W * kZPad * 2);  // conv_in: padded latents
  for (int s = 0; s < 4; ++s) {
    const size_t frame = (static_cast<size_t>(H) << s) * (static_cast<size_t>(W) << s) * C[s] * 2;
    for (int k = 0; k < 4; ++k) take(2 * frame);  // conv1, conv2 of 2 blocks
  }
  take(2ull * (static_cast<size_t>(H) << 3) * (static_cast<size_t>(W) << 3) * C[3] * 2);  // head
  c.total = off;
  return c;
}
}  // namespace

size_t wvae_decode_trunk_cache_bytes(int H, int W, const int* widths) {
  if (H < 1 || W < 1) return 0;
  const int* C = widths ? widths : kDefaultWidths;
  for (int s = 0; s < 4; ++s)
    if (C[s] < 64) return 0;
  return trunk_caches(H, W, C).total;
}

size_t wvae_decode_trunk_workspace_bytes(int T, int H, int W, const int* widths) {
  if (T < 1 || H < 1 || W < 1) return 0;
  const int* C = widths ? widths : kDefaultWidths;
  for (int s = 0; s < 4; ++s)
    if (C[s] < 64) return 0;
  const int F[4] = {T, T, T, T};
  const int Hs[4] = {H, 2 * H, 4 * H, 8 * H}, Ws[4] = {W, 2 * W, 4 * W, 8 * W};
  return trunk_buffers(F, Hs, Ws, C).total;
}

int wvae_decode_video_frames(int T, int continue_chunk) {
  if (T < 1) return 0;
  return continue_chunk ? 4 * T : 4 * T - 3;
}

size_t wvae_decode_video_workspace_bytes(int T, int H, int W, const int* widths) {
  if (T < 1 || H < 1 || W < 1) return 0;
  const int* C = widths ? widths : kDefaultWidths;
  for (int s = 0; s < 4; ++s)
    if (C[s] < 64) return 0;
  const int F[4] = {T, 2 * T, 4 * T, 4 * T};  // a continuing chunk's counts bound the first's
  const int Hs[4] = {H, 2 * H, 4 * H, 8 * H}, Ws[4] = {W, 2 * W, 4 * W, 8 * W};
  return trunk_buffers(F, Hs, Ws, C).total;
}

// Row slab: every stage carries its own rows plus a halo row above and below.
size_t wvae_decode_rows_workspace_bytes(int T, int rows, int W, const int* widths) {
  if (T < 1 || rows < 1 || W < 1) return 0;
  const int* C = widths ? widths : kDefaultWidths;
  for (int s = 0; s < 4; ++s)
    if (C[s] < 64) return 0;
  const int F[4] = {T, T, T, T};
  const int Hs[4] = {rows + 2, 2 * rows + 2, 4 * rows + 2, 8 * rows + 2};
  const int Ws[4] = {W, 2 * W, 4 * W, 8 * W};
  return trunk_buffers(F, Hs, Ws, C).total;
}

namespace {
constexpr int kTrunkLaunches = 22;

// Where the input of one launch of a row-slab decode lives in the workspace
// (the tensor whose halo rows the caller refreshes before that launch).
struct HaloQuery {
  int step = -1;
  int found = 0;
  size_t offset = 0;
  int dims[4] = {0, 0, 0, 0};  // frames, rows (own + 2 halo), columns, channels; bf16
};

// How a decode runs: per-launch events, causal caches of a chunked decode
// (continue_chunk: read the front frames from them, else zeros; they are
// rewritten with this chunk's last two input frames of every causal conv),
// temporal upsampling, a row slab, one launch only, or a halo query.
struct TrunkRun {
  void* const* events = nullptr;
  int n_events = 0;
  void* cache = nullptr;
  size_t cache_bytes = 0;
  int continue_chunk = 0;
  int temporal = 0;
  int rows = 0;            // > 0: a slab of `rows` latent rows (H == rows), one halo row
                           // above and below at every stage
  int only_step = -1;      // >= 0: enqueue launch `only_step` alone
  HaloQuery* query = nullptr;  // enqueue nothing; describe query->step's input
};

wvae_status decode_trunk_impl(const void* const* packed, const float* const* norms, const void* z,
                              void* video, int T, int H, int W, const int* widths,
                              wvae_dtype dtype, void* workspace, size_t ws_bytes,
                              const TrunkRun& run, wvae_stream_t stream) {
  void* const* events = run.events;
  void* cache = run.cache;
  const int continue_chunk = run.continue_chunk;
  const bool query = run.query != nullptr;
  const bool slab = run.rows > 0;
  if (!query && (!packed || !norms || !z || !video || !workspace)) return WVAE_ERR_INVALID_ARG;
  if (cache != nullptr && T < 2) return WVAE_ERR_INVALID_ARG;  // the cache holds two frames
  if (events != nullptr && run.n_events < 2 * kTrunkLaunches) return WVAE_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || W < 1) return WVAE_ERR_INVALID_ARG;
  if (slab && (cache != nullptr || run.temporal)) return WVAE_ERR_UNSUPPORTED;
  if (run.only_step >= kTrunkLaunches) return WVAE_ERR_INVALID_ARG;
  if (dtype != WVAE_BF16) return WVAE_ERR_UNSUPPORTED;
  const int* C = widths ? widths : kDefaultWidths;
  for (int s = 0; s < 4; ++s)
    if (C[s] % 64 != 0 || !bf16_cout_ok(C[s])) return WVAE_ERR_UNSUPPORTED;
  if (!query) {
    for (int i = 0; i < 21; ++i)
      if (!packed[i]) return WVAE_ERR_INVALID_ARG;
    for (int i = 0; i < 34; ++i)
      if (!norms[i]) return WVAE_ERR_INVALID_ARG;
    for (int i = 0; i < 21; ++i)
      if (!a16(packed[i])) return WVAE_ERR_ALIGNMENT;
    if (!a16(z) || !a16(video) || !a16(workspace)) return WVAE_ERR_ALIGNMENT;
  }
  if (continue_chunk && cache == nullptr) return WVAE_ERR_INVALID_ARG;
  // Frames per stage: with temporal upsampling the upsample convs of stages 0
  // and 1 also double the frames (the decode's first frame once).
  const bool first = !continue_chunk;
  int F[4] = {T, T, T, T};
  if (run.temporal) {
    F[1] = first ? 2 * T - 1 : 2 * T;
    F[2] = first ? 2 * F[1] - 1 : 2 * F[1];
    F[3] = F[2];
  }
  // Rows and columns per stage; a slab's tensors carry a halo row on each side.
  int HS[4], WS[4];
  for (int s2 = 0; s2 < 4; ++s2) {
    HS[s2] = slab ? (run.rows << s2) + 2 : H << s2;
    WS[s2] = W << s2;
  }
  const TrunkBuffers B = trunk_buffers(F, HS, WS, C);
  if (!query && ws_bytes < B.total) return WVAE_ERR_WORKSPACE;
  const TrunkCaches K = trunk_caches(H, W, C);
  if (cache != nullptr) {
    if (!a16(cache)) return WVAE_ERR_ALIGNMENT;
    if (run.cache_bytes < K.total) return WVAE_ERR_WORKSPACE;
  }
  DeviceInfo* d = nullptr;
  if (!query) {
    wvae_status st0 = device_info(&d);
    if (st0 != WVAE_OK) return st0;
  }
  wvae_status st = WVAE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int launch = 0;
  // whether launch `launch` is enqueued by this call
  auto exec = [&]() { return !query && (run.only_step < 0 || run.only_step == launch); };
  auto mark = [&](int which) {
    if (events != nullptr && exec())
      cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[2 * launch + which]), s);
  };
  char* ws = static_cast<char*>(workspace);
  // the input of a 3x3 conv whose halo a slab's caller refreshes
  auto note_input = [&](const void* x, int t, int hh, int ww, int cc) {
    if (query && run.query->step == launch) {
      run.query->found = 1;
      run.query->offset = static_cast<size_t>(static_cast<const char*>(x) - ws);
      run.query->dims[0] = t;
      run.query->dims[1] = hh;
      run.query->dims[2] = ww;
      run.query->dims[3] = cc;
    }
  };
  auto conv = [&](const TcConv& c) {
    if (slab && launch > 1) note_input(c.x, c.T, c.H, c.W, c.cin_pad);
    wvae_status r = WVAE_OK;
    if (exec()) {
      mark(0);
      r = run_tc_conv(*d, c, s);
      mark(1);
    }
    ++launch;
    return r;
  };
  // A causal conv of a chunked decode: front frames from cache entry k, then
  // the last two frames of its input x (T frames of `frame` bytes) become the
  // next chunk's entry k.
  int ck = 0;
  auto causal_conv = [&](TcConv c, size_t frame) {
    char* entry = cache != nullptr ? static_cast<char*>(cache) + K.off[ck] : nullptr;
    ++ck;
    if (entry != nullptr && continue_chunk) c.cache = entry;
    wvae_status r = conv(c);
    if (r != WVAE_OK || entry == nullptr) return r;
    return cuda_status(cudaMemcpyAsync(entry, static_cast<const char*>(c.x) + (c.T - 2) * frame,
                                       2 * frame, cudaMemcpyDeviceToDevice, s));
  };
  void* zcl = ws + B.zcl;
  float* h = reinterpret_cast<float*>(ws + B.h);
  __nv_bfloat16* act[2] = {reinterpret_cast<__nv_bfloat16*>(ws + B.act1),
                           reinterpret_cast<__nv_bfloat16*>(ws + B.act2)};
  void* up = ws + B.up;

  // latents NCDHW -> channels-last, channels padded 48 -> 64 (a slab's latents
  // come with their halo rows: the caller reads them from the whole latents)
  if (exec()) {
    mark(0);
    st = cuda_status(launch_ncdhw_to_cl_pad(static_cast<const __nv_bfloat16*>(z),
                                            static_cast<__nv_bfloat16*>(zcl), kZChannels, kZPad, T,
                                            HS[0], W, s));
    mark(1);
  }
  ++launch;
  if (st != WVAE_OK) return st;

  int pi = 0, ni = 0;
  auto next_norm = [&](const float** g, const float** b) {
    *g = norms ? norms[2 * ni] : nullptr;
    *b = norms ? norms[2 * ni + 1] : nullptr;
    ++ni;
  };
  auto next_packed = [&]() { return packed ? packed[pi++] : (++pi, nullptr); };
  int Hs = HS[0], Ws = W;

  // conv_in: residual stream h (fp32) + A1 of stage 0, block 0.
  {
    TcConv c;
    c.x = zcl;
    c.cin_pad = kZPad;
    c.packed = next_packed();
    c.cout = C[0];
    c.T = T; c.H = Hs; c.W = Ws;
    c.ep.out = h;
    c.ep.out_f32 = 1;
    c.ep.act = act[0];
    next_norm(&c.ep.gamma, &c.ep.beta);
    c.ep.eps = 1e-12f;
    st = causal_conv(c, static_cast<size_t>(Hs) * W * kZPad * 2);
    if (st != WVAE_OK) return st;
  }
  for (int stg = 0; stg < 4; ++stg) {
    const int Cs = C[stg];
    const int Ts = F[stg];
    const size_t frame = static_cast<size_t>(Hs) * Ws * Cs * 2;  // bf16 activation frame
    for (int blk = 0; blk < 2; ++blk) {
      // conv1: A1 -> A2 (norm2 in the epilogue)
      TcConv c1;
      c1.x = act[0];
      c1.cin_pad = Cs;
      c1.packed = next_packed();
      c1.cout = Cs;
      c1.T = Ts; c1.H = Hs; c1.W = Ws;
      c1.ep.act = act[1];
      next_norm(&c1.ep.gamma, &c1.ep.beta);
      c1.ep.eps = 1e-12f;
      st = causal_conv(c1, frame);
      if (st != WVAE_OK) return st;
      // conv2: h + conv2(A2) -> h (fp32, in place per voxel) and the next activation
      TcConv c2;
      c2.x = act[1];
      c2.cin_pad = Cs;
      c2.packed = next_packed();
      c2.cout = Cs;
      c2.T = Ts; c2.H = Hs; c2.W = Ws;
      c2.ep.residual = h;
      c2.ep.residual_f32 = 1;
      const bool last_block = blk == 1;
      if (!last_block) {
        c2.ep.out = h;
        c2.ep.out_f32 = 1;
        c2.ep.act = act[0];
        next_norm(&c2.ep.gamma, &c2.ep.beta);
        c2.ep.eps = 1e-12f;
      } else if (stg < 3) {
        // the stage's output feeds only the upsample conv (an MMA operand): bf16
        c2.ep.out = up;
        c2.ep.out_f32 = 0;
      } else {
        // the last block feeds only norm_out + SiLU + head
        c2.ep.act = act[0];
        next_norm(&c2.ep.gamma, &c2.ep.beta);
        c2.ep.eps = 1e-12f;
      }
      st = causal_conv(c2, frame);
      if (st != WVAE_OK) return st;
    }
    if (stg < 3) {
      // nearest 2x upsample + 3x3 conv as four phase convs on the low-res stage output
      TcConv cu;
      cu.x = up;
      cu.cin_pad = Cs;
      cu.packed = next_packed();
      cu.cout = C[stg + 1];
      cu.T = Ts; cu.H = Hs; cu.W = Ws;
      cu.phases = 4;
      if (F[stg + 1] != Ts) cu.tdup = first ? 1 : 2;
      if (slab) {
        // output row 2h + p' of the halo-extended input is row 2h + p' - 1 of the
        // next stage's slab (its own rows and one halo row each side)
        cu.out_row0 = 1;
        cu.out_rows = HS[stg + 1];
      }
      Hs = HS[stg + 1];
      Ws *= 2;
      cu.ep.out = h;
      cu.ep.out_f32 = 1;
      cu.ep.act = act[0];
      next_norm(&cu.ep.gamma, &cu.ep.beta);
      cu.ep.eps = 1e-12f;
      st = conv(cu);
      if (st != WVAE_OK) return st;
    }
  }
  // head: A_out -> causal conv to 12 channels -> pixel-shuffled video.  At 64
  // or 128 channels the head kernel puts the temporal and column taps in N.
  if (C[3] <= 128) {
    char* entry = cache != nullptr ? static_cast<char*>(cache) + K.off[ck] : nullptr;
    ++ck;
    if (slab) note_input(act[0], F[3], Hs, Ws, C[3]);
    const void* pk = next_packed();
    if (exec()) {
      HeadParams hp;
      std::memset(&hp, 0, sizeof(hp));
      const PackedLayout L = packed_layout(kHeadOut, C[3], 3, 3, 3, WVAE_BF16);
      if (!encode_act(&hp.tmA, act[0], C[3], Ws, Hs, F[3], kHeadTileCols, kHeadTileRows + 2))
        return WVAE_ERR_CUDA;
      if (entry != nullptr && continue_chunk) {
        if (!encode_act(&hp.tmC, entry, C[3], Ws, Hs, 2, kHeadTileCols, kHeadTileRows + 2))
          return WVAE_ERR_CUDA;
        hp.has_cache = 1;
      }
      if (!encode_weights(&hp.tmB, pk, L.taps * C[3], L.cout_pad, 16)) return WVAE_ERR_CUDA;
      hp.bias = reinterpret_cast<const float*>(static_cast<const char*>(pk) + L.bias_off);
      hp.video = static_cast<__nv_bfloat16*>(video);
      hp.T = F[3];
      hp.H = Hs;
      hp.W = Ws;
      hp.cin = C[3];
      hp.row0 = slab ? 1 : 0;
      hp.rows_out = slab ? Hs - 2 : Hs;
      hp.tiles_w = (Ws + kHeadOutCols - 1) / kHeadOutCols;
      hp.tiles_h = (Hs + kHeadTileRows - 1) / kHeadTileRows;
      hp.num_tiles = hp.tiles_w * hp.tiles_h;
      hp.err = d->err;
      mark(0);
      st = cuda_status(launch_head_tc(hp, d->num_sms, s));
      mark(1);
    }
    ++launch;
    if (st != WVAE_OK || entry == nullptr || query) return st;
    const size_t frame = static_cast<size_t>(Hs) * Ws * C[3] * 2;
    return cuda_status(cudaMemcpyAsync(entry, reinterpret_cast<const char*>(act[0]) + (F[3] - 2) * frame,
                                       2 * frame, cudaMemcpyDeviceToDevice, s));
  }
  if (slab) return WVAE_ERR_UNSUPPORTED;  // the slab's head needs the head kernel (C3 <= 128)
  TcConv ch;
  ch.x = act[0];
  ch.cin_pad = C[3];
  ch.packed = next_packed();
  ch.cout = kHeadOut;
  ch.T = F[3]; ch.H = Hs; ch.W = Ws;
  ch.ep.video = static_cast<__nv_bfloat16*>(video);
  return causal_conv(ch, static_cast<size_t>(Hs) * Ws * C[3] * 2);
}
}  // namespace

int wvae_decode_trunk_launches(void) { return kTrunkLaunches; }

wvae_status wvae_decode_trunk(const void* const* packed, const float* const* norms, const void* z,
                              void* video, int T, int H, int W, const int* widths,
                              wvae_dtype dtype, void* workspace, size_t ws_bytes,
                              wvae_stream_t stream) {
  return decode_trunk_impl(packed, norms, z, video, T, H, W, widths, dtype, workspace, ws_bytes,
                           TrunkRun{}, stream);
}

wvae_status wvae_decode_trunk_chunk(const void* const* packed, const float* const* norms,
                                    const void* z, void* video, int T, int H, int W,
                                    const int* widths, wvae_dtype dtype, void* workspace,
                                    size_t ws_bytes, void* cache, size_t cache_bytes,
                                    int continue_chunk, wvae_stream_t stream) {
  if (cache == nullptr) return WVAE_ERR_INVALID_ARG;
  TrunkRun run;
  run.cache = cache;
  run.cache_bytes = cache_bytes;
  run.continue_chunk = continue_chunk;
  return decode_trunk_impl(packed, norms, z, video, T, H, W, widths, dtype, workspace, ws_bytes,
                           run, stream);
}

wvae_status wvae_decode_video(const void* const* packed, const float* const* norms, const void* z,
                              void* video, int T, int H, int W, const int* widths,
                              wvae_dtype dtype, void* workspace, size_t ws_bytes, void* cache,
                              size_t cache_bytes, int continue_chunk, wvae_stream_t stream) {
  if (cache == nullptr && continue_chunk) return WVAE_ERR_INVALID_ARG;
  TrunkRun run;
  run.cache = cache;
  run.cache_bytes = cache_bytes;
  run.continue_chunk = continue_chunk;
  run.temporal = 1;
  return decode_trunk_impl(packed, norms, z, video, T, H, W, widths, dtype, workspace, ws_bytes,
                           run, stream);
}

int wvae_decode_rows_steps(void) { return kTrunkLaunches; }

wvae_status wvae_decode_rows_halo(int step, int T, int rows, int W, const int* widths,
                                  size_t* offset, int* dims) {
  if (!offset || !dims || step < 0 || step >= kTrunkLaunches) return WVAE_ERR_INVALID_ARG;
  HaloQuery q;
  q.step = step;
  TrunkRun run;
  run.rows = rows;
  run.query = &q;
  const wvae_status st = decode_trunk_impl(nullptr, nullptr, nullptr, nullptr, T, rows, W, widths,
                                           WVAE_BF16, nullptr, 0, run, nullptr);
  if (st != WVAE_OK) return st;
  *offset = q.found ? q.offset : 0;
  for (int i = 0; i < 4; ++i) dims[i] = q.found ? q.dims[i] : 0;
  return WVAE_OK;
}

wvae_status wvae_decode_rows_step(int step, const void* const* packed, const float* const* norms,
                                  const void* z_rows, void* video_rows, int T, int rows, int W,
                                  const int* widths, wvae_dtype dtype, void* workspace,
                                  size_t ws_bytes, wvae_stream_t stream) {
  if (step < 0 || step >= kTrunkLaunches) return WVAE_ERR_INVALID_ARG;
  TrunkRun run;
  run.rows = rows;
  run.only_step = step;
  return decode_trunk_impl(packed, norms, z_rows, video_rows, T, rows, W, widths, dtype, workspace,
                           ws_bytes, run, stream);
}

wvae_status wvae_decode_trunk_timed(const void* const* packed, const float* const* norms,
                                    const void* z, void* video, int T, int H, int W,
                                    const int* widths, wvae_dtype dtype, void* workspace,
                                    size_t ws_bytes, void* const* events, int n_events,
                                    wvae_stream_t stream) {
  if (events == nullptr) return WVAE_ERR_INVALID_ARG;
  TrunkRun run;
  run.events = events;
  run.n_events = n_events;
  return decode_trunk_impl(packed, norms, z, video, T, H, W, widths, dtype, workspace, ws_bytes,
                           run, stream);
}

// ------------------------------------------------- res block, no allocation
// Scratch for wvae_resblock_noalloc: its A1 and A2 activations.  A file-scope
// device array, so callers that cannot allocate need not; it exists on every
// GPU that loads this library until the process exits.  In host code the
// array's name is not a device address: the address is looked up once per
// device with cudaGetSymbolAddress and passed to the kernels.
}  // extern "C"

namespace wvae {
namespace {
constexpr size_t kNoAllocScratchBytes = 64ull << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device (set-up on the
// first call per device, with that device current).
wvae_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return WVAE_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return WVAE_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return WVAE_OK;
}
}  // namespace
}  // namespace wvae

extern "C" {

wvae_status wvae_resblock_noalloc(const void* x, void* y, int T, int H, int W, int cin, int cout,
                                  const float* gamma1, const float* beta1, const void* w1_packed,
                                  const float* gamma2, const float* beta2, const void* w2_packed,
                                  const void* wsc_packed, wvae_stream_t stream) {
  if (T < 1 || H < 1 || W < 1 || cin < 1 || cout < 1) return WVAE_ERR_INVALID_ARG;
  const size_t need = wvae_resblock_workspace_bytes(T, H, W, cin, cout, WVAE_BF16);
  if (need > kNoAllocScratchBytes) return WVAE_ERR_WORKSPACE;
  if (!x || !y || !gamma1 || !beta1 || !w1_packed || !gamma2 || !beta2 || !w2_packed)
    return WVAE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  wvae_status st = noalloc_scratch(&scratch);
  if (st != WVAE_OK) return st;
  return wvae_resblock(x, y, T, H, W, cin, cout, gamma1, beta1, w1_packed, gamma2, beta2,
                       w2_packed, wsc_packed, WVAE_BF16, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"

/*
 * wvae.h - C ABI of the B200 (sm_100a) Wan-style video-VAE decoder hot path.
 *
 * The operations are those of the Wan2.2 VAE decoder's residual block and the
 * layers around it:
 *   - channel RMS-norm + affine + SiLU ("Opt-in BF16 norm-SiLU fusion for Wan
 *     VAE decoding", TensorRT-LLM issue #19309, section "Feature, motivation
 *     and proposed scope": decoder residual norm1/norm2 and norm_out);
 *   - causal 3x3x3 conv3d with bf16 operands and fp32 accumulation (FastVideo
 *     "Wan2.2 VAE decoder (sm_100a, sm_103a)" README, section "Limits");
 *   - the residual block, the nearest-2x upsample + 3x3 conv, and the decoder
 *     trunk from latents [1, 48, T, H, W] to video [1, 3, T, 16H, 16W], or,
 *     with the decoder's temporal upsampling, [1, 3, 4T - 3, 16H, 16W]
 *     (same README, opening section: 48 latent channels, 16x16 spatial and
 *     4x temporal compression; raw entry points are destination-passing on
 *     the current stream, section "Use").
 *
 * Conventions shared by every entry point:
 *   - Memory: every pointer argument named as a tensor is a DEVICE pointer owned
 *     by the caller; the library never allocates, frees or keeps device memory
 *     (the only device-side state is a 4-byte error word, see
 *     wvae_device_error).  Arrays of pointers (wvae_decode_trunk) are HOST
 *     arrays holding device pointers.
 *   - Layout: activations are batch-1 channels-last [T][H][W][C], contiguous.
 *     The trunk alone takes its latents and returns its video in NCDHW order
 *     ([1][C][T][H][W]) as the FastVideo decoder does.
 *   - Streams: work is enqueued on `stream` (NULL = legacy default stream) and
 *     the call returns without synchronising.  No call blocks on the device.
 *   - Errors: arguments are validated on the host before anything is launched;
 *     a failed check returns a non-zero wvae_status and enqueues nothing.  A
 *     launch failure returns WVAE_ERR_CUDA.  Device-side faults detected by
 *     the kernels (a pipeline wait that exceeded its time limit) are recorded
 *     in the error word and reported by wvae_device_error.
 *   - dtype WVAE_BF16: bf16 activations and weights, fp32 accumulation and
 *     fp32 norm statistics, tensor cores (tcgen05).  WVAE_F32: fp32 storage
 *     and CUDA-core fp32 arithmetic (a precision reference path).
 *   - Pointers must be 16-byte aligned.  In-place operation is allowed only
 *     where stated.
 */
#ifndef WVAE_H
#define WVAE_H

#include <stddef.h>

#if defined(__GNUC__)
#define WVAE_API __attribute__((visibility("default")))
#else
#define WVAE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* wvae_stream_t; /* == cudaStream_t */

typedef enum {
  WVAE_OK = 0,
  WVAE_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, mismatch      */
  WVAE_ERR_UNSUPPORTED = 2,  /* shape/dtype outside what the kernels handle     */
  WVAE_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned                */
  WVAE_ERR_WORKSPACE = 4,    /* workspace / packed buffer smaller than required */
  WVAE_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed            */
  WVAE_ERR_TIMEOUT = 6,      /* a kernel wait exceeded its limit (device word)  */
  WVAE_ERR_NO_DEVICE = 7     /* no sm_100 device is current                     */
} wvae_status;

typedef enum { WVAE_BF16 = 0, WVAE_F32 = 1 } wvae_dtype;

/* Human-readable name of a status code (static string, never NULL). */
WVAE_API const char* wvae_status_string(int status);

/* ABI version: (major << 16) | minor. */
WVAE_API int wvae_version(void);

/*
 * Device error word: returns WVAE_OK if no kernel since the last reset has
 * recorded a fault, else WVAE_ERR_TIMEOUT; *code (may be NULL) receives the raw
 * bit mask.  Synchronises the current device.  reset != 0 clears the word.
 */
WVAE_API wvae_status wvae_device_error(unsigned int* code, int reset);

/* Self-test of the failure detection (the pages define no such call): enqueues
 * one block whose thread waits on a pipeline barrier that nothing ever
 * completes, with a limit of limit_us microseconds (1 .. 1,000,000) instead of
 * the kernels' 2 s.  The wait gives up, records bit 0x10 in the error word and
 * the kernel returns, so the context stays usable; read the outcome with
 * wvae_device_error.  Returns WVAE_ERR_INVALID_ARG for a limit out of range,
 * WVAE_ERR_NO_DEVICE / WVAE_ERR_CUDA as any launch. */
WVAE_API wvae_status wvae_selftest_wait_timeout(unsigned int limit_us, wvae_stream_t stream);

/* ---------------------------------------------------------------- norm-SiLU
 * Channel RMS-norm + affine + SiLU at every voxel v of x [T][H][W][C]:
 *   y[v,c] = SiLU( x[v,c] / max(||x[v,:]||_2, eps) * sqrt(C) * gamma[c] + beta[c] )
 * with SiLU(s) = s / (1 + exp(-s)); statistics in fp32.
 * (TensorRT-LLM issue #19309, "Feature, motivation and proposed scope";
 * FastVideo README "Limits": fp32 RMS-norm statistics.)
 *   x, y     : [T*H*W][C] in `dtype`; y may equal x (in place).
 *   gamma, beta : fp32 [C].
 *   C        : multiple of 8 (bf16) / 4 (fp32), 8 <= C <= 1024.
 *   eps      : > 0 (the decoder uses 1e-12).
 */
WVAE_API wvae_status wvae_norm_silu(const void* x, void* y, const float* gamma, const float* beta,
                           int T, int H, int W, int C, float eps, wvae_dtype dtype,
                           wvae_stream_t stream);

/* ------------------------------------------------------------ weight prepack
 * One-time re-layout of a conv's weights into the tile order the conv kernels
 * read (FastVideo README, "Use": the decoder prepares its weights once).
 * Source: PyTorch order [cout][cin][kt][kh][kw] (fp32 if w_dtype == WVAE_F32,
 * bf16 if WVAE_BF16), device memory; bias fp32 [cout] or NULL (zero).
 * `dtype` selects the compute path the packed blob is for.  The blob is
 * opaque, position-independent and owned by the caller; it can be copied or
 * saved as bytes.  Supported kernel sizes: (3,3,3), (1,3,3), (1,1,1).
 * wvae_conv_packed_bytes returns 0 for unsupported shapes.
 */
WVAE_API size_t wvae_conv_packed_bytes(int cout, int cin, int kt, int kh, int kw, wvae_dtype dtype);
WVAE_API wvae_status wvae_prepack_conv(const void* w, wvae_dtype w_dtype, const float* bias, int cout,
                              int cin, int kt, int kh, int kw, wvae_dtype dtype, void* packed,
                              size_t packed_bytes, wvae_stream_t stream);

/* ------------------------------------------------------------ causal conv3d
 * out[t,h,w,o] = bias[o] + sum_{i,kt,kh,kw} W[o,i,kt,kh,kw] * a[t+kt-(KT-1), h+kh-(KH-1)/2,
 *                                                              w+kw-(KW-1)/2, i]
 * where a = x (or SiLU(norm(x)) when norm_gamma/norm_beta are given), zero
 * outside [0,H)x[0,W), and for frames t' < 0 the previous chunk's frame
 * cache[KT-1+t'] when `cache` is given, else zero (two zero frames in front
 * for KT = 3).  Padding applies after the norm: padded inputs are exactly 0.
 * Optionally out += residual (same layout as y).
 *   x        : [T][H][W][cin] in dtype.   cache: NULL or [KT-1][H][W][cin]
 *              holding the previous chunk's conv INPUT (already normalised).
 *   packed_w : from wvae_prepack_conv for (cout, cin, kt, kh, kw, dtype).
 *   norm_gamma, norm_beta : both NULL (no norm) or both fp32 [cin]; eps 1e-12.
 *   residual : NULL or [T][H][W][cout] in dtype.   y: [T][H][W][cout].
 *   workspace: wvae_causal_conv3d_workspace_bytes(...) bytes (0 without norm).
 * bf16: cin % 64 == 0, cout % 16 == 0 and cout <= 256 or cout == 512.
 * y must not overlap x, cache or residual.
 */
WVAE_API size_t wvae_causal_conv3d_workspace_bytes(int T, int H, int W, int cin, int has_norm,
                                          wvae_dtype dtype);
WVAE_API wvae_status wvae_causal_conv3d(const void* x, const void* cache, const void* packed_w, int T,
                               int H, int W, int cin, int cout, int kt, int kh, int kw,
                               const float* norm_gamma, const float* norm_beta,
                               const void* residual, void* y, wvae_dtype dtype, void* workspace,
                               size_t ws_bytes, wvae_stream_t stream);

/* ------------------------------------------- causal conv3d, Winograd form
 * The same causal 3x3x3 conv as wvae_causal_conv3d (bf16, no norm, no cache),
 * computed as Winograd F(2x2, 3x3) products (Lavin and Gray's minimal
 * filtering) the way the page-3 decoder computes its convs (FastVideo
 * README, "Use": Winograd transforms of the weights; "Performance and
 * memory": the products take 60 % of its GPU time).  Spatially Winograd,
 * temporally direct: the 16 transform planes of the input, V = B^T d B per
 * 4 x 4 tile at stride 2, are multiplied on the tensor cores by the
 * transformed weights U = G g G^T of each temporal tap (fp16 operands, fp32
 * accumulation) and the products go through Y = A^T M A, + bias (+ residual).
 * 2.25x fewer tensor-core FLOPs than the direct conv, at the cost of the
 * planes' memory traffic; fp16 operands keep the direct conv's accuracy.
 *   packed_w: wvae_conv_winograd_packed_bytes(cout, cin) bytes from
 *     wvae_prepack_conv_winograd (weights [cout][cin][3][3][3], fp32 or bf16).
 *   x: [T][H][W][cin] bf16; residual: NULL or [T][H][W][cout] bf16;
 *   y: [T][H][W][cout] bf16 (no overlap with x or residual).
 *   workspace: wvae_causal_conv3d_winograd_workspace_bytes(T, H, W, cin, cout)
 *     bytes: the input planes and the products, fp16
 *     [16][T][ceil(H/2)][ceil(W/2)][C] each.
 * cin % 64 == 0, cout % 16 == 0 and cout <= 256 or cout == 512.
 */
WVAE_API size_t wvae_conv_winograd_packed_bytes(int cout, int cin);
WVAE_API wvae_status wvae_prepack_conv_winograd(const void* w, wvae_dtype w_dtype, const float* bias,
                                                int cout, int cin, void* packed, size_t packed_bytes,
                                                wvae_stream_t stream);
WVAE_API size_t wvae_causal_conv3d_winograd_workspace_bytes(int T, int H, int W, int cin, int cout);
WVAE_API wvae_status wvae_causal_conv3d_winograd(const void* x, const void* packed_w, int T, int H,
                                                 int W, int cin, int cout, const void* residual,
                                                 void* y, void* workspace, size_t ws_bytes,
                                                 wvae_stream_t stream);

/* ------------------------------------------------------------ residual block
 * h = shortcut(x) + conv2(A2(conv1(A1(x)))), A_k = SiLU(norm_k(.)), causal
 * 3x3x3 convs; shortcut = identity when cin == cout, else the 1x1x1 conv
 * packed in wsc_packed (applied to the raw x).  The norm of conv1's output is
 * computed in conv1's epilogue and the shortcut is folded into conv2's
 * reduction, so the block is 3 kernels (norm1, conv1, conv2).
 *   x: [T][H][W][cin], y: [T][H][W][cout] in dtype (y must not overlap x).
 *   w1_packed (cout, cin, 3,3,3), w2_packed (cout, cout, 3,3,3),
 *   wsc_packed (cout, cin, 1,1,1) or NULL iff cin == cout.
 *   gamma1/beta1 fp32 [cin], gamma2/beta2 fp32 [cout].
 *   workspace: wvae_resblock_workspace_bytes(...) bytes.
 */
WVAE_API size_t wvae_resblock_workspace_bytes(int T, int H, int W, int cin, int cout, wvae_dtype dtype);
WVAE_API wvae_status wvae_resblock(const void* x, void* y, int T, int H, int W, int cin, int cout,
                          const float* gamma1, const float* beta1, const void* w1_packed,
                          const float* gamma2, const float* beta2, const void* w2_packed,
                          const void* wsc_packed, wvae_dtype dtype, void* workspace,
                          size_t ws_bytes, wvae_stream_t stream);

/* -------------------------------------------------- upsample + 3x3 conv
 * y[t] = conv3x3( nearest2x(x[t]) ) + bias, per frame, zero border of 1 at the
 * upsampled resolution; u[2h+i, 2w+j] = x[h, w].
 * bf16: computed without materialising u, as four 2x2 "phase" convs on x
 * (the FastVideo README's "phase" weight transform, section "Use"): output
 * pixel (2h+p, 2w+q) reads x rows h+p-1, h+p and columns w+q-1, w+q with the
 * 3x3 taps that land on them summed (in fp32, rounded once to bf16) by
 * wvae_prepack_upsample_conv.  fp32: the reference path materialises u in the
 * workspace and runs the fp32 (1,3,3) conv.
 *   w: PyTorch [cout][cin][1][3][3] (device, fp32 or bf16); bias fp32 [cout] or NULL.
 *   x: [T][H][W][cin], y: [T][2H][2W][cout] in dtype.
 *   packed_w: from wvae_prepack_upsample_conv for (cout, cin, dtype).
 *   workspace: wvae_upsample_conv_workspace_bytes(...) bytes (0 for bf16).
 */
WVAE_API size_t wvae_upsample_conv_packed_bytes(int cout, int cin, wvae_dtype dtype);
WVAE_API wvae_status wvae_prepack_upsample_conv(const void* w, wvae_dtype w_dtype, const float* bias,
                                       int cout, int cin, wvae_dtype dtype, void* packed,
                                       size_t packed_bytes, wvae_stream_t stream);
WVAE_API size_t wvae_upsample_conv_workspace_bytes(int T, int H, int W, int cin, wvae_dtype dtype);
WVAE_API wvae_status wvae_upsample_conv(const void* x, void* y, int T, int H, int W, int cin, int cout,
                               const void* packed_w, wvae_dtype dtype, void* workspace,
                               size_t ws_bytes, wvae_stream_t stream);

/* ------------------------------------------------------------ decoder trunk
 * Wan2.2-shaped decoder trunk on latents z [1][48][T][H][W] (NCDHW, bf16):
 *   conv_in (causal 3x3x3, 48 -> C0)
 *   stage s = 0..3 at resolution (2^s H, 2^s W): 2 residual blocks of width Cs,
 *     then for s < 3 a nearest-2x upsample + 3x3 conv Cs -> C(s+1)
 *   norm_out + SiLU, causal 3x3x3 conv C3 -> 12, 2x2 pixel shuffle
 *   -> video [1][3][T][16H][16W] (NCDHW, bf16), video[c,t,2h+i,2w+j] = out[4c+2i+j].
 *   widths: host int[4] (C0..C3), NULL = {512, 512, 256, 128}; each a multiple of
 *     64 and <= 256 or == 512.
 *   packed: host array of 21 device pointers, in forward order:
 *     [0] conv_in (C0, 48, 3,3,3); per stage s, per block b: conv1 (Cs, Cs, 3,3,3),
 *     conv2 (Cs, Cs, 3,3,3) (wvae_prepack_conv); then for s < 3 the upsample conv
 *     (C(s+1), Cs) from wvae_prepack_upsample_conv; [20] head (12, C3, 3,3,3).
 *   norms: host array of 34 device pointers (fp32), gamma then beta for each norm in
 *     forward order: per stage, per block: norm1, norm2; then norm_out.
 *   workspace: wvae_decode_trunk_workspace_bytes(T, H, W, widths) bytes.
 * Only dtype == WVAE_BF16 is supported.
 */
WVAE_API size_t wvae_decode_trunk_workspace_bytes(int T, int H, int W, const int* widths);
WVAE_API wvae_status wvae_decode_trunk(const void* const* packed, const float* const* norms,
                              const void* z, void* video, int T, int H, int W, const int* widths,
                              wvae_dtype dtype, void* workspace, size_t ws_bytes,
                              wvae_stream_t stream);

/*
 * Per-launch timing of the trunk.  wvae_decode_trunk enqueues exactly
 * wvae_decode_trunk_launches() kernels on `stream`, in this order:
 *   [0] latents NCDHW -> channels-last, [1] conv_in, then per stage s = 0..3:
 *   block 0 conv1, block 0 conv2, block 1 conv1, block 1 conv2 and, for s < 3,
 *   the upsample conv; the last launch is the head.
 * wvae_decode_trunk_timed does the same work and records events[2i] just
 * before and events[2i+1] just after launch i on `stream`.  events: host array
 * of n_events >= 2 * launches cudaEvent_t handles created by the caller
 * (with timing enabled); the library only records them.
 */
WVAE_API int wvae_decode_trunk_launches(void);
WVAE_API wvae_status wvae_decode_trunk_timed(const void* const* packed, const float* const* norms,
                                    const void* z, void* video, int T, int H, int W,
                                    const int* widths, wvae_dtype dtype, void* workspace,
                                    size_t ws_bytes, void* const* events, int n_events,
                                    wvae_stream_t stream);

/*
 * Streaming decode in temporal chunks (the decoder's temporal caching:
 * TensorRT-LLM issue #19309, "Feature, motivation and proposed scope"; the
 * FastVideo decoder decodes a few latent frames per pass, README "Use").
 * Same arguments and work as wvae_decode_trunk on the chunk's T >= 2 latent
 * frames, plus `cache`: a caller-owned device buffer of
 * wvae_decode_trunk_cache_bytes(H, W, widths) bytes (16-byte aligned) holding,
 * for each of the 18 causal 3x3x3 convs (conv_in, the 16 res-block convs, the
 * head), the last two frames of its input.  With continue_chunk == 0 the
 * convs see zero front frames (the first chunk) and the cache's content is
 * ignored; with continue_chunk != 0 they read their front frames from the
 * cache.  Either way the call leaves the cache holding this chunk's last two
 * input frames of every causal conv, so decoding latents chunk by chunk
 * gives the same video as decoding them in one call (the upsample convs are
 * per frame and need no cache).  Besides the 22 kernels of
 * wvae_decode_trunk it enqueues 18 device-to-device copies on `stream`.
 * Returns WVAE_ERR_INVALID_ARG for T < 2 or a NULL cache,
 * WVAE_ERR_WORKSPACE for a short cache, as wvae_decode_trunk otherwise.
 */
WVAE_API size_t wvae_decode_trunk_cache_bytes(int H, int W, const int* widths);
WVAE_API wvae_status wvae_decode_trunk_chunk(const void* const* packed, const float* const* norms,
                                    const void* z, void* video, int T, int H, int W,
                                    const int* widths, wvae_dtype dtype, void* workspace,
                                    size_t ws_bytes, void* cache, size_t cache_bytes,
                                    int continue_chunk, wvae_stream_t stream);

/* ----------------------------------------- video decode with 4T - 3 frames
 * The trunk with the decoder's 4x temporal expansion: latents [1][48][T][H][W]
 * decode to the video [1][3][4T - 3][16H][16W] (FastVideo README, opening
 * section: 4x temporal compression, video [1, 3, 4T - 3, 704, 1248]).  The
 * pages give the frame count, not the layer that makes it; this library
 * reads it as a nearest 2x step in time after the upsample convs of stages 0
 * and 1: the decode's first frame stays one frame, every later frame becomes
 * two consecutive frames (T -> 2T - 1, twice: 4T - 3).  The step rides in
 * those upsample convs' epilogues (each output written to both of its
 * frames), so it costs no launch; stages 1, 2 and 3 run on 2T - 1, 4T - 3
 * and 4T - 3 frames.
 * Arguments as wvae_decode_trunk_chunk, except:
 *   video: [1][3][wvae_decode_video_frames(T, continue_chunk)][16H][16W].
 *   workspace: wvae_decode_video_workspace_bytes(T, H, W, widths) bytes.
 *   cache: NULL for a whole decode (continue_chunk must then be 0); else as
 *     in wvae_decode_trunk_chunk (wvae_decode_trunk_cache_bytes, T >= 2).  A
 *     continuing chunk holds no first frame, so all of its frames double and
 *     it yields 4T frames; chunk by chunk the video equals the whole decode's.
 * wvae_decode_video_frames returns 4T - 3 (continue_chunk == 0) or 4T, 0 for
 * T < 1.  Returns WVAE_ERR_INVALID_ARG for continue_chunk without a cache,
 * as wvae_decode_trunk_chunk otherwise.
 */
WVAE_API int wvae_decode_video_frames(int T, int continue_chunk);
WVAE_API size_t wvae_decode_video_workspace_bytes(int T, int H, int W, const int* widths);
WVAE_API wvae_status wvae_decode_video(const void* const* packed, const float* const* norms,
                                       const void* z, void* video, int T, int H, int W,
                                       const int* widths, wvae_dtype dtype, void* workspace,
                                       size_t ws_bytes, void* cache, size_t cache_bytes,
                                       int continue_chunk, wvae_stream_t stream);

/* -------------------------------------------------- row-slab decode
 * One decode split over ranks by latent rows (the FastVideo decoder spreads
 * one decode over 1-4 GPUs of a node, README "Use" and "Performance and
 * memory"; the pages do not say how it splits the work).  A rank owns the
 * latent rows [r0, r0 + rows) and, at stage s, those rows at 2^s times the
 * resolution; every tensor of its workspace carries its own rows plus one
 * halo row above and one below.  Before each 3x3 conv the halo rows of the
 * conv's INPUT (the activation after norm + SiLU: the frame pads with zeros
 * after the activation) must hold the neighbours' edge rows, or zeros at the
 * frame's top and bottom.  The library runs the decode one launch at a time
 * and says where each launch's input lives, so the caller can fill the halo
 * rows between launches (NCCL point-to-point on the same stream, or copies).
 * Everything else on the path is per voxel and needs no exchange.
 *   wvae_decode_rows_steps(): launches per decode (as wvae_decode_trunk).
 *   wvae_decode_rows_workspace_bytes(T, rows, W, widths): workspace bytes.
 *   wvae_decode_rows_halo(step, ...): before launch `step`, the tensor whose
 *     halo rows must be filled: *offset bytes into the workspace, dims =
 *     {frames, rows + 2 at the stage's resolution, columns, channels}, bf16
 *     channels-last; dims[0] == 0 when the launch needs no exchange (the
 *     latent re-layout and conv_in, whose halo comes with the latents).
 *     Host only: enqueues nothing.
 *   wvae_decode_rows_step(step, ...): enqueue launch `step` of the decode.
 *     z_rows: the rank's latents with their halo rows, [1][48][T][rows + 2][W]
 *     bf16 (rows r0 - 1 .. r0 + rows of the whole latents, zeros outside the
 *     frame); video_rows: [1][3][T][16 rows][16W] bf16, the rank's video rows.
 *     Only widths whose last stage has <= 128 channels.
 * Launching steps 0 .. steps-1 in order, with the halos filled before each,
 * gives the rank's rows of the whole decode's video.
 */
WVAE_API int wvae_decode_rows_steps(void);
WVAE_API size_t wvae_decode_rows_workspace_bytes(int T, int rows, int W, const int* widths);
WVAE_API wvae_status wvae_decode_rows_halo(int step, int T, int rows, int W, const int* widths,
                                           size_t* offset, int* dims);
WVAE_API wvae_status wvae_decode_rows_step(int step, const void* const* packed,
                                           const float* const* norms, const void* z_rows,
                                           void* video_rows, int T, int rows, int W,
                                           const int* widths, wvae_dtype dtype, void* workspace,
                                           size_t ws_bytes, wvae_stream_t stream);

/* ------------------------------------------------- res block, no allocation
 * (No counterpart on the pages: this is a convenience of this library.)
 *
 * wvae_resblock for callers that cannot allocate device memory when they call
 * it and have no workspace to pass in - for example a plugin run by a host
 * engine that owns all device memory and hands its plugins none, or an
 * application that forbids allocation after start-up so that its memory use
 * is fixed and cannot fail mid-run.  Same arguments and result as
 * wvae_resblock with dtype WVAE_BF16, but its scratch (the two activation
 * tensors A1 and A2) lives in a static device array of 64 MiB inside this
 * library, which every GPU that loads the library holds until the process
 * exits.  It calls no allocator.
 *   Size limit: round_up(T*H*W*cin*2, 256) + round_up(T*H*W*cout*2, 256)
 *   <= 64 MiB (the value of wvae_resblock_workspace_bytes for bf16); larger
 *   shapes return WVAE_ERR_WORKSPACE and enqueue nothing.
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   Every call on a device shares the one array, which keeps whatever the
 *   last call left in it (nothing is read before it is written, so nothing
 *   needs clearing).  Calls whose GPU work overlaps - two streams, two host
 *   threads - race on it: serialise them.
 */
WVAE_API wvae_status wvae_resblock_noalloc(const void* x, void* y, int T, int H, int W, int cin,
                                           int cout, const float* gamma1, const float* beta1,
                                           const void* w1_packed, const float* gamma2,
                                           const float* beta2, const void* w2_packed,
                                           const void* wsc_packed, wvae_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* WVAE_H */

/*
 * CPU oracle for the Wan-style video-VAE decoder residual-block hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * definition the CUDA path is checked against.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it; the library
 * under video_diffusion_vae_b200/ never does, and the two share no code.
 *
 * Every tensor is batch 1 in the logical NCDHW order (stored C,T,H,W), every
 * value is an IEEE double and every sum accumulates in double.  Functions
 * follow their definitions term by term; the only freedom taken is the order
 * in which the terms of a sum are added.
 *
 * Sources (web pages gathered on the Wan2.2 VAE decoder):
 *  - "Opt-in BF16 norm-SiLU fusion for Wan VAE decoding" (TensorRT-LLM issue
 *    #19309), section "Feature, motivation and proposed scope": the decoder's
 *    residual norm1/norm2 and norm_out are a channel normalisation, an affine
 *    scaling and a SiLU.
 *  - FastVideo "Wan2.2 VAE decoder (sm_100a, sm_103a)" README, section
 *    "Limits": bf16 weights/activations, fp32 accumulation and fp32 RMS-norm
 *    statistics; the decoder's convs are causal in time (temporal caching is
 *    named in the TensorRT-LLM issue's scope section).
 *  The pages give no formula for the norm or the padding; the readings used
 *  here are the task's own statement of the block: norm over channels
 *  x / max(||x||_2, eps) * sqrt(C) * gamma[c] + beta[c], SiLU(s) = s/(1+e^-s),
 *  a causal conv whose KT-1 missing frames in front are zeros (or the cached
 *  frames of the previous chunk) and whose spatial border is (K-1)/2 zeros.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define IDX4(c, t, h, w, T, H, W) ((((size_t)(c) * (T) + (t)) * (H) + (h)) * (W) + (w))

/* SiLU(s) = s * sigma(s), sigma(s) = 1 / (1 + exp(-s)). */
double orc_silu(double s) { return s / (1.0 + exp(-s)); }

/*
 * Channel RMS-norm + affine (+ SiLU) at every voxel v:
 *   n[v]   = max( sqrt( sum_c x[c,v]^2 ), eps )
 *   s[c,v] = x[c,v] / n[v] * sqrt(C) * gamma[c] + beta[c]
 *   y[c,v] = silu ? SiLU(s[c,v]) : s[c,v]
 * x, y: [C][nvox] (nvox = T*H*W); y may alias x.
 */
void orc_norm_silu(const double* x, double* y, const double* gamma,
                   const double* beta, int C, long nvox, double eps, int silu) {
  const double rootC = sqrt((double)C);
  for (long v = 0; v < nvox; ++v) {
    double ss = 0.0;
    for (int c = 0; c < C; ++c) {
      double xv = x[(size_t)c * nvox + v];
      ss += xv * xv;
    }
    double n = sqrt(ss);
    if (n < eps) n = eps;
    for (int c = 0; c < C; ++c) {
      double s = x[(size_t)c * nvox + v] / n * rootC * gamma[c] + beta[c];
      y[(size_t)c * nvox + v] = silu ? orc_silu(s) : s;
    }
  }
}

/*
 * Causal conv3d, stride 1:
 *   y[o,t,h,w] = bias[o] + sum_{i,kt,kh,kw} wt[o,i,kt,kh,kw]
 *                * a[i, t+kt-(KT-1), h+kh-(KH-1)/2, w+kw-(KW-1)/2]
 * where a[i,t',h',w'] is x inside [0,T)x[0,H)x[0,W); for t' < 0 it is
 * cache[i, KT-1+t', h', w'] when a cache of the previous chunk's last KT-1
 * frames is given ([Cin][KT-1][H][W]) and zero otherwise; outside the
 * spatial range it is zero.  Tap kt = KT-1 is the current frame.  With KT = 1
 * this is a per-frame 2-D conv with zero border.  wt is PyTorch's
 * [Cout][Cin][KT][KH][KW]; bias may be NULL (zero).
 */
typedef struct {
  const double *x, *wt, *bias, *cache;
  double* y;
  int Cin, Cout, T, H, W, KT, KH, KW;
  int o_begin, o_end;
} conv_job;

static double conv_input(const conv_job* j, int i, int ts, int hs, int ws) {
  if (hs < 0 || hs >= j->H || ws < 0 || ws >= j->W) return 0.0;
  if (ts >= 0) return j->x[IDX4(i, ts, hs, ws, j->T, j->H, j->W)];
  if (!j->cache) return 0.0;
  return j->cache[IDX4(i, j->KT - 1 + ts, hs, ws, j->KT - 1, j->H, j->W)];
}

static void* conv_worker(void* arg) {
  const conv_job* j = (const conv_job*)arg;
  const int T = j->T, H = j->H, W = j->W;
  const int PT = j->KT - 1, PH = (j->KH - 1) / 2, PW = (j->KW - 1) / 2;
  const size_t plane = (size_t)T * H * W;
  for (int o = j->o_begin; o < j->o_end; ++o) {
    double* yo = j->y + (size_t)o * plane;
    const double b = j->bias ? j->bias[o] : 0.0;
    for (size_t v = 0; v < plane; ++v) yo[v] = b;
    for (int i = 0; i < j->Cin; ++i)
      for (int kt = 0; kt < j->KT; ++kt)
        for (int kh = 0; kh < j->KH; ++kh)
          for (int kw = 0; kw < j->KW; ++kw) {
            const double wv =
                j->wt[((((size_t)o * j->Cin + i) * j->KT + kt) * j->KH + kh) * j->KW + kw];
            for (int t = 0; t < T; ++t)
              for (int h = 0; h < H; ++h) {
                double* yrow = yo + ((size_t)t * H + h) * W;
                const int ts = t + kt - PT, hs = h + kh - PH;
                for (int w = 0; w < W; ++w)
                  yrow[w] += wv * conv_input(j, i, ts, hs, w + kw - PW);
              }
          }
  }
  return NULL;
}

void orc_causal_conv3d(const double* x, const double* wt, const double* bias,
                       const double* cache, double* y, int Cin, int Cout, int T,
                       int H, int W, int KT, int KH, int KW, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > Cout) nthreads = Cout;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
  conv_job* jobs = (conv_job*)malloc(sizeof(conv_job) * nthreads);
  for (int k = 0; k < nthreads; ++k) {
    conv_job j = {x, wt, bias, cache, y, Cin, Cout, T, H, W, KT, KH, KW,
                  (int)((long)Cout * k / nthreads), (int)((long)Cout * (k + 1) / nthreads)};
    jobs[k] = j;
    pthread_create(&th[k], NULL, conv_worker, &jobs[k]);
  }
  for (int k = 0; k < nthreads; ++k) pthread_join(th[k], NULL);
  free(th);
  free(jobs);
}

/* One output voxel of the same conv: yv[o] = y[o,t,h,w] for every o. */
void orc_causal_conv3d_at(const double* x, const double* wt, const double* bias,
                          const double* cache, double* yv, int Cin, int Cout,
                          int T, int H, int W, int KT, int KH, int KW, int t,
                          int h, int w) {
  conv_job j = {x, wt, bias, cache, NULL, Cin, Cout, T, H, W, KT, KH, KW, 0, Cout};
  const int PT = KT - 1, PH = (KH - 1) / 2, PW = (KW - 1) / 2;
  for (int o = 0; o < Cout; ++o) {
    double acc = bias ? bias[o] : 0.0;
    for (int i = 0; i < Cin; ++i)
      for (int kt = 0; kt < KT; ++kt)
        for (int kh = 0; kh < KH; ++kh)
          for (int kw = 0; kw < KW; ++kw)
            acc += wt[((((size_t)o * Cin + i) * KT + kt) * KH + kh) * KW + kw] *
                   conv_input(&j, i, t + kt - PT, h + kh - PH, w + kw - PW);
    yv[o] = acc;
  }
}

/* Nearest 2x spatial upsample, per frame: y[c,t,2h+i,2w+j] = x[c,t,h,w]. */
void orc_upsample_nearest2x(const double* x, double* y, int C, int T, int H, int W) {
  for (int c = 0; c < C; ++c)
    for (int t = 0; t < T; ++t)
      for (int h = 0; h < 2 * H; ++h)
        for (int w = 0; w < 2 * W; ++w)
          y[IDX4(c, t, h, w, T, 2 * H, 2 * W)] = x[IDX4(c, t, h / 2, w / 2, T, H, W)];
}

/*
 * 2x2 pixel shuffle (PyTorch pixel_shuffle order), per frame:
 *   y[c, t, 2h+i, 2w+j] = x[4c + 2i + j, t, h, w],  x has 4*Cv channels.
 */
void orc_pixel_shuffle2x2(const double* x, double* y, int Cv, int T, int H, int W) {
  for (int c = 0; c < Cv; ++c)
    for (int i = 0; i < 2; ++i)
      for (int j = 0; j < 2; ++j)
        for (int t = 0; t < T; ++t)
          for (int h = 0; h < H; ++h)
            for (int w = 0; w < W; ++w)
              y[IDX4(c, t, 2 * h + i, 2 * w + j, T, 2 * H, 2 * W)] =
                  x[IDX4(4 * c + 2 * i + j, t, h, w, T, H, W)];
}

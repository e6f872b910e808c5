/*
 * CPU oracle for the forward pass of the modality-aware short convolution
 * followed by the Kimi Delta Attention (KDA) scan, as described on the pages
 * about "Chimera: Designing and Chinchilla-Scaling Hybrid Visual Diffusion
 * Transformers".
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call this library.  It shares no code with
 * the CUDA path.  Everything is computed in fp64 from inputs widened exactly
 * from their storage type; nothing is rounded in between.
 *
 * Sources (page, section):
 *  [core]  paper.rainbus.top, section 核心方法: before each KDA update a
 *          modality-aware short convolution (causal 1D for text, 3D for visual
 *          tokens) injects local neighbourhood information into Q/K/V; the
 *          stream is text first, then visual tokens in time-major raster order.
 *  [how]   genai-atlas, section "How it works": the convolution runs separately
 *          per modality -- a causal depthwise 1D conv over the text tokens and a
 *          depthwise 3D conv over the visual tokens reshaped to their
 *          spatiotemporal grid.
 *  [step5] paper.rainbus.top, section 方法步骤详情, step (5):
 *          S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T.
 *  [bg]    paper.rainbus.top, section 前置知识, "Kimi Delta Attention": fixed-size
 *          state, causal scan, channel-wise forget gate alpha_t, scalar write
 *          strength beta_t.
 *  The read-out o_t = S_t^T q_t (no scale on q) is not printed on the pages; it
 *  is the plainest reading of a state that is queried after its update.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t B, N;             /* batch items, tokens per item (text_len + T*Hg*Wg) */
  int64_t text_len;         /* text prefix length L */
  int64_t grid_t, grid_h, grid_w;
  int64_t text_k;           /* causal 1D kernel length over text */
  int64_t vis_kt, vis_kh, vis_kw;  /* 3D kernel extents (odd for centred axes) */
  int64_t vis_causal_t;     /* 0: temporal taps centred; 1: taps on frames t-kt+1..t */
} kdao_conv_shape;

/* ------------------------------------------------------------------------ */
/* thread helper                                                             */
/* ------------------------------------------------------------------------ */
typedef void (*work_fn)(void* ctx, int64_t item);
typedef struct { work_fn fn; void* ctx; int64_t n_items; int64_t stride; int64_t first; } worker_t;

static void* worker_main(void* a) {
  worker_t* w = (worker_t*)a;
  for (int64_t i = w->first; i < w->n_items; i += w->stride) w->fn(w->ctx, i);
  return 0;
}

static void parallel_for(int64_t n_items, int nthreads, work_fn fn, void* ctx) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  if (nthreads > n_items) nthreads = (int)(n_items > 0 ? n_items : 1);
  worker_t ws[512];
  pthread_t th[512];
  for (int t = 0; t < nthreads; ++t) {
    ws[t].fn = fn; ws[t].ctx = ctx; ws[t].n_items = n_items; ws[t].stride = nthreads; ws[t].first = t;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], 0, worker_main, &ws[t]);
  worker_main(&ws[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], 0);
}

/* ------------------------------------------------------------------------ */
/* short convolution  [core], [how]                                          */
/* ------------------------------------------------------------------------ */
/*
 * Text token t < L, channel c (cross-correlation, causal):
 *     y[t,c] = sum_{j=0}^{K-1} w_text[c][j] * x[t-(K-1)+j, c],  x at t' < 0 is 0.
 * Visual token at grid position (tt, hh, ww), stored at index
 * L + (tt*Hg + hh)*Wg + ww, channel c:
 *     y = sum_{a,b,e} w_vis[c][(a*kh + b)*kw + e] * x(tt+a-pt, hh+b-ph, ww+e-pw)
 * with ph = (kh-1)/2, pw = (kw-1)/2, pt = (kt-1)/2 (centred) or kt-1 (causal in
 * time); grid positions outside [0,T)x[0,Hg)x[0,Wg) read 0.  Text never reads
 * visual tokens and visual tokens never read text (per-modality convolution).
 * Batch items are independent.
 */
typedef struct {
  const kdao_conv_shape* s;
  int64_t C, c0, c1;       /* full channel count and the channel range computed */
  const float* x;          /* [B, N, C] */
  const float* w_text;     /* [C][text_k] */
  const float* w_vis;      /* [C][kt*kh*kw] */
  double* y;               /* [B, N, c1-c0] */
  int64_t rows_per_item;
} conv_ctx;

static void conv_rows(void* vctx, int64_t item) {
  conv_ctx* cx = (conv_ctx*)vctx;
  const kdao_conv_shape* s = cx->s;
  const int64_t C = cx->C, c0 = cx->c0, nc = cx->c1 - cx->c0;
  const int64_t N = s->N, L = s->text_len;
  const int64_t T = s->grid_t, Hg = s->grid_h, Wg = s->grid_w;
  const int64_t kt = s->vis_kt, kh = s->vis_kh, kw = s->vis_kw, KV = kt * kh * kw;
  const int64_t pt = s->vis_causal_t ? kt - 1 : (kt - 1) / 2, ph = (kh - 1) / 2, pw = (kw - 1) / 2;
  const int64_t per = cx->rows_per_item;
  const int64_t blocks_per_b = (N + per - 1) / per;
  const int64_t b = item / blocks_per_b;
  const int64_t n0 = (item % blocks_per_b) * per;
  const int64_t n1 = n0 + per < N ? n0 + per : N;
  const float* xb = cx->x + b * N * C;
  double* yb = cx->y + b * N * nc;
  for (int64_t n = n0; n < n1; ++n) {
    for (int64_t ci = 0; ci < nc; ++ci) {
      const int64_t c = c0 + ci;
      double acc = 0.0;
      if (n < L) {
        const int64_t K = s->text_k;
        for (int64_t j = 0; j < K; ++j) {
          int64_t src = n - (K - 1) + j;
          if (src >= 0) acc += (double)cx->w_text[c * K + j] * (double)xb[src * C + c];
        }
      } else {
        int64_t p = n - L;
        int64_t tt = p / (Hg * Wg), hh = (p / Wg) % Hg, ww = p % Wg;
        for (int64_t a = 0; a < kt; ++a) {
          int64_t t2 = tt + a - pt;
          if (t2 < 0 || t2 >= T) continue;
          for (int64_t bb = 0; bb < kh; ++bb) {
            int64_t h2 = hh + bb - ph;
            if (h2 < 0 || h2 >= Hg) continue;
            for (int64_t e = 0; e < kw; ++e) {
              int64_t w2 = ww + e - pw;
              if (w2 < 0 || w2 >= Wg) continue;
              int64_t src = L + (t2 * Hg + h2) * Wg + w2;
              acc += (double)cx->w_vis[c * KV + (a * kh + bb) * kw + e] * (double)xb[src * C + c];
            }
          }
        }
      }
      yb[n * nc + ci] = acc;
    }
  }
}

int kdao_shortconv(const kdao_conv_shape* s, int64_t C, int64_t c0, int64_t c1,
                   const float* x, const float* w_text, const float* w_vis, double* y, int nthreads) {
  if (!s || !x || !w_text || !w_vis || !y) return 1;
  if (s->N != s->text_len + s->grid_t * s->grid_h * s->grid_w) return 2;
  if (c0 < 0 || c1 > C || c0 >= c1) return 3;
  conv_ctx cx = {s, C, c0, c1, x, w_text, w_vis, y, 64};
  int64_t items = s->B * ((s->N + cx.rows_per_item - 1) / cx.rows_per_item);
  parallel_for(items, nthreads, conv_rows, &cx);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* KDA token recurrence  [step5], [bg]                                       */
/* ------------------------------------------------------------------------ */
/*
 * For one head: S in R^{dk x dv}, from S_0 (or zeros).  For t = 0..N-1 in
 * stream order (text, then visual; no reset at the modality boundary):
 *     S <- Diag(alpha_t) S                         alpha_t = exp(log_alpha_t)
 *     u  = beta_t (v_t - S^T k_t)
 *     S <- S + k_t u^T
 *     o_t = S^T q_t
 * which is S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 * followed by the read-out o_t = S_t^T q_t.  Column j of S only ever needs
 * column j of v, so columns are computed independently (blocks of columns run
 * on separate threads).
 */
typedef struct {
  int64_t B, N, dk, dv, j0, j1, jb;
  const double *q, *k, *v, *la, *beta, *S0;
  double *o, *SN;
} scan_ctx;

static void scan_block(void* vctx, int64_t item) {
  scan_ctx* c = (scan_ctx*)vctx;
  const int64_t dk = c->dk, dv = c->dv, N = c->N;
  const int64_t nblk = (c->j1 - c->j0 + c->jb - 1) / c->jb;
  const int64_t b = item / nblk;
  const int64_t ja = c->j0 + (item % nblk) * c->jb;
  const int64_t jz = ja + c->jb < c->j1 ? ja + c->jb : c->j1;
  const int64_t nb = jz - ja;
  double* S = (double*)malloc(sizeof(double) * dk * nb);
  double* u = (double*)malloc(sizeof(double) * nb);
  double* alpha = (double*)malloc(sizeof(double) * dk);
  for (int64_t i = 0; i < dk; ++i)
    for (int64_t j = 0; j < nb; ++j)
      S[i * nb + j] = c->S0 ? c->S0[(b * dk + i) * dv + ja + j] : 0.0;
  for (int64_t t = 0; t < N; ++t) {
    const double* qt = c->q + (b * N + t) * dk;
    const double* kt = c->k + (b * N + t) * dk;
    const double* vt = c->v + (b * N + t) * dv;
    const double* lat = c->la + (b * N + t) * dk;
    const double bt = c->beta[b * N + t];
    for (int64_t i = 0; i < dk; ++i) alpha[i] = exp(lat[i]);
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < nb; ++j) S[i * nb + j] *= alpha[i];
    for (int64_t j = 0; j < nb; ++j) u[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < nb; ++j) u[j] += S[i * nb + j] * kt[i];
    for (int64_t j = 0; j < nb; ++j) u[j] = bt * (vt[ja + j] - u[j]);
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < nb; ++j) S[i * nb + j] += kt[i] * u[j];
    double* ot = c->o + (b * N + t) * dv;
    for (int64_t j = 0; j < nb; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < dk; ++i) acc += S[i * nb + j] * qt[i];
      ot[ja + j] = acc;
    }
  }
  if (c->SN)
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < nb; ++j) c->SN[(b * dk + i) * dv + ja + j] = S[i * nb + j];
  free(S); free(u); free(alpha);
}

/*
 * One head.  q, k, la : [B, N, dk]; v : [B, N, dv]; beta : [B, N];
 * S0, SN : [B, dk, dv] (either may be NULL); o : [B, N, dv].
 * Only columns [j0, j1) of o and SN are written.
 */
int kdao_scan(int64_t B, int64_t N, int64_t dk, int64_t dv,
              const double* q, const double* k, const double* v, const double* la, const double* beta,
              const double* S0, double* o, double* SN, int64_t j0, int64_t j1, int nthreads) {
  if (!q || !k || !v || !la || !beta || !o) return 1;
  if (B < 1 || N < 0 || dk < 1 || dv < 1 || j0 < 0 || j1 > dv || j0 >= j1) return 2;
  scan_ctx c = {B, N, dk, dv, j0, j1, 8, q, k, v, la, beta, S0, o, SN};
  int64_t nblk = (j1 - j0 + c.jb - 1) / c.jb;
  parallel_for(B * nblk, nthreads, scan_block, &c);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* backward pass: the adjoint of the forward above                           */
/* ------------------------------------------------------------------------ */
/*
 * Adjoint of the token recurrence for one head, written out from the forward
 * steps (no source gives the backward; it is the chain rule applied to them).
 * With S~ = Diag(alpha_t) S_{t-1}, u = beta_t (v_t - S~^T k_t), S_t = S~ + k_t u^T,
 * o_t = S_t^T q_t, and dS the gradient reaching S_t from later tokens:
 *     G      = dS + q_t do_t^T                 (total gradient of S_t)
 *     dq_t   = S_t do_t
 *     du     = G^T k_t
 *     dv_t   = beta_t du
 *     dbeta_t= du . (v_t - S~^T k_t)
 *     dk_t   = G u - beta_t S~ du
 *     dS~    = G - beta_t k_t du^T
 *     dla_t  = rowsum(dS~ o S~)               (d alpha / d log alpha = alpha)
 *     dS_{t-1} = Diag(alpha_t) dS~
 * and dS_0 is the gradient left after token 0.  Every state is kept, so this is
 * for small problems only (N * dk * dv doubles per batch item).
 */
typedef struct {
  int64_t N, dk, dv;
  const double *q, *k, *v, *la, *beta, *S0, *dO, *dSN;
  double *dq, *dk_, *dv_, *dla, *dbeta, *dS0;
} scan_bwd_ctx;

static void scan_bwd_item(void* vctx, int64_t b) {
  scan_bwd_ctx* c = (scan_bwd_ctx*)vctx;
  const int64_t N = c->N, dk = c->dk, dv = c->dv, SZ = dk * dv;
  double* states = (double*)malloc(sizeof(double) * SZ * (N + 1));   /* states[t+1] = S_t, states[0] = S_init */
  double* St = (double*)malloc(sizeof(double) * SZ);
  double* G = (double*)malloc(sizeof(double) * SZ);
  double* dS = (double*)malloc(sizeof(double) * SZ);
  double* u = (double*)malloc(sizeof(double) * dv);
  double* r = (double*)malloc(sizeof(double) * dv);
  double* du = (double*)malloc(sizeof(double) * dv);
  double* alpha = (double*)malloc(sizeof(double) * dk);
  for (int64_t x = 0; x < SZ; ++x) states[x] = c->S0 ? c->S0[b * SZ + x] : 0.0;
  /* forward, keeping every state */
  for (int64_t t = 0; t < N; ++t) {
    const double* kt = c->k + (b * N + t) * dk;
    const double* vt = c->v + (b * N + t) * dv;
    const double* lat = c->la + (b * N + t) * dk;
    const double bt = c->beta[b * N + t];
    const double* Sp = states + t * SZ;
    double* Sn = states + (t + 1) * SZ;
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j) Sn[i * dv + j] = exp(lat[i]) * Sp[i * dv + j];
    for (int64_t j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < dk; ++i) acc += Sn[i * dv + j] * kt[i];
      u[j] = bt * (vt[j] - acc);
    }
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j) Sn[i * dv + j] += kt[i] * u[j];
  }
  for (int64_t x = 0; x < SZ; ++x) dS[x] = c->dSN ? c->dSN[b * SZ + x] : 0.0;
  /* backward */
  for (int64_t t = N - 1; t >= 0; --t) {
    const double* qt = c->q + (b * N + t) * dk;
    const double* kt = c->k + (b * N + t) * dk;
    const double* vt = c->v + (b * N + t) * dv;
    const double* lat = c->la + (b * N + t) * dk;
    const double* dot = c->dO + (b * N + t) * dv;
    const double bt = c->beta[b * N + t];
    const double* Sp = states + t * SZ;          /* S_{t-1} */
    const double* Sc = states + (t + 1) * SZ;    /* S_t */
    for (int64_t i = 0; i < dk; ++i) alpha[i] = exp(lat[i]);
    /* St <- S~ = Diag(alpha) S_{t-1};  r = v - S~^T k;  u = beta r */
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j) St[i * dv + j] = alpha[i] * Sp[i * dv + j];
    for (int64_t j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < dk; ++i) acc += St[i * dv + j] * kt[i];
      r[j] = vt[j] - acc;
      u[j] = bt * r[j];
    }
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j) G[i * dv + j] = dS[i * dv + j] + qt[i] * dot[j];
    for (int64_t i = 0; i < dk; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < dv; ++j) acc += Sc[i * dv + j] * dot[j];
      c->dq[(b * N + t) * dk + i] = acc;
    }
    double dbt = 0.0;
    for (int64_t j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < dk; ++i) acc += G[i * dv + j] * kt[i];
      du[j] = acc;
      c->dv_[(b * N + t) * dv + j] = bt * acc;
      dbt += acc * r[j];
    }
    c->dbeta[b * N + t] = dbt;
    for (int64_t i = 0; i < dk; ++i) {
      double a1 = 0.0, a2 = 0.0, a3 = 0.0;
      for (int64_t j = 0; j < dv; ++j) {
        const double g = G[i * dv + j], s = St[i * dv + j];
        const double dst = g - bt * kt[i] * du[j];   /* dS~ */
        a1 += g * u[j];
        a2 += s * du[j];
        a3 += dst * s;
        dS[i * dv + j] = alpha[i] * dst;
      }
      c->dk_[(b * N + t) * dk + i] = a1 - bt * a2;
      c->dla[(b * N + t) * dk + i] = a3;
    }
  }
  if (c->dS0)
    for (int64_t x = 0; x < SZ; ++x) c->dS0[b * SZ + x] = dS[x];
  free(states); free(St); free(G); free(dS); free(u); free(r); free(du); free(alpha);
}

/*
 * One head.  Inputs as in kdao_scan plus dO [B, N, dv] and dSN [B, dk, dv]
 * (NULL: zero).  Outputs dq, dk, dla [B, N, dk], dv [B, N, dv], dbeta [B, N],
 * dS0 [B, dk, dv] (NULL: not written).
 */
int kdao_scan_bwd(int64_t B, int64_t N, int64_t dk, int64_t dv,
                  const double* q, const double* k, const double* v, const double* la, const double* beta,
                  const double* S0, const double* dO, const double* dSN,
                  double* dq, double* dk_, double* dv_, double* dla, double* dbeta, double* dS0, int nthreads) {
  if (!q || !k || !v || !la || !beta || !dO || !dq || !dk_ || !dv_ || !dla || !dbeta) return 1;
  if (B < 1 || N < 0 || dk < 1 || dv < 1) return 2;
  scan_bwd_ctx c = {N, dk, dv, q, k, v, la, beta, S0, dO, dSN, dq, dk_, dv_, dla, dbeta, dS0};
  parallel_for(B, nthreads, scan_bwd_item, &c);
  return 0;
}

/*
 * Adjoint of the short convolution: every tap that read x[src, c] into y[n, c]
 * with weight w sends w * dy[n, c] back to dx[src, c] and x[src, c] * dy[n, c]
 * to its weight.  Threads own disjoint channel ranges, so the scatter is exact.
 * x: [B, N, C] float; dy: [B, N, C] double; dx: [B, N, C], dw_text: [C][text_k],
 * dw_vis: [C][kt*kh*kw], all double and overwritten.
 */
typedef struct {
  const kdao_conv_shape* s;
  int64_t C, cb;
  const float *x, *w_text, *w_vis;
  const double* dy;
  double *dx, *dwt, *dwv;
} conv_bwd_ctx;

static void conv_bwd_channels(void* vctx, int64_t item) {
  conv_bwd_ctx* cx = (conv_bwd_ctx*)vctx;
  const kdao_conv_shape* s = cx->s;
  const int64_t C = cx->C, N = s->N, L = s->text_len;
  const int64_t T = s->grid_t, Hg = s->grid_h, Wg = s->grid_w, K = s->text_k;
  const int64_t kt = s->vis_kt, kh = s->vis_kh, kw = s->vis_kw, KV = kt * kh * kw;
  const int64_t pt = s->vis_causal_t ? kt - 1 : (kt - 1) / 2, ph = (kh - 1) / 2, pw = (kw - 1) / 2;
  const int64_t c0 = item * cx->cb, c1 = c0 + cx->cb < C ? c0 + cx->cb : C;
  for (int64_t c = c0; c < c1; ++c) {
    for (int64_t j = 0; j < K; ++j) cx->dwt[c * K + j] = 0.0;
    for (int64_t j = 0; j < KV; ++j) cx->dwv[c * KV + j] = 0.0;
    for (int64_t b = 0; b < s->B; ++b)
      for (int64_t n = 0; n < N; ++n) cx->dx[(b * N + n) * C + c] = 0.0;
    for (int64_t b = 0; b < s->B; ++b) {
      const float* xb = cx->x + b * N * C;
      const double* dyb = cx->dy + b * N * C;
      double* dxb = cx->dx + b * N * C;
      for (int64_t n = 0; n < N; ++n) {
        const double g = dyb[n * C + c];
        if (n < L) {
          for (int64_t j = 0; j < K; ++j) {
            int64_t src = n - (K - 1) + j;
            if (src < 0) continue;
            dxb[src * C + c] += (double)cx->w_text[c * K + j] * g;
            cx->dwt[c * K + j] += (double)xb[src * C + c] * g;
          }
        } else {
          int64_t p = n - L;
          int64_t tt = p / (Hg * Wg), hh = (p / Wg) % Hg, ww = p % Wg;
          for (int64_t a = 0; a < kt; ++a) {
            int64_t t2 = tt + a - pt;
            if (t2 < 0 || t2 >= T) continue;
            for (int64_t bb = 0; bb < kh; ++bb) {
              int64_t h2 = hh + bb - ph;
              if (h2 < 0 || h2 >= Hg) continue;
              for (int64_t e = 0; e < kw; ++e) {
                int64_t w2 = ww + e - pw;
                if (w2 < 0 || w2 >= Wg) continue;
                int64_t src = L + (t2 * Hg + h2) * Wg + w2, tap = (a * kh + bb) * kw + e;
                dxb[src * C + c] += (double)cx->w_vis[c * KV + tap] * g;
                cx->dwv[c * KV + tap] += (double)xb[src * C + c] * g;
              }
            }
          }
        }
      }
    }
  }
}

int kdao_shortconv_bwd(const kdao_conv_shape* s, int64_t C, const float* x, const float* w_text,
                       const float* w_vis, const double* dy, double* dx, double* dw_text, double* dw_vis,
                       int nthreads) {
  if (!s || !x || !w_text || !w_vis || !dy || !dx || !dw_text || !dw_vis) return 1;
  if (s->N != s->text_len + s->grid_t * s->grid_h * s->grid_w) return 2;
  conv_bwd_ctx cx = {s, C, 8, x, w_text, w_vis, dy, dx, dw_text, dw_vis};
  parallel_for((C + cx.cb - 1) / cx.cb, nthreads, conv_bwd_channels, &cx);
  return 0;
}

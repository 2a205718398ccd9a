/*
 * orthrus_oracle.c -- CPU oracle (test infrastructure only; see the header
 * for the sources, the precision rules and who may use it).
 */
#include "orthrus_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 -> double, exact: a bf16 is the top 16 bits of an IEEE binary32. */
static double widen_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static double load_elem(int dtype, const void* p, int64_t i) {
  if (dtype == ORACLE_F32) return (double)((const float*)p)[i];
  if (dtype == ORACLE_F64) return ((const double*)p)[i];
  return widen_bf16(((const uint16_t*)p)[i]);
}

/* softmax(q.k * scale) v for one query row over an ordered key list.
 * Keys 0..n_cache-1 come from kc/vc (stride D), then n_blk keys from kb/vb
 * (stride blk_stride).  Two passes (max, then exp/sum/weighted sum), double
 * throughout.  [EXPLAINER §二: Q over concat(cache K/V, block K/V)] */
static void attn_row(const double* q, const double* kc, const double* vc,
                     int n_cache, const double* kb, const double* vb,
                     int64_t blk_stride, int n_blk, int D, double scale,
                     double* s /* scratch [n_cache + n_blk] */, double* out) {
  int nk = n_cache + n_blk;
  double m = -INFINITY;
  for (int j = 0; j < nk; ++j) {
    const double* k = j < n_cache ? kc + (int64_t)j * D
                                  : kb + (int64_t)(j - n_cache) * blk_stride;
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q[d] * k[d];
    s[j] = dot * scale;
    if (s[j] > m) m = s[j];
  }
  double l = 0.0;
  for (int j = 0; j < nk; ++j) {
    s[j] = exp(s[j] - m);
    l += s[j];
  }
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (int j = 0; j < nk; ++j) {
    const double* v = j < n_cache ? vc + (int64_t)j * D
                                  : vb + (int64_t)(j - n_cache) * blk_stride;
    for (int d = 0; d < D; ++d) out[d] += s[j] * v[d];
  }
  for (int d = 0; d < D; ++d) out[d] /= l;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int oracle_block_attn(int dtype, int mask_mode, int B, int Hq, int Hkv, int D,
                      int blk, const void* q, const void* k_blk,
                      const void* v_blk, const void* k_cache,
                      const void* v_cache, int cap, const int32_t* ctx_lens,
                      double scale, double* out, int nthreads) {
  if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return -1;
  if (mask_mode != ORACLE_BIDIR_BLOCK && mask_mode != ORACLE_CAUSAL_VERIFY)
    return -1;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || blk < 0 || cap < 0)
    return -1;
  for (int b = 0; b < B; ++b)
    if (ctx_lens[b] < 0 || ctx_lens[b] > cap) return -1;
  const int G = Hq / Hkv;
  set_threads(nthreads);

  /* Work in double: widen one (sequence, kv-head) slice at a time. */
  for (int b = 0; b < B; ++b) {
    const int n = ctx_lens[b];
    for (int g = 0; g < Hkv; ++g) {
      double* kc = (double*)malloc(sizeof(double) * ((size_t)n * D + 1));
      double* vc = (double*)malloc(sizeof(double) * ((size_t)n * D + 1));
      double* kb = (double*)malloc(sizeof(double) * ((size_t)blk * D + 1));
      double* vb = (double*)malloc(sizeof(double) * ((size_t)blk * D + 1));
      const int64_t cbase = ((int64_t)b * Hkv + g) * cap * D;
      for (int64_t t = 0; t < (int64_t)n * D; ++t) {
        kc[t] = load_elem(dtype, k_cache, cbase + t);
        vc[t] = load_elem(dtype, v_cache, cbase + t);
      }
      for (int i = 0; i < blk; ++i)
        for (int d = 0; d < D; ++d) {
          int64_t src = (((int64_t)b * blk + i) * Hkv + g) * D + d;
          kb[(int64_t)i * D + d] = load_elem(dtype, k_blk, src);
          vb[(int64_t)i * D + d] = load_elem(dtype, v_blk, src);
        }
#pragma omp parallel for schedule(dynamic) collapse(2)
      for (int hl = 0; hl < G; ++hl)
        for (int i = 0; i < blk; ++i) {
          const int h = g * G + hl;
          double* qd = (double*)malloc(sizeof(double) * D);
          double* s = (double*)malloc(sizeof(double) * ((size_t)n + blk + 1));
          for (int d = 0; d < D; ++d)
            qd[d] = load_elem(dtype, q, (((int64_t)b * blk + i) * Hq + h) * D + d);
          /* [EXPLAINER §三 mask rule] bidir: whole block; causal: rows <= i */
          int n_blk = mask_mode == ORACLE_BIDIR_BLOCK ? blk : i + 1;
          attn_row(qd, kc, vc, n, kb, vb, D, n_blk, D, scale, s,
                   out + (((int64_t)b * blk + i) * Hq + h) * D);
          free(qd);
          free(s);
        }
      free(kc);
      free(vc);
      free(kb);
      free(vb);
    }
  }
  return 0;
}

/* [EXPLAINER §四 step 2: "the token that should most appear here"] */
int oracle_vocab_argmax(int dtype, const void* logits, int rows, int vocab,
                        int64_t row_stride, int32_t* idx, double* maxval) {
  if (dtype != ORACLE_F32 && dtype != ORACLE_BF16 && dtype != ORACLE_F64) return -1;
  if (rows < 0 || vocab <= 0 || row_stride < vocab) return -1;
  for (int r = 0; r < rows; ++r) {
    int best = -1;
    double bv = 0.0;
    for (int j = 0; j < vocab; ++j) {
      double x = load_elem(dtype, logits, (int64_t)r * row_stride + j);
      if (isnan(x)) continue;
      if (best < 0 || x > bv) { /* strict: the first maximum stays */
        best = j;
        bv = x;
      }
    }
    if (best < 0) { /* all NaN */
      best = 0;
      bv = load_elem(dtype, logits, (int64_t)r * row_stride);
    }
    idx[r] = best;
    if (maxval) maxval[r] = bv;
  }
  return 0;
}

/* [EXPLAINER §四 step 3]: compare left to right, accept while equal, then
 * take the AR token at the first disagreement as the correction and drop the
 * rest; at least one token per round. */
int oracle_consensus(const int32_t* draft, const int32_t* verify, int B,
                     int blk, int32_t* accept_len, int32_t* n_emit,
                     int32_t* emitted, int32_t* next_anchor) {
  if (B < 0 || blk <= 0) return -1;
  for (int b = 0; b < B; ++b) {
    const int32_t* d = draft + (int64_t)b * blk;
    const int32_t* a = verify + (int64_t)b * blk;
    int L = 0;
    while (L < blk && d[L] == a[L]) ++L;
    int ne = L + 1 < blk ? L + 1 : blk;
    accept_len[b] = L;
    n_emit[b] = ne;
    for (int j = 0; j < blk; ++j) emitted[(int64_t)b * blk + j] = j < ne ? a[j] : -1;
    next_anchor[b] = a[ne - 1];
  }
  return 0;
}

/* [EXPLAINER §四 step 3 "update the notebook", §七 constant block state]:
 * only the accepted rows enter the cache; nothing past them is written. */
int oracle_kv_commit(int dtype, void* k_cache, void* v_cache,
                     const void* k_blk, const void* v_blk, int B, int Hkv,
                     int D, int cap, int blk, int32_t* ctx_lens,
                     const int32_t* n_emit) {
  if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return -1;
  const size_t es = dtype == ORACLE_F32 ? 4 : 2;
  for (int b = 0; b < B; ++b) {
    int n = ctx_lens[b], ne = n_emit[b];
    if (ne < 0 || ne > blk || n < 0 || n + ne > cap) return -1;
  }
  for (int b = 0; b < B; ++b) {
    int n = ctx_lens[b], ne = n_emit[b];
    for (int g = 0; g < Hkv; ++g)
      for (int i = 0; i < ne; ++i) {
        int64_t dst = (((int64_t)b * Hkv + g) * cap + n + i) * D;
        int64_t src = (((int64_t)b * blk + i) * Hkv + g) * D;
        memcpy((char*)k_cache + dst * es, (const char*)k_blk + src * es, D * es);
        memcpy((char*)v_cache + dst * es, (const char*)v_blk + src * es, D * es);
      }
    ctx_lens[b] = n + ne;
  }
  return 0;
}

/* ------------------------------------------------------------------ model */

typedef struct {
  const double *attn_norm, *wq, *wk, *wv, *wo, *dq, *dk, *dv, *dout;
  const double *ffn_norm, *w_gate, *w_up, *w_down;
} layer_w;

static int64_t layer_size(const oracle_model_cfg* c) {
  int64_t qd = (int64_t)c->Hq * c->hd, kd = (int64_t)c->Hkv * c->hd;
  int64_t attn = qd * c->d + 2 * kd * c->d + (int64_t)c->d * qd;
  return c->d + 2 * attn + c->d + 3 * (int64_t)c->ffn * c->d;
}

int64_t oracle_model_num_weights(const oracle_model_cfg* c) {
  return (int64_t)c->V * c->d + (int64_t)c->L * layer_size(c) + c->d +
         (int64_t)c->V * c->d;
}

static layer_w get_layer(const oracle_model_cfg* c, const double* w, int l) {
  int64_t qd = (int64_t)c->Hq * c->hd, kd = (int64_t)c->Hkv * c->hd;
  const double* p = w + (int64_t)c->V * c->d + (int64_t)l * layer_size(c);
  layer_w L;
  L.attn_norm = p; p += c->d;
  L.wq = p; p += qd * c->d;
  L.wk = p; p += kd * c->d;
  L.wv = p; p += kd * c->d;
  L.wo = p; p += (int64_t)c->d * qd;
  L.dq = p; p += qd * c->d;
  L.dk = p; p += kd * c->d;
  L.dv = p; p += kd * c->d;
  L.dout = p; p += (int64_t)c->d * qd;
  L.ffn_norm = p; p += c->d;
  L.w_gate = p; p += (int64_t)c->ffn * c->d;
  L.w_up = p; p += (int64_t)c->ffn * c->d;
  L.w_down = p;
  return L;
}

/* y[o] = sum_i W[o][i] x[i], i ascending. */
static void matvec(const double* W, const double* x, int out, int in, double* y) {
  for (int o = 0; o < out; ++o) {
    const double* r = W + (int64_t)o * in;
    double acc = 0.0;
    for (int i = 0; i < in; ++i) acc += r[i] * x[i];
    y[o] = acc;
  }
}

/* RMSNorm: x / sqrt(mean(x^2) + eps) * g */
static void rmsnorm(const double* x, const double* g, int d, double eps, double* y) {
  double ss = 0.0;
  for (int i = 0; i < d; ++i) ss += x[i] * x[i];
  double r = 1.0 / sqrt(ss / d + eps);
  for (int i = 0; i < d; ++i) y[i] = x[i] * r * g[i];
}

/* Rotary embedding, half-split pairing (i, i + hd/2), angle pos * theta^(-2i/hd). */
static void rope(double* x, int hd, int pos, double theta) {
  int h = hd / 2;
  for (int i = 0; i < h; ++i) {
    double ang = (double)pos * pow(theta, -2.0 * i / hd);
    double cs = cos(ang), sn = sin(ang);
    double x1 = x[i], x2 = x[i + h];
    x[i] = x1 * cs - x2 * sn;
    x[i + h] = x2 * cs + x1 * sn;
  }
}

int oracle_model_forward(const oracle_model_cfg* c, const double* w, int view,
                         const int32_t* tokens, int rows,
                         const double* k_cache, const double* v_cache, int cap,
                         int n, double* logits, double* k_blk, double* v_blk,
                         int nthreads) {
  if (view != 0 && view != 1) return -1;
  if (rows <= 0 || n < 0 || n > cap || c->Hq % c->Hkv || c->hd % 2) return -1;
  for (int r = 0; r < rows; ++r)
    if (tokens[r] < 0 || tokens[r] >= c->V) return -1;
  set_threads(nthreads);
  const int d = c->d, hd = c->hd, Hq = c->Hq, Hkv = c->Hkv, G = Hq / Hkv;
  const int qd = Hq * hd, kd = Hkv * hd;
  const double scale = 1.0 / sqrt((double)hd);

  double* x = (double*)calloc((size_t)rows * d, sizeof(double));
  double* hbuf = (double*)calloc((size_t)rows * d, sizeof(double));
  double* q = (double*)calloc((size_t)rows * qd, sizeof(double));
  double* kb = (double*)calloc((size_t)rows * kd, sizeof(double));
  double* vb = (double*)calloc((size_t)rows * kd, sizeof(double));
  double* att = (double*)calloc((size_t)rows * qd, sizeof(double));
  double* ff = (double*)calloc((size_t)rows * 2 * c->ffn, sizeof(double));
  double* tmp = (double*)calloc((size_t)rows * (d > c->V ? d : c->V), sizeof(double));

  for (int r = 0; r < rows; ++r)
    memcpy(x + (int64_t)r * d, w + (int64_t)tokens[r] * d, sizeof(double) * d);

  for (int l = 0; l < c->L; ++l) {
    layer_w Lw = get_layer(c, w, l);
    const double* Wq = view ? Lw.dq : Lw.wq;
    const double* Wk = view ? Lw.dk : Lw.wk;
    const double* Wv = view ? Lw.dv : Lw.wv;
    const double* Wo = view ? Lw.dout : Lw.wo;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
      rmsnorm(x + (int64_t)r * d, Lw.attn_norm, d, c->eps, hbuf + (int64_t)r * d);
      matvec(Wq, hbuf + (int64_t)r * d, qd, d, q + (int64_t)r * qd);
      matvec(Wk, hbuf + (int64_t)r * d, kd, d, kb + (int64_t)r * kd);
      matvec(Wv, hbuf + (int64_t)r * d, kd, d, vb + (int64_t)r * kd);
      for (int h = 0; h < Hq; ++h) rope(q + (int64_t)r * qd + h * hd, hd, n + r, c->rope_theta);
      for (int g = 0; g < Hkv; ++g) rope(kb + (int64_t)r * kd + g * hd, hd, n + r, c->rope_theta);
    }
    if (k_blk) {
      memcpy(k_blk + (int64_t)l * rows * kd, kb, sizeof(double) * rows * kd);
      memcpy(v_blk + (int64_t)l * rows * kd, vb, sizeof(double) * rows * kd);
    }
    /* attention over cache[0,n) then the block (view 0 causal, view 1 bidir) */
    const double* kcl = k_cache + (int64_t)l * Hkv * cap * hd;
    const double* vcl = v_cache + (int64_t)l * Hkv * cap * hd;
#pragma omp parallel for schedule(dynamic) collapse(2)
    for (int r = 0; r < rows; ++r)
      for (int h = 0; h < Hq; ++h) {
        int g = h / G;
        double* s = (double*)malloc(sizeof(double) * ((size_t)n + rows + 1));
        int n_blk = view ? rows : r + 1;
        attn_row(q + (int64_t)r * qd + h * hd, kcl + (int64_t)g * cap * hd,
                 vcl + (int64_t)g * cap * hd, n, kb + g * hd, vb + g * hd, kd,
                 n_blk, hd, scale, s, att + (int64_t)r * qd + h * hd);
        free(s);
      }
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
      double* xr = x + (int64_t)r * d;
      double* tr = tmp + (int64_t)r * d;
      matvec(Wo, att + (int64_t)r * qd, d, qd, tr);
      for (int i = 0; i < d; ++i) xr[i] += tr[i];
      rmsnorm(xr, Lw.ffn_norm, d, c->eps, hbuf + (int64_t)r * d);
      double* gt = ff + (int64_t)r * 2 * c->ffn;
      double* up = gt + c->ffn;
      matvec(Lw.w_gate, hbuf + (int64_t)r * d, c->ffn, d, gt);
      matvec(Lw.w_up, hbuf + (int64_t)r * d, c->ffn, d, up);
      for (int i = 0; i < c->ffn; ++i) gt[i] = gt[i] / (1.0 + exp(-gt[i])) * up[i];
      matvec(Lw.w_down, gt, d, c->ffn, tr);
      for (int i = 0; i < d; ++i) xr[i] += tr[i];
    }
  }
  const double* fnorm = w + (int64_t)c->V * d + (int64_t)c->L * layer_size(c);
  const double* head = fnorm + d;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    rmsnorm(x + (int64_t)r * d, fnorm, d, c->eps, hbuf + (int64_t)r * d);
    matvec(head, hbuf + (int64_t)r * d, c->V, d, logits + (int64_t)r * c->V);
  }
  free(x); free(hbuf); free(q); free(kb); free(vb); free(att); free(ff); free(tmp);
  return 0;
}

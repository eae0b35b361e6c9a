/*
 * orc.c -- CPU oracle of one mixture-of-experts decode layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Plain, slow, fp64.  See orc.h for the equations
 * and for which pages' passages each step follows.  Nothing here is blocked,
 * fused or reordered beyond the per-token definition: every output element is
 * one dot product summed left to right (optionally as `ksplit` contiguous
 * partials, for the split-agreement check).
 */
#include "orc.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "../kdgen/kd_gen.h"

/* ---------------------------------------------------------------- decoders */

double orc_bf16_value(uint16_t bits) {
  /* bf16 is the top half of an IEEE binary32 */
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

double orc_e4m3_value(uint8_t code) {
  /* e4m3fn: sign | 4-bit exponent, bias 7 | 3-bit mantissa; S.1111.111 = NaN */
  int s = code >> 7, ef = (code >> 3) & 15, m = code & 7;
  if (ef == 15 && m == 7) return NAN;
  double v = ef == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, ef - 7);
  return s ? -v : v;
}

/* ------------------------------------------------------------ weight rows */

enum { K_QKV = 1, K_O = 2, K_R = 3, K_G = 4, K_U = 5, K_D = 6 };

typedef struct dims {
  int H, Nqkv, A, E, k, I, S; /* S = n_shared */
} dims;

static dims get_dims(const orc_cfg* c) {
  dims d;
  d.H = c->hidden;
  d.Nqkv = (c->q_heads + 2 * c->kv_heads) * c->head_dim;
  d.A = c->q_heads * c->head_dim;
  d.E = c->n_experts;
  d.k = c->top_k;
  d.I = c->inter;
  d.S = c->n_shared;
  return d;
}

static void kind_shape(const dims* d, int kind, int* R, int* K) {
  switch (kind) {
    case K_QKV: *R = d->Nqkv; *K = d->H; break;
    case K_O:   *R = d->H;    *K = d->A; break;
    case K_R:   *R = d->E;    *K = d->H; break;
    case K_G:
    case K_U:   *R = d->I;    *K = d->H; break;
    default:    *R = d->H;    *K = d->I; break;
  }
}

static uint32_t kind_uid_kind(int kind) {
  switch (kind) {
    case K_QKV: return KDG_QKV;
    case K_O:   return KDG_OPROJ;
    case K_R:   return KDG_ROUTER;
    case K_G:   return KDG_GATE;
    case K_U:   return KDG_UP;
    default:    return KDG_DOWN;
  }
}

/* Rows [r0, r0+n) of a generated matrix, decoded to fp64.
 * bf16: the generator's bf16 bits, decoded.
 * FP8: the scale of each 128 x 128 block needs the whole block's values, so
 * the block's rows are generated in full to find its amax. */
static void gen_rows(const orc_cfg* c, const dims* d, int kind, int expert,
                     int r0, int n, double* dst) {
  int R, K;
  kind_shape(d, kind, &R, &K);
  uint32_t slot = (kind >= K_G) ? (uint32_t)(expert < 0 ? 0 : expert + 1) : 0u;
  uint64_t st = kdg_stream(c->seed, kdg_uid((uint32_t)c->layer_id, kind_uid_kind(kind), slot));
  if (c->wdtype == 0) {
    for (int r = 0; r < n; ++r)
      for (int col = 0; col < K; ++col) {
        uint64_t i = (uint64_t)(r0 + r) * (uint64_t)K + (uint64_t)col;
        dst[(size_t)r * K + col] = orc_bf16_value(kdg_bf16(kdg_value(st, i, KDG_W002)));
      }
    return;
  }
  /* FP8: scale per (row block, column block) */
  int nkb = (K + 127) / 128;
  float* amax = (float*)malloc(sizeof(float) * (size_t)nkb);
  int rb_lo = r0 / 128, rb_hi = (r0 + n - 1) / 128;
  for (int rb = rb_lo; rb <= rb_hi; ++rb) {
    int br0 = rb * 128, br1 = br0 + 128 < R ? br0 + 128 : R;
    for (int kb = 0; kb < nkb; ++kb) amax[kb] = 0.0f;
    for (int r = br0; r < br1; ++r)
      for (int col = 0; col < K; ++col) {
        float v = kdg_value(st, (uint64_t)r * (uint64_t)K + (uint64_t)col, KDG_W002);
        float a = fabsf(v);
        if (a > amax[col / 128]) amax[col / 128] = a;
      }
    for (int r = (br0 > r0 ? br0 : r0); r < br1 && r < r0 + n; ++r)
      for (int col = 0; col < K; ++col) {
        float v = kdg_value(st, (uint64_t)r * (uint64_t)K + (uint64_t)col, KDG_W002);
        float scale = kdg_fp8_scale(amax[col / 128]);
        uint8_t q = kdg_e4m3(kdg_fp8_div(v, scale));
        dst[(size_t)(r - r0) * K + col] = orc_e4m3_value(q) * (double)scale;
      }
  }
  free(amax);
}

static void explicit_rows(const orc_weights* w, const dims* d, int kind, int expert,
                          int r0, int n, double* dst) {
  int R, K;
  kind_shape(d, kind, &R, &K);
  const double* base;
  size_t eoff = (size_t)(expert < 0 ? 0 : d->S + expert);
  switch (kind) {
    case K_QKV: base = w->wqkv; break;
    case K_O:   base = w->wo; break;
    case K_R:   base = w->wr; break;
    case K_G:   base = w->wg + eoff * (size_t)R * K; break;
    case K_U:   base = w->wu + eoff * (size_t)R * K; break;
    default:    base = w->wd + eoff * (size_t)R * K; break;
  }
  memcpy(dst, base + (size_t)r0 * K, sizeof(double) * (size_t)n * K);
}

static void rows(const orc_cfg* c, const orc_weights* w, const dims* d, int kind,
                 int expert, int r0, int n, double* dst) {
  if (w) explicit_rows(w, d, kind, expert, r0, n, dst);
  else gen_rows(c, d, kind, expert, r0, n, dst);
}

/* ------------------------------------------------------------ arithmetic */

/* sum_{j<K} a[j] b[j], as `ksplit` contiguous partial sums added in order */
static double dot(const double* a, const double* b, int K, int ksplit) {
  if (ksplit <= 1) {
    double s = 0.0;
    for (int j = 0; j < K; ++j) s += a[j] * b[j];
    return s;
  }
  double total = 0.0;
  for (int p = 0; p < ksplit; ++p) {
    int lo = (int)((long long)K * p / ksplit), hi = (int)((long long)K * (p + 1) / ksplit);
    double s = 0.0;
    for (int j = lo; j < hi; ++j) s += a[j] * b[j];
    total += s;
  }
  return total;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* y[t, r] = W[r, :] . v[t, :] for all rows r of one matrix and the tokens
 * listed in `tok` (rows of v), row blocks of 128 shared among threads. */
static void matvec(const orc_cfg* c, const orc_weights* w, const dims* d, int kind,
                   int expert, const double* v, int ldv, const int* tok, int ntok,
                   double* y, int ldy, int ksplit, int nthreads) {
  int R, K;
  kind_shape(d, kind, &R, &K);
  int nblk = (R + 127) / 128;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) if (nthreads > 1)
  for (int b = 0; b < nblk; ++b) {
    int r0 = b * 128, n = r0 + 128 <= R ? 128 : R - r0;
    double* wr = (double*)malloc(sizeof(double) * (size_t)n * K);
    rows(c, w, d, kind, expert, r0, n, wr);
    for (int r = 0; r < n; ++r)
      for (int t = 0; t < ntok; ++t)
        y[(size_t)t * ldy + r0 + r] =
            dot(wr + (size_t)r * K, v + (size_t)tok[t] * ldv, K, ksplit);
    free(wr);
  }
}

/* F(v_t) = Wd (silu(Wg v_t) * (Wu v_t)) for the listed tokens; y[t] rows. */
static void swiglu(const orc_cfg* c, const orc_weights* w, const dims* d, int expert,
                   const double* v, int ldv, const int* tok, int ntok, double* y,
                   int ksplit, int nthreads) {
  double* gt = (double*)malloc(sizeof(double) * (size_t)ntok * d->I);
  double* up = (double*)malloc(sizeof(double) * (size_t)ntok * d->I);
  int* iota = (int*)malloc(sizeof(int) * (size_t)ntok);
  for (int t = 0; t < ntok; ++t) iota[t] = t;
  matvec(c, w, d, K_G, expert, v, ldv, tok, ntok, gt, d->I, ksplit, nthreads);
  matvec(c, w, d, K_U, expert, v, ldv, tok, ntok, up, d->I, ksplit, nthreads);
  for (size_t i = 0; i < (size_t)ntok * d->I; ++i) gt[i] = silu(gt[i]) * up[i];
  matvec(c, w, d, K_D, expert, gt, d->I, iota, ntok, y, d->H, ksplit, nthreads);
  free(gt);
  free(up);
  free(iota);
}

/* k largest of l[0..E), descending, ties -> lower index (selection by
 * repeated arg-max over the not yet chosen entries). */
static void topk(const double* l, int E, int k, int* sel) {
  unsigned char* used = (unsigned char*)calloc((size_t)E, 1);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (!used[e] && (best < 0 || l[e] > l[best])) best = e;
    used[best] = 1;
    sel[j] = best;
  }
  free(used);
}

/* The MoE half of the layer for M tokens: router and experts on v (the
 * router/expert input), residual r:
 *   l = Wr v + b;  S = top-k(l);  g = softmax over S
 *   out = r + F_shared(v) + sum_j g_j F_{S_j}(v) */
static void moe_block(const orc_cfg* c, const orc_weights* w, const dims* d, const double* bias,
                      const double* r, const double* v, int M, const int* forced_idx,
                      int ksplit, int nthreads, double* logits_out, int* idx_out,
                      double* gates_out, double* out) {
  int* all = (int*)malloc(sizeof(int) * (size_t)M);
  for (int t = 0; t < M; ++t) all[t] = t;
  /* router logits, selection, renormalised softmax over the selection */
  double* lg = (double*)malloc(sizeof(double) * (size_t)M * d->E);
  matvec(c, w, d, K_R, -1, v, d->H, all, M, lg, d->E, ksplit, nthreads);
  /* selection keys: logits + bias; the gates' logits: the same, or with
   * bias_select_only the unbiased logits */
  double* key = (double*)malloc(sizeof(double) * (size_t)M * d->E);
  for (int t = 0; t < M; ++t)
    for (int e = 0; e < d->E; ++e)
      key[(size_t)t * d->E + e] = lg[(size_t)t * d->E + e] + (bias ? bias[e] : 0.0);
  if (!c->bias_select_only) memcpy(lg, key, sizeof(double) * (size_t)M * d->E);
  int* sel = (int*)malloc(sizeof(int) * (size_t)M * d->k);
  double* g = (double*)malloc(sizeof(double) * (size_t)M * d->k);
  for (int t = 0; t < M; ++t) {
    int* s = sel + (size_t)t * d->k;
    const double* l = lg + (size_t)t * d->E;
    if (forced_idx) memcpy(s, forced_idx + (size_t)t * d->k, sizeof(int) * (size_t)d->k);
    else topk(key + (size_t)t * d->E, d->E, d->k, s);
    double mx = l[s[0]];
    for (int j = 1; j < d->k; ++j) if (l[s[j]] > mx) mx = l[s[j]];
    double den = 0.0;
    for (int j = 0; j < d->k; ++j) den += exp(l[s[j]] - mx);
    for (int j = 0; j < d->k; ++j) g[(size_t)t * d->k + j] = exp(l[s[j]] - mx) / den;
  }

  /* out = r + shared(v) + sum_j g_j routed_{s_j}(v) */
  for (size_t i = 0; i < (size_t)M * d->H; ++i) out[i] = r[i];
  double* y = (double*)malloc(sizeof(double) * (size_t)M * d->H);
  if (d->S == 1) {
    swiglu(c, w, d, -1, v, d->H, all, M, y, ksplit, nthreads);
    for (size_t i = 0; i < (size_t)M * d->H; ++i) out[i] += y[i];
  }
  /* routed experts, one expert at a time over the tokens that selected it;
   * per token the contributions are added in selection order j = 0..k-1 */
  double* yr = (double*)calloc((size_t)M * d->k * d->H, sizeof(double));
  int* tok = (int*)malloc(sizeof(int) * (size_t)M);
  int* slot = (int*)malloc(sizeof(int) * (size_t)M);
  for (int e = 0; e < d->E; ++e) {
    int n = 0;
    for (int t = 0; t < M; ++t)
      for (int j = 0; j < d->k; ++j)
        if (sel[(size_t)t * d->k + j] == e) { tok[n] = t; slot[n] = j; ++n; }
    if (n == 0) continue;
    swiglu(c, w, d, e, v, d->H, tok, n, y, ksplit, nthreads);
    for (int q = 0; q < n; ++q)
      memcpy(yr + ((size_t)tok[q] * d->k + slot[q]) * d->H, y + (size_t)q * d->H,
             sizeof(double) * (size_t)d->H);
  }
  const double rs = c->routed_scale != 0.0 ? c->routed_scale : 1.0;
  for (int t = 0; t < M; ++t)
    for (int j = 0; j < d->k; ++j) {
      double gj = rs * g[(size_t)t * d->k + j];
      const double* yy = yr + ((size_t)t * d->k + j) * d->H;
      for (int h = 0; h < d->H; ++h) out[(size_t)t * d->H + h] += gj * yy[h];
    }
  if (logits_out) memcpy(logits_out, lg, sizeof(double) * (size_t)M * d->E);
  if (idx_out) memcpy(idx_out, sel, sizeof(int) * (size_t)M * d->k);
  if (gates_out) memcpy(gates_out, g, sizeof(double) * (size_t)M * d->k);
  free(key);
  free(all); free(lg); free(sel); free(g); free(y); free(yr); free(tok); free(slot);
}

int orc_layer(const orc_cfg* c, const orc_weights* w, const double* bias,
              const double* x, const double* attn, int M,
              const int* forced_idx, int ksplit, int nthreads,
              double* qkv_out, double* h1_out, double* logits_out, int* idx_out,
              double* gates_out, double* out) {
  if (!c || !x || !attn || !out || M < 0) return -1;
  if (c->n_shared < 0 || c->n_shared > 1 || c->top_k < 1 || c->top_k > c->n_experts) return -1;
  if (M == 0) return 0;
  if (ksplit < 1) ksplit = 1;
  if (nthreads < 1) nthreads = 1;
  dims d = get_dims(c);
  int* all = (int*)malloc(sizeof(int) * (size_t)M);
  for (int t = 0; t < M; ++t) all[t] = t;

  /* fused QKV projection */
  if (qkv_out)
    matvec(c, w, &d, K_QKV, -1, x, d.H, all, M, qkv_out, d.Nqkv, ksplit, nthreads);

  /* h1 = x + Wo attn */
  double* h1 = (double*)malloc(sizeof(double) * (size_t)M * d.H);
  matvec(c, w, &d, K_O, -1, attn, d.A, all, M, h1, d.H, ksplit, nthreads);
  for (size_t i = 0; i < (size_t)M * d.H; ++i) h1[i] += x[i];

  /* router and experts on h1, residual h1 */
  moe_block(c, w, &d, bias, h1, h1, M, forced_idx, ksplit, nthreads, logits_out, idx_out,
            gates_out, out);
  if (h1_out) memcpy(h1_out, h1, sizeof(double) * (size_t)M * d.H);
  free(all); free(h1);
  return 0;
}

/* ------------------------------------------------------------ full layer */

uint8_t orc_e4m3_code(double v) {
  /* e4m3fn: values m * 2^(e-7) (1.m form, e = 1..15, S.1111.111 = NaN) and
   * subnormals m/8 * 2^-6; quantum 2^(E-3) in [2^E, 2^(E+1)), 2^-9 below
   * 2^-6.  Round to nearest, ties to even; beyond 448 saturate to 448. */
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs(v);
  if (a != a) return 0x7F;
  if (a > 448.0) return (uint8_t)(sign | 0x7E);
  if (a == 0.0) return sign;
  int E;
  frexp(a, &E);            /* a = f 2^E, f in [0.5, 1): a in [2^(E-1), 2^E) */
  int e = E - 1;
  double q = e >= -6 ? ldexp(1.0, e - 3) : ldexp(1.0, -9);
  double n = nearbyint(a / q);   /* exact division by a power of two; ties to even */
  double r = n * q;
  if (r > 448.0) return (uint8_t)(sign | 0x7E);
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, -6)) return (uint8_t)(sign | (int)(r / ldexp(1.0, -9)));
  frexp(r, &E);
  e = E - 1;
  int m = (int)(r / ldexp(1.0, e) * 8.0) - 8;
  return (uint8_t)(sign | ((e + 7) << 3) | m);
}

void orc_rmsnorm(const double* x, const double* gamma, int n, double eps, double* y) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = 1.0 / sqrt(ss / (double)n + eps);
  for (int i = 0; i < n; ++i) y[i] = x[i] * r * gamma[i];
}

int orc_attention(const double* q, int ldq, const uint8_t* kc, const uint8_t* vc, double k_scale,
                  double v_scale, int n_seq, int max_ctx, int Hq, int Hkv, int hd,
                  const int* seq, const int* pos, int M, double* out, int ldo) {
  if (Hkv < 1 || Hq % Hkv) return -1;
  int grp = Hq / Hkv;
  double inv = 1.0 / sqrt((double)hd);
  for (int t = 0; t < M; ++t) {
    int s = seq[t], L = pos[t] + 1;
    if (s < 0 || s >= n_seq || pos[t] < 0 || pos[t] >= max_ctx) return -1;
    double* sc = (double*)malloc(sizeof(double) * (size_t)L);
    for (int h = 0; h < Hq; ++h) {
      int gk = h / grp;
      const double* qh = q + (size_t)t * ldq + (size_t)h * hd;
      double mx = -INFINITY;
      for (int j = 0; j < L; ++j) {
        const uint8_t* kr = kc + (((size_t)s * max_ctx + j) * Hkv + gk) * hd;
        double dot = 0.0;
        for (int i = 0; i < hd; ++i) dot += qh[i] * (orc_e4m3_value(kr[i]) * k_scale);
        sc[j] = dot * inv;
        if (sc[j] > mx) mx = sc[j];
      }
      double den = 0.0;
      for (int j = 0; j < L; ++j) { sc[j] = exp(sc[j] - mx); den += sc[j]; }
      double* o = out + (size_t)t * ldo + (size_t)h * hd;
      for (int i = 0; i < hd; ++i) o[i] = 0.0;
      for (int j = 0; j < L; ++j) {
        const uint8_t* vr = vc + (((size_t)s * max_ctx + j) * Hkv + gk) * hd;
        double p = sc[j] / den;
        for (int i = 0; i < hd; ++i) o[i] += p * (orc_e4m3_value(vr[i]) * v_scale);
      }
    }
    free(sc);
  }
  return 0;
}

static void gen_norm(const orc_cfg* c, int kind, int n, double* dst) {
  uint64_t st = kdg_stream(c->seed, kdg_uid((uint32_t)c->layer_id, (uint32_t)kind, 0));
  for (int i = 0; i < n; ++i) dst[i] = orc_bf16_value(kdg_norm_bf16(st, (uint64_t)i));
}

int orc_layer_full(const orc_cfg* c, const orc_weights* w, const double* bias, const double* x,
                   int M, uint8_t* kc, uint8_t* vc, double k_scale, double v_scale, int n_seq,
                   int max_ctx, const int* seq, const int* pos, double eps, int keep_new_kv,
                   const int* forced_idx, int nthreads, double* qkv_out, double* attn_out,
                   double* h1_out, double* v_out, double* logits_out, int* idx_out,
                   double* gates_out, double* out) {
  if (!c || !x || !kc || !vc || !seq || !pos || !out || M < 0) return -1;
  if (c->n_shared < 0 || c->n_shared > 1 || c->top_k < 1 || c->top_k > c->n_experts) return -1;
  if (c->kv_heads < 1 || c->q_heads % c->kv_heads) return -1;
  if (M == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  dims d = get_dims(c);
  const int hd = c->head_dim, Hq = c->q_heads, Hkv = c->kv_heads;
  int* all = (int*)malloc(sizeof(int) * (size_t)M);
  for (int t = 0; t < M; ++t) all[t] = t;
  double* g1 = (double*)malloc(sizeof(double) * (size_t)d.H);
  double* g2 = (double*)malloc(sizeof(double) * (size_t)d.H);
  if (w && w->g1) memcpy(g1, w->g1, sizeof(double) * (size_t)d.H);
  else gen_norm(c, KDG_NORM1, d.H, g1);
  if (w && w->g2) memcpy(g2, w->g2, sizeof(double) * (size_t)d.H);
  else gen_norm(c, KDG_NORM2, d.H, g2);

  /* u = RMSNorm(x) g1;  qkv = Wqkv u */
  double* u = (double*)malloc(sizeof(double) * (size_t)M * d.H);
  for (int t = 0; t < M; ++t) orc_rmsnorm(x + (size_t)t * d.H, g1, d.H, eps, u + (size_t)t * d.H);
  double* qkv = (double*)malloc(sizeof(double) * (size_t)M * d.Nqkv);
  matvec(c, w, &d, K_QKV, -1, u, d.H, all, M, qkv, d.Nqkv, 1, nthreads);

  /* the new tokens' keys and values into the cache (e4m3 of value / scale),
   * unless the caller supplies them */
  if (!keep_new_kv)
    for (int t = 0; t < M; ++t) {
      if (seq[t] < 0 || seq[t] >= n_seq || pos[t] < 0 || pos[t] >= max_ctx) return -1;
      size_t base = (((size_t)seq[t] * max_ctx + pos[t]) * Hkv) * hd;
      const double* kq = qkv + (size_t)t * d.Nqkv + (size_t)Hq * hd;
      const double* vq = kq + (size_t)Hkv * hd;
      for (int i = 0; i < Hkv * hd; ++i) {
        kc[base + i] = orc_e4m3_code(kq[i] / k_scale);
        vc[base + i] = orc_e4m3_code(vq[i] / v_scale);
      }
    }

  /* attention of each token over its sequence's positions 0..pos */
  double* a = (double*)malloc(sizeof(double) * (size_t)M * d.A);
  if (orc_attention(qkv, d.Nqkv, kc, vc, k_scale, v_scale, n_seq, max_ctx, Hq, Hkv, hd, seq, pos,
                    M, a, d.A) != 0)
    return -1;

  /* h1 = x + Wo a;  v = RMSNorm(h1) g2;  MoE on v with residual h1 */
  double* h1 = (double*)malloc(sizeof(double) * (size_t)M * d.H);
  matvec(c, w, &d, K_O, -1, a, d.A, all, M, h1, d.H, 1, nthreads);
  for (size_t i = 0; i < (size_t)M * d.H; ++i) h1[i] += x[i];
  double* v = (double*)malloc(sizeof(double) * (size_t)M * d.H);
  for (int t = 0; t < M; ++t) orc_rmsnorm(h1 + (size_t)t * d.H, g2, d.H, eps, v + (size_t)t * d.H);
  moe_block(c, w, &d, bias, h1, v, M, forced_idx, 1, nthreads, logits_out, idx_out, gates_out,
            out);

  if (qkv_out) memcpy(qkv_out, qkv, sizeof(double) * (size_t)M * d.Nqkv);
  if (attn_out) memcpy(attn_out, a, sizeof(double) * (size_t)M * d.A);
  if (h1_out) memcpy(h1_out, h1, sizeof(double) * (size_t)M * d.H);
  if (v_out) memcpy(v_out, v, sizeof(double) * (size_t)M * d.H);
  free(all); free(g1); free(g2); free(u); free(qkv); free(a); free(h1); free(v);
  return 0;
}

int orc_weight_rows(const orc_cfg* c, int kind, int expert, int row0, int nrows, double* dst) {
  if (!c || !dst || kind < 1 || kind > 6 || nrows < 0 || row0 < 0) return -1;
  dims d = get_dims(c);
  int R, K;
  kind_shape(&d, kind, &R, &K);
  if (row0 + nrows > R) return -1;
  if (nrows == 0) return 0;
  gen_rows(c, &d, kind, expert, row0, nrows, dst);
  return 0;
}

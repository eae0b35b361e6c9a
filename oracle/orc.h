/*
 * orc.h -- CPU oracle of one mixture-of-experts decode layer (test infrastructure).
 *
 * This is the checker, not the product: only the test suite, the package's
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code with the CUDA library except the seeded input generator (kdgen/kd_gen.h),
 * which holds none of the layer's arithmetic.
 *
 * It evaluates, in fp64 with no intermediate rounding, the chain the pages
 * describe for the latency-specialised decode step (wireai.ir "vLLM Blackwell
 * Kimi decode", section "4 key changes": attention input projection, output
 * projection followed by the residual, router scores, shared expert beside the
 * routed experts; bigchange.ai "where the time went": attention, expert
 * selection).  For each token t (rows are independent):
 *
 *   qkv_t    = Wqkv x_t                                   (fused QKV projection)
 *   h1_t     = x_t + Wo a_t                               (o-proj + residual)
 *   l_t      = Wr h1_t + b                                (router logits)
 *   S_t      = indices of the k largest l_t, ties -> lower index
 *   g_{t,e}  = exp(l_e - max_S) / sum_{i in S_t} exp(l_i - max_S),  e in S_t
 *   F_e(v)   = Wd_e ( silu(Wg_e v) * (Wu_e v) ),  silu(z) = z / (1 + e^-z)
 *   out_t    = h1_t + F_shared(h1_t) + sum_{e in S_t} g_{t,e} F_e(h1_t)
 *
 * Two variants of the gating (configuration fields): with bias_select_only
 * the bias enters the selection only, S_t = top-k(Wr h1_t + b) and g over
 * the unbiased logits Wr h1_t (the selection-only expert bias of
 * DeepSeek-V3-style routers); routed_scale s multiplies the routed sum,
 * out_t = h1_t + F_shared(h1_t) + s sum_e g_{t,e} F_e(h1_t).
 *
 * Weights are either given explicitly (fp64 arrays, for hand-built cases) or
 * generated from the seed exactly as the GPU receives them (bf16 values, or
 * FP8 e4m3 codes times the fp32 scale of their 128 x 128 block) and decoded
 * here with this file's own decoders.
 */
#ifndef KD_ORACLE_H
#define KD_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct orc_cfg {
  int hidden;                       /* H                                   */
  int q_heads, kv_heads, head_dim;  /* Nqkv = (q + 2 kv) hd, A = q hd      */
  int n_experts, top_k;             /* E, k                                */
  int n_shared;                     /* 0 or 1                              */
  int inter;                        /* I                                   */
  int wdtype;                       /* 0 = bf16, 1 = FP8 e4m3 + block scale */
  int layer_id;                     /* generator stream id of the layer    */
  uint64_t seed;
  int bias_select_only;             /* 1: the router bias chooses the experts
                                       only; the gates are the softmax of the
                                       unbiased logits over the selection   */
  double routed_scale;              /* factor on the routed experts' sum (0 = 1) */
} orc_cfg;

/* Explicit logical weights, row-major fp64.  Expert arrays hold the shared
 * expert first (when n_shared == 1), then routed experts 0..E-1. */
typedef struct orc_weights {
  const double* wqkv;  /* [Nqkv, H]        */
  const double* wo;    /* [H, A]           */
  const double* wr;    /* [E, H]           */
  const double* wg;    /* [n_shared+E, I, H] */
  const double* wu;    /* [n_shared+E, I, H] */
  const double* wd;    /* [n_shared+E, H, I] */
  const double* g1;    /* [H] RMSNorm gain before attention (full layer), or NULL */
  const double* g2;    /* [H] RMSNorm gain before the MoE (full layer), or NULL   */
} orc_weights;

/* One layer for M tokens.  Returns 0, or -1 on bad arguments.
 *   logits (output) are the biased logits, or with bias_select_only the
 *   unbiased ones.
 *   w          NULL -> weights generated from cfg->seed / cfg->layer_id
 *   bias       [E] additive router bias or NULL
 *   x, attn    [M, H], [M, A]
 *   forced_idx [M, k] selection to use instead of the top-k, or NULL
 *   ksplit     >= 1: every dot product is summed as ksplit contiguous partials
 *   nthreads   >= 1: output rows are shared among threads; results do not
 *              depend on it (each dot product is summed by one thread in order)
 * Outputs (any may be NULL except out): qkv [M,Nqkv], h1 [M,H], logits [M,E],
 *   idx [M,k] (descending logit, ties -> lower index), gates [M,k], out [M,H]. */
int orc_layer(const orc_cfg* cfg, const orc_weights* w, const double* bias,
              const double* x, const double* attn, int M,
              const int* forced_idx, int ksplit, int nthreads,
              double* qkv, double* h1, double* logits, int* idx,
              double* gates, double* out);

/* Decoded logical weight rows [row0, row0+nrows) of one generated matrix, as
 * the layer above uses them.  kind: 1 QKV, 2 O, 3 router, 4 gate, 5 up,
 * 6 down; expert -1 = shared, 0..E-1 routed (ignored for kinds 1..3). */
int orc_weight_rows(const orc_cfg* cfg, int kind, int expert, int row0,
                    int nrows, double* dst);

/* This file's own decoders of the two storage formats, and its e4m3 encoder
 * (round to nearest even, saturating at +-448), written from the format. */
double orc_bf16_value(uint16_t bits);
double orc_e4m3_value(uint8_t code);
uint8_t orc_e4m3_code(double v);

/* ---------------------------------------------------------------- full layer
 * The decode layer with its attention half (an extension beyond the chain
 * above: the pages name the attention core with an FP8 KV cache among the
 * steps of decode -- bigchange.ai "where the time went" -- and the input
 * projections feeding it -- wireai.ir "4 key changes", item 1).  Pre-norm
 * residual form, for token t of sequence seq[t] at position pos[t]:
 *
 *   u_t   = RMSNorm(x_t) g1          RMSNorm(z) = z / sqrt(mean(z^2) + eps)
 *   qkv_t = Wqkv u_t = (q_t [Hq x hd], k_t [Hkv x hd], v_t [Hkv x hd])
 *   K[seq, pos] = e4m3(k_t / k_scale),  V[seq, pos] = e4m3(v_t / v_scale)
 *   o_t,h = sum_{j <= pos} softmax_j(q_t,h . K'_j,g / sqrt(hd)) V'_j,g,
 *           K' = k_scale dec(K), V' = v_scale dec(V), g = h / (Hq / Hkv)
 *   h1_t  = x_t + Wo o_t
 *   v_t   = RMSNorm(h1_t) g2
 *   out_t = h1_t + F_shared(v_t) + sum_{e in S_t} g_e F_e(v_t),  S_t, g from Wr v_t + b
 *
 * Every new key and value is written before any token attends, so tokens of
 * one sequence at consecutive positions (a speculative-verify step) see each
 * other causally.  No positional rotation is applied. */

/* RMSNorm of one row: y = x / sqrt(sum(x^2)/n + eps) * gamma. */
void orc_rmsnorm(const double* x, const double* gamma, int n, double eps, double* y);

/* Attention of M tokens over an e4m3 KV cache [n_seq][max_ctx][Hkv][hd]
 * (codes as given, the new tokens' included).  q row t at q + t*ldq, output
 * row t at out + t*ldo.  Returns 0, or -1 on bad arguments. */
int orc_attention(const double* q, int ldq, const uint8_t* kc, const uint8_t* vc, double k_scale,
                  double v_scale, int n_seq, int max_ctx, int Hq, int Hkv, int hd,
                  const int* seq, const int* pos, int M, double* out, int ldo);

/* The full layer.  kc / vc are read and (unless keep_new_kv) the new tokens'
 * codes written at (seq[t], pos[t]); with keep_new_kv the codes already there
 * are used (the GPU's, for parity checks).  Gains from w->g1 / w->g2 or the
 * generator (kinds KDG_NORM1 / KDG_NORM2).  Outputs (any may be NULL except
 * out): qkv [M,Nqkv], attn [M,A], h1 [M,H], v [M,H] (the MoE input), logits,
 * idx, gates, out [M,H]. */
int orc_layer_full(const orc_cfg* cfg, const orc_weights* w, const double* bias, const double* x,
                   int M, uint8_t* kc, uint8_t* vc, double k_scale, double v_scale, int n_seq,
                   int max_ctx, const int* seq, const int* pos, double eps, int keep_new_kv,
                   const int* forced_idx, int nthreads, double* qkv_out, double* attn_out,
                   double* h1_out, double* v_out, double* logits_out, int* idx_out,
                   double* gates_out, double* out);

#ifdef __cplusplus
}
#endif
#endif

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
} orc_weights;

/* One layer for M tokens.  Returns 0, or -1 on bad arguments.
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

/* This file's own decoders of the two storage formats. */
double orc_bf16_value(uint16_t bits);
double orc_e4m3_value(uint8_t code);

#ifdef __cplusplus
}
#endif
#endif

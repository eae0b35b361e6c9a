/*
 * kd.h -- C ABI of the B200 (sm_100a) mixture-of-experts decode layer library
 * (libkd.so).
 *
 * One call of kd_decode_layer runs one decode step of one transformer layer
 * for M tokens (1..64), the chain described for vLLM's latency-specialised
 * Kimi K3 decode path:
 *   - fused QKV input projection            (wireai.ir "vLLM Blackwell Kimi decode",
 *                                            section "4 key changes", item 1)
 *   - output projection + residual add      (same section, item 2)
 *   - router logits, top-k, renormalised    (same section, item 3;
 *     softmax                                bigchange.ai "where the time went")
 *   - shared SwiGLU expert on a second      (same section, item 3)
 *     stream, overlapping the routed path
 *   - routed SwiGLU experts over the active experts only, weighted combine
 * and the multi-layer loop of a decode step captured in a CUDA graph with the
 * next layer's static weights prefetched into L2 (same section, item 4, and
 * section "extending the pattern to other models").
 *
 * Per token t, with x_t = hidden[t] and a_t = attn_out[t]:
 *   qkv_t = Wqkv x_t ;  h1_t = x_t + Wo a_t ;  l_t = Wr h1_t + b
 *   S_t   = top-k(l_t) (ties -> lower expert id)
 *   g_e   = exp(l_e) / sum_{i in S_t} exp(l_i)            e in S_t
 *   F(v)  = Wd (silu(Wg v) * (Wu v))
 *   hidden[t] <- bf16( h1_t + F_shared(h1_t) + s sum_{e in S_t} g_e F_e(h1_t) )
 * (s = routed_scale, 1 by default; with bias_select_only, S_t = top-k(l + b)
 * and g over the unbiased l -- the selection-only expert bias of
 * DeepSeek-V3-style routers.)
 *
 * Conventions
 *   - Every function returns KD_OK (0) or a negative KD_E* code; the message
 *     of the last failure on the calling thread is kd_last_error().
 *   - Device pointers are plain CUDA device addresses on the layer's device.
 *     `stream` arguments are cudaStream_t values passed as void* (NULL = the
 *     legacy default stream).
 *   - Nothing here falls back to another implementation: unsupported shapes
 *     are rejected with KD_EINVAL / KD_ERANGE.
 */
#ifndef KD_H
#define KD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KD_OK 0
#define KD_EINVAL (-1)       /* null pointer, bad config field                  */
#define KD_ERANGE (-2)       /* M outside 1..max_tokens                          */
#define KD_ECUDA (-3)        /* a CUDA runtime call failed                       */
#define KD_ENOMEM (-4)       /* device or host allocation failed                 */
#define KD_ETIMEOUT (-5)     /* a kernel's bounded wait gave up (device error)   */
#define KD_EDEVICE (-6)      /* other device-side error flag (bad routing)       */

#define KD_WBF16 0           /* bf16 weights                                     */
#define KD_WFP8 1            /* FP8 e4m3 weights, one fp32 scale per 128x128 block */

typedef struct kd_config {
  int hidden;        /* H; multiple of 128                                      */
  int q_heads;       /* attention heads: attn_out width A = q_heads * head_dim  */
  int kv_heads;      /* QKV width = (q_heads + 2 kv_heads) * head_dim            */
  int head_dim;      /* A multiple of 128                                       */
  int n_experts;     /* E routed experts, 1..1024                                */
  int top_k;         /* k, 1..min(E, 16)                                          */
  int n_shared;      /* shared experts: 0 or 1                                   */
  int inter;         /* I expert intermediate size; multiple of 128              */
  int wdtype;        /* KD_WBF16 or KD_WFP8                                      */
  int layer_id;      /* id of the layer in the seeded weight generator           */
  int max_tokens;    /* largest M a call may use, 1..64; sizes the workspaces    */
  const float* router_bias; /* host [E] additive router bias, or NULL; copied    */
  int mma_min_tokens;/* calls with M >= this use the tensor-core (tcgen05) kernels,
                        smaller M the CUDA-core streaming kernels; 0 = default (1:
                        the tensor cores for every M), > 64 = never.            */
  /* Full layer (kd_decode_layer_full); all zero for the layer above.         */
  int full_layer;    /* 1: RMSNorm gains are generated and the layer takes the
                        full-layer call; 0: kd_decode_layer only                */
  float rms_eps;     /* RMSNorm epsilon; 0 = 1e-6                                */
  int kv_n_seq;      /* KV cache geometry: sequences ...                         */
  int kv_max_ctx;    /* ... and positions per sequence                           */
  float k_scale;     /* e4m3 cache scales: dequantised value = code value x scale */
  float v_scale;
  /* Gating variants (both layer kinds); zero keeps the plain gating.         */
  int bias_select_only; /* 1: router_bias chooses the experts only; the gates
                           are the softmax of the unbiased logits over the
                           selection (the logits buffer then holds unbiased
                           logits)                                             */
  float routed_scale;   /* factor on the routed experts' sum; 0 = 1           */
  /* Tensor parallelism: this layer is shard tp_rank of tp_size (0 or 1 = the
     whole layer).  A shard holds q heads [r Hq/R, (r+1) Hq/R) with the kv
     heads they read (QKV rows, o-proj input columns), router rows
     [r E/R, (r+1) E/R) and intermediate rows [r I/R, (r+1) I/R) of every
     expert; it runs the kd_tp_* calls below, not kd_decode_layer.
     Requires q_heads, E and I divisible by tp_size, I/tp_size and the shard's
     o-proj columns multiples of 128; with FP8 weights also E/tp_size and
     head_dim multiples of 128 (the 128 x 128 scale blocks stay whole); no
     full layer.  Otherwise KD_EINVAL.                                        */
  int tp_rank;
  int tp_size;
  /* FP8 expert activations on the tensor cores: e4m3 terms of each activation
     (times its 128 x 128 weight block's scale and a power of two per token
     and tile): 0 or 2 = two terms (~8 significant bits); 1 = one term (W8A8,
     ~4 significant bits, larger error).  Ignored for bf16 weights; other
     values KD_EINVAL.                                                        */
  int fp8_act_terms;
} kd_config;

typedef struct kd_layer kd_layer;
typedef struct kd_stack kd_stack;

/* Allocate one layer on the current CUDA device and generate its weights on
 * the device from (seed, layer_id) with the counter-based generator of
 * kdgen/kd_gen.h (synchronous).  The layer owns weights, workspaces, a side
 * stream and events; *out receives the handle.  Errors: KD_EINVAL for a bad
 * config, KD_ENOMEM, KD_ECUDA; on any error everything allocated so far is
 * released.  Test hooks: with the environment variable KD_TEST_FAIL_ALLOC_AT=n
 * (n >= 1) the n-th device allocation of the call fails as if the device
 * were out of memory; with KD_TEST_STALL_WAIT=1 the layer's tensor-core
 * kernels first wait on a pipeline barrier that nothing completes, so that
 * the bounded wait gives up after its limit (2 s), the kernel stops its roles
 * and returns, and kd_layer_check reports KD_ETIMEOUT (the layer stays
 * usable; the calls' outputs are then undefined). */
int kd_layer_create(const kd_config* cfg, uint64_t seed, kd_layer** out);

/* Release everything kd_layer_create allocated (NULL is ignored).  The caller
 * must make sure no call on the layer is still running on the device. */
void kd_layer_destroy(kd_layer* layer);

/* One decode step of the layer for M tokens, enqueued on `stream`.
 *   hidden_inout  bf16 [M, H] device, row-major: the layer input x on entry,
 *                 the layer output on exit (updated in place, stream-ordered)
 *   attn_out      bf16 [M, q_heads*head_dim] device, row-major (read only)
 * The call makes no host synchronisation and allocates nothing, so it can be
 * captured into a CUDA graph.  Two calls on one layer must not overlap on the
 * device (they share the layer's workspaces).  Errors: KD_EINVAL (null
 * pointers), KD_ERANGE (M outside 1..max_tokens), KD_ECUDA (launch failure).
 * Device-side failures are reported by kd_layer_check. */
int kd_decode_layer(kd_layer* layer, void* hidden_inout, const void* attn_out, int M,
                    void* stream);

/* One decode step of the FULL layer (pre-norm residual block with its
 * attention half) for M tokens, enqueued on `stream`.  Token t belongs to
 * sequence seq[t] and sits at position pos[t] of it:
 *   u = RMSNorm(x) g1;  (q, k, v) = Wqkv u
 *   K[seq, pos] = e4m3(k / k_scale),  V[seq, pos] = e4m3(v / v_scale)
 *   o_h = softmax_j(q_h . K'_j / sqrt(head_dim)) V'_j over j = 0..pos of the
 *         token's sequence, kv head h / (q_heads / kv_heads)
 *   h1 = x + Wo o;  w = RMSNorm(h1) g2;  out = h1 + F_shared(w) + sum g_e F_e(w)
 * with the router on w (bigchange.ai "where the time went": attention with an
 * FP8 KV cache among the steps of decode; wireai.ir "4 key changes", items
 * 1-3).  Every new key and value is written before any token attends, so
 * tokens of one sequence at consecutive positions (a speculative-verify
 * step) see each other causally.  No positional rotation is applied.
 *   hidden_inout  bf16 [M, H] device: x on entry, the layer output on exit
 *   k_cache,      device e4m3 codes [kv_n_seq][kv_max_ctx][kv_heads][head_dim]
 *   v_cache       (caller-owned; the call writes the M new positions)
 *   seq, pos      device int32 [M]; 0 <= seq < kv_n_seq, 0 <= pos < kv_max_ctx
 * The layer must have been created with full_layer = 1, kv_heads >= 1,
 * q_heads / kv_heads in {1, 2, 4, 8} and head_dim 64 or 128.  Same
 * capturability and workspace rules as kd_decode_layer.  Errors: KD_EINVAL
 * (null pointers, a layer without full_layer), KD_ERANGE (M outside
 * 1..max_tokens), KD_ECUDA.  Out-of-range seq / pos entries are skipped on
 * the device (that token's attention output is zero) and reported by
 * kd_layer_check as KD_EDEVICE. */
int kd_decode_layer_full(kd_layer* layer, void* hidden_inout, void* k_cache, void* v_cache,
                         const int* seq, const int* pos, int M, void* stream);

/* ---------------------------------------------------------------- tensor parallel
 * One decode step of a sharded layer (kd_config.tp_size = R > 1) is four
 * calls, with three exchanges between the R shards' calls done by the caller
 * (NCCL, or any other all-reduce / all-gather; the ranks' order of
 * additions is theirs).  The sharding follows wireai.ir "vLLM Blackwell Kimi
 * decode", section "4 key changes", items 2 (o-proj partial sums reduced
 * across GPUs with the residual) and 3 (router scores split among the
 * tensor-parallel ranks).  Exchange buffers (kd_tp_buffers) are
 * layer-owned device memory, fp32 row-major:
 *   p        [M, H]        o-proj partial sum, then (after the caller's
 *                          all-reduce, in place) the sum over shards
 *   lshard   [M, E/R]      this shard's router logits
 *   lfull    [M, E]        all shards' logits side by side, shard r in
 *                          columns [r E/R, (r+1) E/R) (the caller's all-gather)
 *   y        [M, H]        expert partial sum, then (all-reduce, in place) the
 *                          sum over shards
 * Calls (all enqueue on `stream`; M in 1..max_tokens, else KD_ERANGE):
 *   kd_tp_attn     hidden bf16 [M, H] and attn bf16 [M, q_heads head_dim]
 *                  (the whole attention output; the shard reads its heads'
 *                  columns) -> its QKV rows (kd_layer_qkv: bf16 [M, rows],
 *                  q rows of its heads, then k and v of its kv heads) and p.
 *   kd_tp_router   hidden and the summed p -> h1 = x + p (kept), lshard.
 *   kd_tp_moe      lfull -> the selection (identical on every shard), the
 *                  shard's rows of every selected and shared expert -> y
 *                  (without h1).
 *   kd_tp_combine  the summed y -> hidden = bf16(h1 + y), in place.
 * Errors: KD_EINVAL (null or unsharded layer), KD_ERANGE, KD_ECUDA. */
int kd_tp_buffers(const kd_layer* layer, float** p, float** lshard, float** lfull, float** y);
int kd_tp_attn(kd_layer* layer, const void* hidden, const void* attn, int M, void* stream);
int kd_tp_router(kd_layer* layer, const void* hidden, int M, void* stream);
int kd_tp_moe(kd_layer* layer, int M, void* stream);
int kd_tp_combine(kd_layer* layer, void* hidden, int M, void* stream);

/* Synchronise the device and report (then clear) the layer's device error
 * word: KD_OK, KD_ETIMEOUT (a bounded wait inside a kernel gave up) or
 * KD_EDEVICE. */
int kd_layer_check(kd_layer* layer);

/* bf16 [M, (q_heads + 2 kv_heads) * head_dim] QKV projection of the last call
 * (layer-owned device buffer, valid until the next call on the layer). */
const void* kd_layer_qkv(const kd_layer* layer);

/* Enqueue on `stream` an L2 prefetch of the layer's static weights (QKV,
 * o-proj, router, shared expert), at most `max_bytes` of them in that order
 * (0 = the device's L2 size).  Static weights only: activations are never
 * prefetched (wireai.ir, section "validation of AI-generated kernels"). */
int kd_layer_prefetch_l2(const kd_layer* layer, size_t max_bytes, void* stream);

/* Intermediate device buffers of the last call, for tests and tools.
 *   which: KD_T_H1F fp32 [M,H] | KD_T_H1B bf16 [M,H] | KD_T_LOGITS fp32 [M,E]
 *          KD_T_IDX int32 [M,k] | KD_T_GATES fp32 [M,k]
 *          KD_T_COUNTS int32 [E] | KD_T_NACTIVE int32 [1]
 *          KD_T_YSHARED fp32 [M,H] | KD_T_YROUTED fp32 [M*k,H]
 *          (full layer: KD_T_H1F / KD_T_H1B hold the MoE input w = RMSNorm(h1) g2)
 * *dev_ptr receives the layer-owned pointer. */
#define KD_T_H1F 0
#define KD_T_H1B 1
#define KD_T_LOGITS 2
#define KD_T_IDX 3
#define KD_T_GATES 4
#define KD_T_COUNTS 5
#define KD_T_NACTIVE 6
#define KD_T_YSHARED 7
#define KD_T_YROUTED 8
#define KD_T_ATTN 9          /* full layer: fp32 [M, q_heads*head_dim] attention output */
#define KD_T_RESID 10        /* full layer: fp32 [M, H] h1 (residual stream after attention) */
#define KD_T_ACT 11          /* fp32 [M*k, I] routed SwiGLU activations, by (expert, token) position */
#define KD_T_ACTSH 12        /* fp32 [M, I] the shared expert's SwiGLU activations */

int kd_layer_debug_tensor(const kd_layer* layer, int which, void** dev_ptr);

/* Device copy of one generated weight matrix in its LOGICAL layout, for
 * checking the generator: kind 1 QKV [Nqkv,H], 2 o-proj [H,A], 3 router [E,H],
 * 4 gate [I,H], 5 up [I,H], 6 down [H,I]; expert -1 = shared, else routed id.
 * Copies rows [row0, row0+nrows) into dst (host memory): bf16 bits (2 bytes
 * per element) or e4m3 codes (1 byte); for FP8 also the fp32 scales of the
 * rows' 128-row blocks into dst_scales (host, may be NULL). */
int kd_layer_read_weight(const kd_layer* layer, int kind, int expert, int row0, int nrows,
                         void* dst, float* dst_scales);

/* Byte counts used for the HBM roofline: static weight bytes (QKV, o-proj,
 * router, shared expert, with FP8 scales) and the bytes of one routed expert. */
int kd_layer_bytes(const kd_layer* layer, uint64_t* static_bytes, uint64_t* expert_bytes);

/* Number of kernels one kd_decode_layer call with M tokens launches (all of
 * them this library's) -- the per-layer kernel count by which the write-ups
 * compare decode paths (bigchange.ai "where the time went"; wireai.ir
 * "compressing the decode loop with kernel fusion"); for a layer created
 * with full_layer, the count of one kd_decode_layer_full call.  Returns the count
 * (>= 5), or KD_EINVAL for a null layer, KD_ERANGE for M outside
 * 1..max_tokens. */
int kd_layer_launches(const kd_layer* layer, int M);

/* Multi-layer decode step.  kd_stack_create records the layers (not owned)
 * and the token count; kd_stack_run runs layer 0..n-1 in order on `stream`,
 * reading attn_out for layer l at attn_out + l*M*A, and carrying hidden.
 * On the first run (and whenever the pointers change) the sequence is
 * captured into a CUDA graph, which later runs replay; with prefetch != 0,
 * while layer l runs, a side stream prefetches layer l+1's static weights into
 * L2.  The first run of a new pointer set must not itself be inside a stream
 * capture. */
int kd_stack_create(kd_layer* const* layers, int n_layers, int M, int prefetch, kd_stack** out);
int kd_stack_run(kd_stack* stack, void* hidden_inout, const void* attn_out, void* stream);
void kd_stack_destroy(kd_stack* stack);

/* Profiling hook: with n_events == KD_N_TIMING_EVENTS, later kd_decode_layer
 * calls record the caller's events (cudaEvent_t values created with timing)
 * on the call's stream at: [0] start, [1] after the QKV + o-proj kernel,
 * [2] after the router kernel, [3] after the routed gate/up kernel, [4] after
 * the down kernel (routed + shared experts, with the final combine).  While
 * it is on, kernels of the call are not launched as programmatic dependents,
 * so that each interval covers one kernel.  n_events == 0 turns it off.  The
 * events are not owned by the layer.  Errors: KD_EINVAL. */
#define KD_N_TIMING_EVENTS 5
int kd_layer_set_timing_events(kd_layer* layer, void* const* events, int n_events);

/* Router top-k without any device allocation (the pages have no counterpart
 * of this entry point).  For callers that cannot call cudaMalloc from where
 * they run it -- e.g. a host runtime whose device memory all belongs to
 * another allocator, or a plugin that is handed only its input and output
 * buffers: the scratch that the blocks of its one launch hand to each other
 * (router logits, a block counter, the per-expert lists) lives in a
 * file-scope __device__ array of fixed size in the library, held by every
 * GPU that loads it until the process exits, instead of a cudaMalloc'd
 * workspace.
 *   router_w      device, [n_experts, hidden] bf16 (wdtype KD_WBF16) or e4m3
 *                 codes (KD_WFP8), row-major
 *   router_scales device fp32 [ceil(n_experts/128), hidden/128] for KD_WFP8,
 *                 else ignored (may be NULL)
 *   router_bias   device fp32 [n_experts] added to the logits, or NULL
 *   h1            device fp32 [M, hidden]
 *   idx_out       device int32 [M, top_k]: selected experts, descending logit,
 *                 ties -> lower id
 *   gates_out     device fp32 [M, top_k]: softmax renormalised over the top_k
 * Same arithmetic as the CUDA-core router of kd_decode_layer (the one it
 * runs for up to 8 tokens); each call raises that kernel's dynamic shared
 * memory limit to the largest size these limits need (cudaFuncSetAttribute,
 * not an allocation).  Limits: M <= 64
 * (KD_STATIC_MAX_TOKENS), n_experts <= 1024 (KD_STATIC_MAX_EXPERTS),
 * top_k <= 16, hidden <= 8192 (KD_STATIC_MAX_HIDDEN); larger sizes return
 * KD_ERANGE; null pointers, hidden not a multiple of 128 or a bad wdtype
 * KD_EINVAL.  Calls no cudaMalloc / cudaFree.  The first call in a CUDA
 * context looks up the scratch's device address (cudaGetSymbolAddress) for
 * that device and caches it with the context, so make that first call
 * before any stream capture (a call in a new context, e.g. after
 * cudaDeviceReset, looks it up again).  All calls share the scratch and it
 * keeps the last call's contents; calls that overlap on the GPU (other
 * streams, other threads) race on it.  Device-side errors are not
 * reported: the launch has no bounded waits, and the only flag its
 * selection can raise (an out-of-range expert id, which finite logits
 * cannot produce) stays in the scratch. */
#define KD_STATIC_MAX_TOKENS 64
#define KD_STATIC_MAX_EXPERTS 1024
#define KD_STATIC_MAX_HIDDEN 8192
int kd_router_topk_static(const void* router_w, const float* router_scales, int wdtype,
                          const float* router_bias, const float* h1, int M, int hidden,
                          int n_experts, int top_k, int* idx_out, float* gates_out, void* stream);

/* Message of the last failure on the calling thread ("" if none). */
const char* kd_last_error(void);

#ifdef __cplusplus
}
#endif
#endif

// kd_kernels.cuh -- the decode layer's kernels on CUDA cores (GEMV regime) and
// the device-side weight generator.
//
//   gen_bf16_kernel / gen_fp8_kernel  weights from the seeded generator
//   proj_kernel        fused QKV projection + o-proj with residual epilogue
//   router_kernel      fp32 router logits, then (last CTA) top-k, renormalised
//                      softmax and the per-expert token lists
//   gateup_kernel      SwiGLU gate/up of the active experts (or the shared one)
//   down_kernel        down projection of the active experts and the shared one,
//                      with the final combine h1 + shared + gate-weighted routed
//                      outputs -> bf16 done per 64-row block by the CTA that
//                      completes the block
#pragma once

#include "../../kdgen/kd_gen.h"
#include "kd_stream.cuh"

namespace kd {

// ------------------------------------------------------------------ generator

// Rows [lr0, lr0 + R) x columns [lc0, lc0 + K) of a logical matrix with LK
// columns (the whole matrix: lr0 = lc0 = 0, LK = K; a tensor-parallel shard:
// its rows or columns):
// dst[(r*row_mult + row_off) * K + c] = bf16(value(stream, (lr0 + r) LK + lc0 + c)).
static __global__ void gen_bf16_kernel(uint16_t* __restrict__ dst, int R, int K, uint64_t stream,
                                int row_mult, int row_off, uint64_t lr0, uint64_t lc0,
                                uint64_t LK) {
  const uint64_t n = (uint64_t)R * (uint64_t)K;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t r = i / (uint64_t)K, c = i - r * (uint64_t)K;
    dst[(r * row_mult + row_off) * (uint64_t)K + c] =
        kdg_bf16(kdg_value(stream, (lr0 + r) * LK + lc0 + c, KDG_W002));
  }
}

// One 128x128 block per CTA (256 threads): amax -> scale -> e4m3 codes.
// scales: [ceil(R/128), ceil(K/128)] table of these rows and columns.  The
// logical offsets (as for gen_bf16_kernel) are multiples of 128, so that every
// block is a block of the logical matrix.
static __global__ void __launch_bounds__(256) gen_fp8_kernel(uint8_t* __restrict__ dst,
                                                      float* __restrict__ scales, int R, int K,
                                                      uint64_t stream, int row_mult, int row_off,
                                                      uint64_t lr0, uint64_t lc0, uint64_t LK) {
  const int kb = blockIdx.x, rb = blockIdx.y, nkb = gridDim.x;
  __shared__ float wmax[8];
  float v[64];
  float amax = 0.f;
#pragma unroll
  for (int q = 0; q < 64; ++q) {
    const int e = threadIdx.x + 256 * q;
    const int r = rb * 128 + (e >> 7), c = kb * 128 + (e & 127);
    v[q] = 0.f;
    if (r < R && c < K) {
      v[q] = kdg_value(stream, (lr0 + (uint64_t)r) * LK + lc0 + (uint64_t)c, KDG_W002);
      amax = fmaxf(amax, fabsf(v[q]));
    }
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = wmax[0];
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, wmax[w]);
  const float sc = kdg_fp8_scale(amax);
  if (threadIdx.x == 0) scales[rb * nkb + kb] = sc;
#pragma unroll
  for (int q = 0; q < 64; ++q) {
    const int e = threadIdx.x + 256 * q;
    const int r = rb * 128 + (e >> 7), c = kb * 128 + (e & 127);
    if (r < R && c < K)
      dst[((uint64_t)r * row_mult + row_off) * (uint64_t)K + c] = kdg_e4m3(kdg_fp8_div(v[q], sc));
  }
}

// ------------------------------------------------------------------ layer params

struct LayerDev {
  int H, A, Nqkv, E, k, I, S, eb;       // eb = weight element bytes (2 bf16, 1 fp8)
  int nHb, nAb, nIb;                    // 128-blocks along H, A, I
  // Tensor-parallel shard (tp = 1): A, Nqkv and I are the shard's, E stays
  // the number of experts the selection runs over, Er the router rows of this
  // layer (E unsharded), attn_ld the row stride of the attention input (its
  // full width); the o-proj epilogue then writes the partial sum alone, the
  // router no selection, and the combine the fp32 expert sum into tp_y.
  int Er, attn_ld, tp;
  int test_stall;                       // test hook: tensor-core kernels stall first (bounded)
  float* tp_y;                          // [Mmax, H] expert partial sum (shards)
  float* tp_lfull;                      // [Mmax, E] gathered logits (shards)
  const float* rbias;                   // bias of the router rows (bias + first row)
  // weights (physical layouts; see kd_layer.cu)
  const uint8_t* wqkv; const uint8_t* wo; const uint8_t* wr;
  const uint8_t* wgu_sh; const uint8_t* wd_sh;
  const uint8_t* wgu; const uint8_t* wd;   // routed, expert-major
  const float* sqkv; const float* so; const float* sr;
  const float* sgu_sh; const float* sd_sh; const float* sgu; const float* sd;
  const float* bias;                       // [E] or null
  int bias_sel;                            // 1: the bias enters the selection only
  float rscale;                            // factor on the routed experts' sum
  // workspaces
  uint16_t* qkv; float* h1f; uint16_t* h1b;
  float* logits; int* idx; float* gates;
  int* counts; int* offsets; int* perm; int* active; int* n_active;
  float* act; float* act_sh;               // [Mmax*k, I] by position, [Mmax, I] (fp32)
  uint16_t* h1lo;                          // [Mmax, H] bf16(h1 - bf16(h1))   (tensor-core path)
  uint16_t* h1lo2;                         // [Mmax, H] what h1b + h1lo leave of h1 (router)
  uint16_t* act_hi; uint16_t* act_lo;      // [Mmax*k, I] bf16 pair of act    (tensor-core path)
  uint16_t* act_sh_hi; uint16_t* act_sh_lo;// [Mmax, I]
  float* ws_main; float* ws_side;          // split-K partials, main / side stream launches
  unsigned* tcnt_main; unsigned* tcnt_side;// split-K tile arrivals (self-resetting)
  float* yr; float* ysh;                   // [Mmax*k, H] by token*k+slot, [Mmax, H]
  // FP8 tensor-core experts: max |v| per (row, 64 consecutive elements) of
  // their fp32 inputs, [rows][K/64]
  float* h1g;                              // h1 (gate/up input) [Mmax]
  float* actg;                             // routed SwiGLU activations [Mmax*k]
  float* actshg;                           // the shared expert's [Mmax]
  // the residual the combine adds: h1f (the chain with a given attn_out) or
  // h1r (the full layer, where h1f holds the MoE input RMSNorm(h1) g2)
  const float* resid;
  // full layer (kd_decode_layer_full)
  int Hq, Hkv, hd, n_seq, max_ctx, att_ch, att_nch;
  float eps, k_scale, v_scale;
  const uint16_t* g1; const uint16_t* g2;  // RMSNorm gains, bf16 [H]
  float* uf; uint16_t* u_hi; uint16_t* u_lo;   // RMSNorm(x) g1 [Mmax, H]
  float* qkvf;                             // fp32 QKV projection [Mmax, Nqkv]
  float* attnf; uint16_t* attn_hi; uint16_t* attn_lo;   // attention output [Mmax, A]
  float* att_ws; unsigned* att_cnt;        // per-chunk partials, (token, kv head) arrivals
  float* h1r;                              // h1 = x + Wo o [Mmax, H]
  unsigned* rcnt;                          // router blocks done (self-resetting)
  unsigned* err;
};

struct Acts {                              // per-call activations
  const uint16_t* x;                       // [M, H] (layer input)
  const uint16_t* attn;                    // [M, A]
  uint16_t* out;                           // [M, H] (layer output, = x in place)
  int M;
  // full layer: the caller's e4m3 KV cache and each token's (sequence, position)
  uint8_t* kc; uint8_t* vc;
  const int* seq; const int* pos;
};

// The new token's key or value element (row of the fused QKV output past
// the query part) into the e4m3 cache at (seq[j], pos[j]).
KD_DEV void kv_store(const LayerDev& L, const Acts& a, int j, int row, float v) {
  const int qw = L.Hq * L.hd, kw = L.Hkv * L.hd;
  if (row < qw) return;
  int r2 = row - qw;
  const bool isv = r2 >= kw;
  if (isv) r2 -= kw;
  const int s = a.seq[j], p = a.pos[j];
  if (s < 0 || s >= L.n_seq || p < 0 || p >= L.max_ctx) {
    set_error(L.err, ERR_BAD_KV);
    return;
  }
  const float q = __fdiv_rn(v, isv ? L.v_scale : L.k_scale);
  (isv ? a.vc : a.kc)[((size_t)s * L.max_ctx + p) * kw + r2] = (uint8_t)(e4m3x2_rn(q, 0.f) & 0xFFu);
}



KD_DEV int split_lo(int n, int parts, int i) { return (int)(((long long)n * i) / parts); }

// ------------------------------------------------------------------ QKV + o-proj

// MODE 0: QKV + o-proj with residual (the chain with a given attn_out), bf16
// activations x / attn_out.  Full layer: MODE 1 QKV of u = RMSNorm(x) g1
// (fp32), which also writes the new keys / values into the KV cache; MODE 2
// o-proj of the attention output (fp32) + residual x into h1r.
template <int MODE>
struct ProjPlanT {
  const LayerDev* L; Acts a;
  int q0, q1, o0, o1;
  KD_DEV int num_segments() const { return MODE == 0 ? 2 : 1; }
  KD_DEV Seg segment(int i) const {
    Seg s;
    const int which = MODE == 0 ? i : MODE - 1;
    if (which == 0) {
      s.row_bytes = L->H * L->eb; s.w = L->wqkv + (size_t)q0 * s.row_bytes;
      s.nrows = q1 - q0; s.row0 = q0;
    } else {
      s.row_bytes = L->A * L->eb; s.w = L->wo + (size_t)o0 * s.row_bytes;
      s.nrows = o1 - o0; s.row0 = o0;
    }
    s.tok0 = 0; s.ntok = a.M; s.tag = which;
    return s;
  }
  KD_DEV const void* act_row(const Seg& s, int j) const {
    if (MODE == 1) return L->uf + (size_t)j * L->H;
    if (MODE == 2) return L->attnf + (size_t)j * L->A;
    return s.tag == 0 ? (const void*)(a.x + (size_t)j * L->H)
                      : (const void*)(a.attn + (size_t)j * L->attn_ld);
  }
  KD_DEV const float* scale_row(const Seg& s, int row) const {
    return s.tag == 0 ? L->sqkv + (size_t)(row >> 7) * L->nHb : L->so + (size_t)(row >> 7) * L->nAb;
  }
  KD_DEV bool paired() const { return false; }
  KD_DEV void epilogue(const Seg& s, int row, int j, float v) const {
    if (s.tag == 0) {
      L->qkv[(size_t)j * L->Nqkv + row] = f32_to_bf16_bits(v);
      if (MODE == 1) {
        L->qkvf[(size_t)j * L->Nqkv + row] = v;
        kv_store(*L, a, j, row, v);
      }
    } else {
      const size_t o = (size_t)j * L->H + row;
      if (MODE == 0 && L->tp) {   // a shard's o-proj partial sum
        L->h1f[o] = v;
        return;
      }
      const float h = __uint_as_float((uint32_t)a.x[o] << 16) + v;
      if (MODE == 2) {
        L->h1r[o] = h;
      } else {
        L->h1f[o] = h;
        L->h1b[o] = f32_to_bf16_bits(h);
      }
    }
  }
  KD_DEV void epilogue2(const Seg&, int, int, float, float) const {}
  KD_DEV bool wants_segment_done() const { return false; }
  KD_DEV void segment_done(const Seg&) const {}
};
using ProjPlan = ProjPlanT<0>;

// The weights are static, so the first stages are requested before waiting
// for the preceding kernel (programmatic dependent launch); the activations
// are read only after the wait.
template <int WT, int MODE = 0>
__global__ void __launch_bounds__(kThreads, 1) proj_kernel(LayerDev L, Acts a) {
  extern __shared__ uint8_t smem[];
  ProjPlanT<MODE> p;
  p.L = &L; p.a = a;
  p.q0 = split_lo(L.Nqkv, gridDim.x, blockIdx.x); p.q1 = split_lo(L.Nqkv, gridDim.x, blockIdx.x + 1);
  p.o0 = split_lo(L.H, gridDim.x, blockIdx.x); p.o1 = split_lo(L.H, gridDim.x, blockIdx.x + 1);
  stream_run<WT, MODE == 0 ? A_BF16 : A_F32>(p, smem, L.err, true);
}

// ------------------------------------------------------------------ router

// Router logits l = Wr h1 + b from the fp32 h1: CTA b owns expert rows 2b and
// 2b+1; warp w takes row 2b + w/4 and the (w%4)-th quarter of its columns.
// Each lane loads its weight chunks (16 bytes each, up to 8) before waiting
// for h1 (the router weights are static), then forms partial dot products
// with the h1 rows of 4 tokens at a time; the four quarters are added in a
// fixed order.  The CTA that finishes last then runs the selection
// (route_tokens) for every token.
constexpr int kRouterThreads = 256;
constexpr int kRouterRows = 2;
constexpr int kCoreRouterMaxM = 8;   // bf16 layers: the CUDA-core router up to this many tokens

// Accumulate one 16-byte weight chunk against up to kTT fp32 activation rows.
template <int WT>
KD_DEV void router_chunk(const uint4 wv, float scale, const float* const* arow, int col, int nt,
                         float* acc) {
  float w[16];
  if constexpr (WT == W_BF16) {
    w[0] = bf_lo(wv.x); w[1] = bf_hi(wv.x); w[2] = bf_lo(wv.y); w[3] = bf_hi(wv.y);
    w[4] = bf_lo(wv.z); w[5] = bf_hi(wv.z); w[6] = bf_lo(wv.w); w[7] = bf_hi(wv.w);
  } else {
    e4m3x4_to_f32(wv.x, w[0], w[1], w[2], w[3]);
    e4m3x4_to_f32(wv.y, w[4], w[5], w[6], w[7]);
    e4m3x4_to_f32(wv.z, w[8], w[9], w[10], w[11]);
    e4m3x4_to_f32(wv.w, w[12], w[13], w[14], w[15]);
  }
  constexpr int EPC = WTraits<WT>::EPC;
#pragma unroll
  for (int t = 0; t < kTT; ++t) {
    if (t < nt) {
      const float* ap = arow[t] + col;
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int q = 0; q < EPC / 4; ++q) {
        const uint4 a = ld_nc_v4(ap + 4 * q);
        a0 = fmaf(w[4 * q + 0], __uint_as_float(a.x), a0);
        a1 = fmaf(w[4 * q + 1], __uint_as_float(a.y), a1);
        a0 = fmaf(w[4 * q + 2], __uint_as_float(a.z), a0);
        a1 = fmaf(w[4 * q + 3], __uint_as_float(a.w), a1);
      }
      acc[t] = fmaf(a0 + a1, scale, acc[t]);
    }
  }
}


// ------------------------------------------------------------------ selection + dispatch

// Routing of the call in shared memory, built by the router's last CTA from
// the logits (and written to global memory for the expert kernels); the
// CUDA-core gate/up kernel copies it back into shared memory.
struct Route {
  int* sel;      // [M*k] selected expert of (token, slot), descending logit
  float* gv;     // [M*k] its logit
  int* cnt;      // [E] tokens per expert
  int* off;      // [E] exclusive scan of cnt
  int* act;      // [E] active experts in id order
  int* perm;     // [M*k] token*k + slot, sorted by (expert, token*k + slot)
  int* n_act;    // [1]
  int* wsum;     // [2][32] scan scratch
  int* wc;       // [kWalkWarps][E] the selection's per-warp expert counts (selection only)
};

// Warps that place the codes into the per-expert lists (contiguous ranges of
// codes, one per warp).
constexpr int kWalkWarps = 8;

// Ints of a Route in shared memory; the selection (route_tokens) also needs
// its per-warp counts after it.
__host__ __device__ constexpr size_t kRouteSmemInts(int E, int Mk) {
  return (size_t)3 * E + 3 * Mk + 1 + 64;
}
__host__ __device__ constexpr size_t kSelectSmemInts(int E, int Mk) {
  return kRouteSmemInts(E, Mk) + (size_t)kWalkWarps * E;
}

KD_DEV Route carve_route(int* base, int E, int Mk) {
  Route r;
  r.sel = base;
  r.gv = reinterpret_cast<float*>(r.sel + Mk);
  r.perm = r.sel + 2 * Mk;
  r.cnt = r.perm + Mk;
  r.off = r.cnt + E;
  r.act = r.off + E;
  r.n_act = r.act + E;
  r.wsum = r.n_act + 1;
  r.wc = r.wsum + 64;
  return r;
}

// A logit's bits as an unsigned order (sign flipped for positive values, all
// bits for negative ones; -0 ranks with +0) and back.
KD_DEV uint32_t order_bits(float v) {
  uint32_t u = __float_as_uint(v);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
KD_DEV float order_value(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// Top-k of token t by one warp: lane l holds the logits of experts l, l + 32,
// ... (PER of them, PER * 32 >= E) and their selection keys (order bits of
// the logit, plus the bias when it only steers the selection).  A selection
// key ranks by value, then by lower expert id.  Each lane keeps its best
// remaining candidate; a round takes the warp's best with two warp
// reductions (redux.sync max: the order bits, then among the lanes holding
// that value the complemented expert id), and the lane that held it drops it
// and finds its next best.  Then the softmax renormalised over the k
// selected logits, in the same order and arithmetic in every lane.
template <int PER>
KD_DEV void topk_warp(const LayerDev& L, const float* lg, const Route& R, int t,
                      bool write_global) {
  const int lane = threadIdx.x & 31;
  const int k = L.k, E = L.E;
  // with a selection-only bias the logits buffer holds the unbiased logits,
  // which the gates use
  const bool sel_bias = L.bias_sel && L.bias;
  float raw[PER];
  uint32_t hk[PER];
  unsigned live = 0;   // bit qq: expert lane + 32 qq is still a candidate
#pragma unroll
  for (int qq = 0; qq < PER; ++qq) {
    const int e = lane + 32 * qq;
    raw[qq] = e < E ? lg[(size_t)t * E + e] : 0.f;
  }
#pragma unroll
  for (int qq = 0; qq < PER; ++qq) {
    const int e = lane + 32 * qq;
    hk[qq] = order_bits(raw[qq] + (sel_bias && e < E ? __ldg(L.bias + e) : 0.f));
    if (e < E) live |= 1u << qq;
  }
  uint32_t bh = 0;   // this lane's best remaining key: order bits and slot
  int bq = -1;
  auto lane_best = [&]() {
    bh = 0;
    bq = -1;
#pragma unroll
    for (int qq = 0; qq < PER; ++qq)
      if (((live >> qq) & 1u) && (bq < 0 || hk[qq] > bh)) { bh = hk[qq]; bq = qq; }
  };
  lane_best();
  float top = 0.f, den = 0.f;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    const uint32_t lo = bq >= 0 ? ~(uint32_t)(lane + 32 * bq) : 0u;
    const uint32_t bhi = __reduce_max_sync(0xffffffffu, bh);
    const uint32_t blo = __reduce_max_sync(0xffffffffu, bh == bhi ? lo : 0u);
    const int be = (int)~blo;
    float w = 0.f;   // the winner's unbiased logit, in the lane that held it
    if (lane == (be & 31)) {
#pragma unroll
      for (int qq = 0; qq < PER; ++qq)
        if (qq == bq) w = raw[qq];
      live &= ~(1u << bq);
      lane_best();
    }
    const float v = sel_bias ? __shfl_sync(0xffffffffu, w, be & 31) : order_value(bhi);
    if (j == 0 || v > top) {   // the gates' reference value: their largest logit
      den = j == 0 ? 0.f : den * expf(top - v);
      top = v;
    }
    den += expf(v - top);
    if (lane == 0) {
      R.sel[t * k + j] = be;
      R.gv[t * k + j] = v;
    }
  }
  __syncwarp();
  if (write_global)
    for (int j = lane; j < k; j += 32) {
      L.idx[t * k + j] = R.sel[t * k + j];
      L.gates[t * k + j] = expf(R.gv[t * k + j] - top) / den;
    }
}

// Every token's top-k, one token per warp at a time.
template <int PER>
KD_DEV void topk_tokens(const LayerDev& L, const float* lg, const Route& R, int M,
                        bool write_global) {
  for (int t = threadIdx.x >> 5; t < M; t += blockDim.x >> 5)
    topk_warp<PER>(L, lg, R, t, write_global);
}

// Top-k of every token, the renormalised softmax over each selection, and the
// per-expert token lists.  lg: the logits [M, E] (global, or a copy in shared
// memory).
KD_DEV void route_tokens(const LayerDev& L, const float* lg, int M, const Route& R,
                         bool write_global) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = L.k, E = L.E;
  // keys per lane: the smallest of 4, 8, 16, 32 that covers E (E <= 1024)
  if (E <= 128) topk_tokens<4>(L, lg, R, M, write_global);
  else if (E <= 256) topk_tokens<8>(L, lg, R, M, write_global);
  else if (E <= 512) topk_tokens<16>(L, lg, R, M, write_global);
  else topk_tokens<32>(L, lg, R, M, write_global);
  __syncthreads();
  // The codes (token * k + slot) in nwalk contiguous ranges of whole 32-code
  // steps, one per warp.  A step ranks the codes of equal experts with a
  // match; its lowest lane per expert does the bookkeeping.
  const int ncode = M * k;
  const int nwalk = min(kWalkWarps, (int)(blockDim.x >> 5));
  const int span = ((ncode + nwalk - 1) / nwalk + 31) & ~31;
  for (int i = threadIdx.x; i < nwalk * E; i += blockDim.x) R.wc[i] = 0;
  __syncthreads();
  // each warp counts its range's codes per expert
  if (warp < nwalk) {
    int* wc = R.wc + warp * E;
    const int c1 = min(ncode, (warp + 1) * span);
    for (int c0 = warp * span; c0 < c1; c0 += 32) {
      const int c = c0 + lane;
      const int se = c < c1 ? R.sel[c] : 0;
      const bool live = c < c1 && se >= 0 && se < E;
      if (c < c1 && !live) set_error(L.err, ERR_BAD_ROUTE);
      const int e = live ? se : -1 - lane;   // unique dummies
      const unsigned same = __match_any_sync(0xffffffffu, e);
      if (live && (same & ((1u << lane) - 1u)) == 0) wc[e] += __popc(same);
      __syncwarp();
    }
  }
  __syncthreads();
  // per expert: its count, and each warp's first place among its codes
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < nwalk; ++w) {
      const int n = R.wc[w * E + e];
      R.wc[w * E + e] = run;
      run += n;
    }
    R.cnt[e] = run;
  }
  __syncthreads();
  // block-wide exclusive scans of cnt and of (cnt > 0): each thread owns
  // experts [4*tid, 4*tid+4)  (E <= 4 * blockDim.x)
  {
    int c4[4], a4[4], cs = 0, as = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = 4 * threadIdx.x + u;
      c4[u] = e < E ? R.cnt[e] : 0;
      a4[u] = c4[u] > 0;
      cs += c4[u];
      as += a4[u];
    }
    int ci = cs, ai = as;  // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int cv = __shfl_up_sync(0xffffffffu, ci, o), av = __shfl_up_sync(0xffffffffu, ai, o);
      if (lane >= o) { ci += cv; ai += av; }
    }
    if (lane == 31) { R.wsum[warp] = ci; R.wsum[32 + warp] = ai; }
    __syncthreads();
    int cb = 0, ab = 0;
    for (int w2 = 0; w2 < warp; ++w2) { cb += R.wsum[w2]; ab += R.wsum[32 + w2]; }
    int run = cb + ci - cs, arun = ab + ai - as;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = 4 * threadIdx.x + u;
      if (e < E) {
        R.off[e] = run;
        if (a4[u]) R.act[arun] = e;
        if (write_global) {
          L.counts[e] = c4[u];
          L.offsets[e] = run;
          if (a4[u]) L.active[arun] = e;
        }
      }
      run += c4[u];
      arun += a4[u];
    }
    if (threadIdx.x == blockDim.x - 1) {
      *R.n_act = arun;
      if (write_global) {
        L.offsets[E] = run;
        *L.n_active = arun;
      }
    }
  }
  __syncthreads();
  // positions in (expert, code) order: each warp places its range's codes
  if (warp < nwalk) {
    int* wc = R.wc + warp * E;
    const int c1 = min(ncode, (warp + 1) * span);
    for (int c0 = warp * span; c0 < c1; c0 += 32) {
      const int c = c0 + lane;
      const int se = c < c1 ? R.sel[c] : 0;
      const bool live = c < c1 && se >= 0 && se < E;
      const int e = live ? se : -1 - lane;
      const unsigned same = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(same & ((1u << lane) - 1u));
      if (live) {
        const int pos = R.off[e] + wc[e] + rank;
        R.perm[pos] = c;
        if (write_global) L.perm[pos] = c;
      }
      __syncwarp();
      if (live && rank == 0) wc[e] += __popc(same);
      __syncwarp();
    }
  }
  __syncthreads();
}

// Logits done by this block: the block that finishes last (of `nblocks`)
// selects every token's experts and builds the per-expert token lists in
// global memory (route scratch in dynamic shared memory).  All threads call.
KD_DEV void route_last_block(const LayerDev& L, int M, unsigned nblocks) {
  extern __shared__ int route_smem[];
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(L.rcnt, 1u);
    s_last = prev == nblocks - 1;
    if (s_last) *L.rcnt = 0u;   // every block is in: ready for the next call
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const Route R = carve_route(route_smem, L.E, M * L.k);
  route_tokens(L, L.logits, M, R, true);
}

// The routing of the call as the router left it in global memory (only the
// fields the expert kernels read).
KD_DEV Route global_route(const LayerDev& L) {
  Route r{};
  r.perm = L.perm;
  r.cnt = L.counts;
  r.off = L.offsets;
  r.act = L.active;
  r.n_act = L.n_active;
  return r;
}

// The routing of the call, as the router left it in global memory, copied
// into shared memory (all threads call).
KD_DEV void load_route(const LayerDev& L, int M, const Route& R) {
  const int E = L.E, Mk = M * L.k;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    R.cnt[e] = L.counts[e];
    R.off[e] = L.offsets[e];
    R.act[e] = L.active[e];
  }
  for (int c = threadIdx.x; c < Mk; c += blockDim.x) R.perm[c] = L.perm[c];
  if (threadIdx.x == 0) *R.n_act = *L.n_active;
  __syncthreads();
}

template <int WT>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(LayerDev L, int M) {
  constexpr int EPC = WT == W_BF16 ? 8 : 16;
  constexpr int kRouterWChunks = WT == W_BF16 ? 8 : 4;  // 16-byte chunks per lane, H <= 8192
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rloc = warp >> 2, q = warp & 3;
  const int row = blockIdx.x * kRouterRows + rloc;
  const int cq = (L.H * L.eb / 16) / 4;   // chunks per quarter row
  __shared__ float part[kRouterRows][4][64];
  // the router weights are static: load them before waiting for h1
  uint4 w[kRouterWChunks];
  float sc[kRouterWChunks];
  if (row < L.Er) {
    const uint8_t* wrow = L.wr + (size_t)row * L.H * L.eb;
#pragma unroll
    for (int i = 0; i < kRouterWChunks; ++i) {
      const int c = lane + 32 * i;
      if (c < cq) {
        const int ci = q * cq + c;
        w[i] = ld_nc_v4(wrow + (size_t)ci * 16);
        sc[i] = WT == W_FP8 ? __ldg(L.sr + (size_t)(row >> 7) * L.nHb + ((ci * EPC) >> 7)) : 1.f;
      }
    }
  }
  pdl_wait();
  if (row < L.Er) {
    for (int t0 = 0; t0 < M; t0 += kTT) {
      const int nt = M - t0 < kTT ? M - t0 : kTT;
      const float* arow[kTT];
#pragma unroll
      for (int t = 0; t < kTT; ++t) arow[t] = L.h1f + (size_t)(t0 + (t < nt ? t : 0)) * L.H;
      float acc[kTT] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kRouterWChunks; ++i) {
        const int c = lane + 32 * i;
        if (c < cq) router_chunk<WT>(w[i], sc[i], arow, (q * cq + c) * EPC, nt, acc);
      }
#pragma unroll
      for (int t = 0; t < kTT; ++t) {
        float v = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && t < nt) part[rloc][q][t0 + t] = v;
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRouterRows * M; i += kRouterThreads) {
    const int r = i / M, t = i % M, e = blockIdx.x * kRouterRows + r;
    if (e < L.Er)
      L.logits[(size_t)t * L.Er + e] =
          ((part[r][0][t] + part[r][1][t]) + (part[r][2][t] + part[r][3][t])) +
          (L.rbias && !L.bias_sel ? L.rbias[e] : 0.f);
  }
  if (!L.tp) route_last_block(L, M, gridDim.x);   // a shard's selection runs on all shards' logits
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ experts

// Routed mode: CTA b takes pairs / rows [lo, hi) of the concatenation over
// active experts (in expert-id order).  Shared mode: one expert, all tokens.
struct ExpertRange {
  int n_act, per, lo, hi;   // per = units per expert
  KD_DEV int num_segments() const {
    if (hi <= lo) return 0;
    return (hi - 1) / per - lo / per + 1;
  }
  KD_DEV void seg(int i, int& a, int& u0, int& u1) const {
    a = lo / per + i;
    const int b0 = a * per, b1 = b0 + per;
    u0 = (lo > b0 ? lo : b0) - b0;
    u1 = (hi < b1 ? hi : b1) - b0;
  }
};

struct GateUpPlan {
  const LayerDev* L; int M; bool shared; ExpertRange R;
  Route rt;                      // routing of the call (shared memory)
  KD_DEV int num_segments() const { return R.num_segments(); }
  KD_DEV Seg segment(int i) const {
    int a, u0, u1;
    R.seg(i, a, u0, u1);
    Seg s;
    s.row_bytes = L->H * L->eb;
    const size_t estride = (size_t)2 * L->I * s.row_bytes;
    if (shared) {
      s.tag = -1; s.w = L->wgu_sh; s.tok0 = 0; s.ntok = M;
    } else {
      const int e = rt.act[a];
      s.tag = e; s.w = L->wgu + (size_t)e * estride;
      s.tok0 = rt.off[e]; s.ntok = rt.cnt[e];
    }
    s.w += (size_t)(2 * u0) * s.row_bytes;
    s.row0 = 2 * u0;
    s.nrows = 2 * (u1 - u0);
    return s;
  }
  KD_DEV const void* act_row(const Seg& s, int j) const {
    const int t = shared ? j : rt.perm[s.tok0 + j] / L->k;
    return L->h1f + (size_t)t * L->H;
  }
  KD_DEV const float* scale_row(const Seg& s, int prow) const {
    const float* base = shared ? L->sgu_sh : L->sgu + (size_t)s.tag * 2 * L->nIb * L->nHb;
    return base + (size_t)((prow & 1) * L->nIb + ((prow >> 1) >> 7)) * L->nHb;
  }
  KD_DEV bool paired() const { return true; }
  KD_DEV void epilogue(const Seg&, int, int, float) const {}
  KD_DEV void epilogue2(const Seg& s, int i, int j, float g, float u) const {
    float* dst = shared ? L->act_sh + (size_t)j * L->I : L->act + (size_t)(s.tok0 + j) * L->I;
    dst[i] = silu(g) * u;
  }
  KD_DEV bool wants_segment_done() const { return false; }
  KD_DEV void segment_done(const Seg&) const {}
};

// Down projection of every active routed expert and (entry n_act) the shared
// expert, in one launch.
struct DownPlan {
  const LayerDev* L; int M; int n_act; ExpertRange R;
  KD_DEV int num_segments() const { return R.num_segments(); }
  KD_DEV Seg segment(int i) const {
    int a, u0, u1;
    R.seg(i, a, u0, u1);
    Seg s;
    s.row_bytes = L->I * L->eb;
    const size_t estride = (size_t)L->H * s.row_bytes;
    if (a >= n_act) {
      s.tag = -1; s.w = L->wd_sh; s.tok0 = 0; s.ntok = M;
    } else {
      const int e = L->active[a];
      s.tag = e; s.w = L->wd + (size_t)e * estride;
      s.tok0 = L->offsets[e]; s.ntok = L->counts[e];
    }
    s.w += (size_t)u0 * s.row_bytes;
    s.row0 = u0;
    s.nrows = u1 - u0;
    return s;
  }
  KD_DEV const void* act_row(const Seg& s, int j) const {
    return s.tag < 0 ? L->act_sh + (size_t)j * L->I : L->act + (size_t)(s.tok0 + j) * L->I;
  }
  KD_DEV const float* scale_row(const Seg& s, int row) const {
    const float* base = s.tag < 0 ? L->sd_sh : L->sd + (size_t)s.tag * L->nHb * L->nIb;
    return base + (size_t)(row >> 7) * L->nIb;
  }
  KD_DEV bool paired() const { return false; }
  KD_DEV void epilogue(const Seg& s, int h, int j, float v) const {
    if (s.tag < 0) L->ysh[(size_t)j * L->H + h] = v;
    else L->yr[(size_t)L->perm[s.tok0 + j] * L->H + h] = v;
  }
  KD_DEV void epilogue2(const Seg&, int, int, float, float) const {}
  KD_DEV bool wants_segment_done() const { return false; }
  KD_DEV void segment_done(const Seg&) const {}
};

KD_DEV ExpertRange expert_range(int n_act, int per) {
  ExpertRange r;
  r.n_act = n_act; r.per = per;
  const int total = n_act * per;
  r.lo = split_lo(total, gridDim.x, blockIdx.x);
  r.hi = split_lo(total, gridDim.x, blockIdx.x + 1);
  return r;
}

// Routed experts are known only after the router, so the routed launches
// wait for the preceding kernel before reading the routing (and before their
// first weight request); the shared expert's weights are static.
template <int WT>
__global__ void __launch_bounds__(kThreads, 1) gateup_kernel(LayerDev L, int M, int shared) {
  extern __shared__ uint8_t smem[];
  GateUpPlan p;
  p.L = &L; p.M = M; p.shared = shared != 0;
  int n_act = 1;
  if (!shared) {
    pdl_wait();
    pdl_launch_dependents();
    p.rt = carve_route(reinterpret_cast<int*>(smem + kStreamSmem), L.E, M * L.k);
    load_route(L, M, p.rt);
    n_act = *p.rt.n_act;
  }
  p.R = expert_range(n_act, L.I);
  stream_run<WT, A_F32>(p, smem, L.err, shared != 0);
}

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) down_kernel(LayerDev L, int M) {
  extern __shared__ uint8_t smem[];
  pdl_wait();
  pdl_launch_dependents();
  DownPlan p;
  p.L = &L; p.M = M;
  p.n_act = *(volatile int*)L.n_active;
  p.R = expert_range(p.n_act + L.S, L.H);
  stream_run<WT, A_F32>(p, smem, L.err, false);
}

}  // namespace kd

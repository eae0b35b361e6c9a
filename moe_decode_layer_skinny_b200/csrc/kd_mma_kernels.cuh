// kd_mma_kernels.cuh -- the layer's projections on the tensor-core engine
// (kd_mma.cuh), used when a call has enough tokens for the weight tiles to be
// real dense contractions: QKV + o-proj, router (logits, selection and token
// lists in one launch), gate/up, down, and the combine launch.  Same outputs
// as the CUDA-core kernels of kd_kernels.cuh; in addition the epilogues write
// the bf16 terms (h1b/h1lo/h1lo2, act_hi/act_lo) that the next tensor-core
// kernel multiplies.
//
// Tensor maps (one per weight matrix, 128 rows x 128 bytes per box (64 bf16
// or 128 e4m3 K values), 128B swizzle):
//   0 Wqkv [Nqkv, H]   1 Wo [H, A]   2 routed gate/up [E*2I, H]
//   3 routed down [E*H, I]   4 shared gate/up [2I, H]   5 shared down [H, I]
//   6 router [E, H]
#pragma once

#include "kd_kernels.cuh"
#include "kd_mma.cuh"

namespace kd {

// q8 converter warps of the expert kernels: the gate/up B tiles carry two
// scale variants (four e4m3 rows a token), the down ones one (two rows)
constexpr int kGateUpConv = 3;
constexpr int kDownConv = 2;
static_assert(kGateUpConv <= kQ8Conv && kDownConv <= kQ8Conv, "q8 converter tables");

constexpr int kNumMaps = 7;
struct MmaMaps {
  CUtensorMap m[kNumMaps];
};

// Largest token count among the active experts (every thread gets it; all
// threads call).  Lists in global memory: one load round per thread.
KD_DEV int max_tokens_per_expert(const int* cnt, const int* act, int n_act) {
  __shared__ int s_max;
  if (threadIdx.x == 0) s_max = 0;
  __syncthreads();
  int m = 0;
  for (int a = threadIdx.x; a < n_act; a += blockDim.x) m = max(m, cnt[act[a]]);
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(&s_max, m);
  __syncthreads();
  return s_max;
}

// ------------------------------------------------------------------ QKV + o-proj

// MODE 0: QKV + o-proj tiles of one launch (the chain with a given attn_out,
// B = the bf16 inputs).  Full layer: MODE 1 the QKV tiles with B = u =
// RMSNorm(x) g1 as a bf16 hi + lo pair (the epilogue also writes fp32 QKV and
// the new keys / values into the KV cache); MODE 2 the o-proj tiles with B =
// the attention output as hi + lo, residual x, into h1r.
template <bool F8, int MODE = 0>
struct MmaProjPlan {
  static constexpr bool kFp8 = F8;
  static constexpr bool kQ8 = false;
  static constexpr int kConv = 0;
  static constexpr int kVariants = 1;
  // FP8: h1's per-64 maxima for the q8 gate/up kernels (the full layer's
  // come from its second RMSNorm)
  static constexpr bool kGmaxOut = F8 && MODE == 0;
  // FP8: the converter writes the e4m3 tile as bf16 (exact, one term) and
  // puts the block scale on B: (x s) as a bf16 hi + lo pair, so that the
  // products stay exact to ~16 bits (h1 feeds the fp32 router)
  static constexpr int kATerms = 1;
  const LayerDev* L; Acts a; const MmaMaps* maps;
  int nsub;
  int tq, to, cq, co;   // tiles and K chunks per tile of QKV and o-proj
  KD_DEV int num_tiles() const { return tq + to; }
  KD_DEV long long tile_start(int t) const {
    return t <= tq ? (long long)t * cq : (long long)tq * cq + (long long)(t - tq) * co;
  }
  KD_DEV MUnit tile_unit(int t) const {
    MUnit m{};
    const bool q = t < tq;
    m.map = q ? 0 : 1;
    m.lrow = m.row = (q ? t : t - tq) * 128;
    m.tag = q ? 0 : 1;
    m.tok0 = 0;
    m.ntok = a.M;
    return m;
  }
  KD_DEV const CUtensorMap* map(int id) const { return &maps->m[id]; }
  KD_DEV int max_n() const { return a.M; }
  static constexpr int kTerms = MODE == 0 && !F8 ? 1 : 2;
  // B terms gathered from memory (FP8, MODE 0: x; the converter writes the
  // scaled hi + lo over it)
  static constexpr int kGatherTerms = MODE == 0 ? 1 : 2;
  KD_DEV float2 a_scale(const MUnit& m, int kc) const {
    const float sc = m.tag == 0 ? L->sqkv[(size_t)(m.row >> 7) * L->nHb + kc]
                                : L->so[(size_t)(m.row >> 7) * L->nAb + kc];
    return make_float2(sc, sc);
  }
  KD_DEV const uint8_t* b_base(const MUnit& m, int h) const {
    if (MODE == 1) return reinterpret_cast<const uint8_t*>(h ? L->u_lo : L->u_hi);
    if (MODE == 2) return reinterpret_cast<const uint8_t*>(h ? L->attn_lo : L->attn_hi);
    return reinterpret_cast<const uint8_t*>(m.tag == 0 ? a.x : a.attn);
  }
  KD_DEV int b_stride(const MUnit& m) const {
    return (m.tag == 0 ? L->H : (MODE == 0 ? L->attn_ld : L->A)) * 2;
  }
  KD_DEV int b_rowidx(const MUnit&, int j) const { return j; }
  KD_DEV bool paired() const { return false; }
  // the residual x of an o-proj output (none for QKV rows and shard partials)
  KD_DEV float epilogue_in(const MUnit& m, int r, int j) const {
    if (m.tag == 0 || (MODE == 0 && L->tp)) return 0.f;
    return __uint_as_float((uint32_t)__ldg(a.x + (size_t)j * L->H + m.lrow + r) << 16);
  }
  KD_DEV float epilogue(const MUnit& m, int r, int j, float v, float xin) const {
    const int row = m.lrow + r;
    if (m.tag == 0) {
      L->qkv[(size_t)j * L->Nqkv + row] = f32_to_bf16_bits(v);
      if (MODE == 1) {
        L->qkvf[(size_t)j * L->Nqkv + row] = v;
        kv_store(*L, a, j, row, v);
      }
      return v;
    }
    const size_t o = (size_t)j * L->H + row;
    if (MODE == 0 && L->tp) {   // a shard's o-proj partial sum
      L->h1f[o] = v;
      return v;
    }
    const float h = xin + v;
    if (MODE == 2) {
      L->h1r[o] = h;
      return h;
    }
    L->h1f[o] = h;
    store_hilo3(L->h1b, L->h1lo, L->h1lo2, o, h);   // the tensor-core router's three terms
    return h;
  }
  KD_DEV float epilogue2(const MUnit&, int, int, float, float) const { return 0.f; }
  // h1's per-64 maxima: o-proj tiles, groups of 64 rows of h
  KD_DEV bool gmax_tile(const MUnit& m) const { return m.tag == 1; }
  KD_DEV void gmax_store(const MUnit& m, int g, int j, float v) const {
    L->h1g[(size_t)j * (L->H / kQGroup) + m.lrow / kQGroup + g] = v;
  }
  KD_DEV float* ws() const { return L->ws_main; }
  KD_DEV unsigned* tile_cnt() const { return L->tcnt_main; }
  KD_DEV bool wants_unit_done() const { return false; }
  KD_DEV void unit_done(const MUnit&, MmaShared&) const {}
  KD_DEV void after_run(MmaShared&, uint8_t*) const {}
};

template <bool F8, int MODE = 0>
__global__ void __launch_bounds__(F8 ? kMThreadsF8 : kMThreads, 1)
    mma_proj_kernel(LayerDev L, Acts a, const __grid_constant__ MmaMaps maps) {
  extern __shared__ uint8_t smem[];
  MmaProjPlan<F8, MODE> p;
  p.L = &L; p.a = a; p.maps = &maps;
  p.nsub = F8 ? 2 : mma_nsub(a.M, MmaProjPlan<F8, MODE>::kTerms);
  p.tq = MODE == 2 ? 0 : L.Nqkv / 128; p.to = MODE == 1 ? 0 : L.H / 128;
  p.cq = L.H / (64 * p.nsub); p.co = L.A / (64 * p.nsub);
  pdl_wait();
  pdl_launch_dependents();
  mma_run(p, smem, L.err);
}

// ------------------------------------------------------------------ router

// fp32 router logits: the E router rows (ceil(E/128) tiles, rows past E read
// as zeros) against h1 as three bf16 terms, so that every product is exact and
// only the fp32 accumulation rounds.  Launched on a small grid (a few K chunks
// per CTA) to keep the split-K partial sums short.  The CTA that completes
// the last tile then selects every token's experts (top-k, renormalised
// softmax) and builds the per-expert token lists, all within this launch.
template <bool F8>
struct MmaRouterPlan {
  static constexpr bool kFp8 = F8;
  static constexpr bool kQ8 = false;
  static constexpr int kConv = 0;
  static constexpr int kVariants = 1;
  static constexpr bool kGmaxOut = false;
  static constexpr int kATerms = 1;
  const LayerDev* L; int M; const MmaMaps* maps;
  int nsub;
  KD_DEV int num_tiles() const { return (L->E + 127) / 128; }
  KD_DEV long long tile_start(int t) const { return (long long)t * (L->H / (64 * nsub)); }
  KD_DEV MUnit tile_unit(int t) const {
    MUnit m{};
    m.map = 6; m.lrow = m.row = t * 128; m.tag = 0; m.tok0 = 0; m.ntok = M;
    return m;
  }
  KD_DEV const CUtensorMap* map(int id) const { return &maps->m[id]; }
  KD_DEV int max_n() const { return M; }
  static constexpr int kTerms = 3;
  KD_DEV float2 a_scale(const MUnit& m, int kc) const {
    const float sc = L->sr[(size_t)(m.row >> 7) * L->nHb + kc];
    return make_float2(sc, sc);
  }
  KD_DEV const uint8_t* b_base(const MUnit&, int h) const {
    return reinterpret_cast<const uint8_t*>(h == 0 ? L->h1b : h == 1 ? L->h1lo : L->h1lo2);
  }
  KD_DEV int b_stride(const MUnit&) const { return L->H * 2; }
  KD_DEV int b_rowidx(const MUnit&, int j) const { return j; }
  KD_DEV bool paired() const { return false; }
  // the logit bias of the row (added when it is part of the logits)
  KD_DEV float epilogue_in(const MUnit& m, int r, int) const {
    const int e = m.lrow + r;
    return e < L->E && L->bias && !L->bias_sel ? __ldg(L->bias + e) : 0.f;
  }
  KD_DEV float epilogue(const MUnit& m, int r, int j, float v, float b) const {
    const int e = m.lrow + r;
    if (e < L->E) L->logits[(size_t)j * L->E + e] = v + b;
    return v;
  }
  KD_DEV float epilogue2(const MUnit&, int, int, float, float) const { return 0.f; }
  KD_DEV float* ws() const { return L->ws_main; }
  KD_DEV unsigned* tile_cnt() const { return L->tcnt_main; }
  // the CTA that completes the last tile of logits routes the call
  KD_DEV bool wants_unit_done() const { return true; }
  KD_DEV void unit_done(const MUnit&, MmaShared& sh) const {
    __threadfence();
    named_bar_sync(2, 128);
    if (threadIdx.x == 128) {
      const unsigned prev = atomicAdd(L->rcnt, 1u);
      if (prev == (unsigned)num_tiles() - 1) {
        *L->rcnt = 0u;
        sh.misc[2] = 1;
      }
    }
  }
  KD_DEV void after_run(MmaShared& sh, uint8_t* smem) const {
    if (!sh.misc[2]) return;
    __threadfence();
    // the logits into the (now idle) stage ring in one parallel pass, so that
    // the per-token selections read shared memory
    const float* lg = L->logits;
    const int n = M * L->E;
    // ring: [logits copy (if it fits)] [routing scratch]
    const size_t lbytes = ((size_t)n * sizeof(float) + 255) & ~(size_t)255;
    const size_t rbytes = sizeof(int) * kSelectSmemInts(L->E, M * L->k);
    const bool copy = lbytes + rbytes <= (size_t)kMRingBytes && (n & 3) == 0;
    if (copy) {
      // 16-byte loads, eight in flight per thread (the copy is latency-bound)
      float4* cp = reinterpret_cast<float4*>(sh.stage);
      const float4* src = reinterpret_cast<const float4*>(L->logits);
      const int n4 = n >> 2;
      for (int i0 = 0; i0 < n4; i0 += 8 * (int)blockDim.x) {
        float4 t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
          if (i < n4) t[u] = __ldcg(src + i);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
          if (i < n4) cp[i] = t[u];
        }
      }
      __syncthreads();
      lg = reinterpret_cast<const float*>(cp);
    }
    const Route R = carve_route(reinterpret_cast<int*>(sh.stage + (copy ? lbytes : 0)), L->E,
                                M * L->k);
    route_tokens(*L, lg, M, R, true);
  }
};

// 128-K chunks each router CTA streams (sets the router launch's grid: more
// CTAs stream faster, fewer leave fewer split-K partials to add up).
constexpr int kRouterChunksPerCta = 8;

template <bool F8>
__global__ void __launch_bounds__(F8 ? kMThreadsF8 : kMThreads, 1)
    mma_router_kernel(LayerDev L, int M, const __grid_constant__ MmaMaps maps) {
  extern __shared__ uint8_t smem[];
  MmaRouterPlan<F8> p;
  p.L = &L; p.M = M; p.maps = &maps;
  p.nsub = F8 ? 2 : mma_nsub(M, 3);
  pdl_wait();
  mma_run(p, smem, L.err);
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ gate/up

// Routed: tiles of the active experts' interleaved gate/up rows (2I/128 per
// expert); shared: the shared expert's (all M tokens; its own launch on the
// side stream).  bf16 weights: B = h1 as a bf16 hi/lo pair.  FP8 weights
// (q8): the e4m3 tiles as they land, B made from h1 (fp32) per stage with
// the gate rows' and the up rows' block scales (two variants), and the
// SwiGLU activations' per-64 maxima written for the down kernel.
template <bool F8, int NT = kQTerms>
struct MmaGateUpPlan {
  static constexpr int kQT = NT;         // q8: e4m3 terms of an activation (1: W8A8)
  static constexpr bool kFp8 = false;    // no converter warps
  static constexpr bool kQ8 = F8;
  static constexpr int kConv = F8 ? kGateUpConv : 0;   // q8 converter warps
  static constexpr int kVariants = F8 ? 2 : 1;
  static constexpr bool kGmaxOut = F8;
  static constexpr int kATerms = 1;
  const LayerDev* L; int M; bool shared; const MmaMaps* maps; Route rt; int n_act;
  int nsub, nmax;
  KD_DEV int tiles_per() const { return 2 * L->I / 128; }
  KD_DEV int num_tiles() const { return (shared ? 1 : n_act) * tiles_per(); }
  KD_DEV long long tile_start(int t) const {
    return (long long)t * (L->H / (F8 ? 128 : 64 * nsub));
  }
  KD_DEV MUnit tile_unit(int t) const {
    MUnit m{};
    const int a = t / tiles_per(), tt = t % tiles_per();
    if (shared) {
      m.map = 4; m.row = tt * 128; m.tag = -1; m.tok0 = 0; m.ntok = M;
    } else {
      const int e = rt.act[a];
      m.map = 2; m.row = e * 2 * L->I + tt * 128; m.tag = e;
      m.tok0 = rt.off[e]; m.ntok = rt.cnt[e];
    }
    m.lrow = tt * 128;
    return m;
  }
  KD_DEV const CUtensorMap* map(int id) const { return &maps->m[id]; }
  KD_DEV int max_n() const { return nmax; }
  // bf16: hi + lo activations; q8: NT e4m3 terms for each of the two
  // scale variants (B tiles per stage)
  static constexpr int kTerms = F8 ? kVariants * NT : 2;
  KD_DEV const uint8_t* b_base(const MUnit&, int h) const {
    return reinterpret_cast<const uint8_t*>(h ? L->h1lo : L->h1b);
  }
  KD_DEV int b_stride(const MUnit&) const { return L->H * 2; }
  KD_DEV int b_rowidx(const MUnit& m, int j) const {
    return shared ? j : rt.perm[m.tok0 + j] / L->k;
  }
  // q8: rows alternate gate / up, each with its own block scales (logical
  // row block tt / 2); variant 0 = gate, 1 = up
  KD_DEV float w_scale_v(const MUnit& m, int kc, int v) const {
    const int tt = m.lrow >> 7;
    const float* base = shared ? L->sgu_sh : L->sgu + (size_t)m.tag * 2 * L->nIb * L->nHb;
    return __ldg(base + (size_t)v * L->nIb * L->nHb + (size_t)(tt >> 1) * L->nHb + kc);
  }
  KD_DEV const float* x_row(const MUnit& m, int j) const {
    return L->h1f + (size_t)b_rowidx(m, j) * L->H;
  }
  KD_DEV const float* g_row(const MUnit& m, int j) const {
    return L->h1g + (size_t)b_rowidx(m, j) * (L->H / kQGroup);
  }
  KD_DEV int kgroups() const { return L->H / kQGroup; }
  KD_DEV bool paired() const { return true; }
  KD_DEV float epilogue(const MUnit&, int, int, float) const { return 0.f; }
  KD_DEV float epilogue2(const MUnit& m, int p, int j, float g, float u) const {
    const int i = m.lrow / 2 + p;
    const float v = silu(g) * u;
    if (shared) {
      const size_t o = (size_t)j * L->I + i;
      L->act_sh[o] = v;
      if (!F8) store_hilo(L->act_sh_hi, L->act_sh_lo, o, v);
    } else {
      const size_t o = (size_t)(m.tok0 + j) * L->I + i;
      L->act[o] = v;
      if (!F8) store_hilo(L->act_hi, L->act_lo, o, v);
    }
    return v;
  }
  // the activations' per-64 maxima (q8): one group = the tile's 64 outputs
  KD_DEV bool gmax_tile(const MUnit&) const { return true; }
  KD_DEV void gmax_store(const MUnit& m, int, int j, float v) const {
    const int g = m.lrow / 128, nq = L->I / kQGroup;
    if (shared) L->actshg[(size_t)j * nq + g] = v;
    else L->actg[(size_t)(m.tok0 + j) * nq + g] = v;
  }
  KD_DEV float* ws() const { return shared ? L->ws_side : L->ws_main; }
  KD_DEV unsigned* tile_cnt() const { return shared ? L->tcnt_side : L->tcnt_main; }
  KD_DEV bool wants_unit_done() const { return false; }
  KD_DEV void unit_done(const MUnit&, MmaShared&) const {}
  KD_DEV void after_run(MmaShared&, uint8_t*) const {}
};

template <bool F8, int NT = kQTerms>
__global__ void __launch_bounds__(F8 ? q8_threads(kGateUpConv) : kMThreads, 1)
    mma_gateup_kernel(LayerDev L, int M, int shared, const __grid_constant__ MmaMaps maps) {
  extern __shared__ uint8_t smem[];
  MmaGateUpPlan<F8, NT> p;
  p.L = &L; p.M = M; p.shared = shared != 0; p.maps = &maps; p.n_act = 1;
  p.nmax = M;
  if (!shared) {
    pdl_wait();
    pdl_launch_dependents();
    p.rt = global_route(L);   // as the router left it (read through L2)
    p.n_act = *p.rt.n_act;
    p.nmax = max_tokens_per_expert(p.rt.cnt, p.rt.act, p.n_act);
  }
  p.nsub = F8 ? 1 : mma_nsub(p.nmax, 2);
  mma_run(p, smem, L.err);
}

// ------------------------------------------------------------------ down + combine

// Tiles of the active experts' down projections (H/128 per expert) and the
// shared expert's, its M tokens cut into groups of at most shchunk (the
// routed experts' largest token count, rounded up to 16) so that its B tiles
// are no wider than the routed ones: a wide B tile would shrink every stage's
// share of weights in the ring.  B = the SwiGLU activations as a bf16 hi/lo
// pair (q8: the e4m3 terms of the activations).  The epilogue writes each
// expert's rows of its tokens' outputs (yr, ysh); the gate-weighted combine
// into the layer output is the next launch.
template <bool F8, int NT = kQTerms>
struct MmaDownPlan {
  static constexpr int kQT = NT;         // q8: e4m3 terms of an activation (1: W8A8)
  static constexpr bool kFp8 = false;    // no converter warps
  static constexpr bool kQ8 = F8;
  static constexpr int kConv = F8 ? kDownConv : 0;   // q8 converter warps
  static constexpr int kVariants = 1;
  static constexpr bool kGmaxOut = false;
  static constexpr int kATerms = 1;
  const LayerDev* L; int M; int n_act; const MmaMaps* maps;
  int nsub, nmax, shchunk, nsh;
  KD_DEV int tiles_per() const { return L->H / 128; }
  KD_DEV int num_tiles() const { return (n_act + nsh) * tiles_per(); }
  KD_DEV long long tile_start(int t) const {
    return (long long)t * (L->I / (F8 ? 128 : 64 * nsub));
  }
  // The shared expert's tiles are spread evenly through the sequence (tile t
  // is one iff floor((t + 1) S / T) > floor(t S / T), S of the T tiles), so
  // that the CTAs' contiguous ranges share its wider token groups.
  KD_DEV MUnit tile_unit(int t) const {
    MUnit m{};
    const long long T = num_tiles(), S = (long long)nsh * tiles_per();
    const int sb = (int)((long long)t * S / T);   // shared tiles before t
    const bool sh = (int)((long long)(t + 1) * S / T) > sb;
    const int idx = sh ? sb : t - sb;
    const int a = idx / tiles_per(), tt = idx % tiles_per();
    if (sh) {
      const int q = a;
      m.map = 5; m.row = tt * 128; m.tag = -1;
      m.tok0 = q * shchunk; m.ntok = min(shchunk, M - m.tok0);
    } else {
      const int e = L->active[a];
      m.map = 3; m.row = e * L->H + tt * 128; m.tag = e;
      m.tok0 = L->offsets[e]; m.ntok = L->counts[e];
    }
    m.lrow = tt * 128;
    return m;
  }
  KD_DEV const CUtensorMap* map(int id) const { return &maps->m[id]; }
  KD_DEV int max_n() const { return nmax; }
  // bf16: hi + lo activations; q8: NT e4m3 terms
  static constexpr int kTerms = F8 ? NT : 2;
  KD_DEV float w_scale_v(const MUnit& m, int kc, int) const {
    const float* base = m.tag < 0 ? L->sd_sh : L->sd + (size_t)m.tag * L->nHb * L->nIb;
    return __ldg(base + (size_t)(m.lrow >> 7) * L->nIb + kc);
  }
  KD_DEV const float* x_row(const MUnit& m, int j) const {
    return (m.tag < 0 ? L->act_sh : L->act) + (size_t)(m.tok0 + j) * L->I;
  }
  KD_DEV const float* g_row(const MUnit& m, int j) const {
    return (m.tag < 0 ? L->actshg : L->actg) + (size_t)(m.tok0 + j) * (L->I / kQGroup);
  }
  KD_DEV int kgroups() const { return L->I / kQGroup; }
  KD_DEV const uint8_t* b_base(const MUnit& m, int h) const {
    if (m.tag < 0) return reinterpret_cast<const uint8_t*>(h ? L->act_sh_lo : L->act_sh_hi);
    return reinterpret_cast<const uint8_t*>(h ? L->act_lo : L->act_hi);
  }
  KD_DEV int b_stride(const MUnit&) const { return L->I * 2; }
  KD_DEV int b_rowidx(const MUnit& m, int j) const { return m.tok0 + j; }
  KD_DEV bool paired() const { return false; }
  // a routed output's (token, slot) code (loaded for 16 tokens before their
  // stores)
  KD_DEV int epilogue_in(const MUnit& m, int, int j) const {
    return m.tag < 0 ? 0 : __ldg(L->perm + m.tok0 + j);
  }
  KD_DEV float epilogue(const MUnit& m, int r, int j, float v, int code) const {
    const int h = m.lrow + r;
    if (m.tag < 0) L->ysh[(size_t)(m.tok0 + j) * L->H + h] = v;
    else L->yr[(size_t)code * L->H + h] = v;
    return v;
  }
  KD_DEV float epilogue2(const MUnit&, int, int, float, float) const { return 0.f; }
  KD_DEV float* ws() const { return L->ws_main; }
  KD_DEV unsigned* tile_cnt() const { return L->tcnt_main; }
  KD_DEV bool wants_unit_done() const { return false; }
  KD_DEV void unit_done(const MUnit&, MmaShared&) const {}
  KD_DEV void after_run(MmaShared&, uint8_t*) const {}
};

template <bool F8, int NT = kQTerms>
__global__ void __launch_bounds__(F8 ? q8_threads(kDownConv) : kMThreads, 1)
    mma_down_kernel(LayerDev L, int M, const __grid_constant__ MmaMaps maps) {
  extern __shared__ uint8_t smem[];
  pdl_wait();
  pdl_launch_dependents();
  MmaDownPlan<F8, NT> p;
  p.L = &L; p.M = M; p.maps = &maps;
  p.n_act = *(volatile int*)L.n_active;
  p.nmax = max_tokens_per_expert(L.counts, L.active, p.n_act);
  p.shchunk = M;
  p.nsh = 0;
  if (L.S) {
    p.shchunk = min(M, max(16, pad16(p.nmax)));
    p.nsh = (M + p.shchunk - 1) / p.shchunk;
    p.nmax = max(p.nmax, p.shchunk);
  }
  p.nsub = F8 ? 1 : mma_nsub(p.nmax, 2);
  mma_run(p, smem, L.err);
}

}  // namespace kd

namespace kd {

// ------------------------------------------------------------------ combine

// out = bf16(h1 + shared expert + sum_j gate_j * routed expert j), token-major,
// two outputs per thread per step.  The expert outputs were written by the
// down launch that precedes this one.
__global__ void __launch_bounds__(256) combine_kernel(LayerDev L, int M, uint16_t* out) {
  pdl_wait();
  const int H2 = L.H / 2, k = L.k;
  const int n = M * H2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int t = i / H2, h = 2 * (i - t * H2);
    const size_t o = (size_t)t * L.H + h;
    float2 v = L.tp_y ? make_float2(0.f, 0.f) : __ldcg(reinterpret_cast<const float2*>(L.resid + o));
    if (L.S) {
      const float2 y = __ldcg(reinterpret_cast<const float2*>(L.ysh + o));
      v.x += y.x;
      v.y += y.y;
    }
    for (int j = 0; j < k; ++j) {
      const float g = L.rscale * __ldcg(L.gates + t * k + j);
      const float2 y = __ldcg(reinterpret_cast<const float2*>(L.yr + ((size_t)t * k + j) * L.H + h));
      v.x += g * y.x;
      v.y += g * y.y;
    }
    if (L.tp_y) {   // a shard's expert partial sum
      *reinterpret_cast<float2*>(L.tp_y + o) = v;
      continue;
    }
    const uint32_t pair = (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
    *reinterpret_cast<uint32_t*>(out + o) = pair;
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ tensor-parallel shard

// h1 = x + (the o-proj partial sums of all shards, summed in place in h1f by
// the caller), and the copies of h1 the later kernels read: bf16 (FP8
// weights) or the bf16 hi + mid + lo terms, and for FP8 the per-64 maxima.
// One thread per (token, 64 consecutive elements).
__global__ void __launch_bounds__(256) tp_h1_kernel(LayerDev L, const uint16_t* x, int M, int fp8) {
  static_assert(kQGroup == 64, "one thread per group of maxima");
  const int ng = L.H / 64;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * ng) return;
  const int t = i / ng, g = i - t * ng;
  float mx = 0.f;
  for (int u = 0; u < 64; ++u) {
    const size_t o = (size_t)t * L.H + g * 64 + u;
    const float h = __uint_as_float((uint32_t)x[o] << 16) + L.h1f[o];
    L.h1f[o] = h;
    if (fp8) L.h1b[o] = f32_to_bf16_bits(h);
    else store_hilo3(L.h1b, L.h1lo, L.h1lo2, o, h);
    mx = fmaxf(mx, fabsf(h));
  }
  if (fp8 && L.h1g) L.h1g[(size_t)t * (L.H / kQGroup) + g] = mx;
}

// The selection, softmax and token lists of a shard from the gathered logits
// (one CTA; the same on every shard).
__global__ void __launch_bounds__(kRouterThreads) tp_route_kernel(LayerDev L, int M) {
  extern __shared__ int route_smem[];
  const Route R = carve_route(route_smem, L.E, M * L.k);
  route_tokens(L, L.tp_lfull, M, R, true);
}

// hidden = bf16(h1 + the expert partial sums of all shards).
__global__ void __launch_bounds__(256) tp_final_kernel(LayerDev L, uint16_t* out, int M) {
  const size_t n = (size_t)M * L.H;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    out[i] = f32_to_bf16_bits(L.h1f[i] + L.tp_y[i]);
}

}  // namespace kd

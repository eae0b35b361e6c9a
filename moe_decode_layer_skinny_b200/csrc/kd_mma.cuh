// kd_mma.cuh -- tensor-core engine (tcgen05) for token counts where the
// projections are real dense contractions (M >= a few tokens).
//
// Swap-AB: a 128-row weight tile is the MMA's A operand (M = 128) and the
// tokens are its N (padded to a multiple of 16), so one kind::f16 MMA of
// 128 x N x 16 consumes 4 KB of weights.  Per CTA (one per SM), warp roles:
//   warp 0      TMA producer: 2-D tiled loads (128B swizzle) of the weight tile
//               (one or two [128 rows x 64 K] boxes per stage) into a ring
//   warp 1      MMA issuer: owns the TMEM accumulators (two buffers of N fp32
//               columns), issues tcgen05.mma, commits stage releases
//   warps 2-3   B producers: gather the tokens' bf16 rows (64 K at a time)
//               into the stage in the same swizzled K-major layout (q8
//               plans: warp 2 copies the fp32 rows, warp 3 converts them)
//   warps 4-7   epilogue: tcgen05.ld of the accumulator (lane = weight row),
//               then the plan's epilogue, or a split-K partial
//   warps 8-15  FP8 projections only: e4m3 tiles -> scaled bf16 A tiles
//   warps 8 ..  q8 plans: the other converters (the kQ8Conv converters take
//               stages in turn)
// Activations that must stay fp32-accurate come as a sum of bf16 terms, all
// multiplied into the same accumulator: the expert inputs (h1, the SwiGLU
// activations) as hi + lo (hi = bf16(v), lo = bf16(v - hi): ~16 significant
// bits); the router's h1 as hi + mid + lo (all 24 bits of the fp32 value; the
// products with bf16 weights are exact in the fp32 accumulator).
//
// FP8 experts ("q8" plans) take the e4m3 weight tile as TMA lands it, with no
// conversion, into kind::f8f6f4 MMAs (128 x N x 32).  The 128 x 128 block
// scale of the weights cannot sit on an e4m3 operand, so the B producers put
// it on the activations: for each stage (one 128 x 128 weight block) they
// write the live tokens' fp32 activations times (block scale x 2^P) as two
// e4m3 terms, t0 = e4m3(v), t1 = e4m3(v - t0), with one power of two 2^P per
// (token, tile) that puts the largest |activation x block scale| of the tile
// in [128, 256) (from per-64-element maxima the producing kernel writes).
// Gate and up rows of a paired tile have scales of their own, so a paired
// tile gets two B variants.  The B rows are token-major, C = variants x terms
// rows a token (row j C + v kQTerms + h), so that one MMA of N = pad16(C ntok)
// covers them all with little padding.  The accumulators stay in TMEM for the
// whole unit, and the epilogue adds a token's term columns and multiplies by
// 2^-P once.
// Work units are (weight tile, K part); a tile split over several parts is
// summed in part order by the unit that completes it (deterministic).
#pragma once

#include <cuda.h>

#include "kd_common.cuh"

namespace kd {

// ------------------------------------------------------------------ PTX

KD_DEV void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), version 1.
KD_DEV uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);           // start address
  d |= (uint64_t)1u << 16;                            // leading byte offset (16 B, unused)
  d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset
  d |= (uint64_t)1u << 46;                            // version
  d |= (uint64_t)2u << 61;                            // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M = 128.
KD_DEV uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (K-major), fp32 D, M = 128.
KD_DEV uint32_t idesc_e4m3(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

KD_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
KD_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

KD_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

KD_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

KD_DEV void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)acc) : "memory");
}

KD_DEV void mma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)acc) : "memory");
}

// Arrive once on `bar` when every MMA issued so far by this thread completed.
KD_DEV void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

KD_DEV void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

KD_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ engine

constexpr int kMThreads = 256;
constexpr int kMThreadsF8 = 512;      // + 8 converter warps (e4m3 -> bf16 A tiles)
constexpr int kQ8Conv = 4;            // q8: most converter warps (warp 3, then warps 8 ..)
// q8 plans: threads of a CTA with `conv` converter warps (Plan::kConv)
constexpr int q8_threads(int conv) { return 32 * (8 + conv - 1); }
constexpr int kMaxMStages = 16;
constexpr int kATileBytes = 128 * 128;                // 128 rows x 64 bf16 (one swizzle atom wide)
constexpr int kMaxSub = 2;                            // 64-K sub-tiles per stage (at most)
constexpr int kMRingBytes = 222 * 1024;                // stages (+ 3 KB below: 225 KB per CTA)
constexpr int kMaxN = 64;                             // tokens per MMA (N)
constexpr int kMaxTerms = 3;                          // bf16 terms of an activation
constexpr size_t kWsFloatsPerCta = 2 * 128 * 64;     // split-K partial slots of one CTA
constexpr size_t kMmaSmem = (size_t)kMRingBytes + 1024 /*align*/ + 3840 /*barriers, scratch*/;
static_assert(kMmaSmem + 64 <= 227 * 1024, "shared memory per CTA (with the kernels' static bytes)");
constexpr int kQ8AccCols = 256;                       // q8: one accumulator, <= 2 x 2 x 64 columns
constexpr int kQ8TmemCols = 2 * kQ8AccCols;           // q8: two accumulators
// bf16 plans: one accumulator holds every B term's columns side by side
// (term h of token j in column h N + j, N = pad16(ntok)), <= 3 x 64 columns;
// two buffers kBfAccCols apart in the 512 columns the CTA allocates
constexpr int kBfAccCols = 256;
static_assert(kMaxTerms * kMaxN <= kBfAccCols, "bf16 accumulators");
constexpr int kQGroup = 64;                           // activation elements per stored maximum
constexpr int kQTerms = 2;                            // e4m3 terms of a q8 activation (at most;
                                                      // a plan's kQT: 2, or 1 for W8A8)
constexpr int kQ8XBudget = 40 * 1024;                 // q8: bytes of the activation-row ring

// One unit of work: K chunks [kc0, kc0 + nkc) of a 128-row weight tile.
struct MUnit {
  int map;        // tensor map index (plan-defined)
  int row;        // first row of the tile in the tensor map
  int kc0, nkc;   // K chunks (64 elements each)
  int tile;       // tile id within the launch (split-K bookkeeping)
  int part, nparts;
  int tok0, ntok; // token list range (plan-defined meaning)
  int tag;        // plan-defined (matrix, expert)
  int lrow;       // first row of the tile in its logical output (epilogue index)
};

__host__ __device__ inline int pad16(int n) { return (n + 15) & ~15; }

// Stream-K partition of a launch: the K chunks of all tiles, concatenated in
// tile order, are cut into min(gridDim.x, chunks) equal ranges; CTA b takes
// range b.  A
// tile that straddles ranges is computed in parts (one per CTA, part p by
// CTA first_owner + p) and summed, in part order, by the part that finishes
// last.  Only a CTA's first and last unit can be partial, so the partials
// live in two slots per CTA: the tile's part 0 in slot 1 (the end of the
// first owner's range), every later part in slot 0 (the start of its range).  Plan: int num_tiles(); long long
// tile_start(int t) (first chunk of tile t, non-decreasing, tile_start(n) =
// total); MUnit tile_unit(int t) (map, row, tag, lrow, tok0, ntok filled).
template <class Plan>
struct CtaUnits {
  const Plan& plan;
  long long T, G, lo, hi;
  int t, nt;
  KD_DEV explicit CtaUnits(const Plan& p) : plan(p) {
    nt = plan.num_tiles();
    T = plan.tile_start(nt);
    // with fewer chunks than CTAs only the first T CTAs get one chunk each, so
    // that every CTA between two owners of a tile owns part of it
    G = T < (long long)gridDim.x ? T : (long long)gridDim.x;
    const long long b = blockIdx.x;
    lo = b < G ? b * T / G : T;
    hi = b < G ? (b + 1) * T / G : T;
    // first tile whose chunk range reaches past lo
    int a = 0, z = nt;
    while (a < z) {
      const int mid = (a + z) >> 1;
      if (plan.tile_start(mid + 1) <= lo) a = mid + 1;
      else z = mid;
    }
    t = a;
  }
  // CTA owning chunk c: the largest b < G with floor(b*T/G) <= c
  KD_DEV long long owner(long long c) const { return ((c + 1) * G + T - 1) / T - 1; }
  KD_DEV bool next(MUnit& m) {
    if (lo >= hi) return false;
    long long cs = 0, ce = 0;
    for (;; ++t) {
      if (t >= nt) return false;
      cs = plan.tile_start(t);
      ce = plan.tile_start(t + 1);
      if (cs >= hi) return false;
      if (ce > cs) break;
    }
    m = plan.tile_unit(t);
    const long long a = cs > lo ? cs : lo, z = ce < hi ? ce : hi;
    m.kc0 = (int)(a - cs);
    m.nkc = (int)(z - a);
    m.tile = t;
    const long long bf = owner(cs), bl = owner(ce - 1);
    m.nparts = (int)(bl - bf + 1);
    m.part = (int)((long long)blockIdx.x - bf);
    ++t;
    return true;
  }
};

struct MmaShared {
  uint8_t* stage;        // nst x stage_bytes, 1024-aligned
  int nst, stage_bytes;  // stage count and size (A tile + B tile for the launch's largest N)
  // q8: a ring of its own for the activation rows of a stage (the copier
  // refills a slot once a converter is done with it, ahead of the MMAs)
  uint8_t* xring;
  int nxs, xslot;
  // q8: converters that take stages (<= kQ8Conv, nxs and nst).  A converter
  // takes every nconv-th stage and waits for it by phase parity, which stays
  // unambiguous only while no slot or stage comes round twice between two of
  // its stages; the rest idle.
  int nconv;
  int nsub;              // 64-K sub-tiles per stage
  uint64_t* full;        // [nst] B written (64 arrivals), or (FP8 converter) the A tile converted
  uint64_t* afull;       // [nst] bf16 / q8 plans: the A tile landed (TMA transaction count)
  uint64_t* xfull;       // [nxs] q8 plans: a slot's activation rows landed (32 arrivals)
  uint64_t* xempty;      // [nxs] q8 plans: a converter is done with the slot (32 arrivals)
  uint64_t* empty;       // [nst] MMAs of the stage done
  uint64_t* accfull;     // [2] accumulator buffer ready for the epilogue
  uint64_t* accempty;    // [2] epilogue done reading the accumulator
  // B tiles: inside the stages (bf16 weights; bst = stage, boff = the A
  // bytes, bfull / bempty = full / empty) or a ring of their own (FP8)
  uint8_t* bst;
  int nbst, bst_bytes, boff;
  uint64_t* bfull;       // [nbst] B written (64 thread arrivals)
  uint64_t* bempty;      // [nbst] MMAs done with it
  // FP8 weights: e4m3 tiles land in a ring of their own, the converter warps
  // turn them into the stage's bf16 A tile
  uint8_t* raw;          // nraw x kRawBytes
  int nraw;
  uint64_t* rfull;       // [nraw] e4m3 tile landed (tx)
  uint64_t* rempty;      // [nraw] converted
  uint64_t* drain;       // the issuer's MMAs done, after an abort
  uint32_t* tmem_base;
  int* abort_flag;
  int* misc;             // [8] scratch ([0] split-K last part, [2] after-run flag)
  float* qmax;           // [4][16] per-warp column maxima (output group maxima)
  float* qtab;           // [2][kMaxN] q8 epilogue: 2^-P per (variant, token) of the unit
  float* cpm;            // [kQ8Conv][2][kMaxN] q8 converters: 2^P per (variant, token) of the unit
};

// The ring holds as many stages as fit.  A stage covers nsub x 64 K: nsub
// weight sub-tiles [128 rows x 64 K] (16 KB each; with nsub = 2 every row
// contributes 256 contiguous bytes per stage), then nsub B sub-tiles for the
// launch's largest token count (one per bf16 term of the activations).  nsub is 2 when that
// still leaves at least 4 stages, else 1.
__host__ __device__ inline int b_sub_bytes(int n, int terms) { return pad16(n) * 128 * terms; }

__host__ __device__ inline int mma_nsub(int nmax, int terms) {
  return kMRingBytes / (2 * (kATileBytes + b_sub_bytes(nmax, terms))) >= 4 ? 2 : 1;
}

// FP8 weights: one e4m3 tile [128 rows x 128 K] (one scale block) per stage.
// Two or three converted A stages; B tiles get a ring of their own (2-4 deep,
// up to a third of what is left) so that the gathers run ahead; the rest
// holds e4m3 tiles.
constexpr int kRawBytes = 128 * 128;

KD_DEV MmaShared carve_mma_smem(uint8_t* base, int nmax, int terms, int nsub, bool fp8,
                                int aterms, bool q8 = false, int conv = 0) {
  MmaShared s;
  s.nsub = nsub;
  s.stage_bytes = nsub * (aterms * kATileBytes + b_sub_bytes(nmax, terms));   // bf16: A + B
  if (q8) s.stage_bytes = kATileBytes + pad16(terms * nmax) * 128;           // A + packed B
  // q8: slots for the rows' fp32 activations of a 128-K chunk (512 B a row,
  // for the launch's largest token count), as many as fit kQ8XBudget (2 ..
  // kMaxMStages), after the stages
  s.xslot = 0;
  s.nxs = 0;
  s.nconv = 0;
  if (q8) {
    s.xslot = ((nmax + 1) / 2) * 1024;
    const int nx = kQ8XBudget / s.xslot;
    s.nxs = nx < 2 ? 2 : (nx > kMaxMStages ? kMaxMStages : nx);
  }
  uintptr_t p = (reinterpret_cast<uintptr_t>(base) + 1023) & ~uintptr_t(1023);
  s.stage = reinterpret_cast<uint8_t*>(p);
  uint64_t* bars = reinterpret_cast<uint64_t*>(p + (size_t)kMRingBytes);
  s.full = bars;
  s.empty = s.full + kMaxMStages;
  s.rfull = s.empty + kMaxMStages;
  s.rempty = s.rfull + kMaxMStages;
  if (fp8) {
    s.stage_bytes = nsub * aterms * kATileBytes;
    // three converted stages hide the MMA's completion latency (measured: a
    // fourth, which leaves fewer e4m3 slots in flight, is slower)
    s.nst = 3;
    const int bstage = nsub * b_sub_bytes(nmax, terms);
    const int rem = kMRingBytes - s.nst * s.stage_bytes;
    int nb = bstage > 0 ? rem / 3 / bstage : 2;
    nb = nb < 2 ? 2 : (nb > 4 ? 4 : nb);
    s.bst = s.stage + (size_t)s.nst * s.stage_bytes;
    s.nbst = nb;
    s.bst_bytes = bstage;
    s.boff = 0;
    s.bfull = s.rempty + kMaxMStages;
    s.bempty = s.bfull + kMaxMStages;
    s.raw = s.bst + (size_t)nb * bstage;
    s.nraw = (rem - nb * bstage) / kRawBytes;
    if (s.nraw > kMaxMStages) s.nraw = kMaxMStages;
  } else {
    s.nst = (kMRingBytes - s.nxs * s.xslot) / s.stage_bytes;
    if (s.nst > kMaxMStages) s.nst = kMaxMStages;
    s.nconv = conv < s.nxs ? conv : s.nxs;
    if (s.nconv > s.nst) s.nconv = s.nst;
    s.bst = s.stage;
    s.nbst = s.nst;
    s.bst_bytes = s.stage_bytes;
    s.boff = nsub * aterms * kATileBytes;
    s.bfull = s.full;
    s.bempty = s.empty;
    s.raw = nullptr;
    s.nraw = 0;
  }
  s.accfull = s.rempty + 3 * kMaxMStages;
  s.accempty = s.accfull + 2;
  s.tmem_base = reinterpret_cast<uint32_t*>(s.accempty + 2);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_base + 1);
  s.misc = s.abort_flag + 1;
  s.qmax = reinterpret_cast<float*>(s.misc + 8);
  s.qtab = s.qmax + 64;
  s.cpm = s.qtab + 2 * kMaxN;   // ends below 3.7 KB of the 3.75 KB region
  // without a raw ring its barriers serve the A tiles' transactions
  s.afull = s.rfull;
  // q8: the B ring's barriers, unused without a raw ring
  s.xring = s.stage + (size_t)s.nst * s.stage_bytes;
  s.xfull = s.rempty + kMaxMStages;
  s.xempty = s.xfull + kMaxMStages;
  s.drain = reinterpret_cast<uint64_t*>(s.misc + 4);
  return s;
}

// A role's wait on a pipeline barrier: true once the phase completed; false
// after an abort (another role gave up) or after the time limit (this one
// gives up: it raises the abort flag and records the error).  A phase that
// has already completed is taken without reading the flag.
KD_DEV bool mwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity)) return true;
  *abort_flag = 1;
  set_error(err, ERR_WAIT_MMA);
  return false;
}

// Same for waiters off the critical path (the epilogue): sleep between polls
// so that their spinning does not take issue slots from the producers.
KD_DEV bool mwait_lazy(uint64_t* bar, uint32_t parity, volatile int* abort_flag, unsigned* err) {
  if (*abort_flag) return false;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    __nanosleep(200);
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      set_error(err, ERR_WAIT_MMA);
      return false;
    }
  }
  return true;
}

// Plan interface (all methods KD_DEV const):
//   int num_tiles(); long long tile_start(int t); MUnit tile_unit(int t)   (see CtaUnits;
//   a chunk is 64 * nsub K elements, nsub = mma_nsub(max_n(), kTerms))
//   int max_n(); int nsub
//   const CUtensorMap* map(int id)
//   static constexpr int kTerms    bf16 terms of B (1; 2 = hi + lo; 3 = hi + mid + lo)
//   static constexpr int kGatherTerms  (optional, default kTerms) B terms gathered
//                                  from memory; FP8 plans' converter rewrites B
//   static constexpr bool kFp8     A arrives as e4m3 tiles; converter warps write
//                                  them as bf16 (exact) and B as kTerms bf16 terms
//                                  of (gathered sum) x a_scale
//   static constexpr int kATerms   bf16 terms of the converted A tile (1)
//   static constexpr bool kQ8      e4m3 A tiles into kind::f8f6f4 MMAs; B made in-kernel
//   static constexpr int kConv     q8: converter warps (<= kQ8Conv; the CTA has q8_threads(kConv))
//                                  from fp32 rows: int kVariants (1, or 2 for gate / up
//                                  scales), const float* x_row(m, j), const float*
//                                  g_row(m, j) (per-64 maxima), int kgroups(),
//                                  float w_scale_v(m, kc, variant); kTerms = kVariants *
//                                  kQTerms (B tiles per stage)
//   static constexpr bool kGmaxOut  also write the output's per-64 maxima for a q8
//                                  consumer: bool gmax_tile(m), gmax_store(m, group, j, v)
//   const uint8_t* b_base(const MUnit&, int h); int b_stride(const MUnit&) (bytes)
//   int b_rowidx(const MUnit&, int j)   token j's row of term h: base + rowidx * stride
//   bool paired()                  rows are (gate, up) pairs
//   float epilogue(const MUnit&, int row_in_tile, int j, float v)   returns the stored value
//   float epilogue2(const MUnit&, int pair_in_tile, int j, float g, float u)
//   float* ws(); unsigned* tile_cnt()            split-K partials / arrivals
//   bool wants_unit_done(); void unit_done(const MUnit&, MmaShared&)   epilogue warps only
//   void after_run(MmaShared&, uint8_t* smem)   all threads, after the pipeline

template <class Plan>
KD_DEV void mma_producer_a_bf16(const Plan& plan, MmaShared& sh, CtaUnits<Plan>& units,
                                unsigned* err);

// After an abort: wait (bounded, whatever the abort flag says) until the
// last `n` transactions issued on ring `bars` of `nslots` slots have landed,
// so that no TMA write is still in flight when the CTA leaves.
KD_DEV void drain_tx(uint64_t* bars, int nslots, uint32_t issued) {
  const uint32_t n = issued < (uint32_t)nslots ? issued : (uint32_t)nslots;
  for (uint32_t i = issued - n; i < issued; ++i) mbar_wait(&bars[i % nslots], (i / nslots) & 1u);
}

template <class Plan>
KD_DEV void mma_producer_a(const Plan& plan, MmaShared& sh, unsigned* err) {
  uint32_t it = 0;
  CtaUnits<Plan> units(plan);
  MUnit m;
  bool ok = true;
  if constexpr (Plan::kFp8) {
    // e4m3 tiles [128 rows x 128 K bytes] into the raw ring
    while (ok && units.next(m)) {
      const CUtensorMap* map = plan.map(m.map);
      for (int c = 0; c < m.nkc; ++c, ++it) {
        const int s = it % sh.nraw;
        const uint32_t ph = (it / sh.nraw) & 1u;
        if (!mwait(&sh.rempty[s], ph ^ 1u, sh.abort_flag, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&sh.rfull[s], kRawBytes);
        tma_load_2d(sh.raw + (size_t)s * kRawBytes, map, (m.kc0 + c) * 128, m.row, &sh.rfull[s]);
      }
    }
    if (*sh.abort_flag) drain_tx(sh.rfull, sh.nraw, it);
  } else if constexpr (Plan::kQ8) {
    // e4m3 tiles [128 rows x 128 K bytes] straight into the stage (one box)
    while (ok && units.next(m)) {
      const CUtensorMap* map = plan.map(m.map);
      for (int c = 0; c < m.nkc; ++c, ++it) {
        const int s = it % sh.nst;
        const uint32_t ph = (it / sh.nst) & 1u;
        if (!mwait(&sh.empty[s], ph ^ 1u, sh.abort_flag, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&sh.afull[s], kRawBytes);
        tma_load_2d(sh.stage + (size_t)s * sh.stage_bytes, map, (m.kc0 + c) * 128, m.row, &sh.afull[s]);
      }
    }
    if (*sh.abort_flag) drain_tx(sh.afull, sh.nst, it);
  } else {
    while (ok && units.next(m)) {
      const CUtensorMap* map = plan.map(m.map);
      for (int c = 0; c < m.nkc; ++c, ++it) {
        const int s = it % sh.nst;
        const uint32_t ph = (it / sh.nst) & 1u;
        if (!mwait(&sh.empty[s], ph ^ 1u, sh.abort_flag, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&sh.afull[s], sh.nsub * kATileBytes);
        for (int u = 0; u < sh.nsub; ++u)
          tma_load_2d(sh.stage + (size_t)s * sh.stage_bytes + u * kATileBytes, map,
                      ((m.kc0 + c) * sh.nsub + u) * 64, m.row, &sh.afull[s]);
      }
    }
    if (*sh.abort_flag) drain_tx(sh.afull, sh.nst, it);
  }
}

KD_DEV void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes) : "memory");
}
KD_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
KD_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival counts against the barrier's expected count).
KD_DEV void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// B terms a plan gathers from memory (kGatherTerms, else all kTerms).
template <class P, class = void>
struct GatherTerms {
  static constexpr int value = P::kTerms;
};
template <class P>
struct GatherTerms<P, decltype((void)P::kGatherTerms)> {
  static constexpr int value = P::kGatherTerms;
};

// Two warps (64 threads) write the B tile of every stage with cp.async:
// token rows j < ntok (zero-filled up to N), 128 bytes (64 bf16 or 128 e4m3
// K values) each, 16-byte
// chunk c of row r at r*128 + ((c ^ (r & 7)) * 16) -- the 128-byte swizzle
// the A tile has.  Thread t copies chunk t % 8 of rows t / 8, t / 8 + 8, ...
// (so every row it copies has the same swizzle), for every bf16 term.  Each
// thread's copies of a stage arrive on the stage's full barrier when they
// land (no thread waits for them), so every stage of the ring can have
// gathers in flight; the MMA issuer fences the generic-proxy writes against
// the tensor core after its wait.
template <class Plan>
KD_DEV void mma_producer_b(const Plan& plan, MmaShared& sh, unsigned* err) {
  constexpr int nh = Plan::kTerms;
  constexpr int ng = GatherTerms<Plan>::value;   // terms copied (<= nh)
  constexpr int kRows = kMaxN / 8;          // rows per thread (at most)
  const int t = threadIdx.x - 64;           // 0..63
  const int ch = t & 7, rg = t >> 3;
  const uint32_t swz = (uint32_t)((ch ^ rg) * 16);
  uint32_t it = 0;
  CtaUnits<Plan> units(plan);
  MUnit m;
  while (units.next(m)) {
    const int N = pad16(m.ntok);
    const int nr = N >> 3;
    const size_t stride = (size_t)plan.b_stride(m);   // bytes
    // this thread's sources for the whole unit (byte count 0 = zero fill,
    // ~0 = no row)
    const uint8_t* src[ng][kRows];
    uint32_t nb[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int r = rg + 8 * i;
      const bool live = i < nr && r < m.ntok;
      const size_t ro = live ? (size_t)plan.b_rowidx(m, r) * stride : 0;
#pragma unroll
      for (int h = 0; h < ng; ++h) src[h][i] = plan.b_base(m, h) + ro + ch * 16;
      nb[i] = i < nr ? (live ? 16u : 0u) : 0xFFFFFFFFu;
    }
    const int bsub = b_sub_bytes(N, nh);
    for (int c = 0; c < m.nkc; ++c, ++it) {
      const int s = it % sh.nbst;
      const uint32_t ph = (it / sh.nbst) & 1u;
      mwait(&sh.bempty[s], ph ^ 1u, sh.abort_flag, err);
      uint8_t* bt = sh.bst + (size_t)s * sh.bst_bytes + sh.boff + swz;
      for (int u = 0; u < sh.nsub; ++u) {
        const size_t kb = (size_t)((m.kc0 + c) * sh.nsub + u) * 128;   // bytes of K before it
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          if (nb[i] != 0xFFFFFFFFu) {
#pragma unroll
            for (int h = 0; h < ng; ++h)
              cp_async16(bt + u * bsub + h * N * 128 + (rg + 8 * i) * 128, src[h][i] + kb, nb[i]);
          }
        }
      }
      cp_async_arrive_noinc(&sh.bfull[s]);
    }
  }
  cp_async_commit();
  cp_async_wait<0>();   // nothing in flight when the warp leaves
}

// FP8 weights: warps 8-15 turn each e4m3 tile of the raw ring into the
// stage's bf16 A tile (two [128 x 64] sub-tiles in the 128-byte swizzle):
// bf16(decode(e4m3)), exact (every e4m3 value is a bf16 value).  The tile's
// block scale goes on B instead: once the stage's B rows have landed, the
// same warps replace them in place by the kTerms bf16 terms of (the sum of
// the gathered terms) x scale, so that each product is a weight times an
// activation term.  A: thread t takes the 16-byte chunks t, t + 256, ... of
// the 1024 in a tile (row = chunk / 8).  B: the 16-byte chunks of one term
// (the terms lie N rows apart, so a chunk's swizzled place is the same in
// every term), in turn.
template <class Plan>
KD_DEV void mma_converter(const Plan& plan, MmaShared& sh, unsigned* err) {
  constexpr int nh = Plan::kTerms, ng = GatherTerms<Plan>::value;
  static_assert(Plan::kATerms == 1 && !Plan::kQ8, "FP8 converter: one exact A term");
  const int ct = threadIdx.x - 256;
  uint32_t it = 0;
  CtaUnits<Plan> units(plan);
  MUnit m;
  while (units.next(m)) {
    const int N = pad16(m.ntok);
    const int bsub = b_sub_bytes(N, nh);
    const int nchunk = sh.nsub * N * 8;   // 16-byte chunks of one B term per stage
    for (int c = 0; c < m.nkc; ++c, ++it) {
      const int rs = it % sh.nraw, s = it % sh.nst, sb = it % sh.nbst;
      mwait(&sh.rfull[rs], (it / sh.nraw) & 1u, sh.abort_flag, err);
      mwait(&sh.empty[s], ((it / sh.nst) & 1u) ^ 1u, sh.abort_flag, err);
      const uint8_t* raw = sh.raw + (size_t)rs * kRawBytes;
      uint8_t* dst = sh.stage + (size_t)s * sh.stage_bytes;
#pragma unroll 4
      for (int q = 0; q < 4; ++q) {   // unrolled: independent chunks overlap their latencies
        const int p = ct + 256 * q;
        const int r = p >> 3, j = p & 7, sw = r & 7;
        const uint4 w = *reinterpret_cast<const uint4*>(raw + r * 128 + ((j ^ sw) << 4));
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t out[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float v0, v1, v2, v3;
          e4m3x4_to_f32(in[u], v0, v1, v2, v3);
          const __nv_bfloat162 h0 = __floats2bfloat162_rn(v0, v1), h1 = __floats2bfloat162_rn(v2, v3);
          out[2 * u] = *reinterpret_cast<const uint32_t*>(&h0);
          out[2 * u + 1] = *reinterpret_cast<const uint32_t*>(&h1);
        }
        // K bytes 16j .. 16j+15 -> bf16 sub-tile j/4, 16-byte chunks 2(j%4), 2(j%4)+1
        const int j0 = 2 * (j & 3);
        uint8_t* sub = dst + (j >> 2) * kATileBytes + r * 128;
        *reinterpret_cast<uint4*>(sub + ((j0 ^ sw) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
        *reinterpret_cast<uint4*>(sub + (((j0 + 1) ^ sw) << 4)) =
            make_uint4(out[4], out[5], out[6], out[7]);
      }
      // B: (gathered terms) x scale -> nh bf16 terms, in place
      mwait(&sh.bfull[sb], (it / sh.nbst) & 1u, sh.abort_flag, err);
      const float sc = plan.a_scale(m, m.kc0 + c).x;
      uint8_t* bt = sh.bst + (size_t)sb * sh.bst_bytes + sh.boff;
      for (int p = ct; p < nchunk; p += 256) {
        const int u = p / (N * 8);
        uint8_t* c0 = bt + u * bsub + (p - u * N * 8) * 16;
        float v[8];
#pragma unroll
        for (int h = 0; h < ng; ++h) {
          const uint4 t = *reinterpret_cast<const uint4*>(c0 + h * N * 128);
          const uint32_t tw[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(tw[i] << 16), hi = __uint_as_float(tw[i] & 0xFFFF0000u);
            v[2 * i] = h ? v[2 * i] + lo : lo;
            v[2 * i + 1] = h ? v[2 * i + 1] + hi : hi;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= sc;
#pragma unroll
        for (int h = 0; h < nh; ++h) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            o[i] = *reinterpret_cast<const uint32_t*>(&b2);
            v[2 * i] -= __low2float(b2);   // what this term leaves for the next
            v[2 * i + 1] -= __high2float(b2);
          }
          *reinterpret_cast<uint4*>(c0 + h * N * 128) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async_smem();   // generic-proxy writes -> visible to the tensor core
      named_bar_sync(3, 256);
      if (ct == 0) {
        mbar_arrive(&sh.rempty[rs]);
        mbar_arrive(&sh.full[s]);
      }
    }
  }
}

// After an abort: no MMA of the issuing thread may still be running when
// TMEM is freed: it commits them to the drain barrier and waits (bounded).
KD_DEV void drain_mma(MmaShared& sh) {
  if (!*sh.abort_flag) return;
  mma_commit(sh.drain);
  mbar_wait(sh.drain, 0);
}


template <class Plan>
KD_DEV void mma_issuer(const Plan& plan, MmaShared& sh, uint32_t tmem, unsigned* err) {
  constexpr int nterms = Plan::kTerms;
  uint32_t nu_local = 0;
  int s = 0, sb = 0;            // stage and B slot of the stage counter
  uint32_t ph = 0, bph = 0;     // and their phases (counters, no divisions)
  const uint32_t ring0 = smem_u32(sh.stage), bring0 = smem_u32(sh.bst) + sh.boff;
  CtaUnits<Plan> units(plan);
  MUnit m;
  for (; units.next(m); ++nu_local) {
    const int N = pad16(m.ntok);
    // one MMA per K-step for all B terms (their rows lie one after another:
    // N' = nterms N columns, summed by the epilogue)
    const uint32_t idesc_all = idesc_bf16(nterms * N);
    const int buf = nu_local & 1;
    const uint32_t d = tmem + (uint32_t)(buf * kBfAccCols);
    if (!mwait(&sh.accempty[buf], ((nu_local >> 1) & 1u) ^ 1u, sh.abort_flag, err)) break;
    tc_fence_after();
    bool ok = true;
    for (int c = 0; c < m.nkc; ++c) {
      if (Plan::kFp8) {
        ok = mwait(&sh.full[s], ph, sh.abort_flag, err) &&
             mwait(&sh.bfull[sb], bph, sh.abort_flag, err);
      } else {
        ok = mwait(&sh.afull[s], ph, sh.abort_flag, err) &&
             mwait(&sh.full[s], ph, sh.abort_flag, err);
      }
      if (!ok) break;
      fence_proxy_async_smem();   // the B gathers (generic proxy) -> tensor core reads
      tc_fence_after();
      const uint32_t a0 = ring0 + (uint32_t)(s * sh.stage_bytes);
      const uint32_t b0 = bring0 + (uint32_t)(sb * sh.bst_bytes);
      const int bsub = b_sub_bytes(N, nterms);
      if constexpr (!Plan::kFp8) {
        for (int u = 0; u < sh.nsub; ++u) {
          const uint32_t b = b0 + u * bsub;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16(d, sw128_desc(a0 + u * kATileBytes + k * 32), sw128_desc(b + k * 32), idesc_all,
                     c > 0 || u > 0 || k > 0);
        }
      } else {
      // FP8: the converted A tile (one exact term) against every B term in
      // one MMA per K-step, as for bf16 weights; descriptors by adding byte
      // offsets / 16 to the start-address field (shared addresses < 256 KB:
      // the field never carries)
      const uint64_t ad0 = sw128_desc(a0), bd0 = sw128_desc(b0);
      for (int u = 0; u < sh.nsub; ++u) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t bd = bd0 + (uint64_t)((u * bsub + k * 32) >> 4);
          const uint64_t ad = ad0 + (uint64_t)((u * kATileBytes + k * 32) >> 4);
          mma_bf16(d, ad, bd, idesc_all, c > 0 || u > 0 || k > 0);
        }
      }
      }
      mma_commit(&sh.empty[s]);   // the stage is free once these MMAs are done
      if (Plan::kFp8) mma_commit(&sh.bempty[sb]);
      if (++s == sh.nst) { s = 0; ph ^= 1u; }
      if (++sb == sh.nbst) { sb = 0; bph ^= 1u; }
    }
    if (!ok) break;
    mma_commit(&sh.accfull[buf]);
  }
  drain_mma(sh);
}

// q8 plans: per stage (one e4m3 weight tile [128 x 128 K] and a B tile of
// NV x kQTerms x N rows: every (variant, term, token)), four K-steps of 32,
// one MMA each (N = NV kQTerms pad16(ntok) columns); the accumulator lives in
// TMEM for the whole unit (two buffers, alternating between units, as for
// the bf16 plans) and the epilogue adds the term columns.
template <class Plan>
KD_DEV void mma_issuer_q8(const Plan& plan, MmaShared& sh, uint32_t tmem, unsigned* err) {
  constexpr int NV = Plan::kVariants, nh = Plan::kQT;
  uint32_t nu = 0, ph = 0;
  int s = 0;
  const uint32_t ring0 = smem_u32(sh.stage);
  CtaUnits<Plan> units(plan);
  MUnit m;
  for (; units.next(m); ++nu) {
    // one MMA per K-step covers every (token, variant, term) row of the B tile
    const uint32_t idesc = idesc_e4m3(pad16(NV * nh * m.ntok));
    const int buf = nu & 1;
    if (!mwait(&sh.accempty[buf], ((nu >> 1) & 1u) ^ 1u, sh.abort_flag, err)) break;
    tc_fence_after();
    const uint32_t d0 = tmem + (uint32_t)(buf * kQ8AccCols);
    bool ok = true;
    for (int c = 0; c < m.nkc; ++c) {
      ok = mwait(&sh.afull[s], ph, sh.abort_flag, err) &&
           mwait(&sh.full[s], ph, sh.abort_flag, err);
      if (!ok) break;
      // (the converter fenced its B writes against the async proxy before
      // its arrival)
      tc_fence_after();
      const uint32_t a0 = ring0 + (uint32_t)(s * sh.stage_bytes);
      // descriptors by adding byte offsets / 16 to the start-address field
      // (shared addresses < 256 KB: the field never carries)
      const uint64_t ad0 = sw128_desc(a0), bd0 = sw128_desc(a0 + sh.boff);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t off = (uint64_t)((k * 32) >> 4);
        mma_e4m3(d0, ad0 + off, bd0 + off, idesc, c > 0 || k > 0);
      }
      mma_commit(&sh.empty[s]);   // the stage is free once these MMAs are done
      if (++s == sh.nst) { s = 0; ph ^= 1u; }
    }
    if (!ok) break;
    mma_commit(&sh.accfull[buf]);
  }
  drain_mma(sh);
}

// 2^P for token j of a q8 unit and scale variant v (and 2^-P in inv): the
// largest |activation| x weight block scale over the tile's K, from the
// activation's per-64-element maxima, put in [128, 256).
template <class Plan>
KD_DEV float q8_unit_scale(const Plan& plan, const MUnit& m, int j, int v, float& inv) {
  const float* g = plan.g_row(m, j);
  float amax = 0.f;
  const int ng = plan.kgroups();
  for (int q = 0; q < ng; ++q) amax = fmaxf(amax, __ldg(g + q) * plan.w_scale_v(m, q >> 1, v));
  return q_scale(amax, inv);
}

// q8 B producers.  Warp 2 (copier) copies, for every stage, the live token
// rows' fp32 activations of the stage's 128-K chunk with cp.async into a slot
// of the activation ring; each lane's copies arrive on the slot's xfull
// barrier when they land.  The slots are refilled as soon as a converter has
// read them, so the copies run ahead of the weight stages and their latency
// stays off the MMAs' path.  The converter warps (kQ8Conv of them, alternate
// stages) wait for a stage's rows and for its B tile to be free (the MMAs of
// its previous use done), write x times (block scale x 2^P) as kQTerms e4m3
// terms per scale variant, in the 128-byte swizzle, release the slot, and
// arrive on the stage's full barrier.  Rows past ntok are left as they are:
// their MMA columns are not read.
//
// One stage by one converter warp: (row, 8-element piece) pairs p = lane +
// 32 u, row p / 16, piece p % 16 (K elements 8 (p % 16) ..), so that every
// lane has work from two tokens up; pm = the warp's 2^P table of the unit.
template <class Plan>
KD_DEV void q8_convert_stage(const Plan& plan, MmaShared& sh, const MUnit& m, int c, int s,
                             int xsl, const float* pm) {
  constexpr int NV = Plan::kVariants, nh = Plan::kQT, C = NV * nh;
  const int lane = threadIdx.x & 31;
  uint8_t* bt = sh.stage + (size_t)s * sh.stage_bytes + sh.boff;
  const uint8_t* xs = sh.xring + (size_t)xsl * sh.xslot;
  const int kc = m.kc0 + c;
  float ws[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) ws[v] = plan.w_scale_v(m, kc, v);
  const int np = m.ntok * 16;
#pragma unroll 1
  for (int p = lane; p < np; p += 32) {
    const int r = p >> 4, pc = p & 15;
    float x[8];
    {
      const float4* src = reinterpret_cast<const float4*>(xs + (size_t)r * 512 + pc * 32);
      const float4 f0 = src[0], f1 = src[1];
      x[0] = f0.x; x[1] = f0.y; x[2] = f0.z; x[3] = f0.w;
      x[4] = f1.x; x[5] = f1.y; x[6] = f1.z; x[7] = f1.w;
    }
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const float f = ws[v] * pm[v * kMaxN + r];
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = x[e] * f;
#pragma unroll
      for (int h = 0; h < nh; ++h) {
        uint32_t pk[2];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t c2 = e4m3x2_rn(w[2 * e], w[2 * e + 1]);
          if (e & 1) pk[e >> 1] |= c2 << 16;
          else pk[e >> 1] = c2;
          if (h + 1 < nh) {
            const float2 tv = e4m3x2_value(c2);
            w[2 * e] -= tv.x;       // exact: within a factor of two of w (or w)
            w[2 * e + 1] -= tv.y;
          }
        }
        // B row b, 16-byte chunk pc / 2 (swizzled), this piece its half pc % 2
        const int b = r * C + v * nh + h;
        const uint32_t off = (uint32_t)((((pc >> 1) ^ (b & 7)) << 4) | ((pc & 1) << 3));
        *reinterpret_cast<uint2*>(bt + (size_t)b * 128 + off) = make_uint2(pk[0], pk[1]);
      }
    }
  }
  mbar_arrive(&sh.xempty[xsl]);   // the rows are read: the copier may refill the slot
  fence_proxy_async_smem();       // generic-proxy writes -> visible to the tensor core
  mbar_arrive(&sh.full[s]);
}

// Warp 2: the copies (no waiting for them to land).
template <class Plan>
KD_DEV void mma_copier_q8(const Plan& plan, MmaShared& sh, unsigned* err) {
  const int lane = threadIdx.x & 31;
  int xsl = 0;         // slot of the stage counter
  uint32_t xph = 0;    // and its phase
  CtaUnits<Plan> units(plan);
  MUnit m;
  while (units.next(m)) {
    // the unit's row sources (lane j: rows j and j + 32), resolved once per
    // unit and handed out per stage by shuffles
    const unsigned long long r0 =
        lane < m.ntok ? reinterpret_cast<unsigned long long>(plan.x_row(m, lane)) : 0ull;
    const unsigned long long r1 =
        lane + 32 < m.ntok ? reinterpret_cast<unsigned long long>(plan.x_row(m, lane + 32)) : 0ull;
    for (int c = 0; c < m.nkc; ++c) {
      mwait(&sh.xempty[xsl], xph ^ 1u, sh.abort_flag, err);
      uint8_t* xs = sh.xring + (size_t)xsl * sh.xslot;
      const size_t ko = (size_t)(m.kc0 + c) * 512 + lane * 16;
      // no new copies after an abort (one read of the flag for the warp)
      const int nr = __shfl_sync(0xffffffffu, *sh.abort_flag ? 0 : m.ntok, 0);
      for (int r = 0; r < nr; ++r) {   // lane = 16-byte piece of the 512-byte row
        const unsigned long long src = __shfl_sync(0xffffffffu, r < 32 ? r0 : r1, r & 31);
        cp_async16(xs + (size_t)r * 512 + lane * 16, reinterpret_cast<const uint8_t*>(src) + ko, 16u);
      }
      cp_async_arrive_noinc(&sh.xfull[xsl]);
      if (++xsl == sh.nxs) { xsl = 0; xph ^= 1u; }
    }
  }
  cp_async_commit();
  cp_async_wait<0>();   // nothing in flight when the warp leaves
}

// Converter warp cw (warp 3, then warps 8 ..), one of nconv: per unit, the
// 2^P table of its tokens (each token's largest |x| x block scale over the
// tile's groups, put in [128, 256) by q_scale) in a table of its own; then,
// for each stage of the unit that is its own (stage counter mod nconv), wait
// for the rows and for the stage's B tile, convert, release.  The lanes split
// the groups; the block scales are loaded once, and 8 rows' loads are all
// issued before their reductions.
template <class Plan>
KD_DEV void mma_converter_q8(const Plan& plan, MmaShared& sh, int cw, unsigned* err) {
  constexpr int NV = Plan::kVariants;
  const int lane = threadIdx.x & 31;
  if (cw >= sh.nconv) return;
  float* pm = sh.cpm + cw * 2 * kMaxN;
  int own = 0, s = 0, xsl = 0;   // the stage counter's owner, stage, slot
  uint32_t sph = 0, xph = 0;     // and their phases
  CtaUnits<Plan> units(plan);
  MUnit m;
  while (units.next(m)) {
    __syncwarp();   // the previous unit's conversions are done with the table
    {
      constexpr int kG = 4;   // groups per lane (<= 128 groups: K <= 8192)
      const int ng = plan.kgroups();
      float wv[kG][NV];
#pragma unroll
      for (int i = 0; i < kG; ++i) {
        const int q = lane + 32 * i;
#pragma unroll
        for (int v = 0; v < NV; ++v) wv[i][v] = q < ng ? plan.w_scale_v(m, q >> 1, v) : 0.f;
      }
#pragma unroll 1
      for (int r0 = 0; r0 < m.ntok; r0 += 8) {
        float lm[8][NV];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = r0 + rr;
          float g[kG];
          const float* gr = plan.g_row(m, r < m.ntok ? r : 0);
#pragma unroll
          for (int i = 0; i < kG; ++i) {
            const int q = lane + 32 * i;
            g[i] = (r < m.ntok && q < ng) ? __ldg(gr + q) : 0.f;
          }
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < kG; ++i) a = fmaxf(a, g[i] * wv[i][v]);
            lm[rr][v] = a;
          }
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
          for (int v = 0; v < NV; ++v) {
            float amax = lm[rr][v];
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            float inv;
            const float sc = q_scale(amax, inv);
            if (lane == rr && r0 + rr < m.ntok) pm[v * kMaxN + r0 + rr] = sc;
          }
      }
    }
    __syncwarp();
    // stage / slot indices and phases kept as counters (no divisions)
    for (int c = 0; c < m.nkc; ++c) {
      if (own == cw) {
        mwait(&sh.xfull[xsl], xph, sh.abort_flag, err);
        mwait(&sh.empty[s], sph ^ 1u, sh.abort_flag, err);
        q8_convert_stage(plan, sh, m, c, s, xsl, pm);
      }
      if (++own == sh.nconv) own = 0;
      if (++s == sh.nst) { s = 0; sph ^= 1u; }
      if (++xsl == sh.nxs) { xsl = 0; xph ^= 1u; }
    }
  }
}

// Per-64-element maxima of the output for a q8 consumer: this thread's 16
// outputs o (tokens c .. c+15 of its row; with paired rows only the even
// lanes hold one) -> max |o| per (token, group of kQGroup outputs): a group
// is 64 rows (two epilogue warps) of an unpaired tile, or the 64 outputs of
// a paired one (all four).  All four epilogue warps call.
template <class Plan>
KD_DEV void groupmax16(const Plan& plan, const MUnit& m, int lane, int c, const float* o,
                       MmaShared& sh) {
  const int ew = (threadIdx.x >> 5) - 4;
  const bool paired = plan.paired();
  const bool valid = !paired || !(lane & 1);
  float mx[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) mx[j] = (valid && c + j < m.ntok) ? fabsf(o[j]) : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int j = 0; j < 16; ++j) mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], off));
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < 16; ++j) sh.qmax[ew * 16 + j] = mx[j];
  }
  named_bar_sync(2, 128);
  const int g = paired ? 0 : (ew >> 1);
  if (lane < 16 && (paired ? ew == 0 : (ew & 1) == 0) && c + lane < m.ntok) {
    const float* q = sh.qmax + lane;
    const float v = paired ? fmaxf(fmaxf(q[0], q[16]), fmaxf(q[32], q[48]))
                           : fmaxf(q[(2 * g) * 16], q[(2 * g + 1) * 16]);
    plan.gmax_store(m, g, c + lane, v);
  }
  named_bar_sync(2, 128);   // qmax is rewritten by the next chunk
}

// The plan's epilogue for 16 accumulator columns (tokens c .. c+15) of this
// thread's row, then (plans with kGmaxOut) the output's per-64 maxima.
// Plans whose epilogue reads an input per output (a residual) provide
// epilogue_in(m, row, j), and emit16 loads the 16 tokens' inputs before the
// first store (the loads could not move above stores to memory that may alias).
template <class P, class = void>
struct HasEpilogueIn {
  static constexpr bool value = false;
};
template <class P>
struct HasEpilogueIn<P, decltype((void)&P::epilogue_in)> {
  static constexpr bool value = true;
};

template <class Plan>
KD_DEV void emit16(const Plan& plan, const MUnit& m, int row, int lane, int c, const float* v,
                   MmaShared& sh) {
  float o[16];
  if (plan.paired()) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
      o[j] = 0.f;
      if (!(lane & 1) && c + j < m.ntok) o[j] = plan.epilogue2(m, row >> 1, c + j, v[j], other);
    }
  } else if constexpr (HasEpilogueIn<Plan>::value) {
    decltype(plan.epilogue_in(m, row, 0)) in[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) in[j] = c + j < m.ntok ? plan.epilogue_in(m, row, c + j) : 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j] = 0.f;
      if (c + j < m.ntok) o[j] = plan.epilogue(m, row, c + j, v[j], in[j]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j] = 0.f;
      if (c + j < m.ntok) o[j] = plan.epilogue(m, row, c + j, v[j]);
    }
  }
  if constexpr (Plan::kGmaxOut) {
    if (plan.gmax_tile(m)) groupmax16(plan, m, lane, c, o, sh);
  }
}

// Epilogue warps (4..7).  Thread = accumulator lane = row of the tile.  The
// accumulator is read 16 columns at a time (a rolled loop: this code runs a
// few times per unit, so it is kept small for the instruction cache).
template <class Plan>
KD_DEV void mma_epilogue(const Plan& plan, MmaShared& sh, uint32_t tmem, unsigned* err) {
  const int ew = (threadIdx.x >> 5) - 4, lane = threadIdx.x & 31;
  const int row = ew * 32 + lane;
  uint32_t nu_local = 0;
  CtaUnits<Plan> units(plan);
  MUnit m;
  for (; units.next(m); ++nu_local) {
    const int N = pad16(m.ntok);
    const int buf = nu_local & 1;
    mwait_lazy(&sh.accfull[buf], (nu_local >> 1) & 1u, sh.abort_flag, err);
    tc_fence_after();
    const uint32_t ta = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(buf * kBfAccCols);
    // 16 tokens of the accumulator: the sum of the B terms' column blocks
    auto acc16 = [&](int c, float* v) {
      constexpr int NT = Plan::kTerms;
      float t[NT][16];
#pragma unroll
      for (int h = 0; h < NT; ++h) tmem_ld16(ta + (uint32_t)(h * N + c), t[h]);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float a = t[0][j];
#pragma unroll
        for (int h = 1; h < NT; ++h) a += t[h][j];
        v[j] = a;
      }
    };
    bool complete = true;
    int first = 0;
    if (m.nparts > 1) {
      // split-K: park this part, the last part to arrive sums them in order.
      // A slot is [token][row], so that a warp's 32 rows are one 128-byte line.
      const int slot = m.part == 0 ? 1 : 0;
      float* ws = plan.ws() + (size_t)blockIdx.x * kWsFloatsPerCta +
                  (size_t)slot * 128 * kMaxN + row;
#pragma unroll 1
      for (int c = 0; c < N; c += 16) {
        float v[16];
        acc16(c, v);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (c + j < m.ntok) __stcg(ws + (c + j) * 128, v[j]);
      }
      __threadfence();
      named_bar_sync(2, 128);
      if (threadIdx.x == 128) {
        const unsigned prev = atomicAdd(plan.tile_cnt() + m.tile, 1u);
        const bool last = prev == (unsigned)(m.nparts - 1);
        if (last) plan.tile_cnt()[m.tile] = 0u;  // every part is in: ready for reuse
        sh.misc[0] = last;
      }
      named_bar_sync(2, 128);
      complete = sh.misc[0] != 0;
      first = (int)blockIdx.x - m.part;
      if (complete) __threadfence();
    }
    if (complete) {
#pragma unroll 1
      for (int c = 0; c < N; c += 16) {
        float v[16];
        if (m.nparts > 1) {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.f;
          // parts added in part order; four parts' loads in flight at a time
#pragma unroll 1
          for (int p = 0; p < m.nparts; p += 4) {
            float t[4][16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float* src = plan.ws() + (size_t)(first + p + q) * kWsFloatsPerCta +
                                 (size_t)(p + q == 0 ? 1 : 0) * 128 * kMaxN + row + c * 128;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                t[q][j] = (p + q < m.nparts && c + j < m.ntok) ? __ldcg(src + j * 128) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (p + q < m.nparts) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] += t[q][j];
              }
          }
        } else {
          acc16(c, v);
        }
        emit16(plan, m, row, lane, c, v, sh);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.accempty[buf]);
    if (complete && plan.wants_unit_done()) {
      named_bar_sync(2, 128);
      plan.unit_done(m, sh);
    }
  }
}


// q8 epilogue warps (4..7): as mma_epilogue, with the accumulator of this
// thread's variant (gate for even rows, up for odd rows of a paired tile)
// times the token's 2^-P (a per-unit table in shared memory).
template <class Plan>
KD_DEV void mma_epilogue_q8(const Plan& plan, MmaShared& sh, uint32_t tmem, unsigned* err) {
  constexpr int NV = Plan::kVariants;
  const int ew = (threadIdx.x >> 5) - 4, lane = threadIdx.x & 31;
  const int row = ew * 32 + lane, et = threadIdx.x - 128;
  const int myv = NV == 2 ? (row & 1) : 0;
  uint32_t nu_local = 0;
  CtaUnits<Plan> units(plan);
  MUnit m;
  for (; units.next(m); ++nu_local) {
    const int N = pad16(m.ntok);
    const int NC = pad16(NV * Plan::kQT * m.ntok);   // accumulator columns
    const int buf = nu_local & 1;
    // the unit's 2^-P per (variant, token), shared by the four warps
    named_bar_sync(2, 128);   // every warp is done with the previous unit's table
    {
      const int j = et & 63, v = et >> 6;
      if (j < m.ntok && v < NV) {
        float inv;
        q8_unit_scale(plan, m, j, v, inv);
        sh.qtab[v * 64 + j] = inv;
      }
    }
    named_bar_sync(2, 128);
    mwait_lazy(&sh.accfull[buf], (nu_local >> 1) & 1u, sh.abort_flag, err);
    tc_fence_after();
    const uint32_t ta = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(buf * kQ8AccCols);
    const float* qt = sh.qtab + myv * 64;
    // 16 tokens c .. c+15 of this thread's variant: the sum of its term
    // columns (token j's C columns start at j C), scaled.  C loads of 16
    // columns; every lane loads every column (tcgen05.ld is warp-wide).
    auto load16 = [&](int c, float* out) {
      constexpr int C = NV * Plan::kQT, TPL = 16 / C;   // tokens per 16-column load
      float d[C][16];
#pragma unroll
      for (int q = 0; q < C; ++q) {
        if ((c + q * TPL) * C < NC) {
          tmem_ld16(ta + (uint32_t)((c * C) + 16 * q), d[q]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) d[q][i] = 0.f;   // tokens past ntok
        }
      }
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int q = j / TPL, base = (j % TPL) * C;
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < NV; ++v)
          if (v == myv) {
#pragma unroll
            for (int h = 0; h < Plan::kQT; ++h) acc += d[q][base + v * Plan::kQT + h];
          }
        out[j] = acc * qt[c + j];
      }
    };
    bool complete = true;
    int first = 0;
    if (m.nparts > 1) {
      const int slot = m.part == 0 ? 1 : 0;
      float* ws = plan.ws() + (size_t)blockIdx.x * kWsFloatsPerCta +
                  (size_t)slot * 128 * kMaxN + row;
#pragma unroll 1
      for (int c = 0; c < N; c += 16) {
        float v[16];
        load16(c, v);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (c + j < m.ntok) __stcg(ws + (c + j) * 128, v[j]);
      }
      __threadfence();
      named_bar_sync(2, 128);
      if (threadIdx.x == 128) {
        const unsigned prev = atomicAdd(plan.tile_cnt() + m.tile, 1u);
        const bool last = prev == (unsigned)(m.nparts - 1);
        if (last) plan.tile_cnt()[m.tile] = 0u;  // every part is in: ready for reuse
        sh.misc[0] = last;
      }
      named_bar_sync(2, 128);
      complete = sh.misc[0] != 0;
      first = (int)blockIdx.x - m.part;
      if (complete) __threadfence();
    }
    if (complete) {
#pragma unroll 1
      for (int c = 0; c < N; c += 16) {
        float v[16];
        if (m.nparts > 1) {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.f;
#pragma unroll 1
          for (int p = 0; p < m.nparts; p += 4) {
            float t[4][16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float* src = plan.ws() + (size_t)(first + p + q) * kWsFloatsPerCta +
                                 (size_t)(p + q == 0 ? 1 : 0) * 128 * kMaxN + row + c * 128;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                t[q][j] = (p + q < m.nparts && c + j < m.ntok) ? __ldcg(src + j * 128) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (p + q < m.nparts) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] += t[q][j];
              }
          }
        } else {
          load16(c, v);
        }
        emit16(plan, m, row, lane, c, v, sh);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.accempty[buf]);
  }
}

template <class Plan>
KD_DEV void mma_run(const Plan& plan, uint8_t* smem_raw, unsigned* err) {
  MmaShared sh = carve_mma_smem(smem_raw, plan.max_n(), Plan::kTerms, plan.nsub, Plan::kFp8,
                                Plan::kATerms, Plan::kQ8, Plan::kConv);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < sh.nst; ++i) {
      // the converter (FP8 projections), the 64 B threads (A: afull), or the
      // q8 converter warp (32)
      mbar_init(&sh.full[i], Plan::kFp8 ? 1 : (Plan::kQ8 ? 32 : 64));
      mbar_init(&sh.empty[i], 1);
      if (!Plan::kFp8) mbar_init(&sh.afull[i], 1);
    }
    for (int i = 0; i < sh.nxs; ++i) {
      mbar_init(&sh.xfull[i], 32);
      mbar_init(&sh.xempty[i], 32);
    }
    mbar_init(sh.drain, 1);
    if (Plan::kFp8) {
      for (int i = 0; i < sh.nbst; ++i) {
        mbar_init(&sh.bfull[i], 64);
        mbar_init(&sh.bempty[i], 1);
      }
    }
    for (int i = 0; i < sh.nraw; ++i) {
      mbar_init(&sh.rfull[i], 1);
      mbar_init(&sh.rempty[i], 1);
    }

    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.accfull[i], 1);
      mbar_init(&sh.accempty[i], 4);
    }
    *sh.abort_flag = 0;
    sh.misc[2] = 0;
    fence_mbar_init();
  }
  constexpr uint32_t kCols = Plan::kQ8 ? (uint32_t)kQ8TmemCols : (uint32_t)(2 * kBfAccCols);
  static_assert(!Plan::kQ8 || Plan::kVariants * kQTerms * kMaxN <= kQ8AccCols, "q8 accumulators");
  if (warp == 1) tmem_alloc(sh.tmem_base, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sh.tmem_base;
  // test hook: one wait that nothing completes (the drain barrier, which is
  // only ever committed after an abort); it gives up after the limit and
  // raises the abort flag, and the roles below stop at their first blocked wait
  if (plan.L->test_stall && threadIdx.x == 32) mwait(sh.drain, 0, sh.abort_flag, err);
  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) mma_producer_a(plan, sh, err);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) {
      if constexpr (Plan::kQ8) mma_issuer_q8(plan, sh, tmem, err);
      else mma_issuer(plan, sh, tmem, err);
    }
  } else if (warp < 4) {
    if constexpr (Plan::kQ8) {
      if (warp == 2) mma_copier_q8(plan, sh, err);
      else mma_converter_q8(plan, sh, 0, err);
    } else {
      mma_producer_b(plan, sh, err);
    }
  } else if (warp < 8) {
    if constexpr (Plan::kQ8) mma_epilogue_q8(plan, sh, tmem, err);
    else mma_epilogue(plan, sh, tmem, err);
  } else if constexpr (Plan::kFp8) {
    mma_converter(plan, sh, err);
  } else if constexpr (Plan::kQ8) {
    mma_converter_q8(plan, sh, warp - 7, err);   // warps 8 .. 8 + kConv - 2
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
  plan.after_run(sh, smem_raw);
}

}  // namespace kd

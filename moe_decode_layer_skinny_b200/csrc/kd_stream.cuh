// kd_stream.cuh -- weight-streaming GEMV engine on CUDA cores.
//
// One CTA of sixteen warps per SM.  Contiguous runs of weight rows stream from
// HBM into a ring of shared-memory stages with 1-D bulk TMA copies
// (cp.async.bulk, completion counted on one mbarrier per stage).  Each stage
// holds several whole rows; a warp owns one column slice of a subset of them,
// so the activation values it needs are the same for every row and stay in
// registers for a whole segment (up to 4 tokens), and the products use the
// packed fp32 FMA (two IEEE fp32 FMAs per instruction).  Per stage a warp
// writes one lane-reduced partial per (row, slice, token); after the CTA
// barrier that closes the stage the slices are added in a fixed order
// (deterministic) and handed to the plan's epilogue.  The same barrier frees the stage's slot and
// thread 0 immediately refills it with the stage kStages ahead, so there is no
// producer warp and no "empty" barrier.
//
// The work of a launch is a sequence of "segments" (a run of rows of one
// weight matrix against one token list) that the issuing thread and the
// consumers both enumerate from the same plan object.
#pragma once

#include "kd_common.cuh"

namespace kd {

constexpr int kCW = 16;                       // warps per CTA (max column slices per row)
constexpr int kThreads = kCW * 32;
constexpr int kIssuer = kThreads - 32;        // lane 0 of the last warp issues the bulk copies
constexpr int kStageBytes = 57344;            // 56 KB: 4 rows of 7168 bf16
constexpr int kStages = 3;
constexpr int kMaxRps = 64;                   // rows per stage cap
constexpr int kTT = 4;                        // tokens per register pass
constexpr int kPartCap = 8192;                // per-warp partial sums held until the epilogue
constexpr int kMaxChunksLane = 2;             // 16-byte chunks per lane per row slice
constexpr size_t kStreamSmem =
    (size_t)kStages * kStageBytes + kPartCap * sizeof(float) + 2 * kStages * 8 + 16 + 128;

enum WType { W_BF16 = 0, W_FP8 = 1 };
enum AType { A_BF16 = 0, A_F32 = 1 };

template <int WT>
struct WTraits {
  static constexpr int EPC = WT == W_BF16 ? 8 : 16;   // elements per 16-byte chunk
  static constexpr int TT = 2;                        // tokens held in registers at once
};

// One run of rows.  Rows are contiguous in memory (row stride = row_bytes).
struct Seg {
  const uint8_t* w;     // first row
  int row_bytes;        // bytes of one row (multiple of 256)
  int nrows;            // rows in the run (even for paired gate/up runs)
  int row0;             // index of the first row within its matrix (physical)
  int tok0, ntok;       // token list range (meaning is the plan's)
  int tag;              // plan-defined (expert id, matrix id ...)
};

struct StreamShared {
  uint8_t* stage;       // kStages * kStageBytes
  float* part;          // [kPartCap] partials [row][slice][token] since the last epilogue
  uint64_t* full;       // [kStages] stage landed (bulk-copy byte count)
  uint64_t* empty;      // [kStages] every warp finished reading the stage
  int* abort_flag;
};

KD_DEV StreamShared carve_stream_smem(uint8_t* base) {
  StreamShared s;
  uintptr_t p = (reinterpret_cast<uintptr_t>(base) + 127) & ~uintptr_t(127);
  s.stage = reinterpret_cast<uint8_t*>(p);
  p += (size_t)kStages * kStageBytes;
  s.part = reinterpret_cast<float*>(p);
  p += kPartCap * sizeof(float);
  s.full = reinterpret_cast<uint64_t*>(p);
  s.empty = s.full + kStages;
  s.abort_flag = reinterpret_cast<int*>(s.empty + kStages);
  return s;
}

// Bounded wait that gives up immediately once any thread of the CTA aborted.
KD_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                          unsigned* err, unsigned bit) {
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity)) return true;
  *abort_flag = 1;
  set_error(err, bit);
  return false;
}

// Rows per stage for a row of `row_bytes` (even when rows come in pairs).
KD_DEV int rows_per_stage(int row_bytes, bool paired) {
  int r = kStageBytes / row_bytes;
  if (r > kMaxRps) r = kMaxRps;
  if (paired) r &= ~1;
  return r;
}

// ---------------------------------------------------------------- issuer

// Thread 0's cursor over the stage sequence: (segment, first row) pairs in the
// order the consumers take them.
struct Issuer {
  int si = -1, nseg = 0, r = 0, rps = 1;
  uint32_t n = 0;       // stages issued so far
  Seg s;

  template <class Plan>
  KD_DEV void start(const Plan& plan) {
    nseg = plan.num_segments();
    si = -1;
    r = 0;
    s.nrows = 0;
  }

  // Issue the next stage into slot n % kStages; false when none is left.
  template <class Plan>
  KD_DEV bool next(const Plan& plan, StreamShared& sh) {
    while (r >= s.nrows) {
      if (++si >= nseg) return false;
      s = plan.segment(si);
      rps = rows_per_stage(s.row_bytes, plan.paired());
      r = 0;
    }
    const int rows = s.nrows - r < rps ? s.nrows - r : rps;
    const int slot = n % kStages;
    const uint32_t bytes = (uint32_t)rows * (uint32_t)s.row_bytes;
    mbar_arrive_expect_tx(&sh.full[slot], bytes);
    bulk_g2s(sh.stage + (size_t)slot * kStageBytes, s.w + (size_t)r * s.row_bytes, bytes,
             &sh.full[slot]);
    r += rps;
    ++n;
    return true;
  }
};

// ---------------------------------------------------------------- consumer
//
// Plan must provide:
//   int num_segments(), Seg segment(int)
//   const void* act_row(const Seg&, int j)        activation row of token j of the segment
//   const float* scale_row(const Seg&, int row)   FP8: scales of this physical row's block
//   bool paired()                                 rows come in (gate, up) pairs
//   void epilogue(const Seg&, int row, int j, float sum)            unpaired
//   void epilogue2(const Seg&, int pair_row, int j, float g, float u) paired
//   bool wants_segment_done(); void segment_done(const Seg&)
//                                                 called by all threads after a CTA
//                                                 barrier that follows a segment
//
// Geometry of a segment: each row is cut into S column slices (the smallest
// power of two that leaves <= 32*kMaxChunksLane 16-byte chunks per slice);
// warp w takes slice w % S of rows w / S, w / S + G, ... (G = 16 / S row
// groups).  A warp handles its rows four at a time and reduces the four
// partial sums across its lanes together (a transposing butterfly: 6 shuffles
// instead of 20).

KD_DEV int slices_per_row(int row_bytes) {
  const int chunks = row_bytes / 16;
  int S = 1;
  while (S < kCW && chunks / S > 32 * kMaxChunksLane) S *= 2;
  return S;
}

template <int WT>
using ActRegs = f32x2[WTraits<WT>::TT][kMaxChunksLane][WTraits<WT>::EPC / 2];

// Activation values of `nt` tokens at this lane's columns, into registers.
template <int WT, int AT, class Plan>
KD_DEV void load_act_regs(const Plan& plan, const Seg& s, int tok, int nt, int slice0, int cpl,
                          ActRegs<WT>& areg) {
  constexpr int EPC = WTraits<WT>::EPC;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < WTraits<WT>::TT; ++t) {
    const void* ar = plan.act_row(s, tok + (t < nt ? t : 0));
#pragma unroll
    for (int i = 0; i < kMaxChunksLane; ++i) {
      const int c = lane + 32 * i;
      if (t < nt && c < cpl) {
        const int col = (slice0 + c) * EPC;
#pragma unroll
        for (int q = 0; q < EPC / 8; ++q) {
          if constexpr (AT == A_BF16) {
            const uint4 v = ld_nc_v4(static_cast<const uint16_t*>(ar) + col + 8 * q);
            areg[t][i][4 * q + 0] = bf2_to_f2(v.x);
            areg[t][i][4 * q + 1] = bf2_to_f2(v.y);
            areg[t][i][4 * q + 2] = bf2_to_f2(v.z);
            areg[t][i][4 * q + 3] = bf2_to_f2(v.w);
          } else {
            const float* ap = static_cast<const float*>(ar) + col + 8 * q;
            const uint4 v0 = ld_nc_v4(ap), v1 = ld_nc_v4(ap + 4);
            areg[t][i][4 * q + 0] = pack2(__uint_as_float(v0.x), __uint_as_float(v0.y));
            areg[t][i][4 * q + 1] = pack2(__uint_as_float(v0.z), __uint_as_float(v0.w));
            areg[t][i][4 * q + 2] = pack2(__uint_as_float(v1.x), __uint_as_float(v1.y));
            areg[t][i][4 * q + 3] = pack2(__uint_as_float(v1.z), __uint_as_float(v1.w));
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < EPC / 2; ++e) areg[t][i][e] = 0ull;
      }
    }
  }
}

// Sum of four per-lane values over the warp, transposed: lane l receives the
// total of value (l >> 3) & 3.
KD_DEV float reduce4_transposed(float v0, float v1, float v2, float v3) {
  const int lane = threadIdx.x & 31;
  const bool b4 = lane & 16, b3 = lane & 8;
  float k0 = b4 ? v2 : v0, k1 = b4 ? v3 : v1;
  const float s0 = b4 ? v0 : v2, s1 = b4 ? v1 : v3;
  k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
  float k = b3 ? k1 : k0;
  const float sx = b3 ? k0 : k1;
  k += __shfl_xor_sync(0xffffffffu, sx, 8);
  k += __shfl_xor_sync(0xffffffffu, k, 4);
  k += __shfl_xor_sync(0xffffffffu, k, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

// Dot products of up to four rows (stage rows rows[j], -1 = none) with NT
// tokens over this lane's chunks, reduced over the warp: lane l returns the
// sums of row j = (l >> 3) & 3 in res[].
template <int WT, int NT, class Plan>
KD_DEV void batch_dot(const Plan& plan, const Seg& s, int stage_row0, const uint8_t* st,
                      const int (&rows)[4], int slice0, int cpl, const ActRegs<WT>& areg,
                      float (&res)[kTT]) {
  constexpr int EPC = WTraits<WT>::EPC;
  const int lane = threadIdx.x & 31;
  // one accumulator per (row, token); with a single token, one per (row,
  // chunk pair) so that 8 independent FMA chains are in flight
  constexpr int NA = NT == 1 ? 2 : 1;
  f32x2 acc[4][NT][NA];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int u = 0; u < NA; ++u) acc[j][t][u] = 0ull;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (rows[j] < 0) continue;
    const uint8_t* wrow = st + (size_t)rows[j] * s.row_bytes + (size_t)slice0 * 16;
    const float* srow = nullptr;
    if constexpr (WT == W_FP8) srow = plan.scale_row(s, s.row0 + stage_row0 + rows[j]);
#pragma unroll
    for (int i = 0; i < kMaxChunksLane; ++i) {
      const int c = lane + 32 * i;
      if (c < cpl) {
        const uint4 wv = lds_v4(wrow + (size_t)c * 16);
        if constexpr (WT == W_BF16) {
          const f32x2 w0 = bf2_to_f2(wv.x), w1 = bf2_to_f2(wv.y), w2 = bf2_to_f2(wv.z),
                      w3 = bf2_to_f2(wv.w);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            f32x2 a = acc[j][t][i % NA];
            a = ffma2(w0, areg[t][i][0], a);
            a = ffma2(w1, areg[t][i][1], a);
            a = ffma2(w2, areg[t][i][2], a);
            a = ffma2(w3, areg[t][i][3], a);
            acc[j][t][i % NA] = a;
          }
        } else {
          float w[16];
          e4m3x4_to_f32(wv.x, w[0], w[1], w[2], w[3]);
          e4m3x4_to_f32(wv.y, w[4], w[5], w[6], w[7]);
          e4m3x4_to_f32(wv.z, w[8], w[9], w[10], w[11]);
          e4m3x4_to_f32(wv.w, w[12], w[13], w[14], w[15]);
          const float sc = __ldg(srow + (((slice0 + c) * EPC) >> 7));
          const f32x2 sc2 = pack2(sc, sc);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            f32x2 p = 0ull;
#pragma unroll
            for (int e = 0; e < 8; ++e) p = ffma2(pack2(w[2 * e], w[2 * e + 1]), areg[t][i][e], p);
            acc[j][t][i % NA] = ffma2(p, sc2, acc[j][t][i % NA]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 p = unpack2(acc[j][t][0]);
      if (NA == 2) {
        const float2 q = unpack2(acc[j][t][NA - 1]);
        p.x += q.x;
        p.y += q.y;
      }
      v[j] = p.x + p.y;
    }
    res[t] = reduce4_transposed(v[0], v[1], v[2], v[3]);
  }
}

// Epilogue of `n` consecutive rows starting at segment row `row0`, whose lane-
// reduced partials are part[(row * S + slice) * ts + j] (rows relative to
// row0, ts >= nt the token stride): each sum adds its S slices in a fixed
// order (deterministic).
template <class Plan>
KD_DEV void reduce_epilogue(const Plan& plan, const Seg& s, const float* part, int row0, int n,
                            int S, int tok, int nt, int ts) {
  auto sum = [&](int row, int j) {
    const float* p = part + (size_t)row * S * ts + j;
    float v = 0.f;
    for (int sl = 0; sl < S; ++sl) v += p[sl * ts];
    return v;
  };
  if (plan.paired()) {
    const int npair = n >> 1;
    for (int q = threadIdx.x; q < npair * nt; q += kThreads) {
      const int p = nt == 1 ? q : q >> 1, j = nt == 1 ? 0 : q & 1;
      plan.epilogue2(s, (s.row0 + row0) / 2 + p, tok + j, sum(2 * p, j), sum(2 * p + 1, j));
    }
  } else {
    for (int q = threadIdx.x; q < n * nt; q += kThreads) {
      const int row = nt == 1 ? q : q >> 1, j = nt == 1 ? 0 : q & 1;
      plan.epilogue(s, s.row0 + row0 + row, tok + j, sum(row, j));
    }
  }
}

// A warp is done reading a stage: count it on the stage's "empty" barrier.
// The issuing lane waits for all warps and refills the slot at once, without
// waiting for the reductions and the epilogue of the stage.
template <class Plan>
KD_DEV void release_stage(const Plan& plan, StreamShared& sh, Issuer& iss, int slot, uint32_t ph,
                          unsigned* err) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sh.empty[slot]);
  if (threadIdx.x == kIssuer) {
    // after an abort no new copy is issued (the ones in flight are drained
    // before the CTA leaves)
    if (wait_or_abort(&sh.empty[slot], ph, sh.abort_flag, err, ERR_WAIT_EMPTY)) iss.next(plan, sh);
  }
  __syncwarp();  // the issuing lane rejoins its warp before any CTA barrier
}

// One segment.  Tokens are processed TT (= 2) at a time.  With at most TT
// tokens (the common case) their activations are loaded once for the whole
// segment and the warps run through the stages without any CTA barrier: each
// writes its lane-reduced partials into shared memory, and only when
// kPartCap is about to fill (or at the end of the segment) do all warps meet
// to reduce them and run the epilogue.  With more tokens the stage is swept
// once per group of TT tokens, reloading the activations (through L1) for
// every group, and each group is reduced at once.
template <int WT, int AT, class Plan>
KD_DEV void consume_segment(const Plan& plan, StreamShared& sh, Issuer& iss, const Seg& s,
                            uint32_t& it, unsigned* err) {
  constexpr int TT = WTraits<WT>::TT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rps = rows_per_stage(s.row_bytes, plan.paired());
  const int S = slices_per_row(s.row_bytes), G = kCW / S;
  const int cpl = (s.row_bytes / 16) / S;         // chunks per slice (<= 32*kMaxChunksLane)
  const int my_slice = warp % S, my_group = warp / S;
  const int slice0 = my_slice * cpl;
  ActRegs<WT> areg;
  const bool single_pass = s.ntok <= TT;
  const int ntp = single_pass ? (s.ntok > 0 ? s.ntok : 1) : TT;  // token stride of the partials
  if (single_pass) load_act_regs<WT, AT>(plan, s, 0, s.ntok, slice0, cpl, areg);
  int held0 = 0;  // first segment row whose partials wait in sh.part
  for (int r0 = 0; r0 < s.nrows; r0 += rps, ++it) {
    const int n = s.nrows - r0 < rps ? s.nrows - r0 : rps;
    const int slot = it % kStages;
    const uint32_t ph = (it / kStages) & 1u;
    wait_or_abort(&sh.full[slot], ph, sh.abort_flag, err, ERR_WAIT_FULL);
    const uint8_t* st = sh.stage + (size_t)slot * kStageBytes;
    if (!single_pass) held0 = r0;
    float* part = sh.part + (size_t)(r0 - held0) * S * ntp;
    for (int tok = 0; tok < s.ntok; tok += TT) {
      const int nt = s.ntok - tok < TT ? s.ntok - tok : TT;
      if (!single_pass) load_act_regs<WT, AT>(plan, s, tok, nt, slice0, cpl, areg);
      for (int rbase = my_group; rbase < n; rbase += 4 * G) {
        int rows[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) rows[j] = rbase + j * G < n ? rbase + j * G : -1;
        float res[kTT];
        if (nt == 1) batch_dot<WT, 1>(plan, s, r0, st, rows, slice0, cpl, areg, res);
        else batch_dot<WT, TT>(plan, s, r0, st, rows, slice0, cpl, areg, res);
        const int myrow = rbase + ((lane >> 3) & 3) * G;   // the row this lane's sums belong to
        if ((lane & 7) == 0 && myrow < n) {
#pragma unroll
          for (int t = 0; t < TT; ++t)
            if (t < nt) part[(myrow * S + my_slice) * ntp + t] = res[t];
        }
      }
      if (tok + TT >= s.ntok) release_stage(plan, sh, iss, slot, ph, err);
      if (!single_pass) {
        named_bar_sync(1, kThreads);
        reduce_epilogue(plan, s, sh.part, r0, n, S, tok, nt, ntp);
        named_bar_sync(1, kThreads);
      }
    }
    if (s.ntok == 0) release_stage(plan, sh, iss, slot, ph, err);
    if (single_pass && s.ntok > 0) {
      const bool last = r0 + rps >= s.nrows;
      if (last || (r0 + n + rps - held0) * S * ntp > kPartCap) {
        named_bar_sync(1, kThreads);
        reduce_epilogue(plan, s, sh.part, held0, r0 + n - held0, S, 0, s.ntok, ntp);
        named_bar_sync(1, kThreads);  // the partials buffer is reused from the start
        held0 = r0 + n;
      }
    }
  }
}

template <int WT, int AT, class Plan>
KD_DEV void stream_consume(const Plan& plan, StreamShared& sh, Issuer& iss, unsigned* err) {
  uint32_t it = 0;
  const int nseg = plan.num_segments();
  for (int si = 0; si < nseg; ++si) {
    const Seg s = plan.segment(si);
    consume_segment<WT, AT>(plan, sh, iss, s, it, err);
    if (plan.wants_segment_done()) {
      named_bar_sync(1, kThreads);  // every epilogue write of the segment is done
      plan.segment_done(s);
    }
  }
}

// Shared body of every streaming kernel.  With `weights_before_wait` the
// first kStages stages are requested before the programmatic-launch wait:
// only for plans whose segments are static weights known without reading
// anything a preceding kernel writes (activations are read after the wait).
template <int WT, int AT, class Plan>
KD_DEV void stream_run(const Plan& plan, uint8_t* smem_raw, unsigned* err,
                       bool weights_before_wait) {
  StreamShared sh = carve_stream_smem(smem_raw);
  Issuer iss;
  if (threadIdx.x == kIssuer) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], kCW);
    }
    *sh.abort_flag = 0;
    fence_mbar_init();
    if (weights_before_wait) {
      iss.start(plan);
      for (int i = 0; i < kStages; ++i)
        if (!iss.next(plan, sh)) break;
    }
  }
  if (weights_before_wait) {
    pdl_wait();
    pdl_launch_dependents();
  }
  if (threadIdx.x == kIssuer && !weights_before_wait) {
    iss.start(plan);
    for (int i = 0; i < kStages; ++i)
      if (!iss.next(plan, sh)) break;
  }
  __syncthreads();
  stream_consume<WT, AT>(plan, sh, iss, err);
  if (threadIdx.x == kIssuer && *sh.abort_flag) {
    // after an abort: the last stages' bulk copies land before the CTA leaves
    const uint32_t n = iss.n < (uint32_t)kStages ? iss.n : (uint32_t)kStages;
    for (uint32_t i = iss.n - n; i < iss.n; ++i) mbar_wait(&sh.full[i % kStages], (i / kStages) & 1u);
  }
}

}  // namespace kd

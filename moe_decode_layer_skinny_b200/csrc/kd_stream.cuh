// kd_stream.cuh -- weight-streaming GEMV engine on CUDA cores.
//
// One CTA of eight warps per SM.  Contiguous runs of weight rows stream from
// HBM into a ring of shared-memory stages with 1-D bulk TMA copies
// (cp.async.bulk, completion counted on one mbarrier per stage).  Each stage
// holds several whole rows; warp w owns the w-th eighth of the columns of
// every row, so the activation values it needs are the same for every row and
// stay in registers for a whole segment (up to 4 tokens).  Per stage a warp
// forms its partial dot products for all rows, reduces across lanes, and
// writes one partial per (row, token); after the CTA barrier that closes the
// stage the eight partials are added in a fixed order (deterministic) and
// handed to the plan's epilogue.  The same barrier frees the stage's slot and
// thread 0 immediately refills it with the stage kStages ahead, so there is no
// producer warp and no "empty" barrier.
//
// The work of a launch is a sequence of "segments" (a run of rows of one
// weight matrix against one token list) that the issuing thread and the
// consumers both enumerate from the same plan object.
#pragma once

#include "kd_common.cuh"

namespace kd {

constexpr int kCW = 8;                        // warps per CTA = column slices per row
constexpr int kThreads = kCW * 32;
constexpr int kStageBytes = 57344;            // 56 KB: 4 rows of 7168 bf16
constexpr int kStages = 3;
constexpr int kMaxRps = 64;                   // rows per stage cap
constexpr int kTT = 4;                        // tokens per register pass
constexpr int kRedFloats = kMaxRps * kCW * kTT;
constexpr int kMaxChunksLane = 4;             // 16-byte chunks per lane per row (K <= 8192 bf16)
constexpr size_t kStreamSmem =
    (size_t)kStages * kStageBytes + 2 * kRedFloats * sizeof(float) + kStages * 8 + 16 + 128;

enum WType { W_BF16 = 0, W_FP8 = 1 };
enum AType { A_BF16 = 0, A_F32 = 1 };

template <int WT>
struct WTraits {
  static constexpr int EPC = WT == W_BF16 ? 8 : 16;   // elements per 16-byte chunk
  static constexpr int TT = WT == W_BF16 ? 4 : 2;     // tokens held in registers at once
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
  float* red;           // [2][kRedFloats]
  uint64_t* full;       // [kStages] stage landed (bulk-copy byte count)
  int* abort_flag;
};

KD_DEV StreamShared carve_stream_smem(uint8_t* base) {
  StreamShared s;
  uintptr_t p = (reinterpret_cast<uintptr_t>(base) + 127) & ~uintptr_t(127);
  s.stage = reinterpret_cast<uint8_t*>(p);
  p += (size_t)kStages * kStageBytes;
  s.red = reinterpret_cast<float*>(p);
  p += 2 * kRedFloats * sizeof(float);
  s.full = reinterpret_cast<uint64_t*>(p);
  s.abort_flag = reinterpret_cast<int*>(s.full + kStages);
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

template <int WT>
using ActRegs = float[WTraits<WT>::TT][kMaxChunksLane][WTraits<WT>::EPC];

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
            areg[t][i][8 * q + 0] = bf_lo(v.x); areg[t][i][8 * q + 1] = bf_hi(v.x);
            areg[t][i][8 * q + 2] = bf_lo(v.y); areg[t][i][8 * q + 3] = bf_hi(v.y);
            areg[t][i][8 * q + 4] = bf_lo(v.z); areg[t][i][8 * q + 5] = bf_hi(v.z);
            areg[t][i][8 * q + 6] = bf_lo(v.w); areg[t][i][8 * q + 7] = bf_hi(v.w);
          } else {
            const float* ap = static_cast<const float*>(ar) + col + 8 * q;
            const uint4 v0 = ld_nc_v4(ap), v1 = ld_nc_v4(ap + 4);
            areg[t][i][8 * q + 0] = __uint_as_float(v0.x); areg[t][i][8 * q + 1] = __uint_as_float(v0.y);
            areg[t][i][8 * q + 2] = __uint_as_float(v0.z); areg[t][i][8 * q + 3] = __uint_as_float(v0.w);
            areg[t][i][8 * q + 4] = __uint_as_float(v1.x); areg[t][i][8 * q + 5] = __uint_as_float(v1.y);
            areg[t][i][8 * q + 6] = __uint_as_float(v1.z); areg[t][i][8 * q + 7] = __uint_as_float(v1.w);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < EPC; ++e) areg[t][i][e] = 0.f;
      }
    }
  }
}

// Partial dot products of one row slice (this lane's chunks) with NT tokens,
// reduced over the warp's lanes.  Independent accumulators per chunk and two
// interleaved FMA chains per chunk keep the FMA pipe busy.
template <int WT, int NT>
KD_DEV void row_dot(const uint8_t* wslice, const float (&sc)[kMaxChunksLane], int cpl,
                    const ActRegs<WT>& areg, float (&out)[kTT]) {
  const int lane = threadIdx.x & 31;
  float acc[kMaxChunksLane][NT];
#pragma unroll
  for (int i = 0; i < kMaxChunksLane; ++i)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[i][t] = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxChunksLane; ++i) {
    const int c = lane + 32 * i;
    if (c < cpl) {
      const uint4 wv = lds_v4(wslice + (size_t)c * 16);
      if constexpr (WT == W_BF16) {
        const float w[8] = {bf_lo(wv.x), bf_hi(wv.x), bf_lo(wv.y), bf_hi(wv.y),
                            bf_lo(wv.z), bf_hi(wv.z), bf_lo(wv.w), bf_hi(wv.w)};
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float a0 = w[0] * areg[t][i][0], a1 = w[1] * areg[t][i][1];
          a0 = fmaf(w[2], areg[t][i][2], a0); a1 = fmaf(w[3], areg[t][i][3], a1);
          a0 = fmaf(w[4], areg[t][i][4], a0); a1 = fmaf(w[5], areg[t][i][5], a1);
          a0 = fmaf(w[6], areg[t][i][6], a0); a1 = fmaf(w[7], areg[t][i][7], a1);
          acc[i][t] = a0 + a1;
        }
      } else {
        float w[16];
        e4m3x4_to_f32(wv.x, w[0], w[1], w[2], w[3]);
        e4m3x4_to_f32(wv.y, w[4], w[5], w[6], w[7]);
        e4m3x4_to_f32(wv.z, w[8], w[9], w[10], w[11]);
        e4m3x4_to_f32(wv.w, w[12], w[13], w[14], w[15]);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float a0 = w[0] * areg[t][i][0], a1 = w[1] * areg[t][i][1];
#pragma unroll
          for (int e = 2; e < 16; e += 2) {
            a0 = fmaf(w[e], areg[t][i][e], a0);
            a1 = fmaf(w[e + 1], areg[t][i][e + 1], a1);
          }
          acc[i][t] = (a0 + a1) * sc[i];
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float v = acc[0][t];
#pragma unroll
    for (int i = 1; i < kMaxChunksLane; ++i) v += acc[i][t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    out[t] = v;
  }
}

// After every warp wrote its partials of a stage into `red` ([row][slice][t]):
// sum the slices in a fixed order and run the epilogue.
template <class Plan>
KD_DEV void stage_epilogue(const Plan& plan, const Seg& s, const float* red, int n, int stage_row0,
                           int tok, int nt) {
  const int ctid = threadIdx.x;
  if (plan.paired()) {
    const int npair = n >> 1;
    for (int q = ctid; q < npair * nt; q += kThreads) {
      const int p = q / nt, j = q % nt;
      float g = 0.f, u = 0.f;
#pragma unroll
      for (int sl = 0; sl < kCW; ++sl) {
        g += red[((2 * p) * kCW + sl) * kTT + j];
        u += red[((2 * p + 1) * kCW + sl) * kTT + j];
      }
      plan.epilogue2(s, (s.row0 + stage_row0) / 2 + p, tok + j, g, u);
    }
  } else {
    for (int q = ctid; q < n * nt; q += kThreads) {
      const int row = q / nt, j = q % nt;
      float v = 0.f;
#pragma unroll
      for (int sl = 0; sl < kCW; ++sl) v += red[(row * kCW + sl) * kTT + j];
      plan.epilogue(s, s.row0 + stage_row0 + row, tok + j, v);
    }
  }
}

// One segment.  Tokens are processed TT at a time (4 for bf16 weights, 2 for
// FP8): with at most TT tokens (the common case) their activations are loaded
// once for the whole segment; with more, the stage is swept once per group of
// TT tokens, reloading the activations (through L1) for every group.
template <int WT, int AT, class Plan>
KD_DEV void consume_segment(const Plan& plan, StreamShared& sh, Issuer& iss, const Seg& s,
                            uint32_t& it, int& rb, unsigned* err) {
  constexpr int EPC = WTraits<WT>::EPC;
  constexpr int TT = WTraits<WT>::TT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rps = rows_per_stage(s.row_bytes, plan.paired());
  const int cpl = (s.row_bytes / 16) / kCW;       // chunks per slice (<= 32*kMaxChunksLane)
  const int slice0 = warp * cpl;
  ActRegs<WT> areg;
  const bool single_pass = s.ntok <= TT;
  if (single_pass) load_act_regs<WT, AT>(plan, s, 0, s.ntok, slice0, cpl, areg);
  for (int r0 = 0; r0 < s.nrows; r0 += rps, ++it) {
    const int n = s.nrows - r0 < rps ? s.nrows - r0 : rps;
    const int slot = it % kStages;
    const uint32_t ph = (it / kStages) & 1u;
    wait_or_abort(&sh.full[slot], ph, sh.abort_flag, err, ERR_WAIT_FULL);
    const uint8_t* st = sh.stage + (size_t)slot * kStageBytes + (size_t)slice0 * 16;
    for (int tok = 0; tok < s.ntok; tok += TT) {
      const int nt = s.ntok - tok < TT ? s.ntok - tok : TT;
      if (!single_pass) load_act_regs<WT, AT>(plan, s, tok, nt, slice0, cpl, areg);
      float* red = sh.red + rb * kRedFloats;
      for (int row = 0; row < n; ++row) {
        // FP8 block scales of this row at this lane's chunks (static weights)
        float sc[kMaxChunksLane];
#pragma unroll
        for (int i = 0; i < kMaxChunksLane; ++i) sc[i] = 1.f;
        if constexpr (WT == W_FP8) {
          const float* srow = plan.scale_row(s, s.row0 + r0 + row);
#pragma unroll
          for (int i = 0; i < kMaxChunksLane; ++i) {
            const int c = lane + 32 * i;
            sc[i] = c < cpl ? __ldg(srow + (((slice0 + c) * EPC) >> 7)) : 0.f;
          }
        }
        float part[kTT];
        const uint8_t* wrow = st + (size_t)row * s.row_bytes;
        if (nt == 1) row_dot<WT, 1>(wrow, sc, cpl, areg, part);
        else if (TT == 2 || nt == 2) row_dot<WT, 2>(wrow, sc, cpl, areg, part);
        else row_dot<WT, TT>(wrow, sc, cpl, areg, part);
        if (lane == 0) {
#pragma unroll
          for (int t = 0; t < kTT; ++t)
            if (t < nt) red[(row * kCW + warp) * kTT + t] = part[t];
        }
      }
      named_bar_sync(1, kThreads);
      // after the stage's last token group no thread reads it again: refill
      if (threadIdx.x == 0 && tok + TT >= s.ntok) iss.next(plan, sh);
      stage_epilogue(plan, s, red, n, r0, tok, nt);
      rb ^= 1;
    }
    if (s.ntok == 0) {
      named_bar_sync(1, kThreads);
      if (threadIdx.x == 0) iss.next(plan, sh);
    }
  }
}

template <int WT, int AT, class Plan>
KD_DEV void stream_consume(const Plan& plan, StreamShared& sh, Issuer& iss, unsigned* err) {
  uint32_t it = 0;
  int rb = 0;  // reduction buffer parity
  const int nseg = plan.num_segments();
  for (int si = 0; si < nseg; ++si) {
    const Seg s = plan.segment(si);
    consume_segment<WT, AT>(plan, sh, iss, s, it, rb, err);
  }
}

// Shared body of every streaming kernel.
template <int WT, int AT, class Plan>
KD_DEV void stream_run(const Plan& plan, uint8_t* smem_raw, unsigned* err) {
  StreamShared sh = carve_stream_smem(smem_raw);
  Issuer iss;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&sh.full[i], 1);
    *sh.abort_flag = 0;
    fence_mbar_init();
    iss.start(plan);
    for (int i = 0; i < kStages; ++i)
      if (!iss.next(plan, sh)) break;
  }
  __syncthreads();
  stream_consume<WT, AT>(plan, sh, iss, err);
}

}  // namespace kd

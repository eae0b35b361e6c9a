// kd_stream.cuh -- weight-streaming GEMV engine on CUDA cores.
//
// One CTA of eight warps per SM.  Contiguous runs of weight rows stream from
// HBM into a ring of shared-memory stages with 1-D bulk TMA copies
// (cp.async.bulk, completion counted on one mbarrier per stage).  All eight
// warps take each stage as it lands, form dot products of its rows with a few
// token activation rows (kept in registers when there are one or two), reduce
// across lanes and warps in a fixed order (deterministic), and hand each
// (row, token) sum to an epilogue.  The named barrier that closes a stage also
// frees its slot, and thread 0 immediately refills it with the stage
// kStages ahead, so no producer warp or "empty" barrier is needed and each
// thread can hold up to 255 registers.
//
// The work of a launch is a sequence of "segments" (a run of rows of one
// weight matrix against one token list) that the issuing thread and the
// consumers both enumerate from the same plan object.
#pragma once

#include "kd_common.cuh"

namespace kd {

constexpr int kCW = 8;                        // warps per CTA (all consume)
constexpr int kThreads = kCW * 32;
constexpr int kStageBytes = 32768;
constexpr int kStages = 6;
constexpr int kTokBlk = 16;                   // tokens reduced per pass over a stage
constexpr int kTT = 4;                        // tokens accumulated in registers at once
constexpr int kMaxRps = 64;                   // rows per stage cap
constexpr int kRedFloats = kMaxRps * kTokBlk; // rows x slices <= kMaxRps
constexpr size_t kStreamSmem =
    (size_t)kStages * kStageBytes + 2 * kRedFloats * sizeof(float) + kStages * 8 + 16 + 128;

enum WType { W_BF16 = 0, W_FP8 = 1 };
enum AType { A_BF16 = 0, A_F32 = 1 };

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

// rows per stage for a row of `row_bytes` (power of two, <= kMaxRps)
KD_DEV int rows_per_stage(int row_bytes) {
  int r = kStageBytes / row_bytes;
  int p = 1;
  while (p * 2 <= r && p * 2 <= kMaxRps) p *= 2;
  return p;
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
      rps = rows_per_stage(s.row_bytes);
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

// Accumulate dot products of weight chunk (16 bytes at `wp`) with tokens.
template <int WT, int AT>
KD_DEV void chunk_fma(const uint4 wv, float scale, const void* const* arow, int col, int nt,
                      float* acc) {
  if constexpr (WT == W_BF16) {
    float w[8] = {bf_lo(wv.x), bf_hi(wv.x), bf_lo(wv.y), bf_hi(wv.y),
                  bf_lo(wv.z), bf_hi(wv.z), bf_lo(wv.w), bf_hi(wv.w)};
#pragma unroll
    for (int t = 0; t < kTT; ++t) {
      if (t < nt) {
        float s = 0.f;
        if constexpr (AT == A_BF16) {
          uint4 a = ld_nc_v4(static_cast<const uint16_t*>(arow[t]) + col);
          s = fmaf(w[0], bf_lo(a.x), s); s = fmaf(w[1], bf_hi(a.x), s);
          s = fmaf(w[2], bf_lo(a.y), s); s = fmaf(w[3], bf_hi(a.y), s);
          s = fmaf(w[4], bf_lo(a.z), s); s = fmaf(w[5], bf_hi(a.z), s);
          s = fmaf(w[6], bf_lo(a.w), s); s = fmaf(w[7], bf_hi(a.w), s);
        } else {
          const float* ap = static_cast<const float*>(arow[t]) + col;
          uint4 a0 = ld_nc_v4(ap), a1 = ld_nc_v4(ap + 4);
          s = fmaf(w[0], __uint_as_float(a0.x), s); s = fmaf(w[1], __uint_as_float(a0.y), s);
          s = fmaf(w[2], __uint_as_float(a0.z), s); s = fmaf(w[3], __uint_as_float(a0.w), s);
          s = fmaf(w[4], __uint_as_float(a1.x), s); s = fmaf(w[5], __uint_as_float(a1.y), s);
          s = fmaf(w[6], __uint_as_float(a1.z), s); s = fmaf(w[7], __uint_as_float(a1.w), s);
        }
        acc[t] += s;
      }
    }
  } else {
    float w[16];
    e4m3x4_to_f32(wv.x, w[0], w[1], w[2], w[3]);
    e4m3x4_to_f32(wv.y, w[4], w[5], w[6], w[7]);
    e4m3x4_to_f32(wv.z, w[8], w[9], w[10], w[11]);
    e4m3x4_to_f32(wv.w, w[12], w[13], w[14], w[15]);
#pragma unroll
    for (int t = 0; t < kTT; ++t) {
      if (t < nt) {
        float s = 0.f;
        if constexpr (AT == A_BF16) {
          const uint16_t* ap = static_cast<const uint16_t*>(arow[t]) + col;
          uint4 a0 = ld_nc_v4(ap), a1 = ld_nc_v4(ap + 8);
          s = fmaf(w[0], bf_lo(a0.x), s); s = fmaf(w[1], bf_hi(a0.x), s);
          s = fmaf(w[2], bf_lo(a0.y), s); s = fmaf(w[3], bf_hi(a0.y), s);
          s = fmaf(w[4], bf_lo(a0.z), s); s = fmaf(w[5], bf_hi(a0.z), s);
          s = fmaf(w[6], bf_lo(a0.w), s); s = fmaf(w[7], bf_hi(a0.w), s);
          s = fmaf(w[8], bf_lo(a1.x), s); s = fmaf(w[9], bf_hi(a1.x), s);
          s = fmaf(w[10], bf_lo(a1.y), s); s = fmaf(w[11], bf_hi(a1.y), s);
          s = fmaf(w[12], bf_lo(a1.z), s); s = fmaf(w[13], bf_hi(a1.z), s);
          s = fmaf(w[14], bf_lo(a1.w), s); s = fmaf(w[15], bf_hi(a1.w), s);
        } else {
          const float* ap = static_cast<const float*>(arow[t]) + col;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 a = ld_nc_v4(ap + 4 * q);
            s = fmaf(w[4 * q + 0], __uint_as_float(a.x), s);
            s = fmaf(w[4 * q + 1], __uint_as_float(a.y), s);
            s = fmaf(w[4 * q + 2], __uint_as_float(a.z), s);
            s = fmaf(w[4 * q + 3], __uint_as_float(a.w), s);
          }
        }
        acc[t] = fmaf(s, scale, acc[t]);
      }
    }
  }
}

// Consumer side.  Plan must provide:
//   int num_segments(), Seg segment(int)
//   const void* act_row(const Seg&, int j)        activation row of token j of the segment
//   const float* scale_row(const Seg&, int row)   FP8: scales of this physical row's block
//   bool paired()                                 rows come in (gate, up) pairs
//   void epilogue(const Seg&, int row, int j, float sum)            unpaired
//   void epilogue2(const Seg&, int pair_row, int j, float g, float u) paired

// Geometry of one segment as seen by one consumer warp.
struct SegGeom {
  int rps;            // rows per stage
  int wpr;            // warps per row (= K slices)
  int rpw;            // rows per warp
  int chunks_slice;   // 16-byte chunks of one row slice
  int my_slice, my_row0;
};

KD_DEV SegGeom seg_geom(int row_bytes, int warp) {
  SegGeom g;
  g.rps = rows_per_stage(row_bytes);
  g.wpr = g.rps >= kCW ? 1 : kCW / g.rps;
  g.rpw = g.rps >= kCW ? g.rps / kCW : 1;
  g.chunks_slice = (row_bytes / 16) / g.wpr;
  g.my_slice = warp % g.wpr;
  g.my_row0 = (warp / g.wpr) * g.rpw;
  return g;
}

// After every warp wrote its partial sums of a stage into `red`: sum the
// slices in a fixed order and run the epilogue.
template <class Plan>
KD_DEV void stage_epilogue(const Plan& plan, const Seg& s, const float* red, int n, int slices,
                           int stage_row0, int tb, int ntb) {
  const int ctid = threadIdx.x;
  if (plan.paired()) {
    const int npair = n >> 1;
    for (int q = ctid; q < npair * ntb; q += kCW * 32) {
      const int p = q / ntb, j = q % ntb;
      float g = 0.f, u = 0.f;
      for (int sl = 0; sl < slices; ++sl) {
        g += red[((2 * p) * slices + sl) * kTokBlk + j];
        u += red[((2 * p + 1) * slices + sl) * kTokBlk + j];
      }
      plan.epilogue2(s, (s.row0 + stage_row0) / 2 + p, tb + j, g, u);
    }
  } else {
    for (int q = ctid; q < n * ntb; q += kCW * 32) {
      const int row = q / ntb, j = q % ntb;
      float v = 0.f;
      for (int sl = 0; sl < slices; ++sl) v += red[(row * slices + sl) * kTokBlk + j];
      plan.epilogue(s, s.row0 + stage_row0 + row, tb + j, v);
    }
  }
}

constexpr int kMaxChunksLane = 8;   // 16-byte chunks per lane per row slice (K <= 8192 bf16)

// Register path: the segment's T (<= 2) activation rows, restricted to this
// lane's columns, live in registers for the whole segment; each stage costs
// one 16-byte shared load per chunk and T x 8 (or 16) FMAs.
template <int WT, int AT, int T, class Plan>
KD_DEV void consume_segment_reg(const Plan& plan, StreamShared& sh, Issuer& iss, const Seg& s,
                                uint32_t& it, int& rb, unsigned* err) {
  constexpr int EPC = WT == W_BF16 ? 8 : 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SegGeom g = seg_geom(s.row_bytes, warp);
  float areg[T][kMaxChunksLane][EPC];
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const void* ar = plan.act_row(s, t);
#pragma unroll
    for (int i = 0; i < kMaxChunksLane; ++i) {
      const int c = lane + 32 * i;
      if (c < g.chunks_slice) {
        const int col = (g.my_slice * g.chunks_slice + c) * EPC;
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
  for (int r0 = 0; r0 < s.nrows; r0 += g.rps, ++it) {
    const int n = s.nrows - r0 < g.rps ? s.nrows - r0 : g.rps;
    const int slot = it % kStages;
    const uint32_t ph = (it / kStages) & 1u;
    // FP8 block scales of this warp's rows: static weights, so they may be
    // read before the stage's wait.
    float sc[2][kMaxChunksLane];
    if constexpr (WT == W_FP8) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int row = g.my_row0 + rr;
        const float* srow = (rr < g.rpw && row < n) ? plan.scale_row(s, s.row0 + r0 + row) : nullptr;
#pragma unroll
        for (int i = 0; i < kMaxChunksLane; ++i) {
          const int c = lane + 32 * i;
          sc[rr][i] = (srow && c < g.chunks_slice) ? __ldg(srow + (((g.my_slice * g.chunks_slice + c) * EPC) >> 7)) : 0.f;
        }
      }
    }
    wait_or_abort(&sh.full[slot], ph, sh.abort_flag, err, ERR_WAIT_FULL);
    const uint8_t* st = sh.stage + (size_t)slot * kStageBytes;
    float* red = sh.red + rb * kRedFloats;
    for (int rr = 0; rr < g.rpw; ++rr) {
      const int row = g.my_row0 + rr;
      if (row >= n) break;
      const uint8_t* wrow = st + (size_t)row * s.row_bytes + (size_t)g.my_slice * g.chunks_slice * 16;
      float acc[T];
#pragma unroll
      for (int t = 0; t < T; ++t) acc[t] = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxChunksLane; ++i) {
        const int c = lane + 32 * i;
        if (c < g.chunks_slice) {
          const uint4 wv = lds_v4(wrow + (size_t)c * 16);
          if constexpr (WT == W_BF16) {
            const float w[8] = {bf_lo(wv.x), bf_hi(wv.x), bf_lo(wv.y), bf_hi(wv.y),
                                bf_lo(wv.z), bf_hi(wv.z), bf_lo(wv.w), bf_hi(wv.w)};
#pragma unroll
            for (int t = 0; t < T; ++t)
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[t] = fmaf(w[e], areg[t][i][e], acc[t]);
          } else {
            float w[16];
            e4m3x4_to_f32(wv.x, w[0], w[1], w[2], w[3]);
            e4m3x4_to_f32(wv.y, w[4], w[5], w[6], w[7]);
            e4m3x4_to_f32(wv.z, w[8], w[9], w[10], w[11]);
            e4m3x4_to_f32(wv.w, w[12], w[13], w[14], w[15]);
            const float scl = rr == 0 ? sc[0][i] : sc[1][i];
#pragma unroll
            for (int t = 0; t < T; ++t) {
              float p = 0.f;
#pragma unroll
              for (int e = 0; e < 16; ++e) p = fmaf(w[e], areg[t][i][e], p);
              acc[t] = fmaf(p, scl, acc[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < T; ++t) {
        float v = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[(row * g.wpr + g.my_slice) * kTokBlk + t] = v;
      }
    }
    named_bar_sync(1, kCW * 32);
    if (threadIdx.x == 0) iss.next(plan, sh);   // the slot is free: refill it
    stage_epilogue(plan, s, red, n, g.wpr, r0, 0, T);
    rb ^= 1;
  }
}

// General path (any token count): activations read through L1 per stage.
template <int WT, int AT, class Plan>
KD_DEV void consume_segment_l1(const Plan& plan, StreamShared& sh, Issuer& iss, const Seg& s,
                               uint32_t& it, int& rb, unsigned* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int epc = WT == W_BF16 ? 8 : 16;
  const SegGeom g = seg_geom(s.row_bytes, warp);
  for (int r0 = 0; r0 < s.nrows; r0 += g.rps, ++it) {
    const int n = s.nrows - r0 < g.rps ? s.nrows - r0 : g.rps;
    const int slot = it % kStages;
    const uint32_t ph = (it / kStages) & 1u;
    wait_or_abort(&sh.full[slot], ph, sh.abort_flag, err, ERR_WAIT_FULL);
    const uint8_t* st = sh.stage + (size_t)slot * kStageBytes;
    for (int tb = 0; tb < s.ntok; tb += kTokBlk) {
      const int ntb = s.ntok - tb < kTokBlk ? s.ntok - tb : kTokBlk;
      float* red = sh.red + rb * kRedFloats;
      for (int rr = 0; rr < g.rpw; ++rr) {
        const int row = g.my_row0 + rr;
        if (row >= n) break;
        const float* srow = nullptr;
        if constexpr (WT == W_FP8) srow = plan.scale_row(s, s.row0 + r0 + row);
        for (int tg = 0; tg < ntb; tg += kTT) {
          const int nt = ntb - tg < kTT ? ntb - tg : kTT;
          const void* arow[kTT];
#pragma unroll
          for (int t = 0; t < kTT; ++t) arow[t] = plan.act_row(s, tb + tg + (t < nt ? t : 0));
          float acc[kTT];
#pragma unroll
          for (int t = 0; t < kTT; ++t) acc[t] = 0.f;
          const uint8_t* wrow = st + (size_t)row * s.row_bytes;
          for (int c = lane; c < g.chunks_slice; c += 32) {
            const int ci = g.my_slice * g.chunks_slice + c;
            const int col = ci * epc;
            const uint4 wv = lds_v4(wrow + (size_t)ci * 16);
            float scale = 1.f;
            if constexpr (WT == W_FP8) scale = srow[col >> 7];
            chunk_fma<WT, AT>(wv, scale, arow, col, nt, acc);
          }
#pragma unroll
          for (int t = 0; t < kTT; ++t) {
            float v = acc[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[t] = v;
          }
          if (lane == 0) {
#pragma unroll
            for (int t = 0; t < kTT; ++t)
              if (t < nt) red[(row * g.wpr + g.my_slice) * kTokBlk + tg + t] = acc[t];
          }
        }
      }
      named_bar_sync(1, kCW * 32);
      // after the stage's last token block no thread reads it again: refill
      if (threadIdx.x == 0 && tb + kTokBlk >= s.ntok) iss.next(plan, sh);
      stage_epilogue(plan, s, red, n, g.wpr, r0, tb, ntb);
      rb ^= 1;
    }
    if (s.ntok == 0) {
      named_bar_sync(1, kCW * 32);
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
    const bool fits = (s.row_bytes / 16) / seg_geom(s.row_bytes, 0).wpr <= 32 * kMaxChunksLane;
    if (fits && s.ntok == 1) {
      consume_segment_reg<WT, AT, 1>(plan, sh, iss, s, it, rb, err);
    } else if (WT == W_BF16 && fits && s.ntok == 2) {
      consume_segment_reg<WT, AT, 2>(plan, sh, iss, s, it, rb, err);
    } else {
      consume_segment_l1<WT, AT>(plan, sh, iss, s, it, rb, err);
    }
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

// kd_full.cuh -- the attention half of the full decode layer
// (kd_decode_layer_full): the two RMSNorms and decode attention over an FP8
// e4m3 KV cache.  The QKV projection (which also appends the new keys and
// values to the cache) and the o-proj + residual run on the projection
// engines of kd_kernels.cuh / kd_mma_kernels.cuh.
//
//   rmsnorm_in_kernel   u = RMSNorm(x) g1                  x bf16 -> u fp32 + bf16 hi/lo
//   attention_kernel    o = softmax(q K'^T / sqrt(hd)) V'  per (token, kv head, position
//                       chunk); the last chunk to finish of a (token, kv head)
//                       merges the chunks and writes o fp32 + bf16 hi/lo
//   rmsnorm_moe_kernel  w = RMSNorm(h1) g2 into the buffers the router and the
//                       experts read (h1f, bf16 terms, or per-64 maxima for FP8)
#pragma once

#include "kd_mma_kernels.cuh"

namespace kd {

constexpr int kNormThreads = 256;

// Sum of squares of a row, block-wide, in a fixed order (each thread's
// strided elements in order, then a shuffle tree, then the warps in order).
KD_DEV float row_sumsq(float part, float* red) {
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = part;
  __syncthreads();
  float ss = 0.f;
  for (int w = 0; w < kNormThreads / 32; ++w) ss += red[w];
  __syncthreads();
  return ss;
}

// 1 / sqrt(mean + eps) with IEEE square root and division.
KD_DEV float rms_inv(float ss, int n, float eps) {
  return __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)n), eps)));
}

// One CTA per token: u = x / sqrt(mean(x^2) + eps) * g1, as fp32 (CUDA-core
// projection) and as a bf16 hi + lo pair (tensor-core projection).
__global__ void __launch_bounds__(kNormThreads) rmsnorm_in_kernel(LayerDev L, Acts a) {
  __shared__ float red[kNormThreads / 32];
  pdl_wait();
  const int t = blockIdx.x, H = L.H;
  const uint16_t* x = a.x + (size_t)t * H;
  float part = 0.f;
  for (int i = threadIdx.x; i < H; i += kNormThreads) {
    const float v = __uint_as_float((uint32_t)x[i] << 16);
    part = fmaf(v, v, part);
  }
  const float r = rms_inv(row_sumsq(part, red), H, L.eps);
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < H; i += kNormThreads) {
    const float v = __uint_as_float((uint32_t)x[i] << 16);
    const float u = __fmul_rn(__fmul_rn(v, r), __uint_as_float((uint32_t)L.g1[i] << 16));
    const size_t o = (size_t)t * H + i;
    L.uf[o] = u;
    const uint16_t hi = f32_to_bf16_bits(u);
    L.u_hi[o] = hi;
    L.u_lo[o] = f32_to_bf16_bits(u - __uint_as_float((uint32_t)hi << 16));
  }
}

// One CTA per token: w = h1 / sqrt(mean(h1^2) + eps) * g2 into the buffers
// the MoE half reads: h1f (fp32: CUDA-core router and experts), and for the
// tensor-core kernels the bf16 hi / mid / lo terms (bf16 weights) or h1b and
// the maxima of |w| per 64 elements (FP8 weights).  Warp w takes the
// 64-element groups w, w + 8, ...; lane l elements 2l and 2l + 1 of a group.
__global__ void __launch_bounds__(kNormThreads) rmsnorm_moe_kernel(LayerDev L, int fp8) {
  __shared__ float red[kNormThreads / 32];
  pdl_wait();
  const int t = blockIdx.x, H = L.H;
  const float* h = L.h1r + (size_t)t * H;
  float part = 0.f;
  for (int i = threadIdx.x; i < H; i += kNormThreads) part = fmaf(h[i], h[i], part);
  const float r = rms_inv(row_sumsq(part, red), H, L.eps);
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int g = warp; g < H / kQGroup; g += kNormThreads / 32) {
    const int i = g * kQGroup + 2 * lane;
    const size_t o = (size_t)t * H + i;
    const float w0 = __fmul_rn(__fmul_rn(h[i], r), __uint_as_float((uint32_t)L.g2[i] << 16));
    const float w1 = __fmul_rn(__fmul_rn(h[i + 1], r), __uint_as_float((uint32_t)L.g2[i + 1] << 16));
    L.h1f[o] = w0;
    L.h1f[o + 1] = w1;
    store_hilo3(L.h1b, L.h1lo, L.h1lo2, o, w0);
    store_hilo3(L.h1b, L.h1lo, L.h1lo2, o + 1, w1);
    if (!fp8) continue;
    float mx = fmaxf(fabsf(w0), fabsf(w1));
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) L.h1g[(size_t)t * (H / kQGroup) + g] = mx;
  }
}

// ------------------------------------------------------------------ attention

// Sum over the warp of GRP per-lane values, transposed: the first log2(GRP)
// exchange steps each halve the values a lane holds (the lane keeps the
// half its lane bit selects), the rest add across lanes.  Lane l returns the
// total of value hh = bits (4, 3, ...) of l read as a binary number.
template <int GRP>
KD_DEV float reduce_heads(float (&v)[GRP], int lane, int& hh) {
  int n = GRP, bit = 16;
  hh = 0;
#pragma unroll
  for (int lv = 0; (1 << lv) < GRP; ++lv) {
    const int half = n >> 1;
    const bool up = lane & bit;
#pragma unroll
    for (int i = 0; i < GRP / 2; ++i) {
      if (i < half) {
        const float send = up ? v[i] : v[i + half];
        const float keep = up ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
      }
    }
    if (up) hh += half;
    n = half;
    bit >>= 1;
  }
  float y = v[0];
#pragma unroll
  for (int b = 16; b > 0; b >>= 1)
    if (b <= bit) y += __shfl_xor_sync(0xffffffffu, y, b);
  return y;
}

KD_DEV void e4m3x4_dec(uint32_t u, float* f) { e4m3x4_to_f32(u, f[0], f[1], f[2], f[3]); }

// Dims per lane of a head row, and loading them (DPL e4m3 codes).
template <int HD>
KD_DEV void load_kv_codes(const uint8_t* row, int lane, float* f) {
  constexpr int DPL = HD / 32;
  if constexpr (DPL == 4) {
    e4m3x4_dec(*reinterpret_cast<const uint32_t*>(row + 4 * lane), f);
  } else {
    const float2 v = e4m3x2_value(*reinterpret_cast<const uint16_t*>(row + 2 * lane));
    f[0] = v.x;
    f[1] = v.y;
  }
}

// One CTA per (token t, kv head g, chunk c of att_ch positions): scores of
// the GRP query heads of the group for the chunk's positions (pass 1, into
// shared memory), softmax statistics per head (warp h: head h), the
// probability-weighted value rows (pass 2, warps over positions), then the
// warps' sums added in warp order into the chunk's partial (max, sum, acc).
// The chunk that arrives last for (t, g) merges the chunks in chunk order.
// K and V rows are dequantised as code x scale; q carries k_scale / sqrt(hd).
template <int HD, int GRP>
__global__ void __launch_bounds__(256) attention_kernel(LayerDev L, Acts a) {
  extern __shared__ float att_smem[];
  constexpr int DPL = HD / 32;
  const int nch = L.att_nch, CH = L.att_ch;
  const int t = blockIdx.x / (L.Hkv * nch), g = (blockIdx.x / nch) % L.Hkv, c = blockIdx.x % nch;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  const int s = a.seq[t], p = a.pos[t];
  const int A = L.Hq * HD;
  if (s < 0 || s >= L.n_seq || p < 0 || p >= L.max_ctx) {
    // bad sequence / position: this token's heads of group g are zero
    if (c == 0) {
      if (threadIdx.x == 0) set_error(L.err, ERR_BAD_KV);
      for (int i = threadIdx.x; i < GRP * HD; i += blockDim.x) {
        const size_t o = (size_t)t * A + (size_t)g * GRP * HD + i;
        L.attnf[o] = 0.f;
        L.attn_hi[o] = 0;
        L.attn_lo[o] = 0;
      }
    }
    return;
  }
  const int len = p + 1, nct = (len + CH - 1) / CH;
  if (c >= nct) return;
  const int j0 = c * CH, j1 = min(j0 + CH, len), nj = j1 - j0;
  float* sc = att_smem;                        // [CH][GRP] scores, then probabilities
  float* red = att_smem + (size_t)CH * GRP;    // [8 warps][GRP][HD] partial sums
  float* stat = red + 8 * GRP * HD;            // [GRP] max, [GRP] sum
  const int kw = L.Hkv * HD;
  const float qs = __fdiv_rn(L.k_scale, __fsqrt_rn((float)HD));
  float q[GRP][DPL];
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int d = 0; d < DPL; ++d)
      q[h][d] = L.qkvf[(size_t)t * L.Nqkv + (size_t)(g * GRP + h) * HD + lane * DPL + d] * qs;
  const uint8_t* kbase = a.kc + (size_t)s * L.max_ctx * kw + (size_t)g * HD;
  const uint8_t* vbase = a.vc + (size_t)s * L.max_ctx * kw + (size_t)g * HD;
  // pass 1: scores
  for (int j = j0 + warp; j < j1; j += 8) {
    float k[DPL];
    load_kv_codes<HD>(kbase + (size_t)j * kw, lane, k);
    float part[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < DPL; ++d) acc = fmaf(q[h][d], k[d], acc);
      part[h] = acc;
    }
    int hh;
    const float y = reduce_heads<GRP>(part, lane, hh);
    if ((lane & (32 / GRP - 1)) == 0) sc[(j - j0) * GRP + hh] = y;
  }
  __syncthreads();
  // softmax statistics of the chunk, warp h for head h
  if (warp < GRP) {
    float m = -INFINITY;
    for (int j = lane; j < nj; j += 32) m = fmaxf(m, sc[j * GRP + warp]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int j = lane; j < nj; j += 32) {
      const float e = expf(sc[j * GRP + warp] - m);
      sc[j * GRP + warp] = e;
      l += e;
    }
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      stat[warp] = m;
      stat[GRP + warp] = l;
    }
  }
  __syncthreads();
  // pass 2: probability-weighted value rows
  float acc[GRP][DPL];
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int d = 0; d < DPL; ++d) acc[h][d] = 0.f;
  for (int j = j0 + warp; j < j1; j += 8) {
    float v[DPL];
    load_kv_codes<HD>(vbase + (size_t)j * kw, lane, v);
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const float pr = sc[(j - j0) * GRP + h];
#pragma unroll
      for (int d = 0; d < DPL; ++d) acc[h][d] = fmaf(pr, v[d], acc[h][d]);
    }
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int d = 0; d < DPL; ++d) red[((size_t)warp * GRP + h) * HD + lane * DPL + d] = acc[h][d];
  __syncthreads();
  // the chunk's partial: [GRP][HD + 2] (acc, max, sum)
  constexpr int PW = HD + 2;
  float* part = L.att_ws + (((size_t)t * L.Hkv + g) * nch + c) * GRP * PW;
  for (int i = threadIdx.x; i < GRP * HD; i += blockDim.x) {
    const int h = i / HD, d = i % HD;
    float v = 0.f;
    for (int w = 0; w < 8; ++w) v += red[((size_t)w * GRP + h) * HD + d];
    __stcg(part + h * PW + d, v);
  }
  if (threadIdx.x < GRP) {
    __stcg(part + threadIdx.x * PW + HD, stat[threadIdx.x]);
    __stcg(part + threadIdx.x * PW + HD + 1, stat[GRP + threadIdx.x]);
  }
  __threadfence();
  __syncthreads();
  __shared__ int s_last;
  if (threadIdx.x == 0) {
    unsigned* cnt = L.att_cnt + (size_t)t * L.Hkv + g;
    const unsigned prev = atomicAdd(cnt, 1u);
    s_last = prev == (unsigned)(nct - 1);
    if (s_last) *cnt = 0u;   // every chunk is in: ready for the next call
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge the chunks in chunk order: o = sum_c e^(m_c - M) acc_c / sum_c e^(m_c - M) l_c
  const float* base = L.att_ws + ((size_t)t * L.Hkv + g) * nch * GRP * PW;
  for (int i = threadIdx.x; i < GRP * HD; i += blockDim.x) {
    const int h = i / HD, d = i % HD;
    float M = -INFINITY;
    for (int cc = 0; cc < nct; ++cc) M = fmaxf(M, __ldcg(base + ((size_t)cc * GRP + h) * PW + HD));
    float num = 0.f, den = 0.f;
    for (int cc = 0; cc < nct; ++cc) {
      const float* pc = base + ((size_t)cc * GRP + h) * PW;
      const float f = expf(__ldcg(pc + HD) - M);
      num = fmaf(f, __ldcg(pc + d), num);
      den = fmaf(f, __ldcg(pc + HD + 1), den);
    }
    const float o = __fdiv_rn(num, den) * L.v_scale;
    const size_t oi = (size_t)t * A + (size_t)(g * GRP + h) * HD + d;
    L.attnf[oi] = o;
    const uint16_t hi = f32_to_bf16_bits(o);
    L.attn_hi[oi] = hi;
    L.attn_lo[oi] = f32_to_bf16_bits(o - __uint_as_float((uint32_t)hi << 16));
  }
}

// Shared memory of attention_kernel for chunks of `ch` positions.
__host__ __device__ inline size_t attention_smem(int ch, int grp, int hd) {
  return sizeof(float) * ((size_t)ch * grp + (size_t)8 * grp * hd + 2 * grp);
}

}  // namespace kd

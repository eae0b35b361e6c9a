/*
 * kdgen_host.c -- host entry points of the seeded input generator (kd_gen.h),
 * for the Python side: activations, router bias and reference copies of
 * generated weights.  Holds no arithmetic of the decode layer.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "kd_gen.h"

uint64_t kdg_host_mix(uint64_t z) { return kdg_mix(z); }
uint64_t kdg_host_stream(uint64_t seed, uint64_t uid) { return kdg_stream(seed, uid); }
uint64_t kdg_host_uid(uint32_t layer, uint32_t kind, uint32_t slot) { return kdg_uid(layer, kind, slot); }
int32_t kdg_host_ih4(uint64_t u) { return kdg_ih4(u); }

/* fp32 values idx = start .. start+n-1 of one tensor's stream */
void kdg_host_values(uint64_t seed, uint64_t uid, uint64_t start, int64_t n, float c, float* out) {
  uint64_t st = kdg_stream(seed, uid);
  for (int64_t i = 0; i < n; ++i) out[i] = kdg_value(st, start + (uint64_t)i, c);
}

void kdg_host_bf16(const float* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = kdg_bf16(in[i]);
}

void kdg_host_e4m3(const float* in, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = kdg_e4m3(in[i]);
}

/* Activations [M, width] as bf16 bits.  Row t follows a first-order
 * autoregression along the token axis, in fp64:
 *   z_t = ih4 * sqrt(3 / (2^32 - 1)),  x_0 = z_0,
 *   x_t = rho x_{t-1} + sqrt(1 - rho^2) z_t
 * rho = 0 gives independent N(0,1)-like rows.  Stored as bf16(float(x)). */
void kdg_host_activations(uint64_t seed, uint32_t layer, uint32_t kind, int M, int width,
                          double rho, uint16_t* out) {
  uint64_t st = kdg_stream(seed, kdg_uid(layer, kind, 0));
  double unit = sqrt(3.0 / 4294967295.0);
  double inn = sqrt(1.0 - rho * rho);
  double* prev = (double*)malloc(sizeof(double) * (size_t)(width > 0 ? width : 1));
  for (int t = 0; t < M; ++t)
    for (int c = 0; c < width; ++c) {
      double z = (double)kdg_ih4(kdg_bits(st, (uint64_t)t * (uint64_t)width + (uint64_t)c)) * unit;
      double v = t == 0 ? z : rho * prev[c] + inn * z;
      prev[c] = v;
      out[(size_t)t * width + c] = kdg_bf16((float)v);
    }
  free(prev);
}

/* Zipf(s) per-expert router bias: b_e = float(-s * ln(e + 1)), so that
 * exp(b_e) is proportional to (e + 1)^-s and expert 0 is the most favoured. */
void kdg_host_zipf_bias(int E, double s, float* out) {
  for (int e = 0; e < E; ++e) out[e] = (float)(-s * log((double)e + 1.0));
}

/* One logical weight matrix [R, K] of kind/slot as generated (sigma 0.02). */
void kdg_host_weight_bf16(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t slot,
                          int R, int K, uint16_t* out) {
  uint64_t st = kdg_stream(seed, kdg_uid(layer, kind, slot));
  for (int64_t i = 0; i < (int64_t)R * K; ++i) out[i] = kdg_bf16(kdg_value(st, (uint64_t)i, KDG_W002));
}

/* FP8 form of the same matrix: codes [R, K] and scales [ceil(R/128), ceil(K/128)]. */
void kdg_host_weight_fp8(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t slot,
                         int R, int K, uint8_t* codes, float* scales) {
  uint64_t st = kdg_stream(seed, kdg_uid(layer, kind, slot));
  int nrb = (R + 127) / 128, nkb = (K + 127) / 128;
  for (int rb = 0; rb < nrb; ++rb)
    for (int kb = 0; kb < nkb; ++kb) {
      float amax = 0.0f;
      for (int r = rb * 128; r < R && r < rb * 128 + 128; ++r)
        for (int c = kb * 128; c < K && c < kb * 128 + 128; ++c) {
          float a = fabsf(kdg_value(st, (uint64_t)r * K + c, KDG_W002));
          if (a > amax) amax = a;
        }
      float sc = kdg_fp8_scale(amax);
      scales[rb * nkb + kb] = sc;
      for (int r = rb * 128; r < R && r < rb * 128 + 128; ++r)
        for (int c = kb * 128; c < K && c < kb * 128 + 128; ++c)
          codes[(size_t)r * K + c] = kdg_e4m3(kdg_fp8_div(kdg_value(st, (uint64_t)r * K + c, KDG_W002), sc));
    }
}

/* RMSNorm gains [n] of one layer (kind KDG_NORM1 / KDG_NORM2) as bf16 bits. */
void kdg_host_norm_bf16(uint64_t seed, uint32_t layer, uint32_t kind, int n, uint16_t* out) {
  uint64_t st = kdg_stream(seed, kdg_uid(layer, kind, 0));
  for (int i = 0; i < n; ++i) out[i] = kdg_norm_bf16(st, (uint64_t)i);
}

/* Synthetic KV-cache contents: e4m3 codes of fp32(sigma * z) / scale for
 * element ((s * max_ctx + p) * width + c) of one layer's K (KDG_KCACHE) or V
 * (KDG_VCACHE) cache [n_seq][max_ctx][width], z = ih4 * unit (N(0,1)-like). */
void kdg_host_kv_cache(uint64_t seed, uint32_t layer, uint32_t kind, int n_seq, int max_ctx,
                       int width, float sigma, float scale, uint8_t* out) {
  uint64_t st = kdg_stream(seed, kdg_uid(layer, kind, 0));
  int64_t n = (int64_t)n_seq * max_ctx * width;
  for (int64_t i = 0; i < n; ++i) {
    float v = kdg_value(st, (uint64_t)i, KDG_UNIT) * sigma;
    out[i] = kdg_e4m3(kdg_fp8_div(v, scale));
  }
}

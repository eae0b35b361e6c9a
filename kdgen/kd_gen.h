/*
 * kd_gen.h -- counter-based synthetic input generator.
 *
 * This module is shared by the CUDA layer library and by the CPU oracle
 * that checks it.  It holds NO arithmetic of the decode layer itself: it only
 * turns (seed, tensor id, logical element index) into the bits of a weight
 * or activation element, and encodes those values into the storage formats
 * the layer consumes (bf16, or FP8 e4m3 codes plus one fp32 scale per
 * 128 x 128 block).  Decoding those formats and every step of the layer are
 * implemented separately on each side.
 *
 * Definition
 *   mix(z)          = splitmix64 output function applied to z + 0x9E3779B97F4A7C15
 *                     (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *                     generators", OOPSLA 2014; constants of Vigna's public version)
 *   stream(s, uid)  = mix(s XOR uid * 0x9E3779B97F4A7C15)
 *   bits(st, i)     = mix(st + i)           i = logical row-major element index
 *   ih4(u)          = (sum of the four 16-bit fields of u) - 2*65535
 *                     an Irwin-Hall(4) integer: mean 0, variance (2^32-1)/3,
 *                     range +-131070 (exact in fp32)
 *   value           = (float)ih4 * c   -- ONE fp32 multiply, c a fixed fp32 constant
 *                     c = KDG_UNIT  (unit variance) or KDG_W002 (sigma = 0.02)
 *   bf16            = round-to-nearest-even of the fp32 value
 *   norm weight     = bf16(1 + value), c = KDG_W002 (RMSNorm gains near 1)
 *   FP8 (per logical 128x128 block of a weight matrix)
 *                     amax  = max |value| over the block (fp32, exact)
 *                     scale = amax / 448 (IEEE fp32 division), 1 if amax == 0
 *                     code  = e4m3fn(value / scale), round-to-nearest-even,
 *                             saturating to +-448 (no inf/NaN produced)
 *
 * Everything is integer arithmetic plus one fp32 multiply (and, for FP8, one
 * IEEE division), so host and device produce bit-identical results when
 * compiled without fast-math or FMA contraction of the single multiply.
 */
#ifndef KD_GEN_H
#define KD_GEN_H

#include <stdint.h>

#if defined(__CUDACC__)
#define KDG_FN static __host__ __device__ __forceinline__
#else
#define KDG_FN static inline
#endif

#define KDG_GAMMA 0x9E3779B97F4A7C15ULL

/* fp32(sqrt(3 / (2^32 - 1)))         : unit-variance scale for ih4 */
#define KDG_UNIT 0x1.bb67aep-16f
/* fp32(0.02 * sqrt(3 / (2^32 - 1))) : sigma 0.02 scale for ih4    */
#define KDG_W002 0x1.1bc77ap-21f

/* tensor kinds (bits 32..39 of a tensor uid) */
enum {
  KDG_QKV = 1, KDG_OPROJ = 2, KDG_ROUTER = 3,
  KDG_GATE = 4, KDG_UP = 5, KDG_DOWN = 6,
  KDG_NORM1 = 7, KDG_NORM2 = 8,          /* RMSNorm gains before attention / the MoE */
  KDG_HIDDEN_IN = 16, KDG_ATTN_OUT = 17,
  KDG_KCACHE = 18, KDG_VCACHE = 19       /* synthetic KV-cache contents */
};

/* uid of one tensor: layer in bits 40.., kind in 32..39, expert slot in 0..31
 * (slot 0 = not an expert or the shared expert, 1 + e = routed expert e). */
KDG_FN uint64_t kdg_uid(uint32_t layer, uint32_t kind, uint32_t expert_slot) {
  return ((uint64_t)layer << 40) | ((uint64_t)kind << 32) | (uint64_t)expert_slot;
}

KDG_FN uint64_t kdg_mix(uint64_t z) {
  z += KDG_GAMMA;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

KDG_FN uint64_t kdg_stream(uint64_t seed, uint64_t uid) {
  return kdg_mix(seed ^ (uid * KDG_GAMMA));
}

KDG_FN uint64_t kdg_bits(uint64_t stream, uint64_t index) {
  return kdg_mix(stream + index);
}

KDG_FN int32_t kdg_ih4(uint64_t u) {
  int32_t s = (int32_t)(u & 0xFFFFu) + (int32_t)((u >> 16) & 0xFFFFu) +
              (int32_t)((u >> 32) & 0xFFFFu) + (int32_t)((u >> 48) & 0xFFFFu);
  return s - 131070;
}

/* fp32 value of element `index` of the stream, scaled by c (KDG_UNIT or KDG_W002). */
KDG_FN float kdg_value(uint64_t stream, uint64_t index, float c) {
  float z = (float)kdg_ih4(kdg_bits(stream, index)); /* exact: |ih4| < 2^24 */
#if defined(__CUDA_ARCH__)
  return __fmul_rn(z, c);                             /* never contracted */
#else
  return z * c;                                       /* host: -ffp-contract=off */
#endif
}

KDG_FN uint32_t kdg_f32_bits(float f) {
  union { float f; uint32_t u; } v; v.f = f; return v.u;
}

KDG_FN float kdg_bits_f32(uint32_t u) {
  union { float f; uint32_t u; } v; v.u = u; return v.f;
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs). */
KDG_FN uint16_t kdg_bf16(float f) {
  uint32_t b = kdg_f32_bits(f);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

/* RMSNorm gain element `index`: bf16(1 + value(sigma 0.02)). */
KDG_FN uint16_t kdg_norm_bf16(uint64_t stream, uint64_t index) {
#if defined(__CUDA_ARCH__)
  return kdg_bf16(__fadd_rn(1.0f, kdg_value(stream, index, KDG_W002)));
#else
  return kdg_bf16(1.0f + kdg_value(stream, index, KDG_W002));
#endif
}

/* FP8 block scale from a block's amax. */
KDG_FN float kdg_fp8_scale(float amax) {
#if defined(__CUDA_ARCH__)
  return amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
#else
  return amax > 0.0f ? amax / 448.0f : 1.0f;
#endif
}

/* value / scale, IEEE round-to-nearest division, before e4m3 encoding. */
KDG_FN float kdg_fp8_div(float v, float scale) {
#if defined(__CUDA_ARCH__)
  return __fdiv_rn(v, scale);
#else
  return v / scale;
#endif
}

/* fp32 -> e4m3fn code (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * largest finite 448 = 0x7E), round to nearest even, saturating.
 * Finite inputs only.  Quantum of a value in [2^E, 2^(E+1)) is 2^max(E-3,-9). */
KDG_FN uint8_t kdg_e4m3(float f) {
  uint32_t b = kdg_f32_bits(f);
  uint8_t sign = (uint8_t)((b >> 24) & 0x80u);
  uint32_t a = b & 0x7FFFFFFFu;
  if (a == 0u) return sign;
  int32_t E = (int32_t)(a >> 23) - 127;                 /* unbiased exponent */
  uint32_t m24 = (a & 0x7FFFFFu) | 0x800000u;           /* 1.mantissa as integer */
  if ((a >> 23) == 0u) { m24 = a & 0x7FFFFFu; E = -126; } /* fp32 subnormal */
  int32_t qe = E - 3 > -9 ? E - 3 : -9;                 /* quantum exponent */
  int32_t s = 23 - (E - qe);                            /* bits to drop, >= 20 */
  uint32_t n;
  if (s >= 32) {
    n = 0u;
  } else {
    uint32_t keep = m24 >> s;
    uint32_t rem = m24 & ((1u << s) - 1u);
    uint32_t half = 1u << (s - 1);
    n = keep + ((rem > half || (rem == half && (keep & 1u))) ? 1u : 0u);
  }
  if (n == 0u) return sign;
  if (n >= 16u) { n >>= 1; qe += 1; }                   /* mantissa carried out */
  if (qe == -9 && n < 8u) return (uint8_t)(sign | n);   /* subnormal */
  int32_t ef = qe + 10;
  uint32_t m = n - 8u;
  if (ef > 15 || (ef == 15 && m == 7u)) return (uint8_t)(sign | 0x7Eu);
  return (uint8_t)(sign | ((uint32_t)ef << 3) | m);
}

#endif /* KD_GEN_H */

// kd_common.cuh -- sm_100a building blocks shared by the layer's kernels:
// mbarriers with bounded waits, 1-D bulk TMA copies, L2 prefetch, the device
// error word, and bf16 / e4m3 unpacking.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define KD_DEV __device__ __forceinline__

namespace kd {

// Device error word bits (the layer's `err` buffer; read by kd_layer_check).
enum : unsigned {
  ERR_WAIT_FULL = 1u,   // consumer gave up waiting for a weight stage
  ERR_WAIT_EMPTY = 2u,  // producer gave up waiting for a free stage
  ERR_WAIT_MMA = 4u,    // tensor-core pipeline wait gave up
  ERR_BAD_ROUTE = 8u,   // routing produced an out-of-range expert id
  ERR_BAD_KV = 16u,     // full layer: a token's sequence / position outside the KV cache
};

// Every spin-wait gives up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

KD_DEV uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

KD_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

KD_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

KD_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

KD_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

KD_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
               ::"r"(smem_u32(bar)) : "memory");
}

KD_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

KD_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Wait for phase `parity` of an mbarrier to complete; false after the time
// limit (the caller records the error and stops its loop).
KD_DEV bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && globaltimer() - t0 > kWaitLimitNs) return false;
  }
}

// 1-D bulk copy global -> shared, completion counted on `bar` in bytes.
// Both addresses 16-byte aligned, size a multiple of 16.
KD_DEV void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst_smem)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Bring a global range into L2 without a destination (static weights only).
KD_DEV void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

KD_DEV void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

KD_DEV void set_error(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

// Programmatic dependent launch: wait for the preceding grid's memory to be
// visible / let the next grid start its prologue.
KD_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
KD_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// Read-only global load (activations written by an earlier kernel; weights).
// A plain intrinsic so the compiler may batch independent loads.
KD_DEV uint4 ld_nc_v4(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Shared-memory load of a stage written by the bulk-copy engine.  An ordinary
// C++ load: the "memory" clobber of the mbarrier wait that precedes it keeps
// the compiler from hoisting it above the wait.
KD_DEV uint4 lds_v4(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// bf16 pair packed in a u32 -> two fp32 (exact).
KD_DEV float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
KD_DEV float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Four e4m3 codes packed in a u32 -> four fp32 (exact, via f16x2).
KD_DEV void e4m3x4_to_f32(uint32_t u, float& a, float& b, float& c, float& d) {
  uint32_t lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi) : "r"(u));
  __half2 h0 = *reinterpret_cast<__half2*>(&lo);
  __half2 h1 = *reinterpret_cast<__half2*>(&hi);
  float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
  a = f0.x; b = f0.y; c = f1.x; d = f1.y;
}

KD_DEV uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

KD_DEV void store_hilo(uint16_t* hi, uint16_t* lo, size_t o, float v) {
  const uint16_t h = f32_to_bf16_bits(v);
  hi[o] = h;
  lo[o] = f32_to_bf16_bits(v - __uint_as_float((uint32_t)h << 16));
}

// v = hi + mid + lo exactly (each difference is exact in fp32; three 8-bit
// significands cover fp32's 24).
KD_DEV void store_hilo3(uint16_t* hi, uint16_t* mid, uint16_t* lo, size_t o, float v) {
  const uint16_t h = f32_to_bf16_bits(v);
  const float r1 = v - __uint_as_float((uint32_t)h << 16);
  const uint16_t m = f32_to_bf16_bits(r1);
  hi[o] = h;
  mid[o] = m;
  lo[o] = f32_to_bf16_bits(r1 - __uint_as_float((uint32_t)m << 16));
}

KD_DEV float silu(float z) { return z / (1.0f + expf(-z)); }

// Power of two 2^P that puts a group's largest magnitude amax in [128, 256)
// (inside e4m3's range, 448), and its inverse; 1 for an all-zero group.
KD_DEV float q_scale(float amax, float& inv) {
  if (!(amax > 0.f) || !(amax < 3.0e38f)) {
    inv = 1.f;
    return 1.f;
  }
  int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;   // floor(log2 amax), normal amax
  if (e < -126) e = -126;
  int P = 7 - e;
  P = P > 100 ? 100 : (P < -100 ? -100 : P);
  inv = __uint_as_float((uint32_t)(127 - P) << 23);
  return __uint_as_float((uint32_t)(127 + P) << 23);
}

// e4m3 (round to nearest even, saturating) of two values: byte 0 = lo, byte 1 = hi.
KD_DEV uint32_t e4m3x2_rn(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// The two e4m3 codes of e4m3x2_rn back to fp32 (exact).
KD_DEV float2 e4m3x2_value(uint32_t v) {
  uint32_t h;
  const uint16_t b = (uint16_t)v;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b));
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

// Two fp32 values in one 64-bit register, for the packed fp32 FMA of sm_100
// (fma.rn.f32x2: two IEEE fp32 FMAs per instruction).
typedef unsigned long long f32x2;

KD_DEV f32x2 pack2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

KD_DEV float2 unpack2(f32x2 v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}

KD_DEV f32x2 ffma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// bf16 pair (u32) -> packed fp32 pair (exact).
KD_DEV f32x2 bf2_to_f2(uint32_t u) { return pack2(bf_lo(u), bf_hi(u)); }

}  // namespace kd

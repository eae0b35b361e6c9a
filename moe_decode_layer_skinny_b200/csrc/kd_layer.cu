// kd_layer.cu -- runtime of the decode layer and its C ABI (include/kd.h).
//
// HBM layout of one layer (all row-major, K contiguous; elem = 2 bytes bf16
// or 1 byte e4m3; FP8 scales are fp32 per logical 128x128 block):
//   wqkv  [Nqkv, H]          sqkv [Nqkv/128, H/128]
//   wo    [H, A]             so   [H/128, A/128]
//   wr    [E, H]             sr   [ceil(E/128), H/128]
//   wgu   [E][2I, H]  physical row 2i = gate row i, 2i+1 = up row i
//                            sgu  [E][2][I/128][H/128]   (gate blocks, then up)
//   wd    [E][H, I]          sd   [E][H/128][I/128]
//   shared expert: wgu_sh [2I, H], wd_sh [H, I] (same layouts, own scales)
// Workspaces are sized for max_tokens and owned by the layer.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/kd.h"
#include "kd_full.cuh"
#include "kd_kernels.cuh"
#include "kd_mma_kernels.cuh"

using namespace kd;

static thread_local std::string g_err;

static int fail(int code, const char* fmt, const char* a = "", long b = 0) {
  char buf[512];
  snprintf(buf, sizeof buf, fmt, a, b);
  g_err = buf;
  return code;
}

#define KD_CUDA(call)                                                                   \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess) return fail(KD_ECUDA, "%s (line %ld)", cudaGetErrorString(e_), __LINE__); \
  } while (0)

struct kd_layer {
  kd_config cfg{};
  int dev = 0, nsm = 0, maxM = 0;
  size_t l2_bytes = 0;
  LayerDev d{};
  std::vector<void*> allocs;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_h1 = nullptr, ev_sh = nullptr;
  uint64_t static_bytes = 0, expert_bytes = 0;
  int Nqkv = 0, A = 0;
  bool tp = false;       // a tensor-parallel shard (kd_tp_* calls)
  bool w8a8 = false;     // FP8 experts with one e4m3 activation term
  int attn_col0 = 0;     // a shard's first attention-output column
  cudaEvent_t tev[KD_N_TIMING_EVENTS] = {};  // profiling hook (kd_layer_set_timing_events)
  bool timing = false;
  int mma_min = 4;       // calls with M >= mma_min use the tensor-core kernels
  bool has_maps = false;
  MmaMaps maps{};
  size_t ntile = 0;      // split-K tile arrival counters per stream
  // test hook: the n-th device allocation of kd_layer_create fails (0 = none)
  int fail_alloc_at = 0, nalloc = 0;
  // full layer
  bool full = false;
  size_t att_smem = 0;
  int att_ncnt = 0;      // (token, kv head) arrival counters
};

struct kd_stack {
  std::vector<kd_layer*> layers;
  int M = 0, prefetch = 0;
  cudaStream_t cap = nullptr, pf = nullptr;
  std::vector<cudaEvent_t> ev_fork, ev_join;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  void* hidden = nullptr;
  const void* attn = nullptr;
};

extern "C" const char* kd_last_error(void) { return g_err.c_str(); }

// Shared with the other entry-point files of the library.
void kd_set_last_error(const char* msg) { g_err = msg; }

// ------------------------------------------------------------------ helpers

static int dalloc(kd_layer* L, size_t bytes, void** p) {
  if (bytes == 0) bytes = 16;
  if (L->fail_alloc_at > 0 && ++L->nalloc == L->fail_alloc_at) {
    *p = nullptr;
    return fail(KD_ENOMEM, "cudaMalloc of %s%ld bytes failed (injected by KD_TEST_FAIL_ALLOC_AT)", "",
                (long)bytes);
  }
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(KD_ENOMEM, "cudaMalloc of %s%ld bytes failed", "", (long)bytes);
  }
  L->allocs.push_back(*p);
  return KD_OK;
}

template <class T>
static int dalloc_t(kd_layer* L, size_t n, T** p) {
  void* v = nullptr;
  int rc = dalloc(L, n * sizeof(T), &v);
  *p = static_cast<T*>(v);
  return rc;
}

static int ceil128(int x) { return (x + 127) / 128; }

// cuTensorMapEncodeTiled, looked up through the runtime (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map of a row-major weight matrix [rows, K] (bf16 or e4m3 codes): box
// 128 bytes x 128 rows (64 bf16 or 128 e4m3 per row), 128B swizzle.
static bool encode_weight_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, bool fp8) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {fp8 ? 128u : 64u, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Generate rows [lr0, lr0 + R) x columns [lc0, lc0 + K) of one logical
// matrix with LK columns (LK = 0: the whole [R, K] matrix) into `dst` with
// row stride multiplier (physical row = r*mult + off); FP8 writes its block
// scales to `scales`.
static int gen_matrix(const kd_layer* L, uint8_t* dst, float* scales, int R, int K, uint64_t seed,
                      uint32_t kind, uint32_t slot, int mult, int off, cudaStream_t s,
                      int lr0 = 0, int lc0 = 0, int LK = 0) {
  const uint64_t st = kdg_stream(seed, kdg_uid((uint32_t)L->cfg.layer_id, kind, slot));
  const uint64_t lk = LK ? (uint64_t)LK : (uint64_t)K;
  if (L->cfg.wdtype == KD_WBF16) {
    gen_bf16_kernel<<<L->nsm * 8, 256, 0, s>>>(reinterpret_cast<uint16_t*>(dst), R, K, st, mult, off,
                                               (uint64_t)lr0, (uint64_t)lc0, lk);
  } else {
    gen_fp8_kernel<<<dim3(ceil128(K), ceil128(R)), 256, 0, s>>>(dst, scales, R, K, st, mult, off,
                                                                (uint64_t)lr0, (uint64_t)lc0, lk);
  }
  KD_CUDA(cudaGetLastError());
  return KD_OK;
}

// RMSNorm gains: dst[i] = bf16(1 + value(stream, i)).
static __global__ void gen_norm_kernel(uint16_t* dst, int n, uint64_t stream) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    dst[i] = kdg_norm_bf16(stream, (uint64_t)i);
}

typedef void (*AttnKernel)(LayerDev, Acts);

static AttnKernel attention_for(int hd, int grp) {
  if (hd == 128) {
    switch (grp) {
      case 1: return attention_kernel<128, 1>;
      case 2: return attention_kernel<128, 2>;
      case 4: return attention_kernel<128, 4>;
      case 8: return attention_kernel<128, 8>;
    }
  } else if (hd == 64) {
    switch (grp) {
      case 1: return attention_kernel<64, 1>;
      case 2: return attention_kernel<64, 2>;
      case 4: return attention_kernel<64, 4>;
      case 8: return attention_kernel<64, 8>;
    }
  }
  return nullptr;
}

static void free_layer(kd_layer* L) {
  if (!L) return;
  for (void* p : L->allocs) cudaFree(p);
  if (L->side) cudaStreamDestroy(L->side);
  if (L->ev_h1) cudaEventDestroy(L->ev_h1);
  if (L->ev_sh) cudaEventDestroy(L->ev_sh);
  delete L;
}

static bool stream_kernels_configured = false;
constexpr int kMaxAttChunk = 1024;   // attention positions per CTA (at most)

// Routed gate/up CTAs keep the call's routing after the stream area.
static size_t gateup_smem(const LayerDev& d, int M) {
  return kStreamSmem + 16 + sizeof(int) * kRouteSmemInts(d.E, M * d.k);
}
static const size_t kMaxGateupSmem = kStreamSmem + 16 + sizeof(int) * kRouteSmemInts(1024, 64 * 16);

static int configure_kernels() {
  if (stream_kernels_configured) return KD_OK;
  const int smem = (int)kMaxGateupSmem;
  KD_CUDA(cudaFuncSetAttribute(proj_kernel<W_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(proj_kernel<W_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(gateup_kernel<W_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(gateup_kernel<W_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(down_kernel<W_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(down_kernel<W_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int rsmem = (int)(sizeof(int) * kSelectSmemInts(1024, 64 * 16));
  KD_CUDA(cudaFuncSetAttribute(router_kernel<W_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, rsmem));
  KD_CUDA(cudaFuncSetAttribute(router_kernel<W_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, rsmem));
  KD_CUDA(cudaFuncSetAttribute(tp_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, rsmem));
  const int msmem = (int)kMmaSmem;
  KD_CUDA(cudaFuncSetAttribute(mma_proj_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_gateup_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_down_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_router_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_router_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_proj_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_gateup_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_down_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_gateup_kernel<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_down_kernel<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(proj_kernel<W_BF16, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(proj_kernel<W_BF16, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(proj_kernel<W_FP8, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(proj_kernel<W_FP8, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  KD_CUDA(cudaFuncSetAttribute(mma_proj_kernel<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_proj_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_proj_kernel<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  KD_CUDA(cudaFuncSetAttribute(mma_proj_kernel<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, msmem));
  for (int hd : {64, 128})
    for (int grp : {1, 2, 4, 8})
      KD_CUDA(cudaFuncSetAttribute(attention_for(hd, grp), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)attention_smem(kMaxAttChunk, grp, hd)));
  stream_kernels_configured = true;
  return KD_OK;
}

// ------------------------------------------------------------------ create

extern "C" int kd_layer_create(const kd_config* cfg, uint64_t seed, kd_layer** out) {
  if (!cfg || !out) return fail(KD_EINVAL, "kd_layer_create: null argument%s", "");
  *out = nullptr;
  const kd_config& c = *cfg;
  const int A = c.q_heads * c.head_dim, Nqkv = (c.q_heads + 2 * c.kv_heads) * c.head_dim;
  if (c.hidden <= 0 || c.hidden % 128 || c.q_heads <= 0 || c.kv_heads < 0 || c.head_dim <= 0 ||
      A % 128 || Nqkv % 128 || c.n_experts < 1 || c.n_experts > 1024 || c.top_k < 1 ||
      c.top_k > 16 || c.top_k > c.n_experts || c.n_shared < 0 || c.n_shared > 1 || c.inter <= 0 ||
      c.inter % 128 || (c.wdtype != KD_WBF16 && c.wdtype != KD_WFP8) || c.max_tokens < 1 ||
      c.max_tokens > 64 || c.layer_id < 0 || c.mma_min_tokens < 0 ||
      (c.bias_select_only != 0 && c.bias_select_only != 1) || c.fp8_act_terms < 0 ||
      c.fp8_act_terms > 2)
    return fail(KD_EINVAL, "kd_layer_create: unsupported configuration%s", "");
  if (c.hidden * 2 > kStageBytes || A * 2 > kStageBytes || c.inter * 2 > kStageBytes ||
      c.hidden > 8192 || A > 8192 || c.inter > 8192)
    return fail(KD_EINVAL, "kd_layer_create: a weight row exceeds one %s%ld-byte stage", "",
                (long)kStageBytes);
  const int R = c.tp_size > 1 ? c.tp_size : 1, tr = c.tp_size > 1 ? c.tp_rank : 0;
  if (c.tp_size < 0 || c.tp_rank < 0 || (c.tp_size <= 1 && c.tp_rank != 0) || tr >= R)
    return fail(KD_EINVAL, "kd_layer_create: bad tensor-parallel rank%s", "");
  if (R > 1) {
    const bool fp8 = c.wdtype == KD_WFP8;
    // q heads per rank and the kv heads they read (all ranks alike: a rank's
    // q heads never straddle two kv-head groups unevenly)
    const int qr = c.q_heads / R, grp = c.kv_heads > 0 ? c.q_heads / c.kv_heads : 0;
    const bool even = grp > 0 && qr > 0 && (qr % grp == 0 || grp % qr == 0);
    const int kvr = even ? (qr >= grp ? qr / grp : 1) : 0;
    if (!even || ((qr + 2 * kvr) * c.head_dim) % 128 ||
        c.kv_heads < 1 || c.q_heads % c.kv_heads || c.q_heads % R || c.n_experts % R ||
        c.inter % R || (c.inter / R) % 128 || (c.q_heads / R * c.head_dim) % 128 || c.full_layer ||
        (fp8 && ((c.n_experts / R) % 128 || c.head_dim % 128)))
      return fail(KD_EINVAL, "kd_layer_create: unsupported tensor-parallel sharding%s", "");
  }
  if (c.full_layer) {
    const int grp = c.kv_heads > 0 ? c.q_heads / c.kv_heads : 0;
    if (c.full_layer != 1 || c.kv_heads < 1 || c.q_heads % c.kv_heads ||
        (grp != 1 && grp != 2 && grp != 4 && grp != 8) || (c.head_dim != 64 && c.head_dim != 128) ||
        c.kv_n_seq < 1 || c.kv_max_ctx < 1 || !(c.k_scale > 0.f) || !(c.v_scale > 0.f) ||
        c.rms_eps < 0.f)
      return fail(KD_EINVAL, "kd_layer_create: unsupported full-layer configuration%s", "");
  }

  kd_layer* L = new kd_layer();
  L->cfg = c;
  if (const char* f = getenv("KD_TEST_FAIL_ALLOC_AT")) L->fail_alloc_at = atoi(f);
  if (const char* f = getenv("KD_TEST_STALL_WAIT")) L->d.test_stall = atoi(f) == 1;
  L->w8a8 = c.fp8_act_terms == 1;
  L->cfg.router_bias = nullptr;
  L->maxM = c.max_tokens;
  L->mma_min = c.mma_min_tokens > 0 ? c.mma_min_tokens : 1;
  // tensor-parallel shard: its q heads [q0, q1), the kv heads they read
  // [k0, k1), router rows [e0, e0 + Er), expert rows [i0, i0 + Ir)
  const int q0 = c.q_heads * tr / R, q1 = c.q_heads * (tr + 1) / R;
  const int grpq = c.kv_heads > 0 ? c.q_heads / c.kv_heads : 1;
  const int k0 = R > 1 ? q0 / grpq : 0, k1 = R > 1 ? (q1 - 1) / grpq + 1 : c.kv_heads;
  const int Ar = (q1 - q0) * c.head_dim;
  const int Nr = (q1 - q0 + 2 * (k1 - k0)) * c.head_dim;
  const int Er = c.n_experts / R, e0 = Er * tr, Ir = c.inter / R, i0 = Ir * tr;
  L->tp = R > 1;
  L->attn_col0 = q0 * c.head_dim;
  L->Nqkv = Nr;
  L->A = Ar;
  int rc = KD_OK;
#define TRY(x)                 \
  do {                         \
    rc = (x);                  \
    if (rc != KD_OK) {         \
      free_layer(L);           \
      return rc;               \
    }                          \
  } while (0)
#define TRYC(x)                                                                      \
  do {                                                                               \
    cudaError_t e_ = (x);                                                            \
    if (e_ != cudaSuccess) {                                                         \
      free_layer(L);                                                                 \
      return fail(KD_ECUDA, "%s (line %ld)", cudaGetErrorString(e_), __LINE__);      \
    }                                                                                \
  } while (0)
  TRYC(cudaGetDevice(&L->dev));
  TRYC(cudaDeviceGetAttribute(&L->nsm, cudaDevAttrMultiProcessorCount, L->dev));
  int l2 = 0;
  TRYC(cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, L->dev));
  L->l2_bytes = (size_t)l2;
  TRY(configure_kernels());

  LayerDev& d = L->d;
  // (a shard: A, Nqkv, I its own; E the experts the selection runs over; the
  // router generates Er rows)
  const int H = c.hidden, E = c.n_experts, k = c.top_k, M = c.max_tokens;
  const int I = Ir, A_ = Ar, Nq = Nr;
  const int eb = c.wdtype == KD_WBF16 ? 2 : 1;
  const bool fp8 = c.wdtype == KD_WFP8;
  d.H = H; d.A = A_; d.Nqkv = Nq; d.E = E; d.k = k; d.I = I; d.S = c.n_shared; d.eb = eb;
  d.nHb = ceil128(H); d.nAb = ceil128(A_); d.nIb = ceil128(I);
  d.Er = Er; d.attn_ld = A; d.tp = L->tp ? 1 : 0;

  uint8_t *wqkv, *wo, *wr, *wgu_sh = nullptr, *wd_sh = nullptr, *wgu, *wd;
  float *sqkv = nullptr, *so = nullptr, *sr = nullptr, *sgu_sh = nullptr, *sd_sh = nullptr,
        *sgu = nullptr, *sd = nullptr;
  TRY(dalloc_t(L, (size_t)Nq * H * eb, &wqkv));
  TRY(dalloc_t(L, (size_t)H * A_ * eb, &wo));
  TRY(dalloc_t(L, (size_t)Er * H * eb, &wr));
  const size_t gu_bytes = (size_t)2 * I * H * eb, dn_bytes = (size_t)H * I * eb;
  if (c.n_shared) {
    TRY(dalloc_t(L, gu_bytes, &wgu_sh));
    TRY(dalloc_t(L, dn_bytes, &wd_sh));
  }
  TRY(dalloc_t(L, gu_bytes * E, &wgu));
  TRY(dalloc_t(L, dn_bytes * E, &wd));
  const size_t n_sgu = (size_t)2 * d.nIb * d.nHb, n_sd = (size_t)d.nHb * d.nIb;
  if (fp8) {
    TRY(dalloc_t(L, (size_t)ceil128(Nq) * d.nHb, &sqkv));
    TRY(dalloc_t(L, (size_t)d.nHb * d.nAb, &so));
    TRY(dalloc_t(L, (size_t)ceil128(Er) * d.nHb, &sr));
    if (c.n_shared) {
      TRY(dalloc_t(L, n_sgu, &sgu_sh));
      TRY(dalloc_t(L, n_sd, &sd_sh));
    }
    TRY(dalloc_t(L, n_sgu * E, &sgu));
    TRY(dalloc_t(L, n_sd * E, &sd));
  }
  d.wqkv = wqkv; d.wo = wo; d.wr = wr; d.wgu_sh = wgu_sh; d.wd_sh = wd_sh; d.wgu = wgu; d.wd = wd;
  d.sqkv = sqkv; d.so = so; d.sr = sr; d.sgu_sh = sgu_sh; d.sd_sh = sd_sh; d.sgu = sgu; d.sd = sd;

  const size_t sc = fp8 ? sizeof(float) : 0;
  L->static_bytes = (size_t)Nq * H * eb + (size_t)H * A_ * eb + (size_t)Er * H * eb +
                    (c.n_shared ? gu_bytes + dn_bytes : 0) +
                    sc * ((size_t)ceil128(Nq) * d.nHb + (size_t)d.nHb * d.nAb +
                          (size_t)ceil128(Er) * d.nHb + (c.n_shared ? n_sgu + n_sd : 0));
  L->expert_bytes = gu_bytes + dn_bytes + sc * (n_sgu + n_sd);

  float* bias = nullptr;
  if (cfg->router_bias) {
    TRY(dalloc_t(L, (size_t)E, &bias));
    TRYC(cudaMemcpy(bias, cfg->router_bias, sizeof(float) * E, cudaMemcpyHostToDevice));
  }
  d.bias = bias;
  d.rbias = bias ? bias + e0 : nullptr;
  d.bias_sel = c.bias_select_only ? 1 : 0;
  d.rscale = c.routed_scale != 0.f ? c.routed_scale : 1.f;

  TRY(dalloc_t(L, (size_t)M * Nq, &d.qkv));
  TRY(dalloc_t(L, (size_t)M * H, &d.h1f));
  TRY(dalloc_t(L, (size_t)M * H, &d.h1b));
  TRY(dalloc_t(L, (size_t)M * E, &d.logits));
  TRY(dalloc_t(L, (size_t)M * k, &d.idx));
  TRY(dalloc_t(L, (size_t)M * k, &d.gates));
  TRY(dalloc_t(L, (size_t)E, &d.counts));
  TRY(dalloc_t(L, (size_t)E + 1, &d.offsets));
  TRY(dalloc_t(L, (size_t)M * k, &d.perm));
  TRY(dalloc_t(L, (size_t)E, &d.active));
  TRY(dalloc_t(L, 1, &d.n_active));
  TRY(dalloc_t(L, (size_t)M * k * I, &d.act));
  TRY(dalloc_t(L, (size_t)M * I, &d.act_sh));
  TRY(dalloc_t(L, (size_t)M * k * H, &d.yr));
  TRY(dalloc_t(L, (size_t)M * H, &d.ysh));
  TRY(dalloc_t(L, 1, &d.rcnt));
  TRY(dalloc_t(L, (size_t)M * H, &d.h1lo));
  TRY(dalloc_t(L, (size_t)M * H, &d.h1lo2));
  TRY(dalloc_t(L, (size_t)M * k * I, &d.act_hi));
  TRY(dalloc_t(L, (size_t)M * k * I, &d.act_lo));
  TRY(dalloc_t(L, (size_t)M * I, &d.act_sh_hi));
  TRY(dalloc_t(L, (size_t)M * I, &d.act_sh_lo));
  if (fp8) {
    // per-64 maxima of the FP8 tensor-core experts' inputs
    TRY(dalloc_t(L, (size_t)M * (H / kQGroup), &d.h1g));
    TRY(dalloc_t(L, (size_t)M * k * (I / kQGroup), &d.actg));
    TRY(dalloc_t(L, (size_t)M * (I / kQGroup), &d.actshg));
  }
  d.resid = d.h1f;
  if (L->tp) {
    TRY(dalloc_t(L, (size_t)M * H, &d.tp_y));
    TRY(dalloc_t(L, (size_t)M * E, &d.tp_lfull));
  }
  if (c.full_layer) {
    L->full = true;
    d.Hq = c.q_heads; d.Hkv = c.kv_heads; d.hd = c.head_dim;
    d.n_seq = c.kv_n_seq; d.max_ctx = c.kv_max_ctx;
    d.k_scale = c.k_scale; d.v_scale = c.v_scale;
    d.eps = c.rms_eps > 0.f ? c.rms_eps : 1e-6f;
    // positions per attention CTA: about two CTAs per SM for one token
    const int grp = c.q_heads / c.kv_heads;
    int want = (2 * L->nsm + c.kv_heads - 1) / c.kv_heads;
    int ch = (c.kv_max_ctx + want - 1) / want;
    ch = std::max(32, std::min(kMaxAttChunk, (ch + 31) & ~31));
    d.att_ch = ch;
    d.att_nch = (c.kv_max_ctx + ch - 1) / ch;
    L->att_smem = attention_smem(ch, grp, c.head_dim);
    uint16_t *g1, *g2;
    TRY(dalloc_t(L, (size_t)H, &g1));
    TRY(dalloc_t(L, (size_t)H, &g2));
    d.g1 = g1; d.g2 = g2;
    TRY(dalloc_t(L, (size_t)M * H, &d.uf));
    TRY(dalloc_t(L, (size_t)M * H, &d.u_hi));
    TRY(dalloc_t(L, (size_t)M * H, &d.u_lo));
    TRY(dalloc_t(L, (size_t)M * Nqkv, &d.qkvf));
    TRY(dalloc_t(L, (size_t)M * A, &d.attnf));
    TRY(dalloc_t(L, (size_t)M * A, &d.attn_hi));
    TRY(dalloc_t(L, (size_t)M * A, &d.attn_lo));
    TRY(dalloc_t(L, (size_t)M * c.kv_heads * d.att_nch * grp * (c.head_dim + 2), &d.att_ws));
    L->att_ncnt = M * c.kv_heads;
    TRY(dalloc_t(L, (size_t)L->att_ncnt, &d.att_cnt));
    TRYC(cudaMemset(d.att_cnt, 0, sizeof(unsigned) * L->att_ncnt));
    TRY(dalloc_t(L, (size_t)M * H, &d.h1r));
    d.resid = d.h1r;
  }
  TRY(dalloc_t(L, (size_t)L->nsm * kWsFloatsPerCta, &d.ws_main));
  TRY(dalloc_t(L, (size_t)L->nsm * kWsFloatsPerCta, &d.ws_side));
  {
    const size_t ntile = std::max<size_t>({(size_t)(E + 4) * (H / 128), (size_t)(E + 1) * (2 * I / 128),
                                           (size_t)(Nq + H) / 128});
    L->ntile = ntile;
    TRY(dalloc_t(L, ntile, &d.tcnt_main));
    TRY(dalloc_t(L, ntile, &d.tcnt_side));
    TRYC(cudaMemset(d.tcnt_main, 0, sizeof(unsigned) * ntile));
    TRYC(cudaMemset(d.tcnt_side, 0, sizeof(unsigned) * ntile));
  }
  TRYC(cudaMemset(d.rcnt, 0, sizeof(unsigned)));
  TRY(dalloc_t(L, 1, &d.err));
  TRYC(cudaMemset(d.err, 0, sizeof(unsigned)));
  TRYC(cudaMemset(d.n_active, 0, sizeof(int)));
  TRYC(cudaMemset(d.ysh, 0, sizeof(float) * (size_t)M * H));

  // weights from the seeded generator
  cudaStream_t gs = nullptr;
  TRYC(cudaStreamCreateWithFlags(&gs, cudaStreamNonBlocking));
  auto gen = [&](uint8_t* dst, float* s, int R, int K, uint32_t kind, uint32_t slot, int mult,
                 int off) { return gen_matrix(L, dst, s, R, K, seed, kind, slot, mult, off, gs); };
  if (!L->tp) {
    rc = gen(wqkv, sqkv, Nq, H, KDG_QKV, 0, 1, 0);
  } else {
    // a shard's QKV rows: its q heads, then k and v of the kv heads they read
    const int hd = c.head_dim;
    const int seg_l[3] = {q0 * hd, (c.q_heads + k0) * hd, (c.q_heads + c.kv_heads + k0) * hd};
    const int seg_n[3] = {(q1 - q0) * hd, (k1 - k0) * hd, (k1 - k0) * hd};
    int r0 = 0;
    for (int g = 0; g < 3 && rc == KD_OK; ++g) {
      rc = gen_matrix(L, wqkv + (size_t)r0 * H * eb, sqkv ? sqkv + (size_t)(r0 / 128) * d.nHb : nullptr,
                      seg_n[g], H, seed, KDG_QKV, 0, 1, 0, gs, seg_l[g], 0, H);
      r0 += seg_n[g];
    }
  }
  if (rc == KD_OK)
    rc = gen_matrix(L, wo, so, H, A_, seed, KDG_OPROJ, 0, 1, 0, gs, 0, L->attn_col0, A);
  if (rc == KD_OK) rc = gen_matrix(L, wr, sr, Er, H, seed, KDG_ROUTER, 0, 1, 0, gs, e0, 0, H);
  for (int e = (c.n_shared ? -1 : 0); e < E && rc == KD_OK; ++e) {
    uint8_t* gu = e < 0 ? wgu_sh : wgu + (size_t)e * gu_bytes;
    uint8_t* dn = e < 0 ? wd_sh : wd + (size_t)e * dn_bytes;
    float* sg = fp8 ? (e < 0 ? sgu_sh : sgu + (size_t)e * n_sgu) : nullptr;
    float* sdn = fp8 ? (e < 0 ? sd_sh : sd + (size_t)e * n_sd) : nullptr;
    const uint32_t slot = (uint32_t)(e + 1);
    // (a shard: intermediate rows [i0, i0 + I) of gate and up, those columns of down)
    rc = gen_matrix(L, gu, sg, I, H, seed, KDG_GATE, slot, 2, 0, gs, i0, 0, H);
    if (rc == KD_OK)
      rc = gen_matrix(L, gu, sg ? sg + (size_t)d.nIb * d.nHb : nullptr, I, H, seed, KDG_UP, slot, 2, 1,
                      gs, i0, 0, H);
    if (rc == KD_OK) rc = gen_matrix(L, dn, sdn, H, I, seed, KDG_DOWN, slot, 1, 0, gs, 0, i0, c.inter);
  }
  if (rc == KD_OK && c.full_layer) {
    gen_norm_kernel<<<32, 256, 0, gs>>>(const_cast<uint16_t*>(d.g1), H,
                                        kdg_stream(seed, kdg_uid((uint32_t)c.layer_id, KDG_NORM1, 0)));
    gen_norm_kernel<<<32, 256, 0, gs>>>(const_cast<uint16_t*>(d.g2), H,
                                        kdg_stream(seed, kdg_uid((uint32_t)c.layer_id, KDG_NORM2, 0)));
    if (cudaGetLastError() != cudaSuccess) rc = fail(KD_ECUDA, "kd_layer_create: norm generator%s", "");
  }
  cudaError_t se = cudaStreamSynchronize(gs);
  cudaStreamDestroy(gs);
  if (rc != KD_OK) { free_layer(L); return rc; }
  TRYC(se);

  {
    bool ok = encode_weight_map(&L->maps.m[0], wqkv, Nq, H, fp8) &&
              encode_weight_map(&L->maps.m[1], wo, H, A_, fp8) &&
              encode_weight_map(&L->maps.m[2], wgu, (uint64_t)E * 2 * I, H, fp8) &&
              encode_weight_map(&L->maps.m[3], wd, (uint64_t)E * H, I, fp8) &&
              encode_weight_map(&L->maps.m[6], wr, Er, H, fp8);
    if (ok && c.n_shared)
      ok = encode_weight_map(&L->maps.m[4], wgu_sh, 2 * I, H, fp8) &&
           encode_weight_map(&L->maps.m[5], wd_sh, H, I, fp8);
    L->has_maps = ok;
  }

  TRYC(cudaStreamCreateWithFlags(&L->side, cudaStreamNonBlocking));
  TRYC(cudaEventCreateWithFlags(&L->ev_h1, cudaEventDisableTiming));
  TRYC(cudaEventCreateWithFlags(&L->ev_sh, cudaEventDisableTiming));
  d.err = d.err;
  *out = L;
  return KD_OK;
#undef TRY
#undef TRYC
}

extern "C" void kd_layer_destroy(kd_layer* L) {
  if (!L) return;
  cudaDeviceSynchronize();
  free_layer(L);
}

// ------------------------------------------------------------------ decode

static int prefetch_static(const kd_layer* L, size_t max_bytes, cudaStream_t s);

// Launch with programmatic stream serialization: the kernel may start while
// the preceding kernel in the stream finishes; it waits (griddepcontrol.wait)
// before reading anything that kernel wrote.
template <typename... KArgs, typename... Args>
static cudaError_t launch(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                          cudaStream_t s, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

static int launch_layer(kd_layer* L, const Acts& a, cudaStream_t s, const kd_layer* prefetch_next,
                        cudaStream_t pf, cudaEvent_t ev_fork, cudaEvent_t ev_join, bool pdl_first);

extern "C" int kd_decode_layer(kd_layer* L, void* hidden, const void* attn, int M, void* stream) {
  if (!L || !hidden || !attn) return fail(KD_EINVAL, "kd_decode_layer: null argument%s", "");
  if (L->tp) return fail(KD_EINVAL, "kd_decode_layer: a tensor-parallel shard takes kd_tp_*%s", "");
  if (M < 1 || M > L->maxM)
    return fail(KD_ERANGE, "kd_decode_layer: M=%s%ld outside 1..max_tokens", "", (long)M);
  Acts a{};
  a.x = static_cast<const uint16_t*>(hidden);
  a.attn = static_cast<const uint16_t*>(attn);
  a.out = static_cast<uint16_t*>(hidden);
  a.M = M;
  return launch_layer(L, a, static_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, nullptr,
                      false);
}

extern "C" int kd_decode_layer_full(kd_layer* L, void* hidden, void* k_cache, void* v_cache,
                                    const int* seq, const int* pos, int M, void* stream) {
  if (!L || !hidden || !k_cache || !v_cache || !seq || !pos)
    return fail(KD_EINVAL, "kd_decode_layer_full: null argument%s", "");
  if (!L->full)
    return fail(KD_EINVAL, "kd_decode_layer_full: the layer was created without full_layer%s", "");
  if (M < 1 || M > L->maxM)
    return fail(KD_ERANGE, "kd_decode_layer_full: M=%s%ld outside 1..max_tokens", "", (long)M);
  Acts a{};
  a.x = static_cast<const uint16_t*>(hidden);
  a.attn = nullptr;
  a.out = static_cast<uint16_t*>(hidden);
  a.M = M;
  a.kc = static_cast<uint8_t*>(k_cache);
  a.vc = static_cast<uint8_t*>(v_cache);
  a.seq = seq;
  a.pos = pos;
  return launch_layer(L, a, static_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, nullptr,
                      false);
}

// The tensor-core expert kernels for the layer's weight format.
using GateupMmaFn = void (*)(LayerDev, int, int, const MmaMaps);
using DownMmaFn = void (*)(LayerDev, int, const MmaMaps);
static GateupMmaFn gateup_mma_for(const kd_layer* L) {
  if (L->cfg.wdtype != KD_WFP8) return mma_gateup_kernel<false>;
  return L->w8a8 ? mma_gateup_kernel<true, 1> : mma_gateup_kernel<true>;
}
static DownMmaFn down_mma_for(const kd_layer* L) {
  if (L->cfg.wdtype != KD_WFP8) return mma_down_kernel<false>;
  return L->w8a8 ? mma_down_kernel<true, 1> : mma_down_kernel<true>;
}

// The front of the layer up to h1 (and, in the full layer, the MoE input
// w = RMSNorm(h1) g2): the chain with a given attn_out runs QKV and o-proj in
// one launch; the full layer runs RMSNorm -> QKV (+ KV cache append) ->
// attention -> o-proj + residual -> RMSNorm.
static int launch_front(kd_layer* L, const Acts& a, cudaStream_t s, bool pdl_first) {
  const LayerDev& d = L->d;
  const bool fp8 = L->cfg.wdtype == KD_WFP8;
  const int G = L->nsm, M = a.M;
  const bool mma = L->has_maps && M >= L->mma_min;
  const int pthreads = fp8 ? kMThreadsF8 : kMThreads;
  if (!L->full) {
    if (mma)
      KD_CUDA(launch(fp8 ? mma_proj_kernel<true> : mma_proj_kernel<false>, G, pthreads, kMmaSmem, s,
                     pdl_first, d, a, L->maps));
    else
      KD_CUDA(launch(fp8 ? proj_kernel<W_FP8> : proj_kernel<W_BF16>, G, kThreads, kStreamSmem, s,
                     pdl_first, d, a));
    return KD_OK;
  }
  KD_CUDA(launch(rmsnorm_in_kernel, M, kNormThreads, 0, s, pdl_first, d, a));
  if (mma)
    KD_CUDA(launch(fp8 ? mma_proj_kernel<true, 1> : mma_proj_kernel<false, 1>, G, pthreads, kMmaSmem,
                   s, true, d, a, L->maps));
  else
    KD_CUDA(launch(fp8 ? proj_kernel<W_FP8, 1> : proj_kernel<W_BF16, 1>, G, kThreads, kStreamSmem, s,
                   true, d, a));
  KD_CUDA(launch(attention_for(d.hd, d.Hq / d.Hkv), M * d.Hkv * d.att_nch, 256, L->att_smem, s,
                 true, d, a));
  if (mma)
    KD_CUDA(launch(fp8 ? mma_proj_kernel<true, 2> : mma_proj_kernel<false, 2>, G, pthreads, kMmaSmem,
                   s, true, d, a, L->maps));
  else
    KD_CUDA(launch(fp8 ? proj_kernel<W_FP8, 2> : proj_kernel<W_BF16, 2>, G, kThreads, kStreamSmem, s,
                   true, d, a));
  KD_CUDA(launch(rmsnorm_moe_kernel, M, kNormThreads, 0, s, true, d, (int)(fp8 && mma)));
  return KD_OK;
}

static int launch_layer(kd_layer* L, const Acts& a, cudaStream_t s, const kd_layer* next,
                        cudaStream_t pf, cudaEvent_t ev_fork, cudaEvent_t ev_join, bool pdl_first) {
  const LayerDev& d = L->d;
  const bool fp8 = L->cfg.wdtype == KD_WFP8;
  const int M = a.M;
  const int G = L->nsm;
  const size_t sm = kStreamSmem;
  const bool mma = L->has_maps && M >= L->mma_min;
  const size_t msm = kMmaSmem;
  // FP8 projections convert their e4m3 tiles (converter warps); the FP8
  // experts multiply them as they land (with kQ8Conv converter warps for
  // their activation terms)
  const int mthreads = kMThreads;
  const int gthreads = fp8 ? q8_threads(kGateUpConv) : kMThreads;
  const int dthreads = fp8 ? q8_threads(kDownConv) : kMThreads;
  if (L->timing) KD_CUDA(cudaEventRecord(L->tev[0], s));
  // Main stream: projections -> router (logits, selection, token lists in one
  // launch) -> routed gate/up -> down + combine.  Side stream: the shared
  // expert's gate/up, from the end of the projections, joined by an event
  // before the down kernel.  The router releases its dependent launch only
  // when it is done, so the shared gate/up gets the SMs that the router
  // leaves free while the router runs.
  const size_t route_ints = sizeof(int) * kSelectSmemInts(d.E, M * d.k);
  {
    const int rc = launch_front(L, a, s, pdl_first);
    if (rc != KD_OK) return rc;
  }
  if (L->timing) KD_CUDA(cudaEventRecord(L->tev[1], s));
  if (d.S) KD_CUDA(cudaEventRecord(L->ev_h1, s));

  // Up to kCoreRouterMaxM tokens the CUDA-core router (one CTA per two
  // experts) is the faster one: the tensor-core router's small grid is a
  // latency chain.  FP8 router weights go to the tensor cores as exact bf16
  // with the block scale on h1's three terms (the converter warps).
  if (mma && M > kCoreRouterMaxM) {
    const int rsub = fp8 ? 2 : mma_nsub(M, 3);
    const int rchunks = ((d.E + 127) / 128) * (d.H / (64 * rsub));
    const int rgrid = std::max(1, std::min(G, rchunks / (kRouterChunksPerCta * 2 / rsub)));
    if (fp8)
      KD_CUDA(launch(mma_router_kernel<true>, rgrid, kMThreadsF8, msm, s, !L->timing, d, M, L->maps));
    else
      KD_CUDA(launch(mma_router_kernel<false>, rgrid, mthreads, msm, s, !L->timing, d, M, L->maps));
  } else {
    const int rgrid = (d.E + kRouterRows - 1) / kRouterRows;
    KD_CUDA(launch(fp8 ? router_kernel<W_FP8> : router_kernel<W_BF16>, rgrid, kRouterThreads,
                   route_ints, s, !L->timing, d, M));
  }
  if (d.S) {
    KD_CUDA(cudaStreamWaitEvent(L->side, L->ev_h1, 0));
    // one CTA fewer than SMs: the router's last CTA holds its SM for the
    // selection, and a shared gate/up CTA waiting for that SM would start
    // (and end) late and delay the routed gate/up CTA that follows it there
    // (per-CTA clocks: routed starts spread 75-87 us -> 75-76 us at batch 1)
    if (mma)
      KD_CUDA(launch(gateup_mma_for(L), std::max(1, G - 1), gthreads, msm,
                     L->side, false, d, M, 1, L->maps));
    else
      KD_CUDA(launch(fp8 ? gateup_kernel<W_FP8> : gateup_kernel<W_BF16>, G, kThreads, sm, L->side,
                     false, d, M, 1));
    KD_CUDA(cudaEventRecord(L->ev_sh, L->side));
  }
  if (L->timing) KD_CUDA(cudaEventRecord(L->tev[2], s));
  if (mma)
    KD_CUDA(launch(gateup_mma_for(L), G, gthreads, msm, s,
                   !L->timing, d, M, 0, L->maps));
  else
    KD_CUDA(launch(fp8 ? gateup_kernel<W_FP8> : gateup_kernel<W_BF16>, G, kThreads,
                   gateup_smem(d, M), s, !L->timing, d, M, 0));
  if (L->timing) KD_CUDA(cudaEventRecord(L->tev[3], s));
  if (d.S) KD_CUDA(cudaStreamWaitEvent(s, L->ev_sh, 0));
  if (next && pf) {
    // the next layer's static weights into L2 while this layer finishes
    KD_CUDA(cudaEventRecord(ev_fork, s));
    KD_CUDA(cudaStreamWaitEvent(pf, ev_fork, 0));
    int rc = prefetch_static(next, 0, pf);
    if (rc != KD_OK) return rc;
    KD_CUDA(cudaEventRecord(ev_join, pf));
  }
  const bool pdl_down = !L->timing && !d.S && !(next && pf);
  if (mma) {
    // tensor-core down writes each expert's outputs; the combine follows
    KD_CUDA(launch(down_mma_for(L), G, dthreads, msm, s,
                   pdl_down, d, M, L->maps));
    KD_CUDA(launch(combine_kernel, 2 * G, 256, 0, s, !L->timing, d, M, a.out));
  } else {
    // the CUDA-core down writes each expert's outputs too; the combine follows
    KD_CUDA(launch(fp8 ? down_kernel<W_FP8> : down_kernel<W_BF16>, G, kThreads, sm, s, pdl_down, d,
                   M));
    KD_CUDA(launch(combine_kernel, 2 * G, 256, 0, s, !L->timing, d, M, a.out));
  }
  if (L->timing) KD_CUDA(cudaEventRecord(L->tev[4], s));
  if (next && pf) KD_CUDA(cudaStreamWaitEvent(s, ev_join, 0));
  return KD_OK;
}

// ------------------------------------------------------------------ tensor parallel

static int tp_args(const kd_layer* L, int M, const char* fn) {
  if (!L || !L->tp) return fail(KD_EINVAL, "%s: not a tensor-parallel shard", fn);
  if (M < 1 || M > L->maxM) return fail(KD_ERANGE, "%s: M outside 1..max_tokens", fn);
  return KD_OK;
}

extern "C" int kd_tp_buffers(const kd_layer* L, float** p, float** lshard, float** lfull, float** y) {
  if (!L || !L->tp || !p || !lshard || !lfull || !y)
    return fail(KD_EINVAL, "kd_tp_buffers: bad arguments%s", "");
  *p = L->d.h1f;
  *lshard = L->d.logits;
  *lfull = L->d.tp_lfull;
  *y = L->d.tp_y;
  return KD_OK;
}

// Phase 1: the shard's QKV rows and o-proj partial sum (into h1f).
extern "C" int kd_tp_attn(kd_layer* L, const void* hidden, const void* attn, int M, void* stream) {
  int rc = tp_args(L, M, "kd_tp_attn");
  if (rc != KD_OK) return rc;
  if (!hidden || !attn) return fail(KD_EINVAL, "kd_tp_attn: null argument%s", "");
  Acts a{};
  a.x = static_cast<const uint16_t*>(hidden);
  a.attn = static_cast<const uint16_t*>(attn) + L->attn_col0;   // row stride: d.attn_ld
  a.M = M;
  return launch_front(L, a, static_cast<cudaStream_t>(stream), false);
}

// Phase 2: h1 = x + the summed partials; the shard's router logits.
extern "C" int kd_tp_router(kd_layer* L, const void* hidden, int M, void* stream) {
  int rc = tp_args(L, M, "kd_tp_router");
  if (rc != KD_OK) return rc;
  if (!hidden) return fail(KD_EINVAL, "kd_tp_router: null argument%s", "");
  const LayerDev& d = L->d;
  const bool fp8 = L->cfg.wdtype == KD_WFP8;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int ng = M * (d.H / 64);
  KD_CUDA(launch(tp_h1_kernel, (ng + 255) / 256, 256, 0, s, false, d,
                 static_cast<const uint16_t*>(hidden), M, (int)fp8));
  const int rgrid = (d.Er + kRouterRows - 1) / kRouterRows;
  KD_CUDA(launch(fp8 ? router_kernel<W_FP8> : router_kernel<W_BF16>, rgrid, kRouterThreads, 0, s,
                 false, d, M));
  return KD_OK;
}

// Phase 3: the selection from the gathered logits, then the shard's rows of
// the experts (shared on the side stream, as in the whole layer) -> tp_y.
extern "C" int kd_tp_moe(kd_layer* L, int M, void* stream) {
  int rc = tp_args(L, M, "kd_tp_moe");
  if (rc != KD_OK) return rc;
  const LayerDev& d = L->d;
  const bool fp8 = L->cfg.wdtype == KD_WFP8;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int G = L->nsm;
  const bool mma = L->has_maps && M >= L->mma_min;
  const size_t route_ints = sizeof(int) * kSelectSmemInts(d.E, M * d.k);
  KD_CUDA(launch(tp_route_kernel, 1, kRouterThreads, route_ints, s, false, d, M));
  const int gthreads = fp8 ? q8_threads(kGateUpConv) : kMThreads;
  const int dthreads = fp8 ? q8_threads(kDownConv) : kMThreads;
  if (d.S) {
    KD_CUDA(cudaEventRecord(L->ev_h1, s));
    KD_CUDA(cudaStreamWaitEvent(L->side, L->ev_h1, 0));
    if (mma)
      KD_CUDA(launch(gateup_mma_for(L), G, gthreads, kMmaSmem,
                     L->side, false, d, M, 1, L->maps));
    else
      KD_CUDA(launch(fp8 ? gateup_kernel<W_FP8> : gateup_kernel<W_BF16>, G, kThreads, kStreamSmem,
                     L->side, false, d, M, 1));
    KD_CUDA(cudaEventRecord(L->ev_sh, L->side));
  }
  if (mma)
    KD_CUDA(launch(gateup_mma_for(L), G, gthreads, kMmaSmem, s,
                   false, d, M, 0, L->maps));
  else
    KD_CUDA(launch(fp8 ? gateup_kernel<W_FP8> : gateup_kernel<W_BF16>, G, kThreads,
                   gateup_smem(d, M), s, false, d, M, 0));
  if (d.S) KD_CUDA(cudaStreamWaitEvent(s, L->ev_sh, 0));
  if (mma) {
    KD_CUDA(launch(down_mma_for(L), G, dthreads, kMmaSmem, s,
                   false, d, M, L->maps));
    KD_CUDA(launch(combine_kernel, 2 * G, 256, 0, s, false, d, M, (uint16_t*)nullptr));
  } else {
    KD_CUDA(launch(fp8 ? down_kernel<W_FP8> : down_kernel<W_BF16>, G, kThreads, kStreamSmem, s, false,
                   d, M));
    KD_CUDA(launch(combine_kernel, 2 * G, 256, 0, s, false, d, M, (uint16_t*)nullptr));
  }
  return KD_OK;
}

// Phase 4: hidden = bf16(h1 + the summed expert partials).
extern "C" int kd_tp_combine(kd_layer* L, void* hidden, int M, void* stream) {
  int rc = tp_args(L, M, "kd_tp_combine");
  if (rc != KD_OK) return rc;
  if (!hidden) return fail(KD_EINVAL, "kd_tp_combine: null argument%s", "");
  KD_CUDA(launch(tp_final_kernel, 2 * L->nsm, 256, 0, static_cast<cudaStream_t>(stream), false, L->d,
                 static_cast<uint16_t*>(hidden), M));
  return KD_OK;
}

extern "C" int kd_layer_check(kd_layer* L) {
  if (!L) return fail(KD_EINVAL, "kd_layer_check: null layer%s", "");
  KD_CUDA(cudaDeviceSynchronize());
  unsigned e = 0;
  KD_CUDA(cudaMemcpy(&e, L->d.err, sizeof e, cudaMemcpyDeviceToHost));
  if (e == 0) return KD_OK;
  KD_CUDA(cudaMemset(L->d.err, 0, sizeof(unsigned)));
  // an aborted call may have left arrival counters part-way
  KD_CUDA(cudaMemset(L->d.rcnt, 0, sizeof(unsigned)));
  KD_CUDA(cudaMemset(L->d.tcnt_main, 0, sizeof(unsigned) * L->ntile));
  KD_CUDA(cudaMemset(L->d.tcnt_side, 0, sizeof(unsigned) * L->ntile));
  if (L->full) KD_CUDA(cudaMemset(L->d.att_cnt, 0, sizeof(unsigned) * L->att_ncnt));
  if (e & (ERR_WAIT_FULL | ERR_WAIT_EMPTY | ERR_WAIT_MMA))
    return fail(KD_ETIMEOUT, "device: a bounded wait gave up (flags %s0x%lx)", "", (long)e);
  return fail(KD_EDEVICE, "device error flags %s0x%lx", "", (long)e);
}

extern "C" int kd_layer_set_timing_events(kd_layer* L, void* const* events, int n) {
  if (!L || (n != 0 && n != KD_N_TIMING_EVENTS) || (n && !events))
    return fail(KD_EINVAL, "kd_layer_set_timing_events: bad arguments%s", "");
  L->timing = n != 0;
  for (int i = 0; i < KD_N_TIMING_EVENTS; ++i)
    L->tev[i] = n ? static_cast<cudaEvent_t>(events[i]) : nullptr;
  return KD_OK;
}

extern "C" const void* kd_layer_qkv(const kd_layer* L) { return L ? L->d.qkv : nullptr; }

// ------------------------------------------------------------------ L2 prefetch

__global__ void prefetch_kernel(const uint8_t* p0, size_t n0, const uint8_t* p1, size_t n1,
                                const uint8_t* p2, size_t n2, const uint8_t* p3, size_t n3,
                                size_t budget) {
  constexpr size_t kChunk = 32768;
  const uint8_t* ps[4] = {p0, p1, p2, p3};
  size_t ns[4] = {n0, n1, n2, n3};
  size_t base = 0;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t nth = (size_t)gridDim.x * blockDim.x;
  for (int r = 0; r < 4; ++r) {
    if (!ps[r]) continue;
    size_t n = ns[r];
    if (base + n > budget) n = budget > base ? budget - base : 0;
    const size_t nch = (n + kChunk - 1) / kChunk;
    for (size_t c = tid; c < nch; c += nth) {
      const size_t off = c * kChunk;
      size_t len = n - off < kChunk ? n - off : kChunk;
      len &= ~size_t(15);
      if (len) bulk_prefetch_l2(ps[r] + off, (uint32_t)len);
    }
    base += ns[r];
  }
}

static int prefetch_static(const kd_layer* L, size_t max_bytes, cudaStream_t s) {
  const LayerDev& d = L->d;
  const size_t budget = max_bytes ? max_bytes : L->l2_bytes;
  const size_t bqkv = (size_t)d.Nqkv * d.H * d.eb, bo = (size_t)d.H * d.A * d.eb,
               br = (size_t)d.E * d.H * d.eb, bsh = (size_t)2 * d.I * d.H * d.eb;
  prefetch_kernel<<<L->nsm, 128, 0, s>>>(d.wqkv, bqkv, d.wo, bo, d.wr, br, d.wgu_sh,
                                         d.S ? bsh : 0, budget);
  KD_CUDA(cudaGetLastError());
  return KD_OK;
}

extern "C" int kd_layer_prefetch_l2(const kd_layer* L, size_t max_bytes, void* stream) {
  if (!L) return fail(KD_EINVAL, "kd_layer_prefetch_l2: null layer%s", "");
  return prefetch_static(L, max_bytes, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------ introspection

extern "C" int kd_layer_debug_tensor(const kd_layer* L, int which, void** p) {
  if (!L || !p) return fail(KD_EINVAL, "kd_layer_debug_tensor: null argument%s", "");
  const LayerDev& d = L->d;
  switch (which) {
    case KD_T_H1F: *p = d.h1f; break;
    case KD_T_H1B: *p = d.h1b; break;
    case KD_T_LOGITS: *p = d.logits; break;
    case KD_T_IDX: *p = d.idx; break;
    case KD_T_GATES: *p = d.gates; break;
    case KD_T_COUNTS: *p = d.counts; break;
    case KD_T_NACTIVE: *p = d.n_active; break;
    case KD_T_YSHARED: *p = d.ysh; break;
    case KD_T_YROUTED: *p = d.yr; break;
    case KD_T_ATTN: *p = d.attnf; break;
    case KD_T_RESID: *p = d.h1r; break;
    case KD_T_ACT: *p = d.act; break;
    case KD_T_ACTSH: *p = d.act_sh; break;

    default: return fail(KD_EINVAL, "kd_layer_debug_tensor: unknown tensor %s%ld", "", (long)which);
  }
  return KD_OK;
}

extern "C" int kd_layer_read_weight(const kd_layer* L, int kind, int expert, int row0, int nrows,
                                    void* dst, float* dst_scales) {
  if (!L || !dst) return fail(KD_EINVAL, "kd_layer_read_weight: null argument%s", "");
  const LayerDev& d = L->d;
  const int eb = d.eb;
  const bool fp8 = eb == 1;
  const uint8_t* base = nullptr;
  const float* sbase = nullptr;
  int R = 0, K = 0, mult = 1, off = 0;
  if (expert < -1 || expert >= d.E || (expert == -1 && kind >= 4 && !d.S))
    return fail(KD_EINVAL, "kd_layer_read_weight: bad expert %s%ld", "", (long)expert);
  const size_t gu = (size_t)2 * d.I * d.H * eb, dn = (size_t)d.H * d.I * eb;
  const size_t n_sgu = (size_t)2 * d.nIb * d.nHb, n_sd = (size_t)d.nHb * d.nIb;
  switch (kind) {
    case 1: base = d.wqkv; sbase = d.sqkv; R = d.Nqkv; K = d.H; break;
    case 2: base = d.wo; sbase = d.so; R = d.H; K = d.A; break;
    case 3: base = d.wr; sbase = d.sr; R = d.E; K = d.H; break;
    case 4:
    case 5:
      base = expert < 0 ? d.wgu_sh : d.wgu + (size_t)expert * gu;
      sbase = expert < 0 ? d.sgu_sh : (d.sgu ? d.sgu + (size_t)expert * n_sgu : nullptr);
      if (sbase && kind == 5) sbase += (size_t)d.nIb * d.nHb;
      R = d.I; K = d.H; mult = 2; off = kind == 5 ? 1 : 0;
      break;
    case 6:
      base = expert < 0 ? d.wd_sh : d.wd + (size_t)expert * dn;
      sbase = expert < 0 ? d.sd_sh : (d.sd ? d.sd + (size_t)expert * n_sd : nullptr);
      R = d.H; K = d.I;
      break;
    default: return fail(KD_EINVAL, "kd_layer_read_weight: bad kind %s%ld", "", (long)kind);
  }
  if (row0 < 0 || nrows < 0 || row0 + nrows > R)
    return fail(KD_EINVAL, "kd_layer_read_weight: rows out of range%s", "");
  if (nrows == 0) return KD_OK;
  const size_t rb = (size_t)K * eb;
  KD_CUDA(cudaMemcpy2D(dst, rb, base + ((size_t)row0 * mult + off) * rb, rb * mult, rb, nrows,
                       cudaMemcpyDeviceToHost));
  if (fp8 && dst_scales) {
    const int b0 = row0 / 128, b1 = (row0 + nrows - 1) / 128, nkb = ceil128(K);
    KD_CUDA(cudaMemcpy(dst_scales, sbase + (size_t)b0 * nkb, sizeof(float) * (b1 - b0 + 1) * nkb,
                       cudaMemcpyDeviceToHost));
  }
  return KD_OK;
}

extern "C" int kd_layer_launches(const kd_layer* L, int M) {
  if (!L) return fail(KD_EINVAL, "kd_layer_launches: null layer%s", "");
  if (M < 1 || M > L->maxM)
    return fail(KD_ERANGE, "kd_layer_launches: M=%s%ld outside 1..max_tokens", "", (long)M);
  // projections, router, routed gate/up, down, combine, + the shared
  // expert's gate/up; a full layer runs RMSNorm, QKV, attention, o-proj and
  // RMSNorm in place of the projections' launch (the same for every M)
  return 5 + (L->d.S ? 1 : 0) + (L->full ? 4 : 0);
}

extern "C" int kd_layer_bytes(const kd_layer* L, uint64_t* static_bytes, uint64_t* expert_bytes) {
  if (!L) return fail(KD_EINVAL, "kd_layer_bytes: null layer%s", "");
  if (static_bytes) *static_bytes = L->static_bytes;
  if (expert_bytes) *expert_bytes = L->expert_bytes;
  return KD_OK;
}

// ------------------------------------------------------------------ stack + graph

extern "C" int kd_stack_create(kd_layer* const* layers, int n, int M, int prefetch, kd_stack** out) {
  if (!layers || !out || n < 1) return fail(KD_EINVAL, "kd_stack_create: bad arguments%s", "");
  *out = nullptr;
  for (int i = 0; i < n; ++i) {
    if (!layers[i]) return fail(KD_EINVAL, "kd_stack_create: null layer%s", "");
    if (layers[i]->tp) return fail(KD_EINVAL, "kd_stack_create: a tensor-parallel shard%s", "");
    if (M < 1 || M > layers[i]->maxM)
      return fail(KD_ERANGE, "kd_stack_create: M=%s%ld outside a layer's 1..max_tokens", "", (long)M);
    if (layers[i]->d.H != layers[0]->d.H || layers[i]->d.A != layers[0]->d.A)
      return fail(KD_EINVAL, "kd_stack_create: layers of different widths%s", "");
  }
  kd_stack* S = new kd_stack();
  S->layers.assign(layers, layers + n);
  S->M = M;
  S->prefetch = prefetch;
  auto bad = [&](cudaError_t e) {
    if (S->cap) cudaStreamDestroy(S->cap);
    if (S->pf) cudaStreamDestroy(S->pf);
    for (auto ev : S->ev_fork) cudaEventDestroy(ev);
    for (auto ev : S->ev_join) cudaEventDestroy(ev);
    delete S;
    return fail(KD_ECUDA, "kd_stack_create: %s", cudaGetErrorString(e));
  };
  cudaError_t e;
  if ((e = cudaStreamCreateWithFlags(&S->cap, cudaStreamNonBlocking)) != cudaSuccess) return bad(e);
  if ((e = cudaStreamCreateWithFlags(&S->pf, cudaStreamNonBlocking)) != cudaSuccess) return bad(e);
  for (int i = 0; i < n; ++i) {
    cudaEvent_t a, b;
    if ((e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming)) != cudaSuccess) return bad(e);
    S->ev_fork.push_back(a);
    if ((e = cudaEventCreateWithFlags(&b, cudaEventDisableTiming)) != cudaSuccess) return bad(e);
    S->ev_join.push_back(b);
  }
  *out = S;
  return KD_OK;
}

static void stack_drop_graph(kd_stack* S) {
  if (S->exec) cudaGraphExecDestroy(S->exec);
  if (S->graph) cudaGraphDestroy(S->graph);
  S->exec = nullptr;
  S->graph = nullptr;
}

extern "C" int kd_stack_run(kd_stack* S, void* hidden, const void* attn, void* stream) {
  if (!S || !hidden || !attn) return fail(KD_EINVAL, "kd_stack_run: null argument%s", "");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!S->exec || S->hidden != hidden || S->attn != attn) {
    stack_drop_graph(S);
    KD_CUDA(cudaStreamBeginCapture(S->cap, cudaStreamCaptureModeThreadLocal));
    const int n = (int)S->layers.size();
    int rc = KD_OK;
    for (int l = 0; l < n && rc == KD_OK; ++l) {
      kd_layer* L = S->layers[l];
      Acts a{};
      a.x = static_cast<const uint16_t*>(hidden);
      a.attn = reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(attn) +
                                                 (size_t)l * S->M * L->d.A * 2);
      a.out = static_cast<uint16_t*>(hidden);
      a.M = S->M;
      const kd_layer* next = (S->prefetch && l + 1 < n) ? S->layers[l + 1] : nullptr;
      rc = launch_layer(L, a, S->cap, next, next ? S->pf : nullptr, S->ev_fork[l], S->ev_join[l],
                        l > 0);
    }
    cudaGraph_t g = nullptr;
    cudaError_t ce = cudaStreamEndCapture(S->cap, &g);
    if (rc != KD_OK) {
      if (g) cudaGraphDestroy(g);
      return rc;
    }
    KD_CUDA(ce);
    S->graph = g;
    KD_CUDA(cudaGraphInstantiate(&S->exec, g, 0));
    S->hidden = hidden;
    S->attn = attn;
  }
  KD_CUDA(cudaGraphLaunch(S->exec, s));
  return KD_OK;
}

extern "C" void kd_stack_destroy(kd_stack* S) {
  if (!S) return;
  cudaDeviceSynchronize();
  stack_drop_graph(S);
  if (S->cap) cudaStreamDestroy(S->cap);
  if (S->pf) cudaStreamDestroy(S->pf);
  for (auto ev : S->ev_fork) cudaEventDestroy(ev);
  for (auto ev : S->ev_join) cudaEventDestroy(ev);
  delete S;
}

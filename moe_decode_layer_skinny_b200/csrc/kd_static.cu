// kd_static.cu -- router top-k entry point that allocates no device memory.
//
// For callers that cannot call cudaMalloc from where they run this code: for
// example a host runtime whose device memory is entirely owned by another
// allocator (a framework's caching allocator, an inference engine that hands
// plugins only their input and output buffers), or code that may only enqueue
// work.  The logits and the per-expert lists that the blocks of this
// router's one launch hand to each other live in one file-scope __device__
// array of fixed size instead of a cudaMalloc'd workspace.
//
// The array exists once per device for the life of the process.  Host code
// may not pass the array's name to a kernel (on the host it names a stand-in,
// not the device address): the device address is looked up with
// cudaGetSymbolAddress on the first call in each CUDA context (device), with
// that device current, and cached together with the context; a call in a new
// context (after cudaDeviceReset, say) looks it up again.  All calls share
// the array: two calls that overlap on the GPU (different streams, or
// different host threads) race on it.
//
// Device-side errors are not reported: the launch has no bounded waits, and
// the one error flag its selection code can raise (an expert id out of range,
// which finite logits cannot produce) stays in the scratch.  The block
// counter returns to zero at the end of every launch; a launch cannot stop
// part-way short of a fault, which loses the context and the array with it.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/kd.h"
#include "kd_kernels.cuh"

using namespace kd;

namespace {

constexpr int kMaxTok = KD_STATIC_MAX_TOKENS;
constexpr int kMaxExp = KD_STATIC_MAX_EXPERTS;
constexpr int kMaxK = 16;
constexpr int kMaxHidden = 8192;   // router rows held in registers (16-byte chunks per lane)

// logits [64 x 1024] | counts [1024] | offsets [1025] | active [1024]
// | perm [64 x 16] | n_active [1] | err [1] | router blocks done [1]   (4-byte words)
constexpr size_t kWords = (size_t)kMaxTok * kMaxExp + kMaxExp + (kMaxExp + 1) + kMaxExp +
                          (size_t)kMaxTok * kMaxK + 3;

// Every scratch word is written before it is read within a call (logits by
// the logit blocks, lists by the selection), so nothing needs clearing; the
// block-completion counter starts at zero (static storage) and the last
// block of every call puts it back to zero.
static __device__ __align__(256) float g_router_scratch[kWords];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};   // the context the cached address belongs to

// cuCtxGetCurrent through the runtime's driver entry point (no libcuda link).
typedef int (*CtxGetCurrentFn)(void**);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static bool looked = false;
  if (!looked) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
    looked = true;
  }
  return fn;
}

thread_local char g_msg[256];
}  // namespace

// kd_last_error() reports these messages too (defined with the layer API).
void kd_set_last_error(const char* msg);

namespace {
int fail_static(int code) {
  kd_set_last_error(g_msg);
  return code;
}
}  // namespace

extern "C" int kd_router_topk_static(const void* router_w, const float* router_scales,
                                     int wdtype, const float* router_bias, const float* h1,
                                     int M, int hidden, int n_experts, int top_k, int* idx_out,
                                     float* gates_out, void* stream) {
  if (!router_w || !h1 || !idx_out || !gates_out || (wdtype == KD_WFP8 && !router_scales) ||
      (wdtype != KD_WBF16 && wdtype != KD_WFP8) || hidden <= 0 || hidden % 128 || top_k < 1) {
    snprintf(g_msg, sizeof g_msg, "kd_router_topk_static: null pointer or unsupported shape");
    return fail_static(KD_EINVAL);
  }
  if (M < 1 || M > kMaxTok || n_experts < top_k || n_experts > kMaxExp || top_k > kMaxK ||
      hidden > kMaxHidden) {
    snprintf(g_msg, sizeof g_msg,
             "kd_router_topk_static: M=%d experts=%d top_k=%d hidden=%d beyond the static "
             "limits (M <= %d, top_k <= experts <= %d, top_k <= %d, hidden <= %d)",
             M, n_experts, top_k, hidden, kMaxTok, kMaxExp, kMaxK, kMaxHidden);
    return fail_static(KD_ERANGE);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    snprintf(g_msg, sizeof g_msg, "kd_router_topk_static: no usable current device");
    return fail_static(KD_ECUDA);
  }
  void* base = nullptr;
  {
    void* ctx = nullptr;
    CtxGetCurrentFn cur = ctx_get_current();
    if (cur) cur(&ctx);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_router_scratch);
      if (e != cudaSuccess) {
        snprintf(g_msg, sizeof g_msg, "kd_router_topk_static: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(e));
        return fail_static(KD_ECUDA);
      }
      g_scratch_ptr[dev] = p;
      g_scratch_ctx[dev] = ctx;
    }
    base = g_scratch_ptr[dev];
  }
  float* f = static_cast<float*>(base);
  int* w = reinterpret_cast<int*>(f);
  size_t o = (size_t)kMaxTok * kMaxExp;
  LayerDev d{};
  d.H = hidden;
  d.E = n_experts;
  d.k = top_k;
  d.eb = wdtype == KD_WBF16 ? 2 : 1;
  d.nHb = hidden / 128;
  d.wr = static_cast<const uint8_t*>(router_w);
  d.sr = router_scales;
  d.bias = router_bias;
  d.rbias = router_bias;
  d.Er = n_experts;
  d.bias_sel = 0;
  d.rscale = 1.f;
  d.h1f = const_cast<float*>(h1);
  d.logits = f;
  d.idx = idx_out;
  d.gates = gates_out;
  d.counts = w + o; o += kMaxExp;
  d.offsets = w + o; o += kMaxExp + 1;
  d.active = w + o; o += kMaxExp;
  d.perm = w + o; o += (size_t)kMaxTok * kMaxK;
  d.n_active = w + o; o += 1;
  d.err = reinterpret_cast<unsigned*>(w + o); o += 1;
  d.rcnt = reinterpret_cast<unsigned*>(w + o);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // one launch: logits, then the last block selects and builds the lists
  const int rgrid = (n_experts + kRouterRows - 1) / kRouterRows;
  const size_t smem = sizeof(int) * kSelectSmemInts(n_experts, M * top_k);   // <= 57.6 KB
  // the limit for the largest configuration (the layer sets the same one: a
  // kernel's attribute is shared by every caller in the process)
  const int smax = (int)(sizeof(int) * kSelectSmemInts(KD_STATIC_MAX_EXPERTS, kMaxTok * kMaxK));
  cudaError_t e = wdtype == KD_WFP8
      ? cudaFuncSetAttribute(router_kernel<W_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax)
      : cudaFuncSetAttribute(router_kernel<W_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax);
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof g_msg, "kd_router_topk_static: shared memory: %s", cudaGetErrorString(e));
    return fail_static(KD_ECUDA);
  }
  if (wdtype == KD_WFP8) router_kernel<W_FP8><<<rgrid, kRouterThreads, smem, s>>>(d, M);
  else router_kernel<W_BF16><<<rgrid, kRouterThreads, smem, s>>>(d, M);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(g_msg, sizeof g_msg, "kd_router_topk_static: launch: %s", cudaGetErrorString(e));
    return fail_static(KD_ECUDA);
  }
  return KD_OK;
}

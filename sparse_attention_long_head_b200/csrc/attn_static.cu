// Allocation-free variant of vs_sparse_attn_fwd: the plan scratch lives in a
// library-owned static device array instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: plain-C hosts without a
// device memory manager, and plug-ins running inside engines that own every
// byte of device memory through their own pool and forbid extensions from
// calling cudaMalloc (which may also synchronise the device in the middle of
// a latency-critical prefill).  This entry point serves them with a fixed
// scratch array that every GPU loading the library holds until exit.
#include <mutex>

#include "internal.h"

namespace vs {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB

// The scratch itself.  In host code `g_vs_scratch` is only a host-side
// stand-in for the symbol; its device address comes from
// cudaGetSymbolAddress, taken once per device below.
static __device__ __align__(256) unsigned char g_vs_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

// Driver calls that identify the current context (resolved through the
// runtime, so there is no link-time dependency on libcuda).  A context ID is
// unique for the life of the process, so a context created after
// cudaDeviceReset never matches the one an address was taken in.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static void* driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

struct ScratchSlot {
  unsigned long long ctx_id = 0;  // 0: not resolved yet
  void* addr = nullptr;
};
static ScratchSlot g_scratch_slot[kMaxDevices];
static std::mutex g_scratch_mu;

// Resolves the device address of the scratch array for the current device,
// once per (device, context): with that device current, on the first call
// and again whenever the device's context has been replaced.
static cudaError_t scratch_address(void** out) {
  static const auto get_current = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
  static const auto get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  if (!get_current || !get_id) return cudaErrorNotSupported;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  if (ctx == nullptr) {  // no context on this thread yet: the lookup makes the primary one current
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_vs_scratch);
    if (e != cudaSuccess) return e;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch_slot[dev];
  if (slot.ctx_id != id || slot.addr == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_vs_scratch);
    if (e != cudaSuccess) return e;
    slot.addr = p;
    slot.ctx_id = id;
  }
  *out = slot.addr;
  return cudaSuccess;
}

}  // namespace vs

extern "C" vs_status vs_sparse_attn_fwd_static_scratch(
    const void* Q, const void* K, const void* V, vs_dtype dtype, int N, int Hq, int Hkv, int d,
    int64_t q_stride_tok, int64_t kv_stride_tok, float softmax_scale, int H_sel,
    const int32_t* v_idx, int64_t v_ld, const int32_t* v_cnt, const int32_t* s_idx, int64_t s_ld,
    const int32_t* s_cnt, void* O, float* lse, cudaStream_t stream) {
  if (N < 1 || H_sel < 1) return VS_ERR_INVALID_ARG;
  if (vs_attn_workspace_size(N, Hq, H_sel, d) > vs::kStaticScratchBytes) return VS_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (vs::scratch_address(&scratch) != cudaSuccess) return VS_ERR_CUDA;
  return vs_sparse_attn_fwd(Q, K, V, dtype, N, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                            softmax_scale, H_sel, v_idx, v_ld, v_cnt, s_idx, s_ld, s_cnt, O, lse,
                            scratch, vs::kStaticScratchBytes, stream);
}

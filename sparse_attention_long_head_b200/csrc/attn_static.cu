// Allocation-free variant of vs_sparse_attn_fwd: the plan scratch lives in a
// library-owned static device array instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: plain-C hosts without a
// device memory manager, and plug-ins running inside engines that own every
// byte of device memory through their own pool and forbid extensions from
// calling cudaMalloc (which may also synchronise the device in the middle of
// a latency-critical prefill).  This entry point serves them with a fixed
// scratch array that every GPU loading the library holds until exit.
#include <atomic>

#include "internal.h"

namespace vs {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB

// The scratch itself.  In host code `g_vs_scratch` is only a host-side
// stand-in for the symbol; its device address comes from
// cudaGetSymbolAddress, taken once per device below.
static __device__ __align__(256) unsigned char g_vs_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
static std::atomic<void*> g_scratch_addr[kMaxDevices];

// Resolves (once per device, with that device current) the device address of
// the scratch array.
static cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_vs_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
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

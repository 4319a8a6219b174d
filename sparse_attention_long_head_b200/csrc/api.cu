// C ABI of libvs: argument validation, workspace layout and launches.
// Declarations and their documentation: include/vs_prefill.h.
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace vs {

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

void encode_rows_bf16_sw128(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t inner,
                            int64_t rows, int64_t row_stride_elems, CUresult* rc) {
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride_elems * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) *rc = r;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

// One CTA waits on an mbarrier that nothing arrives at, with the same bounded
// wait the kernels use; the timeout is recorded in the status word.
__global__ void wait_selftest_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx w{limit_ns, status, &abort_flag};
  mbar_wait(smem_u32(&bar), 0, w);
  __syncthreads();
}

cudaError_t launch_wait_selftest(int* status, uint64_t limit_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

static bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

static vs_status check_attn_common(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                   int N, int Hq, int Hkv, int d, int64_t qs, int64_t kvs,
                                   float scale, const void* O) {
  if (!Q || !K || !V || !O) return VS_ERR_INVALID_ARG;
  if (dtype != VS_BF16 && dtype != VS_FP32) return VS_ERR_INVALID_ARG;
  if (N < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return VS_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return VS_ERR_UNSUPPORTED;
  if (N > (1 << 24)) return VS_ERR_UNSUPPORTED;
  if (qs < (int64_t)Hq * d || kvs < (int64_t)Hkv * d) return VS_ERR_INVALID_ARG;
  if (qs % 8 != 0 || kvs % 8 != 0) return VS_ERR_UNSUPPORTED;
  if (!(scale >= 0.f) || std::isinf(scale)) return VS_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return VS_ERR_UNSUPPORTED;
  return VS_OK;
}

}  // namespace vs

using namespace vs;

extern "C" {

const char* vs_status_string(vs_status s) {
  switch (s) {
    case VS_OK: return "VS_OK";
    case VS_ERR_INVALID_ARG: return "VS_ERR_INVALID_ARG";
    case VS_ERR_UNSUPPORTED: return "VS_ERR_UNSUPPORTED";
    case VS_ERR_WORKSPACE: return "VS_ERR_WORKSPACE";
    case VS_ERR_CUDA: return "VS_ERR_CUDA";
    case VS_ERR_DEVICE_TIMEOUT: return "VS_ERR_DEVICE_TIMEOUT";
    case VS_ERR_DEVICE_BOUNDS: return "VS_ERR_DEVICE_BOUNDS";
  }
  return "VS_ERR_UNKNOWN";
}

int vs_version(void) { return 100; }

vs_status vs_index_scores(const void* K, const void* V, vs_dtype dtype, int N, int Hkv, int d,
                          int64_t stride_tok, int64_t stride_head, const float* W1,
                          const float* W2, int hidden, float* logits_v, float* logits_s,
                          cudaStream_t stream) {
  if (!K || !V || !W1 || !W2 || !logits_v || !logits_s) return VS_ERR_INVALID_ARG;
  if (dtype != VS_BF16 && dtype != VS_FP32) return VS_ERR_INVALID_ARG;
  if (N < 1 || Hkv < 1 || d < 1 || d > 1024 || hidden < 1 || hidden > 1024)
    return VS_ERR_INVALID_ARG;
  if (stride_head < d || stride_tok < (int64_t)(Hkv - 1) * stride_head + d) return VS_ERR_INVALID_ARG;
  if ((int64_t)N * Hkv > (int64_t)1 << 40) return VS_ERR_UNSUPPORTED;
  if (launch_index_scores(K, V, dtype, N, Hkv, d, stride_tok, stride_head, W1, W2, hidden,
                          logits_v, logits_s, stream) != cudaSuccess)
    return VS_ERR_CUDA;
  return VS_OK;
}

size_t vs_select_workspace_size(int H, int N) {
  (void)H;
  (void)N;
  return kStatusBytes;
}

vs_status vs_select(const float* scores, int H, int N, int64_t ld_scores, vs_select_mode mode,
                    int k_or_cap, double tau, int32_t* idx, int64_t ld_idx, int32_t* count,
                    void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!scores || !idx || !count) return VS_ERR_INVALID_ARG;
  if (H < 1 || H > 65535 || N < 1 || ld_scores < N) return VS_ERR_INVALID_ARG;
  if (N > (1 << 20)) return VS_ERR_UNSUPPORTED;
  if (mode != VS_SELECT_TOPK && mode != VS_SELECT_THRESHOLD && mode != VS_SELECT_MAXFRAC)
    return VS_ERR_INVALID_ARG;
  if (k_or_cap < 1 || k_or_cap > N || ld_idx < k_or_cap) return VS_ERR_INVALID_ARG;
  if (mode != VS_SELECT_TOPK && !(tau > 0.0 && tau <= 1.0)) return VS_ERR_INVALID_ARG;
  const double ln_alpha = mode == VS_SELECT_MAXFRAC ? std::log(tau) : 0.0;
  if (!ws || ws_bytes < vs_select_workspace_size(H, N) || !aligned(ws, 256)) return VS_ERR_WORKSPACE;
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return VS_ERR_CUDA;
  if (launch_select(scores, H, N, ld_scores, mode, k_or_cap, tau, ln_alpha, idx, ld_idx, count, status,
                    stream) != cudaSuccess)
    return VS_ERR_CUDA;
  return VS_OK;
}

size_t vs_select_workspace_size_varlen(int B, int H, int max_seqlen) {
  (void)B;
  (void)H;
  (void)max_seqlen;
  return kStatusBytes;
}

vs_status vs_select_varlen(const float* scores, int total_tokens, int B, const int32_t* cu_seqlens,
                           int max_seqlen, int H, vs_select_mode mode, const int32_t* caps,
                           int cap_max, double tau, int32_t* idx, int64_t ld_idx, int32_t* count,
                           void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!scores || !cu_seqlens || !caps || !idx || !count) return VS_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || (int64_t)B * H > 65535 || max_seqlen < 1 || total_tokens < 1)
    return VS_ERR_INVALID_ARG;
  if (max_seqlen > (1 << 20)) return VS_ERR_UNSUPPORTED;
  if (mode != VS_SELECT_TOPK && mode != VS_SELECT_THRESHOLD && mode != VS_SELECT_MAXFRAC)
    return VS_ERR_INVALID_ARG;
  if (cap_max < 1 || ld_idx < cap_max) return VS_ERR_INVALID_ARG;
  if (mode != VS_SELECT_TOPK && !(tau > 0.0 && tau <= 1.0)) return VS_ERR_INVALID_ARG;
  const double ln_alpha = mode == VS_SELECT_MAXFRAC ? std::log(tau) : 0.0;
  if (!ws || ws_bytes < vs_select_workspace_size_varlen(B, H, max_seqlen) || !aligned(ws, 256))
    return VS_ERR_WORKSPACE;
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return VS_ERR_CUDA;
  if (launch_select(scores, H, max_seqlen, total_tokens, mode, cap_max, tau, ln_alpha, idx, ld_idx,
                    count, status, stream, cu_seqlens, total_tokens, caps, B) != cudaSuccess)
    return VS_ERR_CUDA;
  return VS_OK;
}

size_t vs_attn_workspace_size_ld(int N, int Hq, int H_sel, int d, int64_t v_ld) {
  (void)Hq;
  if (N < 1 || H_sel < 1 || (d != 64 && d != 128) || v_ld < 1) return kStatusBytes;
  const PlanLayout L = PlanLayout::make(N, H_sel);
  const PackedLayout Pk = PackedLayout::make(L, H_sel, d, v_ld);
  return Pk.offset + Pk.bytes;
}

size_t vs_attn_workspace_size(int N, int Hq, int H_sel, int d) {
  (void)Hq;
  (void)d;
  if (N < 1 || H_sel < 1) return kStatusBytes;
  return PlanLayout::make(N, H_sel).total;
}

static vs_status attn_impl(const void* Q, const void* K, const void* V, vs_dtype dtype, int N,
                           int B, int64_t total, const int32_t* cu_seqlens,
                           int Hq, int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                           float softmax_scale, bool sparse, int H_sel, const int32_t* v_idx,
                           int64_t v_ld, const int32_t* v_cnt, const int32_t* s_idx, int64_t s_ld,
                           const int32_t* s_cnt, void* O, float* lse, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
  vs_status st = check_attn_common(Q, K, V, dtype, N, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                                   softmax_scale, O);
  if (st != VS_OK) return st;
  if (sparse) {
    if (!v_idx || !v_cnt || !s_idx || !s_cnt) return VS_ERR_INVALID_ARG;
    if (N > (1 << 22)) return VS_ERR_UNSUPPORTED;  // plan kernel's block-diagonal bitmap
    if (H_sel < 1 || Hq % H_sel != 0 || v_ld < 1 || s_ld < 1) return VS_ERR_INVALID_ARG;
  } else {
    H_sel = 1;
  }
  if (B < 1 || total < 1 || total > INT32_MAX || (B > 1 && !cu_seqlens)) return VS_ERR_INVALID_ARG;
  if (cu_seqlens && dtype != VS_BF16) return VS_ERR_UNSUPPORTED;  // batches: tensor-core path
  if ((int64_t)B * H_sel > 65535) return VS_ERR_UNSUPPORTED;
  const PlanLayout L = PlanLayout::make(N, B * H_sel);
  const size_t need = sparse ? L.total : kStatusBytes;  // the plan alone suffices
  if (!ws || ws_bytes < need || !aligned(ws, 256)) return VS_ERR_WORKSPACE;
  AttnArgs a;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.lse = lse;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.H_sel = H_sel;
  a.B = B;
  a.total = total;
  a.cu_seqlens = cu_seqlens;
  a.q_stride = q_stride_tok;
  a.kv_stride = kv_stride_tok;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(d));
  a.sparse = sparse;
  a.block_mask = nullptr;
  a.v_idx = v_idx;
  a.v_ld = v_ld;
  a.v_cnt = v_cnt;
  a.s_idx = s_idx;
  a.s_ld = s_ld;
  a.s_cnt = s_cnt;
  a.ws = ws;
  a.status = static_cast<int*>(ws);
  a.stream = stream;
  a.pack_vrows = 0;
  a.pack_k = a.pack_v = nullptr;
  if (sparse && dtype == VS_BF16 && PackedLayout::eligible(Hq, Hkv, H_sel)) {
    const PackedLayout Pk = PackedLayout::make(L, B * H_sel, d, v_ld);
    if (ws_bytes >= Pk.offset + Pk.bytes) {  // room to pack the vertical rows
      a.pack_vrows = Pk.vrows;
      a.pack_k = static_cast<char*>(ws) + Pk.offset;
      a.pack_v = static_cast<char*>(ws) + Pk.offset + Pk.bytes / 2;
    }
  }
  if (cudaMemsetAsync(a.status, 0, sizeof(int), stream) != cudaSuccess) return VS_ERR_CUDA;
  if (sparse && launch_plan(a, L) != cudaSuccess) return VS_ERR_CUDA;
  if (a.pack_vrows > 0 && launch_pack(a, L) != cudaSuccess) return VS_ERR_CUDA;
  cudaError_t e = dtype == VS_BF16 ? launch_attn_tc(a, L) : launch_attn_fp32(a, L);
  return e == cudaSuccess ? VS_OK : VS_ERR_CUDA;
}

vs_status vs_sparse_attn_fwd(const void* Q, const void* K, const void* V, vs_dtype dtype, int N,
                             int Hq, int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                             float softmax_scale, int H_sel, const int32_t* v_idx, int64_t v_ld,
                             const int32_t* v_cnt, const int32_t* s_idx, int64_t s_ld,
                             const int32_t* s_cnt, void* O, float* lse, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
  return attn_impl(Q, K, V, dtype, N, 1, N, nullptr, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                   softmax_scale, true, H_sel, v_idx, v_ld, v_cnt, s_idx, s_ld, s_cnt, O, lse,
                   ws, ws_bytes, stream);
}

size_t vs_attn_workspace_size_varlen(int B, int max_seqlen, int H_sel, int d, int64_t v_ld) {
  if (B < 1 || max_seqlen < 1 || H_sel < 1 || (d != 64 && d != 128)) return kStatusBytes;
  const PlanLayout L = PlanLayout::make(max_seqlen, B * H_sel);
  if (v_ld < 1) return L.total;
  const PackedLayout Pk = PackedLayout::make(L, B * H_sel, d, v_ld);
  return Pk.offset + Pk.bytes;
}

vs_status vs_sparse_attn_fwd_varlen(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                    int total_tokens, int B, const int32_t* cu_seqlens,
                                    int max_seqlen, int Hq, int Hkv, int d, int64_t q_stride_tok,
                                    int64_t kv_stride_tok, float softmax_scale, int H_sel,
                                    const int32_t* v_idx, int64_t v_ld, const int32_t* v_cnt,
                                    const int32_t* s_idx, int64_t s_ld, const int32_t* s_cnt,
                                    void* O, float* lse, void* ws, size_t ws_bytes,
                                    cudaStream_t stream) {
  if (!cu_seqlens) return VS_ERR_INVALID_ARG;
  return attn_impl(Q, K, V, dtype, max_seqlen, B, total_tokens, cu_seqlens, Hq, Hkv, d,
                   q_stride_tok, kv_stride_tok, softmax_scale, true, H_sel, v_idx, v_ld, v_cnt,
                   s_idx, s_ld, s_cnt, O, lse, ws, ws_bytes, stream);
}

vs_status vs_dense_attn_fwd_varlen(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                   int total_tokens, int B, const int32_t* cu_seqlens,
                                   int max_seqlen, int Hq, int Hkv, int d, int64_t q_stride_tok,
                                   int64_t kv_stride_tok, float softmax_scale, void* O, float* lse,
                                   void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!cu_seqlens) return VS_ERR_INVALID_ARG;
  return attn_impl(Q, K, V, dtype, max_seqlen, B, total_tokens, cu_seqlens, Hq, Hkv, d,
                   q_stride_tok, kv_stride_tok, softmax_scale, false, 1, nullptr, 0, nullptr,
                   nullptr, 0, nullptr, O, lse, ws, ws_bytes, stream);
}

vs_status vs_dense_attn_fwd(const void* Q, const void* K, const void* V, vs_dtype dtype, int N,
                            int Hq, int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                            float softmax_scale, void* O, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t stream) {
  return attn_impl(Q, K, V, dtype, N, 1, N, nullptr, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                   softmax_scale, false, 1, nullptr, 0, nullptr, nullptr, 0, nullptr, O, lse, ws,
                   ws_bytes, stream);
}

static vs_status aggregate_impl(const void* Q, const void* K, vs_dtype dtype, int N, int B,
                                int64_t total, const int32_t* cu, int Hq, int Hkv, int d,
                                int64_t q_stride_tok, int64_t kv_stride_tok, float softmax_scale,
                                const float* lse, float* A_v, float* A_s, void* ws,
                                size_t ws_bytes, cudaStream_t stream) {
  if (!lse || !A_v || !A_s) return VS_ERR_INVALID_ARG;
  // the checks shared with attention (V and O stand in for K and A_v here)
  vs_status st = check_attn_common(Q, K, K, dtype, N, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                                   softmax_scale, A_v);
  if (st != VS_OK) return st;
  if (B < 1 || total < 1 || total > INT32_MAX) return VS_ERR_INVALID_ARG;
  if (dtype != VS_BF16) return VS_ERR_UNSUPPORTED;
  if ((int64_t)B * Hq * ((N + 127) / 128) >= ((int64_t)1 << 31)) return VS_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < kStatusBytes || !aligned(ws, 256)) return VS_ERR_WORKSPACE;
  AggArgs a;
  a.Q = Q;
  a.K = K;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.B = B;
  a.total = total;
  a.cu_seqlens = cu;
  a.q_stride = q_stride_tok;
  a.kv_stride = kv_stride_tok;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(d));
  a.lse = lse;
  a.Av = A_v;
  a.As = A_s;
  a.status = static_cast<int*>(ws);
  a.stream = stream;
  if (cudaMemsetAsync(a.status, 0, sizeof(int), stream) != cudaSuccess) return VS_ERR_CUDA;
  if (cudaMemsetAsync(A_s, 0, sizeof(float) * (size_t)Hq * (size_t)total, stream) != cudaSuccess)
    return VS_ERR_CUDA;
  return launch_aggregate(a) == cudaSuccess ? VS_OK : VS_ERR_CUDA;
}

vs_status vs_attn_aggregate(const void* Q, const void* K, vs_dtype dtype, int N, int Hq, int Hkv,
                            int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                            float softmax_scale, const float* lse, float* A_v, float* A_s,
                            void* ws, size_t ws_bytes, cudaStream_t stream) {
  return aggregate_impl(Q, K, dtype, N, 1, N, nullptr, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                        softmax_scale, lse, A_v, A_s, ws, ws_bytes, stream);
}

vs_status vs_attn_aggregate_varlen(const void* Q, const void* K, vs_dtype dtype, int total_tokens,
                                   int B, const int32_t* cu_seqlens, int max_seqlen, int Hq,
                                   int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                                   float softmax_scale, const float* lse, float* A_v, float* A_s,
                                   void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!cu_seqlens) return VS_ERR_INVALID_ARG;
  return aggregate_impl(Q, K, dtype, max_seqlen, B, total_tokens, cu_seqlens, Hq, Hkv, d,
                        q_stride_tok, kv_stride_tok, softmax_scale, lse, A_v, A_s, ws, ws_bytes,
                        stream);
}

size_t vs_block_select_workspace_size(int N, int Hkv, int d) {
  if (N < 1 || Hkv < 1 || d < 1) return kStatusBytes;
  return block_select_ws_bytes(N, Hkv, d);
}

size_t vs_block_select_workspace_size_varlen(int B, int max_seqlen, int Hkv, int d) {
  if (B < 1 || max_seqlen < 1 || Hkv < 1 || d < 1) return kStatusBytes;
  return block_select_ws_bytes(max_seqlen, B * Hkv, d);
}

static vs_status block_select_impl(const void* Q, const void* K, vs_dtype dtype, int N, int B,
                                   int64_t total, const int32_t* cu, int Hq, int Hkv, int d,
                                   int64_t q_stride_tok, int64_t kv_stride_tok,
                                   float softmax_scale, double alpha, uint32_t* mask, void* ws,
                                   size_t ws_bytes, cudaStream_t stream) {
  if (!mask) return VS_ERR_INVALID_ARG;
  vs_status st = check_attn_common(Q, K, K, dtype, N, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                                   softmax_scale, mask);
  if (st != VS_OK) return st;
  if (!(alpha > 0.0 && alpha <= 1.0) || B < 1 || total < 1) return VS_ERR_INVALID_ARG;
  if (N > (1 << 18)) return VS_ERR_UNSUPPORTED;
  // work items (sequence, query block, head) are counted in 32 bits
  if ((int64_t)B * ((N + 127) / 128) * Hq >= ((int64_t)1 << 31)) return VS_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < block_select_ws_bytes(N, B * Hkv, d) || !aligned(ws, 256))
    return VS_ERR_WORKSPACE;
  BlockSelectArgs a;
  a.Q = Q;
  a.K = K;
  a.dtype = dtype;
  a.N = N;
  a.B = B;
  a.total = total;
  a.cu_seqlens = cu;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.q_stride = q_stride_tok;
  a.kv_stride = kv_stride_tok;
  a.scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)d);
  a.alpha = alpha;
  a.mask = mask;
  a.ws = ws;
  a.stream = stream;
  // status word and the kernel's work-item counter
  if (cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return VS_ERR_CUDA;
  return launch_block_select(a) == cudaSuccess ? VS_OK : VS_ERR_CUDA;
}

vs_status vs_block_select(const void* Q, const void* K, vs_dtype dtype, int N, int Hq, int Hkv,
                          int d, int64_t q_stride_tok, int64_t kv_stride_tok, float softmax_scale,
                          double alpha, uint32_t* mask, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  return block_select_impl(Q, K, dtype, N, 1, N, nullptr, Hq, Hkv, d, q_stride_tok,
                           kv_stride_tok, softmax_scale, alpha, mask, ws, ws_bytes, stream);
}

vs_status vs_block_select_varlen(const void* Q, const void* K, vs_dtype dtype, int total_tokens,
                                 int B, const int32_t* cu_seqlens, int max_seqlen, int Hq,
                                 int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                                 float softmax_scale, double alpha, uint32_t* mask, void* ws,
                                 size_t ws_bytes, cudaStream_t stream) {
  if (!cu_seqlens) return VS_ERR_INVALID_ARG;
  return block_select_impl(Q, K, dtype, max_seqlen, B, total_tokens, cu_seqlens, Hq, Hkv, d,
                           q_stride_tok, kv_stride_tok, softmax_scale, alpha, mask, ws, ws_bytes,
                           stream);
}

size_t vs_block_attn_workspace_size(int N, int Hq) {
  if (N < 1 || Hq < 1) return kStatusBytes;
  return BlockPlanLayout::make(N, Hq).total;
}

size_t vs_block_attn_workspace_size_varlen(int B, int max_seqlen, int Hq) {
  if (B < 1 || max_seqlen < 1 || Hq < 1) return kStatusBytes;
  return BlockPlanLayout::make(max_seqlen, B * Hq).total;
}

static vs_status block_attn_impl(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                 int N, int B, int64_t total, const int32_t* cu, int Hq, int Hkv,
                                 int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                                 float softmax_scale, const uint32_t* block_mask, void* O,
                                 float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!block_mask) return VS_ERR_INVALID_ARG;
  vs_status st = check_attn_common(Q, K, V, dtype, N, Hq, Hkv, d, q_stride_tok, kv_stride_tok,
                                   softmax_scale, O);
  if (st != VS_OK) return st;
  if (B < 1 || total < 1) return VS_ERR_INVALID_ARG;
  if (dtype != VS_BF16 || N > (1 << 18)) return VS_ERR_UNSUPPORTED;
  const BlockPlanLayout BL = BlockPlanLayout::make(N, B * Hq);
  // per-pair list offsets of every (sequence, head) must fit the kernel's 32-bit index
  if ((int64_t)B * Hq * BL.P * (BL.P + 1) >= ((int64_t)1 << 31)) return VS_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < BL.total || !aligned(ws, 256)) return VS_ERR_WORKSPACE;
  AttnArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.lse = lse;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.H_sel = 1;
  a.B = B;
  a.total = total;
  a.cu_seqlens = cu;
  a.q_stride = q_stride_tok;
  a.kv_stride = kv_stride_tok;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.f / std::sqrt(static_cast<float>(d));
  a.sparse = false;
  a.block_mask = block_mask;
  a.ws = ws;
  a.status = static_cast<int*>(ws);
  a.stream = stream;
  a.pack_vrows = 0;
  const PlanLayout L = PlanLayout::make(N, 1);  // tile and pair counts
  if (cudaMemsetAsync(a.status, 0, sizeof(int), stream) != cudaSuccess) return VS_ERR_CUDA;
  if (launch_block_plan(a) != cudaSuccess) return VS_ERR_CUDA;
  return launch_attn_tc(a, L) == cudaSuccess ? VS_OK : VS_ERR_CUDA;
}

vs_status vs_block_sparse_attn_fwd(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                   int N, int Hq, int Hkv, int d, int64_t q_stride_tok,
                                   int64_t kv_stride_tok, float softmax_scale,
                                   const uint32_t* block_mask, void* O, float* lse, void* ws,
                                   size_t ws_bytes, cudaStream_t stream) {
  return block_attn_impl(Q, K, V, dtype, N, 1, N, nullptr, Hq, Hkv, d, q_stride_tok,
                         kv_stride_tok, softmax_scale, block_mask, O, lse, ws, ws_bytes, stream);
}

vs_status vs_block_sparse_attn_fwd_varlen(const void* Q, const void* K, const void* V,
                                          vs_dtype dtype, int total_tokens, int B,
                                          const int32_t* cu_seqlens, int max_seqlen, int Hq,
                                          int Hkv, int d, int64_t q_stride_tok,
                                          int64_t kv_stride_tok, float softmax_scale,
                                          const uint32_t* block_mask, void* O, float* lse,
                                          void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!cu_seqlens) return VS_ERR_INVALID_ARG;
  return block_attn_impl(Q, K, V, dtype, max_seqlen, B, total_tokens, cu_seqlens, Hq, Hkv, d,
                         q_stride_tok, kv_stride_tok, softmax_scale, block_mask, O, lse, ws,
                         ws_bytes, stream);
}

vs_status vs_read_device_status(const void* ws, cudaStream_t stream, int* flags) {
  if (!ws || !flags) return VS_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return VS_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return VS_ERR_CUDA;
  *flags = v;
  if (v & VS_DEVFLAG_TIMEOUT) return VS_ERR_DEVICE_TIMEOUT;
  if (v & VS_DEVFLAG_BOUNDS) return VS_ERR_DEVICE_BOUNDS;
  return VS_OK;
}

vs_status vs_selftest_wait_timeout(void* ws, uint64_t limit_ns, cudaStream_t stream) {
  if (!ws || !aligned(ws, 256)) return VS_ERR_WORKSPACE;
  if (limit_ns < 1000ull || limit_ns > 10000000000ull) return VS_ERR_INVALID_ARG;
  int* status = static_cast<int*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return VS_ERR_CUDA;
  return launch_wait_selftest(status, limit_ns, stream) == cudaSuccess ? VS_OK : VS_ERR_CUDA;
}

vs_status vs_selftest_exp(const double* x, double* y, int n, cudaStream_t stream) {
  if (!x || !y || n < 1) return VS_ERR_INVALID_ARG;
  return launch_exp_selftest(x, y, n, stream) == cudaSuccess ? VS_OK : VS_ERR_CUDA;
}

}  // extern "C"

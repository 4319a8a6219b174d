// Internal declarations shared by the host API and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "vs_prefill.h"

namespace vs {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s
constexpr size_t kStatusBytes = 256;                      // status word + padding

inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-index-set-head plan data written by the plan kernel into the
// workspace (after the status header).  All sizes depend on N only.
//   vbits  : column bitmap, bit j set iff j is a selected column, padded with
//            zero bits up to 128*T + 128.
//   sbits  : offset bitmap in "reversed" positions: bit (N - o + 128) set iff
//            o is a selected offset; zero elsewhere.  A 128-bit window read at
//            position N - i + 128 + 128*b gives, for row i and key block b,
//            bit c = [ (i - (128b + c)) is a selected offset ], which is 0 for
//            every key in the future of i.
//   vlist  : selected columns ascending, deduplicated (N entries reserved).
//   slist  : selected offsets ascending, deduplicated (N entries reserved).
//   d1list : ascending list of block-diagonal indices d' in [0, T] such that
//            d' or d'-1 is "touched" (a selected offset lies in
//            [128 d - 127, 128 d + 127]).  A 256-row unit at pair p needs key
//            block b iff 2p+1-b is in this list.
//   d1pref : d1pref[x] = #{ d' in d1list : d' < x }, x in [0, T+1].
//   vpair  : vpair[p] = #{ j in vlist : j <= min(256 p + 255, N - 1) }.
//   meta   : [nv, ns, nd1, 0].
struct PlanLayout {
  int N = 0, T = 0, P = 0, H = 0;
  int64_t vbits_words = 0, sbits_words = 0, d1_len = 0, d1pref_len = 0, vpair_len = 0;
  size_t off_meta = 0, off_vbits = 0, off_sbits = 0, off_vlist = 0, off_slist = 0,
         off_d1list = 0, off_d1pref = 0, off_vpair = 0, total = 0;

  __host__ __device__ static PlanLayout make(int N, int H) {
    PlanLayout L;
    L.N = N;
    L.H = H;
    L.T = (N + 127) / 128;
    L.P = (L.T + 1) / 2;
    L.vbits_words = 4 * (int64_t)(L.T + 2);
    L.sbits_words = ((int64_t)N + 512 + 31) / 32 + 2;
    L.d1_len = L.T + 1;
    L.d1pref_len = L.T + 2;
    L.vpair_len = L.P;
    size_t off = 256;  // status header
    auto take = [&](size_t bytes) {
      size_t o = off;
      off = (off + bytes + 255) / 256 * 256;
      return o;
    };
    L.off_meta = take(sizeof(int32_t) * 4 * (size_t)H);
    L.off_vbits = take(sizeof(uint32_t) * (size_t)L.vbits_words * H);
    L.off_sbits = take(sizeof(uint32_t) * (size_t)L.sbits_words * H);
    L.off_vlist = take(sizeof(int32_t) * (size_t)N * H);
    L.off_slist = take(sizeof(int32_t) * (size_t)N * H);
    L.off_d1list = take(sizeof(int32_t) * (size_t)L.d1_len * H);
    L.off_d1pref = take(sizeof(int32_t) * (size_t)L.d1pref_len * H);
    L.off_vpair = take(sizeof(int32_t) * (size_t)L.vpair_len * H);
    L.total = off;
    return L;
  }
};

struct PlanPtrs {
  int32_t* meta;
  uint32_t* vbits;
  uint32_t* sbits;
  int32_t* vlist;
  int32_t* slist;
  int32_t* d1list;
  int32_t* d1pref;
  int32_t* vpair;
};

inline __host__ __device__ PlanPtrs plan_ptrs(const PlanLayout& L, void* ws) {
  char* b = static_cast<char*>(ws);
  PlanPtrs p;
  p.meta = reinterpret_cast<int32_t*>(b + L.off_meta);
  p.vbits = reinterpret_cast<uint32_t*>(b + L.off_vbits);
  p.sbits = reinterpret_cast<uint32_t*>(b + L.off_sbits);
  p.vlist = reinterpret_cast<int32_t*>(b + L.off_vlist);
  p.slist = reinterpret_cast<int32_t*>(b + L.off_slist);
  p.d1list = reinterpret_cast<int32_t*>(b + L.off_d1list);
  p.d1pref = reinterpret_cast<int32_t*>(b + L.off_d1pref);
  p.vpair = reinterpret_cast<int32_t*>(b + L.off_vpair);
  return p;
}

// Optional region after the plan: each index set's selected vertical K and V
// rows packed contiguously ([H_sel][vrows][d] each), so that vertical chunks
// load as ordinary TMA tiles instead of row gathers.  Used when every index
// set's query heads lie in one KV group ((Hq / H_sel) divides Hq / Hkv) and the
// workspace is large enough.
struct PackedLayout {
  int64_t vrows = 0;  // rows per index set, multiple of 128
  size_t offset = 0, bytes = 0;
  static bool eligible(int Hq, int Hkv, int H_sel) {
    const int qs = Hq / H_sel, G = Hq / Hkv;
    return qs >= 1 && G % qs == 0;
  }
  static PackedLayout make(const PlanLayout& L, int H_sel, int d, int64_t v_ld) {
    PackedLayout Pk;
    const int64_t rows = v_ld < L.N ? v_ld : L.N;
    Pk.vrows = (rows + 127) / 128 * 128;
    Pk.offset = (L.total + 1023) / 1024 * 1024;
    Pk.bytes = 2 * (size_t)H_sel * (size_t)Pk.vrows * (size_t)d * 2;
    return Pk;
  }
};

// Sequence b of a packed batch: tokens [tok0, tok0 + Nb) of every tensor.
// Without cu_seqlens the batch is one sequence of maxN tokens.  A malformed
// entry (negative, decreasing, past `total` or longer than maxN) gives an
// empty sequence and returns false (callers flag VS_DEVFLAG_BOUNDS).
__host__ __device__ inline bool seq_range(const int32_t* cu, int64_t total, int maxN, int b,
                                          int64_t& tok0, int& Nb) {
  if (!cu) {
    tok0 = 0;
    Nb = maxN;
    return true;
  }
  const int64_t s = cu[b], e = cu[b + 1];
  if (s < 0 || e < s || e > total || e - s > maxN) {
    tok0 = 0;
    Nb = 0;
    return false;
  }
  tok0 = s;
  Nb = static_cast<int>(e - s);
  return true;
}

// Block-sparse plan in the workspace (after the status header): per (head,
// pair of query blocks) a count, and the kept key blocks of the pair at
// h P (P + 1) + p (p + 1) (at most 2p + 2 of them).
struct BlockPlanLayout {
  int T = 0, P = 0;
  size_t off_cnt = 0, off_list = 0, total = 0;
  __host__ __device__ static BlockPlanLayout make(int N, int Hq) {
    BlockPlanLayout B;
    B.T = (N + 127) / 128;
    B.P = (B.T + 1) / 2;
    B.off_cnt = 256;
    B.off_list = B.off_cnt + (sizeof(int32_t) * (size_t)Hq * B.P + 255) / 256 * 256;
    B.total = B.off_list + sizeof(uint32_t) * (size_t)Hq * B.P * (B.P + 1);
    return B;
  }
};

// Common attention launch description.  A batch of B sequences packed along
// the token axis (cu_seqlens, device, B + 1 offsets; null for one sequence)
// has plan slots b * H_sel + hs, each laid out for N = the longest sequence.
struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  float* lse;
  int N, Hq, Hkv, d, H_sel;  // N: the longest sequence (the only one when B = 1)
  int B;                     // sequences
  int64_t total;             // token rows of Q, K, V, O (= N when B = 1)
  const int32_t* cu_seqlens; // device [B + 1] or null
  int64_t q_stride, kv_stride;
  float scale;
  bool sparse;
  const uint32_t* block_mask;  // block sparse: kept key blocks [Hq][T][W] (else null)
  const int32_t* v_idx;
  int64_t v_ld;
  const int32_t* v_cnt;
  const int32_t* s_idx;
  int64_t s_ld;
  const int32_t* s_cnt;
  void* ws;
  int* status;
  cudaStream_t stream;
  // packed vertical rows (vrows == 0: gather the rows with TMA gather4)
  int64_t pack_vrows;
  void* pack_k;
  void* pack_v;
};

// Ground-truth aggregation launch description (bf16 Q/K).
struct AggArgs {
  const void* Q;
  const void* K;
  int N, Hq, Hkv, d;          // N: the longest sequence (the only one when B = 1)
  int B;                      // sequences packed along the token axis
  int64_t total;              // token rows of Q and K; lse, A_v, A_s are [Hq][total]
  const int32_t* cu_seqlens;  // device [B + 1] or null
  int64_t q_stride, kv_stride;
  float scale;
  const float* lse;
  float* Av;
  float* As;
  int* status;
  cudaStream_t stream;
};

// FlashPrefill-style block pattern discovery (blocks.cu).
struct BlockSelectArgs {
  const void* Q;
  const void* K;
  int dtype, N, Hq, Hkv, d;  // N: the longest sequence (the only one when B = 1)
  int B;                     // sequences packed along the token axis
  int64_t total;             // token rows of Q and K
  const int32_t* cu_seqlens; // device [B + 1] or null
  int64_t q_stride, kv_stride;
  double scale, alpha;
  uint32_t* mask;  // [B][Hq][T][W], T and W of the longest sequence
  void* ws;        // status word, then the block means
  cudaStream_t stream;
};
// workspace of a batch: the block means of B * Hkv (sequence, KV head) pairs
size_t block_select_ws_bytes(int N, int B_Hkv, int d);
cudaError_t launch_block_select(const BlockSelectArgs& a);
cudaError_t launch_exp_selftest(const double* x, double* y, int n, cudaStream_t stream);

// Launchers (return a CUDA error; argument checks are done by the caller).
cudaError_t launch_plan(const AttnArgs& a, const PlanLayout& L);
cudaError_t launch_pack(const AttnArgs& a, const PlanLayout& L);
cudaError_t launch_block_plan(const AttnArgs& a);
cudaError_t launch_attn_tc(const AttnArgs& a, const PlanLayout& L);
cudaError_t launch_attn_fp32(const AttnArgs& a, const PlanLayout& L);
// Batched form: cu (device, B + 1 offsets) and caps (device, B) non-null, N
// the longest sequence, k_or_cap the bound on the caps, scores [H][total].
cudaError_t launch_select(const float* scores, int H, int N, int64_t ld, int mode, int k_or_cap,
                          double tau, double ln_alpha, int32_t* idx, int64_t ld_idx, int32_t* count, int* status,
                          cudaStream_t stream, const int32_t* cu = nullptr, int64_t total = 0,
                          const int32_t* caps = nullptr, int B = 1);
cudaError_t launch_index_scores(const void* K, const void* V, int dtype, int N, int Hkv, int d,
                                int64_t stride_tok, int64_t stride_head, const float* W1,
                                const float* W2, int hidden, float* lv, float* ls,
                                cudaStream_t stream);
cudaError_t launch_wait_selftest(int* status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_aggregate(const AggArgs& a);

// Driver entry point for tensor-map encoding (resolved once through the
// runtime; no link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();
int device_sm_count();
// 2-D bf16 map over `rows` rows of `inner` elements (row stride in elements),
// box of 128 rows x 64 elements, 128-byte swizzle, zero fill past the edges.
// Leaves *rc unchanged on success.
void encode_rows_bf16_sw128(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t inner,
                            int64_t rows, int64_t row_stride_elems, CUresult* rc);

}  // namespace vs

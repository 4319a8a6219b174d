// fp32 CUDA-core path of the vertical-slash attention (and of dense causal
// attention), one warp per (query head, row).  It serves fp32 inputs, where
// the tensor-core path does not apply.
//
// Key set of row i ("VSPrefill ..." Technical Summary, section 2, fused
// kernel merging the vertical and slash index lists): every selected column
// j <= i whose offset i - j is not itself selected, then every key i - o for
// a selected offset o <= i.  The offset test reads the plan's offset bitmap,
// so a key that is both a column and on a selected diagonal is visited once.
// Online softmax in fp32 with accurate expf.
#include "internal.h"

namespace vs {

constexpr int kF32Warps = 8;

struct F32Args {
  const float* Q;
  const float* K;
  const float* V;
  float* O;
  float* lse;
  int N, Hq, Hkv, d, H_sel, G;
  int64_t q_stride, kv_stride;
  float scale;
  bool sparse;
  PlanLayout L;
  PlanPtrs pp;
};

template <int D>
__global__ void __launch_bounds__(32 * kF32Warps) attn_fp32_kernel(F32Args a) {
  constexpr int E = D / 32;  // elements per lane
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * kF32Warps + (threadIdx.x >> 5);
  if (w >= (int64_t)a.N * a.Hq) return;
  const int h = static_cast<int>(w % a.Hq);
  const int i = static_cast<int>(w / a.Hq);
  const int g = h / a.G;
  float q[E], o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = a.Q[(int64_t)i * a.q_stride + (int64_t)h * D + lane + 32 * e];
    o[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  auto visit = [&](int j) {
    const float* kr = a.K + (int64_t)j * a.kv_stride + (int64_t)g * D;
    const float* vr = a.V + (int64_t)j * a.kv_stride + (int64_t)g * D;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) s = fmaf(q[e], kr[lane + 32 * e], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    s *= a.scale;
    const float mn = fmaxf(m, s);
    const float f = expf(m - mn);  // 0 when m = -inf
    const float p = expf(s - mn);
    l = l * f + p;
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = fmaf(p, vr[lane + 32 * e], o[e] * f);
    m = mn;
  };
  if (!a.sparse) {
    for (int j = 0; j <= i; ++j) visit(j);
  } else {
    const int hs = static_cast<int>(((int64_t)h * a.H_sel) / a.Hq);
    const int32_t* meta = a.pp.meta + 4 * hs;
    const int nv = meta[0], ns = meta[1];
    const int32_t* vl = a.pp.vlist + (int64_t)hs * a.N;
    const int32_t* sl = a.pp.slist + (int64_t)hs * a.N;
    const uint32_t* sb = a.pp.sbits + (int64_t)hs * a.L.sbits_words;
    for (int t = 0; t < nv; ++t) {
      const int j = vl[t];
      if (j > i) break;
      const int pos = a.N - (i - j) + 128;
      if ((sb[pos >> 5] >> (pos & 31)) & 1u) continue;  // covered by a slash
      visit(j);
    }
    for (int t = 0; t < ns; ++t) {
      const int off = sl[t];
      if (off > i) break;
      visit(i - off);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e)
    a.O[(int64_t)i * a.q_stride + (int64_t)h * D + lane + 32 * e] = o[e] * inv;
  if (lane == 0 && a.lse) a.lse[(int64_t)h * a.N + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

cudaError_t launch_attn_fp32(const AttnArgs& a, const PlanLayout& L) {
  F32Args k;
  k.Q = static_cast<const float*>(a.Q);
  k.K = static_cast<const float*>(a.K);
  k.V = static_cast<const float*>(a.V);
  k.O = static_cast<float*>(a.O);
  k.lse = a.lse;
  k.N = a.N;
  k.Hq = a.Hq;
  k.Hkv = a.Hkv;
  k.d = a.d;
  k.H_sel = a.sparse ? a.H_sel : 1;
  k.G = a.Hq / a.Hkv;
  k.q_stride = a.q_stride;
  k.kv_stride = a.kv_stride;
  k.scale = a.scale;
  k.sparse = a.sparse;
  k.L = L;
  k.pp = plan_ptrs(L, a.ws);
  const int64_t warps = (int64_t)a.N * a.Hq;
  const int grid = static_cast<int>((warps + kF32Warps - 1) / kF32Warps);
  if (a.d == 128) attn_fp32_kernel<128><<<grid, 32 * kF32Warps, 0, a.stream>>>(k);
  else if (a.d == 64) attn_fp32_kernel<64><<<grid, 32 * kF32Warps, 0, a.stream>>>(k);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace vs

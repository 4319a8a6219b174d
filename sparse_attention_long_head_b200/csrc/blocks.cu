// FlashPrefill-style block pattern discovery on sm_100a.
//
// FlashPrefill summary page, section 2A: a skeleton of uniformly spaced
// queries probes the key blocks, each key block represented by its mean key
// (the geometric mean of the block's attention weights, a monotone proxy of
// their sum); section 2B: for query block I keep key block J when its score
// is at least alpha times the best block's score -- one max reduction, no
// sort, no cumulative sum.  With 128-row blocks and the probes of block I at
// rows 128 I + 8 m (m = 0..15, below N):
//     Score(I, J) = mean_probes softmax_{J' < I}(scale * q . kbar_J')[J],
//     keep J < I iff Score(I, J) >= alpha * max_J' Score(I, J'),
// and the diagonal block is always kept.  Computed in fp64 (the work is a
// few dot products per block pair), so the kept sets follow the definition
// up to rounding order.
//
//   block_mean_kernel: one CTA per (key block, KV head), thread c sums column
//     c of the block's keys -> kbar [Hkv][T][d] fp64 in the workspace.
//   block_score_kernel: one CTA per (query block, head).  The 16 probes sit
//     in shared memory; each thread takes key blocks J = tid, tid + 256, ...
//     Pass 1 keeps a per-probe online max and sum of exponentials, merged
//     across the CTA; pass 2 recomputes the dot products and forms the
//     averaged scores in shared memory; the maximum and the threshold then
//     give the row's bitmask.
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"

namespace vs {

namespace {

constexpr int kProbes = 16;
constexpr int kProbeStride = 8;
constexpr int kScoreThreads = 256;
constexpr int kMaxBlocks = 2048;  // T <= 2048 (N <= 2^18): scores fit in static shared memory

__device__ __forceinline__ double load_kv(const void* p, int dtype, int64_t off) {
  if (dtype == VS_BF16) return (double)__bfloat162float(static_cast<const __nv_bfloat16*>(p)[off]);
  return (double)static_cast<const float*>(p)[off];
}

__global__ void __launch_bounds__(128) block_mean_kernel(const void* K, int dtype, int N, int Hkv,
                                                         int d, int64_t kv_stride, double* kbar) {
  const int J = blockIdx.x, g = blockIdx.y, T = gridDim.x;
  const int64_t j0 = 128 * (int64_t)J, j1 = min((int64_t)N, j0 + 128);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double acc = 0.0;
    for (int64_t j = j0; j < j1; ++j) acc += load_kv(K, dtype, j * kv_stride + (int64_t)g * d + c);
    kbar[((int64_t)g * T + J) * d + c] = acc / (double)(j1 - j0);
  }
}

struct ScoreArgs {
  const void* Q;
  int dtype, N, Hq, Hkv, d, T, W;
  int64_t q_stride;
  double scale, alpha;
  const double* kbar;
  uint32_t* mask;
};

// s[p] = scale * probe_p . kbar_J for the CTA's probes.
__device__ __forceinline__ void probe_dots(const ScoreArgs& a, const double* probes, int np,
                                           const double* kb, double (&s)[kProbes]) {
#pragma unroll
  for (int p = 0; p < kProbes; ++p) s[p] = 0.0;
  for (int c = 0; c < a.d; ++c) {
    const double k = __ldg(kb + c);
#pragma unroll
    for (int p = 0; p < kProbes; ++p) s[p] = fma(probes[p * 128 + c], k, s[p]);
  }
#pragma unroll
  for (int p = 0; p < kProbes; ++p) s[p] = p < np ? a.scale * s[p] : -INFINITY;
}

__global__ void __launch_bounds__(kScoreThreads) block_score_kernel(ScoreArgs a) {
  __shared__ double probes[kProbes * 128];
  __shared__ double score[kMaxBlocks];
  __shared__ double red_m[kScoreThreads / 32][kProbes], red_z[kScoreThreads / 32][kProbes];
  __shared__ double pm[kProbes], pz[kProbes];
  __shared__ double best_w[kScoreThreads / 32];
  __shared__ uint32_t row[kMaxBlocks / 32];
  const int I = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = h / (a.Hq / a.Hkv);
  const double* kbar = a.kbar + (int64_t)g * a.T * a.d;
  int np = 0;
  while (np < kProbes && 128 * (int64_t)I + kProbeStride * np < a.N) ++np;
  for (int e = tid; e < kProbes * 128; e += kScoreThreads) {
    const int p = e / 128, c = e % 128;
    const int64_t i = 128 * (int64_t)I + kProbeStride * p;
    probes[e] = (p < np && c < a.d)
                    ? load_kv(a.Q, a.dtype, i * a.q_stride + (int64_t)h * a.d + c) : 0.0;
  }
  for (int w = tid; w < a.W; w += kScoreThreads) row[w] = 0u;
  __syncthreads();
  // pass 1: per-probe max and sum of exponentials over J < I (online, merged)
  double m[kProbes], z[kProbes];
#pragma unroll
  for (int p = 0; p < kProbes; ++p) {
    m[p] = -INFINITY;
    z[p] = 0.0;
  }
  for (int J = tid; J < I; J += kScoreThreads) {
    double s[kProbes];
    probe_dots(a, probes, np, kbar + (int64_t)J * a.d, s);
#pragma unroll
    for (int p = 0; p < kProbes; ++p) {
      if (p >= np) continue;
      const double mn = fmax(m[p], s[p]);
      z[p] = z[p] * exp(m[p] - mn) + exp(s[p] - mn);
      m[p] = mn;
    }
  }
#pragma unroll
  for (int p = 0; p < kProbes; ++p) {  // warp merge, then across warps
    for (int o = 16; o > 0; o >>= 1) {
      const double mo = __shfl_xor_sync(0xffffffffu, m[p], o);
      const double zo = __shfl_xor_sync(0xffffffffu, z[p], o);
      const double mn = fmax(m[p], mo);
      z[p] = (m[p] == -INFINITY ? 0.0 : z[p] * exp(m[p] - mn)) +
             (mo == -INFINITY ? 0.0 : zo * exp(mo - mn));
      m[p] = mn;
    }
    if (lane == 0) {
      red_m[warp][p] = m[p];
      red_z[warp][p] = z[p];
    }
  }
  __syncthreads();
  if (tid < kProbes) {
    double mm = -INFINITY, zz = 0.0;
    for (int w = 0; w < kScoreThreads / 32; ++w) {
      const double mo = red_m[w][tid], zo = red_z[w][tid];
      const double mn = fmax(mm, mo);
      zz = (mm == -INFINITY ? 0.0 : zz * exp(mm - mn)) + (mo == -INFINITY ? 0.0 : zo * exp(mo - mn));
      mm = mn;
    }
    pm[tid] = mm;
    pz[tid] = zz;
  }
  __syncthreads();
  // pass 2: averaged scores and their maximum
  double best = 0.0;
  for (int J = tid; J < I; J += kScoreThreads) {
    double s[kProbes];
    probe_dots(a, probes, np, kbar + (int64_t)J * a.d, s);
    double acc = 0.0;
#pragma unroll
    for (int p = 0; p < kProbes; ++p)
      if (p < np) acc += exp(s[p] - pm[p]) / pz[p];
    acc /= (double)np;
    score[J] = acc;
    best = fmax(best, acc);
  }
  for (int o = 16; o > 0; o >>= 1) best = fmax(best, __shfl_xor_sync(0xffffffffu, best, o));
  if (lane == 0) best_w[warp] = best;
  __syncthreads();
  double thr = 0.0;
  for (int w = 0; w < kScoreThreads / 32; ++w) thr = fmax(thr, best_w[w]);
  thr *= a.alpha;
  for (int J = tid; J < I; J += kScoreThreads)
    if (score[J] >= thr) atomicOr(&row[J >> 5], 1u << (J & 31));
  if (tid == 0) atomicOr(&row[I >> 5], 1u << (I & 31));  // the diagonal block
  __syncthreads();
  uint32_t* out = a.mask + ((int64_t)h * a.T + I) * a.W;
  for (int w = tid; w < a.W; w += kScoreThreads) out[w] = row[w];
}

}  // namespace

size_t block_select_ws_bytes(int N, int Hkv, int d) {
  const int T = (N + 127) / 128;
  return kStatusBytes + align_up(sizeof(double) * (size_t)Hkv * T * d, 256);
}

cudaError_t launch_block_select(const BlockSelectArgs& a) {
  const int T = (a.N + 127) / 128, W = (T + 31) / 32;
  if (T > kMaxBlocks) return cudaErrorInvalidValue;
  double* kbar = reinterpret_cast<double*>(static_cast<char*>(a.ws) + kStatusBytes);
  block_mean_kernel<<<dim3(T, a.Hkv), 128, 0, a.stream>>>(a.K, a.dtype, a.N, a.Hkv, a.d,
                                                          a.kv_stride, kbar);
  ScoreArgs s{a.Q, a.dtype, a.N, a.Hq, a.Hkv, a.d, T, W, a.q_stride, a.scale, a.alpha, kbar,
              a.mask};
  block_score_kernel<<<dim3(T, a.Hq), kScoreThreads, 0, a.stream>>>(s);
  return cudaGetLastError();
}

}  // namespace vs

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
//     in shared memory; the block means stream through shared memory in
//     chunks of 256 blocks x 16 columns, each thread computing a 4 x 4
//     (blocks x probes) tile of dot products.  Pass 1 keeps a per-probe
//     online max and sum of exponentials, merged across the CTA; pass 2
//     recomputes the dot products and forms the averaged scores in shared
//     memory; the maximum and the threshold then give the row's bitmask.
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
  int cache;  // the pass-1 dot products are kept in shared memory (T <= 1024)
};

// The CTA's dot products s[p][J] = scale * probe_p . kbar_J for J in
// [J0, J0 + 256) (J < I): thread t owns blocks J0 + (t % 64) + 64 x
// (x = 0..3; a warp's 32 blocks then sit 17 doubles apart in the stage, in
// distinct banks) and probes 4 (t / 64) + {0..3} (one value per warp,
// broadcast).  The block means stream through shared memory 16 columns at a
// time (coalesced rows; the next 16 columns are loaded into registers while
// the current ones are used), so every loaded value feeds four fused
// multiply-adds.
constexpr int kJChunk = 256;
constexpr int kCChunk = 16;

template <int D>
__device__ __forceinline__ void chunk_dots(const ScoreArgs& a, const double* probes,
                                           double* kstage, int J0, int I, double (&acc)[4][4]) {
  const int tid = threadIdx.x, jg = tid % 64, pg = tid / 64;
  // this thread stages column tid % 16 of rows J0 + tid / 16 + 16 k (k = 0..15)
  const int cc_ld = tid % kCChunk, jj_ld = tid / kCChunk;
  auto load = [&](int c0, double (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int J = J0 + jj_ld + 16 * k;
      v[k] = J < I ? __ldg(a.kbar + (int64_t)J * D + c0 + cc_ld) : 0.0;
    }
  };
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] = 0.0;
  double nxt[16];
  load(0, nxt);
  for (int c0 = 0; c0 < D; c0 += kCChunk) {
    __syncthreads();  // the previous stage has been read
#pragma unroll
    for (int k = 0; k < 16; ++k) kstage[(jj_ld + 16 * k) * (kCChunk + 1) + cc_ld] = nxt[k];
    __syncthreads();
    if (c0 + kCChunk < D) load(c0 + kCChunk, nxt);  // in flight while this stage is used
#pragma unroll
    for (int cc = 0; cc < kCChunk; ++cc) {
      double pv[4], kv[4];
#pragma unroll
      for (int y = 0; y < 4; ++y) pv[y] = probes[(4 * pg + y) * 128 + c0 + cc];
#pragma unroll
      for (int x = 0; x < 4; ++x) kv[x] = kstage[(jg + 64 * x) * (kCChunk + 1) + cc];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fma(pv[y], kv[x], acc[x][y]);
    }
  }
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] *= a.scale;
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads) block_score_kernel(ScoreArgs a) {
  extern __shared__ double dyn[];  // probes, staged block means, scores, kept dot products
  double* probes = dyn;
  double* kstage = probes + kProbes * 128;
  double* score = kstage + kJChunk * (kCChunk + 1);
  double* sdot = score + kMaxBlocks;  // [kProbes][T] when a.cache
  __shared__ double red_m[kScoreThreads / 32][4], red_z[kScoreThreads / 32][4];
  __shared__ double red_z2[kScoreThreads / 32][kProbes];
  __shared__ double pm[kProbes], pz[kProbes];
  __shared__ double best_w[kScoreThreads / 32];
  __shared__ uint32_t row[kMaxBlocks / 32];
  const int I = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int jg = tid % 64, pg = tid / 64;
  const int g = h / (a.Hq / a.Hkv);
  ScoreArgs b = a;
  b.kbar = a.kbar + (int64_t)g * a.T * D;
  int np = 0;
  while (np < kProbes && 128 * (int64_t)I + kProbeStride * np < a.N) ++np;
  for (int e = tid; e < kProbes * 128; e += kScoreThreads) {
    const int p = e / 128, c = e % 128;
    const int64_t i = 128 * (int64_t)I + kProbeStride * p;
    probes[e] = (p < np && c < D) ? load_kv(a.Q, a.dtype, i * a.q_stride + (int64_t)h * D + c) : 0.0;
  }
  for (int w = tid; w < a.W; w += kScoreThreads) row[w] = 0u;
  if (a.cache) {
    // Kept dot products, the oracle's order of steps: per-probe maximum, then
    // the exponentials once (stored in place) and their sum, then the scores.
    double mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    for (int J0 = 0; J0 < I; J0 += kJChunk) {
      double s[4][4];
      chunk_dots<D>(b, probes, kstage, J0, I, s);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int J = J0 + jg + 64 * x;
        if (J >= I) continue;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          sdot[(4 * pg + y) * a.T + J] = s[x][y];
          mx[y] = fmax(mx[y], s[x][y]);
        }
      }
    }
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      for (int o = 16; o > 0; o >>= 1) mx[y] = fmax(mx[y], __shfl_xor_sync(0xffffffffu, mx[y], o));
      if (lane == 0) red_m[warp][y] = mx[y];
    }
    __syncthreads();
    if (tid < kProbes) pm[tid] = fmax(red_m[2 * (tid / 4)][tid % 4], red_m[2 * (tid / 4) + 1][tid % 4]);
    __syncthreads();
    // exponentials: thread t takes (probe, J) pairs e = t, t + 256, ...
    double zp[kProbes];
#pragma unroll
    for (int p = 0; p < kProbes; ++p) zp[p] = 0.0;
    for (int J = tid; J < I; J += kScoreThreads) {
#pragma unroll
      for (int p = 0; p < kProbes; ++p) {
        if (p >= np) continue;
        const double e = exp(sdot[p * a.T + J] - pm[p]);
        sdot[p * a.T + J] = e;
        zp[p] += e;
      }
    }
#pragma unroll
    for (int p = 0; p < kProbes; ++p) {
      for (int o = 16; o > 0; o >>= 1) zp[p] += __shfl_xor_sync(0xffffffffu, zp[p], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int p = 0; p < kProbes; ++p) red_z2[warp][p] = zp[p];
    }
    __syncthreads();
    if (tid < kProbes) {
      double zz = 0.0;
      for (int w = 0; w < kScoreThreads / 32; ++w) zz += red_z2[w][tid];
      pz[tid] = zz;
    }
    __syncthreads();
    for (int J = tid; J < I; J += kScoreThreads) {
      double t = 0.0;
      for (int p = 0; p < np; ++p) t += sdot[p * a.T + J] / pz[p];
      score[J] = t;
    }
  } else {
  // Recomputed dot products (T > 1024): pass 1 keeps a per-probe online max
  // and sum of exponentials (the four probes of a thread are merged over the
  // 64 threads sharing them); pass 2 forms the averaged scores.
  double m[4], z[4];
#pragma unroll
  for (int y = 0; y < 4; ++y) {
    m[y] = -INFINITY;
    z[y] = 0.0;
  }
  for (int J0 = 0; J0 < I; J0 += kJChunk) {
    double s[4][4];
    chunk_dots<D>(b, probes, kstage, J0, I, s);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      if (J0 + jg + 64 * x >= I) continue;
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const double mn = fmax(m[y], s[x][y]);
        z[y] = z[y] * exp(m[y] - mn) + exp(s[x][y] - mn);
        m[y] = mn;
      }
    }
  }
  auto merge = [](double& m1, double& z1, double m2, double z2) {
    const double mn = fmax(m1, m2);
    z1 = (m1 == -INFINITY ? 0.0 : z1 * exp(m1 - mn)) + (m2 == -INFINITY ? 0.0 : z2 * exp(m2 - mn));
    m1 = mn;
  };
#pragma unroll
  for (int y = 0; y < 4; ++y) {
    for (int o = 16; o > 0; o >>= 1)
      merge(m[y], z[y], __shfl_xor_sync(0xffffffffu, m[y], o), __shfl_xor_sync(0xffffffffu, z[y], o));
    if (lane == 0) {
      red_m[warp][y] = m[y];
      red_z[warp][y] = z[y];
    }
  }
  __syncthreads();
  if (tid < kProbes) {  // probe p = 4 pg + y lives in warps 2 pg, 2 pg + 1
    const int pgp = tid / 4, y = tid % 4;
    double mm = red_m[2 * pgp][y], zz = red_z[2 * pgp][y];
    merge(mm, zz, red_m[2 * pgp + 1][y], red_z[2 * pgp + 1][y]);
    pm[tid] = mm;
    pz[tid] = zz;
  }
  __syncthreads();
  for (int J = tid; J < I; J += kScoreThreads) score[J] = 0.0;
  for (int J0 = 0; J0 < I; J0 += kJChunk) {
    double s[4][4];
    chunk_dots<D>(b, probes, kstage, J0, I, s);
    // sum this thread's four probes, then the four probe groups in order
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      double t = 0.0;
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const int p = 4 * pg + y;
        if (p < np) t += exp(s[x][y] - pm[p]) / pz[p];
      }
      s[x][0] = t;
    }
    for (int q = 0; q < 4; ++q) {
      __syncthreads();
      if (pg == q) {
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int J = J0 + jg + 64 * x;
          if (J < I) score[J] += s[x][0];
        }
      }
    }
  }
  }
  __syncthreads();
  double best = 0.0;
  for (int J = tid; J < I; J += kScoreThreads) {
    score[J] /= (double)np;
    best = fmax(best, score[J]);
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
  const int cache = T <= 1024 ? 1 : 0;
  ScoreArgs s{a.Q,       a.dtype, a.N,     a.Hq, a.Hkv, a.d,    T,    W,
              a.q_stride, a.scale, a.alpha, kbar, a.mask, cache};
  const size_t smem = sizeof(double) * (kProbes * 128 + kJChunk * (kCChunk + 1) + kMaxBlocks +
                                        (cache ? (size_t)kProbes * T : 0));
  auto kern = a.d == 128 ? block_score_kernel<128> : block_score_kernel<64>;
  if (a.d != 128 && a.d != 64) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(T, a.Hq), kScoreThreads, smem, a.stream>>>(s);
  return cudaGetLastError();
}

}  // namespace vs

// The indexer: per token t and KV head g, h = ReLU(W1 [k_t; v_t]) and
// (logit_v, logit_s) = W2 h  ("VSPrefill ..." Technical Summary, section 2,
// VSIndexer: a shared-weight bilayer linear network on concat(K with RoPE, V)
// with separate down-projection heads for the vertical and slash scores).
//
// fp32 CUDA-core GEMM: a CTA computes a 128-row x 256-hidden tile of
// X W1^T (X = the [k; v] rows, fp32 in shared memory, K-loop of 16), then
// applies ReLU and the 2-row down-projection in registers, reducing across
// the 16 threads that share a row with warp shuffles.  Hidden sizes above
// 256 loop over 256-wide slices and accumulate the two outputs.
//
// index_scores_vec_kernel is the same computation for aligned inputs (16-byte
// aligned rows, d a multiple of 16): a CTA takes 128 consecutive tokens of
// one KV head, so its X rows are contiguous and load as 16-byte vectors, W1
// loads as float4, and the next K-chunk is in registers while the current
// one is multiplied.
#include "internal.h"

namespace vs {

constexpr int kIdxRows = 128;
constexpr int kIdxHid = 256;
constexpr int kIdxK = 16;
constexpr int kIdxThreads = 256;

struct IdxArgs {
  const void* K;
  const void* V;
  int dtype, N, Hkv, d;
  int64_t stride_tok, stride_head;
  const float* W1;
  const float* W2;
  int hidden;
  float* lv;
  float* ls;
};

__device__ __forceinline__ float load_x(const IdxArgs& a, const void* base, int64_t off) {
  if (a.dtype == VS_BF16) {
    const uint16_t b = static_cast<const uint16_t*>(base)[off];
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
  return static_cast<const float*>(base)[off];
}

__global__ void __launch_bounds__(kIdxThreads) index_scores_kernel(IdxArgs a) {
  __shared__ float xs[kIdxK][kIdxRows + 4];
  __shared__ float ws[kIdxK][kIdxHid + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads
  const int64_t nrows = (int64_t)a.N * a.Hkv;
  const int64_t row0 = (int64_t)blockIdx.x * kIdxRows;
  const int D2 = 2 * a.d;
  float out_v[8], out_s[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) out_v[r] = out_s[r] = 0.f;

  for (int h0 = 0; h0 < a.hidden; h0 += kIdxHid) {
    float acc[8][16];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[r][c] = 0.f;
    for (int k0 = 0; k0 < D2; k0 += kIdxK) {
      // X tile: 128 rows x kIdxK features (rows = token-major (t, g) pairs)
      for (int e = tid; e < kIdxRows * kIdxK; e += kIdxThreads) {
        const int rr = e / kIdxK, kk = e % kIdxK;
        const int64_t R = row0 + rr;
        float v = 0.f;
        const int c = k0 + kk;
        if (R < nrows && c < D2) {
          const int64_t t = R / a.Hkv, g = R % a.Hkv;
          const int64_t off = t * a.stride_tok + g * a.stride_head;
          v = c < a.d ? load_x(a, a.K, off + c) : load_x(a, a.V, off + (c - a.d));
        }
        xs[kk][rr] = v;
      }
      for (int e = tid; e < kIdxHid * kIdxK; e += kIdxThreads) {
        const int hh = e / kIdxK, kk = e % kIdxK;
        const int u = h0 + hh, c = k0 + kk;
        ws[kk][hh] = (u < a.hidden && c < D2) ? a.W1[(int64_t)u * D2 + c] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < kIdxK; ++kk) {
        float xr[8], wr[16];
#pragma unroll
        for (int r = 0; r < 8; ++r) xr[r] = xs[kk][ty + 16 * r];
#pragma unroll
        for (int c = 0; c < 16; ++c) wr[c] = ws[kk][tx + 16 * c];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[r][c] = fmaf(xr[r], wr[c], acc[r][c]);
      }
      __syncthreads();
    }
    // ReLU + down-projection for this hidden slice
    float w2v[16], w2s[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int u = h0 + tx + 16 * c;
      w2v[c] = u < a.hidden ? a.W2[u] : 0.f;
      w2s[c] = u < a.hidden ? a.W2[a.hidden + u] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float pv = 0.f, ps = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float hv = fmaxf(acc[r][c], 0.f);
        pv = fmaf(w2v[c], hv, pv);
        ps = fmaf(w2s[c], hv, ps);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        pv += __shfl_xor_sync(0xffffffffu, pv, o);
        ps += __shfl_xor_sync(0xffffffffu, ps, o);
      }
      out_v[r] += pv;
      out_s[r] += ps;
    }
  }
  if (tx == 0) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int64_t R = row0 + ty + 16 * r;
      if (R < nrows) {
        const int64_t t = R / a.Hkv, g = R % a.Hkv;
        a.lv[g * a.N + t] = out_v[r];
        a.ls[g * a.N + t] = out_s[r];
      }
    }
  }
}

template <int ESZ>  // input element size: 2 (bf16) or 4 (fp32)
__global__ void __launch_bounds__(kIdxThreads) index_scores_vec_kernel(IdxArgs a) {
  __shared__ float xs[kIdxK][kIdxRows + 4];
  __shared__ float ws[kIdxK][kIdxHid + 4];
  constexpr int PER = 16 / ESZ;                  // elements per 16-byte piece
  constexpr int XP = kIdxRows * kIdxK / PER;     // X pieces per chunk (256 or 512)
  constexpr int XPT = XP / kIdxThreads;          // per thread (1 or 2)
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads
  const int g = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * kIdxRows;
  const int D2 = 2 * a.d;
  float out_v[8], out_s[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) out_v[r] = out_s[r] = 0.f;
  // loads of chunk k0: X piece e = (row, piece), W1 row tid (16 features)
  auto load_x = [&](int k0, uint4 (&xv)[XPT]) {
    const void* base = k0 < a.d ? a.K : a.V;
    const int c0 = k0 < a.d ? k0 : k0 - a.d;
#pragma unroll
    for (int j = 0; j < XPT; ++j) {
      const int e = tid + j * kIdxThreads, rr = e / (kIdxK / PER), pc = e % (kIdxK / PER);
      const int64_t t = t0 + rr;
      xv[j] = make_uint4(0u, 0u, 0u, 0u);
      if (t < a.N)
        xv[j] = __ldg(reinterpret_cast<const uint4*>(
                          static_cast<const uint8_t*>(base) +
                          (t * a.stride_tok + (int64_t)g * a.stride_head + c0) * ESZ) + pc);
    }
  };
  auto load_w = [&](int h0, int k0, float4 (&wv)[4]) {
    const int u = h0 + tid;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      wv[j] = u < a.hidden ? __ldg(reinterpret_cast<const float4*>(a.W1 + (int64_t)u * D2 + k0) + j)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto store_chunk = [&](const uint4 (&xv)[XPT], const float4 (&wv)[4]) {
#pragma unroll
    for (int j = 0; j < XPT; ++j) {
      const int e = tid + j * kIdxThreads, rr = e / (kIdxK / PER), pc = e % (kIdxK / PER);
      const uint32_t w[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
#pragma unroll
      for (int y = 0; y < PER; ++y) {
        const float v = ESZ == 2 ? __uint_as_float(((w[y >> 1] >> (16 * (y & 1))) & 0xffffu) << 16)
                                 : __uint_as_float(w[y]);
        xs[pc * PER + y][rr] = v;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ws[4 * j + 0][tid] = wv[j].x;
      ws[4 * j + 1][tid] = wv[j].y;
      ws[4 * j + 2][tid] = wv[j].z;
      ws[4 * j + 3][tid] = wv[j].w;
    }
  };

  for (int h0 = 0; h0 < a.hidden; h0 += kIdxHid) {
    float acc[8][16];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[r][c] = 0.f;
    uint4 xv[XPT];
    float4 wv[4];
    load_x(0, xv);
    load_w(h0, 0, wv);
    for (int k0 = 0; k0 < D2; k0 += kIdxK) {
      store_chunk(xv, wv);
      __syncthreads();
      if (k0 + kIdxK < D2) {  // the next chunk is in flight while this one is used
        load_x(k0 + kIdxK, xv);
        load_w(h0, k0 + kIdxK, wv);
      }
#pragma unroll 4
      for (int kk = 0; kk < kIdxK; ++kk) {
        float xr[8], wr[16];
#pragma unroll
        for (int r = 0; r < 8; ++r) xr[r] = xs[kk][ty + 16 * r];
#pragma unroll
        for (int c = 0; c < 16; ++c) wr[c] = ws[kk][tx + 16 * c];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[r][c] = fmaf(xr[r], wr[c], acc[r][c]);
      }
      __syncthreads();
    }
    float w2v[16], w2s[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int u = h0 + tx + 16 * c;
      w2v[c] = u < a.hidden ? a.W2[u] : 0.f;
      w2s[c] = u < a.hidden ? a.W2[a.hidden + u] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float pv = 0.f, ps = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float hv = fmaxf(acc[r][c], 0.f);
        pv = fmaf(w2v[c], hv, pv);
        ps = fmaf(w2s[c], hv, ps);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        pv += __shfl_xor_sync(0xffffffffu, pv, o);
        ps += __shfl_xor_sync(0xffffffffu, ps, o);
      }
      out_v[r] += pv;
      out_s[r] += ps;
    }
  }
  if (tx == 0) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int64_t t = t0 + ty + 16 * r;
      if (t < a.N) {
        a.lv[(int64_t)g * a.N + t] = out_v[r];
        a.ls[(int64_t)g * a.N + t] = out_s[r];
      }
    }
  }
}

cudaError_t launch_index_scores(const void* K, const void* V, int dtype, int N, int Hkv, int d,
                                int64_t stride_tok, int64_t stride_head, const float* W1,
                                const float* W2, int hidden, float* lv, float* ls,
                                cudaStream_t stream) {
  IdxArgs a{K, V, dtype, N, Hkv, d, stride_tok, stride_head, W1, W2, hidden, lv, ls};
  const int esz = dtype == VS_BF16 ? 2 : 4;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  const bool vec = d % kIdxK == 0 && (stride_tok * esz) % 16 == 0 && (stride_head * esz) % 16 == 0 &&
                   al16(K) && al16(V) && al16(W1) && (2 * d) % 4 == 0 && N <= (1 << 30);
  if (vec) {
    const dim3 grid((unsigned)((N + kIdxRows - 1) / kIdxRows), (unsigned)Hkv);
    if (esz == 2) index_scores_vec_kernel<2><<<grid, kIdxThreads, 0, stream>>>(a);
    else index_scores_vec_kernel<4><<<grid, kIdxThreads, 0, stream>>>(a);
    return cudaGetLastError();
  }
  const int64_t nrows = (int64_t)N * Hkv;
  const int grid = static_cast<int>((nrows + kIdxRows - 1) / kIdxRows);
  index_scores_kernel<<<grid, kIdxThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace vs

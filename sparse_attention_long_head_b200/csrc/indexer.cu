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
// index_scores_tc_kernel (bf16 inputs, d = 64 or 128, hidden = 128 or 256,
// heads contiguous in a token row, 16-byte aligned rows) runs X W1^T on the
// tensor cores: W1 = hi + lo with hi = bf16(W1) and lo = bf16(W1 - hi)
// (residual below 2^-17 of |W1|), and X W1^T = X hi^T + X lo^T as two bf16
// MMAs with fp32 accumulation (bf16 x bf16 products are exact in fp32).
// Persistent CTAs each keep one 128-unit hidden slice of both parts in shared
// memory (128-byte-swizzled, K-major).  TMA streams the 128-token X tiles
// through a ring of 64-feature boxes; the MMAs accumulate each 128 x 128 tile
// in one of two TMEM accumulators, so that the epilogue of one tile overlaps
// the MMAs of the next.  The epilogue applies ReLU and the slice's share of
// the down-projection and adds it to the logits (zeroed first; at most two
// slices, so the order of the two additions does not change the sum).  A
// device wait that runs out (a correct launch never does) leaves NaN in the
// logits of that tile and of the CTA's later tiles.
//
// index_scores_vec_kernel is the same computation for aligned inputs (16-byte
// aligned rows, d a multiple of 16): a CTA takes 128 consecutive tokens of
// one KV head, so its X rows are contiguous and load as 16-byte vectors, W1
// loads as float4, and the next K-chunk is in registers while the current
// one is multiplied.
#include "internal.h"
#include "ptx.cuh"

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

// Roles of the tensor-core kernel: warp 0 issues the TMA loads, warp 1 owns
// TMEM and issues the MMAs, warps 2..5 run the epilogue (warp w reads TMEM
// lanes 32 (w mod 4) .. 32 (w mod 4) + 31, as the hardware requires).
constexpr int kTcWarps = 6;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kTcEpiThreads = 128;
constexpr uint64_t kTcWaitNs = kDefaultWaitLimitNs;

template <int D>
struct IdxTc {
  static constexpr int KB = 2 * D / 64;                // 64-feature boxes of one [k; v] row
  static constexpr int kBox = 128 * 128;               // bytes of a 128-row x 64-bf16 box
  static constexpr int kStages = D == 128 ? 5 : 8;     // X ring, one box per stage
  static constexpr int kSmem = (2 * KB + kStages) * kBox + 1024;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    index_scores_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, IdxArgs a, int slices) {
  using C = IdxTc<D>;
  constexpr int KB = C::KB, kBox = C::kBox, S = C::kStages;
  extern __shared__ uint8_t dyn_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sW = smem;                  // [2 parts][KB boxes] of the W1 slice
  uint8_t* sR = smem + 2 * KB * kBox;  // X ring: S boxes
  __shared__ float w2s[2][128];
  // full[S], empty[S], accfull[2], accempty[2], drain
  __shared__ __align__(8) uint64_t bars[2 * S + 5];
  __shared__ uint32_t tslot;
  __shared__ int abort_flag, status_sink;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x % slices;   // hidden slice [128 j, 128 j + 128)
  const int D2 = 2 * D;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  // W1 slice -> hi / lo bf16 parts, 8 features (one 16-byte chunk) at a time
  for (int e = tid; e < 128 * (D2 / 8); e += kTcThreads) {
    const int n = e / (D2 / 8), c = (e % (D2 / 8)) * 8;
    const float4* src = reinterpret_cast<const float4*>(a.W1 + (int64_t)(128 * j + n) * D2 + c);
    const float4 f0 = __ldg(src), f1 = __ldg(src + 1);
    const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(f[2 * y]), h1 = __float2bfloat16_rn(f[2 * y + 1]);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(f[2 * y] - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(f[2 * y + 1] - __bfloat162float(h1));
      hi[y] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lo[y] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    const uint32_t off = (c / 64) * kBox + sw128_off(n, (c % 64) / 8);
    *reinterpret_cast<uint4*>(sW + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(sW + KB * kBox + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  for (int e = tid; e < 256; e += kTcThreads)
    w2s[e / 128][e % 128] = a.W2[(e / 128) * a.hidden + 128 * j + e % 128];
  if (tid == 0) {
    for (int i = 0; i < 2 * S; ++i) mbar_init(bar(i), 1);
    mbar_init(bar(2 * S), 1);
    mbar_init(bar(2 * S + 1), 1);
    mbar_init(bar(2 * S + 2), kTcEpiThreads);
    mbar_init(bar(2 * S + 3), kTcEpiThreads);
    mbar_init(bar(2 * S + 4), 1);
    abort_flag = 0;
    status_sink = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tslot), 256);  // two 128-column accumulators
    tmem_relinquish();
  }
  fence_proxy_async_smem();  // the W1 parts, written by threads, are read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  // the index launch has no status word: a timeout shows as NaN logits
  const WaitCtx wc{kTcWaitNs, &status_sink, &abort_flag};
  const int64_t items = (int64_t)((a.N + 127) / 128) * a.Hkv;  // (token tile, KV head)
  const int per = gridDim.x / slices;
  const int64_t first = blockIdx.x / slices;
  const int nmine = first < items ? (int)((items - 1 - first) / per + 1) : 0;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int q = 0;  // boxes issued
      bool live = true;
      for (int i = 0; i < nmine && live; ++i) {
        const int64_t it = first + (int64_t)i * per;
        const int g = (int)(it % a.Hkv);
        const int y = (int)((it / a.Hkv) * 128);
        for (int b = 0; b < KB; ++b) {
          const int st = q % S;
          if (q >= S && !mbar_wait(bar(S + st), (q / S - 1) & 1, wc)) {
            live = false;
            break;
          }
          mbar_arrive_expect_tx(bar(st), kBox);
          tma_load_2d(smem_u32(sR + st * kBox), b < KB / 2 ? &tmK : &tmV, bar(st),
                      g * D + (b % (KB / 2)) * 64, y);
          ++q;
        }
      }
      // copies still in flight land before the CTA exits (at once unless aborted)
      for (int r = q > S ? q - S : 0; r < q; ++r) mbar_wait_drain(bar(r % S), (r / S) & 1, kTcWaitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
      const uint64_t wdesc = sdesc_sw128(smem_u32(sW), 16, 1024);
      int q = 0;  // boxes consumed
      bool live = true;
      for (int i = 0; i < nmine && live; ++i) {
        const int acc = i & 1;
        if (i >= 2 && !mbar_wait(bar(2 * S + 2 + acc), ((i >> 1) - 1) & 1, wc)) break;
        tc_fence_after();
        const uint32_t tacc = tbase + acc * 128;
        for (int b = 0; b < KB; ++b, ++q) {
          const int st = q % S;
          if (!mbar_wait(bar(st), (q / S) & 1, wc)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint64_t xdesc = sdesc_sw128(smem_u32(sR + st * kBox), 16, 1024);
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tacc, xdesc + ((kk * 32) >> 4), wdesc + (((p * KB + b) * kBox + kk * 32) >> 4),
                     idesc, (b | p | kk) ? 1u : 0u);
          mma_commit(bar(S + st));  // the box's slot is free once these MMAs have read it
        }
        if (live) mma_commit(bar(2 * S + acc));
      }
      // every MMA issued has finished before TMEM is released
      mma_commit(bar(2 * S + 4));
      mbar_wait_drain(bar(2 * S + 4), 0, kTcWaitNs);
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    bool live = true;
    for (int i = 0; i < nmine; ++i) {
      const int64_t it = first + (int64_t)i * per;
      const int g = (int)(it % a.Hkv);
      const int64_t t = (it / a.Hkv) * 128 + row;
      const int acc = i & 1;
      float pv = __int_as_float(0x7fc00000), ps = pv;  // NaN unless the tile completes
      // warp-uniform, since tcgen05.ld is a warp-wide instruction
      if (live) live = __all_sync(0xffffffffu, mbar_wait(bar(2 * S + acc), (i >> 1) & 1, wc));
      if (live) {
        tc_fence_after();
        pv = ps = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v[32];
          tmem_ld32(tbase + acc * 128 + ((uint32_t)(quarter * 32) << 16) + 32 * q, v);
          tmem_ld_wait(v);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float h = fmaxf(__uint_as_float(v[c]), 0.f);
            pv = fmaf(w2s[0][32 * q + c], h, pv);
            ps = fmaf(w2s[1][32 * q + c], h, ps);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(2 * S + 2 + acc));
      }
      if (t < a.N) {
        atomicAdd(&a.lv[(int64_t)g * a.N + t], pv);
        atomicAdd(&a.ls[(int64_t)g * a.N + t], ps);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

cudaError_t launch_index_scores(const void* K, const void* V, int dtype, int N, int Hkv, int d,
                                int64_t stride_tok, int64_t stride_head, const float* W1,
                                const float* W2, int hidden, float* lv, float* ls,
                                cudaStream_t stream) {
  IdxArgs a{K, V, dtype, N, Hkv, d, stride_tok, stride_head, W1, W2, hidden, lv, ls};
  const int esz = dtype == VS_BF16 ? 2 : 4;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  const bool tc = dtype == VS_BF16 && (d == 64 || d == 128) && (hidden == 128 || hidden == 256) &&
                  stride_head == d && (stride_tok * 2) % 16 == 0 && al16(K) && al16(V) &&
                  al16(W1);
  if (tc) {
    EncodeTiledFn enc = get_encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap mK, mV;
    CUresult rc = CUDA_SUCCESS;
    encode_rows_bf16_sw128(enc, &mK, K, (int64_t)Hkv * d, N, stride_tok, &rc);
    encode_rows_bf16_sw128(enc, &mV, V, (int64_t)Hkv * d, N, stride_tok, &rc);
    if (rc != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int slices = hidden / 128;
    cudaError_t e = cudaMemsetAsync(lv, 0, sizeof(float) * (size_t)N * Hkv, stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(ls, 0, sizeof(float) * (size_t)N * Hkv, stream);
    if (e != cudaSuccess) return e;
    const int64_t items = ((int64_t)N + 127) / 128 * Hkv;
    int grid = device_sm_count() / slices * slices;
    if ((int64_t)grid > items * slices) grid = (int)(items * slices);
    if (grid < slices) grid = slices;
    if (d == 128) {
      e = cudaFuncSetAttribute(index_scores_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               IdxTc<128>::kSmem);
      if (e != cudaSuccess) return e;
      index_scores_tc_kernel<128><<<grid, kTcThreads, IdxTc<128>::kSmem, stream>>>(mK, mV, a, slices);
    } else {
      e = cudaFuncSetAttribute(index_scores_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               IdxTc<64>::kSmem);
      if (e != cudaSuccess) return e;
      index_scores_tc_kernel<64><<<grid, kTcThreads, IdxTc<64>::kSmem, stream>>>(mK, mV, a, slices);
    }
    return cudaGetLastError();
  }
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

// Ground-truth aggregation of full causal attention weights along vertical
// columns and slash diagonals, on sm_100a.
//
// The VSPrefill pages' distillation target ("VSPrefill ..." Technical
// Summary, section 2, "Distillation Training": a kernel sums the full
// attention weights along columns and diagonals during the block-wise
// computation, never materialising the n x n matrix).  For query head h:
//     A_v[j] = sum_{i >= j} p_ij,   A_s[o] = sum_{i >= o} p_{i, i-o},
// with p_ij = exp(scale * q_i . k_j - LSE_i) and LSE from the dense forward.
//
// Structure (320 threads, one persistent CTA per SM):
//   * A work unit is one (query head h, key block b): the n = T - b query
//     tiles t = b + j of that head against the 128 keys of block b.  The CTA
//     owns the block's 128 column sums, so A_v is written once, without
//     atomics.
//   * Warp 9 loads K(b) once per unit and streams the Q tiles through a
//     two-slot ring (TMA, 128-byte swizzle); warp 8 issues S = Q K^T
//     (tcgen05, M = N = 128).  There is no PV: the pass needs only the
//     weights.
//   * Warps 0-3 take the first half of the unit's tiles, warps 4-7 the
//     second; the issue order alternates between the halves.  Each half is
//     walked from a staggered start (a hash of the unit), so CTAs that run at
//     the same time do not all hit the same diagonal offsets.
//   * TMEM: per group one S buffer (released as soon as it is read) and one
//     128 x 128 fp32 accumulator of the group's weights, row by row.  Column
//     sums are taken from the accumulators once per unit.
//   * Diagonal sums per tile: a thread owns a row r and writes its weights to
//     row r of a shared buffer with rows padded to 129 floats (so the writes
//     of a warp fall in distinct banks).  Thread k then sums the diagonal at
//     local offset -k (elements (i, i + k)) and the one at 128 - k (elements
//     (i, i + k - 128)): walking rows from 128 - k with wrap-around, both are
//     strided runs of 130 floats, again in distinct banks across the warp.
//     The second diagonal of a tile and the first of the next tile of the walk
//     are the same offsets and the same thread, so they are added in a
//     register and sent to A_s with one fp32 atomic.
//   * Every wait is bounded (WaitCtx).  A failed wait is agreed on across a
//     group through bar.red before anyone leaves, so named barriers never
//     wait for a thread that is gone.
#include "internal.h"
#include "ptx.cuh"

namespace vs {

namespace {

constexpr int kAggThreads = 320;
constexpr int kAggWarpMMA = 8;
constexpr int kAggWarpLoad = 9;
constexpr int kAggQSlots = 2;

template <int D>
struct AggCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kRow = 129;                    // padded row of the weight buffer
  static constexpr int kSkewBytes = 128 * kRow * 4;   // one group's weights, fp32
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kAggQSlots * kTileBytes;
  static constexpr int kOffSkew = kOffK + kTileBytes;
  static constexpr int kOffComb = (kOffSkew + 2 * kSkewBytes + 15) / 16 * 16;  // 128 floats
  static constexpr int kOffBar = kOffComb + 512;
  static constexpr int kSmem = kOffBar + 256 + 1024;           // + alignment slack
};

struct AggParams {
  int N, Hq, Hkv, G, T, num_units;  // N, T: of the longest sequence
  int B;                            // sequences
  int64_t total;                    // token rows; lse, A_v, A_s are [Hq][total]
  const int32_t* cu;                // sequence offsets (device) or null
  float scale_log2;
  const float* lse;
  float* Av;
  float* As;
  int* status;
  uint64_t wait_limit_ns;
};

// Unit u: sequences in order, then heads, and within a head the longest
// walks (small b) first.  A key block past its sequence's end has n = 0 and
// is skipped by every role.
struct AggUnit {
  int h, b, n, n0, n1, st0, st1;
  int seq, Nb;    // the unit's sequence and its tokens
  int64_t tok0;   // its first token row
  bool ok_seq;    // false: malformed offsets (the sequence is empty)
};

__device__ __forceinline__ AggUnit agg_unit(const AggParams& P, int u) {
  AggUnit a;
  const int per_seq = P.Hq * P.T;
  a.seq = u / per_seq;
  u -= a.seq * per_seq;
  a.ok_seq = seq_range(P.cu, P.total, P.N, a.seq, a.tok0, a.Nb);
  a.h = u / P.T;
  a.b = u - a.h * P.T;
  a.n = max(0, (a.Nb + 127) / 128 - a.b);
  a.n0 = (a.n + 1) / 2;
  a.n1 = a.n - a.n0;
  const uint32_t x = (uint32_t)a.b * 2654435761u + (uint32_t)a.h * 40503u;
  a.st0 = a.n0 > 0 ? (int)((x >> 8) % (uint32_t)a.n0) : 0;
  a.st1 = a.n1 > 0 ? (int)((x >> 16) % (uint32_t)a.n1) : 0;
  return a;
}

// Tile j of the group's s-th step: a rotation of the group's half.
__device__ __forceinline__ int agg_tile(const AggUnit& a, int grp, int s) {
  if (grp == 0) {
    const int x = s + a.st0;
    return x >= a.n0 ? x - a.n0 : x;
  }
  const int x = s + a.st1;
  return a.n0 + (x >= a.n1 ? x - a.n1 : x);
}

template <int D>
__global__ void __launch_bounds__(kAggThreads, 1)
    agg_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const AggParams P) {
  using C = AggCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  float* skew_all = reinterpret_cast<float*>(smem + C::kOffSkew);
  float* comb = reinterpret_cast<float*>(smem + C::kOffComb);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  enum { B_QFULL = 0, B_QEMPTY = B_QFULL + kAggQSlots, B_KFULL = B_QEMPTY + kAggQSlots,
         B_KEMPTY = B_KFULL + 1, B_SFULL = B_KEMPTY + 1, B_SEMPTY = B_SFULL + 2,
         B_DRAIN = B_SEMPTY + 2, B_END = B_DRAIN + 1 };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + B_END);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kAggQSlots; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
    }
    mbar_init(bar(B_KFULL), 1);
    mbar_init(bar(B_KEMPTY), 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(B_SFULL + g), 1);
      mbar_init(bar(B_SEMPTY + g), 128);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kAggWarpLoad && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == kAggWarpMMA) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const WaitCtx wc{P.wait_limit_ns, P.status, abort_flag};

  if (warp < 8) {
    // ------------------------------------------------ weights and sums
    const int grp = warp >> 2;
    const int r = tid & 127;  // row of the tile this thread owns, and its column k
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + 256 * grp;  // S buffer
    const uint32_t tA = tS + 128;                       // row accumulator
    float* skew = skew_all + grp * 128 * C::kRow;
    float* srow = skew + r * C::kRow;
    const int w4 = warp & 3;  // rows / diagonals 32 w4 .. 32 w4 + 31 of this warp
    const int gbar = 1 + grp;
    uint32_t cnt = 0;  // this group's tiles so far (S buffer phase)
    bool ok = true;
    for (int u = blockIdx.x; u < P.num_units && ok; u += gridDim.x) {
      const AggUnit a = agg_unit(P, u);
      if (a.n == 0) continue;
      const int ng = grp == 0 ? a.n0 : a.n1;
      const float* lse_h = P.lse + (int64_t)a.h * P.total + a.tok0;
      float* As_h = P.As + (int64_t)a.h * P.total + a.tok0;
      {
        uint32_t z[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) z[c] = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_st32(tA + 32 * q, z);
        tmem_st_wait();
      }
      int64_t carry_off = -1;
      float carry = 0.f;
      // this row's LSE for the walk's next tile, loaded a tile ahead
      auto lse_of = [&](int s) -> float {
        const int64_t ii = 128 * (int64_t)(a.b + agg_tile(a, grp, s)) + r;
        return ii < a.Nb ? __ldg(lse_h + ii) : 0.f;
      };
      float lse_next = ng > 0 ? lse_of(0) : 0.f;
      for (int s = 0; s < ng && ok; ++s, ++cnt) {
        const int j = agg_tile(a, grp, s);
        const float lse_i = lse_next;
        if (s + 1 < ng) lse_next = lse_of(s + 1);
        bool w = mbar_wait(bar(B_SFULL + grp), cnt & 1, wc);
        __syncwarp();
        if (!named_bar_and(gbar, 128, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, sr[q]);
        tmem_ld_wait(sr[0]);
        reg_pin(sr[1]);
        reg_pin(sr[2]);
        reg_pin(sr[3]);
        tc_fence_before();
        mbar_arrive(bar(B_SEMPTY + grp));  // the S buffer may be overwritten
        const int64_t i = 128 * (int64_t)(a.b + j) + r;
        // rows past the sequence's end weigh nothing (their Q rows are the next
        // sequence's or zero-filled, so s is finite)
        const float nl = i < a.Nb ? -lse_i * 1.4426950408889634f : -INFINITY;
        if (j == 0) {  // the diagonal tile: keys after the row weigh nothing
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (32 * q + c > r) sr[q][c] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // 16 columns at a time: few live registers
          uint32_t acc[16];
          tmem_ld16(tA + 16 * q, acc);
          float p16[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            p16[c] = ex2_approx(fmaf(__uint_as_float(sr[q >> 1][16 * (q & 1) + c]), P.scale_log2, nl));
            srow[16 * q + c] = p16[c];
          }
          tmem_ld_wait16(acc);
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c] = __float_as_uint(__uint_as_float(acc[c]) + p16[c]);
          tmem_st16(tA + 16 * q, acc);
        }
        named_bar_sync(gbar, 128);
        // Thread k = r: diagonal -k holds (rr, rr + k) for rr < 128 - k, at
        // rr * 130 + k; diagonal 128 - k holds (rr, rr + k - 128) for
        // rr >= 128 - k, at rr * 130 + k - 128.  Visiting rr = 128 - k + m
        // (mod 128) for m = 0 .. 127 puts the lanes of a warp in distinct banks;
        // m < k is the second diagonal, and k spans 32 w4 .. 32 w4 + 31, so
        // only m in [32 w4, 32 w4 + 32) mixes the two within a warp.
        float da = 0.f, db = 0.f;
        {
          const float* pb = skew + (128 - r) * 130 + r - 128;  // m = 0 on diagonal 128 - k
          const float* pa = skew - 129 * r;  // pa + 130 m = (m - k) * 130 + k: diagonal -k
          const int m0 = 32 * w4, m1 = m0 + 32;
#pragma unroll 8
          for (int m = 0; m < m0; ++m) db += pb[130 * m];
#pragma unroll 8
          for (int m = m0; m < m1; ++m) {
            if (m < r) db += pb[130 * m];
            else da += pa[130 * m];
          }
#pragma unroll 8
          for (int m = m1; m < 128; ++m) da += pa[130 * m];
        }
        named_bar_sync(gbar, 128);  // the next tile rewrites the buffer
        tmem_st_wait();             // accumulator stores land before the next loads
        // local offset -r of tile j is global offset 128 j - r; 128 - r is
        // 128 (j + 1) - r, where the next tile of the walk starts
        const int64_t oa = 128 * (int64_t)j - r;
        if (carry_off == oa) {
          da += carry;
        } else if (carry_off >= 0 && carry_off < a.Nb && carry != 0.f) {
          atomicAdd(As_h + carry_off, carry);
        }
        if (oa >= 0 && oa < a.Nb && da != 0.f) atomicAdd(As_h + oa, da);
        carry = db;
        carry_off = r > 0 ? oa + 128 : -1;
      }
      if (ok && carry_off >= 0 && carry_off < a.Nb && carry != 0.f)
        atomicAdd(As_h + carry_off, carry);
      // column sums of this group's accumulator through the skewed buffer
      float cs = 0.f;
      if (ok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t acc[32];
          tmem_ld32(tA + 32 * q, acc);
          tmem_ld_wait(acc);
#pragma unroll
          for (int c = 0; c < 32; ++c) srow[32 * q + c] = __uint_as_float(acc[c]);
        }
      }
      __syncwarp();
      if (!named_bar_and(gbar, 128, ok)) ok = false;
      if (ok) {
#pragma unroll 8
        for (int rr = 0; rr < 128; ++rr) cs += skew[rr * C::kRow + r];
        named_bar_sync(gbar, 128);  // the next unit rewrites the buffer
      }
      // combine the two groups' column sums; group 0 writes A_v
      if (grp == 1) comb[r] = cs;
      __syncwarp();
      if (!named_bar_and(3, 256, ok)) {
        ok = false;
        break;
      }
      if (grp == 0) {
        const int64_t jcol = 128 * (int64_t)a.b + r;
        if (jcol < a.Nb) P.Av[(int64_t)a.h * P.total + a.tok0 + jcol] = cs + comb[r];
      }
      named_bar_sync(3, 256);  // comb is reused by the next unit
    }
  } else if (warp == kAggWarpMMA) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc = sdesc_sw128(smem_u32(sK), 16, 1024);
      uint32_t qseq = 0, kcount = 0, cnt[2] = {0, 0};
      bool ok = true;
      for (int u = blockIdx.x; u < P.num_units && ok; u += gridDim.x) {
        const AggUnit a = agg_unit(P, u);
        if (a.n == 0) continue;
        if (!mbar_wait(bar(B_KFULL), kcount & 1, wc)) { ok = false; break; }
        // the halves alternate: group 0's step s, then group 1's step s
        for (int x = 0; x < a.n && ok; ++x, ++qseq) {
          const int grp = x < 2 * a.n1 ? (x & 1) : 0;  // the last tile of an odd n is group 0's
          const uint32_t qs = qseq % kAggQSlots;
          if (!mbar_wait(bar(B_QFULL + qs), (qseq / kAggQSlots) & 1, wc)) { ok = false; break; }
          if (cnt[grp] > 0 &&
              !mbar_wait(bar(B_SEMPTY + grp), (cnt[grp] - 1) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = qdesc + ((qs * C::kTileBytes) >> 4);
          const uint32_t d = tbase + 256 * grp;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
            mma_ss(d, ad + off, kdesc + off, idesc_qk, kk > 0);
          }
          mma_commit(bar(B_SFULL + grp));
          mma_commit(bar(B_QEMPTY + qs));
          ++cnt[grp];
        }
        if (!ok) break;
        mma_commit(bar(B_KEMPTY));
        ++kcount;
      }
      mma_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0, P.wait_limit_ns);
    }
  } else if (warp == kAggWarpLoad) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t qseq = 0, kcount = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < P.num_units && ok; u += gridDim.x) {
        const AggUnit a = agg_unit(P, u);
        if (!a.ok_seq && a.h == 0 && a.b == 0) atomicOr(P.status, VS_DEVFLAG_BOUNDS);
        if (a.n == 0) continue;
        const int g = a.h / P.G;
        if (kcount > 0 && !mbar_wait(bar(B_KEMPTY), (kcount - 1) & 1, wc)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(B_KFULL), C::kTileBytes);
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_2d(smem_u32(sK + hh * 16384), &tmK, bar(B_KFULL), g * D + 64 * hh,
                      (int)(a.tok0 + 128 * a.b));
        ++kcount;
        for (int x = 0; x < a.n && ok; ++x, ++qseq) {
          const int s = x < 2 * a.n1 ? x >> 1 : x - a.n1;
          const int grp = x < 2 * a.n1 ? (x & 1) : 0;
          const int j = agg_tile(a, grp, s);
          const uint32_t qs = qseq % kAggQSlots;
          if (qseq >= (uint32_t)kAggQSlots &&
              !mbar_wait(bar(B_QEMPTY + qs), ((qseq / kAggQSlots) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(B_QFULL + qs), C::kTileBytes);
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_2d(smem_u32(sQ + qs * C::kTileBytes + hh * 16384), &tmQ, bar(B_QFULL + qs),
                        a.h * D + 64 * hh, (int)(a.tok0 + 128 * (a.b + j)));
        }
      }
      // let every issued copy land before shared memory is released
      const uint32_t first = qseq > (uint32_t)kAggQSlots ? qseq - kAggQSlots : 0;
      for (uint32_t x = first; x < qseq; ++x)
        mbar_wait_drain(bar(B_QFULL + (x % kAggQSlots)), (x / kAggQSlots) & 1, P.wait_limit_ns);
      if (kcount > 0) mbar_wait_drain(bar(B_KFULL), (kcount - 1) & 1, P.wait_limit_ns);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kAggWarpMMA) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int D>
cudaError_t launch_agg_impl(const AggArgs& a) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap mQ, mK;
  CUresult rc = CUDA_SUCCESS;
  encode_rows_bf16_sw128(enc, &mQ, a.Q, (int64_t)a.Hq * D, a.total, a.q_stride, &rc);
  encode_rows_bf16_sw128(enc, &mK, a.K, (int64_t)a.Hkv * D, a.total, a.kv_stride, &rc);
  if (rc != CUDA_SUCCESS) return cudaErrorInvalidValue;
  AggParams P;
  P.N = a.N;
  P.Hq = a.Hq;
  P.Hkv = a.Hkv;
  P.G = a.Hq / a.Hkv;
  P.T = (a.N + 127) / 128;
  P.num_units = a.B * a.Hq * P.T;
  P.B = a.B;
  P.total = a.total;
  P.cu = a.cu_seqlens;
  P.scale_log2 = a.scale * 1.4426950408889634f;
  P.lse = a.lse;
  P.Av = a.Av;
  P.As = a.As;
  P.status = a.status;
  P.wait_limit_ns = kDefaultWaitLimitNs;
  cudaError_t e = cudaFuncSetAttribute(agg_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       AggCfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = P.num_units < device_sm_count() ? P.num_units : device_sm_count();
  agg_kernel<D><<<grid, kAggThreads, AggCfg<D>::kSmem, a.stream>>>(mQ, mK, P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_aggregate(const AggArgs& a) {
  if (a.d == 128) return launch_agg_impl<128>(a);
  if (a.d == 64) return launch_agg_impl<64>(a);
  return cudaErrorInvalidValue;
}

}  // namespace vs

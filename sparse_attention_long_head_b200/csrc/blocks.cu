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
// and the diagonal block is always kept.  Everything is fp64, so the kept
// sets follow the definition up to rounding order.
//
//   block_mean_kernel: one CTA per (key block, KV head); thread c sums column
//     c of the block's keys in row order and writes the mean straight into
//     the operand layout of the fp64 tensor-core MMA below (blocks padded to
//     a multiple of 32 with zeros).
//   block_score_kernel: persistent, one CTA per SM, taking work items (query
//     block, up to four query heads of one KV group: 16 probes each, 8
//     probes per MMA n-tile) heaviest first from a counter.  The dot products
//     are mma.sync m16n8k16 fp64 (16 key blocks x 8 probes x 16 dims per
//     instruction: one instruction where vector code needs 64, at the same
//     fp64 rate).  A producer warp stages each item's probes as fp64 MMA
//     B-fragments in shared memory and streams the block means through a
//     ring of shared-memory stages (two 16-block tiles each) with bulk
//     copies; every tile of a stage feeds all the item's n-tiles.  Eight
//     consumer warps then run three passes per item:
//     pass 1: the dot products (stored in the CTA's scratch) and each
//       probe's maximum;
//     pass 2: e = exp(s - max) back into the scratch, and the sums Z;
//     pass 3: the block scores sum_p e / Z_p in shared memory, then each
//       head's maximum, threshold and bitmask row.
#include <cuda_bf16.h>

#include <cmath>

#include "exp64.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace vs {

namespace {

constexpr int kProbes = 16;
constexpr int kProbeStride = 8;
constexpr int kMaxBlocks = 2048;     // T <= 2048 (N <= 2^18)
constexpr int kBsWarps = 8;          // consumer (MMA) warps
constexpr int kBsThreads = 32 * (kBsWarps + 1);  // + the producer warp
constexpr int kTilesPerStage = 2;    // 16-block tiles per stage
constexpr int kPadBlocks = 16 * kTilesPerStage;
constexpr size_t kCounterOffset = 128;  // work-item counter, inside the status block
constexpr size_t kOneCtaSmem = 120 * 1024;
constexpr size_t kMaxDynSmem = 216 * 1024;  // with the static part, under the 227 KB opt-in limit

__host__ __device__ constexpr int pad_blocks(int T) { return (T + kPadBlocks - 1) / kPadBlocks * kPadBlocks; }

__device__ __forceinline__ double load_kv(const void* p, int dtype, int64_t off) {
  if (dtype == VS_BF16) return (double)__bfloat162float(static_cast<const __nv_bfloat16*>(p)[off]);
  return (double)static_cast<const float*>(p)[off];
}

// Contiguous global -> shared copy of `bytes` (a multiple of 16, both
// addresses 16-byte aligned) completing on mbarrier `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// c += A * B with A 16 x 16 (row), B 16 x 8 (col), fp64.  Lane (g, t) =
// (lane / 4, lane % 4) holds a[i] = A[g + 8 (i % 2)][t + 4 (i / 2)],
// b[i] = B[t + 4 i][g], c[i] = C[g + 8 (i / 2)][2 t + i % 2].
__device__ __forceinline__ void dmma_16816(double (&c)[4], const double (&a)[8],
                                           const double (&b)[4]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f64.f64.f64.f64 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7,%8,%9,%10,%11}, {%12,%13,%14,%15}, {%0,%1,%2,%3};"
      : "+d"(c[0]), "+d"(c[1]), "+d"(c[2]), "+d"(c[3])
      : "d"(a[0]), "d"(a[1]), "d"(a[2]), "d"(a[3]), "d"(a[4]), "d"(a[5]), "d"(a[6]), "d"(a[7]),
        "d"(b[0]), "d"(b[1]), "d"(b[2]), "d"(b[3]));
}

__global__ void exp_selftest_kernel(const double* x, double* y, int n) {
  __shared__ double tab[32];
  exp_table_init(tab);
  __syncthreads();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    y[i] = exp_nonpos(x[i], tab);
}

// Operand layout of the block means, per KV head g: tiles of 16 blocks, and
// per tile D / 16 k-steps of 16 dimensions; a k-step is 4 x [32 lanes][2]
// doubles, entry (j, lane = 4 r + t, e) holding kbar[16 tile + r + 8 e][16 ks
// + 4 j + t], i.e. a lane's A fragment of dmma_16816 as four 16-byte pieces
// that a warp reads as four conflict-free 512-byte rows.
__host__ __device__ __forceinline__ int64_t kbar_frag_off(int D, int Tp, int g, int J, int c) {
  const int tile = J >> 4, r = J & 15, ks = c >> 4, cc = c & 15;
  const int lane = 4 * (r & 7) + (cc & 3), j = cc >> 2, e = r >> 3;
  return (((int64_t)g * (Tp / 16) + tile) * (D / 16) + ks) * 256 + j * 64 + lane * 2 + e;
}

// One CTA per (key block J, KV head g, sequence b) of a batch packed along
// the token axis (cu: B + 1 offsets; null for one sequence of N tokens);
// the means of (b, g) are stored as those of KV head b * Hkv + g.  A
// malformed entry gives an empty sequence (zero means) and the bounds flag.
__global__ void __launch_bounds__(128) block_mean_kernel(const void* K, int dtype, int N, int d,
                                                         int64_t kv_stride, const int32_t* cu,
                                                         int64_t total, int* status,
                                                         double* kbar) {
  const int J = blockIdx.x, g = blockIdx.y, b = blockIdx.z, Tp = gridDim.x, Hkv = gridDim.y;
  int64_t tok0;
  int Nb;
  if (!seq_range(cu, total, N, b, tok0, Nb) && J == 0 && g == 0 && threadIdx.x == 0)
    atomicOr(status, VS_DEVFLAG_BOUNDS);
  const int Tb = (Nb + 127) / 128;
  const int64_t j0 = 128 * (int64_t)J, j1 = min((int64_t)Nb, j0 + 128);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double mean = 0.0;
    if (J < Tb) {
      double acc = 0.0;
      for (int64_t j = j0; j < j1; ++j)
        acc += load_kv(K, dtype, (tok0 + j) * kv_stride + (int64_t)g * d + c);
      mean = acc / (double)(j1 - j0);
    }
    kbar[kbar_frag_off(d, Tp, b * Hkv + g, J, c)] = mean;
  }
}

struct ScoreArgs {
  const void* Q;
  int dtype, N, Hq, Hkv, T, W, Tp, HC;  // HC: query heads per work item (1, 2 or 4)
  int n_items, n_chunks;                // items: (sequence, query block, chunk of HC heads)
  const int32_t* cu;                    // sequence offsets (device) or null
  int64_t total;
  int stages;                           // ring slots: 3, or 4 with two stage classes
  int64_t q_stride;
  double scale, alpha;
  const double* kbar;  // operand layout, [Hkv][Tp / 16 tiles]
  double* scratch;     // per CTA: the scaled dot products of its current item
  int64_t scratch_doubles;
  uint32_t* mask;
  int* status;
  int* counter;  // next work item
  uint64_t wait_limit_ns;
};

// Persistent: one CTA per SM; work items are (query block I, chunk of HC
// query heads), heaviest rows first, claimed from a global counter by the
// producer warp, which also stages each item's probes as fp64 B-fragments
// and streams its block means through the ring, so the next item's data
// arrives while the consumers finish the current one.  Per item the eight
// consumer warps run:
//   pass 1 (MMA): each warp owns one n-tile (8 probes), one or both tiles
//     of each stage and a class of stages (every stage when four heads share
//     an item; else the stage's two tiles go to two warps, and at one head
//     per item every other stage); the MMAs of its next stage are issued
//     before the epilogue of the current one, which stores the scaled dot
//     products in the CTA's scratch and keeps the probes' running maxima;
//   pass 2: e = exp(s - max) back into the scratch, and the sums Z;
//   pass 3: the scores sum_p e / Z_p over each head's 16 probes (two
//     addends, one per n-tile, per block), then each head's maximum,
//     threshold and mask row.  Every scratch entry is written and read back
//     by the same lane, so the passes need no fence.
template <int D, int TPW>
__global__ void __launch_bounds__(kBsThreads, 1) block_score_kernel(const ScoreArgs a) {
  constexpr int KS = D / 16;
  constexpr int kTileDoubles = 16 * D;
  constexpr int kStageDoubles = kTilesPerStage * kTileDoubles;
  constexpr uint32_t kStageBytes = sizeof(double) * kStageDoubles;
  constexpr int kCons = kBsWarps * 32;
  constexpr int TS = kTilesPerStage / TPW;  // warps sharing a stage's tiles
  constexpr int PF = 2;                     // scratch prefetch depth, in stages
  extern __shared__ __align__(128) double dyn[];
  const int NT = 2 * a.HC, WPN = kBsWarps / NT, SR = WPN / TS;
  // ring | bfrag | score: the two double2-accessed buffers first, so that
  // both start on 16-byte boundaries whatever HC * T is
  double* ring = dyn;  // a.stages slots
  // the item's probes as B fragments: per (n-tile, k-step) 2 x [32 lanes][2]
  // doubles, entry (j, lane = 4 g + t, e) = probe 8 (nt % 2) + g of head nt / 2
  // at dimension 16 ks + t + 4 (2 j + e)
  double* bfrag = ring + a.stages * kStageDoubles;
  double* score = bfrag + NT * KS * 128;  // [HC][T]
  __shared__ __align__(8) uint64_t full_bar[4], empty_bar[4], pfull_bar, pempty_bar;
  __shared__ double part[kBsWarps][4 * kProbes];
  __shared__ double st_m[4 * kProbes], st_rz[4 * kProbes];
  __shared__ double red[kBsWarps][4];
  __shared__ int item_slot;
  __shared__ int abort_flag;
  __shared__ double exp_tab[32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), NT * TS);
    }
    mbar_init(smem_u32(&pfull_bar), 1);
    mbar_init(smem_u32(&pempty_bar), kBsWarps);
    abort_flag = 0;
    fence_mbar_init();
  }
  exp_table_init(exp_tab);
  __syncthreads();
  const WaitCtx wc{a.wait_limit_ns, a.status, &abort_flag};
  const int esz = a.dtype == VS_BF16 ? 2 : 4;
  // Item k: sequence b = k / (T n_chunks), then query blocks from the last,
  // heaviest first.  An item whose block lies past its sequence's end
  // (valid = false) only writes zero mask rows.
  auto item_rows = [&](int k, int& b, int64_t& tok0, bool& valid, int& I, int& h0, int& np,
                       int& nsq) {
    const int per_seq = a.T * a.n_chunks;
    b = k / per_seq;
    const int rem = k - b * per_seq;
    I = a.T - 1 - rem / a.n_chunks;
    h0 = (rem % a.n_chunks) * a.HC;
    int Nb;
    seq_range(a.cu, a.total, a.N, b, tok0, Nb);
    valid = 128 * (int64_t)I < Nb;
    np = 0;
    while (valid && np < kProbes && 128 * (int64_t)I + kProbeStride * np < Nb) ++np;
    nsq = valid ? (I + 16 * kTilesPerStage - 1) / (16 * kTilesPerStage) : 0;  // 0 for I = 0
  };

  // ------------------------------------------------------------- producer
  if (warp == kBsWarps) {
    int s = 0;  // stages issued
    bool ok = true;
    for (int it = 0; ok; ++it) {
      int k = 0;
      if (lane == 0) k = atomicAdd(a.counter, 1);
      k = __shfl_sync(0xffffffffu, k, 0);
      // the fragment buffer is free once every consumer warp is past the last item's MMAs
      if (it > 0) {
        bool w = lane == 0 ? mbar_wait(smem_u32(&pempty_bar), (it - 1) & 1, wc) : true;
        if (!__shfl_sync(0xffffffffu, (int)w, 0)) break;
      }
      int I = 0, h0 = 0, np = 0, nsq = 0, bq = 0;
      int64_t tq0 = 0;
      bool valid = false;
      if (k < a.n_items) {
        item_rows(k, bq, tq0, valid, I, h0, np, nsq);
        if (valid && I > 0) {
          // Probe rows (the HC heads' D values are contiguous and 16-byte
          // aligned) in 16-byte pieces, eight per lane in flight, scattered
          // into fragment order; rows past the probes are zeros.
          const int per = 16 / esz;                  // elements per piece
          const int pieces = a.HC * D / per;         // per probe row
          for (int e0 = 0; e0 < kProbes * pieces; e0 += 8 * 32) {
            uint4 v[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const int e = e0 + 32 * x + lane, p = e / pieces;
              v[x] = make_uint4(0u, 0u, 0u, 0u);
              if (e < kProbes * pieces && p < np)
                v[x] = __ldg(reinterpret_cast<const uint4*>(
                                 static_cast<const uint8_t*>(a.Q) +
                                 ((tq0 + 128 * (int64_t)I + kProbeStride * p) * a.q_stride +
                                  (int64_t)h0 * D) * esz) + e % pieces);
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const int e = e0 + 32 * x + lane;
              if (e >= kProbes * pieces) continue;
              const int p = e / pieces, c0 = (e % pieces) * per;
              const uint32_t w[4] = {v[x].x, v[x].y, v[x].z, v[x].w};
              auto put = [&](int c, double val) {
                const int hl = c / D, dim = c % D;
                const int nt = 2 * hl + (p >> 3), cc = dim & 15, i = cc >> 2;
                bfrag[(nt * KS + (dim >> 4)) * 128 + (i >> 1) * 64 + (4 * (p & 7) + (cc & 3)) * 2 +
                      (i & 1)] = val;
              };
              if (esz == 2) {
#pragma unroll
                for (int y = 0; y < 8; ++y)  // bf16 -> fp32 is exact
                  put(c0 + y, (double)__uint_as_float(((w[y >> 1] >> (16 * (y & 1))) & 0xffffu) << 16));
              } else {
#pragma unroll
                for (int y = 0; y < 4; ++y) put(c0 + y, (double)__uint_as_float(w[y]));
              }
            }
          }
        }
      }
      if (lane == 0) item_slot = k;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&pfull_bar));  // release: the fragments and the item
      if (k >= a.n_items) break;
      if (lane == 0) {
        const double* src =
            a.kbar + ((int64_t)bq * a.Hkv + h0 / (a.Hq / a.Hkv)) * (a.Tp / 16) * kTileDoubles;
        for (int q = 0; q < nsq; ++q, ++s) {
          const int slot = s % a.stages, use = s / a.stages;
          if (use > 0 && !mbar_wait(smem_u32(&empty_bar[slot]), (use - 1) & 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(smem_u32(&full_bar[slot]), kStageBytes);
          bulk_load(smem_u32(ring + slot * kStageDoubles), src + (int64_t)q * kStageDoubles,
                    kStageBytes, smem_u32(&full_bar[slot]));
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
    }
    // copies still in flight (after an abort) land before the CTA exits
    if (lane == 0)
      for (int x = max(0, s - a.stages); x < s; ++x)
        mbar_wait_drain(smem_u32(&full_bar[x % a.stages]), (x / a.stages) & 1, a.wait_limit_ns);
    return;
  }

  // ------------------------------------------------------------ consumers
  const int nt = warp % NT, sub = warp / NT;
  const int m0 = (sub % TS) * TPW, cls = sub / TS;  // first tile of a stage; stage class
  const int hl = nt >> 1, pb = 8 * (nt & 1);
  const int gq = lane >> 2, t = lane & 3;
  double* scr = a.scratch + (int64_t)blockIdx.x * a.scratch_doubles;
  // scratch: per (stage, n-tile, tile) 2 x [32 lanes] double2 (a lane's 4 values)
  auto scr_at = [&](int q, int m) {
    return reinterpret_cast<double2*>(scr + (((int64_t)q * NT + nt) * kTilesPerStage + m) * 128) +
           lane;
  };
  int s0 = 0;  // stages consumed before the current item
  for (int it = 0;; ++it) {
    bool ok = mbar_wait(smem_u32(&pfull_bar), it & 1, wc);
    if (!named_bar_and(1, kCons, ok)) break;
    const int k = item_slot;
    if (k >= a.n_items) break;
    int I, h0, np, nsq, bq;
    int64_t tq0;
    bool valid;
    item_rows(k, bq, tq0, valid, I, h0, np, nsq);
    const int sb = s0;
    s0 += nsq;
    // the item's mask rows: heads h0 .. h0 + HC - 1 of sequence bq, block I
    auto mask_row = [&](int x) {
      return a.mask + (((int64_t)bq * a.Hq + h0 + x) * a.T + I) * a.W;
    };
    if (!valid || I == 0) {  // past the sequence's end: nothing; block 0: the diagonal alone
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&pempty_bar));
      for (int e = tid; e < a.HC * a.W; e += kCons) {
        const int x = e / a.W, w = e % a.W;
        mask_row(x)[w] = (valid && w == 0) ? 1u : 0u;
      }
      continue;
    }
    const double2* bsrc = reinterpret_cast<const double2*>(bfrag + nt * KS * 128) + lane;
    // Issues stage q's MMAs into acc[u] (block 16 (2 q + m0 + u) + gq + 8 (i / 2),
    // probe pb + 2 t + i % 2) and releases the stage's slot.
    auto issue = [&](int q, double (&acc)[TPW][4]) -> bool {
      const int s = sb + q, slot = s % a.stages;
      if (!mbar_wait(smem_u32(&full_bar[slot]), (s / a.stages) & 1, wc)) return false;
      const double* sA = ring + slot * kStageDoubles;
#pragma unroll
      for (int u = 0; u < TPW; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[u][i] = 0.0;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const double2 b01 = bsrc[ks * 64], b23 = bsrc[ks * 64 + 32];
        const double bf[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          const double2* src =
              reinterpret_cast<const double2*>(sA + ((m0 + u) * KS + ks) * 256) + lane;
          double af[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const double2 x = src[32 * j];
            af[2 * j] = x.x;
            af[2 * j + 1] = x.y;
          }
          dmma_16816(acc[u], af, bf);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty_bar[slot]));  // release orders the reads
      return true;
    };
    const bool pv0 = pb + 2 * t < np, pv1 = pb + 2 * t + 1 < np;  // this thread's probe columns

    // Pass 1: the dot products into the scratch, and the running maxima.
    double mr[2] = {-INFINITY, -INFINITY};
    {
      double cur[TPW][4], nxt[TPW][4];
      int q = cls;
      if (q < nsq && ok) ok = issue(q, cur);
      for (; q < nsq && ok; q += SR) {
        const int qn = q + SR;
        if (qn < nsq && !issue(qn, nxt)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          const int m = m0 + u;
          double v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = cur[u][i] * a.scale;
          double2* dst = scr_at(q, m);
          dst[0] = make_double2(v[0], v[1]);
          dst[32] = make_double2(v[2], v[3]);
          const int J0 = 16 * (kTilesPerStage * q + m) + gq, J1 = J0 + 8;
          if (J0 < I) {
            if (pv0) mr[0] = fmax(mr[0], v[0]);
            if (pv1) mr[1] = fmax(mr[1], v[1]);
          }
          if (J1 < I) {
            if (pv0) mr[0] = fmax(mr[0], v[2]);
            if (pv1) mr[1] = fmax(mr[1], v[3]);
          }
        }
#pragma unroll
        for (int u = 0; u < TPW; ++u)
#pragma unroll
          for (int i = 0; i < 4; ++i) cur[u][i] = nxt[u][i];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&pempty_bar));  // this warp's MMAs are issued
    // maxima over the 8 lanes sharing a column, then over the n-tile's warps
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) mr[c] = fmax(mr[c], __shfl_xor_sync(0xffffffffu, mr[c], o));
    if (gq == 0) {
      part[sub][hl * kProbes + pb + 2 * t] = mr[0];
      part[sub][hl * kProbes + pb + 2 * t + 1] = mr[1];
    }
    if (!named_bar_and(1, kCons, ok)) break;
    if (tid < a.HC * kProbes) {
      double m = part[0][tid];
      for (int w = 1; w < WPN; ++w) m = fmax(m, part[w][tid]);
      st_m[tid] = m;
    }
    named_bar_sync(1, kCons);

    // Streams this warp's scratch entries (stages q = cls, cls + SR, ...)
    // with PF stages in flight, calling f(q, m, v[4]) per tile and storing v
    // back when `wb`.
    auto sweep = [&](bool wb, auto&& f) {
      double2 buf[PF][2 * TPW];
#pragma unroll
      for (int x = 0; x < PF; ++x) {
        const int q = cls + x * SR;
        if (q < nsq)
#pragma unroll
          for (int u = 0; u < TPW; ++u) {
            buf[x][2 * u] = scr_at(q, m0 + u)[0];
            buf[x][2 * u + 1] = scr_at(q, m0 + u)[32];
          }
      }
      for (int q = cls; q < nsq; q += SR) {
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          double v[4] = {buf[0][2 * u].x, buf[0][2 * u].y, buf[0][2 * u + 1].x,
                         buf[0][2 * u + 1].y};
          f(q, m0 + u, v);
          if (wb) {
            scr_at(q, m0 + u)[0] = make_double2(v[0], v[1]);
            scr_at(q, m0 + u)[32] = make_double2(v[2], v[3]);
          }
        }
#pragma unroll
        for (int x = 0; x + 1 < PF; ++x)
#pragma unroll
          for (int j = 0; j < 2 * TPW; ++j) buf[x][j] = buf[x + 1][j];
        const int qn = q + PF * SR;
        if (qn < nsq)
#pragma unroll
          for (int u = 0; u < TPW; ++u) {
            buf[PF - 1][2 * u] = scr_at(qn, m0 + u)[0];
            buf[PF - 1][2 * u + 1] = scr_at(qn, m0 + u)[32];
          }
      }
    };

    // Pass 2: e = exp(s - max) (0 outside J < I or past the probes) and Z.
    {
      const double pm0 = st_m[hl * kProbes + pb + 2 * t], pm1 = st_m[hl * kProbes + pb + 2 * t + 1];
      double z0 = 0.0, z1 = 0.0;
      sweep(true, [&](int q, int m, double (&v)[4]) {
        const int J0 = 16 * (kTilesPerStage * q + m) + gq, J1 = J0 + 8;
        v[0] = pv0 && J0 < I ? exp_nonpos(v[0] - pm0, exp_tab) : 0.0;
        v[1] = pv1 && J0 < I ? exp_nonpos(v[1] - pm1, exp_tab) : 0.0;
        v[2] = pv0 && J1 < I ? exp_nonpos(v[2] - pm0, exp_tab) : 0.0;
        v[3] = pv1 && J1 < I ? exp_nonpos(v[3] - pm1, exp_tab) : 0.0;
        z0 += v[0] + v[2];
        z1 += v[1] + v[3];
      });
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        z0 += __shfl_xor_sync(0xffffffffu, z0, o);
        z1 += __shfl_xor_sync(0xffffffffu, z1, o);
      }
      if (gq == 0) {
        part[sub][hl * kProbes + pb + 2 * t] = z0;
        part[sub][hl * kProbes + pb + 2 * t + 1] = z1;
      }
    }
    for (int e = tid; e < a.HC * I; e += kCons) score[(e / I) * a.T + e % I] = 0.0;
    named_bar_sync(1, kCons);
    if (tid < a.HC * kProbes) {
      double z = part[0][tid];
      for (int w = 1; w < WPN; ++w) z += part[w][tid];
      st_rz[tid] = 1.0 / z;
    }
    named_bar_sync(1, kCons);

    // Pass 3: block scores (sums over the probes; the mean's 1/np cancels
    // in the comparison with alpha times the best).
    {
      const double r0 = pv0 ? st_rz[hl * kProbes + pb + 2 * t] : 0.0;
      const double r1 = pv1 ? st_rz[hl * kProbes + pb + 2 * t + 1] : 0.0;
      sweep(false, [&](int q, int m, double (&v)[4]) {
        const int J0 = 16 * (kTilesPerStage * q + m) + gq, J1 = J0 + 8;
        double ra = v[0] * r0 + v[1] * r1, rb = v[2] * r0 + v[3] * r1;
        ra += __shfl_xor_sync(0xffffffffu, ra, 1);
        ra += __shfl_xor_sync(0xffffffffu, ra, 2);
        rb += __shfl_xor_sync(0xffffffffu, rb, 1);
        rb += __shfl_xor_sync(0xffffffffu, rb, 2);
        // 0 + x is exact and x + y == y + x, so the order of the two
        // n-tiles' additions does not change the sum
        if (t == 0 && J0 < I) atomicAdd(&score[hl * a.T + J0], ra);
        if (t == 0 && J1 < I) atomicAdd(&score[hl * a.T + J1], rb);
      });
    }
    named_bar_sync(1, kCons);

    // Threshold and bitmask rows of the item's heads.
    double best[4] = {0.0, 0.0, 0.0, 0.0};
    for (int J = tid; J < I; J += kCons)
#pragma unroll
      for (int x = 0; x < 4; ++x)
        if (x < a.HC) best[x] = fmax(best[x], score[x * a.T + J]);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) best[x] = fmax(best[x], __shfl_xor_sync(0xffffffffu, best[x], o));
      if (lane == 0) red[warp][x] = best[x];
    }
    named_bar_sync(1, kCons);
    for (int x = 0; x < a.HC; ++x) {
      double b = red[0][x];
#pragma unroll
      for (int w = 1; w < kBsWarps; ++w) b = fmax(b, red[w][x]);
      const double thr = a.alpha * b;
      const double* sc = score + x * a.T;
      uint32_t* out = mask_row(x);
      for (int w = warp; w < a.W; w += kBsWarps) {
        const int J = 32 * w + lane;
        const bool keep = J == I || (J < I && sc[J] >= thr);
        const uint32_t bits = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) out[w] = bits;
      }
    }
  }
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Per-CTA scratch: every stage's dot products for up to 8 n-tiles.
int64_t scratch_doubles_per_cta(int Tp) { return (int64_t)(Tp / (16 * kTilesPerStage)) * 8 * 256; }

}  // namespace

cudaError_t launch_exp_selftest(const double* x, double* y, int n, cudaStream_t stream) {
  exp_selftest_kernel<<<(n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

size_t block_select_ws_bytes(int N, int B_Hkv, int d) {
  const int T = (N + 127) / 128, Tp = pad_blocks(T), sms = num_sms();
  return kStatusBytes + align_up(sizeof(double) * (size_t)B_Hkv * Tp * d, 256) +
         sizeof(double) * (size_t)(sms > 0 ? sms : 1) * scratch_doubles_per_cta(Tp);
}

cudaError_t launch_block_select(const BlockSelectArgs& a) {
  const int T = (a.N + 127) / 128, W = (T + 31) / 32, Tp = pad_blocks(T);
  if (T > kMaxBlocks || (a.d != 128 && a.d != 64)) return cudaErrorInvalidValue;
  const int sms = num_sms();
  if (sms < 1) return cudaErrorInvalidDevice;
  const int G = a.Hq / a.Hkv;
  const int HC = G % 4 == 0 ? 4 : (G % 2 == 0 ? 2 : 1);
  char* base = static_cast<char*>(a.ws);
  double* kbar = reinterpret_cast<double*>(base + kStatusBytes);
  double* scratch = reinterpret_cast<double*>(
      base + kStatusBytes + align_up(sizeof(double) * (size_t)a.B * a.Hkv * Tp * a.d, 256));
  block_mean_kernel<<<dim3(Tp, a.Hkv, a.B), 128, 0, a.stream>>>(
      a.K, a.dtype, a.N, a.d, a.kv_stride, a.cu_seqlens, a.total, static_cast<int*>(a.ws), kbar);
  ScoreArgs s;
  s.Q = a.Q;
  s.dtype = a.dtype;
  s.N = a.N;
  s.Hq = a.Hq;
  s.Hkv = a.Hkv;
  s.T = T;
  s.W = W;
  s.Tp = Tp;
  s.HC = HC;
  s.n_chunks = a.Hq / HC;
  s.n_items = a.B * T * s.n_chunks;
  s.cu = a.cu_seqlens;
  s.total = a.total;
  s.q_stride = a.q_stride;
  s.scale = a.scale;
  s.alpha = a.alpha;
  s.kbar = kbar;
  s.scratch = scratch;
  s.scratch_doubles = scratch_doubles_per_cta(Tp);
  s.mask = a.mask;
  s.status = static_cast<int*>(a.ws);
  s.counter = reinterpret_cast<int*>(base + kCounterOffset);
  s.wait_limit_ns = kDefaultWaitLimitNs;
  const int NT = 2 * HC, TS = HC == 4 ? 1 : 2, SR = kBsWarps / NT / TS;
  // ring slots: a multiple of the stage-class count SR, as many as fit
  auto dyn_bytes = [&](int stages) {
    return sizeof(double) * ((size_t)stages * kTilesPerStage * 16 * a.d + (size_t)HC * T +
                             (size_t)NT * a.d * 8);
  };
  s.stages = SR == 1 ? 3 : 4;
  if (dyn_bytes(s.stages) > kMaxDynSmem) s.stages = 2;
  const size_t need = dyn_bytes(s.stages);
  if (need > kMaxDynSmem) return cudaErrorInvalidValue;
  // more than half of an SM's shared memory: the persistent grid (one CTA
  // per SM) cannot pile two CTAs onto one SM while another stays idle
  const size_t smem = need > kOneCtaSmem ? need : kOneCtaSmem;
  auto kern = a.d == 128 ? (HC == 4 ? block_score_kernel<128, 2> : block_score_kernel<128, 1>)
                         : (HC == 4 ? block_score_kernel<64, 2> : block_score_kernel<64, 1>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = sms < s.n_items ? sms : s.n_items;
  kern<<<grid, kBsThreads, smem, a.stream>>>(s);
  return cudaGetLastError();
}

}  // namespace vs

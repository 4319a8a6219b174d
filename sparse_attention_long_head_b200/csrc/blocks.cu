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
//     fp64 rate).  Each consumer warp keeps its n-tile's probe fragments in
//     registers; a producer warp streams the block means through a ring of
//     shared-memory stages (two 16-block tiles each) with bulk copies, and
//     every tile of a stage feeds all the item's n-tiles.
//     Pass 1: the dot products, each probe's online maximum and sum of
//     exponentials, and the dot products stored in the CTA's scratch.
//     Pass 2: from the scratch, each probe's normalised exponentials summed
//     over the head's 16 probes give the block scores in shared memory;
//     then the maximum, the threshold and the row's bitmask.
#include <cuda_bf16.h>

#include <cmath>

#include "internal.h"
#include "ptx.cuh"

namespace vs {

namespace {

constexpr int kProbes = 16;
constexpr int kProbeStride = 8;
constexpr int kMaxBlocks = 2048;     // T <= 2048 (N <= 2^18)
constexpr int kBsWarps = 8;          // consumer (MMA) warps
constexpr int kBsThreads = 32 * (kBsWarps + 1);
constexpr int kBsStages = 4;         // shared-memory ring (a multiple of every stage-class count)
constexpr int kTilesPerStage = 2;    // 16-block tiles per stage
constexpr int kPadBlocks = 16 * kTilesPerStage;
constexpr size_t kCounterOffset = 128;  // work-item counter, inside the status block
constexpr size_t kOneCtaSmem = 120 * 1024;

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

__global__ void __launch_bounds__(128) block_mean_kernel(const void* K, int dtype, int N, int T,
                                                         int d, int64_t kv_stride, double* kbar) {
  const int J = blockIdx.x, g = blockIdx.y, Tp = gridDim.x;
  const int64_t j0 = 128 * (int64_t)J, j1 = min((int64_t)N, j0 + 128);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double mean = 0.0;
    if (J < T) {
      double acc = 0.0;
      for (int64_t j = j0; j < j1; ++j) acc += load_kv(K, dtype, j * kv_stride + (int64_t)g * d + c);
      mean = acc / (double)(j1 - j0);
    }
    kbar[kbar_frag_off(d, Tp, g, J, c)] = mean;
  }
}

struct ScoreArgs {
  const void* Q;
  int dtype, N, Hq, Hkv, T, W, Tp, HC;  // HC: query heads per work item (1, 2 or 4)
  int n_items, n_chunks;                // items: (query block, chunk of HC heads)
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

// Online (max, sum of exp(x - max)) merge; symmetric in its two operands, so
// both lanes of a butterfly step end with identical values.
__device__ __forceinline__ void lse_merge(double& m1, double& z1, double m2, double z2) {
  const double mn = fmax(m1, m2);
  if (mn == -INFINITY) return;
  z1 = (m1 == -INFINITY ? 0.0 : z1 * exp(m1 - mn)) + (m2 == -INFINITY ? 0.0 : z2 * exp(m2 - mn));
  m1 = mn;
}

// Persistent: one CTA per SM takes work items (query block I, chunk of HC
// query heads), heaviest rows first, from a global counter.  Per item:
//   pass 1 (MMA): each consumer warp owns one n-tile (8 probes), one or
//     both tiles of each stage, and a class of stages (every stage when four
//     heads share an item, else every other stage with one tile per warp at
//     one head per item); the MMAs of its next stage are issued
//     before the epilogue of the current one, which updates the probes'
//     online (max, sum of exponentials) and stores the scaled dot products
//     in the CTA's scratch (L2-resident, read back by the same lanes);
//   pass 2 (no MMA): the normalised exponentials from the scratch, summed
//     over each head's 16 probes, give the block scores in shared memory;
//   then each head's maximum, threshold and mask row.
// TPW: 16-block tiles of a stage per warp -- 2 when an item has 8 n-tiles
// (four heads), else 1 (the stage's two tiles go to two warps).
template <int D, int TPW>
__global__ void __launch_bounds__(kBsThreads, 1) block_score_kernel(const ScoreArgs a) {
  constexpr int KS = D / 16;
  constexpr int kTileDoubles = 16 * D;
  constexpr int kStageDoubles = kTilesPerStage * kTileDoubles;
  constexpr uint32_t kStageBytes = sizeof(double) * kStageDoubles;
  constexpr int kCons = kBsWarps * 32;
  extern __shared__ __align__(128) double dyn[];
  double* ring = dyn;                                 // kBsStages stages
  double* score = ring + kBsStages * kStageDoubles;   // [HC][T]
  __shared__ __align__(8) uint64_t full_bar[kBsStages], empty_bar[kBsStages];
  __shared__ double part_m[kBsWarps][4 * kProbes], part_z[kBsWarps][4 * kProbes];
  __shared__ double st_m[4 * kProbes], st_rz[4 * kProbes];
  __shared__ double red[kBsWarps];
  __shared__ int item_buf[2];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // n-tiles; warps per n-tile; warps splitting a stage's tiles; stage
  // classes (stage q is consumed by the warps of class q % SR, and since SR
  // divides kBsStages each ring slot serves one class, whose warps wait for
  // the slot's phases in order)
  constexpr int TS = kTilesPerStage / TPW;
  const int NT = 2 * a.HC, WPN = kBsWarps / NT, SR = WPN / TS;
  if (tid == 0) {
    for (int s = 0; s < kBsStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), NT * TS);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  const WaitCtx wc{a.wait_limit_ns, a.status, &abort_flag};
  double* scr = a.scratch + (int64_t)blockIdx.x * a.scratch_doubles;
  int s0 = 0;      // stages issued / consumed before the current item
  int issued = 0;  // producer: stages whose copies were issued
  bool ok = true;  // this thread's bounded waits all succeeded
  for (int it = 0;; ++it) {
    if (tid == 0) item_buf[it & 1] = atomicAdd(a.counter, 1);
    if (__syncthreads_or(!ok)) break;
    const int k = item_buf[it & 1];
    if (k >= a.n_items) break;
    const int I = a.T - 1 - k / a.n_chunks;
    const int h0 = (k % a.n_chunks) * a.HC;
    const int g = h0 / (a.Hq / a.Hkv);
    if (I == 0) {  // no earlier block: the diagonal alone
      for (int e = tid; e < a.HC * a.W; e += blockDim.x) {
        const int hl = e / a.W, w = e % a.W;
        a.mask[((int64_t)(h0 + hl) * a.T) * a.W + w] = w == 0 ? 1u : 0u;
      }
      continue;
    }
    int np = 0;
    while (np < kProbes && 128 * (int64_t)I + kProbeStride * np < a.N) ++np;
    const int nsq = (I + 16 * kTilesPerStage - 1) / (16 * kTilesPerStage);  // stages
    const int sb = s0;
    s0 += nsq;

    if (warp == kBsWarps) {  // producer
      if (lane == 0) {
        const double* src = a.kbar + (int64_t)g * (a.Tp / 16) * kTileDoubles;
        for (int q = 0; q < nsq && ok; ++q) {
          const int s = sb + q, slot = s % kBsStages, use = s / kBsStages;
          if (use > 0 && !mbar_wait(smem_u32(&empty_bar[slot]), (use - 1) & 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(smem_u32(&full_bar[slot]), kStageBytes);
          bulk_load(smem_u32(ring + slot * kStageDoubles), src + (int64_t)q * kStageDoubles,
                    kStageBytes, smem_u32(&full_bar[slot]));
          issued = s + 1;
        }
      }
      continue;
    }

    // ---------------------------------------------------------- consumers
    const int nt = warp % NT, sub = warp / NT;
    const int m0 = (sub % TS) * TPW, cls = sub / TS;  // first tile of the stage; stage class
    const int hl = nt >> 1, pb = 8 * (nt & 1);
    const int gq = lane >> 2, t = lane & 3;
    double bq[KS][4];  // B fragments: probe pb + gq of head h0 + hl
    {
      const int p = pb + gq;
      const int64_t base =
          (128 * (int64_t)I + kProbeStride * p) * a.q_stride + (int64_t)(h0 + hl) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          bq[ks][i] = p < np ? load_kv(a.Q, a.dtype, base + 16 * ks + t + 4 * i) : 0.0;
    }
    // Issues stage q's MMAs into acc[u] (block 16 (2 q + m0 + u) + gq + 8 (i / 2),
    // probe pb + 2 t + i % 2) and releases the stage's slot.
    auto issue = [&](int q, double (&acc)[TPW][4]) -> bool {
      const int s = sb + q, slot = s % kBsStages;
      if (!mbar_wait(smem_u32(&full_bar[slot]), (s / kBsStages) & 1, wc)) return false;
      const double* sA = ring + slot * kStageDoubles;
#pragma unroll
      for (int u = 0; u < TPW; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[u][i] = 0.0;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
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
          dmma_16816(acc[u], af, bq[ks]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty_bar[slot]));  // release orders the reads
      return true;
    };
    // scratch: per (stage, n-tile, tile) 2 x [32 lanes] double2 (a lane's 4
    // values); each entry is written and read back by the same lane
    auto scr_at = [&](int q, int m) {
      return reinterpret_cast<double2*>(scr + (((int64_t)q * NT + nt) * kTilesPerStage + m) * 128) +
             lane;
    };

    // Pass 1: online maximum and sum of exponentials of this thread's two
    // probe columns; the dot products go to the scratch.
    double mr[2] = {-INFINITY, -INFINITY}, zr[2] = {0.0, 0.0};
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
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (pb + 2 * t + c >= np) continue;
            const bool oa = J0 < I, ob = J1 < I;
            const double tm = fmax(oa ? v[c] : -INFINITY, ob ? v[2 + c] : -INFINITY);
            if (tm > mr[c]) {
              zr[c] = mr[c] == -INFINITY ? 0.0 : zr[c] * exp(mr[c] - tm);
              mr[c] = tm;
            }
            if (oa) zr[c] += exp(v[c] - mr[c]);
            if (ob) zr[c] += exp(v[2 + c] - mr[c]);
          }
        }
#pragma unroll
        for (int u = 0; u < TPW; ++u)
#pragma unroll
          for (int i = 0; i < 4; ++i) cur[u][i] = nxt[u][i];
      }
    }
    // over the 8 lanes that share a column, then over the warps of the n-tile
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1)
        lse_merge(mr[c], zr[c], __shfl_xor_sync(0xffffffffu, mr[c], o),
                  __shfl_xor_sync(0xffffffffu, zr[c], o));
    if (gq == 0) {  // one partial per warp of the n-tile
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        part_m[sub][hl * kProbes + pb + 2 * t + c] = mr[c];
        part_z[sub][hl * kProbes + pb + 2 * t + c] = zr[c];
      }
    }
    for (int e = tid; e < a.HC * I; e += kCons) score[(e / I) * a.T + e % I] = 0.0;
    ok = named_bar_and(1, kCons, ok);
    if (!ok) continue;
    if (tid < a.HC * kProbes) {
      double m = part_m[0][tid], z = part_z[0][tid];
      for (int w = 1; w < WPN; ++w) lse_merge(m, z, part_m[w][tid], part_z[w][tid]);
      st_m[tid] = m;
      st_rz[tid] = 1.0 / z;
    }
    named_bar_sync(1, kCons);

    // Pass 2: Score(I, J) sums, two addends (one per n-tile) per (head, J).
    {
      double pm[2], prz[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        pm[c] = st_m[hl * kProbes + pb + 2 * t + c];
        prz[c] = st_rz[hl * kProbes + pb + 2 * t + c];
      }
      double2 cur[2 * TPW], nxt[2 * TPW];
      int q = cls;
      if (q < nsq) {
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          cur[2 * u] = scr_at(q, m0 + u)[0];
          cur[2 * u + 1] = scr_at(q, m0 + u)[32];
        }
      }
      for (; q < nsq; q += SR) {
        const int qn = q + SR;
        if (qn < nsq) {
#pragma unroll
          for (int u = 0; u < TPW; ++u) {
            nxt[2 * u] = scr_at(qn, m0 + u)[0];
            nxt[2 * u + 1] = scr_at(qn, m0 + u)[32];
          }
        }
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          const int m = m0 + u;
          const double v[4] = {cur[2 * u].x, cur[2 * u].y, cur[2 * u + 1].x, cur[2 * u + 1].y};
          const int J0 = 16 * (kTilesPerStage * q + m) + gq, J1 = J0 + 8;
          double ra = 0.0, rb = 0.0;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (pb + 2 * t + c >= np) continue;
            if (J0 < I) ra += exp(v[c] - pm[c]) * prz[c];
            if (J1 < I) rb += exp(v[2 + c] - pm[c]) * prz[c];
          }
          ra += __shfl_xor_sync(0xffffffffu, ra, 1);
          ra += __shfl_xor_sync(0xffffffffu, ra, 2);
          rb += __shfl_xor_sync(0xffffffffu, rb, 1);
          rb += __shfl_xor_sync(0xffffffffu, rb, 2);
          // 0 + x is exact and x + y == y + x, so the order of the two
          // n-tiles' additions does not change the sum
          if (t == 0 && J0 < I) atomicAdd(&score[hl * a.T + J0], ra);
          if (t == 0 && J1 < I) atomicAdd(&score[hl * a.T + J1], rb);
        }
#pragma unroll
        for (int j = 0; j < 2 * TPW; ++j) cur[j] = nxt[j];
      }
    }
    named_bar_sync(1, kCons);

    // Threshold and bitmask, head by head.
    for (int x = 0; x < a.HC; ++x) {
      const double* sc = score + x * a.T;
      double best = 0.0;
      for (int J = tid; J < I; J += kCons) best = fmax(best, sc[J] / (double)np);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) best = fmax(best, __shfl_xor_sync(0xffffffffu, best, o));
      if (lane == 0) red[warp] = best;
      named_bar_sync(1, kCons);
      best = red[0];
#pragma unroll
      for (int w = 1; w < kBsWarps; ++w) best = fmax(best, red[w]);
      const double thr = a.alpha * best;
      uint32_t* out = a.mask + ((int64_t)(h0 + x) * a.T + I) * a.W;
      for (int w = warp; w < a.W; w += kBsWarps) {
        const int J = 32 * w + lane;
        const bool keep = J == I || (J < I && sc[J] / (double)np >= thr);
        const uint32_t bits = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) out[w] = bits;
      }
      named_bar_sync(1, kCons);  // red[] and score[] are reused
    }
  }
  // copies still in flight (after an abort) land before the CTA exits
  if (warp == kBsWarps && lane == 0)
    for (int x = max(0, issued - kBsStages); x < issued; ++x)
      mbar_wait_drain(smem_u32(&full_bar[x % kBsStages]), (x / kBsStages) & 1, a.wait_limit_ns);
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

size_t block_select_ws_bytes(int N, int Hkv, int d) {
  const int T = (N + 127) / 128, Tp = pad_blocks(T), sms = num_sms();
  return kStatusBytes + align_up(sizeof(double) * (size_t)Hkv * Tp * d, 256) +
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
      base + kStatusBytes + align_up(sizeof(double) * (size_t)a.Hkv * Tp * a.d, 256));
  block_mean_kernel<<<dim3(Tp, a.Hkv), 128, 0, a.stream>>>(a.K, a.dtype, a.N, T, a.d, a.kv_stride,
                                                           kbar);
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
  s.n_items = T * s.n_chunks;
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
  // more than half of an SM's shared memory: one CTA per SM, so a CTA's
  // scratch slot (its block index) is never shared
  const size_t need =
      sizeof(double) * ((size_t)kBsStages * kTilesPerStage * 16 * a.d + (size_t)HC * T);
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

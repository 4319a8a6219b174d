// Per-head vertical / slash budget selection (top-k or cumulative mass) on
// sm_100a.
//
// The rule is the VSPrefill pages' budget step ("VSPrefill ..." Technical
// Summary, section 2, Adaptive Inference Pipeline, Dynamic Budgeting: a
// cumulative threshold over the predicted scores decides how many indices to
// keep; the German page's Inferenz-Pipeline phrases it as the number of top-k
// indices needed to keep a given mass).  FlashPrefill's summary page
// (section 1) notes that sorting and cumulative sums are what make such
// selection expensive on GPUs; this kernel therefore never sorts:
//
//   * One thread-block cluster per head (8 CTAs, 16 when there are few
//     heads); each CTA keeps its slice of the scores as order-preserving
//     32-bit keys in shared memory.
//   * Most-significant-digit radix searches (4 passes of 8 bits) find the
//     exact boundary keys.  Per pass every CTA builds 256-bucket histograms
//     (counts, and for the threshold rule fp64 softmax mass); the cluster
//     merges them through distributed shared memory, and every CTA takes the
//     same decision from the same merged data.
//   * The threshold rule keeps k = min(k_threshold, cap) entries, so its mass
//     matters only when the top-cap entries already reach tau * Z.  The kernel
//     takes Z in one pass (fixed-order fp64 sum), runs the count search for
//     the cap, packs the keys at or above the cap's boundary key in index
//     order into a short list (when it fits) and sums the top-cap entries'
//     mass from it; only when that reaches tau * Z does the mass search run,
//     over the same list: every key of the threshold's prefix is in it.  A
//     key's mass is exp(s - s_max) in fp64 (Tang's table-driven method,
//     exp64.cuh).
//   * Each pass's decision is taken by one warp: lane l holds eight buckets
//     of the merged histogram, a shuffle scan of the lanes' sums (counts, or
//     fp64 masses) finds the lane where the target is reached, and that lane
//     walks its eight buckets.
//   * The mass histogram takes no fp64 atomics (shared-memory fp64 atomic
//     adds cost more than half of this kernel's time when they were used,
//     by measurement): each warp owns a private copy; lanes holding
//     the same digit are grouped with a match instruction and summed in a
//     tree over their ranks, and each group's lowest lane adds the sum with
//     a plain read-modify-write (distinct groups touch distinct buckets).
//     The CTA's histogram is the warps' copies added in warp order, so the
//     whole sum is in a fixed order and the selection is deterministic.
//   * FlashPrefill's max-based rule (summary page, section 2B: keep what
//     scores at least alpha times the maximum, no sort and no cumulative sum)
//     is one counting pass after the maximum; the kept entries are all keys
//     at or above a boundary, so unless the cap binds no search runs at all.
//   * A last pass writes the kept indices in ascending order: each warp takes
//     a contiguous range, 32 consecutive keys per step (conflict-free
//     shared-memory reads), and ballots place the kept ones; then -1 pads.
#include <cooperative_groups.h>

#include "exp64.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace vs {

constexpr int kSelThreads = 1024;
constexpr int kSelMaxCluster = 8;
constexpr int kSelCacheKeys = 32768;  // 128 KB of keys per CTA
// dynamic shared memory per CTA (the static part, ~13 KB, stays under the 227 KB limit)
constexpr size_t kSelMaxDynSmem = 208 * 1024;

// Order-preserving key: larger key = earlier in (score desc); NaN -> 0
// (after everything, including -inf); -0.0 is folded onto +0.0.
__device__ __forceinline__ uint32_t fkey(float f) {
  if (f != f) return 0u;
  if (f == 0.f) f = 0.f;
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float fkey_inv(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct SelArgs {
  const float* scores;
  int N;
  int64_t ld;
  int mode;
  int k_or_cap;
  double tau;
  double ln_alpha;  // max-based rule: log(alpha), computed once on the host
  int32_t* idx;
  int64_t ld_idx;
  int32_t* count;
  int* status;
  int chunk;
  int list_cap;  // threshold rule: room for the mass search's candidate keys (after wmass)
  // Batch of sequences (null cu: one score row per head).  Row b * H + h of
  // the grid is sequence b of head h: scores at h * total + cu[b], its cap
  // caps[b] (N: the longest sequence; k_or_cap: the bound on the caps).
  const int32_t* cu;
  int64_t total;
  const int32_t* caps;
  int H;
};

struct SelShared {
  uint32_t cnt_c[2][256];   // count histogram of the top-k (cap) search
  uint32_t cnt_t[2][256];   // count histogram of the threshold search
  double mass_t[2][256];    // mass histogram of the threshold search
  uint32_t tot_cc[256], tot_ct[256];
  double tot_mt[256];
  uint32_t kmax;
  uint32_t npos;
  uint32_t kmin_kept;
  uint32_t gt, eq;
  int bstar_c, bstar_t;
  uint32_t cabove_c, cabove_t, eqcnt_t;
  double mabove_t, target;
  double zpart, mpart;      // this CTA's share of Z, of the top-cap mass
  double exp_tab[32];       // 2^(j/32) for exp_nonpos
  int wred_i[32];
  double wred_d[32];
  uint32_t wg[32], we[32];  // per-warp counts of the compaction
};

// Softmax mass of a key relative to the maximum: 1 for the maximum, 0 for
// NaN.  The mass sums use exp_nonpos (relative error <= 1e-14, masses below
// e^-700 dropped: negligible against sums of at least 1); the "p > 0" test
// of tau = 1 uses the library exp, whose results reach down to the fp64
// subnormals.
__device__ __forceinline__ double pmass(uint32_t key, uint32_t kmax, double smax, const double* tab) {
  if (key == kmax) return 1.0;
  if (key == 0u) return 0.0;
  return exp_nonpos(static_cast<double>(fkey_inv(key)) - smax, tab);
}
__device__ __forceinline__ bool pmass_positive(uint32_t key, uint32_t kmax, double smax) {
  if (key == kmax) return true;
  if (key == 0u) return false;
  return exp(static_cast<double>(fkey_inv(key)) - smax) > 0.0;
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, T* wred, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) wred[warp] = v;
  __syncthreads();
  T r = wred[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = op(r, wred[w]);
  __syncthreads();
  return r;
}

// Sum of v over the lanes in `peers` (this lane's group, from
// __match_any_sync; every lane of the warp calls this).  A binary tree over
// the group's ranks: at step s the lane of rank r (r a multiple of 2s) adds
// the partial sum of rank r + s.  The group's total ends in its lowest lane
// (rank 0).  `steps` = ceil(log2(largest group in the warp)), warp-uniform.
__device__ __forceinline__ double group_sum(unsigned peers, double v, int steps) {
  const int lane = threadIdx.x & 31;
  const int rank = __popc(peers & ((1u << lane) - 1u));
  const unsigned above = lane == 31 ? 0u : peers & ~((2u << lane) - 1u);  // peers after me
  for (int i = 0, st = 1; i < steps; ++i, st <<= 1) {
    unsigned r = above;  // the peer of rank rank + st: the st-th set bit of `above`
    for (int j = 1; j < st && r; ++j) r &= r - 1u;
    const unsigned src = r ? (unsigned)(__ffs(r) - 1) : 32u;
    const double t = __shfl_sync(0xffffffffu, v, src < 32u ? src : (unsigned)lane);
    if ((rank & (2 * st - 1)) == 0 && src < 32u) v += t;
  }
  return v;
}

template <bool CACHE>
__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(SelArgs a) {
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const int C = static_cast<int>(cl.num_blocks());
  const int row_id = blockIdx.y;
  const int tid = threadIdx.x, nt = blockDim.x;
  extern __shared__ uint32_t skeys[];
  __shared__ SelShared sh;
  // per-warp mass histograms [warp][256], after the key cache (threshold rule
  // only), then the candidate keys of the mass search
  double* wmass = reinterpret_cast<double*>(skeys + (CACHE ? (a.chunk + 1) / 2 * 2 : 0));
  uint32_t* clist = reinterpret_cast<uint32_t*>(wmass + (kSelThreads / 32) * 256);
  int ncand = 0;          // candidate keys of this CTA
  bool use_list = false;  // the mass search reads clist (else every key, filtered)

  const float* row = a.scores + (int64_t)row_id * a.ld;
  int N = a.N, chunk = a.chunk, kcap = a.k_or_cap;
  if (a.cu) {
    // One row of a batch; every CTA of the cluster reads the same row, so
    // they all leave here together when it keeps nothing.
    const int b = row_id / a.H, hh = row_id - b * a.H;
    int64_t t0;
    int nb;
    const bool ok_seq = seq_range(a.cu, a.total, a.N, b, t0, nb);
    const int cap = ok_seq && nb > 0 ? __ldg(a.caps + b) : 0;
    const bool ok_cap = nb == 0 || (cap >= 1 && cap <= nb && cap <= a.k_or_cap);
    if ((!ok_seq || !ok_cap) && rank == 0 && tid == 0 && hh == 0)
      atomicOr(a.status, VS_DEVFLAG_BOUNDS);
    if (!ok_seq || !ok_cap || nb == 0) {  // an empty or malformed sequence keeps nothing
      if (rank == 0 && tid == 0) a.count[row_id] = 0;
      return;
    }
    N = nb;
    chunk = (nb + C - 1) / C;
    kcap = cap;
    row = a.scores + (int64_t)hh * a.total + t0;
  }
  const int lo = rank * chunk;
  const int n = max(0, min(N, lo + chunk) - lo);
  auto key_at = [&](int e) -> uint32_t { return CACHE ? skeys[e] : fkey(__ldg(row + lo + e)); };

  if (tid < 32) sh.exp_tab[tid] = exp2((double)tid / 32.0);  // read after the cluster barrier below
  // ---- keys and the cluster-wide maximum key
  uint32_t lmax = 0;
  for (int e = tid; e < n; e += nt) {
    const uint32_t k = fkey(__ldg(row + lo + e));
    if (CACHE) skeys[e] = k;
    lmax = max(lmax, k);
  }
  lmax = block_reduce<int>(static_cast<int>(lmax ^ 0x80000000u), sh.wred_i,
                           [](int x, int y) { return x > y ? x : y; }) ^ 0x80000000u;
  if (tid == 0) sh.kmax = lmax;
  cl.sync();
  uint32_t kmax = 0;
  for (int r = 0; r < C; ++r) kmax = max(kmax, *cl.map_shared_rank(&sh.kmax, r));
  const double smax = static_cast<double>(fkey_inv(kmax));

  // Selection rules:
  //   top-k: the count search for k;
  //   max-based: one counting pass, the count search only if the cap binds;
  //   threshold (tau < 1): k = min(k_threshold, cap), and the mass decides
  //     only when it keeps at most `cap` entries.  So Z comes first (one pass,
  //     a fixed-order sum), then the count search for the cap, then the mass
  //     of the top-cap entries; only when that reaches tau * Z does the mass
  //     search run, and only over the keys at or above the cap's boundary key
  //     (every key of the threshold's prefix is among them).
  int k_count = kcap;
  bool thr = false;              // threshold rule with tau < 1 and a non-NaN maximum
  bool search = true;            // false: the kept set is every key >= kmin_kept
  uint32_t kmin_kept = 0xFFFFFFFFu;
  const double* tab = sh.exp_tab;
  if (a.mode == VS_SELECT_MAXFRAC) {
    // keep r iff key_r == kmax or (double)s_r - s_max >= log(alpha); NaN
    // (key 0) never.  The test is monotone in the key, so the kept entries
    // are the keys >= the smallest kept key.
    uint32_t c = 0, kmin = 0xFFFFFFFFu;
    if (kmax != 0u) {
      for (int e = tid; e < n; e += nt) {
        const uint32_t k = key_at(e);
        if (k != 0u && (k == kmax || static_cast<double>(fkey_inv(k)) - smax >= a.ln_alpha)) {
          ++c;
          kmin = min(kmin, k);
        }
      }
    }
    c = static_cast<uint32_t>(block_reduce<int>(static_cast<int>(c), sh.wred_i,
                                                [](int x, int y) { return x + y; }));
    kmin = block_reduce<int>(static_cast<int>(kmin ^ 0x80000000u), sh.wred_i,
                             [](int x, int y) { return x < y ? x : y; }) ^ 0x80000000u;
    if (tid == 0) {
      sh.npos = c;
      sh.kmin_kept = kmin;
    }
    cl.sync();
    int tot = 0;
    for (int r = 0; r < C; ++r) {
      tot += static_cast<int>(*cl.map_shared_rank(&sh.npos, r));
      kmin_kept = min(kmin_kept, *cl.map_shared_rank(&sh.kmin_kept, r));
    }
    if (kmax == 0u) {  // every score is NaN: keep one entry
      k_count = 1;
    } else if (tot <= kcap) {
      k_count = tot;
      search = false;
    }
  } else if (a.mode == VS_SELECT_THRESHOLD) {
    if (kmax == 0u) {  // every score is NaN: keep one entry
      k_count = 1;
    } else if (a.tau >= 1.0) {  // keep every entry with p > 0
      uint32_t c = 0;
      for (int e = tid; e < n; e += nt) c += pmass_positive(key_at(e), kmax, smax) ? 1u : 0u;
      c = static_cast<uint32_t>(block_reduce<int>(static_cast<int>(c), sh.wred_i,
                                                  [](int x, int y) { return x + y; }));
      if (tid == 0) sh.npos = c;
      cl.sync();
      int tot = 0;
      for (int r = 0; r < C; ++r) tot += static_cast<int>(*cl.map_shared_rank(&sh.npos, r));
      k_count = min(max(tot, 1), kcap);
    } else {
      thr = true;
    }
  }
  double target = 0.0;  // tau * Z
  if (thr) {
    // Z: per-thread partial sums over a fixed stride, a fixed tree over the
    // block, the CTAs' shares added in rank order
    double zp = 0.0;
    for (int e = tid; e < n; e += nt) zp += pmass(key_at(e), kmax, smax, tab);
    zp = block_reduce<double>(zp, sh.wred_d, [](double x, double y) { return x + y; });
    if (tid == 0) sh.zpart = zp;
    cl.sync();
    double z = 0.0;
    for (int r = 0; r < C; ++r) z += *cl.map_shared_rank(&sh.zpart, r);
    target = a.tau * z;
  }

  // Most-significant-digit radix search (4 passes of 8 bits).  Count path:
  // the key of the k_count-th entry.  Mass path: the key where the running
  // mass, in descending key order over the keys >= floor_key, reaches
  // `target`.  Per pass every CTA builds 256-bucket histograms, the cluster
  // merges them through DSMEM and every CTA takes the same decision.
  uint32_t pf_c = 0, pm_c = 0, cab_c = 0;            // count path
  uint32_t pf_t = 0, pm_t = 0, cab_t = 0, eq_t = 0;  // mass path
  double mab_t = 0.0;
  int buf = 0;
  auto radix = [&](bool do_count, bool do_mass, uint32_t floor_key) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      if (tid < 256) {
        sh.cnt_c[buf][tid] = 0;
        sh.cnt_t[buf][tid] = 0;
      }
      if (do_mass)
        for (int i = tid; i < (kSelThreads / 32) * 256; i += nt) wmass[i] = 0.0;
      __syncthreads();
      if (do_count) {
        // run-length aggregation (keys of a pass often fall in one bucket, so
        // a thread accumulates while its bucket repeats and flushes on
        // change; the final flush is reduced across the warp when all lanes
        // agree)
        int cur_c = -1;
        uint32_t rc_c = 0;
        for (int e = tid; e < n; e += nt) {
          const uint32_t k = key_at(e);
          if ((k & pm_c) == pf_c) {
            const int dg = (k >> shift) & 255;
            if (dg != cur_c) {
              if (cur_c >= 0) atomicAdd(&sh.cnt_c[buf][cur_c], rc_c);
              cur_c = dg;
              rc_c = 0;
            }
            ++rc_c;
          }
        }
        __syncwarp();
        const int c0 = __shfl_sync(0xffffffffu, cur_c, 0);
        if (__all_sync(0xffffffffu, cur_c == c0) && c0 >= 0) {
          const uint32_t r = __reduce_add_sync(0xffffffffu, rc_c);
          if ((tid & 31) == 0) atomicAdd(&sh.cnt_c[buf][c0], r);
        } else if (cur_c >= 0) {
          atomicAdd(&sh.cnt_c[buf][cur_c], rc_c);
        }
      }
      // Mass path: a warp takes 32 consecutive keys per step (warp-uniform
      // trip count); lanes with equal digits form a group, whose lowest lane
      // adds the group's count (shared atomic, integer) and mass (the warp's
      // own histogram, plain add: the groups' digits differ).
      if (do_mass) {
        const int lane = tid & 31;
        double* wm = wmass + (tid >> 5) * 256;
        const int mn = use_list ? ncand : n;
        for (int base = tid - lane; base < mn; base += nt) {
          const int e = base + lane;
          int dg = 256;  // 256: not in the searched prefix (or past the end)
          double m = 0.0;
          if (e < mn) {
            const uint32_t k = use_list ? clist[e] : key_at(e);
            if (k >= floor_key && (k & pm_t) == pf_t) {
              dg = (k >> shift) & 255;
              m = pmass(k, kmax, smax, tab);
            }
          }
          if (__all_sync(0xffffffffu, dg == __shfl_sync(0xffffffffu, dg, 0))) {
            if (dg < 256) {  // one digit across the warp
              for (int o = 16; o > 0; o >>= 1) m += __shfl_xor_sync(0xffffffffu, m, o);
              if (lane == 0) {
                atomicAdd(&sh.cnt_t[buf][dg], 32u);
                wm[dg] += m;
              }
            }
            continue;
          }
          const unsigned peers = __match_any_sync(0xffffffffu, dg);
          const int gsize = __popc(peers);
          const int gmax = __reduce_max_sync(0xffffffffu, (unsigned)gsize);
          const int steps = 32 - __clz(gmax - 1);  // ceil(log2(gmax)); 0 for gmax = 1
          m = group_sum(peers, m, steps);
          if (dg < 256 && (peers & ((1u << lane) - 1u)) == 0) {
            atomicAdd(&sh.cnt_t[buf][dg], (uint32_t)gsize);
            wm[dg] += m;
          }
        }
        __syncthreads();
        if (tid < 256) {  // the CTA's histogram: the warps' copies in warp order
          double t = 0.0;
          for (int w = 0; w < kSelThreads / 32; ++w) t += wmass[w * 256 + tid];
          sh.mass_t[buf][tid] = t;
        }
      }
      cl.sync();
      if (tid < 256) {  // merge the cluster's histograms (same order in every CTA)
        uint32_t cc = 0, ct = 0;
        double mt = 0.0;
        for (int r = 0; r < C; ++r) {
          if (do_count) cc += cl.map_shared_rank(&sh.cnt_c[buf][0], r)[tid];
          if (do_mass) {
            ct += cl.map_shared_rank(&sh.cnt_t[buf][0], r)[tid];
            mt += cl.map_shared_rank(&sh.mass_t[buf][0], r)[tid];
          }
        }
        sh.tot_cc[tid] = cc;
        sh.tot_ct[tid] = ct;
        sh.tot_mt[tid] = mt;
      }
      __syncthreads();
      if (do_count && tid < 32) {
        // count path: the first bucket from the top at which the running
        // count reaches k_count.  Lane l holds buckets 255 - 8 l .. 248 - 8 l.
        const int lane = tid;
        uint32_t c[8], tsum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[j] = sh.tot_cc[255 - 8 * lane - j];
          tsum += c[j];
        }
        uint32_t incl = tsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, cab_c + incl >= (uint32_t)k_count);
        if (hit && lane == __ffs(hit) - 1) {
          uint32_t ca = cab_c + incl - tsum;
          int bs = -1;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (bs < 0 && c[j] != 0) {
              if (ca + c[j] >= (uint32_t)k_count) bs = 255 - 8 * lane - j;
              else ca += c[j];
            }
          }
          sh.bstar_c = bs;
          sh.cabove_c = ca;
        }
      }
      if (do_mass && tid >= 32 && tid < 64) {
        // mass path: the first bucket from the top at which the running mass
        // reaches the target.  Lane l holds buckets 255 - 8 l .. 248 - 8 l;
        // an inclusive scan of the lanes' sums finds the lane, which walks its
        // eight buckets.  (Fixed order, the same in every CTA of the cluster.)
        const int lane = tid - 32;
        uint32_t c[8], csum = 0;
        double m[8], msum = 0.0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[j] = sh.tot_ct[255 - 8 * lane - j];
          m[j] = sh.tot_mt[255 - 8 * lane - j];
          csum += c[j];
          msum += m[j];
        }
        uint32_t cincl = csum;
        double mincl = msum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t yc = __shfl_up_sync(0xffffffffu, cincl, o);
          const double ym = __shfl_up_sync(0xffffffffu, mincl, o);
          if (lane >= o) {
            cincl += yc;
            mincl += ym;
          }
        }
        uint32_t cex = __shfl_up_sync(0xffffffffu, cincl, 1);
        double mex = __shfl_up_sync(0xffffffffu, mincl, 1);
        if (lane == 0) {
          cex = 0;
          mex = 0.0;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, mab_t + mincl >= target);
        // no lane reaches it (rounding left the total just short): the last
        // non-empty bucket is the group, with every other bucket above it
        const unsigned nonempty = __ballot_sync(0xffffffffu, csum != 0);
        const int wl = hit ? __ffs(hit) - 1 : (nonempty ? 31 - __clz(nonempty) : 0);
        if (lane == wl) {
          int bs = -1, last_j = -1;
          uint32_t ca = cab_t + cex;
          double ma = mab_t + mex;
          uint32_t ca_last = ca;
          double ma_last = ma;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (bs >= 0 || c[j] == 0) continue;
            if (hit && ma + m[j] >= target) {
              bs = 255 - 8 * lane - j;
            } else {
              last_j = j;
              ca_last = ca;
              ma_last = ma;
              ca += c[j];
              ma += m[j];
            }
          }
          if (bs < 0) {  // the lane's last non-empty bucket
            bs = last_j >= 0 ? 255 - 8 * lane - last_j : 0;
            ca = ca_last;
            ma = ma_last;
          }
          sh.bstar_t = bs;
          sh.cabove_t = ca;
          sh.mabove_t = ma;
          sh.eqcnt_t = sh.tot_ct[bs];
        }
      }
      __syncthreads();
      if (do_count) {
        pf_c |= static_cast<uint32_t>(sh.bstar_c) << shift;
        pm_c |= 255u << shift;
        cab_c = sh.cabove_c;
      }
      if (do_mass) {
        pf_t |= static_cast<uint32_t>(sh.bstar_t) << shift;
        pm_t |= 255u << shift;
        cab_t = sh.cabove_t;
        mab_t = sh.mabove_t;
        eq_t = sh.eqcnt_t;
      }
      buf ^= 1;
    }
  };
  if (search) radix(true, false, 0u);
  uint32_t T = pf_c;
  uint32_t cabove = cab_c;
  int k_target = k_count;
  if (!search) {  // every key > kmin_kept - 1 is kept; no equal-key group to trim
    T = kmin_kept - 1u;
    cabove = static_cast<uint32_t>(k_count);
  }
  if (thr) {
    // The keys at or above the cap's boundary key (scattered over the row)
    // are packed in index order into a short list when it fits: the top-cap
    // mass and, when it reaches tau * Z, the mass search read only them.
    {
      const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
      const int wper = ((n + nw - 1) / nw + 31) / 32 * 32;
      const int wb = min(n, warp * wper), wend = min(n, wb + wper);
      uint32_t c = 0;
      for (int base = wb; base < wend; base += 32) {
        const int e = base + lane;
        c += __popc(__ballot_sync(0xffffffffu, e < wend && key_at(e) >= pf_c));
      }
      if (lane == 0) sh.wg[warp] = c;
      __syncthreads();
      int off = 0;
      for (int w = 0; w < nw; ++w) {
        if (w < warp) off += static_cast<int>(sh.wg[w]);
        ncand += static_cast<int>(sh.wg[w]);
      }
      use_list = ncand <= a.list_cap;
      if (use_list) {
        const unsigned lt = (1u << lane) - 1u;
        for (int base = wb; base < wend; base += 32) {
          const int e = base + lane;
          const uint32_t k = e < wend ? key_at(e) : 0u;
          const bool in = e < wend && k >= pf_c;
          const unsigned m = __ballot_sync(0xffffffffu, in);
          if (in) clist[off + __popc(m & lt)] = k;
          off += __popc(m);
        }
      }
      __syncthreads();
    }
    // mass of the top-cap entries: the keys above the cap's boundary key,
    // and as many copies of that key's mass as the cap keeps
    double mp = 0.0;
    if (use_list) {
      for (int e = tid; e < ncand; e += nt) {
        const uint32_t k = clist[e];
        if (k > pf_c) mp += pmass(k, kmax, smax, tab);
      }
    } else {
      for (int e = tid; e < n; e += nt) {
        const uint32_t k = key_at(e);
        if (k > pf_c) mp += pmass(k, kmax, smax, tab);
      }
    }
    mp = block_reduce<double>(mp, sh.wred_d, [](double x, double y) { return x + y; });
    if (tid == 0) sh.mpart = mp;
    cl.sync();
    double mcap = 0.0;
    for (int r = 0; r < C; ++r) mcap += *cl.map_shared_rank(&sh.mpart, r);
    mcap += static_cast<double>(k_count - static_cast<int>(cab_c)) * pmass(pf_c, kmax, smax, tab);
    if (mcap >= target) {
      // the threshold's prefix ends within the top-cap entries
      radix(false, true, pf_c);
      // within the final group of equal keys every entry has the same mass
      const double pstar = pmass(pf_t, kmax, smax, tab);
      double mm = pstar > 0.0 ? ceil((target - mab_t) / pstar) : static_cast<double>(eq_t);
      mm = fmin(fmax(mm, 1.0), static_cast<double>(eq_t));
      const int k_thr = static_cast<int>(cab_t) + static_cast<int>(mm);
      if (k_thr <= kcap) {
        T = pf_t;
        cabove = cab_t;
        k_target = k_thr;
      }
    }
  }
  const int m_eq = k_target - static_cast<int>(cabove);  // equal keys to keep (smallest indices)

  // ---- ascending compaction across the cluster.  Warp w takes a contiguous
  // range of keys, 32 consecutive keys per step (one per lane: conflict-free
  // shared-memory reads); ballots give each kept key its place.
  const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
  const int wper = ((n + nw - 1) / nw + 31) / 32 * 32;
  const int wb = min(n, warp * wper), wend = min(n, wb + wper);
  const unsigned lt = (1u << lane) - 1u;
  {
    uint32_t g = 0, q = 0;
    for (int base = wb; base < wend; base += 32) {
      const int e = base + lane;
      const uint32_t k = e < wend ? key_at(e) : 0u;
      g += __popc(__ballot_sync(0xffffffffu, e < wend && k > T));
      q += __popc(__ballot_sync(0xffffffffu, e < wend && k == T));
    }
    if (lane == 0) {
      sh.wg[warp] = g;
      sh.we[warp] = q;
    }
  }
  __syncthreads();
  int G = 0, E = 0, Gt = 0, Et = 0;  // this warp's offsets; the CTA's totals
  for (int w = 0; w < nw; ++w) {
    if (w < warp) {
      G += static_cast<int>(sh.wg[w]);
      E += static_cast<int>(sh.we[w]);
    }
    Gt += static_cast<int>(sh.wg[w]);
    Et += static_cast<int>(sh.we[w]);
  }
  if (tid == 0) {
    sh.gt = static_cast<uint32_t>(Gt);
    sh.eq = static_cast<uint32_t>(Et);
  }
  cl.sync();
  int eq_before = 0, sel_before = 0;
  for (int r = 0; r < rank; ++r) {
    const int gr = static_cast<int>(*cl.map_shared_rank(&sh.gt, r));
    const int er = static_cast<int>(*cl.map_shared_rank(&sh.eq, r));
    sel_before += gr + min(er, max(0, m_eq - eq_before));
    eq_before += er;
  }
  int32_t* out = a.idx + (int64_t)row_id * a.ld_idx;
  int pos = sel_before + G + min(E, max(0, m_eq - eq_before));
  int eq_seen = eq_before + E;
  for (int base = wb; base < wend; base += 32) {
    const int e = base + lane;
    const bool in = e < wend;
    const uint32_t k = in ? key_at(e) : 0u;
    const bool isg = in && k > T, ise = in && k == T;
    const unsigned me = __ballot_sync(0xffffffffu, ise);
    const bool keep = isg || (ise && eq_seen + __popc(me & lt) < m_eq);
    const unsigned mk = __ballot_sync(0xffffffffu, keep);
    if (keep) out[pos + __popc(mk & lt)] = lo + e;
    pos += __popc(mk);
    eq_seen += __popc(me);
  }
  // pad [k, k_or_cap) with -1, split over the cluster
  for (int64_t t = (int64_t)k_target + rank * nt + tid; t < kcap; t += (int64_t)C * nt) out[t] = -1;
  if (rank == 0 && tid == 0) a.count[row_id] = k_target;
  cl.sync();  // keep shared memory alive until every remote read is done
}

cudaError_t launch_select(const float* scores, int H, int N, int64_t ld, int mode, int k_or_cap,
                          double tau, double ln_alpha, int32_t* idx, int64_t ld_idx, int32_t* count, int* status,
                          cudaStream_t stream, const int32_t* cu, int64_t total, const int32_t* caps,
                          int B) {
  const int H_seq = H;  // heads of one sequence
  H *= B;               // score rows of the launch
  int C = (N + 4095) / 4096;
  C = C < 1 ? 1 : (C > kSelMaxCluster ? kSelMaxCluster : C);
  {
    // Many rows: a cluster per row at this size needs more than one wave of
    // SMs (one CTA per SM).  Then take the smallest cluster whose CTAs still
    // cache their slice of the keys: it may fit all rows in one wave, and
    // where it does not (a batch of many sequences), fewer CTAs per row spend
    // less on the per-pass cluster barriers.
    int cmin = (N + kSelCacheKeys - 1) / kSelCacheKeys;
    cmin = cmin < 1 ? 1 : cmin;
    const int sms = device_sm_count();
    if (cmin < C && H * C > sms) C = cmin;
  }
  const size_t mass_bytes = mode == VS_SELECT_THRESHOLD ? sizeof(double) * (kSelThreads / 32) * 256 : 0;
  // Room for the threshold rule's candidate list: what is left of the
  // dynamic shared memory, at most one entry per key of the CTA.
  auto list_entries = [&](int chunk_, bool cache_) -> int {
    if (mode != VS_SELECT_THRESHOLD) return 0;
    const size_t used = (cache_ ? sizeof(uint32_t) * ((chunk_ + 1) / 2 * 2) : 0) + mass_bytes;
    const size_t room = used < kSelMaxDynSmem ? (kSelMaxDynSmem - used) / sizeof(uint32_t) : 0;
    return static_cast<int>(room < (size_t)chunk_ ? room : (size_t)chunk_);
  };
  // Few heads leave most SMs idle: split long rows over 16-CTA clusters (a
  // non-portable size: used only when the device can place such a cluster).
  bool wide = C == kSelMaxCluster && H * kSelMaxCluster * 2 <= device_sm_count() &&
              N >= 16 * 4096;
  if (wide) {
    const int chunk16 = (N + 15) / 16;
    const bool cache16 = chunk16 <= kSelCacheKeys;
    auto kern16 = cache16 ? select_kernel<true> : select_kernel<false>;
    cudaLaunchConfig_t probe = {};
    probe.gridDim = dim3(16, H, 1);
    probe.blockDim = dim3(kSelThreads, 1, 1);
    probe.dynamicSmemBytes = (cache16 ? sizeof(uint32_t) * ((chunk16 + 1) / 2 * 2) : 0) + mass_bytes +
                             sizeof(uint32_t) * list_entries(chunk16, cache16);
    cudaLaunchAttribute pa[1];
    pa[0].id = cudaLaunchAttributeClusterDimension;
    pa[0].val.clusterDim.x = 16;
    pa[0].val.clusterDim.y = 1;
    pa[0].val.clusterDim.z = 1;
    probe.attrs = pa;
    probe.numAttrs = 1;
    int nclusters = 0;
    if (cudaFuncSetAttribute(kern16, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)probe.dynamicSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&nclusters, kern16, &probe) != cudaSuccess ||
        nclusters < 1) {
      cudaGetLastError();  // clear a refusal; fall back to the portable size
      wide = false;
    }
  }
  if (wide) C = 16;
  const int chunk = (N + C - 1) / C;
  const bool cache = chunk <= kSelCacheKeys;
  const int list_cap = list_entries(chunk, cache);
  SelArgs a{scores, N,     ld,       mode, k_or_cap, tau,   ln_alpha, idx,
            ld_idx, count, status, chunk, list_cap, cu,  total,    caps, H_seq};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, H, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = (cache ? sizeof(uint32_t) * ((chunk + 1) / 2 * 2) : 0) + mass_bytes +
                         sizeof(uint32_t) * list_cap;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (cache) {
    e = cudaFuncSetAttribute(select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)cfg.dynamicSmemBytes);
    if (e != cudaSuccess) return e;
    if (wide) {
      e = cudaFuncSetAttribute(select_kernel<true>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    e = cudaLaunchKernelEx(&cfg, select_kernel<true>, a);
  } else {
    e = cudaFuncSetAttribute(select_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)cfg.dynamicSmemBytes);
    if (e != cudaSuccess) return e;
    if (wide) {
      e = cudaFuncSetAttribute(select_kernel<false>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    e = cudaLaunchKernelEx(&cfg, select_kernel<false>, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace vs

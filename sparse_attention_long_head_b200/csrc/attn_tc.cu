// Vertical-slash sparse (and dense causal) attention forward on sm_100a.
//
// What is computed follows the VSPrefill summary pages, "VSPrefill ..."
// Technical Summary, section 2: each query attends to the union of the
// selected vertical key columns and the keys at the selected slash offsets
// behind it, inside one FlashAttention-style kernel with no precomputed mask.
// How it is computed is this library's own design for B200:
//
//   * A plan kernel turns the index lists into per-head bitmaps (columns,
//     offsets), an ascending column list, and the list of touched
//     block-diagonals.  No n x n structure is ever built.
//   * The attention kernel is persistent: one CTA per SM walks "units" of 256
//     query rows of one head (two 128-row sub-tiles A and B), KV head by KV
//     head (L2 reuse of K/V), heaviest first within a KV head.
//   * Per unit it streams "items": 128-key blocks loaded by TMA (tiled), or
//     128-column chunks of the vertical list -- as tiles of the packed copy a
//     pack kernel writes before the attention kernel, or, when the workspace
//     has no room for it, gathered row by row with TMA tile::gather4.  Each
//     item is applied to both sub-tiles.
//   * QK^T and PV run on tcgen05 (bf16 in, fp32 accumulate in TMEM); P is
//     written back into TMEM over S and consumed by the TS-form MMA.
//   * Four softmax warps per sub-tile own one row each; the element mask of a
//     key block is four 32-bit words per row read from the offset and column
//     bitmaps, so a key that is both a column and on a selected diagonal is
//     counted once.  Online softmax with lazy rescaling of O (only when the
//     running max grows by more than 2^8).
//   * Per unit the plan picks, in O(1), the cheaper of: every key block of
//     the causal triangle with mask (S or V) ("dense-vs"), or the gathered
//     vertical chunks plus only the key blocks on touched block-diagonals with
//     mask (S and not V) ("split").
//
// Warp roles (320 threads): warps 0-3 softmax/epilogue of sub-tile A, warps
// 4-7 of sub-tile B, warp 8 issues the MMAs (one thread) and owns TMEM,
// warp 9 issues the TMA loads.  Every wait is bounded (see WaitCtx).
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace vs {

// ------------------------------------------------------------------ plan

// Writes, in ascending order, the positions of the set bits of
// bits[0 .. nwords) (bit positions < limit) to out[]; returns the count.
// Whole block participates; `scan` is blockDim.x ints of shared memory.
__device__ int block_bits_to_list(const uint32_t* bits, int64_t nwords, int64_t limit,
                                  int32_t* out, int* scan) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int64_t per = (nwords + nt - 1) / nt;
  const int64_t w0 = tid * per, w1 = min(nwords, w0 + per);
  int c = 0;
  for (int64_t w = w0; w < w1; ++w) c += __popc(bits[w]);
  scan[tid] = c;
  __syncthreads();
  for (int off = 1; off < nt; off <<= 1) {
    int v = tid >= off ? scan[tid - off] : 0;
    __syncthreads();
    scan[tid] += v;
    __syncthreads();
  }
  int pos = scan[tid] - c;
  const int total = scan[nt - 1];
  for (int64_t w = w0; w < w1; ++w) {
    uint32_t x = bits[w];
    while (x) {
      int b = __ffs(x) - 1;
      x &= x - 1;
      int64_t v = w * 32 + b;
      if (v < limit) out[pos] = static_cast<int32_t>(v);
      ++pos;
    }
  }
  __syncthreads();
  return total;
}

struct PlanKernelArgs {
  int N, H_sel;  // N: the longest sequence; slots are b * H_sel + hs
  const int32_t* cu;
  int64_t total;
  const int32_t* v_idx;
  int64_t v_ld;
  const int32_t* v_cnt;
  const int32_t* s_idx;
  int64_t s_ld;
  const int32_t* s_cnt;
  void* ws;
  int* status;
  PlanLayout L;
};

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanKernelArgs a) {
  __shared__ int scan[kPlanThreads];
  __shared__ uint32_t dbits[1026];  // touched block-diagonals, T <= 32768
  __shared__ uint32_t d1bits[1026];
  __shared__ int bad;
  const int hs = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;  // hs: the plan slot
  const PlanLayout& L = a.L;
  PlanPtrs pp = plan_ptrs(L, a.ws);
  uint32_t* vb = pp.vbits + (int64_t)hs * L.vbits_words;
  uint32_t* sb = pp.sbits + (int64_t)hs * L.sbits_words;
  int64_t tok0;
  int N;
  const bool seq_ok = seq_range(a.cu, a.total, a.N, hs / a.H_sel, tok0, N);
  const int T = (N + 127) / 128;
  const int dwords = (T + 2 + 31) / 32;
  for (int64_t w = tid; w < L.vbits_words; w += nt) vb[w] = 0;
  for (int64_t w = tid; w < L.sbits_words; w += nt) sb[w] = 0;
  for (int w = tid; w < dwords; w += nt) dbits[w] = 0;
  if (tid == 0) bad = seq_ok ? 0 : 1;
  __syncthreads();

  int nv_in = a.v_cnt[hs], ns_in = a.s_cnt[hs];
  if (nv_in < 0 || nv_in > a.v_ld) {
    nv_in = nv_in < 0 ? 0 : (int)a.v_ld;
    bad = 1;
  }
  if (ns_in < 0 || ns_in > a.s_ld) {
    ns_in = ns_in < 0 ? 0 : (int)a.s_ld;
    bad = 1;
  }
  for (int t = tid; t < nv_in; t += nt) {
    int j = a.v_idx[(int64_t)hs * a.v_ld + t];
    if (j >= 0 && j < N) atomicOr(&vb[j >> 5], 1u << (j & 31));
    else bad = 1;
  }
  for (int t = tid; t < ns_in; t += nt) {
    int o = a.s_idx[(int64_t)hs * a.s_ld + t];
    if (o >= 0 && o < N) {
      int pos = N - o + 128;
      atomicOr(&sb[pos >> 5], 1u << (pos & 31));
      int dl = o >> 7;
      atomicOr(&dbits[dl >> 5], 1u << (dl & 31));
      if ((o & 127) && dl + 1 < T) atomicOr(&dbits[(dl + 1) >> 5], 1u << ((dl + 1) & 31));
    } else {
      bad = 1;
    }
  }
  __syncthreads();
  if (tid == 0 && bad) atomicOr(a.status, VS_DEVFLAG_BOUNDS);
  // d' in [0, T] is needed iff d' or d'-1 is touched.
  for (int w = tid; w < dwords; w += nt) {
    uint32_t cur = dbits[w], prev = w > 0 ? dbits[w - 1] : 0u;
    d1bits[w] = cur | (cur << 1) | (prev >> 31);
  }
  __syncthreads();
  int32_t* vlist = pp.vlist + (int64_t)hs * L.N;
  int32_t* slist = pp.slist + (int64_t)hs * L.N;
  int32_t* d1list = pp.d1list + (int64_t)hs * L.d1_len;
  int32_t* d1pref = pp.d1pref + (int64_t)hs * L.d1pref_len;
  int32_t* vpair = pp.vpair + (int64_t)hs * L.vpair_len;
  const int nv = block_bits_to_list(vb, (N + 31) / 32, N, vlist, scan);
  // offsets ascending = positions N - o + 128 descending: collect, then reverse.
  int ns = 0;
  {
    // positions live in [129, N + 128]; list them ascending into slist, then
    // map pos -> o = N + 128 - pos and reverse in place.
    ns = block_bits_to_list(sb, L.sbits_words, (int64_t)N + 129, slist, scan);
    for (int t = tid; t < ns / 2; t += nt) {
      int x = slist[t], y = slist[ns - 1 - t];
      slist[t] = N + 128 - y;
      slist[ns - 1 - t] = N + 128 - x;
    }
    if ((ns & 1) && tid == 0) slist[ns / 2] = N + 128 - slist[ns / 2];
    __syncthreads();
  }
  {
    const int nd1 = block_bits_to_list(d1bits, (T + 1 + 31) / 32, (int64_t)T + 1, d1list, scan);
    for (int x = tid; x < L.d1pref_len; x += nt) {
      int lo = 0, hi = nd1;  // lower_bound(d1list, x)
      while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (d1list[mid] < x) lo = mid + 1;
        else hi = mid;
      }
      d1pref[x] = lo;
    }
    for (int p = tid; p < L.P; p += nt) {
      int lim = min(256 * p + 255, N - 1);
      int lo = 0, hi = nv;  // upper_bound(vlist, lim)
      while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (vlist[mid] <= lim) lo = mid + 1;
        else hi = mid;
      }
      vpair[p] = lo;
    }
    if (tid == 0) {
      int32_t* m = pp.meta + 4 * hs;
      m[0] = nv;
      m[1] = ns;
      m[2] = nd1;
      m[3] = 0;
    }
  }
}

cudaError_t launch_plan(const AttnArgs& a, const PlanLayout& L) {
  if (L.T + 2 > 1026 * 32) return cudaErrorInvalidValue;
  PlanKernelArgs k{a.N,   a.H_sel, a.cu_seqlens, a.total, a.v_idx, a.v_ld, a.v_cnt,
                   a.s_idx, a.s_ld,  a.s_cnt,      a.ws,    a.status, L};
  plan_kernel<<<a.B * a.H_sel, kPlanThreads, 0, a.stream>>>(k);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ pack

// Copies each index set's selected K and V rows (ascending column order) into
// [H_sel][vrows][d] buffers, zero-filling the rest of the last 128-row chunk.
// One CTA per (128-row chunk, index set); chunks past the set's count exit.
template <int D>
__global__ void __launch_bounds__(256) pack_kernel(const __nv_bfloat16* K, const __nv_bfloat16* V,
                                                   int64_t kv_stride, int Hq, int Hkv, int H_sel,
                                                   int64_t vrows, PlanLayout L, PlanPtrs pp,
                                                   const int32_t* cu, int64_t total,
                                                   __nv_bfloat16* pk, __nv_bfloat16* pv) {
  const int hs = blockIdx.y, c = blockIdx.x;  // hs: the plan slot
  const int nv = pp.meta[4 * hs + 0];
  if (128 * c >= nv) return;
  int64_t tok0;
  int Nb;
  seq_range(cu, total, L.N, hs / H_sel, tok0, Nb);  // nv == 0 for a malformed entry
  const int g = ((hs % H_sel) * (Hq / H_sel)) / (Hq / Hkv);
  const int32_t* vl = pp.vlist + (int64_t)hs * L.N;
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int e = threadIdx.x; e < 128 * CH; e += blockDim.x) {
    const int r = e / CH, ch = e % CH;
    const int t = 128 * c + r;
    uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (t < nv) {
      const int64_t src = (tok0 + vl[t]) * kv_stride + (int64_t)g * D + ch * 8;
      kk = *reinterpret_cast<const uint4*>(K + src);
      vv = *reinterpret_cast<const uint4*>(V + src);
    }
    const int64_t dst = ((int64_t)hs * vrows + t) * D + ch * 8;
    *reinterpret_cast<uint4*>(pk + dst) = kk;
    *reinterpret_cast<uint4*>(pv + dst) = vv;
  }
}

cudaError_t launch_pack(const AttnArgs& a, const PlanLayout& L) {
  dim3 grid((unsigned)(a.pack_vrows / 128), (unsigned)(a.B * a.H_sel));
  const PlanPtrs pp = plan_ptrs(L, a.ws);
  auto* K = static_cast<const __nv_bfloat16*>(a.K);
  auto* V = static_cast<const __nv_bfloat16*>(a.V);
  auto* pk = static_cast<__nv_bfloat16*>(a.pack_k);
  auto* pv = static_cast<__nv_bfloat16*>(a.pack_v);
  if (a.d == 128)
    pack_kernel<128><<<grid, 256, 0, a.stream>>>(K, V, a.kv_stride, a.Hq, a.Hkv, a.H_sel,
                                                 a.pack_vrows, L, pp, a.cu_seqlens, a.total, pk, pv);
  else
    pack_kernel<64><<<grid, 256, 0, a.stream>>>(K, V, a.kv_stride, a.Hq, a.Hkv, a.H_sel,
                                                a.pack_vrows, L, pp, a.cu_seqlens, a.total, pk, pv);
  return cudaGetLastError();
}

// ------------------------------------------------------------ block plan

// For each (head h, pair p) of query blocks I = 2p, 2p + 1: the ascending
// union of the key blocks kept for either (J <= I each), with bit 30 / 31
// marking the blocks kept for the first / second, and bit 28 / 29 the last
// block kept for the first / second (the attention then knows when a
// sub-tile's accumulation is complete).  One warp per unit; the rows have at
// most 64 words (T <= 2048).
__global__ void __launch_bounds__(32) block_plan_kernel(const uint32_t* mask, int T, int P,
                                                        int32_t* bcnt, uint32_t* blist) {
  const int p = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  const int W = (T + 31) / 32;
  const int IA = 2 * p, IB = 2 * p + 1;
  const uint32_t* ra = mask + ((int64_t)h * T + IA) * W;
  const uint32_t* rb = IB < T ? mask + ((int64_t)h * T + IB) * W : nullptr;
  uint32_t* out = blist + (int64_t)h * P * (P + 1) + (int64_t)p * (p + 1);
  auto upto = [](int w, int last) -> uint32_t {  // bits of word w at positions <= last
    const int k = last - 32 * w;
    return k < 0 ? 0u : (k >= 31 ? 0xffffffffu : ((2u << k) - 1u));
  };
  int base = 0;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int w = w0 + lane;
    uint32_t a = 0u, b = 0u;
    if (w < W) {
      a = ra[w] & upto(w, IA);
      b = rb ? rb[w] & upto(w, min(IB, T - 1)) : 0u;
    }
    const uint32_t u = a | b;
    const int c = __popc(u);
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + incl - c;
    uint32_t x = u;
    while (x) {
      const int bit = __ffs(x) - 1;
      x &= x - 1;
      const uint32_t J = 32u * w + bit;
      out[pos++] = J | (((a >> bit) & 1u) << 30) | (((b >> bit) & 1u) << 31);
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
  if (lane < 2) {  // lane s marks the last entry kept for sub-tile s
    for (int k = base - 1; k >= 0; --k)
      if ((out[k] >> (30 + lane)) & 1u) {
        atomicOr(&out[k], 1u << (28 + lane));
        break;
      }
  }
  if (lane == 0) bcnt[(int64_t)h * P + p] = base;
}

// A batch of B sequences has mask rows and plan slots per (sequence, query
// head), b * Hq + h: the same kernel over B * Hq "heads".
cudaError_t launch_block_plan(const AttnArgs& a) {
  const BlockPlanLayout B = BlockPlanLayout::make(a.N, a.B * a.Hq);
  int32_t* bcnt = reinterpret_cast<int32_t*>(static_cast<char*>(a.ws) + B.off_cnt);
  uint32_t* blist = reinterpret_cast<uint32_t*>(static_cast<char*>(a.ws) + B.off_list);
  block_plan_kernel<<<dim3(B.P, a.B * a.Hq), 32, 0, a.stream>>>(a.block_mask, B.T, B.P, bcnt,
                                                                blist);
  return cudaGetLastError();
}

// ------------------------------------------------------------- attention

constexpr int kAttnThreads = 320;
constexpr int kWarpMMA = 8;
constexpr int kWarpLoad = 9;

enum : int { kModeDense = 0, kModeDenseVS = 1, kModeSplit = 2, kModeBlock = 3 };
// Kernel instantiations: dense causal, vertical-slash sparse, block sparse.
enum : int { kAttnDense = 0, kAttnVS = 1, kAttnBlock = 2 };
enum : int { kItemTile = 0, kItemVChunk = 1 };

template <int D>
struct Cfg {
  static constexpr int kTileBytes = 128 * D * 2;  // one 128-row K or V tile
  static constexpr int kStages = D == 128 ? 4 : 8;
  static constexpr int kQBytes = kTileBytes;
  static constexpr int kData = 2 * kQBytes + kStages * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmem = kData + kBarBytes + 1024;  // + alignment slack
};

struct AttnParams {
  int N, Hq, Hkv, H_sel, T, P, G;  // N, T, P: of the longest sequence
  int num_units;                   // B * Hq * P
  const int32_t* cu;               // sequence offsets (device) or null
  int B;                           // sequences
  int64_t total;                   // token rows of Q, K, V, O
  int64_t q_stride;
  float scale_log2;  // softmax scale * log2(e)
  __nv_bfloat16* O;
  float* lse;
  int* status;
  uint64_t wait_limit_ns;
  PlanLayout L;
  PlanPtrs pp;
  int64_t pack_vrows;  // 0: gather vertical rows; else packed tiles (tmKg/tmVg map them)
  // block sparse: per (head, pair) the count and, at h P (P + 1) + p (p + 1),
  // the ascending kept key blocks of both query blocks (bit 30: kept for the
  // first, bit 31: for the second)
  const int32_t* bcnt;
  const uint32_t* blist;
};

struct UnitInfo {
  int h, hs, g, p, n, mode, nvc, nv, d1start;  // hs: the plan slot b * H_sel + index set
  int b;                                        // the unit's sequence
  int Nb;                                       // its tokens
};

// First token row of the unit's sequence (re-read where needed rather than
// kept live through the tile loop).
__device__ __forceinline__ int64_t unit_tok0(const AttnParams& P, const UnitInfo& ui) {
  return P.cu ? (int64_t)__ldg(P.cu + ui.b) : 0;
}

template <int MODE>
__device__ __forceinline__ UnitInfo unit_info(const AttnParams& P, int u) {
  // Units grouped by KV head (so CTAs running at the same time stream the same
  // K/V and share it in L2), heaviest (largest p) first within a group, the G
  // query heads of a group adjacent.
  // Sequences of a batch come one after another.
  UnitInfo ui;
  const int per_seq = P.Hq * P.P;
  const int bseq = u / per_seq;
  u -= bseq * per_seq;
  int64_t tok0_unused;
  seq_range(P.cu, P.total, P.N, bseq, tok0_unused, ui.Nb);
  ui.b = bseq;
  ui.g = u / (P.G * P.P);
  const int rem = u - ui.g * P.G * P.P;
  ui.p = P.P - 1 - rem / P.G;
  ui.h = ui.g * P.G + rem % P.G;
  ui.hs = bseq * P.H_sel + (int)(((int64_t)ui.h * P.H_sel) / P.Hq);
  const int Tb = (ui.Nb + 127) / 128;
  const int last_b = min(2 * ui.p + 1, Tb - 1);
  const int n_dense = max(0, last_b + 1);  // 0: the pair lies past the sequence's end
  ui.nvc = 0;
  ui.nv = 0;
  ui.d1start = 0;
  if (n_dense == 0) {
    ui.mode = kModeDense;
    ui.n = 0;
    return ui;
  }
  if (MODE == kAttnDense) {
    ui.mode = kModeDense;
    ui.n = n_dense;
    return ui;
  }
  if (MODE == kAttnBlock) {
    const int64_t hb = (int64_t)bseq * P.Hq + ui.h;  // plan slot of (sequence, head)
    ui.mode = kModeBlock;
    ui.n = P.bcnt[hb * P.P + ui.p];
    ui.d1start = (int)(hb * P.P * (P.P + 1) + (int64_t)ui.p * (ui.p + 1));
    return ui;
  }
  const int32_t* d1pref = P.pp.d1pref + (int64_t)ui.hs * P.L.d1pref_len;
  // key block b = 2p+1-d' must lie in [0, last_b]  =>  d' in [2p+1-last_b, 2p+1]
  const int lo = 2 * ui.p + 1 - last_b, hi = 2 * ui.p + 1;
  const int nslash = d1pref[hi + 1] - d1pref[lo];
  const int nvp = P.pp.vpair[(int64_t)ui.hs * P.L.vpair_len + ui.p];
  const int nvc = (nvp + 127) / 128;
  if (nvc + nslash < n_dense) {
    ui.mode = kModeSplit;
    ui.n = nvc + nslash;
    ui.nvc = nvc;
    ui.nv = P.pp.meta[4 * ui.hs + 0];
    ui.d1start = d1pref[lo];
  } else {
    ui.mode = kModeDenseVS;
    ui.n = n_dense;
  }
  return ui;
}

struct Item {
  int kind;
  int b;      // key block (tile) or chunk index (vertical chunk)
  int flags;  // block sparse: bit s set iff the block is kept for sub-tile s,
              // bit 2 + s iff it is the last block kept for sub-tile s
};

__device__ __forceinline__ Item unit_item(const AttnParams& P, const UnitInfo& ui, int k) {
  Item it;
  it.flags = 3;
  if (ui.mode == kModeBlock) {
    const uint32_t e = P.blist[(int64_t)ui.d1start + k];
    it.kind = kItemTile;
    it.b = (int)(e & 0xFFFFu);
    it.flags = (int)((e >> 30) | (((e >> 28) & 3u) << 2));
  } else if (ui.mode != kModeSplit) {
    it.kind = kItemTile;
    it.b = k;
  } else if (k < ui.nvc) {
    it.kind = kItemVChunk;
    it.b = k;
  } else {
    it.kind = kItemTile;
    it.b = 2 * ui.p + 1 - P.pp.d1list[(int64_t)ui.hs * P.L.d1_len + ui.d1start + (k - ui.nvc)];
  }
  return it;
}

__device__ __forceinline__ uint32_t prefix_word(int n, int lo) {
  // bits [0, n - lo) of the 32-bit word covering positions [lo, lo + 32)
  const int k = n - lo;
  return k <= 0 ? 0u : (k >= 32 ? 0xffffffffu : ((1u << k) - 1u));
}

// 128-bit keep-mask of row i for one item; returns false if every key is kept.
template <int MODE>
__device__ __forceinline__ bool item_mask(const AttnParams& P, const UnitInfo& ui, const Item& it,
                                          int i, int t_sub, uint32_t (&w)[4]) {
  if (it.kind == kItemVChunk) {
    const int32_t* base = P.pp.vlist + (int64_t)ui.hs * P.L.N + 128 * it.b;
    const int cnt = min(128, ui.nv - 128 * it.b);
    int n = cnt;
    if (base[cnt - 1] > i) {
      int lo = 0, hi = cnt;
      while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (base[mid] <= i) lo = mid + 1;
        else hi = mid;
      }
      n = lo;
    }
    if (n == 128) return false;
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = prefix_word(n, 32 * q);
    return true;
  }
  const int b = it.b;
  // causal part for the keys of block b: keep c <= i - 128 b
  const bool below = b < t_sub;  // whole block in the past of every row of the sub-tile
  if (MODE == kAttnBlock && !((it.flags >> (t_sub - 2 * ui.p)) & 1)) {  // (callers skip these)
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = 0u;  // not kept for this sub-tile's query block
    return true;
  }
  if (MODE != kAttnVS || ui.mode == kModeDense) {
    if (below) return false;
    const int n = i - 128 * b + 1;
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = prefix_word(n, 32 * q);
    return true;
  }
  // offset window: bit c = [ i - (128 b + c) is a selected offset ]
  const uint32_t* sb = P.pp.sbits + (int64_t)ui.hs * P.L.sbits_words;
  const int64_t pos0 = (int64_t)ui.Nb - i + 128 + 128 * b;
  const uint32_t* sw = sb + (pos0 >> 5);
  const int sh = (int)(pos0 & 31);
  uint32_t x[5];
#pragma unroll
  for (int q = 0; q < 5; ++q) x[q] = __ldg(sw + q);
  uint32_t s[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) s[q] = __funnelshift_r(x[q], x[q + 1], sh);
  const uint32_t* vb = P.pp.vbits + (int64_t)ui.hs * P.L.vbits_words + 4 * b;
  if (ui.mode == kModeDenseVS) {
    const int n = below ? 128 : i - 128 * b + 1;
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = s[q] | (__ldg(vb + q) & prefix_word(n, 32 * q));
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = s[q] & ~__ldg(vb + q);
  }
  return true;
}

// p = 2^(s * scale_log2 - m) for one 128-column row (s is already -inf where
// masked), packed to bf16 pairs and stored over the row's S columns in TMEM
// 32 columns at a time (all of S is already in registers), row sum into ls.
// One call site only: two inlined copies make the compiler spill the row.
__device__ __forceinline__ void exp_tile(const uint32_t (&sr)[4][32], float sl2, float m_base,
                                         uint32_t tS, float& ls) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t pk[16];  // P of 32 columns, stored as soon as it is formed
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      const float x0 = fmaf(__uint_as_float(sr[q][c]), sl2, -m_base);
      const float x1 = fmaf(__uint_as_float(sr[q][c + 1]), sl2, -m_base);
      const float p0 = ex2_approx(x0);
      const float p1 = ex2_approx(x1);
      acc[(c >> 1) & 1] += p0;
      acc[2 + ((c >> 1) & 1)] += p1;
      pk[c / 2] = pack_bf16x2(p0, p1);
    }
    tmem_st16(tS + 16 * q, pk);
  }
  ls = (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <int D, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKg,
                   const __grid_constant__ CUtensorMap tmVg, const AttnParams P) {
  using C = Cfg<D>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + 2 * C::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kData);
  // K/V tiles stream through an S-slot ring in the order K(0), V(0), K(1),
  // V(1), ... of each unit.  They are grouped into stages that complete on one
  // barrier each: [K(0)], [V(0), K(1)], ..., [V(n-2), K(n-1)], [V(n-1)], so
  // that one wait of the MMA issuer covers both tiles a step needs.  Every
  // stage holds at least one tile, so at most S stages are in flight and S
  // stage barriers suffice.
  enum { B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_PFULL = 4, B_OFULL = 6, B_DRAIN = 8,
         B_STAGE = 9, B_EMPTY = 9 + S, B_END = 9 + 2 * S };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + B_END);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_PFULL + s), 128);
      mbar_init(bar(B_OFULL + s), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(B_STAGE + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (MODE == kAttnVS) {
      tma_prefetch_desc(&tmKg);
      tma_prefetch_desc(&tmVg);
    }
  }
  if (warp == kWarpMMA) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const WaitCtx wc{P.wait_limit_ns, P.status, abort_flag};
  if (MODE == kAttnDense && P.cu && blockIdx.x == 0 && tid == 0) {
    // the sparse path's plan kernel checks the offsets; here the first CTA does
    for (int b = 0; b < P.B; ++b) {
      int64_t t0;
      int nb;
      if (!seq_range(P.cu, P.total, P.N, b, t0, nb)) atomicOr(P.status, VS_DEVFLAG_BOUNDS);
    }
  }

  if (warp < 8) {
    // ------------------------------------------------ softmax + epilogue
    const int sub = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + sub * 128;
    const uint32_t tO = tbase + lane_off + 256 + sub * 128;
    uint32_t scnt = 0, ucount = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < P.num_units && ok; u += gridDim.x) {
      const UnitInfo ui = unit_info<MODE>(P, u);
      const int i = 256 * ui.p + 128 * sub + r;
      const int im = max(0, min(i, ui.Nb - 1));
      const int t_sub = 2 * ui.p + sub;
      // output row pointers are formed where they are used (few live registers
      // across the tile loop)
      auto orow_of = [&]() {
        return P.O + (unit_tok0(P, ui) + i) * P.q_stride + (int64_t)ui.h * D;
      };
      auto lrow_of = [&]() { return P.lse + (int64_t)ui.h * P.total + unit_tok0(P, ui) + i; };
      if (ui.n == 0) {
        if (i < ui.Nb) {
          __nv_bfloat16* orow = orow_of();
          for (int c = 0; c < D; c += 8)
            *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
          if (P.lse) *lrow_of() = -INFINITY;
        }
        continue;
      }
      float m_use = -INFINITY, l = 0.f;
      int nproc = 0;  // items this sub-tile has processed
      for (int k = 0; k < ui.n; ++k) {
        const Item it = unit_item(P, ui, k);
        // block sparse: the MMA issuer gives this sub-tile only the blocks it keeps
        if (MODE == kAttnBlock && !((it.flags >> sub) & 1)) continue;
        uint32_t mw[4];
        const bool masked = item_mask<MODE>(P, ui, it, im, t_sub, mw);
        if (!mbar_wait(bar(B_SFULL + sub), scnt & 1, wc)) { ok = false; break; }
        ++scnt;
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, sr[q]);
        tmem_ld_wait(sr[0]);
        reg_pin(sr[1]);
        reg_pin(sr[2]);
        reg_pin(sr[3]);
        if (masked) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (!((mw[q] >> c) & 1u)) sr[q][c] = __float_as_uint(-INFINITY);
        }
        // row max: eight independent chains of three-input max
        float m8[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) m8[t] = -INFINITY;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], __uint_as_float(sr[q][c]),
                                     __uint_as_float(sr[q][c + 1]));
        const float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]),
                               fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
        const float m_cand = mx * P.scale_log2;
        const bool need = m_cand > m_use + 8.0f;
        float factor = 1.f;
        if (need) {
          factor = ex2_approx(m_use - m_cand);  // 0 when m_use = -inf
          m_use = m_cand;
          l *= factor;
        }
        const float m_base = m_use == -INFINITY ? 0.f : m_use;
        float ls = 0.f;
        exp_tile(sr, P.scale_log2, m_base, tS, ls);
        l += ls;
        if (nproc > 0 && __any_sync(0xffffffffu, need)) {
          // O must be rescaled before PV(k) accumulates into it; the previous
          // PV is complete because S(k) was issued after it.
#pragma unroll 1
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * q, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
            tmem_st32(tO + 32 * q, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + sub));
        ++nproc;
      }
      if (!ok) break;
      if (!mbar_wait(bar(B_OFULL + sub), ucount & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      // no key at all (block sparse: possibly no PV, so O holds stale values)
      const bool empty_row = MODE == kAttnBlock && !(l > 0.f);
      __nv_bfloat16* orow = orow_of();
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * q, o);
        tmem_ld_wait(o);
        if (empty_row) {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (i < ui.Nb) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[c + 0]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[c + 4]) * inv_l, __uint_as_float(o[c + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[c + 6]) * inv_l, __uint_as_float(o[c + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + 32 * q + c) = v;
          }
        }
      }
      if (i < ui.Nb && P.lse)
        *lrow_of() =
            l > 0.f ? (m_use + log2f(l)) * 0.6931471805599453f : -INFINITY;
      ++ucount;
    }
  } else if (warp == kWarpMMA) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), kv_addr = smem_u32(sKV);
      uint32_t seq = 0, stg = 0, ucount = 0, pcnt[2] = {0, 0};
      bool ok = true;
      // Descriptors of the tile bases; per-MMA k offsets are compile-time
      // constants added to the 14-bit start-address field (addresses < 256 KB,
      // so the field never carries into its neighbour).
      const uint64_t qdesc = sdesc_sw128(q_addr, 16, 1024);
      const uint64_t kdesc = sdesc_sw128(kv_addr, 16, 1024);
      const uint64_t vdesc = sdesc_sw128(kv_addr, 16384, 1024);
      auto issue_s = [&](int sub, uint32_t slot) {
        const uint64_t ad = qdesc + ((sub * C::kQBytes) >> 4);
        const uint64_t bd = kdesc + ((slot * C::kTileBytes) >> 4);
        const uint32_t d = tbase + sub * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_ss(d, ad + off, bd + off, idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int sub, uint32_t slot, bool acc) {
        const uint64_t bd = vdesc + ((slot * C::kTileBytes) >> 4);
        const uint32_t d = tbase + 256 + sub * 128, a = tbase + sub * 128;
        mma_ts(d, a, bd, idesc_pv, acc ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) mma_ts(d, a + kk * 8, bd + ((kk * 2048) >> 4), idesc_pv, 1u);
      };
      for (int u = blockIdx.x; u < P.num_units && ok; u += gridDim.x) {
        const UnitInfo ui = unit_info<MODE>(P, u);
        if (ui.n == 0) continue;
        if (!mbar_wait(bar(B_QFULL), ucount & 1, wc)) { ok = false; break; }
        if constexpr (MODE == kAttnBlock) {
          // Each sub-tile gets S and PV only for the blocks it keeps; K and V
          // of every listed block stream through the ring as in the other
          // modes.  At the stage [V(k), K(k+1)]: PV(k) for the sub-tiles
          // keeping block k (O complete after a sub-tile's last one), then
          // S(k+1) for those keeping block k+1 -- after the sub-tile's
          // previous PV in issue order, so S never overwrites an unread P.
          int fl = unit_item(P, ui, 0).flags;
          int fl_next = ui.n > 1 ? unit_item(P, ui, 1).flags : 0;
          bool started[2] = {false, false};
          uint32_t kslot = seq % S;
          if (!mbar_wait(bar(B_STAGE + stg % S), (stg / S) & 1, wc)) { ok = false; break; }  // [K(0)]
          ++seq;
          ++stg;
          tc_fence_after();
          for (int sub = 0; sub < 2; ++sub)
            if ((fl >> sub) & 1) {
              issue_s(sub, kslot);
              mma_commit(bar(B_SFULL + sub));
            }
          mma_commit(bar(B_EMPTY + kslot));
          for (int k = 0; k < ui.n && ok; ++k) {
            const int fl_after = k + 2 < ui.n ? unit_item(P, ui, k + 2).flags : 0;  // early load
            if (!mbar_wait(bar(B_STAGE + stg % S), (stg / S) & 1, wc)) { ok = false; break; }
            ++stg;
            const uint32_t vslot = seq % S;
            ++seq;
            if (k + 1 < ui.n) {
              kslot = seq % S;
              ++seq;
            }
            for (int sub = 0; sub < 2; ++sub) {
              if ((fl >> sub) & 1) {
                if (!mbar_wait(bar(B_PFULL + sub), pcnt[sub] & 1, wc)) { ok = false; break; }
                ++pcnt[sub];
                tc_fence_after();
                issue_pv(sub, vslot, started[sub]);
                started[sub] = true;
                if ((fl >> (2 + sub)) & 1) mma_commit(bar(B_OFULL + sub));
              }
              if (k + 1 < ui.n && ((fl_next >> sub) & 1)) {
                issue_s(sub, kslot);
                mma_commit(bar(B_SFULL + sub));
              }
            }
            if (!ok) break;
            mma_commit(bar(B_EMPTY + vslot));
            if (k + 1 < ui.n) mma_commit(bar(B_EMPTY + kslot));
            fl = fl_next;
            fl_next = fl_after;
          }
          if (!ok) break;
          // a sub-tile without kept blocks (rows past the sequence's end, or an
          // empty mask row): its epilogue writes zeros from l = 0
          for (int sub = 0; sub < 2; ++sub)
            if (!started[sub]) mma_commit(bar(B_OFULL + sub));
          mma_commit(bar(B_QEMPTY));
          ++ucount;
          continue;
        }
        uint32_t kslot = seq % S;
        if (!mbar_wait(bar(B_STAGE + stg % S), (stg / S) & 1, wc)) { ok = false; break; }  // [K(0)]
        ++seq;
        ++stg;
        tc_fence_after();
        issue_s(0, kslot);
        mma_commit(bar(B_SFULL + 0));
        issue_s(1, kslot);
        mma_commit(bar(B_SFULL + 1));
        mma_commit(bar(B_EMPTY + kslot));
        for (int k = 0; k < ui.n && ok; ++k) {
          // one wait for V(k) and K(k+1): stage [V(k), K(k+1)] (or [V(n-1)])
          if (!mbar_wait(bar(B_STAGE + stg % S), (stg / S) & 1, wc)) { ok = false; break; }
          ++stg;
          const uint32_t vslot = seq % S;
          ++seq;
          if (k + 1 < ui.n) {
            kslot = seq % S;
            ++seq;
          }
          for (int sub = 0; sub < 2; ++sub) {
            // P(k) of this sub-tile; at k = 0 this also means its rows' previous
            // epilogue has read O (the same threads arrive after it), so PV(0)
            // may overwrite O
            if (!mbar_wait(bar(B_PFULL + sub), pcnt[sub] & 1, wc)) { ok = false; break; }
            ++pcnt[sub];
            tc_fence_after();
            issue_pv(sub, vslot, k > 0);
            if (sub == 1) mma_commit(bar(B_EMPTY + vslot));
            if (k + 1 < ui.n) {
              issue_s(sub, kslot);
              mma_commit(bar(B_SFULL + sub));
              if (sub == 1) mma_commit(bar(B_EMPTY + kslot));
            } else {
              mma_commit(bar(B_OFULL + sub));
            }
          }
        }
        if (!ok) break;
        mma_commit(bar(B_QEMPTY));
        ++ucount;
      }
      // Drain: every MMA issued so far must finish before TMEM is freed.
      mma_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0, P.wait_limit_ns);
    }
  } else if (warp == kWarpLoad) {
    // ------------------------------------------------------- TMA producer
    uint32_t seq = 0, stg = 0, ucount = 0;
    bool ok = true;
    const int nsub64 = D / 64;
    for (int u = blockIdx.x; u < P.num_units && ok; u += gridDim.x) {
      const UnitInfo ui = unit_info<MODE>(P, u);
      if (ui.n == 0) continue;
      if (ucount > 0 && !mbar_wait(bar(B_QEMPTY), (ucount - 1) & 1, wc)) { ok = false; break; }
      const int64_t tok0 = unit_tok0(P, ui);
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_QFULL), 2 * C::kQBytes);
        for (int s = 0; s < 2; ++s)
          for (int h = 0; h < nsub64; ++h)
            tma_load_2d(smem_u32(sQ + s * C::kQBytes + h * 16384), &tmQ, bar(B_QFULL),
                        ui.h * D + 64 * h, (int)(tok0 + 256 * ui.p + 128 * s));
      }
      ++ucount;
      // tile t of the unit: K(t/2) for even t, V(t/2) for odd t; a stage
      // starts at t = 0 and at every odd t, and holds two tiles except the
      // first and the last
      const int ntiles = 2 * ui.n;
      for (int t = 0; t < ntiles && ok; ++t) {
        const int k = t >> 1, kv = t & 1;
        const Item it = unit_item(P, ui, k);
        {
          const uint32_t slot = seq % S;
          if (seq >= (uint32_t)S && !mbar_wait(bar(B_EMPTY + slot), ((seq / S) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar(B_STAGE + stg % S);
          if (t == 0 || kv == 1) {  // first tile of a stage: arm it for all of its bytes
            const int nst = (t == 0 || t == ntiles - 1) ? 1 : 2;
            if (lane == 0) mbar_arrive_expect_tx(fb, nst * C::kTileBytes);
          }
          __syncwarp();
          const uint32_t dst = smem_u32(sKV + slot * C::kTileBytes);
          if (it.kind == kItemTile) {
            if (lane == 0) {
              const CUtensorMap* m = kv ? &tmV : &tmK;
              for (int h = 0; h < nsub64; ++h)
                tma_load_2d(dst + h * 16384, m, fb, ui.g * D + 64 * h, (int)(tok0 + 128 * it.b));
            }
          } else if (P.pack_vrows > 0) {
            if (lane == 0) {
              const CUtensorMap* m = kv ? &tmVg : &tmKg;
              for (int h = 0; h < nsub64; ++h)
                tma_load_2d(dst + h * 16384, m, fb, 64 * h,
                            (int)(ui.hs * P.pack_vrows + 128 * it.b));
            }
          } else {
            const int32_t* base = P.pp.vlist + (int64_t)ui.hs * P.L.N + 128 * it.b;
            const int cnt = min(128, ui.nv - 128 * it.b);
            int rr[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int e = 4 * lane + q;
              rr[q] = (int)tok0 + base[e < cnt ? e : 0];
            }
            const CUtensorMap* m = kv ? &tmVg : &tmKg;
            for (int h = 0; h < nsub64; ++h)
              tma_gather4(dst + h * 16384 + lane * 512, m, fb, ui.g * D + 64 * h, rr[0], rr[1],
                          rr[2], rr[3]);
          }
          ++seq;
          if (t == 0 || kv == 0 || t == ntiles - 1) ++stg;  // the stage's last tile is issued
        }
      }
    }
    // Drain: let every issued copy land before shared memory is released.
    if (lane == 0) {
      const uint32_t first = stg > (uint32_t)S ? stg - S : 0;
      for (uint32_t x = first; x < stg; ++x)
        mbar_wait_drain(bar(B_STAGE + (x % S)), (x / S) & 1, P.wait_limit_ns);
      if (ucount > 0) mbar_wait_drain(bar(B_QFULL), (ucount - 1) & 1, P.wait_limit_ns);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}


static void encode_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, int64_t inner,
                       int64_t rows, int64_t row_stride_elems, uint32_t box_rows, CUresult* rc) {
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) *rc = r;
}

template <int D, int MODE>
static cudaError_t launch_tc_impl(const AttnArgs& a, const PlanLayout& L) {
  constexpr bool SPARSE = MODE == kAttnVS;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap mQ, mK, mV, mKg, mVg;
  CUresult rc = CUDA_SUCCESS;
  encode_map(enc, &mQ, a.Q, (int64_t)a.Hq * D, a.total, a.q_stride, 128, &rc);
  encode_map(enc, &mK, a.K, (int64_t)a.Hkv * D, a.total, a.kv_stride, 128, &rc);
  encode_map(enc, &mV, a.V, (int64_t)a.Hkv * D, a.total, a.kv_stride, 128, &rc);
  if (SPARSE && a.pack_vrows > 0) {  // packed vertical rows: [H_sel * vrows][D] tiles
    encode_map(enc, &mKg, a.pack_k, D, (int64_t)a.B * a.H_sel * a.pack_vrows, D, 128, &rc);
    encode_map(enc, &mVg, a.pack_v, D, (int64_t)a.B * a.H_sel * a.pack_vrows, D, 128, &rc);
  } else {
    encode_map(enc, &mKg, a.K, (int64_t)a.Hkv * D, a.total, a.kv_stride, 1, &rc);
    encode_map(enc, &mVg, a.V, (int64_t)a.Hkv * D, a.total, a.kv_stride, 1, &rc);
  }
  if (rc != CUDA_SUCCESS) return cudaErrorInvalidValue;
  AttnParams P;
  P.N = a.N;
  P.Hq = a.Hq;
  P.Hkv = a.Hkv;
  P.H_sel = SPARSE ? a.H_sel : 1;
  P.T = L.T;
  P.P = L.P;
  P.G = a.Hq / a.Hkv;
  P.num_units = a.B * a.Hq * L.P;
  P.cu = a.cu_seqlens;
  P.B = a.B;
  P.total = a.total;
  P.q_stride = a.q_stride;
  P.scale_log2 = a.scale * 1.4426950408889634f;
  P.O = static_cast<__nv_bfloat16*>(a.O);
  P.lse = a.lse;
  P.status = a.status;
  P.wait_limit_ns = kDefaultWaitLimitNs;
  P.L = L;
  P.pp = plan_ptrs(L, a.ws);
  P.pack_vrows = SPARSE ? a.pack_vrows : 0;
  P.bcnt = nullptr;
  P.blist = nullptr;
  if (MODE == kAttnBlock) {
    const BlockPlanLayout B = BlockPlanLayout::make(a.N, a.B * a.Hq);
    P.bcnt = reinterpret_cast<const int32_t*>(static_cast<const char*>(a.ws) + B.off_cnt);
    P.blist = reinterpret_cast<const uint32_t*>(static_cast<const char*>(a.ws) + B.off_list);
  }
  auto kern = attn_tc_kernel<D, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<D>::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = P.num_units < device_sm_count() ? P.num_units : device_sm_count();
  kern<<<grid, kAttnThreads, Cfg<D>::kSmem, a.stream>>>(mQ, mK, mV, mKg, mVg, P);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const AttnArgs& a, const PlanLayout& L) {
  if (a.block_mask) {
    if (a.d == 128) return launch_tc_impl<128, kAttnBlock>(a, L);
    if (a.d == 64) return launch_tc_impl<64, kAttnBlock>(a, L);
    return cudaErrorInvalidValue;
  }
  if (a.d == 128)
    return a.sparse ? launch_tc_impl<128, kAttnVS>(a, L) : launch_tc_impl<128, kAttnDense>(a, L);
  if (a.d == 64)
    return a.sparse ? launch_tc_impl<64, kAttnVS>(a, L) : launch_tc_impl<64, kAttnDense>(a, L);
  return cudaErrorInvalidValue;
}

}  // namespace vs

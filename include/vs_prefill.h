/*
 * vs_prefill.h -- C ABI of libvs, vertical-slash sparse prefill attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method (VSPrefill summary pages, "VSPrefill: Vertical-Slash Sparse
 * Attention with Lightweight Indexing for Long-Context Prefilling"):
 *   - attention in long-context prefill concentrates on vertical lines (key
 *     columns that every later query attends to) and slash lines (diagonals at
 *     a fixed relative offset o = i - j)  -- Technical Summary, section 2,
 *     "Core Concept: Vertical-Slash Pattern";
 *   - a light indexer predicts one score per column and one per offset from
 *     concat(K with RoPE, V)  -- section 2, "VSIndexer";
 *   - a cumulative threshold on those scores picks the budgets (k_v, k_s)
 *     -- section 2, "Adaptive Inference Pipeline", "Dynamic Budgeting";
 *   - a fused FlashAttention-style kernel attends each query to the union of
 *     the selected columns and the keys at the selected offsets behind it,
 *     without a precomputed mask -- section 2, "Fused Kernel Execution".
 *
 * Conventions for every call:
 *   - Every pointer argument is a DEVICE pointer on the current CUDA device
 *     (except `flags` of vs_read_device_status); the caller owns every buffer (inputs,
 *     outputs, workspace) and the stream.  The library allocates nothing,
 *     keeps no mutable global state (vs_sparse_attn_fwd_static_scratch is the
 *     one documented exception), never writes its inputs and overwrites its
 *     outputs completely.
 *   - Calls are asynchronous on `stream`; selected counts stay on the device,
 *     so select -> attention needs no host synchronisation.
 *   - Host-side argument checks run before anything is launched and return
 *     VS_ERR_INVALID_ARG / VS_ERR_UNSUPPORTED / VS_ERR_WORKSPACE.  A failed
 *     launch returns VS_ERR_CUDA.  Device-side problems (an index outside
 *     [0, N), a count above its row length, a bounded wait that gave up) are
 *     OR-ed into a status word at the start of the workspace; read it with
 *     vs_read_device_status.  Kernels never trap, assert or print.
 *   - Tensors are token-major: element (t, h, c) of Q lives at
 *     Q[t * q_stride_tok + h * d + c]; K and V likewise with kv_stride_tok.
 *     Strides are in elements and must be multiples of 8 (16-byte rows).
 *   - GQA: query head h reads KV head h / (Hq / Hkv) and index-set head
 *     h * H_sel / Hq.
 */
#ifndef VS_PREFILL_H
#define VS_PREFILL_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VS_OK = 0,
  VS_ERR_INVALID_ARG = 1,    /* null pointer, bad size, k/cap/tau out of range */
  VS_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. d not in {64,128}) */
  VS_ERR_WORKSPACE = 3,      /* workspace missing, misaligned or too small */
  VS_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  VS_ERR_DEVICE_TIMEOUT = 5, /* returned by vs_read_device_status */
  VS_ERR_DEVICE_BOUNDS = 6   /* returned by vs_read_device_status */
} vs_status;

typedef enum { VS_SELECT_TOPK = 0, VS_SELECT_THRESHOLD = 1, VS_SELECT_MAXFRAC = 2 } vs_select_mode;

typedef enum { VS_BF16 = 0, VS_FP32 = 1 } vs_dtype;

/* Device status bits (vs_read_device_status `flags`). */
#define VS_DEVFLAG_TIMEOUT 0x1
#define VS_DEVFLAG_BOUNDS 0x2

/* Static, human-readable name of a status code. */
const char* vs_status_string(vs_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int vs_version(void);

/*
 * vs_index_scores -- the indexer: a shared-weight two-layer linear map on
 * concat(K with RoPE, V) producing a vertical and a slash score per position
 * (Technical Summary, section 2, "VSIndexer": input concatenated K and V with
 * RoPE on K, a bilayer linear network with separate down-projection heads for
 * the vertical and slash scores, linear cost in n).  The pages do not fix the
 * exact form; this library reads it as
 *     x = [k_t ; v_t] (2d values, k first),  h = ReLU(W1 x),
 *     logits_v[g][t] = W2[0] . h,  logits_s[g][t] = W2[1] . h,
 * no biases, one weight set shared by all KV heads g.  logits_s[g][t] is the
 * score of slash offset o = t.
 *   K, V      [N, Hkv, d] in `dtype` (VS_BF16 or VS_FP32), token stride
 *             `stride_tok`, head stride `stride_head` (elements).
 *   W1        fp32 [hidden][2d] row-major (device).   W2  fp32 [2][hidden].
 *   hidden    1..1024.
 *   logits_v, logits_s   fp32 [Hkv][N] outputs (device), fully overwritten.
 * Arithmetic: bf16 K/V with d = 64 or 128, hidden = 128 or 256, stride_head
 * = d and 16-byte aligned rows run on the tensor cores.  There W1 is split
 * into two bf16 parts (hi = bf16(W1), lo = bf16(W1 - hi)), the products are
 * exact and the accumulation is fp32; the result is deterministic (at most
 * two partial sums per logit, added onto zero).  Other inputs run in fp32 on
 * the CUDA cores.  The tensor-core kernel's device waits are bounded; a wait
 * that runs out (never on a correct launch) leaves NaN in the logits of the
 * tiles it affects, since this call has no workspace status word.
 */
vs_status vs_index_scores(const void* K, const void* V, vs_dtype dtype, int N, int Hkv, int d,
                          int64_t stride_tok, int64_t stride_head, const float* W1,
                          const float* W2, int hidden, float* logits_v, float* logits_s,
                          cudaStream_t stream);

/*
 * vs_select -- per-head budget selection over a score vector (Technical
 * Summary, section 2, "Dynamic Budgeting": a cumulative-threshold strategy
 * sets the budgets from the predicted importance scores; the German page's
 * Inferenz-Pipeline adds the top-k reading).  One call handles H heads.
 *   scores   fp32 [H][ld_scores] (device), the first N entries of each row used.
 *            Scores are logits: the "mass" of entry r is softmax(scores)_r.
 *   Order    score descending, NaN after -inf, ties to the smaller index.
 *   TOPK     keeps the first k_or_cap entries in that order.
 *   THRESHOLD keeps the smallest prefix in that order whose mass reaches
 *            tau (0 < tau <= 1): p_r = exp(s_r - s_max) in fp64, k is the
 *            smallest k >= 1 with sum_{r<k} p_r >= tau * sum_r p_r; tau = 1
 *            keeps every entry with p_r > 0; then k = min(k, k_or_cap).
 *   MAXFRAC  FlashPrefill's max-based dynamic threshold (FlashPrefill summary
 *            page, section 2B: discard every candidate scoring below alpha
 *            times the best one; no sort, no cumulative sum).  `tau` carries
 *            alpha (0 < alpha <= 1); with the mass reading the rule is
 *            p_r >= alpha, decided in fp64 as
 *              s_r == s_max  or  (double)s_r - (double)s_max >= log(alpha)
 *            (log taken on the host); NaN is never kept, an all-NaN row
 *            keeps one entry; then k = min(k, k_or_cap) in the order above.
 *   idx      int32 [H][ld_idx] (device): for each head the kept indices in
 *            ascending order, then -1 up to k_or_cap (entries past k_or_cap
 *            untouched).  ld_idx >= k_or_cap.
 *   count    int32 [H] (device): kept entries per head.
 *   ws       device workspace of at least vs_select_workspace_size(H, N)
 *            bytes, 256-byte aligned (holds the device status word).
 * Requires 1 <= k_or_cap <= N <= 2^20; tau in (0, 1] for THRESHOLD and
 * MAXFRAC (else VS_ERR_INVALID_ARG).
 * The fp64 mass sums are added in a fixed order (no atomics), so repeated
 * calls with the same H and N on the same device give the same result bit
 * for bit.  That order follows the thread-block cluster the launcher picks,
 * which depends on H, N and the device's SM count: a row selected in a call
 * with another H or N, or on another device, may be summed in another order,
 * and where the decision lies within rounding of tau * sum_r p_r it may then
 * differ by one entry.
 */
size_t vs_select_workspace_size(int H, int N);
vs_status vs_select(const float* scores, int H, int N, int64_t ld_scores, vs_select_mode mode,
                    int k_or_cap, double tau, int32_t* idx, int64_t ld_idx, int32_t* count,
                    void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * vs_select_varlen -- vs_select for B sequences packed along the token axis,
 * in one launch (the budget step of a batched prefill: each sequence's
 * vertical or slash scores select that sequence's index set).
 *   scores     fp32 [H][total_tokens] (device): head h of sequence b is
 *              scores[h * total_tokens + cu_seqlens[b] + j], j < n_b.
 *   cu_seqlens int32 [B + 1] (device), as for vs_sparse_attn_fwd_varlen;
 *              max_seqlen >= every n_b (host; sizes the launch).
 *   caps       int32 [B] (device): k_or_cap of sequence b, 1 <= caps[b] <=
 *              n_b and <= cap_max; cap_max >= 1 and ld_idx >= cap_max.
 *   mode, tau  as for vs_select, applied to every row.
 *   idx        int32 [B * H][ld_idx] (device): row b * H + h as vs_select's
 *              row for that sequence and head (indices from the sequence's
 *              start, ascending, then -1 up to caps[b]; entries past caps[b]
 *              untouched) -- the layout vs_sparse_attn_fwd_varlen reads.
 *   count      int32 [B * H] (device).
 *   ws         device workspace of at least
 *              vs_select_workspace_size_varlen(B, H, max_seqlen) bytes,
 *              256-byte aligned (status word).
 * A sequence with n_b = 0 keeps nothing (count 0, its rows untouched).  A
 * malformed offset or cap empties that sequence the same way and sets
 * VS_DEVFLAG_BOUNDS.  B * H <= 65535; max_seqlen <= 2^20.  The fp64 sums
 * are in a fixed order for a given (B, H, max_seqlen) and device, as for
 * vs_select (the order follows the cluster the launcher picks for B * H rows
 * of max_seqlen, so it may differ from a single-sequence call's).
 */
size_t vs_select_workspace_size_varlen(int B, int H, int max_seqlen);
vs_status vs_select_varlen(const float* scores, int total_tokens, int B, const int32_t* cu_seqlens,
                           int max_seqlen, int H, vs_select_mode mode, const int32_t* caps,
                           int cap_max, double tau, int32_t* idx, int64_t ld_idx, int32_t* count,
                           void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * vs_sparse_attn_fwd -- causal vertical-slash sparse attention forward
 * (Technical Summary, section 2, "Fused Kernel Execution": the vertical and
 * slash index lists are merged on the fly inside a FlashAttention-style
 * kernel, with no precomputed mask).  For query i of query head h:
 *     K_i = { j in V : j <= i }  union  { i - o : o in S, o <= i }
 * (each key once), and O_i = softmax_j(scale * q_i . k_j) over K_i times V;
 * LSE_i = log sum_{j in K_i} exp(scale * q_i . k_j).  An empty K_i gives
 * O_i = 0 and LSE_i = -inf.
 *   Q        [N, Hq, d], K, V [N, Hkv, d], `dtype` (VS_BF16: tensor-core path;
 *            VS_FP32: fp32 CUDA-core path).  d in {64, 128}.  Hq % Hkv == 0.
 *            1 <= N <= 2^22 (dense: 2^24).
 *   softmax_scale   0 selects 1/sqrt(d).
 *   H_sel    number of index sets; Hq % H_sel == 0.
 *   v_idx    int32 [H_sel][v_ld] vertical columns, v_cnt int32 [H_sel];
 *   s_idx    int32 [H_sel][s_ld] slash offsets,   s_cnt int32 [H_sel]
 *            (device; as produced by vs_select: entries in [0, N), the first
 *            cnt entries of each row used; duplicates and order do not matter).
 *   O        [N, Hq, d] in `dtype` with token stride q_stride_tok (output).
 *   lse      fp32 [Hq][N] (output) or NULL.
 *   ws       device workspace, 256-byte aligned, of at least
 *            vs_attn_workspace_size(N, Hq, H_sel, d) bytes (the plan).  With
 *            vs_attn_workspace_size_ld(N, Hq, H_sel, d, v_ld) bytes or more the
 *            selected vertical K/V rows are first packed contiguously and then
 *            loaded as tiles (when every index set's query heads lie in one KV
 *            group); with less they are gathered row by row.  Results are the
 *            same either way.
 */
size_t vs_attn_workspace_size(int N, int Hq, int H_sel, int d);
size_t vs_attn_workspace_size_ld(int N, int Hq, int H_sel, int d, int64_t v_ld);
vs_status vs_sparse_attn_fwd(const void* Q, const void* K, const void* V, vs_dtype dtype, int N,
                             int Hq, int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                             float softmax_scale, int H_sel, const int32_t* v_idx, int64_t v_ld,
                             const int32_t* v_cnt, const int32_t* s_idx, int64_t s_ld,
                             const int32_t* s_cnt, void* O, float* lse, void* ws,
                             size_t ws_bytes, cudaStream_t stream);

/*
 * vs_sparse_attn_fwd_varlen / vs_dense_attn_fwd_varlen -- the same attention
 * over a batch of B independent sequences packed along the token axis
 * (variable-length batched prefill; each sequence attends only to itself).
 *   total_tokens  rows of Q, K, V, O (and columns of lse: lse is fp32
 *            [Hq][total_tokens]); at most 2^31 - 1.
 *   cu_seqlens    int32 [B + 1] (DEVICE): sequence b is tokens
 *            [cu_seqlens[b], cu_seqlens[b + 1]); the offsets must not
 *            decrease, start at >= 0, end at <= total_tokens and give no
 *            sequence longer than max_seqlen.  A malformed entry makes that
 *            sequence empty (its O rows are not written) and sets
 *            VS_DEVFLAG_BOUNDS.
 *   max_seqlen    the longest sequence (sizes the plan; >= 1).
 *   Index sets (sparse): one per (sequence, index-set head): v_idx
 *            [B * H_sel][v_ld] with v_cnt [B * H_sel] (row b * H_sel + hs),
 *            likewise s_idx / s_cnt; positions are relative to the sequence
 *            start (columns and offsets in [0, that sequence's length)).
 *   ws       at least vs_attn_workspace_size_varlen(B, max_seqlen, H_sel, d,
 *            0) bytes (the plan; dense: 256); with v_ld in place of 0, room to
 *            pack the selected vertical rows, as for vs_sparse_attn_fwd.
 *   VS_BF16 only (else VS_ERR_UNSUPPORTED); B * H_sel <= 65535.
 * The pages prefill one sequence at a time; this batching follows their
 * per-sequence definition unchanged.
 */
size_t vs_attn_workspace_size_varlen(int B, int max_seqlen, int H_sel, int d, int64_t v_ld);
vs_status vs_sparse_attn_fwd_varlen(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                    int total_tokens, int B, const int32_t* cu_seqlens,
                                    int max_seqlen, int Hq, int Hkv, int d, int64_t q_stride_tok,
                                    int64_t kv_stride_tok, float softmax_scale, int H_sel,
                                    const int32_t* v_idx, int64_t v_ld, const int32_t* v_cnt,
                                    const int32_t* s_idx, int64_t s_ld, const int32_t* s_cnt,
                                    void* O, float* lse, void* ws, size_t ws_bytes,
                                    cudaStream_t stream);
vs_status vs_dense_attn_fwd_varlen(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                   int total_tokens, int B, const int32_t* cu_seqlens,
                                   int max_seqlen, int Hq, int Hkv, int d, int64_t q_stride_tok,
                                   int64_t kv_stride_tok, float softmax_scale, void* O, float* lse,
                                   void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * vs_block_select -- FlashPrefill's block pattern discovery (FlashPrefill
 * summary page, section 2A: a skeleton of uniformly spaced queries probes
 * every key block through the block's mean key, a proxy that is monotone in
 * the block's total attention weight; section 2B: keep key block J for query
 * block I when its score is at least alpha times the best block's -- no
 * sort, no cumulative sum).  Read as, with 128-row blocks and the probes of
 * block I at rows 128 I + 8 m (m = 0..15, below N):
 *     Score(I, J) = mean over probes q of softmax_{J' < I}(scale q . kbar_J')[J],
 *     J < I kept iff Score(I, J) >= alpha * max_J' Score(I, J'),
 * the diagonal block J = I always kept; computed in fp64.
 *   Q [N, Hq, d], K [N, Hkv, d] (VS_BF16 or VS_FP32; strides as for the
 *            attention calls).  1 <= N <= 2^18.  0 < alpha <= 1.
 *   mask     uint32 [Hq][T][W] output (device), T = ceil(N / 128),
 *            W = ceil(T / 32): bit J of row (h, I) set iff block J is kept.
 *   ws       at least vs_block_select_workspace_size(N, Hkv, d) bytes,
 *            256-byte aligned: status word and work counter, the fp64 block
 *            means, and one dot-product scratch per SM of the current device
 *            (the size depends on that device; a workspace sized on a device
 *            with fewer SMs fails the check with VS_ERR_WORKSPACE).
 */
size_t vs_block_select_workspace_size(int N, int Hkv, int d);
vs_status vs_block_select(const void* Q, const void* K, vs_dtype dtype, int N, int Hq, int Hkv,
                          int d, int64_t q_stride_tok, int64_t kv_stride_tok, float softmax_scale,
                          double alpha, uint32_t* mask, void* ws, size_t ws_bytes,
                          cudaStream_t stream);

/*
 * vs_block_sparse_attn_fwd -- causal attention over kept key blocks
 * (FlashPrefill summary page, section 3: a block-sparse kernel that jumps
 * directly to the next kept block by index).  Query i (block I = i / 128)
 * attends to every key j <= i of every block J kept in row (h, I) of
 * `block_mask` (the layout vs_block_select writes; bits J > I are ignored).
 * O and lse as for vs_sparse_attn_fwd; a row with no kept key gets O = 0 and
 * LSE = -inf.  VS_BF16 only; 1 <= N <= 2^18.
 *   ws       at least vs_block_attn_workspace_size(N, Hq) bytes, 256-byte
 *            aligned (status word and the per-pair block lists).
 */
size_t vs_block_attn_workspace_size(int N, int Hq);
vs_status vs_block_sparse_attn_fwd(const void* Q, const void* K, const void* V, vs_dtype dtype,
                                   int N, int Hq, int Hkv, int d, int64_t q_stride_tok,
                                   int64_t kv_stride_tok, float softmax_scale,
                                   const uint32_t* block_mask, void* O, float* lse, void* ws,
                                   size_t ws_bytes, cudaStream_t stream);

/*
 * vs_block_select_varlen / vs_block_sparse_attn_fwd_varlen -- the block
 * discovery and the block-sparse attention above for B sequences packed along
 * the token axis (batched prefill; FlashPrefill summary page, sections 2A,
 * 2B and 3, applied to each sequence on its own: blocks, probes and the
 * alpha-times-best rule are per sequence, and a sequence attends only to
 * itself).
 *   total_tokens, cu_seqlens, max_seqlen  as for vs_sparse_attn_fwd_varlen
 *            (cu_seqlens on the DEVICE; a malformed entry empties that
 *            sequence and sets VS_DEVFLAG_BOUNDS).
 *   mask / block_mask  uint32 [B][Hq][T][W] with T = ceil(max_seqlen / 128),
 *            W = ceil(T / 32): sequence b's rows of head h at (b * Hq + h) * T;
 *            vs_block_select_varlen writes rows I >= that sequence's block
 *            count as zeros.  Each sequence's rows equal what vs_block_select
 *            writes for that sequence alone (same arithmetic, same order).
 *   O, lse   as for vs_sparse_attn_fwd_varlen (lse fp32 [Hq][total_tokens]).
 *   ws       vs_block_select_workspace_size_varlen(B, max_seqlen, Hkv, d) and
 *            vs_block_attn_workspace_size_varlen(B, max_seqlen, Hq) bytes,
 *            256-byte aligned.
 * Requires 1 <= max_seqlen <= 2^18; VS_ERR_UNSUPPORTED when the batch's
 * per-(sequence, head) block lists would not fit 32-bit offsets.
 */
size_t vs_block_select_workspace_size_varlen(int B, int max_seqlen, int Hkv, int d);
vs_status vs_block_select_varlen(const void* Q, const void* K, vs_dtype dtype, int total_tokens,
                                 int B, const int32_t* cu_seqlens, int max_seqlen, int Hq,
                                 int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                                 float softmax_scale, double alpha, uint32_t* mask, void* ws,
                                 size_t ws_bytes, cudaStream_t stream);
size_t vs_block_attn_workspace_size_varlen(int B, int max_seqlen, int Hq);
vs_status vs_block_sparse_attn_fwd_varlen(const void* Q, const void* K, const void* V,
                                          vs_dtype dtype, int total_tokens, int B,
                                          const int32_t* cu_seqlens, int max_seqlen, int Hq,
                                          int Hkv, int d, int64_t q_stride_tok,
                                          int64_t kv_stride_tok, float softmax_scale,
                                          const uint32_t* block_mask, void* O, float* lse,
                                          void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * vs_sparse_attn_fwd_static_scratch -- vs_sparse_attn_fwd without a
 * caller-provided workspace.  The summary pages have no counterpart to this
 * call; it exists for callers that cannot allocate device memory: plain-C
 * hosts with no device memory manager, and plug-ins inside engines that own
 * every byte of device memory through their own pool and forbid cudaMalloc
 * (which may also synchronise the device mid-prefill).
 *   Same arguments and results as vs_sparse_attn_fwd, minus ws / ws_bytes;
 *   the caller still passes every input and output buffer.
 *   Scratch: one 16 MiB static device array inside libvs, held on every GPU
 *   that loads the library until the process exits.  Calls needing more
 *   (vs_attn_workspace_size(N, Hq, H_sel, d) > 16 MiB) return
 *   VS_ERR_UNSUPPORTED before launching anything.
 *   The first call on a device resolves the array's device address with
 *   cudaGetSymbolAddress (with that device current), and so does the first
 *   call after the device's context has been replaced (cudaDeviceReset): the
 *   address is kept per device together with the ID of the context it was
 *   taken in.  Make the first call on a device (and the first after a reset)
 *   before any stream capture.  No cudaMalloc / cudaFree or other allocating
 *   routine is called.
 *   Every call shares the array, which keeps the last call's contents (the
 *   call clears what it needs to start at zero itself); calls that overlap on
 *   the GPU -- other streams, other host threads -- race on it and must be
 *   serialised by the caller.  The device status word of this call is not
 *   exposed (vs_read_device_status needs a caller-owned workspace).
 */
vs_status vs_sparse_attn_fwd_static_scratch(const void* Q, const void* K, const void* V,
                                            vs_dtype dtype, int N, int Hq, int Hkv, int d,
                                            int64_t q_stride_tok, int64_t kv_stride_tok,
                                            float softmax_scale, int H_sel, const int32_t* v_idx,
                                            int64_t v_ld, const int32_t* v_cnt,
                                            const int32_t* s_idx, int64_t s_ld,
                                            const int32_t* s_cnt, void* O, float* lse,
                                            cudaStream_t stream);

/*
 * vs_dense_attn_fwd -- dense causal attention with the same kernel
 * machinery: the "full attention" the pages measure their speed-ups against
 * (Technical Summary, section 4, Speedup).  Same arguments as
 * vs_sparse_attn_fwd without the index sets; K_i = [0, i].
 */
vs_status vs_dense_attn_fwd(const void* Q, const void* K, const void* V, vs_dtype dtype, int N,
                            int Hq, int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                            float softmax_scale, void* O, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t stream);

/*
 * vs_attn_aggregate -- ground-truth aggregation of the full causal attention
 * weights along vertical columns and slash diagonals: the indexer's
 * distillation target (Technical Summary, section 2, "Distillation Training":
 * a kernel aggregates full attention weights along the columns and diagonals
 * online during block-wise computation, without the n x n matrix).  For query
 * head h, with p_ij = exp(scale * q_i . k_j - LSE_i) over j <= i:
 *     A_v[h][j] = sum_{i >= j} p_ij,    A_s[h][o] = sum_{i >= o} p_{i, i-o},
 * so each row of A_v and of A_s sums to N (normalise by N for the
 * distributions the distillation loss compares).
 *   Q [N, Hq, d], K [N, Hkv, d]: VS_BF16 only (else VS_ERR_UNSUPPORTED);
 *            d in {64, 128}; strides and GQA as for vs_sparse_attn_fwd.
 *   lse      fp32 [Hq][N] (device): the row log-sum-exp of the same dense
 *            causal attention with the same scale, as written by
 *            vs_dense_attn_fwd.  The weights are only as correct as lse.
 *   A_v, A_s fp32 [Hq][N] outputs (device).  A_s is zeroed by the call and
 *            accumulated with fp32 atomics, so its last bits may vary from
 *            run to run; A_v is written once per entry.
 *   ws       device workspace of at least 256 bytes, 256-byte aligned (status
 *            word).
 */
vs_status vs_attn_aggregate(const void* Q, const void* K, vs_dtype dtype, int N, int Hq, int Hkv,
                            int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                            float softmax_scale, const float* lse, float* A_v, float* A_s,
                            void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * vs_attn_aggregate_varlen -- vs_attn_aggregate for B sequences packed along
 * the token axis (each sequence's weights are its own causal softmax; the
 * sums are per sequence, at positions relative to its start).
 *   total_tokens, cu_seqlens, max_seqlen  as for vs_sparse_attn_fwd_varlen
 *            (cu_seqlens on the DEVICE; a malformed entry leaves that
 *            sequence's entries of A_v unwritten and of A_s zero, and sets
 *            VS_DEVFLAG_BOUNDS).
 *   lse      fp32 [Hq][total_tokens] as written by vs_dense_attn_fwd_varlen.
 *   A_v, A_s fp32 [Hq][total_tokens]: sequence b's column j at
 *            h * total_tokens + cu_seqlens[b] + j, its offset o likewise.
 */
vs_status vs_attn_aggregate_varlen(const void* Q, const void* K, vs_dtype dtype, int total_tokens,
                                   int B, const int32_t* cu_seqlens, int max_seqlen, int Hq,
                                   int Hkv, int d, int64_t q_stride_tok, int64_t kv_stride_tok,
                                   float softmax_scale, const float* lse, float* A_v, float* A_s,
                                   void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Device status of the last call that used `ws`: synchronises `stream`,
 * copies the status word to `*flags` (VS_DEVFLAG_* bits) and returns VS_OK,
 * VS_ERR_DEVICE_TIMEOUT or VS_ERR_DEVICE_BOUNDS accordingly.
 */
vs_status vs_read_device_status(const void* ws, cudaStream_t stream, int* flags);

/*
 * Self-test of the device-side wait limit: launches one CTA that waits on an
 * mbarrier nothing will ever arrive at, through the same bounded-wait code the
 * kernels use, giving up after `limit_ns` nanoseconds (1e3..1e10).  Afterwards
 * vs_read_device_status(ws) reports VS_ERR_DEVICE_TIMEOUT.  The CUDA context
 * stays usable.  `ws` needs 256 bytes.
 */
vs_status vs_selftest_wait_timeout(void* ws, uint64_t limit_ns, cudaStream_t stream);

/*
 * Self-test of the fp64 exponential the block discovery uses for e^x, x <= 0
 * (Tang's table-driven method; arguments below -700 give 0): y[i] = e^x[i]
 * for the n device doubles at x (each <= 0 or -inf), written to the device
 * array y.  Asynchronous on `stream`.  VS_ERR_INVALID_ARG for null pointers
 * or n < 1.
 */
vs_status vs_selftest_exp(const double* x, double* y, int n, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VS_PREFILL_H */

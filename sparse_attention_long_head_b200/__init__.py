"""Python binding of libvs (vertical-slash sparse prefill attention, sm_100a).

Argument marshalling only: every step runs in the CUDA kernels of
``libvs.so``; this module passes device pointers, sizes and the current
torch CUDA stream to the C ABI declared in ``include/vs_prefill.h`` and turns
non-OK status codes into ``VsError``.  There is no CPU fallback: if the
library has not been built, importing the binding's functions raises.

Names follow the C ABI (``vs_select``, ``vs_sparse_attn_fwd``, ...).  Tensors
are torch CUDA tensors; layouts are those of the header (token-major
``[N, H, d]`` activations, ``[H, ld]`` index rows).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvs.so")

VS_OK = 0
VS_ERR_INVALID_ARG = 1
VS_ERR_UNSUPPORTED = 2
VS_ERR_WORKSPACE = 3
VS_ERR_CUDA = 4
VS_ERR_DEVICE_TIMEOUT = 5
VS_ERR_DEVICE_BOUNDS = 6

VS_SELECT_TOPK = 0
VS_SELECT_THRESHOLD = 1
VS_SELECT_MAXFRAC = 2
VS_BF16 = 0
VS_FP32 = 1

VS_DEVFLAG_TIMEOUT = 0x1
VS_DEVFLAG_BOUNDS = 0x2

EXPORTS = (
    "vs_status_string", "vs_version", "vs_index_scores", "vs_select_workspace_size", "vs_select",
    "vs_attn_workspace_size", "vs_sparse_attn_fwd", "vs_dense_attn_fwd", "vs_read_device_status",
    "vs_selftest_wait_timeout", "vs_sparse_attn_fwd_static_scratch", "vs_attn_workspace_size_ld",
    "vs_attn_aggregate", "vs_attn_workspace_size_varlen", "vs_sparse_attn_fwd_varlen",
    "vs_dense_attn_fwd_varlen", "vs_block_select_workspace_size", "vs_block_select",
    "vs_block_attn_workspace_size", "vs_block_sparse_attn_fwd", "vs_selftest_exp",
    "vs_block_select_workspace_size_varlen", "vs_block_select_varlen",
    "vs_block_attn_workspace_size_varlen", "vs_block_sparse_attn_fwd_varlen",
    "vs_attn_aggregate_varlen", "vs_select_workspace_size_varlen", "vs_select_varlen",
)


class VsError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libvs.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libvs.so not built at {LIB_PATH}; run "
                              "`python -m sparse_attention_long_head_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, U64, D, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                ctypes.c_double, ctypes.c_float)
        Z = ctypes.c_size_t
        L.vs_status_string.argtypes = [I]
        L.vs_status_string.restype = ctypes.c_char_p
        L.vs_version.argtypes = []
        L.vs_version.restype = I
        L.vs_index_scores.argtypes = [P, P, I, I, I, I, I64, I64, P, P, I, P, P, P]
        L.vs_index_scores.restype = I
        L.vs_select_workspace_size.argtypes = [I, I]
        L.vs_select_workspace_size.restype = Z
        L.vs_select.argtypes = [P, I, I, I64, I, I, D, P, I64, P, P, Z, P]
        L.vs_select.restype = I
        L.vs_select_workspace_size_varlen.argtypes = [I, I, I]
        L.vs_select_workspace_size_varlen.restype = Z
        L.vs_select_varlen.argtypes = [P, I, I, P, I, I, I, P, I, D, P, I64, P, P, Z, P]
        L.vs_select_varlen.restype = I
        L.vs_attn_workspace_size.argtypes = [I, I, I, I]
        L.vs_attn_workspace_size.restype = Z
        L.vs_attn_workspace_size_ld.argtypes = [I, I, I, I, I64]
        L.vs_attn_workspace_size_ld.restype = Z
        L.vs_sparse_attn_fwd.argtypes = [P, P, P, I, I, I, I, I, I64, I64, F, I, P, I64, P, P, I64,
                                         P, P, P, P, Z, P]
        L.vs_sparse_attn_fwd.restype = I
        L.vs_dense_attn_fwd.argtypes = [P, P, P, I, I, I, I, I, I64, I64, F, P, P, P, Z, P]
        L.vs_dense_attn_fwd.restype = I
        L.vs_attn_aggregate.argtypes = [P, P, I, I, I, I, I, I64, I64, F, P, P, P, P, Z, P]
        L.vs_attn_aggregate.restype = I
        L.vs_attn_workspace_size_varlen.argtypes = [I, I, I, I, I64]
        L.vs_attn_workspace_size_varlen.restype = Z
        L.vs_sparse_attn_fwd_varlen.argtypes = [P, P, P, I, I, I, P, I, I, I, I, I64, I64, F, I, P,
                                                I64, P, P, I64, P, P, P, P, Z, P]
        L.vs_sparse_attn_fwd_varlen.restype = I
        L.vs_dense_attn_fwd_varlen.argtypes = [P, P, P, I, I, I, P, I, I, I, I, I64, I64, F, P, P,
                                               P, Z, P]
        L.vs_dense_attn_fwd_varlen.restype = I
        L.vs_block_select_workspace_size.argtypes = [I, I, I]
        L.vs_block_select_workspace_size.restype = Z
        L.vs_block_select.argtypes = [P, P, I, I, I, I, I, I64, I64, F, D, P, P, Z, P]
        L.vs_block_select.restype = I
        L.vs_block_attn_workspace_size.argtypes = [I, I]
        L.vs_block_attn_workspace_size.restype = Z
        L.vs_block_sparse_attn_fwd.argtypes = [P, P, P, I, I, I, I, I, I64, I64, F, P, P, P, P, Z,
                                               P]
        L.vs_block_sparse_attn_fwd.restype = I
        L.vs_block_select_workspace_size_varlen.argtypes = [I, I, I, I]
        L.vs_block_select_workspace_size_varlen.restype = Z
        L.vs_block_select_varlen.argtypes = [P, P, I, I, I, P, I, I, I, I, I64, I64, F, D, P, P, Z,
                                             P]
        L.vs_block_select_varlen.restype = I
        L.vs_block_attn_workspace_size_varlen.argtypes = [I, I, I]
        L.vs_block_attn_workspace_size_varlen.restype = Z
        L.vs_block_sparse_attn_fwd_varlen.argtypes = [P, P, P, I, I, I, P, I, I, I, I, I64, I64, F,
                                                      P, P, P, P, Z, P]
        L.vs_block_sparse_attn_fwd_varlen.restype = I
        L.vs_attn_aggregate_varlen.argtypes = [P, P, I, I, I, P, I, I, I, I, I64, I64, F, P, P,
                                               P, P, Z, P]
        L.vs_attn_aggregate_varlen.restype = I
        L.vs_read_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int)]
        L.vs_read_device_status.restype = I
        L.vs_selftest_wait_timeout.argtypes = [P, U64, P]
        L.vs_selftest_wait_timeout.restype = I
        L.vs_selftest_exp.argtypes = [P, P, I, P]
        L.vs_selftest_exp.restype = I
        L.vs_sparse_attn_fwd_static_scratch.argtypes = [P, P, P, I, I, I, I, I, I64, I64, F, I, P,
                                                        I64, P, P, I64, P, P, P, P]
        L.vs_sparse_attn_fwd_static_scratch.restype = I
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().vs_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != VS_OK:
        raise VsError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return VS_BF16
    if t.dtype == torch.float32:
        return VS_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------ ABI


def vs_version() -> int:
    return lib().vs_version()


def vs_select_workspace_size(H: int, N: int) -> int:
    return lib().vs_select_workspace_size(H, N)


def vs_attn_workspace_size(N: int, Hq: int, H_sel: int, d: int) -> int:
    return lib().vs_attn_workspace_size(N, Hq, H_sel, d)


def vs_attn_workspace_size_ld(N: int, Hq: int, H_sel: int, d: int, v_ld: int) -> int:
    return lib().vs_attn_workspace_size_ld(N, Hq, H_sel, d, v_ld)


def vs_attn_workspace_size_varlen(B: int, max_seqlen: int, H_sel: int, d: int, v_ld: int = 0) -> int:
    return int(lib().vs_attn_workspace_size_varlen(B, max_seqlen, H_sel, d, v_ld))


def vs_index_scores(K, V, W1, W2, logits_v, logits_s, stream=None):
    """K, V [N, Hkv, d] (bf16 or fp32, head stride = d); W1 [hidden, 2d], W2 [2, hidden]
    fp32; writes logits_v / logits_s fp32 [Hkv, N]."""
    N, Hkv, d = K.shape
    _check(lib().vs_index_scores(_ptr(K), _ptr(V), _dtype(K), N, Hkv, d, K.stride(0), K.stride(1),
                                 _ptr(W1), _ptr(W2), W1.shape[0], _ptr(logits_v), _ptr(logits_s),
                                 _stream(stream)), "vs_index_scores")


def vs_select(scores, mode, k_or_cap, tau, idx, count, ws, stream=None):
    """scores fp32 [H, ld >= N] (N = scores.shape[1]); idx int32 [H, ld_idx >= k_or_cap];
    count int32 [H]; ws from vs_select_workspace_size."""
    H, N = scores.shape
    _check(lib().vs_select(_ptr(scores), H, N, scores.stride(0), int(mode), int(k_or_cap),
                           float(tau), _ptr(idx), idx.stride(0), _ptr(count), _ptr(ws), ws.numel(),
                           _stream(stream)), "vs_select")


def vs_select_workspace_size_varlen(B: int, H: int, max_seqlen: int) -> int:
    return lib().vs_select_workspace_size_varlen(B, H, max_seqlen)


def vs_select_varlen(scores, cu_seqlens, max_seqlen, mode, caps, cap_max, tau, idx, count, ws,
                     stream=None):
    """scores fp32 [H, total_tokens] (contiguous rows); cu_seqlens int32 [B + 1] and caps int32
    [B] on the device; idx int32 [B * H, ld_idx >= cap_max]; count int32 [B * H]; ws from
    vs_select_workspace_size_varlen."""
    H, total = scores.shape
    B = cu_seqlens.numel() - 1
    assert scores.stride(1) == 1 and scores.stride(0) == total
    _check(lib().vs_select_varlen(_ptr(scores), total, B, _ptr(cu_seqlens), int(max_seqlen), H,
                                  int(mode), _ptr(caps), int(cap_max), float(tau), _ptr(idx),
                                  idx.stride(0), _ptr(count), _ptr(ws), ws.numel(),
                                  _stream(stream)), "vs_select_varlen")


def vs_sparse_attn_fwd(Q, K, V, v_idx, v_cnt, s_idx, s_cnt, O, lse, ws, softmax_scale=0.0,
                       stream=None):
    """Q [N, Hq, d], K/V [N, Hkv, d], O like Q; index rows [H_sel, ld]; lse fp32 [Hq, N] or None."""
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    _check(lib().vs_sparse_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _dtype(Q), N, Hq, Hkv, d,
                                    Q.stride(0), K.stride(0), float(softmax_scale), v_idx.shape[0],
                                    _ptr(v_idx), v_idx.stride(0), _ptr(v_cnt), _ptr(s_idx),
                                    s_idx.stride(0), _ptr(s_cnt), _ptr(O), _ptr(lse), _ptr(ws),
                                    ws.numel(), _stream(stream)), "vs_sparse_attn_fwd")


def vs_sparse_attn_fwd_static_scratch(Q, K, V, v_idx, v_cnt, s_idx, s_cnt, O, lse,
                                      softmax_scale=0.0, stream=None):
    """vs_sparse_attn_fwd for callers that cannot allocate: uses the library's 16 MiB static
    device scratch instead of a workspace (see include/vs_prefill.h for its limits)."""
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    _check(lib().vs_sparse_attn_fwd_static_scratch(
        _ptr(Q), _ptr(K), _ptr(V), _dtype(Q), N, Hq, Hkv, d, Q.stride(0), K.stride(0),
        float(softmax_scale), v_idx.shape[0], _ptr(v_idx), v_idx.stride(0), _ptr(v_cnt),
        _ptr(s_idx), s_idx.stride(0), _ptr(s_cnt), _ptr(O), _ptr(lse), _stream(stream)),
        "vs_sparse_attn_fwd_static_scratch")


def vs_dense_attn_fwd(Q, K, V, O, lse, ws, softmax_scale=0.0, stream=None):
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    _check(lib().vs_dense_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _dtype(Q), N, Hq, Hkv, d,
                                   Q.stride(0), K.stride(0), float(softmax_scale), _ptr(O),
                                   _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "vs_dense_attn_fwd")


def vs_attn_aggregate(Q, K, lse, A_v, A_s, ws, softmax_scale=0.0, stream=None):
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    _check(lib().vs_attn_aggregate(_ptr(Q), _ptr(K), _dtype(Q), N, Hq, Hkv, d, Q.stride(0),
                                   K.stride(0), float(softmax_scale), _ptr(lse), _ptr(A_v),
                                   _ptr(A_s), _ptr(ws), ws.numel(), _stream(stream)),
           "vs_attn_aggregate")


def vs_sparse_attn_fwd_varlen(Q, K, V, cu_seqlens, max_seqlen, v_idx, v_cnt, s_idx, s_cnt, O, lse,
                              ws, softmax_scale=0.0, stream=None):
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    H_sel = v_idx.shape[0] // B
    _check(lib().vs_sparse_attn_fwd_varlen(
        _ptr(Q), _ptr(K), _ptr(V), _dtype(Q), T, B, _ptr(cu_seqlens), int(max_seqlen), Hq, Hkv, d,
        Q.stride(0), K.stride(0), float(softmax_scale), H_sel, _ptr(v_idx), v_idx.stride(0),
        _ptr(v_cnt), _ptr(s_idx), s_idx.stride(0), _ptr(s_cnt), _ptr(O), _ptr(lse), _ptr(ws),
        ws.numel(), _stream(stream)), "vs_sparse_attn_fwd_varlen")


def vs_dense_attn_fwd_varlen(Q, K, V, cu_seqlens, max_seqlen, O, lse, ws, softmax_scale=0.0,
                             stream=None):
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    _check(lib().vs_dense_attn_fwd_varlen(
        _ptr(Q), _ptr(K), _ptr(V), _dtype(Q), T, B, _ptr(cu_seqlens), int(max_seqlen), Hq, Hkv, d,
        Q.stride(0), K.stride(0), float(softmax_scale), _ptr(O), _ptr(lse), _ptr(ws), ws.numel(),
        _stream(stream)), "vs_dense_attn_fwd_varlen")


def vs_attn_aggregate_varlen(Q, K, cu_seqlens, max_seqlen, lse, A_v, A_s, ws, softmax_scale=0.0,
                             stream=None):
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    _check(lib().vs_attn_aggregate_varlen(
        _ptr(Q), _ptr(K), _dtype(Q), T, B, _ptr(cu_seqlens), int(max_seqlen), Hq, Hkv, d,
        Q.stride(0), K.stride(0), float(softmax_scale), _ptr(lse), _ptr(A_v), _ptr(A_s), _ptr(ws),
        ws.numel(), _stream(stream)), "vs_attn_aggregate_varlen")


def aggregate_varlen(Q, K, V, cu_seqlens, max_seqlen, ws=None, stream=None):
    """Per-sequence column / diagonal sums of a packed batch, fp32 [Hq, total]
    each: the batched dense forward for the row LSE, then the aggregation."""
    T, Hq, _ = Q.shape
    B = cu_seqlens.numel() - 1
    ws = ws if ws is not None else workspace(256, Q.device)
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, T), dtype=torch.float32, device=Q.device)
    wsd = workspace(vs_attn_workspace_size_varlen(B, max_seqlen, 1, Q.shape[2]), Q.device)
    vs_dense_attn_fwd_varlen(Q, K, V, cu_seqlens, max_seqlen, O, lse, wsd, stream=stream)
    A_v = torch.empty((Hq, T), dtype=torch.float32, device=Q.device)
    A_s = torch.empty((Hq, T), dtype=torch.float32, device=Q.device)
    vs_attn_aggregate_varlen(Q, K, cu_seqlens, max_seqlen, lse, A_v, A_s, ws, stream=stream)
    return A_v, A_s


def vs_block_select_workspace_size(N: int, Hkv: int, d: int) -> int:
    return int(lib().vs_block_select_workspace_size(N, Hkv, d))


def vs_block_attn_workspace_size(N: int, Hq: int) -> int:
    return int(lib().vs_block_attn_workspace_size(N, Hq))


def vs_block_select(Q, K, alpha, mask, ws, softmax_scale=0.0, stream=None):
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    _check(lib().vs_block_select(_ptr(Q), _ptr(K), _dtype(Q), N, Hq, Hkv, d, Q.stride(0),
                                 K.stride(0), float(softmax_scale), float(alpha), _ptr(mask),
                                 _ptr(ws), ws.numel(), _stream(stream)), "vs_block_select")


def vs_block_sparse_attn_fwd(Q, K, V, mask, O, lse, ws, softmax_scale=0.0, stream=None):
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    _check(lib().vs_block_sparse_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _dtype(Q), N, Hq, Hkv, d,
                                          Q.stride(0), K.stride(0), float(softmax_scale),
                                          _ptr(mask), _ptr(O), _ptr(lse), _ptr(ws), ws.numel(),
                                          _stream(stream)), "vs_block_sparse_attn_fwd")


def vs_block_select_workspace_size_varlen(B: int, max_seqlen: int, Hkv: int, d: int) -> int:
    return int(lib().vs_block_select_workspace_size_varlen(B, max_seqlen, Hkv, d))


def vs_block_attn_workspace_size_varlen(B: int, max_seqlen: int, Hq: int) -> int:
    return int(lib().vs_block_attn_workspace_size_varlen(B, max_seqlen, Hq))


def vs_block_select_varlen(Q, K, cu_seqlens, max_seqlen, alpha, mask, ws, softmax_scale=0.0,
                           stream=None):
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    _check(lib().vs_block_select_varlen(
        _ptr(Q), _ptr(K), _dtype(Q), T, B, _ptr(cu_seqlens), int(max_seqlen), Hq, Hkv, d,
        Q.stride(0), K.stride(0), float(softmax_scale), float(alpha), _ptr(mask), _ptr(ws),
        ws.numel(), _stream(stream)), "vs_block_select_varlen")


def vs_block_sparse_attn_fwd_varlen(Q, K, V, cu_seqlens, max_seqlen, mask, O, lse, ws,
                                    softmax_scale=0.0, stream=None):
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    _check(lib().vs_block_sparse_attn_fwd_varlen(
        _ptr(Q), _ptr(K), _ptr(V), _dtype(Q), T, B, _ptr(cu_seqlens), int(max_seqlen), Hq, Hkv, d,
        Q.stride(0), K.stride(0), float(softmax_scale), _ptr(mask), _ptr(O), _ptr(lse), _ptr(ws),
        ws.numel(), _stream(stream)), "vs_block_sparse_attn_fwd_varlen")


def block_prefill_varlen(Q, K, V, cu_seqlens, max_seqlen, alpha, stream=None):
    """Batched block prefill: discovery then block-sparse attention per
    sequence; returns (O, lse [Hq, total], mask [B, Hq, T, W])."""
    total, Hq, d = Q.shape
    B = cu_seqlens.numel() - 1
    T = (int(max_seqlen) + 127) // 128
    mask = torch.empty((B, Hq, T, (T + 31) // 32), dtype=torch.int32, device=Q.device)
    ws = workspace(max(vs_block_select_workspace_size_varlen(B, max_seqlen, K.shape[1], d),
                       vs_block_attn_workspace_size_varlen(B, max_seqlen, Hq)), Q.device)
    vs_block_select_varlen(Q, K, cu_seqlens, max_seqlen, alpha, mask, ws, stream=stream)
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, total), dtype=torch.float32, device=Q.device)
    vs_block_sparse_attn_fwd_varlen(Q, K, V, cu_seqlens, max_seqlen, mask, O, lse, ws,
                                    stream=stream)
    return O, lse, mask


def block_prefill(Q, K, V, alpha, stream=None):
    """FlashPrefill-style pattern discovery then block-sparse attention:
    returns (O, lse, mask)."""
    N, Hq, d = Q.shape
    T = (N + 127) // 128
    mask = torch.empty((Hq, T, (T + 31) // 32), dtype=torch.int32, device=Q.device)
    ws = workspace(max(vs_block_select_workspace_size(N, K.shape[1], d),
                       vs_block_attn_workspace_size(N, Hq)), Q.device)
    vs_block_select(Q, K, alpha, mask, ws, stream=stream)
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, N), dtype=torch.float32, device=Q.device)
    vs_block_sparse_attn_fwd(Q, K, V, mask, O, lse, ws, stream=stream)
    return O, lse, mask


def vs_read_device_status(ws, stream=None) -> tuple[int, int]:
    """(status code, flags) of the last call that used ``ws`` (synchronises the stream)."""
    flags = ctypes.c_int(0)
    rc = lib().vs_read_device_status(_ptr(ws), _stream(stream), ctypes.byref(flags))
    return rc, flags.value


def vs_selftest_wait_timeout(ws, limit_ns: int, stream=None):
    _check(lib().vs_selftest_wait_timeout(_ptr(ws), int(limit_ns), _stream(stream)),
           "vs_selftest_wait_timeout")


def vs_selftest_exp(x, y, stream=None):
    _check(lib().vs_selftest_exp(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "vs_selftest_exp")


# ------------------------------------------------------- allocation helpers


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned uint8 device buffer (torch's allocator aligns to 512)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def select(scores, mode, k_or_cap, tau=1.0, ws=None, stream=None):
    """Allocates outputs and runs vs_select -> (idx [H, k_or_cap], count [H])."""
    H, N = scores.shape
    idx = torch.empty((H, k_or_cap), dtype=torch.int32, device=scores.device)
    cnt = torch.empty(H, dtype=torch.int32, device=scores.device)
    ws = workspace(vs_select_workspace_size(H, N), scores.device) if ws is None else ws
    vs_select(scores, mode, k_or_cap, tau, idx, cnt, ws, stream)
    return idx, cnt


def select_varlen(scores, cu_seqlens, max_seqlen, mode, caps, cap_max, tau=1.0, ws=None,
                  stream=None):
    """Allocates outputs and runs vs_select_varlen -> (idx [B * H, cap_max] filled with -1 past
    each row's cap, count [B * H])."""
    H = scores.shape[0]
    B = cu_seqlens.numel() - 1
    idx = torch.full((B * H, cap_max), -1, dtype=torch.int32, device=scores.device)
    cnt = torch.empty(B * H, dtype=torch.int32, device=scores.device)
    if ws is None:
        ws = workspace(vs_select_workspace_size_varlen(B, H, max_seqlen), scores.device)
    vs_select_varlen(scores, cu_seqlens, max_seqlen, mode, caps, cap_max, tau, idx, cnt, ws, stream)
    return idx, cnt


def sparse_attention(Q, K, V, v_idx, v_cnt, s_idx, s_cnt, ws=None, with_lse=True, stream=None):
    N, Hq, d = Q.shape
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, N), dtype=torch.float32, device=Q.device) if with_lse else None
    if ws is None:
        ws = workspace(vs_attn_workspace_size_ld(N, Hq, v_idx.shape[0], d, v_idx.stride(0)),
                       Q.device)
    vs_sparse_attn_fwd(Q, K, V, v_idx, v_cnt, s_idx, s_cnt, O, lse, ws, stream=stream)
    return O, lse


def dense_attention(Q, K, V, ws=None, with_lse=True, stream=None):
    N, Hq, d = Q.shape
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, N), dtype=torch.float32, device=Q.device) if with_lse else None
    ws = workspace(256, Q.device) if ws is None else ws
    vs_dense_attn_fwd(Q, K, V, O, lse, ws, stream=stream)
    return O, lse


def aggregate(Q, K, V=None, lse=None, ws=None, stream=None):
    """Ground-truth column / diagonal sums (A_v, A_s), fp32 [Hq, N] each.

    Runs the dense causal forward first for the row LSE unless ``lse`` is
    given (then V is not needed)."""
    N, Hq, _ = Q.shape
    ws = ws if ws is not None else workspace(256, Q.device)
    if lse is None:
        if V is None:
            raise ValueError("V is needed to compute the LSE")
        O = torch.empty_like(Q)
        lse = torch.empty((Hq, N), dtype=torch.float32, device=Q.device)
        vs_dense_attn_fwd(Q, K, V, O, lse, ws, stream=stream)
        del O
    A_v = torch.empty((Hq, N), dtype=torch.float32, device=Q.device)
    A_s = torch.empty((Hq, N), dtype=torch.float32, device=Q.device)
    vs_attn_aggregate(Q, K, lse, A_v, A_s, ws, stream=stream)
    return A_v, A_s

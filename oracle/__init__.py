"""fp64 CPU oracle for vertical-slash sparse prefill (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path never calls it.

The arithmetic lives in ``vs_oracle.c`` (plain fp64 C, OpenMP over
independent rows only); this module loads it with ctypes and marshals numpy
arrays.  See ``vs_oracle.c`` for the definitions and the page passages each
function follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vs_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

TOPK = 0
THRESHOLD = 1
MAXFRAC = 2


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.or_select.argtypes = [P, i32, i32, i32, dbl, P, P, P]
        lib.or_select.restype = i32
        attn_common = [P, P, P, i32, i32, i32, i32, i32, i64, i64, dbl, i32, P, i64, P, P, i64, P]
        lib.or_attn_rows.argtypes = attn_common + [i32, i32, P, i32, P, P]
        lib.or_attn_rows.restype = None
        lib.or_attn_mask.argtypes = attn_common + [i32, P, P, P]
        lib.or_attn_mask.restype = None
        lib.or_count_pairs.argtypes = [i32, P, i32, P, i32]
        lib.or_count_pairs.restype = i64
        lib.or_index_scores.argtypes = [P, P, i32, i32, i32, i32, i64, i64, P, P, i32, P, i32, P, P]
        lib.or_index_scores.restype = None
        lib.or_aggregate.argtypes = [P, P, i32, i32, i32, i32, i32, i64, i64, dbl, P, i32, i64, i64,
                                     P, P]
        lib.or_aggregate.restype = None
        lib.or_block_select.argtypes = [P, P, i32, i32, i32, i32, i32, i64, i64, dbl, dbl, P, i32,
                                        P, P]
        lib.or_block_select.restype = None
        lib.or_attn_block_rows.argtypes = [P, P, P, i32, i32, i32, i32, i32, i64, i64, dbl, P,
                                           i32, P, i32, P, P]
        lib.or_attn_block_rows.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def select(scores: np.ndarray, mode: int, k_or_cap: int, tau: float = 1.0):
    """One head: returns (idx int32 [k_or_cap] ascending padded -1, count, margin)."""
    s = np.ascontiguousarray(scores, dtype=np.float32)
    idx = np.empty(k_or_cap, np.int32)
    cnt = np.zeros(1, np.int32)
    margin = np.zeros(1, np.float64)
    rc = _load().or_select(_ptr(s), s.size, mode, k_or_cap, float(tau), _ptr(idx), _ptr(cnt),
                           _ptr(margin))
    if rc != 0:
        raise ValueError("invalid select arguments")
    return idx, int(cnt[0]), float(margin[0])


def select_heads(scores: np.ndarray, mode: int, k_or_cap: int, tau: float = 1.0):
    H = scores.shape[0]
    idx = np.empty((H, k_or_cap), np.int32)
    cnt = np.empty(H, np.int32)
    margins = np.empty(H, np.float64)
    for h in range(H):
        idx[h], cnt[h], margins[h] = select(scores[h], mode, k_or_cap, tau)
    return idx, cnt, margins


class _Attn:
    """Marshals the common attention arguments (arrays kept alive here)."""

    def __init__(self, Q, K, V, Hq, Hkv, d, scale, v_idx, v_cnt, s_idx, s_cnt, dense):
        if Q.dtype == np.uint16:
            self.dtype = 0
        elif Q.dtype == np.float32:
            self.dtype = 1
        else:
            raise TypeError("Q/K/V must be bf16 bits (uint16) or float32")
        self.Q = np.ascontiguousarray(Q)
        self.K = np.ascontiguousarray(K)
        self.V = np.ascontiguousarray(V)
        self.N = Q.shape[0]
        self.Hq, self.Hkv, self.d = Hq, Hkv, d
        self.scale = float(scale) if scale else 1.0 / np.sqrt(d)
        if dense or v_idx is None:
            v_idx = np.zeros((1, 1), np.int32)
            v_cnt = np.zeros(1, np.int32)
            s_idx = np.zeros((1, 1), np.int32)
            s_cnt = np.zeros(1, np.int32)
        self.v_idx = np.ascontiguousarray(v_idx, np.int32)
        self.s_idx = np.ascontiguousarray(s_idx, np.int32)
        self.v_cnt = np.ascontiguousarray(v_cnt, np.int32)
        self.s_cnt = np.ascontiguousarray(s_cnt, np.int32)
        self.H_sel = self.v_idx.shape[0]
        self.dense = 1 if dense else 0

    def common(self):
        return [_ptr(self.Q), _ptr(self.K), _ptr(self.V), self.dtype, self.N, self.Hq, self.Hkv,
                self.d, self.Hq * self.d, self.Hkv * self.d, self.scale, self.H_sel,
                _ptr(self.v_idx), self.v_idx.shape[1], _ptr(self.v_cnt), _ptr(self.s_idx),
                self.s_idx.shape[1], _ptr(self.s_cnt)]


def attn_rows(Q, K, V, h, rows, v_idx=None, v_cnt=None, s_idx=None, s_cnt=None, scale=0.0,
              dense=False):
    """Row form for query head h on the given rows -> (O [n,d] f64, LSE [n] f64).

    Q [N,Hq,d], K/V [N,Hkv,d] as bf16 bits (uint16) or float32; index arrays
    [H_sel, ld] ascending with counts [H_sel]."""
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    a = _Attn(Q, K, V, Hq, Hkv, d, scale, v_idx, v_cnt, s_idx, s_cnt, dense)
    rows = np.ascontiguousarray(rows, np.int64)
    O = np.empty((rows.size, d), np.float64)
    lse = np.empty(rows.size, np.float64)
    _load().or_attn_rows(*a.common(), a.dense, int(h), _ptr(rows), rows.size, _ptr(O), _ptr(lse))
    return O, lse


def attn_mask(Q, K, V, h, v_idx, v_cnt, s_idx, s_cnt, scale=0.0, return_mask=False):
    """Explicit-mask form for query head h (all rows; small N)."""
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    a = _Attn(Q, K, V, Hq, Hkv, d, scale, v_idx, v_cnt, s_idx, s_cnt, False)
    O = np.empty((N, d), np.float64)
    lse = np.empty(N, np.float64)
    M = np.empty((N, N), np.uint8) if return_mask else None
    _load().or_attn_mask(*a.common(), int(h), _ptr(O), _ptr(lse),
                         _ptr(M) if M is not None else None)
    return (O, lse, M) if return_mask else (O, lse)


def count_pairs(N: int, v_list, s_list) -> int:
    v = np.ascontiguousarray(v_list, np.int32)
    s = np.ascontiguousarray(s_list, np.int32)
    return int(_load().or_count_pairs(N, _ptr(v), v.size, _ptr(s), s.size))


def index_scores(K, V, W1, W2, toks=None):
    """Indexer logits for the given tokens -> (lv [Hkv,n], ls [Hkv,n]) f64."""
    N, Hkv, d = K.shape
    dtype = 0 if K.dtype == np.uint16 else 1
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    W1 = np.ascontiguousarray(W1, np.float32)
    W2 = np.ascontiguousarray(W2, np.float32)
    toks = np.arange(N, dtype=np.int64) if toks is None else np.ascontiguousarray(toks, np.int64)
    lv = np.empty((Hkv, toks.size), np.float64)
    ls = np.empty((Hkv, toks.size), np.float64)
    _load().or_index_scores(_ptr(K), _ptr(V), dtype, N, Hkv, d, Hkv * d, d, _ptr(W1), _ptr(W2),
                            W1.shape[0], _ptr(toks), toks.size, _ptr(lv), _ptr(ls))
    return lv, ls


def aggregate(Q, K, heads=None, rows=None, scale=0.0):
    """Ground-truth column / diagonal sums of the full causal softmax weights.

    Q [N, Hq, d], K [N, Hkv, d] as bf16 bits (uint16) or float32.  Returns
    (A_v, A_s), each float64 [len(heads), N].  `rows` = (lo, hi) restricts the
    contributing query rows (default all); with hi = N, entries j >= lo of A_v
    and o >= lo of A_s are exact."""
    if Q.dtype == np.uint16:
        dtype = 0
    elif Q.dtype == np.float32:
        dtype = 1
    else:
        raise TypeError("Q/K must be bf16 bits (uint16) or float32")
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    Q = np.ascontiguousarray(Q)
    K = np.ascontiguousarray(K)
    heads = np.arange(Hq, dtype=np.int32) if heads is None else np.ascontiguousarray(heads, np.int32)
    lo, hi = (0, N) if rows is None else rows
    Av = np.empty((heads.size, N), np.float64)
    As = np.empty((heads.size, N), np.float64)
    _load().or_aggregate(_ptr(Q), _ptr(K), dtype, N, Hq, Hkv, d, Hq * d, Hkv * d, float(scale),
                         _ptr(heads), heads.size, int(lo), int(hi), _ptr(Av), _ptr(As))
    return Av, As


def block_select(Q, K, alpha, heads=None, scale=0.0):
    """FlashPrefill-style kept key blocks per query block (see vs_oracle.c).

    Returns (mask uint32 [len(heads), T, W], margin float64 [len(heads)])."""
    dtype = 0 if Q.dtype == np.uint16 else 1
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    Q = np.ascontiguousarray(Q)
    K = np.ascontiguousarray(K)
    heads = np.arange(Hq, dtype=np.int32) if heads is None else np.ascontiguousarray(heads, np.int32)
    T = (N + 127) // 128
    W = (T + 31) // 32
    mask = np.zeros((heads.size, T, W), np.uint32)
    margin = np.zeros(heads.size, np.float64)
    _load().or_block_select(_ptr(Q), _ptr(K), dtype, N, Hq, Hkv, d, Hq * d, Hkv * d, float(scale),
                            float(alpha), _ptr(heads), heads.size, _ptr(mask), _ptr(margin))
    return mask, margin


def attn_block_rows(Q, K, V, h, rows, mask, scale=0.0):
    """Block-sparse causal attention for head h at the given rows; `mask` is
    [Hq, T, W] as from block_select over all heads.  Returns (O [n, d], lse [n])."""
    dtype = 0 if Q.dtype == np.uint16 else 1
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    rows = np.ascontiguousarray(rows, np.int64)
    mask = np.ascontiguousarray(mask, np.uint32)
    O = np.empty((rows.size, d), np.float64)
    lse = np.empty(rows.size, np.float64)
    _load().or_attn_block_rows(_ptr(np.ascontiguousarray(Q)), _ptr(np.ascontiguousarray(K)),
                               _ptr(np.ascontiguousarray(V)), dtype, N, Hq, Hkv, d, Hq * d, Hkv * d,
                               float(scale), _ptr(mask), int(h), _ptr(rows), rows.size, _ptr(O),
                               _ptr(lse))
    return O, lse

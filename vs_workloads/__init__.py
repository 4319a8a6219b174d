"""Seeded synthetic inputs for vertical-slash sparse prefill.

This module only draws numbers: Q/K/V activations with rotary position
embedding applied, per-head vertical/slash score vectors, and indexer
weights.  It contains none of the method's arithmetic (no selection, no
attention, no indexer), so both the CUDA path and the fp64 oracle can take
their inputs from here.

Workloads follow the shapes of the VSPrefill summary pages (Llama-3.1-8B
style attention: 32 query heads, 8 KV heads, head dim 128, 8K-256K prefill;
"VSPrefill: Vertical-Slash Sparse Attention ..." Technical Summary,
section 4 Experimental Results).  The pages evaluate on LongBench / RULER,
which are not available here; these synthetic inputs stand in for them.

Recipe (all draws from numpy ``default_rng``):
  * Q, K, V ~ N(0, 1) drawn in float64, RoPE (rotate-half pairing
    (x_m, x_{m+d/2}), theta_m = base^(-2m/d), positions 0..N-1) applied to
    Q and K in float64, then rounded once to bf16 (round-to-nearest-even).
  * Score vectors are logits l = log(A) rounded to fp32, A from the
    generators below; per-head seed = seed*1000 + head.
  * Indexer weights W1[hidden][2d], W2[2][hidden] ~ N(0, 0.02) in fp32.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

# --------------------------------------------------------------------------
# bf16 helpers (bit patterns stored as uint16)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 directly to bf16 (round-to-nearest-even) -> uint16 bits.

    Rounds the 52-bit mantissa to bf16's 7 explicit bits in one step, so
    there is no double rounding through fp32.  Inputs are finite and far
    from the bf16 overflow / subnormal range (Gaussian draws).
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    b = (b + np.uint64(0x0FFFFFFFFFFF) + lsb) & ~np.uint64(0x1FFFFFFFFFFF)
    f32 = b.view(np.float64).astype(np.float32)  # exact: value has <= 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# Q / K / V


def _rope_tables(pos0: int, n: int, d: int, base: float):
    half = d // 2
    m = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * m / d)
    ang = np.arange(pos0, pos0 + n, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def _draw_chunk(seed: int, tensor_id: int, chunk: int, pos0: int, n: int, H: int, d: int,
                rope_base: float | None) -> np.ndarray:
    rng = np.random.default_rng([seed, tensor_id, chunk])
    x = rng.standard_normal((n, H, d))
    if rope_base is not None:
        c, s = _rope_tables(pos0, n, d, rope_base)
        c = c[:, None, :]
        s = s[:, None, :]
        half = d // 2
        x1 = x[..., :half].copy()
        x2 = x[..., half:].copy()
        x[..., :half] = x1 * c - x2 * s
        x[..., half:] = x2 * c + x1 * s
    return f64_to_bf16_bits(x)


_CHUNK = 4096


def gen_tensor_bf16(seed: int, tensor_id: int, N: int, H: int, d: int,
                    rope_base: float | None, threads: int | None = None) -> np.ndarray:
    """[N, H, d] bf16 bits; deterministic in (seed, tensor_id) and chunked so
    that any N is generated in bounded host memory."""
    out = np.empty((N, H, d), dtype=np.uint16)
    nchunks = (N + _CHUNK - 1) // _CHUNK

    def work(c):
        p0 = c * _CHUNK
        n = min(_CHUNK, N - p0)
        out[p0:p0 + n] = _draw_chunk(seed, tensor_id, c, p0, n, H, d, rope_base)

    threads = threads or min(16, os.cpu_count() or 1)
    if nchunks == 1 or threads == 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def gen_qkv(seed: int, N: int, Hq: int, Hkv: int, d: int, rope_base: float):
    """Q [N,Hq,d], K [N,Hkv,d], V [N,Hkv,d] as bf16 bit arrays."""
    Q = gen_tensor_bf16(seed, 0, N, Hq, d, rope_base)
    K = gen_tensor_bf16(seed, 1, N, Hkv, d, rope_base)
    V = gen_tensor_bf16(seed, 2, N, Hkv, d, None)
    return Q, K, V


def gen_qkv_f32(seed: int, N: int, Hq: int, Hkv: int, d: int, rope_base: float):
    """fp32 variant for the fp32 attention path: the same draws, not rounded."""
    outs = []
    for tid, H, rb in ((0, Hq, rope_base), (1, Hkv, rope_base), (2, Hkv, None)):
        parts = []
        for c in range((N + _CHUNK - 1) // _CHUNK):
            p0 = c * _CHUNK
            n = min(_CHUNK, N - p0)
            rng = np.random.default_rng([seed, tid, c])
            x = rng.standard_normal((n, H, d))
            if rb is not None:
                cs, sn = _rope_tables(p0, n, d, rb)
                cs = cs[:, None, :]
                sn = sn[:, None, :]
                half = d // 2
                x1 = x[..., :half].copy()
                x2 = x[..., half:].copy()
                x[..., :half] = x1 * cs - x2 * sn
                x[..., half:] = x2 * cs + x1 * sn
            parts.append(x.astype(np.float32))
        outs.append(np.concatenate(parts, axis=0))
    return tuple(outs)


# --------------------------------------------------------------------------
# score generators (values A; the selection consumes logits log(A) in fp32)


def _lognormal(rng, n):
    return np.exp(rng.standard_normal(n))


def scores_base(N: int, seed: int):
    """Vertical A_v = LN(0,1) with columns 0-3 x100; slash
    A_s[o] = exp(-o/64) + 0.1*LN(0,1) with offsets 0-15 x100."""
    rng = np.random.default_rng(seed)
    av = _lognormal(rng, N)
    av[:4] *= 100.0
    o = np.arange(N, dtype=np.float64)
    a_s = np.exp(-o / 64.0) + 0.1 * _lognormal(rng, N)
    a_s[:16] *= 100.0
    return av, a_s


def scores_local(N: int, seed: int):
    """'Local' head: few verticals (1e-4*LN floor, columns 0-3 = 100*LN),
    sharply decaying slashes A_s[o] = exp(-o/16) + 1e-6*LN."""
    rng = np.random.default_rng(seed)
    av = 1e-4 * _lognormal(rng, N)
    av[:4] = 100.0 * _lognormal(rng, 4)
    o = np.arange(N, dtype=np.float64)
    a_s = np.exp(-o / 16.0) + 1e-6 * _lognormal(rng, N)
    return av, a_s


def scores_global(N: int, seed: int, structured_slash: bool = False):
    """'Global' head: heavy-tailed verticals A_v ~ Pareto(alpha=1.2, x_m=1);
    slashes from the base generator (or the local one when
    ``structured_slash``)."""
    rng = np.random.default_rng(seed)
    av = rng.pareto(1.2, N) + 1.0
    if structured_slash:
        _, a_s = scores_local(N, seed + 7)
    else:
        _, a_s = scores_base(N, seed + 7)
    return av, a_s


def to_logits(a: np.ndarray) -> np.ndarray:
    with np.errstate(divide="ignore"):
        return np.log(a).astype(np.float32)


# --------------------------------------------------------------------------
# workload registry


@dataclass
class Workload:
    name: str
    N: int
    Hq: int
    Hkv: int
    d: int
    rope_base: float
    seed: int
    select_mode: str            # "topk" | "threshold" | "maxfrac"
    k_v: int                    # top-k budget or cap
    k_s: int
    tau_v: float = 1.0
    tau_s: float = 1.0
    heads: str = "base"         # "base" | "local_global" | "local_global_S"
    indexer: bool = False
    hidden: int = 256
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def select_mode_id(self) -> int:
        """The rule's number in the C ABI and the oracle (0 top-k, 1 threshold, 2 max-based)."""
        return {"topk": 0, "threshold": 1, "maxfrac": 2}[self.select_mode]

    @property
    def H_sel(self) -> int:
        return self.Hkv if self.indexer else self.Hq

    def head_scores(self, h: int):
        """(logit_v, logit_s) fp32 [N] for index-set head h (non-indexer)."""
        s = self.seed * 1000 + h
        if self.heads == "base":
            av, a_s = scores_base(self.N, s)
        else:
            local = h < self.Hq // 2
            if local:
                av, a_s = scores_local(self.N, s)
            else:
                av, a_s = scores_global(self.N, s, structured_slash=self.heads.endswith("_S"))
        return to_logits(av), to_logits(a_s)

    def all_scores(self):
        lv = np.empty((self.H_sel, self.N), np.float32)
        ls = np.empty((self.H_sel, self.N), np.float32)
        for h in range(self.H_sel):
            lv[h], ls[h] = self.head_scores(h)
        return lv, ls

    def qkv(self):
        return gen_qkv(self.seed, self.N, self.Hq, self.Hkv, self.d, self.rope_base)

    def indexer_weights(self):
        rng = np.random.default_rng([self.seed, 99])
        W1 = (0.02 * rng.standard_normal((self.hidden, 2 * self.d))).astype(np.float32)
        W2 = (0.02 * rng.standard_normal((2, self.hidden))).astype(np.float32)
        return W1, W2


WORKLOADS = {
    "tiny_1k": Workload("tiny_1k", 1024, 1, 1, 64, 10000.0, 11, "topk", 32, 32,
                        description="1 head, N=1024, d=64, top-k 32/32"),
    "llama_8k": Workload("llama_8k", 8192, 32, 8, 128, 500000.0, 12, "topk", 1024, 2048,
                         description="32q/8kv, d=128, N=8192, top-k 1024/2048"),
    "llama_32k": Workload("llama_32k", 32768, 32, 8, 128, 500000.0, 13, "threshold", 4096, 4096,
                          tau_v=0.90, tau_s=0.95,
                          description="32q/8kv, d=128, N=32768, threshold 0.90/0.95 cap 4096"),
    "llama_128k": Workload("llama_128k", 131072, 32, 8, 128, 500000.0, 14, "threshold", 8192, 8192,
                           tau_v=0.95, tau_s=0.95, heads="local_global",
                           description="32q/8kv, d=128, N=131072, 16 local + 16 global heads, "
                                       "threshold 0.95 cap 8192"),
    "llama_128k_S": Workload("llama_128k_S", 131072, 32, 8, 128, 500000.0, 14, "threshold", 8192,
                             8192, tau_v=0.95, tau_s=0.95, heads="local_global_S",
                             description="variant of llama_128k whose global heads draw "
                                         "structured (local) slash scores"),
    "llama_128k_maxfrac": Workload("llama_128k_maxfrac", 131072, 32, 8, 128, 500000.0, 14,
                                   "maxfrac", 8192, 8192, tau_v=1e-3, tau_s=1e-3,
                                   heads="local_global",
                                   description="llama_128k's inputs with FlashPrefill's max-based "
                                               "rule: keep mass >= 1e-3 x the largest, cap 8192"),
    "llama_256k_indexer": Workload("llama_256k_indexer", 262144, 32, 8, 128, 500000.0, 15,
                                   "threshold", 16384, 16384, tau_v=0.95, tau_s=0.95, indexer=True,
                                   description="32q/8kv, d=128, N=262144, scores from the "
                                               "2d->256->2 indexer, threshold 0.95 cap 16384"),
}


def small_variant(w: Workload, N: int, Hq: int | None = None, Hkv: int | None = None) -> Workload:
    """Same generators and selection rule at a smaller N (caps scaled)."""
    scale = N / w.N
    Hq = Hq or w.Hq
    Hkv = Hkv or w.Hkv
    return Workload(w.name + f"@{N}", N, Hq, Hkv, w.d, w.rope_base, w.seed, w.select_mode,
                    max(1, min(N, int(math.ceil(w.k_v * scale)))),
                    max(1, min(N, int(math.ceil(w.k_s * scale)))), w.tau_v, w.tau_s, w.heads,
                    w.indexer, w.hidden, w.description + f" (scaled to N={N})")


@dataclass
class BatchWorkload:
    """A batch of independent sequences packed along the token axis
    (variable-length batched prefill).  Sequence b draws its Q/K/V from seed
    seed * 100 + b and its scores from the base generator, seed
    (seed * 100 + b) * 1000 + head; selection per sequence with caps of
    cap_frac x its length (at least 1)."""
    name: str
    lengths: tuple
    Hq: int
    Hkv: int
    d: int
    rope_base: float
    seed: int
    select_mode: str
    cap_frac: float
    tau_v: float = 1.0
    tau_s: float = 1.0
    description: str = ""

    @property
    def select_mode_id(self) -> int:
        return {"topk": 0, "threshold": 1, "maxfrac": 2}[self.select_mode]

    @property
    def H_sel(self) -> int:
        return self.Hq

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lengths)]).astype(np.int32)

    def cap(self, n: int) -> int:
        return max(1, min(n, int(math.ceil(self.cap_frac * n))))

    def qkv(self):
        parts = [gen_qkv(self.seed * 100 + b, n, self.Hq, self.Hkv, self.d, self.rope_base)
                 for b, n in enumerate(self.lengths)]
        return tuple(np.concatenate([p[t] for p in parts]) for t in range(3))

    def scores(self, b: int):
        """(logit_v, logit_s) fp32 [H_sel, n] of sequence b."""
        n = self.lengths[b]
        lv = np.empty((self.H_sel, n), np.float32)
        ls = np.empty((self.H_sel, n), np.float32)
        for h in range(self.H_sel):
            av, a_s = scores_base(n, (self.seed * 100 + b) * 1000 + h)
            lv[h], ls[h] = to_logits(av), to_logits(a_s)
        return lv, ls


BATCH_WORKLOADS = {
    "llama_varlen_mix": BatchWorkload(
        "llama_varlen_mix",
        (32768, 24576, 16384, 16384, 12288, 8192, 8192, 4096, 4096, 2048, 2048, 1024, 1024, 512,
         512, 256, 300),
        32, 8, 128, 500000.0, 16, "threshold", 0.125, tau_v=0.90, tau_s=0.95,
        description="17 sequences of 256-32768 tokens (134,700 in all), 32q/8kv, d=128, "
                    "threshold 0.90/0.95, caps 1/8 of each length"),
}


def plant_block_structure(Qb: np.ndarray, Kb: np.ndarray, seed: int, sinks: int = 3,
                          strength: float = 5.8, local: float = 2.9, period: float = 1024.0,
                          chunk: int = 8192):
    """Block-level attention structure on top of bf16 Q/K bits (returns new
    bits): per KV head a random unit direction u is added to every query of
    its group (x strength) and to the keys of block 0 and `sinks` random
    blocks (x strength), so those blocks act as sinks (a logit bump of about
    strength^2 / sqrt(d)); and slow rotations in four further pairs of
    directions, local * sum_m (cos(w_m t) e_2m + sin(w_m t) e_2m+1) with
    periods period x (1, phi, phi^2, phi^3) (phi the golden ratio, so the
    rotations never realign), are added to queries and keys at position t:
    nearby blocks score higher (a bump of about
    local^2 sum_m cos(w_m (i - j)) / sqrt(d), 4 local^2 / sqrt(d) at i = j).
    The result is rounded to bf16 once (round to nearest even); tokens are
    processed in chunks."""
    N, Hq, d = Qb.shape
    Hkv = Kb.shape[1]
    G = Hq // Hkv
    T = (N + 127) // 128
    rng = np.random.default_rng([seed, 7])
    dirs, sink_blocks = [], []
    for g in range(Hkv):
        basis, _ = np.linalg.qr(rng.standard_normal((d, 9)))
        dirs.append((basis[:, 0], basis[:, 1:9]))
        sink_blocks.append(np.unique(np.concatenate([[0], rng.integers(0, T, sinks)])))
    phi = (1.0 + 5.0 ** 0.5) / 2.0
    w = 2.0 * np.pi / (period * phi ** np.arange(4))
    Qo = np.empty_like(Qb)
    Ko = np.empty_like(Kb)
    for t0 in range(0, N, chunk):
        t1 = min(N, t0 + chunk)
        q = bf16_bits_to_f32(Qb[t0:t1]).astype(np.float64)
        k = bf16_bits_to_f32(Kb[t0:t1]).astype(np.float64)
        t = np.arange(t0, t1, dtype=np.float64)
        rot = np.stack([f(wm * t) for wm in w for f in (np.cos, np.sin)], 1)  # [n, 8]
        blk = np.arange(t0, t1) // 128
        for g in range(Hkv):
            u, e = dirs[g]
            k[np.isin(blk, sink_blocks[g]), g] += strength * u
            k[:, g] += local * rot @ e.T
            for h in range(g * G, (g + 1) * G):
                q[:, h] += strength * u + local * rot @ e.T
        Qo[t0:t1] = f64_to_bf16_bits(q)
        Ko[t0:t1] = f64_to_bf16_bits(k)
    return Qo, Ko


@dataclass
class BlockWorkload:
    """FlashPrefill-style block-sparse prefill of one sequence: Q/K/V from the
    seeded generator with plant_block_structure on Q and K; selection by
    vs_block_select at `alpha`."""
    name: str
    N: int
    Hq: int
    Hkv: int
    d: int
    rope_base: float
    seed: int
    alpha: float
    description: str = ""

    def qkv(self):
        Qb, Kb, Vb = gen_qkv(self.seed, self.N, self.Hq, self.Hkv, self.d, self.rope_base)
        Qb, Kb = plant_block_structure(Qb, Kb, seed=self.seed)
        return Qb, Kb, Vb


BLOCK_WORKLOADS = {
    "flashprefill_32k": BlockWorkload(
        "flashprefill_32k", 32768, 32, 8, 128, 500000.0, 18, 0.3,
        description="flashprefill_128k's recipe at N=32768 (the small profiling case)"),
    "flashprefill_128k": BlockWorkload(
        "flashprefill_128k", 131072, 32, 8, 128, 500000.0, 17, 0.3,
        description="32q/8kv, d=128, N=131072, planted sink + local block structure, block "
                    "pattern discovery at alpha 0.3, block-sparse attention"),
}

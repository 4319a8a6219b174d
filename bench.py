"""Benchmark of the vertical-slash sparse prefill hot path on B200.

One step = one attention layer's whole hot path over one batch of synthetic
input, on the default workload "llama_128k" (Llama-3.1-8B-shaped layer,
32 query / 8 KV heads, d=128, N=131072, 16 local + 16 global heads,
cumulative-threshold selection 0.95 capped at 8192):
    [vs_index_scores (indexer workloads)] -> vs_select (vertical)
    -> vs_select (slash) -> vs_sparse_attn_fwd (plan + attention).

Metric: effective TFLOP/s = 4 * d * P / t, P = number of selected (query,
key) pairs counted exactly from the index sets; ms per layer and the speed-up
over the library's dense causal kernel on the same inputs are reported too.

Prints ONE JSON line on rank 0.  Multi-GPU: one process per GPU (torchrun);
by default every rank runs its own replica of the layer (heads are
independent, there is no exchange step), timing is the max over ranks, value
= all ranks' flops / that time ("scaling": "weak").  --shard heads splits one
layer instead: each rank takes Hkv / N KV heads with their query heads and
index sets (still no exchange step; O stays head-sharded), value = the
layer's flops summed over ranks / the max rank time ("scaling": "strong").

--impl reference times the fp64 CPU oracle (the only other implementation)
on bounded row samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vs_workloads import BATCH_WORKLOADS, BLOCK_WORKLOADS, WORKLOADS, small_variant  # noqa: E402

METRIC = "VS-sparse prefill ms/layer & effective TFLOP/s at 128K; speedup vs dense"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama_128k",
                    choices=sorted(WORKLOADS) + sorted(BATCH_WORKLOADS) + sorted(BLOCK_WORKLOADS))
    ap.add_argument("--dense-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="multi-GPU: a replica of the layer per GPU, or the layer's heads split")
    ap.add_argument("--agg-steps", type=int, default=2,
                    help="timed runs of the ground-truth aggregation pass (0: skip)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--tokens", type=int, default=0,
                    help="run a single-sequence workload at this many tokens instead of its own "
                         "(same generators, caps scaled); for small profiling cases")
    return ap.parse_args()


# ----------------------------------------------------------------- pairs


def pairs_per_set(N: int, vlist: np.ndarray, slist: np.ndarray) -> int:
    """|{(i, j): j <= i, j in V or i - j in S}| = sum_{j in V}(N - j) + sum_{o in S}(N - o)
    - #{(j, o) in V x S : j + o <= N - 1}."""
    v = np.sort(np.asarray(vlist, np.int64))
    s = np.sort(np.asarray(slist, np.int64))
    both = np.searchsorted(s, N - 1 - v, side="right").sum() if v.size and s.size else 0
    return int((N - v).sum() + (N - s).sum() - both)


def row_pairs(i: np.ndarray, vlist, slist) -> np.ndarray:
    """|K_i| for the given rows."""
    v = np.sort(np.asarray(vlist, np.int64))
    s = np.sort(np.asarray(slist, np.int64))
    nv = np.searchsorted(v, i, side="right")
    ns = np.searchsorted(s, i, side="right")
    dup = np.zeros_like(i)
    vset = set(v.tolist())
    for r, row in enumerate(i):
        offs = s[: ns[r]]
        dup[r] = sum(1 for o in offs.tolist() if (row - o) in vset)
    return nv + ns - dup


def total_pairs(N, Hq, vi, vc, si, sc):
    H_sel = vi.shape[0]
    per = [pairs_per_set(N, vi[h, : vc[h]], si[h, : sc[h]]) for h in range(H_sel)]
    return sum(per[(h * H_sel) // Hq] for h in range(Hq)), per


# ----------------------------------------------------------- multi-rank


def dist_env():
    """(world, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity at world 1)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


_CUDART = None


def _cudart():
    """The CUDA runtime torch already loaded (for strided asynchronous copies)."""
    global _CUDART
    if _CUDART is None:
        import ctypes
        import ctypes.util
        path = None
        try:
            import nvidia.cuda_runtime as ncr
            cand = os.path.join(list(ncr.__path__)[0], "lib", "libcudart.so.12")
            path = cand if os.path.exists(cand) else None
        except ImportError:
            pass
        lib = ctypes.CDLL(path or ctypes.util.find_library("cudart"))
        lib.cudaMemcpy2DAsync.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                          ctypes.c_size_t, ctypes.c_size_t, ctypes.c_size_t,
                                          ctypes.c_int, ctypes.c_void_p]
        lib.cudaMemcpy2DAsync.restype = ctypes.c_int
        _CUDART = lib
    return _CUDART


def copy_heads(dst, src, h0, h1, stream):
    """Copy heads [h0, h1) of a token-major [N, H, d] tensor between host
    (pinned) and device, as one strided copy on `stream`."""
    N, H, d = src.shape
    es = src.element_size()
    kind = 1 if dst.is_cuda else 2  # host->device / device->host
    rc = _cudart().cudaMemcpy2DAsync(dst.data_ptr() + h0 * d * es, H * d * es,
                                     src.data_ptr() + h0 * d * es, H * d * es,
                                     (h1 - h0) * d * es, N, kind, stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"cudaMemcpy2DAsync failed ({rc})")


def copy_columns(dst, src, c0, c1, stream):
    """Copy columns [c0, c1) of a row-major [R, C] tensor from pinned host
    memory to the device, as one strided copy on `stream`."""
    R, C = src.shape
    es = src.element_size()
    rc = _cudart().cudaMemcpy2DAsync(dst.data_ptr() + c0 * es, C * es, src.data_ptr() + c0 * es,
                                     C * es, (c1 - c0) * es, R, 1, stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"cudaMemcpy2DAsync failed ({rc})")


def e2e_units(Hkv: int, G: int, head_cost, in_head_ms: float, kv_ms: float, out_head_ms: float,
              launch_ms: float = 0.05):
    """Order of the end-to-end pipeline's units: [(kv_group, h0, h1)].

    A unit is a KV group (its G query heads in one attention call); the first
    and the last group are split into single heads, so compute starts after
    one head's inputs have landed and only one head's output is copied after
    the last compute.  Copies in (Q heads, plus the group's K and V the first
    time), compute and copies out each run in order on their own engine, so
    a schedule's length is that of a three-stage pipeline.  The group order
    with the shortest modelled schedule is taken (every order for up to 8
    groups, else heaviest first).  head_cost[h]: modelled compute ms of query
    head h; in_head_ms / out_head_ms: one head's Q copy in / O copy out;
    kv_ms: one group's K and V copy in."""
    import itertools

    def units_of(order):
        out = []
        for x, g in enumerate(order):
            if G > 1 and Hkv > 1 and (x == 0 or x == len(order) - 1):
                out += [(g, h, h + 1) for h in range(g * G, (g + 1) * G)]
            else:
                out.append((g, g * G, (g + 1) * G))
        return out

    def makespan(units):
        t_in = t_c = t_out = 0.0
        seen = set()
        for g, h0, h1 in units:
            t_in += (h1 - h0) * in_head_ms + (0.0 if g in seen else kv_ms)
            seen.add(g)
            t_c = max(t_c, t_in) + sum(head_cost[h0:h1]) + launch_ms
            t_out = max(t_out, t_c) + (h1 - h0) * out_head_ms
        return t_out

    gcost = [sum(head_cost[g * G:(g + 1) * G]) for g in range(Hkv)]
    heaviest_first = sorted(range(Hkv), key=lambda g: (-gcost[g], g))
    if Hkv > 8:
        return units_of(heaviest_first)
    best = min(itertools.permutations(range(Hkv)),
               key=lambda order: (makespan(units_of(order)), order))
    return units_of(list(best))


def sum_over_ranks(values, device=None):
    """Element-wise sum of a list of floats over all ranks (identity at world 1)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def head_shard(Hq: int, Hkv: int, H_sel: int, world: int, rank: int):
    """Rank `rank`'s part of a head-sharded layer: whole KV groups, so no rank
    needs another's K/V.  Returns (q0, q1, kv0, kv1, s0, s1) half-open ranges
    of query heads, KV heads and index-set heads.  Needs world | Hkv."""
    if Hkv % world != 0:
        raise ValueError(f"head sharding needs the GPU count to divide Hkv={Hkv}")
    kv0, kv1 = rank * Hkv // world, (rank + 1) * Hkv // world
    G = Hq // Hkv
    s_per_q = H_sel / Hq
    q0, q1 = kv0 * G, kv1 * G
    return q0, q1, kv0, kv1, int(q0 * s_per_q), int(q1 * s_per_q)


def time_e2e(e2e_step, stream, flush, steps: int):
    """Device time of `steps` end-to-end steps, as the kernel steps are timed:
    one untimed warm-up step, then each timed step after an L2 flush written
    outside its timed window.  Returns the per-step times in ms."""
    import torch
    e2e_step()
    ts = []
    for _ in range(max(1, steps)):
        flush.zero_()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return ts


E2E_PROTOCOL = ("mean of the timed steps, each after an L2 flush outside its timed window, "
                "after one untimed warm-up step (the device step's protocol)")


def whole_job_value(world: int, flops_per_rank: float, ms: float) -> float:
    """Aggregate effective TFLOP/s: every rank processes one replica of the layer in
    (at most) `ms`, so the job does world x flops in that time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        # raw samples: $VS_CLOCK_DIR if set (to keep them), else the temp directory
        import tempfile
        d = os.environ.get("VS_CLOCK_DIR") or tempfile.gettempdir()
        self.path = os.path.join(d, f"vs_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        # wait (up to 5 s) for the first sample so the timed region is covered
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9:
                rows.append(p)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- peaks


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_rev() -> str:
    """Hash of the attention kernel sources: a committed traffic figure is only
    used while the kernel it was measured on is unchanged."""
    import hashlib
    h = hashlib.sha1()
    for f in ("attn_tc.cu", "ptx.cuh"):
        h.update(open(os.path.join(ROOT, "sparse_attention_long_head_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:12]


def ncu_traffic(workload: str):
    """DRAM bytes (read + write) per attention launch from the committed ncu
    summary for this workload, or None if absent or taken on another kernel."""
    p = os.path.join(ROOT, "profiles", f"attn_traffic_{workload}.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if d.get("kernel_rev") == kernel_rev():
            return d.get("dram_bytes_per_launch")
    return None


# --------------------------------------------------------------- our arm


def vs_config(w, world: int, sharded: bool = False) -> dict:
    """The `config` object of a vertical-slash workload's line (both arms)."""
    return {"workload": w.name, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "H_sel": w.H_sel,
            "select": w.select_mode, "k_v": w.k_v, "k_s": w.k_s, "tau_v": w.tau_v,
            "tau_s": w.tau_s, "indexer": w.indexer,
            "parallelism": f"heads x{world}" if sharded else f"replicas x{world}",
            "l2": "inputs exceed L2 (Q/K/V/O resident in HBM) and a 256 MiB buffer is "
                  "written between timed steps, outside the timed windows"}


def batch_config(w, world: int) -> dict:
    """The `config` object of a batch workload's line (both arms)."""
    return {"workload": w.name, "sequences": len(w.lengths), "tokens": int(w.cu_seqlens[-1]),
            "lengths": list(w.lengths), "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "H_sel": w.H_sel,
            "select": w.select_mode, "cap_frac": w.cap_frac, "tau_v": w.tau_v, "tau_s": w.tau_s,
            "parallelism": f"replicas x{world}",
            "l2": "a 256 MiB buffer is written between timed steps, outside the timed windows"}


def block_config(w, world: int) -> dict:
    """The `config` object of a block-sparse workload's line (both arms)."""
    return {"workload": w.name, "N": w.N, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "alpha": w.alpha,
            "parallelism": f"replicas x{world}",
            "l2": "inputs exceed L2; a 256 MiB buffer is written between timed steps, "
                  "outside the timed windows"}


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import sparse_attention_long_head_b200 as vs

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    dev = torch.device("cuda", torch.cuda.current_device())
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    t0 = time.time()
    Qb, Kb, Vb = w.qkv()
    if w.indexer:
        W1, W2 = w.indexer_weights()
        lv = ls = None
    else:
        lv, ls = w.all_scores()
    gen_s = time.time() - t0
    sharded = args.shard == "heads" and world > 1
    H_sel = w.H_sel
    if sharded:  # this rank's KV groups only
        q0, q1, kv0, kv1, s0, s1 = head_shard(w.Hq, w.Hkv, w.H_sel, world, rank)
        Qb = np.ascontiguousarray(Qb[:, q0:q1])
        Kb = np.ascontiguousarray(Kb[:, kv0:kv1])
        Vb = np.ascontiguousarray(Vb[:, kv0:kv1])
        if lv is not None:
            lv, ls = lv[s0:s1], ls[s0:s1]
        H_sel = s1 - s0

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    mode = w.select_mode_id
    if w.indexer:
        W1d, W2d = torch.from_numpy(W1).to(dev), torch.from_numpy(W2).to(dev)
        LV = torch.empty((Hkv, N), dtype=torch.float32, device=dev)
        LS = torch.empty_like(LV)
    else:
        LV, LS = torch.from_numpy(lv).to(dev), torch.from_numpy(ls).to(dev)
    vi = torch.empty((H_sel, w.k_v), dtype=torch.int32, device=dev)
    si = torch.empty((H_sel, w.k_s), dtype=torch.int32, device=dev)
    vc = torch.empty(H_sel, dtype=torch.int32, device=dev)
    sc = torch.empty(H_sel, dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, N), dtype=torch.float32, device=dev)
    ws_sel = vs.workspace(vs.vs_select_workspace_size(H_sel, N), dev)
    ws_sel2 = vs.workspace(vs.vs_select_workspace_size(H_sel, N), dev)
    ws_att = vs.workspace(vs.vs_attn_workspace_size_ld(N, Hq, H_sel, d, w.k_v), dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    # select x2, plan, pack (when each index set's heads lie in one KV group), attention,
    # plus the indexer; the status-word resets are driver memsets, not counted
    packs = (Hq // Hkv) % (Hq // H_sel) == 0
    launches_per_step = 4 + (1 if packs else 0) + (1 if w.indexer else 0)

    ev = {k: [] for k in ("step0", "idx1", "att0", "att1", "step1")}

    def step(record):
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["step0"].append(e)
        if w.indexer:
            vs.vs_index_scores(K, V, W1d, W2d, LV, LS)
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["idx1"].append(e)
        vs.vs_select(LV, mode, w.k_v, w.tau_v, vi, vc, ws_sel)
        vs.vs_select(LS, mode, w.k_s, w.tau_s, si, sc, ws_sel2)
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["att0"].append(e)
        vs.vs_sparse_attn_fwd(Q, K, V, vi, vc, si, sc, O, lse, ws_att)
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["att1"].append(e)
            ev["step1"].append(e)

    for _ in range(args.warmup):
        flush.zero_()
        step(False)
    torch.cuda.synchronize()
    for ws_ in (ws_sel, ws_sel2, ws_att):
        rc, flags = vs.vs_read_device_status(ws_)
        if rc != vs.VS_OK:
            raise RuntimeError(f"device status {vs.status_string(rc)} flags {flags}")

    # exact pair count from this step's index sets
    vih, vch, sih, sch = (x.cpu().numpy() for x in (vi, vc, si, sc))
    P_total, per_set = total_pairs(N, Hq, vih, vch, sih, sch)
    flops = 4.0 * d * P_total
    dense_flops = 4.0 * d * Hq * N * (N + 1) / 2

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clk:
        for _ in range(args.steps):
            flush.zero_()  # L2 flush outside the timed windows
            step(True)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in zip(ev["step0"], ev["step1"])]
    att_ms = [a.elapsed_time(b) for a, b in zip(ev["att0"], ev["att1"])]
    sel_ms = [a.elapsed_time(b) for a, b in zip(ev["idx1"], ev["att0"])]
    idx_ms = [a.elapsed_time(b) for a, b in zip(ev["step0"], ev["idx1"])]
    ms_step = float(np.mean(step_ms))
    ms_att = float(np.mean(att_ms))
    ms_sel = float(np.mean(sel_ms))
    ms_idx = float(np.mean(idx_ms))
    ms_step, ms_att = max_over_ranks([ms_step, ms_att], dev)
    # the job's flops: every replica's, or the shards' sum
    job_flops = sum_over_ranks([flops], dev)[0] if sharded else world * flops
    value = job_flops / (ms_step * 1e-3) / 1e12

    # the indexer alone, launches queued back to back: the in-step figure above
    # also holds the host's marshalling before its first launch (the GPU waits
    # for it after the L2 flush); the K/V rows it reads exceed L2
    ms_idx_kernel = None
    if w.indexer:
        n_idx = 5
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        flush.zero_()
        vs.vs_index_scores(K, V, W1d, W2d, LV, LS)
        a.record(stream)
        for _ in range(n_idx):
            vs.vs_index_scores(K, V, W1d, W2d, LV, LS)
        b.record(stream)
        b.synchronize()
        ms_idx_kernel = a.elapsed_time(b) / n_idx

    # dense causal kernel on the same inputs (speed-up denominator)
    ws_dense = vs.workspace(256, dev)
    dense_ms = None
    if args.dense_steps > 0:
        Od = torch.empty_like(Q)
        vs.vs_dense_attn_fwd(Q, K, V, Od, None, ws_dense)
        ts = []
        for _ in range(args.dense_steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            vs.vs_dense_attn_fwd(Q, K, V, Od, None, ws_dense)
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        dense_ms = float(np.mean(ts))
        del Od

    # ground-truth aggregation (column / diagonal sums of the full attention
    # weights) on the same inputs, after a dense pass for the row LSE
    agg = None
    if args.agg_steps > 0:
        Od = torch.empty_like(Q)
        lse_d = torch.empty((Hq, N), dtype=torch.float32, device=dev)
        vs.vs_dense_attn_fwd(Q, K, V, Od, lse_d, ws_dense)
        del Od
        A_v = torch.empty((Hq, N), dtype=torch.float32, device=dev)
        A_s = torch.empty_like(A_v)
        vs.vs_attn_aggregate(Q, K, lse_d, A_v, A_s, ws_dense)
        ts = []
        for _ in range(args.agg_steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            vs.vs_attn_aggregate(Q, K, lse_d, A_v, A_s, ws_dense)
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        rc, flags = vs.vs_read_device_status(ws_dense)
        if rc != vs.VS_OK:
            raise RuntimeError(f"aggregate device status {vs.status_string(rc)} flags {flags}")
        agg = {"ms": float(np.mean(ts)), "row_sum_err": float((A_v.sum(1) - N).abs().max() / N)}
        del A_v, A_s, lse_d

    # End to end through the public API with host buffers (pinned).  Work
    # units are KV groups, heaviest first; the first and the last group are
    # split into single query heads, so compute starts after one head's data
    # has landed and only one head's output is copied after the last
    # compute.  Copies in run on one stream, copies out on another, and the
    # units' attention calls alternate over two compute streams, so one
    # call's tail overlaps the next call's start.  Score-vector workloads
    # copy all score rows first and select for every head in two calls;
    # the indexer workload scores and selects per group.  Heads are
    # independent, so the result is the one-call result (checked).
    e2e = None
    if not args.no_e2e:
        hQ = torch.from_numpy(Qb.view(np.int16)).view(torch.bfloat16).pin_memory()
        hK = torch.from_numpy(Kb.view(np.int16)).view(torch.bfloat16).pin_memory()
        hV = torch.from_numpy(Vb.view(np.int16)).view(torch.bfloat16).pin_memory()
        hS = ([] if w.indexer else
              [torch.from_numpy(lv).pin_memory(), torch.from_numpy(ls).pin_memory()])
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in [hQ, hK, hV] + hS)
        d2h = hO.numel() * hO.element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        cs = [stream, torch.cuda.Stream(dev)]
        ws_att2 = [ws_att, vs.workspace(ws_att.numel(), dev)]
        ws_sel2b = [(ws_sel, ws_sel2), (vs.workspace(ws_sel.numel(), dev),
                                        vs.workspace(ws_sel2.numel(), dev))]
        G = Hq // Hkv
        # unit order from a model of the three engines: compute per head from
        # the timed step (ms per selected pair), copies at ~50 GB/s
        ms_pair = ms_att / max(1, P_total)
        head_cost = [ms_pair * per_set[(h * H_sel) // Hq] for h in range(Hq)]
        head_ms = N * d * Q.element_size() / 50e9 * 1e3
        units = e2e_units(Hkv, G, head_cost, head_ms, 2 * head_ms, head_ms)

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            for st in (s_in, cs[1]):
                st.wait_event(start)
            sel_done = None
            if not w.indexer:
                with torch.cuda.stream(s_in):
                    LV.copy_(hS[0], non_blocking=True)
                    LS.copy_(hS[1], non_blocking=True)
                scores_in = torch.cuda.Event()
                scores_in.record(s_in)
                cs[0].wait_event(scores_in)
                vs.vs_select(LV, mode, w.k_v, w.tau_v, vi, vc, ws_sel)
                vs.vs_select(LS, mode, w.k_s, w.tau_s, si, sc, ws_sel2)
                sel_done = torch.cuda.Event()
                sel_done.record(cs[0])
            landed, kv_in = {}, set()
            for u, (g, h0, h1) in enumerate(units):
                if g not in kv_in:
                    copy_heads(K, hK, g, g + 1, s_in)
                    copy_heads(V, hV, g, g + 1, s_in)
                    kv_in.add(g)
                copy_heads(Q, hQ, h0, h1, s_in)
                e = torch.cuda.Event()
                e.record(s_in)
                landed[u] = e
            done, scored = {}, {}
            for u, (g, h0, h1) in enumerate(units):
                st = cs[u % 2]
                wsa = ws_att2[u % 2]
                s0, s1 = h0 * H_sel // Hq, max(h0 * H_sel // Hq + 1, h1 * H_sel // Hq)
                st.wait_event(landed[u])
                with torch.cuda.stream(st):
                    if w.indexer:
                        if g not in scored:
                            # the group's index sets, once, on this unit's stream
                            gs0, gs1 = g * G * H_sel // Hq, (g + 1) * G * H_sel // Hq
                            wa, wb = ws_sel2b[u % 2]
                            vs.vs_index_scores(K[:, g:g + 1], V[:, g:g + 1], W1d, W2d,
                                               LV[gs0:gs1], LS[gs0:gs1], stream=st)
                            vs.vs_select(LV[gs0:gs1], mode, w.k_v, w.tau_v, vi[gs0:gs1],
                                         vc[gs0:gs1], wa, stream=st)
                            vs.vs_select(LS[gs0:gs1], mode, w.k_s, w.tau_s, si[gs0:gs1],
                                         sc[gs0:gs1], wb, stream=st)
                            ev = torch.cuda.Event()
                            ev.record(st)
                            scored[g] = ev
                        else:
                            st.wait_event(scored[g])
                    else:
                        st.wait_event(sel_done)
                    vs.vs_sparse_attn_fwd(Q[:, h0:h1], K[:, g:g + 1], V[:, g:g + 1], vi[s0:s1],
                                          vc[s0:s1], si[s0:s1], sc[s0:s1], O[:, h0:h1],
                                          lse[h0:h1], wsa, stream=st)
                e = torch.cuda.Event()
                e.record(st)
                done[u] = e
            for u, (g, h0, h1) in enumerate(units):
                s_out.wait_event(done[u])
                copy_heads(hO, O, h0, h1, s_out)
            stream.wait_stream(s_out)
            stream.wait_stream(cs[1])

        ts = time_e2e(e2e_step, stream, flush, args.steps)
        # the pipelined result is the one-call result
        O_ref = O.clone()
        step(False)
        torch.cuda.synchronize()
        if not torch.equal(O, O_ref):
            raise RuntimeError("pipelined end-to-end output differs from the one-call output")
        del O_ref
        e2e_ms = max_over_ranks([float(np.mean(ts))], dev)[0]
        e2e = {"value": round(job_flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "protocol": E2E_PROTOCOL,
               "pipeline": "KV groups in the order of the shortest modelled copy-in / compute / "
                           "copy-out schedule (first and last split into heads): copy-in stream, "
                           "two alternating compute streams, copy-out stream"}

    peaks, peak_kind = measured_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    att_tflops = flops / (ms_att * 1e-3) / 1e12
    algo_bytes = (Q.numel() + K.numel() + V.numel() + O.numel()) * 2 + lse.numel() * 4 \
        + (vi.numel() + si.numel()) * 4
    t_roof_ms = max(flops / (peak * 1e12), algo_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    bound = "tensor" if flops / (peak * 1e12) >= algo_bytes / (peaks["hbm_gbs"] * 1e9) else "hbm"
    traffic = ncu_traffic(w.name)
    touched = structural_touched(N, vih, vch, sih, sch, Hq)

    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded generators shaped like the pages' workloads)",
        "config": vs_config(w, world, sharded),
        "ms_per_layer": round(ms_step, 3), "ms_indexer": round(ms_idx, 3) if w.indexer else None,
        "ms_indexer_back_to_back": round(ms_idx_kernel, 3) if w.indexer else None,
        "ms_select": round(ms_sel, 3), "ms_attention": round(ms_att, 3),
        "kernels": kernel_rooflines(w, peaks, N, Hq, Hkv, d, H_sel, flops, algo_bytes, ms_att,
                                    ms_sel, ms_idx_kernel if w.indexer else ms_idx, vih.shape[1],
                                    sih.shape[1], agg),
        "selected_pairs": int(P_total), "density_vs_causal": round(P_total / (Hq * N * (N + 1) / 2), 5),
        "dense_ms": None if dense_ms is None else round(dense_ms, 3),
        "dense_tflops": None if dense_ms is None else round(dense_flops / (dense_ms * 1e-3) / 1e12, 2),
        "speedup_vs_dense": None if dense_ms is None else round(dense_ms / ms_step, 3),
        "structural_ceiling": round(P_total / (touched * 128 * 128), 4) if touched else None,
        "roofline": {"bound": bound, "achieved": round(att_tflops if bound == "tensor" else
                                                       algo_bytes / (ms_att * 1e-3) / 1e9, 2),
                     "peak": peak if bound == "tensor" else peaks["hbm_gbs"],
                     "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                     "frac": round(t_roof_ms / ms_att, 4), "traffic": traffic,
                     "kernel": "vs_sparse_attn_fwd (plan + attn_tc_kernel)",
                     "peak_source": f"{peak_kind} bf16 sustained (MEASURED_PEAKS.json)",
                     "frac_vs_burst_peak": round(flops / (peaks["bf16_tflops"] * 1e12) * 1e3 / ms_att, 4),
                     "t_roof_ms": round(t_roof_ms, 3),
                     # the HBM term against the measured copy rate and the nominal ~8 TB/s
                     "hbm_bytes": int(algo_bytes),
                     "hbm_frac_measured": round(algo_bytes / (peaks["hbm_gbs"] * 1e9) / (ms_att * 1e-3), 5),
                     "hbm_frac_nominal_8tbs": round(algo_bytes / 8e12 / (ms_att * 1e-3), 5)},
        "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "input_gen_s": round(gen_s, 1),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, Qb, Kb, Vb, vih, vch, sih, sch, args.cpu_seconds)
    out["clocks"] = clk.summary()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def kernel_rooflines(w, peaks, N, Hq, Hkv, d, H_sel, flops, att_bytes, ms_att, ms_sel, ms_idx,
                     ld_v, ld_s, agg=None):
    """Per hot-path kernel: achieved vs the roofline that bounds it.
    attention (+plan, +pack): tensor-bound, 4 d P flops; select x2: HBM-bound,
    4 B per score read + 4 B per index slot written; indexer (bf16 rows, the
    tensor-core kernel): 2 (2d hidden + 2 hidden) flops and 2 x 2d bytes of
    [k; v] in plus 8 B of logits out per (token, KV head), bound by the slower
    of the bf16 tensor peak (burst: the kernel is timed alone) and HBM."""
    out = {}
    peak_t = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    t_att = flops / (peak_t * 1e12)
    out["attention"] = {"ms": round(ms_att, 3), "bound": "tensor",
                        "achieved_tflops": round(flops / (ms_att * 1e-3) / 1e12, 2),
                        "frac": round(max(t_att, att_bytes / (peaks["hbm_gbs"] * 1e9)) / (ms_att * 1e-3), 4)}
    sel_bytes = 4.0 * H_sel * N * 2 + 4.0 * H_sel * (ld_v + ld_s)
    out["select_x2"] = {"ms": round(ms_sel, 3), "bound": "hbm",
                        "achieved_gbs": round(sel_bytes / (ms_sel * 1e-3) / 1e9, 1),
                        "frac": round(sel_bytes / (peaks["hbm_gbs"] * 1e9) / (ms_sel * 1e-3), 5)}
    if agg is not None:
        # one exp per causal (query, key) pair; MUFU ex2 runs 16 per clock per SM
        n_exp = Hq * N * (N + 1) / 2
        mufu_peak = 16 * 148 * peaks.get("sm_max_mhz", 1965.0) * 1e6
        out["aggregate"] = {"ms": round(agg["ms"], 3), "bound": "alu (MUFU ex2)",
                            "achieved_gexp_s": round(n_exp / (agg["ms"] * 1e-3) / 1e9, 1),
                            "peak_gexp_s": round(mufu_peak / 1e9, 1),
                            "frac": round(n_exp / mufu_peak / (agg["ms"] * 1e-3), 4),
                            "row_sum_rel_err": agg["row_sum_err"]}
    if w.indexer:
        hidden = w.hidden
        iflops = 2.0 * N * Hkv * (2 * d * hidden + 2 * hidden)
        ibytes = N * Hkv * (2.0 * 2 * d + 8.0) + 4.0 * hidden * (2 * d + 2)
        t_tc = iflops / (peaks["bf16_tflops"] * 1e12)
        t_hbm = ibytes / (peaks["hbm_gbs"] * 1e9)
        out["indexer"] = {"ms": round(ms_idx, 3), "bound": "tensor" if t_tc >= t_hbm else "hbm",
                          "achieved_tflops": round(iflops / (ms_idx * 1e-3) / 1e12, 2),
                          "achieved_gbs": round(ibytes / (ms_idx * 1e-3) / 1e9, 1),
                          "t_roof_ms": round(max(t_tc, t_hbm) * 1e3, 4),
                          "frac": round(max(t_tc, t_hbm) / (ms_idx * 1e-3), 4)}
    return out


def structural_touched(N, vi, vc, si, sc, Hq):
    """128x128 tiles the kernel's cheaper mode touches per head (for the ceiling)."""
    T = (N + 127) // 128
    H_sel = vi.shape[0]
    total = 0
    for h in range(Hq):
        hs = (h * H_sel) // Hq
        v = np.sort(vi[hs, : vc[hs]].astype(np.int64))
        s = np.sort(si[hs, : sc[hs]].astype(np.int64))
        touched = np.zeros(T + 2, bool)
        dl = s >> 7
        touched[dl] = True
        touched[(dl + 1)[(s & 127) != 0]] = True
        d1 = touched.copy()
        d1[1:] |= touched[:-1]
        pref = np.concatenate([[0], np.cumsum(d1)])
        for p in range((T + 1) // 2):
            last_b = min(2 * p + 1, T - 1)
            lo, hi = 2 * p + 1 - last_b, 2 * p + 1
            nslash = pref[hi + 1] - pref[lo]
            nvp = np.searchsorted(v, min(256 * p + 255, N - 1), side="right")
            nsplit = (nvp + 127) // 128 + nslash
            total += 2 * min(nsplit, last_b + 1)
    return total


# ------------------------------------------------------------ CPU baseline


def _cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, Qb, Kb, Vb, vi, vc, si, sc, seconds, seed=0,
                 sets_from="this run's GPU selection"):
    """The fp64 oracle as it stands, timed on a bounded row sample of the same
    workload; scaled to the metric by pair count (oracle effective TFLOP/s)."""
    import oracle
    N, Hq, d = Qb.shape
    H_sel = vi.shape[0]
    rng = np.random.default_rng(seed)
    t_used = 0.0
    pairs = 0
    rows_done = 0
    heads = []
    while t_used < seconds:
        h = int(rng.integers(0, Hq))
        hs = (h * H_sel) // Hq
        rows = np.sort(rng.integers(0, N, 32))
        t0 = time.time()
        oracle.attn_rows(Qb, Kb, Vb, h, rows, vi, vc, si, sc)
        t_used += time.time() - t0
        pairs += int(row_pairs(rows, vi[hs, : vc[hs]], si[hs, : sc[hs]]).sum())
        rows_done += rows.size
        heads.append(h)
    # the dense causal oracle per row, likewise (a few rows spread over the sequence)
    drows = np.sort(rng.integers(N // 2, N, 16))
    t0 = time.time()
    oracle.attn_rows(Qb, Kb, Vb, 0, drows, dense=True)
    dense_row_ms = (time.time() - t0) * 1e3 / drows.size
    dense_pairs_per_row = float(np.mean(drows + 1))
    return {"value": round(4.0 * d * pairs / t_used / 1e12, 6), "unit": UNIT, "cores": _cpu_cores(),
            "kind": "oracle",
            "sample": f"{rows_done} query rows (32 random rows of a random head per draw, "
                      f"{len(set(heads))} heads) of {w.name}, fp64 row-form oracle with OpenMP over "
                      f"rows, {t_used:.1f} s; index sets from {sets_from}",
            "sparse_row_ms": round(t_used * 1e3 / max(rows_done, 1), 4),
            "dense_row_ms": round(dense_row_ms, 4),
            "dense_row_sample": f"16 random rows of the second half, head 0, "
                                f"{dense_pairs_per_row:.0f} keys per row on average"}


def run_reference(args, w):
    """Reference arm: the oracle as it stands on the host cores, rank 0 only."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    Qb, Kb, Vb = w.qkv()
    mode = w.select_mode_id
    if w.indexer:
        W1, W2 = w.indexer_weights()
        toks = np.arange(w.N)
        lv, ls = oracle.index_scores(Kb, Vb, W1, W2, toks)
        lv, ls = lv.astype(np.float32), ls.astype(np.float32)
    else:
        lv, ls = w.all_scores()
    vi, vc, _ = oracle.select_heads(lv, mode, w.k_v, w.tau_v)
    si, sc, _ = oracle.select_heads(ls, mode, w.k_s, w.tau_s)
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    last = None
    for it in range(args.warmup + args.steps):
        last = cpu_baseline(w, Qb, Kb, Vb, vi, vc, si, sc, per_step, seed=it,
                            sets_from="the oracle's own selection")
        if it >= args.warmup:
            vals.append(last["value"])
    value = float(np.mean(vals))
    out = {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
           "data": "synthetic (seeded generators shaped like the pages' workloads)",
           "config": vs_config(w, world),
           "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": last["cores"],
                            "kind": "oracle", "sample": last["sample"] + f"; {per_step:.1f} s per step"},
           "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def batch_oracle_sample(w, Qb, Kb, Vb, sets, seconds, seed=0,
                        sets_from="this run's GPU selection"):
    """The fp64 oracle on random rows of random sequences of a batch workload
    for about `seconds`; effective TFLOP/s by pair count."""
    import oracle
    vih, vch, sih, sch = sets
    cu_h = w.cu_seqlens
    B, H_sel, Hq, d = len(w.lengths), w.H_sel, w.Hq, w.d
    rng = np.random.default_rng(seed)
    t_used, p_done, rows_done = 0.0, 0, 0
    while t_used < seconds:
        b = int(rng.integers(0, B))
        n, t0 = w.lengths[b], int(cu_h[b])
        h = int(rng.integers(0, Hq))
        r = b * H_sel + (h * H_sel) // Hq
        rows = np.sort(rng.integers(0, n, 32))
        sl = slice(t0, t0 + n)
        part = slice(b * H_sel, (b + 1) * H_sel)
        t1 = time.time()
        oracle.attn_rows(Qb[sl], Kb[sl], Vb[sl], h, rows, vih[part], vch[part], sih[part],
                         sch[part])
        t_used += time.time() - t1
        p_done += int(row_pairs(rows, vih[r, : vch[r]], sih[r, : sch[r]]).sum())
        rows_done += rows.size
    return {"value": round(4.0 * d * p_done / t_used / 1e12, 6), "unit": UNIT,
            "cores": _cpu_cores(), "kind": "oracle",
            "sample": f"{rows_done} query rows (32 random rows of a random sequence and head per "
                      f"draw) of {w.name}, fp64 row-form oracle, {t_used:.1f} s; index sets "
                      f"from {sets_from}"}


def run_batch_reference(args, w):
    """Reference arm of a batch workload: the oracle (its own selection per
    sequence) on bounded row samples, rank 0 only."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    Qb, Kb, Vb = w.qkv()
    B, H_sel = len(w.lengths), w.H_sel
    cap_max = w.cap(max(w.lengths))
    vih = np.full((B * H_sel, cap_max), -1, np.int32)
    sih = np.full_like(vih, -1)
    vch = np.zeros(B * H_sel, np.int32)
    sch = np.zeros_like(vch)
    for b, n in enumerate(w.lengths):
        lv, ls = w.scores(b)
        k = w.cap(n)
        vi, vc, _ = oracle.select_heads(lv, w.select_mode_id, k, w.tau_v)
        si, sc, _ = oracle.select_heads(ls, w.select_mode_id, k, w.tau_s)
        vih[b * H_sel:(b + 1) * H_sel, :k], vch[b * H_sel:(b + 1) * H_sel] = vi, vc
        sih[b * H_sel:(b + 1) * H_sel, :k], sch[b * H_sel:(b + 1) * H_sel] = si, sc
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, last = [], None
    for it in range(args.warmup + args.steps):
        last = batch_oracle_sample(w, Qb, Kb, Vb, (vih, vch, sih, sch), per_step, seed=it,
                                   sets_from="the oracle's own selection")
        if it >= args.warmup:
            vals.append(last["value"])
    value = float(np.mean(vals))
    print(json.dumps({
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "impl": "reference",
        "data": "synthetic (seeded generators shaped like the pages' workloads)",
        "config": batch_config(w, world),
        "cpu_baseline": dict(last, value=round(value, 6),
                             sample=last["sample"] + f"; {per_step:.1f} s per step"),
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def run_batch(args, w):
    """A batch of sequences packed along the token axis: per sequence two
    selects, then one batched sparse attention call (the step); value =
    4 d x (selected pairs of every sequence) / step time."""
    import torch
    import torch.distributed as dist
    import sparse_attention_long_head_b200 as vs

    world, rank, local_rank = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    t0 = time.time()
    Qb, Kb, Vb = w.qkv()
    scores = [w.scores(b) for b in range(len(w.lengths))]
    gen_s = time.time() - t0
    to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    T, Hq, d = Q.shape
    B, H_sel, mode = len(w.lengths), w.H_sel, w.select_mode_id
    cu_h = w.cu_seqlens
    cu = torch.from_numpy(cu_h).to(dev)
    max_n = int(max(w.lengths))
    cap_max = w.cap(max_n)
    # scores packed along the token axis: [H_sel][total], sequence b at cu[b]
    LV = torch.from_numpy(np.ascontiguousarray(np.concatenate([lv for lv, _ in scores], 1))).to(dev)
    LS = torch.from_numpy(np.ascontiguousarray(np.concatenate([ls for _, ls in scores], 1))).to(dev)
    caps = torch.tensor([w.cap(n) for n in w.lengths], dtype=torch.int32, device=dev)
    vi = torch.full((B * H_sel, cap_max), -1, dtype=torch.int32, device=dev)
    si = torch.full_like(vi, -1)
    vc = torch.empty(B * H_sel, dtype=torch.int32, device=dev)
    sc = torch.empty_like(vc)
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, T), dtype=torch.float32, device=dev)
    ws_sel = vs.workspace(vs.vs_select_workspace_size_varlen(B, H_sel, max_n), dev)
    ws_att = vs.workspace(vs.vs_attn_workspace_size_varlen(B, max_n, H_sel, d, cap_max), dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = {k: [] for k in ("s0", "a0", "a1")}

    # a step launches 5 kernels: two batched selects, then plan, pack and attention
    def step(record):
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["s0"].append(e)
        vs.vs_select_varlen(LV, cu, max_n, mode, caps, cap_max, w.tau_v, vi, vc, ws_sel)
        vs.vs_select_varlen(LS, cu, max_n, mode, caps, cap_max, w.tau_s, si, sc, ws_sel)
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["a0"].append(e)
        vs.vs_sparse_attn_fwd_varlen(Q, K, V, cu, max_n, vi, vc, si, sc, O, lse, ws_att)
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["a1"].append(e)

    for _ in range(args.warmup):
        flush.zero_()
        step(False)
    torch.cuda.synchronize()
    rc, flags = vs.vs_read_device_status(ws_att)
    if rc != vs.VS_OK:
        raise RuntimeError(f"device status {vs.status_string(rc)} flags {flags}")
    vih, vch, sih, sch = (x.cpu().numpy() for x in (vi, vc, si, sc))
    pairs = 0
    for b, n in enumerate(w.lengths):
        for h in range(Hq):
            r = b * H_sel + (h * H_sel) // Hq
            pairs += pairs_per_set(n, vih[r, : vch[r]], sih[r, : sch[r]])
    flops = 4.0 * d * pairs
    dense_pairs = Hq * sum(n * (n + 1) // 2 for n in w.lengths)
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clk:
        for _ in range(args.steps):
            flush.zero_()
            step(True)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_step = float(np.mean([a.elapsed_time(b) for a, b in zip(ev["s0"], ev["a1"])]))
    ms_att = float(np.mean([a.elapsed_time(b) for a, b in zip(ev["a0"], ev["a1"])]))
    ms_step, ms_att = max_over_ranks([ms_step, ms_att], dev)
    value = whole_job_value(world, flops, ms_step)
    # dense varlen on the same batch (speed-up denominator)
    dense_ms = None
    if args.dense_steps > 0:
        Od = torch.empty_like(Q)
        wsd = vs.workspace(256, dev)
        vs.vs_dense_attn_fwd_varlen(Q, K, V, cu, max_n, Od, None, wsd)
        ts = []
        for _ in range(args.dense_steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            vs.vs_dense_attn_fwd_varlen(Q, K, V, cu, max_n, Od, None, wsd)
            b_.record(stream)
            b_.synchronize()
            ts.append(a.elapsed_time(b_))
        dense_ms = float(np.mean(ts))
        del Od
    # End to end: chunks of consecutive sequences (about a sixth of the tokens
    # each) go through copy-in (their Q, K, V rows and score rows), their
    # selects and one batched attention call, and copy-out of their O rows;
    # consecutive chunks alternate over two compute streams.  Sequences are
    # independent, so the result is the one-call result (checked).
    e2e = None
    if not args.no_e2e:
        hQ, hK, hV = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
                      for x in (Qb, Kb, Vb))
        hLV, hLS = LV.cpu().pin_memory(), LS.cpu().pin_memory()  # packed [H_sel][total]
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV, hLV, hLS))
        d2h = hO.numel() * hO.element_size()
        bounds, acc = [0], 0
        for b, n in enumerate(w.lengths):
            acc += n
            if acc >= T / 6 and b + 1 < B:
                bounds.append(b + 1)
                acc = 0
        bounds.append(B)
        chunks = [(bounds[j], bounds[j + 1]) for j in range(len(bounds) - 1)]
        cu_c = [torch.from_numpy((cu_h[b0:b1 + 1] - cu_h[b0]).astype(np.int32)).to(dev)
                for b0, b1 in chunks]
        lse_c = [torch.empty((Hq, int(cu_h[b1] - cu_h[b0])), dtype=torch.float32, device=dev)
                 for b0, b1 in chunks]
        maxn_c = [int(max(w.lengths[b0:b1])) for b0, b1 in chunks]
        ws_att2 = [ws_att, vs.workspace(ws_att.numel(), dev)]
        ws_sel2 = [ws_sel, vs.workspace(ws_sel.numel(), dev)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        cs = [stream, torch.cuda.Stream(dev)]

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            for st in (s_in, cs[1]):
                st.wait_event(start)
            landed = []
            for b0, b1 in chunks:
                t0, t1 = int(cu_h[b0]), int(cu_h[b1])
                with torch.cuda.stream(s_in):
                    Q[t0:t1].copy_(hQ[t0:t1], non_blocking=True)
                    K[t0:t1].copy_(hK[t0:t1], non_blocking=True)
                    V[t0:t1].copy_(hV[t0:t1], non_blocking=True)
                    copy_columns(LV, hLV, t0, t1, s_in)
                    copy_columns(LS, hLS, t0, t1, s_in)
                e = torch.cuda.Event()
                e.record(s_in)
                landed.append(e)
            done = []
            for j, (b0, b1) in enumerate(chunks):
                st = cs[j % 2]
                st.wait_event(landed[j])
                t0, t1 = int(cu_h[b0]), int(cu_h[b1])
                r0, r1 = b0 * H_sel, b1 * H_sel
                with torch.cuda.stream(st):
                    # the chunk's sequences: their offsets into the packed scores
                    cu_j, caps_j = cu[b0:b1 + 1], caps[b0:b1]
                    vs.vs_select_varlen(LV, cu_j, maxn_c[j], mode, caps_j, cap_max, w.tau_v,
                                        vi[r0:r1], vc[r0:r1], ws_sel2[j % 2], stream=st)
                    vs.vs_select_varlen(LS, cu_j, maxn_c[j], mode, caps_j, cap_max, w.tau_s,
                                        si[r0:r1], sc[r0:r1], ws_sel2[j % 2], stream=st)
                    vs.vs_sparse_attn_fwd_varlen(Q[t0:t1], K[t0:t1], V[t0:t1], cu_c[j], maxn_c[j],
                                                 vi[r0:r1], vc[r0:r1], si[r0:r1], sc[r0:r1],
                                                 O[t0:t1], lse_c[j], ws_att2[j % 2], stream=st)
                e = torch.cuda.Event()
                e.record(st)
                done.append(e)
            for j, (b0, b1) in enumerate(chunks):
                t0, t1 = int(cu_h[b0]), int(cu_h[b1])
                s_out.wait_event(done[j])
                with torch.cuda.stream(s_out):
                    hO[t0:t1].copy_(O[t0:t1], non_blocking=True)
            stream.wait_stream(s_out)
            stream.wait_stream(cs[1])

        ts = time_e2e(e2e_step, stream, flush, args.steps)
        for x in ws_att2:
            rc, flags = vs.vs_read_device_status(x)
            if rc != vs.VS_OK:
                raise RuntimeError(f"device status {vs.status_string(rc)} flags {flags}")
        O_ref = O.clone()
        step(False)
        torch.cuda.synchronize()
        if not torch.equal(O, O_ref):
            raise RuntimeError("pipelined end-to-end output differs from the one-call output")
        del O_ref
        e2e_ms = max_over_ranks([float(np.mean(ts))], dev)[0]
        e2e = {"value": round(whole_job_value(world, flops, e2e_ms), 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "protocol": E2E_PROTOCOL,
               "pipeline": f"{len(chunks)} chunks of consecutive sequences: copy-in stream, two "
                           "alternating compute streams (two batched selects + one batched "
                           "attention call per chunk), copy-out stream"}
    peaks, peak_kind = measured_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    algo_bytes = (Q.numel() + K.numel() + V.numel() + O.numel()) * 2 + lse.numel() * 4 \
        + (vi.numel() + si.numel()) * 4
    t_roof_ms = max(flops / (peak * 1e12), algo_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generators shaped like the pages' workloads)",
        "config": batch_config(w, world),
        "ms_select": round(ms_step - ms_att, 3), "ms_attention": round(ms_att, 3),
        "selected_pairs": int(pairs), "density_vs_causal": round(pairs / dense_pairs, 5),
        "dense_ms": None if dense_ms is None else round(dense_ms, 3),
        "speedup_vs_dense": None if dense_ms is None else round(dense_ms / ms_step, 3),
        "roofline": {"bound": "tensor", "achieved": round(flops / (ms_att * 1e-3) / 1e12, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(t_roof_ms / ms_att, 4),
                     "traffic": None, "kernel": "vs_sparse_attn_fwd_varlen (plan + pack + attn)",
                     "peak_source": f"{peak_kind} bf16 sustained (MEASURED_PEAKS.json)"},
        "e2e": e2e, "gpu_launches": 5 * args.steps, "input_gen_s": round(gen_s, 1),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = batch_oracle_sample(w, Qb, Kb, Vb, (vih, vch, sih, sch),
                                                  args.cpu_seconds)
    out["clocks"] = clk.summary()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def block_pairs(mask: np.ndarray, N: int) -> int:
    """Causal (query, key) pairs inside the kept blocks of a [H, T, W] mask."""
    H, T, _ = mask.shape
    bits = np.unpackbits(np.ascontiguousarray(mask).view(np.uint8), bitorder="little")
    bits = bits.reshape(H, T, -1)[:, :, :T].astype(bool)
    rows = np.minimum(N - 128 * np.arange(T), 128)          # query rows of block I
    cols = np.minimum(N - 128 * np.arange(T), 128)          # keys of block J
    total = 0
    for I in range(T):
        kept = bits[:, I, :I].sum()
        total += int(kept) * 128 * int(rows[I]) if I else 0   # full past blocks (128 keys each)
        diag = int(bits[:, I, I].sum())
        total += diag * int(rows[I]) * (int(rows[I]) + 1) // 2
    return total


def run_blocks(args, w):
    """FlashPrefill-style step: block pattern discovery then block-sparse
    attention; value = 4 d x (causal pairs in the kept blocks) / step time."""
    import torch
    import torch.distributed as dist
    import sparse_attention_long_head_b200 as vs

    world, rank, local_rank = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    t0 = time.time()
    Qb, Kb, Vb = w.qkv()
    gen_s = time.time() - t0
    to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    N, Hq, d = Q.shape
    T = (N + 127) // 128
    mask = torch.zeros((Hq, T, (T + 31) // 32), dtype=torch.int32, device=dev)
    ws = vs.workspace(max(vs.vs_block_select_workspace_size(N, w.Hkv, d),
                          vs.vs_block_attn_workspace_size(N, Hq)), dev)
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, N), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = {k: [] for k in ("s0", "a0", "a1")}

    def step(record):
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["s0"].append(e)
        vs.vs_block_select(Q, K, w.alpha, mask, ws)
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["a0"].append(e)
        vs.vs_block_sparse_attn_fwd(Q, K, V, mask, O, lse, ws)
        if record:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev["a1"].append(e)

    for _ in range(args.warmup):
        flush.zero_()
        step(False)
    torch.cuda.synchronize()
    rc, flags = vs.vs_read_device_status(ws)
    if rc != vs.VS_OK:
        raise RuntimeError(f"device status {vs.status_string(rc)} flags {flags}")
    mask_h = mask.cpu().numpy().view(np.uint32)
    pairs = block_pairs(mask_h, N)
    flops = 4.0 * d * pairs
    dense_pairs = Hq * N * (N + 1) // 2
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clk:
        for _ in range(args.steps):
            flush.zero_()
            step(True)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_step = float(np.mean([a.elapsed_time(b) for a, b in zip(ev["s0"], ev["a1"])]))
    ms_att = float(np.mean([a.elapsed_time(b) for a, b in zip(ev["a0"], ev["a1"])]))
    ms_step, ms_att = max_over_ranks([ms_step, ms_att], dev)
    value = world * flops / (ms_step * 1e-3) / 1e12
    dense_ms = None
    if args.dense_steps > 0:
        Od = torch.empty_like(Q)
        wsd = vs.workspace(256, dev)
        vs.vs_dense_attn_fwd(Q, K, V, Od, None, wsd)
        ts = []
        for _ in range(args.dense_steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            vs.vs_dense_attn_fwd(Q, K, V, Od, None, wsd)
            b_.record(stream)
            b_.synchronize()
            ts.append(a.elapsed_time(b_))
        dense_ms = float(np.mean(ts))
        del Od
    # End to end: the same pipeline as the vertical-slash workload.  Per KV
    # group (its query heads; the first and last group split into heads):
    # copy its Q, K, V in, discover its blocks and run its block-sparse
    # attention, copy its O out; the calls of consecutive units alternate over
    # two compute streams.  Heads are independent, so the result is the
    # one-call result (checked).
    e2e = None
    if not args.no_e2e:
        hQ, hK, hV = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
                      for x in (Qb, Kb, Vb))
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV))
        d2h = hO.numel() * hO.element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        cs = [stream, torch.cuda.Stream(dev)]
        ws2 = [ws, vs.workspace(ws.numel(), dev)]
        G = Hq // w.Hkv
        kept = [int(np.unpackbits(mask_h[h].view(np.uint8)).sum()) for h in range(Hq)]
        ms_disc = ms_step - ms_att
        head_cost = [ms_disc / Hq + ms_att * kept[h] / max(1, sum(kept)) for h in range(Hq)]
        head_ms = N * d * Q.element_size() / 50e9 * 1e3
        units = e2e_units(w.Hkv, G, head_cost, head_ms, 2 * head_ms, head_ms)

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            for st in (s_in, cs[1]):
                st.wait_event(start)
            landed, kv_in = {}, set()
            for u, (g, h0, h1) in enumerate(units):
                if g not in kv_in:
                    copy_heads(K, hK, g, g + 1, s_in)
                    copy_heads(V, hV, g, g + 1, s_in)
                    kv_in.add(g)
                copy_heads(Q, hQ, h0, h1, s_in)
                e = torch.cuda.Event()
                e.record(s_in)
                landed[u] = e
            done = {}
            for u, (g, h0, h1) in enumerate(units):
                st = cs[u % 2]
                st.wait_event(landed[u])
                with torch.cuda.stream(st):
                    vs.vs_block_select(Q[:, h0:h1], K[:, g:g + 1], w.alpha, mask[h0:h1],
                                       ws2[u % 2], stream=st)
                    vs.vs_block_sparse_attn_fwd(Q[:, h0:h1], K[:, g:g + 1], V[:, g:g + 1],
                                                mask[h0:h1], O[:, h0:h1], lse[h0:h1], ws2[u % 2],
                                                stream=st)
                e = torch.cuda.Event()
                e.record(st)
                done[u] = e
            for u, (g, h0, h1) in enumerate(units):
                s_out.wait_event(done[u])
                copy_heads(hO, O, h0, h1, s_out)
            stream.wait_stream(s_out)
            stream.wait_stream(cs[1])

        ts = time_e2e(e2e_step, stream, flush, args.steps)
        for x in ws2:
            rc, flags = vs.vs_read_device_status(x)
            if rc != vs.VS_OK:
                raise RuntimeError(f"device status {vs.status_string(rc)} flags {flags}")
        O_ref = O.clone()
        step(False)
        torch.cuda.synchronize()
        if not torch.equal(O, O_ref):
            raise RuntimeError("pipelined end-to-end output differs from the one-call output")
        del O_ref
        e2e_ms = max_over_ranks([float(np.mean(ts))], dev)[0]
        e2e = {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "protocol": E2E_PROTOCOL,
               "pipeline": "KV groups in the order of the shortest modelled copy-in / compute / "
                           "copy-out schedule (first and last split into heads): copy-in stream, "
                           "two alternating compute streams (block discovery + block-sparse "
                           "attention per unit), copy-out stream"}
    peaks, peak_kind = measured_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    algo_bytes = (Q.numel() + K.numel() + V.numel() + O.numel()) * 2 + lse.numel() * 4
    t_roof_ms = max(flops / (peak * 1e12), algo_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e3
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generators shaped like the pages' workloads)",
        "config": block_config(w, world),
        "ms_select": round(ms_step - ms_att, 3), "ms_attention": round(ms_att, 3),
        "selected_pairs": int(pairs), "density_vs_causal": round(pairs / dense_pairs, 5),
        "dense_ms": None if dense_ms is None else round(dense_ms, 3),
        "speedup_vs_dense": None if dense_ms is None else round(dense_ms / ms_step, 3),
        "roofline": {"bound": "tensor", "achieved": round(flops / (ms_att * 1e-3) / 1e12, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(t_roof_ms / ms_att, 4),
                     "traffic": None, "kernel": "vs_block_sparse_attn_fwd (plan + attn)",
                     "peak_source": f"{peak_kind} bf16 sustained (MEASURED_PEAKS.json)"},
        "e2e": e2e, "gpu_launches": 4 * args.steps, "input_gen_s": round(gen_s, 1),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = block_oracle_sample(w, Qb, Kb, Vb, mask_h, args.cpu_seconds)
    out["clocks"] = clk.summary()
    out["kernels"] = block_kernel_rooflines(N, Hq, d, ms_step - ms_att, ms_att, flops, t_roof_ms,
                                            out["clocks"], torch.cuda.get_device_properties(dev))
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


FP64_FMA_PER_CLK_SM = 64  # fp64 FMA (vector or mma.sync) per clock per SM, measured on the B200


def block_kernel_rooflines(N, Hq, d, ms_disc, ms_att, att_flops, att_roof_ms, clocks, props):
    """Discovery against its fp64 bound: 16 probes x d FMA per (head, query
    block I, key block J < I); the peak is SMs x 64 fp64 FMA/clk x the SM
    clock sampled during the run.  Attention as in the main roofline."""
    T = (N + 127) // 128
    fma = 16.0 * d * Hq * T * (T - 1) / 2
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    peak = props.multi_processor_count * FP64_FMA_PER_CLK_SM * 2 * mhz * 1e6 / 1e12
    achieved = 2 * fma / (ms_disc * 1e-3) / 1e12
    return {
        "discovery": {"ms": round(ms_disc, 3), "bound": "fp64", "achieved_tflops": round(achieved, 2),
                      "peak_tflops": round(peak, 2), "frac": round(achieved / peak, 4),
                      "peak_source": "SMs x 64 fp64 FMA/clk/SM (measured) x sampled SM clock"},
        "attention": {"ms": round(ms_att, 3), "bound": "tensor",
                      "achieved_tflops": round(att_flops / (ms_att * 1e-3) / 1e12, 2),
                      "frac": round(att_roof_ms / ms_att, 4)},
    }


def block_oracle_sample(w, Qb, Kb, Vb, mask, seconds, seed=0,
                        sets_from="this run's GPU selection"):
    """The fp64 oracle's block-sparse rows on random rows of random heads for
    about `seconds`; effective TFLOP/s by pair count."""
    import oracle
    N, Hq, d = Qb.shape
    T = mask.shape[1]
    bits = np.unpackbits(np.ascontiguousarray(mask).view(np.uint8), bitorder="little")
    bits = bits.reshape(mask.shape[0], T, -1)[:, :, :T].astype(bool)
    rng = np.random.default_rng(seed)
    t_used, p_done, rows_done = 0.0, 0, 0
    while t_used < seconds:
        h = int(rng.integers(0, Hq))
        rows = np.sort(rng.integers(0, N, 32))
        t1 = time.time()
        oracle.attn_block_rows(Qb, Kb, Vb, h, rows, mask)
        t_used += time.time() - t1
        for i in rows:
            I = i // 128
            p_done += 128 * int(bits[h, I, :I].sum()) + (int(i - 128 * I + 1) if bits[h, I, I] else 0)
        rows_done += rows.size
    return {"value": round(4.0 * d * p_done / t_used / 1e12, 6), "unit": UNIT,
            "cores": _cpu_cores(), "kind": "oracle",
            "sample": f"{rows_done} query rows (32 random rows of a random head per draw) of "
                      f"{w.name}, fp64 block-sparse row oracle, {t_used:.1f} s; blocks from "
                      f"{sets_from}"}


def run_blocks_reference(args, w):
    """Reference arm of the block workload: the oracle's own block selection
    (on two heads, for time) and its block-sparse rows, rank 0 only."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    Qb, Kb, Vb = w.qkv()
    heads = [0, w.Hq // 2]
    sel, _ = oracle.block_select(Qb, Kb, w.alpha, heads=heads)
    T = sel.shape[1]
    mask = np.zeros((w.Hq, T, sel.shape[2]), np.uint32)
    mask[heads] = sel
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, last = [], None
    for it in range(args.warmup + args.steps):
        # rows of the two selected heads only (their masks are the oracle's)
        Qs = np.ascontiguousarray(Qb[:, heads])
        Ks = np.ascontiguousarray(Kb[:, [h // (w.Hq // w.Hkv) for h in heads]])
        last = block_oracle_sample(w, Qs, Ks, Vb[:, [h // (w.Hq // w.Hkv) for h in heads]],
                                   mask[heads], per_step, seed=it,
                                   sets_from="the oracle's own block selection (2 heads)")
        if it >= args.warmup:
            vals.append(last["value"])
    value = float(np.mean(vals))
    print(json.dumps({
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "impl": "reference",
        "data": "synthetic (seeded generators shaped like the pages' workloads)",
        "config": block_config(w, world),
        "cpu_baseline": dict(last, value=round(value, 6),
                             sample=last["sample"] + f"; {per_step:.1f} s per step"),
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def main():
    args = parse()
    if args.workload in BLOCK_WORKLOADS:
        wb = BLOCK_WORKLOADS[args.workload]
        if args.impl == "reference":
            run_blocks_reference(args, wb)
        else:
            run_blocks(args, wb)
        return
    if args.workload in BATCH_WORKLOADS:
        if args.impl == "reference":
            run_batch_reference(args, BATCH_WORKLOADS[args.workload])
        else:
            run_batch(args, BATCH_WORKLOADS[args.workload])
        return
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = small_variant(w, args.tokens)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()

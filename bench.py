#!/usr/bin/env python
"""SALA layer-group prefill benchmark on B200 (libsala).

One step = one pass of the whole prefill hot path over one batch of
synthetic input: three linear layers (sala_linear_prefill) and one sparse
layer (sala_sparse_select + sala_sparse_prefill), inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload group_256k]
    python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

Under torchrun (N > 1) every rank runs an independent replica of the
single-GPU workload (the path is single-GPU; no collective on the data
path); value = total tokens over all ranks / max-over-ranks time.  Prints
one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from hybrid_sparse_linear_lightning_b200 import workloads as wl  # noqa: E402

METRIC = "SALA layer-group prefill tokens/s at 256K on 1 B200; % bf16 tensor peak"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------------------- algorithmic work

def sparse_attn_flops(w: wl.Workload, N: int) -> float:
    """4 * d * Hq FLOPs per visible (query, key) pair (QK^T and PV), summed over
    the selected blocks of every query block: a full block gives 64*64 pairs,
    the diagonal block 64*65/2."""
    sp = w.sparse
    nb = N // sp.block
    pairs = 0
    for i in range(nb):
        # blocks attended by query block i: initial + local (overlapping near the
        # start) + min(topk, candidates in [n_init, i - n_local])
        first = min(sp.n_init, i + 1)
        local = max(0, i - max(sp.n_init, i - sp.n_local + 1) + 1)
        n = first + local + min(sp.topk, max(0, i - sp.n_local + 1 - sp.n_init))
        pairs += (n - 1) * sp.block * sp.block + sp.block * (sp.block + 1) // 2
    return float(pairs) * 4 * sp.head_dim * sp.q_heads * w.batch


def linear_bytes(w: wl.Workload, N: int) -> float:
    """Compulsory HBM bytes of one linear layer: Q, K, V, G read, O written."""
    e = 2 if w.dtype == "bf16" else 4
    return 5.0 * w.batch * N * w.linear.heads * w.linear.head_dim * e


def select_bytes(w: wl.Workload, N: int) -> float:
    """Q, K read; Q_norm, K_norm (bf16) written; block tables negligible."""
    sp = w.sparse
    e = 2 if w.dtype == "bf16" else 4
    rows = w.batch * N * (sp.q_heads + sp.kv_heads) * sp.head_dim
    return float(rows * (e + 2))


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        sm, mx, reasons = [], [], set()
        for line in self.tmp.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.tmp.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- our arm

class GroupPrefill:
    """Pre-allocated inputs, outputs and workspaces of one layer group."""

    def __init__(self, w: wl.Workload, N: int, dev, sala, lean: bool = False):
        """lean: one output buffer shared by the linear layers, and the sparse
        layer's normalised Q / K carved out of the linear workspace (the calls
        run in order on one stream), so that the 1M-token group fits in HBM
        with every layer's inputs resident."""
        self.w, self.N, self.dev, self.sala = w, N, dev, sala
        ln, sp = w.linear, w.sparse
        B = w.batch
        self.lin_inputs = []
        for l in range(w.n_linear):
            self.lin_inputs.append(wl.layer_inputs(w, l, dev, seqlen=N))
            torch.cuda.empty_cache()
        self.sp_inputs = wl.layer_inputs(w, w.n_linear, dev, seqlen=N)
        torch.cuda.empty_cache()
        self.lam = torch.tensor(wl.lam_schedule(ln), dtype=torch.float32, device=dev)
        self.wt = wl.rms_weights(ln.head_dim, dev)
        if lean:
            shared = torch.empty_like(self.lin_inputs[0][0])
            self.lin_out = [shared] * w.n_linear
        else:
            self.lin_out = [torch.empty_like(x[0]) for x in self.lin_inputs]
        self.ld = sala.linear_desc(B, N, ln.heads, ln.head_dim, ln.chunk, w.torch_dtype)
        self.sd = sala.sparse_desc(B, N, sp.q_heads, sp.kv_heads, sp.head_dim, sp.block, sp.topk,
                                   sp.n_init, sp.n_local, w.torch_dtype)
        self.lws = sala.workspace(sala.sala_linear_workspace_size(self.ld), dev)
        self.sws = sala.workspace(sala.sala_sparse_workspace_size(self.sd), dev)
        nb = N // sp.block
        nq = B * N * sp.q_heads * sp.head_dim
        nk = B * N * sp.kv_heads * sp.head_dim
        if lean and self.lws.numel() >= 2 * (nq + nk) + 256:
            off = (2 * nq + 255) // 256 * 256
            self.qn = self.lws[:2 * nq].view(torch.bfloat16).view(B, N, sp.q_heads, sp.head_dim)
            self.kn = self.lws[off:off + 2 * nk].view(torch.bfloat16).view(B, N, sp.kv_heads,
                                                                           sp.head_dim)
        else:
            self.qn = torch.empty((B, N, sp.q_heads, sp.head_dim), dtype=torch.bfloat16,
                                  device=dev)
            self.kn = torch.empty((B, N, sp.kv_heads, sp.head_dim), dtype=torch.bfloat16,
                                  device=dev)
        self.kbar = torch.empty((B, nb, sp.kv_heads, sp.head_dim), dtype=torch.float32, device=dev)
        self.idx = torch.empty((B, sp.kv_heads, nb, sala.sala_sparse_index_width(self.sd)),
                               dtype=torch.int32, device=dev)
        self.sp_out = torch.empty_like(self.sp_inputs[0])
        self.timers = None

    def calls(self):
        s = self.sala
        res = []
        for l in range(self.w.n_linear):
            q, k, v, g = self.lin_inputs[l]
            res.append(("linear_prefill", lambda q=q, k=k, v=v, g=g, l=l: s.sala_linear_prefill(
                self.ld, q, k, v, g, self.lam, self.wt, self.wt, None, None, self.lin_out[l],
                self.lws)))
        q, k, v, g = self.sp_inputs
        res.append(("sparse_select", lambda: s.sala_sparse_select(
            self.sd, q, k, self.wt, self.wt, self.qn, self.kn, self.kbar, self.idx, self.sws)))
        res.append(("sparse_prefill", lambda: s.sala_sparse_prefill(
            self.sd, self.qn, self.kn, v, g, self.idx, self.sp_out)))
        return res

    def step(self, timed_calls=None):
        for name, fn in self.calls():
            if timed_calls is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
            st = fn()
            if st != 0:
                raise RuntimeError(f"{name}: {self.sala.status_string(st)}")
            if timed_calls is not None:
                e1.record()
                timed_calls.append((name, e0, e1))


class ShardedGroupPrefill:
    """One rank's head shard of a layer group (``--shard heads``): linear
    heads [lo, hi) of every linear layer and the q heads of its sparse-layer
    shard, with the kv group's block-mean query sums all-reduced over NCCL
    where a group spans several ranks.  Inputs are the rank's slices of the
    seeded full tensors (each drawn in full, sliced, then freed)."""

    def __init__(self, w: wl.Workload, N: int, dev, rank: int, ws: int):
        from hybrid_sparse_linear_lightning_b200 import shard
        ln, sp = w.linear, w.sparse
        self.w, self.N = w, N
        self.grp = shard.ShardedGroup(rank, ws, ln.heads, sp.q_heads, sp.kv_heads,
                                      shard.group_subgroups(ws, sp.kv_heads))
        lo, hi = self.grp.lin
        self.lin_inputs = []
        for l in range(w.n_linear):
            full = wl.layer_inputs(w, l, dev, seqlen=N)
            self.lin_inputs.append([t[:, :, lo:hi].contiguous() for t in full])
            del full
            torch.cuda.empty_cache()
        s_ = self.grp.sp
        full = wl.layer_inputs(w, w.n_linear, dev, seqlen=N)
        self.sp_inputs = [full[0][:, :, s_.q_lo:s_.q_hi].contiguous(),
                          full[1][:, :, s_.kv_lo:s_.kv_hi].contiguous(),
                          full[2][:, :, s_.kv_lo:s_.kv_hi].contiguous(),
                          full[3][:, :, s_.q_lo:s_.q_hi].contiguous()]
        del full
        torch.cuda.empty_cache()
        self.lam = torch.tensor(wl.lam_schedule(ln)[lo:hi], dtype=torch.float32, device=dev)
        self.wt = wl.rms_weights(ln.head_dim, dev)

    def step(self, timed_calls=None):
        w, sp = self.w, self.w.sparse
        for l in range(w.n_linear):
            q, k, v, g = self.lin_inputs[l]
            self.grp.linear(q, k, v, g, self.lam, self.wt, self.wt, chunk=w.linear.chunk)
        q, k, v, g = self.sp_inputs
        self.grp.sparse(q, k, v, g, self.wt, self.wt, block=sp.block, topk=sp.topk,
                        n_init=sp.n_init, n_local=sp.n_local)


def run_sharded(args):
    """Strong scaling: one layer group split by heads over the ranks."""
    rank, ws, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from hybrid_sparse_linear_lightning_b200 import sala
    w = wl.WORKLOADS[args.workload]
    N = args.seqlen or w.seqlen
    grp = ShardedGroupPrefill(w, N, dev, rank, ws)
    for _ in range(args.warmup):
        grp.step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(ws)
    torch.cuda.synchronize()
    l0 = sala.sala_kernel_launch_count()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        grp.step()
    e1.record()
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), ws)
    if sala.sala_get_device_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    value = w.batch * N * args.steps / (ms / 1e3)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic N(0,1) inputs, seeded (no trained weights)",
            "config": dict(config_of(w, N, ws), parallelism=f"heads x{ws}"),
            "gpu_launches": sala.sala_kernel_launch_count() - l0, "clocks": clk}), flush=True)
    if ws > 1:
        dist.destroy_process_group()


KERNEL_SOURCES = {
    "sparse_prefill": "sparse_tc.cuh",
    "linear_prefill": "linear_seg_tc.cuh",
    "sparse_select": "select.cuh",
}


def code_hash(text: str) -> str:
    """Hash of a CUDA source with comments removed and whitespace collapsed,
    so that edits to comments alone keep stored counters valid."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def kernel_source_hash(call: str) -> str:
    path = os.path.join(ROOT, "hybrid_sparse_linear_lightning_b200", "csrc", KERNEL_SOURCES[call])
    with open(path, encoding="utf-8") as f:
        return code_hash(f.read())


def kernel_traffic(workload: str, call: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            tr = json.load(f)
    except (OSError, ValueError):
        return None
    ent = tr.get(workload, {}).get(call)
    if not ent or ent.get("source_sha256_16") != kernel_source_hash(call):
        return None
    return ent.get("dram_bytes_per_launch")


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return rank, ws, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """Max of a per-rank time over all ranks (device tensor under NCCL, host
    tensor under gloo)."""
    if ws <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank_step: int, steps: int, max_ms: float, ws: int) -> float:
    """Whole-job tokens/s of `ws` independent replicas timed by the slowest."""
    return tokens_per_rank_step * ws * steps / (max_ms / 1e3)


CPU_SAMPLE_TOKENS = 4096        # linear layer: tokens of the timed sample (all heads)
CPU_SAMPLE_BLOCKS = 8           # sparse layer: query blocks of the timed sample


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        return len(os.sched_getaffinity(0))


def cpu_baseline_sample(w: wl.Workload):
    """Time the oracle as it stands on one bounded sample of the workload
    (the same sample in both arms of the benchmark).

    Linear part: one linear layer, all heads, over the first
    CPU_SAMPLE_TOKENS tokens (its work per token is constant).  Sparse part:
    the last CPU_SAMPLE_BLOCKS query blocks of a sequence long enough that
    they take the full top-k selection, through the oracle's row form (only
    those blocks' queries are normalised; every key is, as the selection
    needs).  Returns layer-group tokens/s extrapolated by per-token work, the
    thread count, a description and the seconds the sample took.
    """
    import numpy as np
    import oracle
    ln, sp = w.linear, w.sparse
    f64 = lambda t: t.to(torch.float64).numpy()
    T = CPU_SAMPLE_TOKENS
    q, k, v, g = (f64(x) for x in wl.layer_inputs(w, 0, "cpu", seqlen=T))
    lam = np.asarray(wl.lam_schedule(ln))
    wt = np.ones(ln.head_dim)
    t0 = time.perf_counter()
    oracle.linear_layer(q, k, v, g, lam, wt, wt, chunk=ln.chunk)
    t_lin = (time.perf_counter() - t0) / T
    need = (sp.topk + sp.n_init + sp.n_local) * sp.block
    Ns = max(4096, 2 * need)
    nq = CPU_SAMPLE_BLOCKS
    nb = Ns // sp.block
    rows = list(range(nb - nq, nb))
    q, k, v, g = (f64(x) for x in wl.layer_inputs(w, w.n_linear, "cpu", seqlen=Ns))
    cat = lambda x: np.concatenate([x[:, i * sp.block:(i + 1) * sp.block] for i in rows], axis=1)
    t0 = time.perf_counter()
    oracle.sparse_layer_rows(cat(q), cat(g), rows, k, v, wt, wt, block=sp.block, topk=sp.topk,
                             n_init=sp.n_init, n_local=sp.n_local)
    t_sp = (time.perf_counter() - t0) / (nq * sp.block)
    per_token = w.n_linear * t_lin + t_sp
    desc = (f"oracle (numpy fp64) on host cores: linear layer x{w.n_linear} timed on 1 layer x "
            f"{ln.heads} heads x {T} tokens; sparse layer timed on the last {nq} query blocks "
            f"of a {Ns}-token sequence (full top-{sp.topk} selection over every earlier block); "
            f"layer-group tokens/s extrapolated by per-token work")
    return 1.0 / per_token, cpu_threads(), desc, t_lin * T + t_sp * nq * sp.block


def config_of(w: wl.Workload, N: int, ws: int) -> dict:
    """The workload description both arms print."""
    return {"workload": w.name, "seq_len": N, "batch": w.batch,
            "layers": f"{w.n_linear} linear + 1 sparse",
            "heads": w.linear.heads, "kv_heads": w.sparse.kv_heads,
            "head_dim": w.linear.head_dim, "chunk": w.linear.chunk,
            "block": w.sparse.block, "topk": w.sparse.topk,
            "n_init": w.sparse.n_init, "n_local": w.sparse.n_local,
            "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
            "l2": "inputs larger than L2 (no flush needed)"}


def time_group(w: wl.Workload, N: int, dev, sala, steps: int, warmup: int, ws: int = 1,
               lean: bool = False, clocks=None):
    """Warm up, then time `steps` group steps with CUDA events on the
    launching stream (barrier + synchronize on both sides).  Returns the
    GroupPrefill, the max-over-ranks elapsed ms, per-call event times and
    the number of library launches in the timed region."""
    grp = GroupPrefill(w, N, dev, sala, lean=lean)
    torch.cuda.synchronize()
    for _ in range(warmup):
        grp.step()
    torch.cuda.synchronize()
    if sala.sala_get_device_status() != 0:
        raise RuntimeError("device status word set during warm-up")
    if clocks is not None:
        clocks.start()
    barrier(ws)
    torch.cuda.synchronize()
    launches0 = sala.sala_kernel_launch_count()
    timed = []
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        grp.step(timed)
    end.record()
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop() if clocks is not None else None
    launches = sala.sala_kernel_launch_count() - launches0
    elapsed_ms = max_over_ranks(start.elapsed_time(end), ws)
    if sala.sala_get_device_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    per_call = {}
    for name, e0, e1 in timed:
        per_call.setdefault(name, []).append(e0.elapsed_time(e1))
    return grp, elapsed_ms, per_call, launches, clk


def call_rooflines(w: wl.Workload, N: int, per_call: dict, steps: int, peaks: dict) -> dict:
    """Per-call achieved work against the measured peaks.  The calls are
    timed in windows of milliseconds inside a sub-second region, so the
    tensor-bound call is rated against the burst bf16 peak (the sustained
    figure is given beside it)."""
    work = {
        "linear_prefill": ("hbm", linear_bytes(w, N)),
        "sparse_select": ("hbm", select_bytes(w, N)),
        "sparse_prefill": ("tensor", sparse_attn_flops(w, N)),
    }
    calls = {}
    for name, ts in per_call.items():
        avg = sum(ts) / len(ts)
        bound, amount = work[name]
        c = {"ms": round(avg, 4), "launches_per_step": len(ts) // steps, "bound": bound}
        if bound == "hbm":
            ach = amount / (avg / 1e3) / 1e9
            c.update(achieved=round(ach, 2), peak=peaks["hbm_gbs"], unit="GB/s",
                     frac=round(ach / peaks["hbm_gbs"], 4))
        else:
            ach = amount / (avg / 1e3) / 1e12
            c.update(achieved=round(ach, 2), peak=peaks["bf16_tflops"], unit="TFLOP/s",
                     frac=round(ach / peaks["bf16_tflops"], 4),
                     frac_of_sustained=round(ach / peaks["bf16_tflops_sustained"], 4))
        calls[name] = c
    tot = sum(c["ms"] * c["launches_per_step"] for c in calls.values())
    for c in calls.values():
        c["share"] = round(c["ms"] * c["launches_per_step"] / tot, 4)
    return calls


def per_config_entry(w, N, elapsed_ms, steps, per_call, peaks, ws, note=None):
    calls = call_rooflines(w, N, per_call, steps, peaks)
    ms = elapsed_ms / steps
    e = {"workload": w.name, "seq_len": N, "topk": w.sparse.topk, "steps": steps,
         "ms_per_step": round(ms, 4),
         "tokens_per_s": round(replica_throughput(w.batch * N, steps, elapsed_ms, ws), 1),
         "calls": calls}
    if note:
        e["note"] = note
    return e


PER_CONFIG = [("group_32k", 10, False), ("group_128k", 5, False), ("group_1m", 3, True)]

# fp32 FMA throughput of the CUDA cores: 148 SMs x 128 FMA lanes x 2 FLOP x
# 1.965 GHz (unit counts and maximum clock of the B200)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def token_softmax_flops(w: wl.Workload, N: int) -> float:
    """Work of the token-level selection variant: two passes (log-sum-exp,
    then probabilities) of 2 * d FLOP per (query row, candidate block), over
    64 * Hq query rows per query block, for the blocks that rank (fewer
    slots than candidates)."""
    sp = w.sparse
    nb = N // sp.block
    cand = 0
    for i in range(nb):
        n = max(0, i - sp.n_local + 1 - sp.n_init)
        if 0 < min(sp.topk, n) < n:
            cand += n
    return 2.0 * 2 * sp.head_dim * sp.block * sp.q_heads * cand * w.batch


def time_selection_variant(w: wl.Workload, dev, sala, steps: int = 5, warmup: int = 3):
    """sala_sparse_select with SALA_SELECT_TOKEN_SOFTMAX on the workload's
    sparse layer (CUDA events around each call)."""
    sp = w.sparse
    N = w.seqlen
    q, k, _, _ = wl.layer_inputs(w, w.n_linear, dev)
    wt = wl.rms_weights(sp.head_dim, dev)
    d = sala.sparse_desc(w.batch, N, sp.q_heads, sp.kv_heads, sp.head_dim, sp.block, sp.topk,
                         sp.n_init, sp.n_local, w.torch_dtype,
                         selection=sala.SALA_SELECT_TOKEN_SOFTMAX)
    nb = N // sp.block
    outs = (torch.empty_like(q), torch.empty_like(k),
            torch.empty((w.batch, nb, sp.kv_heads, sp.head_dim), dtype=torch.float32, device=dev),
            torch.empty((w.batch, sp.kv_heads, nb, sala.sala_sparse_index_width(d)),
                        dtype=torch.int32, device=dev))
    wsp = sala.workspace(sala.sala_sparse_workspace_size(d), dev)
    for _ in range(warmup):
        assert sala.sala_sparse_select(d, q, k, wt, wt, *outs, wsp) == 0
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        assert sala.sala_sparse_select(d, q, k, wt, wt, *outs, wsp) == 0
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    if sala.sala_get_device_status() != 0:
        raise RuntimeError("device status word set in the selection variant")
    ms = sum(a.elapsed_time(b) for a, b in ts) / steps
    tf = token_softmax_flops(w, N) / (ms / 1e3) / 1e12
    return {"workload": w.name, "selection": "token_softmax", "ms": round(ms, 4),
            "bound": "alu", "achieved": round(tf, 2), "peak": round(FP32_ALU_TFLOPS, 1),
            "unit": "TFLOP/s", "frac": round(tf / FP32_ALU_TFLOPS, 4),
            "peak_source": "fp32 FMA lanes x SMs x max clock (no measured fp32 peak)"}


BLOCK_HIDDEN, BLOCK_FFN = 4096, 16384     # synthetic decoder-block widths (pages give none)


def block_group_gemm_flops(w: wl.Workload, N: int, hidden=BLOCK_HIDDEN, ffn=BLOCK_FFN) -> float:
    """Dense GEMM work of one group of decoder blocks: q, k, v, gate and
    output projections and the SwiGLU FFN (2 FLOP per multiply-add)."""
    ln, sp = w.linear, w.sparse
    d = ln.head_dim
    lin = 2 * hidden * (2 * ln.heads * d + 2 * ln.heads * d) + 2 * ln.heads * d * hidden
    spa = 2 * hidden * (2 * sp.q_heads * d + 2 * sp.kv_heads * d) + 2 * sp.q_heads * d * hidden
    ffn_f = 2 * hidden * 2 * ffn + 2 * ffn * hidden
    return float(w.batch * N) * (w.n_linear * (lin + ffn_f) + spa + ffn_f)


def time_block_group(w: wl.Workload, N: int, dev, sala, peaks, steps=3, warmup=2):
    """A layer group of full decoder blocks (sala_block_prefill x 4) on a
    residual stream x [1, N, 4096] fp32, synthetic weights; CUDA events."""
    ln, sp = w.linear, w.sparse
    d = ln.head_dim
    hidden = ln.heads * d
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    bufs = [torch.randn((w.batch, N, hidden), generator=gen, device=dev), None]
    bufs[1] = torch.empty_like(bufs[0])
    bd = sala.BlockDesc(hidden, BLOCK_FFN, 1e-6)
    ld = sala.linear_desc(w.batch, N, ln.heads, d, ln.chunk, w.torch_dtype)
    sd = sala.sparse_desc(w.batch, N, sp.q_heads, sp.kv_heads, d, sp.block, sp.topk, sp.n_init,
                          sp.n_local, w.torch_dtype)
    layers = []
    for l in range(w.n_linear + 1):
        kind_lin = l < w.n_linear
        wt = wl.block_weights(hidden, BLOCK_FFN, ln.heads if kind_lin else sp.q_heads,
                              ln.heads if kind_lin else sp.kv_heads, d, l, dev, seed=w.seed)
        layers.append((ld if kind_lin else None, None if kind_lin else sd, wt, sala.block_weights(wt)))
    ws = sala.workspace(max(sala.sala_block_workspace_size(bd, a, b) for a, b, _, _ in layers), dev)
    lam = torch.tensor(wl.lam_schedule(ln), dtype=torch.float32, device=dev)

    def step():
        for l, (a, b, _, bw) in enumerate(layers):
            st = sala.sala_block_prefill(bd, a, b, bw, lam if a is not None else None,
                                         bufs[l % 2], bufs[(l + 1) % 2], None, ws)
            if st != 0:
                raise RuntimeError("sala_block_prefill: " + sala.status_string(st))

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    if sala.sala_get_device_status() != 0:
        raise RuntimeError("device status word set in the block group")
    ms = e0.elapsed_time(e1) / steps
    gemm = block_group_gemm_flops(w, N) / (ms / 1e3) / 1e12
    return {"workload": w.name, "seq_len": N, "hidden": hidden, "ffn": BLOCK_FFN,
            "ms_per_step": round(ms, 3), "tokens_per_s": round(w.batch * N / (ms / 1e3), 1),
            "gemm_tflops_over_step": round(gemm, 1),
            "gemm_frac_of_burst_bf16": round(gemm / peaks["bf16_tflops"], 4),
            "note": "3 linear + 1 sparse decoder blocks, synthetic weights; GEMMs in cuBLASLt"}


def run_ours(args):
    rank, ws, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from hybrid_sparse_linear_lightning_b200 import sala
    w = wl.WORKLOADS[args.workload]
    N = args.seqlen or w.seqlen
    peaks, peak_kind = load_peaks()
    clocks = ClockSampler(local)
    grp, elapsed_ms, per_call, launches, clk = time_group(w, N, dev, sala, args.steps,
                                                          args.warmup, ws, clocks=clocks)
    ms_per_step = elapsed_ms / args.steps
    value = replica_throughput(w.batch * N, args.steps, elapsed_ms, ws)
    calls = call_rooflines(w, N, per_call, args.steps, peaks)
    dom = max(calls, key=lambda n: calls[n]["share"])
    traffic = kernel_traffic(args.workload, dom)
    d = calls[dom]
    roofline = {"bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"],
                "unit": d["unit"], "frac": d["frac"], "traffic": traffic, "kernel": dom,
                "peak_source": f"{peak_kind} ({'burst bf16' if d['bound'] == 'tensor' else 'HBM copy'})"}
    if "frac_of_sustained" in d:
        roofline["frac_of_sustained"] = d["frac_of_sustained"]

    # end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(grp, args, ws)
    del grp
    torch.cuda.empty_cache()

    # the other layer-group workloads (parity cases at their own sizes)
    per_config = {w.name: per_config_entry(w, N, elapsed_ms, args.steps, per_call, peaks, ws)}
    if not args.no_per_config:
        for name, steps, lean in PER_CONFIG:
            if name == w.name:
                continue
            wc = wl.WORKLOADS[name]
            g2, el, pc, _, _ = time_group(wc, wc.seqlen, dev, sala, steps, 3, ws, lean=lean)
            del g2
            torch.cuda.empty_cache()
            note = ("one output buffer shared by the three linear layers and the sparse "
                    "layer's normalised Q/K in the linear workspace (memory)") if lean else None
            per_config[name] = per_config_entry(wc, wc.seqlen, el, steps, pc, peaks, ws, note)

    variants = None
    if not args.no_per_config:
        variants = [time_selection_variant(wl.WORKLOADS["group_32k"], dev, sala)]
        torch.cuda.empty_cache()

    blocks = None
    if not args.no_blocks:
        blocks = []
        for name in ("group_32k", "group_256k"):
            blocks.append(time_block_group(wl.WORKLOADS[name], wl.WORKLOADS[name].seqlen, dev,
                                           sala, peaks))
            torch.cuda.empty_cache()

    dec = None
    if args.decode_steps > 0:
        dec = run_decode(wl.WORKLOADS["group_1m"], args.decode_steps, dev, sala, peaks, ws)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        vals, threads, desc, secs = [], 1, "", 0.0
        for _ in range(args.cpu_samples):
            v, threads, desc, s_ = cpu_baseline_sample(w)
            vals.append(v)
            secs += s_
        cpu = {"value": round(len(vals) / sum(1.0 / v for v in vals), 2), "unit": UNIT,
               "cores": threads, "kind": "oracle",
               "sample": desc + f"; {len(vals)} samples, harmonic mean",
               "sample_seconds": round(secs, 2)}

    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic N(0,1) inputs, seeded (no trained weights)",
            "config": config_of(w, N, ws),
            "roofline": roofline, "calls": calls,
            "tensor_frac_of_step": round(sparse_attn_flops(w, N) / (ms_per_step / 1e3) / 1e12
                                         / peaks["bf16_tflops"], 4),
            "e2e": e2e, "gpu_launches": launches, "clocks": clk, "cpu_baseline": cpu,
            "per_config": per_config, "selection_variants": variants, "blocks": blocks,
            "decode": dec,
        }
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def decode_bytes(w: wl.Workload, cur_len: int) -> float:
    """Compulsory HBM bytes of one decode step at cache length cur_len:
    linear states read + written, the complete blocks' key means read, the
    selected blocks' keys and values read (dominant terms)."""
    ln, sp = w.linear, w.sparse
    st = 2.0 * w.n_linear * w.batch * ln.heads * ln.head_dim * ln.head_dim * 4
    nb = cur_len // sp.block
    kb = float(w.batch * nb * sp.kv_heads * sp.head_dim * 4)
    sel = min(nb + 1, sp.topk + sp.n_init + sp.n_local)
    kv = float(w.batch * sp.kv_heads * sel * sp.block * sp.head_dim * 2 * 2)
    return st + kb + kv


def run_decode(w: wl.Workload, steps: int, dev, sala, peaks, ws):
    """Prefill the 1M-token group layer by layer (keeping only the linear
    states and the sparse layer's key / value caches), then time `steps`
    decode tokens through the C ABI with CUDA events: replayed from a CUDA
    graph (the device time of the step), and launched one call at a time
    from Python (host-bound)."""
    N = w.seqlen
    ln, sp = w.linear, w.sparse
    B, H, D = w.batch, ln.heads, ln.head_dim
    # room for the warm-up tokens, the graph-timed steps and up to 64 eager steps
    cap = N + ((steps + 64 + 3 + sp.block - 1) // sp.block + 1) * sp.block
    lam = torch.tensor(wl.lam_schedule(ln), dtype=torch.float32, device=dev)
    wt = wl.rms_weights(D, dev)
    states = []
    for l in range(w.n_linear):
        q, k, v, g = wl.layer_inputs(w, l, dev)
        out, st = sala.linear_prefill(q, k, v, g, lam, wt, wt, chunk=ln.chunk, want_state=True)
        states.append(st)
        del q, k, v, g, out
        torch.cuda.empty_cache()
    q, k, v, g = wl.layer_inputs(w, w.n_linear, dev)
    k_cache = torch.zeros((B, cap, sp.kv_heads, D), dtype=torch.bfloat16, device=dev)
    v_cache = torch.zeros_like(k_cache)
    kbar = torch.zeros((B, cap // sp.block, sp.kv_heads, D), dtype=torch.float32, device=dev)
    ksum = torch.zeros((B, sp.kv_heads, D), dtype=torch.float32, device=dev)
    qn, kn, kb, idx = sala.sparse_select(q, k, wt, wt, block=sp.block, topk=sp.topk,
                                         n_init=sp.n_init, n_local=sp.n_local)
    k_cache[:, :N] = kn
    v_cache[:, :N] = v
    kbar[:, :N // sp.block] = kb
    del q, k, v, g, qn, kn, kb, idx
    torch.cuda.empty_cache()
    ld = sala.linear_desc(B, 64, H, D, ln.chunk, w.torch_dtype)
    sd = sala.sparse_desc(B, 64, sp.q_heads, sp.kv_heads, D, sp.block, sp.topk, sp.n_init,
                          sp.n_local, w.torch_dtype)
    dd = sala.DecodeDesc(ld, sd, w.n_linear, cap)
    wsd = sala.workspace(sala.sala_decode_workspace_size(dd), dev)
    toks = [wl.decode_inputs(w, s, dev) for s in range(steps + 3)]
    outs = [torch.empty_like(t[0]) for t in toks[0]]
    ios = [sala.make_decode_io(t, outs, states, [lam] * w.n_linear, wt, wt) for t in toks]

    def step(s, pos):
        r = sala.sala_decode_step(dd, ios[s], k_cache, v_cache, kbar, ksum, pos, wsd)
        if r != 0:
            raise RuntimeError("decode: " + sala.status_string(r))

    for s in range(3):                       # warm-up tokens
        step(s, N + s)
    torch.cuda.synchronize()
    if sala.sala_get_device_status() != 0:
        raise RuntimeError("device status word set during decode warm-up")
    # The timed steps are captured into one CUDA graph (each step's launches
    # with its own token position and buffers) and replayed, so the per-step
    # host call overhead is not part of the device time.
    base = N + 3
    graph = None
    try:
        cs = torch.cuda.Stream()
        cs.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cs):
            for s in range(steps):
                step(s + 3, base + s)
    except RuntimeError as e:               # capture not available: time eager launches
        graph = None
        print(f"decode: graph capture failed ({e}); timing eager launches", file=sys.stderr)
        torch.cuda.synchronize()
    l0 = sala.sala_kernel_launch_count()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    if graph is not None:
        graph.replay()
    else:
        for s in range(steps):
            step(s + 3, base + s)
    e1.record()
    torch.cuda.synchronize()
    if sala.sala_get_device_status() != 0:
        raise RuntimeError("device status word set during decode")
    ms = max_over_ranks(e0.elapsed_time(e1), ws)
    launches = (sala.sala_kernel_launch_count() - l0) if graph is None else None
    # the same steps launched one call at a time from Python (host-bound figure)
    # need the caches rolled back: time them on the next positions instead
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    n_eager = min(steps, 64)
    e2.record()
    for s in range(n_eager):
        step(s + 3, base + steps + s)
    e3.record()
    torch.cuda.synchronize()
    eager_us = e2.elapsed_time(e3) * 1e3 / n_eager
    us = ms * 1e3 / steps
    byts = sum(decode_bytes(w, base + s) for s in range(steps)) / steps
    gbs = byts / (us * 1e-6) / 1e9
    return {"workload": w.name, "context": N, "steps": steps, "us_per_step": round(us, 2),
            "timing": "CUDA graph of the timed steps" if graph is not None else "eager launches",
            "eager_us_per_step": round(eager_us, 2),
            "tokens_per_s": round(ws * 1e6 / us, 1), "bytes_per_step": int(byts),
            "achieved_GBps": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
            "launches_per_step": 1,
            "launches_counted": launches}


def run_e2e(grp: GroupPrefill, args, ws):
    """Same step through the C ABI with host buffers: every layer's inputs
    are copied from pinned host memory and every layer's output read back
    inside the timed region.  Copies run on two side streams so that the
    host-to-device copy of layer l+1 and the read-back of layer l-1 overlap
    the computation of layer l (PCIe is full duplex); events order each
    buffer's reuse across layers and steps."""
    w, N = grp.w, grp.N
    host_in = []
    for tens in grp.lin_inputs + [grp.sp_inputs]:
        host_in.append([t.to("cpu").pin_memory() for t in tens])
    host_out = [o.to("cpu").pin_memory() for o in grp.lin_out + [grp.sp_out]]
    dev_in = grp.lin_inputs + [grp.sp_inputs]
    dev_out = grp.lin_out + [grp.sp_out]
    h2d = sum(t.numel() * t.element_size() for ts in host_in for t in ts)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    steps = max(1, min(args.steps, args.e2e_steps))
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    calls = grp.calls()
    # layer l = calls of linear layer l; the sparse layer is select + prefill
    layers = [[c] for c in calls[:w.n_linear]] + [calls[w.n_linear:]]
    n = len(layers)
    read_done = [None] * n      # compute finished reading layer l's inputs
    out_done = [None] * n       # read-back of layer l's output finished

    def one():
        ev_in = []
        for l in range(n):
            with torch.cuda.stream(s_in):
                if read_done[l] is not None:
                    s_in.wait_event(read_done[l])
                for h, d in zip(host_in[l], dev_in[l]):
                    d.copy_(h, non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_in)
                ev_in.append(e)
        for l in range(n):
            comp.wait_event(ev_in[l])
            if out_done[l] is not None:
                comp.wait_event(out_done[l])
            for name, fn in layers[l]:
                st = fn()
                if st != 0:
                    raise RuntimeError(f"{name}: {grp.sala.status_string(st)}")
            e = torch.cuda.Event()
            e.record(comp)
            read_done[l] = e
            with torch.cuda.stream(s_out):
                s_out.wait_event(e)
                host_out[l].copy_(dev_out[l], non_blocking=True)
                e2 = torch.cuda.Event()
                e2.record(s_out)
                out_done[l] = e2

    one()
    torch.cuda.synchronize()
    barrier(ws)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(comp)
    s_in.wait_event(s)
    for _ in range(steps):
        one()
    comp.wait_stream(s_out)
    e.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), ws)
    barrier(ws)
    return {"value": round(w.batch * N * ws * steps / (ms / 1e3), 1), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "overlap": "H2D of layer l+1 and D2H of layer l-1 overlap layer l"}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    N = args.seqlen or w.seqlen
    for _ in range(args.warmup):
        cpu_baseline_sample(w)
    vals, secs = [], 0.0
    threads, desc = 1, ""
    for _ in range(args.steps):
        v, threads, desc, s = cpu_baseline_sample(w)
        vals.append(v)
        secs += s
    value = len(vals) / sum(1.0 / v for v in vals)
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT,
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        # time the oracle would take for one whole step (extrapolated by work)
        "warmup": args.warmup, "ms_per_step": round(w.batch * N / value * 1e3, 1),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic N(0,1) inputs, seeded (no trained weights)",
        "config": config_of(w, N, 1),
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": threads,
                         "kind": "oracle", "sample": desc + "; one sample per step",
                         "sample_seconds": round(secs, 2)},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="group_256k", choices=list(wl.WORKLOADS))
    ap.add_argument("--seqlen", type=int, default=0, help="override the workload length")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-samples", type=int, default=4,
                    help="oracle samples timed for cpu_baseline (a few seconds each)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other layer-group workloads")
    ap.add_argument("--no-blocks", action="store_true",
                    help="skip timing the full decoder-block groups")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="replicas: one independent group per GPU (weak scaling); heads: one "
                         "group split by heads over the GPUs (strong scaling)")
    ap.add_argument("--decode-steps", type=int, default=256,
                    help="decode tokens timed after a 1M-token prefill (0: skip)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.shard == "heads":
        run_sharded(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

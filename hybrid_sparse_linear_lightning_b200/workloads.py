"""Workload definitions and seeded synthetic inputs.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds only shapes, parameters and random-number draws: no arithmetic of the
attention method lives here.

The five workloads follow the pages' usage: a SALA layer group is three
linear (Lightning-style) layers and one sparse (InfLLM-V2-style) layer, the
1:3 sparse:linear mix of the MiniCPM-SALA paper (section 2.1); 256K tokens is
the length of the paper's 3.5x time-to-first-token comparison and 1M tokens
the longest context it runs.  Inputs are synthetic: Q, K, V and the gate are
i.i.d. N(0, 1) (no trained projections exist), RMSNorm weights are 1.

Seeding: the tensors of layer ``l`` of a workload with seed ``s`` are drawn in
the order Q, K, V, G from a ``torch.Generator`` seeded with ``s * 100 + l`` on
the device where they are made, as fp32, then cast to the workload dtype.
Consumers that compare two computations always copy the same generated
tensors, so the two sides see identical bits.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class LinearShape:
    heads: int
    head_dim: int
    chunk: int
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    scale: float = 1.0
    lam_kind: str = "schedule"      # "const", "schedule" or "half_one"
    lam_const: float = 0.99


@dataclasses.dataclass(frozen=True)
class SparseShape:
    q_heads: int
    kv_heads: int
    head_dim: int
    block: int
    topk: int
    n_init: int
    n_local: int
    rms_eps: float = 1e-6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    batch: int
    seqlen: int
    dtype: str                  # "f32" or "bf16"
    n_linear: int
    linear: LinearShape
    sparse: SparseShape
    salient_key_frac: float = 0.0   # fraction of key rows scaled by salient_key_mult
    salient_key_mult: float = 8.0
    decode_steps: int = 0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


def lam_schedule(shape: LinearShape) -> List[float]:
    """Per-head decay factors of a linear layer (an input of the workload).

    "schedule": lam_h = 1 - 2^(-5 - h/4) (real division), h = 0..H-1.
    "half_one": heads h >= H/2 use lam = 1, the others the schedule.
    "const": every head uses ``lam_const``.
    """
    H = shape.heads
    if shape.lam_kind == "const":
        return [float(shape.lam_const)] * H
    sched = [1.0 - 2.0 ** (-5.0 - h / 4.0) for h in range(H)]
    if shape.lam_kind == "half_one":
        return [1.0 if h >= H // 2 else sched[h] for h in range(H)]
    return sched


_LIN128 = LinearShape(heads=32, head_dim=128, chunk=64)

WORKLOADS = {
    # Tiny correctness case: one linear + one sparse layer, fp32, seed 0.
    "tiny_2k_f32": Workload(
        name="tiny_2k_f32", seed=0, batch=1, seqlen=2048, dtype="f32", n_linear=1,
        linear=LinearShape(heads=4, head_dim=64, chunk=64, lam_kind="const", lam_const=0.99),
        sparse=SparseShape(q_heads=4, kv_heads=1, head_dim=64, block=64, topk=4, n_init=1,
                           n_local=2)),
    # One layer group at 32K tokens.
    "group_32k": Workload(
        name="group_32k", seed=1, batch=1, seqlen=32768, dtype="bf16", n_linear=3,
        linear=_LIN128,
        sparse=SparseShape(q_heads=32, kv_heads=2, head_dim=128, block=64, topk=16, n_init=1,
                           n_local=2)),
    # 128K tokens, half the linear heads with lam = 1, 1% salient key rows.
    "group_128k": Workload(
        name="group_128k", seed=2, batch=1, seqlen=131072, dtype="bf16", n_linear=3,
        linear=dataclasses.replace(_LIN128, lam_kind="half_one"),
        sparse=SparseShape(q_heads=32, kv_heads=2, head_dim=128, block=64, topk=32, n_init=1,
                           n_local=2),
        salient_key_frac=0.01),
    # 256K tokens: the length of the pages' time-to-first-token comparison.
    "group_256k": Workload(
        name="group_256k", seed=3, batch=1, seqlen=262144, dtype="bf16", n_linear=3,
        linear=_LIN128,
        sparse=SparseShape(q_heads=32, kv_heads=2, head_dim=128, block=64, topk=64, n_init=1,
                           n_local=4)),
    # 1M tokens, then 256 decode steps.
    "group_1m": Workload(
        name="group_1m", seed=4, batch=1, seqlen=1048576, dtype="bf16", n_linear=3,
        linear=_LIN128,
        sparse=SparseShape(q_heads=32, kv_heads=2, head_dim=128, block=64, topk=64, n_init=1,
                           n_local=4),
        decode_steps=256),
}

WORKLOAD_ORDER = ["tiny_2k_f32", "group_32k", "group_128k", "group_256k", "group_1m"]


def with_seqlen(w: Workload, seqlen: int, name: Optional[str] = None) -> Workload:
    """Same workload at another sequence length (parity cases at reduced size)."""
    return dataclasses.replace(w, seqlen=seqlen, name=name or f"{w.name}@{seqlen}")


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def layer_inputs(w: Workload, layer: int, device="cpu", seqlen: Optional[int] = None,
                 batch: Optional[int] = None):
    """Q, K, V, G of layer ``layer`` (0..n_linear-1 linear, n_linear = sparse).

    Shapes [B, N, heads, d] (K and V use the kv heads in the sparse layer),
    drawn N(0, 1) in fp32 in the order Q, K, V, G, then cast to the workload
    dtype.  When the workload asks for salient keys, a Bernoulli mask per
    (batch, token, kv head) from a second generator (seed 1 + 100 * layer)
    multiplies those key rows by ``salient_key_mult``.
    """
    N = seqlen or w.seqlen
    B = batch or w.batch
    g = _gen(device, w.seed * 100 + layer)
    if layer < w.n_linear:
        hq = hk = w.linear.heads
        d = w.linear.head_dim
    else:
        hq, hk, d = w.sparse.q_heads, w.sparse.kv_heads, w.sparse.head_dim
    dt = w.torch_dtype
    out = []
    # each tensor is cast as soon as it is drawn (same values as drawing all
    # four first: the draws come from one generator in the same order), so
    # at most one fp32 tensor is alive at a time
    for which, heads in enumerate((hq, hk, hk, hq)):
        t = torch.randn((B, N, heads, d), generator=g, device=device, dtype=torch.float32)
        if which == 1 and w.salient_key_frac > 0:
            g2 = _gen(device, 1 + 100 * layer)
            mask = torch.rand((B, N, hk, 1), generator=g2, device=device) < w.salient_key_frac
            t = torch.where(mask, t * w.salient_key_mult, t)
        out.append(t.to(dt))
        del t
    return out


def decode_inputs(w: Workload, step: int, device="cpu"):
    """Per-layer one-token inputs of decode step ``step``: a list over layers
    of (q, k, v, g), each [B, heads, d], drawn N(0, 1) from a generator seeded
    with ``w.seed * 100000 + 1000 + step``."""
    g = _gen(device, w.seed * 100000 + 1000 + step)
    res = []
    for layer in range(w.n_linear + 1):
        if layer < w.n_linear:
            hq = hk = w.linear.heads
            d = w.linear.head_dim
        else:
            hq, hk, d = w.sparse.q_heads, w.sparse.kv_heads, w.sparse.head_dim
        ts = [torch.randn((w.batch, h, d), generator=g, device=device, dtype=torch.float32)
              .to(w.torch_dtype) for h in (hq, hk, hk, hq)]
        res.append(ts)
    return res


def rms_weights(d: int, device="cpu"):
    """RMSNorm weights of every workload: all ones (no trained weights)."""
    return torch.ones(d, dtype=torch.float32, device=device)


def block_weights(hidden: int, ffn: int, q_heads: int, kv_heads: int, head_dim: int, layer: int,
                  device="cpu", seed: int = 0):
    """Synthetic weights of one decoder block (no trained weights exist):
    bf16 projections in the [out, in] layout drawn N(0, 1) / sqrt(in) from a
    generator seeded with ``seed * 100 + 50 + layer`` (in the order wq, wk, wv,
    wg, wo, w13, w2), all-ones norms.  The sub-block outputs are then of the
    residual stream's order of magnitude."""
    g = _gen(device, seed * 100 + 50 + layer)

    def lin(out, inp):
        return (torch.randn((out, inp), generator=g, device=device) / inp ** 0.5).to(torch.bfloat16)
    w = {"wq": lin(q_heads * head_dim, hidden), "wk": lin(kv_heads * head_dim, hidden),
         "wv": lin(kv_heads * head_dim, hidden), "wg": lin(q_heads * head_dim, hidden),
         "wo": lin(hidden, q_heads * head_dim), "w13": lin(2 * ffn, hidden), "w2": lin(hidden, ffn)}
    ones = lambda n: torch.ones(n, dtype=torch.float32, device=device)
    w.update(norm_attn=ones(hidden), norm_ffn=ones(hidden), qk_norm_q=ones(head_dim),
             qk_norm_k=ones(head_dim))
    return w

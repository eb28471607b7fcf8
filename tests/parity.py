"""Shared helpers of the GPU parity tests: run libsala and the oracle on the
same seeded inputs and compare.  Tolerance for floating outputs:
max|gpu - oracle| / max|oracle| <= 1e-2 (bf16 operands, fp32 accumulation).
Block indices must be identical to the oracle's (ranked in fp64) except
inside the tie window: a block may differ only when its oracle score lies
within 1e-3 * max(|s_k|, |s_k+1|) (+ 1e-6 * row max |s|) of the k-th
selected candidate's score s_k.  Attention outputs are compared on every
checked row, against the oracle's attention over the GPU's own index list
(validated first), so rows that differ inside the tie window are checked
too."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from hybrid_sparse_linear_lightning_b200 import workloads as wl

TOL = 1e-2
TIE_REL = 1e-3
TIE_ABS_FRAC = 1e-6


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(got, ref, mask=None) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if mask is None:
        mask = np.isfinite(ref)
    d = np.abs(got[mask] - ref[mask])
    assert np.all(np.isfinite(got[mask])), "non-finite GPU output"
    return float(d.max() / max(np.abs(ref[mask]).max(), 1e-30))


def _check_row(gr, rr, s, i, topk, n_init, n_local, where):
    """One index row of query block i: GPU list gr, oracle list rr, oracle
    scores s (fp64, over all blocks).  Returns 1 if the two differ inside the
    tie window, 0 if identical; raises AssertionError otherwise."""
    gr = [int(j) for j in gr]
    rr = [int(j) for j in rr]
    n = oracle.selected_count(i, topk, n_init, n_local)
    assert all(j == -1 for j in gr[n:]), (where, gr)
    sel = gr[:n]
    assert sel == sorted(set(sel)) and all(0 <= j <= i for j in sel), (where, gr)
    if gr == rr:
        return 0
    s = np.asarray(s, np.float64)
    cand = np.arange(n_init, i - n_local + 1)
    cs = np.sort(s[cand])[::-1]
    kk = min(topk, len(cand))
    sk = cs[kk - 1]
    sk1 = cs[kk] if kk < len(cand) else sk
    win = TIE_REL * max(abs(sk), abs(sk1)) + TIE_ABS_FRAC * np.abs(cs).max()
    for j in set(gr[:n]) ^ set(rr[:n]):
        assert abs(s[j] - sk) <= win, (where, j, s[j], sk, win)
    return 1


def check_index_rows(gpu_idx, ref_idx, scores, topk, n_init, n_local, rows=None):
    """Compare index rows [B, Hkv, nb, W] (scores [B, Hkv, nb, nb]); returns
    the number of rows that differed inside the tie window."""
    B, Hkv, nb, W = ref_idx.shape
    rows = range(nb) if rows is None else rows
    return sum(_check_row(gpu_idx[b, g, i], ref_idx[b, g, i], scores[b, g, i], i, topk, n_init,
                          n_local, (b, g, i))
               for b in range(B) for g in range(Hkv) for i in rows)


def check_index_subset(gpu_idx_rows, ref_idx_rows, scores_rows, rows, topk, n_init, n_local):
    """The same for row-subset arrays: gpu_idx_rows / ref_idx_rows
    [B, Hkv, R, W] and scores_rows [B, Hkv, R, nb] of query blocks ``rows``."""
    B, Hkv = ref_idx_rows.shape[:2]
    return sum(_check_row(gpu_idx_rows[b, g, r], ref_idx_rows[b, g, r], scores_rows[b, g, r], i,
                          topk, n_init, n_local, (b, g, i))
               for b in range(B) for g in range(Hkv) for r, i in enumerate(rows))


def lam_tensor(w: wl.Workload, device):
    return torch.tensor(wl.lam_schedule(w.linear), dtype=torch.float32, device=device)


def block_rows(t: torch.Tensor, rows, block=64) -> np.ndarray:
    """Tokens of query blocks ``rows`` of a [B, N, H, d] device tensor, in that
    order, as fp64 [B, R*block, H, d] (copied block by block)."""
    return np.concatenate([f64(t[:, i * block:(i + 1) * block]) for i in rows], axis=1)

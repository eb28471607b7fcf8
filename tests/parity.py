"""Shared helpers of the GPU parity tests: run libsala and the oracle on the
same seeded inputs and compare.  Tolerance for floating outputs:
max|gpu - oracle| / max|oracle| <= 1e-2 (bf16 operands, fp32 accumulation).
Block indices must be identical except inside the tie window: a block may
differ only when its oracle score lies within 1e-3 * max(|s_k|, |s_k+1|)
(+ 1e-6 * row max |s|) of the k-th selected candidate's score s_k."""
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


def check_index_rows(gpu_idx, ref_idx, scores, topk, n_init, n_local, rows=None):
    """Compare index rows [B, Hkv, nb, W]; returns the number of rows that
    differed inside the tie window.  Raises AssertionError otherwise."""
    B, Hkv, nb, W = ref_idx.shape
    rows = range(nb) if rows is None else rows
    n_tie = 0
    for b in range(B):
        for g in range(Hkv):
            for i in rows:
                gr = [int(j) for j in gpu_idx[b, g, i]]
                rr = [int(j) for j in ref_idx[b, g, i]]
                n = oracle.selected_count(i, topk, n_init, n_local)
                assert all(j == -1 for j in gr[n:]), (b, g, i, gr)
                sel = gr[:n]
                assert sel == sorted(set(sel)) and all(0 <= j <= i for j in sel), (b, g, i, gr)
                if gr == rr:
                    continue
                # differ: only inside the tie window of the k-th candidate score
                s = np.asarray(scores[b, g, i], np.float64)
                cand = np.arange(n_init, i - n_local + 1)
                cs = np.sort(s[cand])[::-1]
                kk = min(topk, len(cand))
                sk = cs[kk - 1]
                sk1 = cs[kk] if kk < len(cand) else sk
                win = TIE_REL * max(abs(sk), abs(sk1)) + TIE_ABS_FRAC * np.abs(cs).max()
                diff = set(gr[:n]) ^ set(rr[:n])
                for j in diff:
                    assert abs(s[j] - sk) <= win, (b, g, i, j, s[j], sk, win)
                n_tie += 1
    return n_tie


def lam_tensor(w: wl.Workload, device):
    return torch.tensor(wl.lam_schedule(w.linear), dtype=torch.float32, device=device)

"""The algorithmic work bench.py divides by, checked against independent
counts: visible (query, key) pairs of the sparse layer counted from the
oracle's own index lists on small inputs, and the source hash that keys the
stored DRAM counters."""
import numpy as np
import pytest

import bench
import oracle
from hybrid_sparse_linear_lightning_b200 import workloads as wl


def _visible_pairs(idx, block):
    """Count (query, key) pairs a causal block-sparse layer attends to, from
    index lists [B, Hkv, nb, width] (one kv head is enough: all share it)."""
    nb = idx.shape[2]
    pairs = 0
    for i in range(nb):
        for j in idx[0, 0, i]:
            if j < 0:
                continue
            pairs += block * (block + 1) // 2 if j == i else block * block
    return pairs


@pytest.mark.parametrize("topk,n_init,n_local,nb", [(4, 1, 2, 24), (64, 1, 4, 80), (3, 2, 3, 9),
                                                    (0, 1, 1, 7)])
def test_sparse_flops_match_selected_blocks(topk, n_init, n_local, nb):
    import dataclasses
    w = wl.WORKLOADS["tiny_2k_f32"]
    sp = dataclasses.replace(w.sparse, topk=topk, n_init=n_init, n_local=n_local)
    w = dataclasses.replace(w, sparse=sp, batch=1)
    N = nb * sp.block
    rng = np.random.default_rng(3)
    d = sp.head_dim
    q = rng.standard_normal((1, N, sp.q_heads, d))
    k = rng.standard_normal((1, N, sp.kv_heads, d))
    ones = np.ones(d)
    _, _, _, idx, _ = oracle.sparse_select(q, k, ones, ones, block=sp.block, topk=topk,
                                           n_init=n_init, n_local=n_local)
    pairs = _visible_pairs(idx, sp.block)
    assert bench.sparse_attn_flops(w, N) == pairs * 4 * d * sp.q_heads


def test_linear_and_select_bytes():
    w = wl.WORKLOADS["group_256k"]
    N = w.seqlen
    assert bench.linear_bytes(w, N) == 5 * N * 32 * 128 * 2
    assert bench.select_bytes(w, N) == N * (32 + 2) * 128 * (2 + 2)


def test_code_hash_ignores_comments_only():
    a = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    b = "/* doc */ int f(int x) {\n  // comment\n  return x + 1;\n}\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench.code_hash(a) == bench.code_hash(b)
    assert bench.code_hash(a) != bench.code_hash(c)

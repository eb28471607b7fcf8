"""Full-size parity in the benchmark's launch configuration (256K-token layer
group, 1M-token decode context), checked on outputs the oracle can afford:
whole heads of a linear layer, sampled query blocks of the sparse layer, and
single decode tokens against a 1M-token cache."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_sparse_linear_lightning_b200 import workloads as wl
from tests.parity import TOL, check_index_rows, f64, lam_tensor, rel_err

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def sala(cuda_device):
    from hybrid_sparse_linear_lightning_b200 import sala as s
    return s


def test_linear_256k_whole_heads(sala):
    """Linear layer at 262144 tokens, 32 heads: heads 0 (fastest decay) and
    31 (slowest) over the whole sequence, outputs and final state."""
    dev = torch.device("cuda")
    w = wl.WORKLOADS["group_256k"]
    q, k, v, g = wl.layer_inputs(w, 0, dev)
    lam = lam_tensor(w, dev)
    wt = wl.rms_weights(128, dev)
    out, st = sala.linear_prefill(q, k, v, g, lam, wt, wt, chunk=w.linear.chunk, want_state=True)
    torch.cuda.synchronize()
    assert sala.sala_get_device_status() == 0
    heads = [0, 31]
    sub = lambda t: f64(t[:, :, heads])
    ref, S = oracle.linear_layer(sub(q), sub(k), sub(v), sub(g), f64(lam)[heads], f64(wt), f64(wt),
                                 chunk=w.linear.chunk)
    assert rel_err(sub(out), ref) <= TOL
    assert rel_err(f64(st[:, heads]), S) <= TOL


def test_sparse_256k_sampled_blocks(sala):
    """Sparse layer at 262144 tokens (4096 blocks, top-64 + 1 + 4): the
    selection and the output of 24 query blocks (first, last and random)."""
    dev = torch.device("cuda")
    w = wl.WORKLOADS["group_256k"]
    sp = w.sparse
    q, k, v, g = wl.layer_inputs(w, w.n_linear, dev)
    wt = wl.rms_weights(128, dev)
    qn, kn, kbar, idx = sala.sparse_select(q, k, wt, wt, block=sp.block, topk=sp.topk,
                                           n_init=sp.n_init, n_local=sp.n_local)
    out = sala.sparse_prefill(qn, kn, v, g, idx, block=sp.block, topk=sp.topk, n_init=sp.n_init,
                              n_local=sp.n_local)
    torch.cuda.synchronize()
    assert sala.sala_get_device_status() == 0
    nb = w.seqlen // sp.block
    rng = np.random.default_rng(0)
    rows = sorted(set([0, 1, 2, 70, nb - 1, nb - 2]) | set(rng.choice(nb, 18, replace=False).tolist()))
    ref, (qh, kh, kb, ridx, scores) = oracle.sparse_layer(
        f64(q), f64(k), f64(v), f64(g), f64(wt), f64(wt), block=sp.block, topk=sp.topk,
        n_init=sp.n_init, n_local=sp.n_local, query_blocks=rows)
    gidx = idx.cpu().numpy()
    check_index_rows(gidx, ridx, scores, sp.topk, sp.n_init, sp.n_local, rows)
    assert rel_err(f64(kbar), np.transpose(kb, (0, 2, 1, 3))) <= 1e-5
    G = sp.q_heads // sp.kv_heads
    got, want = f64(out), ref
    for i in rows:
        sl = slice(i * sp.block, (i + 1) * sp.block)
        for gg in range(sp.kv_heads):
            if np.array_equal(gidx[0, gg, i], ridx[0, gg, i]):
                hs = slice(gg * G, (gg + 1) * G)
                assert rel_err(got[:, sl, hs], want[:, sl, hs]) <= TOL, (i, gg)


def test_sparse_decode_1m_context(sala):
    """Sparse-layer decode tokens against the 1M-token cache of a real
    prefill (1048576 tokens, 16384 blocks, top-64 + 1 + 4)."""
    dev = torch.device("cuda")
    w = wl.WORKLOADS["group_1m"]
    sp, ln = w.sparse, w.linear
    N, D = w.seqlen, 128
    cap = N + 128
    q, k, v, g = wl.layer_inputs(w, w.n_linear, dev)
    wt = wl.rms_weights(D, dev)
    qn, kn, kb, idx = sala.sparse_select(q, k, wt, wt, block=sp.block, topk=sp.topk,
                                         n_init=sp.n_init, n_local=sp.n_local)
    k_cache = torch.zeros((1, cap, sp.kv_heads, D), dtype=torch.bfloat16, device=dev)
    v_cache = torch.zeros_like(k_cache)
    kbar = torch.zeros((1, cap // 64, sp.kv_heads, D), dtype=torch.float32, device=dev)
    ksum = torch.zeros((1, sp.kv_heads, D), dtype=torch.float32, device=dev)
    k_cache[:, :N] = kn
    v_cache[:, :N] = v
    kbar[:, :N // 64] = kb
    k_hist, v_hist = f64(k), f64(v)
    del q, g, qn, kn, kb, idx
    torch.cuda.empty_cache()
    # linear layers start from zero state here: only the sparse output is compared
    H = ln.heads
    lam = lam_tensor(w, dev)
    states = [torch.zeros((1, H, D, D), dtype=torch.float32, device=dev) for _ in range(w.n_linear)]
    ld = sala.linear_desc(1, 64, H, D)
    sd = sala.sparse_desc(1, 64, sp.q_heads, sp.kv_heads, D, topk=sp.topk, n_init=sp.n_init,
                          n_local=sp.n_local)
    dd = sala.DecodeDesc(ld, sd, w.n_linear, cap)
    ws = sala.workspace(sala.sala_decode_workspace_size(dd), dev)
    for s in range(2):
        pos = N + s
        tok = wl.decode_inputs(w, s, dev)
        outs = [torch.empty_like(t[0]) for t in tok]
        io = sala.make_decode_io(tok, outs, states, [lam] * w.n_linear, wt, wt)
        assert sala.sala_decode_step(dd, io, k_cache, v_cache, kbar, ksum, pos, ws) == 0
        torch.cuda.synchronize()
        tq, tk, tv, tg = (f64(t) for t in tok[w.n_linear])
        k_hist = np.concatenate([k_hist, tk[:, None]], axis=1)
        v_hist = np.concatenate([v_hist, tv[:, None]], axis=1)
        ro, _ = oracle.decode_sparse_step(k_hist, v_hist, tq, tg, f64(wt), f64(wt), pos,
                                          topk=sp.topk, n_init=sp.n_init, n_local=sp.n_local)
        assert rel_err(f64(outs[w.n_linear]), ro) <= TOL
    assert sala.sala_get_device_status() == 0

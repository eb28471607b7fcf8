"""Full-size parity on every layer-group workload, in the launch configuration
the benchmark times (32K, 128K, 256K and 1M tokens; 32 q heads, 2 kv heads,
head_dim 128), checked on outputs the fp64 oracle can afford:

* linear layers: whole heads over the whole sequence (outputs and final
  state), chosen to cover the fastest and slowest decay and, in the 128K
  workload, the heads with lambda = 1;
* the sparse layer: every query block at 32K, sampled query blocks (first,
  last, random) at the longer lengths, through the oracle's row forms.  The
  selected indices are checked against the oracle's fp64 ranking within the
  tie window, and every checked row's output against the oracle's attention
  over the GPU's own (validated) index list;
* decode after a real 1M-token prefill of all four layers: linear outputs
  and states and the sparse output of each token.
"""
import numpy as np
import pytest
import torch

import oracle
from hybrid_sparse_linear_lightning_b200 import workloads as wl
from tests.parity import (TOL, block_rows, check_index_subset, f64, lam_tensor, rel_err)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def sala(cuda_device):
    from hybrid_sparse_linear_lightning_b200 import sala as s
    return s


def _linear_whole_heads(sala, w, layer, heads):
    """One linear layer at the workload's full length; heads `heads` compared
    whole.  Returns the GPU's final state (all heads) and the oracle's
    (the compared heads)."""
    dev = torch.device("cuda")
    q, k, v, g = wl.layer_inputs(w, layer, dev)
    lam = lam_tensor(w, dev)
    wt = wl.rms_weights(w.linear.head_dim, dev)
    out, st = sala.linear_prefill(q, k, v, g, lam, wt, wt, chunk=w.linear.chunk, want_state=True)
    torch.cuda.synchronize()
    assert sala.sala_get_device_status() == 0
    sub = lambda t: f64(t[:, :, heads])
    ref, S = oracle.linear_layer(sub(q), sub(k), sub(v), sub(g), f64(lam)[heads], f64(wt), f64(wt),
                                 chunk=w.linear.chunk)
    e_out, e_st = rel_err(sub(out), ref), rel_err(f64(st[:, heads]), S)
    print(f"linear {w.name} layer {layer} heads {heads}: output err {e_out:.2e}, "
          f"state err {e_st:.2e}")
    assert e_out <= TOL, (layer, heads, e_out)
    assert e_st <= TOL, (layer, heads, e_st)
    del q, k, v, g, out
    torch.cuda.empty_cache()
    return st, S


def _sparse_rows(sala, w, rows):
    """The sparse layer at full length; query blocks `rows` compared.
    Returns the device tensors the decode cache is built from."""
    dev = torch.device("cuda")
    sp = w.sparse
    q, k, v, g = wl.layer_inputs(w, w.n_linear, dev)
    wt = wl.rms_weights(sp.head_dim, dev)
    qn, kn, kbar, idx = sala.sparse_select(q, k, wt, wt, block=sp.block, topk=sp.topk,
                                           n_init=sp.n_init, n_local=sp.n_local)
    out = sala.sparse_prefill(qn, kn, v, g, idx, block=sp.block, topk=sp.topk, n_init=sp.n_init,
                              n_local=sp.n_local)
    torch.cuda.synchronize()
    assert sala.sala_get_device_status() == 0
    kf, vf = f64(k), f64(v)
    q_rows, g_rows = block_rows(q, rows, sp.block), block_rows(g, rows, sp.block)
    _, (qh, kh, kb, ridx, scores) = oracle.sparse_layer_rows(
        q_rows, g_rows, rows, kf, vf, f64(wt), f64(wt), block=sp.block, topk=sp.topk,
        n_init=sp.n_init, n_local=sp.n_local)
    gidx = idx.cpu().numpy()[:, :, rows]
    n_tie = check_index_subset(gidx, ridx, scores, rows, sp.topk, sp.n_init, sp.n_local)
    assert rel_err(f64(kbar), np.transpose(kb, (0, 2, 1, 3))) <= 1e-5
    assert rel_err(f64(kn), kh) <= TOL
    assert rel_err(block_rows(qn, rows, sp.block), qh) <= TOL
    want = oracle.sigmoid(g_rows) * oracle.sparse_attention_rows(qh, kh, vf, gidx, rows, sp.block)
    assert rel_err(block_rows(out, rows, sp.block), want) <= TOL
    # ties are rare: at most a few percent of the checked rows
    assert n_tie <= max(2, len(rows) * sp.kv_heads // 20), n_tie
    return dict(k=k, v=v, kn=kn, kbar=kbar, kf=kf, vf=vf)


def _sample_rows(nb, n_random, seed):
    rng = np.random.default_rng(seed)
    fixed = {0, 1, 2, 3, 70, nb // 2, nb - 3, nb - 2, nb - 1}
    return sorted(fixed | set(rng.choice(nb, n_random, replace=False).tolist()))


def test_group_32k_all_layers(sala):
    """32768 tokens, top-16 + 1 + 2: linear heads 0, 15, 16, 31 of all three
    linear layers whole; every query block of the sparse layer."""
    w = wl.WORKLOADS["group_32k"]
    for layer in range(w.n_linear):
        _linear_whole_heads(sala, w, layer, [0, 15, 16, 31])
    _sparse_rows(sala, w, list(range(w.seqlen // w.sparse.block)))


def test_group_128k_lambda_one_and_salient_keys(sala):
    """131072 tokens, heads 16..31 with lambda = 1 (no decay over 128K
    tokens), 1% of key rows scaled x8 before the norm, top-32 + 1 + 2: linear
    heads 0, 15 (decayed) and 16, 31 (lambda = 1) of all three layers whole;
    48 sampled query blocks of the sparse layer."""
    w = wl.WORKLOADS["group_128k"]
    assert wl.lam_schedule(w.linear)[16] == 1.0 and wl.lam_schedule(w.linear)[15] < 1.0
    for layer in range(w.n_linear):
        _linear_whole_heads(sala, w, layer, [0, 15, 16, 31])
    _sparse_rows(sala, w, _sample_rows(w.seqlen // w.sparse.block, 40, 2))


def test_group_256k(sala):
    """262144 tokens, top-64 + 1 + 4: linear heads 0 (fastest decay) and 31
    (slowest) of the first linear layer whole; 32 sampled query blocks."""
    w = wl.WORKLOADS["group_256k"]
    _linear_whole_heads(sala, w, 0, [0, 31])
    _sparse_rows(sala, w, _sample_rows(w.seqlen // w.sparse.block, 24, 0))


def test_group_1m_prefill_then_decode(sala):
    """1048576 tokens: all four layers prefilled (linear heads 0 and 31 of
    each layer whole, with final states; 24 sampled sparse query blocks),
    then decode tokens through the C ABI starting from those states and the
    sparse layer's 1M-token cache: linear outputs and states, sparse output."""
    dev = torch.device("cuda")
    w = wl.WORKLOADS["group_1m"]
    sp, ln = w.sparse, w.linear
    N, D, H = w.seqlen, ln.head_dim, ln.heads
    heads = [0, 31]
    states, ref_states = [], []
    for layer in range(w.n_linear):
        st, S = _linear_whole_heads(sala, w, layer, heads)
        states.append(st)
        ref_states.append(S)
    r = _sparse_rows(sala, w, _sample_rows(N // sp.block, 15, 4))
    steps = 3
    cap = N + 2 * sp.block
    k_cache = torch.zeros((1, cap, sp.kv_heads, D), dtype=torch.bfloat16, device=dev)
    v_cache = torch.zeros_like(k_cache)
    kbar = torch.zeros((1, cap // sp.block, sp.kv_heads, D), dtype=torch.float32, device=dev)
    ksum = torch.zeros((1, sp.kv_heads, D), dtype=torch.float32, device=dev)
    k_cache[:, :N] = r["kn"]
    v_cache[:, :N] = r["v"]
    kbar[:, :N // sp.block] = r["kbar"]
    k_hist, v_hist = f64(r["k"]), r["vf"]
    del r
    torch.cuda.empty_cache()
    lam = lam_tensor(w, dev)
    wt = wl.rms_weights(D, dev)
    gpu_start = [f64(s) for s in states]          # every head, as the GPU prefill left it
    ld = sala.linear_desc(1, 64, H, D)
    sd = sala.sparse_desc(1, 64, sp.q_heads, sp.kv_heads, D, topk=sp.topk, n_init=sp.n_init,
                          n_local=sp.n_local)
    dd = sala.DecodeDesc(ld, sd, w.n_linear, cap)
    ws = sala.workspace(sala.sala_decode_workspace_size(dd), dev)
    for s in range(steps):
        pos = N + s
        tok = wl.decode_inputs(w, s, dev)
        outs = [torch.empty_like(t[0]) for t in tok]
        io = sala.make_decode_io(tok, outs, states, [lam] * w.n_linear, wt, wt)
        assert sala.sala_decode_step(dd, io, k_cache, v_cache, kbar, ksum, pos, ws) == 0
        torch.cuda.synchronize()
        assert sala.sala_get_device_status() == 0
        for l in range(w.n_linear):
            tq, tk, tv, tg = (f64(t) for t in tok[l])
            # all heads, from the GPU's own prefill state
            ro, gpu_start[l] = oracle.decode_linear_step(gpu_start[l], tq, tk, tv, tg, f64(lam),
                                                         f64(wt), f64(wt), pos)
            assert rel_err(f64(outs[l]), ro) <= TOL, (s, l)
            # the compared heads, from the oracle's own 1M-token prefill state
            ro, ref_states[l] = oracle.decode_linear_step(
                ref_states[l], tq[:, heads], tk[:, heads], tv[:, heads], tg[:, heads],
                f64(lam)[heads], f64(wt), f64(wt), pos)
            assert rel_err(f64(outs[l][:, heads]), ro) <= TOL, (s, l)
        tq, tk, tv, tg = (f64(t) for t in tok[w.n_linear])
        k_hist = np.concatenate([k_hist, tk[:, None]], axis=1)
        v_hist = np.concatenate([v_hist, tv[:, None]], axis=1)
        ro, _ = oracle.decode_sparse_step(k_hist, v_hist, tq, tg, f64(wt), f64(wt), pos,
                                          topk=sp.topk, n_init=sp.n_init, n_local=sp.n_local)
        assert rel_err(f64(outs[w.n_linear]), ro) <= TOL, s
    for l in range(w.n_linear):
        assert rel_err(f64(states[l][:, heads]), ref_states[l]) <= TOL
        assert rel_err(f64(states[l]), gpu_start[l]) <= TOL


def test_linear_lambda_one_1m(sala):
    """lambda = 1 (no decay) over 1048576 tokens, the case where the state
    grows the most and its bf16 copy (the B operand of Q' S) is most
    exposed: heads 16 and 31 of a linear layer whose upper half of heads use
    lambda = 1, compared whole (outputs and final state)."""
    import dataclasses
    w = wl.WORKLOADS["group_1m"]
    w = dataclasses.replace(w, linear=dataclasses.replace(w.linear, lam_kind="half_one"))
    assert wl.lam_schedule(w.linear)[16] == 1.0
    _linear_whole_heads(sala, w, 0, [16, 31])

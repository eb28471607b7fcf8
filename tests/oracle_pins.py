"""Pins of the oracle against facts that do not come from the oracle itself.

Each ``check_*`` takes an oracle module and raises ``AssertionError`` when the
oracle disagrees with a closed form, a library routine, a brute-force search
or an invariant.  ``test_oracle_pins.py`` runs them on the real oracle (all
must pass) and on mutated copies of it with planted mistakes (at least one
must fail for every mutant), which shows that the pins can see such mistakes.

The pages print no worked numeric example, so there is no page value to pin
against; the pins are mathematical.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch

RTOL = 1e-10


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------- norms / rope

def check_rms_norm_closed_form(orc):
    # x = [3, 4]: mean of squares 12.5, so x_hat = x / sqrt(12.5).
    x = np.array([[3.0, 4.0]])
    got = orc.rms_norm(x, np.array([2.0, 0.5]), eps=0.0)
    want = np.array([[3.0 / math.sqrt(12.5) * 2.0, 4.0 / math.sqrt(12.5) * 0.5]])
    assert _rel(got, want) < 1e-14, (got, want)
    # eps enters under the root: x = [1, 1] -> 1 / sqrt(1 + eps)
    got = orc.rms_norm(np.ones((1, 2)), np.ones(2), eps=0.25)
    assert _rel(got, np.full((1, 2), 1.0 / math.sqrt(1.25))) < 1e-14


def check_rms_norm_invariants(orc):
    x = _rng(1).standard_normal((3, 5, 2, 16))
    y = orc.rms_norm(x, np.ones(16), eps=0.0)
    assert _rel(np.mean(y * y, axis=-1), np.ones((3, 5, 2))) < 1e-13
    # scale invariance (with the default eps it holds to ~eps)
    assert _rel(orc.rms_norm(8.0 * x, np.ones(16), eps=0.0), y) < 1e-13
    assert _rel(orc.rms_norm(8.0 * x, np.ones(16)), orc.rms_norm(x, np.ones(16))) < 1e-5


def check_rope_complex(orc):
    # d = 4, rotate-half pairs (0, 2) and (1, 3) turn by p*theta_0 and p*theta_1,
    # theta_i = base^(-2i/d): with base 10000, theta_0 = 1 and theta_1 = 1/100.
    x = _rng(2).standard_normal((1, 6, 1, 4))
    pos = np.array([0, 1, 2, 5, 100, 12345])
    y = orc.apply_rope(x, pos, 10000.0)
    for t, p in enumerate(pos):
        for i, th in ((0, 1.0), (1, 0.01)):
            z = complex(x[0, t, 0, i], x[0, t, 0, i + 2]) * complex(math.cos(p * th), math.sin(p * th))
            assert abs(y[0, t, 0, i] - z.real) < 1e-9 and abs(y[0, t, 0, i + 2] - z.imag) < 1e-9


def check_rope_invariants(orc):
    r = _rng(3)
    d = 32
    q = r.standard_normal((1, 1, 1, d))
    k = r.standard_normal((1, 1, 1, d))
    # p = 0 is the identity; norms are kept
    assert _rel(orc.apply_rope(q, [0], 10000.0), q) < 1e-15
    y = orc.apply_rope(np.repeat(q, 4, axis=1), [3, 77, 1000, 262143], 10000.0)
    assert _rel(np.linalg.norm(y, axis=-1), np.full((1, 4, 1), np.linalg.norm(q))) < 1e-12
    # <R_m q, R_n k> depends only on m - n
    dots = []
    for m, n in ((10, 3), (107, 100), (5007, 5000)):
        a = orc.apply_rope(q, [m], 10000.0)
        b = orc.apply_rope(k, [n], 10000.0)
        dots.append(float(np.sum(a * b)))
    assert max(dots) - min(dots) < 1e-9, dots


def check_sigmoid(orc):
    assert abs(float(orc.sigmoid(0.0)) - 0.5) < 1e-16
    assert abs(float(orc.sigmoid(40.0)) - 1.0) < 1e-16
    assert abs(float(orc.sigmoid(-2.0)) - 1.0 / (1.0 + math.exp(2.0))) < 1e-16


# --------------------------------------------------------------------------- linear attention

def _lin_inputs(seed, B=2, N=37, H=3, dk=8, dv=5):
    r = _rng(seed)
    q = r.standard_normal((B, N, H, dk))
    k = r.standard_normal((B, N, H, dk))
    v = r.standard_normal((B, N, H, dv))
    S0 = r.standard_normal((B, H, dk, dv))
    lam = np.array([0.9, 1.0, 0.5])[:H]
    return q, k, v, S0, lam


def check_linear_brute_force(orc):
    # Hand-expanded recurrence, scalar loops: o_t = q_t (sum_s lam^(t-s) k_s^T v_s + lam^(t+1) S0)
    q, k, v, S0, lam = _lin_inputs(4, B=1, N=5, H=2, dk=3, dv=2)
    o, S = orc.linear_attention_chunked(q, k, v, lam, chunk=2, scale=0.5, state_in=S0)
    for h in range(2):
        for t in range(5):
            for j in range(2):
                acc = 0.0
                for i in range(3):
                    st = lam[h] ** (t + 1) * S0[0, h, i, j]
                    for s in range(t + 1):
                        st += lam[h] ** (t - s) * k[0, s, h, i] * v[0, s, h, j]
                    acc += q[0, t, h, i] * st
                assert abs(o[0, t, h, j] - 0.5 * acc) < 1e-12
        for i in range(3):
            for j in range(2):
                st = lam[h] ** 5 * S0[0, h, i, j] + sum(
                    lam[h] ** (4 - s) * k[0, s, h, i] * v[0, s, h, j] for s in range(5))
                assert abs(S[0, h, i, j] - st) < 1e-12


def check_linear_three_forms(orc):
    q, k, v, S0, lam = _lin_inputs(5)
    o_r, S_r = orc.linear_attention_recurrent(q, k, v, lam, 0.7, S0)
    o_q = orc.linear_attention_quadratic(q, k, v, lam, 0.7, S0)
    assert _rel(o_q, o_r) < RTOL
    for C in (1, 4, 16, 37, 64):
        o_c, S_c = orc.linear_attention_chunked(q, k, v, lam, C, 0.7, S0)
        assert _rel(o_c, o_r) < RTOL, C
        assert _rel(S_c, S_r) < RTOL, C


def check_linear_special_lambdas(orc):
    q, k, v, _, _ = _lin_inputs(6, H=2)
    # lam = 1: prefix sums of outer products
    o, S = orc.linear_attention_chunked(q, k, v, np.ones(2), 8)
    P = np.cumsum(np.einsum("bnhk,bnhv->bnhkv", k, v), axis=1)
    assert _rel(o, np.einsum("bnhk,bnhkv->bnhv", q, P)) < RTOL
    assert _rel(S, P[:, -1]) < RTOL
    # lam = 0: o_t = (q_t . k_t) v_t and the state is the last outer product
    o, S = orc.linear_attention_chunked(q, k, v, np.zeros(2), 8)
    assert _rel(o, np.sum(q * k, axis=-1, keepdims=True) * v) < RTOL
    assert _rel(S, np.einsum("bhk,bhv->bhkv", k[:, -1], v[:, -1])) < RTOL


def check_linear_segments(orc):
    # Resumable prefill: two halves with the carried state equal one pass.
    q, k, v, S0, lam = _lin_inputs(7, N=64)
    o, S = orc.linear_attention_chunked(q, k, v, lam, 16, 1.0, S0)
    o1, S1 = orc.linear_attention_chunked(q[:, :24], k[:, :24], v[:, :24], lam, 16, 1.0, S0)
    o2, S2 = orc.linear_attention_chunked(q[:, 24:], k[:, 24:], v[:, 24:], lam, 16, 1.0, S1)
    assert _rel(np.concatenate([o1, o2], axis=1), o) < RTOL
    assert _rel(S2, S) < RTOL


def check_linear_layer_gate_rope(orc):
    r = _rng(8)
    B, N, H, d = 1, 40, 2, 8
    q, k, v = (r.standard_normal((B, N, H, d)) for _ in range(3))
    lam = np.array([0.95, 1.0])
    w = np.ones(d)
    # gate 0 halves the output; a large gate passes it through
    out0, _ = orc.linear_layer(q, k, v, np.zeros((B, N, H, d)), lam, w, w, chunk=16)
    outp, _ = orc.linear_layer(q, k, v, np.full((B, N, H, d), 60.0), lam, w, w, chunk=16)
    assert _rel(out0, 0.5 * outp) < 1e-14
    # the layer = RMSNorm, then RoPE at pos0 + t, then attention (independent assembly)
    pos0 = 1000
    qh = np.empty_like(q)
    kh = np.empty_like(k)
    half = d // 2
    for t in range(N):
        for h in range(H):
            for x, dst in ((q, qh), (k, kh)):
                vec = x[0, t, h] / math.sqrt(np.mean(x[0, t, h] ** 2) + 1e-6)
                for i in range(half):
                    ang = (pos0 + t) * 10000.0 ** (-2.0 * i / d)
                    z = complex(vec[i], vec[i + half]) * complex(math.cos(ang), math.sin(ang))
                    dst[0, t, h, i], dst[0, t, h, i + half] = z.real, z.imag
    want, _ = orc.linear_attention_recurrent(qh, kh, v, lam)
    got, _ = orc.linear_layer(q, k, v, np.full((B, N, H, d), 60.0), lam, w, w, chunk=16, pos0=pos0)
    assert _rel(got, want) < 1e-12


# --------------------------------------------------------------------------- selection

def check_block_means_and_scores(orc):
    # ramp: mean of a block of consecutive integers is its midpoint
    x = np.arange(12, dtype=np.float64).reshape(1, 12, 1, 1) * np.ones((1, 1, 1, 2))
    m = orc.block_means(x, 4)
    assert _rel(m[0, 0, :, 0], [1.5, 5.5, 9.5]) < 1e-15
    # hand example: d = 4, group of 2 q heads, one kv head
    qbar = np.zeros((1, 2, 2, 4))
    kbar = np.zeros((1, 1, 2, 4))
    qbar[0, 0, 1] = [1, 0, 0, 0]
    qbar[0, 1, 1] = [0, 2, 0, 0]
    kbar[0, 0, 0] = [1, 1, 0, 0]
    kbar[0, 0, 1] = [0, 0, 3, -1]
    s = orc.block_scores(qbar, kbar)
    assert abs(s[0, 0, 1, 0] - 3.0 / 2.0) < 1e-15      # (1*1 + 2*1) / sqrt(4)
    assert abs(s[0, 0, 1, 1]) < 1e-15
    assert s[0, 0, 0, 1] == -np.inf                      # non-causal
    # GQA grouping: heads 0..G-1 go to kv head 0, G..2G-1 to kv head 1
    qbar = np.zeros((1, 4, 1, 2))
    kbar = np.ones((1, 2, 1, 2))
    qbar[0, 1, 0, 0] = 1.0
    qbar[0, 2, 0, 1] = 5.0
    s = orc.block_scores(qbar, kbar)
    assert abs(s[0, 0, 0, 0] - 1.0 / math.sqrt(2)) < 1e-15
    assert abs(s[0, 1, 0, 0] - 5.0 / math.sqrt(2)) < 1e-15


def check_selection_exhaustive(orc):
    r = _rng(9)
    nb, topk, n_init, n_local = 12, 3, 1, 2
    for trial in range(6):
        sc = r.standard_normal((1, 1, nb, nb))
        idx = orc.select_blocks(sc, topk, n_init, n_local)
        for b in range(nb):
            cand = list(range(n_init, b - n_local + 1))
            best = ()
            if cand:
                kk = min(topk, len(cand))
                best = max(itertools.combinations(cand, kk), key=lambda c: sum(sc[0, 0, b, j] for j in c))
            want = sorted(set(range(min(n_init, b + 1))) | set(range(max(0, b - n_local + 1), b + 1))
                          | set(best))
            row = [int(j) for j in idx[0, 0, b] if j >= 0]
            assert row == want, (b, row, want)
            assert len(row) == orc.selected_count(b, topk, n_init, n_local)
            assert all(j == -1 for j in idx[0, 0, b, len(row):])


def check_selection_ties(orc):
    # equal scores: the lower block index wins
    nb = 10
    sc = np.zeros((1, 1, nb, nb))
    sc[0, 0, 9, :] = [0, 1.0, 2.0, 1.0, 1.0, 2.0, 1.0, 0, 0, 0]
    idx = orc.select_blocks(sc, 3, 1, 2, rows=[9])
    assert [int(j) for j in idx[0, 0, 9] if j >= 0] == [0, 1, 2, 5, 8, 9]
    # more slots than candidates: everything causal is taken
    assert [int(j) for j in orc.select_blocks(sc, 50, 1, 2, rows=[9])[0, 0, 9] if j >= 0] == list(range(10))


def check_sparse_select_exhaustive(orc):
    # The whole selection stage on raw inputs against an independent
    # computation: block means of hand-normalised rows, group-summed queries,
    # then the best-scoring candidate subset by exhaustive search (fp64).
    r = _rng(15)
    B, N, Hq, Hkv, d, blk = 1, 14 * 8, 4, 2, 8, 8
    q = r.standard_normal((B, N, Hq, d))
    k = r.standard_normal((B, N, Hkv, d))
    w = np.ones(d)
    topk, n_init, n_local = 3, 1, 2
    _, _, _, idx, _ = orc.sparse_select(q, k, w, w, block=blk, topk=topk, n_init=n_init,
                                        n_local=n_local)
    nrm = lambda x: x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + 1e-6)
    nb = N // blk
    for g in range(Hkv):
        kb = [np.mean(nrm(k[0, j * blk:(j + 1) * blk, g]), axis=0) for j in range(nb)]
        for i in range(nb):
            qg = sum(np.mean(nrm(q[0, i * blk:(i + 1) * blk, h]), axis=0)
                     for h in (2 * g, 2 * g + 1))
            cand = list(range(n_init, i - n_local + 1))
            best = ()
            if cand:
                best = max(itertools.combinations(cand, min(topk, len(cand))),
                           key=lambda c: sum(float(kb[j] @ qg) for j in c))
            want = sorted(set(range(min(n_init, i + 1))) | set(range(max(0, i - n_local + 1), i + 1))
                          | set(best))
            assert [int(j) for j in idx[0, g, i] if j >= 0] == want, (g, i)


def check_sparse_rows_forms(orc):
    # The row forms compute the same definitions as the full forms on the
    # chosen query blocks (block numbers, causality and selection included).
    r = _rng(16)
    B, N, Hq, Hkv, d, blk = 2, 24 * 16, 6, 2, 16, 16
    q, g = (r.standard_normal((B, N, Hq, d)) for _ in range(2))
    k, v = (r.standard_normal((B, N, Hkv, d)) for _ in range(2))
    w = 1.0 + 0.1 * r.standard_normal(d)
    kw = dict(block=blk, topk=3, n_init=1, n_local=2)
    full, (qh, kh, kbar, idx, scores) = orc.sparse_layer(q, k, v, g, w, w, **kw)
    rows = [23, 0, 9, 4, 17]
    cat = lambda x: np.concatenate([x[:, i * blk:(i + 1) * blk] for i in rows], axis=1)
    out, (qh_r, kh_r, kbar_r, idx_r, sc_r) = orc.sparse_layer_rows(cat(q), cat(g), rows, k, v,
                                                                   w, w, **kw)
    assert _rel(out, cat(full)) < 1e-13
    assert np.array_equal(idx_r, idx[:, :, rows])
    assert np.array_equal(sc_r, scores[:, :, rows])
    assert _rel(kbar_r, kbar) < 1e-15 and _rel(qh_r, cat(qh)) < 1e-15


def check_token_softmax_selection(orc):
    # Token-level variant against an independent brute force: scalar loops
    # for the scores, an explicit softmax per (token, head), the importance
    # sums, and the best-scoring candidate subset by exhaustive search.
    r = _rng(17)
    B, blk, nb, Hq, Hkv, d = 1, 4, 9, 4, 2, 4
    N = blk * nb
    q = r.standard_normal((B, N, Hq, d))
    k = r.standard_normal((B, N, Hkv, d))
    w = np.ones(d)
    topk, n_init, n_local = 2, 1, 2
    _, _, _, idx, imp = orc.select_token_softmax(q, k, w, w, block=blk, topk=topk, n_init=n_init,
                                                 n_local=n_local)
    def nrm(x):
        s_ = math.sqrt(sum(v * v for v in x) / len(x) + 1e-6)
        return [v / s_ for v in x]
    G = Hq // Hkv
    for g in range(Hkv):
        kb = []
        for j in range(nb):
            rows_ = [nrm(list(k[0, j * blk + t, g])) for t in range(blk)]
            kb.append([sum(rr[e] for rr in rows_) / blk for e in range(d)])
        for i in range(nb):
            cand = list(range(n_init, i - n_local + 1))
            tot = {j: 0.0 for j in cand}
            for t in range(blk):
                for h in range(g * G, (g + 1) * G):
                    qq = nrm(list(q[0, i * blk + t, h]))
                    z = {j: sum(qq[e] * kb[j][e] for e in range(d)) / math.sqrt(d) for j in cand}
                    den = sum(math.exp(v) for v in z.values())
                    for j in cand:
                        tot[j] += math.exp(z[j]) / den
            for j in cand:
                assert abs(imp[0, g, i, j] - tot[j]) < 1e-12, (g, i, j)
            best = ()
            if cand:
                best = max(itertools.combinations(cand, min(topk, len(cand))),
                           key=lambda c: sum(tot[j] for j in c))
            want = sorted(set(range(min(n_init, i + 1))) | set(range(max(0, i - n_local + 1), i + 1))
                          | set(best))
            assert [int(j) for j in idx[0, g, i] if j >= 0] == want, (g, i)


def check_token_softmax_single_query(orc):
    # One query token per block and one q head per kv head: the softmax is
    # monotonic in the score, so the variant ranks candidates exactly as the
    # block-mean rule does.
    r = _rng(18)
    q = r.standard_normal((1, 40, 2, 8))
    k = r.standard_normal((1, 40, 2, 8))
    w = np.ones(8)
    kw = dict(block=1, topk=5, n_init=1, n_local=3)
    _, _, _, idx_v, _ = orc.select_token_softmax(q, k, w, w, **kw)
    _, _, _, idx_m, _ = orc.sparse_select(q, k, w, w, **kw)
    assert np.array_equal(idx_v, idx_m)


# --------------------------------------------------------------------------- sparse attention
# --------------------------------------------------------------------------- sparse attention

def _sdpa(q, k, v, mask=None, causal=False, scale=None):
    """torch SDPA in fp64 on [B, N, H, d] with GQA expansion (library routine)."""
    G = q.shape[2] // k.shape[2]
    Q = torch.from_numpy(np.ascontiguousarray(np.transpose(q, (0, 2, 1, 3))))
    K = torch.from_numpy(np.ascontiguousarray(np.transpose(k, (0, 2, 1, 3)))).repeat_interleave(G, dim=1)
    V = torch.from_numpy(np.ascontiguousarray(np.transpose(v, (0, 2, 1, 3)))).repeat_interleave(G, dim=1)
    M = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=M, is_causal=causal, scale=scale)
    return np.transpose(o.numpy(), (0, 2, 1, 3))


def _sparse_inputs(seed, B=1, N=512, Hq=4, Hkv=2, d=16):
    r = _rng(seed)
    return (r.standard_normal((B, N, Hq, d)), r.standard_normal((B, N, Hkv, d)),
            r.standard_normal((B, N, Hkv, d)))


def check_sparse_dense_limit(orc):
    # top-k covering every block: dense causal softmax attention
    q, k, v = _sparse_inputs(10)
    w = np.ones(16)
    g = np.full(q.shape, 60.0)
    out, (qh, kh, _, _, _) = orc.sparse_layer(q, k, v, g, w, w, block=32, topk=64, n_init=1, n_local=2)
    want = _sdpa(orc.rms_norm(q, w), orc.rms_norm(k, w), v, causal=True)
    assert _rel(out, want) < 1e-12


def check_sparse_block_diagonal(orc):
    # k = 0, no initial block, one local block: causal attention inside each block
    q, k, v = _sparse_inputs(11, N=256)
    w = np.ones(16)
    qh, kh, _, idx, _ = orc.sparse_select(q, k, w, w, block=64, topk=0, n_init=0, n_local=1)
    o = orc.sparse_attention(qh, kh, v, idx, 64)
    for i in range(4):
        sl = slice(64 * i, 64 * (i + 1))
        assert _rel(o[:, sl], _sdpa(qh[:, sl], kh[:, sl], v[:, sl], causal=True)) < 1e-12
    # the first query sees only the first key: o = v
    assert _rel(o[:, 0], np.repeat(v[:, 0], 2, axis=1)) < 1e-14


def check_sparse_masked_sdpa(orc):
    # general selection: SDPA with the boolean mask built from the index lists
    q, k, v = _sparse_inputs(12, N=512, Hq=6, Hkv=2)
    w = np.ones(16)
    qh, kh, _, idx, _ = orc.sparse_select(q, k, w, w, block=32, topk=3, n_init=1, n_local=2)
    o = orc.sparse_attention(qh, kh, v, idx, 32)
    N, Hq, Hkv, blk = 512, 6, 2, 32
    mask = np.zeros((1, Hq, N, N), dtype=bool)
    for h in range(Hq):
        gkv = h // (Hq // Hkv)
        for t in range(N):
            for j in idx[0, gkv, t // blk]:
                if j >= 0:
                    mask[0, h, t, j * blk:(j + 1) * blk] = True
            mask[0, h, t, t + 1:] = False
    assert _rel(o, _sdpa(qh, kh, v, mask=mask)) < 1e-12


# --------------------------------------------------------------------------- decode

def check_decode_linear(orc):
    r = _rng(13)
    B, N, H, d = 1, 48, 2, 8
    q, k, v, g = (r.standard_normal((B, N + 1, H, d)) for _ in range(4))
    lam = np.array([0.9, 1.0])
    w = np.ones(d)
    full, _ = orc.linear_layer(q, k, v, g, lam, w, w, chunk=16)
    _, S = orc.linear_layer(q[:, :N], k[:, :N], v[:, :N], g[:, :N], lam, w, w, chunk=16)
    o, _ = orc.decode_linear_step(S, q[:, N], k[:, N], v[:, N], g[:, N], lam, w, w, N)
    assert _rel(o, full[:, N]) < 1e-12


def check_decode_sparse(orc):
    r = _rng(14)
    B, Hq, Hkv, d, blk = 1, 4, 2, 16, 16
    N = 5 * blk + 6
    q, g = (r.standard_normal((B, N, Hq, d)) for _ in range(2))
    k, v = (r.standard_normal((B, N, Hkv, d)) for _ in range(2))
    w = np.ones(d)
    # top-k covering all blocks: dense causal attention of the last token
    o, _ = orc.decode_sparse_step(k, v, q[:, -1], g[:, -1], w, w, N - 1, block=blk, topk=64,
                                  n_init=1, n_local=2)
    dense = _sdpa(orc.rms_norm(q, w), orc.rms_norm(k, w), v, causal=True)[:, -1]
    assert _rel(o, orc.sigmoid(g[:, -1]) * dense) < 1e-12
    # real selection: exhaustive search over the complete candidate blocks
    for topk in (1, 2):
        o, idx = orc.decode_sparse_step(k, v, q[:, -1], g[:, -1], w, w, N - 1, block=blk,
                                        topk=topk, n_init=1, n_local=2, score_dtype=np.float64)
        kh = orc.rms_norm(k, w)
        qh = orc.rms_norm(q[:, -1], w)
        for gg in range(Hkv):
            qg = qh[0, 2 * gg] + qh[0, 2 * gg + 1]
            cand = list(range(1, (N - 1) // blk - 2 + 1))
            sc = {j: float(np.mean(kh[0, j * blk:(j + 1) * blk, gg], axis=0) @ qg) for j in cand}
            best = max(itertools.combinations(cand, topk), key=lambda c: sum(sc[j] for j in c))
            want = sorted({0, 4, 5} | set(best))
            assert [int(j) for j in idx[0, gg] if j >= 0] == want


def check_silu(orc):
    assert orc.silu(0.0) == 0.0
    assert abs(float(orc.silu(2.0)) - 2.0 / (1.0 + math.exp(-2.0))) < 1e-15
    assert abs(float(orc.silu(-40.0))) < 1e-15


def check_sala_block_assembly(orc):
    # The block against an independent scalar assembly on a tiny case: pre-
    # norm, projections, the (already pinned) attention, output projection
    # and residual, pre-norm, SwiGLU, residual.
    r = _rng(19)
    B, N, Hq, d, ff = 1, 8, 2, 4, 6
    hid = Hq * d
    x = r.standard_normal((B, N, hid))
    w = {"norm_attn": 1 + 0.1 * r.standard_normal(hid), "wq": r.standard_normal((hid, hid)) / 3,
         "wk": r.standard_normal((hid, hid)) / 3, "wv": r.standard_normal((hid, hid)) / 3,
         "wg": r.standard_normal((hid, hid)) / 3, "qk_q": np.ones(d), "qk_k": np.ones(d),
         "wo": r.standard_normal((hid, hid)) / 3, "norm_ffn": 1 + 0.1 * r.standard_normal(hid),
         "w1": r.standard_normal((ff, hid)) / 3, "w3": r.standard_normal((ff, hid)) / 3,
         "w2": r.standard_normal((hid, ff)) / 3}
    lam = np.array([0.9, 1.0])
    y = orc.sala_block(x, w, "linear", q_heads=Hq, kv_heads=Hq, head_dim=d, lam=lam, chunk=4)
    def mv(m, v_):
        return [sum(m[i][j] * v_[j] for j in range(len(v_))) for i in range(len(m))]
    def nrm(v_, wt):
        s_ = math.sqrt(sum(e * e for e in v_) / len(v_) + 1e-6)
        return [e / s_ * wt[i] for i, e in enumerate(v_)]
    xs = [list(x[0, t]) for t in range(N)]
    proj = {k_: [mv(w[k_], nrm(xs[t], w["norm_attn"])) for t in range(N)]
            for k_ in ("wq", "wk", "wv", "wg")}
    rs = lambda key: np.array(proj[key]).reshape(1, N, Hq, d)
    a, _ = orc.linear_layer(rs("wq"), rs("wk"), rs("wv"), rs("wg"), lam, np.ones(d), np.ones(d),
                            chunk=4)
    for t in range(N):
        h = [xs[t][i] + e for i, e in enumerate(mv(w["wo"], list(a[0, t].reshape(-1))))]
        hn = nrm(h, w["norm_ffn"])
        u, g3 = mv(w["w1"], hn), mv(w["w3"], hn)
        s_ = [u[i] / (1 + math.exp(-u[i])) * g3[i] for i in range(ff)]
        want = [h[i] + e for i, e in enumerate(mv(w["w2"], s_))]
        assert max(abs(y[0, t, i] - want[i]) for i in range(hid)) < 1e-10, t


ALL_CHECKS = [
    check_rms_norm_closed_form, check_rms_norm_invariants, check_rope_complex,
    check_rope_invariants, check_sigmoid, check_linear_brute_force, check_linear_three_forms,
    check_linear_special_lambdas, check_linear_segments, check_linear_layer_gate_rope,
    check_block_means_and_scores, check_selection_exhaustive, check_selection_ties,
    check_sparse_select_exhaustive, check_sparse_rows_forms,
    check_token_softmax_selection, check_token_softmax_single_query,
    check_sparse_dense_limit, check_sparse_block_diagonal, check_sparse_masked_sdpa,
    check_decode_linear, check_decode_sparse, check_silu, check_sala_block_assembly,
]

"""fp64 CPU oracle of the SALA prefill / decode attention path (test infrastructure).

Source pages and what each fixes:

* MiniCPM-SALA paper, zh translation (bittide.aicompass.dev), summary and
  abstract: the model interleaves Lightning linear-attention layers with
  InfLLM-V2 sparse-attention layers at 1:3, applies QK normalisation in every
  layer, uses RoPE only in the linear layers and puts an output gate after
  each attention block.  Section 2.1 (model architecture): linear layers have
  constant-size state, sparse layers model long-range dependencies.
* acgfav.com press article, section "SALA 混合架构": linear layers use
  Lightning Attention at O(N); sparse layers use InfLLM-V2, where a
  fine-grained block selection lets each query attend to a small set of key
  blocks; HyPE keeps RoPE in linear layers and uses NoPE in sparse layers, so
  the sparse KV cache carries no position.
* intelliparadigm.com blog, section 2.2 (HyPE) and yunpan.plus post,
  section 二.2 (HyPE): the same RoPE / NoPE split.

None of the pages prints a formula.  The readings taken here (each stated at
its function) are the plainest ones consistent with the pages:

* QK normalisation is RMSNorm over head_dim per (token, head), eps 1e-6, with
  one weight vector for Q and one for K, applied before RoPE.
* RoPE is the rotate-half form, theta_i = base^(-2i/d), position = pos0 + t.
* Lightning linear attention: o_t = scale * q_t S_t, S_t = lam S_{t-1} + k_t^T v_t
  (no denominator, no extra normaliser), per-head decay lam, computed
  chunk-wise: intra-chunk (Q K^T . D) V with D_ij = lam^(i-j) for j <= i, plus
  the inter-chunk term lam^(i+1) q_i S_prev and the state carry
  S <- lam^C S + sum_j lam^(C-1-j) k_j^T v_j.
* Output gate: out = sigmoid(g) * o, g a tensor of the output's shape.
* InfLLM-V2-style selection: block keys/queries are the means of the
  normalised NoPE keys/queries over non-overlapping blocks of B_s tokens; the
  score of key block j for query block b and kv head g is
  <sum over the group's q heads of qbar_b^h, kbar_j^g> / sqrt(d); each query
  block takes the initial blocks [0, n_init), the local blocks
  [b-n_local+1, b] and the top-k of the remaining causal candidates
  [n_init, b-n_local] (ties to the lower block index), emitted in ascending
  order and padded with -1.
* Exact softmax attention (scale 1/sqrt(d)) of each query over the keys of
  its selected blocks at positions <= its own.

All arithmetic is fp64, the block-selection decision included: the selected
index sets are exact for the fp64 scores, and an implementation that ranks
in lower precision may differ from them only where the k-th and (k+1)-th
candidate scores lie within a relative 1e-3 of each other (the tolerance
stated for the selected indices).  ``score_dtype`` can still be lowered for
experiments; nothing on the test path does so.

Full-size inputs (up to 1M tokens, 32 query heads) do not fit in host memory
as fp64 arrays, so the sparse layer also has ``*_rows`` forms that take the
queries of a chosen subset of query blocks only; they compute the same
definitions for those blocks (pinned against the full forms).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "rms_norm", "rope_cos_sin", "apply_rope", "sigmoid",
    "linear_attention_chunked", "linear_attention_recurrent",
    "linear_attention_quadratic", "linear_layer",
    "block_means", "block_scores", "select_row", "select_blocks",
    "selected_count", "sparse_attention", "sparse_select", "sparse_layer",
    "sparse_attention_rows", "sparse_select_rows", "sparse_layer_rows",
    "token_softmax_importance", "select_token_softmax",
    "decode_linear_step", "decode_sparse_step",
    "silu", "sala_block",
]

F64 = np.float64


# ---------------------------------------------------------------------------
# QK normalisation, RoPE, gate
# ---------------------------------------------------------------------------

def rms_norm(x, w, eps=1e-6, dtype=F64):
    """QK normalisation "applied globally" (paper summary; abstract).

    Reading: RMSNorm over the last axis (head_dim) of each (token, head)
    vector, x / sqrt(mean(x^2) + eps) * w, with w of shape [d].
    """
    x = np.asarray(x, dtype=dtype)
    w = np.asarray(w, dtype=dtype)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + dtype(eps)) * w


def rope_cos_sin(positions, d, base):
    """Angles of rotate-half RoPE (HyPE keeps RoPE in the linear layers:
    acgfav.com "SALA 混合架构"; intelliparadigm.com section 2.2).

    theta_i = base^(-2i/d) for i in [0, d/2); angle = position * theta_i.
    Returns (cos, sin), each [len(positions), d/2], fp64.
    """
    half = d // 2
    i = np.arange(half, dtype=F64)
    theta = np.power(F64(base), -2.0 * i / d)
    ang = np.asarray(positions, dtype=F64)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x, positions, base):
    """Rotate dims (i, i + d/2) of x [B, N, H, d] by position * theta_i."""
    x = np.asarray(x, dtype=F64)
    d = x.shape[-1]
    half = d // 2
    c, s = rope_cos_sin(positions, d, base)
    c = c[None, :, None, :]
    s = s[None, :, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def sigmoid(x):
    """Output gate nonlinearity (output gate after each block: paper summary)."""
    x = np.asarray(x, dtype=F64)
    return 1.0 / (1.0 + np.exp(-x))


# ---------------------------------------------------------------------------
# Lightning-style linear attention (three formulations)
# ---------------------------------------------------------------------------

def _state0(state_in, B, H, dk, dv):
    if state_in is None:
        return np.zeros((B, H, dk, dv), dtype=F64)
    return np.array(state_in, dtype=F64, copy=True)


def linear_attention_chunked(q, k, v, lam, chunk, scale=1.0, state_in=None, heads=None):
    """Chunk-wise causal linear attention (Lightning Attention, O(N): acgfav.com
    "SALA 混合架构"; paper section 2.1: constant-size state).

    q, k: [B, N, H, dk]; v: [B, N, H, dv]; lam: [H] decay per head.
    For each chunk of C tokens (the last may be shorter):
        O_intra = (Q_c K_c^T . D) V_c,  D_ij = lam^(i-j) for j <= i, else 0
        O_inter = diag(lam^(i+1)) Q_c S_prev
        S_new   = lam^C S_prev + (diag(lam^(C-1-j)) K_c)^T V_c
    Returns (o [B, N, H, dv] scaled by ``scale``, S_final [B, H, dk, dv]).
    ``heads`` restricts the work to a subset (other heads left NaN / zero).
    """
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    lam = np.asarray(lam, F64)
    B, N, H, dk = q.shape
    dv = v.shape[-1]
    S_all = _state0(state_in, B, H, dk, dv)
    o = np.full((B, N, H, dv), np.nan, dtype=F64)
    hs = range(H) if heads is None else heads
    for b in range(B):
        for h in hs:
            S = S_all[b, h]
            la = lam[h]
            for c0 in range(0, N, chunk):
                c1 = min(N, c0 + chunk)
                L = c1 - c0
                Qc = q[b, c0:c1, h]
                Kc = k[b, c0:c1, h]
                Vc = v[b, c0:c1, h]
                ii = np.arange(L)
                diff = ii[:, None] - ii[None, :]
                D = np.where(diff >= 0, np.power(la, np.maximum(diff, 0)), 0.0)
                o_intra = ((Qc @ Kc.T) * D) @ Vc
                o_inter = np.power(la, ii + 1)[:, None] * (Qc @ S)
                o[b, c0:c1, h] = scale * (o_intra + o_inter)
                S = np.power(la, L) * S + (np.power(la, L - 1 - ii)[:, None] * Kc).T @ Vc
            S_all[b, h] = S
    return o, S_all


def linear_attention_recurrent(q, k, v, lam, scale=1.0, state_in=None):
    """Token-by-token form of the same recurrence: S_t = lam S_{t-1} + k_t^T v_t,
    o_t = scale * q_t S_t.  Used to cross-check the chunked form."""
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    B, N, H, dk = q.shape
    dv = v.shape[-1]
    S_all = _state0(state_in, B, H, dk, dv)
    o = np.empty((B, N, H, dv), dtype=F64)
    for b in range(B):
        for h in range(H):
            S = S_all[b, h]
            for t in range(N):
                S = lam[h] * S + np.outer(k[b, t, h], v[b, t, h])
                o[b, t, h] = scale * (q[b, t, h] @ S)
            S_all[b, h] = S
    return o, S_all


def linear_attention_quadratic(q, k, v, lam, scale=1.0, state_in=None):
    """Quadratic masked form: O = ((Q K^T) . M) V + diag(lam^(t+1)) Q S_in with
    M_ts = lam^(t-s) for s <= t.  Used to cross-check the chunked form."""
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    B, N, H, dk = q.shape
    dv = v.shape[-1]
    S0 = _state0(state_in, B, H, dk, dv)
    t = np.arange(N)
    diff = t[:, None] - t[None, :]
    o = np.empty((B, N, H, dv), dtype=F64)
    for b in range(B):
        for h in range(H):
            M = np.where(diff >= 0, np.power(lam[h], np.maximum(diff, 0)), 0.0)
            A = (q[b, :, h] @ k[b, :, h].T) * M
            o[b, :, h] = scale * (A @ v[b, :, h]
                                  + np.power(lam[h], t + 1)[:, None] * (q[b, :, h] @ S0[b, h]))
    return o


def linear_layer(q, k, v, g, lam, wq, wk, *, chunk=64, pos0=0, rope_base=10000.0,
                 eps=1e-6, scale=1.0, state_in=None, heads=None):
    """One linear SALA layer: QK-RMSNorm, RoPE (linear layers keep RoPE under
    HyPE), chunked linear attention, sigmoid output gate.

    Returns (out [B, N, H, dv], S_final [B, H, dk, dv]).
    """
    N = np.shape(q)[1]
    pos = pos0 + np.arange(N)
    qh = apply_rope(rms_norm(q, wq, eps), pos, rope_base)
    kh = apply_rope(rms_norm(k, wk, eps), pos, rope_base)
    o, S = linear_attention_chunked(qh, kh, v, lam, chunk, scale, state_in, heads)
    return sigmoid(g) * o, S


# ---------------------------------------------------------------------------
# InfLLM-V2-style block selection
# ---------------------------------------------------------------------------

def block_means(x, block, dtype=F64):
    """Mean over each non-overlapping block of ``block`` tokens.

    x: [B, N, H, d] (N a multiple of block) -> [B, H, N/block, d].
    """
    x = np.asarray(x, dtype)
    B, N, H, d = x.shape
    nb = N // block
    xb = x[:, : nb * block].reshape(B, nb, block, H, d)
    m = xb.sum(axis=2, dtype=dtype) / dtype(block)
    return np.ascontiguousarray(np.transpose(m, (0, 2, 1, 3)))


def block_scores(qbar, kbar, dtype=F64, rows=None):
    """Block scores s[b, g, i, j] = <sum_{h in G(g)} qbar_i^h, kbar_j^g> / sqrt(d).

    qbar: [B, Hq, nq, d] per-head query block means; kbar: [B, Hkv, nb, d].
    Query heads h with h // (Hq/Hkv) == g form the group G(g) (GQA).
    Entries with j > i (non-causal) are -inf.  Query block r of qbar is
    block ``rows[r]`` of the sequence (default: block r, nq == nb).
    """
    qbar = np.asarray(qbar, dtype)
    kbar = np.asarray(kbar, dtype)
    B, Hq, nq, d = qbar.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    G = Hq // Hkv
    qg = qbar.reshape(B, Hkv, G, nq, d).sum(axis=2, dtype=dtype)
    s = np.einsum("bgid,bgjd->bgij", qg, kbar) / dtype(math.sqrt(d))
    qi = np.arange(nq) if rows is None else np.asarray(rows)
    causal = np.arange(nb)[None, :] <= qi[:, None]
    return np.where(causal[None, None], s, -np.inf)


def selected_count(b, topk, n_init, n_local):
    """Number of blocks query block b attends to under the reading above."""
    init = set(range(0, min(n_init, b + 1)))
    local = set(range(max(0, b - n_local + 1), b + 1))
    n_cand = max(0, b - n_local + 1 - n_init)
    return len(init | local) + min(topk, n_cand)


def select_row(scores_row, b, topk, n_init, n_local):
    """Selected blocks of query block b (ascending list of ints).

    Initial blocks [0, n_init) and local blocks [b-n_local+1, b] (clipped to
    [0, b]) are always kept; the top-k of the candidates [n_init, b-n_local]
    by score, ties to the lower block index, are added.
    """
    init = set(range(0, min(n_init, b + 1)))
    local = set(range(max(0, b - n_local + 1), b + 1))
    lo, hi = n_init, b - n_local  # inclusive candidate range
    chosen = set()
    if hi >= lo and topk > 0:
        cand = np.arange(lo, hi + 1)
        sc = np.asarray(scores_row)[cand]
        order = np.lexsort((cand, -sc))  # primary: score desc; secondary: index asc
        chosen = set(int(j) for j in cand[order[:topk]])
    return sorted(init | local | chosen)


def select_blocks(scores, topk, n_init, n_local, rows=None):
    """Index lists [B, Hkv, nb, topk + n_init + n_local] int32, -1 padded.

    ``rows`` (optional iterable of query blocks) restricts the work; other rows
    are left filled with -2.
    """
    B, Hkv, nb, _ = scores.shape
    width = topk + n_init + n_local
    idx = np.full((B, Hkv, nb, width), -2, dtype=np.int32)
    rs = range(nb) if rows is None else rows
    for b in range(B):
        for g in range(Hkv):
            for i in rs:
                sel = select_row(scores[b, g, i], i, topk, n_init, n_local)
                idx[b, g, i, :] = -1
                idx[b, g, i, : len(sel)] = sel
    return idx


def _selection_inputs(x, w, eps, block, sd, exact):
    """Block means of the normalised rows of x in the precision ``sd`` of the
    ranking (the fp64 normalised values themselves when sd is fp64)."""
    xs = exact if sd is F64 else rms_norm(np.asarray(x, sd), np.asarray(w, sd), eps, dtype=sd)
    return block_means(xs, block, sd)


def sparse_select(q, k, wq, wk, *, block=64, topk=16, n_init=1, n_local=2, eps=1e-6,
                  score_dtype=F64, rows=None):
    """Selection stage of the sparse layer (NoPE: no RoPE in sparse layers).

    Returns (q_hat, k_hat, kbar, idx, scores): q_hat / k_hat / kbar in fp64,
    scores [B, Hkv, nb, nb] and idx [B, Hkv, nb, W] ranked in ``score_dtype``
    (fp64 by default) throughout (normalisation, block means, group sum, dot
    product).  ``rows`` restricts the index lists to those query blocks.
    """
    qh = rms_norm(q, wq, eps)
    kh = rms_norm(k, wk, eps)
    kbar = block_means(kh, block)
    sd = score_dtype
    scores = block_scores(_selection_inputs(q, wq, eps, block, sd, qh),
                          _selection_inputs(k, wk, eps, block, sd, kh), sd)
    idx = select_blocks(scores, topk, n_init, n_local, rows)
    return qh, kh, kbar, idx, scores


def sparse_select_rows(q_rows, rows, k, wq, wk, *, block=64, topk=16, n_init=1, n_local=2,
                       eps=1e-6, score_dtype=F64):
    """Selection of the query blocks ``rows`` only.

    q_rows: [B, R*block, Hq, d], the raw queries of query blocks rows[0..R)
    in that order; k: [B, N, Hkv, d] all raw keys.  Same definitions as
    ``sparse_select`` restricted to those blocks.  Returns (q_hat_rows,
    k_hat, kbar, idx [B, Hkv, R, W], scores [B, Hkv, R, nb]).
    """
    rows = [int(i) for i in rows]
    qh = rms_norm(q_rows, wq, eps)
    kh = rms_norm(k, wk, eps)
    kbar = block_means(kh, block)
    sd = score_dtype
    scores = block_scores(_selection_inputs(q_rows, wq, eps, block, sd, qh),
                          _selection_inputs(k, wk, eps, block, sd, kh), sd, rows=rows)
    B, Hkv = scores.shape[:2]
    idx = np.full((B, Hkv, len(rows), topk + n_init + n_local), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            for r, i in enumerate(rows):
                sel = select_row(scores[b, g, r], i, topk, n_init, n_local)
                idx[b, g, r, : len(sel)] = sel
    return qh, kh, kbar, idx, scores


def token_softmax_importance(qh_rows, kbar, rows, block, n_init, n_local):
    """Block importance of the token-level selection variant.

    Reading of the InfLLM-V2 block selection that the pages name (paper
    summary and section 2.1; acgfav.com "SALA 混合架构": "fine-grained block
    selection"): every query token t of query block i and every q head h of
    kv group g scores each candidate key block j in [n_init, i - n_local]
    against that block's mean normalised key, z = <q^_t^h, kbar_j^g> / sqrt(d);
    the scores of one (token, head) are turned into a distribution over the
    candidate blocks by a softmax; the importance of block j for query block
    i is the probability mass all tokens of the block and all heads of the
    group give it: I[b, g, r, j] = sum_{t in block rows[r]} sum_{h in G(g)}
    softmax_j(z_t^h)(j).  Non-candidates are -inf.

    qh_rows: [B, R*block, Hq, d] normalised queries of blocks rows[0..R);
    kbar: [B, Hkv, nb, d].  Returns [B, Hkv, R, nb] (fp64).
    """
    qh_rows = np.asarray(qh_rows, F64)
    kbar = np.asarray(kbar, F64)
    B, _, Hq, d = qh_rows.shape
    Hkv, nb = kbar.shape[1], kbar.shape[2]
    G = Hq // Hkv
    imp = np.full((B, Hkv, len(rows), nb), -np.inf, dtype=F64)
    for b in range(B):
        for g in range(Hkv):
            for r, i in enumerate(rows):
                cand = np.arange(n_init, i - n_local + 1)
                if len(cand) == 0:
                    continue
                Q = qh_rows[b, r * block:(r + 1) * block, g * G:(g + 1) * G].reshape(-1, d)
                z = (Q @ kbar[b, g, cand].T) / math.sqrt(d)          # [T*G, C]
                z = z - z.max(axis=1, keepdims=True)
                p = np.exp(z)
                p = p / p.sum(axis=1, keepdims=True)
                imp[b, g, r, cand] = p.sum(axis=0)
    return imp


def select_token_softmax(q, k, wq, wk, *, block=64, topk=16, n_init=1, n_local=2, eps=1e-6,
                         rows=None):
    """Selection stage of the token-level variant (``token_softmax_importance``),
    with the same initial / local blocks, top-k rule and tie-break as
    ``select_row``.  Returns (q_hat, k_hat, kbar, idx, importance); ``rows``
    restricts the work to those query blocks (importance rows then follow
    ``rows``; idx keeps all nb rows, others -2)."""
    qh = rms_norm(q, wq, eps)
    kh = rms_norm(k, wk, eps)
    kbar = block_means(kh, block)
    B, N, Hq, d = qh.shape
    nb = N // block
    rs = list(range(nb)) if rows is None else [int(i) for i in rows]
    q_rows = np.concatenate([qh[:, i * block:(i + 1) * block] for i in rs], axis=1)
    imp = token_softmax_importance(q_rows, kbar, rs, block, n_init, n_local)
    Hkv = kbar.shape[1]
    idx = np.full((B, Hkv, nb, topk + n_init + n_local), -2, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            for r, i in enumerate(rs):
                sel = select_row(imp[b, g, r], i, topk, n_init, n_local)
                idx[b, g, i, :] = -1
                idx[b, g, i, : len(sel)] = sel
    return qh, kh, kbar, idx, imp


# ---------------------------------------------------------------------------
# Gathered block-sparse attention
# ---------------------------------------------------------------------------

def sparse_attention_rows(qh_rows, kh, v, idx_rows, rows, block, scale=None):
    """Exact softmax attention of the query blocks ``rows`` over their
    selected key blocks.

    qh_rows: [B, R*block, Hq, d] normalised queries of blocks rows[0..R) in
    that order; kh, v: [B, N, Hkv, d]; idx_rows: [B, Hkv, R, W] their index
    lists (-1 padded).  Query t of block i (= rows[r]) and head h (kv head
    h // (Hq/Hkv)) attends to every key s in a selected block with s <= t,
    logits scaled by ``scale`` (default 1/sqrt(d)).  Returns [B, R*block, Hq, dv].
    """
    qh_rows = np.asarray(qh_rows, F64)
    kh = np.asarray(kh, F64)
    v = np.asarray(v, F64)
    B, _, Hq, d = qh_rows.shape
    Hkv = kh.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((B, len(rows) * block, Hq, v.shape[-1]), dtype=F64)
    for b in range(B):
        for g in range(Hkv):
            for r, i in enumerate(rows):
                sel = [int(j) for j in idx_rows[b, g, r] if j >= 0]
                pos = np.concatenate([np.arange(j * block, (j + 1) * block) for j in sel])
                K = kh[b, pos, g]                      # [L, d]
                V = v[b, pos, g]
                t = np.arange(i * block, (i + 1) * block)
                Q = qh_rows[b, r * block:(r + 1) * block, g * G:(g + 1) * G]   # [T, G, d]
                T = Q.shape[0]
                logits = (Q.reshape(T * G, d) @ K.T).reshape(T, G, -1) * scale
                mask = pos[None, :] <= t[:, None]       # [T, L]
                logits = np.where(mask[:, None, :], logits, -np.inf)
                m = logits.max(axis=-1, keepdims=True)
                p = np.exp(logits - m)
                p = p / p.sum(axis=-1, keepdims=True)
                o[b, r * block:(r + 1) * block, g * G:(g + 1) * G] = \
                    (p.reshape(T * G, -1) @ V).reshape(T, G, -1)
    return o


def sparse_attention(qh, kh, v, idx, block, scale=None, query_blocks=None):
    """Exact softmax attention of each query over its selected key blocks.

    qh: [B, N, Hq, d] normalised queries; kh, v: [B, N, Hkv, d]; idx as from
    ``select_blocks``.  The definition is ``sparse_attention_rows`` applied
    to every query block (or to ``query_blocks``); the others are left NaN.
    """
    qh = np.asarray(qh, F64)
    B, N, Hq, d = qh.shape
    nb = N // block
    rows = list(range(nb)) if query_blocks is None else [int(i) for i in query_blocks]
    o = np.full((B, N, Hq, np.shape(v)[-1]), np.nan, dtype=F64)
    if not rows:
        return o
    q_rows = np.concatenate([qh[:, i * block:(i + 1) * block] for i in rows], axis=1)
    o_rows = sparse_attention_rows(q_rows, kh, v, np.asarray(idx)[:, :, rows], rows, block, scale)
    for r, i in enumerate(rows):
        o[:, i * block:(i + 1) * block] = o_rows[:, r * block:(r + 1) * block]
    return o


def sparse_layer(q, k, v, g, wq, wk, *, block=64, topk=16, n_init=1, n_local=2,
                 eps=1e-6, scale=None, score_dtype=F64, query_blocks=None):
    """One sparse SALA layer: QK-RMSNorm without RoPE (NoPE), block selection,
    gathered exact attention, sigmoid output gate.

    Returns (out, (q_hat, k_hat, kbar, idx, scores)).
    """
    qh, kh, kbar, idx, scores = sparse_select(
        q, k, wq, wk, block=block, topk=topk, n_init=n_init, n_local=n_local, eps=eps,
        score_dtype=score_dtype, rows=query_blocks)
    o = sparse_attention(qh, kh, v, idx, block, scale, query_blocks)
    return sigmoid(g) * o, (qh, kh, kbar, idx, scores)


def sparse_layer_rows(q_rows, g_rows, rows, k, v, wq, wk, *, block=64, topk=16, n_init=1,
                      n_local=2, eps=1e-6, scale=None, score_dtype=F64):
    """``sparse_layer`` for the query blocks ``rows`` only: q_rows / g_rows
    are the raw queries / gate values of those blocks ([B, R*block, Hq, d],
    in the order of ``rows``); k, v cover the whole sequence.

    Returns (out_rows, (q_hat_rows, k_hat, kbar, idx_rows, scores_rows)).
    """
    qh, kh, kbar, idx, scores = sparse_select_rows(
        q_rows, rows, k, wq, wk, block=block, topk=topk, n_init=n_init, n_local=n_local,
        eps=eps, score_dtype=score_dtype)
    o = sparse_attention_rows(qh, kh, v, idx, rows, block, scale)
    return sigmoid(g_rows) * o, (qh, kh, kbar, idx, scores)


# ---------------------------------------------------------------------------
# Decode (one new token)
# ---------------------------------------------------------------------------

def decode_linear_step(S, q, k, v, g, lam, wq, wk, pos, *, rope_base=10000.0, eps=1e-6,
                       scale=1.0):
    """One decode token of a linear layer (constant-size state, paper section 2.1).

    S: [B, H, dk, dv]; q, k, g: [B, H, d]; v: [B, H, dv]; pos: its position.
    S_new = lam S + k_hat^T v;  out = sigmoid(g) * scale * q_hat S_new.
    Returns (out [B, H, dv], S_new).
    """
    qh = apply_rope(rms_norm(np.asarray(q)[:, None], wq, eps), [pos], rope_base)[:, 0]
    kh = apply_rope(rms_norm(np.asarray(k)[:, None], wk, eps), [pos], rope_base)[:, 0]
    lam = np.asarray(lam, F64)
    S_new = lam[None, :, None, None] * np.asarray(S, F64) + \
        np.einsum("bhk,bhv->bhkv", kh, np.asarray(v, F64))
    o = scale * np.einsum("bhk,bhkv->bhv", qh, S_new)
    return sigmoid(g) * o, S_new


def decode_sparse_step(k_hist, v_hist, q, g, wq, wk, pos, *, block=64, topk=64, n_init=1,
                       n_local=4, eps=1e-6, scale=None, score_dtype=F64):
    """One decode token of the sparse layer at position ``pos``.

    k_hist, v_hist: raw keys / values of positions [0, pos] ([B, pos+1, Hkv, d]),
    the last row being the new token.  The query "block" is the single new
    token: its group query is sum_{h in G(g)} q_hat^h; the scored candidates
    are the complete blocks [n_init, b - n_local] with b = pos // block; the
    block holding ``pos`` is local; attention is exact over the selected
    blocks' keys at positions <= pos.  Returns (out [B, Hq, d], idx).
    """
    k_hist = np.asarray(k_hist)
    B, L, Hkv, d = k_hist.shape
    assert L == pos + 1
    q = np.asarray(q)
    Hq = q.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    kh = rms_norm(k_hist, wk, eps)
    qh = rms_norm(q, wq, eps)                                    # [B, Hq, d]
    sd = score_dtype
    kh_s = rms_norm(np.asarray(k_hist, sd), np.asarray(wk, sd), eps, dtype=sd)
    qh_s = rms_norm(np.asarray(q, sd), np.asarray(wq, sd), eps, dtype=sd)
    nb_done = L // block
    kbar_s = block_means(kh_s[:, : nb_done * block], block, sd) if nb_done else None
    bcur = pos // block
    width = topk + n_init + n_local
    idx = np.full((B, Hkv, width), -1, dtype=np.int32)
    o = np.empty((B, Hq, np.asarray(v_hist).shape[-1]), dtype=F64)
    v_hist = np.asarray(v_hist, F64)
    for b in range(B):
        for gg in range(Hkv):
            qg = qh_s[b, gg * G:(gg + 1) * G].sum(axis=0, dtype=sd)
            row = np.full(bcur + 1, -np.inf, dtype=sd)
            if kbar_s is not None:
                nscore = min(nb_done, bcur + 1)
                row[:nscore] = (kbar_s[b, gg, :nscore] @ qg) / sd(math.sqrt(d))
            sel = select_row(row, bcur, topk, n_init, n_local)
            idx[b, gg, : len(sel)] = sel
            pos_list = np.concatenate([np.arange(j * block, min((j + 1) * block, L)) for j in sel])
            K = kh[b, pos_list, gg]
            V = v_hist[b, pos_list, gg]
            logits = qh[b, gg * G:(gg + 1) * G] @ K.T * scale       # [G, Lsel]
            m = logits.max(axis=-1, keepdims=True)
            p = np.exp(logits - m)
            p /= p.sum(axis=-1, keepdims=True)
            o[b, gg * G:(gg + 1) * G] = p @ V
    return sigmoid(g) * o, idx


# ---------------------------------------------------------------------------
# Full decoder block around the attention (synthetic weights)
# ---------------------------------------------------------------------------

def silu(x):
    """x * sigmoid(x), the gate of the SwiGLU feed-forward network."""
    x = np.asarray(x, F64)
    return x / (1.0 + np.exp(-x))


def sala_block(x, w, kind, *, q_heads, kv_heads, head_dim, eps=1e-6, lam=None, chunk=64,
               pos0=0, rope_base=10000.0, block=64, topk=16, n_init=1, n_local=2):
    """One SALA decoder block: attention sub-block and feed-forward sub-block,
    each pre-normalised and added to the residual stream.

    The pages fix the block structure only in words: every attention block
    (linear or sparse) is followed by an FFN block (MiniCPM-SALA paper,
    section 2.1), the attention output passes an output gate (summary).  The
    rest is the plainest reading for a model of this family: RMSNorm before
    each sub-block, bias-free projections q, k, v, gate from the normalised
    input, the attention of this module (``linear_layer`` or
    ``sparse_layer``), an output projection added to the residual, and a
    SwiGLU FFN (silu(h W1^T) * (h W3^T)) W2^T added to the residual.

    x: [B, N, hidden]; w: dict with norm_attn [hidden], wq [Hq*d, hidden],
    wk / wv [Hkv*d, hidden], wg [Hq*d, hidden], qk_q / qk_k [d] (QK-RMSNorm
    weights), wo [hidden, Hq*d], norm_ffn [hidden], w1 / w3 [ffn, hidden],
    w2 [hidden, ffn] (torch Linear layout: [out, in]).  kind "linear" uses
    q_heads for k and v too.  Returns y [B, N, hidden].
    """
    x = np.asarray(x, F64)
    B, N, hidden = x.shape
    W = {key: np.asarray(val, F64) for key, val in w.items()}
    xn = rms_norm(x, W["norm_attn"], eps)
    hk = q_heads if kind == "linear" else kv_heads
    q = (xn @ W["wq"].T).reshape(B, N, q_heads, head_dim)
    k = (xn @ W["wk"].T).reshape(B, N, hk, head_dim)
    v = (xn @ W["wv"].T).reshape(B, N, hk, head_dim)
    g = (xn @ W["wg"].T).reshape(B, N, q_heads, head_dim)
    if kind == "linear":
        a, _ = linear_layer(q, k, v, g, lam, W["qk_q"], W["qk_k"], chunk=chunk, pos0=pos0,
                            rope_base=rope_base, eps=eps)
    else:
        a, _ = sparse_layer(q, k, v, g, W["qk_q"], W["qk_k"], block=block, topk=topk,
                            n_init=n_init, n_local=n_local, eps=eps)
    h = x + a.reshape(B, N, q_heads * head_dim) @ W["wo"].T
    hn = rms_norm(h, W["norm_ffn"], eps)
    return h + (silu(hn @ W["w1"].T) * (hn @ W["w3"].T)) @ W["w2"].T

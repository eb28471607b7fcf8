"""The oracle against its pins, and the pins against planted mistakes (CPU only)."""
import importlib.util
import os
import sys
import types

import pytest

import oracle
from tests import oracle_pins as pins

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "sala_oracle.py")


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(oracle)


# Planted mistakes: (description, original text, mutated text).  Each is a
# plausible slip (a dropped term, a wrong sign or index, a transposed operand);
# the pins must reject every one of them.
MUTANTS = [
    ("rmsnorm drops the square", "np.mean(x * x, axis=-1", "np.mean(np.abs(x), axis=-1"),
    ("rmsnorm eps outside the root", "np.sqrt(ms + dtype(eps))", "(np.sqrt(ms) + dtype(eps))"),
    ("rope sign flipped", "x1 * c - x2 * s, x2 * c + x1 * s", "x1 * c + x2 * s, x2 * c - x1 * s"),
    ("rope theta exponent", "-2.0 * i / d", "-1.0 * i / d"),
    ("rope interleaved pairs", "x1 = x[..., :half]", "x1 = x[..., 0::2]"),
    ("inter-chunk decay off by one", "np.power(la, ii + 1)[:, None]", "np.power(la, ii)[:, None]"),
    ("state carry decay off by one", "np.power(la, L - 1 - ii)", "np.power(la, L - ii)"),
    ("chunk state decay dropped", "S = np.power(la, L) * S +", "S = S +"),
    ("intra-chunk mask not causal", "np.where(diff >= 0, np.power(la, np.maximum(diff, 0)), 0.0)\n"
     "                o_intra", "np.power(la, np.abs(diff))\n                o_intra"),
    ("state transposed", "(Qc @ S)", "(Qc @ S.T[:S.shape[0], :S.shape[1]] if S.shape[0] == S.shape[1] else Qc @ S)"),
    ("gate missing", "state_in, heads)\n    return sigmoid(g) * o, S", "state_in, heads)\n    return o, S"),
    ("scores not scaled", "/ dtype(math.sqrt(d))", "/ dtype(1.0)"),
    ("group mapping interleaved", "qg = qbar.reshape(B, Hkv, G, nq, d)", "qg = qbar.reshape(B, G, Hkv, nq, d).swapaxes(1, 2)"),
    ("tie-break to higher index", "np.lexsort((cand, -sc))", "np.lexsort((-cand, -sc))"),
    ("local window one short", "local = set(range(max(0, b - n_local + 1), b + 1))\n    lo, hi",
     "local = set(range(max(0, b - n_local + 2), b + 1))\n    lo, hi"),
    ("candidates overlap local", "lo, hi = n_init, b - n_local", "lo, hi = n_init, b - 1"),
    ("causal mask off by one", "mask = pos[None, :] <= t[:, None]", "mask = pos[None, :] < t[:, None] + 2"),
    ("softmax scale missing", "scale = 1.0 / math.sqrt(d)\n    o = np.empty(", "scale = 1.0\n    o = np.empty("),
    ("sparse gqa mapping", "Q = qh_rows[b, r * block:(r + 1) * block, g * G:(g + 1) * G]   # [T, G, d]",
     "Q = qh_rows[b, r * block:(r + 1) * block, g::Hkv]   # [T, G, d]"),
    ("token softmax gqa mapping", "Q = qh_rows[b, r * block:(r + 1) * block, g * G:(g + 1) * G].reshape(-1, d)",
     "Q = qh_rows[b, r * block:(r + 1) * block, g::Hkv].reshape(-1, d)"),
    ("row scores ignore the block numbers", "qi = np.arange(nq) if rows is None else np.asarray(rows)",
     "qi = np.arange(nq)"),
    ("row attention uses the row number as the block", "t = np.arange(i * block, (i + 1) * block)",
     "t = np.arange(r * block, (r + 1) * block)"),
    ("selection ranked on unnormalised queries",
     "xs = exact if sd is F64 else", "xs = np.asarray(x, sd) if sd is F64 else"),
    ("decode state update order", "S_new = lam[None, :, None, None] * np.asarray(S, F64) + \\\n"
     "        np.einsum(\"bhk,bhv->bhkv\", kh, np.asarray(v, F64))",
     "S_new = lam[None, :, None, None] * (np.asarray(S, F64) + \\\n"
     "        np.einsum(\"bhk,bhv->bhkv\", kh, np.asarray(v, F64)))"),
    ("token softmax over all blocks", "cand = np.arange(n_init, i - n_local + 1)\n                if len(cand) == 0:",
     "cand = np.arange(0, i + 1)\n                if len(cand) == 0:"),
    ("token importance without the softmax", "p = p / p.sum(axis=1, keepdims=True)\n                imp",
     "p = z\n                imp"),
    ("block ffn gate and up swapped", "(silu(hn @ W[\"w1\"].T) * (hn @ W[\"w3\"].T))",
     "(silu(hn @ W[\"w3\"].T) * (hn @ W[\"w1\"].T))"),
    ("block residual dropped", "h = x + a.reshape(B, N, q_heads * head_dim) @ W[\"wo\"].T",
     "h = a.reshape(B, N, q_heads * head_dim) @ W[\"wo\"].T"),
    ("decode query group sum", "qg = qh_s[b, gg * G:(gg + 1) * G].sum(axis=0, dtype=sd)",
     "qg = qh_s[b, gg * G]"),
]


def _load_mutant(src, name):
    mod = types.ModuleType(name)
    mod.__file__ = ORACLE_SRC
    exec(compile(src, ORACLE_SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("desc,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(desc, orig, mut):
    with open(ORACLE_SRC) as f:
        src = f.read()
    assert src.count(orig) == 1, f"mutation anchor not found exactly once: {desc}"
    mod = _load_mutant(src.replace(orig, mut), "oracle_mutant")
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(mod)
        except Exception as e:  # AssertionError, or the mutant crashing
            failed.append((check.__name__, type(e).__name__))
    assert failed, f"no pin caught the planted mistake: {desc}"

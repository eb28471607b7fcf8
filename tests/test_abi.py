"""libsala C ABI on the host: the library loads, exports every declared entry
point, and rejects bad arguments before touching the device (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sala.h")

sala = pytest.importorskip("hybrid_sparse_linear_lightning_b200.sala")

FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced by a rejected call
MISALIGNED = ctypes.c_void_p(0x10008)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sala_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(sala.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sala.EXPORTED)


def test_version_and_strings():
    assert sala.sala_version() >= 100
    for code in range(7):
        assert sala.status_string(code) and sala.status_string(code) != "unknown status"


def _lin(**kw):
    base = dict(batch=1, seqlen=2048, heads=4, head_dim=64, chunk=64)
    base.update(kw)
    return sala.linear_desc(base.pop("batch"), base.pop("seqlen"), base.pop("heads"),
                            base.pop("head_dim"), base.pop("chunk"))


def _call_linear(d, ptr=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return sala.LIB.sala_linear_prefill(ctypes.byref(d), ptr, ptr, ptr, ptr, ptr, ptr, ptr,
                                        None, None, ptr, ws, ws_bytes, None)


def test_linear_validation():
    assert _call_linear(_lin(head_dim=96)) == sala.SALA_ERR_UNSUPPORTED
    assert _call_linear(_lin(seqlen=100)) == sala.SALA_ERR_UNSUPPORTED      # not a chunk multiple
    assert _call_linear(_lin(batch=0)) == sala.SALA_ERR_INVALID_ARG
    assert _call_linear(_lin(), ptr=None) == sala.SALA_ERR_INVALID_ARG
    assert _call_linear(_lin(), ptr=MISALIGNED) == sala.SALA_ERR_INVALID_ARG
    d = _lin()
    need = sala.sala_linear_workspace_size(d)
    assert need > 0
    assert _call_linear(d, ws_bytes=need - 1) == sala.SALA_ERR_WORKSPACE
    assert sala.LIB.sala_linear_prefill(None, *([FAKE] * 10), FAKE, 1 << 40, None) == \
        sala.SALA_ERR_INVALID_ARG
    assert sala.sala_linear_workspace_size(_lin(head_dim=96)) == 0


def _sp(**kw):
    base = dict(batch=1, seqlen=2048, q_heads=4, kv_heads=1, head_dim=64, block=64, topk=4,
                n_init=1, n_local=2, selection=sala.SALA_SELECT_BLOCK_MEAN)
    base.update(kw)
    return sala.SparseDesc(base["batch"], base["seqlen"], base["q_heads"], base["kv_heads"],
                           base["head_dim"], base["block"], base["topk"], base["n_init"],
                           base["n_local"], sala.SALA_BF16, 1e-6, 0.0, base["selection"])


def _call_select(d, ptr=FAKE, ws_bytes=1 << 40):
    return sala.LIB.sala_sparse_select(ctypes.byref(d), ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr,
                                       FAKE, ws_bytes, None)


def test_sparse_validation():
    assert _call_select(_sp(q_heads=6, kv_heads=4)) == sala.SALA_ERR_INVALID_ARG
    assert _call_select(_sp(n_local=0)) == sala.SALA_ERR_INVALID_ARG
    assert _call_select(_sp(topk=-1)) == sala.SALA_ERR_INVALID_ARG
    assert _call_select(_sp(block=32)) == sala.SALA_ERR_UNSUPPORTED
    assert _call_select(_sp(seqlen=2000)) == sala.SALA_ERR_UNSUPPORTED
    assert _call_select(_sp(head_dim=80)) == sala.SALA_ERR_UNSUPPORTED
    assert _call_select(_sp(), ptr=MISALIGNED) == sala.SALA_ERR_INVALID_ARG
    d = _sp()
    assert sala.sala_sparse_index_width(d) == 7
    need = sala.sala_sparse_workspace_size(d)
    assert need >= 32 * 64 * 4
    assert _call_select(d, ws_bytes=need - 1) == sala.SALA_ERR_WORKSPACE
    assert sala.LIB.sala_sparse_prefill(ctypes.byref(_sp(head_dim=80)), *([FAKE] * 6), None, 0,
                                        None) == sala.SALA_ERR_UNSUPPORTED
    # selection rule: unknown value, token-softmax beyond its 8192-block limit
    assert _call_select(_sp(selection=2)) == sala.SALA_ERR_INVALID_ARG
    assert _call_select(_sp(selection=1, seqlen=64 * 8193)) == sala.SALA_ERR_UNSUPPORTED
    assert sala.sala_sparse_workspace_size(_sp(selection=1)) > 0


def test_decode_validation():
    d = sala.DecodeDesc(_lin(), _sp(), 3, 4096)
    assert sala.sala_decode_workspace_size(d) > 0
    io = sala.DecodeIO()
    # cur_len beyond the cache
    assert sala.LIB.sala_decode_step(ctypes.byref(d), ctypes.byref(io), FAKE, FAKE, FAKE, FAKE,
                                     4096, FAKE, 1 << 40, None) == sala.SALA_ERR_INVALID_ARG
    # missing per-layer pointers
    assert sala.LIB.sala_decode_step(ctypes.byref(d), ctypes.byref(io), FAKE, FAKE, FAKE, FAKE,
                                     10, FAKE, 1 << 40, None) == sala.SALA_ERR_INVALID_ARG
    bad = sala.DecodeDesc(_lin(), _sp(), 0, 4096)
    assert sala.sala_decode_workspace_size(bad) == 0
    bad = sala.DecodeDesc(_lin(), _sp(), 3, 100)      # capacity not a block multiple
    assert sala.sala_decode_workspace_size(bad) == 0
    bad = sala.DecodeDesc(_lin(), _sp(selection=1), 3, 4096)   # prefill-only selection rule
    assert sala.sala_decode_workspace_size(bad) == 0

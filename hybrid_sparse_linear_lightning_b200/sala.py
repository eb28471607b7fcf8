"""Thin ctypes binding of libsala (include/sala.h).

Argument marshalling only: every step of the attention path runs in the
library's CUDA kernels.  torch tensors are passed as raw device pointers;
the caller (or the ``*_alloc`` helpers here) owns all memory.  Importing this
module loads ``libsala.so`` from the package directory and raises when it is
missing: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsala.so")

SALA_OK = 0
SALA_ERR_INVALID_ARG = 1
SALA_ERR_UNSUPPORTED = 2
SALA_ERR_CUDA = 3
SALA_ERR_TIMEOUT = 4
SALA_ERR_WORKSPACE = 5
SALA_ERR_DEVICE_FAULT = 6
SALA_F32 = 0
SALA_BF16 = 1
SALA_SELECT_BLOCK_MEAN = 0
SALA_SELECT_TOKEN_SOFTMAX = 1
SALA_MAX_LAYERS = 8

EXPORTED = [
    "sala_sparse_index_width", "sala_linear_workspace_size", "sala_linear_prefill",
    "sala_sparse_workspace_size", "sala_sparse_select", "sala_sparse_prefill",
    "sala_decode_workspace_size", "sala_decode_step", "sala_status_string",
    "sala_get_device_status", "sala_version", "sala_kernel_launch_count",
    "sala_sparse_select_noalloc", "sala_selftest_bounded_wait",
    "sala_sparse_select_begin", "sala_sparse_select_finish",
    "sala_block_workspace_size", "sala_block_prefill",
]
NOALLOC_SCRATCH_BYTES = 4 << 20


class SalaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class LinearDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("chunk", ctypes.c_int), ("dtype", ctypes.c_int),
                ("pos0", ctypes.c_int64), ("rope_base", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("scale", ctypes.c_float)]


class SparseDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("q_heads", ctypes.c_int),
                ("kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("block", ctypes.c_int),
                ("topk", ctypes.c_int), ("n_init", ctypes.c_int), ("n_local", ctypes.c_int),
                ("dtype", ctypes.c_int), ("rms_eps", ctypes.c_float), ("scale", ctypes.c_float),
                ("selection", ctypes.c_int)]


class DecodeDesc(ctypes.Structure):
    _fields_ = [("lin", LinearDesc), ("sp", SparseDesc), ("n_linear", ctypes.c_int),
                ("cache_capacity", ctypes.c_int64)]


class BlockDesc(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("ffn", ctypes.c_int), ("rms_eps", ctypes.c_float)]


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("norm_attn", "wq", "wk", "wv", "wg", "qk_norm_q", "qk_norm_k", "wo", "norm_ffn",
                 "w13", "w2")]


_PA = ctypes.c_void_p * SALA_MAX_LAYERS


class DecodeIO(ctypes.Structure):
    _fields_ = [("q", _PA), ("k", _PA), ("v", _PA), ("gate", _PA), ("wq", _PA), ("wk", _PA),
                ("lambda_", _PA), ("lin_state", _PA), ("out", _PA)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsala.so not built at {LIB_PATH}; run "
                          "`python -m hybrid_sparse_linear_lightning_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    S = ctypes.c_size_t
    I = ctypes.c_int
    sig = {
        "sala_sparse_index_width": (I, [P]),
        "sala_linear_workspace_size": (S, [P]),
        "sala_linear_prefill": (I, [P] + [P] * 10 + [P, S, P]),
        "sala_sparse_workspace_size": (S, [P]),
        "sala_sparse_select": (I, [P] + [P] * 8 + [P, S, P]),
        "sala_sparse_prefill": (I, [P] + [P] * 6 + [P, S, P]),
        "sala_decode_workspace_size": (S, [P]),
        "sala_decode_step": (I, [P, P, P, P, P, P, ctypes.c_int64, P, S, P]),
        "sala_status_string": (ctypes.c_char_p, [I]),
        "sala_get_device_status": (I, [P]),
        "sala_version": (I, []),
        "sala_kernel_launch_count": (ctypes.c_uint64, []),
        "sala_sparse_select_noalloc": (I, [P] + [P] * 8 + [P]),
        "sala_selftest_bounded_wait": (I, [P]),
        "sala_sparse_select_begin": (I, [P] + [P] * 8 + [P]),
        "sala_sparse_select_finish": (I, [P, P, P, P, P]),
        "sala_block_workspace_size": (S, [P, P, P]),
        "sala_block_prefill": (I, [P, P, P, P, P, P, P, P, P, S, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


LIB = _load()


def status_string(s: int) -> str:
    return LIB.sala_status_string(int(s)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, what: str):
    if status != SALA_OK:
        raise SalaError(status, what)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return SALA_F32
    if dt == torch.bfloat16:
        return SALA_BF16
    raise ValueError(f"unsupported dtype {dt}")


def linear_desc(batch, seqlen, heads, head_dim, chunk=64, dtype=torch.bfloat16, pos0=0,
                rope_base=10000.0, rms_eps=1e-6, scale=1.0) -> LinearDesc:
    return LinearDesc(batch, seqlen, heads, head_dim, chunk, dtype_code(dtype), pos0,
                      rope_base, rms_eps, scale)


def sparse_desc(batch, seqlen, q_heads, kv_heads, head_dim, block=64, topk=16, n_init=1,
                n_local=2, dtype=torch.bfloat16, rms_eps=1e-6, scale=0.0,
                selection=SALA_SELECT_BLOCK_MEAN) -> SparseDesc:
    return SparseDesc(batch, seqlen, q_heads, kv_heads, head_dim, block, topk, n_init, n_local,
                      dtype_code(dtype), rms_eps, scale, selection)


# ---------------------------------------------------------------------------- raw entry points

def sala_linear_workspace_size(d: LinearDesc) -> int:
    return int(LIB.sala_linear_workspace_size(ctypes.byref(d)))


def sala_linear_prefill(d: LinearDesc, q, k, v, gate, lam, wq, wk, state_in, state_out, out,
                        workspace, stream=None) -> int:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return LIB.sala_linear_prefill(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(gate),
                                   _ptr(lam), _ptr(wq), _ptr(wk), _ptr(state_in),
                                   _ptr(state_out), _ptr(out), _ptr(workspace), ws_bytes,
                                   _stream(stream))


def sala_sparse_workspace_size(d: SparseDesc) -> int:
    return int(LIB.sala_sparse_workspace_size(ctypes.byref(d)))


def sala_sparse_index_width(d: SparseDesc) -> int:
    return int(LIB.sala_sparse_index_width(ctypes.byref(d)))


def sala_sparse_select(d: SparseDesc, q, k, wq, wk, q_norm, k_norm, kbar, idx, workspace,
                       stream=None) -> int:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return LIB.sala_sparse_select(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(wq), _ptr(wk),
                                  _ptr(q_norm), _ptr(k_norm), _ptr(kbar), _ptr(idx),
                                  _ptr(workspace), ws_bytes, _stream(stream))


def sala_sparse_select_noalloc(d: SparseDesc, q, k, wq, wk, q_norm, k_norm, kbar, idx,
                               stream=None) -> int:
    """sala_sparse_select without a workspace: for callers that cannot allocate
    device memory.  Its scratch is a fixed 4 MiB array inside the library
    (shapes needing more return SALA_ERR_WORKSPACE); calls on one device must
    not overlap on the GPU."""
    return LIB.sala_sparse_select_noalloc(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(wq), _ptr(wk),
                                          _ptr(q_norm), _ptr(k_norm), _ptr(kbar), _ptr(idx),
                                          _stream(stream))


def sala_sparse_select_begin(d: SparseDesc, q, k, wq, wk, q_norm, k_norm, kbar, qsum,
                             stream=None) -> int:
    return LIB.sala_sparse_select_begin(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(wq), _ptr(wk),
                                        _ptr(q_norm), _ptr(k_norm), _ptr(kbar), _ptr(qsum),
                                        _stream(stream))


def sala_sparse_select_finish(d: SparseDesc, qsum, kbar, idx, stream=None) -> int:
    return LIB.sala_sparse_select_finish(ctypes.byref(d), _ptr(qsum), _ptr(kbar), _ptr(idx),
                                         _stream(stream))


def sala_sparse_prefill(d: SparseDesc, q_norm, k_norm, v, gate, idx, out, workspace=None,
                        stream=None) -> int:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return LIB.sala_sparse_prefill(ctypes.byref(d), _ptr(q_norm), _ptr(k_norm), _ptr(v),
                                   _ptr(gate), _ptr(idx), _ptr(out), _ptr(workspace), ws_bytes,
                                   _stream(stream))


def sala_block_workspace_size(b: BlockDesc, lin: Optional[LinearDesc] = None,
                              sp: Optional[SparseDesc] = None) -> int:
    return int(LIB.sala_block_workspace_size(ctypes.byref(b), None if lin is None else ctypes.byref(lin),
                                             None if sp is None else ctypes.byref(sp)))


def block_weights(w: dict) -> BlockWeights:
    """ctypes view of a dict of device tensors (keys as BlockWeights' fields;
    the tensors must stay alive while it is used)."""
    bw = BlockWeights()
    for name, _ in BlockWeights._fields_:
        setattr(bw, name, _ptr(w[name]).value)
    bw._keep = w
    return bw


def sala_block_prefill(b: BlockDesc, lin: Optional[LinearDesc], sp: Optional[SparseDesc],
                       w: BlockWeights, lam, x, y, state_out, workspace, stream=None) -> int:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return LIB.sala_block_prefill(ctypes.byref(b), None if lin is None else ctypes.byref(lin),
                                  None if sp is None else ctypes.byref(sp), ctypes.byref(w),
                                  _ptr(lam), _ptr(x), _ptr(y), _ptr(state_out), _ptr(workspace),
                                  ws_bytes, _stream(stream))


def sala_decode_workspace_size(d: DecodeDesc) -> int:
    return int(LIB.sala_decode_workspace_size(ctypes.byref(d)))


def sala_decode_step(d: DecodeDesc, io: DecodeIO, k_cache, v_cache, kbar, ksum, cur_len: int,
                     workspace, stream=None) -> int:
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return LIB.sala_decode_step(ctypes.byref(d), ctypes.byref(io), _ptr(k_cache), _ptr(v_cache),
                                _ptr(kbar), _ptr(ksum), int(cur_len), _ptr(workspace), ws_bytes,
                                _stream(stream))


def sala_get_device_status(stream=None) -> int:
    return int(LIB.sala_get_device_status(_stream(stream)))


def sala_selftest_bounded_wait(stream=None) -> int:
    return int(LIB.sala_selftest_bounded_wait(_stream(stream)))


def sala_version() -> int:
    return int(LIB.sala_version())


def sala_kernel_launch_count() -> int:
    return int(LIB.sala_kernel_launch_count())


# ---------------------------------------------------------------------------- tensor helpers

def workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def linear_prefill(q, k, v, gate, lam, wq, wk, *, chunk=64, pos0=0, rope_base=10000.0,
                   rms_eps=1e-6, scale=1.0, state_in=None, want_state=False, ws=None,
                   out=None, stream=None):
    """One linear layer forward; returns (out, state_out or None)."""
    B, N, H, D = q.shape
    d = linear_desc(B, N, H, D, chunk, q.dtype, pos0, rope_base, rms_eps, scale)
    if out is None:
        out = torch.empty_like(q)
    st_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device) if want_state else None
    if ws is None:
        ws = workspace(sala_linear_workspace_size(d), q.device)
    _check(sala_linear_prefill(d, q, k, v, gate, lam, wq, wk, state_in, st_out, out, ws, stream),
           "sala_linear_prefill")
    return out, st_out


def sparse_select(q, k, wq, wk, *, block=64, topk=16, n_init=1, n_local=2, rms_eps=1e-6,
                  selection=SALA_SELECT_BLOCK_MEAN, ws=None, outs=None, stream=None):
    """Selection stage; returns (q_norm, k_norm, kbar, idx)."""
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    d = sparse_desc(B, N, Hq, Hkv, D, block, topk, n_init, n_local, q.dtype, rms_eps,
                    selection=selection)
    if outs is None:
        nb = N // block
        outs = (torch.empty((B, N, Hq, D), dtype=torch.bfloat16, device=q.device),
                torch.empty((B, N, Hkv, D), dtype=torch.bfloat16, device=q.device),
                torch.empty((B, nb, Hkv, D), dtype=torch.float32, device=q.device),
                torch.empty((B, Hkv, nb, sala_sparse_index_width(d)), dtype=torch.int32,
                            device=q.device))
    if ws is None:
        ws = workspace(sala_sparse_workspace_size(d), q.device)
    _check(sala_sparse_select(d, q, k, wq, wk, *outs, ws, stream), "sala_sparse_select")
    return outs


def sparse_prefill(q_norm, k_norm, v, gate, idx, *, block=64, topk=16, n_init=1, n_local=2,
                   scale=0.0, out=None, ws=None, stream=None):
    """Gathered sparse attention + gate; returns out (dtype of v)."""
    B, N, Hq, D = q_norm.shape
    Hkv = k_norm.shape[2]
    d = sparse_desc(B, N, Hq, Hkv, D, block, topk, n_init, n_local, v.dtype, scale=scale)
    if out is None:
        out = torch.empty((B, N, Hq, D), dtype=v.dtype, device=v.device)
    _check(sala_sparse_prefill(d, q_norm, k_norm, v, gate, idx, out, ws, stream),
           "sala_sparse_prefill")
    return out


def make_decode_io(layers: Sequence, outs: Sequence, states: Sequence, lams: Sequence,
                   wq: torch.Tensor, wk: torch.Tensor) -> DecodeIO:
    """layers: per layer (q, k, v, g); outs: per layer out tensors; states /
    lams: per linear layer.  The same RMSNorm weights serve every layer."""
    io = DecodeIO()
    keep = []
    for l, (q, k, v, g) in enumerate(layers):
        for name, t in (("q", q), ("k", k), ("v", v), ("gate", g), ("wq", wq), ("wk", wk),
                        ("out", outs[l])):
            getattr(io, name)[l] = t.data_ptr()
            keep.append(t)
    for l, (s, lam) in enumerate(zip(states, lams)):
        io.lin_state[l] = s.data_ptr()
        io.lambda_[l] = lam.data_ptr()
    io._keep = keep
    return io

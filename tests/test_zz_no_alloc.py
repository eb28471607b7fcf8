"""The allocation-free selection entry point against the workspace one.

sala_sparse_select_noalloc serves callers that cannot allocate device
memory (an allocator-free runtime, a memory pool that refuses new
allocations): its scratch is a fixed array compiled into the library instead
of a caller workspace.  This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from hybrid_sparse_linear_lightning_b200 import workloads as wl

sala = pytest.importorskip("hybrid_sparse_linear_lightning_b200.sala")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 512K tokens x 2 kv heads x 128 dims of fp32 block sums need 8 MiB > 4 MiB;
    # rejected on the host before anything is launched.
    d = sala.sparse_desc(1, 524288, 32, 2, 128, topk=64, n_init=1, n_local=4)
    assert sala.sala_sparse_workspace_size(d) > sala.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)
    st = sala.LIB.sala_sparse_select_noalloc(ctypes.byref(d), *([fake] * 8), None)
    assert st == sala.SALA_ERR_WORKSPACE


def _run_both(w, seqlen):
    dev = torch.device("cuda")
    sp = w.sparse
    q, k, _, _ = wl.layer_inputs(w, w.n_linear, dev, seqlen=seqlen)
    wt = wl.rms_weights(sp.head_dim, dev)
    d = sala.sparse_desc(w.batch, seqlen, sp.q_heads, sp.kv_heads, sp.head_dim, sp.block,
                         sp.topk, sp.n_init, sp.n_local, w.torch_dtype)
    ref = sala.sparse_select(q, k, wt, wt, block=sp.block, topk=sp.topk, n_init=sp.n_init,
                             n_local=sp.n_local)
    outs = [torch.full_like(t, -7) for t in ref]
    st = sala.sala_sparse_select_noalloc(d, q, k, wt, wt, *outs)
    assert st == sala.SALA_OK, sala.status_string(st)
    torch.cuda.synchronize()
    assert sala.sala_get_device_status() == sala.SALA_OK
    return ref, outs


@pytest.mark.gpu
def test_noalloc_matches_workspace_select_on_two_calls(cuda_device):
    # first call: the largest shape that fits (exactly 4 MiB of scratch);
    # second call: another shape and other inputs (another seed), same array
    for name, seqlen in (("group_256k", 262144), ("group_32k", 32768)):
        ref, got = _run_both(wl.WORKLOADS[name], seqlen)
        qn, kn, kbar, idx = ref
        gq, gk, gkbar, gidx = got
        # same kernels on the same inputs: identical bits, scratch location aside
        assert torch.equal(gq, qn)
        assert torch.equal(gk, kn)
        assert torch.equal(gkbar, kbar)
        assert torch.equal(gidx, idx)

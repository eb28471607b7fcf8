"""Head-sharded prefill plumbing on CPU: two gloo ranks run their head shards
of one linear and one sparse layer through `shard.ShardedGroup`, with the
fp64 oracle standing in for the CUDA kernels (the backend interface of the
module), exchange the sparse layer's block-mean query sums over the kv
group's ranks, gather the heads, and must reproduce the unsharded oracle
layers.  Covers both splits: a kv group spread over the two ranks (the
all-reduce path) and whole kv groups per rank."""
import math
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleBackend:
    """The backend interface of shard.ShardedGroup computed by the oracle (fp64)."""

    def __init__(self, oracle):
        self.o = oracle

    def linear_prefill(self, q, k, v, g, lam, wq, wk, *, chunk, pos0=0, state_in=None,
                       want_state=False):
        out, S = self.o.linear_layer(q.numpy(), k.numpy(), v.numpy(), g.numpy(), lam.numpy(),
                                     wq.numpy(), wk.numpy(), chunk=chunk, pos0=pos0,
                                     state_in=None if state_in is None else state_in.numpy())
        return torch.from_numpy(out), torch.from_numpy(S) if want_state else None

    def select_begin(self, q, k, wq, wk, *, block, topk, n_init, n_local):
        o = self.o
        qh = o.rms_norm(q.numpy(), wq.numpy())
        kh = o.rms_norm(k.numpy(), wk.numpy())
        kbar = o.block_means(kh, block)                      # [B, Hkv, nb, d]
        qbar = o.block_means(qh, block)                      # [B, Hq, nb, d]
        B, Hq, nb, d = qbar.shape
        Hkv = kbar.shape[1]
        qsum = qbar.reshape(B, Hkv, Hq // Hkv, nb, d).sum(axis=2)
        return dict(qh=qh, kh=kh, kbar=kbar, qsum=torch.from_numpy(np.ascontiguousarray(qsum)),
                    block=block, topk=topk, n_init=n_init, n_local=n_local)

    def select_finish(self, sel):
        # the summed group query against the block means: the block-mean rule
        scores = self.o.block_scores(sel["qsum"].numpy(), sel["kbar"])
        return self.o.select_blocks(scores, sel["topk"], sel["n_init"], sel["n_local"])

    def sparse_prefill(self, sel, v, g, idx):
        o = self.o
        att = o.sparse_attention(sel["qh"], sel["kh"], v.numpy(), idx, sel["block"])
        return torch.from_numpy(o.sigmoid(g.numpy()) * att)


def _inputs(Hq, Hkv, H=4, N=512, d=16, seed=5):
    r = np.random.default_rng(seed)
    lin = [torch.from_numpy(r.standard_normal((1, N, H, d))) for _ in range(4)]
    sp = [torch.from_numpy(r.standard_normal((1, N, h, d))) for h in (Hq, Hkv, Hkv, Hq)]
    lam = torch.from_numpy(np.array([0.9, 0.99, 1.0, 0.5][:H]))
    return lin, sp, lam, torch.ones(d, dtype=torch.float64)


def _worker(rank, world, port, Hq, Hkv, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import oracle
    from hybrid_sparse_linear_lightning_b200 import shard
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        lin, sp, lam, w = _inputs(Hq, Hkv)
        subgroups = shard.group_subgroups(world, Hkv)
        grp = shard.ShardedGroup(rank, world, lin[0].shape[2], Hq, Hkv, subgroups,
                                 backend=OracleBackend(oracle))
        lo, hi = grp.lin
        ql, kl, vl, gl = (t[:, :, lo:hi].contiguous() for t in lin)
        lin_out, _ = grp.linear(ql, kl, vl, gl, lam[lo:hi], w, w, chunk=16)
        s = grp.sp
        sq, sk, sv, sg = sp
        sp_out, _ = grp.sparse(sq[:, :, s.q_lo:s.q_hi].contiguous(),
                               sk[:, :, s.kv_lo:s.kv_hi].contiguous(),
                               sv[:, :, s.kv_lo:s.kv_hi].contiguous(),
                               sg[:, :, s.q_lo:s.q_hi].contiguous(), w, w, block=32, topk=3,
                               n_init=1, n_local=2)
        lin_all = shard.gather_heads(lin_out, world)
        sp_all = shard.gather_heads(sp_out, world)
        if rank == 0:
            ref_lin, _ = oracle.linear_layer(*(t.numpy() for t in lin), lam.numpy(), w.numpy(),
                                             w.numpy(), chunk=16)
            ref_sp, _ = oracle.sparse_layer(*(t.numpy() for t in sp), w.numpy(), w.numpy(),
                                            block=32, topk=3, n_init=1, n_local=2)
            q.put((float(np.abs(lin_all.numpy() - ref_lin).max()),
                   float(np.abs(sp_all.numpy() - ref_sp).max()), s.group_ranks))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("Hq,Hkv", [(8, 1), (8, 2)])
def test_head_sharded_group_gloo(Hq, Hkv):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + (os.getpid() % 500) + Hkv
    procs = [ctx.Process(target=_worker, args=(r, 2, port, Hq, Hkv, q)) for r in range(2)]
    for p in procs:
        p.start()
    e_lin, e_sp, ranks = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert e_lin < 1e-12 and e_sp < 1e-12, (e_lin, e_sp)
    assert len(ranks) == (2 if Hkv == 1 else 1)      # the all-reduce path ran when the group split


def test_shard_layout():
    from hybrid_sparse_linear_lightning_b200 import shard
    assert shard.head_range(32, 4, 3) == (24, 32)
    s = shard.sparse_shard(32, 2, 8, 5)              # 4 ranks per kv group, 4 q heads each
    assert (s.q_lo, s.q_hi, s.kv_lo, s.kv_hi, s.group_ranks) == (20, 24, 1, 2, (4, 5, 6, 7))
    s = shard.sparse_shard(32, 2, 2, 1)              # one whole kv group per rank
    assert (s.q_lo, s.q_hi, s.kv_lo, s.kv_hi, s.group_ranks) == (16, 32, 1, 2, (1,))
    with pytest.raises(ValueError):
        shard.sparse_shard(32, 2, 3, 0)
    assert math.isclose(sum(shard.head_range(32, 8, r)[1] - shard.head_range(32, 8, r)[0]
                            for r in range(8)), 32)

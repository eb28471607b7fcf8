"""Head-sharded layer-group prefill over several GPUs (one process per GPU).

The linear layers' heads are independent recurrences, so a rank computes the
heads [lo, hi) of every linear layer from its slice of the inputs and needs
nothing from the others.  The sparse layer's q heads are split the same way;
a kv group (the q heads sharing one key / value head and one block
selection) is either held whole by a rank (world <= kv heads) or spread over
world / kv_heads ranks.  In the second case the selection of the group
needs the block-mean queries summed over ALL its q heads: each rank forms
the sum over its own heads (sala_sparse_select_begin), the ranks of the
group all-reduce it, and each ranks the blocks from the total
(sala_sparse_select_finish) -- the one exchange on the path.  Attention of
a rank's q heads then needs only its group's keys and values, which every
rank of the group holds.  Outputs stay sharded by head; ``gather_heads``
assembles [B, N, H, d] when a caller needs every head.

The compute goes through a backend object (``LibsalaBackend`` by default:
the C ABI on this rank's GPU) so that the orchestration can be exercised on
CPU processes with another backend.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch
import torch.distributed as dist


@dataclasses.dataclass(frozen=True)
class SparseShard:
    q_lo: int             # this rank's q heads [q_lo, q_hi)
    q_hi: int
    kv_lo: int            # the kv heads [kv_lo, kv_hi) those q heads use
    kv_hi: int
    group_ranks: tuple    # ranks that share this rank's kv group (len 1: no exchange)


def head_range(heads: int, world: int, rank: int):
    """Contiguous heads [lo, hi) of `rank` when `heads` are split over `world`."""
    if heads % world:
        raise ValueError(f"{heads} heads do not split over {world} ranks")
    n = heads // world
    return rank * n, (rank + 1) * n


def sparse_shard(q_heads: int, kv_heads: int, world: int, rank: int) -> SparseShard:
    """Split of the sparse layer: whole kv groups per rank when world <= kv
    heads, else world / kv_heads ranks per group, each with a contiguous
    share of the group's q heads."""
    if q_heads % kv_heads:
        raise ValueError("q heads must be a multiple of kv heads")
    G = q_heads // kv_heads
    if world <= kv_heads:
        if kv_heads % world:
            raise ValueError(f"{kv_heads} kv heads do not split over {world} ranks")
        kv_lo, kv_hi = head_range(kv_heads, world, rank)
        return SparseShard(kv_lo * G, kv_hi * G, kv_lo, kv_hi, (rank,))
    if world % kv_heads or G % (world // kv_heads):
        raise ValueError(f"{q_heads}/{kv_heads} heads do not split over {world} ranks")
    rpg = world // kv_heads
    g = rank // rpg
    per = G // rpg
    lo = g * G + (rank % rpg) * per
    return SparseShard(lo, lo + per, g, g + 1, tuple(range(g * rpg, (g + 1) * rpg)))


def group_subgroups(world: int, kv_heads: int):
    """The process groups of the ranks sharing a kv group (world > kv heads),
    created in the same order on every rank; None where no exchange is needed."""
    if world <= kv_heads or world == 1:
        return {}
    rpg = world // kv_heads
    groups = {}
    for g in range(kv_heads):
        ranks = list(range(g * rpg, (g + 1) * rpg))
        groups[tuple(ranks)] = dist.new_group(ranks)
    return groups


class LibsalaBackend:
    """The C ABI on this rank's current CUDA device."""

    def __init__(self):
        from hybrid_sparse_linear_lightning_b200 import sala
        self.sala = sala

    def linear_prefill(self, q, k, v, g, lam, wq, wk, *, chunk, pos0=0, state_in=None,
                       want_state=False):
        return self.sala.linear_prefill(q, k, v, g, lam, wq, wk, chunk=chunk, pos0=pos0,
                                        state_in=state_in, want_state=want_state)

    def select_begin(self, q, k, wq, wk, *, block, topk, n_init, n_local):
        s = self.sala
        B, N, Hq, D = q.shape
        Hkv = k.shape[2]
        d = s.sparse_desc(B, N, Hq, Hkv, D, block, topk, n_init, n_local, q.dtype)
        nb = N // block
        qn = torch.empty((B, N, Hq, D), dtype=torch.bfloat16, device=q.device)
        kn = torch.empty((B, N, Hkv, D), dtype=torch.bfloat16, device=q.device)
        kbar = torch.empty((B, nb, Hkv, D), dtype=torch.float32, device=q.device)
        qsum = torch.empty((B, nb, Hkv, D), dtype=torch.float32, device=q.device)
        st = s.sala_sparse_select_begin(d, q, k, wq, wk, qn, kn, kbar, qsum)
        if st != s.SALA_OK:
            raise s.SalaError(st, "sala_sparse_select_begin")
        return dict(desc=d, q_norm=qn, k_norm=kn, kbar=kbar, qsum=qsum)

    def select_finish(self, sel):
        s = self.sala
        d = sel["desc"]
        nb = d.seqlen // d.block
        idx = torch.empty((d.batch, d.kv_heads, nb, s.sala_sparse_index_width(d)),
                          dtype=torch.int32, device=sel["qsum"].device)
        st = s.sala_sparse_select_finish(d, sel["qsum"], sel["kbar"], idx)
        if st != s.SALA_OK:
            raise s.SalaError(st, "sala_sparse_select_finish")
        return idx

    def sparse_prefill(self, sel, v, g, idx):
        d = sel["desc"]
        return self.sala.sparse_prefill(sel["q_norm"], sel["k_norm"], v, g, idx, block=d.block,
                                        topk=d.topk, n_init=d.n_init, n_local=d.n_local)


class ShardedGroup:
    """One rank's share of a head-sharded layer group.

    rank / world: this process's place; subgroups: ``group_subgroups`` (pass
    the same dict on every rank).  Inputs handed to the methods are this
    rank's slices ([B, N, heads of the shard, d]); outputs are too.
    """

    def __init__(self, rank: int, world: int, heads: int, q_heads: int, kv_heads: int,
                 subgroups: Optional[dict] = None, backend=None):
        self.rank, self.world = rank, world
        self.lin = head_range(heads, world, rank)
        self.sp = sparse_shard(q_heads, kv_heads, world, rank)
        self.subgroups = subgroups or {}
        self.backend = backend or LibsalaBackend()

    def linear(self, q, k, v, g, lam_local, wq, wk, *, chunk=64, pos0=0, state_in=None,
               want_state=False):
        return self.backend.linear_prefill(q, k, v, g, lam_local, wq, wk, chunk=chunk, pos0=pos0,
                                           state_in=state_in, want_state=want_state)

    def sparse(self, q, k, v, g, wq, wk, *, block=64, topk=16, n_init=1, n_local=2):
        sel = self.backend.select_begin(q, k, wq, wk, block=block, topk=topk, n_init=n_init,
                                        n_local=n_local)
        ranks = self.sp.group_ranks
        if len(ranks) > 1:
            # the kv group's block-mean queries summed over all its q heads
            dist.all_reduce(sel["qsum"], op=dist.ReduceOp.SUM, group=self.subgroups[ranks])
        idx = self.backend.select_finish(sel)
        return self.backend.sparse_prefill(sel, v, g, idx), idx


def gather_heads(local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """[B, N, h, d] shards of equal h on every rank -> [B, N, world * h, d]
    (rank order = head order)."""
    if world == 1:
        return local
    parts: List[torch.Tensor] = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    return torch.cat(parts, dim=2)

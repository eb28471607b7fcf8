"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The SALA path is single-GPU; `bench.py --gpus N` runs N independent replicas
under torchrun with no collective on the data path.  These tests cover the
host-side parts: the max-over-ranks timing, the whole-job throughput and
the reference arm's rank-0-only behaviour."""
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        my_ms = 100.0 + 50.0 * rank              # rank 1 is the slow replica
        mx = bench.max_over_ranks(my_ms, world)
        val = bench.replica_throughput(262144, 5, mx, world)
        bench.barrier(world)
        q.put((rank, mx, val))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slowest replica's time; throughput counts both replicas
    assert [r[1] for r in res] == [150.0, 150.0]
    assert res[0][2] == pytest.approx(262144 * 2 * 5 / 0.150)
    assert res[0][2] == res[1][2]


def test_reference_arm_rank_nonzero_exits_silently():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_rank0(capsys):
    """The oracle arm on rank 0: one JSON line whose step time is the
    extrapolated time of a whole step at its own throughput."""
    import json
    import types
    import bench
    os.environ.pop("RANK", None)
    bench.run_reference(types.SimpleNamespace(workload="group_256k", seqlen=0, steps=1, warmup=0))
    line = capsys.readouterr().out.strip().splitlines()[-1]
    d = json.loads(line)
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    tokens = 262144
    assert d["ms_per_step"] == pytest.approx(tokens / d["value"] * 1e3, rel=1e-3)
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"

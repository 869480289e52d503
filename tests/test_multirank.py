"""The multi-GPU path of bench.py is "replicas only": every rank runs its own layer, the
ranks meet at barriers around the timed region, the slowest rank's time is the job's,
and rank 0 alone reports.  These checks run that host logic as two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    import bench
    local = [1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)]        # per-rank timings (ms)
    dist.barrier()
    got = bench.max_over_ranks(local, world, "cpu")
    dist.barrier()
    q.put((rank, got, bench.job_rate(2.0, world, got[0])))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    by_rank = {r: (got, rate) for r, got, rate in results}
    assert set(by_rank) == {0, 1}
    for got, rate in by_rank.values():
        assert got == [2.0, 10.0, 1.0]                          # element-wise max over the ranks
        assert rate == pytest.approx(2.0 * 2 / (2.0e-3))        # both replicas' work / slowest time


def test_reference_arm_other_ranks_exit_without_work():
    import subprocess
    import sys
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""

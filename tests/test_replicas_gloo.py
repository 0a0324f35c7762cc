"""Multi-process host logic of the data-parallel bench path, on CPU with
the gloo backend (world size 2): max-over-ranks timing, whole-job rate and
per-rank input seeds."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from bitlinear_bitnet_linear_b200 import replicas
    replicas.init("gloo", timeout_s=60)
    r, w, _ = replicas.rank_info()
    ms = 1.0 + r                                   # rank 1 is the slower one
    ms_max = replicas.max_over_ranks(ms)
    rate = replicas.whole_job_rate(1000.0, w, ms_max * 1e-3)
    replicas.barrier()
    q.put((r, w, ms_max, rate, replicas.replica_seed(7, r)))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_max_timing_and_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(2))
    for r, w, ms_max, rate, seed in res:
        assert w == 2 and ms_max == 2.0                  # the slowest rank's time
        assert rate == pytest.approx(1000.0 * 2 / 2e-3)  # all units / max time
    assert res[0][4] != res[1][4]                       # independent input streams


def test_single_process_is_identity():
    from bitlinear_bitnet_linear_b200 import replicas
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.whole_job_rate(10.0, 1, 2.0) == 5.0

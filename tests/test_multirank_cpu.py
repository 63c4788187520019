"""The N > 1 logic of bench.py on CPU with two gloo ranks: the step time is the maximum
over ranks and the job throughput counts every rank's tokens."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [12.5, 20.0][rank]
    got = bench.max_over_ranks(local_ms, dist, "cpu")
    tput = bench.job_tokens_per_s(world, 8192, 10, got)
    q.put((rank, got, tput))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tput in res:
        assert got == pytest.approx(20.0)
        assert tput == pytest.approx(2 * 8192 * 10 / 0.020)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.job_tokens_per_s(1, 100, 2, 1000.0) == pytest.approx(200.0)


def test_reference_arm_nonzero_rank_exits_without_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args) == 0

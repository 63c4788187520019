"""The N > 1 logic on CPU with two gloo ranks: the step time of bench.py is the maximum
over ranks, the job throughput counts every rank's tokens, and the data-parallel step
(token shards + one all-reduce of dtheta) reproduces the full-batch gradient."""
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


def _dp_worker(rank, world, port, q):
    import numpy as np
    import torch
    import torch.distributed as dist

    from oracle import poetx_ref as ref
    from orthogonal_reparameterized_cnp_b200 import dp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    n, m, b, k, T = 16, 24, 4, 4, 11
    rng = np.random.default_rng(5)
    x = rng.standard_normal((T, n))
    dy = rng.standard_normal((T, m))
    W0 = rng.standard_normal((m, n)) / np.sqrt(n)
    tP = rng.standard_normal((n // b, b * (b - 1) // 2)) * 0.1
    tR = rng.standard_normal((m // b, b * (b - 1) // 2)) * 0.1
    pP, _ = ref.make_perm(1, n)
    pR, _ = ref.make_perm(2, m)
    t0, cnt = dp.token_shard(T, world, rank)
    out = ref.full_step(x[t0:t0 + cnt], W0, tP, tR, dy[t0:t0 + cnt], pP, pR, b, k)
    dth = torch.from_numpy(np.concatenate([out["dtheta_P"], out["dtheta_R"]]))
    dp.allreduce_dtheta(dth)
    q.put((rank, cnt, dth.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def test_data_parallel_dtheta_equals_full_batch():
    import numpy as np

    from oracle import poetx_ref as ref
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [6, 5]  # T = 11 split 6 + 5
    n, m, b, k, T = 16, 24, 4, 4, 11
    rng = np.random.default_rng(5)
    x = rng.standard_normal((T, n))
    dy = rng.standard_normal((T, m))
    W0 = rng.standard_normal((m, n)) / np.sqrt(n)
    tP = rng.standard_normal((n // b, b * (b - 1) // 2)) * 0.1
    tR = rng.standard_normal((m // b, b * (b - 1) // 2)) * 0.1
    pP, _ = ref.make_perm(1, n)
    pR, _ = ref.make_perm(2, m)
    full = ref.full_step(x, W0, tP, tR, dy, pP, pR, b, k)
    want = np.concatenate([full["dtheta_P"], full["dtheta_R"]])
    for _, _, got in res:
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_token_shards_cover_the_batch():
    from orthogonal_reparameterized_cnp_b200 import dp
    for T, world in [(8192, 8), (11, 2), (5, 8), (0, 3)]:
        spans = [dp.token_shard(T, world, r) for r in range(world)]
        assert sum(c for _, c in spans) == T
        assert all(spans[r][0] + spans[r][1] == spans[r + 1][0] for r in range(world - 1))
        assert max(c for _, c in spans) - min(c for _, c in spans) <= 1
    with pytest.raises(ValueError):
        dp.token_shard(8, 2, 2)

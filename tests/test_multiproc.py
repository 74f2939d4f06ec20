"""The multi-rank path of the benchmark on CPU: two gloo ranks (one process each, as torchrun
launches them) agree on the max of their timings, draw independent batches, and the whole-job
throughput counts every rank's tokens over the slowest rank's time.  The recurrence itself has no
cross-rank exchange (independent sequences), so nothing else crosses ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        t_local = [1.5, 4.25][rank]
        t_max = bench.max_over_ranks(t_local, world)
        cfg = workloads.CONFIGS["tiny"]
        seed = bench.rank_seed(cfg["seed"], rank)
        inp = workloads.config_inputs("tiny", seed=seed)
        # checksum of this rank's batch, gathered to compare across ranks
        csum = torch.tensor([float(inp["q"].double().sum()), float(inp["v"].double().sum())])
        gathered = [torch.zeros(2, dtype=csum.dtype) for _ in range(world)]
        dist.all_gather(gathered, csum)
        dist.barrier()
        q.put((rank, t_max, seed, [g.tolist() for g in gathered]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [4.25, 4.25]          # max over ranks, seen by every rank
    assert res[0][2] != res[1][2]                        # independent seeds
    g = res[0][3]
    assert g == res[1][3] and g[0] != g[1]               # distinct batches, same view on both ranks


def test_aggregate_counts_all_ranks_over_slowest():
    import bench
    assert bench.aggregate_tokens_per_s(1000, 4, 2.0) == pytest.approx(4000 / 2e-3)
    assert bench.max_over_ranks(3.0, 1) == 3.0

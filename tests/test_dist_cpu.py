"""Multi-rank host logic of bench.py on CPU: 2 gloo ranks (no GPU).

Each rank must draw its own batch (weak scaling), the step time is the max
over ranks and the ideal work is summed over ranks.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from attention_flashattention_fwd_04_b200 import workloads as W
        t = bench.max_over_ranks(1.0 + rank, world)
        s = bench.sum_over_ranks(10.0 * (rank + 1), world)
        seed = bench.shard_seed(W.PREFILL_CONFIGS["tiny"].seed, rank)
        cfg = W.PREFILL_CONFIGS["tiny"]
        mine = W.PrefillConfig(cfg.name, cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.d, cfg.causal, seed)
        qsum = float(W.make_prefill_inputs(mine)[0].float().sum())
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, torch.tensor([qsum], dtype=torch.float64))
        q.put((rank, t, s, seed, [float(x) for x in sums]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_rank_timing_and_sharding():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, t, s, seed, sums in res:
        assert t == 2.0          # max over ranks
        assert s == 30.0         # sum over ranks
    assert res[0][3] != res[1][3]             # different seeds ...
    assert res[0][4][0] != res[0][4][1]       # ... give different batches

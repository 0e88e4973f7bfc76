"""The N>1 host logic of bench.py on CPU with world-size-2 gloo ranks: every rank
runs its own token batch, the barrier holds, and the reported time is the max
over ranks (weak scaling: value = all ranks' tokens / that time)."""
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


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    got = bench.max_over_ranks(10.0 * (rank + 1), world)
    # per-rank batches come from different seeds: the x of rank 0 and rank 1 differ
    from expert_ffn_layer_moe_b200.inputs import CONFIGS, make_inputs
    x = make_inputs(CONFIGS["tiny"], seed=rank, weights=False)["x"]
    dist.destroy_process_group()
    q.put((rank, got, float(x.float().sum())))


@pytest.mark.timeout(180)
def test_two_gloo_ranks_time_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]
    assert res[0][2] != res[1][2]

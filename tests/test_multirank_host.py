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


def _ep_rank_main(rank, world, port, q):
    """The --ep bench path's host side on a gloo rank: its inputs (own batch, own expert
    slice), the exchange with the oracle as the local experts, the max over ranks of
    the step time and the JSON line."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    from expert_ffn_layer_moe_b200 import ep
    from expert_ffn_layer_moe_b200.inputs import MoEConfig, make_inputs
    from tests._bf16 import to_u16
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    cfg = MoEConfig("epb", N=16, H=64, I=32, E=4 * world, k=2)
    x, Wg, bias, W = bench.ep_local_inputs(cfg, rank, world, "cpu")
    full = make_inputs(cfg, seed=0)
    L = cfg.E // world
    sliced = all(torch.equal(W[n], full[n][rank * L:(rank + 1) * L]) for n in ("W1", "W3", "W2"))
    xu = to_u16(x)
    l32 = oracle.router_logits(xu, Wg.numpy()).astype(np.float32)
    idx, w = oracle.topk(l32, cfg.k)
    counts, _, r2t, t2r = oracle.dispatch(idx, cfg.E)
    xp = torch.from_numpy(oracle.permute_rows(xu, r2t).view(np.int16))

    def ffn(x_loc, offs):
        return torch.from_numpy(oracle.expert_ffn(x_loc.numpy().view(np.uint16), offs.numpy(), to_u16(W["W1"]),
                                                  to_u16(W["W3"]), to_u16(W["W2"])))

    def scatter(src, dst_row, dst):
        dst[dst_row.long()] = src
        return dst

    stats = []
    y, _ = ep.exchange_ffn(xp, torch.from_numpy(counts), cfg.E, ffn, scatter, stats=stats)
    out = oracle.combine(y.numpy(), t2r, w)
    ref = oracle.layer_given_logits(xu, l32, to_u16(full["W1"]), to_u16(full["W3"]), to_u16(full["W2"]), cfg.k)
    ms = bench.max_over_ranks(1.0 + rank, world)           # the slowest rank's step time
    line = bench.ep_line(cfg, world, 5, 3, ms, "collective", stats[0].rows_sent, stats[0].rows_received, 2.0 * ms)
    dist.destroy_process_group()
    q.put((rank, sliced, bool(np.array_equal(out, ref)), line["value"], line["e2e"]["value"],
           line["config"]["parallelism"]))


@pytest.mark.timeout(180)
def test_two_gloo_ranks_expert_parallel_bench_path():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, sliced, exact, value, e2e, par in res:
        assert sliced and exact
        assert value == 2 * 16 / 2.0e-3                     # both ranks' tokens over the slower rank's 2 ms
        assert e2e == 2 * 16 / 4.0e-3
        assert par.startswith("ep2: experts split 8/2")

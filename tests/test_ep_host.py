"""Expert parallelism on CPU: the exchange plan, and the whole exchange over gloo ranks.

[MoE-latency] "跨 GPU 时,激活要出门": tokens whose experts live on other GPUs send
their rows there and get the outputs back (all-to-all).  The plan is checked by hand
on a small case and by its invariants on random counts; the exchange runs as 2 and 4
gloo ranks (each with its own token batch and E/G experts, the oracle as each rank's
local expert compute and torch indexing as its row scatter) and must give every rank
the bit-exact output of the one-device oracle layer on its batch.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from expert_ffn_layer_moe_b200 import ep


def test_plan_by_hand():
    # G = 2 ranks, E = 4 experts (rank 0: experts 0, 1; rank 1: experts 2, 3)
    counts = [[1, 2, 0, 3],   # rank 0's rows per expert
              [2, 0, 1, 1]]   # rank 1's
    p0 = ep.exchange_plan(counts, 0)
    assert p0.send_splits == [3, 3] and p0.recv_splits == [3, 2]
    assert p0.local_offsets.tolist() == [0, 3, 5]
    # received: (src 0: e0 r0, e1 r0, e1 r1), (src 1: e0 r0, e0 r1); expert-major with
    # the source order inside an expert: e0 <- s0 r0, s1 r0, s1 r1; e1 <- s0 r0, s0 r1
    assert p0.recv_to_local.tolist() == [0, 3, 4, 1, 2]
    assert p0.local_to_recv.tolist() == [0, 3, 4, 1, 2]
    p1 = ep.exchange_plan(counts, 1)
    assert p1.send_splits == [2, 2] and p1.recv_splits == [3, 2]
    assert p1.local_offsets.tolist() == [0, 1, 5]
    # received: (src 0: e3 x3), (src 1: e2, e3) -> e2 <- s1; e3 <- s0 x3, s1
    assert p1.recv_to_local.tolist() == [1, 2, 3, 0, 4]
    with pytest.raises(ValueError):
        ep.exchange_plan(np.ones((2, 3)), 0)          # 3 experts do not split over 2 ranks
    with pytest.raises(ValueError):
        ep.exchange_plan(counts, 2)                   # no rank 2


@pytest.mark.parametrize("G,E", [(1, 8), (2, 8), (4, 16), (8, 256)])
def test_plan_invariants(G, E):
    rng = np.random.default_rng(G * 100 + E)
    counts = rng.integers(0, 6, size=(G, E))
    counts[0, : E // G] = 0                       # a rank whose experts get nothing from rank 0
    plans = [ep.exchange_plan(counts, r) for r in range(G)]
    L = E // G
    for r, p in enumerate(plans):
        # what r sends to d is what d receives from r; sends cover r's rows, in x_perm order
        assert sum(p.send_splits) == counts[r].sum()
        for d in range(G):
            assert p.send_splits[d] == plans[d].recv_splits[r] == counts[r, d * L:(d + 1) * L].sum()
        n = sum(p.recv_splits)
        assert p.local_offsets[-1] == n and np.all(np.diff(p.local_offsets) == counts[:, r * L:(r + 1) * L].sum(0))
        assert sorted(p.recv_to_local.tolist()) == list(range(n))           # a permutation
        assert np.array_equal(p.local_to_recv[p.recv_to_local], np.arange(n))
        # stable: inside each local expert the received rows keep their received order
        expert_of = np.repeat(np.arange(L), np.diff(p.local_offsets))
        recv_expert = expert_of[p.recv_to_local]
        for e in range(L):
            pos = np.flatnonzero(recv_expert == e)
            assert np.all(np.diff(p.recv_to_local[pos]) == 1)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from expert_ffn_layer_moe_b200.inputs import MoEConfig, make_inputs
    from tests._bf16 import to_u16

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    cfg = MoEConfig("ep", N=24, H=64, I=32, E=4 * world, k=3)
    wts = make_inputs(cfg, seed=0)                               # the same weights on every rank
    x = to_u16(make_inputs(cfg, seed=10 + rank, weights=False)["x"])   # each rank its own batch
    W1, W3, W2 = (to_u16(wts[n]) for n in ("W1", "W3", "W2"))
    Wg = wts["W_gate"].numpy()
    l32 = oracle.router_logits(x, Wg).astype(np.float32)
    idx, w = oracle.topk(l32, cfg.k)
    counts, _, r2t, t2r = oracle.dispatch(idx, cfg.E)
    xp = oracle.permute_rows(x, r2t)
    L = cfg.E // world
    mine = slice(rank * L, (rank + 1) * L)

    def ffn(x_loc, offsets):
        y = oracle.expert_ffn(x_loc.numpy().view(np.uint16), offsets.numpy(), W1[mine], W3[mine], W2[mine])
        return torch.from_numpy(y)

    def scatter(src, dst_row, dst):
        dst[dst_row.long()] = src
        return dst

    stats = []
    y, plan = ep.exchange_ffn(torch.from_numpy(xp.view(np.int16)), torch.from_numpy(counts), cfg.E, ffn, scatter,
                              stats=stats)
    out = oracle.combine(y.numpy(), t2r, w)
    ref = oracle.layer_given_logits(x, l32, W1, W3, W2, cfg.k)
    dist.destroy_process_group()
    q.put((rank, bool(np.array_equal(out, ref)), stats[0].rows_sent, stats[0].rows_received, plan.recv_splits))


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_exchange_gives_the_one_device_layer(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=200) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[1] for r in res), res
    assert all(r[2] == 24 * 3 for r in res)                    # every rank sends all its N*k rows
    assert sum(r[3] for r in res) == world * 24 * 3            # and all of them arrive somewhere
    assert any(r[4][r[0]] < r[3] for r in res)                 # rows really crossed ranks


def test_plan_empty_batches_and_slices():
    p = ep.exchange_plan(np.zeros((4, 8), np.int64), 2)           # nobody routes anything
    assert p.send_splits == [0] * 4 and p.recv_splits == [0] * 4
    assert p.local_offsets.tolist() == [0, 0, 0] and p.recv_to_local.size == 0 and p.local_to_recv.size == 0
    import torch
    W = torch.arange(8 * 3).reshape(8, 3)
    assert ep.local_experts(W, 1, 4).tolist() == W[2:4].tolist()
    with pytest.raises(ValueError):
        ep.local_experts(W, 0, 3)                                  # 8 experts over 3 ranks


def test_exchange_skips_rows_without_an_expert():
    """Rows past the counted ones (assignments without a valid expert) are neither sent
    nor written back: a one-rank gloo group, identity experts."""
    import datetime

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=30))
    try:
        x = torch.arange(5 * 4, dtype=torch.int32).reshape(5, 4)
        counts = torch.tensor([1, 0, 3], dtype=torch.int32)      # 4 counted rows of 5

        def ffn(x_loc, offsets):
            assert offsets.tolist() == [0, 1, 1, 4]
            return x_loc.to(torch.float64) * 2

        def scatter(src, dst_row, dst):
            dst[dst_row.long()] = src
            return dst

        y, plan = ep.exchange_ffn(x, counts, 3, ffn, scatter)
        assert plan.send_splits == [4] and plan.recv_splits == [4]
        assert torch.equal(y[:4], x[:4].to(torch.float64) * 2)
    finally:
        dist.destroy_process_group()


def test_peer_offsets_follow_the_all_to_all_order():
    counts = np.array([[1, 2, 0, 3],    # rank 0's rows per expert (rank 0: experts 0,1; rank 1: 2,3)
                       [2, 0, 1, 1]])   # rank 1's
    send0, back0 = ep.peer_offsets(counts, 0)
    send1, back1 = ep.peer_offsets(counts, 1)
    # rank 0 sends rows [0,3) to itself at row 0 and rows [3,6) to rank 1 at row 0
    assert send0 == [(0, 0, 3), (3, 0, 3)]
    # rank 1 sends rows [0,2) to rank 0 after rank 0's own 3 rows, rows [2,4) to itself after rank 0's 3
    assert send1 == [(0, 3, 2), (2, 3, 2)]
    # outputs go back to where the rows came from: rank 0 returns rows [3,5) of what it got to rank 1 row 0
    assert back0 == [(0, 0, 3), (3, 0, 2)]
    assert back1 == [(0, 3, 3), (3, 2, 2)]


class MemmapPeers:
    """Stand-in for CudaPeers on CPU: each rank's buffers are files mapped by every rank
    (the 'handle' is the path), copies write into the mapping, and the fence flushes
    and meets the others at a gloo barrier -- the same protocol without a GPU."""

    def __init__(self, root, tag):
        import torch.distributed as dist
        self.dist = dist
        self.world, self.rank = dist.get_world_size(), dist.get_rank()
        self.root, self.tag, self.n = root, tag, 0
        self.maps = {}

    def alloc(self, rows, words):
        import torch
        path = os.path.join(self.root, f"{self.tag}_r{self.rank}_b{self.n}.bin")
        self.n += 1
        mm = np.memmap(path, dtype=np.int32, mode="w+", shape=(max(1, rows), words))
        self.maps[path] = mm
        return torch.from_numpy(mm)

    def share(self, buf):
        path = next(p for p, m in self.maps.items() if m.ctypes.data == buf.data_ptr())
        paths = [None] * self.world
        self.dist.all_gather_object(paths, (path, buf.shape))
        return paths

    def copy(self, dst, row, src):
        path, shape = dst
        if path not in self.maps:
            self.maps[path] = np.memmap(path, dtype=np.int32, mode="r+", shape=tuple(shape))
        self.maps[path][row:row + src.shape[0]] = src.numpy()

    def fence(self):
        for m in self.maps.values():
            m.flush()
        self.dist.barrier()

    def close(self):
        self.dist.barrier()


def _rank_main_peer(rank, world, port, root, q):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from expert_ffn_layer_moe_b200.inputs import MoEConfig, make_inputs
    from tests._bf16 import to_u16

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    cfg = MoEConfig("ep", N=20, H=64, I=32, E=2 * world, k=2)
    wts = make_inputs(cfg, seed=1)
    W1, W3, W2 = (to_u16(wts[n]) for n in ("W1", "W3", "W2"))
    L = cfg.E // world
    mine = slice(rank * L, (rank + 1) * L)

    def ffn(x_loc, offsets):
        return torch.from_numpy(oracle.expert_ffn(x_loc.numpy().view(np.uint16), offsets.numpy(), W1[mine],
                                                  W3[mine], W2[mine]))

    def scatter(src, dst_row, dst):
        dst[dst_row.long()] = src
        return dst

    # rows travel as 32-bit words: bf16 x rows are H/2 words, the oracle's fp64 outputs 2H
    tr = ep.PeerCopyTransport(MemmapPeers(root, "t"), max_rows=cfg.N * cfg.k, words_in=cfg.H // 2,
                              words_out=2 * cfg.H)
    ok = True
    for step in range(3):  # the buffers are reused from step to step
        x = to_u16(make_inputs(cfg, seed=20 + 7 * rank + step, weights=False)["x"])
        l32 = oracle.router_logits(x, wts["W_gate"].numpy()).astype(np.float32)
        idx, w = oracle.topk(l32, cfg.k)
        counts, _, r2t, t2r = oracle.dispatch(idx, cfg.E)
        xp = torch.from_numpy(oracle.permute_rows(x, r2t).view(np.int16))   # bf16 rows as their bits
        y_p, _ = ep.exchange_ffn(xp, torch.from_numpy(counts), cfg.E, ffn, scatter, transport=tr)
        y_c, _ = ep.exchange_ffn(xp, torch.from_numpy(counts), cfg.E, ffn, scatter)
        out = oracle.combine(y_p.numpy(), t2r, w)
        ref = oracle.layer_given_logits(x, l32, W1, W3, W2, cfg.k)
        ok = ok and bool(np.array_equal(out, ref)) and torch.equal(y_p, y_c)
    tr.close()
    dist.destroy_process_group()
    q.put((rank, ok))


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 3])
def test_peer_copy_exchange_equals_the_all_to_all(world, tmp_path):
    """The peer-copy transport, its buffers reused over three steps on gloo ranks with
    file-mapped stand-ins for the GPUs' shared buffers: bit-identical expert outputs to
    the all-to-all, and every rank's layer equals the one-device oracle layer."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_peer, args=(r, world, port, str(tmp_path), q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=200) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[1] for r in res), res


def test_peer_copy_moves_bits_of_fp32_rows(tmp_path):
    """fp32 rows (the GPU path's expert outputs) and bf16 rows travel as raw words: the
    return copy must not convert values.  One gloo rank, file-mapped buffers."""
    import datetime

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=30))
    try:
        x = torch.randn(6, 8).to(torch.bfloat16)
        counts = torch.tensor([2, 4], dtype=torch.int32)

        def ffn(x_loc, offsets):
            return x_loc.float() * 3.0 + 0.25          # fp32 outputs with fractional bits

        def scatter(src, dst_row, dst):
            dst[dst_row.long()] = src
            return dst

        tr = ep.PeerCopyTransport(MemmapPeers(str(tmp_path), "f"), max_rows=6, words_in=4, words_out=8)
        y, _ = ep.exchange_ffn(x, counts, 2, ffn, scatter, transport=tr)
        tr.close()
        assert y.dtype == torch.float32 and torch.equal(y, x.float() * 3.0 + 0.25)
    finally:
        dist.destroy_process_group()

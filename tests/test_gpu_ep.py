"""Expert parallelism on one GPU: the row scatter kernel, and the EP layer on a
one-rank NCCL group (route, permute, the exchange to itself, the local experts, the
combine) against the oracle given the GPU's logits.

[MoE-latency] "跨 GPU 时,激活要出门".  Runs with more ranks need more GPUs than a
test here has; the multi-rank exchange is covered on CPU by tests/test_ep_host.py.
"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from expert_ffn_layer_moe_b200 import ep, moe
from expert_ffn_layer_moe_b200.inputs import MoEConfig
from tests._bf16 import dec
from tests.test_gpu_parity import assert_close, cuda_inputs, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,cols", [(torch.bfloat16, 64), (torch.bfloat16, 200 * 8), (torch.float32, 64)])
def test_scatter_rows_bit_exact(dtype, cols):
    g = torch.Generator().manual_seed(cols)
    rows = 333
    src = torch.randn((rows, cols), generator=g).to(dtype)
    perm = torch.randperm(rows + 20, generator=g)[:rows].to(torch.int32)
    perm[::7] = -1                                               # skipped rows
    perm[1::11] = rows + 20 + 5                                  # targets past dst: skipped too
    dst = torch.full((rows + 20, cols), 7.0).to(dtype)
    got = moe.moe_scatter_rows(src.cuda(), perm.cuda(), dst.cuda())
    torch.cuda.synchronize()
    want = dst.clone()
    keep = (perm >= 0) & (perm < rows + 20)
    want[perm[keep].long()] = src[keep]
    assert torch.equal(got.cpu().view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                       want.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("cfg", [
    MoEConfig("ep1", N=300, H=256, I=192, E=8, k=2),
    MoEConfig("ep1_decode", N=7, H=512, I=256, E=16, k=4),       # empty experts, a few rows each
])
def test_ep_layer_one_rank_matches_oracle(cfg):
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = cuda_inputs(cfg, seed=5)
        stats = []
        out = ep.moe_layer_forward_ep(t["x"], t["W_gate"], ep.local_experts(t["W1"], 0, 1),
                                      ep.local_experts(t["W3"], 0, 1), ep.local_experts(t["W2"], 0, 1), cfg.k,
                                      bias=t["bias"], stats=stats)
        # the same router call as inside the layer, now keeping its logits (same path, same bits)
        logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
        moe.moe_route(t["x"], t["W_gate"], cfg.k, bias=t["bias"], logits=logits)
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == 0
        assert stats[0].rows_sent == stats[0].rows_received == cfg.N * cfg.k
        ref = oracle.layer_given_logits(host(t["x"]), host(logits), host(t["W1"]), host(t["W3"]), host(t["W2"]),
                                        cfg.k)
        assert_close(dec(host(out)), dec(ref), f"{cfg.name} ep out")
    finally:
        dist.destroy_process_group()


def test_ep_layer_skips_an_out_of_range_expert_index():
    """A caller-supplied choice with an index outside [0, E): that assignment has no
    row, its slot of the returned y is never written, and the combine must skip it.
    The output must equal the oracle over the valid picks (the bad pick given weight 0
    on a valid expert, which adds exactly nothing) and the error word must say
    MOE_DEVERR_BAD_EXPERT_INDEX."""
    cfg = MoEConfig("ep1_bad", N=96, H=256, I=128, E=8, k=2)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = cuda_inputs(cfg, seed=9)
        idx, w, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k)
        bad_tokens = [3, 40, 95]
        idx_bad = idx.clone()
        for tok in bad_tokens:
            idx_bad[tok, 1] = cfg.E + 5 if tok != 40 else -2
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == 0
        out = ep.moe_layer_forward_ep(t["x"], t["W_gate"], ep.local_experts(t["W1"], 0, 1),
                                      ep.local_experts(t["W3"], 0, 1), ep.local_experts(t["W2"], 0, 1), cfg.k,
                                      routing=(idx_bad, w))
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == moe.MOE_DEVERR_BAD_EXPERT_INDEX

        # oracle: the bad pick moved to a valid expert with weight 0
        idx_ref = host(idx_bad).copy()
        w_ref = host(w).astype(np.float64)
        for tok in bad_tokens:
            idx_ref[tok, 1] = 0 if idx_ref[tok, 0] != 0 else 1
            w_ref[tok, 1] = 0.0
        counts, offsets, r2t, t2r = oracle.dispatch(idx_ref, cfg.E)
        x_perm = oracle.permute_rows(host(t["x"]), r2t)
        y = oracle.expert_ffn(x_perm, offsets, host(t["W1"]), host(t["W3"]), host(t["W2"]))
        ref = oracle.combine(y, t2r, w_ref)
        assert_close(dec(host(out)), dec(ref), "ep out with skipped picks")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("transport", ["collective", "peer_copy"])
def test_ep_layer_one_rank_both_transports(transport):
    """A one-rank NCCL group with either transport (the peer copies then go into the
    rank's own buffers): same bits as each other and the oracle's layer."""
    cfg = MoEConfig("ep1_tr", N=200, H=256, I=192, E=8, k=2)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = cuda_inputs(cfg, seed=13)
        tr = None
        if transport == "peer_copy":
            tr = ep.PeerCopyTransport(ep.CudaPeers(), max_rows=cfg.N * cfg.k, words_in=cfg.H // 2, words_out=cfg.H)
        outs = []
        for _ in range(2):  # the second step reuses the transport's buffers
            outs.append(ep.moe_layer_forward_ep(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k,
                                                transport=tr))
        if tr is not None:
            tr.close()
        logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
        moe.moe_route(t["x"], t["W_gate"], cfg.k, logits=logits)
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == 0
        assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
        ref = oracle.layer_given_logits(host(t["x"]), host(logits), host(t["W1"]), host(t["W3"]), host(t["W2"]),
                                        cfg.k)
        assert_close(dec(host(outs[0])), dec(ref), f"ep {transport}")
    finally:
        dist.destroy_process_group()


def _two_process_rank(rank, port, q):
    """One of two processes on the same GPU: gloo for the host-side plan and barriers,
    the rows moved by the library's copies into the other process's IPC-mapped buffers.
    The processes never wait on each other on the device."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from expert_ffn_layer_moe_b200 import ep, moe
    from expert_ffn_layer_moe_b200.inputs import MoEConfig, make_inputs
    from tests._bf16 import to_u16
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=2,
                                timeout=datetime.timedelta(seconds=60))
        cfg = MoEConfig("ep2", N=96, H=256, I=128, E=8, k=2)
        w = make_inputs(cfg, seed=3)
        x = make_inputs(cfg, seed=40 + rank, weights=False)["x"].cuda()
        Wg = w["W_gate"].cuda()
        W1, W3, W2 = (ep.local_experts(w[n], rank, 2).contiguous().cuda() for n in ("W1", "W3", "W2"))
        idx, wt, _ = moe.moe_route(x, Wg, cfg.k)
        p = moe.moe_permute(x, idx, cfg.E)

        def ffn(x_loc, offs):
            return moe.moe_expert_ffn(x_loc, offs, W1, W3, W2)

        tr = ep.PeerCopyTransport(ep.CudaPeers(), max_rows=cfg.N * cfg.k, words_in=cfg.H // 2, words_out=cfg.H)
        outs = []
        for _ in range(2):
            y, _ = ep.exchange_ffn(p["x_perm"], p["counts"].cpu(), cfg.E, ffn, moe.moe_scatter_rows, transport=tr)
            outs.append(moe.moe_combine(y, p["token_to_row"], wt))
        tr.close()
        torch.cuda.synchronize()
        err = moe.moe_get_device_error()
        logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
        moe.moe_route(x, Wg, cfg.k, logits=logits)
        ref = oracle.layer_given_logits(to_u16(x.cpu()), logits.cpu().numpy(), to_u16(w["W1"]), to_u16(w["W3"]),
                                        to_u16(w["W2"]), cfg.k)
        same = bool(torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)))
        g = to_u16(outs[0].cpu())
        from tests._bf16 import dec
        a, b = dec(g), dec(ref)
        close = bool(np.all(np.abs(a - b) <= 2e-2 * np.abs(b) + 2e-3))
        dist.destroy_process_group()
        q.put((rank, err, same, close, None))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, -1, False, False, repr(e)))


def test_ep_two_processes_on_one_gpu_peer_copies():
    """Two ranks as two processes sharing one GPU: the peer-copy transport's buffers
    are exported and imported through CUDA IPC (a process cannot import its own
    handle, so this is the only way one GPU exercises the import), rows move by
    moe_copy_async, and the ranks meet only at host barriers.  Each rank's layer must
    match the oracle and repeat bit for bit."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_two_process_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert all(r[4] is None for r in res), res
    assert all(r[1] == 0 and r[2] and r[3] for r in res), res

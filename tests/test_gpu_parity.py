"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bars: routing indices, counts, offsets, row maps and permuted rows bit-exact
(the oracle picks experts from the GPU's fp32 logits, so both sides take that
integer decision in the same precision); logits within a float64-derived bound;
routing weights within a few fp32 ulp; h, y and out within
|d| <= 2e-2*|ref| + 2e-3 with bf16 rounding at the same points.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from expert_ffn_layer_moe_b200 import moe
from expert_ffn_layer_moe_b200.inputs import CONFIGS, MoEConfig, make_inputs
from tests._bf16 import dec, to_u16

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2e-2, 2e-3


def assert_close(g, w, what):
    """|got - want| <= 2e-2*|want| + 2e-3, elementwise (float arrays)."""
    g = np.asarray(g, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    bad = np.abs(g - w) > RTOL * np.abs(w) + ATOL
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at "
                           f"{np.argwhere(bad)[0].tolist()}: got {g[bad][0]} want {w[bad][0]}")


def cuda_inputs(cfg, seed=0, gen_device="cpu"):
    t = make_inputs(cfg, seed=seed, device=gen_device)
    return {n: (v.cuda() if v is not None else None) for n, v in t.items()}


def host(t):
    if t is None:
        return None
    t = t.detach().cpu()
    return to_u16(t) if t.dtype == torch.bfloat16 else t.numpy()


def run_layer(cfg, t, **kw):
    logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
    out = moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, bias=t["bias"],
                                   Ws1=t.get("Ws1"), Ws3=t.get("Ws3"), Ws2=t.get("Ws2"), logits=logits, **kw)
    assert moe.moe_get_device_error() == 0
    return out, logits


def check_layer_against_oracle(cfg, t, out, logits, tokens=None):
    """Compare out (and routing) for `tokens` (default: all) with the oracle fed
    the same inputs and the GPU's fp32 logits."""
    sel = slice(None) if tokens is None else tokens
    x = host(t["x"])[sel]
    l32 = host(logits)[sel]
    ref = oracle.layer_given_logits(x, l32, host(t["W1"]), host(t["W3"]), host(t["W2"]), cfg.k,
                                    Ws1=host(t.get("Ws1")), Ws3=host(t.get("Ws3")), Ws2=host(t.get("Ws2")))
    assert_close(dec(host(out)[sel]), dec(ref), f"{cfg.name} out")


def check_logits(cfg, t, logits):
    l64 = oracle.router_logits(host(t["x"]), host(t["W_gate"]), host(t["bias"]))
    xd = dec(host(t["x"]))
    scale = np.abs(xd) @ np.abs(host(t["W_gate"]).astype(np.float64))
    bound = 2.0 ** -20 * scale + 1e-6
    assert np.all(np.abs(host(logits) - l64) <= bound)


# --------------------------------------------------------------- the steps ---

def test_route_matches_oracle():
    cfg = CONFIGS["tiny"]
    t = cuda_inputs(cfg)
    logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
    idx, w, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k, logits=logits)
    torch.cuda.synchronize()
    check_logits(cfg, t, logits)
    ref_idx, ref_w = oracle.topk(host(logits), cfg.k)
    assert np.array_equal(host(idx), ref_idx)
    assert np.allclose(host(w), ref_w, rtol=4 * 2.0 ** -23, atol=1e-7)


# (N, H, E, k, workspace, logits buffer).  Paths: no workspace and no logits buffer ->
# the fused one-kernel path; a logits buffer alone -> the split path with one slice of
# H; a workspace -> the split path with up to H/512 slices of H (small N) or the
# tensor-core path (N >= 256 and N*E >= 32768).  Where the split would use one slice
# and E <= 16 the fused kernel runs instead (e.g. H=512, E=8).
ROUTE_CASES = [
    # fused
    (203, 512, 8, 2, False, False), (203, 512, 160, 6, False, False), (1, 2048, 128, 8, False, False),
    (37, 768, 37, 3, False, False),
    # split, one slice of H (logits buffer, no workspace)
    (203, 512, 160, 6, False, True), (1, 2048, 128, 8, False, True), (203, 512, 8, 2, False, True),
    # split with slices of H
    (203, 512, 8, 2, True, True), (203, 512, 128, 8, True, True), (203, 512, 37, 3, True, True),
    (203, 512, 1, 1, True, True), (203, 512, 256, 8, True, True), (1, 2048, 128, 8, True, True),
    (16, 2048, 128, 8, True, True), (156, 6144, 8, 2, True, True), (5, 4096, 160, 6, True, True),
    (3, 1536, 256, 8, True, False), (128, 2048, 128, 8, True, False),
    # tensor cores
    (1000, 512, 128, 8, True, True), (512, 512, 160, 6, True, True), (4096, 512, 8, 2, True, True),
    (300, 512, 256, 8, True, True), (777, 512, 37, 3, True, True), (1024, 2048, 128, 8, True, False),
    # tensor cores, tokens on the M side, one thread per token ranking expert-major logits
    (16411, 256, 128, 8, True, True), (16411, 256, 37, 3, True, False), (16384, 512, 256, 8, True, True),
]


def check_picks_without_logits(cfg, t, idx, w):
    """Routing returned without its logits: the picks must equal the top-k of the
    float64 logits wherever that top-k is decided by more than the fp32 error bound
    (the (k+1)-th logit and each consecutive pick apart by more than it); the weights
    match the float64 softmax of the picks."""
    l64 = oracle.router_logits(host(t["x"]), host(t["W_gate"]), host(t["bias"]))
    scale = np.abs(dec(host(t["x"]))) @ np.abs(host(t["W_gate"]).astype(np.float64))
    bound = 2.0 ** -20 * scale.max(axis=1) + 1e-6
    order = np.lexsort((np.broadcast_to(np.arange(cfg.E), l64.shape), -l64), axis=1)
    k = cfg.k
    top = np.take_along_axis(l64, order[:, : min(k + 1, cfg.E)], axis=1)
    gaps = -np.diff(top, axis=1)
    clear = (gaps > 2 * bound[:, None]).all(axis=1)
    got = host(idx)
    assert clear.mean() > 0.5, "inputs too tied to check"
    assert np.array_equal(got[clear], order[clear, :k])
    picked = np.take_along_axis(l64, got.astype(np.int64), axis=1)
    ref_w = np.exp(picked - picked[:, :1])
    ref_w /= ref_w.sum(axis=1, keepdims=True)
    assert np.allclose(host(w), ref_w, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("N,H,E,k,use_ws,with_logits", ROUTE_CASES)
def test_route_shapes_and_bias(N, H, E, k, use_ws, with_logits):
    cfg = MoEConfig("route", N=N, H=H, I=64, E=E, k=k)
    t = cuda_inputs(cfg, seed=4)
    bias = torch.linspace(-0.5, 0.5, E, device="cuda")
    logits = torch.empty((cfg.N, E), dtype=torch.float32, device="cuda") if with_logits else None
    idx, w, _ = moe.moe_route(t["x"], t["W_gate"], k, bias=bias, logits=logits, use_workspace=use_ws)
    torch.cuda.synchronize()
    t["bias"] = bias
    if with_logits:
        check_logits(cfg, t, logits)
        ref_idx, ref_w = oracle.topk(host(logits), k)
        assert np.array_equal(host(idx), ref_idx)
        assert np.allclose(host(w), ref_w, rtol=4 * 2.0 ** -23, atol=1e-7)
    else:
        check_picks_without_logits(cfg, t, idx, w)


def test_kernel_launch_counter_counts_a_layer():
    """The host-side launch count moves by the kernels one layer call runs.  At the
    tiny shape (128 assignments): the one-kernel router, the kernel that dispatches and
    copies the rows of a small batch, the two grouped GEMMs and the combine.  Through
    the separate steps the same work is six launches: router, single-block dispatch,
    row scatter, two GEMMs, combine."""
    cfg = CONFIGS["tiny"]
    t = cuda_inputs(cfg)
    n0 = moe.moe_kernel_launches()
    run_layer(cfg, t)
    assert moe.moe_kernel_launches() - n0 == 5
    n0 = moe.moe_kernel_launches()
    idx, w, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k, use_workspace=False)
    p = moe.moe_permute(t["x"], idx, cfg.E)
    y = moe.moe_expert_ffn(p["x_perm"], p["offsets"], t["W1"], t["W3"], t["W2"])
    moe.moe_combine(y, p["token_to_row"], w)
    assert moe.moe_kernel_launches() - n0 == 6


def test_route_paths_agree_on_logits():
    """The tensor-core logits (three-term bf16 split of W_gate) and the CUDA-core fp32
    logits agree to fp32 accuracy; most expert choices coincide."""
    cfg = MoEConfig("paths", N=2048, H=1024, I=64, E=128, k=8)
    t = cuda_inputs(cfg, seed=6)
    la = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
    lb = torch.empty_like(la)
    ia, _, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k, logits=la, use_workspace=True)
    ib, _, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k, logits=lb, use_workspace=False)
    torch.cuda.synchronize()
    scale = torch.from_numpy(np.abs(dec(host(t["x"]))) @ np.abs(host(t["W_gate"]).astype(np.float64)))
    d = (la - lb).abs().double().cpu()
    assert bool((d <= 2.0 ** -19 * scale + 1e-6).all())
    assert (ia == ib).float().mean().item() > 0.99


def test_route_ties_lower_index_first():
    # all-zero hidden states: every logit equals the bias, with exact ties
    N, H, E, k = 5, 256, 16, 4
    x = torch.zeros((N, H), dtype=torch.bfloat16, device="cuda")
    Wg = torch.randn((H, E), device="cuda")
    bias = torch.tensor([0, 1, 1, 0, 2, 2, 2, 0, -1, 1, 0, 0, 2, 0, 0, 1], dtype=torch.float32, device="cuda")
    idx, w, _ = moe.moe_route(x, Wg, k, bias=bias)
    torch.cuda.synchronize()
    assert host(idx).tolist() == [[4, 5, 6, 12]] * N
    assert np.allclose(host(w), 0.25, rtol=0, atol=1e-7)


@pytest.mark.parametrize("N", [5, 1500, 17000])
def test_route_ties_on_every_path(N):
    """Exact ties at every size, so that each top-k form meets them: the fused and split
    paths (small N), the tensor-core path with token-major partial logits (N < 16384) and
    with expert-major ones ranked one thread per token (N >= 16384).  x is zero, so
    every logit is the bias: ties between the picks, a tie straddling the k-th place, and
    -0 against +0."""
    H, E, k = 256, 32, 8
    x = torch.zeros((N, H), dtype=torch.bfloat16, device="cuda")
    Wg = torch.randn((H, E), device="cuda")
    b = [0.0] * E
    for e, v in {3: 2.0, 9: 2.0, 17: 2.0, 30: 1.5, 1: 1.0, 12: 1.0, 20: 1.0, 25: 1.0, 26: 1.0}.items():
        b[e] = v
    b[5], b[6] = -0.0, 0.0                      # -0 == +0: the lower index first
    bias = torch.tensor(b, dtype=torch.float32, device="cuda")
    logits = torch.empty((N, E), dtype=torch.float32, device="cuda")
    idx, w, _ = moe.moe_route(x, Wg, k, bias=bias, logits=logits)
    torch.cuda.synchronize()
    want = [3, 9, 17, 30, 1, 12, 20, 25]          # 1.0 ties: 1, 12, 20, 25 make it, 26 does not
    assert host(idx).tolist() == [want] * N
    ref_idx, ref_w = oracle.topk(host(logits), k)
    assert np.array_equal(host(idx), ref_idx)
    assert np.allclose(host(w), ref_w, rtol=4 * 2.0 ** -23, atol=1e-7)


@pytest.mark.parametrize("N,E,k", [(64, 8, 2), (1000, 160, 6), (3000, 128, 8), (7, 4, 4), (1, 1, 1),
                                   (128, 64, 8), (129, 64, 8), (256, 128, 8),  # one block up to 1024 rows
                                   (4095, 256, 8), (4096, 256, 8)])  # 128 blocks of 256, then 32 of 1024
def test_permute_bit_exact(N, E, k):
    H = 128
    g = torch.Generator().manual_seed(N + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(N)]).to(torch.int32)
    idx[: N // 3, 0] = 0                           # a hot expert
    x = (torch.randn((N, H), generator=g) * 3).to(torch.bfloat16)
    res = moe.moe_permute(x.cuda(), idx.cuda(), E)
    torch.cuda.synchronize()
    counts, offsets, r2t, t2r = oracle.dispatch(idx.numpy(), E)
    assert np.array_equal(host(res["counts"]), counts)
    assert np.array_equal(host(res["offsets"]), offsets)
    assert np.array_equal(host(res["row_to_token"]), r2t)
    assert np.array_equal(host(res["token_to_row"]), t2r)
    assert np.array_equal(host(res["x_perm"]), oracle.permute_rows(to_u16(x), r2t))
    assert moe.moe_get_device_error() == 0


def test_permute_bad_index_reports_without_trap():
    N, H, E, k = 40, 64, 4, 2
    idx = torch.randint(0, E, (N, k), dtype=torch.int32)
    idx[:, 1] = (idx[:, 0] + 1) % E
    idx[7, 1] = 9                                  # outside [0, E)
    idx[12, 0] = -3
    x = torch.randn((N, H)).to(torch.bfloat16).cuda()
    res = moe.moe_permute(x, idx.cuda(), E)
    assert moe.moe_get_device_error() == 1         # MOE_DEVERR_BAD_EXPERT_INDEX
    assert moe.moe_get_device_error() == 0         # read clears it
    t2r = host(res["token_to_row"])
    assert t2r[7, 1] == -1 and t2r[12, 0] == -1
    assert host(res["offsets"])[-1] == N * k - 2


def test_expert_ffn_matches_oracle_tiny():
    cfg = CONFIGS["tiny"]
    t = cuda_inputs(cfg)
    idx, w, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k)
    p = moe.moe_permute(t["x"], idx, cfg.E)
    y = moe.moe_expert_ffn(p["x_perm"], p["offsets"], t["W1"], t["W3"], t["W2"])
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 0
    ref = oracle.expert_ffn(host(p["x_perm"]), host(p["offsets"]), host(t["W1"]), host(t["W3"]), host(t["W2"]))
    assert_close(host(y), ref, "y_perm")


def test_expert_ffn_bad_offsets_report_and_skip_their_groups():
    """Offsets that are not monotone, or that reach past R, mark their groups bad:
    the kernels set MOE_DEVERR_BAD_OFFSETS, run no tile of those groups (rows that
    belong to no valid group keep their prior contents), finish without a hang, and
    the valid groups' rows still match the oracle."""
    E, R, H, I = 4, 128, 256, 192
    g = torch.Generator().manual_seed(11)
    x_perm = (torch.randn((R, H), generator=g)).to(torch.bfloat16)
    W1 = (torch.randn((E, I, H), generator=g) / H ** 0.5).to(torch.bfloat16)
    W3 = (torch.randn((E, I, H), generator=g) / H ** 0.5).to(torch.bfloat16)
    W2 = (torch.randn((E, H, I), generator=g) / I ** 0.5).to(torch.bfloat16)
    # group 0 rows [0, 40); group 1 [40, 200) reaches past R; group 2 [200, 90) runs
    # backwards; group 3 rows [90, 128).  Rows 40..89 belong to no valid group.
    offsets = torch.tensor([0, 40, 200, 90, 128], dtype=torch.int32)
    sentinel = 12345.0
    y = torch.full((R, H), sentinel, dtype=torch.float32, device="cuda")
    assert moe.moe_get_device_error() == 0
    moe.moe_expert_ffn(x_perm.cuda(), offsets.cuda(), W1.cuda(), W3.cuda(), W2.cuda(), y_perm=y)
    assert moe.moe_get_device_error() == moe.MOE_DEVERR_BAD_OFFSETS
    assert moe.moe_get_device_error() == 0         # read clears it
    got = host(y)
    assert np.all(got[40:90] == sentinel)          # no tile of a bad group ran
    xp = to_u16(x_perm)
    ref0 = oracle.expert_ffn(xp[0:40], np.array([0, 40, 40, 40, 40], np.int32), to_u16(W1), to_u16(W3),
                             to_u16(W2))
    ref3 = oracle.expert_ffn(xp[90:128], np.array([0, 0, 0, 0, 38], np.int32), to_u16(W1), to_u16(W3),
                             to_u16(W2))
    assert_close(got[0:40], ref0, "group 0 rows")
    assert_close(got[90:128], ref3, "group 3 rows")


def test_combine_matches_oracle():
    N, H, k, R = 50, 192, 3, 150
    g = torch.Generator().manual_seed(2)
    y = torch.randn((R, H), generator=g)
    t2r = torch.randperm(R, generator=g).to(torch.int32).reshape(N, k)
    w = torch.softmax(torch.randn((N, k), generator=g), 1).to(torch.float32)
    s = torch.randn((N, H), generator=g)
    for shared in (None, s):
        out = moe.moe_combine(y.cuda(), t2r.cuda(), w.cuda(), None if shared is None else shared.cuda())
        ref = oracle.combine(y.numpy(), t2r.numpy(), w.numpy().astype(np.float64),
                             None if shared is None else s.numpy())
        assert_close(dec(host(out)), dec(ref), "combine")


# -------------------------------------------------------------- full layer ---

def test_layer_tiny_matches_oracle():
    cfg = CONFIGS["tiny"]
    t = cuda_inputs(cfg)
    out, logits = run_layer(cfg, t)
    check_logits(cfg, t, logits)
    check_layer_against_oracle(cfg, t, out, logits)


LAYER_SHAPES = [
    # several token tiles per expert with a ragged tail, K loop of 5, feature tiles 2.5 and 1.5
    MoEConfig("ragged", N=300, H=320, I=192, E=5, k=2),
    # mean 12 rows per expert -> 32-row token tiles
    MoEConfig("narrow", N=48, H=256, I=256, E=16, k=4),
    # mean ~100 rows -> 128-row tiles
    MoEConfig("wide", N=400, H=256, I=384, E=8, k=2),
    # mean ~400 rows -> 256-row tiles for W2
    MoEConfig("wider", N=800, H=192, I=128, E=4, k=2),
    # one expert, top-1: a dense SwiGLU FFN
    MoEConfig("dense", N=77, H=128, I=256, E=1, k=1),
    # shared experts on top of routed ones
    MoEConfig("shared", N=90, H=256, I=128, E=6, k=2, Is=192),
    # few tiles and a long K: the W2 GEMM splits K and the combine adds the slices
    MoEConfig("splitk", N=64, H=256, I=2048, E=4, k=2),
    # the largest expert count and top-k the library takes
    MoEConfig("maxEk", N=512, H=256, I=128, E=256, k=8),
    # k == E: every token visits every expert
    MoEConfig("allexperts", N=96, H=192, I=192, E=4, k=4),
    # the smallest widths (one 64-column K block, one feature half-tile)
    MoEConfig("narrowest", N=40, H=64, I=64, E=3, k=2),
    # 192-row token tiles on CTA pairs (the widest tile below 256)
    MoEConfig("tile192", N=1200, H=128, I=128, E=8, k=1),
]


@pytest.mark.parametrize("cfg", LAYER_SHAPES, ids=lambda c: c.name)
def test_layer_gathered_rows_equal_the_permuted_copy(cfg):
    """The W1/W3 GEMM either reads the permuted copy x_perm or gathers each row from x
    through row_to_token (tile::gather4); the two must give the same bits."""
    t = cuda_inputs(cfg, seed=21)
    prev = moe.moe_set_gather_mode(moe.MOE_GATHER_OFF)
    try:
        copy, lc = run_layer(cfg, t)
        moe.moe_set_gather_mode(moe.MOE_GATHER_ON)
        gathered, lg = run_layer(cfg, t)
    finally:
        moe.moe_set_gather_mode(prev)
    torch.cuda.synchronize()
    assert torch.equal(lc, lg)
    assert torch.equal(copy.view(torch.int16), gathered.view(torch.int16))


@pytest.mark.parametrize("cfg", LAYER_SHAPES, ids=lambda c: c.name)
def test_layer_shapes_match_oracle(cfg):
    t = cuda_inputs(cfg, seed=1)
    out, logits = run_layer(cfg, t)
    check_layer_against_oracle(cfg, t, out, logits)


def test_layer_skewed_routing_with_empty_experts():
    cfg = MoEConfig("skew", N=256, H=256, I=256, E=12, k=2)
    t = cuda_inputs(cfg, seed=5)
    # experts 0 and 1 take every token; the others stay empty
    t["bias"] = torch.tensor([50.0, 40.0] + [-50.0] * 10, device="cuda")
    out, logits = run_layer(cfg, t)
    check_layer_against_oracle(cfg, t, out, logits)


def test_layer_empty_batch_is_a_no_op():
    cfg = CONFIGS["tiny"]
    t = cuda_inputs(cfg)
    out = torch.full((0, cfg.H), 7, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward_ex(t["x"][:0], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, out=out)
    assert moe.moe_get_device_error() == 0


@pytest.mark.parametrize("cfg", [CONFIGS["tiny"], MoEConfig("graph", N=300, H=256, I=384, E=16, k=4)])
def test_layer_replays_from_a_cuda_graph(cfg):
    """The explicit call only enqueues kernels on its stream (no allocation, no host
    synchronisation), so one step captured as a CUDA graph replays to the same bits."""
    t = cuda_inputs(cfg, seed=2)
    ws = torch.empty(moe.moe_workspace_bytes(cfg.N, cfg.H, cfg.I, cfg.E, cfg.k, 0), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((cfg.N, cfg.H), dtype=torch.bfloat16, device="cuda")

    def step():
        moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, ws=ws, out=out,
                                 stream=torch.cuda.current_stream())

    step()
    torch.cuda.synchronize()
    eager = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 0
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    del g


def test_layer_is_deterministic():
    cfg = MoEConfig("det", N=500, H=256, I=256, E=8, k=2)
    t = cuda_inputs(cfg, seed=9)
    a, _ = run_layer(cfg, t)
    b, _ = run_layer(cfg, t)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_short_form_with_host_buffers_matches_explicit_form():
    cfg = CONFIGS["tiny"]
    t = cuda_inputs(cfg)
    ref = moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k)
    x_host = t["x"].cpu().pin_memory()
    out_host = moe.moe_layer_forward(x_host, t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k)
    assert out_host.device.type == "cpu"
    assert torch.equal(out_host.view(torch.int16), ref.cpu().view(torch.int16))
    out_dev = moe.moe_layer_forward(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k)
    assert torch.equal(out_dev.view(torch.int16), ref.view(torch.int16))


def test_mixtral_decode_full_size_every_token():
    """The Mixtral-8x22B-shaped decode layer at full size through the benchmark's launch
    path: routing maps bit-exact, and every one of the 156 tokens' outputs against the
    oracle (its threaded build: the same arithmetic per row, spread over the host's
    cores)."""
    cfg = CONFIGS["mixtral_8x22b_decode"]
    t = cuda_inputs(cfg, gen_device="cuda")
    out, logits = run_layer(cfg, t)
    idx, w, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k)
    p = moe.moe_permute(t["x"], idx, cfg.E)
    ref_idx, _ = oracle.topk(host(logits), cfg.k)
    assert np.array_equal(host(idx), ref_idx)
    counts, offsets, r2t, t2r = oracle.dispatch(ref_idx, cfg.E)
    assert np.array_equal(host(p["offsets"]), offsets)
    assert np.array_equal(host(p["row_to_token"]), r2t)
    assert counts.sum() / cfg.E == 39
    oracle.set_threads(os.cpu_count() or 1)
    try:
        check_layer_against_oracle(cfg, t, out, logits)
    finally:
        oracle.set_threads(1)


@pytest.mark.parametrize("cfg", [
    MoEConfig("micro", N=4100, H=256, I=128, E=64, k=8),              # halves of 2048 and 2052 tokens
    MoEConfig("micro_k6", N=6000, H=128, I=192, E=48, k=6),            # halves of 2560 and 3440 tokens
    MoEConfig("micro_shared", N=4096, H=128, I=192, E=16, k=8, Is=128),  # shared experts: runs in one piece
])
def test_layer_in_two_microbatches_gives_the_same_bits(cfg):
    """The layer with its expert GEMMs run as two micro-batches of tokens (the second
    half's row copies and the first half's combine on the library's second stream) gives
    the bits of the one-piece layer, logits included, and replays the same from a CUDA
    graph (the second stream joins the capture)."""
    t = cuda_inputs(cfg, seed=31)
    prev = moe.moe_set_microbatches(1)
    try:
        one, l1 = run_layer(cfg, t)
        moe.moe_set_microbatches(2)
        two, l2 = run_layer(cfg, t)
        torch.cuda.synchronize()
        assert torch.equal(l1, l2)
        assert torch.equal(one.view(torch.int16), two.view(torch.int16))
        ws = torch.empty(moe.moe_workspace_bytes(cfg.N, cfg.H, cfg.I, cfg.E, cfg.k, cfg.Is), dtype=torch.uint8,
                         device="cuda")
        out = torch.zeros_like(one)

        def step():
            moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, Ws1=t.get("Ws1"),
                                     Ws3=t.get("Ws3"), Ws2=t.get("Ws2"), ws=ws, out=out,
                                     stream=torch.cuda.current_stream())
        step()
        torch.cuda.synchronize()
        out.zero_()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == 0
        assert torch.equal(out.view(torch.int16), one.view(torch.int16))
        del g
    finally:
        moe.moe_set_microbatches(prev)


SIDE_CASES = [
    MoEConfig("side", N=700, H=256, I=128, E=8, k=2, Is=192),
    MoEConfig("side_e32", N=800, H=384, I=192, E=32, k=6, Is=256),
    MoEConfig("side_ragged", N=300, H=256, I=192, E=16, k=2, Is=320),     # ragged shared feature tiles
]


@pytest.mark.parametrize("cfg", SIDE_CASES, ids=lambda c: c.name)
def test_shared_experts_on_the_side_stream_give_the_same_bits(cfg):
    """The shared experts forked onto the library's second stream at the start of the
    call and joined before the combine: the same bits as on the caller's stream, eager and
    replayed from a CUDA graph (the second stream joins the capture)."""
    t = cuda_inputs(cfg, seed=17)
    prev = moe.moe_set_shared_stream(False)
    try:
        one, l1 = run_layer(cfg, t)
        moe.moe_set_shared_stream(True)
        two, l2 = run_layer(cfg, t)
        torch.cuda.synchronize()
        assert torch.equal(l1, l2)
        assert torch.equal(one.view(torch.int16), two.view(torch.int16))
        ws = torch.empty(moe.moe_workspace_bytes(cfg.N, cfg.H, cfg.I, cfg.E, cfg.k, cfg.Is), dtype=torch.uint8,
                         device="cuda")
        out = torch.zeros_like(one)

        def step():
            moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, Ws1=t["Ws1"],
                                     Ws3=t["Ws3"], Ws2=t["Ws2"], ws=ws, out=out, stream=torch.cuda.current_stream())
        step()
        torch.cuda.synchronize()
        out.zero_()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == 0
        assert torch.equal(out.view(torch.int16), one.view(torch.int16))
        del g
    finally:
        moe.moe_set_shared_stream(prev)



DECODE_SHAPES = [
    # (shape, mode): AUTO takes the GEMV kernels for 2*N*k <= E (H <= 2048, I <= 1024); ON up to 512 rows
    (MoEConfig("dec_one", N=1, H=512, I=256, E=32, k=8), moe.MOE_DECODE_AUTO),
    (MoEConfig("dec_qwen_shape", N=4, H=2048, I=768, E=128, k=8), moe.MOE_DECODE_AUTO),
    (MoEConfig("dec_qwen_8", N=8, H=2048, I=768, E=128, k=8), moe.MOE_DECODE_AUTO),
    (MoEConfig("dec_wide_h", N=2, H=8192, I=2048, E=64, k=4), moe.MOE_DECODE_ON),     # rows staged nowhere
    (MoEConfig("dec_long_rows", N=4, H=5120, I=1536, E=160, k=6), moe.MOE_DECODE_ON),  # several load rounds
    (MoEConfig("dec_qwen_16", N=16, H=2048, I=768, E=128, k=8), moe.MOE_DECODE_ON),
    (MoEConfig("dec_ragged", N=5, H=320, I=192, E=160, k=6), moe.MOE_DECODE_AUTO),   # rows and K not multiples of 256
    (MoEConfig("dec_shared", N=3, H=256, I=128, E=64, k=4, Is=192), moe.MOE_DECODE_AUTO),
    (MoEConfig("dec_crowded", N=40, H=256, I=128, E=8, k=2), moe.MOE_DECODE_ON),     # ~10 tokens per expert
    (MoEConfig("dec_max", N=64, H=128, I=64, E=256, k=8), moe.MOE_DECODE_ON),        # 512 rows, every expert
    (MoEConfig("dec_dense", N=3, H=256, I=128, E=1, k=1), moe.MOE_DECODE_ON),        # one expert, top-1
    (MoEConfig("dec_router_fused", N=2, H=192, I=128, E=16, k=2), moe.MOE_DECODE_AUTO),  # the one-kernel router picks
]


@pytest.mark.parametrize("cfg,mode", DECODE_SHAPES, ids=[c.name for c, _ in DECODE_SHAPES])
def test_decode_gemv_layer_matches_oracle(cfg, mode):
    """The decode form of the layer (W1/W3 + SwiGLU and W2 + combine as CUDA-core GEMVs,
    each pick's x row read directly, the top-k finished inside the first) against the
    oracle on every token, with a router bias; the routing maps bit-exact; deterministic
    from call to call and under CUDA-graph replay; the launch count shows the form ran
    (router partials and two GEMV kernels: three, against five or more for the grouped
    GEMMs)."""
    t = cuda_inputs(cfg, seed=37)
    t["bias"] = torch.linspace(-0.3, 0.3, cfg.E, device="cuda")
    prev = moe.moe_set_decode_gemv(mode)
    try:
        n0 = moe.moe_kernel_launches()
        out, logits = run_layer(cfg, t)
        launches = moe.moe_kernel_launches() - n0
        torch.cuda.synchronize()
        check_layer_against_oracle(cfg, t, out, logits)
        if cfg.Is == 0:
            assert launches == 3, launches
        idx, _, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k, bias=t["bias"])
        ref_idx, _ = oracle.topk(host(logits), cfg.k)
        assert np.array_equal(host(idx), ref_idx)
        again, _ = run_layer(cfg, t)
        torch.cuda.synchronize()
        assert torch.equal(again.view(torch.int16), out.view(torch.int16))
        ws = torch.empty(moe.moe_workspace_bytes(cfg.N, cfg.H, cfg.I, cfg.E, cfg.k, cfg.Is), dtype=torch.uint8,
                         device="cuda")
        o2 = torch.zeros_like(out)

        def step():
            moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, bias=t["bias"],
                                     Ws1=t.get("Ws1"), Ws3=t.get("Ws3"), Ws2=t.get("Ws2"), ws=ws, out=o2,
                                     stream=torch.cuda.current_stream())
        step()
        torch.cuda.synchronize()
        o2.zero_()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_get_device_error() == 0
        assert torch.equal(o2.view(torch.int16), out.view(torch.int16))
        del g
    finally:
        moe.moe_set_decode_gemv(prev)


def test_decode_gemv_and_grouped_gemm_agree():
    """The same decode batch through the GEMV kernels and through the grouped GEMMs:
    identical routing, and outputs that differ only by the summation order inside each
    dot product (a few bf16 ulps at most)."""
    cfg = MoEConfig("dec_agree", N=8, H=1024, I=512, E=64, k=8)
    t = cuda_inputs(cfg, seed=41)
    prev = moe.moe_set_decode_gemv(moe.MOE_DECODE_ON)
    try:
        a, la = run_layer(cfg, t)
        moe.moe_set_decode_gemv(moe.MOE_DECODE_OFF)
        b, lb = run_layer(cfg, t)
        torch.cuda.synchronize()
        assert torch.equal(la, lb)
        d = (a.float() - b.float()).abs()
        assert bool((d <= 2.0 ** -6 * b.float().abs() + 1e-3).all()), float(d.max())
    finally:
        moe.moe_set_decode_gemv(prev)

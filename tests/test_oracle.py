"""Pins for the CPU oracle, each against something other than the oracle itself.

CPU only.  Sources of truth used here: hand-worked fixtures under
tests/golden/ (each cites the page and section it follows), torch's own bf16
conversion, float64 BLAS products, full sorts, numpy's stable argsort, dense
evaluation of every expert on every token, and invariants of the method.
"""
import math
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from expert_ffn_layer_moe_b200.inputs import CONFIGS, MoEConfig, make_inputs
from tests._bf16 import dec, enc, to_u16, ulp_diff

GOLD = Path(__file__).parent / "golden"


def _rows(name):
    for line in (GOLD / name).read_text().splitlines():
        line = line.strip()
        if line and not line.startswith("#"):
            yield line


def small_layer(N=24, H=64, I=32, E=4, k=2, Is=0, seed=3):
    cfg = MoEConfig("pin", N=N, H=H, I=I, E=E, k=k, Is=Is)
    t = make_inputs(cfg, seed=seed)
    return cfg, {n: (to_u16(v) if v is not None and v.dtype == torch.bfloat16 else
                     (None if v is None else v.numpy())) for n, v in t.items()}


def dense_swiglu(xd, W1d, W3d, W2d):
    """Dense SwiGLU FFN in float64 with torch's silu and BLAS products,
    rounding h to bf16 (the second GEMM's operand); y stays float64."""
    x = torch.from_numpy(xd)
    g = x @ torch.from_numpy(W1d).T
    u = x @ torch.from_numpy(W3d).T
    h = dec(enc((F.silu(g) * u).numpy()))
    return (torch.from_numpy(h) @ torch.from_numpy(W2d).T).numpy()


# ------------------------------------------------------------------ bf16 ----

def test_bf16_rounding_golden():
    for line in _rows("bf16_rounding.txt"):
        val, bits = line.split()[:2]
        assert oracle.round_to_bf16(float.fromhex(val)) == int(bits, 16), line


def test_bf16_rounding_matches_torch_on_fp32_values():
    g = torch.Generator().manual_seed(11)
    mant = torch.rand(20000, generator=g, dtype=torch.float64) + 1.0
    ex = torch.randint(-140, 128, (20000,), generator=g)
    v = (mant * torch.pow(2.0, ex.to(torch.float64))).to(torch.float32)
    v[::2] *= -1
    # exact midpoints between bf16 neighbours, where ties-to-even decides
    mid = (torch.randint(0, 2 ** 15, (4000,), generator=g, dtype=torch.int32) << 16) | 0x8000
    v = torch.cat([v, mid.view(torch.float32)])
    v = v[torch.isfinite(v)]
    want = to_u16(v.to(torch.bfloat16))
    got = oracle.round_to_bf16(v.to(torch.float64).numpy())
    assert np.array_equal(got, want)


def test_bf16_decode_all_patterns():
    u = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f64(u)
    want = dec(u)
    finite = np.isfinite(want)
    assert np.array_equal(got[finite], want[finite])
    assert np.array_equal(np.isnan(got), np.isnan(want))


# ---------------------------------------------------------------- router ----

def test_logits_match_float64_product():
    cfg = CONFIGS["tiny"]
    t = make_inputs(cfg, seed=0, weights=False)
    bias = torch.linspace(-1, 1, cfg.E, dtype=torch.float32)
    got = oracle.router_logits(to_u16(t["x"]), t["W_gate"].numpy(), bias.numpy())
    xd = t["x"].to(torch.float64)
    want = (xd @ t["W_gate"].to(torch.float64) + bias.to(torch.float64)).numpy()
    scale = (xd.abs() @ t["W_gate"].to(torch.float64).abs()).numpy() + 1.0
    assert np.all(np.abs(got - want) <= 1e-13 * scale)


def test_topk_golden_ties():
    for line in _rows("topk_ties.txt"):
        k, logits, want = [p.strip() for p in line.split("|")]
        l = np.array([[float(v) for v in logits.split()]], dtype=np.float32)
        idx, w = oracle.topk(l, int(k))
        assert idx[0].tolist() == [int(v) for v in want.split()], line


def test_topk_matches_full_sort():
    g = np.random.default_rng(5)
    N, E = 200, 37
    # coarse values force many exact ties
    l = (g.integers(-6, 6, size=(N, E)) * 0.5).astype(np.float32)
    for k in (1, 2, 5, E):
        idx, _ = oracle.topk(l, k)
        for t in range(N):
            order = sorted(range(E), key=lambda e: (-float(l[t, e]), e))
            assert idx[t].tolist() == order[:k]


def test_topk_weights_closed_forms():
    g = np.random.default_rng(6)
    l = g.standard_normal((64, 16)).astype(np.float32)
    _, w1 = oracle.topk(l, 1)
    assert np.all(w1 == 1.0)
    idx, w2 = oracle.topk(l, 2)
    l0 = l[np.arange(64), idx[:, 0]].astype(np.float64)
    l1 = l[np.arange(64), idx[:, 1]].astype(np.float64)
    assert np.allclose(w2[:, 0], 1.0 / (1.0 + np.exp(l1 - l0)), rtol=1e-15, atol=0)
    # softmax over all E renormalised over the picks equals the stated form
    idx, w6 = oracle.topk(l, 6)
    p = np.exp(l.astype(np.float64) - l.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    pk = np.take_along_axis(p, idx.astype(np.int64), 1)
    assert np.allclose(w6, pk / pk.sum(1, keepdims=True), rtol=1e-13, atol=0)
    assert np.allclose(w6.sum(1), 1.0, rtol=0, atol=1e-15)
    assert np.all(np.diff(w6, axis=1) <= 0)
    # the golden two-expert weights (hand-worked layer)
    rows = dict(r.split(maxsplit=1) for r in _rows("tiny_layer_by_hand.txt"))
    _, w = oracle.topk(np.array([[1.0, -1.0]], np.float32), 2)
    assert np.allclose(w[0], [float(v) for v in rows["w"].split()], rtol=1e-15, atol=0)


# -------------------------------------------------------------- dispatch ----

def test_dispatch_matches_stable_argsort():
    g = np.random.default_rng(7)
    N, E, k = 300, 9, 3
    idx = np.stack([g.permutation(E)[:k] for _ in range(N)]).astype(np.int32)
    idx[:40] = [0, 1, 2]                              # a hot expert group
    counts, offsets, r2t, t2r = oracle.dispatch(idx, E)
    order = np.argsort(idx.ravel(), kind="stable")    # assignment ids sorted by expert
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(r2t, order // k)
    inv = np.empty_like(order)
    inv[order] = np.arange(N * k)
    assert np.array_equal(t2r.ravel(), inv)


def test_dispatch_invariants_and_empty_experts():
    g = np.random.default_rng(8)
    N, E, k = 50, 12, 2
    idx = np.stack([g.choice([1, 4, 7, 9], size=k, replace=False) for _ in range(N)]).astype(np.int32)
    counts, offsets, r2t, t2r = oracle.dispatch(idx, E)
    assert counts.sum() == N * k and offsets[-1] == N * k
    assert all(counts[e] == 0 for e in range(E) if e not in (1, 4, 7, 9))
    assert np.all(np.diff(offsets) >= 0)
    assert sorted(t2r.ravel().tolist()) == list(range(N * k))      # bijection
    assert np.array_equal(r2t[t2r], np.repeat(np.arange(N)[:, None], k, 1))
    for e in range(E):
        seg = r2t[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)                            # stable, ascending token


def test_dispatch_rejects_bad_index():
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, 5]], np.int32), 4)
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, -1]], np.int32), 4)


def test_mixtral_worked_example_mean_rows():
    """156 tokens, 8 experts, top-2: 312 assignments, 39 rows per expert on
    average (MegaScale-Infer summary, section "核心问题")."""
    fx = dict(r.split() for r in _rows("mixtral_worked_example.txt"))
    cfg = CONFIGS["mixtral_8x22b_decode"]
    assert (cfg.N, cfg.E, cfg.k) == (int(fx["tokens"]), int(fx["experts"]), int(fx["top_k"]))
    t = make_inputs(cfg, seed=0, weights=False)
    l64 = oracle.router_logits(to_u16(t["x"]), t["W_gate"].numpy())
    idx, _ = oracle.topk(l64.astype(np.float32), cfg.k)
    counts, offsets, _, _ = oracle.dispatch(idx, cfg.E)
    assert counts.sum() == int(fx["assignments"])
    assert counts.sum() / cfg.E == float(fx["mean_rows_per_expert"])
    assert float(fx["ffn_mfu"]) == cfg.k / cfg.E


def test_permute_rows_copies_bits():
    cfg, t = small_layer()
    idx, _ = oracle.topk(oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32), cfg.k)
    _, _, r2t, _ = oracle.dispatch(idx, cfg.E)
    assert np.array_equal(oracle.permute_rows(t["x"], r2t), t["x"][r2t])


# ------------------------------------------------------------ expert FFN ----

def test_swiglu_ffn_matches_dense_float64():
    cfg, t = small_layer(N=8, H=96, I=48, E=2)
    W1, W3, W2 = t["W1"][1], t["W3"][1], t["W2"][1]
    want = dense_swiglu(dec(t["x"]), dec(W1), dec(W3), dec(W2))
    got = np.stack([oracle.swiglu_ffn(t["x"][i], W1, W3, W2) for i in range(cfg.N)])
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)


def test_layer_by_hand():
    rows = dict(r.split(maxsplit=1) for r in _rows("tiny_layer_by_hand.txt"))
    b = lambda *v: np.array(v, np.float32).astype(np.float64)
    x = enc(np.array([[1.0, 0.0]]))
    Wg = np.array([[1.0, -1.0], [0.0, 0.0]], np.float32)
    W1 = enc(np.array([[[2.0, 0.0]], [[-1.0, 0.0]]]))
    W3 = enc(np.array([[[1.0, 0.0]], [[4.0, 0.0]]]))
    W2 = enc(np.array([[[1.0], [-0.5]], [[1.0], [2.0]]]))
    out, logits = oracle.layer(x, Wg, W1, W3, W2, k=2)
    assert logits.tolist() == [[1.0, -1.0]]
    res = oracle.layer_given_logits(x, logits, W1, W3, W2, 2, extras=True)
    assert res["idx"][0].tolist() == [int(v) for v in rows["idx"].split()]
    r0, r1 = res["token_to_row"][0]
    assert res["y_perm"][r0].tolist() == [float(v) for v in rows["y0"].split()]
    assert res["y_perm"][r1].tolist() == [float(v) for v in rows["y1"].split()]
    assert out[0].tolist() == [int(v, 16) for v in rows["out"].split()]
    Ws1 = enc(np.array([[1.0, 0.0]])); Ws3 = enc(np.array([[1.0, 0.0]]))
    Ws2 = enc(np.array([[1.0], [1.0]]))
    out_s, _ = oracle.layer(x, Wg, W1, W3, W2, k=2, Ws1=Ws1, Ws3=Ws3, Ws2=Ws2)
    assert out_s[0].tolist() == [int(v, 16) for v in rows["out_shared"].split()]


def test_layer_equals_dense_masked_evaluation():
    """Run every expert on every token, weight by the routing mask and sum in
    pick order: the sparse dispatch/permute/combine path must agree."""
    cfg, t = small_layer(N=20, H=64, I=32, E=5, k=3)
    l32 = oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32)
    out = oracle.layer_given_logits(t["x"], l32, t["W1"], t["W3"], t["W2"], cfg.k)
    idx, w = oracle.topk(l32, cfg.k)
    xd = dec(t["x"])
    Y = np.stack([dense_swiglu(xd, dec(t["W1"][e]), dec(t["W3"][e]), dec(t["W2"][e]))
                  for e in range(cfg.E)])                         # [E, N, H]
    acc = np.zeros((cfg.N, cfg.H))
    for j in range(cfg.k):
        acc += w[:, j:j + 1] * Y[idx[:, j], np.arange(cfg.N)]
    d = ulp_diff(out, enc(acc))
    assert d.max() <= 1 and (d == 0).mean() > 0.99


def test_single_expert_top1_is_dense_swiglu():
    cfg, t = small_layer(N=16, H=64, I=96, E=1, k=1)
    out, _ = oracle.layer(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], k=1)
    want = enc(dense_swiglu(dec(t["x"]), dec(t["W1"][0]), dec(t["W3"][0]), dec(t["W2"][0])))
    d = ulp_diff(out, want)
    assert d.max() <= 1 and (d == 0).mean() > 0.99


def test_shared_expert_alone_is_dense_swiglu():
    cfg, t = small_layer(N=12, H=64, I=32, E=3, k=2, Is=48)
    W2zero = np.zeros_like(t["W2"])
    out, _ = oracle.layer(t["x"], t["W_gate"], t["W1"], t["W3"], W2zero, k=2,
                          Ws1=t["Ws1"], Ws3=t["Ws3"], Ws2=t["Ws2"])
    want = enc(dense_swiglu(dec(t["x"]), dec(t["Ws1"]), dec(t["Ws3"]), dec(t["Ws2"])))
    d = ulp_diff(out, want)
    assert d.max() <= 1 and (d == 0).mean() > 0.99


def test_expert_relabelling_is_invisible():
    cfg, t = small_layer(N=16, H=64, I=32, E=6, k=2)
    out, _ = oracle.layer(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], k=2)
    pi = np.array([3, 5, 0, 2, 1, 4])
    out_p, _ = oracle.layer(t["x"], t["W_gate"][:, pi], t["W1"][pi], t["W3"][pi], t["W2"][pi], k=2)
    assert np.array_equal(out, out_p)


def test_w2_scaling_by_two_is_exact():
    cfg, t = small_layer(N=10, H=64, I=32, E=4, k=2)
    l32 = oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32)
    out = oracle.layer_given_logits(t["x"], l32, t["W1"], t["W3"], t["W2"], 2)
    out2 = oracle.layer_given_logits(t["x"], l32, t["W1"], t["W3"], enc(2.0 * dec(t["W2"])), 2)
    assert np.array_equal(dec(out2), 2.0 * dec(out))


def test_layer_routes_with_its_own_fp32_logits():
    cfg, t = small_layer(N=10, H=64, I=32, E=4, k=2)
    out, l32 = oracle.layer(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], k=2)
    assert np.array_equal(l32, oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32))
    assert np.array_equal(out, oracle.layer_given_logits(t["x"], l32, t["W1"], t["W3"], t["W2"], 2))


def test_qwen3_30b_shape_matches_parameter_arithmetic():
    """The MoE-latency article, section "内存按总参数算": Qwen3-30B-A3B holds
    30.5B parameters, 8 of 128 experts per token, 48 layers, about 61 GB at
    2 bytes per parameter.  The expert stacks of the Qwen3-30B-shaped layer
    must fit inside that total."""
    c = CONFIGS["qwen3_30b_a3b"]
    expert_params = c.E * 3 * c.H * c.I * 48
    assert c.E == 128 and c.k == 8
    assert 0.9 * 30.5e9 < expert_params < 30.5e9
    assert abs(30.5e9 * 2 / 1e9 - 61) < 0.5


# ------------------------------------------------------------- fp8 weights ----
# [MoE-latency] "优化从测量开始": quantized weights are their own experiment.
# The e4m3 format is pinned against torch's float8_e4m3fn (an independent
# implementation of the same OCP format) and against nearest-value search.

def test_e4m3_decode_every_code_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    want = codes.view(torch.float8_e4m3fn).double().numpy()
    got = oracle.fp8_to_f64(codes.numpy())
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(want[ok]))
    # the format's landmarks: smallest subnormal, smallest normal, one, largest; NaN only at 0x7F/0xFF
    assert got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6 and got[0x38] == 1.0 and got[0x7E] == 448.0
    assert set(np.flatnonzero(np.isnan(got)).tolist()) == {0x7F, 0xFF}


def test_e4m3_encode_is_nearest_with_ties_to_even_code():
    finite = [c for c in range(0x7F)]                       # 0x00 .. 0x7E, non-negative
    vals = oracle.fp8_to_f64(np.array(finite, np.uint8))
    assert np.all(np.diff(vals) > 0)                         # codes order the values
    # every value encodes to its own code; every midpoint to the neighbour with an even code
    assert np.array_equal(oracle.fp8_from_f32(vals.astype(np.float32)), np.array(finite, np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (vals[:-1] + vals[1:]) / 2)   # midpoints exact in fp32
    got = oracle.fp8_from_f32(mids)
    lo = np.array(finite[:-1], np.uint8)
    want = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    assert np.array_equal(got, want)
    # negative side mirrors; past 448 saturates at 448
    assert np.array_equal(oracle.fp8_from_f32(-vals[1:].astype(np.float32)), np.array(finite[1:], np.uint8) | 0x80)
    assert oracle.fp8_from_f32(np.array([464.0, 1e9, -1e9], np.float32)).tolist() == [0x7E, 0x7E, 0xFE]


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-14, 6, 100000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.fp8_from_f32(x), want)


def test_quantizer_scale_codes_and_error_bound():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((40, 192)) * np.exp(rng.uniform(-6, 3, (40, 1)))).astype(np.float32)
    W[7] = 0.0                                                    # an all-zero row
    Wb = enc(W)
    q, sc = oracle.quantize_rows_fp8(Wb)
    Wd = dec(Wb)
    assert sc[7] == 1.0 and not q[7].any()
    amax = np.abs(Wd).max(axis=1)
    nz = amax > 0
    assert np.array_equal(sc[nz], (amax[nz].astype(np.float32) / np.float32(448)).astype(np.float32))
    # each nonzero row's largest magnitude lands on +-448
    top = np.abs(Wd).argmax(axis=1)
    assert all((q[r, top[r]] & 0x7F) == 0x7E for r in np.flatnonzero(nz))
    # the rounding step is torch's e4m3 conversion of the fp32 quotient
    quot = (Wd.astype(np.float32) / sc[:, None]).astype(np.float32)
    assert np.array_equal(q, torch.from_numpy(quot).to(torch.float8_e4m3fn).view(torch.uint8).numpy())
    # reconstruction: within half an e4m3 step (2^-4 relative, 2^-10 absolute in the subnormals) of the weight
    rec = oracle.fp8_to_f64(q) * sc[:, None].astype(np.float64)
    err = np.abs(rec - Wd)
    bound = (2.0 ** -4 * np.abs(Wd) + 2.0 ** -10 * sc[:, None]) * (1 + 2.0 ** -20)
    assert np.all(err <= bound)


def _grid_weights(rng, shape, jlo=-14, jhi=-6):
    """bf16 rows that are e4m3 values times a power of two 2^j per row (j in
    [jlo, jhi)), each row holding +-448 times that power: the per-row quantizer
    represents them exactly."""
    pos = oracle.fp8_to_f64(np.arange(1, 0x7F, dtype=np.uint8))
    v = rng.choice(pos, size=shape) * rng.choice([-1.0, 1.0], size=shape)
    v[..., 0] = 448.0 * rng.choice([-1.0, 1.0], size=shape[:-1])
    j = rng.integers(jlo, jhi, size=shape[:-1] + (1,))
    return enc((v * np.exp2(j)).astype(np.float32))


def test_fp8_layer_equals_bf16_layer_on_exactly_representable_weights():
    cfg, t = small_layer(N=18, H=64, I=32, E=4, k=2)
    rng = np.random.default_rng(9)
    W1 = _grid_weights(rng, (cfg.E, cfg.I, cfg.H))
    W3 = _grid_weights(rng, (cfg.E, cfg.I, cfg.H))
    W2 = _grid_weights(rng, (cfg.E, cfg.H, cfg.I))
    q1, s1 = oracle.quantize_rows_fp8(W1)
    q3, s3 = oracle.quantize_rows_fp8(W3)
    q2, s2 = oracle.quantize_rows_fp8(W2)
    assert np.array_equal(enc((oracle.fp8_to_f64(q1) * s1[..., None]).astype(np.float32)), W1)
    l32 = oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32)
    want = oracle.layer_given_logits(t["x"], l32, W1, W3, W2, cfg.k)
    got = oracle.layer_given_logits_fp8(t["x"], l32, q1, s1, q3, s3, q2, s2, cfg.k)
    assert np.array_equal(got, want)
    xp = t["x"][np.arange(cfg.N).repeat(1)]
    off = np.array([0, 5, 9, 9, cfg.N], np.int32)
    assert np.array_equal(oracle.expert_ffn_fp8(xp, off, q1, s1, q3, s3, q2, s2),
                          oracle.expert_ffn(xp, off, W1, W3, W2))


def test_fp8_layer_error_against_bf16_is_quantization_sized():
    """Ordinary weights: the fp8 layer differs from the bf16 layer by about the
    e4m3 step (2^-4 relative) averaged over the sums, far less than the outputs."""
    cfg, t = small_layer(N=24, H=128, I=64, E=4, k=2)
    l32 = oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32)
    want = dec(oracle.layer_given_logits(t["x"], l32, t["W1"], t["W3"], t["W2"], cfg.k))
    qs = [oracle.quantize_rows_fp8(t[n]) for n in ("W1", "W3", "W2")]
    got = dec(oracle.layer_given_logits_fp8(t["x"], l32, *qs[0], *qs[1], *qs[2], cfg.k))
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert 1e-3 < rel < 5e-2


# ---------------------------------------------- fp8 weights and fp8 activations
# [MoE-latency] "优化从测量开始": activations quantized beside the weights, with the
# error measured.  Each pin reduces the activation-quantized experts to something
# pinned above (the weight-only fp8 experts, a float64 BLAS product) or to an exact
# invariant of per-row scaling.

def _fp8_experts(t):
    return [a for n in ("W1", "W3", "W2") for a in oracle.quantize_rows_fp8(t[n])]


def _ffn_case(R=20, H=128, I=64, E=4, seed=3):
    cfg, t = small_layer(N=R, H=H, I=I, E=E, k=1, seed=seed)
    off = np.array([0, 6, 6, 13, R], np.int32)             # one empty group, ragged others
    return cfg, t, _fp8_experts(t), off


def test_fp8_acts_exact_x_rows_give_the_weight_only_h():
    """x rows the quantizer represents exactly (a power-of-two scale per row): the
    quantized W1/W3 step gives the weight-only h bit for bit, and the weight-only
    option of the extended function is the weight-only experts pinned above."""
    cfg, t, q, off = _ffn_case()
    xg = _grid_weights(np.random.default_rng(11), (cfg.N, cfg.H), -8, -4)
    y0, h0 = oracle.expert_ffn_fp8_ex(xg, off, *q, quantize_acts=False)
    _, h1 = oracle.expert_ffn_fp8_ex(xg, off, *q, quantize_acts=True)
    assert np.array_equal(h1, h0)
    assert np.array_equal(y0, oracle.expert_ffn_fp8(xg, off, *q))
    # ordinary rows are not exact: h moves by about the e4m3 step averaged over the sums
    x = t["x"]
    _, hw = oracle.expert_ffn_fp8_ex(x, off, *q, quantize_acts=False)
    _, ha = oracle.expert_ffn_fp8_ex(x, off, *q, quantize_acts=True)
    d = np.linalg.norm(dec(ha) - dec(hw)) / np.linalg.norm(dec(hw))
    assert 1e-3 < d < 5e-2, d


def test_fp8_acts_exact_h_rows_give_the_blas_product():
    """h rows given in the exactly representable form: the quantized W2 step equals
    the weight-only one, and both equal a float64 BLAS product of the given h with
    the dequantized W2 of each row's expert."""
    cfg, t, q, off = _ffn_case()
    rng = np.random.default_rng(12)
    xg = _grid_weights(rng, (cfg.N, cfg.H), -8, -4)
    hg = _grid_weights(rng, (cfg.N, cfg.I), -6, -2)
    y0, _ = oracle.expert_ffn_fp8_ex(xg, off, *q, quantize_acts=False, h_given=hg)
    y1, _ = oracle.expert_ffn_fp8_ex(xg, off, *q, quantize_acts=True, h_given=hg)
    assert np.array_equal(y1, y0)
    W2d = oracle.fp8_to_f64(q[4]) * q[5][..., None].astype(np.float64)
    for e in range(cfg.E):
        r = slice(off[e], off[e + 1])
        assert np.allclose(y1[r], dec(hg[r]) @ W2d[e].T, rtol=1e-12, atol=1e-14)


def _dequant_rows(a):
    qa, sa = oracle.quantize_rows_fp8(a)
    return oracle.fp8_to_f64(qa) * sa[:, None].astype(np.float64)


def test_fp8_acts_steps_read_the_quantizer_output():
    """Ordinary activations: the experts' output equals a float64 BLAS statement
    that feeds each GEMM the pinned quantizer's dequantized rows -- x for W1/W3,
    the experts' own bf16 h for W2 -- with the dequantized weights."""
    cfg, t, q, off = _ffn_case()
    y, h = oracle.expert_ffn_fp8_ex(t["x"], off, *q, quantize_acts=True)
    W1d, W3d, W2d = (oracle.fp8_to_f64(q[i]) * q[i + 1][..., None].astype(np.float64) for i in (0, 2, 4))
    xq, hq = _dequant_rows(t["x"]), _dequant_rows(h)
    for e in range(cfg.E):
        if off[e] == off[e + 1]:
            continue
        r = slice(off[e], off[e + 1])
        g, u = xq[r] @ W1d[e].T, xq[r] @ W3d[e].T
        assert ulp_diff(h[r], enc(g / (1 + np.exp(-g)) * u)).max() <= 1
        assert np.allclose(y[r], hq[r] @ W2d[e].T, rtol=1e-12, atol=1e-14)
    # and those are not the unquantized rows
    assert not np.allclose(xq, dec(t["x"]), rtol=1e-3) and not np.allclose(hq, dec(h), rtol=1e-3)


def test_fp8_acts_quantize_the_bf16_h_and_use_a_given_one():
    """Handing back the experts' own bf16 h changes nothing (the quantizer reads h
    after its bf16 rounding); a different given h changes the output."""
    cfg, t, q, off = _ffn_case()
    y, h = oracle.expert_ffn_fp8_ex(t["x"], off, *q, quantize_acts=True)
    yg, _ = oracle.expert_ffn_fp8_ex(t["x"], off, *q, quantize_acts=True, h_given=h)
    assert np.array_equal(yg, y)
    h2 = h.copy()
    h2[3] = enc(-dec(h[3]))
    y2, _ = oracle.expert_ffn_fp8_ex(t["x"], off, *q, quantize_acts=True, h_given=h2)
    assert np.array_equal(y2[3], -y[3]) and np.array_equal(np.delete(y2, 3, 0), np.delete(y, 3, 0))


def test_fp8_acts_per_row_power_of_two_scaling_of_h_is_exact():
    """Scaling each given h row by its own power of two scales that row's scale and
    nothing else, so each output row scales by the same power exactly; a scale
    along the wrong axis, or shared between rows, would change the codes."""
    cfg, t, q, off = _ffn_case()
    _, h = oracle.expert_ffn_fp8_ex(t["x"], off, *q, quantize_acts=True)
    m = np.random.default_rng(13).integers(-3, 4, cfg.N).astype(np.float64)
    hs = enc((dec(h) * np.exp2(m)[:, None]).astype(np.float32))
    assert np.array_equal(dec(hs), dec(h) * np.exp2(m)[:, None])
    y, _ = oracle.expert_ffn_fp8_ex(t["x"], off, *q, quantize_acts=True, h_given=h)
    ys, _ = oracle.expert_ffn_fp8_ex(t["x"], off, *q, quantize_acts=True, h_given=hs)
    assert np.array_equal(ys, y * np.exp2(m)[:, None])


def test_fp8_acts_layer_is_its_steps_and_reads_h_in_assignment_order():
    """The layer = pinned top-k, dispatch and combine around the quantized experts;
    a given h in assignment order (row t*k + j) lands on the right permuted rows;
    without activation quantization it is the weight-only fp8 layer."""
    cfg, t = small_layer(N=24, H=128, I=64, E=4, k=2)
    q = _fp8_experts(t)
    l32 = oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32)
    idx, w = oracle.topk(l32, cfg.k)
    _, offsets, r2t, t2r = oracle.dispatch(idx, cfg.E)
    assert not np.array_equal(t2r.ravel(), np.arange(cfg.N * cfg.k))
    y, h = oracle.expert_ffn_fp8_ex(oracle.permute_rows(t["x"], r2t), offsets, *q, quantize_acts=True)
    out = oracle.layer_given_logits_fp8_ex(t["x"], l32, *q, cfg.k, quantize_acts=True)
    assert np.array_equal(out, oracle.combine(y, t2r, w))
    h_tok = h[t2r.ravel()]
    out_g = oracle.layer_given_logits_fp8_ex(t["x"], l32, *q, cfg.k, quantize_acts=True, h_given=h_tok)
    assert np.array_equal(out_g, out)
    assert np.array_equal(oracle.layer_given_logits_fp8_ex(t["x"], l32, *q, cfg.k, quantize_acts=False),
                          oracle.layer_given_logits_fp8(t["x"], l32, *q, cfg.k))


def test_fp8_acts_layer_error_against_bf16_is_quantization_sized():
    cfg, t = small_layer(N=24, H=128, I=64, E=4, k=2)
    l32 = oracle.router_logits(t["x"], t["W_gate"]).astype(np.float32)
    want = dec(oracle.layer_given_logits(t["x"], l32, t["W1"], t["W3"], t["W2"], cfg.k))
    got = dec(oracle.layer_given_logits_fp8_ex(t["x"], l32, *_fp8_experts(t), cfg.k, quantize_acts=True))
    w8 = dec(oracle.layer_given_logits_fp8(t["x"], l32, *_fp8_experts(t), cfg.k))
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    rel_w8 = np.linalg.norm(w8 - want) / np.linalg.norm(want)
    assert rel_w8 < rel < 8e-2, (rel, rel_w8)


def test_threaded_build_gives_the_serial_builds_bits():
    """The OpenMP build spreads independent tokens and rows over threads; each row's
    arithmetic is unchanged, so every output (logits, picks, weights, maps, fp64 expert
    rows, out, with shared experts and fp8 activations too) must be bit-identical to
    the serial build's."""
    cfg = MoEConfig("mt", N=37, H=128, I=192, E=16, k=4, Is=128)
    t = make_inputs(cfg, seed=3)
    x, Wg = to_u16(t["x"]), t["W_gate"].numpy()
    W1, W3, W2 = to_u16(t["W1"]), to_u16(t["W3"]), to_u16(t["W2"])
    Ws = [to_u16(t[n]) for n in ("Ws1", "Ws3", "Ws2")]

    def run():
        l64 = oracle.router_logits(x, Wg)
        out, l32 = oracle.layer(x, Wg, W1, W3, W2, cfg.k, Ws1=Ws[0], Ws3=Ws[1], Ws2=Ws[2])
        ex = oracle.layer_given_logits(x, l32, W1, W3, W2, cfg.k, Ws1=Ws[0], Ws3=Ws[1], Ws2=Ws[2], extras=True)
        q = [oracle.quantize_rows_fp8(W.reshape(-1, W.shape[-1])) for W in (W1, W3, W2)]
        qq = [(c.reshape(W.shape), s_.reshape(W.shape[:-1])) for (c, s_), W in zip(q, (W1, W3, W2))]
        a8 = oracle.expert_ffn_fp8_ex(oracle.permute_rows(x, ex["row_to_token"]), ex["offsets"], *qq[0], *qq[1],
                                      *qq[2], quantize_acts=1)
        return [l64, out, l32] + [ex[n] for n in sorted(ex)] + list(a8 if isinstance(a8, tuple) else (a8,))

    try:
        assert oracle.set_threads(1) == 1
        serial = run()
        assert oracle.set_threads(4) == 4
        threaded = run()
    finally:
        oracle.set_threads(1)
    assert len(serial) == len(threaded)
    for a, b in zip(serial, threaded):
        a, b = np.asarray(a), np.asarray(b)
        assert a.dtype == b.dtype and a.shape == b.shape
        assert a.tobytes() == b.tobytes()


def test_skew4x_scale_is_the_calibrated_one():
    """The 4x-mean skew reading's bias scale in the input recipe is the value the
    calibration script (oracle routing on the seeded inputs) recorded."""
    from expert_ffn_layer_moe_b200.inputs import SKEW4X_BIAS_SCALE, SKEW4X_LOAD_BAND
    rec = dict(l.split() for l in (Path(__file__).parent / "golden" / "skew4x_bias_scale.txt").read_text()
               .splitlines() if l and not l.startswith("#"))
    assert float(rec["bias_scale"]) == SKEW4X_BIAS_SCALE
    assert SKEW4X_LOAD_BAND[0] <= float(rec["max_over_mean_load"]) <= SKEW4X_LOAD_BAND[1]
    assert CONFIGS["qwen3_235b_a22b_skew4x"].bias_scale == SKEW4X_BIAS_SCALE

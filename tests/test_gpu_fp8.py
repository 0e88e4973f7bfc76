"""GPU parity of the fp8 (e4m3) expert-weight path against the oracle.

[MoE-latency] "优化从测量开始": quantized weights are an experiment of their own,
with their numerical error measured.  Bars: the quantizer's bytes and scales
bit-exact against the oracle's; the fp8 layer against the oracle's fp8 layer
(the same e4m3 codes and scales) within |d| <= 2e-2*|ref| + 2e-3; its distance
from the bf16 layer reported and bounded by the quantization step.
"""
import numpy as np
import pytest
import torch

import oracle
from expert_ffn_layer_moe_b200 import moe
from expert_ffn_layer_moe_b200.inputs import CONFIGS, MoEConfig
from tests._bf16 import dec
from tests.test_gpu_parity import assert_close, cuda_inputs, host

pytestmark = pytest.mark.gpu


def quantized(t):
    """GPU-quantized routed weights: dict name -> (codes, scales) on the device."""
    return {n: moe.moe_quantize_fp8(t[n]) for n in ("W1", "W3", "W2")}


def run_fp8_layer(cfg, t, q, **kw):
    logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
    out = moe.moe_layer_forward_fp8_ex(t["x"], t["W_gate"], *q["W1"], *q["W3"], *q["W2"], cfg.k, bias=t["bias"],
                                       Ws1=t.get("Ws1"), Ws3=t.get("Ws3"), Ws2=t.get("Ws2"), logits=logits, **kw)
    assert moe.moe_get_device_error() == 0
    return out, logits


def check_fp8_layer(cfg, t, q, out, logits, tokens=None):
    sel = slice(None) if tokens is None else tokens
    hq = {n: (host(c), host(s)) for n, (c, s) in q.items()}
    ref = oracle.layer_given_logits_fp8(host(t["x"])[sel], host(logits)[sel], *hq["W1"], *hq["W3"], *hq["W2"],
                                        cfg.k, Ws1=host(t.get("Ws1")), Ws3=host(t.get("Ws3")),
                                        Ws2=host(t.get("Ws2")))
    assert_close(dec(host(out)[sel]), dec(ref), f"{cfg.name} fp8 out")


@pytest.mark.parametrize("shape", [(4, 192, 256), (3, 64, 64), (2, 1000, 640)])
def test_quantizer_bit_exact(shape):
    g = torch.Generator().manual_seed(sum(shape))
    W = torch.randn(shape, generator=g) * torch.exp(torch.empty(shape[:-1] + (1,)).uniform_(-8, 4, generator=g))
    W[0, 1] = 0.0                                     # an all-zero row
    W[-1, -1, 3] = 3.0e38                             # a huge magnitude (bf16 range)
    Wb = W.to(torch.bfloat16)
    q, sc = moe.moe_quantize_fp8(Wb.cuda())
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_rows_fp8(host(Wb))
    assert np.array_equal(host(sc), rs)
    assert np.array_equal(host(q), rq)


def test_expert_ffn_fp8_matches_oracle():
    cfg = MoEConfig("ffn8", N=150, H=256, I=320, E=6, k=2)
    t = cuda_inputs(cfg, seed=2)
    q = quantized(t)
    idx, w, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k)
    p = moe.moe_permute(t["x"], idx, cfg.E)
    y = moe.moe_expert_ffn_fp8(p["x_perm"], p["offsets"], *q["W1"], *q["W3"], *q["W2"])
    torch.cuda.synchronize()
    hq = {n: (host(c), host(s)) for n, (c, s) in q.items()}
    ref = oracle.expert_ffn_fp8(host(p["x_perm"]), host(p["offsets"]), *hq["W1"], *hq["W3"], *hq["W2"])
    assert_close(host(y), ref, "fp8 y_perm")


def test_layer_fp8_tiny_matches_oracle():
    cfg = CONFIGS["tiny"]
    t = cuda_inputs(cfg)
    q = quantized(t)
    out, logits = run_fp8_layer(cfg, t, q)
    check_fp8_layer(cfg, t, q, out, logits)


@pytest.mark.parametrize("cfg", [
    MoEConfig("ragged", N=300, H=320, I=192, E=5, k=2),        # several tiles, ragged tails
    MoEConfig("narrow", N=48, H=256, I=256, E=16, k=4),        # 32-row tiles on single CTAs
    MoEConfig("wide", N=400, H=256, I=384, E=8, k=2),          # 128-row tiles
    MoEConfig("wider", N=800, H=192, I=128, E=4, k=2),         # 256-row tiles
    MoEConfig("shared", N=90, H=256, I=128, E=6, k=2, Is=192),  # bf16 shared experts beside fp8 routed ones
    MoEConfig("splitk", N=64, H=256, I=2048, E=4, k=2),        # W2 splits K; long fp8 ring walk
    MoEConfig("maxEk", N=512, H=256, I=128, E=256, k=8),
    MoEConfig("narrowest", N=40, H=64, I=64, E=3, k=2),
])
def test_layer_fp8_shapes_match_oracle(cfg):
    t = cuda_inputs(cfg, seed=1)
    q = quantized(t)
    out, logits = run_fp8_layer(cfg, t, q)
    check_fp8_layer(cfg, t, q, out, logits)


def test_subnormal_e4m3_weights_are_widened_exactly():
    """Weights whose codes are e4m3 subnormals (m * 2^-9 times the row scale): x is
    zero on the one column holding each row's largest weight, and the first W1/W3 row
    is zero (so h[0] = 0), so every output comes from subnormal codes alone -- a
    widening that flushed them would give zeros."""
    cfg = MoEConfig("sub", N=32, H=64, I=64, E=1, k=1)
    t = cuda_inputs(cfg, seed=4)
    g = torch.Generator().manual_seed(4)

    def sub_rows(rows, cols):
        m = torch.randint(1, 8, (rows, cols), generator=g).float() * torch.where(
            torch.rand((rows, cols), generator=g) < 0.5, -1.0, 1.0)
        w = m * 2.0 ** -9 * 2.0 ** 9         # row scale 2^9: the codes are m * 2^-9
        w[:, 0] = 448.0 * 2.0 ** 9           # the row maximum on column 0
        return w.to(torch.bfloat16)

    W1, W3, W2 = sub_rows(64, 64), sub_rows(64, 64), sub_rows(64, 64)
    W1[0] = 0
    W3[0] = 0
    t["W1"], t["W3"], t["W2"] = (w.unsqueeze(0).cuda() for w in (W1, W3, W2))
    x = t["x"].clone()
    x[:, 0] = 0
    t["x"] = x
    q = quantized(t)
    codes = host(q["W1"][0])[1:, 1:]
    assert np.all((codes & 0x78) == 0) and np.all((codes & 0x07) != 0)   # exponent field 0, nonzero
    out, logits = run_fp8_layer(cfg, t, q)
    assert float(dec(host(out)).__abs__().max()) > 1.0
    check_fp8_layer(cfg, t, q, out, logits)


def test_layer_fp8_is_deterministic():
    cfg = MoEConfig("det8", N=500, H=256, I=256, E=8, k=2)
    t = cuda_inputs(cfg, seed=9)
    q = quantized(t)
    a, _ = run_fp8_layer(cfg, t, q)
    b, _ = run_fp8_layer(cfg, t, q)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_layer_fp8_error_against_bf16_layer():
    """The measured cost of the experiment: the fp8 layer's distance from the bf16
    layer on the same inputs is of the e4m3 step's size (2^-4 relative per weight,
    averaged down over the sums), and the routing is identical (same logits)."""
    cfg = MoEConfig("err8", N=256, H=512, I=384, E=8, k=2)
    t = cuda_inputs(cfg, seed=3)
    q = quantized(t)
    out8, l8 = run_fp8_layer(cfg, t, q)
    logits = torch.empty_like(l8)
    out16 = moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, logits=logits)
    torch.cuda.synchronize()
    assert torch.equal(l8, logits)
    a, b = dec(host(out8)), dec(host(out16))
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-3 < rel < 5e-2, rel


def test_mixtral_decode_fp8_full_size_sampled():
    """The benchmark's fp8 line: full-size workload, a seeded token sample against
    the oracle fed the GPU's codes and scales."""
    cfg = CONFIGS["mixtral_8x22b_decode"]
    t = cuda_inputs(cfg, gen_device="cuda")
    q = quantized(t)
    for n in ("W1", "W3", "W2"):
        del t[n]
    torch.cuda.empty_cache()
    out, logits = run_fp8_layer(cfg, t, q)
    sample = np.sort(np.random.default_rng(1).choice(cfg.N, 4, replace=False))
    check_fp8_layer(cfg, t, q, out, logits, tokens=sample)

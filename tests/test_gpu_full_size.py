"""GPU parity at the full workload sizes (the shapes of the models' MoE layers).

For each workload: the whole layer runs once through moe_layer_forward_ex (the
benchmark's launch path); the expert choice for every token is checked
bit-exact against the oracle fed the GPU's fp32 logits, the full dispatch maps
bit-exact against the oracle's dispatch, and the outputs of a seeded sample of
tokens (tokens are independent once routed) against the oracle within
|d| <= 2e-2*|ref| + 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from expert_ffn_layer_moe_b200 import moe
from expert_ffn_layer_moe_b200.inputs import CONFIGS, QWEN3_30B_TOKEN_SWEEP
from tests._bf16 import dec, to_u16

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2e-2, 2e-3

WORKLOADS = ([CONFIGS["deepseek_v2"], CONFIGS["qwen3_235b_a22b_skew"]] +
             [CONFIGS["qwen3_30b_a3b"].with_tokens(n) for n in QWEN3_30B_TOKEN_SWEEP])


def _host(t):
    if t is None:
        return None
    t = t.detach().cpu()
    return to_u16(t) if t.dtype == torch.bfloat16 else t.numpy()


@pytest.mark.parametrize("cfg", WORKLOADS, ids=lambda c: c.name)
def test_full_size_layer_sampled(cfg):
    from expert_ffn_layer_moe_b200.inputs import make_inputs
    t = make_inputs(cfg, seed=0, device="cuda")
    logits = torch.empty((cfg.N, cfg.E), dtype=torch.float32, device="cuda")
    out = moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, bias=t["bias"],
                                   Ws1=t["Ws1"], Ws3=t["Ws3"], Ws2=t["Ws2"], logits=logits)
    assert moe.moe_get_device_error() == 0

    # routing and dispatch of every token, bit-exact, on the logits the router produced
    rlogits = torch.empty_like(logits)
    idx, w, _ = moe.moe_route(t["x"], t["W_gate"], cfg.k, bias=t["bias"], logits=rlogits)
    p = moe.moe_permute(t["x"], idx, cfg.E)
    torch.cuda.synchronize()
    assert torch.equal(rlogits, logits)        # the layer's router runs the same path
    l32 = _host(logits)
    ref_idx, ref_w = oracle.topk(l32, cfg.k)
    assert np.array_equal(_host(idx), ref_idx)
    assert np.allclose(_host(w), ref_w, rtol=4 * 2.0 ** -23, atol=1e-7)
    counts, offsets, r2t, t2r = oracle.dispatch(ref_idx, cfg.E)
    assert np.array_equal(_host(p["counts"]), counts)
    assert np.array_equal(_host(p["offsets"]), offsets)
    assert np.array_equal(_host(p["row_to_token"]), r2t)
    assert np.array_equal(_host(p["token_to_row"]), t2r)

    # outputs of a seeded token sample
    sample = np.sort(np.random.default_rng(1).choice(cfg.N, min(cfg.N, 4), replace=False))
    ref = oracle.layer_given_logits(_host(t["x"])[sample], l32[sample], _host(t["W1"]), _host(t["W3"]),
                                    _host(t["W2"]), cfg.k, Ws1=_host(t["Ws1"]), Ws3=_host(t["Ws3"]),
                                    Ws2=_host(t["Ws2"]))
    g, wnt = dec(_host(out)[sample]), dec(ref)
    bad = np.abs(g - wnt) > RTOL * np.abs(wnt) + ATOL
    assert not bad.any(), f"{bad.sum()} of {bad.size} sampled outputs outside tolerance"

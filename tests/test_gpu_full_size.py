"""GPU parity at the full workload sizes (the shapes of the models' MoE layers).

For each workload: the whole layer runs once through moe_layer_forward_ex (the
benchmark's launch path); the expert choice for every token is checked
bit-exact against the oracle fed the GPU's fp32 logits, the full dispatch maps
bit-exact against the oracle's dispatch, and the outputs of at least 64 tokens
(tokens are independent once routed) against the oracle within
|d| <= 2e-2*|ref| + 2e-3.  The tokens are chosen, from the oracle's own
dispatch, so that the checked rows include the two hottest experts' first and
last rows and rows at every 16-, 32- and 64-row boundary near the ends of those
groups (the last ragged token tile, both halves of a CTA pair's tile, the
32-row epilogue chunks), the first and last rows of the emptiest non-empty expert, and a
seeded random fill; every checked row passes through every K slice and feature
tile of both GEMMs.  The oracle runs its threaded build (same arithmetic per row)
on all the host's cores.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from expert_ffn_layer_moe_b200 import moe
from expert_ffn_layer_moe_b200.inputs import CONFIGS, QWEN3_30B_TOKEN_SWEEP
from tests._bf16 import dec, to_u16

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2e-2, 2e-3
MIN_TOKENS = 64

WORKLOADS = ([CONFIGS["deepseek_v2"], CONFIGS["qwen3_235b_a22b_skew"]] +
             ([CONFIGS["qwen3_235b_a22b_skew4x"]] if "qwen3_235b_a22b_skew4x" in CONFIGS else []) +
             [CONFIGS["qwen3_30b_a3b"].with_tokens(n) for n in QWEN3_30B_TOKEN_SWEEP])


def _host(t):
    if t is None:
        return None
    t = t.detach().cpu()
    return to_u16(t) if t.dtype == torch.bfloat16 else t.numpy()


def pick_tokens(counts, offsets, row_to_token, N, seed=1):
    """Tokens whose rows sit at the places a tiled kernel gets wrong first (see the
    module docstring), topped up with seeded random tokens to MIN_TOKENS."""
    rows = set()
    order = np.argsort(-counts, kind="stable")
    for e in order[:2]:
        c = int(counts[e])
        if c == 0:
            continue
        lo = int(offsets[e])
        for r in (0, 1, 15, 16, 31, 32, 63, 64, 127, 128, 255, 256):
            if r < c:
                rows.add(lo + r)
        for back in (1, 2, 16, 17, 32, 33, 64, 65):
            if c - back >= 0:
                rows.add(lo + c - back)
        last_tile = (c - 1) // 256 * 256            # the last tile of the widest token tile
        rows.update(lo + r for r in range(last_tile, min(c, last_tile + 3)))
    nonzero = np.flatnonzero(counts)
    emptiest = nonzero[np.argmin(counts[nonzero])]
    lo, hi = int(offsets[emptiest]), int(offsets[emptiest + 1])
    rows.update(range(lo, min(hi, lo + 8)))      # its first and last rows (all of them when few)
    rows.update(range(max(lo, hi - 8), hi))
    toks = set(int(row_to_token[r]) for r in rows)
    rng = np.random.default_rng(seed)
    for t in rng.permutation(N):
        if len(toks) >= min(N, MIN_TOKENS):
            break
        toks.add(int(t))
    return np.array(sorted(toks))


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
    if cfg.name.startswith("qwen3_235b_a22b_skew4x"):
        from expert_ffn_layer_moe_b200.inputs import SKEW4X_LOAD_BAND
        ratio = counts.max() / (counts.sum() / cfg.E)
        assert SKEW4X_LOAD_BAND[0] <= ratio <= SKEW4X_LOAD_BAND[1], ratio

    # outputs of the chosen tokens
    sample = pick_tokens(counts, offsets, r2t, cfg.N)
    assert len(sample) >= min(cfg.N, MIN_TOKENS)
    oracle.set_threads(os.cpu_count() or 1)
    try:
        ref = oracle.layer_given_logits(_host(t["x"])[sample], l32[sample], _host(t["W1"]), _host(t["W3"]),
                                        _host(t["W2"]), cfg.k, Ws1=_host(t["Ws1"]), Ws3=_host(t["Ws3"]),
                                        Ws2=_host(t["Ws2"]))
    finally:
        oracle.set_threads(1)
    g, wnt = dec(_host(out)[sample]), dec(ref)
    bad = np.abs(g - wnt) > RTOL * np.abs(wnt) + ATOL
    assert not bad.any(), f"{bad.sum()} of {bad.size} checked outputs outside tolerance"

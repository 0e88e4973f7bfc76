"""Linear time model of the expert FFN, fitted to these kernels.

FinDEP review ("FinDEP: Efficient MoE Inference with Fine-Grained Scheduling of
Disaggregated Expert Parallelism"), section "核心公式": the MoE layer's time is
modelled as linear in the tokens each expert receives, t_e(m_e) = a_e + b_e * m_e,
with coefficients collected offline by microbenchmarks and a fit quality (R^2)
reported for its GEMM model.  This module measures the two grouped GEMMs of this
library (W1/W3 with SwiGLU, then W2) over a sweep of batch sizes at one layer shape,
takes m_e = N*k/E (mean rows per expert), and fits t = a + b*m by least squares -- over
every point, and over the points where all experts receive rows (the model's premise).
Because small batches leave experts untouched (their weights are then not streamed), it
also fits t = c0 + c1*touched + c2*m_e.

    python -m expert_ffn_layer_moe_b200.perfmodel [--config qwen3_30b_a3b] [--tokens 1,16,...]

prints one JSON object: the per-N measurements and the fits with their R^2.
"""
from __future__ import annotations

import argparse
import json
import statistics
from typing import Dict, List, Sequence, Tuple

import numpy as np


def fit_linear(m: Sequence[float], t: Sequence[float]) -> Tuple[float, float, float]:
    """Least-squares fit t ~ a + b*m; returns (a, b, R^2).

    R^2 = 1 - SS_res / SS_tot (1.0 when all t are equal and fitted exactly)."""
    x = np.asarray(m, dtype=np.float64)
    y = np.asarray(t, dtype=np.float64)
    if x.size < 2:
        raise ValueError("need at least two points")
    A = np.stack([np.ones_like(x), x], axis=1)
    (a, b), *_ = np.linalg.lstsq(A, y, rcond=None)
    resid = y - (a + b * x)
    ss_res = float(resid @ resid)
    ss_tot = float(((y - y.mean()) ** 2).sum())
    r2 = 1.0 - ss_res / ss_tot if ss_tot > 0 else 1.0
    return float(a), float(b), float(r2)


def fit_multilinear(cols: Sequence[Sequence[float]], t: Sequence[float]) -> Tuple[List[float], float]:
    """Least-squares fit t ~ c0 + c1*cols[0] + c2*cols[1] + ...; returns (coefficients, R^2)."""
    y = np.asarray(t, dtype=np.float64)
    A = np.stack([np.ones_like(y)] + [np.asarray(c, dtype=np.float64) for c in cols], axis=1)
    coef, *_ = np.linalg.lstsq(A, y, rcond=None)
    resid = y - A @ coef
    ss_tot = float(((y - y.mean()) ** 2).sum())
    return [float(v) for v in coef], (1.0 - float(resid @ resid) / ss_tot if ss_tot > 0 else 1.0)


def measure(config: str, tokens: Sequence[int], steps: int = 10, warmup: int = 3) -> List[Dict]:
    """CUDA-event times of the layer and of its two grouped GEMMs at each N (the grouped
    GEMMs at every N: the decode kernels, which the layer takes for a few tokens, are
    another model and stay off here)."""
    from expert_ffn_layer_moe_b200 import moe

    prev = moe.moe_set_decode_gemv(moe.MOE_DECODE_OFF)
    try:
        return _measure(config, tokens, steps, warmup)
    finally:
        moe.moe_set_decode_gemv(prev)


def _measure(config: str, tokens: Sequence[int], steps: int, warmup: int) -> List[Dict]:
    import torch

    from expert_ffn_layer_moe_b200 import moe
    from expert_ffn_layer_moe_b200.inputs import CONFIGS, make_inputs

    base = CONFIGS[config]
    out = []
    weights = make_inputs(base.with_tokens(1), seed=0, device="cuda")
    for n in tokens:
        cfg = base.with_tokens(n)
        x = make_inputs(cfg, seed=0, device="cuda", weights=False)["x"]
        t = dict(weights, x=x)
        ws = torch.empty(moe.moe_workspace_bytes(cfg.N, cfg.H, cfg.I, cfg.E, cfg.k, cfg.Is), dtype=torch.uint8,
                         device="cuda")
        o = torch.empty((cfg.N, cfg.H), dtype=torch.bfloat16, device="cuda")
        stream = torch.cuda.current_stream()

        def step(events=None):
            moe.moe_layer_forward_ex(t["x"], t["W_gate"], t["W1"], t["W3"], t["W2"], cfg.k, bias=t["bias"],
                                     Ws1=t["Ws1"], Ws3=t["Ws3"], Ws2=t["Ws2"], ws=ws, out=o, stream=stream,
                                     phase_events=events)

        for _ in range(warmup):
            step()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(moe.PHASES) + 1)] for _ in range(steps)]
        for e in evs:
            for ev in e:
                ev.record(stream)
        torch.cuda.synchronize()
        for i in range(steps):
            step(evs[i])
        torch.cuda.synchronize()
        if moe.moe_get_device_error(stream) != 0:
            raise RuntimeError("device error during the sweep")
        ph = {p: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, p in enumerate(moe.PHASES)}
        counts = moe.moe_permute(t["x"], moe.moe_route(t["x"], t["W_gate"], cfg.k, bias=t["bias"])[0],
                                 cfg.E)["counts"]
        out.append({"N": n, "m_e": cfg.R / cfg.E, "touched": int((counts > 0).sum().item()),
                    "gemm_ms": ph["gemm13"] + ph["gemm2"], "layer_ms": sum(ph.values()), "phase_ms": ph})
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="qwen3_30b_a3b")
    ap.add_argument("--tokens", default="1,16,64,128,256,512,1024,2048,4096,8192")
    ap.add_argument("--steps", type=int, default=10)
    args = ap.parse_args()
    tokens = [int(v) for v in args.tokens.split(",")]
    rows = measure(args.config, tokens, steps=args.steps)
    a, b, r2 = fit_linear([r["m_e"] for r in rows], [r["gemm_ms"] for r in rows])
    la, lb, lr2 = fit_linear([r["m_e"] for r in rows], [r["layer_ms"] for r in rows])
    full = [r for r in rows if r["touched"] == max(q["touched"] for q in rows)]
    fa, fb, fr2 = fit_linear([r["m_e"] for r in full], [r["gemm_ms"] for r in full]) if len(full) >= 2 else (0, 0, 0)
    coef, mr2 = fit_multilinear([[r["touched"] for r in rows], [r["m_e"] for r in rows]],
                                [r["gemm_ms"] for r in rows])
    print(json.dumps({"config": args.config, "points": rows,
                      "expert_ffn_fit": {"alpha_ms": a, "beta_ms_per_row": b, "r2": r2},
                      "expert_ffn_fit_all_experts_active": {"alpha_ms": fa, "beta_ms_per_row": fb, "r2": fr2,
                                                            "points": len(full)},
                      "expert_ffn_fit_touched_and_rows": {"const_ms": coef[0], "ms_per_touched_expert": coef[1],
                                                          "ms_per_row_per_expert": coef[2], "r2": mr2},
                      "layer_fit": {"alpha_ms": la, "beta_ms_per_row": lb, "r2": lr2}}))


if __name__ == "__main__":
    main()

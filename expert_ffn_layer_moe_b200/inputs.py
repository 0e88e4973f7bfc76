"""Seeded synthetic inputs for the MoE expert layer.

This module is shared by the CUDA path's tests and benchmark and by the oracle's
tests.  It holds workload shapes and random-number recipes only; none of the
layer's arithmetic (routing, dispatch, the expert FFN, combine) lives here.

Recipe (every tensor):
  * generator: ``torch.Generator(device).manual_seed(seed * 1000 + tensor_id)``,
    tensor ids x=1, W_gate=2, W1=3, W3=4, W2=5, Ws1=6, Ws3=7, Ws2=8, expert-rank
    permutation=9;
  * values: ``randn`` in fp32, multiplied by the stated standard deviation, then
    rounded to bf16 by round-to-nearest-even (``Tensor.to(torch.bfloat16)``);
    W_gate and the optional bias stay fp32;
  * x ~ N(0, 1); W_gate ~ N(0, 1/H); W1, W3, Ws1, Ws3 ~ N(0, 1/H);
    W2, Ws2 ~ N(0, 1/I) (std = 1/sqrt(fan_in));
  * expert weight stacks are drawn one expert at a time, in expert order, from
    the tensor's one generator (so a 7 GB stack never needs a 14 GB fp32 temp);
  * the skewed workload adds a router bias b_e = 2 * ln(1 / rank_e ** 1.2) with
    rank_e = 1 + randperm(E)[e] (a Zipf s=1.2 profile over a seeded expert
    order), multiplied by ``bias_scale``: 1 for the bias as written (the hottest
    expert then takes every token), SKEW4X_BIAS_SCALE for the reading in which the
    hottest expert takes 4x the mean load (the scale was bisected on the seeded
    inputs, made on a CUDA device, with the oracle's routing, until max/mean load
    lay in SKEW4X_LOAD_BAND; tests/golden/calibrate_skew4x.py).

The same (config, seed, device) always gives the same bits; CPU and CUDA
generators give different streams, so a test that needs the oracle to see the
GPU's inputs copies the tensors, never regenerates them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

TENSOR_IDS = {"x": 1, "W_gate": 2, "W1": 3, "W3": 4, "W2": 5,
              "Ws1": 6, "Ws3": 7, "Ws2": 8, "perm": 9}


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    """Shape of one MoE layer workload.

    N tokens of width H; E routed experts, each a SwiGLU FFN with
    intermediate width I; each token picks k experts; Is > 0 adds always-on
    shared experts (their intermediate widths concatenated into one of Is).
    """
    name: str
    N: int
    H: int
    I: int
    E: int
    k: int
    Is: int = 0
    skew: bool = False
    bias_scale: float = 1.0

    @property
    def R(self) -> int:
        """Assignment rows: every token contributes k (token, expert) pairs."""
        return self.N * self.k

    def with_tokens(self, N: int) -> "MoEConfig":
        return dataclasses.replace(self, name=f"{self.name.split('@')[0]}@N={N}", N=N)


# The skewed workload's bias scale at which the hottest expert's load is about 4x the
# mean (measured 3.9512 with every one of the 128 experts touched).
SKEW4X_BIAS_SCALE = 0.0938
SKEW4X_LOAD_BAND = (3.9, 4.1)

# Workload shapes named after the models whose MoE layers they mimic.
CONFIGS: Dict[str, MoEConfig] = {
    "tiny": MoEConfig("tiny", N=64, H=256, I=512, E=8, k=2),
    "mixtral_8x22b_decode": MoEConfig("mixtral_8x22b_decode", N=156, H=6144, I=16384, E=8, k=2),
    "deepseek_v2": MoEConfig("deepseek_v2", N=4096, H=5120, I=1536, E=160, k=6, Is=3072),
    "qwen3_30b_a3b": MoEConfig("qwen3_30b_a3b", N=1024, H=2048, I=768, E=128, k=8),
    "qwen3_235b_a22b_skew": MoEConfig("qwen3_235b_a22b_skew", N=16384, H=4096, I=1536,
                                      E=128, k=8, skew=True),
    "qwen3_235b_a22b_skew4x": MoEConfig("qwen3_235b_a22b_skew4x", N=16384, H=4096, I=1536,
                                        E=128, k=8, skew=True, bias_scale=SKEW4X_BIAS_SCALE),
}
QWEN3_30B_TOKEN_SWEEP = (1, 16, 128, 1024, 8192)


def _gen(device: torch.device, seed: int, name: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + TENSOR_IDS[name])
    return g


def _randn_bf16(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def _expert_stack(E: int, rows: int, cols: int, std: float, g: torch.Generator, device) -> torch.Tensor:
    out = torch.empty((E, rows, cols), dtype=torch.bfloat16, device=device)
    for e in range(E):
        out[e] = _randn_bf16((rows, cols), std, g, device)
    return out


def skew_bias(E: int, seed: int = 0, scale: float = 1.0, device="cpu") -> torch.Tensor:
    """Per-expert router bias b_e = 2*ln(rank_e**-1.2), times ``scale`` (fp32)."""
    g = _gen(torch.device("cpu"), seed, "perm")
    rank = torch.randperm(E, generator=g).to(torch.float64) + 1.0
    b = 2.0 * torch.log(1.0 / rank.pow(1.2)) * scale
    return b.to(torch.float32).to(device)


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu",
                weights: bool = True) -> Dict[str, Optional[torch.Tensor]]:
    """All inputs of one layer call: x, W_gate, bias, W1, W3, W2, Ws1, Ws3, Ws2.

    Layouts: x [N,H] bf16; W_gate [H,E] fp32; bias [E] fp32 or None;
    W1, W3 [E,I,H] bf16; W2 [E,H,I] bf16; Ws1, Ws3 [Is,H] bf16 and
    Ws2 [H,Is] bf16 or None when Is == 0.  ``weights=False`` skips the expert
    stacks (router-only uses).
    """
    device = torch.device(device)
    N, H, I, E, Is = cfg.N, cfg.H, cfg.I, cfg.E, cfg.Is
    out: Dict[str, Optional[torch.Tensor]] = {}
    out["x"] = _randn_bf16((N, H), 1.0, _gen(device, seed, "x"), device)
    out["W_gate"] = torch.randn((H, E), generator=_gen(device, seed, "W_gate"),
                                device=device, dtype=torch.float32) * (1.0 / math.sqrt(H))
    out["bias"] = skew_bias(E, seed, cfg.bias_scale, device) if cfg.skew else None
    if weights:
        out["W1"] = _expert_stack(E, I, H, 1.0 / math.sqrt(H), _gen(device, seed, "W1"), device)
        out["W3"] = _expert_stack(E, I, H, 1.0 / math.sqrt(H), _gen(device, seed, "W3"), device)
        out["W2"] = _expert_stack(E, H, I, 1.0 / math.sqrt(I), _gen(device, seed, "W2"), device)
        if Is > 0:
            out["Ws1"] = _randn_bf16((Is, H), 1.0 / math.sqrt(H), _gen(device, seed, "Ws1"), device)
            out["Ws3"] = _randn_bf16((Is, H), 1.0 / math.sqrt(H), _gen(device, seed, "Ws3"), device)
            out["Ws2"] = _randn_bf16((H, Is), 1.0 / math.sqrt(Is), _gen(device, seed, "Ws2"), device)
        else:
            out["Ws1"] = out["Ws3"] = out["Ws2"] = None
    return out


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """The uint16 storage of a bf16 tensor (same bytes, viewed as int16)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16)

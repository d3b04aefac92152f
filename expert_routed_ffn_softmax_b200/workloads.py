"""Seeded synthetic workloads for the routed MoE FFN layer.

This module only draws random numbers and names the layer shapes; it holds none
of the layer's arithmetic, so the CUDA path, the CPU oracle, the tests and the
benchmark can all take their inputs from here without sharing any computation.

Shapes follow the Gemma-4-26B-A4B MoE block as the pages describe it: hidden 2816,
128 experts with top-8 routing, expert intermediate 704, bf16 (cann-recipes-infer
"Gemma-4-26B-A4B 模型优化报告" §1 模型概况; Gemma-4-26B-A4B-NVFP4 Ascend verification
report §2.1 模型架构参数).

Recipe (every config):
  * weights come from ``numpy.random.default_rng(seed)`` drawn in this order:
    W_router [H,E], W_gate [E,H,I], W_up [E,H,I], W_down [E,I,H]; each is drawn
    as float32 N(0,1), scaled by 0.02 in float32 and rounded to bf16 (RNE);
  * x [T,H] comes from a second ``default_rng(seed)`` stream: float32 N(0,1)
    rounded to bf16, so configs that share (H,E,I) share one weight set;
  * the skewed config adds a per-expert router bias b_e = 2*ln(1/(e+1)),
    evaluated in float64 and rounded once to float32.
"""
from __future__ import annotations

import dataclasses
import functools
import math

import numpy as np
import torch

WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int          # tokens
    H: int          # hidden size
    E: int          # experts
    k: int          # experts per token
    I: int          # expert intermediate size
    skew_bias: bool = False

    @property
    def pairs(self) -> int:
        return self.T * self.k


def _gemma(name: str, T: int, skew: bool = False) -> MoEConfig:
    return MoEConfig(name, T, 2816, 128, 8, 704, skew)


CONFIGS: dict[str, MoEConfig] = {
    "tiny": MoEConfig("tiny", 16, 256, 8, 2, 128),
    "decode": _gemma("decode", 8),
    "prefill": _gemma("prefill", 2048),
    "skewed": _gemma("skewed", 16384, skew=True),
}
SWEEP_T = (1, 8, 64, 512, 4096, 32768)
for _t in SWEEP_T:
    CONFIGS[f"sweep_T{_t}"] = _gemma(f"sweep_T{_t}", _t)


def bf16_from_f32(a: np.ndarray) -> torch.Tensor:
    """float32 numpy array -> bf16 torch tensor, round-to-nearest-even."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def skew_bias(E: int) -> torch.Tensor:
    """b_e = 2*ln(1/(e+1)) in float64, rounded once to float32."""
    b = np.array([2.0 * math.log(1.0 / (e + 1)) for e in range(E)], dtype=np.float64)
    return torch.from_numpy(b.astype(np.float32))


@functools.lru_cache(maxsize=2)
def _weights(H: int, E: int, I: int, seed: int) -> tuple[torch.Tensor, ...]:
    rng = np.random.default_rng(seed)
    std = np.float32(WEIGHT_STD)

    def draw(shape):
        a = rng.standard_normal(size=shape, dtype=np.float32)
        a *= std
        return bf16_from_f32(a)

    w_router = draw((H, E))
    w_gate = draw((E, H, I))
    w_up = draw((E, H, I))
    w_down = draw((E, I, H))
    return w_router, w_gate, w_up, w_down


def make_weights(cfg: MoEConfig, seed: int = 0) -> dict:
    """Weights of one MoE layer as contiguous CPU tensors (bf16; bias float32 or None)."""
    w_router, w_gate, w_up, w_down = _weights(cfg.H, cfg.E, cfg.I, seed)
    return {
        "w_router": w_router,
        "w_gate": w_gate,
        "w_up": w_up,
        "w_down": w_down,
        "bias": skew_bias(cfg.E) if cfg.skew_bias else None,
    }


DENSE_I = 2112   # intermediate of the dense MLP that runs beside the MoE in every layer


def make_dense_weights(H: int, I: int, seed: int = 0) -> dict:
    """Weights of the dense GEGLU MLP beside the MoE: w_gate, w_up [H,I], w_down [I,H], bf16,
    N(0, 0.02^2) from their own stream (seed + 1000), so the MoE weights do not change."""
    rng = np.random.default_rng(seed + 1000)
    std = np.float32(WEIGHT_STD)

    def draw(shape):
        a = rng.standard_normal(size=shape, dtype=np.float32)
        a *= std
        return bf16_from_f32(a)

    w_gate = draw((H, I))
    w_up = draw((H, I))
    w_down = draw((I, H))
    return {"w_gate": w_gate, "w_up": w_up, "w_down": w_down}


def make_x(cfg: MoEConfig, seed: int = 0, T: int | None = None) -> torch.Tensor:
    """Token activations x [T,H] bf16 on the CPU."""
    T = cfg.T if T is None else T
    rng = np.random.default_rng(seed)
    return bf16_from_f32(rng.standard_normal(size=(T, cfg.H), dtype=np.float32))


def make_inputs(cfg: MoEConfig, seed: int = 0) -> dict:
    d = make_weights(cfg, seed)
    d["x"] = make_x(cfg, seed)
    return d


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw uint16 bit patterns of a contiguous bf16 CPU tensor (a view, no copy)."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)

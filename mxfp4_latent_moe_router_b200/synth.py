"""Seeded synthetic inputs for the latent-MoE decode block.

This module only draws random numbers and packs them into the canonical
storage layouts of ``include/moe.h``; it holds none of the block's arithmetic
(no dequantisation, no routing, no matmul).  Both the CUDA path and the CPU
oracle receive exactly the arrays built here.

Workloads (sizes and distributions of the five decode shapes the layer is
measured on; the pages fix only "small-batch decode, batch 1-64" and the
speculative-verify shape of 16 requests x 8 draft tokens):

* ``tiny``  B=1,   H=512,  L=256,  E=16,  k=2, I=128,  I_s=256, softmax top-2
* ``b1``    B=1,   H=7168, L=2048, E=384, k=8, I=2048, I_s=2048, sigmoid+bias top-8
* ``b8``    B=8,   same shapes, near-uniform routing
* ``b64``   B=64,  same shapes
* ``b128``  B=128 (16 requests x 8 draft positions), Zipf(1.1)-skewed routing
  imposed through the per-expert selection bias.

Distributions: x ~ N(0,1); every dense bf16 weight ~ N(0, 0.02); e2m1 codes
uniform over all 16 codes; e8m0 scale exponents uniform over an integer range
({-6..-3} for ``tiny``, {-8..-4} otherwise).  The selection bias is N(0, 0.01)
for the uniform-routing shapes and ``-beta*ln(rank)`` over a seeded
permutation for the Zipf shape.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1


@dataclasses.dataclass(frozen=True)
class Shape:
    name: str
    tokens: int            # B
    hidden: int            # H
    latent: int            # L
    num_experts: int       # E
    top_k: int             # k
    expert_inter: int      # I
    shared_inter: int      # I_s (0: no shared expert)
    score_fn: int          # SCORE_SOFTMAX / SCORE_SIGMOID
    renormalize: int = 1
    routed_scale: float = 1.0
    scale_exp_lo: int = -8  # e8m0 exponent range (inclusive)
    scale_exp_hi: int = -4
    routing: str = "uniform"  # "uniform" | "zipf"
    seed: int = 0


# Zipf exponent of the speculative-verify shape and the bias strength that
# produces it.  The bias slope was chosen by sweeping beta with the oracle's
# router on this workload (tests/golden/calibrate_zipf.py); the fitted
# log-log slope of the per-expert token histogram is recorded there.
ZIPF_S = 1.1
ZIPF_BETA = 0.13

SHAPES = {
    "tiny": Shape("tiny", 1, 512, 256, 16, 2, 128, 256, SCORE_SOFTMAX,
                  scale_exp_lo=-6, scale_exp_hi=-3, seed=1000),
    "b1": Shape("b1", 1, 7168, 2048, 384, 8, 2048, 2048, SCORE_SIGMOID, seed=1001),
    "b8": Shape("b8", 8, 7168, 2048, 384, 8, 2048, 2048, SCORE_SIGMOID, seed=1002),
    "b64": Shape("b64", 64, 7168, 2048, 384, 8, 2048, 2048, SCORE_SIGMOID, seed=1003),
    "b128": Shape("b128", 128, 7168, 2048, 384, 8, 2048, 2048, SCORE_SIGMOID,
                  routing="zipf", seed=1004),
}
SHAPE_ORDER = ["tiny", "b1", "b8", "b64", "b128"]


def custom_shape(name: str, tokens: int, hidden: int, latent: int, num_experts: int,
                 top_k: int, expert_inter: int, shared_inter: int, score_fn: int,
                 seed: int = 7, **kw) -> Shape:
    return Shape(name, tokens, hidden, latent, num_experts, top_k, expert_inter,
                 shared_inter, score_fn, seed=seed, **kw)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float array -> uint16 bf16 bit patterns (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def _codes(rng: np.random.Generator, rows: int, k: int, experts: int) -> np.ndarray:
    # two uniform 4-bit codes per byte: element 2t in the low nibble of byte t
    return rng.integers(0, 256, size=(experts, rows, k // 2), dtype=np.uint8)


def _scales(rng: np.random.Generator, rows: int, k: int, experts: int,
            lo: int, hi: int) -> np.ndarray:
    e = rng.integers(lo, hi + 1, size=(experts, rows, k // 32), dtype=np.int32)
    return (e + 127).astype(np.uint8)


def make_weights(shape: Shape, instance: int = 0) -> dict:
    """Canonical-layout weights (see ``include/moe.h``), as numpy arrays."""
    H, L, E, I, Is = shape.hidden, shape.latent, shape.num_experts, shape.expert_inter, shape.shared_inter
    rng = np.random.default_rng([shape.seed, 1, instance])
    w = {
        "router_w": _normal_bf16(rng, (H, E), 0.02),
        "w_in": _normal_bf16(rng, (H, L), 0.02),
        "w_out": _normal_bf16(rng, (L, H), 0.02),
        "gu_codes": _codes(rng, 2 * I, L, E),
        "gu_scales": _scales(rng, 2 * I, L, E, shape.scale_exp_lo, shape.scale_exp_hi),
        "dn_codes": _codes(rng, L, I, E),
        "dn_scales": _scales(rng, L, I, E, shape.scale_exp_lo, shape.scale_exp_hi),
    }
    if Is > 0:
        w["sh_gate"] = _normal_bf16(rng, (H, Is), 0.02)
        w["sh_up"] = _normal_bf16(rng, (H, Is), 0.02)
        w["sh_down"] = _normal_bf16(rng, (Is, H), 0.02)
    if shape.score_fn == SCORE_SIGMOID:
        if shape.routing == "zipf":
            rank = rng.permutation(E).astype(np.float64) + 1.0
            w["router_bias"] = (-ZIPF_BETA * np.log(rank)).astype(np.float32)
        else:
            w["router_bias"] = (rng.standard_normal(E) * 0.01).astype(np.float32)
    else:
        w["router_bias"] = None
    return w


def make_x(shape: Shape, tokens: int | None = None, step: int = 0) -> np.ndarray:
    """Token activations x[B, H] as bf16 bits, N(0,1)."""
    B = shape.tokens if tokens is None else tokens
    rng = np.random.default_rng([shape.seed, 2, step])
    return _normal_bf16(rng, (B, shape.hidden), 1.0)


def weight_bytes(shape: Shape) -> dict:
    """Storage bytes of each weight group (algorithmic traffic per use)."""
    H, L, E, I, Is = shape.hidden, shape.latent, shape.num_experts, shape.expert_inter, shape.shared_inter
    dense = 2 * (H * E + H * L + L * H + 3 * H * Is)
    per_expert = (2 * I * L + L * I) // 2 + (2 * I * L + L * I) // 32
    return {"dense": dense, "per_expert": per_expert, "bias": 4 * E}


def expected_distinct(shape: Shape) -> float:
    E, k, B = shape.num_experts, shape.top_k, shape.tokens
    return E * (1.0 - (1.0 - k / E) ** B)


__all__ = ["Shape", "SHAPES", "SHAPE_ORDER", "make_weights", "make_x", "weight_bytes",
           "custom_shape", "to_bf16_bits", "SCORE_SOFTMAX", "SCORE_SIGMOID", "expected_distinct",
           "ZIPF_S", "ZIPF_BETA"]

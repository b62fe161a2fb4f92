"""Seeded synthetic inputs for the quantized MoE expert matmul.

This module only draws random numbers and rounds them to bf16 storage; it holds
none of the method's arithmetic (no quantization, routing, matmul or SwiGLU).
Both the CUDA path and the CPU oracle consume what it returns.

Every tensor is drawn from its own numpy ``SeedSequence`` keyed by
``(seed, tag, index)`` so that one expert's weights can be regenerated without
drawing the others.  bf16 tensors are returned as ``uint16`` bit patterns
(round-to-nearest-even from the float32 draw).

Workload shapes (the pages' workloads: GPT-OSS-20B, DeepSeek-V2-Lite, a
Switch-style ternary model, an lm_head-sized linear; their weights are not
needed, these synthetic tensors stand in for them):

* ``tiny``     H=512, I=1024, E=8, top-2, FC1 INT2 / FC2 INT4, block 64, T=1.
* ``linear``   K=5120 -> N=17408 (or 248320), group 128, INT2 or INT4.
* ``v2lite``   H=2048, I=1408, E=64 top-6 + 2 shared experts, INT4/INT4,
               +2.0 on 4 "hot" experts' logits.
* ``ternary``  d=2048, d_ff=6144, E=128, top-1, ternary FC1 and FC2.
* ``prefill``  T=4096, H=2048, I=768, E=128 top-8, FC1 INT2 / FC2 INT4,
               expert biases N(0, 0.01), Zipf(1.1)-skewed router offsets.
"""
from __future__ import annotations

import dataclasses
import numpy as np

TAG_FC1, TAG_FC2, TAG_B1, TAG_B2, TAG_X, TAG_LOGITS, TAG_HOT, TAG_ZIPF, TAG_LINEAR, TAG_SIGNS = range(10)


def f32_to_bf16_bits(a) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, tag: int, index: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(tag), int(index)]))


def normal_bf16(seed: int, tag: int, index: int, shape, std: float) -> np.ndarray:
    g = _rng(seed, tag, index)
    return f32_to_bf16_bits(g.standard_normal(shape, dtype=np.float32) * np.float32(std))


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    H: int
    I: int
    E: int
    k: int
    n_shared: int
    fc1_fmt: str          # "int2" | "int4" | "ternary"
    fc2_fmt: str
    block: int = 64
    bias: bool = False
    hot_experts: int = 0  # number of experts whose logits get +hot_boost
    hot_boost: float = 0.0
    zipf_s: float = 0.0   # Zipf exponent for the per-expert logit offset (0 = none)
    w_std: float = 0.02
    b_std: float = 0.01

    @property
    def n_experts_total(self) -> int:
        return self.E + self.n_shared


TINY = MoEConfig("tiny", H=512, I=1024, E=8, k=2, n_shared=0, fc1_fmt="int2", fc2_fmt="int4")
V2LITE = MoEConfig("v2lite", H=2048, I=1408, E=64, k=6, n_shared=2, fc1_fmt="int4",
                   fc2_fmt="int4", hot_experts=4, hot_boost=2.0)
TERNARY = MoEConfig("ternary", H=2048, I=6144, E=128, k=1, n_shared=0, fc1_fmt="ternary",
                    fc2_fmt="ternary")
PREFILL = MoEConfig("prefill", H=2048, I=768, E=128, k=8, n_shared=0, fc1_fmt="int2",
                    fc2_fmt="int4", bias=True, zipf_s=1.1)
CONFIGS = {c.name: c for c in (TINY, V2LITE, TERNARY, PREFILL)}


def expert_fc1(cfg: MoEConfig, seed: int, e: int) -> np.ndarray:
    """FC1 of expert e (routed 0..E-1, shared E..E+n_shared-1): bf16 bits [2I, H],
    gate and up rows interleaved (row 2j = gate j, row 2j+1 = up j)."""
    return normal_bf16(seed, TAG_FC1, e, (2 * cfg.I, cfg.H), cfg.w_std)


def expert_fc2(cfg: MoEConfig, seed: int, e: int) -> np.ndarray:
    """FC2 (down) of expert e: bf16 bits [H, I]."""
    return normal_bf16(seed, TAG_FC2, e, (cfg.H, cfg.I), cfg.w_std)


def expert_b1(cfg: MoEConfig, seed: int, e: int) -> np.ndarray:
    return normal_bf16(seed, TAG_B1, e, (2 * cfg.I,), cfg.b_std)


def expert_b2(cfg: MoEConfig, seed: int, e: int) -> np.ndarray:
    return normal_bf16(seed, TAG_B2, e, (cfg.H,), cfg.b_std)


def tokens(cfg_H: int, seed: int, T: int, index: int = 0) -> np.ndarray:
    """x: bf16 bits [T, H], N(0, 1)."""
    return normal_bf16(seed, TAG_X, index, (T, cfg_H), 1.0)


def router_logits(cfg: MoEConfig, seed: int, T: int, index: int = 0) -> np.ndarray:
    """fp32 [T, E] router logits N(0,1), plus the workload's structure:

    * hot experts: +hot_boost on the first ``hot_experts`` entries of a seeded
      permutation of the experts, so several tokens share an expert;
    * Zipf skew: offset_e = -s * ln(rank_e) with rank_e in 1..E from a seeded
      permutation, i.e. a softmax prior proportional to rank^-s.
    """
    g = _rng(seed, TAG_LOGITS, index)
    lg = g.standard_normal((T, cfg.E), dtype=np.float32)
    if cfg.hot_experts:
        hot = _rng(seed, TAG_HOT).permutation(cfg.E)[: cfg.hot_experts]
        lg[:, hot] += np.float32(cfg.hot_boost)
    if cfg.zipf_s:
        rank = _rng(seed, TAG_ZIPF).permutation(cfg.E) + 1
        lg += (-cfg.zipf_s * np.log(rank.astype(np.float64))).astype(np.float32)[None, :]
    return lg


def shared_logit_tokens(cfg: MoEConfig, seed: int, M: int) -> np.ndarray:
    """M tokens that all carry the same router logits (row 0 of router_logits),
    so every selected expert receives exactly M tokens: the tokens-per-expert
    axis of the decode sweep."""
    row = router_logits(cfg, seed, 1)
    return np.repeat(row, M, axis=0)


def linear_weight(seed: int, N: int, K: int, std: float = 0.02, index: int = 0) -> np.ndarray:
    """Single quantized linear: bf16 bits [N, K]."""
    return normal_bf16(seed, TAG_LINEAR, index, (N, K), std)


def rht_signs(seed: int, H: int) -> np.ndarray:
    """The random signs d [H] (float32, +1 or -1) of the channel layer's
    randomized Hadamard rotation: a draw the method makes once at load time."""
    return np.where(_rng(seed, TAG_SIGNS).random(H) < 0.5, -1.0, 1.0).astype(np.float32)

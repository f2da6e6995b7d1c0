"""Seeded synthetic inputs for the NVFP4 W4A16 MoE FFN layer.

This module draws random numbers and packs them into the canonical byte
layout that both the CUDA path and the CPU oracle consume. It holds none of
the layer's arithmetic: no decoding of E2M1 / E4M3, no routing, no matmul.
The only rounding it does is turning freshly drawn floats into storage types
(float32 -> bfloat16 and float32 -> float8_e4m3fn through torch's casts), which
is how the input bytes are made, not how they are consumed.

Canonical layout (all row-major, little-endian):

  router_w     uint16 (bf16 bits) [E][H]
  router_bias  float32 [E] or None
  gate_codes   uint8 [E][I][H/2]   element 2c in the low nibble of byte c
  up_codes     uint8 [E][I][H/2]
  gate_scales  uint8 (e4m3 bits) [E][I][H/16]   one scale per 16 consecutive K
  up_scales    uint8 [E][I][H/16]
  gate_global, up_global  float32 [E]   per-tensor multiplier
  down_codes   uint8 [E][H][I/2]
  down_scales  uint8 [E][H][I/16]
  down_global  float32 [E]
  x            uint16 (bf16 bits) [T][H]

Workload recipe (sizes and distributions of the five layer shapes):

  * NVFP4 codes: every nibble uniform over the 16 E2M1 codes, i.e. uniform
    random bytes (both +0 and -0 occur).
  * Block scales: u ~ U[-4, 2], scale = float8_e4m3fn(2**u) (round to nearest
    even), so scale bytes fall in 0x18..0x48.
  * Per-tensor scale: 0.05 for the tiny layer, 0.02 otherwise, one per
    (expert, projection).
  * Router weights: N(0, 0.02) for the tiny layer, N(0, 1) otherwise; x: N(0, 1).
  * Zipf routing (batched decode): an fp32 router bias makes expert load follow
    Zipf(s) over the experts: p_r ~ r^-s over ranks r = 1..E given to the
    experts by a seeded permutation; bias_e = beta * ln p_r(e) with
    beta = sigma_l * sqrt(6) / pi, sigma_l = router_std * x_std * sqrt(H) the
    analytic std of the unbiased logits (the Gumbel scale that turns the
    bias into top-1 Zipf load).
  * Shared expert (optional): one SwiGLU FFN of width Is = m * I in the same
    formats and distributions as a routed expert (codes uniform, scales
    2**U[-4, 2], per-tensor scale as the routed experts').
  * Residual: N(0, 1) bf16 [T][H]. RMS-norm weight gamma: U[0.5, 1.5] bf16 [H].

Shared-expert layout (canonical, row-major): shared_gate_codes / shared_up_codes
uint8 [Is][H/2], shared_gate_scales / shared_up_scales [Is][H/16],
shared_down_codes [H][Is/2], shared_down_scales [H][Is/16], and the three
per-tensor multipliers as fp32 arrays of one element.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    H: int
    I: int
    E: int
    k: int
    T: tuple
    seeds: tuple
    global_scale: float
    router_std: float
    x_std: float = 1.0
    zipf_s: Optional[float] = None


# The five workload shapes. Sizes follow the layer descriptions of the
# spec workload list; each one is a seeded synthetic layer.
SHAPES: Dict[int, LayerShape] = {
    0: LayerShape("tiny", H=512, I=1024, E=8, k=2, T=(4,), seeds=(0,),
                  global_scale=0.05, router_std=0.02),
    1: LayerShape("decode", H=2048, I=768, E=128, k=8, T=(1, 8), seeds=(1, 2, 3),
                  global_scale=0.02, router_std=1.0),
    2: LayerShape("batched_decode_zipf", H=2048, I=768, E=128, k=8, T=(256,), seeds=(4,),
                  global_scale=0.02, router_std=1.0, zipf_s=1.1),
    3: LayerShape("prefill", H=4096, I=1536, E=128, k=8, T=(8192,), seeds=(5,),
                  global_scale=0.02, router_std=1.0),
    4: LayerShape("large_sweep", H=4096, I=2688, E=256, k=8, T=(1, 32, 256, 2048, 7234),
                  seeds=(6, 7, 8, 9, 10), global_scale=0.02, router_std=1.0),
}


def custom_shape(H: int, I: int, E: int, k: int, *, global_scale: float = 0.05,
                 router_std: float = 1.0, x_std: float = 1.0,
                 zipf_s: Optional[float] = None, name: str = "custom") -> LayerShape:
    return LayerShape(name, H=H, I=I, E=E, k=k, T=(), seeds=(), global_scale=global_scale,
                      router_std=router_std, x_std=x_std, zipf_s=zipf_s)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _random_bytes(rng: np.random.Generator, n: int) -> np.ndarray:
    # full-range 64-bit draws are the generator's raw outputs (the same stream as
    # bit_generator.random_raw), produced without per-call overhead
    words = rng.integers(0, np.iinfo(np.uint64).max, (n + 7) // 8, dtype=np.uint64, endpoint=True)
    return words.view(np.uint8)[:n]


def _bf16_bits_normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    f = rng.standard_normal(int(np.prod(shape)), dtype=np.float32) * np.float32(std)
    return torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).reshape(shape)


def _e4m3_bits_loguniform(rng: np.random.Generator, n: int, lo: float = -4.0, hi: float = 2.0,
                          chunk: int = 1 << 25) -> np.ndarray:
    out = np.empty(n, dtype=np.uint8)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        u = rng.random(m, dtype=np.float32) * np.float32(hi - lo) + np.float32(lo)
        v = torch.from_numpy(np.exp2(u))
        out[s:s + m] = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return out


def make_layer(shape: LayerShape, seed: int) -> Dict[str, Optional[np.ndarray]]:
    """One seeded layer in the canonical layout (host numpy arrays)."""
    H, I, E = shape.H, shape.I, shape.E
    assert H % 2 == 0 and I % 2 == 0
    r = _rng(seed, 0xA11CE)
    layer: Dict[str, Optional[np.ndarray]] = {}
    layer["router_w"] = _bf16_bits_normal(r, (E, H), shape.router_std)
    for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
        layer[f"{name}_codes"] = _random_bytes(r, E * rows * (K // 2)).reshape(E, rows, K // 2)
        layer[f"{name}_scales"] = _e4m3_bits_loguniform(r, E * rows * (K // 16)).reshape(E, rows, K // 16)
        layer[f"{name}_global"] = np.full(E, shape.global_scale, dtype=np.float32)
    if shape.zipf_s is not None:
        rz = _rng(seed, 0x21DF)
        ranks = rz.permutation(E) + 1                      # rank of expert e
        p = ranks.astype(np.float64) ** (-shape.zipf_s)
        p /= p.sum()
        sigma_l = shape.router_std * shape.x_std * math.sqrt(H)
        beta = sigma_l * math.sqrt(6.0) / math.pi
        layer["router_bias"] = (beta * np.log(p)).astype(np.float32)
    else:
        layer["router_bias"] = None
    return layer


def make_shared(shape: LayerShape, seed: int, Is: int) -> Dict[str, np.ndarray]:
    """Seeded shared expert of width Is (canonical layout, host numpy arrays)."""
    H = shape.H
    assert Is % 16 == 0 and Is > 0
    r = _rng(seed, 0x5EED, Is)
    out: Dict[str, np.ndarray] = {}
    for name, rows, K in (("gate", Is, H), ("up", Is, H), ("down", H, Is)):
        out[f"shared_{name}_codes"] = _random_bytes(r, rows * (K // 2)).reshape(rows, K // 2)
        out[f"shared_{name}_scales"] = _e4m3_bits_loguniform(r, rows * (K // 16)).reshape(rows, K // 16)
        out[f"shared_{name}_global"] = np.full(1, shape.global_scale, dtype=np.float32)
    return out


def make_residual(shape: LayerShape, seed: int, T: int) -> np.ndarray:
    """Seeded residual stream, bf16 bits [T][H]."""
    return _bf16_bits_normal(_rng(seed, 0x2E5, T), (T, shape.H), 1.0)


def make_norm_weight(shape: LayerShape, seed: int) -> np.ndarray:
    """Seeded RMS-norm gamma, bf16 bits [H], uniform on [0.5, 1.5]."""
    f = _rng(seed, 0x4042).random(shape.H, dtype=np.float32) + np.float32(0.5)
    return torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def make_x(shape: LayerShape, seed: int, T: int, stream: int = 0) -> np.ndarray:
    """Seeded activations x, bf16 bits [T][H]."""
    r = _rng(seed, 0xB0B, T, stream)
    return _bf16_bits_normal(r, (T, shape.H), shape.x_std)


def layer_digest(layer: Dict[str, Optional[np.ndarray]]) -> Dict[str, str]:
    out = {}
    for k, v in sorted(layer.items()):
        out[k] = "none" if v is None else hashlib.sha256(np.ascontiguousarray(v).tobytes()).hexdigest()[:16]
    return out


LAYER_KEYS: List[str] = ["router_w", "router_bias", "gate_codes", "up_codes", "gate_scales",
                         "up_scales", "gate_global", "up_global", "down_codes", "down_scales",
                         "down_global"]

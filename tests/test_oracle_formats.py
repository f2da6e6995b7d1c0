"""Pins for the oracle's number-format routines (CPU only).

E2M1 / E4M3 values are pinned to the OCP MX / OFP8 format tables stored in
tests/golden/formats.txt and, for all 256 E4M3 bytes, to torch's own
float8_e4m3fn decoder (a library routine). The bf16 rounding is pinned to
hand-worked cases, including one where rounding through fp32 first would give
a different answer, and to torch's fp32 -> bf16 conversion on fp32 inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "formats.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, code, val = line.split()
            rows.append((fmt, int(code, 16), float(val)))
    return rows


def test_golden_format_tables(oracle_mod):
    rows = _golden()
    assert sum(1 for r in rows if r[0] == "e2m1") == 16
    for fmt, code, val in rows:
        got = oracle_mod.e2m1(code) if fmt == "e2m1" else oracle_mod.e4m3(code)
        if math.isnan(val):
            assert math.isnan(got), (fmt, hex(code))
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), (fmt, hex(code), got, val)


def test_e4m3_all_bytes_match_torch(oracle_mod):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for b in range(256):
        got, want = oracle_mod.e4m3(b), ref[b].item()
        if math.isnan(want):
            assert math.isnan(got), hex(b)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (hex(b), got, want)


@pytest.mark.parametrize("value,bits", [
    (1.0, 0x3F80),
    (-2.5, 0xC020),
    (1.0 + 2.0 ** -8, 0x3F80),                 # exact midpoint, ties to even (down)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),             # exact midpoint, ties to even (up)
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),    # just above the midpoint; via fp32 it would be 0x3F80
    (2.0 ** -130, 0x0008),                     # bf16 subnormal, exact
    (2.0 ** -134, 0x0000),                     # half the smallest subnormal: ties to even -> 0
    (3 * 2.0 ** -134, 0x0002),                 # 1.5 quanta: ties to even -> 2 quanta
    (3.4e38, 0x7F80),                          # above max + half ulp -> inf
    (3.38e38, 0x7F7E),                         # below bf16 max, rounds within range
    (-0.0, 0x8000),
    (0.0, 0x0000),
    (float("inf"), 0x7F80),
    (float("-inf"), 0xFF80),
])
def test_round_bf16_hand_cases(oracle_mod, value, bits):
    assert oracle_mod.round_bf16(value) == bits


def test_round_bf16_nan(oracle_mod):
    b = oracle_mod.round_bf16(float("nan"))
    assert (b & 0x7F80) == 0x7F80 and (b & 0x7F) != 0


def test_round_bf16_matches_torch_on_fp32_values(oracle_mod):
    rng = np.random.default_rng(123)
    f = np.concatenate([
        rng.standard_normal(3000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-38).astype(np.float32),   # subnormal range
        (rng.standard_normal(1000) * 1e37).astype(np.float32),
    ])
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for v, w in zip(f.tolist(), want.tolist()):
        assert oracle_mod.round_bf16(float(np.float32(v))) == w, v


def test_bf16_to_float_roundtrip(oracle_mod):
    for bits in (0x3F80, 0xC020, 0x0001, 0x7F7F, 0x8000):
        assert oracle_mod.round_bf16(oracle_mod.bf16_to_float(bits)) == bits

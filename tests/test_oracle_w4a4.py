"""Pin the oracle's NVFP4 activation quantisation and its W4A4 forward (CPU only).

* E2M1 rounding against a brute-force nearest-code search (ties to the even code), over every
  grid point, every midpoint, points next to them and saturation.
* E4M3 rounding against torch's float8_e4m3fn cast (round to nearest even), scales clamped to 448.
* The row quantiser: exact round trip of rows built from representable values, every element's
  dequantised value the nearest grid point times its block's scale (brute force), zero rows.
* The W4A4 forward against a dense numpy computation that quantises with the brute-force
  rounding above, decodes the weights in one vectorised pass and uses fp64 matmuls.
"""
import numpy as np
import pytest
import torch

from nvfp4_weight_only_route_b200 import synth

import test_oracle_bruteforce as bf

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e2m1_brute(v):
    """Nearest of the 16 codes, ties to the code with an even mantissa bit; saturating."""
    a = min(abs(v), 6.0)
    d = np.abs(GRID - a)
    best = np.flatnonzero(d == d.min())
    c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
    return (8 if v < 0 else 0) | c


def _e4m3_torch(v):
    return int(torch.tensor([min(v, 448.0)], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).item())


def _f32(v):
    return float(np.float32(v))


def test_e2m1_rounding_matches_brute_force(oracle_mod):
    mids = (GRID[1:] + GRID[:-1]) / 2
    pts = np.concatenate([GRID, mids, np.nextafter(mids, 0), np.nextafter(mids, 10), [6.5, 7.0, 100.0, 1e-9]])
    for v in np.concatenate([pts, -pts]):
        assert oracle_mod.e2m1_rne(float(v)) == _e2m1_brute(float(v)), v


def test_e4m3_rounding_matches_torch(oracle_mod):
    rng = np.random.default_rng(3)
    vals = [0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -6, 1.0625, 1.1875, 447.0, 448.0, 460.0]
    vals += list(np.exp2(rng.uniform(-11, 9, 400)).astype(np.float32))
    for v in vals:
        v = _f32(v)
        assert oracle_mod.e4m3_rne(v) == _e4m3_torch(v), v
    assert oracle_mod.e4m3_rne(1e6) == 0x7E       # clamped to 448


def test_row_of_representable_values_round_trips_exactly(oracle_mod):
    """amax = 2688 * 2^j gives g = 2^j; a block whose largest magnitude is 6 s_b g gets scale
    s_b; its elements E2M1 * s_b * g come back bit for bit."""
    rng = np.random.default_rng(5)
    K, j = 64, -3
    g = 2.0 ** j
    sbs = [448.0, 0.5, 2.0, 0.1875]      # E4M3 values (0.1875 = 1.5 * 2^-3); block 0 holds the row max
    v = np.zeros(K)
    for b in range(K // 16):
        codes = rng.integers(0, 16, 16)
        v[16 * b:16 * b + 16] = np.array([bf.E2M1_TABLE[c] for c in codes]) * sbs[b] * g
        v[16 * b] = 6.0 * sbs[b] * g                        # the block's largest: 6 s_b g
    assert v[0] == 2688.0 * g                                # the row's largest: 6 * 448 * g
    codes, scales, gq, deq = oracle_mod.quant_act_row(v)
    assert gq == g
    assert np.array_equal(deq, v)


def test_row_quantisation_is_nearest_grid_point(oracle_mod):
    rng = np.random.default_rng(9)
    for seed in range(4):
        v = rng.standard_normal(128).astype(np.float32).astype(np.float64) * (10.0 ** (seed - 2))
        v[rng.integers(0, 128, 5)] = 0.0
        codes, scales, g, deq = oracle_mod.quant_act_row(v)
        amax = np.float32(np.max(np.abs(v)))
        assert g == _f32(amax / np.float32(2688.0))
        six_g = np.float32(6.0) * np.float32(g)
        for b in range(8):
            blk = v[16 * b:16 * b + 16]
            ratio = np.float32(np.max(np.abs(blk))) / six_g
            assert scales[b] == _e4m3_torch(float(ratio))
            sbv = torch.tensor([scales[b]], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
            S = np.float32(sbv) * np.float32(g)
            for i in range(16):
                c = _e2m1_brute(float(np.float32(blk[i]) / S)) if S > 0 else 0
                assert codes[16 * b + i] == c
                assert deq[16 * b + i] == bf.E2M1_TABLE[c] * sbv * g


def test_zero_row(oracle_mod):
    codes, scales, g, deq = oracle_mod.quant_act_row(np.zeros(32))
    assert g == 1.0 and not codes.any() and not scales.any() and not deq.any()


def _quant_rows_brute(rows):
    out = np.empty_like(rows)
    for r in range(rows.shape[0]):
        v = rows[r]
        g = np.float32(np.float32(np.max(np.abs(v))) / np.float32(2688.0)) if np.any(v) else np.float32(1.0)
        six_g = np.float32(6.0) * g
        for b in range(v.shape[0] // 16):
            blk = v[16 * b:16 * b + 16]
            sb = _e4m3_torch(float(np.float32(np.max(np.abs(blk))) / six_g))
            sbv = torch.tensor([sb], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
            S = np.float32(sbv) * g
            for i in range(16):
                c = _e2m1_brute(float(np.float32(blk[i]) / S)) if S > 0 else 0
                out[r, 16 * b + i] = bf.E2M1_TABLE[c] * sbv * float(g)
    return out


@pytest.mark.parametrize("H,I,E,k,T,seed", [(64, 32, 4, 2, 3, 61), (32, 64, 8, 3, 2, 62)])
def test_w4a4_forward_matches_dense(oracle_mod, H, I, E, k, T, seed):
    shape = synth.custom_shape(H, I, E, k, router_std=1.0)
    layer = synth.make_layer(shape, seed)
    x = synth.make_x(shape, seed, T)
    r = oracle_mod.forward(layer, x, top_k=k, intermediates=True, act_fp4=True)
    b = bf.brute_force(layer, x, k)                              # routing is the W4A16 one
    assert np.array_equal(r["ids"], b["ids"])
    xq = _quant_rows_brute(bf._bf16(x))
    Wg = bf._decode_matrix(layer["gate_codes"], layer["gate_scales"], layer["gate_global"])
    Wu = bf._decode_matrix(layer["up_codes"], layer["up_scales"], layer["up_global"])
    Wd = bf._decode_matrix(layer["down_codes"], layer["down_scales"], layer["down_global"])
    out64 = np.zeros((T, H))
    for t in range(T):
        for s in range(k):
            e = r["ids"][t, s]
            G = np.float32(xq[t] @ Wg[e].T)
            U = np.float32(xq[t] @ Wu[e].T)
            v = G.astype(np.float64) / (1.0 + np.exp(-G.astype(np.float64))) * U.astype(np.float64)
            a = bf._bf16(bf._to_bf16_bits(v))
            assert np.array_equal(bf._bf16(r["a"][t, s]), a) or np.mean(bf._bf16(r["a"][t, s]) == a) > 0.95
            aq = _quant_rows_brute(bf._bf16(r["a"][t, s])[None, :])[0]
            out64[t] += r["g"][t, s] * (aq @ Wd[e].T)
    assert np.allclose(r["out64"], out64, rtol=1e-12, atol=1e-12 * np.max(np.abs(out64)))


def test_w4a4_differs_from_w4a16_by_the_quantisation_only(oracle_mod):
    """Same routing; outputs close to W4A16's (4-bit activations lose ~2 bits), not equal."""
    shape = synth.custom_shape(64, 32, 4, 2, router_std=1.0)
    layer = synth.make_layer(shape, 63)
    x = synth.make_x(shape, 63, 4)
    a16 = oracle_mod.forward(layer, x, top_k=2, intermediates=True)
    a4 = oracle_mod.forward(layer, x, top_k=2, intermediates=True, act_fp4=True)
    assert np.array_equal(a16["ids"], a4["ids"])
    assert not np.array_equal(a16["out64"], a4["out64"])
    assert np.max(np.abs(a16["out64"] - a4["out64"])) < 0.5 * np.max(a16["S"])

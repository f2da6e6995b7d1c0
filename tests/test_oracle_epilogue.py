"""Pin the oracle's steps around the routed path: the shared expert, the residual add and
the RMS norm of the layer output (CPU only).

* The shared expert, residual and norm are checked against an independent dense numpy
  computation (weights decoded in one vectorised pass, one fp64 matmul per projection,
  the norm through torch's ``rms_norm`` in fp64), which shares nothing with the oracle's
  loops.
* Closed forms: zero expert weights leave exactly the residual; a constant row normalises
  to +-1 when eps = 0; the norm is invariant to scaling its input.
* The identity the CUDA path relies on: a shared expert of width 2I equals the sum of its
  two halves of width I (its down projection split along the reduction dimension).
"""
import numpy as np
import pytest
import torch

from nvfp4_weight_only_route_b200 import synth

import test_oracle_bruteforce as bf


def _shared_dense(sh, x_bits):
    x = bf._bf16(x_bits)
    Wg = bf._decode_matrix(sh["shared_gate_codes"][None], sh["shared_gate_scales"][None], sh["shared_gate_global"])[0]
    Wu = bf._decode_matrix(sh["shared_up_codes"][None], sh["shared_up_scales"][None], sh["shared_up_global"])[0]
    Wd = bf._decode_matrix(sh["shared_down_codes"][None], sh["shared_down_scales"][None], sh["shared_down_global"])[0]
    G = (x @ Wg.T).astype(np.float32)
    U = (x @ Wu.T).astype(np.float32)
    v = G.astype(np.float64) / (1.0 + np.exp(-G.astype(np.float64))) * U.astype(np.float64)
    a_bits = bf._to_bf16_bits(v)
    a = bf._bf16(a_bits)
    return dict(v=v, a_bits=a_bits, y=a @ Wd.T, yabs=np.abs(a) @ np.abs(Wd).T)


def _norm_dense(v_bits, gamma_bits, eps):
    v = torch.from_numpy(bf._bf16(v_bits))
    n = torch.nn.functional.rms_norm(v, (v.shape[1],), eps=eps)
    return (n * torch.from_numpy(bf._bf16(gamma_bits))).numpy()


def _check_bf16_near(got_bits, want64, slack=0.0):
    """bf16 bits equal the RNE rounding of want64, except next to a midpoint (the dense
    side rounds through a library path)."""
    got = bf._bf16(got_bits)
    q = bf._bf16_quantum(want64)
    assert np.all(np.abs(got - want64) <= 0.5 * q * (1 + 1e-9) + slack)


def _layer(H, I, E, k, Is, seed):
    shape = synth.custom_shape(H, I, E, k, router_std=1.0)
    layer = synth.make_layer(shape, seed)
    if Is:
        layer.update(synth.make_shared(shape, seed, Is))
        # distinct per-tensor multipliers, so that a projection reading another's shows
        for name, v in (("gate", 0.05), ("up", 0.07), ("down", 0.03)):
            layer[f"shared_{name}_global"] = np.full(1, v, np.float32)
    return shape, layer


@pytest.mark.parametrize("H,I,E,k,Is,T,seed", [
    (64, 32, 4, 2, 32, 3, 21),
    (32, 64, 8, 3, 128, 2, 22),
    (48, 80, 5, 2, 160, 4, 23),     # K not a multiple of 32
])
def test_shared_expert_residual_and_norm_match_dense(oracle_mod, H, I, E, k, Is, T, seed):
    shape, layer = _layer(H, I, E, k, Is, seed)
    x = synth.make_x(shape, seed, T)
    res = synth.make_residual(shape, seed, T)
    gamma = synth.make_norm_weight(shape, seed)
    eps = 1e-6
    r = oracle_mod.forward(layer, x, top_k=k, intermediates=True, residual=res, norm_w=gamma, eps=eps)
    b = bf.brute_force(layer, x, k)
    d = _shared_dense(layer, x)
    # the shared expert's a: equal except next to a bf16 midpoint
    diff = r["a_sh"] != d["a_bits"]
    if diff.any():
        q = bf._bf16_quantum(d["v"][diff])
        frac = np.abs(d["v"][diff] / q - np.floor(d["v"][diff] / q) - 0.5)
        assert np.all(frac < 2.0 ** -14)
    exact_a = not diff.any()
    if exact_a:
        assert np.allclose(r["y_sh"], d["y"], rtol=0, atol=1e-12 * np.max(np.abs(d["y"])))
    # out64 = routed + shared + residual; S = routed + shared absolute sums
    want = b["out64"] + d["y"] + bf._bf16(res)
    S = b["S"] + d["yabs"]
    assert np.allclose(r["S"], S, rtol=1e-12, atol=1e-300)
    tol = (1e-12 if exact_a else 2.0 ** -7) * S + 1e-12
    assert np.all(np.abs(r["out64"] - want) <= tol)
    _check_bf16_near(r["out"], want, tol)
    # the norm reads the rounded output
    _check_bf16_near(r["out_norm"], _norm_dense(r["out"], gamma, eps))


def test_residual_only_when_expert_weights_are_zero(oracle_mod):
    """All codes zero: every expert output is 0, so the layer output is the residual, bit for bit."""
    shape, layer = _layer(64, 32, 4, 2, 64, 31)
    for key in ("gate_codes", "up_codes", "down_codes", "shared_down_codes"):
        layer[key] = np.zeros_like(layer[key])
    x = synth.make_x(shape, 31, 5)
    res = synth.make_residual(shape, 31, 5)
    r = oracle_mod.forward(layer, x, top_k=2, residual=res)
    assert np.array_equal(r["out"], res)


def test_residual_adds_exactly(oracle_mod):
    """With and without the residual, out64 differs by the residual's value (to fp64 rounding)."""
    shape, layer = _layer(64, 32, 4, 2, 0, 32)
    x = synth.make_x(shape, 32, 4)
    res = synth.make_residual(shape, 32, 4)
    a = oracle_mod.forward(layer, x, top_k=2)
    b = oracle_mod.forward(layer, x, top_k=2, residual=res)
    assert np.allclose(b["out64"] - a["out64"], bf._bf16(res), rtol=0, atol=1e-12 * (1 + np.abs(a["out64"])))


@pytest.mark.parametrize("c", [0.75, -3.0, 2.0 ** -20, 1000.0])
def test_norm_of_constant_row_is_sign_when_eps_is_zero(oracle_mod, c):
    H = 64
    v = np.full((2, H), oracle_mod.round_bf16(c), dtype=np.uint16)
    ones = np.full(H, 0x3F80, dtype=np.uint16)
    out = oracle_mod.rms_norm(v, ones, 0.0)
    assert np.all(out == (0xBF80 if c < 0 else 0x3F80))


def test_norm_eps_enters_under_the_root(oracle_mod):
    """Constant row c, gamma 1: out = bf16(c / sqrt(c^2 + eps)) -- eps inside the square root."""
    H = 32
    c, eps = 0.5, 0.0625
    v = np.full((1, H), oracle_mod.round_bf16(c), dtype=np.uint16)
    ones = np.full(H, 0x3F80, dtype=np.uint16)
    want = oracle_mod.round_bf16(c / np.sqrt(c * c + eps))
    assert np.all(oracle_mod.rms_norm(v, ones, eps) == want)


def test_norm_is_scale_invariant_and_applies_gamma_per_column(oracle_mod):
    """rms_norm(2^j v) == rms_norm(v) for eps = 0 (powers of two scale exactly), and gamma
    multiplies column h only."""
    H = 48
    rng = np.random.default_rng(7)
    v = bf._to_bf16_bits(rng.standard_normal((3, H))).reshape(3, H)
    gamma = bf._to_bf16_bits(rng.uniform(0.5, 1.5, H))
    v4 = bf._to_bf16_bits(bf._bf16(v) * 4.0).reshape(3, H)
    a = oracle_mod.rms_norm(v, gamma, 0.0)
    assert np.array_equal(a, oracle_mod.rms_norm(v4, gamma, 0.0))
    g2 = gamma.copy()
    g2[5] = oracle_mod.round_bf16(2.0 * bf._bf16(gamma[5:6])[0])
    b = oracle_mod.rms_norm(v, g2, 0.0)
    assert np.array_equal(np.delete(a, 5, axis=1), np.delete(b, 5, axis=1))
    assert np.allclose(bf._bf16(b[:, 5]), 2.0 * bf._bf16(a[:, 5]), rtol=2.0 ** -7)


def test_shared_expert_of_width_2I_is_the_sum_of_its_halves(oracle_mod):
    """Split the shared expert's intermediate rows (gate/up rows, down columns) into two
    halves: the two half-width experts' outputs add up to the full one's (fp64 rounding)."""
    H, I = 64, 32
    shape, layer = _layer(H, I, 4, 1, 2 * I, 41)
    x = synth.make_x(shape, 41, 3)
    full = oracle_mod.forward(layer, x, top_k=1, intermediates=True)
    halves = []
    for j in range(2):
        lj = dict(layer)
        for name in ("gate", "up"):
            lj[f"shared_{name}_codes"] = np.ascontiguousarray(layer[f"shared_{name}_codes"][j * I:(j + 1) * I])
            lj[f"shared_{name}_scales"] = np.ascontiguousarray(layer[f"shared_{name}_scales"][j * I:(j + 1) * I])
        lj["shared_down_codes"] = np.ascontiguousarray(layer["shared_down_codes"][:, j * I // 2:(j + 1) * I // 2])
        lj["shared_down_scales"] = np.ascontiguousarray(layer["shared_down_scales"][:, j * I // 16:(j + 1) * I // 16])
        halves.append(oracle_mod.forward(lj, x, top_k=1, intermediates=True))
    assert np.array_equal(np.concatenate([h["a_sh"] for h in halves], axis=1), full["a_sh"])
    assert np.allclose(halves[0]["y_sh"] + halves[1]["y_sh"], full["y_sh"], rtol=0,
                       atol=1e-12 * np.max(np.abs(full["y_sh"])))

"""Closed-form pins for the oracle's layer arithmetic (CPU only).

Each case is small enough to be worked by hand; the expected numbers are
written out below with their derivation, not recomputed by the test.
"""
import math

import numpy as np

from layer_builders import bf16_bits, constant_layer, unit_x

# The hand-worked 16-element block: bytes 10 32 54 76 98 BA DC FE hold codes
# 0..15 in element order (element 2c in the low nibble of byte c), scale byte
# 0x3C = 1.5, per-tensor scale 0.05.
BLOCK = np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], dtype=np.uint8)
# E2M1 codes 0..15 times 1.5 * 0.05 = 0.075:
BLOCK_DEQ = [0.0, 0.0375, 0.075, 0.1125, 0.15, 0.225, 0.3, 0.45,
             -0.0, -0.0375, -0.075, -0.1125, -0.15, -0.225, -0.3, -0.45]


def _block_layer():
    H = I = 16
    L = constant_layer(H, I, 1)
    L["gate_codes"][:] = BLOCK
    L["gate_scales"][:] = 0x3C
    L["gate_global"][:] = 0.05
    return L


def test_hand_worked_block_dot_first_half(oracle_mod):
    L = _block_layer()
    x = bf16_bits([[1.0] * 8 + [0.0] * 8])
    r = oracle_mod.forward(L, x, top_k=1, intermediates=True)
    # sum of codes 0..7 = 18; 18 * 1.5 * fp32(0.05) = 1.350000020116..., whose nearest
    # fp32 is fp32(1.35) = 1.35000002384185791015625.
    assert r["G"][0, 0, 0] == np.float32(1.35)
    assert np.all(r["G"][0, 0, :] == np.float32(1.35))


def test_hand_worked_block_dot_all_ones_cancels(oracle_mod):
    L = _block_layer()
    x = bf16_bits([[1.0] * 16])
    r = oracle_mod.forward(L, x, top_k=1, intermediates=True)
    assert np.all(r["G"][0, 0, :] == 0.0)


def test_hand_worked_block_each_element(oracle_mod):
    L = _block_layer()
    for c in range(16):
        x = unit_x(1, 16, col=c)
        r = oracle_mod.forward(L, x, top_k=1, intermediates=True)
        got = float(r["G"][0, 0, 0])
        assert abs(got - BLOCK_DEQ[c]) <= 1e-7 * max(abs(BLOCK_DEQ[c]), 1e-30), (c, got)


def test_swiglu_chain_gate1_up2(oracle_mod):
    # One expert, x = e_0, all weights exact: G = 1, U = 2.
    # silu(1) * 2 = 2e/(e+1) = 1.46211715726...; bf16 grid on [1,2) is 1/128:
    # 187.15/128 -> 187/128 = 1.4609375. Down weights all 1: y = 64 * 1.4609375 = 93.5.
    L = constant_layer(16, 64, 1, gate_code=0x2, up_code=0x4, down_code=0x2)
    r = oracle_mod.forward(L, unit_x(1, 16), top_k=1, intermediates=True)
    assert np.all(r["G"] == 1.0) and np.all(r["U"] == 2.0)
    assert np.all(r["a"] == bf16_bits([1.4609375])[0])
    assert np.all(r["out"] == bf16_bits([93.5])[0])
    assert np.allclose(r["out64"], 93.5, rtol=0, atol=0)


def test_swiglu_chain_gate2_up1(oracle_mod):
    # silu applies to the gate only: G = 2, U = 1 -> silu(2) = 1.76159415595...,
    # 225.48/128 -> 225/128 = 1.7578125; y = 64 * 1.7578125 = 112.5.
    L = constant_layer(16, 64, 1, gate_code=0x4, up_code=0x2, down_code=0x2)
    r = oracle_mod.forward(L, unit_x(1, 16), top_k=1, intermediates=True)
    assert np.all(r["out"] == bf16_bits([112.5])[0])


def test_per_tensor_scales_are_per_projection(oracle_mod):
    # gate 1.0 * 0.5, up 1.0 * 4.0: silu(0.5) * 4 = 1.24491866240...; 159.35/128 -> 159/128.
    # down 1.0 * 0.25: y = 64 * 159/128 * 0.25 = 19.875 (exact in bf16: quantum 1/8 on [16,32)).
    L = constant_layer(16, 64, 1, gate_code=0x2, up_code=0x2, down_code=0x2,
                       gate_global=0.5, up_global=4.0, down_global=0.25)
    r = oracle_mod.forward(L, unit_x(1, 16), top_k=1, intermediates=True)
    assert np.all(r["G"] == 0.5) and np.all(r["U"] == 4.0)
    assert np.all(r["a"] == bf16_bits([159 / 128])[0])
    assert np.all(r["out"] == bf16_bits([19.875])[0])


def test_block_scales_apply_per_16_elements(oracle_mod):
    # x = ones on H=32; gate codes 1.0 everywhere, block 0 scale 1.0 (0x38), block 1
    # scale 2.0 (0x40): G = 16*1 + 16*2 = 48. Up codes 1.0 with scale 1.0: U = 32.
    L = constant_layer(32, 16, 1, gate_code=0x2, up_code=0x2, down_code=0x2)
    L["gate_scales"][:, :, 1] = 0x40
    x = bf16_bits([[1.0] * 32])
    r = oracle_mod.forward(L, x, top_k=1, intermediates=True)
    assert np.all(r["G"] == 48.0) and np.all(r["U"] == 32.0)


def test_two_expert_weighted_combine(oracle_mod):
    # Router: expert 0's row is e_0, expert 1's row is zero, x = e_0:
    # logits (1, 0); g = (e/(e+1), 1/(e+1)) = (0.731058578630..., 0.268941421369...).
    # Expert 0: gate 1, up 2 -> y0 = 93.5; expert 1: gate 2, up 1 -> y1 = 112.5.
    # out = 0.7310585786 * 93.5 + 0.2689414214 * 112.5 = 98.6098870... -> bf16 (quantum 0.5) 98.5.
    H, I, E = 16, 64, 2
    rows = np.zeros((E, H), np.float32)
    rows[0, 0] = 1.0
    L = constant_layer(H, I, E, gate_code=[0x2, 0x4], up_code=[0x4, 0x2], down_code=0x2, router_rows=rows)
    r = oracle_mod.forward(L, unit_x(1, H), top_k=2, intermediates=True)
    assert r["ids"].tolist() == [[0, 1]]
    assert r["logits"].tolist() == [[1.0, 0.0]]
    e = math.e
    assert abs(r["g"][0, 0] - e / (e + 1)) < 1e-15 and abs(r["g"][0, 1] - 1 / (e + 1)) < 1e-15
    assert np.all(r["out"] == bf16_bits([98.5])[0])
    assert abs(r["out64"][0, 0] - 98.60988700602991) < 1e-9
    # k = 1 keeps only expert 0 with weight 1.
    r1 = oracle_mod.forward(L, unit_x(1, H), top_k=1, intermediates=True)
    assert r1["ids"].tolist() == [[0]] and r1["g"].tolist() == [[1.0]]
    assert np.all(r1["out"] == bf16_bits([93.5])[0])


def test_router_bias_shifts_selection(oracle_mod):
    H, I, E = 16, 16, 4
    rows = np.zeros((E, H), np.float32)
    rows[:, 0] = [1.0, 2.0, 3.0, 4.0]
    L = constant_layer(H, I, E, router_rows=rows, bias=[10.0, 0.0, 0.0, 0.0])
    r = oracle_mod.forward(L, unit_x(1, H), top_k=2, intermediates=True)
    assert r["logits"].tolist() == [[11.0, 2.0, 3.0, 4.0]]
    assert r["ids"].tolist() == [[0, 3]]


def test_exact_ties_go_to_lower_index(oracle_mod):
    H, I, E = 16, 16, 6
    rows = np.zeros((E, H), np.float32)
    rows[[1, 2, 4], 0] = 0.5          # three identical rows
    rows[5, 0] = -1.0
    L = constant_layer(H, I, E, router_rows=rows)
    r = oracle_mod.forward(L, unit_x(1, H), top_k=4, intermediates=True)
    assert r["ids"].tolist() == [[1, 2, 4, 0]]
    # the three tied experts share one weight; expert 0 (logit 0) gets exp(-0.5) of it
    g = r["g"][0]
    assert g[0] == g[1] == g[2]
    assert abs(g[3] / g[0] - math.exp(-0.5)) < 1e-15


def test_k_equals_E_selects_every_expert(oracle_mod):
    H, I, E = 16, 16, 5
    rows = np.zeros((E, H), np.float32)
    rows[:, 0] = [0.25, -1.0, 3.0, 0.25, 2.0]
    L = constant_layer(H, I, E, router_rows=rows)
    r = oracle_mod.forward(L, unit_x(1, H), top_k=5, intermediates=True)
    assert r["ids"].tolist() == [[2, 4, 0, 3, 1]]
    assert abs(r["g"].sum() - 1.0) < 1e-15


def test_empty_batch(oracle_mod):
    L = constant_layer(16, 16, 2)
    r = oracle_mod.forward(L, np.zeros((0, 16), np.uint16), top_k=1)
    assert r["out"].shape == (0, 16)


def test_gate_and_up_are_rounded_to_fp32_before_silu(oracle_mod):
    # x = (1, 2^-30, 0, ...): in fp64 G = 1 + 2^-30 and U = u*(1 + 2^-30), u the up
    # tensor's scale; rounded to fp32 they are exactly 1 and u.
    # u = 1.0392677783966064 (an fp32 number) puts silu(1)*u = 0.75976562489...
    # = 194.49999997 * 2^-8, just under the midpoint of two bf16 values, so
    # a = 194/256 = 0.7578125. Without the fp32 rounding, silu(1+2^-30)*u*(1+2^-30)
    # is 194.5000004 quanta and a would be 195/256.
    u = 1.0392677783966064
    L = constant_layer(16, 16, 1, gate_code=0x2, up_code=0x2, down_code=0x2, up_global=u)
    x = bf16_bits([[1.0, 2.0 ** -30] + [0.0] * 14])
    r = oracle_mod.forward(L, x, top_k=1, intermediates=True)
    assert np.all(r["G"] == 1.0) and np.all(r["U"] == np.float32(u))
    assert np.all(r["a"] == bf16_bits([0.7578125])[0])

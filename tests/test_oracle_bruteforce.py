"""Pin the oracle against an independent dense-equivalent computation (CPU only).

The brute force below decodes every expert's weights in one vectorised numpy
pass (E2M1 through the OCP table, E4M3 through torch's float8 decoder), runs
ALL experts on ALL tokens with fp64 matmuls, and masks by the routing. It
shares nothing with the oracle's per-expert loop nest, so a transposed
operand, a wrong row stride, a dropped term or a mixed-up projection in
either one shows up as a mismatch.
"""
import numpy as np
import pytest
import scipy.special
import torch

from nvfp4_weight_only_route_b200 import synth

E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
                       -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def _decode_matrix(codes, scales, glob):
    E, R, Kh = codes.shape
    K = Kh * 2
    nib = np.empty((E, R, K), dtype=np.uint8)
    nib[:, :, 0::2] = codes & 0x0F
    nib[:, :, 1::2] = codes >> 4
    sc = torch.from_numpy(np.ascontiguousarray(scales)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return E2M1_TABLE[nib] * np.repeat(sc, 16, axis=2) * glob.astype(np.float64)[:, None, None]


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def _to_bf16_bits(v64):
    return torch.from_numpy(np.ascontiguousarray(v64)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def brute_force(layer, x_bits, k):
    x = _bf16(x_bits)                                     # [T,H]
    Wr = _bf16(layer["router_w"])                         # [E,H]
    l = (x @ Wr.T).astype(np.float32)
    if layer.get("router_bias") is not None:
        l = l + layer["router_bias"][None, :]
    T, E = l.shape
    order = np.argsort(-l.astype(np.float64), axis=1, kind="stable")
    ids = order[:, :k]
    sel = np.take_along_axis(l.astype(np.float64), ids, axis=1)
    g = scipy.special.softmax(sel, axis=1)
    gw = np.zeros((T, E))
    np.put_along_axis(gw, ids, g, axis=1)
    mask = np.zeros((T, E), dtype=bool)
    np.put_along_axis(mask, ids, True, axis=1)

    Wg = _decode_matrix(layer["gate_codes"], layer["gate_scales"], layer["gate_global"])  # [E,I,H]
    Wu = _decode_matrix(layer["up_codes"], layer["up_scales"], layer["up_global"])
    Wd = _decode_matrix(layer["down_codes"], layer["down_scales"], layer["down_global"])  # [E,H,I]
    G = np.einsum("th,eih->tei", x, Wg).astype(np.float32)
    U = np.einsum("th,eih->tei", x, Wu).astype(np.float32)
    v = G.astype(np.float64) / (1.0 + np.exp(-G.astype(np.float64))) * U.astype(np.float64)
    a_bits = _to_bf16_bits(v)          # via fp32: may differ from a direct rounding at midpoints
    a = _bf16(a_bits)
    y = np.einsum("tei,ehi->teh", a, Wd)
    yabs = np.einsum("tei,ehi->teh", np.abs(a), np.abs(Wd))
    out64 = np.einsum("te,teh->th", gw, y)
    S = np.einsum("te,teh->th", gw, yabs)
    return dict(logits=l, ids=ids, g=g, G=G, U=U, v=v, a_bits=a_bits, y=y, out64=out64, S=S, mask=mask)


def _bf16_quantum(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _check(oracle_mod, layer, x, k):
    r = oracle_mod.forward(layer, x, top_k=k, intermediates=True)
    b = brute_force(layer, x, k)
    T = x.shape[0]
    # Routing: identical logits, identical ids, weights to fp64 rounding.
    assert np.array_equal(r["logits"], b["logits"])
    assert np.array_equal(r["ids"], b["ids"])
    assert np.allclose(r["g"], b["g"], rtol=1e-14, atol=0)
    assert np.allclose(r["g"].sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # Gate / up per selected pair: fp32 results from two summation orders agree
    # to within one fp32 ulp (almost always exactly).
    Gb = np.take_along_axis(b["G"], b["ids"][:, :, None], axis=1)
    Ub = np.take_along_axis(b["U"], b["ids"][:, :, None], axis=1)
    for got, want in ((r["G"], Gb), (r["U"], Ub)):
        ulp = np.spacing(np.abs(want).astype(np.float32))
        assert np.all(np.abs(got.astype(np.float64) - want.astype(np.float64)) <= ulp)
        assert np.mean(got == want) > 0.99
    # SwiGLU output a: equal, except where rounding through fp32 (the brute force's
    # library route) and rounding the fp64 value directly (the oracle) legitimately differ:
    # only next to a bf16 midpoint.
    ab = np.take_along_axis(b["a_bits"], b["ids"][:, :, None], axis=1)
    diff = r["a"] != ab
    if diff.any():
        v = np.take_along_axis(b["v"], b["ids"][:, :, None], axis=1)[diff]
        q = _bf16_quantum(v)
        frac = np.abs(v / q - np.floor(v / q) - 0.5)
        assert np.all(frac < 2.0 ** -14), "a differs away from a bf16 midpoint"
    # Down + combine: compare fp64 pre-rounding output and the rounded one.
    exact_a = not diff.any()
    tol = (1e-12 if exact_a else 2.0 ** -7) * b["S"] + 1e-12
    assert np.all(np.abs(r["out64"] - b["out64"]) <= tol)
    assert np.allclose(r["S"], b["S"], rtol=1e-12, atol=1e-300)
    yb = np.take_along_axis(b["y"], b["ids"][:, :, None], axis=1)
    if exact_a:
        assert np.allclose(r["y"], yb, rtol=0, atol=1e-12 * np.max(np.abs(yb)))
    out_r = _bf16(r["out"])
    q = _bf16_quantum(b["out64"])
    assert np.all(np.abs(out_r - b["out64"]) <= 0.5 * q + tol)
    return r, b


@pytest.mark.parametrize("H,I,E,k,T,seed", [
    (32, 32, 4, 1, 3, 11),
    (64, 32, 4, 2, 4, 12),
    (32, 64, 8, 3, 2, 13),
    (64, 64, 8, 8, 1, 14),     # k = E
    (48, 80, 5, 2, 5, 15),     # K not a multiple of 32
])
def test_oracle_matches_brute_force_tiny(oracle_mod, H, I, E, k, T, seed):
    shape = synth.custom_shape(H, I, E, k, global_scale=0.05, router_std=1.0)
    layer = synth.make_layer(shape, seed)
    # distinct per-tensor scales per expert and projection, to catch mix-ups
    rng = np.random.default_rng(seed)
    for n in ("gate_global", "up_global", "down_global"):
        layer[n] = rng.uniform(0.01, 0.1, size=E).astype(np.float32)
    x = synth.make_x(shape, seed, T)
    _check(oracle_mod, layer, x, k)


def test_oracle_matches_brute_force_with_bias(oracle_mod):
    shape = synth.custom_shape(64, 32, 8, 2, global_scale=0.05, router_std=1.0, zipf_s=1.1)
    layer = synth.make_layer(shape, 21)
    assert layer["router_bias"] is not None
    _check(oracle_mod, layer, synth.make_x(shape, 21, 6), 2)


def test_oracle_matches_brute_force_tiny_layer_shape(oracle_mod):
    """The tiny workload layer (H=512, I=1024, E=8, top-2, T=4, seed 0) in full."""
    shape = synth.SHAPES[0]
    layer = synth.make_layer(shape, 0)
    x = synth.make_x(shape, 0, 4)
    _check(oracle_mod, layer, x, shape.k)


def test_routing_invariants_large_router(oracle_mod):
    """Routing on the decode layer shape: ids equal a stable argsort of -logits,
    logits equal fp32 of an fp64 matmul, weights are a softmax summing to 1."""
    shape = synth.SHAPES[1]
    E, H = shape.E, shape.H
    rng = np.random.default_rng(5)
    layer = synth.make_layer(synth.custom_shape(H, 16, E, shape.k, router_std=1.0), 3)
    x = synth.make_x(shape, 3, 16)
    r = oracle_mod.forward(layer, x, top_k=shape.k, intermediates=True)
    l_ref = (_bf16(x) @ _bf16(layer["router_w"]).T).astype(np.float32)
    assert np.array_equal(r["logits"], l_ref)
    ids_ref = np.argsort(-r["logits"].astype(np.float64), axis=1, kind="stable")[:, :shape.k]
    assert np.array_equal(r["ids"], ids_ref)
    for t in range(x.shape[0]):
        assert len(set(r["ids"][t].tolist())) == shape.k
        sel = r["logits"][t, r["ids"][t]]
        assert np.all(np.diff(sel) <= 0)
    assert np.allclose(r["g"].sum(axis=1), 1.0, atol=1e-15, rtol=0)
    del rng

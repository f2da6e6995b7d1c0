"""The oracle's routing-only entry point (CPU only).

``oracle.route`` runs the oracle's routing step by itself, so that whole large
batches can have every token's routing checked against it. It must give what
``oracle.forward`` gives for routing (the same step, the same arithmetic), and
it is pinned independently: the logits against a dense fp64 matrix product
rounded once to fp32, the ids against a stable argsort (ties to the lower
expert index), the weights against a softmax over the selected logits.
"""
import numpy as np
import pytest

from nvfp4_weight_only_route_b200 import synth


def _bf16(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


CASES = [
    ("tiny", 0, 0, 4),
    ("decode_t8", 1, 1, 8),
    ("decode_t1", 1, 2, 1),
    ("zipf", 2, 4, 48),
]


@pytest.mark.parametrize("name,shape_idx,seed,T", CASES)
def test_route_equals_forward_routing(oracle_mod, name, shape_idx, seed, T):
    s = synth.SHAPES[shape_idx]
    layer = synth.make_layer(s, seed)
    x = synth.make_x(s, seed, T)
    f = oracle_mod.forward(layer, x, top_k=s.k, intermediates=True)
    r = oracle_mod.route(layer, x, top_k=s.k)
    assert np.array_equal(r["logits"], f["logits"])
    assert np.array_equal(r["ids"], f["ids"])
    assert np.array_equal(r["g"], f["g"])


@pytest.mark.parametrize("with_bias", [False, True])
def test_route_pinned_to_dense_product_argsort_and_softmax(oracle_mod, with_bias):
    H, E, k, T = 256, 64, 6, 40
    shape = synth.custom_shape(H, 16, E, k, router_std=1.0, zipf_s=1.1 if with_bias else None)
    layer = synth.make_layer(shape, 31)
    x = synth.make_x(shape, 31, T)
    r = oracle_mod.route(layer, x, top_k=k)
    # logits: one fp32 rounding of the exact dot product (every bf16*bf16 product is exact
    # in fp64, and these sums stay far from fp32 rounding boundaries), plus the fp32 bias
    l_ref = (_bf16(x) @ _bf16(layer["router_w"]).T).astype(np.float32)
    if with_bias:
        l_ref = l_ref + layer["router_bias"][None, :]
    assert np.array_equal(r["logits"], l_ref)
    # ids: descending logits, ties to the lower expert index = a stable argsort of -logits
    ids_ref = np.argsort(-l_ref.astype(np.float64), axis=1, kind="stable")[:, :k]
    assert np.array_equal(r["ids"], ids_ref)
    # weights: softmax over the k selected logits
    sel = np.take_along_axis(l_ref.astype(np.float64), ids_ref, axis=1)
    e = np.exp(sel - sel[:, :1])
    assert np.allclose(r["g"], e / e.sum(axis=1, keepdims=True), rtol=1e-14, atol=0)
    assert np.allclose(r["g"].sum(axis=1), 1.0, rtol=0, atol=1e-15)


def test_route_exact_ties_go_to_the_lower_index(oracle_mod):
    H, E, k = 64, 8, 3
    shape = synth.custom_shape(H, 16, E, k, router_std=1.0)
    layer = synth.make_layer(shape, 5)
    rw = layer["router_w"].copy()
    rw[2] = rw[6] = rw[1]              # experts 1, 2, 6 have identical logits
    layer["router_w"] = rw
    x = synth.make_x(shape, 5, 64)
    r = oracle_mod.route(layer, x, top_k=k)
    for t in range(64):
        chosen = [e for e in r["ids"][t] if e in (1, 2, 6)]
        # whenever some of the three tie into the top k, the lower indices come first
        assert chosen == sorted(chosen)
        assert chosen == [1, 2, 6][:len(chosen)]


def test_route_k_equals_e_returns_every_expert(oracle_mod):
    H, E = 64, 8
    shape = synth.custom_shape(H, 16, E, E, router_std=1.0)
    layer = synth.make_layer(shape, 9)
    x = synth.make_x(shape, 9, 5)
    r = oracle_mod.route(layer, x, top_k=E)
    assert np.array_equal(np.sort(r["ids"], axis=1), np.tile(np.arange(E), (5, 1)))

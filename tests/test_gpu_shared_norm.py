"""The shared expert, the residual add and the RMS norm (tfmoe_forward_add_norm) against the
oracle, on the GPU through the C ABI.

The layer output out is checked against the oracle's fp64 value within the layer tolerance
(4e-3 * S + 1e-3 plus the final rounding; S includes the shared expert's absolute sums). The
norm is checked on the GPU's own out: out_norm must equal the oracle's RMS norm of that same
bf16 row (both sides compute the products in fp64 and round once), so any difference is a
rounding flip next to a bf16 midpoint.
"""
import numpy as np
import pytest

from nvfp4_weight_only_route_b200 import synth

from gpu_harness import bf16_to_f64, check_output

pytestmark = pytest.mark.gpu


def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _layer(H, I, E, k, m, seed, zipf=False):
    shape = synth.custom_shape(H, I, E, k, global_scale=0.02, router_std=1.0, zipf_s=1.1 if zipf else None)
    layer = synth.make_layer(shape, seed)
    if m:
        layer.update(synth.make_shared(shape, seed, m * I))
        for name, v in (("gate", 0.02), ("up", 0.03), ("down", 0.015)):
            layer[f"shared_{name}_global"] = np.full(1, v, np.float32)
    return shape, layer


def _run(layer, shape, x, m, flags=0, residual=None, norm_w=None, eps=1e-6, in_place=False, plain=False):
    torch = _cuda()
    from nvfp4_weight_only_route_b200 import tfmoe
    T = x.shape[0]
    L = tfmoe.MoELayer(shape.H, shape.I, shape.E, shape.k, T, has_router_bias=layer.get("router_bias") is not None,
                       flags=flags, shared_intermediate=m * shape.I, norm_eps=eps)
    try:
        L.load_weights(tfmoe.layer_to_device(layer))
        xd = torch.from_numpy(x.view(np.int16)).cuda()
        rd = None if residual is None else torch.from_numpy(residual.view(np.int16)).cuda()
        gd = None if norm_w is None else torch.from_numpy(norm_w.view(np.int16)).cuda()
        if plain:
            out = torch.empty((T, shape.H), dtype=torch.int16, device="cuda")
            L.forward(xd, out, T=T)
            on = None
        elif in_place:
            out, on = L.forward_add_norm(xd, residual=rd, norm_w=gd, out=rd)
        else:
            out, on = L.forward_add_norm(xd, residual=rd, norm_w=gd)
        assert L.sync_status() == 0, tfmoe.last_error()
        kx = shape.k + m
        res = {"out": out.view(torch.int16).cpu().numpy().view(np.uint16),
               "ids": L.buffer_tensor(tfmoe.BUF_TOPK_IDS, torch.int32, (T, kx)).cpu().numpy(),
               "g": L.buffer_tensor(tfmoe.BUF_TOPK_WEIGHTS, torch.float32, (T, kx)).cpu().numpy(),
               "counts": L.buffer_tensor(tfmoe.BUF_EXPERT_COUNTS, torch.int32, (shape.E + m,)).cpu().numpy()}
        if on is not None:
            res["out_norm"] = on.view(torch.int16).cpu().numpy().view(np.uint16)
        return res
    finally:
        L.close()


def _check(oracle_mod, layer, shape, x, m, g, residual=None, norm_w=None, eps=1e-6):
    o = oracle_mod.forward(layer, x, top_k=shape.k, intermediates=True, residual=residual, norm_w=norm_w, eps=eps)
    T, k, E = x.shape[0], shape.k, shape.E
    assert np.array_equal(g["ids"][:, :k], o["ids"])
    assert np.array_equal(g["ids"][:, k:], np.tile(E + np.arange(m), (T, 1)))
    assert np.all(g["g"][:, k:] == 1.0)
    assert np.allclose(g["g"][:, :k], o["g"], rtol=2e-6, atol=1e-7)
    assert np.all(g["counts"][E:] == T)
    assert np.array_equal(g["counts"][:E], np.bincount(o["ids"].ravel(), minlength=E))
    check_output(g["out"], o)
    if norm_w is not None:
        want = oracle_mod.rms_norm(g["out"], norm_w, eps)
        same = g["out_norm"] == want
        assert np.mean(same) >= 0.9999, f"only {np.mean(same):.6f} of normed outputs equal the oracle's norm"
        gv, wv = bf16_to_f64(g["out_norm"]), bf16_to_f64(want)
        assert np.all(np.abs(gv - wv) <= 2.0 ** -7 * np.abs(wv) + 1e-30), "a normed output is off by more than one ulp"
    return o


@pytest.mark.parametrize("regime", ["auto", "gemv", "mma"])
def test_decode_with_shared_expert_residual_and_norm(oracle_mod, regime):
    from nvfp4_weight_only_route_b200 import tfmoe
    flags = {"auto": 0, "gemv": tfmoe.FLAG_FORCE_GEMV, "mma": tfmoe.FLAG_FORCE_MMA}[regime]
    shape, layer = _layer(2048, 768, 128, 8, 1, 51)
    x = synth.make_x(shape, 51, 8)
    res = synth.make_residual(shape, 51, 8)
    gam = synth.make_norm_weight(shape, 51)
    g = _run(layer, shape, x, 1, flags=flags, residual=res, norm_w=gam)
    _check(oracle_mod, layer, shape, x, 1, g, residual=res, norm_w=gam)


@pytest.mark.parametrize("regime", ["auto", "gemv", "mma"])
@pytest.mark.parametrize("T", [1, 37])
def test_two_shared_slots_ragged_batch(oracle_mod, regime, T):
    from nvfp4_weight_only_route_b200 import tfmoe
    flags = {"auto": 0, "gemv": tfmoe.FLAG_FORCE_GEMV, "mma": tfmoe.FLAG_FORCE_MMA}[regime]
    shape, layer = _layer(384, 192, 6, 3, 2, 52)
    x = synth.make_x(shape, 52, T)
    res = synth.make_residual(shape, 52, T)
    gam = synth.make_norm_weight(shape, 52)
    g = _run(layer, shape, x, 2, flags=flags, residual=res, norm_w=gam, eps=1e-5)
    _check(oracle_mod, layer, shape, x, 2, g, residual=res, norm_w=gam, eps=1e-5)


def test_large_batch_plan_with_shared_expert(oracle_mod):
    """601 tokens x (8 + 1) slots: the multi-CTA plan counts the shared slot in every segment."""
    shape, layer = _layer(512, 256, 16, 8, 1, 53, zipf=True)
    x = synth.make_x(shape, 53, 601)
    res = synth.make_residual(shape, 53, 601)
    gam = synth.make_norm_weight(shape, 53)
    g = _run(layer, shape, x, 1, residual=res, norm_w=gam)
    _check(oracle_mod, layer, shape, x, 1, g, residual=res, norm_w=gam)


def test_residual_updated_in_place_without_norm(oracle_mod):
    shape, layer = _layer(512, 256, 8, 2, 1, 54)
    x = synth.make_x(shape, 54, 20)
    res = synth.make_residual(shape, 54, 20)
    g = _run(layer, shape, x, 1, residual=res.copy(), in_place=True)
    assert "out_norm" not in g
    _check(oracle_mod, layer, shape, x, 1, g, residual=res)


def test_norm_without_residual_and_no_shared_expert(oracle_mod):
    shape, layer = _layer(512, 256, 8, 2, 0, 55)
    x = synth.make_x(shape, 55, 24)
    gam = synth.make_norm_weight(shape, 55)
    g = _run(layer, shape, x, 0, norm_w=gam, eps=1e-3)
    _check(oracle_mod, layer, shape, x, 0, g, norm_w=gam, eps=1e-3)


def test_plain_forward_includes_the_shared_expert(oracle_mod):
    shape, layer = _layer(512, 256, 8, 2, 1, 56)
    x = synth.make_x(shape, 56, 5)
    g = _run(layer, shape, x, 1, plain=True)
    _check(oracle_mod, layer, shape, x, 1, g)


def test_add_norm_rejects_partial_overlap():
    torch = _cuda()
    from nvfp4_weight_only_route_b200 import tfmoe
    shape, layer = _layer(512, 256, 8, 2, 0, 57)
    L = tfmoe.MoELayer(shape.H, shape.I, shape.E, shape.k, 8)
    try:
        L.load_weights(tfmoe.layer_to_device(layer))
        buf = torch.zeros((16, shape.H), dtype=torch.int16, device="cuda")
        x = torch.from_numpy(synth.make_x(shape, 57, 8).view(np.int16)).cuda()
        lib = tfmoe.load_library()
        # residual and out overlap without being the same array
        st = lib.tfmoe_forward_add_norm(L.handle, x.data_ptr(), 8, buf[0].data_ptr(), None, buf[1].data_ptr(), None,
                                        torch.cuda.current_stream().cuda_stream)
        assert st == tfmoe.ERR_INVALID_ARG
        # norm weights without an out_norm
        gam = torch.zeros(shape.H, dtype=torch.int16, device="cuda")
        st = lib.tfmoe_forward_add_norm(L.handle, x.data_ptr(), 8, None, gam.data_ptr(), buf[8].data_ptr(), None,
                                        torch.cuda.current_stream().cuda_stream)
        assert st == tfmoe.ERR_INVALID_ARG
    finally:
        L.close()

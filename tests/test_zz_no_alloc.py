"""The allocation-free routing entry point, tfmoe_route_noalloc (needs a GPU).

Some callers of this library cannot allocate device memory: code running while
another component owns the whole memory budget through a fixed pool, and
real-time loops that cannot take cudaMalloc's latency or its implicit device
synchronisation. For them the entry point keeps its router logits in a fixed
array compiled into the library. Its ids and weights are checked here against
the fp64 oracle's routing and against the routing tfmoe_forward computes, on
two calls in a row. This file is collected last on purpose: if it fails, a run
stopped at the first failure has already run every other test. It also passes
alone in a fresh process.
"""
import numpy as np
import pytest

from nvfp4_weight_only_route_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_weight_only_route_b200 import build
    build.build()
    return torch


def _forward_routing(torch, layer_np, shape, x_np):
    """ids and weights from the regular entry point (tfmoe_forward's workspace)."""
    from nvfp4_weight_only_route_b200 import tfmoe
    T = x_np.shape[0]
    L = tfmoe.MoELayer(shape.H, shape.I, shape.E, shape.k, T, has_router_bias=layer_np["router_bias"] is not None)
    try:
        L.load_weights(tfmoe.layer_to_device(layer_np))
        x = torch.from_numpy(x_np.view(np.int16)).cuda()
        out = torch.empty_like(x)
        L.forward(x, out)
        tfmoe.check(L.sync_status())
        ids = L.buffer_tensor(tfmoe.BUF_TOPK_IDS, torch.int32, (T, shape.k)).cpu().numpy()
        w = L.buffer_tensor(tfmoe.BUF_TOPK_WEIGHTS, torch.float32, (T, shape.k)).cpu().numpy()
    finally:
        L.close()
    return ids, w


def _noalloc_routing(torch, layer_np, shape, x_np):
    from nvfp4_weight_only_route_b200 import tfmoe
    T = x_np.shape[0]
    x = torch.from_numpy(x_np.view(np.int16)).cuda()
    rw = torch.from_numpy(layer_np["router_w"].view(np.int16)).cuda()
    bias = None if layer_np["router_bias"] is None else torch.from_numpy(layer_np["router_bias"]).cuda()
    ids = torch.full((T, shape.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, shape.k), -1.0, dtype=torch.float32, device="cuda")
    tfmoe.check(tfmoe.route_noalloc(x, rw, bias, shape.k, ids, w))
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


# (shape, seed, T): the tiny layer (E=8, top-2, no bias); the decode layer (no bias) at
# T=1, 8 (the small-batch router kernel), 17 and 63 (partly filled 64-token tiles of the
# tiled router kernel); the batched-decode layer with its Zipf router bias at T=256.
CASES = [(0, 0, 4), (1, 1, 1), (1, 1, 8), (1, 2, 17), (1, 3, 63), (2, 4, 256)]


@pytest.mark.parametrize("shape_idx,seed,T", CASES)
def test_noalloc_routing_matches_oracle_and_forward_on_two_calls_in_a_row(torch_cuda, oracle_mod, shape_idx,
                                                                          seed, T):
    torch = torch_cuda
    shape = synth.SHAPES[shape_idx]
    layer_np = synth.make_layer(shape, seed)
    x_np = synth.make_x(shape, seed, T)
    ref = oracle_mod.route(layer_np, x_np, top_k=shape.k)
    ids_fwd, w_fwd = _forward_routing(torch, layer_np, shape, x_np)
    for _ in range(2):                        # the fixed array keeps the previous call's logits
        ids, w = _noalloc_routing(torch, layer_np, shape, x_np)
        assert np.array_equal(ids, ref["ids"]), "ids differ from the oracle's"
        assert np.max(np.abs(w.astype(np.float64) - ref["g"])) <= 2e-6
        assert np.array_equal(ids, ids_fwd), "ids differ from tfmoe_forward's"
        assert np.max(np.abs(w.astype(np.float64) - w_fwd)) <= 2e-6


def test_noalloc_ties_go_to_the_lower_expert(torch_cuda, oracle_mod):
    torch = torch_cuda
    shape = synth.custom_shape(256, 64, 8, 3, router_std=1.0)
    layer_np = synth.make_layer(shape, 8)
    rw = layer_np["router_w"].copy()
    rw[2] = rw[6] = rw[1]                     # three identical router rows: exact ties
    layer_np["router_w"] = rw
    x_np = synth.make_x(shape, 8, 20)
    ref = oracle_mod.route(layer_np, x_np, top_k=3)
    assert any(len({1, 2, 6} & set(r.tolist())) >= 2 for r in ref["ids"]), "fixture should produce ties"
    ids, w = _noalloc_routing(torch, layer_np, shape, x_np)
    assert np.array_equal(ids, ref["ids"])


def test_noalloc_rejects_batches_beyond_the_fixed_scratch(torch_cuda):
    torch = torch_cuda
    from nvfp4_weight_only_route_b200 import tfmoe
    E, H, k = 256, 64, 2
    T = tfmoe.ROUTE_NOALLOC_MAX_LOGITS // E + 1
    x = torch.zeros((T, H), dtype=torch.int16, device="cuda")
    rw = torch.zeros((E, H), dtype=torch.int16, device="cuda")
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    st = tfmoe.route_noalloc(x, rw, None, k, ids, w)
    assert st == tfmoe.ERR_INVALID_ARG
    assert "fixed scratch" in tfmoe.last_error()

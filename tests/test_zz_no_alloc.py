"""The allocation-free routing entry point (tfmoe_route_noalloc) matches the
routing that tfmoe_forward produces (needs a GPU).

It exists for callers that cannot allocate device memory -- a fixed memory
pool owned by someone else, real-time loops that cannot afford cudaMalloc's
latency or implicit synchronisation -- so it keeps its logits in a fixed array
inside the library. This file is collected last on purpose: if it fails, a run
stopped at the first failure has already run every other test. It must pass
alone in a fresh process as well.
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


def _reference_routing(torch, layer_np, shape, x_np):
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


def test_noalloc_routing_matches_forward_on_two_calls_in_a_row(torch_cuda):
    torch = torch_cuda
    cases = []
    s2 = synth.SHAPES[2]                       # batched decode with a Zipf router bias, T=256
    cases.append((synth.make_layer(s2, 4), s2, synth.make_x(s2, 4, 256)))
    s1 = synth.SHAPES[1]                       # decode, T=8 (the small-T router kernel)
    cases.append((synth.make_layer(s1, 1), s1, synth.make_x(s1, 1, 8)))
    for layer_np, shape, x_np in cases:        # two calls in a row, different sizes and kernels
        ids_ref, w_ref = _reference_routing(torch, layer_np, shape, x_np)
        ids, w = _noalloc_routing(torch, layer_np, shape, x_np)
        assert np.array_equal(ids, ids_ref)
        assert np.max(np.abs(w.astype(np.float64) - w_ref)) <= 2e-6


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

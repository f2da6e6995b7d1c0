"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Routing must match bit-exactly; every output element must satisfy
|gpu - oracle| <= 4e-3 * S + 1e-3 with S = sum_s g_s * sum_j |a_s[j] * w[h,j]|.
Small layers are compared in full. On the full-size prefill and large layers
the routing (logits, ids, weights) of every token is compared with the
oracle's routing step, and the layer output on a seeded sample of tokens
(each token's output depends only on its own row).
"""
import numpy as np
import pytest

from nvfp4_weight_only_route_b200 import synth

from gpu_harness import GpuLayerRun, check_intermediates, check_logits, check_output, check_routing, logit_bound
from layer_builders import bf16_bits

pytestmark = pytest.mark.gpu

REGIMES = {"gemv": 1, "mma": 2, "auto": 0}     # descriptor flags: FORCE_GEMV = 1, FORCE_MMA = 2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_weight_only_route_b200 import build
    build.build()


def _full_check(oracle_mod, layer, x, H, I, E, k, flags, max_tokens=None):
    T = x.shape[0]
    run = GpuLayerRun(layer, H, I, E, k, max_tokens or max(T, 1), flags=flags)
    try:
        g = run.forward(x)
    finally:
        run.close()
    o = oracle_mod.forward(layer, x, top_k=k, intermediates=True)
    check_routing(g, o, E, k, logit_bound(x, layer["router_w"], layer.get("router_bias")))
    check_intermediates(g, o, k)
    return check_output(g["out"], o)


@pytest.mark.parametrize("regime", sorted(REGIMES))
def test_tiny_layer(oracle_mod, regime):
    s = synth.SHAPES[0]
    layer = synth.make_layer(s, 0)
    x = synth.make_x(s, 0, 4)
    _full_check(oracle_mod, layer, x, s.H, s.I, s.E, s.k, REGIMES[regime])


@pytest.mark.parametrize("regime", sorted(REGIMES))
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_decode_layer(oracle_mod, seed, regime):
    s = synth.SHAPES[1]
    layer = synth.make_layer(s, seed)
    for T in s.T:
        x = synth.make_x(s, seed, T)
        _full_check(oracle_mod, layer, x, s.H, s.I, s.E, s.k, REGIMES[regime])


@pytest.mark.parametrize("regime", sorted(REGIMES))
def test_batched_decode_zipf(oracle_mod, regime):
    s = synth.SHAPES[2]
    layer = synth.make_layer(s, 4)
    x = synth.make_x(s, 4, 256)
    _full_check(oracle_mod, layer, x, s.H, s.I, s.E, s.k, REGIMES[regime])


@pytest.mark.parametrize("regime", sorted(REGIMES))
@pytest.mark.parametrize("H,I,E,k,T", [
    (384, 192, 6, 3, 1),       # 3 row tiles, 3 K tiles, ragged everything
    (384, 192, 6, 3, 37),
    (256, 320, 5, 2, 100),
    (128, 64, 4, 1, 9),        # smallest supported tile counts
    (512, 128, 8, 8, 13),      # k == E: every expert selected
])
def test_ragged_shapes(oracle_mod, regime, H, I, E, k, T):
    shape = synth.custom_shape(H, I, E, k, global_scale=0.05, router_std=1.0)
    layer = synth.make_layer(shape, 100 + T)
    x = synth.make_x(shape, 100 + T, T)
    _full_check(oracle_mod, layer, x, H, I, E, k, REGIMES[regime])


def _wide_range_x(T, H, seed):
    """Activations whose 16-element blocks span ~2^32: in every row, block 0 holds one
    element near 2^20 and fifteen near 2^-12; the other blocks are N(0, 1). Elements
    more than 2^28 below their group's largest are not exact f16 values after the
    power-of-two scaling of the 16-bit operand, so this checks that the loss stays
    inside the tolerance in both regimes."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H)).astype(np.float32)
    sign = np.where(rng.random((T, 16)) < 0.5, -1.0, 1.0).astype(np.float32)
    x[:, 0] = sign[:, 0] * np.float32(2.0 ** 20) * (1.0 + rng.random(T).astype(np.float32) / 4)
    x[:, 1:16] = sign[:, 1:] * np.float32(2.0 ** -12) * (1.0 + rng.random((T, 15)).astype(np.float32))
    return bf16_bits(x).reshape(T, H)


@pytest.mark.parametrize("regime", ["gemv", "mma"])
@pytest.mark.parametrize("H,I,E,k,T", [(384, 192, 6, 3, 37), (256, 320, 5, 2, 100)])
def test_wide_dynamic_range_activations(oracle_mod, regime, H, I, E, k, T):
    shape = synth.custom_shape(H, I, E, k, global_scale=0.05, router_std=1.0)
    layer = synth.make_layer(shape, 200 + T)
    x = _wide_range_x(T, H, 200 + T)
    _full_check(oracle_mod, layer, x, H, I, E, k, REGIMES[regime])


@pytest.mark.parametrize("H,I,E,k,T", [(256, 128, 32, 12, 40), (256, 128, 64, 20, 33)])
def test_large_top_k_on_the_tensor_core_router(oracle_mod, H, I, E, k, T):
    """k above 8 with more than 16 tokens: the tensor-core router's epilogue keeps 16 or 32 lower
    bounds (a looser, still valid threshold than the k-th), and the refinement selects k of the
    exact candidates."""
    shape = synth.custom_shape(H, I, E, k, global_scale=0.05, router_std=1.0)
    layer = synth.make_layer(shape, 300 + k)
    x = synth.make_x(shape, 300 + k, T)
    _full_check(oracle_mod, layer, x, H, I, E, k, REGIMES["auto"])


def test_router_exact_path_for_extreme_exponents(oracle_mod):
    """The exact router recomputation forms bf16 x bf16 products in fp32 when every product is
    a normal fp32 number, and in fp64 otherwise. Token 3 holds one element of 2^-120 (its
    products would be fp32 subnormals) and token 11 one of 2^126 (they could overflow); both
    must take the fp64 path, every other token the fp32-product one, and the routing of all
    40 tokens must equal the oracle's routing step bit for bit (ids and selected logits)."""
    import torch
    from nvfp4_weight_only_route_b200 import tfmoe
    H, I, E, k, T = 512, 256, 16, 4, 40
    shape = synth.custom_shape(H, I, E, k, global_scale=0.05, router_std=1.0)
    layer = synth.make_layer(shape, 77)
    # column 7 of the router weights at +-0.5, so that 2^126 there keeps every logit finite
    rw = layer["router_w"].copy()
    rw[:, 7] = np.where(rw[:, 7] & 0x8000, 0xBF00, 0x3F00).astype(np.uint16)
    layer["router_w"] = rw
    xf = (synth.make_x(shape, 77, T).astype(np.uint32) << 16).view(np.float32).copy()
    xf[3, 5] = np.float32(2.0 ** -120)
    xf[11, 7] = np.float32(2.0 ** 126)
    x = bf16_bits(xf).reshape(T, H)
    L = tfmoe.MoELayer(H, I, E, k, T)
    try:
        L.load_weights(tfmoe.layer_to_device(layer))
        xd = torch.from_numpy(x.view(np.int16)).cuda()
        out = torch.empty_like(xd)
        L.forward(xd, out)
        torch.cuda.synchronize()
        ids = L.buffer_tensor(tfmoe.BUF_TOPK_IDS, torch.int32, (T, k)).cpu().numpy()
        logits = L.buffer_tensor(tfmoe.BUF_LOGITS, torch.float32, (T, E)).cpu().numpy()
    finally:
        L.close()
    r = oracle_mod.route(layer, x, top_k=k)
    assert np.array_equal(ids, r["ids"])
    assert np.array_equal(np.take_along_axis(logits, r["ids"], 1), np.take_along_axis(r["logits"], r["ids"], 1))


@pytest.mark.parametrize("regime", sorted(REGIMES))
def test_single_expert_holds_every_token(oracle_mod, regime):
    H, I, E, k, T = 256, 128, 8, 2, 40
    shape = synth.custom_shape(H, I, E, k, global_scale=0.05, router_std=0.02)
    layer = synth.make_layer(shape, 7)
    bias = np.zeros(E, np.float32)
    bias[5] = 1000.0
    layer["router_bias"] = bias
    x = synth.make_x(shape, 7, T)
    _full_check(oracle_mod, layer, x, H, I, E, k, REGIMES[regime])


@pytest.mark.parametrize("regime", sorted(REGIMES))
def test_exact_logit_ties(oracle_mod, regime):
    H, I, E, k, T = 256, 128, 8, 3, 16
    shape = synth.custom_shape(H, I, E, k, global_scale=0.05, router_std=1.0)
    layer = synth.make_layer(shape, 8)
    rw = layer["router_w"].copy()
    rw[2] = rw[6] = rw[1]                 # three identical router rows: exact ties
    layer["router_w"] = rw
    x = synth.make_x(shape, 8, T)
    o = oracle_mod.forward(layer, x, top_k=k, intermediates=True)
    assert any(len({1, 2, 6} & set(r.tolist())) >= 2 for r in o["ids"]), "fixture should produce ties"
    _full_check(oracle_mod, layer, x, H, I, E, k, REGIMES[regime])


def test_zero_tokens_launches_nothing(oracle_mod):
    import torch
    s = synth.SHAPES[0]
    run = GpuLayerRun(synth.make_layer(s, 0), s.H, s.I, s.E, s.k, 4)
    try:
        x = torch.zeros((1, s.H), dtype=torch.int16, device="cuda")
        out = torch.full((1, s.H), 7, dtype=torch.int16, device="cuda")
        run.layer.forward(x, out, T=0)
        assert run.layer.last_launch_count() == 0
        assert int(out[0, 0]) == 7
    finally:
        run.close()


def test_max_tokens_and_over_limit(oracle_mod):
    import torch
    from nvfp4_weight_only_route_b200 import tfmoe
    s = synth.SHAPES[0]
    layer = synth.make_layer(s, 0)
    x = synth.make_x(s, 0, 6)
    _full_check(oracle_mod, layer, x, s.H, s.I, s.E, s.k, 0, max_tokens=6)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, 6)
    try:
        xt = torch.zeros((7, s.H), dtype=torch.int16, device="cuda")
        out = torch.zeros((7, s.H), dtype=torch.int16, device="cuda")
        with pytest.raises(tfmoe.TfmoeError) as ei:
            run.layer.forward(xt, out, T=7)
        assert ei.value.status == tfmoe.ERR_INVALID_ARG
        with pytest.raises(tfmoe.TfmoeError) as ei:
            run.layer.forward(xt, xt, T=2)          # out overlaps x
        assert ei.value.status == tfmoe.ERR_INVALID_ARG
        with pytest.raises(tfmoe.TfmoeError) as ei:   # misaligned x
            tfmoe.check(run.layer.forward_raw(xt.data_ptr() + 2, 1, out.data_ptr(), 0))
        assert ei.value.status == tfmoe.ERR_INVALID_ARG
    finally:
        run.close()


def test_forward_before_load_is_rejected():
    import torch
    from nvfp4_weight_only_route_b200 import tfmoe
    L = tfmoe.MoELayer(128, 64, 4, 1, 4)
    try:
        x = torch.zeros((1, 128), dtype=torch.int16, device="cuda")
        with pytest.raises(tfmoe.TfmoeError) as ei:
            L.forward(x, torch.zeros_like(x))
        assert ei.value.status == tfmoe.ERR_NOT_LOADED
    finally:
        L.close()


def test_deterministic_bytes(oracle_mod):
    s = synth.SHAPES[2]
    layer = synth.make_layer(s, 4)
    x = synth.make_x(s, 4, 256)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, 256)
    try:
        a = run.forward(x, intermediates=False)["out"]
        b = run.forward(x, intermediates=False)["out"]
    finally:
        run.close()
    assert a.tobytes() == b.tobytes()


def test_forward_host_matches_device(oracle_mod):
    import torch
    s = synth.SHAPES[1]
    layer = synth.make_layer(s, 1)
    x = synth.make_x(s, 1, 8)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, 8)
    try:
        dev = run.forward(x, intermediates=False)["out"]
        xh = torch.from_numpy(x.view(np.int16)).pin_memory()
        oh = torch.empty((8, s.H), dtype=torch.int16).pin_memory()
        stream = torch.cuda.Stream()
        run.layer.forward_host(xh, oh, stream=stream)
        assert np.array_equal(oh.numpy().view(np.uint16), dev)
        # another input (pageable buffers), then the first again: no state leaks between calls
        x2 = synth.make_x(s, 11, 8)
        dev2 = run.forward(x2, intermediates=False)["out"]
        oh2 = torch.empty((8, s.H), dtype=torch.int16)
        run.layer.forward_host(torch.from_numpy(x2.view(np.int16)), oh2, stream=stream)
        assert np.array_equal(oh2.numpy().view(np.uint16), dev2)
        run.layer.forward_host(xh, oh, stream=stream)
        assert np.array_equal(oh.numpy().view(np.uint16), dev)
        assert run.layer.last_launch_count() > 0
    finally:
        run.close()


def test_debug_checks_report_clean(oracle_mod):
    s = synth.SHAPES[1]
    layer = synth.make_layer(s, 2)
    x = synth.make_x(s, 2, 8)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, 8, flags=4)
    try:
        g = run.forward(x)
    finally:
        run.close()
    o = oracle_mod.forward(layer, x, top_k=s.k, intermediates=True)
    check_routing(g, o, s.E, s.k, logit_bound(x, layer["router_w"], layer.get("router_bias")))
    check_output(g["out"], o)


def _sampled_check(oracle_mod, run, layer, x, k, n_sample, seed):
    T = x.shape[0]
    g = run.forward(x, intermediates=True)
    # routing of every token against the oracle's routing step: bit-exact logits and ids
    r = oracle_mod.route(layer, x, top_k=k)
    n_ids = int(np.sum(np.any(g["ids"] != r["ids"], axis=1)))
    assert n_ids == 0, f"{n_ids} of {T} tokens select other experts than the oracle"
    check_logits(g["logits"], r["logits"], r["ids"], logit_bound(x, layer["router_w"], layer.get("router_bias")))
    assert np.max(np.abs(g["g"].astype(np.float64) - r["g"])) <= 2e-6
    rng = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([[0, T - 1], rng.choice(T, size=min(T, n_sample), replace=False)]))
    o = oracle_mod.forward(layer, x[idx], top_k=k, intermediates=True)
    assert np.array_equal(o["ids"], r["ids"][idx])
    # the plan of the whole batch: rows ordered by (expert, pair index)
    ids_all = g["ids"].ravel()
    E = g["counts"].shape[0]
    counts = np.bincount(ids_all, minlength=E)
    assert np.array_equal(g["counts"], counts)
    assert np.array_equal(g["offsets"], np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(g["perm"], np.argsort(ids_all, kind="stable"))
    assert np.array_equal(g["inv"][g["perm"]], np.arange(T * k))
    return check_output(g["out"][idx], o)


def test_prefill_layer_sampled(oracle_mod):
    s = synth.SHAPES[3]
    layer = synth.make_layer(s, 5)
    x = synth.make_x(s, 5, 8192)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, 8192)
    try:
        _sampled_check(oracle_mod, run, layer, x, s.k, 24, 5)
    finally:
        run.close()


@pytest.mark.parametrize("seed", synth.SHAPES[4].seeds)
def test_large_layer_sweep_sampled(oracle_mod, seed):
    """One large-sweep layer per seed (6..10), every T of the sweep."""
    s = synth.SHAPES[4]
    layer = synth.make_layer(s, seed)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, max(s.T))
    try:
        for T in s.T:
            x = synth.make_x(s, seed, T)
            _sampled_check(oracle_mod, run, layer, x, s.k, 6, 1000 * seed + T)
    finally:
        run.close()
        del layer


@pytest.mark.gpu
@pytest.mark.parametrize("regime", ["auto", "gemv"])
def test_large_batch_plan(oracle_mod, regime):
    """More than 4096 (token, expert) pairs: the plan is built by the multi-CTA scan; 601
    tokens leave a ragged last segment of one token."""
    s = synth.custom_shape(H=256, I=128, E=64, k=8)
    layer = synth.make_layer(s, 21)
    x = synth.make_x(s, 21, 601)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, 601, flags=REGIMES[regime])
    try:
        g = run.forward(x, intermediates=True)
        o = oracle_mod.forward(layer, x, top_k=s.k, intermediates=True)
        check_routing(g, o, s.E, s.k, logit_bound(x, layer["router_w"], layer.get("router_bias")))
        check_output(g["out"], o)
    finally:
        run.close()


def test_forced_timeout_reports_and_next_forward_is_clean(oracle_mod):
    """The failure path of a bounded device wait, made to run out on purpose: with
    TFMOE_FLAG_TEST_TIMEOUT one thread of the GEMV gate/up kernel's first CTA waits 1 ms
    on a barrier that nothing completes, takes the timeout path (error word, abort,
    drain of its copies in flight), and tfmoe_sync_status reports TFMOE_ERR_TIMEOUT.
    The context stays usable: the next forwards match the oracle."""
    from nvfp4_weight_only_route_b200 import tfmoe
    import torch
    s = synth.SHAPES[1]
    layer = synth.make_layer(s, 3)
    x = synth.make_x(s, 3, 8)
    bad = tfmoe.MoELayer(s.H, s.I, s.E, s.k, 8, flags=tfmoe.FLAG_TEST_TIMEOUT)
    try:
        bad.load_weights(tfmoe.layer_to_device(layer))
        xd = torch.from_numpy(x.view(np.int16)).cuda()
        out = torch.empty_like(xd)
        for _ in range(2):
            bad.forward(xd, out)
            assert bad.sync_status() == tfmoe.ERR_TIMEOUT
            assert "timed out" in tfmoe.last_error()
        assert bad.sync_status() == tfmoe.OK          # the word was cleared by the report
    finally:
        bad.close()
    _full_check(oracle_mod, layer, x, s.H, s.I, s.E, s.k, 0)


@pytest.mark.parametrize("value", [float("inf"), float("-inf")])
def test_debug_checks_flag_non_finite_logits(oracle_mod, value):
    """A non-finite activation (an input outside the contract, made on the host) gives
    non-finite router logits; with TFMOE_FLAG_DEBUG_CHECKS the routing kernels set the
    non-finite-logit bit and tfmoe_sync_status reports TFMOE_ERR_DEVICE. The next clean
    input on the same handle reports OK and matches the oracle."""
    from nvfp4_weight_only_route_b200 import tfmoe
    s = synth.SHAPES[1]
    layer = synth.make_layer(s, 2)
    run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, 8, flags=tfmoe.FLAG_DEBUG_CHECKS)
    try:
        for T in (8, 40):                     # the fused decode routing and the split router + top-k
            x = synth.make_x(s, 2, T)
            xf = ((x.astype(np.uint32) << 16).view(np.float32)).copy()
            xf[T // 2, 100] = value
            xbad = bf16_bits(xf).reshape(T, s.H)
            import torch
            xd = torch.from_numpy(xbad.view(np.int16)).cuda()
            out = torch.empty_like(xd)
            if T > 8:
                run.close()
                run = GpuLayerRun(layer, s.H, s.I, s.E, s.k, T, flags=tfmoe.FLAG_DEBUG_CHECKS)
            run.layer.forward(xd, out)
            assert run.layer.sync_status() == tfmoe.ERR_DEVICE
            assert "0x8" in tfmoe.last_error()
            g = run.forward(x)                # clean input: status OK (checked inside), oracle parity
            o = oracle_mod.forward(layer, x, top_k=s.k, intermediates=True)
            check_routing(g, o, s.E, s.k, logit_bound(x, layer["router_w"], layer.get("router_bias")))
            check_output(g["out"], o)
    finally:
        run.close()


def test_handles_of_different_shapes_coexist(oracle_mod):
    """Several handles of different layer shapes live in one process: one created later
    with a smaller layer must not break launches of an earlier, larger one (per-kernel
    settings such as the shared-memory limit are process-wide)."""
    big_s = synth.custom_shape(H=512, I=1024, E=8, k=2, global_scale=0.05, router_std=1.0)
    small_s = synth.custom_shape(H=128, I=64, E=4, k=1, global_scale=0.05, router_std=1.0)
    big_l, small_l = synth.make_layer(big_s, 41), synth.make_layer(small_s, 42)
    big = GpuLayerRun(big_l, 512, 1024, 8, 2, 40, flags=REGIMES["gemv"])
    small = GpuLayerRun(small_l, 128, 64, 4, 1, 40, flags=REGIMES["gemv"])
    try:
        for T in (5, 33):
            for run, layer, s in ((big, big_l, big_s), (small, small_l, small_s)):
                x = synth.make_x(s, 40 + T, T)
                g = run.forward(x)
                o = oracle_mod.forward(layer, x, top_k=s.k, intermediates=True)
                check_routing(g, o, s.E, s.k, logit_bound(x, layer["router_w"], layer.get("router_bias")))
                check_output(g["out"], o)
    finally:
        small.close()
        big.close()

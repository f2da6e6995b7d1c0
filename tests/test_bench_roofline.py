"""The bench's algorithmic work and roofline arithmetic (CPU only), checked against the
formulas of the measurement plan and against numbers of a recorded decode run."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_roofline_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_work_per_forward_decode_layer():
    b = _load_bench()
    H, I, E, k, T = 2048, 768, 128, 8, 8
    # one expert's three projections: 3 H I weights at 0.5 + 1/16 bytes each
    assert 3 * H * I * b.NVFP4_BYTES_PER_WEIGHT == 2_654_208
    nbytes, flops = b.work_per_forward(51.625, T, H, I, E, k)
    assert nbytes == pytest.approx(51.625 * 2_654_208 + E * H * 2 + T * H * 4)
    assert flops == 2 * T * k * 3 * H * I + 2 * T * H * E == 608_174_080
    # a recorded decode line: 137,613,312 algorithmic bytes per forward at 51.625 active experts
    assert nbytes == pytest.approx(137_613_312.0)


def test_gemv_roofline_is_weight_bytes_over_time():
    b = _load_bench()
    H, I = 2048, 768
    r = b.roofline_for("gemv_gate_up", 28.097362383037595, H, I, 51.0, 0.0, 0.0, 6555.5, 1636.3, True, 95639040, "t")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["algorithmic_bytes_per_launch"] == 51 * 2 * I * H * 0.5625 == 90_243_072
    assert r["achieved"] == pytest.approx(90_243_072 / 28.097362383037595e-6 / 1e9)
    assert r["frac"] == pytest.approx(0.48994, abs=1e-4)       # the recorded decode line
    assert r["traffic"] == 95639040 and r["peak_source"].startswith("measured")
    d = b.roofline_for("gemv_down", 10.0, H, I, 2.0, 0, 0, 6555.5, 1636.3, False, None, "t")
    assert d["algorithmic_bytes_per_launch"] == 2 * H * I * 0.5625 and d["peak_source"] == "fallback"


def test_tensor_core_roofline_follows_arithmetic_intensity():
    b = _load_bench()
    H, I = 4096, 1536
    # prefill gate/up: 65,536 pairs over all 128 experts -> tensor bound
    r = b.roofline_for("mma_gate_up", 1735.2, H, I, 0, 65536.0, 128.0, 6555.5, 1636.3, True, None, "t")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["algorithmic_flops_per_launch"] == pytest.approx(2 * 65536 * 2 * I * H)
    assert r["frac"] == pytest.approx(2 * 65536 * 2 * I * H / 1735.2e-6 / 1e12 / 1636.3)
    # a few tokens per expert stream weights -> HBM bound, on the weight bytes
    r = b.roofline_for("mma_down", 50.0, H, I, 0, 500.0, 100.0, 6555.5, 1636.3, True, None, "t")
    assert r["bound"] == "hbm"
    assert r["algorithmic_bytes_per_launch"] == pytest.approx(100 * H * I * 0.5625)
    # the switch sits at the ratio of the peaks: FLOPs per weight byte = 2 m / 0.5625 for m tokens per expert
    ridge = 1636.3e12 / 6555.5e9
    m_lo, m_hi = ridge * 0.5625 / 2 * 0.99, ridge * 0.5625 / 2 * 1.01
    assert b.roofline_for("mma_down", 1.0, H, I, 0, m_lo, 1.0, 6555.5, 1636.3, True, None, "")["bound"] == "hbm"
    assert b.roofline_for("mma_down", 1.0, H, I, 0, m_hi, 1.0, 6555.5, 1636.3, True, None, "")["bound"] == "tensor"


def test_other_kernels_report_no_fraction():
    b = _load_bench()
    r = b.roofline_for("combine", 3.0, 2048, 768, 0, 0, 0, 6555.5, 1636.3, True, None, "t")
    assert r["frac"] is None and r["achieved"] is None and r["avg_launch_us"] == 3.0


def test_both_arms_name_the_workload_alike():
    b = _load_bench()
    assert (b.workload_label("decode", 2048, 768, 128, 8, 8, (1, 2, 3))
            == "decode: H=2048 I=768 E=128 top-8 T=8 tokens/forward, seeds [1, 2, 3] rotated")


def test_shared_norm_workload_is_registered_and_labelled():
    b = _load_bench()
    assert "decode_shared_norm" in b.PER_CONFIG and b.SHARED_NORM["decode_shared_norm"] == 1
    si, T, seeds = b.WORKLOADS["decode_shared_norm"]
    assert (si, T) == b.WORKLOADS["decode"][:2]
    label = b.workload_label("decode_shared_norm", 2048, 768, 128, 8, T, seeds)
    assert "shared expert Is=768" in label and "tfmoe_forward_add_norm" in label
    assert "shared" not in b.workload_label("decode", 2048, 768, 128, 8, T, seeds)
    assert b.regime_of("decode_shared_norm") == "hbm"


def test_add_norm_layer_passes_its_buffers_and_delegates():
    """The bench's wrapper drives tfmoe_forward_add_norm with its own residual, norm weights and
    out_norm, and hands every other attribute to the layer (no GPU: a recording fake)."""
    b = _load_bench()

    class Buf:
        def __init__(self, p):
            self.p = p

        def data_ptr(self):
            return self.p

    calls = []

    class Lib:
        def tfmoe_forward_add_norm(self, *a):
            calls.append(a)
            return 0

    class Layer:
        lib, handle = Lib(), 77

        def last_launch_count(self):
            return 5

    w = b.AddNormLayer(Layer(), Buf(100), Buf(200), Buf(300))
    assert w.forward_raw(1000, 8, 2000, 9) == 0
    assert calls == [(77, 1000, 8, 100, 200, 2000, 300, 9)]
    assert w.last_launch_count() == 5 and w.handle == 77

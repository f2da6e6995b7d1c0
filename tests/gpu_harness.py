"""Run the CUDA layer through the C ABI and compare it with the oracle.

Everything compared here is checked against values the oracle computes from
the same seeded inputs; nothing expected comes from the CUDA path.
"""
from __future__ import annotations

import numpy as np

BF16_ULP_REL = 2.0 ** -7


def bf16_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class GpuLayerRun:
    def __init__(self, layer_np, H, I, E, k, max_tokens, flags=0, gemv_max_tokens=0):
        import torch
        from nvfp4_weight_only_route_b200 import tfmoe
        self.torch = torch
        self.tfmoe = tfmoe
        self.H, self.I, self.E, self.k = H, I, E, k
        self.layer = tfmoe.MoELayer(H, I, E, k, max_tokens, has_router_bias=layer_np.get("router_bias") is not None,
                                    flags=flags, gemv_max_tokens=gemv_max_tokens)
        dev = tfmoe.layer_to_device(layer_np)
        self.layer.load_weights(dev)
        del dev
        torch.cuda.synchronize()

    def forward(self, x_np, intermediates=True):
        torch, tfmoe = self.torch, self.tfmoe
        T = x_np.shape[0]
        x = torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).cuda()
        out = torch.empty((T, self.H), dtype=torch.int16, device="cuda")
        self.layer.forward(x, out, T=T)
        st = self.layer.sync_status()
        assert st == 0, tfmoe.last_error()
        res = {"out": out.cpu().numpy().view(np.uint16), "launches": self.layer.last_launch_count()}
        if intermediates and T > 0:
            P = T * self.k
            L = self.layer
            res["logits"] = L.buffer_tensor(tfmoe.BUF_LOGITS, torch.float32, (T, self.E)).cpu().numpy()
            res["ids"] = L.buffer_tensor(tfmoe.BUF_TOPK_IDS, torch.int32, (T, self.k)).cpu().numpy()
            res["g"] = L.buffer_tensor(tfmoe.BUF_TOPK_WEIGHTS, torch.float32, (T, self.k)).cpu().numpy()
            res["counts"] = L.buffer_tensor(tfmoe.BUF_EXPERT_COUNTS, torch.int32, (self.E,)).cpu().numpy()
            res["offsets"] = L.buffer_tensor(tfmoe.BUF_EXPERT_OFFSETS, torch.int32, (self.E + 1,)).cpu().numpy()
            res["perm"] = L.buffer_tensor(tfmoe.BUF_PERM, torch.int32, (P,)).cpu().numpy()
            res["inv"] = L.buffer_tensor(tfmoe.BUF_INV, torch.int32, (P,)).cpu().numpy()
            res["regime"] = L.buffer_tensor(tfmoe.BUF_REGIME, torch.int32, (self.E,)).cpu().numpy()
            res["act"] = L.buffer_tensor(tfmoe.BUF_ACT, torch.int16, (P, self.I)).cpu().numpy().view(np.uint16)
            res["y"] = L.buffer_tensor(tfmoe.BUF_EXPERT_OUT, torch.float32, (P, self.H)).cpu().numpy()
        return res

    def close(self):
        self.layer.close()


def logit_bound(x_bits, w_bits, bias=None):
    """The bound on |approximate - exact| router logit the library states for the experts it
    does not recompute exactly: (H + 34) 2^-22 ||x_t|| ||w_e|| + 2^-21 |bias_e| (with a 1 %
    margin)."""
    xf, wf = bf16_to_f64(x_bits), bf16_to_f64(w_bits)
    H = xf.shape[1]
    b = 0.0 if bias is None else 2.0 ** -21 * np.abs(np.asarray(bias, np.float64))[None, :]
    return ((H + 34) * 2.0 ** -22 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) + b) * 1.01 + 1e-6


def check_logits(g_logits, o_logits, ids, bound=None):
    """The logits of the selected experts are bit-exact. Every other entry is either exact or,
    for batches routed through the tensor-core approximation, within `bound` of it."""
    sel_g = np.take_along_axis(g_logits, ids, axis=1)
    sel_o = np.take_along_axis(o_logits, ids, axis=1)
    n_bad = int(np.sum(sel_g != sel_o))
    assert n_bad == 0, f"{n_bad} router logits of selected experts differ from the oracle"
    diff = np.abs(g_logits.astype(np.float64) - o_logits.astype(np.float64))
    if bound is None:
        assert np.all(diff == 0), f"{int(np.sum(diff != 0))} router logits differ from the oracle"
    else:
        assert np.all(diff <= bound), f"router logits off by more than the stated bound: {float(np.max(diff / bound)):.3f}"


def check_routing(g, o, E, k, bound=None):
    """Router logits (selected ones bit-exact), ids (bit-exact), weights; then the expert
    permutation."""
    T = o["ids"].shape[0]
    assert np.array_equal(g["ids"], o["ids"]), "top-k ids differ from the oracle"
    check_logits(g["logits"], o["logits"], o["ids"], bound)
    assert np.max(np.abs(g["g"].astype(np.float64) - o["g"])) <= 2e-6
    ids = o["ids"].ravel()
    counts = np.bincount(ids, minlength=E)
    assert np.array_equal(g["counts"], counts)
    offs = np.concatenate([[0], np.cumsum(counts)])
    assert np.array_equal(g["offsets"], offs)
    perm = np.argsort(ids, kind="stable")           # rows ordered by (expert, pair index)
    assert np.array_equal(g["perm"], perm)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(T * k)
    assert np.array_equal(g["inv"], inv)


def check_intermediates(g, o, k):
    perm = g["perm"]
    I = o["a"].shape[2]
    H = o["y"].shape[2]
    a_o = o["a"].reshape(-1, I)[perm]
    a_g = g["act"]
    va, vg = bf16_to_f64(a_o), bf16_to_f64(a_g)
    exact = np.mean(a_o == a_g)
    assert exact >= 0.98, f"only {exact:.4f} of SwiGLU outputs equal the oracle's"
    # differences beyond a rounding flip must be explained by fp32-vs-fp64 accumulation
    big = np.abs(va - vg) > 2 * BF16_ULP_REL * np.maximum(np.abs(va), np.abs(vg)) + 1e-6
    assert np.mean(big) < 1e-4, f"{int(big.sum())} SwiGLU outputs differ by more than two bf16 ulps"
    y_o = o["y"].reshape(-1, H)[perm]
    yabs = o["yabs"].reshape(-1, H)[perm]
    err = np.abs(g["y"].astype(np.float64) - y_o)
    tol = 4e-3 * yabs + 1e-3
    assert np.all(err <= tol), f"expert outputs: max err/tol {np.max(err / tol):.3f}"


def bf16_half_ulp(v):
    """Half the bf16 quantum at |v| (the error of one final round-to-nearest)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 0.5 * 2.0 ** (np.floor(np.log2(a)) - 7)


def check_output(g_out, o):
    """|gpu - oracle| <= 4e-3*S + 1e-3 applied to the computed value: the GPU's bf16
    output against the oracle's unrounded fp64 output, plus the half ulp of the one
    final bf16 rounding (both sides round once; two independent roundings of values
    that differ by less than the bound can land one bf16 ulp apart, which on layers
    with little cancellation exceeds 4e-3*S)."""
    g = bf16_to_f64(g_out)
    err = np.abs(g - o["out64"])
    tol = 4e-3 * o["S"] + 1e-3 + bf16_half_ulp(np.maximum(np.abs(g), np.abs(o["out64"])))
    worst = float(np.max(err / tol)) if err.size else 0.0
    assert np.all(err <= tol), f"output outside |gpu-oracle| <= 4e-3*S + 1e-3 (+ final rounding): worst {worst:.3f}"
    # the oracle's own bf16 output must agree with the GPU's except for rounding flips
    flips = g != bf16_to_f64(o["out"])
    assert np.all(np.abs(g - bf16_to_f64(o["out"]))[flips] <= 2 * bf16_half_ulp(g[flips]) + 4e-3 * o["S"][flips] + 1e-3)
    return worst

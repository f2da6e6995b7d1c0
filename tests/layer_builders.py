"""Hand-built layers in the canonical layout, for closed-form tests."""
import numpy as np
import torch


def bf16_bits(values):
    return torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def constant_layer(H, I, E, *, gate_code=0x2, up_code=0x4, down_code=0x2, scale_byte=0x38,
                   gate_global=1.0, up_global=1.0, down_global=1.0, router_rows=None, bias=None):
    """Every gate/up/down element of every expert holds one E2M1 code, every block
    scale one E4M3 byte; the codes may be given per expert as lists."""
    def codes(code, rows, K):
        code = np.broadcast_to(np.asarray(code, dtype=np.uint8).reshape(-1, 1, 1), (E, 1, 1))
        byte = (code | (code << 4)).astype(np.uint8)
        return np.ascontiguousarray(np.broadcast_to(byte, (E, rows, K // 2)))

    def scales(rows, K):
        return np.full((E, rows, K // 16), scale_byte, dtype=np.uint8)

    if router_rows is None:
        router_rows = np.zeros((E, H), dtype=np.float32)
    layer = {
        "router_w": bf16_bits(router_rows).reshape(E, H),
        "router_bias": None if bias is None else np.asarray(bias, dtype=np.float32),
        "gate_codes": codes(gate_code, I, H), "up_codes": codes(up_code, I, H),
        "gate_scales": scales(I, H), "up_scales": scales(I, H),
        "gate_global": np.full(E, gate_global, np.float32) if np.isscalar(gate_global) else np.asarray(gate_global, np.float32),
        "up_global": np.full(E, up_global, np.float32) if np.isscalar(up_global) else np.asarray(up_global, np.float32),
        "down_codes": codes(down_code, H, I), "down_scales": scales(H, I),
        "down_global": np.full(E, down_global, np.float32) if np.isscalar(down_global) else np.asarray(down_global, np.float32),
    }
    return layer


def unit_x(T, H, col=0, value=1.0):
    x = np.zeros((T, H), dtype=np.float32)
    x[:, col] = value
    return bf16_bits(x).reshape(T, H)

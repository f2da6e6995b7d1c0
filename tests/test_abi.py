"""The C-ABI library loads and exports what include/tfmoe.h declares; host-side
argument checks work without a GPU (no kernel is launched here)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tfmoe.h")


@pytest.fixture(scope="module")
def tf():
    from nvfp4_weight_only_route_b200 import build, tfmoe
    build.build()
    tfmoe.load_library()
    return tfmoe


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TFMOE_API\s+[\w\s\*]+?\b(tfmoe_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("tfmoe_create", "tfmoe_load_weights", "tfmoe_forward", "tfmoe_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(tf):
    lib = ctypes.CDLL(tf.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(tf.EXPORTED) == declared_functions()


def test_struct_layout_matches_header(tf):
    src = """
#include <stdio.h>
#include <stddef.h>
#include "tfmoe.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu\\n", sizeof(tfmoe_layer_desc), offsetof(tfmoe_layer_desc, gemv_max_tokens),
         sizeof(tfmoe_weights), offsetof(tfmoe_weights, down_global), offsetof(tfmoe_layer_desc, shared_intermediate),
         offsetof(tfmoe_layer_desc, norm_eps), offsetof(tfmoe_weights, shared_down_global));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        got = [int(v) for v in subprocess.check_output([exe]).split()]
    want = [ctypes.sizeof(tf.LayerDesc), tf.LayerDesc.gemv_max_tokens.offset,
            ctypes.sizeof(tf.Weights), tf.Weights.down_global.offset, tf.LayerDesc.shared_intermediate.offset,
            tf.LayerDesc.norm_eps.offset, tf.Weights.shared_down_global.offset]
    assert got == want


def _create(tf, **kw):
    d = dict(hidden=512, intermediate=256, num_experts=8, top_k=2, max_tokens=4, has_router_bias=0,
             flags=0, gemv_max_tokens=0, shared_intermediate=0, norm_eps=1e-6)
    d.update(kw)
    desc = tf.LayerDesc(**d)
    h = ctypes.c_void_p()
    st = tf.load_library().tfmoe_create(ctypes.byref(desc), ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("kw,status", [
    (dict(hidden=500), 1), (dict(intermediate=0), 1), (dict(top_k=9), 1), (dict(top_k=0), 1),
    (dict(max_tokens=0), 1), (dict(flags=3), 1), (dict(flags=0x100), 1),
    (dict(hidden=528), 5), (dict(intermediate=80), 5), (dict(num_experts=300, top_k=2), 5),
    # limits of the library: the reduction length a GEMV task's scale copy covers (256 tiles of 64),
    # top_k <= 32 (one warp per token in top-k), 32-bit offsets of the permuted activation rows
    (dict(hidden=16384 + 128), 5), (dict(intermediate=16384 + 64), 5),
    (dict(num_experts=64, top_k=33), 5),
    (dict(max_tokens=(1 << 31) // 8, top_k=8, num_experts=8), 5),
    (dict(hidden=4096, max_tokens=131072, top_k=8, num_experts=8), 5),
    # the shared expert: a multiple of the routed width; its slots count against E and k
    (dict(shared_intermediate=128), 1), (dict(shared_intermediate=-256), 1),
    (dict(norm_eps=-1.0), 1), (dict(norm_eps=float("nan")), 1), (dict(norm_eps=float("inf")), 1),
    (dict(num_experts=255, shared_intermediate=512), 5),
    (dict(num_experts=64, top_k=31, shared_intermediate=512), 5),
])
def test_create_rejects_bad_descriptors_without_gpu(tf, kw, status):
    st, h = _create(tf, **kw)
    assert st == status and not h.value
    assert tf.last_error()


def test_create_null_arguments(tf):
    lib = tf.load_library()
    h = ctypes.c_void_p()
    assert lib.tfmoe_create(None, ctypes.byref(h)) == tf.ERR_INVALID_ARG
    desc = tf.LayerDesc(512, 256, 8, 2, 4, 0, 0, 0)
    assert lib.tfmoe_create(ctypes.byref(desc), None) == tf.ERR_INVALID_ARG


def test_injected_allocation_failure(tf, monkeypatch):
    monkeypatch.setenv("TFMOE_FAIL_ALLOC", "1")
    st, h = _create(tf)
    assert st == tf.ERR_OOM and not h.value
    assert "injected" in tf.last_error()


def test_null_handle_calls(tf):
    lib = tf.load_library()
    assert lib.tfmoe_forward(None, None, 1, None, None) == tf.ERR_INVALID_ARG
    assert lib.tfmoe_forward_host(None, None, 1, None, None) == tf.ERR_INVALID_ARG
    assert lib.tfmoe_forward_add_norm(None, None, 1, None, None, None, None, None) == tf.ERR_INVALID_ARG
    assert lib.tfmoe_load_weights(None, None) == tf.ERR_INVALID_ARG
    assert lib.tfmoe_sync_status(None, None) == tf.ERR_INVALID_ARG
    p, n = ctypes.c_void_p(), ctypes.c_size_t()
    assert lib.tfmoe_get_buffer(None, 0, ctypes.byref(p), ctypes.byref(n)) == tf.ERR_INVALID_ARG
    assert lib.tfmoe_last_launch_count(None) == 0
    lib.tfmoe_destroy(None)

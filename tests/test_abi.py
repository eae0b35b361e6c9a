"""The C ABI library loads on a machine without a GPU, exports every symbol
include/kd.h declares, and rejects bad arguments on the host (no device
calls are made on these paths)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kd():
    from moe_decode_layer_skinny_b200 import build
    build.build()
    import moe_decode_layer_skinny_b200 as kd
    kd.lib()
    return kd


def declared_functions():
    src = ""
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src += open(os.path.join(ROOT, "include", f)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(kd_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_binding_exports(kd):
    decl = declared_functions()
    assert "kd_decode_layer" in decl and "kd_layer_create" in decl
    assert set(decl) == set(kd.EXPORTS)


def test_library_exports_every_declared_symbol(kd):
    L = ctypes.CDLL(kd.SO_PATH)
    for name in declared_functions():
        assert hasattr(L, name), name


def test_host_side_argument_errors(kd):
    L = kd.lib()
    h = ctypes.c_void_p()
    assert L.kd_layer_create(None, 0, ctypes.byref(h)) == kd.KD_EINVAL
    # invalid configurations are rejected before any device call
    bad = [dict(hidden=100), dict(top_k=0), dict(top_k=9, n_experts=8), dict(max_tokens=65),
           dict(max_tokens=0), dict(wdtype=7), dict(n_shared=2), dict(inter=96), dict(n_experts=2000),
           dict(hidden=32768), dict(mma_min_tokens=-1), dict(bias_select_only=3)]
    for b in bad:
        f = dict(hidden=256, q_heads=4, kv_heads=1, head_dim=64, n_experts=8, top_k=2,
                 n_shared=1, inter=128, wdtype=0, layer_id=0, max_tokens=4, router_bias=None,
                 mma_min_tokens=0)
        f.update(b)
        cfg = kd._Config(**f)
        assert L.kd_layer_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == kd.KD_EINVAL, b
        assert kd.lib().kd_last_error().decode()
    # full-layer geometry the attention kernels do not take
    for b in [dict(head_dim=96), dict(kv_heads=0), dict(q_heads=6, kv_heads=2, head_dim=128),
              dict(kv_n_seq=0), dict(kv_max_ctx=0), dict(k_scale=0.0), dict(full_layer=2)]:
        f = dict(hidden=256, q_heads=4, kv_heads=1, head_dim=64, n_experts=8, top_k=2,
                 n_shared=1, inter=128, wdtype=0, layer_id=0, max_tokens=4, router_bias=None,
                 mma_min_tokens=0, full_layer=1, rms_eps=0.0, kv_n_seq=2, kv_max_ctx=16,
                 k_scale=0.01, v_scale=0.01)
        f.update(b)
        cfg = kd._Config(**f)
        assert L.kd_layer_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == kd.KD_EINVAL, b
    assert L.kd_decode_layer(None, None, None, 1, None) == kd.KD_EINVAL
    assert L.kd_decode_layer_full(None, None, None, None, None, None, 1, None) == kd.KD_EINVAL
    assert L.kd_layer_check(None) == kd.KD_EINVAL
    assert L.kd_layer_qkv(None) is None
    assert L.kd_layer_bytes(None, None, None) == kd.KD_EINVAL
    assert L.kd_layer_launches(None, 1) == kd.KD_EINVAL
    assert L.kd_layer_prefetch_l2(None, 0, None) == kd.KD_EINVAL
    assert L.kd_layer_set_timing_events(None, None, 0) == kd.KD_EINVAL
    assert L.kd_stack_create(None, 0, 1, 0, ctypes.byref(h)) == kd.KD_EINVAL
    assert L.kd_stack_run(None, None, None, None) == kd.KD_EINVAL
    assert L.kd_router_topk_static(None, None, 0, None, None, 1, 256, 8, 2, None, None, None) == kd.KD_EINVAL
    L.kd_layer_destroy(None)
    L.kd_stack_destroy(None)
    assert "kd_router_topk_static" in kd.lib().kd_last_error().decode()


def test_product_path_does_not_touch_the_oracle():
    # the package and bench's GPU arm never import oracle/; only tests, smoke
    # and the CPU-baseline leg do
    pkg = os.path.join(ROOT, "moe_decode_layer_skinny_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "orc.h" not in txt, f

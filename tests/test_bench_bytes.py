"""The algorithmic byte counts behind bench.py's HBM roofline, for the
H=7168 layer: each weight matrix's bytes written out from its shape."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import moe_decode_layer_skinny_b200 as kd  # noqa: E402
from kdgen import K2  # noqa: E402

MB = 1024 * 1024


def test_bf16_kernel_bytes_batch1():
    spec = kd.LayerSpec.from_dims(K2, wdtype=0)
    kb = bench.kernel_bytes(spec, n_active=8)
    # QKV 10240 x 7168 and o-proj 7168 x 8192, 2 bytes each
    assert kb["proj"] == (10240 * 7168 + 7168 * 8192) * 2
    assert kb["router"] == 256 * 7168 * 2
    # per routed expert: gate + up 2 x 2048 x 7168, down 7168 x 2048
    assert kb["gateup"] == 8 * 2 * 2048 * 7168 * 2
    # the down launch also streams the shared expert's down projection
    assert kb["down"] == 9 * 7168 * 2048 * 2
    assert kb["gateup"] == 469762048   # the figure profiles/traffic.json compares with


def test_fp8_kernel_bytes_count_block_scales():
    spec = kd.LayerSpec.from_dims(K2, wdtype=1)
    kb = bench.kernel_bytes(spec, n_active=1)
    scales = lambda r, k: ((r + 127) // 128) * ((k + 127) // 128) * 4
    assert kb["proj"] == 10240 * 7168 + 7168 * 8192 + scales(10240, 7168) + scales(7168, 8192)
    assert kb["gateup"] == 2 * 2048 * 7168 + 2 * scales(2048, 7168)
    assert kb["down"] == 2 * (7168 * 2048 + scales(7168, 2048))

"""kd_router_topk_static: the router top-k for callers that cannot allocate
device memory (a runtime whose device memory belongs to another allocator, a
plugin handed only its inputs and outputs).  Its scratch is a fixed
__device__ array inside the library; here its output is checked, through the
C ABI, against the router of kd_decode_layer on the same weights and h1, on
two calls in a row, and the device's free memory is checked to be the same
before and after a call.  This file is collected last on purpose."""
import gc

import numpy as np
import pytest

import kdgen
from kdgen import K2, TINY, Dims
from kdtest import fetch, torch_bf16

pytestmark = pytest.mark.gpu


def _case(kd, torch, dims, wdtype, bias, M):
    # the layer's CUDA-core router (the tensor-core one rounds differently)
    spec = kd.LayerSpec.from_dims(dims, wdtype=wdtype, max_tokens=M, router_bias=bias,
                                  mma_min_tokens=1000)
    layer = kd.Layer(spec, seed=0)
    try:
        x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, dims.hidden, 0.3)
        a = kdgen.activations(0, 0, kdgen.ATTN_OUT, M, dims.attn, 0.3)
        h = torch_bf16(x)
        layer.decode(h, torch_bf16(a), M)
        torch.cuda.synchronize()
        layer.check()
        E, k, H = dims.n_experts, dims.top_k, dims.hidden
        ref_idx = fetch(layer.debug_ptr(kd.T_IDX), (M, k), np.int32)
        ref_gates = fetch(layer.debug_ptr(kd.T_GATES), (M, k), np.float32)
        h1 = torch.from_numpy(fetch(layer.debug_ptr(kd.T_H1F), (M, H), np.float32)).cuda()
        if wdtype == kd.KD_WBF16:
            wr = torch_bf16(layer.read_weight(3, -1, 0, E))
            sc = None
        else:
            codes, scales = layer.read_weight(3, -1, 0, E)
            wr = torch.from_numpy(codes).cuda()
            sc = torch.from_numpy(scales).cuda()
        b = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
        idx = torch.full((M, k), -1, dtype=torch.int32, device="cuda")
        gates = torch.zeros((M, k), dtype=torch.float32, device="cuda")
        for call in range(2):
            idx.fill_(-1)
            gates.zero_()
            gc.collect()   # objects of earlier tests freed now, not inside the window
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info()[0]
            alloc0 = torch.cuda.memory_allocated()
            kd.router_topk_static(wr, sc, wdtype, b, h1, M, H, E, k, idx, gates)
            torch.cuda.synchronize()
            if call == 1:   # the first call may load the library's module
                assert torch.cuda.mem_get_info()[0] == free0
            assert torch.cuda.memory_allocated() == alloc0
            assert np.array_equal(idx.cpu().numpy(), ref_idx)
            assert np.abs(gates.cpu().numpy() - ref_gates).max() < 1e-4
    finally:
        layer.close()


def test_static_router_matches_layer_router(torch_cuda):
    import moe_decode_layer_skinny_b200 as kd
    torch = torch_cuda
    _case(kd, torch, TINY, kd.KD_WBF16, kdgen.zipf_bias(8, 1.1), 13)
    _case(kd, torch, Dims(256, 4, 1, 64, 16, 4, 1, 128), kd.KD_WFP8, None, 5)
    _case(kd, torch, K2, kd.KD_WBF16, None, 8)


def test_static_router_rejects_sizes_beyond_its_scratch(torch_cuda):
    import moe_decode_layer_skinny_b200 as kd
    torch = torch_cuda
    h1 = torch.zeros((65, 256), dtype=torch.float32, device="cuda")
    wr = torch.zeros((2048, 256), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((65, 16), dtype=torch.int32, device="cuda")
    g = torch.zeros((65, 16), dtype=torch.float32, device="cuda")
    for M, E, k, H in [(65, 8, 2, 256), (4, 1025, 2, 256), (4, 64, 17, 256), (4, 8, 2, 8320)]:
        # through the C ABI directly (the binding would refuse the short buffers)
        rc = kd.lib().kd_router_topk_static(wr.data_ptr(), None, kd.KD_WBF16, None, h1.data_ptr(),
                                            M, H, E, k, idx.data_ptr(), g.data_ptr(), None)
        assert rc == kd.KD_ERANGE, (M, E, k, H)
        assert "static limits" in kd.lib().kd_last_error().decode()
    # the binding checks its tensors before the call
    with pytest.raises(ValueError):
        kd.router_topk_static(wr, None, kd.KD_WBF16, None, h1[:, :128], 4, 256, 8, 2, idx, g)
    with pytest.raises(ValueError):
        kd.router_topk_static(wr, None, kd.KD_WBF16, None, h1, 4, 256, 8, 2, idx.long(), g)

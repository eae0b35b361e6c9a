"""Failure detection on the GPU without a fault: a bounded wait that runs out.

With KD_TEST_STALL_WAIT=1 the layer's tensor-core kernels first wait on a
pipeline barrier that nothing completes.  The wait gives up after its limit
(2 s), raises the CTA's abort flag and records the error; every role stops at
its first blocked wait, drains what it has in flight (TMA loads, MMAs, cp.async
copies) and returns.  The host reads KD_ETIMEOUT from kd_layer_check, and the
context stays usable: another layer on the same device then gives the same
bits as before the stalled call."""
import time

import numpy as np
import pytest

import kdgen
from kdtest import torch_bf16, torch_bits

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_device_stays_usable(torch_cuda, monkeypatch):
    import moe_decode_layer_skinny_b200 as kd
    torch = torch_cuda
    dims, M = kdgen.TINY, 4   # M >= 3: the tensor-core kernels
    x = kdgen.activations(0, 0, kdgen.HIDDEN_IN, M, dims.hidden)
    a = kdgen.activations(0, 0, kdgen.ATTN_OUT, M, dims.attn)
    good = kd.Layer(kd.LayerSpec.from_dims(dims, max_tokens=M), seed=0)
    monkeypatch.setenv("KD_TEST_STALL_WAIT", "1")
    stalled = kd.Layer(kd.LayerSpec.from_dims(dims, max_tokens=M), seed=0)
    monkeypatch.delenv("KD_TEST_STALL_WAIT")
    try:
        h = torch_bf16(x)
        good.decode(h, torch_bf16(a), M)
        good.check()
        ref = torch_bits(h)

        h2 = torch_bf16(x)
        t0 = time.time()
        stalled.decode(h2, torch_bf16(a), M)
        with pytest.raises(kd.KdError) as e:
            stalled.check()          # synchronises: every stalled kernel gave up
        assert e.value.code == kd.KD_ETIMEOUT
        assert time.time() - t0 >= 1.9   # the limit, not an early exit
        # the error word was read and cleared; the device answers
        torch.cuda.synchronize()
        h3 = torch_bf16(x)
        good.decode(h3, torch_bf16(a), M)
        good.check()
        assert np.array_equal(torch_bits(h3), ref)
    finally:
        stalled.close()
        good.close()

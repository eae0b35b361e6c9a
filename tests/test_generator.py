"""Pins of the seeded input generator (kdgen): published splitmix64 outputs,
moments of the Irwin-Hall(4) normal, and its bf16 / e4m3 encoders against
torch's own conversions."""
import numpy as np
import pytest
import torch

import kdgen


def test_splitmix64_published_sequence():
    # splitmix64 seeded with state 0 (Steele, Lea & Flood 2014; Vigna's public
    # reference implementation) yields these first three outputs.  Our mix(z)
    # is the output function applied to z + gamma, so output n = mix(n * gamma).
    gamma = 0x9E3779B97F4A7C15
    expect = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    for n, e in enumerate(expect):
        assert kdgen.mix((n * gamma) & (2**64 - 1)) == e


def test_ih4_is_sum_of_four_fields():
    L = kdgen.lib()
    rng = np.random.default_rng(1)
    for u in rng.integers(0, 2**63, 200, dtype=np.int64).tolist() + [0, 2**64 - 1]:
        u = int(u) & (2**64 - 1)
        s = sum((u >> (16 * i)) & 0xFFFF for i in range(4)) - 131070
        assert L.kdg_host_ih4(u) == s


def test_unit_normal_moments():
    v = kdgen.values(0, kdgen.uid(0, kdgen.HIDDEN_IN), 0, 2_000_000, kdgen.UNIT).astype(np.float64)
    assert abs(v.mean()) < 2e-3
    assert abs(v.var() - 1.0) < 3e-3
    # Irwin-Hall(4) rescaled is bounded by sqrt(3) * 2 = 3.4641...
    assert np.abs(v).max() <= 131070 * kdgen.UNIT * (1 + 1e-7)
    # the constant is fp32(sqrt(3/(2^32-1)))
    assert kdgen.UNIT == float(np.float32(np.sqrt(3.0 / (2**32 - 1))))
    assert kdgen.W002 == float(np.float32(0.02 * np.sqrt(3.0 / (2**32 - 1))))


def test_weight_sigma():
    v = kdgen.values(0, kdgen.uid(0, kdgen.QKV), 0, 1_000_000, kdgen.W002).astype(np.float64)
    assert abs(v.std() - 0.02) < 1e-4


def test_streams_differ_by_uid_and_seed():
    a = kdgen.values(0, kdgen.uid(0, kdgen.GATE, 1), 0, 1000)
    b = kdgen.values(0, kdgen.uid(0, kdgen.GATE, 2), 0, 1000)
    c = kdgen.values(1, kdgen.uid(0, kdgen.GATE, 1), 0, 1000)
    d = kdgen.values(0, kdgen.uid(1, kdgen.GATE, 1), 0, 1000)
    for o in (b, c, d):
        assert abs(np.corrcoef(a, o)[0, 1]) < 0.15
        assert not np.array_equal(a, o)


def test_bf16_matches_torch_rne():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32),
        (rng.standard_normal(10_000) * 1e-30).astype(np.float32),
        # exact ties between two bf16 neighbours
        ((np.arange(1, 5000, dtype=np.uint32) << 16) | 0x8000).view(np.float32),
        ((np.arange(1, 5000, dtype=np.uint32) << 16) | 0x7FFF).view(np.float32),
    ])
    ours = kdgen.to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_e4m3_matches_torch_in_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.uniform(-448, 448, 200_000).astype(np.float32),
        (rng.standard_normal(100_000) * 0.01).astype(np.float32),   # subnormal range
        # every code's value and every midpoint between neighbouring codes
        np.array([float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float())
                  for c in range(256) if (c & 0x7F) != 0x7F], np.float32),
    ])
    vals = np.sort(np.unique(np.abs(torch.arange(0, 127, dtype=torch.uint8)
                                    .view(torch.float8_e4m3fn).float().numpy())))
    mids = ((vals[1:].astype(np.float64) + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.float32([0.0, -0.0, 448.0, -448.0])])
    ours = kdgen.to_e4m3_codes(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # +-0: torch keeps the sign bit, so do we
    assert np.array_equal(ours, ref)


def test_e4m3_saturates():
    x = np.float32([449.0, 464.0, 1e6, 3e38, -500.0, -1e9])
    codes = kdgen.to_e4m3_codes(x)
    assert list(codes) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_fp8_block_quantisation():
    codes, scales = kdgen.weight_fp8(0, 0, kdgen.GATE, 1, 256, 384)
    ref = kdgen.values(0, kdgen.uid(0, kdgen.GATE, 1), 0, 256 * 384, kdgen.W002).reshape(256, 384)
    deq = (torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy())
    for rb in range(2):
        for kb in range(3):
            blk = ref[rb * 128:(rb + 1) * 128, kb * 128:(kb + 1) * 128]
            amax = np.abs(blk).max()
            assert scales[rb, kb] == np.float32(amax) / np.float32(448.0)
            d = deq[rb * 128:(rb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert np.abs(d).max() <= 448.0
            # the block's largest element lands on the largest code
            assert np.abs(d).max() == 448.0
            err = np.abs(d * scales[rb, kb] - blk)
            # half a quantum: 2^-4 relative for normal values, 2^-10 * scale below
            bound = np.maximum(np.abs(blk) * 2.0**-4, 2.0**-10 * scales[rb, kb]) * (1 + 1e-6)
            assert np.all(err <= bound)


def test_activation_correlation():
    a = kdgen.activations(0, 0, kdgen.HIDDEN_IN, 64, 7168, 0.9)
    x = kdgen.bf16_bits_to_f32(a).astype(np.float64)
    r = np.mean([np.corrcoef(x[t], x[t + 1])[0, 1] for t in range(63)])
    assert abs(r - 0.9) < 0.01
    assert abs(x.var() - 1.0) < 0.02
    b = kdgen.activations(0, 0, kdgen.HIDDEN_IN, 64, 7168, 0.0)
    y = kdgen.bf16_bits_to_f32(b).astype(np.float64)
    r0 = np.mean([np.corrcoef(y[t], y[t + 1])[0, 1] for t in range(63)])
    assert abs(r0) < 0.01
    # first row is the innovation itself for any rho
    assert np.array_equal(a[0], b[0])


def test_zipf_bias():
    b = kdgen.zipf_bias(256, 1.1)
    e = np.arange(256)
    assert np.array_equal(b, (-1.1 * np.log(e + 1.0)).astype(np.float32))
    w = np.exp(b.astype(np.float64))
    assert np.allclose(w / w[0], (e + 1.0) ** -1.1)

"""Writes tiny_seed0.txt: the oracle's output on the tiny workload (seed 0).

A regression anchor for the oracle; it calls only ``oracle/`` and ``kdgen``.
Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import kdgen  # noqa: E402
import oracle  # noqa: E402

w = kdgen.WORKLOADS["tiny"]
x = kdgen.bf16_bits_to_f32(w.hidden_in()).astype(np.float64)
a = kdgen.bf16_bits_to_f32(w.attn_out()).astype(np.float64)
r = oracle.layer(w.dims, x, a, nthreads=1)
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_seed0.txt"), "w") as f:
    f.write("# tiny workload (hidden 256, 8 experts, top-2, M=1, bf16, seed 0): fp64 oracle output\n")
    f.write("# written by tests/golden/make_golden.py from oracle/ only\n")
    f.write("idx: " + " ".join(str(int(v)) for v in r["idx"][0]) + "\n")
    f.write("gates: " + " ".join(repr(float(v)) for v in r["gates"][0]) + "\n")
    f.write("out: " + " ".join(repr(float(v)) for v in r["out"][0]) + "\n")

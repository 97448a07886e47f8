"""The FMA-pipe exp2 of the attention kernel: its coefficient table comes from
the committed generator, and its error bound holds (CPU, float32 Horner
evaluation mirroring the device code; the device evaluation itself is checked
against CUDA's exp2 in test_gpu_parity.py)."""
import os
import re
import subprocess
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "attention_state_reuse_partition_b200", "csrc")


def _table():
    text = open(os.path.join(CSRC, "as_device.cuh")).read()
    return [np.float32(float(v)) for v in re.findall(r"EXP2_C\d = ([-+0-9.e]+)f;", text)]


def test_table_matches_generator():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "gen_exp2_poly.py")], capture_output=True,
                         text=True, check=True).stdout
    gen = [np.float32(float(v)) for v in re.findall(r"EXP2_C\d = ([-+0-9.e]+)f;", out)]
    assert len(gen) == 5 and gen == _table()


def _exp2_poly_f32(x):
    c = _table()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = c[4]
    for a in (c[3], c[2], c[1], c[0]):
        p = (p * f + a).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-124.9, 9.0, 2_000_001, dtype=np.float32)
    y = _exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1)) < 4e-6


def test_clamp_and_masked_inputs():
    y = _exp2_poly_f32(np.array([-np.inf, -1000.0, -125.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y < 3e-38)

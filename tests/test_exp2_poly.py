"""The FMA-pipe exponential available for part of the softmax columns (CPU only).

Replays the kernel's float32 recipe (exp2_poly3_x2: each lane of the packed
pair takes the same steps; constants read from the CUDA source) and
checks it against the exact 2^x: relative error below 1e-4 wherever 2^x is a
normal float, a finite positive result everywhere (very negative inputs are
clamped), and results far below every probability that matters for inputs
under the clamp."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_lvsa_b200", "csrc", "attn_fwd.cuh")


def kernel_recipe():
    src = open(SRC).read()
    body = src[src.index("exp2_poly3_x2(uint64_t xp) {"):]
    body = body[:body.index("\n}")]
    clamp = float(re.search(r"fmaxf\(a, (-?[0-9.]+)f\)", body).group(1))
    pair = r"f2pack\(([0-9.]+)f, \1f\)"      # the same constant in both lanes
    m = re.search(r"ffma2\(" + pair + r", f,\s*f2pack\(([0-9.]+)f, \2f\)\)", body)
    c3, c2 = float(m.group(1)), float(m.group(2))
    c1, c0 = [float(v) for v in re.findall(r"ffma2\(q, f, f2pack\(([0-9.]+)f, \1f\)\)", body)]
    f32 = np.float32

    def exp2(x):
        x = np.maximum(x.astype(f32), f32(clamp))
        t = (x + f32(12582912.0)).astype(f32)
        j = (t - f32(12582912.0)).astype(f32)
        fr = (x - j).astype(f32)
        p = (f32(c3) * fr + f32(c2)).astype(f32)       # fmaf rounds once; difference is below 1 ulp
        p = (p * fr + f32(c1)).astype(f32)
        p = (p * fr + f32(c0)).astype(f32)
        bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
        return bits.astype(np.uint32).view(np.float32), clamp
    return exp2


def test_relative_error_and_range():
    exp2 = kernel_recipe()
    x = np.linspace(-300.0, 10.0, 3_000_001).astype(np.float32)
    y, clamp = exp2(x)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    ref = np.exp2(x.astype(np.float64))
    normal = x >= clamp
    rel = np.abs(y[normal] - ref[normal]) / ref[normal]
    assert rel.max() < 1e-4, rel.max()
    # below the clamp the result is tiny (2^clamp), never larger
    assert np.all(y[~normal] <= 2.0 ** (clamp + 0.5))

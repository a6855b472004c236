"""The FMA-pipe exponential of the attention kernel: its constants are the
Remez minimax cubic for 2^f on [-1/2, 1/2], and the full construction (range
reduction, cubic, exponent-field add), emulated here in fp32 with numpy,
stays within 1e-4 relative of 2^x over the softmax's argument range."""
import os
import re

import numpy as np

from rank_latent_attention_mixer_b200 import exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def kernel_constants():
    src = open(os.path.join(ROOT, "rank_latent_attention_mixer_b200", "csrc", "kernels_tc.cuh")).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", src).group(1)) for i in range(4)]


def test_kernel_constants_are_the_remez_fit():
    assert kernel_constants() == exp2_poly.coefficients_f32()
    assert exp2_poly.max_rel_error_f32() < 8e-5


def emulate(x):
    """fp32 emulation of ex2_fma_pair for one lane."""
    f32 = np.float32
    c0, c1, c2, c3 = (f32(v) for v in kernel_constants())
    x = np.maximum(x.astype(f32), f32(-120))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    f = (x - n).astype(f32)                      # exact (fma with -1 in the kernel)
    q = ((c3 * f + c2).astype(f32) * f + c1).astype(f32)
    q = (q * f + c0).astype(f32)
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_construction_matches_exp2():
    x = np.concatenate([np.linspace(-119.9, 8.0, 400001), np.array([-0.5, 0.5, -1.5, 1.5, 0.0, 8.0])])
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    assert np.all(np.isfinite(y))
    assert np.abs(y / ref - 1).max() < 1e-4


def test_clamp_below_range():
    y = emulate(np.array([-1000.0, -np.inf, -200.0], dtype=np.float32))
    assert np.all(y >= 0) and np.all(y < 2.0 ** -118)

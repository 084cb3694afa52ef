"""The FMA-pipe base-2 exponential of the attention kernel: its constants are
the Remez minimax fit that geometry_routed_block_b200/exp2_poly.py derives, and
the kernel's float32 operation sequence (emulated here step by step) stays
within 1e-4 relative error of 2^x over the range the softmax feeds it. CPU."""
import os
import re

import numpy as np

from geometry_routed_block_b200 import exp2_poly

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "geometry_routed_block_b200", "csrc", "attn_common.cuh")


def kernel_constants():
    text = open(SRC).read()
    return [float(re.search(rf"EXP2_C{i} = ([0-9.eE+-]+)f;", text).group(1)) for i in range(4)]


def test_constants_match_the_remez_fit():
    c, err = exp2_poly.remez_relative()
    assert err < 8e-5
    got = kernel_constants()
    assert np.allclose(got, np.asarray(c, np.float32), rtol=0, atol=1e-7)


def _fma32(a, b, c):
    # a float32 fused multiply-add: exact product and sum in float64 (exact for
    # float32 inputs up to the final rounding), one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def device_exp2(x):
    c0, c1, c2, c3 = (np.float32(v) for v in kernel_constants())
    x = np.maximum(x.astype(np.float32), np.float32(-120.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t + np.float32(-12582912.0)).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.int32).astype(np.int64) + ((t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_device_sequence_error_bound():
    x = np.concatenate([np.linspace(-119.9, 8.0, 400001, dtype=np.float32),
                        np.arange(-119, 9, dtype=np.float32),             # integers
                        np.arange(-119, 9, dtype=np.float32) + 0.5])      # ties
    got = device_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_clamp_below_range_is_tiny_and_positive():
    got = device_exp2(np.array([-1000.0, -200.0, -121.0], np.float32))
    assert (got > 0).all() and (got < 1e-35).all()

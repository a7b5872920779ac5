"""The polynomial 2^x of the prefill softmax (Cody-Waite reduction and a
degree-3 minimax polynomial on [0, 1)): the kernel's constants are the Remez
fit of paged_kv_cache_481_b200/exp2_poly.py, and the fp32 evaluation as the
kernel performs it (floor by the 1.5 * 2^23 round-down trick, Horner with
fused multiply-adds, exponent-field add) stays within 1e-4 relative of 2^x
over the range the softmax uses, x in [-40, 8]."""
import os
import re

import numpy as np

from paged_kv_cache_481_b200 import exp2_poly

HDR = os.path.join(os.path.dirname(os.path.dirname(__file__)), "paged_kv_cache_481_b200", "csrc",
                   "prefill_kernel.cuh")


def _kernel_coeffs():
    src = open(HDR).read()
    return [float(re.search(rf"kExp2C{k} = ([0-9.eE+-]+)f;", src).group(1)) for k in range(4)]


def test_kernel_constants_are_the_remez_fit():
    fit, max_rel = exp2_poly.fit()
    assert max_rel < 1e-4
    np.testing.assert_allclose(_kernel_coeffs(), fit, rtol=1e-9)


def _emulate(x):
    """The kernel's steps in fp32 (numpy float32; fma emulated in float64 and
    rounded once)."""
    c = np.asarray(_kernel_coeffs(), dtype=np.float32)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126))
    magic = np.float32(12582912.0)
    t = np.floor(x.astype(np.float64) + np.float64(magic)).astype(np.float32)  # round-down add
    j = (t - magic).astype(np.float32)
    f = (x.astype(np.float64) - j.astype(np.float64)).astype(np.float32)
    q = np.float64(c[3])
    for k in (2, 1, 0):
        q = (q * f.astype(np.float64) + np.float64(c[k])).astype(np.float32).astype(np.float64)
    q = q.astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_emulated_exp2_within_bound():
    x = np.concatenate([np.linspace(-40, 8, 400001), np.arange(-40, 9, dtype=np.float64),
                        np.arange(-40, 9) - 2.0 ** -20]).astype(np.float32)
    got = _emulate(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_emulated_exp2_floor_trick_and_limits():
    # integers come out exact up to the polynomial's value at 0
    xs = np.arange(-20, 9, dtype=np.float32)
    np.testing.assert_allclose(_emulate(xs), np.exp2(xs) * np.float32(_kernel_coeffs()[0]), rtol=1e-7)
    # far below the range: (almost) zero, never negative or NaN
    tiny = _emulate(np.array([-126.0, -127.0, -200.0, -1e30], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1e-37)

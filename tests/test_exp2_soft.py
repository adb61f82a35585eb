"""CPU check of the attention kernel's software exp2 (exp2_soft in attn_sm100.cu) against exp2.

The test re-executes the kernel's exact operation sequence in fp32 (clamp, floor via the 1.5*2^23
round-down add, polynomial from exp2_poly.cuh in Horner form, integer add of n into the exponent
field) and checks it against numpy's exp2 over the whole input range the softmax produces
(x in [-inf, 8]): relative error within the fitted bound for x >= -126, finite and below 2^-125
below that, never NaN.
"""
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "sparse_rank_hybrid_b200", "csrc")


def _coeffs():
    src = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    c = {int(k): np.float32(float(v)) for k, v in re.findall(r"SLRA_EXP2_C(\d) ([-0-9.e+]+)f", src)}
    return [c[k] for k in sorted(c)]


def _clamp_value():
    src = open(os.path.join(CSRC, "attn_sm100.cu")).read()
    m = re.search(r"float exp2_soft\(float x\) \{\s*x = fmaxf\(x, (-?[0-9.]+)f\);", src)
    return np.float32(float(m.group(1)))


def exp2_soft(x):
    c = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), _clamp_value())
    n = np.floor(x).astype(np.float32)                       # add.rm(x, 1.5*2^23) - 1.5*2^23
    t_bits = (np.int64(0x4B400000) + n.astype(np.int64)).astype(np.uint32)
    f = (x - n).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + ((t_bits.astype(np.uint64) << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_exp2_soft_accuracy_and_range():
    x = np.concatenate([np.linspace(-126, 8, 2_000_001, dtype=np.float32),
                        np.float32([-126.0, -125.5, -1e-7, 0.0, 1e-7, 0.999999, 1.0, 7.9999, 8.0])])
    y = exp2_soft(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(y))
    ok = x >= -125.0  # normal results
    rel = np.abs(y[ok] / ref[ok] - 1)
    assert rel.max() < 1e-4, rel.max()
    assert np.all(y[~ok] >= 0) and np.all(y[~ok] < 2.0 ** -124)


def test_exp2_soft_masked_and_very_negative_inputs():
    x = np.float32([-np.inf, -1e30, -1000.0, -200.0, -127.0, -126.5])
    y = exp2_soft(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2.0 ** -124)

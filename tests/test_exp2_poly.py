"""The FMA-pipe exp2 of the attention kernel, emulated step by step in float32.

The kernel forms 2^x for one pair in eight of the softmax exponentials without
the MUFU unit: j = rint(x) by adding 1.5 * 2^23, f = x - j, a degree-3
polynomial for 2^f, and j added to the exponent bits.  This reads its
constants from the kernel source, repeats each float32 step (a fused
multiply-add rounds once), and checks the result against exact 2^x over the
whole range the softmax feeds it, and that the constants are the Remez fit.
"""
import os
import re

import numpy as np

from kv_cached_segment_b200.fit_exp2_poly import remez_exp2

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cached_segment_b200", "csrc", "attn_device.cuh")


def _constants():
    text = open(SRC).read()
    c = [float(re.search(rf"constexpr float kPc{k} = ([0-9.eE+-]+)f;", text).group(1))
         for k in range(4)]
    shifter = float(re.search(r"constexpr float kShifter = ([0-9.]+)f;", text).group(1))
    return np.float32(c), np.float32(shifter)


def _fma32(a, b, c):
    # a * b is exact in float64 for float32 inputs; one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def kernel_exp2(x):
    c, shifter = _constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + shifter).astype(np.float32)
    jf = (t - shifter).astype(np.float32)
    fr = _fma32(jf, np.float32(-1.0), x)
    p = _fma32(np.full_like(fr, c[3]), fr, np.full_like(fr, c[2]))
    p = _fma32(p, fr, np.full_like(fr, c[1]))
    p = _fma32(p, fr, np.full_like(fr, c[0]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    # the softmax feeds x <= 16 (larger values are caught and redone); below
    # -125 the clamp gives 2^-125, which is 0 for every purpose here
    x = np.concatenate([np.linspace(-125.0, 16.0, 2_000_001),
                        np.arange(-125, 17).astype(np.float64) + 0.5])
    x32 = x.astype(np.float32)
    got = kernel_exp2(x32).astype(np.float64)
    want = np.exp2(x32.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 8e-5          # the fit's 7.5e-5 plus float32 evaluation
    assert rel.max() < 2.0 ** -9     # well inside the rounding step of the bf16 P


def test_integer_arguments_scale_by_exact_powers_of_two():
    # f = 0 for every integer x, so all of them share the polynomial's value
    # at 0 (p(0) = kPc0, within the fit's error of 1), scaled by exactly 2^x
    x = np.arange(-120, 17).astype(np.float32)
    got = kernel_exp2(x).astype(np.float64)
    ratio = got / np.exp2(x.astype(np.float64))
    assert np.all(ratio == ratio[0]) and abs(ratio[0] - 1.0) < 8e-5


def test_clamp_below_minus_125():
    # anything below -125 becomes 2^-125 (times p(0)): a positive normal
    # float that no P of interest is compared with
    got = kernel_exp2(np.float32([-126.0, -1e4, -np.inf, -125.0]))
    assert np.all(got == got[-1]) and abs(float(got[-1]) / 2.0 ** -125 - 1.0) < 8e-5


def test_constants_are_the_remez_fit():
    coef, err = remez_exp2()
    c, _ = _constants()
    assert np.array_equal(coef.astype(np.float32), c)
    assert err < 7.5e-5

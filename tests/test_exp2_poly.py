"""The FMA-pipe exp2 used by the attention backward (f2_exp2_poly in
csrc/common.cuh), emulated step by step in float32 on the CPU with the
coefficients read from the header: Cody-Waite split x = rint(x) + f via the
1.5 * 2^23 shift, the cubic for 2^f, and the integer add into the exponent
field.  Its relative error must stay far below bf16's half-ulp (2^-9), the
precision P is stored in."""
import pathlib
import re

import numpy as np

HDR = pathlib.Path(__file__).resolve().parents[1] / "gpt_pretraining_step_b200" / "csrc" / "common.cuh"


def _coefficients():
    src = HDR.read_text()
    body = src[src.index("f2_exp2_poly(uint64_t x)"):]
    body = body[:body.index("\n}\n")]
    vals = re.findall(r"f2_pack\(([0-9.eE+-]+)f, \1f\)", body)
    nums = [float(v) for v in vals]
    magic = nums[0]
    c3, c2, c1, c0 = nums[1], nums[2], nums[3], nums[4]
    return magic, (c0, c1, c2, c3)


def _emulate(x):
    magic, (c0, c1, c2, c3) = _coefficients()
    x = np.asarray(x, dtype=np.float32)
    t = (x + np.float32(magic)).astype(np.float32)
    f = (x - (t - np.float32(magic)).astype(np.float32)).astype(np.float32)
    p = (np.float32(c3) * f + np.float32(c2)).astype(np.float32)
    p = (p * f + np.float32(c1)).astype(np.float32)
    p = (p * f + np.float32(c0)).astype(np.float32)
    # 32-bit integer add, wrapping like the device's
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(
        0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_header_constants_are_the_remez_fit():
    magic, c = _coefficients()
    assert magic == 12582912.0
    assert abs(c[0] - 1) < 1e-4 and abs(c[1] - np.log(2)) < 1e-3


def test_relative_error_over_the_softmax_range():
    # above 2^-125 the result is a normal float; the softmax arguments are <= ~0
    x = np.concatenate([np.linspace(-125, 1, 2_000_001), -np.logspace(-8, 2, 10001), [0.0, -0.5, 0.5, -1.0]])
    x = x.astype(np.float32)
    got = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1e-4, rel.max()


def test_bottom_of_the_range_is_tiny_and_nonnegative():
    # the caller clamps at -126: the result there loses the implicit bit but
    # stays a nonnegative value below 2^-125, i.e. an exponential that is zero
    # for every sum it enters
    x = np.linspace(-126, -125, 10001).astype(np.float32)
    got = _emulate(x)
    assert (got >= 0).all() and (got < 2.0 ** -124).all()


def test_integer_and_half_integer_points():
    for n in range(-125, 2):
        assert abs(_emulate(np.float32(n)) / 2.0 ** n - 1) < 1e-4
        assert abs(_emulate(np.float32(n + 0.5)) / 2.0 ** (n + 0.5) - 1) < 1e-4

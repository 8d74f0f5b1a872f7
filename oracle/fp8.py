"""fp8 e4m3 per-tensor quantisation (fp64 reference).

TEST INFRASTRUCTURE ONLY: see the package header.

"Como Treinar Seu Próprio ChatGPT por 50 Dólares?", section "3. Gerenciamento
de Precisão": with --fp8 most layers become Float8Linear with per-tensor
scaling.  Reading: dynamic per-tensor scale = 448 / amax(|x|) of the tensor
being quantised, values rounded to the nearest e4m3 number (ties to an even
mantissa), saturated at +-448; the product of two quantised operands is
divided by both scales.

e4m3 (no infinities): sign, 4 exponent bits with bias 7, 3 mantissa bits;
exponent field 0 holds subnormals m * 2^-9, the code with every exponent and
mantissa bit set is NaN, so the largest finite value is 1.75 * 2^8 = 448.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_grid():
    """All non-negative finite e4m3 values with their 7-bit codes, ascending."""
    vals, codes = [], []
    for e in range(16):
        for m in range(8):
            code = (e << 3) | m
            if code == 0x7F:
                continue                      # NaN
            if e == 0:
                val = m * 2.0 ** -9
            else:
                val = (1.0 + m / 8.0) * 2.0 ** (e - 7)
            vals.append(val)
            codes.append(code)
    order = np.argsort(vals)
    return np.array(vals)[order], np.array(codes)[order]


_GRID, _CODES = e4m3_grid()


def round_e4m3(x):
    """Nearest e4m3 value (ties to even mantissa), saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_GRID, a, side="left"), 0, len(_GRID) - 1)
    lo = np.clip(hi - 1, 0, len(_GRID) - 1)
    dlo = a - _GRID[lo]
    dhi = _GRID[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((_CODES[hi] & 1) == 0))
    r = np.where(pick_hi, _GRID[hi], _GRID[lo])
    return np.sign(x) * r


def scale_for(x):
    amax = float(np.max(np.abs(x)))
    return E4M3_MAX / amax if amax > 0 else 1.0


def quantise(x):
    """(q, scale): q = round_e4m3(x * scale) holds e4m3 values as fp64."""
    s = scale_for(x)
    return round_e4m3(np.asarray(x, dtype=np.float64) * s), s


def fp8_matmul(x, w):
    """x @ w with both operands quantised per tensor, product rescaled."""
    qx, sx = quantise(x)
    qw, sw = quantise(w)
    return (qx @ qw) / (sx * sw)

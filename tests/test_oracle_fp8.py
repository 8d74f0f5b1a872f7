"""Pins of the e4m3 quantiser against the format definition and torch's cast (CPU)."""
import numpy as np
import pytest

from oracle import fp8


def test_grid_shape():
    vals, codes = fp8.e4m3_grid()
    assert len(vals) == 127                       # 0 plus 126 finite positives
    assert vals[0] == 0.0 and vals[1] == 2.0 ** -9 and vals[-1] == 448.0
    assert np.all(np.diff(vals) > 0)


def test_matches_torch_cast_in_range():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 50, rng.uniform(-448, 448, 20000),
                        rng.standard_normal(5000) * 1e-3])
    mine = fp8.round_e4m3(x)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    x32 = x.astype(np.float32).astype(np.float64)
    mine32 = fp8.round_e4m3(x32)
    assert np.array_equal(mine32, ref)
    assert np.abs(mine - mine32).max() <= 2.0 ** -9 * 448


def test_ties_to_even_and_saturation():
    # 1 + 1/16 lies halfway between 1 (mantissa 0) and 1.125 (mantissa 1)
    assert fp8.round_e4m3(1.0 + 1 / 16) == 1.0
    assert fp8.round_e4m3(1.125 + 1 / 16) == 1.25
    assert fp8.round_e4m3(1e6) == 448.0 and fp8.round_e4m3(-1e6) == -448.0


def test_per_tensor_scale_hits_max():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 64))
    q, s = fp8.quantise(x)
    assert np.abs(q).max() == 448.0
    assert np.abs(q / s - x).max() <= np.abs(x).max() / 448 * 16   # half an ulp at the top

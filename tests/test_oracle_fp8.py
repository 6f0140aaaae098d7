"""Pins of the FP8 (e4m3) oracle against the format's definition as a library implements
it (torch.float8_e4m3fn) and against closed forms -- not against the oracle itself."""
import numpy as np
import pytest
import torch

from oracle import fp8q as Q


def test_grid_matches_the_library_decoding():
    vals, codes = Q.e4m3_positive_values()
    assert len(vals) == 127 and vals[0] == 0.0 and vals[-1] == 448.0
    assert vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6          # first subnormal, first normal
    lib = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    assert np.array_equal(lib.numpy()[codes], vals)
    assert np.all(np.diff(vals) > 0)


def _lib_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_rounding_matches_the_library_on_ties_and_neighbours():
    vals, _ = Q.e4m3_positive_values()
    mids = (vals[:-1] + vals[1:]) / 2                       # exact ties (all float32-exact)
    eps = np.float32(1e-3)
    xs = np.concatenate([vals, mids, mids * (1 + 2 ** -20), mids * (1 - 2 ** -20)])
    xs = xs[xs <= 448.0].astype(np.float32).astype(np.float64)
    xs = np.concatenate([xs, -xs])
    assert np.array_equal(Q.round_e4m3(xs), _lib_round(xs))
    assert Q.round_e4m3(1.0625) == 1.0 and Q.round_e4m3(1.1875) == 1.25     # ties to even
    assert Q.round_e4m3(2.0 ** -10) == 0.0 and Q.round_e4m3(3 * 2.0 ** -11) == 2.0 ** -9


def test_rounding_matches_the_library_on_random_values():
    g = np.random.default_rng(0)
    x = (g.standard_normal(20000) * np.exp(g.uniform(-12, 5, 20000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0].astype(np.float64)
    assert np.array_equal(Q.round_e4m3(x), _lib_round(x))


@pytest.mark.parametrize("amax,e", [(448.0, 0), (448.0000001, 1), (224.0, -1), (224.0001, 0),
                                    (1.0, -8), (0.875, -9), (0.0, 0), (1e6, 12)])
def test_scale_exponent_closed_form(amax, e):
    assert Q.pow2_scale_exponent(amax) == e
    if amax > 0:
        assert amax <= 448.0 * 2.0 ** e and amax > 448.0 * 2.0 ** (e - 1)


def test_quantize_rows_tight_scale_and_error_bound():
    g = np.random.default_rng(1)
    x = g.standard_normal((50, 3, 16)) * np.exp(g.uniform(-5, 5, (50, 3, 1)))
    x[7, 1] = 0.0
    x8, s = Q.quantize_rows(x)
    assert s.shape == (50, 3)
    a8 = np.abs(x8).max(axis=-1)
    nz = np.abs(x).max(axis=-1) > 0
    ratio = np.abs(x).max(axis=-1)[nz] / s[nz]               # before rounding: in (224, 448]
    assert np.all(ratio > 224.0) and np.all(ratio <= 448.0)
    assert np.all(a8 <= 448.0) and np.all(a8[nz] >= 224.0) and np.all(x8[7, 1] == 0)
    xr = x8 * s[..., None]
    normal = np.abs(x / s[..., None]) >= 2.0 ** -6
    rel = np.abs(xr - x) / np.where(normal, np.abs(x), 1.0)
    assert np.all(rel[normal] <= 2.0 ** -4)
    assert np.all(np.abs(xr - x)[~normal & (x != 0)] <= 2.0 ** -10 * np.broadcast_to(s[..., None], x.shape)[~normal & (x != 0)])
    # exact round trip for values already on the scaled grid
    x8b, sb = Q.quantize_rows(xr)
    assert np.array_equal(x8b * sb[..., None], xr)


def test_quantize_per_head_uses_one_scale_per_head():
    g = np.random.default_rng(2)
    x = g.standard_normal((6, 40, 4, 8))                       # [slots, T, H, d]
    x[:, :, 2] *= 100.0
    x8, s = Q.quantize_per_head(x)
    assert s.shape == (4,)
    for h in range(4):
        assert s[h] == 2.0 ** Q.pow2_scale_exponent(np.abs(x[:, :, h]).max())
        assert np.abs(x8[:, :, h]).max() <= 448.0
    assert s[2] > s[0]
    assert np.allclose(x8 * s[None, None, :, None], x, rtol=2.0 ** -4, atol=2.0 ** -10 * s.max())

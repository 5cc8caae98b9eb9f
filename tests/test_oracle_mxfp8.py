"""Pins for oracle.mxfp8 (the MXFP8 quantiser kept for a block-scaled expert path): the
E4M3 grid built from its bit fields, brute-force nearest-value rounding, torch's float8
cast, and the block-scale rule of the OCP MX v1.0 specification."""
import numpy as np
import pytest
import torch

from oracle import mxfp8 as mx


def e4m3_grid():
    """Every non-negative finite E4M3 value from its bit fields (exponent field E with
    bias 7, mantissa field M): E = 0 is subnormal, (E, M) = (15, 7) is NaN.  Returns
    (values, mantissa fields), sorted by value."""
    vals, mants = [], []
    for E in range(16):
        for M in range(8):
            if E == 15 and M == 7:
                continue
            v = (M / 8.0) * 2.0 ** -6 if E == 0 else (1.0 + M / 8.0) * 2.0 ** (E - 7)
            vals.append(v)
            mants.append(M)
    order = np.argsort(vals, kind="stable")
    return np.array(vals)[order], np.array(mants)[order]


def brute_nearest(v):
    """Nearest grid value by exhaustive search, ties to the even mantissa field, clamped
    to the largest finite value."""
    grid, mant = e4m3_grid()
    out = []
    for x in np.atleast_1d(v):
        a = min(abs(float(x)), grid[-1])
        d = np.abs(grid - a)
        cand = np.nonzero(d == d.min())[0]
        pick = cand[0] if len(cand) == 1 else [c for c in cand if mant[c] % 2 == 0][0]
        out.append(np.copysign(grid[pick], x))
    return np.array(out)


def test_grid_size_and_extremes():
    grid, _ = e4m3_grid()
    assert len(grid) == 127                      # zero, 7 subnormals, 119 normals
    assert grid[-1] == mx.E4M3_MAX == 448.0
    assert grid[1] == 2.0 ** -9 and grid[8] == 2.0 ** -6


def test_every_grid_value_round_trips():
    grid, _ = e4m3_grid()
    assert np.array_equal(mx.e4m3_round(grid), grid)
    assert np.array_equal(mx.e4m3_round(-grid), -grid)


def test_midpoints_round_to_the_even_mantissa():
    grid, mant = e4m3_grid()
    mids = (grid[:-1] + grid[1:]) / 2
    want = np.where(mant[:-1] % 2 == 0, grid[:-1], grid[1:])
    assert np.array_equal(mx.e4m3_round(mids), want)


def test_brute_force_nearest_on_random_values():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-448, 448, 400), rng.uniform(-1, 1, 300) * 2.0 ** -6,
                        np.exp2(rng.uniform(-12, 9.5, 300)) * rng.choice([-1, 1], 300)])
    assert np.array_equal(mx.e4m3_round(v), brute_nearest(v))


def test_overflow_clamps_to_448():
    v = np.array([448.0, 449.0, 463.9, 464.0, 465.0, 480.0, 511.9, 1e6])
    assert np.array_equal(mx.e4m3_round(v), np.full(v.shape, 448.0))
    assert np.array_equal(mx.e4m3_round(-v), np.full(v.shape, -448.0))
    assert np.isnan(mx.e4m3_round([np.nan])[0])


def test_matches_torch_float8_cast_in_range():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(2000) * 50.0, rng.standard_normal(500) * 2.0 ** -8])
    v = np.clip(v, -448.0, 448.0)
    ref = torch.from_numpy(v).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    # float64 -> float32 first (as torch's cast takes it); the float32 rounding cannot move
    # a value across an E4M3 rounding boundary except at exact float32 ties, not drawn here
    assert np.array_equal(mx.e4m3_round(v.astype(np.float32).astype(np.float64)), ref)


def test_block_scale_rule():
    rng = np.random.default_rng(2)
    for e in (-20, -3, 0, 5, 20):
        x = rng.standard_normal((4, 128)) * 2.0 ** e
        q, s = mx.quantize_mxfp8(x)
        assert s.shape == (4, 4)
        amax = np.abs(x).reshape(4, 4, 32).max(axis=-1)
        r = amax / np.exp2(s)
        assert np.all((r >= 256) & (r < 512))
        # q is on the E4M3 grid and is the element-wise rounding of x / 2^s
        assert np.array_equal(q, mx.e4m3_round(x / np.repeat(np.exp2(s), 32, axis=-1)))
    q, s = mx.quantize_mxfp8(np.zeros((2, 32)))
    assert np.all(s == -127) and np.all(q == 0)


def test_quantise_other_axis_and_dequantise():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 5))
    q0, s0 = mx.quantize_mxfp8(x, axis=0)
    q1, s1 = mx.quantize_mxfp8(x.T, axis=-1)
    assert np.array_equal(q0, q1.T) and np.array_equal(s0, s1.T)
    d = mx.dequantize_mxfp8(q0, s0, axis=0)
    # relative error of an element below the block maximum: at most half a quantum of
    # its binade (2^-4 relative), or the clamp of the [448, 512) range (at most 1/8)
    assert np.all(np.abs(d - x) <= np.abs(x) * 2.0 ** -3 + np.exp2(np.repeat(s0, 32, axis=0)) * 2.0 ** -9)


def test_blocked_axis_must_be_a_multiple_of_32():
    with pytest.raises(ValueError):
        mx.quantize_mxfp8(np.ones((2, 48)))

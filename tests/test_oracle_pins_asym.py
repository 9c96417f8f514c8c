"""Pins of the oracle's asymmetric RTN with clipping (DuQuant, Knowl 12:
per-token asymmetric activations, per-channel asymmetric weights, clipping
ratios on the extremes; step (gamma max - beta min) / (2^b - 1)) against
hand-worked values, bounds, special cases and a brute-force expansion of the
zero-point product (no GPU)."""
import numpy as np
import pytest

import oracle
from rotation_bit_quantization_randomized_b200 import synth


def test_hand_worked_row_no_clip():
    # lo = -1, hi = 2, d = 3/15 = 0.2, z = rint(5) = 5; x/d = -5, 0, 2.5 (even -> 2), 10
    x = np.array([[-1.0, 0.0, 0.5, 2.0]])
    u, d, z, r = oracle.quantize_asym(x, 1.0)
    assert abs(d[0] - 0.2) <= 1e-15 and z[0] == 5 and r[0] == 27
    np.testing.assert_array_equal(u[0], [0, 5, 7, 15])
    np.testing.assert_allclose(d[0] * (u[0] - z[0]), [-1.0, 0.0, 0.4, 2.0], atol=1e-14)


def test_hand_worked_row_clipped():
    # clip 0.5: lo = -0.5, hi = 1, d = 0.1, z = 5; x/d + z = -5, 5, 10, 25 -> clamp to [0, 15]
    x = np.array([[-1.0, 0.0, 0.5, 2.0]])
    u, d, z, r = oracle.quantize_asym(x, 0.5)
    assert abs(d[0] - 0.1) <= 1e-15 and z[0] == 5 and r[0] == 30
    np.testing.assert_array_equal(u[0], [0, 5, 10, 15])


def test_symmetric_row_zero_point_and_step():
    # min = -max: d = 2 max / 15, z = rint(7.5) = 8 (ties to even)
    x = np.array([[-3.0, 1.0, 3.0, 0.25]])
    u, d, z, r = oracle.quantize_asym(x, 1.0)
    assert abs(d[0] - 6.0 / 15) <= 1e-15 and z[0] == 8
    assert u[0, 0] == 0 and u[0, 2] == 15      # -7.5 + 8 -> 0 (even), 7.5 + 8 = 15.5 -> 16 -> clamp 15


def test_bound_inside_clipped_range_and_clamp_outside():
    x = synth.random_f16((32, 512), 21, dist="student_t3")
    xr = oracle.rotate(x, synth.signs(512, 21), 0)
    for clip in (1.0, 0.9, 0.8):
        u, d, z, r = oracle.quantize_asym(xr, clip)
        assert u.min() >= 0 and u.max() <= 15
        np.testing.assert_array_equal(u.astype(np.int64).sum(axis=1), r)
        lo = clip * xr.min(axis=1, keepdims=True)
        hi = clip * xr.max(axis=1, keepdims=True)
        xh = d[:, None] * (u - z[:, None])
        inside = (xr >= lo) & (xr <= hi)
        err = np.abs(xr - xh)
        assert np.all(err[inside] <= (d[:, None] / 2 * (1 + 1e-12) + 1e-15).repeat(512, 1)[inside])
        # outside the clipped range the code saturates at the end of the grid
        assert np.all(u[xr > hi] == 15) and np.all(u[xr < lo] == 0)
        if clip == 1.0:
            assert inside.all()


def test_zero_and_constant_rows_give_zero_codes():
    x = np.zeros((2, 8))
    x[1] = 2.5
    u, d, z, r = oracle.quantize_asym(x, 0.9)
    np.testing.assert_array_equal(d, 0.0)
    np.testing.assert_array_equal(z, 0)
    np.testing.assert_array_equal(u, 0)
    np.testing.assert_array_equal(r, 0)


def test_dequant_asym_equals_brute_force_expansion():
    rng = np.random.default_rng(47)
    M, N, K = 5, 7, 128
    ua = rng.integers(0, 16, size=(M, K)).astype(np.int8)
    uw = rng.integers(0, 16, size=(N, K)).astype(np.int8)
    za = rng.integers(-3, 19, size=M)
    zw = rng.integers(-3, 19, size=N)
    da = rng.random(M) + 0.1
    dw = rng.random(N) * 1e-2 + 1e-3
    acc = oracle.int_gemm(ua, uw, 0)
    y, y16 = oracle.dequant_asym(acc, K, da, za, ua.astype(np.int64).sum(1), dw, zw, uw.astype(np.int64).sum(1))
    for m in range(M):
        for n in range(N):
            ref = sum(da[m] * (int(ua[m, k]) - za[m]) * dw[n] * (int(uw[n, k]) - zw[n]) for k in range(K))
            assert abs(y[m, n] - ref) <= 1e-12 * max(1.0, abs(ref))
            assert y16[m, n] == np.float16(ref).view(np.uint16)


def test_linear_asym_error_bound_tiny_workload():
    # x'.w' - xh.wh = (x' - xh).w' + xh.(w' - wh): |y - x.w| <= (da/2) sum|w'| + (dw/2) sum|xh| with clip 1
    w_ = synth.TINY
    x = synth.activations(w_)
    W = synth.weights(w_, 256)
    s = synth.signs(w_.K, w_.seed)
    out = oracle.linear_asym(x, W, s, 1.0, 1.0, 0)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    xh = out["da"][:, None] * ((oracle.unpack(out["qa"]) & 0x0F) - out["za"][:, None])
    wr = oracle.rotate(W, s, 0)
    bound = (out["da"][:, None] / 2) * np.abs(wr).sum(1)[None, :] + \
        (out["dw"][None, :] / 2) * np.abs(xh).sum(1)[:, None]
    assert np.all(np.abs(out["y"] - ref) <= bound * (1 + 1e-9) + 1e-9)
    assert np.max(np.abs(out["y"] - ref)) < 0.25 * np.max(np.abs(ref))


@pytest.mark.parametrize("bad", [0.0, -0.5, 1.5])
def test_clip_ratio_range_is_checked(bad):
    with pytest.raises(ValueError):
        oracle.quantize_asym(np.ones((1, 4)), bad)


def test_quantize_asym_with_own_step_and_zero_reproduces_codes_and_hand_values():
    x = synth.random_f16((16, 256), 23, dist="laplace").astype(np.float64)
    u, d, z, r = oracle.quantize_asym(x, 0.9)
    np.testing.assert_array_equal(oracle.quantize_asym_with(x, d, z), u)
    # hand values: d = 0.5, z = 3: x/d = -10, -1.5 (even -> -2), 0.6, 30 -> +3, clamp
    got = oracle.quantize_asym_with(np.array([[-5.0, -0.75, 0.3, 15.0]]), np.array([0.5]), np.array([3]))
    np.testing.assert_array_equal(got[0], [0, 1, 4, 15])

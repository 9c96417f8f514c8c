"""Pins of the oracle's 6-bit RTN variant against closed forms, hand-worked
values, brute force and error bounds (no GPU).

QuaRot's summary (Elamur Research, "Key points") reports that plain
round-to-nearest is close to lossless at 6 and 8 bits without calibration;
the ISTA record abstract names 4 bits as the headline width of the same
recipe.  At 6 bits: scale s = max|row| / 31, codes clamp(rint(v / s), -32,
31) with ties to even, one signed byte per code.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from rotation_bit_quantization_randomized_b200 import synth


@pytest.mark.parametrize("n", [256, 4096])
def test_spike_closed_form_6bit(n):
    # x = c e_k: every |x'| = c/sqrt(n), scale c/(31 sqrt(n)), codes 31 s_k H[k, :]
    c, k = 5.0, 77
    s = synth.signs(n, 26)
    x = np.zeros((1, n), np.float16)
    x[0, k] = c
    codes, sc = oracle.quantize_bits(oracle.rotate(x, s, 0), 6)
    assert abs(sc[0] - c / (31 * np.sqrt(n))) <= 1e-16
    H = scipy.linalg.hadamard(n)
    np.testing.assert_array_equal(codes[0], 31 * s[k] * H[k])


def test_quantizer_6bit_error_bound_range_and_absmax():
    x = synth.random_f16((64, 1024), 27, dist="student_t3")
    xr = oracle.rotate(x, synth.signs(1024, 27), 0)
    codes, sc = oracle.quantize_bits(xr, 6)
    np.testing.assert_allclose(sc, np.abs(xr).max(axis=1) / 31, rtol=1e-15)
    err = np.abs(xr - codes * sc[:, None])
    assert np.all(err <= sc[:, None] / 2 * (1 + 1e-12))
    assert codes.min() >= -31 and codes.max() <= 31         # per-row scale never needs the clamp
    j = np.argmax(np.abs(xr), axis=1)
    np.testing.assert_array_equal(np.abs(codes[np.arange(64), j]), 31)
    # the grid is 31/7 times finer than the 4-bit one
    _, sc4 = oracle.quantize(xr, 0)
    np.testing.assert_allclose(sc4 / sc, 31 / 7, rtol=1e-12)


def test_quantizer_6bit_hand_worked_ties_and_zero_row():
    # scale 31 / 31 = 1: ties go to the even neighbour
    xr = np.array([[31.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 0.0, -30.5, 30.5, 12.49],
                   [0.0] * 11])
    codes, sc = oracle.quantize_bits(xr, 6)
    assert sc[0] == 1.0 and sc[1] == 0.0
    np.testing.assert_array_equal(codes[0], [31, 2, 4, -2, 0, 0, 2, 0, -30, 30, 12])
    np.testing.assert_array_equal(codes[1], 0)


def test_quantizer_6bit_clamp_with_small_scale():
    # under a supplied scale of 1 the codes saturate at -32 and 31
    xr = np.array([[40.0, -40.0, 31.6, -31.6, -32.4, 7.0]])
    codes = oracle.quantize_bits_with_scales(xr, np.array([1.0]), 6)
    np.testing.assert_array_equal(codes[0], [31, -32, 31, -32, -32, 7])


def test_quantizer_6bit_idempotent():
    x = synth.random_f16((16, 512), 28, dist="laplace")
    codes, sc = oracle.quantize_bits(oracle.rotate(x, synth.signs(512, 28), 0), 6)
    codes2, sc2 = oracle.quantize_bits(codes * sc[:, None], 6)
    np.testing.assert_array_equal(codes, codes2)
    np.testing.assert_allclose(sc2, sc, rtol=1e-15)


def test_int_gemm_6bit_codes_brute_force():
    rng = np.random.default_rng(66)
    qa = rng.integers(-32, 32, size=(3, 128)).astype(np.int8)
    qw = rng.integers(-32, 32, size=(5, 128)).astype(np.int8)
    brute = np.array([[sum(int(a) * int(b) for a, b in zip(qa[m], qw[n])) for n in range(5)] for m in range(3)])
    np.testing.assert_array_equal(oracle.int_gemm(qa, qw, 0), brute)


def test_linear6_error_bound_and_between_int4_and_int8():
    # |y - x.w| <= (s_a/2) sum|w'| + (s_w/2) sum|x'| + K s_a s_w / 4 with the
    # 6-bit scales; the result lies between the 4-bit and 8-bit ones in error
    w_ = synth.TINY
    x = synth.activations(w_)
    W = synth.weights(w_, 256)
    s = synth.signs(w_.K, w_.seed)
    xr = oracle.rotate(x, s, 0)
    wr = oracle.rotate(W, s, 0)
    qa, sa = oracle.quantize_bits(xr, 6)
    qw, sw = oracle.quantize_bits(wr, 6)
    y, _ = oracle.dequant_linear(oracle.int_gemm(qa, qw, 0), sa, sw, 0)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    bound = (sa[:, None] / 2) * np.abs(wr).sum(1)[None, :] + \
        (sw[None, :] / 2) * np.abs(xr).sum(1)[:, None] + w_.K * sa[:, None] * sw[None, :] / 4
    assert np.all(np.abs(y - ref) <= bound * (1 + 1e-9))
    err6 = np.max(np.abs(y - ref))
    err4 = np.max(np.abs(oracle.linear(x, W, s, 0, 0)["y"] - ref))
    err8 = np.max(np.abs(oracle.linear8(x, W, s, 0)["y"] - ref))
    assert err8 < err6 < err4

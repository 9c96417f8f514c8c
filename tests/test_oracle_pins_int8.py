"""Pins of the oracle's 8-bit RTN variant against closed forms, hand-worked
values, brute force and error bounds (no GPU).

The INT8 variant is the same recipe as the INT4 path at a wider code: QuaRot
(ISTA record abstract) names 4-bit as the headline and reports that higher
widths of the same round-to-nearest scheme are lossless without calibration
(Elamur Research summary, "Key points").  Scale s = max|row| / 127, codes
clamp(rint(v / s), -128, 127) with ties to even, one signed byte per code.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from rotation_bit_quantization_randomized_b200 import synth


@pytest.mark.parametrize("n", [256, 8192])
def test_spike_closed_form_8bit(n):
    # x = c e_k: every |x'| = c/sqrt(n), scale c/(127 sqrt(n)), codes 127 s_k H[k, :]
    c, k = 3.0, 201
    s = synth.signs(n, 16)
    x = np.zeros((1, n), np.float16)
    x[0, k] = c
    codes, sc, _ = oracle.rotate_quant8(x, s, 0)
    assert abs(sc[0] - c / (127 * np.sqrt(n))) <= 1e-16
    H = oracle.sylvester(n) if n > 1024 else scipy.linalg.hadamard(n)
    np.testing.assert_array_equal(codes[0], 127 * s[k] * H[k])


def test_quantizer_8bit_error_bound_range_and_absmax():
    x = synth.random_f16((64, 1024), 17, dist="student_t3")
    xr = oracle.rotate(x, synth.signs(1024, 17), 0)
    codes, sc = oracle.quantize_bits(xr, 8)
    np.testing.assert_allclose(sc, np.abs(xr).max(axis=1) / 127, rtol=1e-15)
    err = np.abs(xr - codes * sc[:, None])
    assert np.all(err <= sc[:, None] / 2 * (1 + 1e-12))
    assert codes.min() >= -127 and codes.max() <= 127       # per-row scale never needs the clamp
    j = np.argmax(np.abs(xr), axis=1)
    np.testing.assert_array_equal(np.abs(codes[np.arange(64), j]), 127)
    # 16x finer grid than 4 bits: the INT4 error bound is 127/7 times wider
    _, sc4 = oracle.quantize(xr, 0)
    np.testing.assert_allclose(sc4 / sc, 127 / 7, rtol=1e-12)


def test_quantizer_8bit_hand_worked_ties_and_zero_row():
    xr = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 0.0, -126.5, 126.5],
                   [0.0] * 10])
    codes, sc = oracle.quantize_bits(xr, 8)
    assert sc[0] == 1.0 and sc[1] == 0.0
    np.testing.assert_array_equal(codes[0], [127, 2, 4, -2, 0, 0, 2, 0, -126, 126])
    np.testing.assert_array_equal(codes[1], 0)


def test_quantizer_8bit_clamp_with_small_scale():
    # v / s = +-200 and +-127.6 under a supplied scale of 1: clamp to [-128, 127]
    xr = np.array([[200.0, -200.0, 127.6, -127.6, -128.4, 3.0]])
    codes = oracle.quantize_bits_with_scales(xr, np.array([1.0]), 8)
    np.testing.assert_array_equal(codes[0], [127, -128, 127, -128, -128, 3])


def test_quantizer_8bit_idempotent():
    x = synth.random_f16((16, 256), 18)
    codes, sc = oracle.quantize_bits(oracle.rotate(x, synth.signs(256, 18), 0), 8)
    codes2, sc2 = oracle.quantize_bits(codes * sc[:, None], 8)
    np.testing.assert_array_equal(codes, codes2)
    np.testing.assert_allclose(sc2, sc, rtol=1e-15)


def test_general_width_at_4_bits_is_the_int4_quantizer():
    x = synth.random_f16((8, 512), 19, dist="laplace")
    xr = oracle.rotate(x, synth.signs(512, 19), 0)
    c4, s4 = oracle.quantize(xr, 0)
    cb, sb = oracle.quantize_bits(xr, 4)
    np.testing.assert_array_equal(c4, cb)
    np.testing.assert_array_equal(s4, sb)


def _brute(qa, qw):
    M, K = qa.shape
    N = qw.shape[0]
    out = [[0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            s = 0
            for k in range(K):
                s += int(qa[m, k]) * int(qw[n, k])
            out[m][n] = s
    return np.array(out, np.int64)


def test_int_gemm_8bit_codes_brute_force_and_extremes():
    rng = np.random.default_rng(46)
    qa = rng.integers(-128, 128, size=(3, 256)).astype(np.int8)
    qw = rng.integers(-128, 128, size=(4, 256)).astype(np.int8)
    np.testing.assert_array_equal(oracle.int_gemm(qa, qw, 0), _brute(qa, qw))
    K = 8192
    a = np.full((1, K), -128, np.int8)
    w = np.stack([np.full(K, -128, np.int8), np.full(K, 127, np.int8)])
    np.testing.assert_array_equal(oracle.int_gemm(a, w, 0)[0], [16384 * K, -16256 * K])


def test_linear8_error_bound_tiny_workload():
    # |y - x.w| <= (s_a/2) sum|w'| + (s_w/2) sum|x'| + K s_a s_w / 4 with the
    # 8-bit scales, and the result is much closer than the INT4 one
    w_ = synth.TINY
    x = synth.activations(w_)
    W = synth.weights(w_, 256)
    s = synth.signs(w_.K, w_.seed)
    out = oracle.linear8(x, W, s, 0)
    xr = oracle.rotate(x, s, 0)
    wr = oracle.rotate(W, s, 0)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    sa, sw = out["sa"], out["sw"]
    bound = (sa[:, None] / 2) * np.abs(wr).sum(1)[None, :] + \
        (sw[None, :] / 2) * np.abs(xr).sum(1)[:, None] + w_.K * sa[:, None] * sw[None, :] / 4
    assert np.all(np.abs(out["y"] - ref) <= bound * (1 + 1e-9))
    err8 = np.max(np.abs(out["y"] - ref))
    err4 = np.max(np.abs(oracle.linear(x, W, s, 0, 0)["y"] - ref))
    assert err8 < err4 / 4

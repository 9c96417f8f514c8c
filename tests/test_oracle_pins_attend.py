"""Pins of the oracle's decode-attention tail (softmax over the decode scores,
then the product with the INT4 value cache) against closed forms and
invariants (no GPU): uniform scores average the dequantized values, a
dominant score selects one token, two tokens weigh by the logistic of their
score gap, a constant shift of the scores changes nothing, and query head hq
reads KV head hq / (Hq / Hkv)."""
import numpy as np

import oracle


def _values(B, T, H, D, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(-8, 8, size=(B, T, H, D)).astype(np.int8)
    scales = (rng.random((B, T, H)) * 0.1 + 0.01).astype(np.float16)
    return oracle.pack(codes), scales.view(np.uint16), codes, scales.astype(np.float64)


def test_uniform_scores_average_the_values():
    vq, vs, codes, s = _values(2, 37, 2, 128, 1)
    out = oracle.kv_attend(np.full((2, 4, 37), 0.75), vq, vs)
    deq = codes * s[..., None]                           # [B, T, H, D]
    for b in range(2):
        for hq in range(4):
            np.testing.assert_allclose(out[b, hq], deq[b, :, hq // 2].mean(axis=0), rtol=0, atol=1e-12)


def test_dominant_score_selects_its_token():
    vq, vs, codes, s = _values(1, 50, 1, 128, 2)
    sc = np.zeros((1, 3, 50))
    sc[0, 0, 17] = 1e4                                  # exp(-1e4 / sqrt(128)) underflows to 0
    sc[0, 1, 0] = 1e4
    sc[0, 2, 49] = 1e4
    out = oracle.kv_attend(sc, vq, vs)
    for hq, t in ((0, 17), (1, 0), (2, 49)):
        np.testing.assert_array_equal(out[0, hq], codes[0, t, 0] * s[0, t, 0])


def test_two_tokens_logistic_weights():
    vq, vs, codes, s = _values(1, 2, 1, 128, 3)
    g = 3.0
    sc = np.array([[[g * np.sqrt(128.0), 0.0]]])       # gap of g after the 1/sqrt(D) scale
    p0 = 1.0 / (1.0 + np.exp(-g))
    out = oracle.kv_attend(sc, vq, vs)
    ref = p0 * codes[0, 0, 0] * s[0, 0, 0] + (1 - p0) * codes[0, 1, 0] * s[0, 1, 0]
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-13, atol=1e-15)


def test_shift_invariance_and_gqa_mapping():
    vq, vs, codes, s = _values(1, 64, 4, 128, 4)
    rng = np.random.default_rng(5)
    sc = rng.standard_normal((1, 16, 64)) * 20
    a = oracle.kv_attend(sc, vq, vs)
    b = oracle.kv_attend(sc + 123.25, vq, vs)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    # the four query heads of KV head h read only KV head h: equal scores give equal outputs
    sc2 = np.repeat(sc[:, :1], 16, axis=1)
    c = oracle.kv_attend(sc2, vq, vs)
    for hq in range(16):
        np.testing.assert_array_equal(c[0, hq], c[0, 4 * (hq // 4)])
    assert not np.allclose(c[0, 0], c[0, 4])

"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests re-types the oracle's formula or re-calls its own routine
as the expected value: each compares it to an independent object (a textbook
matrix, scipy's Hadamard, numpy's fp16 conversion, a closed form, a
brute-force loop, an invariant or an error bound).  Each test names the
mistake it is there to catch.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from rotation_bit_quantization_randomized_b200 import synth


def _f16(a):
    return np.asarray(a, np.float64).astype(np.float16)


# --------------------------------------------------------------------------
# Hadamard matrix
# --------------------------------------------------------------------------

def test_sylvester_h8_textbook(golden):
    rows, _ = golden("sylvester_h8.txt")
    np.testing.assert_array_equal(oracle.sylvester(8), np.array(rows, np.int8))


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024])
def test_sylvester_matches_scipy(n):
    # scipy.linalg.hadamard builds the same Sylvester-ordered matrix
    np.testing.assert_array_equal(oracle.sylvester(n), scipy.linalg.hadamard(n).astype(np.int8))


@pytest.mark.parametrize("n", [2, 64, 1024])
def test_hadamard_orthogonal_exact(n):
    H = oracle.sylvester(n).astype(np.int64)
    np.testing.assert_array_equal(H @ H.T, n * np.eye(n, dtype=np.int64))


def test_hadamard_8192_sampled_rows_orthogonal():
    n = 8192
    H = oracle.sylvester(n)
    rows = synth.sample_rows(n, 48, 7)
    Hs = H[rows].astype(np.int64)
    np.testing.assert_array_equal(Hs @ Hs.T, n * np.eye(len(rows), dtype=np.int64))
    # sampled rows against the closed form (-1)^popcount(k & l)
    l = np.arange(n)
    for k in rows[:8]:
        pc = np.array([bin(int(k) & int(j)).count("1") for j in l])
        np.testing.assert_array_equal(H[k], np.where(pc % 2 == 0, 1, -1))


# --------------------------------------------------------------------------
# fast transform and rotation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_fwht_equals_dense_sylvester(n):
    v = np.random.default_rng(n).standard_normal((5, n))
    ref = v @ scipy.linalg.hadamard(n).astype(np.float64)
    got = oracle.fwht(v)
    assert np.max(np.abs(got - ref)) <= 1e-14 * max(1.0, np.max(np.abs(ref)))


@pytest.mark.parametrize("n", [128, 1024, 8192])
def test_fwht_involution(n):
    # (H/sqrt n)^2 = I: catches a wrong butterfly sign or a dropped stage
    v = np.random.default_rng(1).standard_normal((3, n))
    back = oracle.fwht(oracle.fwht(v)) / n
    assert np.max(np.abs(back - v)) <= 1e-12


@pytest.mark.parametrize("K,hb", [(256, 0), (128, 0), (512, 128), (384, 128)])
def test_rotate_fast_equals_dense(K, hb):
    x = synth.random_f16((4, K), 11)
    s = synth.signs(K, 3)
    a = oracle.rotate(x, s, hb)
    b = oracle.rotate(x, s, hb, dense=True)
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))


@pytest.mark.parametrize("K", [256, 4096])
def test_rotate_matches_scipy_product_with_signs(K):
    # x' = (x diag(s)) H / sqrt(K): catches signs applied after H, or H^T/H mixups
    x = synth.random_f16((3, K), 5)
    s = synth.signs(K, 9)
    H = scipy.linalg.hadamard(K).astype(np.float64)
    ref = (x.astype(np.float64) * s) @ H / np.sqrt(K)
    got = oracle.rotate(x, s, 0)
    assert np.max(np.abs(got - ref)) <= 1e-11 * np.max(np.abs(ref))


@pytest.mark.parametrize("K", [256, 11008])
def test_block_rotation_equals_kron(K):
    # I_{K/128} (x) H_128 / sqrt(128): each block rotated on its own
    x = synth.random_f16((2, K), 21, dist="laplace")
    s = synth.signs(K, 4)
    Hb = scipy.linalg.hadamard(128).astype(np.float64) / np.sqrt(128)
    xs = x.astype(np.float64) * s
    ref = np.concatenate([xs[:, b:b + 128] @ Hb for b in range(0, K, 128)], axis=1)
    got = oracle.rotate(x, s, 128)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("n", [8, 256, 8192])
def test_rotate_basis_vectors(n):
    # e_k -> s_k * H[k, :] / sqrt(n)
    s = synth.signs(n, 2)
    ks = [0, 1, n // 2 + 1, n - 1]
    x = np.zeros((len(ks), n), np.float16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    got = oracle.rotate(x, s, 0)
    H = scipy.linalg.hadamard(n) if n <= 1024 else oracle.sylvester(n)
    for i, k in enumerate(ks):
        np.testing.assert_allclose(got[i], s[k] * H[k] / np.sqrt(n), rtol=0, atol=1e-15)


def test_rotate_constant_vector():
    # c * 1 with unit signs -> sqrt(n) * c * e_0
    n = 1024
    x = np.full((1, n), 0.5, np.float16)
    got = oracle.rotate(x, np.ones(n, np.int8), 0)[0]
    assert abs(got[0] - 0.5 * np.sqrt(n)) <= 1e-12
    assert np.max(np.abs(got[1:])) <= 1e-12


def test_rotate_preserves_norm():
    x = synth.random_f16((6, 4096), 8, dist="student_t3")
    s = synth.signs(4096, 8)
    got = oracle.rotate(x, s, 0)
    np.testing.assert_allclose(np.linalg.norm(got, axis=1),
                               np.linalg.norm(x.astype(np.float64), axis=1), rtol=1e-12)


@pytest.mark.parametrize("K,hb", [(256, 0), (4096, 0), (1024, 128)])
def test_computational_invariance(K, hb):
    # DuQuant Knowl 1: Y = XW = (XG)(G^-1 W); with G = diag(s) H/sqrt(n) orthogonal,
    # rotating both x and the rows of W leaves x W^T unchanged.
    x = synth.random_f16((5, K), 31, dist="student_t3")
    w = synth.random_f16((7, K), 32, scale=0.02)
    s = synth.signs(K, 33)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    got = oracle.rotate(x, s, hb) @ oracle.rotate(w, s, hb).T
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))


# --------------------------------------------------------------------------
# quantizer
# --------------------------------------------------------------------------

def test_spike_fixture(golden):
    _, kv = golden("spike_n8.txt")
    n = int(kv["n"][0])
    x = np.array([[float(t) for t in kv["x"]]], np.float16)
    s = np.array([int(t) for t in kv["signs"]], np.int8)
    xr = oracle.rotate(x, s, 0)
    np.testing.assert_allclose(xr[0], [float(t) for t in kv["rotated"]], rtol=0, atol=1e-15)
    codes, sc = oracle.quantize(xr, 0)
    assert abs(sc[0] - float(kv["scale"][0])) <= 1e-16
    np.testing.assert_array_equal(codes[0], [int(t) for t in kv["codes"]])
    np.testing.assert_array_equal(oracle.pack(codes)[0], [int(t, 16) for t in kv["packed_hex"]])
    assert n == 8


@pytest.mark.parametrize("n", [256, 8192])
def test_spike_closed_form(n):
    # x = c e_k: every |x'| = c/sqrt(n), scale c/(7 sqrt(n)), codes +-7 = 7 s_k H[k, :]
    c, k = 3.0, 77
    s = synth.signs(n, 6)
    x = np.zeros((1, n), np.float16)
    x[0, k] = c
    packed, sc, xr = oracle.rotate_quant(x, s, 0, 0)
    assert abs(sc[0] - c / (7 * np.sqrt(n))) <= 1e-15
    H = oracle.sylvester(n) if n > 1024 else scipy.linalg.hadamard(n)
    np.testing.assert_array_equal(oracle.unpack(packed)[0], 7 * s[k] * H[k])


def test_quantizer_error_bound_and_range():
    x = synth.random_f16((64, 1024), 12, dist="student_t3")
    xr = oracle.rotate(x, synth.signs(1024, 12), 0)
    codes, sc = oracle.quantize(xr, 0)
    err = np.abs(xr - codes * sc[:, None])
    assert np.all(err <= sc[:, None] / 2 * (1 + 1e-12))
    assert codes.min() >= -8 and codes.max() <= 7
    # the absmax element of each row maps to +-7
    j = np.argmax(np.abs(xr), axis=1)
    np.testing.assert_array_equal(np.abs(codes[np.arange(64), j]), 7)


def test_quantizer_group_scale_is_fp16_of_absmax_over_7():
    x = synth.random_f16((8, 512), 13, dist="laplace")
    xr = oracle.rotate(x, synth.signs(512, 13), 128)
    codes, sc16 = oracle.quantize(xr, 128)
    amax = np.abs(xr.reshape(8, 4, 128)).max(axis=2)
    np.testing.assert_array_equal(sc16, _f16(amax / 7).view(np.uint16))
    s = sc16.view(np.float16).astype(np.float64)
    err = np.abs(xr.reshape(8, 4, 128) - codes.reshape(8, 4, 128) * s[:, :, None])
    assert np.all(err <= s[:, :, None] / 2 * (1 + 1e-12))


def test_quantizer_idempotent():
    x = synth.random_f16((16, 256), 14)
    codes, sc = oracle.quantize(oracle.rotate(x, synth.signs(256, 14), 0), 0)
    codes2, sc2 = oracle.quantize(codes * sc[:, None], 0)
    np.testing.assert_array_equal(codes, codes2)
    np.testing.assert_allclose(sc2, sc, rtol=1e-15)


def test_quantizer_ties_to_even_and_zero_row():
    xr = np.array([[7.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 0.0],
                   [0.0] * 8])
    codes, sc = oracle.quantize(xr, 0)
    assert sc[0] == 1.0 and sc[1] == 0.0
    np.testing.assert_array_equal(codes[0], [7, 2, 4, -2, 0, 0, 2, 0])
    np.testing.assert_array_equal(codes[1], 0)


def test_quantizer_clamps_when_fp16_scale_is_subnormal():
    # amax/7 = 1.4 * 2^-24 rounds to the subnormal 2^-24; v/s = +-9.8 -> clamp to 7 / -8
    a = 7 * 1.4 * 2.0 ** -24
    xr = np.zeros((1, 128))
    xr[0, 0], xr[0, 1], xr[0, 2] = a, -a, a / 9.8 * 2.0
    codes, sc16 = oracle.quantize(xr, 128)
    assert sc16[0, 0] == 1          # bit pattern of 2^-24
    assert codes[0, 0] == 7 and codes[0, 1] == -8 and codes[0, 2] == 2


def test_quantizer_zero_fp16_scale_gives_zero_codes():
    xr = np.zeros((1, 128))
    xr[0, :4] = [1e-9, -1e-9, 5e-10, 0.0]       # amax/7 underflows fp16 to 0
    codes, sc16 = oracle.quantize(xr, 128)
    assert sc16[0, 0] == 0
    np.testing.assert_array_equal(codes, 0)


# --------------------------------------------------------------------------
# packing and fp16
# --------------------------------------------------------------------------

def test_pack_unpack_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    c = oracle.unpack(b)
    np.testing.assert_array_equal(oracle.pack(c), b)
    lo = (b & 0xF).astype(np.int16)
    hi = (b >> 4).astype(np.int16)
    np.testing.assert_array_equal(c[0::2], np.where(lo >= 8, lo - 16, lo))
    np.testing.assert_array_equal(c[1::2], np.where(hi >= 8, hi - 16, hi))


def test_pack_nibble_order():
    # element 2i -> bits 0-3, element 2i+1 -> bits 4-7, two's complement
    np.testing.assert_array_equal(oracle.pack(np.array([1, -2, -8, 7], np.int8)), [0xE1, 0x78])


def test_f16_decode_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.f16_to_f64(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_f16_encode_matches_numpy():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 6, 200000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25,
                  3 * 2.0 ** -26, 2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]),
    ])
    # every fp16 value and the midpoints between neighbours (exact ties)
    v = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2
    x = np.concatenate([x, v, -v, mids, -mids])
    np.testing.assert_array_equal(oracle.f64_to_f16(x), x.astype(np.float16).view(np.uint16))


# --------------------------------------------------------------------------
# integer product and dequantization
# --------------------------------------------------------------------------

def _brute_gemm(qa, qw, group):
    M, K = qa.shape
    N = qw.shape[0]
    G = 1 if group == 0 else K // group
    w = K if group == 0 else group
    out = [[[0] * G for _ in range(N)] for _ in range(M)]
    for m in range(M):
        for n in range(N):
            for g in range(G):
                s = 0
                for k in range(g * w, (g + 1) * w):
                    s += int(qa[m, k]) * int(qw[n, k])
                out[m][n][g] = s
    return np.array(out, np.int64)


@pytest.mark.parametrize("group", [0, 128])
def test_int_gemm_brute_force(group):
    qa = synth.random_codes((3, 256), 40)
    qw = synth.random_codes((5, 256), 41)
    got = oracle.int_gemm(qa, qw, group)
    ref = _brute_gemm(qa, qw, group)
    np.testing.assert_array_equal(got.reshape(ref.shape), ref)


def test_int_gemm_identity_weights():
    qa = synth.random_codes((4, 128), 42)
    got = oracle.int_gemm(qa, np.eye(128, dtype=np.int8), 0)
    np.testing.assert_array_equal(got, qa.astype(np.int64))


def test_int_gemm_extremes_exact():
    # |acc| reaches 64 K: all -8 against all -8
    K = 8192
    qa = np.full((2, K), -8, np.int8)
    qw = np.full((3, K), -8, np.int8)
    qw[1] = 7
    got = oracle.int_gemm(qa, qw, 0)
    np.testing.assert_array_equal(got[:, 0], 64 * K)
    np.testing.assert_array_equal(got[:, 1], -56 * K)


def test_single_group_reduces_to_per_token():
    qa = synth.random_codes((6, 128), 43)
    qw = synth.random_codes((9, 128), 44)
    np.testing.assert_array_equal(oracle.int_gemm(qa, qw, 128)[:, :, 0], oracle.int_gemm(qa, qw, 0))


def test_dequant_linear_brute_force():
    rng = np.random.default_rng(45)
    acc = rng.integers(-5000, 5000, size=(3, 4, 2))
    sa = rng.random((3, 2))
    sw = rng.random((4, 2))
    y, y16 = oracle.dequant_linear(acc, sa, sw, group=128)
    for m in range(3):
        for n in range(4):
            ref = sum(float(acc[m, n, g]) * float(sa[m, g]) * float(sw[n, g]) for g in range(2))
            assert abs(y[m, n] - ref) <= 1e-12 * abs(ref)
            assert y16[m, n] == np.float16(ref).view(np.uint16)


def test_linear_error_bound_tiny_workload():
    # Composition pin (invariance + RTN bounds): with x' = q_a s_a + e_a, w' = q_w s_w + e_w,
    # |y - x.w| <= (s_a/2) sum|w'| + (s_w/2) sum|x'| + K s_a s_w / 4.
    w_ = synth.TINY
    x = synth.activations(w_)
    W = synth.weights(w_, 256)
    s = synth.signs(w_.K, w_.seed)
    out = oracle.linear(x, W, s, 0, 0)
    xr = oracle.rotate(x, s, 0)
    wr = oracle.rotate(W, s, 0)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    sa, sw = out["sa"], out["sw"]
    bound = (sa[:, None] / 2) * np.abs(wr).sum(1)[None, :] + \
        (sw[None, :] / 2) * np.abs(xr).sum(1)[:, None] + w_.K * sa[:, None] * sw[None, :] / 4
    assert np.all(np.abs(out["y"] - ref) <= bound * (1 + 1e-9))
    # and the bound is not vacuous: the error is far below |x||w|
    assert np.max(np.abs(out["y"] - ref)) < 0.25 * np.max(np.abs(ref)) + 1.0


# --------------------------------------------------------------------------
# KV cache
# --------------------------------------------------------------------------

def test_kv_quant_properties():
    c = synth.KV_70B
    k, v, q, s = synth.kv_inputs(c, batch=1)
    k, v = k[:, :32], v[:, :32]
    kq, ks, vq, vs = oracle.kv_quant(k, v, s)
    H128 = scipy.linalg.hadamard(128).astype(np.float64) / np.sqrt(128)
    kr = np.einsum("bthd,hd,de->bthe", k.astype(np.float64), s.astype(np.float64), H128)
    for rot, codes_p, sc in ((kr, kq, ks), (v.astype(np.float64), vq, vs)):
        codes = oracle.unpack(codes_p)
        amax = np.abs(rot).max(axis=-1)
        np.testing.assert_array_equal(sc, _f16(amax / 7).view(np.uint16))
        sv = sc.view(np.float16).astype(np.float64)
        assert np.all(np.abs(rot - codes * sv[..., None]) <= sv[..., None] / 2 * (1 + 1e-12))
        j = np.argmax(np.abs(rot), axis=-1)
        assert np.all(np.abs(np.take_along_axis(codes, j[..., None], -1)) >= 7)


def test_kv_scores_against_numpy():
    c = synth.KV_70B
    k, v, q, s = synth.kv_inputs(c, batch=2)
    k, v = k[:, :40], v[:, :40]
    kq, ks, _, _ = oracle.kv_quant(k, v, s)
    got = oracle.kv_scores(q, s, kq, ks)
    H128 = scipy.linalg.hadamard(128).astype(np.float64) / np.sqrt(128)
    grp = c.Hq // c.Hkv
    sq = np.repeat(s, grp, axis=0).astype(np.float64)          # [Hq, D]
    qr = np.einsum("bhd,hd,de->bhe", q.astype(np.float64), sq, H128)
    kd = oracle.unpack(kq) * ks.view(np.float16).astype(np.float64)[..., None]  # [B,T,H,D]
    kd = np.repeat(kd, grp, axis=2)                              # [B,T,Hq,D]
    ref = np.einsum("bhd,bthd->bht", qr, kd)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_kv_scores_spike_query_closed_form():
    # q = c e_j on every head: q' = c s_h[j] H[j]/sqrt(D); one key row of all-7 codes
    B, T, H, D, Hq = 1, 3, 2, 128, 4
    s = np.stack([synth.signs(D, 70), synth.signs(D, 71)])
    q = np.zeros((B, Hq, D), np.float16)
    j, c = 5, 2.0
    q[:, :, j] = c
    codes = np.zeros((B, T, H, D), np.int8)
    codes[0, 1] = 7
    kq = oracle.pack(codes)
    ks = np.full((B, T, H), np.float16(0.25)).view(np.uint16)
    got = oracle.kv_scores(q, s, kq, ks)
    Hm = scipy.linalg.hadamard(D)
    for hq in range(Hq):
        h = hq // (Hq // H)
        expect = c * s[h, j] * Hm[j].sum() / np.sqrt(D) * 7 * 0.25
        assert abs(got[0, hq, 1] - expect) <= 1e-12
        assert got[0, hq, 0] == 0 and got[0, hq, 2] == 0


def test_quantize_with_given_scales_matches_own_scales():
    # with the oracle's own scales the two routes agree; with halved scales codes saturate
    x = synth.random_f16((4, 256), 50)
    xr = oracle.rotate(x, synth.signs(256, 50), 0)
    codes, sc = oracle.quantize(xr, 0)
    np.testing.assert_array_equal(oracle.quantize_with_scales(xr, sc, 0), codes)
    xg = oracle.rotate(x, synth.signs(256, 51), 128)
    cg, sg = oracle.quantize(xg, 128)
    np.testing.assert_array_equal(oracle.quantize_with_scales(xg, sg, 128), cg)
    half = oracle.quantize_with_scales(xr, sc / 2, 0)
    j = np.argmax(np.abs(xr), axis=1)
    assert set(np.unique(half[np.arange(4), j])) <= {-8, 7}

"""Parity of the fused decode step quarot_kv_decode_attention with the oracle's
two steps, kv_attend(kv_scores(...)): query rotation, scores against the INT4
key cache, softmax of scores / sqrt(128), product with the INT4 value cache
(QuaRot abstract: the KV cache in 4 bits; DuQuant Knowl 12: Hadamard on the
query-key product, attention output x quantized values).

Tolerance, per output row (b, hq).  The kernel's scores differ from the
oracle's by at most

    eps_s = 2^-15 * max_t ks[t] * 8 * sum_d |q'[d]|

(the fp32 rotation of the query, its split into two fp16 parts carrying 22
bits, the fp32 sum of 128 exact products on the tensor core with at most 127
roundings of partial sums bounded by sum_d |q'[d] code[d] ks|, and the
scaling), i.e. 4x the sum of those bounds.  Softmax weights p of scores
perturbed by at most eps move by sum_t |dp_t| <= 2 eps / sqrt(128) in total,
so the output moves by at most that times max_t |vs_t code_t|.  The value
product itself is the attention tail's convex combination in fp32, bounded as
in the test of quarot_kv_decode_attend by 4 (T + 32) 2^-24 max_t |vs_t code_t|
(the weights' two-part fp16 split adds 2^-22 relative).  The weights come from
the hardware base-2 exponential (ex2.approx, a few ulp): with each weight off
by at most eps_x = 2^-21 relative, the normalized output moves by at most
2 eps_x max_t |vs_t code_t| (the rescale factors' errors cancel between the
accumulator and the sum of weights).  So

    |out - ref| <= (4 (T + 32) 2^-24 + 2^-20 + 2 eps_s / sqrt(128)) max_t |vs_t code_t|.
"""
import numpy as np
import pytest
import torch

import oracle
from rotation_bit_quantization_randomized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import __graft_entry__
    __graft_entry__.build()
    from rotation_bit_quantization_randomized_b200 import binding
    return binding


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _ok(q):
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0


def _bound(qh, s, kq, ks, vq, vs):
    B, Hq, D = qh.shape
    H = kq.shape[2]
    G = Hq // H
    T = kq.shape[1]
    # rotated queries in fp64: per-head block rotation of the [Hq * D] row
    qr = oracle.rotate(qh.reshape(B, Hq * D), np.repeat(s, G, axis=0).reshape(-1), 128).reshape(B, Hq, D)
    qsum = np.abs(qr).sum(axis=2)                                                   # [B, Hq]
    ksmax = np.repeat(oracle.f16_to_f64(ks).max(axis=1), G, axis=1)                 # [B, Hq]
    eps_s = 2.0 ** -15 * ksmax * 8.0 * qsum
    vmax = np.abs(oracle.unpack(vq).astype(np.float64) * oracle.f16_to_f64(vs)[..., None]).max(axis=(1, 3))
    vmax = np.repeat(vmax, G, axis=1)                                               # [B, Hq]
    return ((4.0 * (T + 32) * 2.0 ** -24 + 2.0 ** -20 + 2.0 * eps_s / np.sqrt(128.0)) * vmax)[..., None] + 1e-30


def _decode_check(q, qh, s, kq, ks, vq, vs):
    got = q.quarot_kv_decode_attention(_dev(qh), _dev(s), _dev(kq), _dev(ks.view(np.float16)), _dev(vq),
                                       _dev(vs.view(np.float16)))
    _ok(q)
    got = got.cpu().numpy().astype(np.float64)
    ref = oracle.kv_attend(oracle.kv_scores(qh, s, kq, ks), vq, vs)
    bound = _bound(qh, s, kq, ks, vq, vs)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), f"max error / bound {np.max(err / bound):.3f}"
    return got, ref, float(np.max(err / bound))


def _cache(rng, B, T, H, kscale=1.0):
    k = (rng.standard_normal((B, T, H, 128)) * kscale).astype(np.float16)
    v = rng.standard_normal((B, T, H, 128)).astype(np.float16)
    k[..., 5] *= np.float16(15.0)                     # an outlier key channel per head
    s = np.stack([synth.signs(128, 40 + hh) for hh in range(H)])
    kq, ks, vq, vs = oracle.kv_quant(k, v, s)
    return s, kq, ks, vq, vs


@pytest.mark.parametrize("B,T,H,G", [(1, 1, 8, 8), (1, 7, 8, 8), (2, 64, 8, 8), (2, 127, 4, 8), (1, 128, 2, 8),
                                      (1, 129, 2, 8), (2, 1000, 8, 8), (1, 2048, 8, 8), (1, 513, 2, 1),
                                      (2, 65, 4, 16), (1, 300, 3, 2), (1, 129, 2, 4), (1, 5000, 1, 16),
                                      (3, 257, 2, 8), (1, 4097, 2, 8)])
def test_decode_matches_oracle(q, B, T, H, G):
    rng = np.random.default_rng(11 * T + G + B)
    s, kq, ks, vq, vs = _cache(rng, B, T, H)
    qh = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    _decode_check(q, qh, s, kq, ks, vq, vs)


def test_decode_zero_query_averages_the_values(q):
    # all scores 0: uniform weights, the output is the mean dequantized value row
    rng = np.random.default_rng(5)
    B, T, H, G = 2, 300, 2, 8
    s, kq, ks, vq, vs = _cache(rng, B, T, H)
    qh = np.zeros((B, H * G, 128), np.float16)
    got, _, _ = _decode_check(q, qh, s, kq, ks, vq, vs)
    mean = (oracle.unpack(vq).astype(np.float64) * oracle.f16_to_f64(vs)[..., None]).mean(axis=1)   # [B, H, D]
    np.testing.assert_allclose(got, np.repeat(mean, G, axis=1), rtol=0, atol=1e-5 * np.abs(mean).max())


@pytest.mark.parametrize("qscale", [1e-4, 30.0, 3000.0])
def test_decode_query_magnitudes(q, qscale):
    # tiny queries (nearly uniform weights), large ones (one dominant token per head)
    rng = np.random.default_rng(int(qscale) + 9)
    B, T, H, G = 1, 700, 2, 8
    s, kq, ks, vq, vs = _cache(rng, B, T, H)
    qh = (rng.standard_normal((B, H * G, 128)) * qscale).astype(np.float16)
    _decode_check(q, qh, s, kq, ks, vq, vs)


def test_decode_equals_two_step_path(q):
    # the fused step and quarot_kv_decode_attend(quarot_kv_decode_scores(...)) agree
    rng = np.random.default_rng(21)
    B, T, H, G = 2, 1500, 8, 8
    s, kq, ks, vq, vs = _cache(rng, B, T, H)
    qh = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    args = (_dev(qh), _dev(s), _dev(kq), _dev(ks.view(np.float16)))
    fused = q.quarot_kv_decode_attention(*args, _dev(vq), _dev(vs.view(np.float16)))
    two = q.quarot_kv_decode_attend(q.quarot_kv_decode_scores(*args), _dev(vq), _dev(vs.view(np.float16)))
    _ok(q)
    bound = torch.from_numpy(2.0 * _bound(qh, s, kq, ks, vq, vs)).cuda()
    assert torch.all((fused.double() - two.double()).abs() <= bound)


def test_decode_full_size_sampled_batches(q):
    # the 70B GQA shape, B 64 x T 2048 x Hkv 8, 64 query heads, through the
    # device's own KV write; the oracle checks 3 sampled batches
    c = synth.KV_70B
    k, v, qh, s = synth.kv_inputs(c)
    kq, ks, vq, vs = q.quarot_kv_quant(_dev(k), _dev(v), _dev(s))
    got = q.quarot_kv_decode_attention(_dev(qh), _dev(s), kq, ks, vq, vs)
    _ok(q)
    rows = synth.sample_rows(c.B, 3, c.seed)
    kq_n, vq_n = kq.cpu().numpy()[rows], vq.cpu().numpy()[rows]
    ks_n, vs_n = ks.cpu().numpy().view(np.uint16)[rows], vs.cpu().numpy().view(np.uint16)[rows]
    ref = oracle.kv_attend(oracle.kv_scores(qh[rows], s, kq_n, ks_n), vq_n, vs_n)
    bound = _bound(qh[rows], s, kq_n, ks_n, vq_n, vs_n)
    err = np.abs(got.cpu().numpy()[rows].astype(np.float64) - ref)
    assert np.all(err <= bound), f"max error / bound {np.max(err / bound):.3f}"


@pytest.mark.parametrize("B,T", [(1, 2048), (16, 2048), (2, 1000)])
def test_decode_back_to_back(q, B, T):
    # many launches on one stream with no synchronization between them: the
    # same bytes as a lone launch, and no bounded wait runs out
    rng = np.random.default_rng(B + T)
    H, G = 8, 8
    s, kq, ks, vq, vs = _cache(rng, B, T, H)
    qh = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    args = (_dev(qh), _dev(s), _dev(kq), _dev(ks.view(np.float16)), _dev(vq), _dev(vs.view(np.float16)))
    ref = q.quarot_kv_decode_attention(*args)
    _ok(q)
    out = torch.empty_like(ref)
    for _ in range(60):
        q.quarot_kv_decode_attention(*args, out)
    _ok(q)
    assert torch.equal(out, ref)

"""Parity of the rest of the INT4 decode attention step, quarot_kv_decode_attend:
softmax over the tokens of scores / sqrt(128), times the dequantized INT4 value
cache, grouped-query heads (QuaRot abstract: the KV cache in 4 bits; DuQuant,
Knowl 12: the attention-output x value product on quantized values).

Tolerance.  The output row is a convex combination of dequantized value rows
(the weights are positive and sum to one), computed in fp32: each weight
carries a few roundings (the scaled score, its exponential, the normalising
sum over T terms, two products) and the T-term fp32 accumulation adds at most
T roundings of partial sums bounded by max|V|.  So

    |out - out_ref| <= 4 (T + 32) 2^-24 max_t |vs[t] * code[t, :]|

over the head's tokens, which the test states per output row."""
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


def _attend_check(q, scores32, vq, vs):
    B, Hq, T = scores32.shape
    H = vq.shape[2]
    got = q.quarot_kv_decode_attend(_dev(scores32), _dev(vq), _dev(vs.view(np.float16)))
    _ok(q)
    got = got.cpu().numpy().astype(np.float64)
    ref = oracle.kv_attend(scores32.astype(np.float64), vq, vs)
    vmax = np.abs(oracle.unpack(vq).astype(np.float64) * oracle.f16_to_f64(vs)[..., None]).max(axis=(1, 3))  # [B, H]
    vmax = np.repeat(vmax, Hq // H, axis=1)[..., None]                                          # [B, Hq, 1]
    bound = 4.0 * (T + 32) * 2.0 ** -24 * vmax + 1e-30
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), f"max error / bound {np.max(err / bound):.3f}"
    return float(np.max(err / bound))


def _values(rng, B, T, H):
    v = rng.standard_normal((B, T, H, 128)).astype(np.float16)
    k = np.zeros_like(v)
    s = np.ones((H, 128), np.int8)
    _, _, vq, vs = oracle.kv_quant(k, v, s)
    return vq, vs


@pytest.mark.parametrize("B,T,H,G", [(1, 1, 8, 8), (1, 7, 8, 8), (2, 64, 8, 8), (2, 1000, 8, 8),
                                      (1, 513, 2, 1), (2, 65, 4, 16), (1, 300, 3, 2), (1, 129, 2, 4),
                                      (1, 1500, 2, 8), (1, 5000, 1, 16), (3, 257, 2, 8)])
def test_attend_matches_oracle(q, B, T, H, G):
    rng = np.random.default_rng(7 * T + G)
    vq, vs = _values(rng, B, T, H)
    scores = (rng.standard_normal((B, H * G, T)) * 30).astype(np.float32)
    _attend_check(q, scores, vq, vs)


def test_attend_one_token_returns_its_value_row(q):
    rng = np.random.default_rng(3)
    vq, vs = _values(rng, 2, 1, 4)
    scores = rng.standard_normal((2, 8, 1)).astype(np.float32) * 100
    got = q.quarot_kv_decode_attend(_dev(scores), _dev(vq), _dev(vs.view(np.float16)))
    _ok(q)
    row = oracle.unpack(vq).astype(np.float64) * oracle.f16_to_f64(vs)[..., None]       # [2, 1, 4, 128]
    expect = np.repeat(row[:, 0], 2, axis=1)                                              # [2, 8, 128]
    np.testing.assert_array_equal(got.cpu().numpy().astype(np.float64), expect)


def test_attend_dominant_score_and_uniform_scores(q):
    rng = np.random.default_rng(5)
    B, T, H, G = 1, 300, 2, 4
    vq, vs = _values(rng, B, T, H)
    scores = np.zeros((B, H * G, T), np.float32)
    scores[0, :G, 123] = 1.0e4             # heads of KV head 0 pick token 123
    _attend_check(q, scores, vq, vs)
    got = q.quarot_kv_decode_attend(_dev(scores), _dev(vq), _dev(vs.view(np.float16))).cpu().numpy()
    _ok(q)
    rows = oracle.unpack(vq).astype(np.float64) * oracle.f16_to_f64(vs)[..., None]
    np.testing.assert_allclose(got[0, :G], np.repeat(rows[0, 123, 0][None], G, 0), rtol=0, atol=1e-6)
    # KV head 1: all scores equal -> the plain mean of the value rows
    np.testing.assert_allclose(got[0, G:], np.repeat(rows[0, :, 1].mean(0)[None], G, 0),
                               rtol=0, atol=4 * (T + 32) * 2.0 ** -24 * np.abs(rows[0, :, 1]).max())


@pytest.mark.parametrize("slope", [1.0, -1.0])
def test_attend_running_maximum_across_chunks(q, slope):
    """Scores that rise (or fall) along the tokens: with a rising ramp every
    chunk of every token slice raises the running maximum, so the rescaling of
    the partial sums is exercised at each step."""
    rng = np.random.default_rng(11)
    B, T, H, G = 1, 6000, 2, 8
    vq, vs = _values(rng, B, T, H)
    ramp = slope * np.linspace(0.0, 400.0, T)
    scores = (ramp[None, None, :] + rng.standard_normal((B, H * G, T)) * 5).astype(np.float32)
    _attend_check(q, scores, vq, vs)


def test_attend_empty_batch_is_a_no_op(q):
    out = torch.full((0, 8, 128), 7.0, device="cuda")
    q.quarot_kv_decode_attend(torch.empty((0, 8, 5), device="cuda"),
                              torch.empty((0, 5, 1, 64), dtype=torch.uint8, device="cuda"),
                              torch.empty((0, 5, 1), dtype=torch.float16, device="cuda"), out=out)
    _ok(q)


def test_attend_full_size_on_oracle_scores(q):
    """The llama2-70b decode workload (Hkv 8, 64 query heads, T 2048, D 128) on
    a batch slice: keys and values written by the oracle's KV quantizer, scores
    from the oracle's decode scores, so the whole decode attention step is
    checked on realistic inputs (outlier key channels, Gaussian values)."""
    c = synth.KV_70B
    k, v, qh, s = synth.kv_inputs(c, batch=4)
    kq, ks, vq, vs = oracle.kv_quant(k, v, s)
    scores = oracle.kv_scores(qh, s, kq, ks).astype(np.float32)
    _attend_check(q, scores, vq, vs)

"""Parity of the INT4 KV-cache path: quarot_kv_quant and quarot_kv_decode_scores."""
import numpy as np
import pytest
import torch

import oracle
from parity import check_codes
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


def _kv_check(q, k, v, s, rows=None):
    kq, ks, vq, vs = q.quarot_kv_quant(_dev(k), _dev(v), _dev(s))
    _ok(q)
    B, T, H, D = k.shape
    kq = kq.cpu().numpy().reshape(B * T, H * D // 2)
    vq = vq.cpu().numpy().reshape(B * T, H * D // 2)
    ks = ks.cpu().numpy().view(np.uint16).reshape(B * T, H)
    vs = vs.cpu().numpy().view(np.uint16).reshape(B * T, H)
    kf = k.reshape(B * T, H * D)
    vf = v.reshape(B * T, H * D)
    if rows is not None:
        kf, vf, kq, vq, ks, vs = kf[rows], vf[rows], kq[rows], vq[rows], ks[rows], vs[rows]
    # keys: per-head rotation = block rotation of the [H*D] row with the concatenated signs
    check_codes(kq, ks, oracle.rotate(kf, s.reshape(-1), D), D)
    check_codes(vq, vs, oracle.f16_to_f64(vf), D)


@pytest.mark.parametrize("B,T,H", [(1, 5, 8), (2, 64, 8), (3, 33, 1), (1, 17, 40), (3, 2001, 8), (1, 700, 16)])
def test_kv_quant_matches_oracle(q, B, T, H):
    rng = np.random.default_rng(B * 100 + T + H)
    k = (rng.standard_normal((B, T, H, 128)) * 2).astype(np.float16)
    v = rng.standard_normal((B, T, H, 128)).astype(np.float16)
    k[0, 0, 0, 5] = 40.0
    v[0, 0, 0] = 0                         # zero value row
    s = np.stack([synth.signs(128, 20 + h) for h in range(H)])
    _kv_check(q, k, v, s)


def test_kv_quant_full_size_sampled(q):
    c = synth.KV_70B
    k, v, _, s = synth.kv_inputs(c)
    rows = synth.sample_rows(c.B * c.T, 256, c.seed)
    _kv_check(q, k, v, s, rows)


def _scores_check(q, qh, s, kq, ks, tol=1e-5):
    got = q.quarot_kv_decode_scores(_dev(qh), _dev(s), _dev(kq), _dev(ks.view(np.float16)))
    _ok(q)
    got = got.cpu().numpy().astype(np.float64)
    ref = oracle.kv_scores(qh, s, kq, ks)
    # fp32 rotation (7 exact-order stages) and a 128-term fp32 sum: error well
    # under 1e-5 of the largest |score| of the row
    scale = np.abs(ref).max(axis=-1, keepdims=True) + 1e-30
    err = np.abs(got - ref) / scale
    assert err.max() <= tol, f"max scaled error {err.max():.3e}"


@pytest.mark.parametrize("B,T,H,G", [(1, 7, 8, 8), (2, 1000, 8, 8), (1, 513, 2, 1), (2, 64, 4, 16),
                                      (1, 300, 3, 2), (1, 128, 2, 4)])
def test_kv_scores_matches_oracle(q, B, T, H, G):
    rng = np.random.default_rng(T + G)
    k = (rng.standard_normal((B, T, H, 128))).astype(np.float16)
    v = np.zeros_like(k)
    s = np.stack([synth.signs(128, 40 + h) for h in range(H)])
    kq, ks, _, _ = oracle.kv_quant(k, v, s)
    qh = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    _scores_check(q, qh, s, kq, ks)


@pytest.mark.parametrize("qscale", [0.0, 1e-6, 1e-3, 300.0])
def test_kv_scores_query_magnitudes(q, qscale):
    """Zero, tiny and large queries: the scores must keep their relative
    accuracy at every scale (a zero query gives exactly zero scores)."""
    rng = np.random.default_rng(int(qscale * 1e6) % 1000 + 3)
    B, T, H, G = 1, 200, 2, 8
    k = rng.standard_normal((B, T, H, 128)).astype(np.float16)
    s = np.stack([synth.signs(128, 60 + h) for h in range(H)])
    kq, ks, _, _ = oracle.kv_quant(k, np.zeros_like(k), s)
    qh = (rng.standard_normal((B, H * G, 128)) * qscale).astype(np.float16)
    if qscale == 0.0:
        got = q.quarot_kv_decode_scores(_dev(qh), _dev(s), _dev(kq), _dev(ks.view(np.float16)))
        _ok(q)
        np.testing.assert_array_equal(got.cpu().numpy(), 0.0)
    else:
        _scores_check(q, qh, s, kq, ks)


def test_kv_scores_full_size_sampled(q):
    c = synth.KV_70B
    k, v, qh, s = synth.kv_inputs(c, batch=4)
    kq, ks, _, _ = oracle.kv_quant(k, v, s)
    _scores_check(q, qh, s, kq, ks)


@pytest.mark.parametrize("B,T", [(1, 2048), (4, 2048), (2, 1000), (3, 129)])
def test_kv_scores_back_to_back(q, B, T):
    # many launches on one stream with no synchronization between them: every
    # one gives the same bytes as a lone launch and no wait runs out (a
    # hand-off barrier that could run two phases ahead of its waiter would
    # show here as a timeout)
    rng = np.random.default_rng(B * T)
    H, G = 8, 8
    k = rng.standard_normal((B, T, H, 128)).astype(np.float16)
    s = np.stack([synth.signs(128, 40 + h) for h in range(H)])
    kq, ks, _, _ = oracle.kv_quant(k, np.zeros_like(k), s)
    qh = rng.standard_normal((B, H * G, 128)).astype(np.float16)
    args = (_dev(qh), _dev(s), _dev(kq), _dev(ks.view(np.float16)))
    ref = q.quarot_kv_decode_scores(*args)
    _ok(q)
    out = torch.empty_like(ref)
    for _ in range(60):
        q.quarot_kv_decode_scores(*args, out)
    _ok(q)
    assert torch.equal(out, ref)

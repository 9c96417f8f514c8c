"""Parity of the 8-bit variant (quarot_rotate_quant_i8, quarot_int8_gemm_s32,
quarot_int8_linear, quarot_rotate_quant_linear_i8) with the oracle.

Integer results from identical codes must be bit-exact; the quantizer follows
the code rule of tests/parity.py at 8 bits; fp16 outputs follow the output
rule against the oracle's fp64 product of the same codes and scales.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import check_codes_bits, check_f16_output
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


QCASES = [
    # (K, had_block, M)
    (128, 0, 3), (256, 0, 37), (1024, 0, 17), (4096, 0, 70), (8192, 0, 45),
    (128, 128, 257), (1024, 128, 19), (11008, 128, 11), (28672, 128, 5), (384, 128, 130),
]


@pytest.mark.parametrize("K,hb,M", QCASES)
def test_rotate_quant_i8_matches_oracle(q, K, hb, M):
    x = synth.random_f16((M, K), 500 + K + M, dist="student_t3", scale=2.0)
    s = synth.signs(K, K + hb + 1)
    qc, sc = q.quarot_rotate_quant_i8(_dev(x), _dev(s), hb)
    _ok(q)
    check_codes_bits(qc.cpu().numpy(), sc.cpu().numpy().astype(np.float64), oracle.rotate(x, s, hb), 8)


@pytest.mark.parametrize("K,hb", [(8192, 0), (11008, 128)])
def test_rotate_quant_i8_zero_spike_constant_rows(q, K, hb):
    x = synth.random_f16((5, K), 9, dist="laplace")
    x[1] = 0
    x[2] = 0
    x[2, 77] = 3.0
    x[3] = np.float16(-0.5)
    x[4, ::2] = np.float16(60000.0)
    s = synth.signs(K, 8)
    qc, sc = q.quarot_rotate_quant_i8(_dev(x), _dev(s), hb)
    _ok(q)
    scn = sc.cpu().numpy().astype(np.float64)
    assert scn[1] == 0 and np.all(qc.cpu().numpy()[1] == 0)
    check_codes_bits(qc.cpu().numpy(), scn, oracle.rotate(x, s, hb), 8)


S32_SHAPES = [(128, 256, 128), (1, 8, 128), (200, 264, 384), (300, 520, 1024), (129, 256, 8192),
              (257, 1000, 256), (64, 4096, 512), (4500, 2248, 128)]


@pytest.mark.parametrize("M,N,K", S32_SHAPES)
def test_int8_s32_bit_exact(q, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    ca = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    cw = rng.integers(-128, 128, size=(N, K)).astype(np.int8)
    acc = q.quarot_int8_gemm_s32(_dev(ca), _dev(cw))
    _ok(q)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), oracle.int_gemm(ca, cw))


def test_int8_s32_extremes(q):
    # |acc| up to 2^14 K: -128 x -128 and -128 x 127 over K = 65536 stay inside int32
    K = 65536
    ca = np.full((130, K), -128, np.int8)
    ca[1] = 127
    cw = np.full((16, K), -128, np.int8)
    cw[3] = 127
    cw[5, ::2] = 127
    acc = q.quarot_int8_gemm_s32(_dev(ca), _dev(cw))
    _ok(q)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), oracle.int_gemm(ca, cw))


def _prep8(x, W, s, hb):
    qa, sa, _ = oracle.rotate_quant8(x, s, hb)
    qw, sw, _ = oracle.rotate_quant8(W, s, hb)
    return qa, sa.astype(np.float32), qw, sw.astype(np.float32)


def _ref8(qa, sa, qw, sw):
    acc = oracle.int_gemm(qa, qw, 0)
    y, _ = oracle.dequant_linear(acc, sa.astype(np.float64), sw.astype(np.float64), 0)
    return y


@pytest.mark.parametrize("M,N,K,hb", [
    (16, 256, 256, 0), (130, 264, 1024, 0), (1, 8, 128, 0), (257, 512, 4096, 0), (200, 520, 11008, 128),
    (33, 128, 8192, 0),
])
def test_int8_linear_matches_oracle(q, M, N, K, hb):
    x = synth.random_f16((M, K), 600 + M, dist="student_t3")
    W = synth.random_f16((N, K), 601 + N, scale=0.02)
    s = synth.signs(K, 602)
    qa, sa, qw, sw = _prep8(x, W, s, hb)
    y = q.quarot_int8_linear(_dev(qa), _dev(sa), _dev(qw), _dev(sw))
    _ok(q)
    check_f16_output(y.cpu().numpy(), _ref8(qa, sa, qw, sw))


@pytest.mark.parametrize("wid", [1, 2])
def test_int8_fused_equals_separate_and_oracle(q, wid):
    w = synth.LINEARS[wid]
    rows = min(w.M, 160)
    N = w.Ns[0]
    x = synth.activations(w, rows=rows)
    W = synth.weights(w, N)
    s = synth.signs(w.K, w.seed)
    hb = w.had_block
    xt, Wt, st = _dev(x), _dev(W), _dev(s)
    qw, sw = q.quarot_rotate_quant_i8(Wt, st, hb)
    y = q.quarot_rotate_quant_linear_i8(xt, st, qw, sw, hb)
    qa, sa = q.quarot_rotate_quant_i8(xt, st, hb)
    y2 = q.quarot_int8_linear(qa, sa, qw, sw)
    _ok(q)
    assert torch.equal(y, y2)
    check_codes_bits(qa.cpu().numpy(), sa.cpu().numpy().astype(np.float64), oracle.rotate(x, s, hb), 8)
    check_codes_bits(qw.cpu().numpy(), sw.cpu().numpy().astype(np.float64), oracle.rotate(W, s, hb), 8)
    # the device codes and scales through the oracle's product give the device output
    ref = _ref8(qa.cpu().numpy(), sa.cpu().numpy(), qw.cpu().numpy(), sw.cpu().numpy())
    check_f16_output(y.cpu().numpy(), ref)


def test_int8_llama2_70b_slice_sampled_rows(q):
    # 4096 tokens of the 70B prefill shape through the fused INT8 path; oracle on sampled rows
    w = synth.LLAMA2_70B
    x = synth.activations(w, rows=4096)
    s = synth.signs(w.K, w.seed)
    W = synth.weights(w, w.Ns[0])
    qw, sw, _ = oracle.rotate_quant8(W, s, 0)
    del W
    y = q.quarot_rotate_quant_linear_i8(_dev(x), _dev(s), _dev(qw), _dev(sw.astype(np.float32)), 0)
    qa, sa = q.quarot_rotate_quant_i8(_dev(x), _dev(s), 0)
    _ok(q)
    rows = synth.sample_rows(4096, 6, w.seed)
    qa_n = qa.cpu().numpy()[rows]
    sa_n = sa.cpu().numpy()[rows]
    check_codes_bits(qa_n, sa_n.astype(np.float64), oracle.rotate(x[rows], s, 0), 8)
    ref = _ref8(qa_n, sa_n, qw, sw.astype(np.float32))
    check_f16_output(y.cpu().numpy()[rows], ref)

"""Parity of the 6-bit variant (quarot_rotate_quant_i6, and the INT8 tensor-core
linear fed with 6-bit codes through quarot_rotate_quant_linear_i6) with the
oracle.

The quantizer follows the code rule of tests/parity.py at 6 bits; integer
products of identical codes are bit-exact; fp16 outputs follow the output
rule against the oracle's fp64 product of the device's own codes and scales.
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
    (128, 0, 5), (256, 0, 37), (2048, 0, 19), (4096, 0, 70), (8192, 0, 45),
    (128, 128, 131), (11008, 128, 13), (384, 128, 129),
]


@pytest.mark.parametrize("K,hb,M", QCASES)
def test_rotate_quant_i6_matches_oracle(q, K, hb, M):
    x = synth.random_f16((M, K), 700 + K + M, dist="student_t3", scale=2.0)
    s = synth.signs(K, K + hb + 3)
    qc, sc = q.quarot_rotate_quant_i6(_dev(x), _dev(s), hb)
    _ok(q)
    qn = qc.cpu().numpy()
    assert qn.min() >= -31 and qn.max() <= 31
    check_codes_bits(qn, sc.cpu().numpy().astype(np.float64), oracle.rotate(x, s, hb), 6)


def test_rotate_quant_i6_zero_spike_and_constant_rows(q):
    K = 4096
    x = synth.random_f16((4, K), 19, dist="laplace")
    x[1] = 0
    x[2] = 0
    x[2, 301] = -7.0
    x[3] = np.float16(0.25)
    s = synth.signs(K, 20)
    qc, sc = q.quarot_rotate_quant_i6(_dev(x), _dev(s), 0)
    _ok(q)
    qn, scn = qc.cpu().numpy(), sc.cpu().numpy().astype(np.float64)
    assert scn[1] == 0 and np.all(qn[1] == 0)
    # a spike: every code is 31 times the sign of its Hadamard entry (closed form)
    H2 = oracle.sylvester(K)[301]
    np.testing.assert_array_equal(qn[2], (-31 * s[301] * H2).astype(np.int8))
    check_codes_bits(qn, scn, oracle.rotate(x, s, 0), 6)


@pytest.mark.parametrize("wid", [1, 2])
def test_int6_fused_equals_separate_and_oracle(q, wid):
    w = synth.LINEARS[wid]
    rows = min(w.M, 160)
    N = w.Ns[0]
    x = synth.activations(w, rows=rows)
    W = synth.weights(w, N)
    s = synth.signs(w.K, w.seed)
    hb = w.had_block
    xt, Wt, st = _dev(x), _dev(W), _dev(s)
    qw, sw = q.quarot_rotate_quant_i6(Wt, st, hb)
    y = q.quarot_rotate_quant_linear_i6(xt, st, qw, sw, hb)
    qa, sa = q.quarot_rotate_quant_i6(xt, st, hb)
    y2 = q.quarot_int8_linear(qa, sa, qw, sw)
    acc = q.quarot_int8_gemm_s32(qa, qw)
    _ok(q)
    assert torch.equal(y, y2)
    qa_n, qw_n = qa.cpu().numpy(), qw.cpu().numpy()
    check_codes_bits(qa_n, sa.cpu().numpy().astype(np.float64), oracle.rotate(x, s, hb), 6)
    check_codes_bits(qw_n, sw.cpu().numpy().astype(np.float64), oracle.rotate(W, s, hb), 6)
    ref_acc = oracle.int_gemm(qa_n, qw_n, 0)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), ref_acc)
    ref, _ = oracle.dequant_linear(ref_acc, sa.cpu().numpy().astype(np.float64),
                                   sw.cpu().numpy().astype(np.float64), 0)
    check_f16_output(y.cpu().numpy(), ref)

"""Parity of the tensor-core INT4 GEMM (quarot_int4_gemm_s32, quarot_int4_linear).

Inputs are produced by the oracle (codes and scales from seeded data), so the
GEMM is checked in isolation from the quantizer: int32 accumulators must be
bit-exact, fp16 outputs within the output rule of tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import check_f16_output
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


S32_SHAPES = [(128, 256, 128), (1, 8, 128), (200, 264, 384), (300, 520, 1024), (129, 256, 8192),
              (257, 1000, 256), (64, 4096, 512), (4500, 2248, 128)]


@pytest.mark.parametrize("M,N,K", S32_SHAPES)
def test_s32_bit_exact_random_codes(q, M, N, K):
    ca = synth.random_codes((M, K), M + K)
    cw = synth.random_codes((N, K), N + K + 1)
    acc = q.quarot_int4_gemm_s32(_dev(oracle.pack(ca)), _dev(oracle.pack(cw)))
    _ok(q)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), oracle.int_gemm(ca, cw))


def test_s32_extremes(q):
    K = 8192
    ca = np.full((130, K), -8, np.int8)
    ca[1] = 7
    cw = np.full((264, K), -8, np.int8)
    cw[3] = 7
    cw[5, ::2] = 7
    acc = q.quarot_int4_gemm_s32(_dev(oracle.pack(ca)), _dev(oracle.pack(cw)))
    _ok(q)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), oracle.int_gemm(ca, cw))


def _prep(x, W, s, hb, group):
    """Oracle codes and scales for both operands (scales as the library stores them)."""
    qa, sa, _ = oracle.rotate_quant(x, s, hb, group)
    qw, sw, _ = oracle.rotate_quant(W, s, hb, group)
    if group == 0:
        sa = sa.astype(np.float32)
        sw = sw.astype(np.float32)
    return qa, sa, qw, sw


def _linear(q, qa, sa, qw, sw, group):
    sat = _dev(sa.view(np.float16) if group else sa)
    swt = _dev(sw.view(np.float16) if group else sw)
    y = q.quarot_int4_linear(_dev(qa), sat, _dev(qw), swt, group)
    _ok(q)
    return y.cpu().numpy()


def _ref(qa, sa, qw, sw, group):
    acc = oracle.int_gemm(oracle.unpack(qa), oracle.unpack(qw), group)
    sa64 = sa.astype(np.float64) if group == 0 else sa
    sw64 = sw.astype(np.float64) if group == 0 else sw
    y, _ = oracle.dequant_linear(acc, sa64, sw64, group)
    return y


@pytest.mark.parametrize("M,N,K,hb,group", [
    (16, 256, 256, 0, 0), (130, 264, 1024, 0, 0), (1, 8, 128, 0, 0), (257, 512, 4096, 0, 0),
    (64, 256, 128, 128, 128), (130, 136, 1024, 128, 128), (200, 520, 11008, 128, 128),
    (33, 128, 8192, 0, 128),
])
def test_linear_fp16_matches_oracle(q, M, N, K, hb, group):
    x = synth.random_f16((M, K), 300 + M, dist="student_t3")
    W = synth.random_f16((N, K), 301 + N, scale=0.02)
    s = synth.signs(K, 302)
    qa, sa, qw, sw = _prep(x, W, s, hb, group)
    check_f16_output(_linear(q, qa, sa, qw, sw, group), _ref(qa, sa, qw, sw, group))


@pytest.mark.parametrize("wid", [1, 2, 3])
def test_workload_shapes(q, wid):
    w = synth.LINEARS[wid]
    rows = min(w.M, 192)
    x = synth.activations(w, rows=rows)
    s = synth.signs(w.K, w.seed)
    for N in w.Ns:
        W = synth.weights(w, N)
        qa, sa, qw, sw = _prep(x, W, s, w.had_block, w.group)
        check_f16_output(_linear(q, qa, sa, qw, sw, w.group), _ref(qa, sa, qw, sw, w.group))


def test_llama2_70b_full_size_sampled_rows(q):
    # full 32768 x 28672 x 8192 GEMM on oracle codes; oracle outputs on sampled rows
    w = synth.LLAMA2_70B
    x = synth.activations(w)
    s = synth.signs(w.K, w.seed)
    W = synth.weights(w, w.Ns[0])
    qa, sa, qw, sw = _prep(x, W, s, 0, 0)
    del x, W
    y = _linear(q, qa, sa, qw, sw, 0)
    rows = synth.sample_rows(w.M, 8, w.seed)
    check_f16_output(y[rows], _ref(qa[rows], sa[rows], qw, sw, 0))

"""Parity of the asymmetric INT4 variant (quarot_rotate_quant_asym,
quarot_uint4_gemm_s32, quarot_int4_linear_asym) with the oracle: the
quantizer under the asymmetric code rule of tests/parity.py, the unsigned
integer product bit-exact, fp16 outputs under the output rule."""
import numpy as np
import pytest
import torch

import oracle
from parity import check_codes_asym, check_f16_output
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


@pytest.mark.parametrize("K,M,clip", [(256, 37, 0.9), (512, 33, 1.0), (1024, 17, 0.8), (4096, 70, 0.9),
                                      (8192, 45, 0.9), (8192, 3, 1.0)])
def test_rotate_quant_asym_matches_oracle(q, K, M, clip):
    x = synth.random_f16((M, K), 700 + K + M, dist="student_t3", scale=2.0)
    s = synth.signs(K, K + 7)
    qp, d, z, r = q.quarot_rotate_quant_asym(_dev(x), _dev(s), clip)
    _ok(q)
    check_codes_asym(qp.cpu().numpy(), d.cpu().numpy(), z.cpu().numpy(), r.cpu().numpy(),
                     oracle.rotate(x, s, 0), clip)


def test_rotate_quant_asym_zero_spike_constant_rows(q):
    K = 8192
    x = synth.random_f16((5, K), 11, dist="laplace")
    x[1] = 0
    x[2] = 0
    x[2, 77] = 3.0                    # spike: every |x'| equal, two values
    x[3] = np.float16(-0.5)           # constant row: rotates to a single spike
    x[4, ::2] = np.float16(60000.0)
    s = synth.signs(K, 12)
    qp, d, z, r = q.quarot_rotate_quant_asym(_dev(x), _dev(s), 0.9)
    _ok(q)
    dn = d.cpu().numpy()
    assert dn[1] == 0 and z.cpu().numpy()[1] == 0 and r.cpu().numpy()[1] == 0
    check_codes_asym(qp.cpu().numpy(), dn, z.cpu().numpy(), r.cpu().numpy(), oracle.rotate(x, s, 0), 0.9)


S32_SHAPES = [(128, 256, 128), (1, 8, 128), (200, 264, 384), (129, 256, 8192), (257, 1000, 256), (4500, 2248, 128)]


@pytest.mark.parametrize("M,N,K", S32_SHAPES)
def test_uint4_s32_bit_exact(q, M, N, K):
    rng = np.random.default_rng(M + 3 * N + K)
    pa = rng.integers(0, 256, size=(M, K // 2)).astype(np.uint8)
    pw = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
    acc = q.quarot_uint4_gemm_s32(_dev(pa), _dev(pw))
    _ok(q)
    ua = oracle.unpack(pa) & 0x0F
    uw = oracle.unpack(pw) & 0x0F
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), oracle.int_gemm(ua, uw))


def test_uint4_s32_extremes(q):
    K = 65536
    pa = np.full((130, K // 2), 0xFF, np.uint8)      # all codes 15
    pa[1] = 0x00
    pw = np.full((16, K // 2), 0xFF, np.uint8)
    pw[3, ::2] = 0x0F
    acc = q.quarot_uint4_gemm_s32(_dev(pa), _dev(pw))
    _ok(q)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64),
                                  oracle.int_gemm(oracle.unpack(pa) & 0x0F, oracle.unpack(pw) & 0x0F))


def _prep(x, W, s, ca, cw):
    qa, da, za, ra, _ = oracle.rotate_quant_asym(x, s, ca, 0)
    qw, dw, zw, rw, _ = oracle.rotate_quant_asym(W, s, cw, 0)
    f32 = lambda a: np.asarray(a, np.float32)
    i32 = lambda a: np.asarray(a, np.int32)
    return (qa, f32(da), i32(za), i32(ra)), (qw, f32(dw), i32(zw), i32(rw))


def _ref(A, Wq, K):
    qa, da, za, ra = A
    qw, dw, zw, rw = Wq
    acc = oracle.int_gemm(oracle.unpack(qa) & 0x0F, oracle.unpack(qw) & 0x0F)
    y, _ = oracle.dequant_asym(acc, K, da.astype(np.float64), za, ra, dw.astype(np.float64), zw, rw)
    return y


@pytest.mark.parametrize("M,N,K", [(16, 256, 256), (130, 264, 1024), (1, 8, 256), (257, 520, 4096), (33, 128, 8192)])
def test_linear_asym_matches_oracle(q, M, N, K):
    x = synth.random_f16((M, K), 800 + M, dist="student_t3")
    W = synth.random_f16((N, K), 801 + N, scale=0.02)
    s = synth.signs(K, 802)
    A, Wq = _prep(x, W, s, 0.9, 0.8)
    y = q.quarot_int4_linear_asym(*(_dev(a) for a in A), *(_dev(w) for w in Wq))
    _ok(q)
    check_f16_output(y.cpu().numpy(), _ref(A, Wq, K))


def test_asym_device_path_end_to_end(q):
    # device quantizer on both operands, device linear; the oracle's product of
    # the device codes gives the device output, and the codes obey the rule
    w = synth.LLAMA2_7B
    x = synth.activations(w, rows=160)
    W = synth.weights(w, w.Ns[0])
    s = synth.signs(w.K, w.seed)
    xa = q.quarot_rotate_quant_asym(_dev(x), _dev(s), 0.9)
    wa = q.quarot_rotate_quant_asym(_dev(W), _dev(s), 0.8)
    y = q.quarot_int4_linear_asym(*xa, *wa)
    _ok(q)
    A = tuple(t.cpu().numpy() for t in xa)
    Wq = tuple(t.cpu().numpy() for t in wa)
    check_codes_asym(*A, oracle.rotate(x, s, 0), 0.9)
    check_codes_asym(*Wq, oracle.rotate(W, s, 0), 0.8)
    check_f16_output(y.cpu().numpy(), _ref(A, Wq, w.K))

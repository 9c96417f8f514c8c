"""Parity of the full Kronecker rotation for K = 11008 = 344 * 32 fused with
INT4 RTN (quarot_rotate_quant_kron) against the oracle's rotate_kron +
quantize: x' = (x diag(s)) (H_344 (x) H_32) / sqrt(K), H_344 a Paley factor
(QuaRot summary, Elamur Research, Summary and Key points; References item 24
for non-power-of-two factors).  The code and scale rules are those of the
other rotation kernels (parity.check_codes): the kernel sums in fp32 on the
tensor cores, the oracle in fp64, so codes may differ only at near-ties."""
import numpy as np
import pytest
import torch

import oracle
from parity import check_codes
from rotation_bit_quantization_randomized_b200 import synth

pytestmark = pytest.mark.gpu
K = 11008


@pytest.fixture(scope="module")
def q():
    import __graft_entry__
    __graft_entry__.build()
    from rotation_bit_quantization_randomized_b200 import binding
    return binding


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(q, x, s, group):
    qa, sc = q.quarot_rotate_quant_kron(_dev(x), _dev(s), group)
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    sc = sc.cpu().numpy()
    return qa.cpu().numpy(), (sc if group == 0 else sc.view(np.uint16))


@pytest.mark.parametrize("group", [0, 128])
@pytest.mark.parametrize("M", [1, 3, 4, 5, 64, 150, 301])
def test_kron_matches_oracle(q, M, group):
    x = synth.random_f16((M, K), 500 + M, dist="laplace")
    x[:, [17, 4000, 9001]] *= 40                      # a few outlier channels
    s = synth.signs(K, 77 + M)
    qa, sc = _run(q, x, s, group)
    check_codes(qa, sc, oracle.rotate_kron(x, s), group)


@pytest.mark.parametrize("group", [0, 128])
def test_kron_full_size_sampled(q, group):
    """The down-projection workload (2048 tokens, Laplace activations with 4
    channels x500): every row through the kernel in the launch the benchmark
    times, 96 sampled rows through the oracle."""
    w = synth.DOWN_PROJ
    x = synth.activations(w)
    s = synth.signs(K, w.seed)
    qa, sc = _run(q, x, s, group)
    rows = synth.sample_rows(w.M, 96, w.seed)
    check_codes(qa[rows], sc[rows], oracle.rotate_kron(x[rows], s), group)


def test_kron_edge_rows(q):
    """Zero rows (zero scale, zero codes), a single spike (spread evenly over
    all 11008 outputs), constant rows and negative-zero inputs."""
    x = np.zeros((6, K), np.float16)
    x[1, 123] = 1000.0
    x[2, :] = 1.0
    x[3, :] = np.float16(-0.0)
    x[4, ::2] = -3.0
    x[5] = synth.random_f16((1, K), 9)[0]
    s = synth.signs(K, 5)
    for group in (0, 128):
        qa, sc = _run(q, x, s, group)
        check_codes(qa, sc, oracle.rotate_kron(x, s), group)
        np.testing.assert_array_equal(qa[0], 0)
        np.testing.assert_array_equal(qa[3], 0)


def test_kron_empty_is_a_no_op(q):
    x = torch.empty((0, K), dtype=torch.float16, device="cuda")
    s = torch.ones(K, dtype=torch.int8, device="cuda")
    qa, sc = q.quarot_rotate_quant_kron(x, s, 0)
    torch.cuda.synchronize()
    assert qa.shape == (0, K // 2)


def test_kron_linear_end_to_end(q):
    """Computational invariance through the full rotation: x and W rotated by
    the same R (W's rows through the same kernel, one fp32 scale per output
    channel), the INT4 GEMM, and the result against x W^T in fp64 within the
    bound that the two quantization errors give."""
    M, N = 64, 256
    x = synth.random_f16((M, K), 61, dist="laplace")
    W = (np.random.default_rng(62).standard_normal((N, K)) * 0.02).astype(np.float16)
    s = synth.signs(K, 63)
    qa, sa = q.quarot_rotate_quant_kron(_dev(x), _dev(s), 0)
    qw, sw = q.quarot_rotate_quant_kron(_dev(W), _dev(s), 0)
    y = q.quarot_int4_linear(qa, sa, qw, sw, 0)
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    y = y.cpu().numpy().astype(np.float64)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    xr = oracle.rotate_kron(x, s)
    wr = oracle.rotate_kron(W, s)
    sa_ = sa.cpu().numpy().astype(np.float64)
    sw_ = sw.cpu().numpy().astype(np.float64)
    # x'.w' - xh.wh = (x' - xh).w' + xh.(w' - wh), |x' - xh| <= sa/2 (a near-tie
    # flip adds at most 1e-3 sa), |xh| <= |x'| + sa/2; plus the fp16 rounding of y
    bound = 1.01 * ((sa_[:, None] / 2) * np.abs(wr).sum(1)[None, :] +
                    (sw_[None, :] / 2) * (np.abs(xr).sum(1)[:, None] + K * sa_[:, None] / 2))
    bound = bound + 1e-3 * np.abs(ref) + 1e-3
    assert np.all(np.abs(y - ref) <= bound)

"""Parity of quarot_rotate_quant (rotation + INT4 RTN + packing) with the oracle."""
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


def _run(q, x, s, hb, group):
    xt = torch.from_numpy(x).cuda()
    st = torch.from_numpy(s).cuda()
    qp, sc = q.quarot_rotate_quant(xt, st, hb, group)
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    scn = sc.cpu().numpy()
    return qp.cpu().numpy(), (scn.view(np.uint16) if group else scn.astype(np.float64))


CASES = [
    # (K, had_block, group, M)
    (128, 0, 0, 1), (128, 0, 128, 130), (256, 0, 0, 37), (256, 0, 128, 64),
    (512, 0, 0, 33), (1024, 0, 0, 17), (2048, 0, 128, 9), (4096, 0, 0, 70),
    (4096, 0, 128, 5), (8192, 0, 0, 45), (8192, 0, 128, 3),
    (128, 128, 0, 257), (1024, 128, 128, 50), (1024, 128, 0, 19), (11008, 128, 128, 40),
    (11008, 128, 0, 11), (28672, 128, 128, 6), (28672, 128, 0, 5), (384, 128, 0, 130),
]


@pytest.mark.parametrize("K,hb,group,M", CASES)
def test_rotate_quant_matches_oracle(q, K, hb, group, M):
    x = synth.random_f16((M, K), 100 + K + M, dist="student_t3", scale=2.0)
    s = synth.signs(K, K + hb)
    qp, sc = _run(q, x, s, hb, group)
    xr = oracle.rotate(x, s, hb)
    check_codes(qp, sc, xr, group)


@pytest.mark.parametrize("K,hb,group", [(8192, 0, 0), (256, 0, 128), (11008, 128, 128), (11008, 128, 0)])
def test_zero_and_spike_rows(q, K, hb, group):
    M = 6
    x = synth.random_f16((M, K), 7, dist="laplace")
    x[1] = 0                               # all-zero row: scales 0, codes 0
    x[2] = 0
    x[2, 77] = 3.0                         # single spike: every |x'| equal within its block
    x[3] = 0
    x[3, :] = np.float16(-0.5)             # constant row
    x[4, ::2] = np.float16(60000.0)        # near the fp16 limit
    s = synth.signs(K, 5)
    qp, sc = _run(q, x, s, hb, group)
    xr = oracle.rotate(x, s, hb)
    check_codes(qp, sc, xr, group)
    assert np.all(qp[1] == 0)
    if group == 0:
        assert sc[1] == 0.0


@pytest.mark.parametrize("wid", [1, 2, 3, 4])
def test_workload_shapes_leading_rows(q, wid):
    w = synth.LINEARS[wid]
    rows = min(w.M, 96)
    x = synth.activations(w, rows=rows)
    s = synth.signs(w.K, w.seed)
    qp, sc = _run(q, x, s, w.had_block, w.group)
    check_codes(qp, sc, oracle.rotate(x, s, w.had_block), w.group)


def test_llama2_70b_full_size_sampled_rows(q):
    # the full 32768 x 8192 activation, as the benchmark runs it; oracle on sampled rows
    w = synth.LLAMA2_70B
    x = synth.activations(w)
    s = synth.signs(w.K, w.seed)
    qp, sc = _run(q, x, s, w.had_block, w.group)
    rows = synth.sample_rows(w.M, 48, w.seed)
    xr = oracle.rotate(x[rows], s, 0)
    check_codes(qp[rows], sc[rows], xr, 0)


def test_packed_layout_matches_oracle_pack(q):
    # bytes are the oracle's own packing of the checked codes (nibble order)
    x = synth.random_f16((8, 256), 3)
    s = synth.signs(256, 3)
    qp, sc = _run(q, x, s, 0, 0)
    xr = oracle.rotate(x, s, 0)
    codes = oracle.quantize_with_scales(xr, sc, 0)
    np.testing.assert_array_equal(qp, oracle.pack(codes))

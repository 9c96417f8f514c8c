"""The fused entry point quarot_rotate_quant_linear: the same bytes as the two
separate calls; the activation and weight codes the device produced obey the
code rule; and every output element matches the oracle's fp64 product of the
device's own codes and scales under the fp16 output rule (the quantizer is
checked by the code rule, the product element by element)."""
import numpy as np
import pytest
import torch

import oracle
from parity import check_codes, check_f16_output
from rotation_bit_quantization_randomized_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import __graft_entry__
    __graft_entry__.build()
    from rotation_bit_quantization_randomized_b200 import binding
    return binding


def _scales_np(t, group):
    """Device scales as the oracle takes them: fp64 per row, or fp16 bit patterns per group."""
    a = t.cpu().numpy()
    return a.view(np.uint16) if group else a.astype(np.float64)


def _oracle_product(qa, sa, qw, sw, group):
    """The oracle's dequantized product of packed codes and their scales."""
    acc = oracle.int_gemm(oracle.unpack(qa), oracle.unpack(qw), group)
    y, _ = oracle.dequant_linear(acc, sa, sw, group)
    return y


@pytest.mark.parametrize("wid", [1, 2, 3])
def test_fused_equals_separate_and_oracle(q, wid):
    w = synth.LINEARS[wid]
    rows = min(w.M, 160)
    N = w.Ns[0]
    x = synth.activations(w, rows=rows)
    W = synth.weights(w, N)
    s = synth.signs(w.K, w.seed)
    xt, Wt, st = (torch.from_numpy(a).cuda() for a in (x, W, s))
    qw, sw = q.quarot_rotate_quant(Wt, st, w.had_block, w.group)
    y = q.quarot_rotate_quant_linear(xt, st, qw, sw, w.had_block, w.group)
    qa, sa = q.quarot_rotate_quant(xt, st, w.had_block, w.group)
    y2 = q.quarot_int4_linear(qa, sa, qw, sw, w.group)
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    assert torch.equal(y, y2)

    qa_n, qw_n = qa.cpu().numpy(), qw.cpu().numpy()
    sa_n, sw_n = _scales_np(sa, w.group), _scales_np(sw, w.group)
    check_codes(qa_n, sa_n, oracle.rotate(x, s, w.had_block), w.group)
    check_codes(qw_n, sw_n, oracle.rotate(W, s, w.had_block), w.group)
    check_f16_output(y.cpu().numpy(), _oracle_product(qa_n, sa_n, qw_n, sw_n, w.group))


def test_fused_llama2_70b_full_size_sampled_rows(q):
    # the full 32768 x 8192 -> 28672 launch of the fused entry; the oracle
    # checks sampled token rows against every output channel, and sampled
    # weight rows against the code rule
    w = synth.LLAMA2_70B
    N = w.Ns[0]
    x = synth.activations(w)
    s = synth.signs(w.K, w.seed)
    W = synth.weights(w, N)
    st = torch.from_numpy(s).cuda()
    Wt = torch.from_numpy(W).cuda()
    qw, sw = q.quarot_rotate_quant(Wt, st, 0, 0)
    del Wt
    xt = torch.from_numpy(x).cuda()
    y = q.quarot_rotate_quant_linear(xt, st, qw, sw, 0, 0)
    qa, sa = q.quarot_rotate_quant(xt, st, 0, 0)
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    del xt

    rows = synth.sample_rows(w.M, 8, w.seed)
    wrows = synth.sample_rows(N, 64, w.seed + 5)
    qa_n = qa.cpu().numpy()[rows]
    sa_n = sa.cpu().numpy()[rows].astype(np.float64)
    qw_n = qw.cpu().numpy()
    sw_n = sw.cpu().numpy().astype(np.float64)
    check_codes(qa_n, sa_n, oracle.rotate(x[rows], s, 0), 0)
    check_codes(qw_n[wrows], sw_n[wrows], oracle.rotate(W[wrows], s, 0), 0)
    check_f16_output(y.cpu().numpy()[rows], _oracle_product(qa_n, sa_n, qw_n, sw_n, 0))


def test_fused_empty_and_workspace_size(q):
    M, K, N = 0, 256, 256
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    s = torch.ones(K, dtype=torch.int8, device="cuda")
    qw = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y = q.quarot_rotate_quant_linear(x, s, qw, sw)
    assert y.shape == (0, N)
    assert q.quarot_rotate_quant_linear_workspace(2048, 4096, 0) == 2048 * 2048 + 2048 * 4

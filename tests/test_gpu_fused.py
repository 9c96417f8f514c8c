"""The fused entry point quarot_rotate_quant_linear: same bytes as the two
separate calls, and the oracle's linear output wherever the device's codes
equal the oracle's."""
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

    # the weight and activation codes the device produced obey the code rule ...
    sa_n = sa.cpu().numpy()
    sw_n = sw.cpu().numpy()
    sa_n = sa_n.view(np.uint16) if w.group else sa_n.astype(np.float64)
    sw_n = sw_n.view(np.uint16) if w.group else sw_n.astype(np.float64)
    check_codes(qa.cpu().numpy(), sa_n, oracle.rotate(x, s, w.had_block), w.group)
    check_codes(qw.cpu().numpy(), sw_n, oracle.rotate(W, s, w.had_block), w.group)
    # ... and rows whose codes match the oracle's exactly give the oracle's output
    ref = oracle.linear(x, W, s, w.had_block, w.group)
    same_w = np.array_equal(qw.cpu().numpy(), ref["qw"])
    same_rows = np.all(qa.cpu().numpy() == ref["qa"], axis=1)
    assert same_rows.mean() > 0.9
    yg = y.cpu().numpy().astype(np.float64)[same_rows]
    yr = ref["y"][same_rows]
    if same_w:
        check_f16_output(yg, yr)
    else:
        # a few weight codes flipped at near-ties: assess the rows as a whole
        rel = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
        assert rel <= 2e-3, f"relative Frobenius error {rel:.3e}"


def test_fused_empty_and_workspace_size(q):
    M, K, N = 0, 256, 256
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    s = torch.ones(K, dtype=torch.int8, device="cuda")
    qw = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y = q.quarot_rotate_quant_linear(x, s, qw, sw)
    assert y.shape == (0, N)
    assert q.quarot_rotate_quant_linear_workspace(2048, 4096, 0) == 2048 * 2048 + 2048 * 4

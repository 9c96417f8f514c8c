"""The bounded-wait path of the kernels, exercised without faulting anything.

quarot_test_wait_timeout runs the KV value-row quantizer with the copy of one
tile never issued and a 1 ms limit on every wait: the CTA that owns that tile
must give up, record QUAROT_ERR_DEVICE_TIMEOUT, wait for the copies it did
issue and exit.  The test checks that the status is reported once (and then
cleared), that the other CTAs' rows are still quantized correctly, that the
withheld tile's rows were never written, and that the context stays usable:
a normal KV write afterwards is parity-green with a clean status.
"""
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


def test_withheld_copy_times_out_and_context_stays_usable(q):
    rows, withheld = 128 * 600, 5
    v = synth.random_f16((rows, 128), 91)
    vt = torch.from_numpy(v).cuda()
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    qc, sc = q.quarot_test_wait_timeout(vt, withheld, 1_000_000)
    assert q.quarot_get_device_status() == 5          # QUAROT_ERR_DEVICE_TIMEOUT ...
    assert q.quarot_get_device_status() == 0          # ... reported once, then cleared

    qn, scn = qc.cpu().numpy(), sc.cpu().numpy()
    # the aborted CTA wrote nothing of the withheld tile (outputs were zeroed)
    blk = slice(128 * withheld, 128 * (withheld + 1))
    assert np.all(scn[blk] == 0) and np.all(qn[blk] == 0)
    # tiles 0..4 belong to other CTAs (the grid has at least one CTA per SM)
    # and follow the code rule: value rows are their own 128-element groups
    ok = slice(0, 128 * withheld)
    check_codes(qn[ok], scn[ok].view(np.uint16), oracle.f16_to_f64(v[ok]), 128)

    # the context is usable: a normal KV write is parity-green, status clean
    B, T, H, D = 2, 300, 8, 128
    k = synth.random_f16((B, T, H, D), 92)
    vv = synth.random_f16((B, T, H, D), 93)
    s = np.stack([synth.signs(D, 94 + h) for h in range(H)])
    kq, ks, vq, vs = q.quarot_kv_quant(torch.from_numpy(k).cuda(), torch.from_numpy(vv).cuda(),
                                       torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    kq = kq.cpu().numpy().reshape(B * T, H * D // 2)
    vq = vq.cpu().numpy().reshape(B * T, H * D // 2)
    ks = ks.cpu().numpy().view(np.uint16).reshape(B * T, H)
    vs = vs.cpu().numpy().view(np.uint16).reshape(B * T, H)
    # keys: the per-head rotation is the block rotation of the [H*D] row with
    # the concatenated signs; values are not rotated
    check_codes(kq, ks, oracle.rotate(k.reshape(B * T, H * D), s.reshape(-1), D), D)
    check_codes(vq, vs, oracle.f16_to_f64(vv.reshape(B * T, H * D)), D)

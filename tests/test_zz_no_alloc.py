"""quarot_rotate_quant_linear_noalloc against the allocating fused entry point.

The allocation-free entry point is for callers that cannot give the library
device memory (no allocator of their own on this path, or a request loop that
must not call cudaMalloc / cudaFree).  It must give the same output as
quarot_rotate_quant_linear, call after call, while reusing its built-in
scratch.  This file sorts last so that a run stopping at its first failure has
run every other test already.
"""
import ctypes

import pytest
import torch

from rotation_bit_quantization_randomized_b200 import synth


@pytest.fixture(scope="module")
def q():
    import __graft_entry__
    __graft_entry__.build()
    from rotation_bit_quantization_randomized_b200 import binding
    return binding


def _noalloc(q, x, s, qw, sw, hb, group, out, stream):
    P = ctypes.c_void_p
    return q.lib.quarot_rotate_quant_linear_noalloc(
        P(x.data_ptr()), x.shape[0], x.shape[1], P(s.data_ptr()), hb, group, P(qw.data_ptr()),
        P(sw.data_ptr()), qw.shape[0], P(out.data_ptr()), P(stream))


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_on_two_calls(q):
    # first call: per-token H_4096 (7B shape); second: block I x H_128 with groups (down-proj)
    stream = torch.cuda.current_stream().cuda_stream
    for w, rows in ((synth.LLAMA2_7B, 512), (synth.DOWN_PROJ, 256)):
        x = torch.from_numpy(synth.activations(w, rows=rows)).cuda()
        W = torch.from_numpy(synth.weights(w, w.Ns[0])).cuda()
        s = torch.from_numpy(synth.signs(w.K, w.seed)).cuda()
        qw, sw = q.quarot_rotate_quant(W, s, w.had_block, w.group)
        ref = q.quarot_rotate_quant_linear(x, s, qw, sw, w.had_block, w.group)
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(q, x, s, qw, sw, w.had_block, w.group, out, stream) == 0
        torch.cuda.synchronize()
        assert q.quarot_get_device_status() == 0
        # the same kernels on the same inputs: the same bytes
        assert torch.equal(out, ref)


@pytest.mark.gpu
def test_noalloc_at_the_scratch_limit(q):
    # 4092 tokens x K 8192 with per-token scales need exactly 16 MiB: accepted
    stream = torch.cuda.current_stream().cuda_stream
    w = synth.LLAMA2_70B
    M, N = 4092, 256
    assert q.quarot_rotate_quant_linear_workspace(M, w.K, 0) == 16 * 1024 * 1024
    x = torch.from_numpy(synth.activations(w, rows=M)).cuda()
    W = torch.from_numpy(synth.weights(w, N)).cuda()
    s = torch.from_numpy(synth.signs(w.K, w.seed)).cuda()
    qw, sw = q.quarot_rotate_quant(W, s, 0, 0)
    ref = q.quarot_rotate_quant_linear(x, s, qw, sw, 0, 0)
    out = torch.full_like(ref, float("nan"))
    assert _noalloc(q, x, s, qw, sw, 0, 0, out, stream) == 0
    torch.cuda.synchronize()
    assert q.quarot_get_device_status() == 0
    assert torch.equal(out, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch(q):
    A = ctypes.c_void_p(0x10000)
    # 8192 tokens x K 8192 need 32 MiB + scales > 16 MiB: rejected before any device work
    assert q.lib.quarot_rotate_quant_linear_noalloc(A, 8192, 8192, A, 0, 0, A, A, 256, A, None) == 2
    assert "16777216" in q.lib.quarot_last_error().decode()
    # one token past the limit (4093 x K 8192: 16 MiB + 4 KiB) is rejected too
    assert q.lib.quarot_rotate_quant_linear_noalloc(A, 4093, 8192, A, 0, 0, A, A, 256, A, None) == 2
    assert q.lib.quarot_rotate_quant_linear_noalloc(A, 0, 8192, A, 0, 0, A, A, 256, A, None) == 0

"""Guard bands around every output: each entry point writes into buffers cut
from the middle of a larger allocation whose 4 KiB before and after are
filled with a canary pattern, on ragged sizes (token counts that end inside a
tile, odd head counts, odd T); after the call the canaries must be intact,
the device status clean, and every floating-point output free of the NaN
poison the buffer was filled with (so the kernel wrote all of it).  With
compute-sanitizer unavailable, this is the check that no kernel stores past
the ends of its outputs."""
import numpy as np
import pytest
import torch

from rotation_bit_quantization_randomized_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5


@pytest.fixture(scope="module")
def q():
    import __graft_entry__
    __graft_entry__.build()
    from rotation_bit_quantization_randomized_b200 import binding
    # the library the binding loaded is the one it names (normal or bounds-checking)
    assert binding.lib.quarot_debug_bounds() == (1 if binding.DEBUG_BOUNDS else 0)
    return binding


class Guarded:
    """Typed buffers carved out of one allocation, each between two canary bands."""

    def __init__(self):
        self.parts = []

    def __call__(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.empty(GUARD + nbytes + GUARD, dtype=torch.uint8, device="cuda")
        raw[:GUARD] = CANARY
        raw[GUARD + nbytes:] = CANARY
        raw[GUARD:GUARD + nbytes] = 0xFF          # NaN in fp16 / fp32
        view = raw[GUARD:GUARD + nbytes].view(dtype).view(shape)
        self.parts.append((raw, nbytes, view))
        return view

    def check(self, q):
        torch.cuda.synchronize()
        assert q.quarot_get_device_status() == 0
        for raw, nbytes, view in self.parts:
            assert bool(torch.all(raw[:GUARD] == CANARY)), "store before the start of an output"
            assert bool(torch.all(raw[GUARD + nbytes:] == CANARY)), "store past the end of an output"
            if view.dtype in (torch.float16, torch.float32) and view.numel():
                assert not bool(torch.isnan(view).any()), "output not fully written"


def _x(M, K, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((M, K)).astype(np.float16)).cuda()


def _s(K, seed):
    return torch.from_numpy(synth.signs(K, seed)).cuda()


@pytest.mark.parametrize("M,K,hb,group", [(17, 256, 0, 0), (129, 4096, 0, 0), (17, 256, 0, 128),
                                          (3, 384, 128, 0), (130, 384, 128, 128), (1, 8192, 0, 0)])
def test_rotate_quant_guards(q, M, K, hb, group):
    g = Guarded()
    x, s = _x(M, K, M + K), _s(K, 3)
    qp = g((M, K // 2), torch.uint8)
    sc = g((M,), torch.float32) if group == 0 else g((M, K // 128), torch.float16)
    q.quarot_rotate_quant(x, s, hb, group, qp, sc)
    if group == 0:
        q.quarot_rotate_quant_i8(x, s, hb, g((M, K), torch.int8), g((M,), torch.float32))
        q.quarot_rotate_quant_i6(x, s, hb, g((M, K), torch.int8), g((M,), torch.float32))
        if hb == 0:
            q.quarot_rotate_quant_asym(x, s, 0.9, 0, g((M, K // 2), torch.uint8), g((M,), torch.float32),
                                       g((M,), torch.int32), g((M,), torch.int32))
    g.check(q)


@pytest.mark.parametrize("M,group", [(17, 0), (5, 128)])
def test_kron_guards(q, M, group):
    K = 11008
    g = Guarded()
    x, s = _x(M, K, 7), _s(K, 8)
    sc = g((M,), torch.float32) if group == 0 else g((M, K // 128), torch.float16)
    q.quarot_rotate_quant_kron(x, s, group, g((M, K // 2), torch.uint8), sc)
    g.check(q)


@pytest.mark.parametrize("M,N,K,group", [(17, 264, 256, 0), (300, 520, 1024, 0), (33, 136, 512, 128)])
def test_linear_guards(q, M, N, K, group):
    g = Guarded()
    s = _s(K, 11)
    x, W = _x(M, K, 12), (_x(N, K, 13) * 0.05).half()
    qw, sw = q.quarot_rotate_quant(W, s, 0, group)
    qa, sa = q.quarot_rotate_quant(x, s, 0, group)
    q.quarot_int4_linear(qa, sa, qw, sw, group, g((M, N), torch.float16))
    if group == 0:
        q.quarot_int4_gemm_s32(qa, qw, g((M, N), torch.int32))
        ws = g((q.quarot_rotate_quant_linear_workspace(M, K, 0),), torch.uint8)
        q.quarot_rotate_quant_linear(x, s, qw, sw, 0, 0, ws, g((M, N), torch.float16))
        q.quarot_rotate_quant_linear_noalloc(x, s, qw, sw, g((M, N), torch.float16))
        qw8, sw8 = q.quarot_rotate_quant_i8(W, s)
        qa8, sa8 = q.quarot_rotate_quant_i8(x, s)
        q.quarot_int8_linear(qa8, sa8, qw8, sw8, g((M, N), torch.float16))
        q.quarot_int8_gemm_s32(qa8, qw8, g((M, N), torch.int32))
        ws8 = g((q.quarot_rotate_quant_linear_i8_workspace(M, K),), torch.uint8)
        q.quarot_rotate_quant_linear_i8(x, s, qw8, sw8, 0, ws8, g((M, N), torch.float16))
        qw6, sw6 = q.quarot_rotate_quant_i6(W, s)
        ws6 = g((q.quarot_rotate_quant_linear_i8_workspace(M, K),), torch.uint8)
        q.quarot_rotate_quant_linear_i6(x, s, qw6, sw6, 0, ws6, g((M, N), torch.float16))
        ua = q.quarot_rotate_quant_asym(x, s, 0.9)
        uw = q.quarot_rotate_quant_asym(W, s, 1.0)
        q.quarot_uint4_gemm_s32(ua[0], uw[0], g((M, N), torch.int32))
        q.quarot_int4_linear_asym(*ua, *uw, g((M, N), torch.float16))
    else:
        ws = g((q.quarot_rotate_quant_linear_workspace(M, K, group),), torch.uint8)
        q.quarot_rotate_quant_linear(x, s, qw, sw, 0, group, ws, g((M, N), torch.float16))
    g.check(q)


@pytest.mark.parametrize("B,T,H,G", [(2, 65, 3, 8), (1, 129, 2, 4), (3, 300, 1, 16), (1, 1, 8, 1)])
def test_kv_guards(q, B, T, H, G):
    g = Guarded()
    rng = np.random.default_rng(T + H)
    k = torch.from_numpy(rng.standard_normal((B, T, H, 128)).astype(np.float16)).cuda()
    v = torch.from_numpy(rng.standard_normal((B, T, H, 128)).astype(np.float16)).cuda()
    qh = torch.from_numpy(rng.standard_normal((B, H * G, 128)).astype(np.float16)).cuda()
    s = torch.from_numpy(np.stack([synth.signs(128, 40 + i) for i in range(H)])).cuda()
    kq, ks = g((B, T, H, 64), torch.uint8), g((B, T, H), torch.float16)
    vq, vs = g((B, T, H, 64), torch.uint8), g((B, T, H), torch.float16)
    q.quarot_kv_quant(k, v, s, kq, ks, vq, vs)
    scores = q.quarot_kv_decode_scores(qh, s, kq, ks, g((B, H * G, T), torch.float32))
    q.quarot_kv_decode_attend(scores, vq, vs, g((B, H * G, 128), torch.float32))
    q.quarot_kv_decode_attention(qh, s, kq, ks, vq, vs, g((B, H * G, 128), torch.float32))
    g.check(q)

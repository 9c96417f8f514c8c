"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/quarot.h declares, and rejects bad arguments before
touching the device."""
import ctypes

import pytest

import __graft_entry__


@pytest.fixture(scope="module")
def q():
    __graft_entry__.build()
    from rotation_bit_quantization_randomized_b200 import binding
    return binding


def test_library_exports_every_header_function(q):
    names = q.header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(q.lib, n), f"libquarot.so does not export {n}"


def test_status_strings(q):
    for code, name in q.STATUS.items():
        assert q.status_string(code) == name
    assert q.status_string(99) == "QUAROT_ERR_UNKNOWN"


P = ctypes.c_void_p
A16 = P(0x10000)           # aligned fake pointer, never dereferenced: validation fails first
MIS = P(0x10008)


def _rq(q, x=A16, M=4, K=256, signs=A16, hb=0, group=0, out=A16, sc=A16):
    return q.lib.quarot_rotate_quant(x, M, K, signs, hb, group, out, sc, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=-1), 1), (dict(hb=64), 1), (dict(group=64), 1),
    (dict(K=384), 2), (dict(K=16384), 2), (dict(K=64), 2), (dict(hb=128, K=200), 2),
    (dict(hb=128, K=65536 + 128), 2),
    (dict(x=None), 1), (dict(sc=None), 1), (dict(x=MIS), 3), (dict(out=MIS), 3),
])
def test_rotate_quant_rejects(q, kw, status):
    assert _rq(q, **kw) == status


def test_rotate_quant_empty_is_ok_without_launch(q):
    assert _rq(q, M=0, x=None, out=None, sc=None, signs=None) == 0


def _lin(q, qa=A16, sa=A16, M=4, qw=A16, sw=A16, N=256, K=256, group=0, out=A16):
    return q.lib.quarot_int4_linear(qa, sa, M, qw, sw, N, K, group, out, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=-2), 1), (dict(N=0), 1), (dict(group=7), 1), (dict(N=100), 2), (dict(K=200), 2),
    (dict(K=65536 + 128), 2), (dict(qa=None), 1), (dict(sw=None), 1), (dict(out=MIS), 3),
    (dict(sa=MIS), 3),
])
def test_int4_linear_rejects(q, kw, status):
    assert _lin(q, **kw) == status


def test_int4_linear_empty_is_ok(q):
    assert _lin(q, M=0, qa=None, sa=None, out=None) == 0


def test_gemm_s32_rejects(q):
    assert q.lib.quarot_int4_gemm_s32(A16, 4, A16, 12, 256, A16, None) == 2
    assert q.lib.quarot_int4_gemm_s32(None, 4, A16, 16, 256, A16, None) == 1
    assert q.lib.quarot_int4_gemm_s32(A16, 0, A16, 16, 256, A16, None) == 0


def test_workspace_size(q):
    f = q.lib.quarot_rotate_quant_linear_workspace
    assert f(0, 256, 0) == 0
    assert f(16, 256, 0) == 2048 + 256          # codes, then 16 fp32 scales rounded to 256
    assert f(16, 256, 128) == 2048 + 256        # 16 x 2 fp16 scales
    assert f(1000, 4096, 0) == 2048000 + 4096
    assert f(2048, 11008, 128) % 256 == 0


def test_fused_rejects_small_or_misaligned_workspace(q):
    f = q.lib.quarot_rotate_quant_linear
    need = q.lib.quarot_rotate_quant_linear_workspace(16, 256, 0)
    assert f(A16, 16, 256, A16, 0, 0, A16, A16, 256, A16, need - 1, A16, None) == 1
    assert f(A16, 16, 256, A16, 0, 0, A16, A16, 256, P(0x10010), need, A16, None) == 3


def test_kv_rejects(q):
    kv = q.lib.quarot_kv_quant
    assert kv(A16, A16, 1, 4, 8, 64, A16, A16, A16, A16, A16, None) == 2
    assert kv(A16, A16, 1, 4, 0, 128, A16, A16, A16, A16, A16, None) == 1
    assert kv(A16, A16, 0, 4, 8, 128, None, None, None, None, None, None) == 0
    sc = q.lib.quarot_kv_decode_scores
    assert sc(A16, 12, A16, A16, A16, 1, 16, 8, 128, A16, None) == 2     # Hq % Hkv != 0
    assert sc(A16, 64 * 8, A16, A16, A16, 1, 16, 8, 128, A16, None) == 2  # group of 64
    assert sc(A16, 64, A16, A16, A16, 1, 16, 8, 64, A16, None) == 2      # D != 128
    assert sc(A16, 64, A16, A16, A16, 1, 0, 8, 128, None, None) == 0     # no tokens: no launch
    at = q.lib.quarot_kv_decode_attend
    assert at(A16, 1, 64, A16, A16, 16, 8, 64, A16, None) == 2       # D != 128
    assert at(A16, 1, 12, A16, A16, 16, 8, 128, A16, None) == 2      # Hq % Hkv != 0
    assert at(A16, 1, 24, A16, A16, 16, 8, 128, A16, None) == 2      # group of 3
    assert at(A16, 1, 64, A16, A16, 0, 8, 128, A16, None) == 1       # no tokens
    assert at(A16, 1, 64, A16, None, 16, 8, 128, A16, None) == 1
    assert at(A16, 1, 64, MIS, A16, 16, 8, 128, A16, None) == 3
    assert at(None, 0, 64, None, None, 16, 8, 128, None, None) == 0  # empty batch: no launch


def test_kron_entry_point_rejects_and_factor_matches_oracle(q):
    import numpy as np
    import oracle
    kr = q.lib.quarot_rotate_quant_kron
    assert kr(A16, 4, 11008 - 128, A16, 0, A16, A16, None) == 2     # only K = 11008
    assert kr(A16, 4, 11008, A16, 64, A16, A16, None) == 1          # group 0 or 128
    assert kr(A16, -1, 11008, A16, 0, A16, A16, None) == 1
    assert kr(A16, 4, 11008, None, 0, A16, A16, None) == 1
    assert kr(MIS, 4, 11008, A16, 0, A16, A16, None) == 3
    assert kr(None, 0, 11008, None, 0, None, None, None) == 0       # empty: no launch
    assert q.lib.quarot_kron_factor(172, A16) == 2
    # the library's factor (squares enumerated) equals the oracle's (Euler's
    # criterion): two independent routes to the same Paley matrix
    h = q.quarot_kron_factor(344).numpy()
    np.testing.assert_array_equal(h, oracle.paley(7, 3))


def test_binding_raises_on_error(q):
    import torch
    x = torch.zeros((4, 384), dtype=torch.float16)
    s = torch.ones(384, dtype=torch.int8)
    with pytest.raises(q.QuarotError, match="UNSUPPORTED_SHAPE"):
        q.quarot_rotate_quant(x, s)


def test_int8_entry_points_reject(q):
    rq8 = q.lib.quarot_rotate_quant_i8
    assert rq8(A16, 4, 384, A16, 0, A16, A16, None) == 2          # not a power of two
    assert rq8(A16, 4, 256, A16, 64, A16, A16, None) == 1         # had_block
    assert rq8(A16, 4, 256, A16, 0, MIS, A16, None) == 3
    assert rq8(None, 0, 256, None, 0, None, None, None) == 0      # empty: no launch
    lin8 = q.lib.quarot_int8_linear
    assert lin8(A16, A16, 4, A16, A16, 100, 256, A16, None) == 2  # N % 8
    assert lin8(A16, A16, 4, A16, A16, 256, 200, A16, None) == 2  # K % 128
    assert lin8(A16, None, 4, A16, A16, 256, 256, A16, None) == 1
    assert lin8(None, None, 0, A16, A16, 256, 256, None, None) == 0
    s32 = q.lib.quarot_int8_gemm_s32
    assert s32(A16, 4, A16, 12, 256, A16, None) == 2
    assert s32(A16, 4, A16, 16, 256, MIS, None) == 3
    ws = q.lib.quarot_rotate_quant_linear_i8_workspace
    assert ws(0, 256) == 0
    assert ws(16, 256) == 4096 + 256                               # int8 codes, then fp32 scales
    f = q.lib.quarot_rotate_quant_linear_i8
    need = ws(16, 256)
    assert f(A16, 16, 256, A16, 0, A16, A16, 256, A16, need - 1, A16, None) == 1
    assert f(A16, 16, 256, A16, 0, A16, A16, 256, P(0x10010), need, A16, None) == 3


def test_timeout_entry_rejects(q):
    A = ctypes.c_void_p(0x10000)
    f = q.lib.quarot_test_wait_timeout
    assert f(A, 0, A, A, 0, 1_000_000, None) == 1             # no rows
    assert f(A, 256, A, A, 2, 1_000_000, None) == 1           # tile 2 of 2
    assert f(A, 256, A, A, -1, 1_000_000, None) == 1
    assert f(A, 256, A, A, 0, 10, None) == 1                  # limit too short
    assert f(A, 256, A, A, 0, 3_000_000_000, None) == 1       # limit too long
    assert f(ctypes.c_void_p(0x10008), 256, A, A, 0, 1_000_000, None) == 3


def test_mma_probe_rejects(q):
    n = ctypes.c_int64(0)
    assert q.lib.quarot_probe_mma_i8(0, 0, ctypes.byref(n), None) == 1
    assert q.lib.quarot_probe_mma_i8((1 << 22) + 1, 1, ctypes.byref(n), None) == 1
    assert q.lib.quarot_probe_mma_i8(10, 0, None, None) == 1
    assert q.lib.quarot_probe_mma_i8(10, 3, ctypes.byref(n), None) == 1
    assert q.lib.quarot_probe_mma_i8(10, -1, ctypes.byref(n), None) == 1
    assert "operands" in q.lib.quarot_last_error().decode()


def test_fused_decode_rejects(q):
    f = q.lib.quarot_kv_decode_attention
    assert f(A16, 64, A16, A16, A16, A16, A16, 1, 16, 8, 64, A16, None) == 2      # D != 128
    assert f(A16, 12, A16, A16, A16, A16, A16, 1, 16, 8, 128, A16, None) == 2     # Hq % Hkv != 0
    assert f(A16, 24, A16, A16, A16, A16, A16, 1, 16, 8, 128, A16, None) == 2     # group of 3
    assert f(A16, 64, A16, A16, A16, A16, A16, 1, 0, 8, 128, A16, None) == 1      # no tokens
    assert f(A16, 64, A16, A16, None, A16, A16, 1, 16, 8, 128, A16, None) == 1
    assert f(A16, 64, A16, A16, A16, MIS, A16, 1, 16, 8, 128, A16, None) == 3
    assert f(None, 64, None, None, None, None, None, 0, 16, 8, 128, None, None) == 0   # empty batch


def test_bounds_checking_build(q):
    # the twin library compiled with QUAROT_DEBUG_BOUNDS says so; the normal one does not
    from rotation_bit_quantization_randomized_b200 import build_lib
    dbg = ctypes.CDLL(build_lib.LIB_DEBUG)
    dbg.quarot_debug_bounds.restype = ctypes.c_int
    assert dbg.quarot_debug_bounds() == 1
    assert q.lib.quarot_debug_bounds() == (1 if q.DEBUG_BOUNDS else 0)
    assert q.status_string(7) == "QUAROT_ERR_DEVICE_BOUNDS"

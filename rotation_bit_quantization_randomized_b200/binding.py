"""ctypes binding of libquarot (include/quarot.h), same entry-point names.

Argument marshalling only: tensors become device pointers and sizes, the
current torch stream becomes the cudaStream_t, and a non-zero status raises
QuarotError.  Every step of the computation runs in the library's kernels;
there is no fallback of any kind, and importing this module raises if the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QUAROT_DEBUG_BOUNDS=1 in the environment selects the bounds-checking build
# (libquarot_dbg.so: every kernel checks its output stores; see
# quarot_debug_bounds in include/quarot.h)
DEBUG_BOUNDS = os.environ.get("QUAROT_DEBUG_BOUNDS", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libquarot_dbg.so" if DEBUG_BOUNDS else "libquarot.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "quarot.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'`")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_SZ = ctypes.c_size_t
_SIGS = {
    "quarot_rotate_quant": ([_P, _I64, _I64, _P, _INT, _INT, _P, _P, _P], _INT),
    "quarot_int4_linear": ([_P, _P, _I64, _P, _P, _I64, _I64, _INT, _P, _P], _INT),
    "quarot_int4_gemm_s32": ([_P, _I64, _P, _I64, _I64, _P, _P], _INT),
    "quarot_rotate_quant_linear_workspace": ([_I64, _I64, _INT], _SZ),
    "quarot_rotate_quant_linear": ([_P, _I64, _I64, _P, _INT, _INT, _P, _P, _I64, _P, _SZ, _P, _P], _INT),
    "quarot_rotate_quant_linear_noalloc": ([_P, _I64, _I64, _P, _INT, _INT, _P, _P, _I64, _P, _P], _INT),
    "quarot_rotate_quant_i8": ([_P, _I64, _I64, _P, _INT, _P, _P, _P], _INT),
    "quarot_int8_linear": ([_P, _P, _I64, _P, _P, _I64, _I64, _P, _P], _INT),
    "quarot_int8_gemm_s32": ([_P, _I64, _P, _I64, _I64, _P, _P], _INT),
    "quarot_rotate_quant_linear_i8_workspace": ([_I64, _I64], _SZ),
    "quarot_rotate_quant_linear_i8": ([_P, _I64, _I64, _P, _INT, _P, _P, _I64, _P, _SZ, _P, _P], _INT),
    "quarot_rotate_quant_i6": ([_P, _I64, _I64, _P, _INT, _P, _P, _P], _INT),
    "quarot_rotate_quant_linear_i6": ([_P, _I64, _I64, _P, _INT, _P, _P, _I64, _P, _SZ, _P, _P], _INT),
    "quarot_rotate_quant_asym": ([_P, _I64, _I64, _P, _INT, ctypes.c_float, _P, _P, _P, _P, _P], _INT),
    "quarot_uint4_gemm_s32": ([_P, _I64, _P, _I64, _I64, _P, _P], _INT),
    "quarot_int4_linear_asym": ([_P, _P, _P, _P, _I64, _P, _P, _P, _P, _I64, _I64, _P, _P], _INT),
    "quarot_kv_quant": ([_P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P], _INT),
    "quarot_kv_decode_scores": ([_P, _I64, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P], _INT),
    "quarot_rotate_quant_kron": ([_P, _I64, _I64, _P, _I64, _P, _P, _P], _INT),
    "quarot_kron_factor": ([_I64, _P], _INT),
    "quarot_kv_decode_attend": ([_P, _I64, _I64, _P, _P, _I64, _I64, _I64, _P, _P], _INT),
    "quarot_kv_decode_attention": ([_P, _I64, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P], _INT),
    "quarot_probe_mma_i8": ([_I64, _INT, _P, _P], _INT),
    "quarot_test_wait_timeout": ([_P, _I64, _P, _P, _I64, ctypes.c_uint64, _P], _INT),
    "quarot_get_device_status": ([_P], _INT),
    "quarot_status_string": ([_INT], ctypes.c_char_p),
    "quarot_last_error": ([], ctypes.c_char_p),
    "quarot_debug_bounds": ([], _INT),
}
for _name, (_args, _ret) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _ret

STATUS = {0: "QUAROT_OK", 1: "QUAROT_ERR_INVALID_ARG", 2: "QUAROT_ERR_UNSUPPORTED_SHAPE",
          3: "QUAROT_ERR_MISALIGNED", 4: "QUAROT_ERR_CUDA", 5: "QUAROT_ERR_DEVICE_TIMEOUT",
          6: "QUAROT_ERR_NO_DEVICE", 7: "QUAROT_ERR_DEVICE_BOUNDS"}


class QuarotError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib.quarot_last_error().decode(errors="replace")
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}")


def header_functions():
    """Names of the functions include/quarot.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(quarot_\w+)\s*\(", text)))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous (row-major)")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        if not torch.cuda.is_available():
            return ctypes.c_void_p(0)      # argument errors are reported before any launch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, status: int):
    if status != 0:
        raise QuarotError(fn, status)


def status_string(status: int) -> str:
    return lib.quarot_status_string(status).decode()


# --------------------------------------------------------------------------- entry points

def quarot_rotate_quant(x: torch.Tensor, signs: torch.Tensor, had_block: int = 0, group: int = 0,
                        q_packed: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                        stream=None):
    """x fp16 [M, K] -> (q_packed uint8 [M, K/2], scales fp32 [M] or fp16 [M, K/128])."""
    M, K = x.shape
    dev = x.device
    if q_packed is None:
        q_packed = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = (torch.empty((M,), dtype=torch.float32, device=dev) if group == 0
                  else torch.empty((M, K // 128), dtype=torch.float16, device=dev))
    _check("quarot_rotate_quant",
           lib.quarot_rotate_quant(_ptr(x), M, K, _ptr(signs), had_block, group, _ptr(q_packed),
                                   _ptr(scales), _stream(stream)))
    return q_packed, scales


def quarot_int4_linear(qa: torch.Tensor, s_a: torch.Tensor, qw: torch.Tensor, s_w: torch.Tensor,
                       group: int = 0, out: Optional[torch.Tensor] = None, stream=None):
    """Packed INT4 [M, K/2] x packed INT4 [N, K/2]^T with scales -> fp16 [M, N]."""
    M, Kh = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=qa.device)
    _check("quarot_int4_linear",
           lib.quarot_int4_linear(_ptr(qa), _ptr(s_a), M, _ptr(qw), _ptr(s_w), N, 2 * Kh, group,
                                  _ptr(out), _stream(stream)))
    return out


def quarot_int4_gemm_s32(qa: torch.Tensor, qw: torch.Tensor, acc: Optional[torch.Tensor] = None,
                         stream=None):
    """Exact int32 [M, N] = codes(qa) . codes(qw)^T."""
    M, Kh = qa.shape
    N = qw.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=qa.device)
    _check("quarot_int4_gemm_s32",
           lib.quarot_int4_gemm_s32(_ptr(qa), M, _ptr(qw), N, 2 * Kh, _ptr(acc), _stream(stream)))
    return acc


def quarot_rotate_quant_linear_workspace(M: int, K: int, group: int = 0) -> int:
    return int(lib.quarot_rotate_quant_linear_workspace(M, K, group))


def quarot_rotate_quant_linear(x: torch.Tensor, signs: torch.Tensor, qw: torch.Tensor, s_w: torch.Tensor,
                               had_block: int = 0, group: int = 0, workspace: Optional[torch.Tensor] = None,
                               out: Optional[torch.Tensor] = None, stream=None):
    """Fused online path: rotate + quantize x, then the INT4 linear; fp16 [M, N]."""
    M, K = x.shape
    N = qw.shape[0]
    need = quarot_rotate_quant_linear_workspace(M, K, group)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check("quarot_rotate_quant_linear",
           lib.quarot_rotate_quant_linear(_ptr(x), M, K, _ptr(signs), had_block, group, _ptr(qw), _ptr(s_w), N,
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _ptr(out), _stream(stream)))
    return out


def quarot_rotate_quant_linear_noalloc(x: torch.Tensor, signs: torch.Tensor, qw: torch.Tensor,
                                       s_w: torch.Tensor, out: torch.Tensor, had_block: int = 0, group: int = 0,
                                       stream=None):
    """The fused path on the library's built-in scratch; the caller supplies every
    buffer, including `out` (fp16 [M, N]), and nothing is allocated."""
    M, K = x.shape
    N = qw.shape[0]
    _check("quarot_rotate_quant_linear_noalloc",
           lib.quarot_rotate_quant_linear_noalloc(_ptr(x), M, K, _ptr(signs), had_block, group, _ptr(qw),
                                                  _ptr(s_w), N, _ptr(out), _stream(stream)))
    return out


def quarot_rotate_quant_i8(x: torch.Tensor, signs: torch.Tensor, had_block: int = 0,
                           q: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None, stream=None):
    """x fp16 [M, K] -> (q int8 [M, K], scales fp32 [M]): the 8-bit variant."""
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check("quarot_rotate_quant_i8",
           lib.quarot_rotate_quant_i8(_ptr(x), M, K, _ptr(signs), had_block, _ptr(q), _ptr(scales),
                                      _stream(stream)))
    return q, scales


def quarot_int8_linear(qa: torch.Tensor, s_a: torch.Tensor, qw: torch.Tensor, s_w: torch.Tensor,
                       out: Optional[torch.Tensor] = None, stream=None):
    """INT8 [M, K] x INT8 [N, K]^T with fp32 scales -> fp16 [M, N]."""
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=qa.device)
    _check("quarot_int8_linear",
           lib.quarot_int8_linear(_ptr(qa), _ptr(s_a), M, _ptr(qw), _ptr(s_w), N, K, _ptr(out), _stream(stream)))
    return out


def quarot_int8_gemm_s32(qa: torch.Tensor, qw: torch.Tensor, acc: Optional[torch.Tensor] = None, stream=None):
    """Exact int32 [M, N] = qa . qw^T for int8 codes."""
    M, K = qa.shape
    N = qw.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=qa.device)
    _check("quarot_int8_gemm_s32",
           lib.quarot_int8_gemm_s32(_ptr(qa), M, _ptr(qw), N, K, _ptr(acc), _stream(stream)))
    return acc


def quarot_rotate_quant_linear_i8_workspace(M: int, K: int) -> int:
    return int(lib.quarot_rotate_quant_linear_i8_workspace(M, K))


def quarot_rotate_quant_linear_i8(x: torch.Tensor, signs: torch.Tensor, qw: torch.Tensor, s_w: torch.Tensor,
                                  had_block: int = 0, workspace: Optional[torch.Tensor] = None,
                                  out: Optional[torch.Tensor] = None, stream=None):
    """Fused online INT8 path: rotate + 8-bit quantize x, then the INT8 linear; fp16 [M, N]."""
    M, K = x.shape
    N = qw.shape[0]
    need = quarot_rotate_quant_linear_i8_workspace(M, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check("quarot_rotate_quant_linear_i8",
           lib.quarot_rotate_quant_linear_i8(_ptr(x), M, K, _ptr(signs), had_block, _ptr(qw), _ptr(s_w), N,
                                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                                             _ptr(out), _stream(stream)))
    return out


def quarot_rotate_quant_i6(x: torch.Tensor, signs: torch.Tensor, had_block: int = 0,
                           q: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None, stream=None):
    """x fp16 [M, K] -> (q int8 [M, K] in [-31, 31], scales fp32 [M]): the 6-bit variant."""
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check("quarot_rotate_quant_i6",
           lib.quarot_rotate_quant_i6(_ptr(x), M, K, _ptr(signs), had_block, _ptr(q), _ptr(scales),
                                      _stream(stream)))
    return q, scales


def quarot_rotate_quant_linear_i6(x: torch.Tensor, signs: torch.Tensor, qw: torch.Tensor, s_w: torch.Tensor,
                                  had_block: int = 0, workspace: Optional[torch.Tensor] = None,
                                  out: Optional[torch.Tensor] = None, stream=None):
    """Fused online 6-bit path: rotate + 6-bit quantize x, then the INT8 linear; fp16 [M, N]."""
    M, K = x.shape
    N = qw.shape[0]
    need = quarot_rotate_quant_linear_i8_workspace(M, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check("quarot_rotate_quant_linear_i6",
           lib.quarot_rotate_quant_linear_i6(_ptr(x), M, K, _ptr(signs), had_block, _ptr(qw), _ptr(s_w), N,
                                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                                             _ptr(out), _stream(stream)))
    return out


def quarot_rotate_quant_asym(x: torch.Tensor, signs: torch.Tensor, clip: float, had_block: int = 0, q=None, d=None,
                             z=None, r=None, stream=None):
    """x fp16 [M, K] -> (q_packed uint8 [M, K/2] unsigned nibbles, steps fp32 [M],
    zero points int32 [M], code row sums int32 [M]); outputs may be passed in."""
    M, K = x.shape
    dev = x.device
    q = torch.empty((M, K // 2), dtype=torch.uint8, device=dev) if q is None else q
    d = torch.empty((M,), dtype=torch.float32, device=dev) if d is None else d
    z = torch.empty((M,), dtype=torch.int32, device=dev) if z is None else z
    r = torch.empty((M,), dtype=torch.int32, device=dev) if r is None else r
    _check("quarot_rotate_quant_asym",
           lib.quarot_rotate_quant_asym(_ptr(x), M, K, _ptr(signs), had_block, float(clip), _ptr(q), _ptr(d),
                                        _ptr(z), _ptr(r), _stream(stream)))
    return q, d, z, r


def quarot_uint4_gemm_s32(qa: torch.Tensor, qw: torch.Tensor, acc: Optional[torch.Tensor] = None, stream=None):
    """Exact int32 [M, N] = sum_k u_a u_w of unsigned nibble codes."""
    M, Kh = qa.shape
    N = qw.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=qa.device)
    _check("quarot_uint4_gemm_s32",
           lib.quarot_uint4_gemm_s32(_ptr(qa), M, _ptr(qw), N, 2 * Kh, _ptr(acc), _stream(stream)))
    return acc


def quarot_int4_linear_asym(qa, s_a, z_a, r_a, qw, s_w, z_w, r_w, out: Optional[torch.Tensor] = None,
                            stream=None):
    """The asymmetric INT4 linear layer -> fp16 [M, N]."""
    M, Kh = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=qa.device)
    _check("quarot_int4_linear_asym",
           lib.quarot_int4_linear_asym(_ptr(qa), _ptr(s_a), _ptr(z_a), _ptr(r_a), M, _ptr(qw), _ptr(s_w), _ptr(z_w),
                                       _ptr(r_w), N, 2 * Kh, _ptr(out), _stream(stream)))
    return out


def quarot_kv_quant(k: torch.Tensor, v: torch.Tensor, signs: torch.Tensor, kq=None, ks=None, vq=None, vs=None,
                    stream=None):
    """k, v fp16 [B, T, Hkv, D] -> (kq, ks, vq, vs): packed codes [B, T, Hkv, D/2], fp16 scales [B, T, Hkv]."""
    B, T, H, D = k.shape
    dev = k.device
    kq = kq if kq is not None else torch.empty((B, T, H, D // 2), dtype=torch.uint8, device=dev)
    vq = vq if vq is not None else torch.empty((B, T, H, D // 2), dtype=torch.uint8, device=dev)
    ks = ks if ks is not None else torch.empty((B, T, H), dtype=torch.float16, device=dev)
    vs = vs if vs is not None else torch.empty((B, T, H), dtype=torch.float16, device=dev)
    _check("quarot_kv_quant",
           lib.quarot_kv_quant(_ptr(k), _ptr(v), B, T, H, D, _ptr(signs), _ptr(kq), _ptr(ks), _ptr(vq), _ptr(vs),
                               _stream(stream)))
    return kq, ks, vq, vs


def quarot_kv_decode_scores(q: torch.Tensor, signs: torch.Tensor, kq: torch.Tensor, ks: torch.Tensor,
                            scores: Optional[torch.Tensor] = None, stream=None):
    """q fp16 [B, Hq, D] against the INT4 key cache -> fp32 scores [B, Hq, T]."""
    B, Hq, D = q.shape
    _, T, H, _ = kq.shape
    if scores is None:
        scores = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    _check("quarot_kv_decode_scores",
           lib.quarot_kv_decode_scores(_ptr(q), Hq, _ptr(signs), _ptr(kq), _ptr(ks), B, T, H, D, _ptr(scores),
                                       _stream(stream)))
    return scores


def quarot_rotate_quant_kron(x: torch.Tensor, signs: torch.Tensor, group: int = 0,
                             q: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None, stream=None):
    """Full Kronecker rotation (K = 11008 = 344 * 32) + INT4 RTN + packing -> (q [M, K/2] uint8, scales)."""
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device) if group == 0 else \
            torch.empty((M, K // 128), dtype=torch.float16, device=x.device)
    _check("quarot_rotate_quant_kron",
           lib.quarot_rotate_quant_kron(_ptr(x), M, K, _ptr(signs), group, _ptr(q), _ptr(scales), _stream(stream)))
    return q, scales


def quarot_kron_factor(m: int = 344):
    """The library's Hadamard factor of order m (host int8 tensor [m, m])."""
    h = torch.empty((m, m), dtype=torch.int8)
    _check("quarot_kron_factor", lib.quarot_kron_factor(m, h.data_ptr()))
    return h


def quarot_kv_decode_attend(scores: torch.Tensor, vq: torch.Tensor, vs: torch.Tensor,
                            out: Optional[torch.Tensor] = None, stream=None):
    """scores fp32 [B, Hq, T], vq [B, T, Hkv, 64], vs fp16 [B, T, Hkv] -> fp32 [B, Hq, 128]."""
    B, Hq, T = scores.shape
    Hkv = vq.shape[2]
    if out is None:
        out = torch.empty((B, Hq, 128), dtype=torch.float32, device=scores.device)
    _check("quarot_kv_decode_attend",
           lib.quarot_kv_decode_attend(_ptr(scores), B, Hq, _ptr(vq), _ptr(vs), T, Hkv, 128, _ptr(out),
                                       _stream(stream)))
    return out


def quarot_kv_decode_attention(q: torch.Tensor, signs: torch.Tensor, kq: torch.Tensor, ks: torch.Tensor,
                               vq: torch.Tensor, vs: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """One fused decode step: q fp16 [B, Hq, 128] against the INT4 K and V caches
    [B, T, Hkv, 64] (+ fp16 scales [B, T, Hkv]) -> fp32 [B, Hq, 128]."""
    B, Hq, D = q.shape
    _, T, H, _ = kq.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    _check("quarot_kv_decode_attention",
           lib.quarot_kv_decode_attention(_ptr(q), Hq, _ptr(signs), _ptr(kq), _ptr(ks), _ptr(vq), _ptr(vs), B, T, H,
                                          D, _ptr(out), _stream(stream)))
    return out


def quarot_probe_mma_i8(steps: int, stream=None, operands: int = 0) -> int:
    """Launches the dense INT8 tensor-pipe probe on zero (0), pseudo-random
    byte (1) or pseudo-random high-nibble 4-bit (2) operands; returns the
    integer operations it performs (time it on the stream with CUDA events)."""
    pairs = ctypes.c_int64(0)
    _check("quarot_probe_mma_i8", lib.quarot_probe_mma_i8(steps, operands, ctypes.byref(pairs), _stream(stream)))
    return int(pairs.value) * steps * 4 * 2 * 256 * 256 * 32


def quarot_test_wait_timeout(v: torch.Tensor, withheld_tile: int, wait_limit_ns: int,
                             q: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None, stream=None):
    """The value-row quantizer over v fp16 [rows, 128] with the copy of one
    128-row tile withheld and every wait bounded by wait_limit_ns (tests the
    timeout path); returns (q [rows, 64], scales fp16 [rows])."""
    rows = v.shape[0]
    if q is None:
        q = torch.zeros((rows, 64), dtype=torch.uint8, device=v.device)
    if scales is None:
        scales = torch.zeros((rows,), dtype=torch.float16, device=v.device)
    _check("quarot_test_wait_timeout",
           lib.quarot_test_wait_timeout(_ptr(v), rows, _ptr(q), _ptr(scales), withheld_tile, wait_limit_ns,
                                        _stream(stream)))
    return q, scales


def quarot_get_device_status(stream=None) -> int:
    """Synchronizes `stream` (the whole device when None) and returns, then
    clears, the library's device error word (0 = no bounded wait gave up)."""
    return int(lib.quarot_get_device_status(None if stream is None else _stream(stream)))

"""CPU oracle for the QuaRot online rotation + INT4 hot path (numpy front end).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the CPU-baseline
leg of the benchmark may import this package; the product library never does.
It is independent of the CUDA library (no shared code, headers or tables).
The arithmetic lives in quarot_oracle.c (fp64 / int64); this module only
marshals numpy arrays into it and composes its steps in the method's order:

    x' = (x * diag(s)) * H / sqrt(n)             randomized Hadamard rotation
    s_x = max|x'| / 7, q = clamp(rint(x'/s), -8, 7)   symmetric INT4 RTN
    pack: byte i = q[2i] (bits 0-3) | q[2i+1] (bits 4-7)
    acc = qa . qw^T  (int64), y = acc * s_x[t] * s_w[n]  (fp64, then fp16)

Sources: QuaRot (ISTA record abstract; Elamur Research summary, "Summary" and
"Key points"), the onlyaistuff.com QuaRot article (randomized Hadamard), and
DuQuant (chapterpal) Knowl 1, 2 and 12 for invariance, block-128 rotations and
the per-head Hadamard on the attention path.  Each C function states the
reading it takes where the pages are silent.
"""
import ctypes
import os

import numpy as np

from . import build_oracle

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        sigs = {
            "qo_sylvester": [I64, P],
            "qo_paley": [ctypes.c_int, ctypes.c_int, P],
            "qo_rotate_kron": [P, I64, I64, P, ctypes.c_int, ctypes.c_int, P],
            "qo_fwht": [P, I64],
            "qo_rotate": [P, I64, I64, P, I64, P],
            "qo_rotate_dense": [P, I64, I64, P, I64, P],
            "qo_quantize": [P, I64, I64, I64, P, P, P],
            "qo_quantize_with_scales": [P, I64, I64, I64, P, P],
            "qo_quantize_bits": [P, I64, I64, ctypes.c_int, P, P],
            "qo_quantize_asym": [P, I64, I64, ctypes.c_int, ctypes.c_double, P, P, P, P],
            "qo_dequant_asym": [P, I64, I64, I64, P, P, P, P, P, P, P, P],
            "qo_quantize_asym_with": [P, I64, I64, ctypes.c_int, P, P, P],
            "qo_quantize_bits_with_scales": [P, I64, I64, ctypes.c_int, P, P],
            "qo_pack": [P, I64, P],
            "qo_unpack": [P, I64, P],
            "qo_int_gemm": [P, P, I64, I64, I64, I64, P],
            "qo_dequant_linear": [P, I64, I64, I64, P, P, P, P],
            "qo_kv_quant": [P, P, I64, I64, I64, I64, P, P, P, P, P],
            "qo_kv_scores": [P, I64, I64, I64, I64, I64, P, P, P, P],
            "qo_kv_attend": [P, I64, I64, I64, I64, I64, P, P, P],
            "qo_f16_to_f64_array": [P, I64, P],
            "qo_f64_to_f16_array": [P, I64, P],
            "qo_max_threads": [],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.qo_f16_to_f64_array.restype = None
        L.qo_f64_to_f16_array.restype = None
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def max_threads() -> int:
    return int(lib().qo_max_threads())


# --- fp16 ------------------------------------------------------------------

def f16_bits(x):
    """fp16 array (or bits) -> uint16 bit patterns."""
    x = np.asarray(x)
    if x.dtype == np.float16:
        return np.ascontiguousarray(x).view(np.uint16)
    return _c(x, np.uint16)


def f16_to_f64(bits):
    b = f16_bits(bits)
    out = np.empty(b.shape, np.float64)
    lib().qo_f16_to_f64_array(_p(b), b.size, _p(out))
    return out


def f64_to_f16(x):
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().qo_f64_to_f16_array(_p(x), x.size, _p(out))
    return out


# --- rotation --------------------------------------------------------------

def sylvester(n: int) -> np.ndarray:
    H = np.empty((n, n), np.int8)
    _check(lib().qo_sylvester(n, _p(H)), "sylvester")
    return H


def fwht(v) -> np.ndarray:
    """Unnormalized transform of each row of v (last axis, power-of-two length)."""
    v = _c(v, np.float64).copy()
    n = v.shape[-1]
    flat = v.reshape(-1, n)
    for r in range(flat.shape[0]):
        row = flat[r]
        _check(lib().qo_fwht(_p(row), n), "fwht")
    return v


def rotate(x16, signs, had_block: int = 0, dense: bool = False) -> np.ndarray:
    """x' = (x * diag(s)) * R for each row of the fp16 matrix x16 [M, K]."""
    xb = f16_bits(x16)
    M, K = xb.shape
    s = _c(signs, np.int8)
    assert s.shape == (K,)
    out = np.empty((M, K), np.float64)
    fn = lib().qo_rotate_dense if dense else lib().qo_rotate
    _check(fn(_p(xb), M, K, _p(s), had_block, _p(out)), "rotate")
    return out


def paley(p: int, e: int = 1) -> np.ndarray:
    """Paley's first-construction Hadamard matrix of order p^e + 1 (p^e = 3 mod 4), int8 +-1."""
    n = p ** e + 1
    H = np.empty((n, n), np.int8)
    _check(lib().qo_paley(p, e, _p(H)), "paley")
    return H


def rotate_kron(x16, signs, p: int = 7, e: int = 3) -> np.ndarray:
    """x' = (x * diag(s)) * (H_m (x) H_n) / sqrt(K), m = p^e + 1 (Paley), n = K / m
    (Sylvester).  The default factor is the one for K = 11008 = 344 * 32."""
    xb = f16_bits(x16)
    M, K = xb.shape
    s = _c(signs, np.int8)
    assert s.shape == (K,)
    out = np.empty((M, K), np.float64)
    _check(lib().qo_rotate_kron(_p(xb), M, K, _p(s), p, e, _p(out)), "rotate_kron")
    return out


def rotate_quant_kron(x16, signs, group: int = 0, p: int = 7, e: int = 3):
    """The full-rotation activation step: Kronecker rotation, quantize, pack."""
    xr = rotate_kron(x16, signs, p, e)
    codes, sc = quantize(xr, group)
    return pack(codes), sc, xr


# --- quantizer -------------------------------------------------------------

def quantize(xr, group: int = 0):
    """Returns (codes int8 [M, K], scales): fp64 [M] if group == 0, else fp16 bits [M, K/group]."""
    xr = _c(xr, np.float64)
    M, K = xr.shape
    codes = np.empty((M, K), np.int8)
    if group == 0:
        sc = np.empty((M,), np.float64)
        _check(lib().qo_quantize(_p(xr), M, K, 0, _p(codes), _p(sc), None), "quantize")
    else:
        sc = np.empty((M, K // group), np.uint16)
        _check(lib().qo_quantize(_p(xr), M, K, group, _p(codes), None, _p(sc)), "quantize")
    return codes, sc


def quantize_with_scales(xr, scales, group: int = 0) -> np.ndarray:
    """RTN codes of xr [M, K] under given scales (fp64 [M], or fp16 bits [M, K/group])."""
    xr = _c(xr, np.float64)
    M, K = xr.shape
    sc = _c(scales_to_f64(scales), np.float64)
    codes = np.empty((M, K), np.int8)
    _check(lib().qo_quantize_with_scales(_p(xr), M, K, group, _p(sc), _p(codes)), "quantize_with_scales")
    return codes


def quantize_bits(xr, bits: int):
    """Per-row symmetric RTN at `bits` bits: (codes int8 [M, K], scales fp64 [M]),
    s = max|row| / (2^(bits-1) - 1)."""
    xr = _c(xr, np.float64)
    M, K = xr.shape
    codes = np.empty((M, K), np.int8)
    sc = np.empty((M,), np.float64)
    _check(lib().qo_quantize_bits(_p(xr), M, K, bits, _p(codes), _p(sc)), "quantize_bits")
    return codes, sc


def quantize_bits_with_scales(xr, scales, bits: int) -> np.ndarray:
    """RTN codes at `bits` bits of xr [M, K] under given per-row fp64 scales."""
    xr = _c(xr, np.float64)
    M, K = xr.shape
    sc = _c(scales_to_f64(scales), np.float64)
    codes = np.empty((M, K), np.int8)
    _check(lib().qo_quantize_bits_with_scales(_p(xr), M, K, bits, _p(sc), _p(codes)), "quantize_bits_with_scales")
    return codes


def rotate_quant8(x16, signs, had_block: int = 0):
    """The INT8 activation step: rotate, then per-row RTN at 8 bits (codes stay
    one byte each).  Returns (codes int8 [M, K], scales fp64 [M], x')."""
    xr = rotate(x16, signs, had_block)
    codes, sc = quantize_bits(xr, 8)
    return codes, sc, xr


def linear8(x16, w16, signs, had_block: int = 0):
    """The INT8 prefill linear: both operands rotated and quantized per row at
    8 bits, then the integer product and the dequantized fp16 output."""
    qa, sa, _ = rotate_quant8(x16, signs, had_block)
    qw, sw, _ = rotate_quant8(w16, signs, had_block)
    acc = int_gemm(qa, qw, 0)
    y, y16 = dequant_linear(acc, sa, sw, 0)
    return dict(qa=qa, sa=sa, qw=qw, sw=sw, acc=acc, y=y, y16=y16)


def quantize_asym(xr, clip: float, bits: int = 4):
    """Per-row asymmetric RTN with clipping: (codes int8 in [0, 2^bits-1] [M, K],
    step fp64 [M], zero point int64 [M], code row sums int64 [M])."""
    xr = _c(xr, np.float64)
    M, K = xr.shape
    codes = np.empty((M, K), np.int8)
    d = np.empty((M,), np.float64)
    z = np.empty((M,), np.int64)
    r = np.empty((M,), np.int64)
    _check(lib().qo_quantize_asym(_p(xr), M, K, bits, float(clip), _p(codes), _p(d), _p(z), _p(r)),
           "quantize_asym")
    return codes, d, z, r


def quantize_asym_with(xr, step, zero, bits: int = 4) -> np.ndarray:
    """Asymmetric RTN codes of xr [M, K] under given per-row steps and zero points."""
    xr = _c(xr, np.float64)
    M, K = xr.shape
    codes = np.empty((M, K), np.int8)
    _check(lib().qo_quantize_asym_with(_p(xr), M, K, bits, _p(_c(step, np.float64)), _p(_c(zero, np.int64)),
                                       _p(codes)), "quantize_asym_with")
    return codes


def dequant_asym(acc, K, da, za, ra, dw, zw, rw):
    """y = da dw (acc - zw ra - za rw + K za zw).  Returns (y fp64, y fp16 bits)."""
    acc = _c(np.asarray(acc, np.int64), np.int64)
    M, N = acc.shape
    y = np.empty((M, N), np.float64)
    y16 = np.empty((M, N), np.uint16)
    _check(lib().qo_dequant_asym(_p(acc), M, N, K, _p(_c(da, np.float64)), _p(_c(za, np.int64)),
                                 _p(_c(ra, np.int64)), _p(_c(dw, np.float64)), _p(_c(zw, np.int64)),
                                 _p(_c(rw, np.int64)), _p(y), _p(y16)), "dequant_asym")
    return y, y16


def rotate_quant_asym(x16, signs, clip: float, had_block: int = 0):
    """Rotate, then per-row asymmetric 4-bit RTN with clipping, packed (low nibble =
    even element).  Returns (packed, step, zero, rowsum, x')."""
    xr = rotate(x16, signs, had_block)
    codes, d, z, r = quantize_asym(xr, clip, 4)
    return pack(codes), d, z, r, xr


def linear_asym(x16, w16, signs, clip_a: float = 0.9, clip_w: float = 0.8, had_block: int = 0):
    """The asymmetric INT4 linear: activations per token (clip_a), weights per
    output channel (clip_w), integer product of the unsigned codes and the
    zero-point-corrected dequantized output."""
    qa, da, za, ra, _ = rotate_quant_asym(x16, signs, clip_a, had_block)
    qw, dw, zw, rw, _ = rotate_quant_asym(w16, signs, clip_w, had_block)
    ua = unpack(qa) & 0x0F
    uw = unpack(qw) & 0x0F
    acc = int_gemm(ua, uw, 0)
    K = ua.shape[1]
    y, y16 = dequant_asym(acc, K, da, za, ra, dw, zw, rw)
    return dict(qa=qa, da=da, za=za, ra=ra, qw=qw, dw=dw, zw=zw, rw=rw, acc=acc, y=y, y16=y16)


def pack(codes) -> np.ndarray:
    c = _c(codes, np.int8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] // 2,), np.uint8)
    _check(lib().qo_pack(_p(c), c.size, _p(out)), "pack")
    return out


def unpack(packed) -> np.ndarray:
    p = _c(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.int8)
    _check(lib().qo_unpack(_p(p), p.size * 2, _p(out)), "unpack")
    return out


def rotate_quant(x16, signs, had_block: int = 0, group: int = 0):
    """The full activation step: rotate, quantize, pack.  Returns (packed, scales, x')."""
    xr = rotate(x16, signs, had_block)
    codes, sc = quantize(xr, group)
    return pack(codes), sc, xr


# --- integer product -------------------------------------------------------

def int_gemm(qa, qw, group: int = 0) -> np.ndarray:
    """acc[m, n(, g)] = sum_k qa[m, k] qw[n, k] over each group (int64)."""
    qa = _c(qa, np.int8)
    qw = _c(qw, np.int8)
    M, K = qa.shape
    N, K2 = qw.shape
    assert K == K2
    G = 1 if group == 0 else K // group
    acc = np.empty((M, N, G), np.int64)
    _check(lib().qo_int_gemm(_p(qa), _p(qw), M, N, K, group, _p(acc)), "int_gemm")
    return acc[:, :, 0] if group == 0 else acc


def scales_to_f64(sc):
    """fp64 scales pass through; fp16 bit patterns (or fp16 arrays) decode exactly."""
    sc = np.asarray(sc)
    if sc.dtype in (np.uint16, np.float16):
        return f16_to_f64(sc)
    return _c(sc, np.float64)


def dequant_linear(acc, sa, sw, group: int = 0):
    """y = acc * sa[m] * sw[n] (or the group sum).  Returns (y fp64, y fp16 bits)."""
    acc = np.asarray(acc, np.int64)
    if group == 0:
        M, N = acc.shape
        G = 1
        acc = acc.reshape(M, N, 1)
    else:
        M, N, G = acc.shape
    acc = _c(acc, np.int64)
    sa64 = scales_to_f64(sa).reshape(M, G)
    sw64 = scales_to_f64(sw).reshape(N, G)
    sa64 = _c(sa64, np.float64)
    sw64 = _c(sw64, np.float64)
    y = np.empty((M, N), np.float64)
    y16 = np.empty((M, N), np.uint16)
    _check(lib().qo_dequant_linear(_p(acc), M, N, G, _p(sa64), _p(sw64), _p(y), _p(y16)),
           "dequant_linear")
    return y, y16


def weight_prep(w16, signs, had_block: int = 0, group: int = 0):
    """Offline weight step: rotate the rows of W with the same signs and Hadamard
    (QuaRot summary: most rotations are fused into the weights), then quantize
    per output channel (group 0) or per 128-group.  Returns (packed, scales)."""
    packed, sc, _ = rotate_quant(w16, signs, had_block, group)
    return packed, sc


def linear(x16, w16, signs, had_block: int = 0, group: int = 0):
    """The whole prefill linear: both operands rotated and quantized, then the
    integer product and the dequantized fp16 output."""
    qa_p, sa, _ = rotate_quant(x16, signs, had_block, group)
    qw_p, sw = weight_prep(w16, signs, had_block, group)
    acc = int_gemm(unpack(qa_p), unpack(qw_p), group)
    y, y16 = dequant_linear(acc, sa, sw, group)
    return dict(qa=qa_p, sa=sa, qw=qw_p, sw=sw, acc=acc, y=y, y16=y16)


# --- KV cache --------------------------------------------------------------

def kv_quant(k16, v16, signs):
    """k16, v16: fp16 [B, T, H, D]; signs [H, D].  Returns packed codes and fp16-bit scales."""
    kb = f16_bits(k16)
    vb = f16_bits(v16)
    B, T, H, D = kb.shape
    s = _c(signs, np.int8)
    assert s.shape == (H, D)
    kc = np.empty((B, T, H, D), np.int8)
    vc = np.empty((B, T, H, D), np.int8)
    ks = np.empty((B, T, H), np.uint16)
    vs = np.empty((B, T, H), np.uint16)
    _check(lib().qo_kv_quant(_p(kb), _p(vb), B, T, H, D, _p(s), _p(kc), _p(ks), _p(vc), _p(vs)),
           "kv_quant")
    return pack(kc), ks, pack(vc), vs


def kv_scores(q16, signs, kq_packed, ks):
    """q16 fp16 [B, Hq, D]; kq_packed [B, T, H, D/2]; ks fp16 bits [B, T, H] -> fp64 [B, Hq, T]."""
    qb = f16_bits(q16)
    B, Hq, D = qb.shape
    kc = unpack(kq_packed)
    _, T, H, _ = kc.shape
    s = _c(signs, np.int8)
    ks64 = _c(scales_to_f64(ks), np.float64)
    out = np.empty((B, Hq, T), np.float64)
    _check(lib().qo_kv_scores(_p(qb), B, Hq, H, D, T, _p(s), _p(kc), _p(ks64), _p(out)),
           "kv_scores")
    return out


def kv_attend(scores, vq_packed, vs):
    """scores [B, Hq, T] (any float); vq_packed [B, T, H, D/2]; vs fp16 bits [B, T, H]
    -> fp64 [B, Hq, D]: softmax(scores / sqrt(D)) over T times the dequantized values."""
    sc = _c(np.asarray(scores, np.float64), np.float64)
    B, Hq, T = sc.shape
    vc = unpack(vq_packed)
    _, T2, H, D = vc.shape
    assert T2 == T
    vs64 = _c(scales_to_f64(vs), np.float64)
    out = np.empty((B, Hq, D), np.float64)
    _check(lib().qo_kv_attend(_p(sc), B, Hq, H, D, T, _p(vc), _p(vs64), _p(out)), "kv_attend")
    return out

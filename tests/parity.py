"""Parity rules between the CUDA library and the CPU oracle.

 * Integer and byte results (int32 accumulators from identical codes, packed
   bytes from identical codes) must be bit-exact.
 * Scales: a per-token / per-channel fp32 scale within 1e-6 relative of the
   oracle's fp64 max|x'|/7.  An fp16 group scale equal to the oracle's fp16
   scale, or one fp16 step away only when the oracle's exact max|x'|/7 lies
   within 1e-5 (relative) of the rounding midpoint between the two: both are
   then correct roundings of a near-tie.
 * Codes: once a scale has passed that check, the expected codes are the
   oracle's RTN of its own fp64 rotated values under that scale.  A device
   code may differ from them only by +-1, only where the oracle's v/s lies
   within 1e-3 of a rounding boundary, and in at most 1e-4 of the elements.
   (The kernel rotates in fp32, the oracle in fp64; the decision can flip
   only at such near-ties.)  Values lying exactly on a boundary (v/s = k + 1/2
   to fp64 precision, which structured inputs such as constant rows produce
   in bulk) have two correct roundings -- any perturbation of s in either
   direction picks one -- so either is accepted there and such elements are
   not counted against the 1e-4 budget.
 * fp16 outputs: max relative error 2e-3 against the oracle's fp64 product,
   relative to max(|y_ref|, 1e-2 * rms(y_ref row)) so that outputs near zero
   (which any rounding order perturbs by more than 2e-3 of themselves) are
   measured on the row's scale.
"""
import numpy as np

import oracle


def unpack_codes(packed) -> np.ndarray:
    return oracle.unpack(np.asarray(packed, np.uint8))


def check_scales(gpu_scales, xr, group):
    """Returns the device scales as fp64 once they pass the scale rule."""
    M, K = xr.shape
    if group == 0:
        amax = np.abs(xr).max(axis=1)
        ref = amax / 7.0
        got = np.asarray(gpu_scales, np.float64)
        rel = np.abs(got - ref) / np.maximum(ref, 1e-300)
        bad = (rel > 1e-6) & ~((ref == 0) & (got == 0))
        assert not np.any(bad), f"per-token scales off: max rel {rel[bad].max():.3e} at rows {np.nonzero(bad)[0][:5]}"
        return got
    G = K // group
    amax = np.abs(xr.reshape(M, G, group)).max(axis=2)
    exact = amax / 7.0
    ref16 = oracle.f64_to_f16(exact)
    got16 = np.asarray(gpu_scales).view(np.uint16).reshape(M, G)
    diff = got16.astype(np.int64) - ref16.astype(np.int64)
    off = diff != 0
    if np.any(off):
        assert np.all(np.abs(diff[off]) == 1), "fp16 scales more than one step off"
        a = oracle.f16_to_f64(got16[off])
        b = oracle.f16_to_f64(ref16[off])
        mid = (a + b) / 2
        near = np.abs(exact[off] - mid) <= 1e-5 * np.abs(mid)
        assert np.all(near), "fp16 scale differs from the oracle away from a rounding near-tie"
    return got16


def check_codes(gpu_packed, gpu_scales, xr, group, max_frac=1e-4):
    """Applies the scale and code rules; returns the number of near-tie flips."""
    sc = check_scales(gpu_scales, xr, group)
    expect = oracle.quantize_with_scales(xr, sc, group)
    got = unpack_codes(gpu_packed).reshape(xr.shape)
    d = got.astype(np.int16) - expect.astype(np.int16)
    flips = d != 0
    n = int(flips.sum())
    if n == 0:
        return 0
    assert np.all(np.abs(d[flips]) == 1), "codes differ by more than one step"
    M, K = xr.shape
    s = oracle.scales_to_f64(sc)
    s_el = np.repeat(s.reshape(M, -1), K if group == 0 else group, axis=1)
    t = np.where(s_el > 0, xr / np.where(s_el > 0, s_el, 1.0), 0.0)
    dist = np.abs(t - (np.floor(t) + 0.5))
    assert np.all(dist[flips] < 1e-3), f"code flips away from near-ties (max dist {dist[flips].max():.3e})"
    # exact ties are decided with the oracle's own scale (fp64 max|x'|/7 per row,
    # or the checked fp16 group scale)
    if group == 0:
        s0 = np.abs(xr).max(axis=1, keepdims=True) / 7.0
        t0 = np.where(s0 > 0, xr / np.where(s0 > 0, s0, 1.0), 0.0)
    else:
        t0 = t
    exact_tie = np.abs(t0 - (np.floor(t0) + 0.5)) <= 1e-9 * np.maximum(1.0, np.abs(t0))
    counted = int((flips & ~exact_tie).sum())
    assert counted <= max_frac * got.size, f"{counted} near-tie code flips in {got.size} elements"
    return n


def check_f16_output(y_gpu_f16, y_ref, tol=2e-3):
    y = np.asarray(y_gpu_f16, np.float16).astype(np.float64)
    ref = np.asarray(y_ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    denom = np.maximum(np.abs(ref), 1e-2 * rms)
    denom = np.where(denom > 0, denom, 1.0)
    err = np.abs(y - ref) / denom
    assert np.all(np.isfinite(y)), "non-finite outputs"
    worst = float(err.max()) if err.size else 0.0
    assert worst <= tol, f"max relative error {worst:.3e} > {tol}"
    return worst


def check_codes_bits(gpu_codes, gpu_scales, xr, bits, max_frac=1e-4):
    """The scale and code rules for per-row codes of `bits` bits stored one per
    byte (the 8-bit variant): scale within 1e-6 relative of the oracle's fp64
    max|x'| / (2^(bits-1) - 1); codes equal the oracle's RTN under the device
    scale, or +-1 only at near-ties (same budget and exact-tie rule as the
    INT4 check).  Returns the number of flips."""
    qmax = float((1 << (bits - 1)) - 1)
    M, K = xr.shape
    amax = np.abs(xr).max(axis=1)
    ref = amax / qmax
    got_s = np.asarray(gpu_scales, np.float64)
    rel = np.abs(got_s - ref) / np.maximum(ref, 1e-300)
    bad = (rel > 1e-6) & ~((ref == 0) & (got_s == 0))
    assert not np.any(bad), f"per-row scales off: max rel {rel[bad].max():.3e}"
    expect = oracle.quantize_bits_with_scales(xr, got_s, bits)
    got = np.asarray(gpu_codes).view(np.int8).reshape(M, K)
    d = got.astype(np.int16) - expect.astype(np.int16)
    flips = d != 0
    n = int(flips.sum())
    if n == 0:
        return 0
    assert np.all(np.abs(d[flips]) == 1), "codes differ by more than one step"
    t = np.where(got_s[:, None] > 0, xr / np.where(got_s[:, None] > 0, got_s[:, None], 1.0), 0.0)
    dist = np.abs(t - (np.floor(t) + 0.5))
    assert np.all(dist[flips] < 1e-3), f"code flips away from near-ties (max dist {dist[flips].max():.3e})"
    s0 = ref[:, None]
    t0 = np.where(s0 > 0, xr / np.where(s0 > 0, s0, 1.0), 0.0)
    exact_tie = np.abs(t0 - (np.floor(t0) + 0.5)) <= 1e-9 * np.maximum(1.0, np.abs(t0))
    counted = int((flips & ~exact_tie).sum())
    assert counted <= max_frac * got.size, f"{counted} near-tie code flips in {got.size} elements"
    return n


def check_codes_asym(gpu_packed, gpu_step, gpu_zero, gpu_rowsum, xr, clip, max_frac=1e-4):
    """Rules for the asymmetric 4-bit quantizer (per row: step from the clipped
    min/max, zero point, unsigned codes, code sum).
     * step within 1e-6 relative of the oracle's fp64 step;
     * zero point equal to the oracle's, or one away only where the oracle's
       -lo/step lies within 1e-4 of a rounding boundary (both are correct
       roundings of a near-tie);
     * codes: the oracle's RTN under the device's step and zero point, +-1
       only within 1e-3 of a rounding boundary, at most max_frac of elements
       (exact ties excluded, as in the symmetric rule);
     * the code sum equals the sum of the device's own codes."""
    M, K = xr.shape
    u_o, d_o, z_o, _ = oracle.quantize_asym(xr, clip)
    d = np.asarray(gpu_step, np.float64)
    z = np.asarray(gpu_zero, np.int64)
    rel = np.abs(d - d_o) / np.maximum(d_o, 1e-300)
    bad = (rel > 1e-6) & ~((d_o == 0) & (d == 0))
    assert not np.any(bad), f"steps off: max rel {rel[bad].max():.3e}"
    dz = z - z_o
    if np.any(dz != 0):
        assert np.all(np.abs(dz[dz != 0]) == 1), "zero points more than one away"
        lo = clip * xr.min(axis=1)
        t = np.where(d_o > 0, -lo / np.where(d_o > 0, d_o, 1.0), 0.0)
        dist = np.abs(t - (np.floor(t) + 0.5))
        assert np.all(dist[dz != 0] < 1e-4), "zero point differs away from a rounding near-tie"
    got = (oracle.unpack(np.asarray(gpu_packed, np.uint8)) & 0x0F).astype(np.int64).reshape(M, K)
    np.testing.assert_array_equal(got.sum(axis=1), np.asarray(gpu_rowsum, np.int64))
    expect = oracle.quantize_asym_with(xr, d, z).astype(np.int64)
    diff = got - expect
    flips = diff != 0
    if not np.any(flips):
        return 0
    assert np.all(np.abs(diff[flips]) == 1), "codes differ by more than one step"
    t = np.where(d[:, None] > 0, xr / np.where(d[:, None] > 0, d[:, None], 1.0), 0.0)
    dist = np.abs(t - (np.floor(t) + 0.5))
    assert np.all(dist[flips] < 1e-3), f"code flips away from near-ties (max dist {dist[flips].max():.3e})"
    exact_tie = dist <= 1e-9 * np.maximum(1.0, np.abs(t))
    counted = int((flips & ~exact_tie).sum())
    assert counted <= max_frac * got.size, f"{counted} near-tie code flips in {got.size} elements"
    return int(flips.sum())

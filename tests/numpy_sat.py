"""Saturation counts restated in plain numpy fp32 arithmetic.

The oracle and the kernels both report how many elements of a quantisation
call had a pre-clamp magnitude |fp32(x * s)| more than one fp32 ulp above the
encoding's largest finite value (the observable form of the silent clipping
that "FP8 su GPU AMD: ..." (ai-radar.it), section "La correttezza del formato
viene prima del tuning", warns about when a tensor is scaled against the wrong
maximum).  This module computes that count a third way, with numpy's IEEE fp32
division and multiplication, so that the exact value can be pinned at any
size.  It shares nothing with the oracle or the CUDA library.
"""
import numpy as np

ENC_MAX = {0: 448.0, 1: 240.0}  # e4m3fn, e4m3fnuz largest finite values


def _f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _threshold(fmt):
    return np.nextafter(np.float32(ENC_MAX[fmt]), np.float32(np.inf))


def _scales(amax, smax):
    return (np.float32(smax) / np.maximum(amax, np.float32(1e-12))).astype(np.float32)


def rowwise(x_bits, fmt, scale_max=0.0, chunk=4096):
    """Count for a rowwise call on bf16 patterns x_bits [rows, cols]."""
    smax = scale_max if scale_max > 0 else ENC_MAX[fmt]
    thr = _threshold(fmt)
    total = 0
    for r0 in range(0, x_bits.shape[0], chunk):
        x = _f32(x_bits[r0:r0 + chunk])
        s = _scales(np.abs(x).max(axis=1), smax)
        y = (x * s[:, None]).astype(np.float32)
        total += int((np.abs(y) > thr).sum())
    return total


def colwise_jagged(x_bits, offsets, fmt, scale_max=0.0):
    """Count for a jagged column-wise call (offsets: cumulative group ends)."""
    smax = scale_max if scale_max > 0 else ENC_MAX[fmt]
    thr = _threshold(fmt)
    rows = x_bits.shape[0]
    total = 0
    start = 0
    for end in np.asarray(offsets, np.int64):
        end = min(max(int(end), start), rows)
        if end > start:
            x = _f32(x_bits[start:end])
            s = _scales(np.abs(x).max(axis=0), smax)
            y = (x * s[None, :]).astype(np.float32)
            total += int((np.abs(y) > thr).sum())
        start = end
    return total

"""bfloat16 round-to-nearest-even, written out from the IEEE 754 definition.

Test infrastructure: part of the fp64 CPU oracle. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm
may import it. The CUDA path never does.

bfloat16 is binary32 with the low 16 fraction bits dropped: 1 sign bit,
8 exponent bits (bias 127, the same range as binary32) and 7 stored
fraction bits, i.e. 8 significant bits.  For a finite real x with
|x| >= 2^-126 the spacing of representable values next to x is
2^(floor(log2|x|) - 7); below 2^-126 (subnormals) the spacing is the
fixed 2^-133.  Rounding to nearest with ties to the even neighbour is
``rint(x / q) * q`` with q that spacing, because ``x / q`` is exact in
binary64 (q is a power of two) and ``numpy.rint`` rounds half to even.
A result of magnitude >= 2^128 is out of range and becomes +-inf.

These values are returned as float64 numbers (every bfloat16 is exactly
representable in binary64), so the rest of the oracle can keep working in
binary64 on the very values a bfloat16 tensor holds.
"""
import numpy as np

_EMIN = -126          # smallest normal exponent of binary32 / bfloat16
_FRAC_BITS = 7        # stored fraction bits of bfloat16
_OVERFLOW = 2.0 ** 128


def bf16_round(x):
    """Round float64 values to the nearest bfloat16 (ties to even); float64 out."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    finite = np.isfinite(ax)
    safe = np.where(finite & (ax > 0), ax, 1.0)
    _, e2 = np.frexp(safe)                       # safe = m * 2**e2, m in [0.5, 1)
    expo = np.maximum(e2 - 1, _EMIN)             # floor(log2|x|), clamped to the subnormal range
    q = np.ldexp(1.0, expo - _FRAC_BITS)         # spacing of bfloat16 values near |x|
    y = np.rint(safe / q) * q
    y = np.where(y >= _OVERFLOW, np.inf, y)
    y = np.where(ax > 0, y, 0.0)
    y = np.where(finite, y, ax)                  # inf stays inf, nan stays nan
    return np.copysign(y, x)


def bf16_bits(x):
    """bfloat16 bit patterns (uint16) of float64 values that are already bfloat16."""
    v = np.asarray(x, dtype=np.float64)
    r = bf16_round(v)
    if not np.array_equal(r[np.isfinite(v)], v[np.isfinite(v)]):
        raise ValueError("bf16_bits: values are not bfloat16-representable")
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(bits):
    """float64 values of uint16 bfloat16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_ulp(x):
    """Spacing of bfloat16 values at |x| (the unit in the last place)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    safe = np.where(ax > 0, ax, 2.0 ** _EMIN)
    _, e2 = np.frexp(safe)
    return np.ldexp(1.0, np.maximum(e2 - 1, _EMIN) - _FRAC_BITS)

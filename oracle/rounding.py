"""Rounding of float64 values onto a binary floating-point format (fp16, bf16).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

A binary format with ``p`` significand bits (implicit bit included), minimum
normal exponent ``emin`` and largest finite value ``vmax`` represents, in the
binade [2**E, 2**(E+1)) with E >= emin, exactly the multiples of
``ulp(E) = 2**(E - p + 1)``; below 2**emin (subnormals) the spacing stays
``ulp(emin)``.  Rounding ``x`` therefore means: find E = max(floor(log2|x|), emin),
divide by ulp(E) (exact: a power of two), round the quotient to an integer with
the chosen rule, multiply back.  Overflow past ``vmax`` gives +-inf for
round-to-nearest (IEEE-754 section 4.3 / 7.4 behaviour).

The scale formats of the pages' methods use two binary16-sized formats:

* fp16 (IEEE binary16): p = 11, emin = -14, vmax = 65504.
* bf16 (bfloat16):      p = 8,  emin = -126, vmax = (2 - 2**-7) * 2**127.

Pinned by ``tests/test_oracle.py``: against numpy's float64 -> float16 cast and
torch's float32 -> bfloat16 cast (library routines) on random values, exact ties
and subnormals, and against hand-listed boundary values.
"""

import numpy as np

FP16 = dict(p=11, emin=-14, vmax=65504.0)
BF16 = dict(p=8, emin=-126, vmax=float((2.0 - 2.0 ** -7) * 2.0 ** 127))


def _round(x, p, emin, vmax, mode):
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    # frexp: ax = m * 2**e with 0.5 <= m < 1, so floor(log2 ax) = e - 1 exactly.
    _, e = np.frexp(ax)
    E = np.maximum(e.astype(np.int64) - 1, emin)
    shift = (p - 1) - E  # x * 2**shift has its unit in the last place at 1
    scaled = np.ldexp(x, shift)
    if mode == "rne":
        r = np.rint(scaled)  # numpy rint is round-half-to-even
    elif mode == "down":
        r = np.floor(scaled)
    elif mode == "up":
        r = np.ceil(scaled)
    else:
        raise ValueError(mode)
    out = np.ldexp(r, -shift)
    out = np.where(ax == 0.0, x, out)  # keep signed zeros untouched
    if mode == "rne":
        out = np.where(np.abs(out) > vmax, np.copysign(np.inf, x), out)
    elif mode == "up":
        out = np.where(out > vmax, np.inf, np.where(out < -vmax, -vmax, out))
    else:
        out = np.where(out < -vmax, -np.inf, np.where(out > vmax, vmax, out))
    return out


def fp16_rne(x):
    """Round float64 ``x`` to the nearest fp16 value, ties to even."""
    return _round(x, mode="rne", **FP16)


def bf16_rne(x):
    """Round float64 ``x`` to the nearest bf16 value, ties to even."""
    return _round(x, mode="rne", **BF16)


def bf16_down(x):
    """Round float64 ``x`` toward -inf onto the bf16 grid."""
    return _round(x, mode="down", **BF16)


def bf16_up(x):
    """Round float64 ``x`` toward +inf onto the bf16 grid."""
    return _round(x, mode="up", **BF16)


def fp16_bits(v):
    """uint16 bit patterns of values already representable in fp16."""
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits(v):
    """uint16 bit patterns of values already representable in bf16."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def fp16_value(bits):
    """float64 values of fp16 bit patterns."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_value(bits):
    """float64 values of bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)

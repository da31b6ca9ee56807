"""bfloat16 bit patterns <-> float64, written out from the format's definition.

bfloat16 is the upper 16 bits of an IEEE-754 binary32: 1 sign bit, 8 exponent
bits, 7 stored mantissa bits.  Widening is exact (append 16 zero bits);
narrowing rounds to nearest, ties to even, the rounding the pages leave open and
the plainest reading for "bf16 output".  Part of the oracle (test
infrastructure only).
"""

import numpy as np


def bf16_bits_to_f64(bits):
    """Exact value of each bf16 bit pattern (uint16 array) as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x):
    """Round float64 values to bf16, nearest-even, returning uint16 patterns.

    Done in two exact-enough stages: float64 -> the two neighbouring bf16 values
    are found from the binary32 pattern of x truncated toward zero, and the
    nearer one is chosen in float64 arithmetic (ties -> even mantissa).  No
    double rounding: the comparison uses the float64 value itself.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat = x.reshape(-1)
    o = out.reshape(-1)
    for start in range(0, flat.size, 1 << 22):
        v = flat[start:start + (1 << 22)]
        # binary32 truncation toward zero of v (exact neighbours bracket v)
        f32 = v.astype(np.float32)  # nearest binary32
        f32 = np.where(np.abs(f32.astype(np.float64)) > np.abs(v),
                       np.nextafter(f32, np.float32(0)), f32).astype(np.float32)
        u = f32.view(np.uint32)
        lo_bits = (u >> np.uint32(16)).astype(np.uint32)          # |lo| <= |v|
        hi_bits = lo_bits + np.uint32(1)                            # next bf16 away from 0
        lo = bf16_bits_to_f64(lo_bits.astype(np.uint16))
        hi = bf16_bits_to_f64(hi_bits.astype(np.uint16))
        dlo = np.abs(v - lo)
        dhi = np.abs(hi - v)
        pick_hi = (dhi < dlo) | ((dhi == dlo) & ((lo_bits & np.uint32(1)) == 1))
        # exact bf16 values (v == lo) stay lo
        pick_hi &= (dlo != 0)
        res = np.where(pick_hi, hi_bits, lo_bits).astype(np.uint16)
        # keep the sign of zero / negative values: lo_bits already carry the sign
        o[start:start + v.size] = res
    return out


def bf16_ulp_distance(bits_a, bits_b):
    """Number of representable bf16 values between two patterns (0 = equal).

    +0 and -0 count as equal.  Patterns are mapped to a monotone integer line
    (sign-magnitude -> two's complement) before subtracting.
    """
    a = np.asarray(bits_a, dtype=np.uint16).astype(np.int32)
    b = np.asarray(bits_b, dtype=np.uint16).astype(np.int32)

    def line(v):
        mag = v & 0x7FFF
        return np.where(v & 0x8000, -mag, mag)

    return np.abs(line(a) - line(b))

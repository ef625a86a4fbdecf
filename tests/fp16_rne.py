"""IEEE 754 binary16 round-to-nearest-even of fp32 bit patterns, written from
the format's definition with integer arithmetic only (sign, 8-bit exponent
and 23-bit fraction in; sign, 5-bit exponent biased by 15 and 10-bit
fraction out; results below 2^-14 are subnormal multiples of 2^-24, results
of magnitude 65520 and above overflow to infinity).  Independent of numpy's
and CUDA's conversions, which the tests check against it.  NaN inputs are
out of its scope."""
import numpy as np


def fp16_bits_rne(u32: np.ndarray) -> np.ndarray:
    u = np.asarray(u32, dtype=np.uint32).astype(np.int64)
    sign = (u >> 31) & 1
    exp = (u >> 23) & 0xFF
    frac = u & 0x7FFFFF
    S = np.where(exp > 0, frac | (1 << 23), frac)           # significand: value = S * 2^(e - 23)
    e = np.where(exp > 0, exp - 127, -126)
    # bits of S dropped: 13 in the fp16 normal range (e >= -14), more below it
    shift = np.minimum(np.where(e >= -14, 13, 13 + (-14 - e)), 40)
    r = S >> shift
    rem = S & ((np.int64(1) << shift) - 1)
    half = np.int64(1) << (shift - 1)
    up = (rem > half) | ((rem == half) & ((r & 1) == 1))
    r = r + up.astype(np.int64)
    normal = e >= -14
    # normal: r holds 11 bits (implicit bit included); a carry to 2^11 moves up a binade
    carry = normal & (r >= (1 << 11))
    r = np.where(carry, r >> 1, r)
    e2 = np.where(carry, e + 1, e)
    nbits = ((e2 + 15) << 10) | (r & 0x3FF)
    # subnormal: r counts 2^-24 (r == 1024 is 2^-14, the smallest normal: the same bits)
    bits = np.where(normal, nbits, r)
    bits = np.where(normal & (e2 > 15), 0x7C00, bits)        # overflow
    bits = np.where(exp == 0xFF, 0x7C00, bits)               # infinity (NaN excluded by callers)
    return ((sign << 15) | bits).astype(np.uint16)


def stratified_fp32_patterns(rng: np.random.Generator) -> np.ndarray:
    """fp32 bit patterns (no NaN) that stress the conversion: every exponent
    with fraction tails at, just below and just above the rounding point of
    the fp16 spacing for that exponent (including the subnormal range),
    exact fp16 values, overflow and underflow edges, and random patterns."""
    out = []
    for ex in range(0, 255):
        e = ex - 127 if ex > 0 else -126
        sh = 13 if e >= -14 else min(13 + (-14 - e), 24)
        hi = rng.integers(0, 1 << max(0, 23 - sh), 16, dtype=np.uint64) << np.uint64(sh) if sh < 23 else np.zeros(16, np.uint64)
        half = np.uint64(1) << np.uint64(sh - 1) if sh >= 1 else np.uint64(0)
        for tail in (np.uint64(0), half - np.uint64(1), half, half + np.uint64(1),
                     (np.uint64(1) << np.uint64(sh)) - np.uint64(1)):
            fr = (hi | tail) & np.uint64(0x7FFFFF)
            for s in (0, 1):
                out.append((np.uint64(s) << np.uint64(31)) | (np.uint64(ex) << np.uint64(23)) | fr)
    out.append(rng.integers(0, 1 << 32, 200000, dtype=np.uint64))
    u = np.concatenate([np.atleast_1d(x) for x in out]).astype(np.uint32)
    f = u.view(np.float32)
    return u[~np.isnan(f)]

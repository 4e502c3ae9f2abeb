"""Element and scale number formats, written as plain nearest-value searches.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

E2M1 ("DeepSeek-V4.1-Flash-NVFP4", §二): one sign bit, two exponent bits, one
mantissa bit; the eight magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Code bits
are ``s e1 e0 m`` so the magnitude code is the index into that list.

E4M3 (the NVFP4 block-scale type; the QAT page, §2.1, gives its maximum as
448): bias 7, three mantissa bits, subnormals m * 2^-9, 0x7F is NaN and is
never produced here.

UE8M0 (the MXFP4 block-scale type, "DeepSeek-V4.1-Flash-NVFP4" §三): an
unsigned power of two 2^(c-127); c = 255 is NaN.

Rounding reading (the pages are silent): round to nearest, ties to the code
whose mantissa LSB is 0 (= the even code), saturate to the largest finite
value.  The sign of an E2M1 result is the input's sign bit even when the
magnitude rounds to zero.

Every encoder is a nearest-value search over the format's own value list,
done exactly in fp64 (each fp32 input and each format value is exact in fp64,
so distances and the tie test are exact).
"""
import numpy as np

# The page's table: magnitude index -> value.
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def e2m1_decode(codes):
    """4-bit codes (uint8 in 0..15) -> float64 values."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where(codes & 8, -mag, mag)


def _nearest_code(absval, values):
    """Index of the nearest entry of the ascending ``values`` (float64) to each
    non-negative ``absval``; ties go to the even index; above the last value
    the last index (saturation)."""
    absval = np.asarray(absval, dtype=np.float64)
    n = len(values)
    hi = np.searchsorted(values, absval, side="left")  # first values[hi] >= absval
    hi = np.clip(hi, 0, n - 1)
    lo = np.clip(hi - 1, 0, n - 1)
    d_lo = absval - values[lo]
    d_hi = values[hi] - absval
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    # absval beyond the largest value: saturate (satfinite)
    idx = np.where(absval >= values[-1], n - 1, idx)
    return idx.astype(np.uint8)


def e2m1_encode(v):
    """fp32 array -> 4-bit E2M1 codes (uint8), RNE with ties to even, satfinite,
    sign bit copied from the input (so -0.0 and small negatives give code 8)."""
    v = np.asarray(v, dtype=np.float32)
    mag = _nearest_code(np.abs(v.astype(np.float64)), E2M1_MAGNITUDES)
    sign = np.signbit(v).astype(np.uint8) << 3
    return (mag | sign).astype(np.uint8)


def _e4m3_values():
    vals = []
    for c in range(0x7F):  # 0x00 .. 0x7E, 0x7F is NaN
        e, m = c >> 3, c & 7
        if e == 0:
            vals.append(m * 2.0 ** -9)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


E4M3_VALUES = _e4m3_values()  # ascending; index == code


def e4m3_decode(codes):
    """E4M3 byte codes (positive, 0..0x7E) -> float64; 0x7F -> NaN."""
    codes = np.asarray(codes, dtype=np.uint8)
    c = codes & 0x7F
    out = E4M3_VALUES[np.minimum(c, 0x7E)]
    out = np.where(c == 0x7F, np.nan, out)
    return np.where(codes & 0x80, -out, out)


def e4m3_encode_pos(v):
    """Non-negative fp32 array -> E4M3 byte codes, RNE ties to even, saturating
    at 448 (0x7E).  Used for block scales, which are never negative."""
    v = np.asarray(v, dtype=np.float32)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("e4m3_encode_pos: negative or NaN input")
    return _nearest_code(v.astype(np.float64), E4M3_VALUES)


def e4m3_encode(v):
    """fp32 array -> signed E4M3 byte codes (the MXFP8 element type): RNE ties
    to even, saturating at +-448, sign bit copied from the input (so -0.0 and
    negatives that round to zero give 0x80)."""
    v = np.asarray(v, dtype=np.float32)
    if np.any(np.isnan(v)):
        raise ValueError("e4m3_encode: NaN input")
    mag = _nearest_code(np.abs(v.astype(np.float64)), E4M3_VALUES)
    sign = np.signbit(v).astype(np.uint8) << 7
    return (mag | sign).astype(np.uint8)


def ue8m0_decode(codes):
    """UE8M0 byte codes -> float64 2^(c-127); 255 -> NaN."""
    codes = np.asarray(codes, dtype=np.int64)
    out = np.ldexp(1.0, codes - 127)
    return np.where(codes == 255, np.nan, out)


def floor_log2_f32(a):
    """Exact floor(log2(a)) of positive fp32 values (subnormals included):
    frexp writes a = m * 2^e with 0.5 <= m < 1 exactly, so floor(log2 a) = e-1."""
    a = np.asarray(a, dtype=np.float32).astype(np.float64)
    if np.any(a <= 0):
        raise ValueError("floor_log2_f32: non-positive input")
    _, e = np.frexp(a)
    return e.astype(np.int64) - 1


def pack_nibbles(codes):
    """[..., 2n] 4-bit codes -> [..., n] bytes; element 2j in the low nibble of
    byte j (the float4_e2m1fn_x2 convention the page names)."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[..., 0::2] & 0xF) | ((codes[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed):
    """[..., n] bytes -> [..., 2n] 4-bit codes (low nibble first)."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def bf16_bits_to_f32(bits):
    """uint16 bf16 bit patterns -> fp32 (exact widening)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f64_to_bf16_rne(x):
    """fp64 -> bf16 bit patterns (uint16) with one round-to-nearest-even step
    taken directly from fp64 (no intermediate fp32 rounding)."""
    x = np.asarray(x, dtype=np.float64)
    # Round to 8 significant bits (bf16 precision) with RNE using frexp.
    m, e = np.frexp(x)  # x = m * 2^e, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)  # 8 significant bits
    r = np.round(scaled)  # numpy rounds half to even
    y = np.ldexp(r, e - 8)
    # bf16 shares fp32's exponent range; below the normal range the bf16 grid
    # is fixed at 2^-133, handle it by rounding on that grid.
    small = np.abs(x) < 2.0 ** -126
    y = np.where(small, np.round(x * 2.0 ** 133) * 2.0 ** -133, y)
    y32 = y.astype(np.float32)  # exact: y already has <= 8 significant bits
    return (y32.view(np.uint32) >> 16).astype(np.uint16)

"""NVFP4 and MXFP4 quantizers, dequantizers and the MXFP4 -> NVFP4 scale remap.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Blocks run along the last (reduction, K) axis: 16 consecutive elements for
NVFP4 ("DeepSeek-V4.1-Flash-NVFP4", §二, group_size 16), 32 for MXFP4 (same
page §三; "DeepSeek-V4 architecture" §6.3, 1x32 tiles).

NVFP4 two-level scaling (same page §二: a block scale brings each group into
[-6, 6], a tensor-level scale sits above it).  The exact rule is the plainest
one consistent with E4M3 block scales (max 448) and E2M1 elements (max 6):

    g    = amax(tensor) / (448 * 6)                    fp32, tensor "decode" scale
    d    = 6 * g                                       fp32
    sf   = E4M3_RNE(amax(block) / d)                   fp32 division, then encode
    s    = dec(sf) * g                                 fp32
    r    = 1 / s   (0 when s == 0)                     fp32
    code = E2M1_RNE(x * r)                             fp32 product, then encode

Every step is one IEEE fp32 operation with round-to-nearest-even, in exactly
this order; numpy float32 array arithmetic is IEEE RN, so the oracle takes
each integer decision (an E4M3 or E2M1 code) in the same precision as the
device.  Dequantization is val(code) * dec(sf) * g in fp64.

MXFP4 (OCP-style shared exponent): per 32-block, X = floor(log2 amax) - 2,
clamped to [-127, 127], scale byte X + 127, code = E2M1_RNE(x * 2^-X); an
all-zero block gets scale byte 0.

MXFP4 -> NVFP4 remap (same page §一 point 2 and §六 convert script: lossless
re-expression of every MX block scale): per tensor, e_max = the largest MX
exponent among blocks holding a nonzero magnitude code; g = 2^(e_max - 8);
each such block with exponent e gets the E4M3 scale 2^(e - e_max + 8) in both
of its 16-element halves (exactly representable while e - e_max + 8 >= -9);
blocks whose codes are all (signed) zeros get scale 0; codes are unchanged.
A tensor whose exponent span would need an E4M3 power below 2^-9 cannot be
remapped losslessly and is reported as a range error.

Lossy-span fallback ("DeepSeek-V4 architecture" §6.3 says the conversion is
lossless only while the ratio of the scale factors stays under a threshold;
it gives no rule beyond it).  Reading: a live block whose exact E4M3 power
2^k would fall below 2^-9 (k < -9) is re-quantized from its dequantized
values, val(c) * 2^e in fp32 (exact), by the NVFP4 rule above at the
tensor's fixed g, one 16-element half at a time.  Every other block is
remapped exactly as in the lossless case.  (Under that rule such a block's
amax_b / (6g) is at most 2^-10, which rounds to the E4M3 code 0: its scales
become 0 and its codes sign|0.)

MXFP8 (the W4A8 activation format: "DeepSeek-V4 FP4 QAT" §4.3 recommends FP8
activations against FP4 weights, and §4.2 keeps the power-of-two block scale
of the MX format).  Reading: the MXFP4 rule above with the E4M3 element
type, whose largest power of two is 2^8: per 32-block X = floor(log2 amax) - 8
clamped to [-127, 127], scale byte X + 127 (0 for an all-zero block),
element = E4M3_RNE_satfinite(x * 2^-X) with the input's sign bit.

FP4 -> FP8 widening (same page §4.2, steps 3-4): every E2M1 value is exactly
an E4M3 value, so each 4-bit code maps to the E4M3 byte of the same value and
the UE8M0 block scales carry over unchanged; nothing is rounded.
"""
import numpy as np

from .formats import (
    e2m1_decode,
    e2m1_encode,
    e4m3_decode,
    e4m3_encode,
    e4m3_encode_pos,
    floor_log2_f32,
    pack_nibbles,
    ue8m0_decode,
    unpack_nibbles,
)

NV_BLOCK = 16
MX_BLOCK = 32
NV_G_DIVISOR = np.float32(448.0 * 6.0)  # 2688


def nv_global_scale(x):
    """g = amax(|x|) / 2688 in fp32 (0 for an all-zero tensor)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    return np.float32(amax / NV_G_DIVISOR)


def nvfp4_quantize(x, g=None):
    """x: fp32 [rows, cols] (bf16 values widened exactly), cols % 16 == 0.
    g: fp32 tensor decode scale; None -> dynamic (nv_global_scale(x)).
    Returns (packed codes uint8 [rows, cols/2], sf uint8 [rows, cols/16], g)."""
    x = np.asarray(x, dtype=np.float32)
    rows, cols = x.shape
    assert cols % NV_BLOCK == 0
    g = nv_global_scale(x) if g is None else np.float32(g)
    xb = x.reshape(rows, cols // NV_BLOCK, NV_BLOCK)
    amax_b = np.max(np.abs(xb), axis=2).astype(np.float32)
    d = np.float32(np.float32(6.0) * g)
    if d == 0:
        sf = np.zeros(amax_b.shape, dtype=np.uint8)
    else:
        with np.errstate(over="ignore"):
            q = (amax_b / d).astype(np.float32)
        q = np.minimum(q, np.float32(np.finfo(np.float32).max))  # inf -> saturates to 448
        sf = e4m3_encode_pos(q)
    s = (e4m3_decode(sf).astype(np.float32) * g).astype(np.float32)
    with np.errstate(divide="ignore"):
        r = np.where(s == 0, np.float32(0), np.float32(1.0) / s).astype(np.float32)
    v = (xb * r[:, :, None]).astype(np.float32)
    codes = e2m1_encode(v).reshape(rows, cols)
    return pack_nibbles(codes), sf, g


def nvfp4_dequantize(packed, sf, g):
    """fp64 [rows, cols] = val(code) * dec(sf) * g."""
    codes = unpack_nibbles(packed)
    rows, cols = codes.shape
    vals = e2m1_decode(codes).reshape(rows, cols // NV_BLOCK, NV_BLOCK)
    scale = e4m3_decode(sf).astype(np.float64) * np.float64(g)
    return (vals * scale[:, :, None]).reshape(rows, cols)


def mxfp4_quantize(x):
    """x: fp32 [rows, cols], cols % 32 == 0.
    Returns (packed codes uint8 [rows, cols/2], UE8M0 scale bytes [rows, cols/32])."""
    x = np.asarray(x, dtype=np.float32)
    rows, cols = x.shape
    assert cols % MX_BLOCK == 0
    xb = x.reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    amax = np.max(np.abs(xb), axis=2)
    zero = amax == 0
    X = np.zeros(amax.shape, dtype=np.int64)
    X[~zero] = floor_log2_f32(amax[~zero]) - 2
    X = np.clip(X, -127, 127)
    scale_codes = np.where(zero, 0, X + 127).astype(np.uint8)
    # x * 2^-X as one fp32 multiply: exact in fp64, then a single RN to fp32.
    # (an all-zero block has X = 0, so v keeps each zero's sign)
    v = np.ldexp(xb.astype(np.float64), -X[:, :, None]).astype(np.float32)
    codes = e2m1_encode(v).reshape(rows, cols)
    return pack_nibbles(codes), scale_codes


def mxfp4_dequantize(packed, scale_codes):
    codes = unpack_nibbles(packed)
    rows, cols = codes.shape
    vals = e2m1_decode(codes).reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    return (vals * ue8m0_decode(scale_codes)[:, :, None]).reshape(rows, cols)


MXFP8_EMAX = 8  # floor(log2(448))


def mxfp8_quantize(x):
    """x: fp32 [rows, cols], cols % 32 == 0.
    Returns (E4M3 codes uint8 [rows, cols], UE8M0 scale bytes [rows, cols/32])."""
    x = np.asarray(x, dtype=np.float32)
    rows, cols = x.shape
    assert cols % MX_BLOCK == 0
    xb = x.reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    amax = np.max(np.abs(xb), axis=2)
    zero = amax == 0
    X = np.zeros(amax.shape, dtype=np.int64)
    X[~zero] = floor_log2_f32(amax[~zero]) - MXFP8_EMAX
    X = np.clip(X, -127, 127)
    scale_codes = np.where(zero, 0, X + 127).astype(np.uint8)
    v = np.ldexp(xb.astype(np.float64), -X[:, :, None]).astype(np.float32)  # one RN to fp32
    return e4m3_encode(v).reshape(rows, cols), scale_codes


def mxfp8_dequantize(codes, scale_codes):
    codes = np.asarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    vals = e4m3_decode(codes).reshape(rows, cols // MX_BLOCK, MX_BLOCK)
    return (vals * ue8m0_decode(scale_codes)[:, :, None]).reshape(rows, cols)


def e2m1_to_e4m3(packed):
    """Packed E2M1 codes [rows, cols/2] -> E4M3 bytes [rows, cols] of the same
    values (sign included): the E4M3 encoding of each decoded E2M1 value."""
    codes = unpack_nibbles(packed)
    return e4m3_encode(e2m1_decode(codes).astype(np.float32))


class RemapRangeError(ValueError):
    """An MX tensor's exponent span is too wide for a lossless E4M3 remap."""


def e4m3_power_of_two(k):
    """E4M3 byte holding exactly 2^k for integer k in [-9, 8]."""
    k = np.asarray(k, dtype=np.int64)
    if np.any(k < -9) or np.any(k > 8):
        raise RemapRangeError("power of two outside E4M3's exact range")
    return np.where(k >= -6, (k + 7) << 3, 1 << np.maximum(k + 9, 0)).astype(np.uint8)


def pow2_f32(e):
    """2^e as an exact fp32 (normal or subnormal), e in [-149, 127]."""
    return np.float32(np.ldexp(1.0, int(e)))


def mx_to_nv(packed, mx_scales, num_tensors=1):
    """Remap MXFP4 block scales to NVFP4 (E4M3 per 16 + fp32 g per tensor).

    packed: uint8 [num_tensors * rows, cols/2]; mx_scales: uint8 [.., cols/32].
    The leading axis is split evenly into ``num_tensors`` tensors.
    Returns (nv_sf uint8 [.., cols/16], g fp32 [num_tensors]).  Codes are
    unchanged (the caller keeps ``packed``).  Raises RemapRangeError."""
    packed = np.asarray(packed, dtype=np.uint8)
    mx_scales = np.asarray(mx_scales, dtype=np.uint8)
    total_rows, half_cols = packed.shape
    cols = half_cols * 2
    assert total_rows % num_tensors == 0
    if np.any(mx_scales == 255):
        raise ValueError("UE8M0 NaN scale in input")
    rows = total_rows // num_tensors
    codes = unpack_nibbles(packed).reshape(total_rows, cols // MX_BLOCK, MX_BLOCK)
    live = np.any((codes & 7) != 0, axis=2)  # a nonzero magnitude in the block
    e = mx_scales.astype(np.int64) - 127
    nv_sf = np.zeros((total_rows, cols // NV_BLOCK), dtype=np.uint8)
    gs = np.zeros(num_tensors, dtype=np.float32)
    for t in range(num_tensors):
        sl = slice(t * rows, (t + 1) * rows)
        lt, et = live[sl], e[sl]
        if not np.any(lt):
            gs[t] = np.float32(0)
            continue
        e_max = int(np.max(et[lt]))
        k = np.where(lt, et - e_max + 8, 0)
        if np.any(k[lt] < -9):
            raise RemapRangeError(f"tensor {t}: exponent span {e_max - int(np.min(et[lt]))} > 17")
        sf_blk = np.where(lt, e4m3_power_of_two(np.clip(k, -9, 8)), 0).astype(np.uint8)
        nv_sf[sl, 0::2] = sf_blk
        nv_sf[sl, 1::2] = sf_blk
        gs[t] = pow2_f32(e_max - 8)
    return nv_sf, gs


def mx_to_nv_lossy(packed, mx_scales, num_tensors=1):
    """MXFP4 -> NVFP4 remap that re-quantizes the blocks below E4M3's range
    (the lossy-span fallback above) instead of refusing the tensor.

    Returns (codes uint8 [.., cols/2], nv_sf uint8 [.., cols/16],
    g fp32 [num_tensors], lossy int64 [num_tensors] = re-quantized 32-blocks).
    A UE8M0 NaN byte is still an error."""
    packed = np.asarray(packed, dtype=np.uint8)
    mx_scales = np.asarray(mx_scales, dtype=np.uint8)
    total_rows, half_cols = packed.shape
    cols = half_cols * 2
    assert total_rows % num_tensors == 0
    if np.any(mx_scales == 255):
        raise ValueError("UE8M0 NaN scale in input")
    rows = total_rows // num_tensors
    codes = unpack_nibbles(packed).reshape(total_rows, cols // MX_BLOCK, MX_BLOCK).copy()
    live = np.any((codes & 7) != 0, axis=2)
    e = mx_scales.astype(np.int64) - 127
    nv_sf = np.zeros((total_rows, cols // NV_BLOCK), dtype=np.uint8)
    gs = np.zeros(num_tensors, dtype=np.float32)
    lossy = np.zeros(num_tensors, dtype=np.int64)
    for t in range(num_tensors):
        r0 = t * rows
        lt = live[r0:r0 + rows]
        if not np.any(lt):
            continue
        e_max = int(np.max(e[r0:r0 + rows][lt]))
        g = pow2_f32(e_max - 8)
        gs[t] = g
        for r in range(r0, r0 + rows):
            for j in range(cols // MX_BLOCK):
                if not live[r, j]:
                    continue
                k = int(e[r, j]) - e_max + 8
                if k >= -9:
                    nv_sf[r, 2 * j] = nv_sf[r, 2 * j + 1] = e4m3_power_of_two(k)
                    continue
                lossy[t] += 1
                # the block's dequantized values (exact in fp32: at least 2^-128 in
                # magnitude when nonzero), re-quantized by the NVFP4 rule at g
                x = (e2m1_decode(codes[r, j]) * np.ldexp(1.0, int(e[r, j]))).astype(np.float32)
                pc, sf, _ = nvfp4_quantize(x.reshape(1, MX_BLOCK), g=g)
                codes[r, j] = unpack_nibbles(pc)[0]
                nv_sf[r, 2 * j:2 * j + 2] = sf[0]
    return pack_nibbles(codes.reshape(total_rows, cols)), nv_sf, gs, lossy

"""W4A4 block-scaled GEMM: dequantize both operands in fp64, then matmul.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

"DeepSeek-V4.1-Flash-NVFP4", §二: the W4A4 product runs on 4-bit operands and
multiplies each block's scale back in the accumulator.  Mathematically that
is exactly  C = (g_a * g_b) * sum_k val(a_ik) dec(sfa) val(b_jk) dec(sfb),
i.e. the product of the two dequantized matrices; the oracle computes that
product in fp64 (numpy matmul is the library step) with A [M,K] and B [N,K]
both stored K-major, C = A_dq @ B_dq^T.

Tolerance for an fp32 result (stated with the workload): elementwise
|C - C_ref| <= 1e-4 * (|A_dq| @ |B_dq|^T)_ij.  A bf16 result must be within
one bf16 ulp of RNE_bf16(C_ref).
"""
import numpy as np

from .quant import mxfp4_dequantize, mxfp8_dequantize, nvfp4_dequantize

FP32_REL_TOL = 1e-4


def nvfp4_gemm_ref(a_packed, a_sf, a_g, b_packed, b_sf, b_g):
    """fp64 C [M, N] and the error-bound matrix |A_dq| @ |B_dq|^T."""
    a = nvfp4_dequantize(a_packed, a_sf, a_g)
    b = nvfp4_dequantize(b_packed, b_sf, b_g)
    return a @ b.T, np.abs(a) @ np.abs(b).T


def mxfp4_gemm_ref(a_packed, a_scales, b_packed, b_scales):
    """MXFP4 x MXFP4 ("DeepSeek-V4.1-Flash-NVFP4" §三: one UE8M0 scale per 32
    elements): fp64 C = A_dq @ B_dq^T and the bound matrix |A_dq| @ |B_dq|^T."""
    a = mxfp4_dequantize(a_packed, a_scales)
    b = mxfp4_dequantize(b_packed, b_scales)
    return a @ b.T, np.abs(a) @ np.abs(b).T


def w4a8_gemm_ref(a_codes, a_scales, b, b_scales, b_is_fp8=False):
    """FP8 x FP4 ("DeepSeek-V4 FP4 QAT" §4.3: FP4 weights against FP8
    activations): A MXFP8 (E4M3 codes [M,K], UE8M0 per 32), B MXFP4 (packed
    [N,K/2], UE8M0 per 32) or, with b_is_fp8, MXFP8 like A.  fp64
    C = A_dq @ B_dq^T and the bound matrix |A_dq| @ |B_dq|^T."""
    a = mxfp8_dequantize(a_codes, a_scales)
    bd = mxfp8_dequantize(b, b_scales) if b_is_fp8 else mxfp4_dequantize(b, b_scales)
    return a @ bd.T, np.abs(a) @ np.abs(bd).T


def bf16_ulp(x_bf16_as_f64):
    """Spacing of the bf16 grid at each (bf16-representable) value."""
    x = np.abs(np.asarray(x_bf16_as_f64, dtype=np.float64))
    _, e = np.frexp(x)
    ulp = np.ldexp(1.0, e - 8)
    return np.where(x < 2.0 ** -126, 2.0 ** -133, ulp)

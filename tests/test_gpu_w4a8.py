"""W4A8 ("DeepSeek-V4 FP4 QAT", §4.2-4.3: FP8 activations against FP4
weights) on tcgen05 kind::mxf8f6f4, against the oracle.

Quantizers and the FP4 -> FP8 widening are bit-exact.  GEMM bars as for the
FP4 GEMMs: fp32 output |C - C_ref| <= 1e-4 * (|A_dq| |B_dq|^T)_ij, bf16
output within 1 ulp of RNE_bf16(C_ref) (or that bound plus one ulp where
cancellation makes it larger); the integer special case is exact."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import layouts as LY
from oracle import quant as Q
from tests._util import bf16_bits, bf16_ulps_apart, f32, tiled_const

pytestmark = pytest.mark.gpu


def _lib():
    import fp4_block_scaled_03_b200 as fp4

    return fp4


def _edge_activations(rows, cols, seed):
    """N(0,1) bf16 with planted edge blocks: all zeros, signed zeros, bf16
    subnormals, an amax a hair below a power of two (the saturating top of the
    E4M3 range), and huge and tiny magnitudes."""
    x = synth.activations_bf16((rows, cols), seed=seed, device="cuda").float()
    if rows >= 4 and cols >= 64:
        x[0, :32] = 0.0
        x[0, 32:64] = -0.0
        x[1, :32] = torch.arange(32, device="cuda") * 2.0 ** -133  # bf16 subnormals
        x[2, :32] = torch.linspace(-1, 1, 32, device="cuda") * 1.99
        x[2, 5] = 1.9921875  # amax -> scaled value 509.9 > 448: saturates
        x[3, :32] *= 2.0 ** 100
        x[3, 32:64] *= 2.0 ** -100
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols,tiled", [(5, 128, False), (130, 384, True), (257, 4096, True), (64, 96, False)])
def test_mxfp8_quantize_bit_exact(rows, cols, tiled):
    fp4 = _lib()
    x = _edge_activations(rows, cols, seed=rows + cols)
    codes, sc = fp4.quantize_mxfp8(x, tiled=tiled)
    rc, rs = Q.mxfp8_quantize(f32(x))
    assert np.array_equal(codes.cpu().numpy(), rc)
    s = sc.cpu().numpy()
    if tiled:
        s = LY.sf_from_mma(s, rows, cols, block=32)
    assert np.array_equal(s, rs)


@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 4096), (1024, 2048)])
def test_e2m1_to_e4m3_bit_exact(rows, cols):
    fp4 = _lib()
    codes = synth.random_codes((rows, cols // 2), seed=rows, device="cuda")
    got = fp4.e2m1_to_e4m3(codes).cpu().numpy()
    assert np.array_equal(got, Q.e2m1_to_e4m3(codes.cpu().numpy()))


def _int_codes(M, K, seed):
    """E4M3 bytes of integers in [-16, 16] (exact in E4M3) and the integers."""
    a_int = np.random.default_rng(seed).integers(-16, 17, (M, K))
    return torch.from_numpy(F.e4m3_encode(a_int.astype(np.float32))).cuda(), a_int


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (200, 264, 384), (300, 520, 1152)])
def test_w4a8_integer_gemm_bit_exact(M, N, K):
    fp4 = _lib()
    a, a_int = _int_codes(M, K, M)
    b = synth.random_codes((N, K // 2), seed=N + 4, device="cuda")
    a_sc = tiled_const(fp4.fp4_sf_tiled_bytes(M, K) // 2, 127)
    b_sc = tiled_const(fp4.fp4_sf_tiled_bytes(N, K) // 2, 127)
    c = fp4.gemm(a, a_sc, None, b, b_sc, None, M, N, K, w4a8=True).cpu().numpy().astype(np.float64)
    b_twice = np.rint(2 * F.e2m1_decode(F.unpack_nibbles(b.cpu().numpy()))).astype(np.int64)
    assert np.array_equal(2 * c, (a_int @ b_twice.T).astype(np.float64))


def _check_bf16(c_bits, C, bound):
    ref_bits = F.f64_to_bf16_rne(C)
    ok = bf16_ulps_apart(c_bits, ref_bits) <= 1
    got = F.bf16_bits_to_f32(c_bits).astype(np.float64)
    ok |= np.abs(got - C) <= G.FP32_REL_TOL * bound + G.bf16_ulp(got)
    return ok


def _operands(M, N, K, seed):
    fp4 = _lib()
    a_bf = _edge_activations(M, K, seed)
    b_bf = synth.weights_bf16((N, K), 0.02, 0.005, 30.0, seed=seed + 1, device="cuda")
    a_c, a_s = fp4.quantize_mxfp8(a_bf, tiled=True)
    b_c, b_s = fp4.quantize_mx(b_bf, tiled=True)
    ra = Q.mxfp8_quantize(f32(a_bf))
    rb = Q.mxfp4_quantize(f32(b_bf))
    return (a_c, a_s, b_c, b_s), ra, rb


@pytest.mark.parametrize("M,N,K,out", [(128, 256, 512, "f32"), (333, 136, 1152, "f32"), (64, 520, 384, "bf16"),
                                       (512, 512, 4096, "bf16"), (1, 8, 128, "f32")])
def test_w4a8_gemm_within_bound(M, N, K, out):
    fp4 = _lib()
    (a_c, a_s, b_c, b_s), ra, rb = _operands(M, N, K, seed=M + N + K)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    c = fp4.gemm(a_c, a_s, None, b_c, b_s, None, M, N, K, out_dtype=dt, w4a8=True)
    C, bound = G.w4a8_gemm_ref(*ra, *rb)
    if out == "f32":
        err = np.abs(c.cpu().numpy().astype(np.float64) - C)
        assert np.all(err <= G.FP32_REL_TOL * bound), float((err / np.maximum(bound, 1e-300)).max())
    else:
        ok = _check_bf16(bf16_bits(c), C, bound)
        assert ok.all(), int((~ok).sum())


@pytest.mark.parametrize("M,N,K", [(256, 512, 1024), (77, 264, 640)])
def test_w4a8_widened_fp8_weights_agree(M, N, K):
    """The same weights run packed (FP4 B, unpacked by TMA) and widened to
    FP8 on the device: both within the bound of the one oracle product (the
    widening is value-exact, so the oracle's two forms are equal)."""
    fp4 = _lib()
    (a_c, a_s, b_c, b_s), ra, rb = _operands(M, N, K, seed=K)
    c4 = fp4.gemm(a_c, a_s, None, b_c, b_s, None, M, N, K, w4a8=True).cpu().numpy().astype(np.float64)
    b8 = fp4.e2m1_to_e4m3(b_c)
    c8 = fp4.gemm(a_c, a_s, None, b8, b_s, None, M, N, K, w4a8=True, b_fp8=True).cpu().numpy().astype(np.float64)
    C, bound = G.w4a8_gemm_ref(*ra, *rb)
    for c in (c4, c8):
        assert np.all(np.abs(c - C) <= G.FP32_REL_TOL * bound)


def test_w4a8_4096_cubed_bf16_sampled():
    """The dense W4A8 GEMM in the bench's launch configuration: activations
    MXFP8-quantized on the device, MXFP4 weights N(0,0.02) + 0.5% x30, bf16
    out; a block of rows and columns checked against the oracle."""
    M = N = K = 4096
    fp4 = _lib()
    a_bf = synth.activations_bf16((M, K), seed=0, device="cuda")
    b_bf = synth.weights_bf16((N, K), 0.02, 0.005, 30.0, seed=1, device="cuda")
    a_c, a_s = fp4.quantize_mxfp8(a_bf, tiled=True)
    b_c, b_s = fp4.quantize_mx(b_bf, tiled=True)
    c = fp4.gemm(a_c, a_s, None, b_c, b_s, None, M, N, K, out_dtype=torch.bfloat16, w4a8=True)
    rows = np.sort(np.random.default_rng(1).choice(M, 96, replace=False))
    cols = np.sort(np.random.default_rng(2).choice(N, 160, replace=False))
    ra = Q.mxfp8_quantize(f32(a_bf)[rows])
    rb = Q.mxfp4_quantize(f32(b_bf)[cols])
    C, bound = G.w4a8_gemm_ref(*ra, *rb)
    ok = _check_bf16(bf16_bits(c)[np.ix_(rows, cols)], C, bound)
    assert ok.all(), int((~ok).sum())

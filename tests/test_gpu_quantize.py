"""GPU quantizers and the MX->NV remap against the oracle: codes, scales and
global scales must match bit for bit."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import layouts as LY
from oracle import quant as Q
from tests._util import f32, f32_bits_equal, np_u8

pytestmark = pytest.mark.gpu


def _lib():
    import fp4_block_scaled_03_b200 as fp4

    return fp4


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (128, 512), (200, 1024), (1000, 7168)])
def test_nv_dynamic_canonical_bit_exact(rows, cols):
    x = synth.activations_bf16((rows, cols), seed=rows * 7 + cols, device="cuda")
    codes, sf, g = _lib().quantize_nv(x)
    rc, rs, rg = Q.nvfp4_quantize(f32(x))
    assert f32_bits_equal(g.cpu().numpy(), [rg])
    assert np.array_equal(np_u8(sf), rs)
    assert np.array_equal(np_u8(codes), rc)


@pytest.mark.parametrize("rows,cols", [(5, 64), (130, 256), (257, 4096)])
def test_nv_tiled_layout_bit_exact(rows, cols):
    x = synth.weights_bf16((rows, cols), 0.02, 0.005, 30.0, seed=11 + rows, device="cuda")
    codes, sf_t, g = _lib().quantize_nv(x, tiled=True)
    rc, rs, rg = Q.nvfp4_quantize(f32(x))
    assert f32_bits_equal(g.cpu().numpy(), [rg])
    assert np.array_equal(np_u8(codes), rc)
    assert np.array_equal(LY.sf_from_mma(np_u8(sf_t), rows, cols), rs)


def test_nv_static_scale_and_exact_ties():
    """Blocks whose scale is a power of two put x*(1/s) exactly on every E2M1
    rounding tie (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) and on +-0 and tiny
    negatives; the device must take the same decisions as the oracle."""
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -0.0]
    rows = []
    for j in range(-8, 9):
        blk = np.array([6.0] + ties, dtype=np.float64) * 2.0**j
        rows.append(blk)
        blk2 = blk.copy()
        blk2[1:4] = [-1e-3 * 2.0**j, 7.0 * 2.0**j, 1.0e-30]  # tiny negative, saturation, tiny positive
        rows.append(blk2)
    x_np = np.stack(rows).astype(np.float32)
    x = torch.from_numpy(x_np).to(torch.bfloat16).cuda()
    g = torch.tensor([1.0], dtype=torch.float32)
    codes, sf, _ = _lib().quantize_nv(x, g=g)
    rc, rs, _ = Q.nvfp4_quantize(f32(x), g=np.float32(1.0))
    assert np.array_equal(np_u8(sf), rs)
    assert np.array_equal(np_u8(codes), rc)
    # and the tie decisions are the reading's (ties to the even code)
    dq = F.e2m1_decode(F.unpack_nibbles(rc))[0::2, 1:8]
    assert np.allclose(dq[8], [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0])  # j = 0 row


def test_nv_zero_tensor():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    x[1] = -0.0
    codes, sf, g = _lib().quantize_nv(x)
    rc, rs, rg = Q.nvfp4_quantize(f32(x))
    assert g.item() == 0.0 and rg == 0
    assert np.array_equal(np_u8(sf), rs) and np.array_equal(np_u8(codes), rc)


def test_nv_full_size_sampled_rows():
    """Pro-shaped activation [16384, 7168] in the launch the bench times:
    dynamic g over the whole tensor, then sampled rows checked exactly."""
    T, H = 16384, 7168
    x = synth.activations_bf16((T, H), seed=3, device="cuda")
    codes, sf, g = _lib().quantize_nv(x)
    xf = f32(x)
    rg = Q.nv_global_scale(xf)
    assert f32_bits_equal(g.cpu().numpy(), [rg])
    rows = np.random.default_rng(0).choice(T, 48, replace=False)
    rows = np.concatenate([rows, [0, T - 1]])
    rc, rs, _ = Q.nvfp4_quantize(xf[rows], g=rg)
    assert np.array_equal(np_u8(codes[torch.from_numpy(rows).cuda()]), rc)
    assert np.array_equal(np_u8(sf[torch.from_numpy(rows).cuda()]), rs)


@pytest.mark.parametrize("rows,cols", [(1, 32), (5, 96), (256, 4096)])
def test_mx_bit_exact(rows, cols):
    x = synth.weights_bf16((rows, cols), 0.02, 0.005, 30.0, seed=rows + cols, device="cuda")
    codes, sc = _lib().quantize_mx(x)
    rc, rs = Q.mxfp4_quantize(f32(x))
    assert np.array_equal(np_u8(sc), rs)
    assert np.array_equal(np_u8(codes), rc)


def test_mx_extreme_exponents():
    base = synth.activations_bf16((8, 64), seed=5, device="cuda").float()
    scale = torch.tensor([2.0**-130, 2.0**-126, 2.0**-100, 1.0, 2.0**60, 2.0**120, 2.0**126, 0.0],
                         device="cuda")[:, None]
    x = (base * scale).to(torch.bfloat16)
    codes, sc = _lib().quantize_mx(x)
    rc, rs = Q.mxfp4_quantize(f32(x))
    assert np.array_equal(np_u8(sc), rs)
    assert np.array_equal(np_u8(codes), rc)


def test_remap_bit_exact_and_lossless():
    nt, rows, cols = 4, 64, 256
    w = synth.weights_bf16((nt * rows, cols), 0.02, 0.005, 30.0, seed=9, device="cuda")
    w[: rows] *= 64  # tensor 0 has its own range
    codes, sc = _lib().quantize_mx(w)
    nv, g = _lib().mx_to_nv(codes, sc, nt)
    rc, rs = Q.mxfp4_quantize(f32(w))
    rnv, rg = Q.mx_to_nv(rc, rs, nt)
    assert np.array_equal(np_u8(nv), rnv)
    assert f32_bits_equal(g.cpu().numpy(), rg)
    for t in range(nt):
        sl = slice(t * rows, (t + 1) * rows)
        assert np.array_equal(Q.mxfp4_dequantize(rc[sl], rs[sl]), Q.nvfp4_dequantize(rc[sl], np_u8(nv)[sl], rg[t]))


def test_remap_refuses_wide_span():
    fp4 = _lib()
    rows, cols = 4, 64
    codes = torch.full((2 * rows, cols // 2), 0x11, dtype=torch.uint8, device="cuda")
    sc = torch.full((2 * rows, cols // 32), 127, dtype=torch.uint8, device="cuda")
    sc[rows + 1, 0] = 127 - 18  # tensor 1 spans 18 octaves
    nv = torch.full((2 * rows, cols // 16), 0xAB, dtype=torch.uint8, device="cuda")
    g = torch.empty(2, dtype=torch.float32, device="cuda")
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.fp4_mx_to_nv(codes, sc, rows, cols, 2, nv, g)
    assert ei.value.code == 4
    gh = g.cpu().numpy()
    assert gh[0] == np.float32(2.0**-8) and np.isnan(gh[1])
    assert torch.all(nv[rows:] == 0xAB)  # the refused tensor's scales are untouched
    assert fp4.fp4_get_device_status() == 0


def test_remap_tiled_layout():
    nt, rows, cols = 3, 64, 192  # rows not a multiple of 128: each tensor padded on its own
    w = synth.weights_bf16((nt * rows, cols), 0.02, 0.005, 30.0, seed=12, device="cuda")
    codes, sc = _lib().quantize_mx(w)
    nv_t, g = _lib().mx_to_nv(codes, sc, nt, tiled=True)
    rc, rs = Q.mxfp4_quantize(f32(w))
    rnv, rg = Q.mx_to_nv(rc, rs, nt)
    tb = _lib().fp4_sf_tiled_bytes(rows, cols)
    for t in range(nt):
        got = LY.sf_from_mma(np_u8(nv_t[t * tb:(t + 1) * tb]), rows, cols)
        assert np.array_equal(got, rnv[t * rows:(t + 1) * rows])
    assert f32_bits_equal(g.cpu().numpy(), rg)


def _wide_span_mx(nt, rows, cols, seed):
    """MX codes and UE8M0 scales whose tensors span far more than 17 octaves
    (tensor 1 stays inside the lossless span), with some dead blocks."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (nt * rows, cols // 2), dtype=np.uint8)
    e = rng.integers(-90, 40, (nt * rows, cols // 32))
    e[rows:2 * rows] = rng.integers(-6, 8, (rows, cols // 32))
    dead = rng.random((nt * rows, cols // 32)) < 0.05
    for r, j in zip(*np.nonzero(dead)):
        codes[r, 16 * j:16 * j + 16] = 0x88 if (r + j) % 2 else 0x00  # signed zeros only
    return codes, (e + 127).astype(np.uint8)


@pytest.mark.parametrize("tiled", [False, True])
@pytest.mark.parametrize("inplace", [False, True])
def test_remap_lossy_bit_exact(tiled, inplace):
    """fp4_mx_to_nv_codes with FP4_MX2NV_ALLOW_LOSSY: codes, scales, globals
    and re-quantized block counts equal the oracle's lossy remap bit for bit
    (several tensors, rows not a multiple of 128, spans up to 129 octaves)."""
    fp4 = _lib()
    nt, rows, cols = 3, 96, 192
    codes, sc = _wide_span_mx(nt, rows, cols, seed=11 + 2 * tiled + inplace)
    c_d = torch.from_numpy(codes.copy()).cuda()
    s_d = torch.from_numpy(sc).cuda()
    oc, nv, g, lossy = fp4.mx_to_nv_codes(c_d, s_d, nt, tiled=tiled, allow_lossy=True,
                                          out_codes=c_d if inplace else None)
    rc, rsf, rg, rl = Q.mx_to_nv_lossy(codes, sc, nt)
    assert np.array_equal(np_u8(oc), rc)
    if inplace:
        assert oc.data_ptr() == c_d.data_ptr()
    if tiled:
        tb = fp4.fp4_sf_tiled_bytes(rows, cols)
        for t in range(nt):
            got = LY.sf_from_mma(np_u8(nv[t * tb:(t + 1) * tb]), rows, cols)
            assert np.array_equal(got, rsf[t * rows:(t + 1) * rows])
    else:
        assert np.array_equal(np_u8(nv), rsf)
    assert f32_bits_equal(g.cpu().numpy(), rg)
    assert np.array_equal(lossy.cpu().numpy(), rl)
    assert rl[0] > 0 and rl[1] == 0 and rl[2] > 0
    assert fp4.fp4_get_device_status() == 0


def test_remap_codes_without_lossy_flag_matches_lossless_remap():
    """Without the flag, fp4_mx_to_nv_codes is fp4_mx_to_nv plus a code copy:
    the wide tensors are refused (FP4_ERR_RANGE, NaN global, codes and scales
    untouched) and the tensor inside the span is remapped exactly."""
    fp4 = _lib()
    nt, rows, cols = 3, 64, 128
    codes, sc = _wide_span_mx(nt, rows, cols, seed=5)
    c_d = torch.from_numpy(codes).cuda()
    s_d = torch.from_numpy(sc).cuda()
    oc = torch.full_like(c_d, 0x5A)
    nv = torch.full((nt * rows, cols // 16), 0xAB, dtype=torch.uint8, device="cuda")
    g = torch.empty(nt, dtype=torch.float32, device="cuda")
    lossy = torch.full((nt,), -1, dtype=torch.int64, device="cuda")
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.fp4_mx_to_nv_codes(c_d, s_d, rows, cols, nt, oc, nv, g, lossy, 0)
    assert ei.value.code == 4
    gh = g.cpu().numpy()
    assert np.isnan(gh[0]) and np.isnan(gh[2])
    sl = slice(rows, 2 * rows)
    rnv, rg = Q.mx_to_nv(codes[sl], sc[sl], 1)
    assert np.array_equal(np_u8(nv[sl]), rnv) and f32_bits_equal(gh[1:2], rg)
    assert np.array_equal(np_u8(oc[sl]), codes[sl])
    assert torch.all(oc[:rows] == 0x5A) and torch.all(nv[:rows] == 0xAB)
    assert lossy.cpu().tolist() == [0, 0, 0]
    assert fp4.fp4_get_device_status() == 0


def test_remap_lossy_still_refuses_nan_scale():
    fp4 = _lib()
    rows, cols = 4, 64
    c_d = torch.full((2 * rows, cols // 2), 0x11, dtype=torch.uint8, device="cuda")
    s_d = torch.full((2 * rows, cols // 32), 127, dtype=torch.uint8, device="cuda")
    s_d[rows, 1] = 255
    oc = torch.empty_like(c_d)
    nv = torch.empty((2 * rows, cols // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(2, dtype=torch.float32, device="cuda")
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.fp4_mx_to_nv_codes(c_d, s_d, rows, cols, 2, oc, nv, g, None, fp4.FP4_MX2NV_ALLOW_LOSSY)
    assert ei.value.code == 4
    gh = g.cpu().numpy()
    assert gh[0] == np.float32(2.0**-8) and np.isnan(gh[1])

"""The MoE layer at the benchmark's full sizes, in the launch configuration
bench.py times, checked against the oracle on sampled tokens.

The layer is built exactly as the bench builds it (per-expert seeded weights,
calibrated h scales); the oracle regenerates only the sampled tokens' experts
from the same seeds, quantizes them itself, and computes those tokens'
outputs in fp64.  Bar: within 1 bf16 ulp, plus the w2 GEMM bound, the
combine's fp32-sum bound, and what rounding decisions inside the w13 error
band can move (as in test_gpu_moe.test_layer_end_to_end)."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import gemm as G
from oracle import moe as MO
from oracle import quant as Q
from tests import moe_case
from tests._util import bf16_bits, bf16_ulps_apart

pytestmark = pytest.mark.gpu


def _h_tol(xr, w1, w3, gate, up, h):
    bg = np.abs(xr) @ np.abs(w1).T
    bu = np.abs(xr) @ np.abs(w3).T
    return 1.1 * G.FP32_REL_TOL * bg * np.abs(up) + np.abs(MO.silu(gate)) * G.FP32_REL_TOL * bu + \
        4e-7 * np.abs(h) + 1e-30


@pytest.mark.parametrize("workload,tokens", [("pro", [0, 9999]), ("decode", [63]), ("flash", [17]), ("flashmx", [5]),
                                             ("flashw4a8", [2049]), ("pro128k", [131071])])
def test_layer_full_size_sampled_tokens(workload, tokens):
    import bench

    b = bench.MoeBench(workload, seed=0)
    b.step()
    torch.cuda.synchronize()
    assert b.fp4.fp4_get_device_status() == 0
    T, H, I, E, k, zipf, sigma, _ = bench.WORKLOADS[workload]
    xf = b.x.float().cpu().numpy()
    if b.w4a8:
        x_dq = Q.mxfp8_dequantize(*Q.mxfp8_quantize(xf[tokens]))
    elif b.mx:
        x_dq = Q.mxfp4_dequantize(*Q.mxfp4_quantize(xf[tokens]))
    else:
        g = Q.nv_global_scale(xf)
        x_dq = Q.nvfp4_dequantize(*Q.nvfp4_quantize(xf[tokens], g=g))
    ids = b.ids.cpu().numpy()[tokens]
    wts = b.w.cpu().numpy()[tokens].astype(np.float64)
    hg = b.h_g.cpu().numpy()

    def oracle_weights(e):
        w13 = synth.weights_bf16((2 * I, H), sigma, 0.005, 30.0, seed=1000 * 2 + e, device="cuda").float().cpu().numpy()
        w2 = synth.weights_bf16((H, I), sigma, 0.005, 30.0, seed=1000 * 3 + e, device="cuda").float().cpu().numpy()
        if b.mx:
            d13, d2 = Q.mxfp4_dequantize(*Q.mxfp4_quantize(w13)), Q.mxfp4_dequantize(*Q.mxfp4_quantize(w2))
        elif workload == "flash":  # MX weights remapped to NVFP4 (lossless)
            def via_remap(w):
                c, sc = Q.mxfp4_quantize(w)
                nv, gg = Q.mx_to_nv(c, sc, 1)
                return Q.nvfp4_dequantize(c, nv, gg[0])
            d13, d2 = via_remap(w13), via_remap(w2)
        else:
            d13, d2 = Q.nvfp4_dequantize(*Q.nvfp4_quantize(w13)), Q.nvfp4_dequantize(*Q.nvfp4_quantize(w2))
        w1, w3 = MO.deinterleave_w13(d13)
        return (w1, w3, d2)

    cache = {}
    experts_w = [[cache.setdefault(int(e), oracle_weights(int(e))) for e in row] for row in ids]
    g_h = None if b.mx else [[hg[int(e)] for e in row] for row in ids]
    fmt = "w4a8" if b.w4a8 else "mx" if b.mx else "nv"
    ref, slack, sum_abs = moe_case.oracle_token_rows(x_dq, experts_w, wts, g_h, fmt, _h_tol)
    got_bits = bf16_bits(b.out)[tokens]
    got = F.bf16_bits_to_f32(got_bits).astype(np.float64)
    ulps = bf16_ulps_apart(got_bits, F.f64_to_bf16_rne(ref))
    ok = (ulps <= 1) | (np.abs(got - ref) <= G.bf16_ulp(np.abs(ref)) + slack + k * 2.0**-24 * sum_abs)
    assert ok.all(), int((~ok).sum())
    print(f"{workload}: {float((ulps <= 1).mean()):.5f} of sampled outputs within 1 bf16 ulp")

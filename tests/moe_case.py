"""Builds one seeded MoE test case on the GPU (through the library) and its
oracle mirror on the host (through oracle/ only, from the same bf16 inputs).

Weights: w13 [E, 2I, H] bf16 drawn directly in the fused order (rows 32j..32j+15
are gate rows, 32j+16..32j+31 up rows), w2 [E, H, I]; each expert's matrix is
NVFP4-quantized with its own dynamic tensor scale (NV) or MXFP4-quantized and
remapped (MX)."""
import numpy as np
import torch

import synth
from oracle import moe as MO
from oracle import quant as Q
from tests._util import f32


class Case:
    pass


def build(T, H, I, E, k, seed=0, zipf=0.0, h_g=1e-3, w_sigma=0.02, w_frac=0.005, w_factor=30.0, fmt="nv",
          oracle_experts=None, counts=None):
    import fp4_block_scaled_03_b200 as fp4

    c = Case()
    c.T, c.H, c.I, c.E, c.k = T, H, I, E, k
    dev = "cuda"
    c.x = synth.activations_bf16((T, H), seed=seed, device=dev)
    if counts is not None:  # prescribed top-1 routing
        assert k == 1 and len(counts) == E and sum(counts) == T
        c.ids, c.w, c.counts = synth.router_fixed_counts(counts, seed=seed + 1, device=dev)
    else:
        c.ids, c.w, c.counts = synth.router(T, E, k, seed=seed + 1, zipf_s=zipf, device=dev)
    w13 = synth.weights_bf16((E * 2 * I, H), w_sigma, w_frac, w_factor, seed=seed + 2, device=dev)
    w2 = synth.weights_bf16((E * H, I), w_sigma, w_frac, w_factor, seed=seed + 3, device=dev)
    c.w13_codes = torch.empty((E * 2 * I, H // 2), dtype=torch.uint8, device=dev)
    c.w2_codes = torch.empty((E * H, I // 2), dtype=torch.uint8, device=dev)
    div = 2 if fmt in ("mx", "w4a8") else 1  # MX: one scale per 32 elements
    c.fmt = fmt
    c.w13_sf = torch.empty(fp4.fp4_sf_tiled_bytes(E * 2 * I, H) // div, dtype=torch.uint8, device=dev)
    c.w2_sf = torch.empty(fp4.fp4_sf_tiled_bytes(E * H, I) // div, dtype=torch.uint8, device=dev)
    c.w13_g = torch.empty(E, dtype=torch.float32, device=dev)
    c.w2_g = torch.empty(E, dtype=torch.float32, device=dev)
    s13 = fp4.fp4_sf_tiled_bytes(2 * I, H) // div
    s2 = fp4.fp4_sf_tiled_bytes(H, I) // div
    for e in range(E):
        for (wb, codes, sf, g, rows, cols, sfb) in ((w13, c.w13_codes, c.w13_sf, c.w13_g, 2 * I, H, s13),
                                                     (w2, c.w2_codes, c.w2_sf, c.w2_g, H, I, s2)):
            sl = slice(e * rows, (e + 1) * rows)
            if fmt == "nv":
                cc, ss, gg = fp4.quantize_nv(wb[sl], tiled=True)
                codes[sl] = cc
                sf[e * sfb:(e + 1) * sfb] = ss
                g[e] = gg[0]
            elif fmt in ("mx", "w4a8"):  # MXFP4 weights (w4a8: with MXFP8 activations)
                cc, ss = fp4.quantize_mx(wb[sl], tiled=True)
                codes[sl] = cc
                sf[e * sfb:(e + 1) * sfb] = ss
                g[e] = 1.0
            else:
                raise ValueError(fmt)
    c.h_g = torch.full((E,), h_g, dtype=torch.float32, device=dev)
    c.weights = fp4.MoeWeightSet(c.w13_codes, c.w13_sf, c.w13_g, c.w2_codes, c.w2_sf, c.w2_g, c.h_g)
    # host copies for the oracle
    c.x_f32 = f32(c.x)
    c.ids_np = c.ids.cpu().numpy()
    c.w_np = c.w.cpu().numpy()
    c.w13_bf = w13
    c.w2_bf = w2
    c.h_g_np = np.full(E, np.float32(h_g), dtype=np.float32)
    return c


def oracle_expert_weights(c, e):
    """Dequantized fp64 (W1 [I,H], W3 [I,H], W2 [H,I]) of expert e, quantized
    by the oracle from the same bf16 weights."""
    I, H = c.I, c.H
    w13 = f32(c.w13_bf[e * 2 * I:(e + 1) * 2 * I])
    w2 = f32(c.w2_bf[e * H:(e + 1) * H])
    if getattr(c, "fmt", "nv") in ("mx", "w4a8"):
        q13, q2 = Q.mxfp4_quantize(w13), Q.mxfp4_quantize(w2)
        w1, w3 = MO.deinterleave_w13(Q.mxfp4_dequantize(*q13))
        return w1, w3, Q.mxfp4_dequantize(*q2), q13, q2
    q13 = Q.nvfp4_quantize(w13)
    q2 = Q.nvfp4_quantize(w2)
    d13 = Q.nvfp4_dequantize(*q13)
    w1, w3 = MO.deinterleave_w13(d13)
    return w1, w3, Q.nvfp4_dequantize(*q2), q13, q2


def oracle_x(c):
    if getattr(c, "fmt", "nv") == "w4a8":
        xq = Q.mxfp8_quantize(c.x_f32)
        return xq, Q.mxfp8_dequantize(*xq)
    if getattr(c, "fmt", "nv") == "mx":
        xq = Q.mxfp4_quantize(c.x_f32)
        return xq, Q.mxfp4_dequantize(*xq)
    xq = Q.nvfp4_quantize(c.x_f32)
    return xq, Q.nvfp4_dequantize(*xq)


def oracle_token_rows(x_dq_rows, experts_w, slot_weights, g_h, fmt, h_tol_fn):
    """Oracle output rows of a few tokens and the per-element slack the
    layer bar allows (see test_gpu_moe.test_layer_end_to_end).

    x_dq_rows: fp64 [n, H]; experts_w: per token, a list of k (w1, w3, w2)
    dequantized fp64 matrices; slot_weights: fp64 [n, k]; g_h: per token, a
    list of k h tensor scales (NV) or None (MX)."""
    from oracle import formats as F
    from oracle import gemm as G

    n, H = x_dq_rows.shape
    ref = np.zeros((n, H))
    slack = np.zeros((n, H))
    sum_abs = np.zeros((n, H))
    for t in range(n):
        for s, (w1, w3, w2) in enumerate(experts_w[t]):
            xr = x_dq_rows[t:t + 1]
            gate, up = xr @ w1.T, xr @ w3.T
            h = MO.swiglu(gate, up)
            tol = h_tol_fn(xr, w1, w3, gate, up, h)
            blk = 32 if fmt in ("mx", "w4a8") else 16
            if fmt == "w4a8":  # MXFP8 h: one E4M3 byte per element, magnitude in bits 0-6
                hc, hs = Q.mxfp8_quantize(h.astype(np.float32))
                h_dq = Q.mxfp8_dequantize(hc, hs)
                lo_c, lo_s = Q.mxfp8_quantize((h - tol).astype(np.float32))
                hi_c, hi_s = Q.mxfp8_quantize((h + tol).astype(np.float32))
                mid = hc & 0x7F
                unstable = ~((lo_s == hs) & (hi_s == hs) & ((lo_c & 0x7F) == mid).reshape(1, -1, blk).all(2) &
                             ((hi_c & 0x7F) == mid).reshape(1, -1, blk).all(2))
                # a different decision in the band moves an element by at most the
                # block's largest coded magnitude: 448 x 2^X <= 2 amax
                amax_hi = (np.abs(h) + tol).reshape(1, -1, blk).max(2)
                dh = np.repeat(np.where(unstable, 2.0 * amax_hi, 0.0), blk, axis=1)
                wt = float(slot_weights[t, s])
                y = wt * (h_dq @ w2.T)
                ref[t] += y[0]
                sum_abs[t] += np.abs(y[0])
                slack[t] += (abs(wt) * (dh @ np.abs(w2).T) + G.FP32_REL_TOL * abs(wt) * (np.abs(h_dq) @ np.abs(w2).T))[0]
                continue
            if fmt == "mx":
                hc, hs = Q.mxfp4_quantize(h.astype(np.float32))
                h_dq = Q.mxfp4_dequantize(hc, hs)
                q = lambda v: Q.mxfp4_quantize(v)  # noqa: E731
            else:
                g = np.float32(g_h[t][s])
                hc, hs, _ = Q.nvfp4_quantize(h.astype(np.float32), g=g)
                h_dq = Q.nvfp4_dequantize(hc, hs, g)
                q = lambda v: Q.nvfp4_quantize(v, g=g)[:2]  # noqa: E731
            lo_c, lo_s = q((h - tol).astype(np.float32))
            hi_c, hi_s = q((h + tol).astype(np.float32))
            mid = F.unpack_nibbles(hc) & 7
            unstable = ~((lo_s == hs) & (hi_s == hs) &
                         ((F.unpack_nibbles(lo_c) & 7) == mid).reshape(1, -1, blk).all(2) &
                         ((F.unpack_nibbles(hi_c) & 7) == mid).reshape(1, -1, blk).all(2))
            # largest magnitude a band value can be coded with: 6 x the next scale up
            amax_hi = (np.abs(h) + tol).reshape(1, -1, blk).max(2)
            step = np.where(unstable, 12.0 * 2.0 * amax_hi, 0.0)
            dh = np.repeat(step, blk, axis=1)
            wt = float(slot_weights[t, s])
            y = wt * (h_dq @ w2.T)
            ref[t] += y[0]
            sum_abs[t] += np.abs(y[0])
            slack[t] += (abs(wt) * (dh @ np.abs(w2).T) + G.FP32_REL_TOL * abs(wt) * (np.abs(h_dq) @ np.abs(w2).T))[0]
    return ref, slack, sum_abs

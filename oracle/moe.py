"""Routed-expert MoE layer: dispatch, W4A4 expert FFN (w1/w3 -> SwiGLU ->
re-quantize -> w2), combine.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Pins: the pages print no worked example of an expert or a layer.
expert_ffn_ref, expert_ffn_ref_mx and expert_ffn_ref_w4a8 are pinned by a
case worked by hand (tests/golden/expert_ffn_hand.txt): gates of +-100 (or
+-128) make SiLU exact in fp64 and every re-quantization lossless, so y is
a sum of small integers.  route, topk_softmax and combine_ref are pinned by
a library stable sort, brute force and hand-worked sums.

Sources: "DeepSeek-V4 FP4 QAT" page §3.1 (simplified MoE forward: each token
goes to its top-k experts, the expert outputs are summed); "DeepSeek-V4
architecture" §2.1 (Pro: 384 routed experts, 6 active) and §5.1 (SwiGLU
feed-forward layers); "DeepSeek-V4.1-Flash-NVFP4" §三 (the quantized experts'
three projections w1, w2, w3) and §一 point 3 (W4A4: activations are 4-bit
too, so the intermediate is re-quantized before w2).

Readings where the pages are silent (restated with the oracle so a reader can
check them here): h = silu(x W1^T) * (x W3^T) with silu(z) = z / (1 + e^-z);
the activation x is NVFP4-quantized with a dynamic per-call tensor scale; h
is NVFP4-quantized with a static per-expert scale g_h[e] supplied by the
caller; routed rows are ordered by (expert, token, slot) (a stable sort of
the flattened expert ids); the combine weights each slot's output by the
caller's top-k weight (1.0 when none is given) and sums slots in order 0..k-1.
"""
import numpy as np

from .formats import f64_to_bf16_rne
from .quant import (mxfp4_dequantize, mxfp4_quantize, mxfp8_dequantize, mxfp8_quantize, nvfp4_dequantize,
                    nvfp4_quantize)


def route(expert_ids, num_experts):
    """expert_ids int [T, k] -> (counts [E], offsets [E+1], perm [R], inv [T, k]).

    perm[r] is the flat index t*k+s of the r-th routed row in (expert, t, s)
    order; inv[t, s] is the row that slot s of token t went to.  Raises on ids
    outside [0, E)."""
    ids = np.asarray(expert_ids, dtype=np.int64)
    T, k = ids.shape
    flat = ids.reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= num_experts):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=num_experts).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    perm = np.argsort(flat, kind="stable").astype(np.int64)
    inv = np.empty(flat.size, dtype=np.int64)
    inv[perm] = np.arange(flat.size)
    return counts, offsets, perm, inv.reshape(T, k)


def topk_softmax(logits, k):
    """Router top-k ("DeepSeek-V4 FP4 QAT" §3.1: each token picks its top-k
    experts): expert ids = the k largest logits, ties to the lower expert id
    (a stable sort of -logits); weights = softmax over the k chosen logits,
    in fp64.  logits fp32 [T, E] -> (ids int64 [T, k], weights fp64 [T, k])."""
    z = np.asarray(logits, dtype=np.float32).astype(np.float64)
    order = np.argsort(-z, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(z, order, axis=1)
    e = np.exp(sel - sel[:, :1])
    return order.astype(np.int64), e / e.sum(axis=1, keepdims=True)


def silu(z):
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def swiglu(gate, up):
    return silu(gate) * up


def expert_ffn_ref(x_dq_rows, w1_dq, w3_dq, w2_dq, g_h):
    """One expert on a set of dequantized activation rows (fp64 [n, H]).

    Returns dict with gate, up, h (fp64), the NVFP4 codes/scales of h (taken
    from h rounded once to fp32, the precision the re-quantizer works in), the
    dequantized h and y = h_dq @ W2^T (fp64)."""
    gate = x_dq_rows @ w1_dq.T
    up = x_dq_rows @ w3_dq.T
    h = swiglu(gate, up)
    h_codes, h_sf, _ = nvfp4_quantize(h.astype(np.float32), g=g_h)
    h_dq = nvfp4_dequantize(h_codes, h_sf, g_h)
    y = h_dq @ w2_dq.T
    return dict(gate=gate, up=up, h=h, h_codes=h_codes, h_sf=h_sf, h_dq=h_dq, y=y)


def expert_ffn_ref_mx(x_dq_rows, w1_dq, w3_dq, w2_dq):
    """MXFP4 variant of expert_ffn_ref: h is re-quantized to MXFP4 (one
    power-of-two scale per 32 elements, no tensor scale) from h rounded once
    to fp32."""
    gate = x_dq_rows @ w1_dq.T
    up = x_dq_rows @ w3_dq.T
    h = swiglu(gate, up)
    h_codes, h_sc = mxfp4_quantize(h.astype(np.float32))
    h_dq = mxfp4_dequantize(h_codes, h_sc)
    y = h_dq @ w2_dq.T
    return dict(gate=gate, up=up, h=h, h_codes=h_codes, h_sc=h_sc, h_dq=h_dq, y=y)


def expert_ffn_ref_w4a8(x_dq_rows, w1_dq, w3_dq, w2_dq):
    """W4A8 variant ("DeepSeek-V4 FP4 QAT" §4.3: FP8 activations, FP4
    weights): x_dq_rows are the dequantized MXFP8 activations, the weights
    dequantized MXFP4; h is re-quantized to MXFP8 (E4M3 elements, one
    power-of-two scale per 32) from h rounded once to fp32."""
    gate = x_dq_rows @ w1_dq.T
    up = x_dq_rows @ w3_dq.T
    h = swiglu(gate, up)
    h_codes, h_sc = mxfp8_quantize(h.astype(np.float32))
    h_dq = mxfp8_dequantize(h_codes, h_sc)
    y = h_dq @ w2_dq.T
    return dict(gate=gate, up=up, h=h, h_codes=h_codes, h_sc=h_sc, h_dq=h_dq, y=y)


def combine_ref(y_rows, inv, topk_weights=None):
    """out[t] = sum_s w[t,s] * y[inv[t,s]] in fp64, then one RNE to bf16.
    Returns (fp64 sum, bf16 bit patterns)."""
    y_rows = np.asarray(y_rows, dtype=np.float64)
    T, k = inv.shape
    w = np.ones((T, k)) if topk_weights is None else np.asarray(topk_weights, dtype=np.float64)
    out = np.zeros((T, y_rows.shape[1]), dtype=np.float64)
    for s in range(k):
        out += w[:, s : s + 1] * y_rows[inv[:, s]]
    return out, f64_to_bf16_rne(out)


def interleave_w13(w1, w3, group=16):
    """Stack gate (w1) and up (w3) rows [I, H] into one [2I, H] matrix whose
    rows alternate 16 gate rows, 16 up rows (the fused w13 operand order)."""
    I, H = w1.shape
    assert I % group == 0
    out = np.empty((2 * I, H), dtype=w1.dtype)
    v = out.reshape(I // group, 2, group, H)
    v[:, 0] = w1.reshape(I // group, group, H)
    v[:, 1] = w3.reshape(I // group, group, H)
    return out


def deinterleave_w13(w13, group=16):
    """Inverse of interleave_w13: [2I, H] -> (w1 [I, H], w3 [I, H])."""
    two_i, H = w13.shape
    I = two_i // 2
    v = w13.reshape(I // group, 2, group, H)
    return v[:, 0].reshape(I, H), v[:, 1].reshape(I, H)

"""Router ("DeepSeek-V4 FP4 QAT" §3.1: tokens go to their top-k experts;
"DeepSeek-V4 architecture" §2.1: top-6 of 384): the bf16 gate GEMM on tcgen05
kind::f16 and the fused gate + top-k call, against the oracle.

bf16 GEMM: exact for small integers; otherwise |C - C_ref| <= 1e-4 *
(|A| |B|^T)_ij.  Router: logits within that bound of the fp64 oracle; the
expert choice is an integer decision made on the logits, so it is checked
bit-exactly against the oracle's top-k applied to the same fp32 logits the
device produced, and the weights within 2e-6 relative (fp32 softmax)."""
import numpy as np
import pytest
import torch

import synth
from oracle import gemm as G
from oracle import moe as MO

pytestmark = pytest.mark.gpu


def _lib():
    import fp4_block_scaled_03_b200 as fp4

    return fp4


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 264, 320), (1, 8, 128)])
def test_gemm_bf16_integer_exact(M, N, K):
    rng = np.random.default_rng(M + N)
    a = rng.integers(-8, 9, (M, K))
    b = rng.integers(-8, 9, (N, K))
    at = torch.from_numpy(a).to(torch.bfloat16).cuda()
    bt = torch.from_numpy(b).to(torch.bfloat16).cuda()
    c = _lib().gemm_bf16(at, bt).cpu().numpy().astype(np.float64)
    assert np.array_equal(c, (a @ b.T).astype(np.float64))


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (333, 136, 1088), (1000, 384, 7168)])
def test_gemm_bf16_within_bound(M, N, K):
    a = synth.activations_bf16((M, K), seed=M, device="cuda")
    b = synth.weights_bf16((N, K), 0.02, 0.005, 30.0, seed=N, device="cuda")
    c = _lib().gemm_bf16(a, b).cpu().numpy().astype(np.float64)
    af, bf = a.double().cpu().numpy(), b.double().cpu().numpy()
    C, bound = af @ bf.T, np.abs(af) @ np.abs(bf).T
    err = np.abs(c - C)
    assert np.all(err <= G.FP32_REL_TOL * bound), float((err / np.maximum(bound, 1e-300)).max())


@pytest.mark.parametrize("T,H,E,k", [(1000, 1024, 64, 6), (300, 7168, 384, 6), (7, 512, 8, 2)])
def test_router_gate_and_topk(T, H, E, k):
    fp4 = _lib()
    x = synth.activations_bf16((T, H), seed=T, device="cuda")
    wg = synth.weights_bf16((E, H), 0.02, 0.0, 1.0, seed=E, device="cuda")
    logits, ids, w = fp4.router(x, wg, k)
    assert fp4.fp4_get_device_status() == 0
    xf, wf = x.double().cpu().numpy(), wg.double().cpu().numpy()
    L, bound = xf @ wf.T, np.abs(xf) @ np.abs(wf).T
    lg = logits.cpu().numpy()
    assert np.all(np.abs(lg.astype(np.float64) - L) <= G.FP32_REL_TOL * bound)
    rid, rw = MO.topk_softmax(lg, k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=0)
    # and the choice is a top-k of the exact logits up to the GEMM bound
    for t in range(T):
        sel = set(rid[t].tolist())
        rest = [e for e in range(E) if e not in sel]
        if rest:
            tol = 2 * G.FP32_REL_TOL * bound[t].max()
            assert min(L[t, list(sel)]) >= max(L[t, rest]) - tol


@pytest.mark.parametrize("T,H,E,k", [(16384, 1024, 384, 6), (3000, 512, 64, 8), (100, 512, 64, 6), (0, 512, 64, 6)])
def test_router_route_fused_equals_router_then_route(T, H, E, k):
    """fp4_moe_router_route (the routing's count pass done by the top-k
    kernel) gives the same ids, weights, logits and routing tables, bit for
    bit, as fp4_moe_router followed by fp4_moe_route."""
    fp4 = _lib()
    x = synth.activations_bf16((max(T, 1), H), seed=T + 1, device="cuda")[:T]
    wg = synth.weights_bf16((E, H), 0.02, 0.0, 1.0, seed=E + 2, device="cuda")
    R = T * k
    scratch = torch.empty(max(fp4.fp4_moe_route_scratch_bytes(R, E), 4), dtype=torch.uint8, device="cuda")

    def tables():
        return dict(logits=torch.full((max(T, 1), E), -7.0, device="cuda"),
                    ids=torch.full((max(T, 1), k), -7, dtype=torch.int32, device="cuda"),
                    w=torch.full((max(T, 1), k), -7.0, device="cuda"),
                    counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
                    offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
                    toffs=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
                    perm=torch.full((max(R, 1),), -7, dtype=torch.int32, device="cuda"),
                    inv=torch.full((max(R, 1),), -7, dtype=torch.int32, device="cuda"))

    a, b = tables(), tables()
    fp4.fp4_moe_router_route(x, T, H, wg, E, k, a["logits"], a["ids"], a["w"], a["counts"], a["offsets"], a["toffs"],
                             a["perm"], a["inv"], scratch)
    fp4.fp4_moe_router(x, T, H, wg, E, k, b["logits"], b["ids"], b["w"])
    fp4.fp4_moe_route(b["ids"], T, k, E, b["counts"], b["offsets"], b["toffs"], b["perm"], b["inv"], scratch)
    assert fp4.fp4_get_device_status() == 0
    for name in a:
        assert torch.equal(a[name], b[name]), name
    if T:
        assert int(a["offsets"][E]) == R

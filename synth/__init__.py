"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the quantizers, the GEMM or the MoE layer:
it only draws random tensors with torch generators and shapes them like the
workloads (expert-shaped weights with outliers, Gaussian activations, Gaussian
router logits with an optional Zipf popularity skew, top-k selection of the
drawn logits).  Both the CUDA path and the oracle consume what it returns; the
oracle always receives host copies.

Recipes (one seed per call; ``torch.Generator`` on the target device):
  weights      fp32 N(0, sigma) -> outliers: exactly round(p * n) distinct
               positions chosen uniformly, multiplied by ``factor`` (sign kept)
               -> rounded to bf16.
  activations  bf16 N(0, 1).
  router       logits z[t, e] + log p_e with z ~ N(0, 1) and p_e proportional
               to rank(e)^-s under a seeded random rank permutation (s = 0 is
               uniform); expert_ids = the k largest logits per token, ties to
               the lower expert id; weights = softmax over the k chosen logits.
"""
import torch


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights_bf16(shape, sigma, outlier_frac, outlier_factor, seed, device="cpu"):
    """Expert-shaped weights: N(0, sigma) with a fraction of entries scaled."""
    g = _gen(seed, device)
    w = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * sigma
    n = w.numel()
    cnt = int(round(outlier_frac * n))
    if cnt > 0:
        idx = torch.randperm(n, generator=g, device=device)[:cnt]
        flat = w.view(-1)
        flat[idx] = flat[idx] * outlier_factor
    return w.to(torch.bfloat16)


def activations_bf16(shape, seed, device="cpu", std=1.0):
    g = _gen(seed, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def router(T, E, k, seed, zipf_s=0.0, device="cpu"):
    """Return (expert_ids int32 [T, k], topk_weights fp32 [T, k], counts int64 [E])."""
    g = _gen(seed, device)
    z = torch.randn((T, E), generator=g, device=device, dtype=torch.float32)
    if zipf_s > 0:
        ranks = torch.randperm(E, generator=g, device=device).to(torch.float64) + 1.0
        p = ranks.pow(-zipf_s)
        p = p / p.sum()
        z = z + torch.log(p).to(torch.float32)[None, :]
    # top-k with ties to the lower id: stable descending sort
    order = torch.sort(z, dim=1, descending=True, stable=True).indices[:, :k]
    ids = order.to(torch.int32)
    sel = torch.gather(z, 1, order)
    w = torch.softmax(sel, dim=1).to(torch.float32)
    counts = torch.bincount(ids.reshape(-1).to(torch.int64), minlength=E)
    return ids, w, counts


def router_fixed_counts(counts, seed, device="cpu"):
    """Top-1 routing with prescribed per-expert row counts, tokens in a seeded
    random order, weights uniform in [0.25, 1).  Returns the same triple as
    router()."""
    g = _gen(seed, device)
    ids = torch.cat([torch.full((int(n),), e, dtype=torch.int32, device=device) for e, n in enumerate(counts)])
    ids = ids[torch.randperm(ids.numel(), generator=g, device=device)].reshape(-1, 1)
    w = (0.25 + 0.75 * torch.rand((ids.shape[0], 1), generator=g, device=device)).to(torch.float32)
    c = torch.tensor([int(n) for n in counts], dtype=torch.int64, device=device)
    return ids, w, c


def random_codes(shape_bytes, seed, device="cpu"):
    """Uniform random packed FP4 bytes (every code equally likely)."""
    g = _gen(seed, device)
    return torch.randint(0, 256, shape_bytes, generator=g, device=device, dtype=torch.int32).to(torch.uint8)


def random_e4m3_scales(shape, seed, lo=0x20, hi=0x48, device="cpu"):
    """Random E4M3 scale bytes in [lo, hi) (defaults span 2^-3 .. 2^2)."""
    g = _gen(seed, device)
    return torch.randint(lo, hi, shape, generator=g, device=device, dtype=torch.int32).to(torch.uint8)

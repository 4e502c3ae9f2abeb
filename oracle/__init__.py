"""Plain, slow CPU oracle for the NVFP4 / MXFP4 W4A4 MoE expert path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
legs of ``bench.py`` use it.  It shares no code with the CUDA path: the
number formats, rounding rules, scale rules, layouts and the GEMM are all
written out here again, from the pages' definitions, in numpy.

Sources (cited by page title and section):
  * "DeepSeek-V4.1-Flash-NVFP4" model-card digest, §二 (the E2M1 value table,
    packing two codes per byte, NVFP4 group of 16 with a block scale under a
    tensor-level scale) and §一 / §六 (the lossless MXFP4 -> NVFP4 remap).
  * same page, §三 (which layers: routed experts w1/w2/w3; MXFP4 = one
    UE8M0 scale per 32 elements).
  * "DeepSeek-V4 architecture" page, §6.3 (1x32 MX tiles) and §5.1 (SwiGLU
    feed-forward layers); §2.1 (Pro shape: 384 experts, 6 active).
  * "DeepSeek-V4 FP4 QAT" page, §3.1 (simplified MoE forward: per-token
    top-k experts, outputs summed); §4.2 (FP4 -> FP8 widening without loss)
    and §4.3 (FP8 activations against FP4 weights: W4A8).

Modules:
  formats  -- E2M1 / E4M3 / UE8M0 encoders and decoders (brute-force nearest)
  quant    -- NVFP4, MXFP4 and MXFP8 quantizers, dequantizers, MXFP4->NVFP4
              remap, E2M1 -> E4M3 widening
  layouts  -- the tensor-core scale-factor tile layout (permutation only)
  gemm     -- fp64 dequantize-then-matmul GEMMs (NVFP4, MXFP4, W4A8) and
              their error bound
  moe      -- routing (stable sort), SwiGLU expert FFN, combine

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against something other than itself (the pages' table, a library cast,
exhaustive brute force, closed-form integer GEMMs, invariants).  The
exhaustive 2^32 sweeps live in ``oracle/sweep.c``.  The pages print no
worked example of an expert; the expert FFN (``moe.expert_ffn_ref`` and its
MXFP4 / W4A8 variants) is pinned by a case worked by hand
(``tests/golden/expert_ffn_hand.txt``) where SiLU and every re-quantization
are exact, so a swapped gate/up, a missing SiLU or a transposed W2 fails.
"""

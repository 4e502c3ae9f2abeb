"""Failure detection without a GPU fault.

Every mbarrier wait in the GEMM pipeline is bounded by a wall-clock limit.
Shrinking the limit to 1 ns makes the first wait that is not already
satisfied run out: the kernel must record FP4_ERR_DEVICE_TIMEOUT in the
device status word, let its in-flight copies and MMAs finish, free tensor
memory and return.  The context must stay usable: with the default limit
restored, the same GEMM gives the same result as before.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    import fp4_block_scaled_03_b200 as fp4

    M = N = K = 1024
    a = synth.random_codes((M, K // 2), seed=1, device="cuda")
    b = synth.random_codes((N, K // 2), seed=2, device="cuda")
    asf = synth.random_e4m3_scales((fp4.fp4_sf_tiled_bytes(M, K),), seed=3, lo=0x30, hi=0x40, device="cuda")
    bsf = synth.random_e4m3_scales((fp4.fp4_sf_tiled_bytes(N, K),), seed=4, lo=0x30, hi=0x40, device="cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    ref = fp4.gemm(a, asf, one, b, bsf, one, M, N, K)
    assert fp4.fp4_get_device_status() == 0
    fp4.fp4_set_wait_limit_ns(1)
    try:
        fp4.gemm(a, asf, one, b, bsf, one, M, N, K)
        st = fp4.fp4_get_device_status()
    finally:
        fp4.fp4_set_wait_limit_ns(0)
    assert st == 7  # FP4_ERR_DEVICE_TIMEOUT
    again = fp4.gemm(a, asf, one, b, bsf, one, M, N, K)
    assert fp4.fp4_get_device_status() == 0
    assert torch.equal(again, ref)

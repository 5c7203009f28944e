"""Failure detection without a GPU fault: every pipeline wait in the decode
GEMV, the GEMM and the grouped quantize is bounded by the launch's wait limit.  With
the copy stall test hook on, the copy warp issues no copies (a flag that
nothing sets), so every compute warp's wait for a stage must run out after
the (short) wait limit: the call must set Q4_STATUS_TIMEOUT and return, and
after switching the hook off, restoring the limit and re-zeroing the
workspace, the next call is correct."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_matmul_close, bits, oracle_state

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("qtype,bs,dq,N,K", [("nf4", 64, True, 4096, 8192), ("int4_asym", 128, False, 4096, 8192)])
def test_gemv_wait_limit_times_out_and_recovers(oracle, qtype, bs, dq, N, K):
    """The decode kernel's two instance sets: NF4 (with INT4 symmetric) and
    INT4 asymmetric (zero-point window)."""
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4
    g = torch.Generator().manual_seed(5)
    M = 4
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).half()
    st = q4.quantize(W.cuda(), bs, qtype, dq)
    q4.clear_device_status()
    try:
        q4.set_wait_limit_ns(200_000)  # 0.2 ms
        q4.set_copy_stall(True)
        q4.gemv(A.cuda(), st)
        torch.cuda.synchronize()
        assert q4.last_device_status() & 2  # Q4_STATUS_TIMEOUT
    finally:
        q4.set_copy_stall(False)
        q4.set_wait_limit_ns(0)
        q4.reset_workspaces()
        q4.clear_device_status()
    y = q4.gemv(A.cuda(), st)
    rows = np.arange(0, N, 61)
    ost = oracle_state(oracle, W, bs, {"nf4": 0, "int4_asym": 2}[qtype], dq)
    w16 = oracle.dequantize(ost, False).reshape(N, K)[rows]
    ref = oracle.matmul(bits(A), False, w16, False, M, len(rows), K)
    assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)
    assert q4.last_device_status() == 0


@pytest.mark.parametrize("dq", [True, False])
def test_grouped_quantize_wait_limit_times_out_and_recovers(oracle, dq):
    """The grouped quantize's consumer warps wait for ring stages that the
    stalled producer never fills: Q4_STATUS_TIMEOUT, then a correct call."""
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4
    from gpu_helpers import assert_state_equal
    g = torch.Generator().manual_seed(6)
    Ws = [torch.randn(N, K, generator=g).mul(0.02).bfloat16() for N, K in [(1024, 4096), (3000, 1024)]]
    q4.clear_device_status()
    try:
        q4.set_wait_limit_ns(200_000)
        q4.set_copy_stall(True)
        q4.quantize_grouped([W.cuda() for W in Ws], 64, "nf4", dq)
        torch.cuda.synchronize()
        assert q4.last_device_status() & 2
    finally:
        q4.set_copy_stall(False)
        q4.set_wait_limit_ns(0)
        q4.reset_workspaces()
        q4.clear_device_status()
    sts = q4.quantize_grouped([W.cuda() for W in Ws], 64, "nf4", dq)
    for W, st in zip(Ws, sts):
        assert_state_equal(st, oracle_state(oracle, W, 64, 0, dq))
    assert q4.last_device_status() == 0


@pytest.mark.parametrize("M,N,K", [(512, 1024, 2048), (700, 10240, 512)])
def test_gemm_wait_limit_times_out_and_recovers(oracle, M, N, K):
    """The GEMM's MMA and dequant warps wait for tiles that the stalled
    producer never copies: Q4_STATUS_TIMEOUT, the kernel returns (waiting
    for its issued MMAs before it frees the tensor memory), and a following
    call is correct.  The first shape runs 256-token tiles, the second
    512-token tiles (two rings for the producer to drain)."""
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4
    g = torch.Generator().manual_seed(7)
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).bfloat16()
    st = q4.quantize(W.cuda(), 64, "nf4", True)
    q4.clear_device_status()
    try:
        q4.set_wait_limit_ns(200_000)
        q4.set_copy_stall(True)
        q4.gemm(A.cuda(), st)
        torch.cuda.synchronize()
        assert q4.last_device_status() & 2
    finally:
        q4.set_copy_stall(False)
        q4.set_wait_limit_ns(0)
        q4.clear_device_status()
    y = q4.gemm(A.cuda(), st)
    rows = np.arange(0, N, 37)
    ost = oracle_state(oracle, W, 64, 0, True)
    w16 = oracle.dequantize(ost, True).reshape(N, K)[rows]
    ref = oracle.matmul(bits(A), True, w16, True, M, len(rows), K)
    assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)
    assert q4.last_device_status() == 0

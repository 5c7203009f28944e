"""GPU parity on the method's degenerate cases and at the largest sizes:
blocks of zeros, negative zeros, constants, a single spike, one-sided
values, subnormals only and near-maximum magnitudes; and one matrix of more
than 2^31 elements.  States and dequantized weights bit-exact with the CPU
oracle; GEMV and GEMM within the matmul tolerance of its binary64 product."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_matmul_close, assert_state_equal, bits, oracle_state

pytestmark = pytest.mark.gpu

QT = {"nf4": 0, "int4_sym": 1, "int4_asym": 2}
K_DEG = 1024  # columns: a whole number of blocks at every blocksize


@pytest.fixture(scope="module")
def q4():
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4 as m
    assert torch.cuda.is_available()
    m.clear_device_status()
    return m


def degenerate_rows(dtype, B, seed, large=True):
    """One row per kind of block (every block of a row is of that kind),
    plus random rows so that the matrix spans several 16-row groups."""
    g = torch.Generator().manual_seed(seed)
    K = K_DEG
    tiny = 2.0 ** -24 if dtype == torch.float16 else 2.0 ** -133  # smallest subnormal
    big = 60000.0 if dtype == torch.float16 else 1.0e38
    u = lambda: torch.rand(K, generator=g) * 0.9 + 0.1
    rows = [
        torch.zeros(K),                                   # all zero: the scale is 0
        torch.full((K,), -0.0),                           # negative zeros
        torch.full((K,), 0.125),                          # constant positive
        torch.full((K,), -3.0),                           # constant negative
        u(),                                              # all positive (INT4 asym: z = 0)
        -u(),                                             # all negative (INT4 asym: z = 15)
        torch.where(torch.arange(K) % 2 == 0, 1.0, -1.0),  # symmetric +-c
        torch.randint(1, 100, (K,), generator=g).float() * tiny * torch.where(torch.rand(K, generator=g) < 0.5, -1.0, 1.0),
    ]
    spike = torch.zeros(K)
    spike[torch.arange(0, K, B) + (torch.arange(K // B) * 7) % B] = -0.75  # one nonzero per block
    rows.append(spike)
    if large:
        rows.append((torch.randn(K, generator=g) * big / 4).clamp(-big, big))  # near the format's maximum
        rows[-1][::B] = big
    while len(rows) % 16:
        rows.append(torch.randn(K, generator=g) * 0.02)
    return torch.stack(rows).to(dtype)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("qtype,dq", [("nf4", False), ("nf4", True), ("int4_sym", False), ("int4_asym", False)])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
def test_degenerate_blocks_bit_exact(q4, oracle, dtype, qtype, dq, bs):
    W = degenerate_rows(dtype, bs, seed=bs + 5 * QT[qtype] + (1 if dq else 0))
    ost = oracle_state(oracle, W, bs, QT[qtype], dq)
    st = q4.quantize(W.cuda(), bs, qtype, dq)
    assert_state_equal(st, ost)
    (stg,) = q4.quantize_grouped([W.cuda()], bs, qtype, dq)
    assert_state_equal(stg, ost)
    for out in (torch.float16, torch.bfloat16):
        d = q4.dequantize(st, out)
        assert np.array_equal(bits(d), oracle.dequantize(ost, out == torch.bfloat16))
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0


@pytest.mark.parametrize("qtype,dq", [("nf4", True), ("int4_sym", False), ("int4_asym", False)])
def test_degenerate_blocks_gemv_gemm(q4, oracle, qtype, dq):
    """The consumers on zero, constant, one-sided, spike and subnormal
    blocks (magnitudes that keep the outputs finite)."""
    bs = 128 if qtype != "nf4" else 64
    W = degenerate_rows(torch.bfloat16, bs, seed=40 + QT[qtype], large=False)
    N, K = W.shape
    ost = oracle_state(oracle, W, bs, QT[qtype], dq)
    st = q4.quantize(W.cuda(), bs, qtype, dq)
    g = torch.Generator().manual_seed(41)
    for M in (1, 4, 16):
        A = torch.randn(M, K, generator=g).half()
        y = q4.gemv(A.cuda(), st)
        assert_matmul_close(y, oracle.gemv_reference(bits(A), False, ost, N, K))
    A = torch.randn(64, K, generator=g).bfloat16()
    y = q4.gemm(A.cuda(), st)
    w16 = oracle.dequantize(ost, True)
    assert_matmul_close(y, oracle.matmul(bits(A), True, w16, True, 64, N, K))
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0


def test_matrix_over_2g_elements(q4, oracle):
    """W[65552, 32768] bf16 ~ N(0, 0.02): 2,148,007,936 elements, past 2^31
    (element 2^31 starts row 65536).  NF4 blocksize 64 through the single
    and the grouped quantizer, dequantize, the decode GEMV at M = 1 and the
    GEMM at M = 64, checked on sampled rows that include both sides of the
    2^31 boundary and the last row."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    N, K, B = 65552, 32768, 64
    assert N * K > 2 ** 31
    W = wl.gaussian((N, K), 0.02, torch.bfloat16, 77, device="cuda")
    st = q4.quantize(W, B, "nf4", False)
    (stg,) = q4.quantize_grouped([W], B, "nf4", False)
    torch.cuda.synchronize()
    assert torch.equal(st.packed, stg.packed) and torch.equal(st.absmax, stg.absmax)
    del stg
    rows = [0, 1, 32767, 40000, 65535, 65536, 65537, N - 1]
    osts = [oracle.quantize(bits(W[r]), True, B, 0, False) for r in rows]
    packed = st.packed.view(N, K // 2)
    absmax = st.absmax.view(N, K // B)
    for r, o in zip(rows, osts):
        assert np.array_equal(packed[r].cpu().numpy(), o.packed), f"packed codes differ in row {r}"
        assert np.array_equal(absmax[r].cpu().numpy().view(np.uint32), o.absmax.view(np.uint32)), \
            f"absmax differs in row {r}"
    d = q4.dequantize(st, torch.bfloat16)
    for r, o in zip(rows, osts):
        assert np.array_equal(bits(d[r]), oracle.dequantize(o, True)), f"dequantized row {r} differs"
    del d, W
    torch.cuda.empty_cache()
    idx = torch.tensor(rows, device="cuda")
    a1 = wl.activation(1, K, torch.float16, 78)
    y1 = q4.gemv(a1.cuda(), st)
    ref1 = np.concatenate([oracle.gemv_reference(bits(a1), False, o, 1, K) for o in osts], axis=1)
    assert_matmul_close(y1[:, idx], ref1)
    a64 = wl.activation(64, K, torch.bfloat16, 79)
    y64 = q4.gemm(a64.cuda(), st)
    w16 = np.concatenate([oracle.dequantize(o, True) for o in osts])
    ref64 = oracle.matmul(bits(a64), True, w16, True, 64, len(rows), K)
    assert_matmul_close(y64[:, idx], ref64)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0

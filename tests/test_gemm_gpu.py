"""GPU parity of the tcgen05 W4A16 GEMM against the oracle (C ABI)."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_matmul_close, bits, oracle_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4():
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4 as m
    m.clear_device_status()
    return m


def _case(q4, oracle, M, N, K, a_dtype=torch.bfloat16, dq=True, seed=0, out_dtype=None, rows=None):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).to(a_dtype)
    st = q4.quantize(W.cuda(), 64, "nf4", dq)
    ost = oracle_state(oracle, W, 64, 0, dq)
    y = q4.gemm(A.cuda(), st, out_dtype)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    if rows is None:
        ref = oracle.gemv_reference(bits(A), a_dtype == torch.bfloat16, ost, N, K)
        return y, ref
    w16 = oracle.dequantize(ost, a_dtype == torch.bfloat16).reshape(N, K)[rows]
    ref = oracle.matmul(bits(A), a_dtype == torch.bfloat16, w16, a_dtype == torch.bfloat16, M,
                        len(rows), K)
    return y[:, torch.from_numpy(rows).cuda()], ref


def test_gemm_one_tile(q4, oracle):
    y, ref = _case(q4, oracle, 256, 256, 64)
    assert_matmul_close(y, ref)


def test_gemm_split_k_few_tiles(q4, oracle):
    """One matrix of few tiles (M = 512, N = 2048, K = 4608: 32 tiles for
    many more SMs): the launch cuts tiles into k halves whose partials meet
    in the workspace.  Against the oracle, bit-identical on repeat, the
    workspace left zeroed, and within tolerance of the uncut launch."""
    import ctypes
    g = torch.Generator().manual_seed(12)
    M, N, K = 512, 2048, 4608
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).bfloat16()
    st = q4.quantize(W.cuda(), 64, "nf4", True)
    ost = oracle_state(oracle, W, 64, 0, True)
    arr = (ctypes.POINTER(q4._CState) * 1)(ctypes.pointer(st.c_struct()))
    wsz = ctypes.c_size_t(0)
    assert q4.library().q4_gemm_workspace_size(1, arr, M, ctypes.byref(wsz)) == 0
    assert wsz.value > 0  # the plan cuts tiles
    a = A.cuda()
    ys = [q4.gemm(a, st) for _ in range(3)]
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])
    rows = np.arange(0, N, 7)
    w16 = oracle.dequantize(ost, True).reshape(N, K)[rows]
    ref = oracle.matmul(bits(A), True, w16, True, M, len(rows), K)
    assert_matmul_close(ys[0][:, torch.from_numpy(rows).cuda()], ref)
    # the arrival counters (the workspace's first 64 KB) are left zeroed
    ws = q4._workspace(a.device, "gemm", wsz.value)
    assert int(ws[:65536].count_nonzero()) == 0
    # the uncut launch (no workspace) gives the same product within tolerance
    y1 = torch.empty_like(ys[0])
    assert q4.library().q4_gemm(a.data_ptr(), 1, M, ctypes.pointer(st.c_struct()), y1.data_ptr(), 1,
                                None, 0, None) == 0
    torch.cuda.synchronize()
    assert_matmul_close(y1[:, torch.from_numpy(rows).cuda()], ref)


def _sampled_case(q4, oracle, M, N, K, seed, rows):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).bfloat16()
    st = q4.quantize(W.cuda(), 64, "nf4", True)
    ost = oracle_state(oracle, W, 64, 0, True)
    w16 = oracle.dequantize(ost, True).reshape(N, K)[rows]
    ref = oracle.matmul(bits(A), True, w16, True, M, len(rows), K)
    return A.cuda(), st, ref


def test_gemm_tall_tiles_ragged_half(q4, oracle):
    """512-token tiles whose last tile's second half lies wholly past M:
    M = 700, N = 10240, K = 512.  The planner takes the tall tiles here (160
    tall tiles, the busiest CTA at 272 weighted units, against 320 for 240
    half-height tiles), so tokens 512 .. 699 run as a lone first half and
    the second half is neither loaded nor multiplied."""
    M, N, K = 700, 10240, 512
    rows = np.concatenate([np.arange(0, N, 37), np.arange(N - 40, N)])
    a, st, ref = _sampled_case(q4, oracle, M, N, K, 21, rows)
    y = q4.gemm(a, st)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)


def test_gemm_tall_tiles_ragged_rows(q4, oracle):
    """512-token tiles over a weight matrix whose last tile is ragged (M =
    700, N = 9440 = 73 x 128 + 96, K = 512: 148 tall tiles, the planner's
    pick); the rows past N are neither stored nor let into the result."""
    M, N, K = 700, 9440, 512
    rows = np.concatenate([np.arange(0, N, 53), np.arange(N - 112, N)])
    a, st, ref = _sampled_case(q4, oracle, M, N, K, 25, rows)
    y = q4.gemm(a, st)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)


def test_gemm_tall_tiles_f16_fp32_out(q4, oracle):
    """512-token tiles with fp16 activations and fp32 output (M = 600, N =
    10240, K = 512: 160 tall tiles, the second of each column a lone first
    half of 88 tokens); the fp32 output differs from the binary64 product
    only by the fp32 accumulation order."""
    M, N, K = 600, 10240, 512
    g = torch.Generator().manual_seed(23)
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).half()
    st = q4.quantize(W.cuda(), 64, "nf4", True)
    ost = oracle_state(oracle, W, 64, 0, True)
    rows = np.concatenate([np.arange(0, N, 41), np.arange(N - 24, N)])
    w16 = oracle.dequantize(ost, False).reshape(N, K)[rows]
    ref = oracle.matmul(bits(A), False, w16, False, M, len(rows), K)
    y = q4.gemm(A.cuda(), st, torch.float32)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    fro, mx = assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)
    assert fro < 1e-5


def test_gemm_round_robin_ragged_groups(q4, oracle):
    """A launch of too many tiles for a list (M = 5000, N = 27648, K = 256:
    10 x 216 tall tiles) is dealt round robin with the m-tiles taken four
    at a time; 10 m-tiles leave a last group of two.  Sampled rows and
    tokens, including the last of each, against the oracle."""
    M, N, K = 5000, 27648, 256
    rows = np.concatenate([np.arange(0, N, 211), np.arange(N - 8, N)])
    a, st, ref = _sampled_case(q4, oracle, M, N, K, 24, rows)
    y = q4.gemm(a, st)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    toks = np.concatenate([np.arange(0, M, 97), np.arange(M - 8, M)])
    sel = y[torch.from_numpy(toks).cuda()][:, torch.from_numpy(rows).cuda()]
    assert_matmul_close(sel, ref[toks])


def test_gemm_tall_tiles_split_k(q4, oracle):
    """512-token tiles cut into k halves: M = 1000, N = 2560, K = 16384.  40
    tall tiles of 256 k-blocks leave most SMs idle; cut, their 80 halves
    (busiest CTA 4896 weighted units) beat both the uncut tall tiles (8704)
    and the 80 half-height tiles (5120; cut, 160 halves overflow the SMs).
    Against the oracle, bit-identical on repeat, counters left zeroed."""
    import ctypes
    M, N, K = 1000, 2560, 16384
    rows = np.concatenate([np.arange(0, N, 29), np.arange(N - 16, N)])
    a, st, ref = _sampled_case(q4, oracle, M, N, K, 22, rows)
    arr = (ctypes.POINTER(q4._CState) * 1)(ctypes.pointer(st.c_struct()))
    wsz = ctypes.c_size_t(0)
    assert q4.library().q4_gemm_workspace_size(1, arr, M, ctypes.byref(wsz)) == 0
    assert wsz.value > 0  # the plan cuts tiles
    ys = [q4.gemm(a, st) for _ in range(2)]
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    assert torch.equal(ys[0], ys[1])
    assert_matmul_close(ys[0][:, torch.from_numpy(rows).cuda()], ref)
    ws = q4._workspace(a.device, "gemm", wsz.value)
    assert int(ws[:65536].count_nonzero()) == 0


def test_gemm_exact_small_integers(q4, oracle):
    """A in {-1, 0, 1}, every block's maximum 1 (so w^ is the bf16 level),
    K = 64, fp32 output: each partial sum of the tensor cores is exactly
    representable in binary32 (the terms' magnitudes span under 2^17 ulps),
    so Y equals the oracle's binary64 product exactly."""
    g = torch.Generator().manual_seed(9)
    M, N, K = 40, 64, 64
    L = torch.tensor(oracle.nf4_levels())
    codes = torch.randint(0, 16, (N, K), generator=g)
    W = L[codes]
    W[:, 0] = 1.0  # the block absmax
    W = W.bfloat16()
    A = torch.randint(-1, 2, (M, K), generator=g).bfloat16()
    st = q4.quantize(W.cuda(), 64, "nf4", False)
    ost = oracle_state(oracle, W, 64, 0, False)
    y = q4.gemm(A.cuda(), st, torch.float32)
    torch.cuda.synchronize()
    ref = oracle.matmul(bits(A), True, oracle.dequantize(ost, True), True, M, N, K)
    assert np.array_equal(y.cpu().double().numpy(), ref)


def test_gemm_fp32_out_tight(q4, oracle):
    """fp32 output: the only difference from the binary64 reference is the
    fp32 accumulation order, far below the tolerance."""
    y, ref = _case(q4, oracle, 256, 512, 1024, out_dtype=torch.float32, seed=1)
    fro, mx = assert_matmul_close(y, ref)
    assert fro < 1e-5


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (100, 512, 256), (300, 272, 1088),
                                   (513, 768, 4096)])
def test_gemm_ragged(q4, oracle, M, N, K):
    y, ref = _case(q4, oracle, M, N, K, seed=M + N)
    assert_matmul_close(y, ref)


@pytest.mark.parametrize("a_dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("dq", [False, True])
def test_gemm_dtypes(q4, oracle, a_dtype, dq):
    y, ref = _case(q4, oracle, 384, 512, 512, a_dtype=a_dtype, dq=dq, seed=3)
    assert_matmul_close(y, ref)


def test_gemm_prefill_7b_layer_m512(q4, oracle):
    """Prefill config: the 7B layer shapes, NF4 double-quant weights, bf16
    activations at M = 512, one grouped launch; every output of the layer
    against the oracle's binary64 product (about 200 GFLOP on the host)."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    Ws = wl.layer_weights(wl.LAYER_7B, 0.02, seed=300)
    sts = [q4.quantize(W.cuda(), 64, "nf4", True) for W in Ws]
    osts = [oracle_state(oracle, W, 64, 0, True) for W in Ws]
    M = 512
    As = [wl.activation(M, K, torch.bfloat16, seed=400 + i) for i, (_, N, K) in enumerate(wl.LAYER_7B)]
    ys = q4.gemm_grouped([a.cuda() for a in As], sts)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    for (name, N, K), a, y, ost in zip(wl.LAYER_7B, As, ys, osts):
        w16 = oracle.dequantize(ost, True)
        ref = oracle.matmul(bits(a), True, w16, True, M, N, K)
        assert_matmul_close(y, ref)


@pytest.mark.parametrize("M", [2048, 8192])
def test_gemm_prefill_7b_layer_large_m(q4, oracle, M):
    """Prefill config at M = 2048 and 8192 tokens: one grouped launch over the
    7B layer; checked on a deterministic sample of 64 token rows x 256 output
    columns per matrix (the oracle's binary64 product of those)."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    Ws = wl.layer_weights(wl.LAYER_7B, 0.02, seed=310)
    sts = [q4.quantize(W.cuda(), 64, "nf4", True) for W in Ws]
    osts = [oracle_state(oracle, W, 64, 0, True) for W in Ws]
    rng = np.random.default_rng(M)
    As = [wl.activation(M, K, torch.bfloat16, seed=410 + i) for i, (_, N, K) in enumerate(wl.LAYER_7B)]
    ys = q4.gemm_grouped([a.cuda() for a in As], sts)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    for (name, N, K), a, y, ost in zip(wl.LAYER_7B, As, ys, osts):
        rows = np.sort(rng.choice(N, 256, replace=False))
        toks = np.sort(rng.choice(M, 64, replace=False))
        w16 = oracle.dequantize(ost, True).reshape(N, K)[rows]
        a16 = bits(a).reshape(M, K)[toks]
        ref = oracle.matmul(a16, True, w16, True, len(toks), len(rows), K)
        sub = y[torch.from_numpy(toks).cuda()][:, torch.from_numpy(rows).cuda()]
        assert_matmul_close(sub, ref)


@pytest.mark.parametrize("qtype,dq", [("nf4", False), ("nf4", True), ("int4_sym", False), ("int4_asym", False)])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
def test_gemm_formats_and_blocksizes(q4, oracle, qtype, dq, bs):
    """Every state format the quantizer makes, at every blocksize: ragged M
    and N (a partial 256-row and 128-column tile), K = 4608 so that the
    row's window of 16 block scales turns over (144 blocks at B = 32, 18 at
    B = 256); against the oracle's binary64 product of its dequantized
    weights (w^ exactly as q4_dequantize gives it)."""
    QT = {"nf4": 0, "int4_sym": 1, "int4_asym": 2}[qtype]
    g = torch.Generator().manual_seed(bs + 7 * QT)
    M, N, K = 300, 272, 4608
    W = torch.randn(N, K, generator=g).mul(0.02)
    W.view(-1)[::701] *= 15  # outliers: wide block ranges
    W = W.bfloat16()
    A = torch.randn(M, K, generator=g).bfloat16()
    st = q4.quantize(W.cuda(), bs, qtype, dq)
    ost = oracle_state(oracle, W, bs, QT, dq)
    y = q4.gemm(A.cuda(), st)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0
    w16 = oracle.dequantize(ost, True).reshape(N, K)
    ref = oracle.matmul(bits(A), True, w16, True, M, N, K)
    assert_matmul_close(y, ref)


def test_gemm_grouped_int4_asym_layer(q4, oracle):
    """One grouped launch over the 7B layer's shapes in INT4 asymmetric
    group-128 (the format the decode GEMV also takes), M = 512; sampled
    output columns against the oracle."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    Ws = wl.layer_weights(wl.LAYER_7B, 0.02, seed=320)
    sts = [q4.quantize(W.cuda(), 128, "int4_asym", False) for W in Ws]
    rng = np.random.default_rng(3)
    M = 512
    As = [wl.activation(M, K, torch.bfloat16, seed=420 + i) for i, (_, N, K) in enumerate(wl.LAYER_7B)]
    ys = q4.gemm_grouped([a.cuda() for a in As], sts)
    torch.cuda.synchronize()
    for W, (name, N, K), a, y in zip(Ws, wl.LAYER_7B, As, ys):
        ost = oracle_state(oracle, W, 128, 2, False)
        rows = np.sort(rng.choice(N, 64, replace=False))
        w16 = oracle.dequantize(ost, True).reshape(N, K)[rows]
        ref = oracle.matmul(bits(a), True, w16, True, M, len(rows), K)
        assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)

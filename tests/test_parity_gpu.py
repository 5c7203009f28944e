"""GPU parity: quantize / dequantize bit-exact, GEMV within tolerance, against
the CPU oracle on identical seeded inputs, called through the C ABI."""
import numpy as np
import pytest
import torch

from gpu_helpers import (assert_matmul_close, assert_state_equal, bits, is_bf16, oracle_state)

pytestmark = pytest.mark.gpu

QT = {"nf4": 0, "int4_sym": 1, "int4_asym": 2}


@pytest.fixture(scope="module")
def q4():
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4 as m
    assert torch.cuda.is_available()
    m.clear_device_status()
    return m


def dev(t):
    return t.to("cuda")


# ------------------------------------------------------------- quantize -----

def test_tiny_nf4_config(q4, oracle):
    """fp16 W[256,512] ~ N(0,0.02), seed 0, NF4 blocksize 64, no double quant;
    quantize -> pack -> dequantize bit-exact; GEMV with x[512] ~ N(0,1)."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    W = wl.tiny_weight(0)
    x = wl.tiny_activation(1)
    st = q4.quantize(dev(W), 64, "nf4", False)
    ost = oracle_state(oracle, W, 64, 0, False)
    assert_state_equal(st, ost)
    d = q4.dequantize(st)
    assert np.array_equal(bits(d), oracle.dequantize(ost, False))
    y = q4.gemv(dev(x), st)
    ref = oracle.gemv_reference(bits(x), False, ost, 256, 512)
    assert_matmul_close(y, ref)
    torch.cuda.synchronize()
    assert q4.last_device_status() == 0


@pytest.mark.parametrize("qtype,bs,dq", [("nf4", 64, True), ("int4_sym", 128, False),
                                         ("int4_asym", 128, False)])
def test_scheme_config_4096_outliers(q4, oracle, qtype, bs, dq):
    """bf16 W[4096,4096] ~ N(0,0.02) with 0.1% x20 outliers; the three schemes."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    W = wl.outlier_weight(4096, 4096, seed=0)
    st = q4.quantize(dev(W), bs, qtype, dq)
    ost = oracle_state(oracle, W, bs, QT[qtype], dq)
    assert_state_equal(st, ost)
    for out_dt in (torch.bfloat16, torch.float16):
        d = q4.dequantize(st, out_dt)
        assert np.array_equal(bits(d), oracle.dequantize(ost, out_dt == torch.bfloat16))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("qtype", ["nf4", "int4_sym", "int4_asym"])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
def test_quantize_ragged_shapes(q4, oracle, dtype, qtype, bs):
    """Several tiles plus ragged tails: n not a multiple of the block or of a
    256-block chunk, odd n, a single element, and wide-range values."""
    g = torch.Generator().manual_seed(bs * 7 + QT[qtype])
    shapes = [(1, 1), (3, 5), (17, 33), (7, 1001), (257, 300), (96, 4096 + 64)]
    for rows, cols in shapes:
        W = (torch.randn(rows, cols, generator=g) *
             torch.exp(torch.randn(rows, cols, generator=g) * 2)).to(dtype)
        W[0, 0] = 0.0
        dq = qtype == "nf4"
        for use_dq in ([False, True] if dq else [False]):
            st = q4.quantize(dev(W), bs, qtype, use_dq)
            ost = oracle_state(oracle, W, bs, QT[qtype], use_dq)
            assert_state_equal(st, ost)
            d = q4.dequantize(st, dtype)
            assert np.array_equal(bits(d), oracle.dequantize(ost, is_bf16(W)))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_nearest_coding_exhaustive_16bit_on_gpu(q4, oracle, dtype):
    """Every finite 16-bit value w paired with block maxima c from a spread of
    magnitudes (blocks [w, c] of size 2... as 32-blocks padded with zeros):
    codes bit-exact with the oracle."""
    allbits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(dtype)
    vals = allbits[torch.isfinite(allbits.float())]
    for c in [1.0, 0.7, 3.0e-3, 1234.5, 6.0e-5]:
        cc = torch.tensor(c, dtype=torch.float32).to(dtype)
        v = vals[vals.float().abs() <= cc.float()]
        blocks = torch.zeros(v.numel(), 32, dtype=dtype)
        blocks[:, 0] = v
        blocks[:, 1] = cc
        st = q4.quantize(dev(blocks), 32, "nf4", False)
        ost = oracle_state(oracle, blocks, 32, 0, False)
        assert_state_equal(st, ost)
        st = q4.quantize(dev(blocks), 32, "int4_sym", False)
        assert_state_equal(st, oracle_state(oracle, blocks, 32, 1, False))


def test_nonfinite_input_sets_status(q4):
    W = torch.randn(64, 64).half()
    W[3, 5] = float("inf")
    q4.clear_device_status()
    q4.quantize(dev(W), 64, "nf4", False)
    torch.cuda.synchronize()
    assert q4.last_device_status() & 1
    q4.clear_device_status()
    assert q4.last_device_status() == 0


def test_double_quant_mean_many_chunks(q4, oracle):
    """More 256-block chunks than one CTA run: the pairwise mean crosses CTAs."""
    W = torch.randn(4099, 8192, generator=torch.Generator().manual_seed(2)).mul(0.015).bfloat16()
    st = q4.quantize(dev(W), 64, "nf4", True)
    assert_state_equal(st, oracle_state(oracle, W, 64, 0, True))
    st2 = q4.quantize(dev(W), 64, "nf4", True)  # the workspace was left clean
    assert torch.equal(st.absmax_mean, st2.absmax_mean) and torch.equal(st.absmax_q, st2.absmax_q)


def test_host_rejects_bad_arguments(q4):
    W = dev(torch.randn(64, 64).half())
    with pytest.raises(q4.Q4Error):
        q4.quantize(W, 48)
    with pytest.raises(q4.Q4Error):
        q4.quantize(W, 64, "int4_sym", True)
    with pytest.raises(q4.Q4Error):
        base = dev(torch.randn(64 * 64 + 8).half())
        q4.quantize(base[1:64 * 64 + 1].view(64, 64), 64)  # not 16-byte aligned
    st = q4.quantize(W, 64)
    with pytest.raises(q4.Q4Error):
        q4.gemv(dev(torch.randn(33, 64).half()), st)    # M > 32


# ------------------------------------------------------------------ GEMV -----

def _gemv_case(q4, oracle, N, K, M, a_dtype, dq, bs=64, seed=0, out_dtype=None):
    g = torch.Generator().manual_seed(seed)
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).to(a_dtype)
    st = q4.quantize(dev(W), bs, "nf4", dq)
    ost = oracle_state(oracle, W, bs, 0, dq)
    y = q4.gemv(dev(A), st, out_dtype)
    ref = oracle.gemv_reference(bits(A), a_dtype == torch.bfloat16, ost, N, K)
    return y, ref


@pytest.mark.parametrize("M", [1, 2, 4, 7, 8, 9, 16, 17, 31, 32])
def test_gemv_batch_sizes(q4, oracle, M):
    y, ref = _gemv_case(q4, oracle, 512, 2048 + 64, M, torch.float16, True, seed=M)
    assert_matmul_close(y, ref)


@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("a_dtype", [torch.float16, torch.bfloat16])
def test_gemv_blocksizes_dtypes(q4, oracle, bs, a_dtype):
    for M in (1, 16):
        y, ref = _gemv_case(q4, oracle, 272, 3072, M, a_dtype, bs == 64, bs=bs, seed=bs + M)
        assert_matmul_close(y, ref)


@pytest.mark.parametrize("M", [20, 32])
@pytest.mark.parametrize("a_dtype,out_dtype", [(torch.bfloat16, None), (torch.float16, torch.float32),
                                               (torch.bfloat16, torch.float32)])
def test_gemv_large_batch_grouped_dtypes(q4, oracle, M, a_dtype, out_dtype):
    """16 < M <= 32 in one pass (four activation tiles of 8): a grouped call
    over two matrices of different shapes, with 16-bit and fp32 outputs."""
    g = torch.Generator().manual_seed(M)
    shapes = [(384, 1024), (272, 3072)]
    Ws = [torch.randn(N, K, generator=g).mul(0.02).bfloat16() for N, K in shapes]
    As = [torch.randn(M, K, generator=g).to(a_dtype) for N, K in shapes]
    sts = [q4.quantize(dev(W), 64, "nf4", True) for W in Ws]
    ys = q4.gemv_grouped([dev(A) for A in As], sts, out_dtype)
    for (N, K), W, A, y in zip(shapes, Ws, As, ys):
        assert y.shape == (M, N) and y.dtype == (out_dtype or a_dtype)
        ost = oracle_state(oracle, W, 64, 0, True)
        ref = oracle.gemv_reference(bits(A), a_dtype == torch.bfloat16, ost, N, K)
        assert_matmul_close(y, ref)


@pytest.mark.parametrize("M", [1, 5, 13, 29])
def test_gemv_ragged_group_split_tiles(q4, oracle, M):
    """Shapes that leave partial 256-row tiles, 16-row groups cut by N, K not
    a multiple of the 128-k chunk, and tiles split across CTAs (seven
    matrices of different shapes in one launch)."""
    g = torch.Generator().manual_seed(300 + M)
    shapes = [(5, 64), (17, 192), (300, 1088), (257, 2112), (1000, 960), (16, 4096), (512, 64)]
    Ws = [torch.randn(N, K, generator=g).mul(0.05).bfloat16() for N, K in shapes]
    As = [torch.randn(M, K, generator=g).half() for N, K in shapes]
    sts = [q4.quantize(dev(W), 64, "nf4", True) for W in Ws]
    for _ in range(2):  # the second call reuses the workspace the first left
        ys = q4.gemv_grouped([dev(A) for A in As], sts)
        for (N, K), W, A, y in zip(shapes, Ws, As, ys):
            ost = oracle_state(oracle, W, 64, 0, True)
            ref = oracle.gemv_reference(bits(A), False, ost, N, K)
            assert_matmul_close(y, ref)
    assert q4.last_device_status() == 0


@pytest.mark.parametrize("M", [1, 16, 24])
@pytest.mark.parametrize("a_dtype", [torch.float16, torch.bfloat16])
def test_gemv_int4_sym(q4, oracle, a_dtype, M):
    """INT4 symmetric, group 128 (the scheme-coverage format): the decode
    kernel with the integer codebook -8..7 and the group scale in place of
    c~, against the oracle's dequantize + binary64 matmul."""
    g = torch.Generator().manual_seed(128 + M)
    N, K = 400, 4096 + 128
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    A = torch.randn(M, K, generator=g).to(a_dtype)
    st = q4.quantize(dev(W), 128, "int4_sym", False)
    ost = oracle_state(oracle, W, 128, 1, False)
    assert_state_equal(st, ost)
    y = q4.gemv(dev(A), st)
    ref = oracle.gemv_reference(bits(A), a_dtype == torch.bfloat16, ost, N, K)
    assert_matmul_close(y, ref)


@pytest.mark.parametrize("M", [1, 16, 24, 32])
@pytest.mark.parametrize("a_dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("bs", [32, 128])
def test_gemv_int4_asym(q4, oracle, a_dtype, M, bs):
    """INT4 asymmetric (robotsatlas.com "INT4": [0, 15] with an integer
    zero-point), with offset weights so the zero-points vary: the kernel's
    s (sum a q - z sum a) against the oracle's dequantize + binary64 matmul."""
    g = torch.Generator().manual_seed(256 + M + bs)
    N, K = 400, 4096 + 2 * bs
    W = (torch.randn(N, K, generator=g) * 0.02 + torch.randn(N, 1, generator=g) * 0.02).bfloat16()
    A = torch.randn(M, K, generator=g).to(a_dtype)
    st = q4.quantize(dev(W), bs, "int4_asym", False)
    ost = oracle_state(oracle, W, bs, 2, False)
    assert_state_equal(st, ost)
    z = np.concatenate([ost.zero & 15, ost.zero >> 4])
    assert len(np.unique(z)) > 4
    y = q4.gemv(dev(A), st)
    ref = oracle.gemv_reference(bits(A), a_dtype == torch.bfloat16, ost, N, K)
    assert_matmul_close(y, ref)


def test_gemv_grouped_rejects_mixed_formats(q4):
    """One grouped launch takes one format: a second matrix with another
    double-quant flag or quantization type is rejected on the host, before
    any launch."""
    W = dev(torch.randn(256, 512).half())
    a = q4.quantize(W, 64, "nf4", True)
    b = q4.quantize(W, 64, "nf4", False)
    c = q4.quantize(W, 64, "int4_sym", False)
    A = [dev(torch.randn(1, 512).half()) for _ in range(2)]
    for pair in ((a, b), (a, c), (c, a)):
        with pytest.raises(q4.Q4Error):
            q4.gemv_grouped(A, list(pair))
    assert q4.last_device_status() == 0


def test_gemv_fp32_output_tight(q4, oracle):
    """fp32 output against the unrounded reference: the fused path's own error
    (fp16 codebook values, fp32 accumulation) stays far below the tolerance."""
    y, ref = _gemv_case(q4, oracle, 1024, 4096, 4, torch.float16, True, out_dtype=torch.float32)
    fro, mx = assert_matmul_close(y, ref)
    assert fro < 5e-4


def test_gemv_exact_small_integers(q4, oracle):
    """A in {-1,0,1}, power-of-two block maxima, K = 64: the fp32 result is
    exact, so Y equals the reference exactly."""
    g = torch.Generator().manual_seed(4)
    N, K = 64, 64
    L = torch.tensor(oracle.nf4_levels())
    codes = torch.randint(0, 16, (N, K), generator=g)
    scale = 2.0 ** torch.randint(-3, 3, (N, 1), generator=g).float()
    W = (L[codes] * scale)
    W[:, 0] = scale[:, 0]  # the block absmax is the power of two
    W = W.half()
    A = torch.randint(-1, 2, (3, K), generator=g).half()
    st = q4.quantize(dev(W), 64, "nf4", False)
    ost = oracle_state(oracle, W, 64, 0, False)
    assert_state_equal(st, ost)
    y = q4.gemv(dev(A), st, torch.float32)
    ref = oracle.gemv_reference(bits(A), False, ost, N, K)
    assert np.array_equal(y.cpu().double().numpy(), ref)


def test_gemv_grouped_7b_layer(q4, oracle):
    """Llama-2-7B-shaped decode layer (q/k/v/o 4096x4096, gate/up 11008x4096,
    down 4096x11008), bf16 weights ~ N(0,0.02) -> NF4 blocksize 64 with double
    quant, fp16 activations at M = 1, 4, 16, one grouped launch; checked on
    sampled output rows of every matrix."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    Ws = wl.layer_weights(wl.LAYER_7B, 0.02, seed=100)
    sts = [q4.quantize(dev(W), 64, "nf4", True) for W in Ws]
    osts = [oracle_state(oracle, W, 64, 0, True) for W in Ws]
    for st, ost in zip(sts, osts):
        assert_state_equal(st, ost)
    rng = np.random.default_rng(0)
    for M in (1, 4, 16):
        As = [wl.activation(M, K, torch.float16, seed=200 + M + i) for i, (_, N, K) in enumerate(wl.LAYER_7B)]
        ys = q4.gemv_grouped([dev(a) for a in As], sts)
        for (name, N, K), a, y, ost in zip(wl.LAYER_7B, As, ys, osts):
            rows = np.sort(rng.choice(N, 384, replace=False))
            w16 = oracle.dequantize(ost, False).reshape(N, K)[rows]
            ref = oracle.matmul(bits(a), False, w16, False, M, len(rows), K)
            assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)


def test_gemv_repeat_calls_are_bit_identical(q4, oracle):
    """The split-K partial sums are added in a fixed order and the workspace
    is left zeroed: identical calls give identical bits, at every batch size
    and output type (17..32 rows use four column tiles)."""
    g = torch.Generator().manual_seed(6)
    W = dev(torch.randn(4096, 11008, generator=g).mul(0.02).bfloat16())
    st = q4.quantize(W, 64, "nf4", True)
    for M in (1, 4, 16, 24):
        A = dev(torch.randn(M, 11008, generator=g).half())
        for out_dt in (torch.float16, torch.float32):
            ys = [q4.gemv(A, st, out_dt) for _ in range(3)]
            torch.cuda.synchronize()
            assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2]), (M, out_dt)


def test_gemv_workspace_reuse_across_batch_sizes(q4, oracle):
    """One cached workspace serves every batch size in turn: each call leaves
    it zeroed, so a later call of another M (a different layout of partial
    sums and counters) still gets the right answer."""
    g = torch.Generator().manual_seed(8)
    N, K = 1024, 11008
    W = torch.randn(N, K, generator=g).mul(0.02).bfloat16()
    st = q4.quantize(dev(W), 64, "nf4", True)
    ost = oracle_state(oracle, W, 64, 0, True)
    rows = np.arange(0, N, 7)
    w16 = oracle.dequantize(ost, False).reshape(N, K)[rows]
    for M in (16, 1, 32, 8, 17, 4, 16, 1):
        A = torch.randn(M, K, generator=g).half()
        y = q4.gemv(dev(A), st)
        ref = oracle.matmul(bits(A), False, w16, False, M, len(rows), K)
        assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)


def test_gemv_workspace_left_zeroed_across_shapes(q4, oracle):
    """The partial-row slots and the counters sit at offsets that depend on
    M and on the group, so one cached workspace serves every call only if
    each call leaves all of it zeroed: alternate batch sizes and groups of
    different shapes on one workspace (large M first, then small)."""
    g = torch.Generator().manual_seed(12)
    shapes = [(1024, 2048), (256, 4096), (2048, 1024)]
    Ws = [torch.randn(N, K, generator=g).mul(0.02).bfloat16() for N, K in shapes]
    sts = [q4.quantize(dev(W), 64, "nf4", True) for W in Ws]
    osts = [oracle_state(oracle, W, 64, 0, True) for W in Ws]
    for M, idx in [(32, [0, 1, 2]), (1, [1]), (16, [2, 0]), (8, [0]), (32, [1]), (4, [0, 1, 2]), (1, [2])]:
        As = [torch.randn(M, shapes[i][1], generator=g).half() for i in idx]
        ys = q4.gemv_grouped([dev(a) for a in As], [sts[i] for i in idx])
        for i, a, y in zip(idx, As, ys):
            N, K = shapes[i]
            ref = oracle.gemv_reference(bits(a), False, osts[i], N, K)
            assert_matmul_close(y, ref)
    ws = q4._ws.get((torch.cuda.current_device(), "gemv"))
    torch.cuda.synchronize()
    assert ws is not None and int(ws.count_nonzero().item()) == 0


@pytest.mark.parametrize("qtype,bs,dq", [("nf4", 64, True), ("nf4", 32, False), ("nf4", 256, True),
                                         ("int4_sym", 128, False), ("int4_asym", 128, False)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_quantize_grouped_equals_single_and_oracle(q4, oracle, qtype, bs, dq, dtype):
    """One grouped launch over matrices of different (ragged) shapes gives,
    bit for bit, the states q4.quantize gives for each and the oracle's;
    twice in a row (the workspace is left zeroed)."""
    g = torch.Generator().manual_seed(40 + bs)
    shapes = [(300, 1024), (17, 96), (1024, 4096), (5, 7), (2048, 1088)]
    Ws = [(torch.randn(N, K, generator=g) * 0.02).to(dtype) for N, K in shapes]
    Ws[2].view(-1)[::997] *= 20
    for _ in range(2):
        sts = q4.quantize_grouped([dev(W) for W in Ws], bs, qtype, dq)
        torch.cuda.synchronize()
        for W, st in zip(Ws, sts):
            assert_state_equal(st, oracle_state(oracle, W, bs, QT[qtype], dq))
            single = q4.quantize(dev(W), bs, qtype, dq)
            assert_state_equal(single, oracle_state(oracle, W, bs, QT[qtype], dq))
    ws = q4._ws.get((torch.cuda.current_device(), "quantize"))
    if ws is not None:
        assert int(ws.count_nonzero().item()) == 0


def test_quantize_grouped_7b_layer_mean_many_chunks(q4, oracle):
    """The 7B layer in one grouped call: matrices of 1024 and 2752 chunks, so
    the double-quant mean crosses subtrees of 2048 chunk sums."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    Ws = wl.layer_weights(wl.LAYER_7B, 0.02, seed=300)
    sts = q4.quantize_grouped([dev(W) for W in Ws], 64, "nf4", True)
    for W, st in zip(Ws, sts):
        assert_state_equal(st, oracle_state(oracle, W, 64, 0, True))


@pytest.mark.gpu
@pytest.mark.parametrize("qtype,bs,dq", [("nf4", 64, True), ("nf4", 32, False), ("int4_sym", 128, False),
                                         ("int4_asym", 256, False)])
@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_dequantize_grouped_equals_single_and_oracle(q4, oracle, qtype, bs, dq, out_dtype):
    """One grouped dequantize launch over ragged shapes (spans that end
    mid-matrix, matrices smaller than one span) writes, bit for bit, what
    q4.dequantize writes for each matrix and what the oracle computes."""
    g = torch.Generator().manual_seed(70 + bs)
    shapes = [(3, 256), (300, 1024), (1, 256), (1024, 4096), (17, 768), (2048, 1280)]
    Ws = [(torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16) for N, K in shapes]
    sts = q4.quantize_grouped([dev(W) for W in Ws], bs, qtype, dq)
    outs = q4.dequantize_grouped(sts, out_dtype)
    torch.cuda.synchronize()
    for W, st, o in zip(Ws, sts, outs):
        single = q4.dequantize(st, out_dtype)
        assert torch.equal(o.view(torch.int16), single.view(torch.int16))
        ost = oracle_state(oracle, W, bs, QT[qtype], dq)
        assert np.array_equal(bits(o), oracle.dequantize(ost, out_dtype == torch.bfloat16))


# ------------------------------------------------------- binary16 scales --
# robotsatlas.com, "INT4", "Components": the per-group scale "usually stored
# in FP16".

@pytest.mark.parametrize("qtype", ["int4_sym", "int4_asym"])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_fp16_scales_quantize_dequantize(q4, oracle, qtype, bs, dtype):
    """Binary16 group scales: the single and the grouped quantize give the
    oracle's state bit for bit (codes taken against the rounded scale) on
    ragged shapes with tiny and large groups; dequantize is bit-exact too."""
    g = torch.Generator().manual_seed(90 + bs)
    shapes = [(300, 1024), (17, 96 * 2), (5, 7 * 32)]
    Ws = [torch.randn(N, K, generator=g) * 0.02 for N, K in shapes]
    Ws[0][3] *= 1e-5  # scales that round to binary16 subnormals
    Ws[0][5] *= 3e3
    Ws = [W.to(dtype) for W in Ws]
    grouped = q4.quantize_grouped([dev(W) for W in Ws], bs, qtype, False, scale_f16=True)
    for W, gst in zip(Ws, grouped):
        ost = oracle_state(oracle, W, bs, QT[qtype], False, scale_f16=True)
        assert_state_equal(gst, ost)
        st = q4.quantize(dev(W), bs, qtype, False, scale_f16=True)
        assert_state_equal(st, ost)
        for out_dt in (torch.float16, torch.bfloat16):
            d = q4.dequantize(st, out_dt)
            assert np.array_equal(bits(d), oracle.dequantize(ost, out_dt == torch.bfloat16))


@pytest.mark.parametrize("qtype,M", [("int4_sym", 1), ("int4_sym", 16), ("int4_sym", 24),
                                     ("int4_asym", 4), ("int4_asym", 32)])
def test_fp16_scales_gemv(q4, oracle, qtype, M):
    """Both decode kernels read binary16 scales: the GEMV of a binary16-scale
    state against the oracle's product of its dequantized weights."""
    g = torch.Generator().manual_seed(95 + M)
    N, K = 1000, 4096
    W = (torch.randn(N, K, generator=g) * 0.02).bfloat16()
    A = torch.randn(M, K, generator=g).half()
    st = q4.quantize(dev(W), 128, qtype, False, scale_f16=True)
    ost = oracle_state(oracle, W, 128, QT[qtype], False, scale_f16=True)
    y = q4.gemv(dev(A), st)
    ref = oracle.gemv_reference(bits(A), False, ost, N, K)
    assert_matmul_close(y, ref)


@pytest.mark.parametrize("qtype", ["int4_sym", "int4_asym"])
def test_fp16_scales_gemm(q4, oracle, qtype):
    """The GEMM reads binary16 scales; against the oracle at M = 300."""
    g = torch.Generator().manual_seed(99)
    M, N, K = 300, 272, 4608
    W = (torch.randn(N, K, generator=g) * 0.02).bfloat16()
    A = torch.randn(M, K, generator=g).bfloat16()
    st = q4.quantize(dev(W), 64, qtype, False, scale_f16=True)
    ost = oracle_state(oracle, W, 64, QT[qtype], False, scale_f16=True)
    y = q4.gemm(dev(A), st)
    w16 = oracle.dequantize(ost, True).reshape(N, K)
    ref = oracle.matmul(bits(A), True, w16, True, M, N, K)
    assert_matmul_close(y, ref)

"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and its host-side logic (state sizes, codebook, decision
thresholds) agrees with the pages and the oracle.  No kernel runs here."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from conftest import ROOT, read_golden

HEADER = os.path.join(ROOT, "include", "q4.h")


@pytest.fixture(scope="session")
def lib():
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4
    return q4.library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"Q4_API\s+(?:int|const char \*)\s*(q4_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for want in ["q4_quantize", "q4_dequantize", "q4_gemv", "q4_gemm", "q4_state_sizes"]:
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    out = os.popen(f"nm -D --defined-only {lib._name}").read()
    exported = set(re.findall(r" T (q4_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    # nothing else leaks out of the library's C ABI
    assert exported == set(names)
    for n in names:
        assert hasattr(lib, n)


def test_strerror(lib):
    assert lib.q4_strerror(0) == b"ok"
    for code in range(-7, 0):
        assert lib.q4_strerror(code) not in (b"ok", b"unknown error")


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_no_cpu_fallback(lib):
    from bit_blockwise_weight_absmax_b200 import q4
    assert lib.q4_check_device() == -4  # Q4_ERR_NO_DEVICE
    w = torch.zeros(64, 64, dtype=torch.float16)
    with pytest.raises(q4.Q4Error):
        q4.quantize(w)


def test_codebook_is_the_printed_table(lib):
    from bit_blockwise_weight_absmax_b200 import q4
    got = np.array(q4.nf4_levels(), dtype=np.float32)
    want = np.array([float(r[0]) for r in read_golden("nf4_levels.txt")], dtype=np.float32)
    assert got.tobytes() == want.tobytes()


def test_thresholds_reproduce_oracle_nearest_coding(lib, oracle):
    """code = #{i : x >= t_i} with the library's derived thresholds equals the
    oracle's brute-force argmin on every finite fp16/bf16 value in [-1, 1]
    and around every threshold."""
    from bit_blockwise_weight_absmax_b200 import q4
    t = np.array(q4.nf4_thresholds(), dtype=np.float32)
    assert np.all(np.diff(t) > 0)
    bits = np.arange(65536, dtype=np.uint32)
    xs = [bits.astype(np.uint16).view(np.float16).astype(np.float32), (bits << 16).view(np.float32)]
    near = []
    for v in t:
        g = v
        for _ in range(4):
            g = np.nextafter(g, np.float32(-2))
        for _ in range(9):
            near.append(g)
            g = np.nextafter(g, np.float32(2))
    xs.append(np.array(near, dtype=np.float32))
    x = np.concatenate(xs)
    x = x[np.isfinite(x) & (np.abs(x) <= 1)]
    x = np.unique(x)
    codes_t = (x[:, None] >= t[None, :]).sum(1)
    # oracle: quantize blocks [x, 1.0] as binary32 values via its per-element coder
    idx = np.linspace(0, x.size - 1, 4000).astype(int)
    for j in idx:
        assert codes_t[j] == oracle.nf4_code(float(x[j])), x[j]
    for v in near:
        assert (np.float32(v) >= t).sum() == oracle.nf4_code(float(v))


@pytest.mark.parametrize("qtype", [0, 1, 2])
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
def test_state_sizes_match_oracle_storage(lib, oracle, qtype, bs):
    from bit_blockwise_weight_absmax_b200 import q4
    for n in [1, 7, 64, 1000, 256 * 512, 4096 * 4096 + 3]:
        for dq in ([False, True] if qtype == 0 else [False]):
            sz = q4.state_sizes(qtype, n, bs, dq)
            nb = -(-n // bs)
            assert sz[0] == (n + 1) // 2 and sz[1] == 4 * nb
            resident = sz[0] + (sz[3] + sz[4] + sz[5] if dq else sz[1] + sz[2])
            assert resident * 8 / n == pytest.approx(oracle.storage_bits_per_param(qtype, bs, dq, n=n))


def test_state_sizes_storage_arithmetic(lib):
    """learn.pranaymahendrakar.com: 4 + 32/64 = 4.5 bits/param, near 4.127 with
    double quantization (7B-layer-sized tensor)."""
    from bit_blockwise_weight_absmax_b200 import q4
    n = 4096 * 4096
    sz = q4.state_sizes("nf4", n, 64, False)
    assert (sz[0] + sz[1]) * 8 / n == 4.5
    sz = q4.state_sizes("nf4", n, 64, True)
    bits = (sz[0] + sz[3] + sz[4] + sz[5]) * 8 / n
    assert abs(bits - 4.127) < 5e-4


def test_invalid_arguments_rejected_on_host(lib):
    from bit_blockwise_weight_absmax_b200 import q4
    out = (ctypes.c_size_t * 6)()
    assert lib.q4_state_sizes(0, 100, 48, 0, out) == -1     # blocksize
    assert lib.q4_state_sizes(1, 100, 64, 1, out) == -1     # DQ only for NF4
    assert lib.q4_state_sizes(3, 100, 64, 0, out) == -1     # qtype
    assert lib.q4_state_sizes(0, 0, 64, 0, out) == -2       # empty
    with pytest.raises(q4.Q4Error):
        q4.state_sizes("int4_sym", 100, 64, True)


def _fake_state(qtype, rows, cols, bs, dq):
    """A q4_state whose device pointers are placeholders: the host-side
    checks below never dereference them."""
    from bit_blockwise_weight_absmax_b200 import q4
    s = q4._CState()
    s.qtype, s.src_dtype, s.rows, s.cols, s.n = qtype, 1, rows, cols, rows * cols
    s.blocksize, s.double_quant, s.dq_group = bs, int(dq), 256
    s.packed, s.absmax = 0x10000, 0x20000
    s.zero = 0x30000 if qtype == 2 else None
    if dq:
        s.absmax_q, s.absmax_scale, s.absmax_mean = 0x40000, 0x50000, 0x60000
    return s


def _gemv(lib, states, M):
    from bit_blockwise_weight_absmax_b200 import q4
    n = len(states)
    arr = (ctypes.POINTER(q4._CState) * n)(*[ctypes.pointer(s) for s in states])
    ptrs = (ctypes.c_void_p * n)(*([0x70000] * n))
    return lib.q4_gemv_grouped(n, ptrs, arr, ptrs, M, 0, 0, ctypes.c_void_p(0x80000), 1 << 30, None)


def test_gemv_workspace_sizes_per_format(lib):
    """Both decode kernels run one pass for every M <= 32: their slots hold
    8, 16 or 32 columns (M <= 8, <= 16, <= 32).  M outside 1..32 is
    refused."""
    from bit_blockwise_weight_absmax_b200 import q4

    def sizes(qt, bs, dq):
        sts = [_fake_state(qt, 4096, 4096, bs, dq), _fake_state(qt, 11008, 4096, bs, dq)]
        arr = (ctypes.POINTER(q4._CState) * 2)(*[ctypes.pointer(s) for s in sts])

        def size(M):
            out = ctypes.c_size_t(0)
            assert lib.q4_gemv_workspace_size(2, arr, M, ctypes.byref(out)) == 0
            return out.value
        out = ctypes.c_size_t(0)
        assert lib.q4_gemv_workspace_size(2, arr, 33, ctypes.byref(out)) == -2
        assert lib.q4_gemv_workspace_size(2, arr, 0, ctypes.byref(out)) == -2
        return size
    nf4 = sizes(0, 64, True)
    assert nf4(1) == nf4(8) < nf4(9) == nf4(16) < nf4(17) == nf4(32)
    asym = sizes(2, 128, False)
    assert asym(1) == asym(8) < asym(9) == asym(16) < asym(17) == asym(32)


def test_quantize_grouped_workspace_sizes(lib):
    """The grouped quantize needs a workspace only with double quantization:
    256 bytes of counters plus one fp64 sum per 256-block chunk of each
    matrix (256-byte aligned); a matrix of more than 65536 chunks is a shape
    error there (2^30 weights at blocksize 64), and fine without it."""
    def size(shapes, bs, dq):
        n = len(shapes)
        rows = (ctypes.c_int64 * n)(*[r for r, _ in shapes])
        cols = (ctypes.c_int64 * n)(*[c for _, c in shapes])
        out = ctypes.c_size_t(0)
        rc = lib.q4_quantize_grouped_workspace_size(n, rows, cols, bs, 0, int(dq), ctypes.byref(out))
        return rc, out.value
    assert size([(4096, 4096), (11008, 4096)], 64, False) == (0, 0)
    # 1024 and 2752 chunks -> 8192 and 22016 bytes
    assert size([(4096, 4096), (11008, 4096)], 64, True) == (0, 256 + 8192 + 22016)
    assert size([(1, 5)], 64, True) == (0, 256 + 256)
    assert size([(65536, 65536 * 256 * 64 // 65536)], 64, True)[0] == 0          # 65536 chunks
    assert size([(65537, 65536 * 256 * 64 // 65536)], 64, True)[0] == -2         # one row more
    assert size([(65537, 65536 * 256 * 64 // 65536)], 64, False) == (0, 0)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_gemv_host_checks_before_the_device(lib):
    """The GEMV's format checks run on the host, matrix by matrix, before
    any device work: NF4, INT4 symmetric and INT4 asymmetric states pass them
    and stop at the missing GPU; mixed formats in one group are Q4_ERR_ARG;
    M outside 1..32 is a shape error; K not a multiple of the blocksize is
    a shape error."""
    nf4 = _fake_state(0, 256, 512, 64, True)
    sym = _fake_state(1, 256, 512, 128, False)
    asym = _fake_state(2, 256, 512, 128, False)
    assert _gemv(lib, [asym], 1) == -4           # Q4_ERR_NO_DEVICE
    assert _gemv(lib, [asym], 24) == -4
    assert _gemv(lib, [nf4], 1) == -4
    assert _gemv(lib, [sym], 16) == -4
    assert _gemv(lib, [nf4], 32) == -4
    assert _gemv(lib, [nf4, sym], 4) == -1
    assert _gemv(lib, [nf4], 33) == -2
    assert _gemv(lib, [nf4], 0) == -2
    assert _gemv(lib, [_fake_state(0, 256, 96, 64, False)], 1) == -2


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_gemm_host_checks_before_the_device(lib):
    """The GEMM takes every format and blocksize: each passes the host checks
    and stops at the missing GPU; a grouped call of mixed formats or
    blocksizes is Q4_ERR_ARG; K not a multiple of 64 or of the blocksize,
    or N not a multiple of 16, is a shape error."""
    from bit_blockwise_weight_absmax_b200 import q4
    P = ctypes.POINTER(q4._CState)

    def gemm(states, M=512):
        n = len(states)
        arr = (P * n)(*[ctypes.pointer(st) for st in states])
        ptrs = (ctypes.c_void_p * n)(*([0x70000] * n))
        return lib.q4_gemm_grouped(n, ptrs, arr, ptrs, M, 1, 1, None, 0, None)
    for qt, dq in ((0, False), (0, True), (1, False), (2, False)):
        for bs in (32, 64, 128, 256):
            assert gemm([_fake_state(qt, 256, 1024, bs, dq)]) == -4  # Q4_ERR_NO_DEVICE
    assert gemm([_fake_state(0, 256, 1024, 64, True), _fake_state(1, 256, 1024, 64, False)]) == -1
    assert gemm([_fake_state(1, 256, 1024, 64, False), _fake_state(1, 256, 1024, 128, False)]) == -1
    assert gemm([_fake_state(1, 256, 96, 32, False)]) == -2      # K % 64
    assert gemm([_fake_state(1, 256, 384, 256, False)]) == -2    # K % B
    assert gemm([_fake_state(2, 250, 1024, 128, False)]) == -2   # N % 16


def test_gemm_workspace_size_host_checks(lib):
    """The GEMM workspace size takes the same shape and format checks as
    the GEMM (mixed formats Q4_ERR_ARG, K % 64 a shape error) before it
    asks for the device (its plan depends on the SM count)."""
    from bit_blockwise_weight_absmax_b200 import q4
    P = ctypes.POINTER(q4._CState)

    def size(states, M=512):
        arr = (P * len(states))(*[ctypes.pointer(st) for st in states])
        out = ctypes.c_size_t(7)
        return lib.q4_gemm_workspace_size(len(states), arr, M, ctypes.byref(out))
    assert size([_fake_state(0, 256, 1024, 64, True)]) == -4  # Q4_ERR_NO_DEVICE
    assert size([_fake_state(0, 256, 1024, 64, True), _fake_state(1, 256, 1024, 64, False)]) == -1
    assert size([_fake_state(1, 256, 96, 32, False)]) == -2
    assert size([_fake_state(0, 256, 1024, 64, True)], M=0) == -2
    arr = (P * 1)(ctypes.pointer(_fake_state(0, 256, 1024, 64, True)))
    assert lib.q4_gemm_workspace_size(1, arr, 512, None) == -1


def _plan(lib, shapes, M, sms=148, ws=2 ** 64 - 1):
    """q4_gemm_plan_info over fake NF4 (B=64, double-quantized) states of
    the given (N, K) shapes: (return code, tile_m, grid, cut tiles)."""
    from bit_blockwise_weight_absmax_b200 import q4
    P = ctypes.POINTER(q4._CState)
    sts = [_fake_state(0, N, K, 64, True) for N, K in shapes]
    arr = (P * len(sts))(*[ctypes.pointer(st) for st in sts])
    tm, grid, cut = ctypes.c_int32(-7), ctypes.c_int32(-7), ctypes.c_int64(-7)
    rc = lib.q4_gemm_plan_info(len(sts), arr, M, sms, ws, ctypes.byref(tm), ctypes.byref(grid), ctypes.byref(cut))
    return rc, tm.value, grid.value, cut.value


def test_gemm_plan_tile_height_and_cuts(lib):
    """The GEMM's host planner (no device): 512-token tiles when there are
    enough of them to fill the SMs, 256-token tiles for M <= 256 and for
    launches of few tiles, k-cuts only with a workspace and only where they
    take at least a tenth off the busiest CTA."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    layer = [(N, K) for _, N, K in wl.LAYER_7B]
    # the 7B layer at prefill sizes: 332 (1328) tall tiles, none cut
    assert _plan(lib, layer, 512) == (0, 512, 148, 0)
    assert _plan(lib, layer, 2048) == (0, 512, 148, 0)
    # M <= 256: one token half per tile either way, so two accumulators
    assert _plan(lib, layer, 64)[:2] == (0, 256)
    assert _plan(lib, layer, 256)[:2] == (0, 256)
    # one 4096 x 4096 matrix at M = 512: 32 tall tiles would leave 116 SMs
    # idle; 64 half-height tiles cut in k give 128 items
    assert _plan(lib, [(4096, 4096)], 512) == (0, 256, 128, 64)
    assert _plan(lib, [(4096, 4096)], 512, ws=0) == (0, 256, 64, 0)  # no workspace, no cuts
    # the GPU tests' shapes for the tall tiles' lone first half and cut tall tiles
    assert _plan(lib, [(10240, 512)], 700) == (0, 512, 148, 0)
    assert _plan(lib, [(10240, 512)], 600)[:2] == (0, 512)
    assert _plan(lib, [(9440, 512)], 700) == (0, 512, 148, 0)  # a ragged last weight tile
    assert _plan(lib, [(1024, 2048)], 512)[:2] == (0, 256)  # the timeout test's other shape
    # more tiles than a list holds: whole tall tiles round robin
    assert _plan(lib, [(27648, 256)], 5000) == (0, 512, 148, 0)
    assert _plan(lib, [(2560, 16384)], 1000) == (0, 512, 80, 40)
    # fewer SMs: the same layer still takes tall tiles, and the grid follows
    assert _plan(lib, layer, 512, sms=74) == (0, 512, 74, 0)
    # cuts only within the workspace: 64 KB of counters, then one 512 KB
    # fp32 slot per cut tile (128 weight rows x 512 tokens x two halves)
    need = 65536 + 64 * 524288
    assert _plan(lib, [(4096, 4096)], 512, ws=need) == (0, 256, 128, 64)
    assert _plan(lib, [(4096, 4096)], 512, ws=need - 1) == (0, 256, 64, 0)
    # argument and shape checks, before any device is asked for
    assert _plan(lib, layer, 512, sms=0)[0] == -1
    assert _plan(lib, layer, 512, sms=1025)[0] == -1
    assert _plan(lib, layer, 0)[0] == -2
    assert _plan(lib, [(4096, 4000)], 512)[0] == -2  # K % 64


def test_grouped_calls_reject_a_null_entry_before_any_use(lib):
    """A NULL state, activation or output pointer in any entry of a grouped
    call is Q4_ERR_ARG, found before the library reads any entry (a NULL
    second state used to be dereferenced while sizing the workspace)."""
    from bit_blockwise_weight_absmax_b200 import q4
    good = _fake_state(0, 256, 512, 64, True)
    P = ctypes.POINTER(q4._CState)
    for M in (1, 24):
        arr = (P * 2)(ctypes.pointer(good), P())
        ptrs = (ctypes.c_void_p * 2)(0x70000, 0x70000)
        assert lib.q4_gemv_grouped(2, ptrs, arr, ptrs, M, 0, 0, ctypes.c_void_p(0x80000), 1 << 30, None) == -1
        assert lib.q4_gemm_grouped(2, ptrs, arr, ptrs, 512, 1, 1, None, 0, None) == -1
        arr = (P * 2)(ctypes.pointer(good), ctypes.pointer(good))
        for bad in ((ctypes.c_void_p * 2)(0x70000, None),):
            assert lib.q4_gemv_grouped(2, bad, arr, ptrs, M, 0, 0, ctypes.c_void_p(0x80000), 1 << 30, None) == -1
            assert lib.q4_gemv_grouped(2, ptrs, arr, bad, M, 0, 0, ctypes.c_void_p(0x80000), 1 << 30, None) == -1
            assert lib.q4_gemm_grouped(2, bad, arr, ptrs, 512, 1, 1, None, 0, None) == -1
            assert lib.q4_gemm_grouped(2, ptrs, arr, bad, 512, 1, 1, None, 0, None) == -1


def test_binary16_scale_sizes_and_checks(lib, oracle):
    """Q4_SCALE_F16 (INT4 only): the scale buffer is 2 bytes per block, the
    rest of the state unchanged, and the sizes match the oracle's storage
    count; NF4 with the flag is Q4_ERR_ARG, and so is a state that claims
    binary16 scales for NF4."""
    from bit_blockwise_weight_absmax_b200 import q4
    out = (ctypes.c_size_t * 6)()
    n, bs = 100_000, 128
    nb = -(-n // bs)
    for qt in (1, 2):
        assert lib.q4_state_sizes(qt | 0x100, n, bs, 0, out) == 0
        assert out[1] == 2 * nb
        total = sum(out)
        bits = oracle.storage_bits_per_param(qt, bs, False, n, scale_f16=True)
        assert abs(8 * total / n - bits) < 1e-12
    assert lib.q4_state_sizes(0 | 0x100, n, bs, 0, out) == -1
    assert lib.q4_state_sizes(1 | 0x100, n, bs, 1, out) == -1
    st = _fake_state(0, 256, 512, 64, False)
    st.scale_f16 = 1
    P = ctypes.POINTER(q4._CState)
    arr = (P * 1)(ctypes.pointer(st))
    ptrs = (ctypes.c_void_p * 1)(0x70000)
    assert lib.q4_gemm_grouped(1, ptrs, arr, ptrs, 512, 1, 1, None, 0, None) == -1

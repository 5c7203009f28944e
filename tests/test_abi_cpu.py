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

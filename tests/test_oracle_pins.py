"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle's own formulas.

Each test names what pins it: printed values (tests/golden/), library
routines (numpy / torch conversions and matmul), exact rational arithmetic
(fractions.Fraction), closed forms, invariants and brute force on tiny inputs.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def golden_levels():
    return np.array([float(r[0]) for r in read_golden("nf4_levels.txt")], dtype=np.float32)


def golden_storage():
    return {r[0]: float(r[1]) for r in read_golden("storage_arithmetic.txt")}


# ---------------------------------------------------------------- codebook --

def test_codebook_is_the_printed_table(oracle):
    """n4n.ai "Conceptual NF4 dequantization": 16 levels, -1, 0, +1 exact."""
    L = oracle.nf4_levels()
    G = golden_levels()
    assert L.tobytes() == G.tobytes()
    assert np.all(np.diff(L) > 0)
    assert L[0] == -1.0 and L[7] == 0.0 and L[15] == 1.0
    assert (L < 0).sum() == 7 and (L > 0).sum() == 8  # asymmetric: 7 below, 8 above zero


# ------------------------------------------------------- nearest coding ----

def boundary_code(x: float, L) -> int:
    """Nearest level via decision boundaries in exact rationals.

    Independent of argmin: code = number of midpoints strictly below x, plus
    one for a midpoint equal to x whose upper neighbour has the smaller
    magnitude (the tie rule: the level nearer zero wins)."""
    fx = Fraction(float(x))
    code = 0
    for i in range(15):
        lo, hi = Fraction(float(L[i])), Fraction(float(L[i + 1]))
        m = (lo + hi) / 2
        if fx > m or (fx == m and abs(hi) < abs(lo)):
            code += 1
    return code


def _all_16bit(dtype_name):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    if dtype_name == "fp16":
        vals = bits.view(np.float16).astype(np.float32)
    else:
        vals = (bits.astype(np.uint32) << 16).view(np.float32)
    ok = np.isfinite(vals) & (np.abs(vals) <= 1.0)
    return bits[ok], vals[ok]


@pytest.mark.parametrize("dt", ["fp16", "bf16"])
def test_nearest_coding_exhaustive_16bit(oracle, dt):
    """Every finite 16-bit w with |w| <= 1, in blocks [w, 1.0] (so c = 1 and
    x = w): the code equals the exact-rational boundary count."""
    L = golden_levels()
    bits, vals = _all_16bit(dt)
    one = np.float16(1.0).view(np.uint16) if dt == "fp16" else np.uint16(0x3F80)
    blocks = np.empty(2 * bits.size, dtype=np.uint16)
    blocks[0::2] = bits
    blocks[1::2] = one
    st = oracle.quantize(blocks, dt == "bf16", 2, oracle.QT_NF4)
    codes = st.codes()[0::2]
    # exact boundaries, vectorised in binary64 (midpoints of adjacent binary32
    # levels are exact in binary64); ties checked separately below
    mids = np.array([(float(L[i]) + float(L[i + 1])) / 2 for i in range(15)])
    for i in range(15):
        assert Fraction(mids[i]) == (Fraction(float(L[i])) + Fraction(float(L[i + 1]))) / 2
    v = vals.astype(np.float64)
    expect = (v[:, None] > mids[None, :]).sum(1)
    tie = v[:, None] == mids[None, :]
    upper_smaller = np.abs(L[1:].astype(np.float64)) < np.abs(L[:-1].astype(np.float64))
    expect += (tie & upper_smaller[None, :]).sum(1)
    assert np.array_equal(codes, expect)
    # the vectorised count agrees with the rational one on a spread sample
    for j in range(0, vals.size, 997):
        assert boundary_code(vals[j], L) == expect[j]


def test_nearest_coding_at_fp32_boundaries(oracle):
    """At, below and above every midpoint, as binary32 inputs x."""
    L = golden_levels()
    xs = []
    for i in range(15):
        m = (float(L[i]) + float(L[i + 1])) / 2
        f = np.float32(m)
        for d in range(-3, 4):
            g = f
            step = np.float32(np.inf) if d > 0 else np.float32(-np.inf)
            for _ in range(abs(d)):
                g = np.nextafter(g, step)
            xs.append(g)
    for x in xs:
        assert oracle.nf4_code(float(x)) == boundary_code(float(x), L), x


def test_tie_goes_to_smaller_magnitude(oracle):
    """Exactly representable midpoints: the level nearer zero wins."""
    L = golden_levels()
    hit = 0
    for i in range(15):
        m = (Fraction(float(L[i])) + Fraction(float(L[i + 1]))) / 2
        if Fraction(float(np.float32(float(m)))) != m:
            continue
        hit += 1
        want = i if abs(L[i]) < abs(L[i + 1]) else i + 1
        assert oracle.nf4_code(float(m)) == want
    # -1/-0.696 ... at least the zero-adjacent pairs are exactly representable
    assert hit >= 1


@pytest.mark.parametrize("B", [2, 4, 8])
def test_nearest_coding_random_tiny_blocks(oracle, B):
    """Random fp16 blocks: x = fl32(w / c) (numpy IEEE division), then the
    exact-rational nearest level."""
    L = golden_levels()
    rng = np.random.default_rng(100 + B)
    w = (rng.standard_normal(B * 400) * rng.choice([1e-3, 0.02, 1.0, 300.0], B * 400))
    w16 = w.astype(np.float16)
    st = oracle.quantize(w16.view(np.uint16), False, B, oracle.QT_NF4)
    codes = st.codes()
    wf = w16.astype(np.float32).reshape(-1, B)
    c = np.abs(wf).max(1)
    assert np.array_equal(st.absmax, c)  # absmax is exact: the max of 16-bit values
    with np.errstate(invalid="ignore"):
        x = np.where(c[:, None] == 0, np.float32(0), wf / c[:, None]).reshape(-1)
    expect = np.array([boundary_code(v, L) for v in x])
    assert np.array_equal(codes, expect)


def test_absmax_element_maps_to_endpoint(oracle):
    w = torch.randn(64 * 50, generator=torch.Generator().manual_seed(3)).mul(0.02).half()
    st = oracle.quantize(w.numpy().view(np.uint16), False, 64, oracle.QT_NF4)
    wf = w.float().numpy().reshape(-1, 64)
    codes = st.codes().reshape(-1, 64)
    i = np.abs(wf).argmax(1)
    top = codes[np.arange(codes.shape[0]), i]
    sign = np.sign(wf[np.arange(wf.shape[0]), i])
    assert np.all(np.where(sign > 0, top == 15, top == 0))


def test_zero_block(oracle):
    w = np.zeros(128, dtype=np.float16)
    w[5] = -0.0
    st = oracle.quantize(w.view(np.uint16), False, 64, oracle.QT_NF4)
    assert np.all(st.absmax == 0) and np.all(st.codes() == 7)
    d = oracle.dequantize(st, False).view(np.float16)
    assert np.all(d == 0)


# --------------------------------------------------------- grid round trip --

@pytest.mark.parametrize("dt", ["fp16", "bf16"])
def test_grid_values_round_trip_exactly(oracle, dt):
    """Inputs already on the grid, w = cvt(c * L_k) with power-of-two c and
    the absmax element present: quantize -> dequantize returns them."""
    L = golden_levels()
    tt = torch.float16 if dt == "fp16" else torch.bfloat16
    for c in [1.0, 0.5, 2.0 ** -6, 8.0, 2.0 ** 10]:
        vals = torch.tensor(np.float32(c) * L, dtype=torch.float32).to(tt)
        block = torch.cat([vals, vals.flip(0), vals, vals.flip(0)])  # 64 elements
        bits = block.view(torch.int16).numpy().view(np.uint16)
        st = oracle.quantize(bits, dt == "bf16", 64, oracle.QT_NF4)
        assert st.absmax[0] == np.float32(c)
        codes = st.codes()
        assert np.array_equal(codes[:16], np.arange(16))
        back = oracle.dequantize(st, dt == "bf16")
        assert np.array_equal(back, bits)


@pytest.mark.parametrize("dt", ["fp16", "bf16"])
def test_quantize_is_idempotent(oracle, dt):
    """codes(Q(DQ(Q(W)))) == codes(Q(W)) and the absmax is preserved (no
    block so small that c * L_k underflows the 16-bit format)."""
    tt = torch.float16 if dt == "fp16" else torch.bfloat16
    w = torch.randn(256 * 64, generator=torch.Generator().manual_seed(9)).mul(0.02).to(tt)
    bits = w.view(torch.int16).numpy().view(np.uint16)
    st1 = oracle.quantize(bits, dt == "bf16", 64, oracle.QT_NF4)
    back = oracle.dequantize(st1, dt == "bf16")
    st2 = oracle.quantize(back, dt == "bf16", 64, oracle.QT_NF4)
    assert np.array_equal(st1.codes(), st2.codes())
    assert np.array_equal(st1.absmax, st2.absmax)


# ------------------------------------------------------------------ pack ----

def test_packing_low_nibble_first(oracle):
    """n4n.ai dequantize_nf4 unpacks `p & 0xF` then `(p >> 4) & 0xF`: element
    2j is the low nibble of byte j.  Odd n: the last high nibble is 0."""
    L = golden_levels()
    vals = np.array([L[3], L[12], L[0], L[15], L[7]], dtype=np.float16)  # c = 1 via L[15]
    st = oracle.quantize(vals.view(np.uint16), False, 64, oracle.QT_NF4)
    assert list(st.packed) == [3 | (12 << 4), 0 | (15 << 4), 7]


def test_snippet_restatement_matches_fp32_product(oracle):
    """A numpy restatement of the page's dequantize_nf4 (NF4_VALUES[idx]
    viewed per block times the block scale), in binary32, equals the
    oracle's product before rounding, bit for bit."""
    w = torch.randn(64 * 40 + 64, generator=torch.Generator().manual_seed(5)).mul(0.02).half()
    st = oracle.quantize(w.numpy().view(np.uint16), False, 64, oracle.QT_NF4)
    NF4_VALUES = golden_levels()
    p = st.packed
    indices = np.stack([p & 0xF, (p >> 4) & 0xF], axis=-1).reshape(-1)
    snippet = NF4_VALUES[indices].reshape(-1, 64) * st.absmax.reshape(-1, 1)
    assert snippet.dtype == np.float32
    assert np.array_equal(snippet.reshape(-1).view(np.uint32),
                          oracle.dequantize_f32(st).view(np.uint32))
    # and the 16-bit output is that product rounded once (numpy's cast)
    assert np.array_equal(snippet.reshape(-1).astype(np.float16).view(np.uint16),
                          oracle.dequantize(st, False))


def test_ragged_tail_block(oracle):
    n = 64 * 3 + 17
    w = torch.randn(n, generator=torch.Generator().manual_seed(4)).mul(0.02).half()
    st = oracle.quantize(w.numpy().view(np.uint16), False, 64, oracle.QT_NF4)
    assert st.absmax.size == 4 and st.packed.size == (n + 1) // 2
    assert st.absmax[3] == np.abs(w[192:].float().numpy()).max()
    assert (st.packed[-1] >> 4) == 0  # odd n: final high nibble is padding


# --------------------------------------------------------------- INT4 sym ---

def test_int4_sym_scale_and_levels(oracle):
    """n4n.ai "INT4 symmetric": levels -8..7, scale max|w|/7."""
    w = torch.randn(128 * 64, generator=torch.Generator().manual_seed(11)).mul(0.02).bfloat16()
    bits = w.view(torch.int16).numpy().view(np.uint16)
    st = oracle.quantize(bits, True, 128, oracle.QT_INT4_SYM)
    wf = w.float().numpy().reshape(-1, 128)
    c = np.abs(wf).max(1)
    s = st.absmax
    # s is max|w|/7 up to the one rounding of the division
    assert np.all(np.abs(s.astype(np.float64) * 7 - c) <= np.spacing(c.astype(np.float32)) * 4)
    q = st.codes().astype(np.int16).reshape(-1, 128)
    q = np.where(q >= 8, q - 16, q)
    assert q.min() >= -7 and q.max() <= 7  # -8 is never produced
    i = np.abs(wf).argmax(1)
    top = q[np.arange(q.shape[0]), i]
    assert np.all(np.abs(top) == 7)
    # brute force: q is the integer in [-8, 7] nearest x = fl32(w/s), ties even
    x = (wf / s[:, None]).astype(np.float32)
    for r in range(0, x.shape[0], 7):
        for j in range(0, 128, 5):
            fx = Fraction(float(x[r, j]))
            best = min(range(-8, 8), key=lambda k: (abs(fx - k), k % 2))
            assert q[r, j] == best
    # dequantization: one binary32 multiply, one rounding (numpy) to bf16 bits
    deq = oracle.dequantize(st, True)
    prod = (q.astype(np.float32) * s[:, None]).reshape(-1)
    want = torch.from_numpy(prod).bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(deq, want)


# -------------------------------------------------------------- INT4 asym ---

def test_int4_asym_zero_point(oracle):
    """robotsatlas "INT4": range fit into [0, 15] with an integer zero-point."""
    g = torch.Generator().manual_seed(12)
    w = (torch.randn(128 * 64, generator=g) * 0.02 + 0.01).half()
    w[:128] = torch.rand(128, generator=g).half()  # an all-positive group: mn = 0
    w[128:256] = -torch.rand(128, generator=g).half()  # all negative: mx = 0
    w[300] = 0.0
    st = oracle.quantize(w.numpy().view(np.uint16), False, 128, oracle.QT_INT4_ASYM)
    nb = 64
    z = np.stack([st.zero & 0xF, st.zero >> 4], -1).reshape(-1)[:nb].astype(np.int32)
    q = st.codes().astype(np.int32).reshape(nb, 128)
    wf = w.float().numpy().reshape(nb, 128)
    s = st.absmax
    assert z.min() >= 0 and z.max() <= 15 and q.min() >= 0 and q.max() <= 15
    assert z[0] == 0 and z[1] == 15
    # zero encodes exactly: the element w = 0 has q == z and dequantizes to 0
    assert q[300 // 128, 300 % 128] == z[300 // 128]
    deq = oracle.dequantize(st, False).view(np.float16).astype(np.float32).reshape(nb, 128)
    assert deq[300 // 128, 300 % 128] == 0.0
    # min / max elements map to 0 / 15 (within rint) for mixed-sign groups
    for b in range(2, nb):
        assert q[b, wf[b].argmin()] == 0
        assert q[b, wf[b].argmax()] in (14, 15)
    # brute force: q = argmin over 0..15 of |x - (q - z)|, x = fl32(w / s), ties even
    for b in range(0, nb, 5):
        x = (wf[b] / s[b]).astype(np.float32)
        for j in range(0, 128, 9):
            fx = Fraction(float(x[j]))
            best = min(range(16), key=lambda k: (abs(fx - (k - z[b])), (k - z[b]) % 2))
            assert q[b, j] == best
    # dequantization: (q - z) * s, one multiply, one rounding (numpy)
    prod = ((q - z[:, None]).astype(np.float32) * s[:, None]).astype(np.float16)
    assert np.array_equal(prod.astype(np.float32), deq)


# -------------------------------------------------------- double quantization

def test_pairwise_sum_order(oracle):
    """The fixed order: adjacent pairs level by level, odd last carried up."""
    assert oracle.pairwise_sum([1.0, 2.0, 3.0]) == 6.0
    # (1e16 + 1) + (-1e16 + 1) = 1e16 + (-1e16) = 0, where a left-to-right sum gives 1
    assert oracle.pairwise_sum([1e16, 1.0, -1e16, 1.0]) == 0.0
    # five values: ((a + b) + (c + d)) + e
    a, b, c, d, e = 2.0 ** 53, 1.0, 1.0, 0.0, 1.0
    assert oracle.pairwise_sum([a, b, c, d, e]) == ((a + b) + (c + d)) + e
    assert oracle.pairwise_sum([7.5]) == 7.5


def test_double_quant_state(oracle):
    """learn.pranaymahendrakar.com: the block scales are quantized to 8 bits
    in blocks of 256; the mean is subtracted first."""
    w = torch.randn(1000 * 64 + 40, generator=torch.Generator().manual_seed(21)).mul(0.02)
    w[::997] *= 20
    w = w.bfloat16()
    bits = w.view(torch.int16).numpy().view(np.uint16)
    st = oracle.quantize(bits, True, 64, oracle.QT_NF4, double_quant=True)
    nb = st.nb
    assert nb == 1001 and st.absmax_q.size == nb and st.absmax_scale.size == 4
    # mean: the exact rational sum, rounded to binary64 then binary32
    S = sum(Fraction(float(v)) for v in st.absmax)
    assert oracle.pairwise_sum(st.absmax.astype(np.float64)) == float(S)  # exact here
    mu = np.float32(float(S / nb))
    assert st.absmax_mean[0] == mu
    # per group: |q2| = 127 at the largest deviation; |c~ - c| <= s2/2 + rounding
    for g in range(4):
        cs = st.absmax[g * 256:(g + 1) * 256]
        qs = st.absmax_q[g * 256:(g + 1) * 256].astype(np.int32)
        s2 = st.absmax_scale[g]
        dev = np.abs(cs.astype(np.float64) - float(mu))
        assert abs(qs[dev.argmax()]) == 127
        assert np.float32(dev.max() / 127) == s2 or abs(dev.max() / 127 - s2) <= np.spacing(s2) * 2
        ct = (qs.astype(np.float32) * s2) + mu
        assert np.all(np.abs(ct.astype(np.float64) - cs) <= s2 / 2 + 4 * np.spacing(np.float32(cs.max())))
    # NF4 codes come from the original c, so they equal the no-DQ codes
    st0 = oracle.quantize(bits, True, 64, oracle.QT_NF4)
    assert np.array_equal(st0.codes(), st.codes()) and np.array_equal(st0.absmax, st.absmax)
    # dequantization uses c~: numpy restatement, one multiply, one rounding
    L = golden_levels()
    ctil = (st.absmax_q.astype(np.float32) * np.repeat(st.absmax_scale, 256)[:nb]) + st.absmax_mean[0]
    prod = L[st.codes()] * np.repeat(ctil, 64)[: st.n]
    want = torch.from_numpy(prod.astype(np.float32)).bfloat16().view(torch.int16).numpy()
    assert np.array_equal(oracle.dequantize(st, True), want.view(np.uint16))


# ------------------------------------------------------- 16-bit conversions -

def test_half_and_bf16_decode_all_patterns(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.half_to_float(int(b)) for b in bits], dtype=np.float32)
    fin = np.isfinite(want)
    assert np.array_equal(got[fin], want[fin]) and np.all(np.isnan(got[np.isnan(want)]))
    wantb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    gotb = np.array([oracle.bf16_to_float(int(b)) for b in bits], dtype=np.float32)
    fin = np.isfinite(wantb)
    assert np.array_equal(gotb[fin], wantb[fin]) and np.all(np.isnan(gotb[np.isnan(wantb)]))


def test_float_to_16bit_rounding(oracle):
    """binary32 -> binary16 / bfloat16, ties to even: numpy and torch casts."""
    rng = np.random.default_rng(7)
    xs = [rng.standard_normal(20000).astype(np.float32) * s for s in (1e-6, 1e-3, 1, 1e3, 6e4)]
    h = np.arange(0, 0x7C00, 7, dtype=np.uint16).view(np.float16).astype(np.float32)
    mids = ((h[:-1].astype(np.float64) + h[1:]) / 2).astype(np.float32)  # many exact ties
    edge = np.array([65504, 65519.996, 65520, 65536, 1e38, 2 ** -24, 2 ** -25, 3 * 2 ** -26,
                     2 ** -14, 2 ** -133, 2 ** -134, 3.389e38, 3.3895e38, 0, -0.0], np.float32)
    x = np.concatenate(xs + [mids, -mids, edge, -edge])
    got = np.array([oracle.float_to_half(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, x.astype(np.float16).view(np.uint16))
    gotb = np.array([oracle.float_to_bf16(float(v)) for v in x], dtype=np.uint16)
    wantb = torch.from_numpy(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(gotb, wantb)


# ------------------------------------------------------------------ matmul --

def test_matmul_exact_small_integers(oracle):
    """A in {-1, 0, 1}, W small integers times a power of two: exact."""
    rng = np.random.default_rng(3)
    M, N, K = 3, 7, 64
    A = rng.integers(-1, 2, size=(M, K)).astype(np.float16)
    W = (rng.integers(-8, 8, size=(N, K)) * 0.25).astype(np.float16)
    y = oracle.matmul(A.view(np.uint16), False, W.view(np.uint16), False, M, N, K)
    want = A.astype(np.int64 if False else np.float64) @ W.astype(np.float64).T
    assert np.array_equal(y, want)
    rows = np.array([6, 0, 3])
    y2 = oracle.matmul(A.view(np.uint16), False, W.view(np.uint16), False, M, N, K, rows)
    assert np.array_equal(y2, want[:, rows])


def test_matmul_matches_numpy_fp64(oracle):
    g = torch.Generator().manual_seed(8)
    A = torch.randn(4, 300, generator=g).bfloat16()
    W = torch.randn(50, 300, generator=g).mul(0.02).bfloat16()
    y = oracle.matmul(A.view(torch.int16).numpy().view(np.uint16), True,
                      W.view(torch.int16).numpy().view(np.uint16), True, 4, 50, 300)
    want = A.double().numpy() @ W.double().numpy().T
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------ storage arithmetic --

def test_storage_arithmetic_matches_pages(oracle):
    G = golden_storage()
    nodq = oracle.storage_bits_per_param(oracle.QT_NF4, 64, False)
    dq = oracle.storage_bits_per_param(oracle.QT_NF4, 64, True)
    assert nodq - 4 == G["nf4_b64_absmax_bits"]
    assert abs((dq - 4) - G["nf4_b64_dq_overhead_bits_approx"]) < 5e-4
    assert abs(dq - G["nf4_b64_dq_total_bits_approx"]) < 5e-4
    assert abs((nodq - dq) - G["dq_saving_bits_approx"]) < 0.05
    # 7B: 14.00 GB at fp16, 3.67 GB at 4.2 bits, 3.8x
    p = G["params_7b"]
    assert f"{p * 2 / 1e9:.2f}" == f"{G['fp16_gb_7b']:.2f}"
    gb42 = p * G["int4_bits_7b"] / 8 / 1e9
    assert f"{gb42:.2f}" == f"{G['int4_gb_7b']:.2f}"
    assert f"{(p * 2 / 1e9) / gb42:.1f}" == f"{G['compression_7b']:.1f}"
    # our NF4 + DQ format at the same 7e9 parameters is below the page's 4.2-bit figure
    assert p * dq / 8 / 1e9 < G["int4_gb_7b"]
    # the 70B-shaped stack, exact state sizes: inside "~35-40 GB", near "~37 GB"
    from bit_blockwise_weight_absmax_b200.workloads import LAYER_70B, N_LAYERS_70B
    total_bits = sum(oracle.storage_bits_per_param(oracle.QT_NF4, 64, True, n=N * K) * N * K
                     for _, N, K in LAYER_70B) * N_LAYERS_70B
    gb = total_bits / 8 / 1e9
    assert G["int4_gb_70b_lo"] <= gb <= G["int4_gb_70b_hi"]
    assert abs(gb - G["int4_gb_70b_approx"]) < 2.5
    params70 = sum(N * K for _, N, K in LAYER_70B) * N_LAYERS_70B
    assert abs(params70 * 2 / 1e9 - G["fp16_gb_70b"]) < 5  # "140 GB" at fp16
    # n4n.ai metadata table: fp16 scales, 8 Gi params / g * 2 bytes (MiB), % of 4000 MB
    for g, key in [(128, "meta_g128"), (64, "meta_g64"), (32, "meta_g32")]:
        mib = G["meta_params"] / 1e9 * 2 ** 30 / g * 2 / 2 ** 20
        assert mib == G[key + "_mb"]
        assert round(mib / (G["meta_weights_gb"] * 1000) * 100, 1) == G[key + "_pct"]


# ------------------------------------- INT4 asym: closed forms, exactly -----
# robotsatlas.com, "INT4", "How it works": each group's range is fit into
# [0, 15]; "Components" (Zero-point): an integer offset lets a group whose
# values are not centred on zero use all 16 levels.  With the range widened
# to include 0 (so 0 stays exactly representable), the scale is the range
# over the 15 steps between level 0 and level 15, and the zero-point is the
# level that 0 falls on.  These pins evaluate that closed form with exact
# rationals on the exact 16-bit inputs, rounding to binary32 only where a
# binary32 operation stands: the difference, the quotient by 15, -mn / s.

def _rne32(x: Fraction) -> Fraction:
    """Round an exact rational to the nearest binary32 (ties to even)."""
    if x == 0:
        return Fraction(0)
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)  # subnormal quantum below 2^-126
    quantum = Fraction(2) ** (e - 23)
    r = round(a / quantum)  # Python rounds a Fraction half to even
    return (r * quantum) if x > 0 else -(r * quantum)


def _keep(x: Fraction) -> Fraction:
    return x


def _to_half(x: Fraction) -> Fraction:
    """The binary16 value nearest to the binary32 value x (numpy's IEEE
    conversion, ties to even, overflow to infinity)."""
    h = np.float16(float(x))
    return Fraction(float(h)) if np.isfinite(h) else h


def int4_asym_pin_failures(wf: np.ndarray, st, scale_round=_keep) -> list:
    """Every closed-form check that the state of INT4 asymmetric groups
    (rows of `wf`, the exact binary32 values of the 16-bit inputs) fails.
    scale_round: the storage rounding of s (binary16 scales: codes and
    zero-points are formed against the rounded s)."""
    nb, B = wf.shape
    z = np.stack([st.zero & 0xF, st.zero >> 4], -1).reshape(-1)[:nb].astype(np.int64)
    q = st.codes().astype(np.int64).reshape(nb, B)
    bad = []
    for b in range(nb):
        vals = [Fraction(float(v)) for v in wf[b]]
        mn, mx = min(min(vals), Fraction(0)), max(max(vals), Fraction(0))
        s = scale_round(_rne32(_rne32(mx - mn) / 15))
        if not isinstance(s, Fraction):  # binary16 overflow: every quotient is 0
            if not np.isinf(st.absmax[b]) or z[b] != 0 or np.any(q[b] != 0):
                bad.append(("inf-scale", b))
            continue
        if Fraction(float(st.absmax[b])) != s:
            bad.append(("scale", b))
            continue
        if s == 0:
            if z[b] != 0 or np.any(q[b] != 0):
                bad.append(("zero-range", b))
            continue
        zz = min(max(round(_rne32(-mn / s)), 0), 15)
        if z[b] != zz:
            bad.append(("zero-point", b))
            continue
        # the dequantized ends of the level range sit within s/2 (plus the
        # binary32 roundings of s) of the widened group minimum and maximum;
        # a binary16 s may be off by half its ulp, 15 times over
        slack = s / 2 + abs(mx - mn) * Fraction(1, 2 ** 22)
        if scale_round is not _keep:
            slack += 15 * s / 2 ** 11 + Fraction(15, 2 ** 25)
        if abs(-zz * s - mn) > slack or abs((15 - zz) * s - mx) > slack:
            bad.append(("endpoints", b))
        for j in range(B):
            qq = min(max(round(_rne32(vals[j] / s)) + zz, 0), 15)
            if q[b, j] != qq:
                bad.append(("code", b, j))
                break
    return bad


def _asym_groups(dt, seed):
    """Groups of 32 covering the cases the rule distinguishes: centred and
    offset Gaussians, all-positive and all-negative groups (the widening to
    0), constant and all-zero groups, tiny and large magnitudes."""
    g = torch.Generator().manual_seed(seed)
    B = 32
    rows = [torch.randn(B, generator=g) * 0.02 + off for off in (0.0, 0.01, -0.015, 0.05)]
    rows += [torch.rand(B, generator=g) * 0.3 + 0.01, -(torch.rand(B, generator=g) * 0.3 + 0.01)]
    rows += [torch.full((B,), 0.125), torch.zeros(B), torch.randn(B, generator=g) * 1e-4,
             torch.randn(B, generator=g) * 300.0]
    rows += [torch.randn(B, generator=g) * s for s in torch.rand(40, generator=g).mul(4).exp().tolist()]
    w = torch.stack(rows).to(dt)
    return w, B


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_int4_asym_scale_and_zero_point_closed_form(oracle, dt):
    """s = fl32(fl32(mx - mn) / 15) and z = clamp(rint(fl32(-mn / s)), 0, 15)
    on every group, exactly; the levels 0 and 15 dequantize to within s/2 of
    the widened group minimum and maximum."""
    w, B = _asym_groups(dt, 31)
    bits = w.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    st = oracle.quantize(bits, dt == torch.bfloat16, B, oracle.QT_INT4_ASYM)
    assert int4_asym_pin_failures(w.float().numpy(), st) == []


def _mutated_oracle(tmp_path, old, new):
    """The oracle source with one planted mistake, built into its own .so."""
    import ctypes
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle_module_file()), "q4_oracle.c")).read()
    assert src.count(old) == 1, old
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", str(path),
                    "-o", str(so), "-lm"], check=True, capture_output=True)
    lib = ctypes.CDLL(str(so))
    P = ctypes.c_void_p
    lib.oracle_quantize.argtypes = [P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, P, P, P, P, P, P]
    lib.oracle_quantize.restype = None
    return lib


def oracle_module_file():
    import oracle as o
    return o.__file__


@pytest.mark.parametrize("old,new", [
    ("float s = (mx - mn) / 15.0f;", "float s = (mx - mn) / 16.0f;"),
    ("z = clampi((int)rintf(-mn / s), 0, 15);", "z = clampi((int)floorf(-mn / s), 0, 15);"),
    ("q = clampi((int)rintf(to_f32(w[j], is_bf16) / s) + z, 0, 15);",
     "q = clampi((int)floorf(to_f32(w[j], is_bf16) / s) + z, 0, 15);"),
    ("float mn = 0.0f, mx = 0.0f;", "float mn = 3e38f, mx = -3e38f;"),
])
def test_int4_asym_pins_catch_planted_mistakes(oracle, tmp_path, old, new):
    """Each plausible slip in the asymmetric rule (divisor 16, floor for the
    zero-point or the code, no widening to include 0), planted in a copy of
    the oracle, fails the closed-form pins."""
    import ctypes
    w, B = _asym_groups(torch.float16, 31)
    bits = np.ascontiguousarray(w.view(torch.int16).numpy().view(np.uint16).reshape(-1))
    lib = _mutated_oracle(tmp_path, old, new)
    n = bits.size
    nb = n // B
    st = oracle.State(oracle.QT_INT4_ASYM, n, B, 0, np.zeros(n // 2, np.uint8), np.zeros(nb, np.float32),
                      np.zeros((nb + 1) // 2, np.uint8), None, None, None)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    lib.oracle_quantize(p(bits), 0, n, B, oracle.QT_INT4_ASYM, 0, p(st.packed), p(st.absmax),
                        p(st.zero), None, None, None)
    assert int4_asym_pin_failures(w.float().numpy(), st) != []



# ---------------------------------------------------------------- fp16 scales --
# robotsatlas.com, "INT4", "Components": the per-group scale is usually stored
# in FP16.  Reading: s is rounded to binary16 when formed and the codes (and
# the zero-point) are computed against the rounded s.

def test_oracle_binary16_rounding_is_ieee(oracle):
    """The oracle's own binary32 -> binary16 conversion (written from the
    format's definition) equals numpy's IEEE conversion on random patterns
    over the whole binary32 range and on the cases that decide rounding:
    exact halfway points between neighbouring binary16 values (both
    parities), the subnormal range, and the overflow threshold."""
    rng = np.random.default_rng(12)
    f = rng.integers(0, 2 ** 32, 60000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    f = f[np.isfinite(f)]
    h = np.arange(0, 0x7C00, 37, dtype=np.uint16).view(np.float16).astype(np.float64)
    halves = (h[:-1] + h[1:]) / 2  # exact in binary32 for these magnitudes
    edge = np.array([65504.0, 65519.99, 65520.0, 65536.0, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.5,
                     2.0 ** -26, 6.1e-5, 6.097555e-05, 1e-8, 0.0], dtype=np.float64)
    vals = np.concatenate([f.astype(np.float64), halves, edge, -halves, -edge]).astype(np.float32)
    want = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.float_to_half(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)


def int4_sym_pin_failures(wf: np.ndarray, st, scale_round=_keep) -> list:
    """Closed-form checks of INT4 symmetric groups: s = round(fl32(c / 7)),
    q = clamp(rint(fl32(w / s)), -8, 7) as a two's-complement nibble."""
    nb, B = wf.shape
    q = st.codes().astype(np.int64).reshape(nb, B)
    bad = []
    for b in range(nb):
        vals = [Fraction(float(v)) for v in wf[b]]
        c = max(abs(v) for v in vals)
        s = scale_round(_rne32(c / 7))
        if not isinstance(s, Fraction):
            if not np.isinf(st.absmax[b]) or np.any(q[b] != 0):
                bad.append(("inf-scale", b))
            continue
        if Fraction(float(st.absmax[b])) != s:
            bad.append(("scale", b))
            continue
        for j in range(B):
            qq = 0 if s == 0 else min(max(round(_rne32(vals[j] / s)), -8), 7)
            if q[b, j] != (qq & 15):
                bad.append(("code", b, j))
                break
    return bad


def _fp16_scale_groups(dt, seed):
    """_asym_groups plus groups whose scale leaves the binary16 range: tiny
    ones (s rounds to a subnormal or to 0) and, for bf16, huge ones (s
    overflows to infinity)."""
    w, B = _asym_groups(dt, seed)
    g = torch.Generator().manual_seed(seed + 1)
    extra = [torch.randn(B, generator=g) * 1e-6, torch.randn(B, generator=g) * 3e-8]
    if dt == torch.bfloat16:
        extra += [torch.randn(B, generator=g) * 1e6]
    return torch.cat([w, torch.stack(extra).to(dt)]), B


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_int4_fp16_scale_closed_forms(oracle, dt):
    """With binary16 scales, every group's stored scale is the binary16
    rounding of the binary32 rule, and its codes (and zero-point) are the
    closed forms computed against that rounded scale; the stored patterns
    are the binary16 of the stored values."""
    w, B = _fp16_scale_groups(dt, 37)
    bits = w.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    wf = w.float().numpy()
    sym = oracle.quantize(bits, dt == torch.bfloat16, B, oracle.QT_INT4_SYM, scale_f16=True)
    assert int4_sym_pin_failures(wf, sym, _to_half) == []
    asym = oracle.quantize(bits, dt == torch.bfloat16, B, oracle.QT_INT4_ASYM, scale_f16=True)
    assert int4_asym_pin_failures(wf, asym, _to_half) == []
    for st in (sym, asym):
        assert np.array_equal(st.scale_f16_bits(), st.absmax.astype(np.float16).view(np.uint16))
    # and the binary32 pins still hold without the option
    assert int4_sym_pin_failures(wf, oracle.quantize(bits, dt == torch.bfloat16, B, oracle.QT_INT4_SYM)) == []


@pytest.mark.parametrize("old,new", [
    # codes against the unrounded s, only the stored scale rounded
    ("      if (scale_f16) s = oracle_half_to_float(oracle_float_to_half(s));\n      absmax[b] = s;",
     "      absmax[b] = scale_f16 ? oracle_half_to_float(oracle_float_to_half(s)) : s;"),
    # the option ignored in the asymmetric rule
    ("      if (scale_f16) s = oracle_half_to_float(oracle_float_to_half(s));\n      int z = 0;",
     "      int z = 0;"),
])
def test_fp16_scale_pins_catch_planted_mistakes(oracle, tmp_path, old, new):
    """A planted slip in the binary16-scale rule fails the closed-form pins."""
    import ctypes
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle_module_file()), "q4_oracle.c")).read()
    assert src.count(old) == 1, old
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", str(path),
                    "-o", str(so), "-lm"], check=True, capture_output=True)
    lib = ctypes.CDLL(str(so))
    P = ctypes.c_void_p
    lib.oracle_quantize_s.argtypes = [P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, P, P, P, P, P, P]
    lib.oracle_quantize_s.restype = None
    w, B = _fp16_scale_groups(torch.float16, 37)
    bits = np.ascontiguousarray(w.view(torch.int16).numpy().view(np.uint16).reshape(-1))
    n = bits.size
    nb = n // B
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    fails = 0
    for qt in (oracle.QT_INT4_SYM, oracle.QT_INT4_ASYM):
        st = oracle.State(qt, n, B, 0, np.zeros(n // 2, np.uint8), np.zeros(nb, np.float32),
                          np.zeros((nb + 1) // 2, np.uint8), None, None, None, 1)
        lib.oracle_quantize_s(p(bits), 0, n, B, qt, 0, 1, p(st.packed), p(st.absmax), p(st.zero), None,
                              None, None)
        pin = int4_sym_pin_failures if qt == oracle.QT_INT4_SYM else int4_asym_pin_failures
        fails += len(pin(w.float().numpy(), st, _to_half))
    assert fails > 0

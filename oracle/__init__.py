"""The CPU oracle for blockwise 4-bit weight quantization and its matmul consumer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``bit_blockwise_weight_absmax_b200``) never does,
and the two share no code.

The arithmetic lives in ``q4_oracle.c`` (plain scalar C, binary32/binary64,
no FMA contraction); this module compiles it with gcc on first use and wraps
it with numpy.  Every function follows the pages cited in that file:

* learn.pranaymahendrakar.com, "Loading a model in 4-bit", section
  "Block-wise quantisation, stated exactly" -- contiguous blocks, absmax c,
  nearest of 16 levels after dividing by c, w^ = c * Q[i], double
  quantization of the block scales in blocks of 256 to 8 bits;
* n4n.ai, "What is 4-bit quantization and why does it matter?", code block
  "Conceptual NF4 dequantization" -- the 16 levels and the low-nibble-first
  unpacking; paragraph "INT4 symmetric" -- levels -8..7, scale max|w|/7;
* robotsatlas.com, "INT4", "How it works" / "Components" -- [0,15] with an
  integer zero-point, [-8,7] without;
* mbrenndoerfer.com, "INT4 Quantization > Practical Implementation with
  bitsandbytes" -- dequantize to the 16-bit compute dtype, then matmul.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_LIB = os.path.join(_HERE, "libq4oracle.so")

QT_NF4, QT_INT4_SYM, QT_INT4_ASYM = 0, 1, 2
QTYPES = {"nf4": QT_NF4, "int4_sym": QT_INT4_SYM, "int4_asym": QT_INT4_ASYM}
DQ_GROUP = 256


def build(force: bool = False) -> str:
    """Compile q4_oracle.c into libq4oracle.so (gcc, -ffp-contract=off)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    base = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
            "-D_GNU_SOURCE"]
    tmp = _LIB + ".tmp%d" % os.getpid()
    try:
        subprocess.run(base + ["-fopenmp", _SRC, "-o", tmp, "-lm"], check=True,
                       capture_output=True)
    except subprocess.CalledProcessError:
        subprocess.run(base + [_SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        _lib.oracle_quantize.argtypes = [P, i32, i64, i32, i32, i32, P, P, P, P, P, P]
        _lib.oracle_quantize.restype = None
        _lib.oracle_quantize_s.argtypes = [P, i32, i64, i32, i32, i32, i32, P, P, P, P, P, P]
        _lib.oracle_quantize_s.restype = None
        _lib.oracle_dequantize.argtypes = [P, P, P, P, P, P, i64, i32, i32, i32, i32, P]
        _lib.oracle_dequantize.restype = None
        _lib.oracle_dequantize_f32.argtypes = [P, P, P, P, P, P, i64, i32, i32, i32, P]
        _lib.oracle_dequantize_f32.restype = None
        _lib.oracle_matmul.argtypes = [P, i32, i64, P, i32, i64, i64, P, i64, P]
        _lib.oracle_matmul.restype = None
        _lib.oracle_nf4_code.argtypes = [ctypes.c_float]
        _lib.oracle_nf4_code.restype = i32
        _lib.oracle_nf4_level.argtypes = [i32]
        _lib.oracle_nf4_level.restype = ctypes.c_float
        _lib.oracle_pairwise_sum.argtypes = [P, i64]
        _lib.oracle_pairwise_sum.restype = ctypes.c_double
        _lib.oracle_half_to_float.argtypes = [ctypes.c_uint16]
        _lib.oracle_half_to_float.restype = ctypes.c_float
        _lib.oracle_bf16_to_float.argtypes = [ctypes.c_uint16]
        _lib.oracle_bf16_to_float.restype = ctypes.c_float
        _lib.oracle_float_to_half.argtypes = [ctypes.c_float]
        _lib.oracle_float_to_half.restype = ctypes.c_uint16
        _lib.oracle_float_to_bf16.argtypes = [ctypes.c_float]
        _lib.oracle_float_to_bf16.restype = ctypes.c_uint16
        _lib.oracle_set_threads.argtypes = [i32]
        _lib.oracle_set_threads.restype = i32
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(t: int) -> int:
    """Set the OpenMP thread count (<= 0 keeps it); returns the count in use."""
    return lib().oracle_set_threads(int(t))


def nf4_levels() -> np.ndarray:
    return np.array([lib().oracle_nf4_level(i) for i in range(16)], dtype=np.float32)


def nf4_code(x: float) -> int:
    return lib().oracle_nf4_code(float(x))


def pairwise_sum(v) -> float:
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64)).copy()
    return lib().oracle_pairwise_sum(_ptr(a), a.size)


@dataclass
class State:
    """Quantized tensor as the oracle produces it (numpy, host)."""
    qtype: int
    n: int
    blocksize: int
    double_quant: int
    packed: np.ndarray             # uint8 [ceil(n/2)]
    absmax: np.ndarray             # float32 [nb]
    zero: np.ndarray | None        # uint8 [ceil(nb/2)] (INT4_ASYM)
    absmax_q: np.ndarray | None    # int8 [nb] (double_quant)
    absmax_scale: np.ndarray | None  # float32 [ceil(nb/256)]
    absmax_mean: np.ndarray | None   # float32 [1]
    scale_f16: int = 0               # INT4: the scale is a binary16 value (absmax holds it as fp32)

    def scale_f16_bits(self) -> np.ndarray:
        """The stored binary16 scales (uint16 [nb]) of a scale_f16 state."""
        return np.array([lib().oracle_float_to_half(float(v)) for v in self.absmax], dtype=np.uint16)

    @property
    def nb(self) -> int:
        return (self.n + self.blocksize - 1) // self.blocksize

    def codes(self) -> np.ndarray:
        """Unpacked 4-bit codes, element j = nibble j (low nibble first)."""
        out = np.empty(2 * self.packed.size, dtype=np.uint8)
        out[0::2] = self.packed & 0xF
        out[1::2] = self.packed >> 4
        return out[: self.n]


def quantize(w_bits: np.ndarray, is_bf16: bool, blocksize: int, qtype: int,
             double_quant: bool = False, scale_f16: bool = False) -> State:
    """Quantize n 16-bit floats given as raw uint16 bit patterns (flattened).
    scale_f16 (INT4 only): binary16 scales, codes against the rounded scale."""
    w = np.ascontiguousarray(w_bits.reshape(-1).view(np.uint16))
    n = w.size
    nb = (n + blocksize - 1) // blocksize
    ng = (nb + DQ_GROUP - 1) // DQ_GROUP
    packed = np.zeros((n + 1) // 2, dtype=np.uint8)
    absmax = np.zeros(nb, dtype=np.float32)
    zero = np.zeros((nb + 1) // 2, dtype=np.uint8) if qtype == QT_INT4_ASYM else None
    dq = bool(double_quant) and qtype == QT_NF4
    absmax_q = np.zeros(nb, dtype=np.int8) if dq else None
    absmax_scale = np.zeros(ng, dtype=np.float32) if dq else None
    absmax_mean = np.zeros(1, dtype=np.float32) if dq else None
    sf = int(bool(scale_f16) and qtype != QT_NF4)
    lib().oracle_quantize_s(_ptr(w), int(is_bf16), n, blocksize, qtype, int(dq), sf, _ptr(packed),
                            _ptr(absmax), _ptr(zero), _ptr(absmax_q), _ptr(absmax_scale),
                            _ptr(absmax_mean))
    return State(qtype, n, blocksize, int(dq), packed, absmax, zero, absmax_q, absmax_scale,
                 absmax_mean, sf)


def dequantize(st: State, out_bf16: bool) -> np.ndarray:
    """Dequantize to raw 16-bit patterns (uint16 [n])."""
    out = np.empty(st.n, dtype=np.uint16)
    lib().oracle_dequantize(_ptr(st.packed), _ptr(st.absmax), _ptr(st.zero), _ptr(st.absmax_q),
                            _ptr(st.absmax_scale), _ptr(st.absmax_mean), st.n, st.blocksize,
                            st.qtype, st.double_quant, int(out_bf16), _ptr(out))
    return out


def dequantize_f32(st: State) -> np.ndarray:
    """The binary32 product c * Q[code] for every element, before rounding."""
    out = np.empty(st.n, dtype=np.float32)
    lib().oracle_dequantize_f32(_ptr(st.packed), _ptr(st.absmax), _ptr(st.zero),
                                _ptr(st.absmax_q), _ptr(st.absmax_scale), _ptr(st.absmax_mean),
                                st.n, st.blocksize, st.qtype, st.double_quant, _ptr(out))
    return out


def matmul(a_bits: np.ndarray, a_bf16: bool, w_bits: np.ndarray, w_bf16: bool, M: int, N: int,
           K: int, rows: np.ndarray | None = None) -> np.ndarray:
    """Y = A . W^T in binary64; A [M,K], W [N,K] as raw 16-bit patterns.

    Returns float64 [M, len(rows)] (or [M, N] when rows is None)."""
    a = np.ascontiguousarray(a_bits.reshape(-1).view(np.uint16))
    w = np.ascontiguousarray(w_bits.reshape(-1).view(np.uint16))
    assert a.size == M * K and w.size == N * K
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    R = N if r is None else r.size
    y = np.empty((M, R), dtype=np.float64)
    lib().oracle_matmul(_ptr(a), int(a_bf16), M, _ptr(w), int(w_bf16), N, K, _ptr(r),
                        0 if r is None else r.size, _ptr(y))
    return y


def gemv_reference(a_bits, a_bf16, st: State, N: int, K: int, rows=None) -> np.ndarray:
    """Fused dequant-matmul reference: dequantize to A's dtype, then binary64 matmul."""
    M = a_bits.size // K
    w16 = dequantize(st, a_bf16)
    return matmul(a_bits, a_bf16, w16, a_bf16, M, N, K, rows)


def half_to_float(h: int) -> float:
    return lib().oracle_half_to_float(h)


def bf16_to_float(b: int) -> float:
    return lib().oracle_bf16_to_float(b)


def float_to_half(f: float) -> int:
    return lib().oracle_float_to_half(f)


def float_to_bf16(f: float) -> int:
    return lib().oracle_float_to_bf16(f)


def storage_bits_per_param(qtype: int, blocksize: int, double_quant: bool,
                           n: int | None = None, scale_f16: bool = False) -> float:
    """Bits per parameter of the resident format (codes + block state).

    Asymptotic (n None): 4 + per-block state / blocksize.  NF4 without double
    quantization keeps one fp32 absmax per block (learn.pranaymahendrakar.com,
    "Block-wise quantisation, stated exactly": 32/64 = 0.5 bits); with it,
    one int8 per block plus one fp32 scale per 256 blocks and one fp32 mean.
    INT4 with scale_f16 keeps one binary16 scale per block.
    """
    if n is None:
        if qtype == QT_NF4 and double_quant:
            return 4.0 + 8.0 / blocksize + 32.0 / (blocksize * DQ_GROUP)
        extra = (16.0 if scale_f16 else 32.0) / blocksize
        if qtype == QT_INT4_ASYM:
            extra += 4.0 / blocksize
        return 4.0 + extra
    nb = (n + blocksize - 1) // blocksize
    bits = 8 * ((n + 1) // 2)
    if qtype == QT_NF4 and double_quant:
        bits += 8 * nb + 32 * ((nb + DQ_GROUP - 1) // DQ_GROUP) + 32
    else:
        bits += (16 if scale_f16 else 32) * nb
        if qtype == QT_INT4_ASYM:
            bits += 8 * ((nb + 1) // 2)
    return bits / n

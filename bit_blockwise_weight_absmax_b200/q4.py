"""ctypes binding of libq4.so (include/q4.h).

Argument marshalling only: every step of quantization, dequantization and the
fused matmuls runs in the library's sm_100a kernels.  torch supplies device
memory (the state buffers, outputs and workspaces are torch tensors) and the
current CUDA stream.  There is no CPU fallback: without the built library or
without a B200 every op raises Q4Error.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq4.so")

NF4, INT4_SYM, INT4_ASYM = 0, 1, 2
SCALE_F16 = 0x100  # OR into an INT4 qtype: binary16 group scales
F16, BF16, F32 = 0, 1, 2
QTYPES = {"nf4": NF4, "int4_sym": INT4_SYM, "int4_asym": INT4_ASYM}
_DT = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32}
_DT_INV = {v: k for k, v in _DT.items()}
DQ_GROUP = 256


class Q4Error(RuntimeError):
    pass


class _CState(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int32), ("src_dtype", ctypes.c_int32), ("n", ctypes.c_int64),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("blocksize", ctypes.c_int32), ("double_quant", ctypes.c_int32),
                ("dq_group", ctypes.c_int32), ("scale_f16", ctypes.c_int32),
                ("packed", ctypes.c_void_p), ("absmax", ctypes.c_void_p), ("zero", ctypes.c_void_p),
                ("absmax_q", ctypes.c_void_p), ("absmax_scale", ctypes.c_void_p),
                ("absmax_mean", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()


def library():
    """Load libq4.so (built in-tree by ``bit_blockwise_weight_absmax_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise Q4Error(f"{LIB_PATH} is not built: run `python -m "
                          "bit_blockwise_weight_absmax_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        SP = ctypes.POINTER(_CState)
        sig = {
            "q4_state_sizes": ([i32, i64, i32, i32, ctypes.POINTER(sz)], i32),
            "q4_quantize_workspace_size": ([i32, i64, i32, i32, ctypes.POINTER(sz)], i32),
            "q4_quantize": ([P, i32, i64, i64, i32, i32, i32, SP, P, sz, P], i32),
            "q4_quantize_grouped_workspace_size": ([i32, ctypes.POINTER(i64), ctypes.POINTER(i64), i32, i32, i32,
                                                    ctypes.POINTER(sz)], i32),
            "q4_quantize_grouped": ([i32, ctypes.POINTER(P), i32, ctypes.POINTER(i64), ctypes.POINTER(i64), i32, i32,
                                     i32, ctypes.POINTER(SP), P, sz, P], i32),
            "q4_dequantize": ([SP, P, i32, P], i32),
            "q4_dequantize_grouped": ([i32, ctypes.POINTER(SP), ctypes.POINTER(P), i32, P], i32),
            "q4_gemv_workspace_size": ([i32, ctypes.POINTER(SP), i64, ctypes.POINTER(sz)], i32),
            "q4_gemv": ([P, i32, i64, SP, P, i32, P, sz, P], i32),
            "q4_gemv_grouped": ([i32, ctypes.POINTER(P), ctypes.POINTER(SP), ctypes.POINTER(P), i64,
                                 i32, i32, P, sz, P], i32),
            "q4_gemm_workspace_size": ([i32, ctypes.POINTER(SP), i64, ctypes.POINTER(ctypes.c_size_t)], i32),
            "q4_gemm_plan_info": ([i32, ctypes.POINTER(SP), i64, i32, ctypes.c_size_t, ctypes.POINTER(i32),
                                   ctypes.POINTER(i32), ctypes.POINTER(i64)], i32),
            "q4_gemm": ([P, i32, i64, SP, P, i32, P, ctypes.c_size_t, P], i32),
            "q4_gemm_grouped": ([i32, ctypes.POINTER(P), ctypes.POINTER(SP), ctypes.POINTER(P), i64,
                                 i32, i32, P, ctypes.c_size_t, P], i32),
            "q4_device_status": ([ctypes.POINTER(i32)], i32),
            "q4_clear_device_status": ([], i32),
            "q4_set_wait_limit_ns": ([ctypes.c_uint64], i32),
            "q4_set_copy_stall": ([i32], i32),
            "q4_check_device": ([], i32),
            "q4_nf4_levels": ([ctypes.POINTER(ctypes.c_float)], i32),
            "q4_nf4_thresholds": ([ctypes.POINTER(ctypes.c_float)], i32),
            "q4_strerror": ([i32], ctypes.c_char_p),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
        return lib


def _check(rc: int, what: str):
    if rc != 0:
        msg = library().q4_strerror(rc).decode()
        raise Q4Error(f"{what}: {msg} (code {rc})")


def _require_gpu(t: torch.Tensor | None = None):
    if not torch.cuda.is_available():
        raise Q4Error("no CUDA device: libq4 has no CPU fallback")
    if t is not None and not t.is_cuda:
        raise Q4Error("tensor must be on a CUDA device")
    _check(library().q4_check_device(), "q4_check_device")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------ state ----

@dataclass
class Q4State:
    """A quantized weight [rows, cols] and its device buffers (torch tensors)."""
    qtype: int
    src_dtype: torch.dtype
    rows: int
    cols: int
    blocksize: int
    double_quant: bool
    packed: torch.Tensor
    absmax: torch.Tensor | None  # with double quantization no consumer reads it
    zero: torch.Tensor | None = None
    absmax_q: torch.Tensor | None = None
    absmax_scale: torch.Tensor | None = None
    absmax_mean: torch.Tensor | None = None
    scale_f16: bool = False  # INT4: absmax holds binary16 scales

    @property
    def n(self) -> int:
        return self.rows * self.cols

    @property
    def device(self):
        return self.packed.device

    def c_struct(self) -> _CState:
        """The C view of the state, built once and rebuilt only when a buffer
        or a field has changed."""
        key = (self.qtype, self.src_dtype, self.rows, self.cols, self.blocksize, self.double_quant, self.scale_f16,
               self.packed.data_ptr(), None if self.absmax is None else self.absmax.data_ptr(),
               None if self.zero is None else self.zero.data_ptr(),
               None if self.absmax_q is None else self.absmax_q.data_ptr(),
               None if self.absmax_scale is None else self.absmax_scale.data_ptr(),
               None if self.absmax_mean is None else self.absmax_mean.data_ptr())
        cached = self.__dict__.get("_cs")
        if cached is not None and cached[0] == key:
            return cached[1]
        s = self._build_c_struct()
        self.__dict__["_cs"] = (key, s)
        return s

    def _build_c_struct(self) -> _CState:
        s = _CState()
        s.qtype = self.qtype
        s.src_dtype = _DT[self.src_dtype]
        s.n = self.n
        s.rows = self.rows
        s.cols = self.cols
        s.blocksize = self.blocksize
        s.double_quant = int(self.double_quant)
        s.dq_group = DQ_GROUP
        s.scale_f16 = int(self.scale_f16)
        s.packed = self.packed.data_ptr()
        s.absmax = None if self.absmax is None else self.absmax.data_ptr()
        s.zero = None if self.zero is None else self.zero.data_ptr()
        s.absmax_q = None if self.absmax_q is None else self.absmax_q.data_ptr()
        s.absmax_scale = None if self.absmax_scale is None else self.absmax_scale.data_ptr()
        s.absmax_mean = None if self.absmax_mean is None else self.absmax_mean.data_ptr()
        return s

    def release_absmax(self):
        """Drop the fp32 block absmax of a double-quantized state: the
        consumers read the 8-bit codes, their scales and the mean instead, so
        the fp32 copy (0.5 bit per weight at blocksize 64) is only needed to
        inspect the state."""
        if not self.double_quant:
            raise Q4Error("the fp32 absmax is the block scale of a state without double quantization")
        self.absmax = None

    def held_bytes(self) -> int:
        """Device bytes of every buffer the state still holds."""
        return sum(t.numel() * t.element_size() for t in (self.packed, self.absmax, self.zero, self.absmax_q,
                                                         self.absmax_scale, self.absmax_mean) if t is not None)

    def resident_bytes(self) -> int:
        """Bytes of the format a consumer reads (codes + block state); with
        double quantization the fp32 absmax kept for inspection is excluded."""
        b = self.packed.numel()
        if self.double_quant:
            b += self.absmax_q.numel() + 4 * self.absmax_scale.numel() + 4
        else:
            b += self.absmax.numel() * self.absmax.element_size()
            if self.zero is not None:
                b += self.zero.numel()
        return b


def state_sizes(qtype, n: int, blocksize: int, double_quant: bool) -> tuple:
    qt = QTYPES[qtype] if isinstance(qtype, str) else int(qtype)
    out = (ctypes.c_size_t * 6)()
    _check(library().q4_state_sizes(qt, n, blocksize, int(double_quant), out), "q4_state_sizes")
    return tuple(out)


def nf4_levels() -> list:
    out = (ctypes.c_float * 16)()
    _check(library().q4_nf4_levels(out), "q4_nf4_levels")
    return list(out)


def nf4_thresholds() -> list:
    out = (ctypes.c_float * 15)()
    _check(library().q4_nf4_thresholds(out), "q4_nf4_thresholds")
    return list(out)


def last_device_status() -> int:
    v = ctypes.c_int32(0)
    _check(library().q4_device_status(ctypes.byref(v)), "q4_device_status")
    return v.value


def clear_device_status():
    _check(library().q4_clear_device_status(), "q4_clear_device_status")


def set_wait_limit_ns(ns: int):
    """Bound (ns) of every device-side wait of later launches; 0 = default 2 s."""
    _check(library().q4_set_wait_limit_ns(int(ns)), "q4_set_wait_limit_ns")


def set_copy_stall(on: bool):
    """Test hook: while on, the decode GEMV issues no weight copies, so its
    stage waits run out after the wait limit (Q4_STATUS_TIMEOUT)."""
    _check(library().q4_set_copy_stall(int(bool(on))), "q4_set_copy_stall")


def reset_workspaces():
    """Zero-fill every cached workspace again (needed after a call ended with
    Q4_STATUS_TIMEOUT, which leaves its workspace undefined)."""
    for t in _ws.values():
        t.zero_()


# -------------------------------------------------------------- workspaces --
# Workspaces must start zero-filled; every call leaves them zeroed again, so
# one buffer per (device, kind) is reused.  Calls on different streams that
# overlap in time must not share a workspace.
_ws: dict = {}


def _workspace(device, kind: str, nbytes: int) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    key = (device.index if device.index is not None else torch.cuda.current_device(), kind)
    t = _ws.get(key)
    if t is None or t.numel() < nbytes:
        t = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _ws[key] = t
    return t


# ------------------------------------------------------------------- ops ----

def quantize(W: torch.Tensor, blocksize: int = 64, qtype="nf4", double_quant: bool = False,
             stream=None, out: Q4State | None = None, scale_f16: bool = False) -> Q4State:
    """Blockwise 4-bit quantization of a 2-D fp16/bf16 CUDA tensor.

    `out` reuses the buffers of an earlier state of the same shape and format
    (no allocation: the call can be captured in a CUDA graph).  scale_f16
    (INT4 only): binary16 group scales, the codes taken against them."""
    _require_gpu(W)
    if W.dtype not in (torch.float16, torch.bfloat16) or W.dim() != 2:
        raise Q4Error("W must be a 2-D float16/bfloat16 tensor")
    W = W.contiguous()
    qt = QTYPES[qtype] if isinstance(qtype, str) else int(qtype)
    qt_arg = qt | (SCALE_F16 if scale_f16 else 0)
    rows, cols = W.shape
    n = rows * cols
    dev = W.device
    if out is not None:
        if (out.qtype, out.rows, out.cols, out.blocksize, out.double_quant, out.scale_f16) != \
                (qt, rows, cols, blocksize, bool(double_quant), bool(scale_f16)):
            raise Q4Error("out= state has a different shape or format")
        if out.absmax is None:
            raise Q4Error("out= state has released its absmax buffer, which quantize writes")
        out.src_dtype = W.dtype
    st = out if out is not None else _new_state(qt, W.dtype, rows, cols, blocksize, double_quant, dev, scale_f16)
    wsz = ctypes.c_size_t(0)
    _check(library().q4_quantize_workspace_size(qt_arg, n, blocksize, int(double_quant), ctypes.byref(wsz)),
           "q4_quantize_workspace_size")
    ws = _workspace(dev, "quantize", wsz.value)
    cs = st.c_struct()
    _check(library().q4_quantize(_ptr(W), _DT[W.dtype], rows, cols, blocksize, qt_arg, int(double_quant),
                                 ctypes.byref(cs), _ptr(ws), 0 if ws is None else ws.numel(),
                                 _stream(stream)), "q4_quantize")
    return st


def _new_state(qt, dtype, rows, cols, blocksize, double_quant, dev, scale_f16=False) -> Q4State:
    sz = state_sizes(qt | (SCALE_F16 if scale_f16 else 0), rows * cols, blocksize, double_quant)
    return Q4State(qt, dtype, rows, cols, blocksize, bool(double_quant),
                   packed=torch.empty(sz[0], dtype=torch.uint8, device=dev),
                   absmax=(torch.empty(sz[1] // 2, dtype=torch.float16, device=dev) if scale_f16 else
                           torch.empty(sz[1] // 4, dtype=torch.float32, device=dev)),
                   zero=torch.empty(sz[2], dtype=torch.uint8, device=dev) if sz[2] else None,
                   absmax_q=torch.empty(sz[3], dtype=torch.int8, device=dev) if sz[3] else None,
                   absmax_scale=torch.empty(sz[4] // 4, dtype=torch.float32, device=dev) if sz[4] else None,
                   absmax_mean=torch.empty(1, dtype=torch.float32, device=dev) if sz[5] else None,
                   scale_f16=bool(scale_f16))


def quantize_grouped(Ws, blocksize: int = 64, qtype="nf4", double_quant: bool = False, stream=None,
                     outs=None, scale_f16: bool = False) -> list:
    """Quantize several 2-D weights of one dtype and one format in one launch
    (plus one second-level launch with double quantization); the states are
    bit for bit those of quantize() on each weight.  `outs` reuses earlier
    states of the same shapes and format (no allocation)."""
    _require_gpu(Ws[0])
    qt = QTYPES[qtype] if isinstance(qtype, str) else int(qtype)
    qt_arg = qt | (SCALE_F16 if scale_f16 else 0)
    dtype = Ws[0].dtype
    for W in Ws:
        if W.dtype != dtype or W.dim() != 2 or W.dtype not in (torch.float16, torch.bfloat16):
            raise Q4Error("weights must be 2-D float16/bfloat16 tensors of one dtype")
    Ws = [W.contiguous() for W in Ws]
    dev = Ws[0].device
    if outs is None:
        outs = [_new_state(qt, dtype, W.shape[0], W.shape[1], blocksize, double_quant, dev, scale_f16)
                for W in Ws]
    else:
        for st, W in zip(outs, Ws):
            if (st.qtype, st.rows, st.cols, st.blocksize, st.double_quant, st.scale_f16) != \
                    (qt, W.shape[0], W.shape[1], blocksize, bool(double_quant), bool(scale_f16)) \
                    or st.absmax is None:
                raise Q4Error("outs= states have a different shape or format")
            st.src_dtype = dtype
    n = len(Ws)
    rows = (ctypes.c_int64 * n)(*[W.shape[0] for W in Ws])
    cols = (ctypes.c_int64 * n)(*[W.shape[1] for W in Ws])
    wsz = ctypes.c_size_t(0)
    _check(library().q4_quantize_grouped_workspace_size(n, rows, cols, blocksize, qt_arg, int(double_quant),
                                                         ctypes.byref(wsz)), "q4_quantize_grouped_workspace_size")
    ws = _workspace(dev, "quantize", wsz.value)
    structs = [st.c_struct() for st in outs]
    arr = _struct_array(structs)
    wp = (ctypes.c_void_p * n)(*[W.data_ptr() for W in Ws])
    _check(library().q4_quantize_grouped(n, wp, _DT[dtype], rows, cols, blocksize, qt_arg, int(double_quant), arr,
                                         _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)),
           "q4_quantize_grouped")
    return outs


def dequantize(st: Q4State, dtype: torch.dtype | None = None, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    _require_gpu(st.packed)
    dtype = dtype or st.src_dtype
    if out is None:
        out = torch.empty(st.rows, st.cols, dtype=dtype, device=st.device)
    cs = st.c_struct()
    _check(library().q4_dequantize(ctypes.byref(cs), _ptr(out), _DT[dtype], _stream(stream)),
           "q4_dequantize")
    return out


def dequantize_grouped(states, dtype: torch.dtype | None = None, outs=None, stream=None) -> list:
    """q4.dequantize of several states of one format in one launch."""
    _require_gpu(states[0].packed)
    dtype = dtype or states[0].src_dtype
    if outs is None:
        outs = [torch.empty(st.rows, st.cols, dtype=dtype, device=st.device) for st in states]
    structs = [st.c_struct() for st in states]
    n = len(states)
    arr = _struct_array(structs)
    op = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    _check(library().q4_dequantize_grouped(n, arr, op, _DT[dtype], _stream(stream)), "q4_dequantize_grouped")
    return outs


_gemv_ws_need = {}  # (shapes and formats of the group, M) -> workspace bytes


_struct_arrays = {}


def _struct_array(structs):
    """The C array of pointers to these state structs, built once per tuple
    of structs (c_struct() returns the same object while a state is
    unchanged; the cache holds the structs, so their ids stay theirs)."""
    key = tuple(id(s) for s in structs)
    hit = _struct_arrays.get(key)
    if hit is not None:
        return hit[1]
    arr = (ctypes.POINTER(_CState) * len(structs))(*[ctypes.pointer(s) for s in structs])
    if len(_struct_arrays) >= 256:
        _struct_arrays.clear()
    _struct_arrays[key] = (tuple(structs), arr)
    return arr


def _gemv_workspace(states, structs, M, device):
    arr = _struct_array(structs)
    key = (tuple((s.rows, s.cols, s.blocksize, s.qtype, s.double_quant) for s in states), M)
    need = _gemv_ws_need.get(key)
    if need is None:
        n = ctypes.c_size_t(0)
        _check(library().q4_gemv_workspace_size(len(structs), arr, M, ctypes.byref(n)),
               "q4_gemv_workspace_size")
        need = _gemv_ws_need[key] = n.value
    return arr, _workspace(device, "gemv", need)


def gemv_grouped(As, states, out_dtype: torch.dtype | None = None, outs=None, stream=None):
    """Y_i = A_i . W^_i^T for each i in one launch; A_i [M, K_i], 1 <= M <= 32."""
    _require_gpu(As[0])
    M = As[0].shape[0]
    a_dtype = As[0].dtype
    out_dtype = out_dtype or a_dtype
    structs = [s.c_struct() for s in states]
    arr, ws = _gemv_workspace(states, structs, M, As[0].device)
    if outs is None:
        outs = [torch.empty(M, s.rows, dtype=out_dtype, device=As[0].device) for s in states]
    a_ptrs = (ctypes.c_void_p * len(As))(*[a.data_ptr() for a in As])
    y_ptrs = (ctypes.c_void_p * len(As))(*[y.data_ptr() for y in outs])
    for a, s in zip(As, states):
        if a.dtype != a_dtype or a.shape != (M, s.cols) or not a.is_contiguous():
            raise Q4Error("activations must be contiguous [M, K] of one dtype")
    _check(library().q4_gemv_grouped(len(As), a_ptrs, arr, y_ptrs, M, _DT[a_dtype], _DT[out_dtype],
                                     _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)),
           "q4_gemv_grouped")
    return outs


def gemv(A: torch.Tensor, st: Q4State, out_dtype: torch.dtype | None = None, out=None,
         stream=None) -> torch.Tensor:
    return gemv_grouped([A], [st], out_dtype, None if out is None else [out], stream)[0]


def gemm_grouped(As, states, out_dtype: torch.dtype | None = None, outs=None, stream=None):
    """Y_i = A_i . W^_i^T for each i, tcgen05 W4A16 GEMM, one persistent launch."""
    _require_gpu(As[0])
    M = As[0].shape[0]
    a_dtype = As[0].dtype
    out_dtype = out_dtype or a_dtype
    structs = [s.c_struct() for s in states]
    arr = _struct_array(structs)
    if outs is None:
        outs = [torch.empty(M, s.rows, dtype=out_dtype, device=As[0].device) for s in states]
    for a, s in zip(As, states):
        if a.dtype != a_dtype or a.shape != (M, s.cols) or not a.is_contiguous():
            raise Q4Error("activations must be contiguous [M, K] of one dtype")
    a_ptrs = (ctypes.c_void_p * len(As))(*[a.data_ptr() for a in As])
    y_ptrs = (ctypes.c_void_p * len(As))(*[y.data_ptr() for y in outs])
    # the workspace that lets the launch cut tiles in k where that evens out
    # the CTAs' work (cached per device; zero-filled, left zeroed)
    wsz = ctypes.c_size_t(0)
    _check(library().q4_gemm_workspace_size(len(As), arr, M, ctypes.byref(wsz)), "q4_gemm_workspace_size")
    ws = _workspace(As[0].device, "gemm", wsz.value)
    _check(library().q4_gemm_grouped(len(As), a_ptrs, arr, y_ptrs, M, _DT[a_dtype], _DT[out_dtype],
                                     _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)),
           "q4_gemm_grouped")
    return outs


def gemm(A: torch.Tensor, st: Q4State, out_dtype: torch.dtype | None = None, out=None,
         stream=None) -> torch.Tensor:
    return gemm_grouped([A], [st], out_dtype, None if out is None else [out], stream)[0]

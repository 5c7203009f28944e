"""q4_quantize_noalloc: the quantize entry point for callers that cannot
allocate device memory (it takes its workspace from a fixed static array in
the library instead of from the caller).

Called through the C ABI, its output state must equal q4_quantize's exactly
(quantization is bit-exact everywhere in this library), on two calls in a
row, so that whatever the first call leaves in the shared static array does
not leak into the second.  This file sorts last so that a stop-at-first-
failure run has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _fresh_state(q4, W, blocksize, qtype, dq):
    sz = q4.state_sizes(qtype, W.numel(), blocksize, dq)
    dev = W.device
    return q4.Q4State(
        q4.QTYPES[qtype], W.dtype, W.shape[0], W.shape[1], blocksize, dq,
        packed=torch.full((sz[0],), 0xAB, dtype=torch.uint8, device=dev),
        absmax=torch.full((sz[1] // 4,), float("nan"), dtype=torch.float32, device=dev),
        zero=torch.zeros(sz[2], dtype=torch.uint8, device=dev) if sz[2] else None,
        absmax_q=torch.zeros(sz[3], dtype=torch.int8, device=dev) if sz[3] else None,
        absmax_scale=torch.zeros(sz[4] // 4, dtype=torch.float32, device=dev) if sz[4] else None,
        absmax_mean=torch.full((1,), -1.0, dtype=torch.float32, device=dev) if sz[5] else None)


def _call_noalloc(q4, lib, W, st):
    cs = st.c_struct()
    rc = lib.q4_quantize_noalloc(ctypes.c_void_p(W.data_ptr()), q4._DT[W.dtype], st.rows, st.cols,
                                 st.blocksize, st.qtype, int(st.double_quant), ctypes.byref(cs),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.q4_strerror(rc)


def _same(a, b):
    if a is None or b is None:
        return a is None and b is None
    return torch.equal(a.view(torch.uint8) if a.dtype == torch.float32 else a,
                       b.view(torch.uint8) if b.dtype == torch.float32 else b)


@pytest.mark.parametrize("qtype,dq,dtype", [("nf4", True, torch.bfloat16), ("nf4", True, torch.float16),
                                            ("nf4", False, torch.bfloat16),
                                            ("int4_asym", False, torch.float16)])
def test_noalloc_matches_q4_quantize_twice(qtype, dq, dtype):
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4
    lib = q4.library()
    lib.q4_quantize_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.POINTER(q4._CState), ctypes.c_void_p]
    lib.q4_quantize_noalloc.restype = ctypes.c_int32
    g = torch.Generator().manual_seed(77)
    # two different inputs, so the second call cannot pass by repeating the first
    Ws = [(torch.randn(4099, 2048, generator=g) * 0.02).to(dtype).cuda(),
          (torch.randn(1000, 4160, generator=g) * 0.05).to(dtype).cuda()]
    for W in Ws:
        ref = q4.quantize(W, 64, qtype, dq)
        st = _fresh_state(q4, W, 64, qtype, dq)
        _call_noalloc(q4, lib, W, st)
        torch.cuda.synchronize()
        for f in ("packed", "absmax", "zero", "absmax_q", "absmax_scale", "absmax_mean"):
            assert _same(getattr(st, f), getattr(ref, f)), f
    # the library's state size for the largest DQ workspace fits the array
    need = ctypes.c_size_t(0)
    lib.q4_quantize_workspace_size(0, 1 << 34, 64, 1, ctypes.byref(need))
    assert 0 < need.value <= 32768

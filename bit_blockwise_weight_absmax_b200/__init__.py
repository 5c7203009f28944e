"""Blockwise 4-bit weight quantization (NF4 absmax / INT4 sym / INT4 asym with
zero-point, double quantization of the absmax) and its fused consumers
(dequantize, dequant-GEMV for decode, W4A16 tcgen05 GEMM for prefill) as
hand-written sm_100a CUDA kernels behind the C-ABI library ``libq4.so``.

The Python layer only marshals arguments (torch provides device memory and
streams).  Importing this package loads nothing; the first call of an op
loads ``libq4.so`` and fails loudly if the library or a B200 is missing.
"""
_BINDING = {
    "Q4State", "Q4Error", "NF4", "INT4_SYM", "INT4_ASYM", "F16", "BF16", "quantize", "quantize_grouped",
    "dequantize", "dequantize_grouped", "gemv", "gemv_grouped", "gemm", "gemm_grouped", "state_sizes", "nf4_levels",
    "nf4_thresholds", "last_device_status", "clear_device_status", "library",
}


def __getattr__(name):
    if name in _BINDING:
        from . import q4
        return getattr(q4, name)
    raise AttributeError(name)

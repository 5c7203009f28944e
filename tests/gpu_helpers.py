"""Helpers shared by the GPU parity tests: moving seeded inputs between torch
and the oracle's raw 16-bit representation, and the matmul tolerance check."""
import numpy as np
import torch

# Tolerance of the fused matmuls against the oracle's binary64 product of A
# and the 16-bit dequantized weights, rounded once to the output dtype.
REL_FRO = 1e-3
MAX_ABS = 1e-2


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 patterns of a 16-bit float tensor (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def is_bf16(t: torch.Tensor) -> bool:
    return t.dtype == torch.bfloat16


def round_to(y: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Round a binary64 array once to dtype, returned as binary64."""
    if dtype == torch.float16:
        return y.astype(np.float16).astype(np.float64)
    if dtype == torch.float32:
        return y.astype(np.float32).astype(np.float64)
    return torch.from_numpy(y).to(torch.bfloat16).double().numpy()


def matmul_errors(y_gpu: torch.Tensor, y_ref: np.ndarray):
    """(relative Frobenius error, max abs error / max|Y_ref|) of the GPU
    output against the reference rounded once to the output dtype."""
    y = y_gpu.detach().double().cpu().numpy().reshape(y_ref.shape)
    r = round_to(y_ref, y_gpu.dtype)
    fro = np.linalg.norm(y - r) / max(np.linalg.norm(r), 1e-300)
    mx = np.abs(y - r).max() / max(np.abs(y_ref).max(), 1e-300)
    return fro, mx


def assert_matmul_close(y_gpu, y_ref, rel_fro=REL_FRO, max_abs=MAX_ABS):
    fro, mx = matmul_errors(y_gpu, y_ref)
    assert np.all(np.isfinite(y_gpu.detach().float().cpu().numpy()))
    assert fro <= rel_fro and mx <= max_abs, (fro, mx)
    return fro, mx


def assert_state_equal(st, ost):
    """GPU state (Q4State) equals the oracle state bit for bit."""
    assert np.array_equal(st.packed.cpu().numpy(), ost.packed), "packed codes differ"
    if getattr(ost, "scale_f16", 0):
        assert st.scale_f16 and st.absmax.dtype == torch.float16
        assert np.array_equal(st.absmax.cpu().numpy().view(np.uint16), ost.scale_f16_bits()), \
            "binary16 scale differs"
    else:
        assert np.array_equal(st.absmax.cpu().numpy().view(np.uint32), ost.absmax.view(np.uint32)), \
            "absmax / scale differs"
    if ost.zero is not None:
        assert np.array_equal(st.zero.cpu().numpy(), ost.zero), "zero-points differ"
    if ost.absmax_q is not None:
        assert np.array_equal(st.absmax_q.cpu().numpy(), ost.absmax_q), "double-quant codes differ"
        assert np.array_equal(st.absmax_scale.cpu().numpy().view(np.uint32),
                              ost.absmax_scale.view(np.uint32)), "double-quant scales differ"
        assert np.array_equal(st.absmax_mean.cpu().numpy().view(np.uint32),
                              ost.absmax_mean.view(np.uint32)), "double-quant mean differs"


def oracle_state(oracle, W: torch.Tensor, blocksize, qtype, dq, scale_f16=False):
    return oracle.quantize(bits(W), is_bf16(W), blocksize, qtype, dq, scale_f16)

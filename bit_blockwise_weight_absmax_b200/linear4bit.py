"""A Linear4bit-style module over the C ABI: an nn.Linear whose weight is held
as blockwise 4-bit codes (NF4 absmax with optional double quantization, INT4
symmetric, or INT4 asymmetric with zero-points), and whose forward pass is the
fused consumer.

learn.pranaymahendrakar.com, "Loading a model in 4-bit", "Where the accuracy
goes": a 4-bit linear layer keeps its weight quantized and dequantizes it to
the compute dtype for the matmul; the output head and the normalisation
layers stay in 16 bits.  Here the dequantization is fused into the kernels:
up to 32 rows of activations run the decode GEMV, more rows the W4A16
tcgen05 GEMM (every format and blocksize; N % 16 == 0 and K % 64 == 0),
other shapes run the GEMV 32 rows at a time.  A format neither consumer
takes is refused when the module is built.  All compute is on the GPU; there is no CPU path.
"""
from __future__ import annotations

import torch

from . import q4

GEMV_MAX_ROWS = 32


class Linear4bit(torch.nn.Module):
    """y = x . W^T + b with W held as a Q4State (see q4.quantize)."""

    def __init__(self, state: q4.Q4State, bias: torch.Tensor | None = None,
                 compute_dtype: torch.dtype = torch.float16):
        super().__init__()
        if compute_dtype not in (torch.float16, torch.bfloat16):
            raise q4.Q4Error("compute_dtype must be torch.float16 or torch.bfloat16")
        why = unsupported_reason(state)
        if why:
            raise q4.Q4Error(f"Linear4bit cannot run this state: {why}")
        self.state = state
        self.in_features = state.cols
        self.out_features = state.rows
        self.compute_dtype = compute_dtype
        self.bias = None if bias is None else torch.nn.Parameter(bias.detach().to(compute_dtype),
                                                                 requires_grad=False)

    @classmethod
    def from_linear(cls, lin: torch.nn.Linear, blocksize: int = 64, qtype: str = "nf4",
                    double_quant: bool = True, compute_dtype: torch.dtype = torch.float16,
                    keep_absmax: bool = False) -> "Linear4bit":
        """Quantize an nn.Linear's weight (on its CUDA device) once, at load
        time.  With double quantization the fp32 block absmax, which no
        consumer reads, is released unless `keep_absmax`."""
        qt = q4.QTYPES[qtype] if isinstance(qtype, str) else int(qtype)
        why = unsupported_reason_of(qt, blocksize, lin.in_features)
        if why:
            raise q4.Q4Error(f"Linear4bit cannot run this format: {why}")
        w = lin.weight.detach()
        if w.dtype not in (torch.float16, torch.bfloat16):
            w = w.to(torch.bfloat16)
        st = q4.quantize(w.contiguous(), blocksize, qt, double_quant)
        if double_quant and not keep_absmax:
            st.release_absmax()
        return cls(st, lin.bias, compute_dtype)

    def _gemm_ok(self) -> bool:
        st = self.state
        return st.rows % 16 == 0 and st.cols % 64 == 0 and st.cols % st.blocksize == 0

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if x.shape[-1] != self.in_features:
            raise q4.Q4Error(f"expected last dimension {self.in_features}, got {x.shape[-1]}")
        lead = x.shape[:-1]
        a = x.reshape(-1, self.in_features).to(self.compute_dtype).contiguous()
        T = a.shape[0]
        # with a bias the product stays fp32 until the bias is added, so the
        # output is rounded to the compute dtype once
        acc = torch.float32 if self.bias is not None else self.compute_dtype
        if T == 0:
            y = a.new_empty(0, self.out_features, dtype=acc)
        elif T <= GEMV_MAX_ROWS:
            y = q4.gemv(a, self.state, acc)
        elif self._gemm_ok():
            y = q4.gemm(a, self.state, acc)
        else:
            y = torch.cat([q4.gemv(a[i:i + GEMV_MAX_ROWS].contiguous(), self.state, acc)
                           for i in range(0, T, GEMV_MAX_ROWS)])
        if self.bias is not None:
            y = (y + self.bias.float()).to(self.compute_dtype)
        return y.reshape(*lead, self.out_features)

    def extra_repr(self) -> str:
        st = self.state
        kind = {q4.NF4: "nf4", q4.INT4_SYM: "int4_sym", q4.INT4_ASYM: "int4_asym"}[st.qtype]
        return (f"in_features={self.in_features}, out_features={self.out_features}, {kind}, "
                f"blocksize={st.blocksize}, double_quant={st.double_quant}, "
                f"compute_dtype={self.compute_dtype}")


def unsupported_reason_of(qtype: int, blocksize: int, in_features: int) -> str | None:
    """Why the fused consumers cannot run a format, or None when they can:
    the GEMV takes NF4, INT4 symmetric and INT4 asymmetric states with whole
    blocks per row (in_features % blocksize == 0)."""
    if qtype not in (q4.NF4, q4.INT4_SYM, q4.INT4_ASYM):
        return f"unknown qtype {qtype}"
    if blocksize not in (32, 64, 128, 256):
        return f"blocksize {blocksize} is not 32, 64, 128 or 256"
    if in_features % blocksize:
        return f"in_features {in_features} is not a multiple of the blocksize {blocksize}"
    return None


def unsupported_reason(st: q4.Q4State) -> str | None:
    return unsupported_reason_of(st.qtype, st.blocksize, st.cols)


def memory_footprint(module: torch.nn.Module) -> int:
    """Bytes a module holds: every distinct parameter and buffer (a weight
    tied between two layers counts once) plus the buffers of every
    Linear4bit's quantized state."""
    total = 0
    seen = set()
    for t in list(module.parameters()) + list(module.buffers()):
        if id(t) not in seen:
            seen.add(id(t))
            total += t.numel() * t.element_size()
    for m in module.modules():
        if isinstance(m, Linear4bit):
            total += m.state.held_bytes()
    return total


def linears_to_replace(module: torch.nn.Module, skip=("lm_head",)) -> list:
    """Qualified names of the nn.Linear submodules that replace_linear swaps:
    every nn.Linear except those whose own name is in `skip` (the output head
    stays in 16 bits)."""
    names = []
    for name, m in module.named_modules():
        if isinstance(m, torch.nn.Linear) and name.rsplit(".", 1)[-1] not in skip:
            names.append(name)
    return names


def replace_linear(module: torch.nn.Module, skip=("lm_head",), **kw) -> torch.nn.Module:
    """Swap the module's nn.Linear layers (except `skip`) for Linear4bit in
    place, quantizing each weight once; keyword arguments go to
    Linear4bit.from_linear.  Returns the module."""
    for name in linears_to_replace(module, skip):
        parent_name, _, child = name.rpartition(".")
        parent = module.get_submodule(parent_name) if parent_name else module
        setattr(parent, child, Linear4bit.from_linear(getattr(parent, child), **kw))
    return module

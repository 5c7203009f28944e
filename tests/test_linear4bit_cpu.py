"""Host logic of the Linear4bit module: which layers replace_linear swaps,
argument checks, and that a forward pass without a GPU fails loudly (there
is no CPU path)."""
import pytest
import torch

from bit_blockwise_weight_absmax_b200 import linear4bit, q4


class _Toy(torch.nn.Module):
    def __init__(self):
        super().__init__()
        self.embed = torch.nn.Embedding(10, 64)
        self.layers = torch.nn.ModuleList([torch.nn.ModuleDict({
            "q_proj": torch.nn.Linear(64, 64),
            "mlp": torch.nn.Sequential(torch.nn.Linear(64, 128), torch.nn.GELU(), torch.nn.Linear(128, 64)),
        }) for _ in range(2)])
        self.norm = torch.nn.LayerNorm(64)
        self.lm_head = torch.nn.Linear(64, 10)


def test_linears_to_replace_keeps_head_embeddings_norms():
    names = linear4bit.linears_to_replace(_Toy())
    assert names == ["layers.0.q_proj", "layers.0.mlp.0", "layers.0.mlp.2",
                     "layers.1.q_proj", "layers.1.mlp.0", "layers.1.mlp.2"]
    assert "lm_head" in linear4bit.linears_to_replace(_Toy(), skip=())


def _dummy_state(qtype=q4.NF4, cols=64, blocksize=64):
    z = torch.zeros(4 * cols // 2, dtype=torch.uint8)
    return q4.Q4State(qtype, torch.float16, 4, cols, blocksize, False, z, torch.zeros(4 * cols // blocksize))


def test_rejects_fp32_compute_dtype():
    with pytest.raises(q4.Q4Error):
        linear4bit.Linear4bit(_dummy_state(), compute_dtype=torch.float32)


def test_forward_without_gpu_fails_loudly():
    m = linear4bit.Linear4bit(_dummy_state())
    assert m.in_features == 64 and m.out_features == 4
    with pytest.raises(q4.Q4Error):
        m(torch.zeros(2, 64))
    with pytest.raises(q4.Q4Error):
        m(torch.zeros(2, 7))  # wrong width is caught before any kernel call


def test_refuses_formats_no_consumer_runs():
    """A state the GEMV/GEMM cannot consume is refused when the module is
    built, not at its first forward pass."""
    with pytest.raises(q4.Q4Error, match="multiple"):
        linear4bit.Linear4bit(_dummy_state(q4.NF4, 96, 64))
    with pytest.raises(q4.Q4Error, match="multiple"):
        linear4bit.Linear4bit.from_linear(torch.nn.Linear(96, 8), 64, "nf4")
    with pytest.raises(q4.Q4Error, match="blocksize"):
        linear4bit.Linear4bit(_dummy_state(q4.NF4, 96, 48))
    for qt in (q4.NF4, q4.INT4_SYM, q4.INT4_ASYM):
        linear4bit.Linear4bit(_dummy_state(qt, 128, 128))


def test_state_c_struct_is_cached_and_rebuilt_on_change():
    """The binding builds a state's C struct once and rebuilds it when a
    buffer is replaced (the cache is keyed by every pointer and field)."""
    st = _dummy_state()
    a = st.c_struct()
    assert st.c_struct() is a
    assert a.packed == st.packed.data_ptr() and a.rows == 4 and a.cols == 64
    st.packed = torch.zeros(16, dtype=torch.uint8)
    b = st.c_struct()
    assert b is not a and b.packed == st.packed.data_ptr()
    st.blocksize = 32
    assert st.c_struct().blocksize == 32

"""Memory footprint of replace_linear's 4-bit model against the pages.

learn.pranaymahendrakar.com, "Loading a model in 4-bit": "The walkthrough"
prints 269 MB at fp16 and 110 MB at 4 bits for the 135M-parameter demo
model, and "Block-wise quantisation, stated exactly" says NF4 with double
quantization is near 4.127 bits per parameter, a ~3.9x ratio that appears
only when the linear layers dominate, while the demo reached 2.4x because
the embeddings, the output head and the norms stay 16-bit.  Here the
replacement is planned on the meta device (no memory, no GPU): every linear
that replace_linear swaps becomes a Linear4bit whose state has the sizes
q4_state_sizes gives, with the fp32 absmax released as from_linear does."""
import torch

from bit_blockwise_weight_absmax_b200 import linear4bit, q4
from bit_blockwise_weight_absmax_b200 import workloads as wl
from model_layouts import DecoderSkeleton


def _plan_4bit(model, blocksize=64):
    for name in linear4bit.linears_to_replace(model):
        parent_name, _, child = name.rpartition(".")
        parent = model.get_submodule(parent_name) if parent_name else model
        lin = getattr(parent, child)
        N, K = lin.out_features, lin.in_features
        sz = q4.state_sizes("nf4", N * K, blocksize, True)
        meta = lambda n, dt: torch.empty(n, dtype=dt, device="meta")
        st = q4.Q4State(q4.NF4, torch.float16, N, K, blocksize, True, packed=meta(sz[0], torch.uint8),
                        absmax=None, absmax_q=meta(sz[3], torch.int8),
                        absmax_scale=meta(sz[4] // 4, torch.float32), absmax_mean=meta(1, torch.float32))
        setattr(parent, child, linear4bit.Linear4bit(st, None))
    return model


def _ratio(layout):
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    fp16 = linear4bit.memory_footprint(DecoderSkeleton(layout))
    b4 = linear4bit.memory_footprint(_plan_4bit(DecoderSkeleton(layout)))
    return fp16, b4


def test_small_model_footprint_is_the_demo_ratio():
    """135M-class layout (tied head, 16-bit embeddings): 269 MB at fp16, about
    110 MB at 4 bits, the page's 2.4x."""
    fp16, b4 = _ratio(wl.LAYOUT_135M)
    assert round(fp16 / 1e6) == 269
    assert abs(b4 / 1e6 - 110) < 3
    assert round(fp16 / b4, 1) == 2.4


def test_large_model_footprint_approaches_the_format_ratio():
    """Llama-70B-shaped layout: the linears dominate, so the whole-model ratio
    nears the format's own 16 / 4.127 = 3.9x (embeddings and head keep it
    a little below); the 4-bit model is inside the pages' 35-40 GB."""
    fp16, b4 = _ratio(wl.LAYOUT_70B)
    fmt = 16 / (8 * (q4.state_sizes("nf4", 8192 * 8192, 64, True)[0] +
                     sum(q4.state_sizes("nf4", 8192 * 8192, 64, True)[3:])) / (8192 * 8192))
    assert round(fmt, 1) == 3.9
    assert 3.7 < fp16 / b4 < fmt
    assert 35 <= b4 / 1e9 <= 40
    assert abs(fp16 / 1e9 - 140) < 5

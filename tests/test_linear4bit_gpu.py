"""Linear4bit on a B200: every forward route (decode GEMV up to 32 rows,
tcgen05 GEMM above, GEMV in 32-row pieces for other formats) against the
oracle's dequantize + binary64 matmul, plus replace_linear on a small model."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_matmul_close, bits, oracle_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import linear4bit, q4
    assert torch.cuda.is_available()
    return linear4bit, q4


@pytest.mark.parametrize("T", [1, 8, 32, 33, 100])
@pytest.mark.parametrize("fmt", [("nf4", 64, True), ("int4_sym", 128, False), ("int4_asym", 128, False)])
def test_linear4bit_forward_routes(mods, oracle, T, fmt):
    linear4bit, q4 = mods
    qtype, bs, dq = fmt
    g = torch.Generator().manual_seed(T + bs)
    N, K = 272, 1024
    lin = torch.nn.Linear(K, N)
    with torch.no_grad():
        lin.weight.copy_(torch.randn(N, K, generator=g) * 0.02)
        lin.bias.copy_(torch.randn(N, generator=g))
    lin = lin.to(torch.bfloat16).cuda()
    m = linear4bit.Linear4bit.from_linear(lin, bs, qtype, dq, compute_dtype=torch.bfloat16)
    x = torch.randn(T, K, generator=g).bfloat16()
    y = m(x.cuda().view(1, T, K))
    assert y.shape == (1, T, N) and y.dtype == torch.bfloat16
    ost = oracle_state(oracle, lin.weight.detach().cpu(), bs, {"nf4": 0, "int4_sym": 1, "int4_asym": 2}[qtype], dq)
    ref = oracle.gemv_reference(bits(x), True, ost, N, K)
    ref = ref + lin.bias.detach().float().cpu().double().numpy()[None, :]
    assert_matmul_close(y.view(T, N), ref)


def test_replace_linear_on_a_small_model(mods):
    """Swap a small model's linears: the 4-bit model equals the same model
    run on the dequantized weights (fp32 reference), stays near the 16-bit
    model (NF4 error of two layers, about 0.13 relative), keeps lm_head."""
    linear4bit, q4 = mods
    torch.manual_seed(0)
    model = torch.nn.Sequential(torch.nn.Linear(256, 512), torch.nn.GELU(), torch.nn.Linear(512, 256))
    with torch.no_grad():
        for lin in (model[0], model[2]):
            lin.weight.normal_(0, 0.05)
            lin.bias.normal_(0, 0.1)
    model.lm_head = torch.nn.Linear(256, 64)
    model = model.half().cuda()
    x = torch.randn(4, 256, device="cuda").half()
    with torch.no_grad():
        ref16 = model[2](model[1](model[0](x))).float()
    linear4bit.replace_linear(model)
    assert isinstance(model[0], linear4bit.Linear4bit) and isinstance(model[2], linear4bit.Linear4bit)
    assert type(model.lm_head) is torch.nn.Linear
    with torch.no_grad():
        y = model[2](model[1](model[0](x))).float()
        W0 = q4.dequantize(model[0].state, torch.float16).float()
        W2 = q4.dequantize(model[2].state, torch.float16).float()
        h = torch.nn.functional.gelu((x.float() @ W0.T + model[0].bias.float()).half().float())
        ref = (h.half().float() @ W2.T + model[2].bias.float())
    rel = ((y - ref).norm() / ref.norm()).item()
    assert rel < 5e-3, rel
    rel16 = ((y - ref16).norm() / ref16.norm()).item()
    assert rel16 < 0.25, rel16
    assert q4.last_device_status() == 0


def test_replace_linear_footprint_small_model(mods):
    """learn.pranaymahendrakar.com, "Loading a model in 4-bit": the 135M demo
    goes from 269 MB at fp16 to about 110 MB, 2.4x, because embeddings, the
    tied output head and the norms stay 16-bit.  The same layout, quantized
    for real by replace_linear (NF4, blocksize 64, double quantization), holds
    exactly the bytes the planned CPU footprint gives, and still runs."""
    linear4bit, q4 = mods
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    from model_layouts import DecoderSkeleton
    torch.manual_seed(0)
    model = DecoderSkeleton(wl.LAYOUT_135M, device="cuda", dtype=torch.float16)
    fp16 = linear4bit.memory_footprint(model)
    linear4bit.replace_linear(model, blocksize=64, qtype="nf4", double_quant=True)
    b4 = linear4bit.memory_footprint(model)
    assert type(model.lm_head) is torch.nn.Linear
    assert model.lm_head.weight is model.embed_tokens.weight
    assert round(fp16 / 1e6) == 269 and abs(b4 / 1e6 - 110) < 3
    assert round(fp16 / b4, 1) == 2.4
    blk = model.layers[0]
    assert isinstance(blk.down_proj, linear4bit.Linear4bit) and blk.down_proj.state.absmax is None
    x = torch.randn(3, 576, device="cuda").half()
    y = blk.down_proj(blk.gate_proj(x))
    assert y.shape == (3, 576) and torch.isfinite(y).all()
    assert q4.last_device_status() == 0

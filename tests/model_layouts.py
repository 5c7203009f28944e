"""A decoder-only model skeleton (embeddings, attention and MLP linears,
RMS-norm weights, output head) built from a layout in workloads.py, for the
Linear4bit memory-footprint checks.  Weights are random or on the meta
device: only shapes matter."""
import torch


class _Block(torch.nn.Module):
    def __init__(self, h, inter, heads, kv, device, dtype):
        super().__init__()
        hd = h // heads
        lin = lambda i, o: torch.nn.Linear(i, o, bias=False, device=device, dtype=dtype)
        self.q_proj, self.k_proj, self.v_proj, self.o_proj = lin(h, h), lin(h, kv * hd), lin(h, kv * hd), lin(h, h)
        self.gate_proj, self.up_proj, self.down_proj = lin(h, inter), lin(h, inter), lin(inter, h)
        self.input_norm = torch.nn.Parameter(torch.ones(h, device=device, dtype=dtype))
        self.post_norm = torch.nn.Parameter(torch.ones(h, device=device, dtype=dtype))


class DecoderSkeleton(torch.nn.Module):
    def __init__(self, layout, device="meta", dtype=torch.float16):
        super().__init__()
        h = layout["hidden"]
        self.embed_tokens = torch.nn.Embedding(layout["vocab"], h, device=device, dtype=dtype)
        self.layers = torch.nn.ModuleList([_Block(h, layout["inter"], layout["heads"], layout["kv_heads"],
                                                  device, dtype) for _ in range(layout["layers"])])
        self.norm = torch.nn.Parameter(torch.ones(h, device=device, dtype=dtype))
        self.lm_head = torch.nn.Linear(h, layout["vocab"], bias=False, device=device, dtype=dtype)
        if layout["tied"]:
            self.lm_head.weight = self.embed_tokens.weight

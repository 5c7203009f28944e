"""Llama-70B-shaped load-time quantize + decode over the whole 80-layer stack
(q 8192x8192, k/v 1024x8192, o 8192x8192, gate/up 28672x8192, down
8192x28672; shape templates only, synthetic N(0, 0.015) bf16 weights).

Each layer's weights are generated on the device from a seed, quantized to
NF4 blocksize 64 with double quantization and freed, so only the ~35 GB of
packed state stays resident.  Layers 0, 1, 39 and 79 are checked bit for bit
against the oracle (all state arrays) and their decode GEMV at M = 1, 8, 32
on sampled output rows; the GEMV then runs over the full stack at each M."""
import os

import numpy as np
import pytest
import torch

from gpu_helpers import assert_matmul_close, assert_state_equal, bits

pytestmark = pytest.mark.gpu

STD = 0.015
SEED = 70000
CHECK_LAYERS = (0, 1, 39, 79)
DECODE_M = (1, 8, 32)
SAMPLED_ROWS = 192


@pytest.fixture(scope="module")
def q4():
    from bit_blockwise_weight_absmax_b200 import build
    build.build()
    from bit_blockwise_weight_absmax_b200 import q4 as m
    assert torch.cuda.is_available()
    m.clear_device_status()
    return m


def _layer(wl, layer, device):
    """The seven bf16 weights of one layer (seed per layer and matrix)."""
    return [wl.gaussian((N, K), STD, torch.bfloat16, SEED + 16 * layer + i, device)
            for i, (_, N, K) in enumerate(wl.LAYER_70B)]


def test_70b_stack_quantize_and_decode(q4, oracle):
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    oracle.set_threads(os.cpu_count() or 1)
    rng = np.random.default_rng(70)
    stack = []
    for layer in range(wl.N_LAYERS_70B):
        Ws = _layer(wl, layer, "cuda")
        sts = [q4.quantize(W, 64, "nf4", True) for W in Ws]
        if layer in CHECK_LAYERS:
            for (name, N, K), W, st in zip(wl.LAYER_70B, Ws, sts):
                ost = oracle.quantize(bits(W), True, 64, 0, True)
                assert_state_equal(st, ost)
                # dequantized weights in the compute dtype of the decode GEMV
                # (fp16): bit-exact on every element
                deq = q4.dequantize(st, torch.float16)
                odeq = oracle.dequantize(ost, False)
                assert np.array_equal(bits(deq), odeq), (layer, name)
                rows = np.sort(rng.choice(N, SAMPLED_ROWS, replace=False))
                w16 = odeq.reshape(N, K)[rows].copy()
                del odeq
                for M in DECODE_M:
                    A = wl.activation(M, K, torch.float16, seed=SEED + 1000 * layer + M)
                    y = q4.gemv(A.cuda(), st)
                    ref = oracle.matmul(bits(A), False, w16, False, M, len(rows), K)
                    assert_matmul_close(y[:, torch.from_numpy(rows).cuda()], ref)
                del deq
        del Ws
        stack.append(sts)
    packed = sum(st.resident_bytes() for sts in stack for st in sts)
    assert 35.0e9 < packed < 35.7e9  # ~35.3 GB of packed weights and state
    assert q4.last_device_status() == 0

    # decode GEMV over the full stack, one grouped launch per layer
    for M in DECODE_M:
        A = [wl.activation(M, K, torch.float16, seed=SEED + 7 + M).cuda() for _, N, K in wl.LAYER_70B]
        outs = None
        for sts in stack:
            outs = q4.gemv_grouped(A, sts)
        torch.cuda.synchronize()
        assert all(torch.isfinite(y.float()).all().item() for y in outs)
        # the last layer's grouped result equals single-matrix calls up to
        # the order of the fp32 partial-sum additions
        for a, st, y in zip(A, stack[-1], outs):
            y1 = q4.gemv(a, st)
            d = (y1.float() - y.float()).abs().max().item()
            assert d <= 1e-3 * max(y1.float().abs().max().item(), 1e-30)
    assert q4.last_device_status() == 0

"""Benchmark of the blockwise 4-bit quantization hot path on B200.

One step = one pass of every hot-path operation over the Llama-2-7B-shaped
decoder layer (q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008):
  1. load-time quantize of L distinct layer copies (bf16 ~ N(0, 0.02) ->
     NF4 blocksize 64 with double quantization of the absmax), one grouped
     launch per layer plus its second-level launch;
  2. fused dequant-GEMV of every layer copy at decode batch M = 1, 4, 16
     (fp16 activations ~ N(0, 1), fp32 accumulate, fp16 out), one grouped
     launch per layer;
  3. dequantize of every layer copy to bf16, one grouped launch per layer;
  4. W4A16 tcgen05 GEMM of every layer copy at prefill M = 512 (bf16).
The L = 4 copies (~2 GB of inputs) rotate, so every kernel reads data that
was last touched more than the 126 MB L2 ago.  `value` is the headline
metric: GEMV effective HBM TB/s = algorithmic bytes (packed weights + block
state + activations + outputs) / device time of the GEMV launches; quantize
GB/s (input bytes / time) and every kernel's roofline are reported beside it.

Multi-GPU: the path does not shard (a single-GPU format and kernels); with
--gpus N every rank runs an independent replica (weak scaling) and the
whole-job value is the sum of bytes over the max time across ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "4-bit GEMV effective HBM TB/s (7B shapes, batch 1-16); quantize GB/s"
UNIT = "TB/s"
WORKLOAD = "llama2-7b-layer-nf4-b64-dq"
DECODE_M = (1, 4, 16)
PREFILL_M = 512
N_COPIES = 4


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the kernel on one layer of this workload, keyed by the
# SHA-256 of the kernel source it was taken on: a changed source reports null.
# Outputs still dirty in L2 when the kernel ends are not counted as writes.
NCU_TRAFFIC = {
    "gemm": ("bit_blockwise_weight_absmax_b200/csrc/gemm.cuh",
             "131690000b067cfa5b54292cd0fcbaaca0955854007702fa36d49b37172ba8dd", 142_834_176 + 19_374_592),
    "gemv": ("bit_blockwise_weight_absmax_b200/csrc/gemv_small.cuh",
             "e1c37f32b32c6306cbcee77f09a0121d152d14267279be05e5e7aa0ea42ff327", 108_468_224 + 3_651_840),
}


def _ncu_traffic(kernel):
    import hashlib
    if kernel not in NCU_TRAFFIC:
        return None
    path, digest, nbytes = NCU_TRAFFIC[kernel]
    with open(os.path.join(ROOT, path), "rb") as f:
        return nbytes if hashlib.sha256(f.read()).hexdigest() == digest else None


def _peaks():
    """The roofline denominators: the measured copy bandwidth and bf16 GEMM
    rates of MEASURED_PEAKS.json when it is present and readable, else the
    recipe's fallback figures (the source says which, and why)."""
    fallback = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return fallback
    try:
        with open(p) as f:
            d = json.load(f)
        out = {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
               "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
               "source": "measured"}
    except (OSError, ValueError, KeyError, TypeError) as e:
        return dict(fallback, source=f"fallback (MEASURED_PEAKS.json unreadable: {type(e).__name__})")
    if min(out["hbm_gbs"], out["bf16_tflops"], out["bf16_tflops_sustained"]) <= 0:
        return dict(fallback, source="fallback (MEASURED_PEAKS.json holds a non-positive peak)")
    return out


def layer_state_bytes(shapes, blocksize=64):
    """Resident NF4 + double-quant bytes of one layer (codes, int8 absmax
    codes, fp32 second-level scales, fp32 mean)."""
    tot = 0
    for _, N, K in shapes:
        n = N * K
        nb = -(-n // blocksize)
        tot += (n + 1) // 2 + nb + 4 * (-(-nb // 256)) + 4
    return tot


def gemv_bytes(shapes, M):
    return layer_state_bytes(shapes) + sum(2 * M * K + 2 * M * N for _, N, K in shapes)


def workload_config(L, world):
    """The `config` of both arms' JSON lines: the 7B-layer workload."""
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    n_params = sum(N * K for _, N, K in wl.LAYER_7B)
    state_b = layer_state_bytes(wl.LAYER_7B)
    return {"workload": WORKLOAD, "decode_M": list(DECODE_M), "prefill_M": PREFILL_M,
            "layer_copies": L, "blocksize": 64, "double_quant": True,
            "l2": f"{L} rotating layer copies (~{L * 2 * n_params / 1e9:.1f} GB bf16 + "
                  f"{L * state_b / 1e6:.0f} MB packed) > 126 MB L2",
            "parallelism": f"replicas x{world}"}


# ------------------------------------------------------------- replicas --
def max_over_ranks(values, world, device=None):
    """Element-wise max over all ranks of per-rank device times (ms): the
    slowest replica sets the whole job's time.  Identity at world size 1."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank, world, max_ms):
    """Units per second of the whole job: every rank's units over the
    slowest rank's time (weak scaling: each replica does the same work)."""
    return world * units_per_rank / (max_ms / 1e3)


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"q4_bench_clocks_rank{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded)}


# ------------------------------------------------------------- CPU oracle ---
def cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), else the platform's."""
    import platform
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def oracle_sample(rows_per_matrix=16, quantize_layer=True, seed=0, threads=None):
    """Time the oracle on a bounded sample of the same workload and scale it
    to one whole layer.  Quantize: NF4 + DQ of the full layer (all seven
    matrices) when `quantize_layer`, else of the 4096x4096 q matrix.  GEMV:
    the reference (dequantize + binary64 matmul) of the first
    `rows_per_matrix` output rows of every matrix at M = 1, 4, 16; each
    matrix's time is scaled by N / rows to the full matrix, and the value is
    the layer's algorithmic GEMV bytes over the scaled time, summed over M
    like the GPU arm.  Returns (TB/s, quantize GB/s, threads, description,
    seconds spent, scaled ms of the whole layer's GEMVs at the three M)."""
    import numpy as np
    import torch

    import oracle
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    threads = oracle.set_threads(threads or os.cpu_count() or 1)
    t0 = time.perf_counter()
    q_bytes, tq = 0, 0.0
    for i, (_, N, K) in enumerate(wl.LAYER_7B if quantize_layer else wl.LAYER_7B[:1]):
        W = wl.gaussian((N, K), 0.02, torch.bfloat16, seed + 100 + i)
        wb = W.view(torch.int16).numpy().view(np.uint16).reshape(-1)
        del W
        t = time.perf_counter()
        oracle.quantize(wb, True, 64, oracle.QT_NF4, True)
        tq += time.perf_counter() - t
        q_bytes += wb.size * 2
    q_gbs = q_bytes / tq / 1e9
    t_full = {M: 0.0 for M in DECODE_M}
    for i, (_, N, K) in enumerate(wl.LAYER_7B):
        r = min(rows_per_matrix, N)
        Wr = wl.gaussian((r, K), 0.02, torch.bfloat16, seed + 1 + i)
        st = oracle.quantize(Wr.view(torch.int16).numpy().view(np.uint16).reshape(-1), True, 64,
                             oracle.QT_NF4, True)
        for M in DECODE_M:
            A = wl.activation(M, K, torch.float16, seed + 50 + i)
            ab = A.view(torch.int16).numpy().view(np.uint16).reshape(-1)
            t = time.perf_counter()
            oracle.gemv_reference(ab, False, st, r, K)
            t_full[M] += (time.perf_counter() - t) * N / r
    tb = sum(gemv_bytes(wl.LAYER_7B, M) for M in DECODE_M) / sum(t_full.values()) / 1e12
    whole = all(rows_per_matrix >= N for _, N, K in wl.LAYER_7B)
    gemv_part = ("GEMV reference (dequantize + fp64 matmul) of the whole layer at M=1,4,16" if whole else
                 f"GEMV reference (dequantize + fp64 matmul) of the first {rows_per_matrix} output rows "
                 f"of each of the 7 layer matrices at M=1,4,16, each matrix's time scaled by N/rows "
                 f"to the whole layer")
    desc = (f"oracle on {threads} host threads: NF4+DQ quantize of "
            f"{'the whole 7B layer (7 matrices, 202M bf16 weights)' if quantize_layer else 'the 4096x4096 q matrix'}"
            f"; {gemv_part}")
    return tb, q_gbs, threads, desc, time.perf_counter() - t0, sum(t_full.values()) * 1e3


def run_reference(args, rank, world):
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    vals, qs, ms, wall = [], [], [], []
    for i in range(warm + steps):
        t0 = time.perf_counter()
        tb, qg, thr, desc, secs, est_ms = oracle_sample(rows_per_matrix=args.ref_rows, quantize_layer=False,
                                                       seed=i)
        if i >= warm:
            wall.append((time.perf_counter() - t0) * 1e3)
            vals.append(tb)
            qs.append(qg)
            ms.append(est_ms)
    v = statistics.mean(vals)
    # ms_per_step: the wall time of one step as it ran (the bounded sample);
    # the whole-layer GEMV time that sample scales to is a separate key
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": statistics.mean(wall),
            "layer_gemv_ms_estimate": statistics.mean(ms), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64", "data": "synthetic",
            "config": workload_config(args.copies, world),
            "quantize_gbs": statistics.mean(qs),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": thr, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm --
def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from bit_blockwise_weight_absmax_b200 import q4
    from bit_blockwise_weight_absmax_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    shapes = wl.LAYER_7B
    peaks = _peaks()
    L = args.copies

    # ---- inputs resident in HBM before timing (seeded, generated on device)
    Ws = [[wl.gaussian((N, K), 0.02, torch.bfloat16, 1000 * l + i + 17 * rank, dev)
           for i, (_, N, K) in enumerate(shapes)] for l in range(L)]
    A_dec = {M: [wl.activation(M, K, torch.float16, 7000 + 10 * M + i, dev) for i, (_, N, K) in enumerate(shapes)]
             for M in DECODE_M}
    A_pre = [wl.activation(PREFILL_M, K, torch.bfloat16, 9000 + i, dev) for i, (_, N, K) in enumerate(shapes)]
    states = [[q4.quantize(w, 64, "nf4", True) for w in layer] for layer in Ws]
    y_dec = {M: [[torch.empty(M, N, dtype=torch.float16, device=dev) for _, N, K in shapes]
                 for _ in range(L)] for M in DECODE_M}
    deq_out = [torch.empty(N, K, dtype=torch.bfloat16, device=dev) for _, N, K in shapes]
    y_pre = [torch.empty(PREFILL_M, N, dtype=torch.bfloat16, device=dev) for _, N, K in shapes]
    torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)
    n_params = sum(N * K for _, N, K in shapes)

    # Every phase is one CUDA graph of library launches (captured once after
    # an eager warm-up), so no host-side marshalling falls inside a timed
    # interval; graphs replay back to back on one stream.
    def ph_quantize():
        for l in range(L):
            q4.quantize_grouped(Ws[l], 64, "nf4", True, outs=states[l])

    def ph_gemv(M):
        for l in range(L):
            q4.gemv_grouped(A_dec[M], states[l], outs=y_dec[M][l])

    def ph_dequantize():
        for l in range(L):
            q4.dequantize_grouped(states[l], torch.bfloat16, outs=deq_out)

    def ph_gemm():
        for l in range(L):
            q4.gemm_grouped(A_pre, states[l], outs=y_pre)

    fns = {"quantize": ph_quantize}
    for M in DECODE_M:
        fns[f"gemv_m{M}"] = (lambda M=M: ph_gemv(M))
    fns["dequantize"] = ph_dequantize
    fns["gemm"] = ph_gemm
    phases = list(fns)
    # one grouped launch per layer (quantize: plus its second-level launch)
    launches = {"quantize": L * 2, "dequantize": L, "gemm": L}
    for M in DECODE_M:
        launches[f"gemv_m{M}"] = L
    launches_per_step = sum(launches.values())
    if args.profile:
        # a short eager run of one phase for a profiler capture (no timing)
        for _ in range(1 + args.steps):
            fns[args.profile]()
        torch.cuda.synchronize()
        if rank == 0:
            print(json.dumps({"profile": args.profile, "launches": launches[args.profile] * (1 + args.steps)}))
        return
    for f in fns.values():
        f()
    torch.cuda.synchronize()
    graphs = {}
    for name, f in fns.items():
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            f()
        graphs[name] = g
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step(rec):
        for name in phases:
            e0, e1 = ev(), ev()
            e0.record(stream)
            graphs[name].replay()
            e1.record(stream)
            rec[name].append((e0, e1))

    for _ in range(args.warmup):
        step({p: [] for p in phases})
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    rec = {p: [] for p in phases}
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for _ in range(args.steps):
        step(rec)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()

    total_ms = t_start.elapsed_time(t_end)
    ph_ms = {p: sum(a.elapsed_time(b) for a, b in rec[p]) for p in phases}
    gemv_B = {M: gemv_bytes(shapes, M) * L * args.steps for M in DECODE_M}
    gemv_ms = sum(ph_ms[f"gemv_m{M}"] for M in DECODE_M)
    q_in_bytes = 2 * n_params * L * args.steps
    state_b = layer_state_bytes(shapes)
    q_alg_bytes = (2 * n_params + state_b) * L * args.steps
    deq_alg_bytes = (state_b + 2 * n_params) * L * args.steps
    gemm_flops = 2 * PREFILL_M * n_params * L * args.steps

    # max over ranks of the device times; value = all ranks' bytes / that time
    vec = max_over_ranks([total_ms, gemv_ms] + [ph_ms[p] for p in phases], world, dev)
    total_ms, gemv_ms = vec[0], vec[1]
    ph_ms = {p: vec[2 + i] for i, p in enumerate(phases)}

    value = whole_job_rate(sum(gemv_B.values()), world, gemv_ms) / 1e12
    # effective TB/s counts weights + state + A + Y; weight_tb_s the packed
    # weights and their state alone
    per_m = {f"M={M}": {"tb_s": gemv_B[M] / (ph_ms[f"gemv_m{M}"] / 1e3) / 1e12,
                        "weight_tb_s": gemv_B[M] * layer_state_bytes(shapes) / gemv_bytes(shapes, M)
                                       / (ph_ms[f"gemv_m{M}"] / 1e3) / 1e12,
                        "us_per_layer": ph_ms[f"gemv_m{M}"] * 1e3 / (L * args.steps),
                        "bytes_per_layer": gemv_bytes(shapes, M)} for M in DECODE_M}
    hbm = peaks["hbm_gbs"]
    quant_gbs = q_in_bytes / (ph_ms["quantize"] / 1e3) / 1e9
    rooflines = {
        "quantize": {"bound": "hbm", "achieved": q_alg_bytes / (ph_ms["quantize"] / 1e3) / 1e9,
                     "peak": hbm, "unit": "GB/s"},
        "gemv": {"bound": "hbm", "achieved": sum(gemv_B.values()) / (gemv_ms / 1e3) / 1e9, "peak": hbm,
                 "unit": "GB/s"},
        "dequantize": {"bound": "hbm", "achieved": deq_alg_bytes / (ph_ms["dequantize"] / 1e3) / 1e9,
                       "peak": hbm, "unit": "GB/s"},
        # each GEMM launch runs ~0.3 ms at full clocks, not a seconds-long
        # power-capped loop: the burst cuBLAS figure is its peak
        "gemm": {"bound": "tensor", "achieved": gemm_flops / (ph_ms["gemm"] / 1e3) / 1e12,
                 "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"},
    }
    for r in rooflines.values():
        r["frac"] = r["achieved"] / r["peak"]
    dominant = max(["quantize", "dequantize", "gemm"] + ["gemv"],
                   key=lambda k: gemv_ms if k == "gemv" else ph_ms[k])
    dom = dict(rooflines[dominant])
    dom["kernel"] = dominant
    dom["launch_us"] = (gemv_ms if dominant == "gemv" else ph_ms[dominant]) * 1e3 / (
        args.steps * (L * len(DECODE_M) if dominant == "gemv" else launches[dominant]))
    dom["traffic"] = _ncu_traffic(dominant)
    dom["traffic_unit"] = "bytes per launch (ncu, one layer)"
    dom["peak_source"] = (f"{peaks['source']} "
                          f"({'bf16_tflops, burst: launches of ~0.3 ms' if dom['bound'] == 'tensor' else 'hbm_gbs'})")

    # ---- end to end through the public API: pinned host activations in,
    # results back to host, weights resident (quantized at load time)
    e2e = None
    if not args.no_e2e:
        # every activation of a step (each M, each layer copy, each matrix)
        # lives in one pinned host buffer and every output in another; per
        # batch size one host-to-device and one device-to-host transfer on a
        # copy stream, ordered by events against the GEMVs, so a batch
        # size's copies overlap the others' GEMVs (batch sizes run 1, 16, 4:
        # the first input and the last output exposed are small)
        order = [1, 16, 4] if sorted(DECODE_M) == [1, 4, 16] else list(DECODE_M)
        a_sizes = [(M, l, i, M * K) for M in order for l in range(L) for i, (_, N, K) in enumerate(shapes)]
        y_sizes = [(M, l, i, M * N) for M in order for l in range(L) for i, (_, N, K) in enumerate(shapes)]
        host_a = torch.empty(sum(n for *_, n in a_sizes), dtype=torch.float16).pin_memory()
        host_y = torch.empty(sum(n for *_, n in y_sizes), dtype=torch.float16).pin_memory()
        dev_a = torch.empty(host_a.numel(), dtype=torch.float16, device=dev)
        dev_y = torch.empty(host_y.numel(), dtype=torch.float16, device=dev)
        a_views, y_views, a_span, y_span, off = {}, {}, {}, {}, 0
        for M, l, i, n in a_sizes:
            K = shapes[i][2]
            host_a[off:off + n].copy_(A_dec[M][i].reshape(-1).cpu())
            a_views[(M, l, i)] = dev_a[off:off + n].view(M, K)
            a_span[M] = (a_span.get(M, (off, off))[0], off + n)
            off += n
        off = 0
        for M, l, i, n in y_sizes:
            y_views[(M, l, i)] = dev_y[off:off + n].view(M, shapes[i][1])
            y_span[M] = (y_span.get(M, (off, off))[0], off + n)
            off += n
        args_e2e = {(M, l): ([a_views[(M, l, i)] for i in range(len(shapes))],
                             [y_views[(M, l, i)] for i in range(len(shapes))])
                    for M in order for l in range(L)}
        h2d = host_a.numel() * 2
        d2h = host_y.numel() * 2
        copy_stream = torch.cuda.Stream(device=dev)

        def e2e_step():
            a_in, y_out = {}, {}
            with torch.cuda.stream(copy_stream):
                for M in order:
                    a0, a1 = a_span[M]
                    dev_a[a0:a1].copy_(host_a[a0:a1], non_blocking=True)
                    a_in[M] = torch.cuda.Event()
                    a_in[M].record(copy_stream)
            for M in order:
                stream.wait_event(a_in[M])
                for l in range(L):
                    a_l, y_l = args_e2e[(M, l)]
                    q4.gemv_grouped(a_l, states[l], outs=y_l, stream=stream)
                y_out[M] = torch.cuda.Event()
                y_out[M].record(stream)
            with torch.cuda.stream(copy_stream):
                for M in order:
                    copy_stream.wait_event(y_out[M])
                    y0, y1 = y_span[M]
                    host_y[y0:y1].copy_(dev_y[y0:y1], non_blocking=True)
            stream.wait_stream(copy_stream)
            copy_stream.synchronize()  # the step's results are on the host
        for _ in range(max(1, args.warmup)):
            e2e_step()
        e0, e1 = ev(), ev()
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0]
        e2e = {"value": whole_job_rate(sum(gemv_B.values()), world, e2e_ms) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "what": "q4.gemv_grouped at M=1,4,16 over the resident layer copies; every step copies all "
                       "its activations from pinned host memory (one transfer per batch size) and reads "
                       "every output back (one transfer per batch size) on a copy stream that overlaps "
                       "the other batch sizes' GEMVs; the host waits for each step's results"}

    # ---- the pages' own method, timed beside the fused path on the same
    # resident states: dequantize every weight to a 16-bit buffer, then a
    # library (cuBLAS) matmul.  Same algorithmic bytes / flops as the fused
    # phases, so the ratio is the fusion's gain.
    unfused = None
    if not args.no_unfused:
        w16 = {dt: [torch.empty(N, K, dtype=dt, device=dev) for _, N, K in shapes]
               for dt in (torch.float16, torch.bfloat16)}

        def un_gemv(M):
            for l in range(L):
                for st, w, a, y in zip(states[l], w16[torch.float16], A_dec[M], y_dec[M][l]):
                    q4.dequantize(st, torch.float16, out=w)
                    torch.matmul(a, w.t(), out=y)

        def un_gemm():
            for l in range(L):
                for st, w, a, y in zip(states[l], w16[torch.bfloat16], A_pre, y_pre):
                    q4.dequantize(st, torch.bfloat16, out=w)
                    torch.matmul(a, w.t(), out=y)

        ufns = {f"gemv_m{M}": (lambda M=M: un_gemv(M)) for M in DECODE_M}
        ufns["gemm"] = un_gemm
        for f in ufns.values():
            f()
        torch.cuda.synchronize()
        ugraphs = {}
        for name, f in ufns.items():
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                f()
            ugraphs[name] = g
        for g in ugraphs.values():
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ums = {}
        for name, g in ugraphs.items():
            e0, e1 = ev(), ev()
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            ums[name] = e0.elapsed_time(e1)
        uv = max_over_ranks([ums[n] for n in ufns], world, dev)
        ums = dict(zip(ufns, uv))
        ugemv_ms = sum(ums[f"gemv_m{M}"] for M in DECODE_M)
        unfused = {
            "what": "q4.dequantize of every weight to a 16-bit buffer, then torch.matmul (cuBLAS), "
                    "per matrix; same workload, bytes and flops as the fused phases",
            "gemv_tb_s": whole_job_rate(sum(gemv_B.values()), world, ugemv_ms) / 1e12,
            "gemv_us_per_layer": {f"M={M}": ums[f"gemv_m{M}"] * 1e3 / (L * args.steps) for M in DECODE_M},
            "gemm_tflops": whole_job_rate(gemm_flops, world, ums["gemm"]) / 1e12,
            "fused_speedup": {"gemv": ugemv_ms / gemv_ms, "gemm": ums["gemm"] / ph_ms["gemm"]},
        }
        del w16, ugraphs

    # ---- the larger configurations, outside the step: prefill GEMM at
    # M = 2048 / 8192 on the resident 7B-layer states, and the 70B stack
    large = None
    if not args.no_large:
        large = {"prefill_gemm": prefill_large(states, shapes, dev, peaks["bf16_tflops"]),
                 "stack70b": stack70b(max(3, min(args.steps, 10)), args.warmup, dev)}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        tb, qg, thr, desc, secs, _ = oracle_sample(rows_per_matrix=args.cpu_rows)
        cpu = {"value": tb, "unit": UNIT, "cores": thr, "kind": "oracle", "sample": desc,
               "quantize_gbs": qg, "seconds": round(secs, 1), "cpu_model": cpu_model()}
        # the same oracle on one thread, on a smaller sample (the q matrix's
        # quantize, 16 output rows per matrix for the GEMV reference)
        tb1, qg1, thr1, desc1, secs1, _ = oracle_sample(rows_per_matrix=16, quantize_layer=False, threads=1)
        cpu["single_thread"] = {"value": tb1, "unit": UNIT, "cores": thr1, "quantize_gbs": qg1, "sample": desc1,
                                "seconds": round(secs1, 1)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic (seeded Gaussian weights of 7B-layer shapes; no checkpoint)",
            "config": workload_config(L, world),
            "quantize_gbs": quant_gbs,
            "gemv_per_m": per_m,
            "phase_ms_per_step": {p: ph_ms[p] / args.steps for p in phases},
            "roofline": dom,
            "rooflines": rooflines,
            "gpu_launches": launches_per_step * args.steps,
            "launches_per_step": launches,
            "clocks": clk,
            "e2e": e2e,
            "unfused_baseline": unfused,
            "large_configs": large,
            "cpu_baseline": cpu,
            "peaks": peaks,
        }
        print(json.dumps(line), flush=True)


def prefill_large(states_l, shapes, dev, peak_tflops, reps=3):
    """The prefill GEMM at the larger batch sizes of the 7B-layer workload
    (M = 2048 and 8192, bf16 activations ~ N(0, 1)): one grouped launch per
    resident layer copy, captured in a CUDA graph, timed with CUDA events."""
    import torch

    from bit_blockwise_weight_absmax_b200 import q4
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    n_params = sum(N * K for _, N, K in shapes)
    out = {}
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for M in (2048, 8192):
        A = [wl.activation(M, K, torch.bfloat16, 9100 + M + i, dev) for i, (_, N, K) in enumerate(shapes)]
        Y = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _, N, K in shapes]

        def rnd():
            for sts in states_l:
                q4.gemm_grouped(A, sts, outs=Y)
        rnd()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            rnd()
        g.replay()
        e0, e1 = ev(), ev()
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / (reps * len(states_l))
        tf = 2 * M * n_params / (ms / 1e3) / 1e12
        out[f"M={M}"] = {"tflops": tf, "us_per_layer": ms * 1e3, "frac_of_bf16_burst": tf / peak_tflops}
        del g, A, Y
    return out


def stack70b(steps, warmup, dev):
    """The Llama-70B-shaped stack (80 layers; shape templates, synthetic
    N(0, 0.015) bf16 weights generated per layer on the device, quantized to
    NF4 blocksize 64 with double quantization, bf16 freed): load-time
    quantize rate (CUDA events around each layer's grouped quantize) and the
    decode GEMV over the whole stack, one grouped launch per layer, at
    M = 1, 8, 32.  Returns a dict."""
    import torch

    from bit_blockwise_weight_absmax_b200 import q4
    from bit_blockwise_weight_absmax_b200 import workloads as wl
    shapes = wl.LAYER_70B
    ev = lambda: torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    stack, qev = [], []
    for layer in range(wl.N_LAYERS_70B):
        Ws = [wl.gaussian((N, K), 0.015, torch.bfloat16, 70000 + 16 * layer + i, dev)
              for i, (_, N, K) in enumerate(shapes)]
        # the layer's states are allocated before the timed launch (an
        # allocation inside it would time the host, not the kernel); the
        # first layer also sizes the workspace, untimed
        sts = [q4._new_state(q4.QTYPES["nf4"], torch.bfloat16, N, K, 64, True, dev) for _, N, K in shapes]
        if layer == 0:
            q4.quantize_grouped(Ws, 64, "nf4", True, outs=sts)
        e0, e1 = ev(), ev()
        e0.record()
        q4.quantize_grouped(Ws, 64, "nf4", True, outs=sts)
        e1.record()
        qev.append((e0, e1))
        for st in sts:
            st.release_absmax()  # a resident model keeps only what the consumers read
        stack.append(sts)
        del Ws
    torch.cuda.synchronize()
    load_s = time.perf_counter() - t0
    q_ms = sum(a.elapsed_time(b) for a, b in qev)
    n_params = wl.N_LAYERS_70B * sum(N * K for _, N, K in shapes)
    resident = sum(st.resident_bytes() for sts in stack for st in sts)
    per_m = {}
    for M in (1, 8, 32):
        A = [wl.activation(M, K, torch.float16, 7 + i, dev) for i, (_, N, K) in enumerate(shapes)]
        Y = [[torch.empty(M, N, dtype=torch.float16, device=dev) for _, N, K in shapes] for _ in stack]

        def token_step():
            for sts, ys in zip(stack, Y):
                q4.gemv_grouped(A, sts, outs=ys)
        token_step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            token_step()
        for _ in range(max(3, warmup)):
            g.replay()
        e0, e1 = ev(), ev()
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        nbytes = wl.N_LAYERS_70B * gemv_bytes(shapes, M)
        per_m[f"M={M}"] = {"ms_per_token_step": ms, "tb_s": nbytes / (ms / 1e3) / 1e12,
                           "bytes_per_token_step": nbytes}
        del g, Y
    del stack
    torch.cuda.empty_cache()
    return {"workload": "llama-70b-stack-80-layers-nf4-b64-dq", "resident_gb": resident / 1e9,
            "quantize_gbs": 2 * n_params / (q_ms / 1e3) / 1e9, "quantize_ms": q_ms,
            "load_s_with_generation": load_s, "steps": steps, "gemv_per_m": per_m}


def run_stack70b(args):
    """--stack70b: only the 70B-stack block, as its own JSON line."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = stack70b(args.steps, args.warmup, dev)
    d.update({"metric": "70B-stack decode GEMV effective HBM TB/s", "unit": "TB/s"})
    print(json.dumps(d), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="q4", choices=["q4", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--stack70b", action="store_true",
                    help="time the decode GEMV over the Llama-70B-shaped 80-layer stack instead (one JSON line)")
    ap.add_argument("--no-unfused", action="store_true",
                    help="skip timing the unfused dequantize-then-cuBLAS baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=11008,
                    help="output rows per matrix in the timed oracle sample (cpu_baseline); "
                         "the default covers every row of the layer")
    ap.add_argument("--ref-rows", type=int, default=64,
                    help="output rows per matrix in each step of --impl reference")
    ap.add_argument("--no-large", action="store_true",
                    help="skip the prefill GEMM at M = 2048 / 8192 and the 70B-stack block")
    ap.add_argument("--profile", default=None,
                    help="run one phase eagerly (quantize, gemv_m1, gemv_m4, gemv_m16, dequantize, "
                         "gemm) --steps+1 times for a profiler capture; prints no metric")
    ap.add_argument("--copies", type=int, default=N_COPIES,
                    help="distinct layer copies that rotate through the step")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.stack70b:
        if rank == 0:
            run_stack70b(args)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

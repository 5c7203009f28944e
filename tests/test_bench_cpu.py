"""The replica path of bench.py on CPU: world size 2 over gloo.

The hot path does not shard (one GPU holds a whole 70B stack), so with
--gpus N every rank runs an independent replica and the only cross-rank
step is the max of the device times.  These tests run that step, and the
reference arm's rank gating, as two gloo processes on 127.0.0.1."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r took (r + 1) ms for phase 0 and (10 - r) ms for phase 1
        mx = bench.max_over_ranks([rank + 1.0, 10.0 - rank], world)
        rate = bench.whole_job_rate(1e9, world, mx[0])
        # the reference arm: rank 0 alone works; the others return at once
        class A:
            steps, warmup = 0, 0
        skipped = bench.run_reference(A, rank, world) is None if rank else True
        q.put((rank, mx, rate, skipped))
    finally:
        dist.destroy_process_group()


def test_replicas_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(2))
    for rank, mx, rate, skipped in got:
        assert mx == [2.0, 10.0]                 # the slowest rank per phase
        assert rate == pytest.approx(2 * 1e9 / 2e-3)  # both ranks' units over the max time
        assert skipped


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.5, 4.0], 1) == [3.5, 4.0]
    assert bench.whole_job_rate(5e8, 1, 2.0) == pytest.approx(2.5e11)


def test_reference_arm_json_line(capsys):
    """The reference arm (the oracle on the host) prints one JSON line with
    the contract's keys and the same config as the GPU arm."""
    import json

    import bench

    class A:
        steps, warmup, copies, ref_rows = 1, 0, bench.N_COPIES, 16
    bench.run_reference(A, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["config"] == bench.workload_config(bench.N_COPIES, 1)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # ms_per_step is the step's measured wall time, not the whole-layer estimate
    assert 0 < line["ms_per_step"] < line["layer_gemv_ms_estimate"]


def test_peaks_measured_fallback_and_unreadable(tmp_path, monkeypatch):
    """The roofline denominators: MEASURED_PEAKS.json when present and
    readable, else the recipe's fallback, with the reason in `source`."""
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._peaks() == {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                              "source": "fallback"}
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text('{"hbm_gbs": 6542.1, "bf16_tflops": 1641.8, "bf16_tflops_sustained": 1367.1}')
    p = bench._peaks()
    assert p["source"] == "measured" and (p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"]) == (
        6542.1, 1641.8, 1367.1)
    f.write_text('{"hbm_gbs": 6542.1, "bf16_tflops": 1641.8}')  # no sustained figure: the burst one
    assert bench._peaks()["bf16_tflops_sustained"] == 1641.8
    for bad in ('{"hbm_gbs": 6542.1}', "not json", '{"hbm_gbs": "x", "bf16_tflops": 1}',
                '{"hbm_gbs": 0, "bf16_tflops": 1641.8}'):
        f.write_text(bad)
        p = bench._peaks()
        assert p["source"].startswith("fallback (") and p["hbm_gbs"] == 6650.0, bad

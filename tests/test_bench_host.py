"""Host-side logic of bench.py: cross-rank aggregation over gloo (2 ranks, CPU) and the JSON helpers."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    # rank r timed (r+1) seconds for 10*(r+1) units of work
    t, u = bench.aggregate(float(rank + 1), 10.0 * (rank + 1))
    bench.barrier()
    out[rank] = (t, u)
    dist.destroy_process_group()


def test_aggregate_max_time_sum_units_over_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    # every rank sees the slowest rank's time and the work of all ranks
    assert res == {0: (2.0, 30.0), 1: (2.0, 30.0)}


def test_aggregate_single_process_is_identity():
    import bench
    assert bench.aggregate(1.5, 7.0) == (1.5, 7.0)


def test_reference_arm_rank_nonzero_does_nothing(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_warmup_floor():
    import bench
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_traffic_is_null_when_kernel_changed(tmp_path, monkeypatch):
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1")
    digest = bench.source_digest(["k.cuh"])
    (tmp_path / "profiles" / "p.txt").write_text("source_digest: %s\ndram_bytes_per_launch_full_workload: 123\n" % digest)
    assert bench.profiled_traffic("p.txt", ["k.cuh"]) == 123.0
    src.write_text("kernel v2")
    assert bench.profiled_traffic("p.txt", ["k.cuh"]) is None


def test_cost_model_arithmetic():
    # alpha F + beta M with alpha, beta the reciprocal peaks; the roofline is the larger term
    import bench
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    c = bench.cost_model(2e12, 1e10, 0.004, peaks, standard_bytes=3e10)
    assert abs(c["predicted_ms"] - (2.0 + 2.0)) < 1e-9          # 2e12 / 1e15 s + 1e10 / 5e12 s
    assert abs(c["roofline_ms"] - 2.0) < 1e-9
    assert abs(c["measured_over_predicted"] - 1.0) < 1e-9
    assert abs(c["standard_predicted_ms"] - 8.0) < 1e-9           # 2 ms + 3e10 / 5e12 s
    assert abs(c["predicted_speedup_vs_standard"] - 2.0) < 1e-9


def test_standard_traffic_counts_every_pair():
    import bench
    from seeded_inputs import workloads as W
    w = W.CFG2C  # causal: the standard implementation still forms every (query, key) pair
    assert bench.standard_bytes(w) == w.bytes() + 4 * 16 * 2048 * 2048 * 12


def test_flop_convention():
    # two matrix products at 2 FLOP per multiply-add; a causal mask halves the count
    # (the convention of the 2-simplicial article, "model design")
    from seeded_inputs import workloads as W
    assert W.CFG2.flops() == 4.0 * 4 * 16 * 2048 * 2048 * 64
    assert W.CFG2C.flops() == W.CFG2.flops() / 2


def test_reference_arm_prints_one_contract_line():
    # The reference arm (the CPU oracle) end to end: one JSON line with the contract's keys,
    # measured on a bounded sample (about a second of oracle work here).
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-seconds", "1"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["unit"] == "TFLOP/s"
    assert d["config"]["workload"].startswith("cfg4")  # the same workload as the headline of our arm
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_roofline_reports_both_denominators():
    # achieved = algorithmic FLOPs / mean launch time, against the measured burst peak and the spec figure
    import bench
    r = bench.tensor_roofline("k", 2e12, 1e9, 0.002, {"bf16_tflops": 1600.0}, "measured", 3e9, "p.txt")
    assert r["achieved"] == 1000.0 and r["unit"] == "TFLOP/s" and r["bound"] == "tensor"
    assert r["frac"] == 0.625 and r["peak"] == 1600.0
    assert r["spec_peak"] == 2250.0 and abs(r["spec_frac"] - 1000.0 / 2250.0) < 1e-4
    assert r["traffic"] == 3e9 and r["traffic_over_algorithmic_bytes"] == 3.0
    h = bench.hbm_roofline("d", 6e9, 0.001, {"hbm_gbs": 6000.0}, "measured", None)
    assert h["achieved"] == 6000.0 and h["frac"] == 1.0 and h["spec_frac"] == 0.75 and h["traffic"] is None


def test_every_prefill_workload_is_described_and_defined():
    import bench
    from seeded_inputs import workloads as W
    for name in bench.PREFILL_WORKLOADS:
        w = bench.workload(name)
        assert w.name == name and bench.DESCRIBE[name].startswith(name + ":")
        assert bench.kernel_name(w).startswith("sdpa_fwd_bf16_kernel<%d," % w.d)
    assert bench.kernel_name(W.CFG3W).endswith(",2>") and bench.kernel_name(W.CFG3).endswith(",1>")

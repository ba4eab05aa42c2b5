"""The JSON line bench.py prints: every key the benchmark contract names, with the right types.

report() is fed synthetic stage times (no GPU); the oracle timing is replaced by a
stub so the test stays fast.
"""
import argparse
import json

import pytest

import bench
from sparse_moe_layer_03_b200 import inputs as I


@pytest.mark.parametrize("fused,exchange", [(True, False), (False, False), (True, True)])
def test_report_has_the_contract_keys(monkeypatch, fused, exchange):
    monkeypatch.setattr(bench, "calibrated_tokens", lambda w, inp, s: 128)
    monkeypatch.setattr(bench, "oracle_rate", lambda w, inp, n: (700.0, 0.18, 8))
    w = I.WORKLOADS["xl2_8e2a_512"]
    args = argparse.Namespace(steps=20, warmup=5, workload="xl2_8e2a_512", adaln="off", fuse_combine="on",
                              global_aux="on" if exchange else "off")
    stages = {"route": [0.03] * 20, "dispatch": [0.05] * 20, "gemm1": [1.1] * 20}
    if exchange:
        stages["balance_exchange"] = [0.01] * 20
    if fused:
        stages["gemm2_combine"] = [1.12] * 20
    else:
        stages.update(gemm2=[1.08] * 20, combine=[0.06] * 20)
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 5}
    r = bench.report(args, w, None, stages, 2.3, 2.5, clocks, 1, {})
    line = json.loads(json.dumps(r))                     # one JSON-serialisable object
    for k, t in [("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                 ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool), ("scaling", str),
                 ("dtype", str), ("data", str), ("config", dict), ("roofline", dict), ("cpu_baseline", dict),
                 ("e2e", dict), ("gpu_launches", int), ("clocks", dict)]:
        assert isinstance(line[k], t), k
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s" and line["scaling"] == "weak"
    assert line["vs_baseline"] is None
    assert abs(line["value"] - w.T / 2.3e-3) < 1.0
    assert line["config"]["workload"] == w.name
    rf = line["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s" and abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    assert "traffic" in rf
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 8 and cb["unit"] == "tokens/s" and cb["sample"]
    e2e = line["e2e"]
    assert e2e["unit"] == "tokens/s" and e2e["h2d_bytes_per_step"] == w.T * w.D * 2
    assert e2e["d2h_bytes_per_step"] == w.T * w.D * 2 + 4
    assert line["gpu_launches"] == ((5 if fused else 6) + (2 if exchange else 0)) * 20
    assert ("balance_exchange" in line["stages"]) == exchange
    assert line["config"]["balance_loss"].startswith("whole batch" if exchange else "per rank")
    assert set(line["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    nom = line["vs_nominal"]
    assert abs(nom["gemm_frac"] - line["gemm_tflops"] / 2250.0) < 2e-3
    assert abs(nom["mem_stages_frac"] - line["mem_stages_GBps"] / 8000.0) < 2e-3


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2", "--steps", "1"])


def test_report_fp16_and_per_image_loss(monkeypatch):
    import dataclasses
    monkeypatch.setattr(bench, "calibrated_tokens", lambda w, inp, s: 128)
    monkeypatch.setattr(bench, "oracle_rate", lambda w, inp, n: (700.0, 0.18, 8))
    w = dataclasses.replace(I.WORKLOADS["xl2_8e2a_512"], dtype="f16")
    args = argparse.Namespace(steps=10, warmup=3, workload="xl2_8e2a_512", adaln="off", fuse_combine="on",
                              global_aux="off", seq_len=1024, dtype="f16")
    stages = {"route": [0.04] * 10, "dispatch": [0.05] * 10, "gemm1": [1.1] * 10, "gemm2_combine": [1.12] * 10}
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5}
    line = json.loads(json.dumps(bench.report(args, w, None, stages, 2.31, 2.5, clocks, 1, {})))
    assert line["dtype"] == "f16"
    assert line["roofline"]["traffic"] is None                 # DRAM counters were taken on the bf16 build
    assert "fp16" in line["roofline"]["peak_source"]
    assert line["gpu_launches"] == (5 + 1) * 10                 # + the per-image loss kernel
    assert "mean over images of 1024" in line["config"]["balance_loss"]
    assert line["e2e"]["h2d_bytes_per_step"] == w.T * w.D * 2


def test_bench_refuses_inconsistent_loss_options():
    with pytest.raises(SystemExit):
        bench.main(["--global-aux", "on", "--seq-len", "1024"])
    with pytest.raises(SystemExit):
        bench.main(["--seq-len", "1000"])


def test_reference_arm_line_on_the_host(monkeypatch):
    # the reference arm is the oracle on the host cores: it runs here as it does on the GPU machine
    monkeypatch.setattr(bench, "calibrated_tokens", lambda w, inp, s: 64)
    w = I.WORKLOADS["s2_8e2a_f32"]
    args = argparse.Namespace(steps=1, warmup=3)
    line = json.loads(json.dumps(bench.run_reference(args, w, 0, 1)))
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["config"]["workload"] == w.name
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and "64" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_gpus_mismatch_with_launcher_is_refused(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "2", "--steps", "1", "--warmup", "3"])


def test_gpus_without_launcher_relaunches_under_torchrun(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    seen = {}

    def fake_call(cmd):
        seen["cmd"] = cmd
        return 0
    monkeypatch.setattr(bench.subprocess, "call", fake_call)
    with pytest.raises(SystemExit) as ei:
        bench.main(["--gpus", "4", "--steps", "7", "--warmup", "3"])
    assert ei.value.code == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-6:] == ["--gpus", "4", "--steps", "7", "--warmup", "3"]


def test_traffic_is_null_once_the_gemm_sources_change(monkeypatch):
    key = ("xl2_8e2a_512", "gemm1")
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {key: 123})
    monkeypatch.setattr(bench, "TRAFFIC_SOURCES_SHA", bench.gemm_sources_sha())
    assert bench.measured_traffic(*key) == 123
    monkeypatch.setattr(bench, "TRAFFIC_SOURCES_SHA", "0" * 16)
    assert bench.measured_traffic(*key) is None

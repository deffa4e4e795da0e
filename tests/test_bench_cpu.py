"""bench.py's host side on CPU: the reference arm's JSON line, its rank rule, the clock
summary and the shared workload description (no GPU)."""

import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=timeout)


def test_reference_arm_line():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
              "--cpu-sample-seconds", "2"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    bench = _bench_module()
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["cpu_baseline"]["nproc"] >= 1
    assert set(line["cpu_baseline"]["stage_seconds"]) == {"gram", "prepare", "sweep"}
    assert sum(line["cpu_baseline"]["stage_seconds"].values()) == pytest.approx(
        line["ms_per_step"] / 1e3, rel=0.05, abs=2e-3)
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    from post_weight_quantization_solve_b200 import synth
    wl = synth.WORKLOADS["tiny"]
    assert line["config"]["workload"] == bench.workload_desc(wl, synth.num_chunks(wl))


def test_reference_arm_other_ranks_print_nothing():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
             env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_workload_description_names_the_headline_shape():
    bench = _bench_module()
    from post_weight_quantization_solve_b200 import synth
    wl = synth.WORKLOADS["mlp_up_w3"]
    d = bench.workload_desc(wl, synth.num_chunks(wl))
    assert d.startswith("mlp_up_w3: K=4096 N=14336 tokens=2097152 (chunks 32x65536) W3")
    cae = synth.WORKLOADS["gptaq_cae"]
    assert bench.workload_desc(cae, synth.num_chunks(cae)).endswith("gptaq cae")


@pytest.mark.parametrize("reasons,expect", [
    (["Not Active", "Not Active", "Not Active", "Active"], ["sw_power_cap"]),
    (["Active", "Not Active", "Not Active", "Not Active"], ["hw_slowdown"]),
    (["Not Active"] * 4, []),
])
def test_clock_summary(reasons, expect):
    bench = _bench_module()
    cs = bench.ClockSampler(0)
    row = ", ".join(["0", "{sm}", "1965", "700.5", "0x0"] + reasons)
    cs.lines = [row.format(sm=v) for v in (1800, 1500, 1650)] + ["garbage", "0, N/A, 1965"]
    out = cs.summary()
    assert out["sm_mhz"] == 1650 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == expect
    assert out["samples"] == 3

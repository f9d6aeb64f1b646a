"""bench.py keeps its one-line JSON contract: a tiny run of the default workload prints exactly one line
with the metric, the throughput, the roofline of the dominant kernel, the oracle's CPU baseline, the
end-to-end figure, the clocks and the launch count; the reference arm prints its own line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=600):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                       timeout=timeout)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


@pytest.mark.gpu
def test_default_workload_line():
    d = _run("--scale", "0.01", "--steps", "3", "--warmup", "3", "--cpu-seconds", "0.3", "--e2e-steps", "2")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "clocks",
                "gpu_launches"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3 and d["value"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and isinstance(d["config"]["workload"], str)
    r = d["roofline"]
    assert r["bound"] in ("hbm", "tensor", "alu") and r["unit"] in ("GB/s", "TFLOP/s")
    assert r["achieved"] > 0 and r["peak"] > 0 and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    assert d["gpu_launches"] > 0
    assert d["dtype"] == "f32"


@pytest.mark.gpu
def test_default_line_carries_every_configuration():
    """The default workload's line also reports C1, C2, C3 and C5 (each from its own run of the script) with
    their roofline and CPU baseline, and the streaming window sweep ({0}, [-2,6], [-8,8])."""
    d = _run("--scale", "0.01", "--steps", "3", "--warmup", "3", "--cpu-seconds", "0.3", "--no-e2e",
             "--with-configs", "--config-steps", "3", timeout=900)
    assert set(d["configs"]) == {"act_f32", "act_bf16", "kv_bf16", "bev_f16"}
    for name, e in d["configs"].items():
        assert "error" not in e, name
        assert e["value"] > 0 and e["unit"] == "GB/s" and e["roofline"]["frac"] > 0
        assert e["cpu_baseline"]["kind"] == "oracle" and e["workload"].startswith(name)
    assert e["dtype"] == "f16" and d["configs"]["act_bf16"]["dtype"] == "bf16"
    sw = d["window_sweep_ms"]
    assert set(sw["search"]) == {"[0,0]", "[-2,6]", "[-8,8]"} and sw["two_pass_over_max_scaling"]["[0,0]"] == 1.0


@pytest.mark.gpu
@pytest.mark.parametrize("workload,dtype", [("act_bf16", "bf16"), ("bev_f16", "f16")])
def test_line_dtype_follows_the_workload(workload, dtype):
    """The line's dtype is the element type of the workload it measured."""
    d = _run("--workload", workload, "--scale", "0.05", "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
             "--no-e2e")
    assert d["dtype"] == dtype and d["config"]["workload"].startswith(workload)


def test_reference_arm_line():
    """The reference arm is the oracle on the host: no GPU needed."""
    d = _run("--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "act_f32", timeout=300)
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["dtype"] == "f32"


def test_workload_dtypes():
    """Both arms label a line with its workload's element type."""
    sys.path.insert(0, ROOT)
    import bench
    assert [bench.workload_dtype(w) for w in ("stream_f32", "act_f32", "act_bf16", "kv_bf16", "bev_f16")] == \
        ["f32", "f32", "bf16", "bf16", "f16"]


@pytest.mark.parametrize("workload,extra", [("kv_decode", []), ("kv_decode_layers", ["--kv-layers", "2"])])
def test_decode_reference_arm_lines(workload, extra):
    """The decode workloads' reference arms (the oracle's appends on the host) keep the same contract."""
    d = _run("--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", workload, *extra, timeout=300)
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"].startswith(workload)


@pytest.mark.gpu
def test_attention_workload_line():
    """The FP4-attention line: the fused call and the chain timed, the faster one sets `value`, and the
    end-to-end figure copies q, k and v in and O back every step."""
    d = _run("--workload", "attn_nvfp4", "--scale", "0.125", "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
             "--e2e-steps", "3")
    for key in ("metric", "value", "unit", "ms_per_step", "dtype", "config", "roofline", "e2e", "clocks",
                "gpu_launches", "fused"):
        assert key in d, key
    assert d["unit"] == "TFLOP/s" and d["value"] > 0 and d["gpu_launches"] > 0
    assert d["fused"]["status"] == 0 and d["fused"]["max_abs_diff_vs_chain"] < 1e-5
    H, Tq, Tk, D = (d["config"][k] for k in ("H", "Tq", "Tk", "D"))
    assert d["e2e"]["h2d_bytes_per_step"] == 2 * H * D * (Tq + 2 * Tk) and d["e2e"]["value"] > 0
    assert d["e2e"]["d2h_bytes_per_step"] == 4 * H * Tq * D

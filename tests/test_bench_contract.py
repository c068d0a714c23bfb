"""The bench.py JSON line on one GPU: every field of the contract, with its type
and the relations between fields that hold by construction."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_bench_line_carries_the_contract_fields():
    cmd = [sys.executable, "bench.py", "--workload", "varlen_b32_hq32_hkv8_d128_p64_l512to4096",
           "--steps", "20", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["unit"] == "tokens/s"
    assert d["scaling"] in ("weak", "strong") and d["data"] == "synthetic"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    # tokens/s is the batch's q rows per step over the step time
    cfg = d["config"]
    assert cfg["workload"] == "varlen_b32_hq32_hkv8_d128_p64_l512to4096"
    assert d["value"] == pytest.approx(cfg["batch"] * cfg["q_len"] / (d["ms_per_step"] / 1e3), rel=1e-6)
    rf = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in rf, k
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s"
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"], rel=1e-9)
    assert 0.05 < rf["frac"] < 1.5
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == "tokens/s"
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    # our kernels only: the persistent kernel and its prologue each step
    assert d["gpu_launches"] >= d["steps"]
    ck = d["clocks"]
    assert ck["sm_max_mhz"] > 0 and isinstance(ck["reasons"], list)
    # every workload, timed in the same run, each with its L2 policy
    wls = d["workloads"]
    assert set(wls) == {"tiny_b2_gqa4_d64_p16", "varlen_b32_hq32_hkv8_d128_p64_l512to4096",
                        "b128_hq32_hkv8_d128_p16_l8192_bf16",
                        "longctx_b4_hq16_hkv4_d256_p128_l32768_peaked",
                        "fp8_verify_b64_q4_hq64_hkv8_d128_p128_w4096",
                        "nvfp4_b128_hq32_hkv8_d128_p16_l8192"}
    assert wls["nvfp4_b128_hq32_hkv8_d128_p16_l8192"]["extra"]
    assert wls["nvfp4_b128_hq32_hkv8_d128_p16_l8192"]["kv_dtype"] == "nvfp4"
    for name, e in wls.items():
        for k in ("ms_per_step", "tokens_per_s", "gb_s", "frac_of_copy", "frac_of_8tbs_spec",
                  "kernel", "splits", "l2", "clocks", "avg_launch_ms", "timing", "launched",
                  "algorithmic_bytes_per_step", "cpu_baseline"):
            assert k in e, (name, k)
        assert e["gb_s"] == pytest.approx(
            e["algorithmic_bytes_per_step"] / (e["avg_launch_ms"] / 1e3) / 1e9, rel=1e-9)
        assert e["frac_of_copy"] == pytest.approx(e["gb_s"] / rf["peak"], rel=1e-9)
        assert e["tokens_per_s"] == pytest.approx(
            e["batch"] * e["q_len"] / (e["ms_per_step"] / 1e3), rel=1e-6)
        assert e["cpu_baseline"]["kind"] == "oracle" and e["cpu_baseline"]["value"] > 0
        if name.startswith("tiny"):
            assert e["l2"].startswith("flushed") and e["timing"] == "host-launched"
        else:
            assert e["timing"].startswith("one CUDA graph")
            if name.startswith("b128") or name.startswith("nvfp4"):
                assert e["l2"].startswith("no flush")
            else:
                assert e["l2"].startswith("rotating")
        assert e["launched"]["ms_per_step"] > 0
    top = wls[cfg["workload"]]
    assert top["top_level"] and top["ms_per_step"] == d["ms_per_step"]

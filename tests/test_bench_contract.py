"""The bench's JSON contract, checked on the CPU through its reference arm (the oracle on a bounded
sample) and its FLOP accounting."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_attention_flops_full_and_causal():
    from mxfp4_bit_attention_b200 import inputs
    b = _bench_module()
    w = inputs.WORKLOADS["720p"]
    assert b.attention_flops(w, False) == 4.0 * 40 * 75600 * 75600 * 128
    assert b.attention_flops(w, True) == 4.0 * 40 * (75600 * 75601 / 2) * 128
    assert b.whole_job_tflops(2, 1e12, 1000.0) == pytest.approx(2.0)


@pytest.mark.parametrize("extra", [[], ["--causal"]])
def test_reference_arm_json_line(extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "1", "--warmup", "1", "--cpu-sample-seconds", "0.5"] + extra
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "TFLOPS" and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny" and line["config"]["causal"] == bool(extra)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] > 0
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_recorded_traffic_is_keyed_to_the_kernel_source(tmp_path, monkeypatch):
    """The committed DRAM-traffic record is used only while the kernel sources hash to the value it
    was captured on; any other source gives no traffic figure."""
    b = _bench_module()
    rec = {"mxattn_fwd_wide_kernel": {"kernel_source_hash": "0123456789abcdef",
                                      "per_workload": {"720p": 1.25e9, "480p": 5.5e8}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "attn_fwd_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    monkeypatch.setattr(b, "kernel_source_hash", lambda key_tile=128: "0123456789abcdef")
    assert b.recorded_traffic("720p", 128) == 1.25e9
    assert b.recorded_traffic("joint", 128) is None
    assert b.recorded_traffic("720p", 64) is None  # no record for the 64-key kernel
    monkeypatch.setattr(b, "kernel_source_hash", lambda key_tile=128: "ffffffffffffffff")
    assert b.recorded_traffic("720p", 128) is None


def test_gpus_n_without_torchrun_starts_n_ranks():
    """`bench.py --gpus 2` started directly (no RANK in the environment) starts two ranks under
    torch.distributed.run on 127.0.0.1 itself; with the reference arm (no GPU needed) rank 0 prints
    the one JSON line, reporting the world size it ran under, and the other rank exits 0."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--workload",
           "tiny", "--steps", "1", "--warmup", "0", "--cpu-sample-seconds", "0.5"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2

"""Host logic of bench.py that needs no GPU: the clock-sample summary (throttle reasons
the timing rules reject), the device-code hash that decides whether the recorded ncu
traffic still applies, and the traffic lookup."""
import importlib.util
import json
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _summary(bench, tmp_path, lines):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    return s.summary()


def test_clock_summary_median_max_and_reasons(bench, tmp_path):
    idle = "Not Active"
    rows = [f"0, {mhz}, 1965, 600.0 W, 0x0, {idle}, {idle}, {idle}, {cap}"
            for mhz, cap in ((1965, idle), (1950, "Active"), (1965, idle), (1800, idle), (1965, idle))]
    out = _summary(bench, tmp_path, rows + ["garbage line", "0, n/a, 1965, x, y, a, b, c, d"])
    assert out["sm_mhz"] == 1965 and out["sm_max_mhz"] == 1965 and out["samples"] == 5
    assert out["reasons"] == ["sw_power_cap"]
    rows[2] = f"0, 1500, 1965, 700 W, 0x0, Active, {idle}, Active, {idle}"
    out = _summary(bench, tmp_path, rows)
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_summary_without_samples_is_none(bench, tmp_path):
    assert _summary(bench, tmp_path, []) is None


def _fake_root(tmp_path):
    root = tmp_path / "root"
    (root / "ternary_rank_weight_b200" / "csrc").mkdir(parents=True)
    (root / "profiles").mkdir()
    for name in ("externd.cu", "externd_kernels.cuh"):
        shutil.copy(os.path.join(ROOT, "ternary_rank_weight_b200", "csrc", name),
                    root / "ternary_rank_weight_b200" / "csrc" / name)
    return root


def test_device_code_hash_ignores_comments_and_host_code(bench, tmp_path, monkeypatch):
    root = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    cu = root / "ternary_rank_weight_b200" / "csrc" / "externd.cu"
    src = cu.read_text()
    base = bench._kernel_source_hash()
    assert base == bench._kernel_source_hash()
    cu.write_text("// a new comment line\n\n" + src.replace("struct ProbIn", "// host note\nstruct ProbIn", 1))
    assert bench._kernel_source_hash() == base
    host = src.index("struct ProbIn")
    cu.write_text(src[:host] + src[host:] + "\nint host_only_addition() { return 1; }\n")
    assert bench._kernel_source_hash() == base
    dev = src.index("__global__")
    cu.write_text(src[:dev] + "__device__ int device_only_addition() { return 2; }\n" + src[dev:])
    assert bench._kernel_source_hash() != base


def test_traffic_record_applies_only_to_its_source(bench, tmp_path, monkeypatch):
    root = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    rec = {"source_sha256": bench._kernel_source_hash(), "dram_bytes_per_launch_scaled": {"wl": 123.0}}
    (root / "profiles" / "als_kernel_traffic.json").write_text(json.dumps(rec))
    assert bench._ncu_traffic("wl") == 123.0
    assert bench._ncu_traffic("other") is None
    rec["source_sha256"] = "0" * 64
    (root / "profiles" / "als_kernel_traffic.json").write_text(json.dumps(rec))
    assert bench._ncu_traffic("wl") is None


def test_reference_arm_prints_once_on_rank_zero(tmp_path):
    """`bench.py --impl reference` under several ranks: rank 0 times the oracle on a bounded
    sample and prints one JSON line with the contract's keys; every other rank exits 0 silently."""
    import subprocess
    import sys
    base = dict(os.environ, WORLD_SIZE="2", MASTER_ADDR="127.0.0.1", MASTER_PORT="29555")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "0",
           "--workload", "iid_256x256_mu2_tau0.7", "--ref-budget", "1"]
    r1 = subprocess.run(cmd, env=dict(base, RANK="1", LOCAL_RANK="1"), capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, env=dict(base, RANK="0", LOCAL_RANK="0"), capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0
    lines = [l for l in r0.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0

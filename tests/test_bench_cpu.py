"""Host-side pieces of bench.py that need no GPU: the clock record's parsing and
the reference arm (the oracle timed on the host cores) with its JSON line."""
import datetime
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _row(t, sm, reasons=(), ts=True):
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    flags = ["Active" if n in reasons else "Not Active" for n in names]
    cols = ["0", str(sm), "1965", "950.12", "0x0000000000000000", *flags]
    if ts:
        cols.append(datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3])
    return ", ".join(cols)


def _sampler(tmp_path, lines, t0=None, t1=None):
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(lines) + "\n")
    s = bench.ClockSampler(0)
    s.path = str(path)
    s.t0, s.t1 = t0, t1
    return s


def test_clock_summary_keeps_only_the_timed_region(tmp_path):
    t0 = 1_800_000_000.0
    t1 = t0 + 0.1
    lines = [_row(t0 - 1.0, 1200, ("hw_slowdown",)),          # before: idle and throttled
             _row(t0 + 0.00, 1965),
             _row(t0 + 0.04, 1950, ("sw_power_cap",)),
             _row(t0 + 0.08, 1965),
             _row(t1 + 1.0, 900, ("hw_thermal_slowdown",))]     # after
    got = _sampler(tmp_path, lines, t0, t1).summary()
    assert got["in_timed_region"] is True
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1965.0
    assert got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]


def test_clock_summary_falls_back_to_all_samples(tmp_path):
    # rows without a timestamp column, or no sample inside a very short window
    lines = [_row(0, 1965, ts=False), _row(0, 1800, ("hw_slowdown",), ts=False)]
    got = _sampler(tmp_path, lines, 1.0, 2.0).summary()
    assert got["in_timed_region"] is False
    assert got["samples"] == 2
    assert got["reasons"] == ["hw_slowdown"]
    t0 = 1_800_000_000.0
    got = _sampler(tmp_path, [_row(t0 - 5, 1965), _row(t0 + 5, 1965)], t0, t0 + 0.01).summary()
    assert got["in_timed_region"] is False and got["samples"] == 2


def test_clock_summary_missing_file(tmp_path):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "absent.csv")
    assert s.summary() is None


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one JSON
    line with the same metric and workload as the GPU arm."""
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] >= 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["vs_baseline"] is None
    assert line["config"]["workload"] == bench.WORKLOAD
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_under_two_ranks(rank):
    """Launched as two ranks, the reference arm runs and prints on rank 0 only (n_gpus
    the world size); the other rank exits 0 without work or output."""
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank))
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3", "--gpus", "2"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    if rank == 0:
        line = json.loads(res.stdout.strip().splitlines()[-1])
        assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    else:
        assert res.stdout.strip() == ""


FAKE_SMI = r'''#!{python}
import datetime, sys, time
args = sys.argv[1:]
query = [a for a in args if a.startswith("--query-gpu=")][0].split("=", 1)[1]
ms = int(args[args.index("-lms") + 1])
mode = "{mode}"
if mode == "refuse_timestamp" and "timestamp" in query:
    sys.exit(2)
if mode == "slow":
    time.sleep(4)
while True:
    cols = ["0", "1965", "1965", "900.00", "0x0000000000000000"] + ["Not Active"] * 4
    if "timestamp" in query:
        cols.append(datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3])
    print(", ".join(cols), flush=True)
    time.sleep(ms / 1000.0)
'''


def _fake_smi(tmp_path, monkeypatch, mode):
    d = tmp_path / f"bin_{mode}"
    d.mkdir()
    exe = d / "nvidia-smi"
    exe.write_text(FAKE_SMI.format(python=sys.executable, mode=mode))
    exe.chmod(0o755)
    monkeypatch.setenv("PATH", f"{d}{os.pathsep}{os.environ.get('PATH', '')}")
    monkeypatch.setenv("QLORA_CLOCKS_CSV", str(tmp_path / f"clocks_{mode}.csv"))


@pytest.mark.parametrize("mode", ["ok", "refuse_timestamp", "slow"])
def test_clock_sampler_process_paths(tmp_path, monkeypatch, mode):
    """The sampler against a stand-in nvidia-smi: timestamped samples inside the
    block; a refused timestamped query falls back to the plain fields; a slow first
    sample is waited for (up to 3 s) and not taken for a refusal."""
    import time
    _fake_smi(tmp_path, monkeypatch, mode)
    c = bench.ClockSampler(0)
    with c:
        time.sleep(0.3)
    got = c.summary()
    assert c.proc is None and c.fh is None
    if mode == "ok":
        assert c.interval == 20 and got["in_timed_region"] is True and got["samples"] >= 3
        assert got["sm_mhz"] == 1965.0 and got["reasons"] == []
    elif mode == "refuse_timestamp":
        assert c.interval == 200 and got["in_timed_region"] is False and got["samples"] >= 1
    else:
        assert c.interval == 20 and got is None


def test_smi_device_id_follows_cuda_visible_devices():
    assert bench.smi_device_id(0, None) == "0"
    assert bench.smi_device_id(1, "3,5") == "5"
    assert bench.smi_device_id(0, "GPU-0a1b2c3d-0000-1111-2222-333344445555") == \
        "GPU-0a1b2c3d-0000-1111-2222-333344445555"
    assert bench.smi_device_id(2, "3,5") == "2"          # out of range: the index itself
    assert bench.smi_device_id(0, "all") == "0"          # not an index or a UUID
    assert bench.smi_device_id(0, "") == "0"


def _fake_tree(tmp_path, kernel_text):
    csrc = tmp_path / "bit_nf4_quantized_19_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gemm_kernel.cuh").write_text(kernel_text)
    (csrc / "common.cuh").write_text("// shared helpers\n")
    (csrc / "qlora_nf4.cu").write_text("qlora_status launch_gemm(int x) {\n  return x;\n}\n")
    (tmp_path / "profiles").mkdir()
    return tmp_path


def test_traffic_is_reported_only_for_the_sources_it_was_captured_on(tmp_path, monkeypatch):
    root = _fake_tree(tmp_path, "// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    h1 = bench.source_hash("qlora_gemm_kernel")
    (root / "profiles" / "traffic.json").write_text(
        json.dumps({"qlora_gemm_kernel": {"source_hash": h1, "bytes_per_launch": 1.5e9}}))
    assert bench.traffic_for("qlora_gemm_kernel") == 1.5e9
    # any change to the kernel's header (or its launcher) makes the stored figure stale
    (root / "bit_nf4_quantized_19_b200" / "csrc" / "gemm_kernel.cuh").write_text("// kernel v2\n")
    assert bench.source_hash("qlora_gemm_kernel") != h1
    assert bench.traffic_for("qlora_gemm_kernel") is None
    (root / "bit_nf4_quantized_19_b200" / "csrc" / "gemm_kernel.cuh").write_text("// kernel v1\n")
    (root / "bit_nf4_quantized_19_b200" / "csrc" / "qlora_nf4.cu").write_text(
        "qlora_status launch_gemm(int x) {\n  return x + 1;\n}\n")
    assert bench.traffic_for("qlora_gemm_kernel") is None


def test_traffic_missing_file_or_kernel_reads_null(tmp_path, monkeypatch):
    root = _fake_tree(tmp_path, "// kernel\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.traffic_for("qlora_gemm_kernel") is None
    (root / "profiles" / "traffic.json").write_text("{}")
    assert bench.traffic_for("qlora_gemm_kernel") is None

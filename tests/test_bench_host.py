"""Host-side logic of bench.py, on CPU: the clock summary, the multi-rank
helpers over a world-size-2 gloo group, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_clock_summary_counts_only_the_timed_window():
    cs = bench.ClockSampler(0)
    cs.source = "nvml"
    cs.max_mhz = 1965.0
    cs.t_start, cs.t_stop = 10.0, 11.0
    cs.samples = [(9.5, 500.0, 0x8),            # before the window: ignored (hw_slowdown)
                  (10.1, 1900.0, 0x0), (10.5, 1965.0, 0x4), (10.9, 1950.0, 0x0),
                  (11.5, 300.0, 0x40)]          # after the window: ignored
    s = cs.summary()
    assert s["sm_mhz"] == 1950.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 3


def test_clock_summary_names_every_slowdown_reason():
    cs = bench.ClockSampler(0)
    cs.source = "nvml"
    cs.t_start, cs.t_stop = 0.0, 1.0
    cs.samples = [(0.5, 1000.0, 0x8 | 0x20 | 0x40 | 0x80 | 0x1)]  # 0x1 (idle) is not reported
    assert cs.summary()["reasons"] == ["hw_power_brake_slowdown", "hw_slowdown",
                                       "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples_says_so():
    cs = bench.ClockSampler(0)
    cs.source = "nvml"
    cs.t_start, cs.t_stop = 0.0, 1.0
    assert cs.summary()["reasons"] == ["not recorded"]
    smi = bench.ClockSampler(0)
    smi.smi_lines = ["0, 1965, 1965, 700.5, 0x4, Not Active, Not Active, Not Active, Active"]
    s = smi.summary()
    assert s["sm_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    bench.barrier(world)
    m = bench.max_over_ranks(1.5 + rank, world)  # each rank's own time; the max is reported
    bench.barrier(world)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
        f.write(repr(m))


def test_max_over_ranks_on_two_gloo_ranks(tmp_path):
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    assert [float(open(tmp_path / f"r{r}").read()) for r in range(2)] == [2.5, 2.5]


def test_max_over_ranks_is_identity_for_one_rank():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_on_a_nonzero_rank_prints_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(type("A", (), {"cpu_tokens": 64, "warmup": 3, "steps": 1})())
    assert capsys.readouterr().out == ""


@pytest.mark.timeout(300)
def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--cpu-tokens", "128"],
                       capture_output=True, text=True, timeout=280, cwd=ROOT,
                       env={**os.environ, "RANK": "0"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"

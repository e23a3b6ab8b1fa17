"""CPU checks of the bench's host-side accounting and clock sampling (no GPU)."""

import os
import stat

import numpy as np

import bench


def _allowed_entries(n, k):
    """Count the allowed (row, key) pairs of one segment straight from the mask rule:
    key j is visible to row i when j == i or j < min(i, n)."""
    T = n + k
    return sum(1 for i in range(T) for j in range(T) if j == i or j < min(i, n))


def test_prefill_flops_counts_the_allowed_entries():
    past, cand, H, D = [5, 0, 7, 3], [3, 4, 0, 9], 2, 32
    entries = sum(_allowed_entries(n, k) for n, k in zip(past, cand))
    assert bench.prefill_flops(past, cand, H, D) == 4.0 * D * H * entries


def test_decode_flops_and_bytes():
    past, cand, H, D = [10, 0, 3], [2, 5, 1], 4, 64
    # every candidate scores its request's n pool keys plus itself
    assert bench.decode_flops(past, cand, H, D) == 4.0 * D * H * (2 * 11 + 5 * 1 + 1 * 4)
    # pool K/V rows once, candidate q/k/v once, output once (fp32 here)
    assert bench.decode_bytes(past, cand, H, D, 4) == 2 * 13 * H * D * 2 + 3 * 8 * H * D * 2 + 8 * H * D * 4


def test_prefill_traffic_scales_with_tokens_or_is_null():
    a = bench.prefill_traffic(1000, 8, 128)
    b = bench.prefill_traffic(3000, 8, 128)
    if a is None:
        assert b is None          # the kernel source changed since the capture
    else:
        assert abs(b - 3 * a) < 1e-6 * b
    assert bench.prefill_traffic(1000, 2, 32) is None   # no capture for this shape


def test_clock_sampler_reads_fake_nvidia_smi(tmp_path, monkeypatch):
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/bash\n"
                    "while true; do echo '0, 1900, 1965, 700.5, 0x4, Not Active, Not Active, Not Active, Active'; "
                    "sleep 0.02; done\n")
    fake.chmod(fake.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    c = bench.ClockSampler(0)
    c.start()
    r = c.stop()
    assert r is not None and r["samples"] >= 1
    assert r["sm_mhz"] == 1900.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    c = bench.ClockSampler(0)
    c.start()
    assert c.stop() is None


def test_reference_arm_prints_one_oracle_line():
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, bench.__file__, "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("tiny_prefill_B2_H2_D32")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_gpus_flag_relaunches_one_rank_per_gpu():
    """--gpus N without a launcher starts N ranks through torch's launcher on 127.0.0.1."""
    cmd = bench.relaunch_command(["--gpus", "4", "--steps", "5"], 4, port=29555)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert cmd[cmd.index("--nproc-per-node") + 1] == "4"
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[cmd.index("--master-port") + 1] == "29555"
    assert cmd[cmd.index("--master-port") + 2].endswith("bench.py")
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"]


def test_gpus_flag_must_match_the_launcher(monkeypatch):
    """Under a launcher, --gpus that disagrees with WORLD_SIZE is an error, never ignored."""
    import pytest
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit) as e:
        bench.main(["--gpus", "4", "--workload", "tiny"])
    assert e.value.code == 2


def test_reference_arm_with_several_gpus_runs_once():
    """The oracle arm under --gpus 2 without a launcher runs on the host once and prints one line."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, bench.__file__, "--impl", "reference", "--gpus", "2", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1 and json.loads(lines[0])["impl"] == "reference"

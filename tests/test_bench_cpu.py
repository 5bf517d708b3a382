"""bench.py on the CPU: the argument checks and the reference arm (the fp64 oracle) for every
pass, on the smallest workload (no GPU needed)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=600):
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          timeout=timeout, cwd=ROOT)
    return proc


@pytest.mark.parametrize("pass_", ["fwd", "bwd", "rope", "fp8", "bwd_rope"])
def test_reference_arm_prints_one_json_line(pass_):
    proc = run_bench("--impl", "reference", "--pass", pass_, "--workload", "cfg1", "--steps", "2", "--warmup", "3")
    assert proc.returncode == 0, proc.stderr
    lines = [l for l in proc.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("cfg1")


def test_warmup_below_three_is_refused():
    proc = run_bench("--impl", "reference", "--warmup", "2", "--steps", "1")
    assert proc.returncode != 0
    assert "--warmup" in proc.stderr


def test_reference_arm_under_two_ranks_prints_on_rank_zero_only():
    """Launched by torchrun with N > 1, the reference arm runs on rank 0 alone (the oracle on the
    host cores); the other ranks exit 0 without work or output."""
    outs = {}
    for rank in (0, 1):
        env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank))
        proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                               "--workload", "cfg1", "--steps", "1", "--warmup", "3"],
                              capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
        assert proc.returncode == 0, proc.stderr
        outs[rank] = [l for l in proc.stdout.splitlines() if l.strip()]
    assert outs[1] == []
    assert len(outs[0]) == 1
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2


def test_clock_sampler_parses_nvidia_smi_rows(tmp_path, monkeypatch):
    """The clock record of the timed region, from a stand-in nvidia-smi on PATH that prints
    four samples (one idle) in the query's CSV form and then waits to be stopped."""
    sys.path.insert(0, ROOT)
    import bench

    fake = tmp_path / "nvidia-smi"
    rows = ["0, 1965, 1965, 120.5, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
            "0, 1900, 1965, 560.0, 100, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1880, 1965, 571.5, 100, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1920, 1965, 540.0, 99, 0x0, Not Active, Not Active, Not Active, Not Active"]
    fake.write_text("#!/bin/sh\n" + "".join(f"echo '{r}'\n" for r in rows) + "exec sleep 30\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    sampler = bench.ClockSampler(0)
    path = sampler.path
    rec = sampler.stop()
    assert rec["samples"] == 3                      # the idle row is left out
    assert rec["sm_mhz"] == 1900.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["power_w_max"] == 571.5
    assert not os.path.exists(path)


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("PATH", str(tmp_path))
    sampler = bench.ClockSampler(0)
    path = sampler.path
    rec = sampler.stop()
    assert rec["samples"] == 0 and rec["reasons"] == ["nvidia-smi unavailable"]
    assert not os.path.exists(path)


def test_reference_arm_loads_none_of_the_libraries_own_code():
    """The reference arm is the fp64 oracle alone: it must not map the CUDA library (nor import
    the package that loads it), and it prints the same `config` object as the CUDA arm."""
    code = ("import sys; sys.argv=['bench.py']; import bench; "
            "bench.main(['--impl','reference','--workload','cfg1','--steps','1','--warmup','3']); "
            "maps=open('/proc/self/maps').read(); "
            "print('MAPPED' if 'libattn_fwd' in maps else 'CLEAN'); "
            "print('PKG' if 'tiled_attention_forward_03_b200' in sys.modules else 'NOPKG')")
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr
    out = proc.stdout.splitlines()
    assert out[-2:] == ["CLEAN", "NOPKG"]
    line = json.loads(out[0])
    sys.path.insert(0, ROOT)
    import bench
    from attn_inputs import get_workload

    assert line["config"] == bench.bench_config(get_workload("cfg1"), "fwd", 1)

"""bench.py under torchrun with 2 ranks on the CPU.

The reference arm (the fp64 oracle) needs no GPU, so the multi-rank launch
path of the benchmark contract can run here: rank 0 alone runs and prints
one JSON line, the other rank exits 0 without work.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_reference_arm_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_port()), "bench.py", "--gpus", "2",
           "--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "8"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["metric"].startswith("TP-MLP fwd+bwd")


def test_clock_sampler_keeps_the_marked_samples(tmp_path, monkeypatch):
    """The clock record covers the timed steps only: samples written before
    mark() (start-up, warm-up) are left out, and the throttle reasons are
    read from the kept ones.  A stand-in nvidia-smi prints 900 MHz until a
    flag file appears and 1500 MHz with sw_power_cap after it."""
    import time
    flag = tmp_path / "timed"
    fake = tmp_path / "nvidia-smi"
    fake.write_text(
        "#!/bin/sh\n"
        "i=0\n"
        "while [ $i -lt 300 ]; do\n"
        f"  if [ -e {flag} ]; then echo '0, 1500, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active';\n"
        "  else echo '0, 900, 1965, 300.0, 0x0, Not Active, Not Active, Not Active, Not Active'; fi\n"
        "  i=$((i+1)); sleep 0.01\n"
        "done\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}:{os.environ['PATH']}")
    sys.path.insert(0, ROOT)
    import bench
    with bench.ClockSampler(0) as clk:
        assert clk._lines() >= 1            # sampling is live on entry
        time.sleep(0.4)                     # "warm-up": 900 MHz samples
        flag.touch()
        time.sleep(0.05)
        clk.mark()
        time.sleep(0.15)                    # "timed steps": 1500 MHz samples
    s = clk.summary()
    assert s["sm_mhz"] == 1500.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] >= 3

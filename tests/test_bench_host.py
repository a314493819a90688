"""bench.py's host side on CPU: the reference arm's JSON line (the CPU oracle
timed on a small workload), its silence on ranks other than 0, the N-rank
launch that `--gpus N` starts by itself, and the parsing of the nvidia-smi
clock samples that accompany every timed run."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          timeout=600, env=e, cwd=ROOT)


def test_reference_arm_line_on_tiny_workload():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "f64" and d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_silently():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "1"],
             env={"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_clock_rows_summary():
    rows = [
        "1965, 1965, 450.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "1410, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "1395, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "[N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]\n",
        "garbage line\n",
    ]
    s = bench.summarize_clock_rows(rows)
    assert s["sm_mhz"] == 1410.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 4
    hot = bench.summarize_clock_rows(
        ["1200, 1965, 700, 0x8, Active, Not Active, Active, Not Active\n"])
    assert hot["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_clock_rows([]) is None


def test_torchrun_command_for_n_ranks():
    argv = bench.torchrun_argv(["--gpus", "4", "--steps", "3"], 4, 29555, limit_s=600)
    assert argv[:4] == ["timeout", "-k", "60", "600"]
    i = argv.index("torch.distributed.run")
    assert argv[i - 1] == "-m" and "--nnodes=1" in argv and "--nproc-per-node=4" in argv
    assert "--master-addr=127.0.0.1" in argv and "--master-port=29555" in argv
    assert argv[-4:] == ["--gpus", "4", "--steps", "3"] and argv[-5].endswith("bench.py")


def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` without a launcher starts two ranks (here the CPU
    reference arm, which rank 0 alone runs): one JSON line, n_gpus = 2."""
    e = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "1"], capture_output=True, text=True,
                       timeout=600, env=e, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2

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


def test_layer_roofline_counts_the_algorithmic_work():
    """FLOPs of the kept and shared rows through both MLP layers; minimum bytes
    of x, W_g, the touched experts' weights, y and routing metadata; the slower
    of the two against each peak set."""
    from sparse_mixture_experts_gate_b200.workloads import WORKLOADS
    w = WORKLOADS["e64"]
    kept, touched, ms = 40000, 65, 0.8
    peaks = {"bf16": 1000.0, "bf16_sustained": 800.0, "hbm_gbs": 5000.0, "source": "test"}
    r = bench.layer_roofline(w, kept, touched, ms, peaks)
    rows = kept + w.S * w.T
    flops = 2.0 * rows * w.F * (w.d + w.O)
    bytes_min = (w.T * w.d * 2 + w.E * w.d * 4 + touched * (w.F * w.d + w.O * w.F) * 2 + w.T * w.O * 2
                 + w.T * w.k * 12)
    assert r["flops"] == flops and r["bytes_min"] == bytes_min
    t = ms / 1e3
    t_flop, t_bytes = flops / 1e15, bytes_min / 5e12
    assert r["bound"] == ("tensor" if t_flop >= t_bytes else "hbm")
    assert abs(r["layer_roofline_frac"] - max(t_flop, t_bytes) / t) < 1e-12
    assert abs(r["layer_roofline_frac_sustained"] - max(flops / 8e14, t_bytes) / t) < 1e-12
    t_spec = max(flops / (bench.SPEC_BF16_TFLOPS * 1e12), bytes_min / (bench.SPEC_HBM_GBS * 1e9))
    assert abs(r["layer_roofline_frac_spec_sheet"] - t_spec / t) < 1e-12
    assert abs(r["expert_gemm_tflops"] - flops / t / 1e12) < 1e-9


def test_committed_traffic_scales_the_capture_and_checks_the_source(tmp_path, monkeypatch):
    """The DRAM traffic of a scaled capture is scaled by the rows processed, and
    is withheld when the expert-GEMM source differs from the captured one or the
    workload was resized."""
    import hashlib
    from sparse_mixture_experts_gate_b200.workloads import WORKLOADS
    src = tmp_path / "sparse_mixture_experts_gate_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "gemm_pair.cu").write_text("// kernel source\n")
    sha = hashlib.sha256(b"// kernel source\n").hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "grouped_gemm_pair_e256_traffic.txt").write_text(
        f"# a capture\nkernel_source_sha256: {sha}\ncapture_rows: 1000\ndram_bytes_per_launch_pair: 2.5e9\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    w = WORKLOADS["e256"]
    assert bench.committed_traffic(w, 4000) == 2.5e9 * 4
    assert bench.committed_traffic(w.with_(T=1024), 4000) is None  # resized workload
    (src / "gemm_pair.cu").write_text("// edited kernel source\n")
    assert bench.committed_traffic(w, 4000) is None  # source changed since the capture

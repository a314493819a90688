#!/usr/bin/env python
"""Benchmark of the sparse top-k MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload e256] [--impl ours|reference]

A step is one layer forward plus its statistics (moe_forward + moe_aux_stats
through the C ABI) over one batch of synthetic tokens already resident in HBM.
The default workload is the largest configuration, "e256" (T=32768, d=7168,
d_ff=2048, E=256, k=8, one shared expert, Swish, C_f=1.25, credit statistics).
Its inputs are larger than L2 (x 470 MB, expert weights 15 GB), so no L2 flush
is needed between steps.

With N > 1 (one process per GPU under torchrun) every rank runs its own replica
on its own batch (weak scaling, no collective on the data path); the timed
region is bracketed by barriers and the max over ranks is reported.

`--gpus N` without a launcher starts the N ranks itself (torch.distributed.run
on 127.0.0.1, bounded by `timeout`).

Rank 0 prints one JSON line: whole-job tokens/s, the layer and expert-GEMM
roofline fractions measured with CUDA events inside the timed region (against
the burst bf16 peak, the sustained one beside it), the end-to-end number with
host buffers, the CPU-oracle baseline and the SM clocks. Under "configs" the
same line carries the device measurement of the other named configurations
(tiny, default, e64, decode), each timed the same way after the headline one.
`--impl reference` times the CPU oracle (the reference arm) instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s; expert GEMM TFLOP/s and % of B200 roofline"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="e256")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="time the headline workload only")
    # Smaller variants of a workload, for profiler captures of the same kernels.
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling)")
    ap.add_argument("--experts", type=int, default=None, help="override E (profiling)")
    ap.add_argument("--dff", type=int, default=None, help="override d_ff (profiling the router at full E and d)")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm_gbs=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarize_clock_rows(lines)


def summarize_clock_rows(lines):
    """Median SM clock, max clock and the throttle reasons seen, from
    nvidia-smi CSV rows of ClockSampler.FIELDS (no header, no units)."""
    rows = [[p.strip() for p in line.split(",")] for line in lines]
    rows = [r for r in rows if len(r) >= 8]
    if not rows:
        return None
    sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
    mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": reasons, "samples": len(rows)}


def gpu_id_for(dev) -> str:
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[dev]
        return str(dev)


# ---------------------------------------------------------------- CPU oracle sample

def oracle_sample(w, x_rows, w_gate, b_gate, sel_bias, noise_rows, token_loss_rows, expert_source):
    """Times the CPU oracle over a T_s-token batch of workload `w` (its own
    capacity at T_s). `expert_source(experts)` returns host copies of the touched
    experts' w1/b1/w2/b2. Returns (seconds, tokens)."""
    import oracle
    T_s = x_rows.shape[0]
    ws = w.with_(T=T_s)
    inp = dict(x=x_rows, w_gate=w_gate, b_gate=b_gate, sel_bias=sel_bias, noise=noise_rows,
               token_loss=token_loss_rows)
    # Untimed pre-pass: which experts does this sample touch?
    h = oracle.router_logits(x_rows, w_gate, b_gate)
    key = oracle.selection_keys(h.astype("float32"), noise_rows if w.top_k_method == "noisy" else None,
                                sel_bias if w.use_selection_bias else None)
    idx = oracle.topk(key, w.k)
    inp.update(expert_source(sorted(set(idx.ravel().tolist()) | set(range(w.E, w.E + w.S)))))
    t0 = time.perf_counter()
    oracle.forward(ws, inp)
    return time.perf_counter() - t0, T_s


def cpu_sample_from_device(w, inp, T_s):
    import torch
    sl = slice(0, T_s)
    cpu = lambda t: None if t is None else t[sl].cpu() if t.dim() and t.shape[0] == w.T else t.cpu()

    def experts(es):
        return {k: {e: inp[k][e].cpu() for e in es} for k in ("w1", "b1", "w2", "b2")}

    return oracle_sample(w, inp["x"][sl].cpu(), inp["w_gate"].cpu(),
                         None if inp.get("b_gate") is None else inp["b_gate"].cpu(),
                         None if inp.get("sel_bias") is None else inp["sel_bias"].cpu(),
                         None if inp.get("noise") is None else inp["noise"][sl].cpu(),
                         None if inp.get("token_loss") is None else inp["token_loss"][sl].cpu(), experts)


def oracle_threads():
    import oracle
    return oracle.max_threads()


# ---------------------------------------------------------------- our arm

SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0


def layer_roofline(w, kept, touched, ms_step, peaks):
    """Roofline numbers of one layer step from the algorithmic work: expert-GEMM
    FLOPs (kept + shared rows) and minimum bytes (x once, W_g, the weights of
    experts with a kept row, y once, routing metadata). The layer's ideal time
    is the slower of the FLOPs at the bf16 tensor peak and the bytes at the HBM
    peak; the burst tensor peak is the headline denominator (a step timed over a
    fraction of a second), the sustained one is reported beside it."""
    rows = kept + w.S * w.T
    flops = 2.0 * rows * w.F * (w.d + w.O)
    es = 2 if w.dtype == "bf16" else 4
    bytes_min = (w.T * w.d * es + w.E * w.d * 4 + touched * (w.F * w.d + w.O * w.F) * es + w.T * w.O * es
                 + w.T * w.k * 12)
    t = ms_step / 1e3
    t_flop = flops / (peaks["bf16"] * 1e12)
    t_flop_s = flops / (peaks["bf16_sustained"] * 1e12)
    t_bytes = bytes_min / (peaks["hbm_gbs"] * 1e9)
    # The spec-sheet figures (dense bf16 2250 TFLOP/s, HBM3e 8000 GB/s), beside the measured ones.
    t_spec = max(flops / (SPEC_BF16_TFLOPS * 1e12), bytes_min / (SPEC_HBM_GBS * 1e9))
    return {"flops": flops, "bytes_min": bytes_min, "bound": "tensor" if t_flop >= t_bytes else "hbm",
            "expert_gemm_tflops": flops / t / 1e12, "hbm_gbs": bytes_min / t / 1e9,
            "layer_roofline_frac": max(t_flop, t_bytes) / t,
            "layer_roofline_frac_sustained": max(t_flop_s, t_bytes) / t,
            "layer_roofline_frac_spec_sheet": t_spec / t,
            "hbm_frac": t_bytes / t}


def measure(w, args, dev, rank, world, headline):
    """Times one workload: an instrumented eager loop (per-stage CUDA events
    recorded by the library), then the step replayed as a CUDA graph (the
    timed number), then, for the headline workload, the end-to-end pipeline
    with host buffers. Every rank runs the same collectives in the same order."""
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_gate_b200 import binding
    from sparse_mixture_experts_gate_b200.binding import MoELayer
    from sparse_mixture_experts_gate_b200.workloads import make_inputs, make_tokens

    inp = make_inputs(w, "cuda")
    if rank > 0:  # each replica routes its own batch of tokens
        inp.update(make_tokens(w, "cuda", seed=w.seed + 7919 * rank))
    layer = MoELayer(w, inp)
    # The weights stay fixed over the run: the router matrix is split into its
    # bf16 planes once (moe_prepare_router), as a serving process does after
    # loading or updating weights, instead of in every forward.
    layer.prepare_router()
    T = w.T
    x, noise, tl = inp["x"], inp.get("noise"), inp.get("token_loss")
    out = layer.alloc_outputs(T)
    layer.workspace(T)
    stream = torch.cuda.current_stream()
    fits_l2 = not inputs_exceed_l2(w)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if fits_l2 else None

    def step():
        layer.forward(x, noise=noise, out=out)
        layer.aux_stats(out, token_loss=tl)

    W = max(args.warmup, 3)
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if layer.device_status() != 0:
        raise RuntimeError(f"{w.name}: device status reports a timeout")
    kept = int(out["count_kept"].sum().item())
    touched = int((out["count_kept"] > 0).sum().item()) + w.S
    launches_per_step = layer.launch_count()

    # Per-stage times from the library's stage events (eager launches).
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(binding.MOE_TIMING_EVENTS)] for _ in range(K)]
    for row in evs:  # materialise the event handles
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        if flush is not None:
            flush.fill_(i & 0xFF)
        binding.moe_set_timing_events(layer.handle, [e.cuda_event for e in evs[i]])
        step()
    end.record(stream)
    torch.cuda.synchronize()
    binding.moe_set_timing_events(layer.handle, None)
    stage = {n: [] for n in binding.STAGES}
    for row in evs:
        for j, n in enumerate(binding.STAGES):
            stage[n].append(row[j].elapsed_time(row[j + 1]))
    eager_steps = [row[0].elapsed_time(row[-1]) for row in evs]

    # The timed number: the step replayed as one CUDA graph (the same kernels on
    # the same buffers, without per-launch host overhead).
    graph = binding.StepGraph(layer, x, noise=noise, token_loss=tl, out=out)
    for _ in range(W):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id_for(dev.index))
    clocks.start()
    time.sleep(0.3)
    if flush is None:
        start.record(stream)
        for _ in range(K):
            graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
        ms = start.elapsed_time(end)
    else:
        # The layer's data fits in L2: before every timed step a 256 MB write
        # (twice L2) evicts it, outside the step's own events.
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in ev)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    if layer.device_status() != 0:
        raise RuntimeError(f"{w.name}: device status reports a timeout")
    ms_t = torch.tensor([ms], device=dev)
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    stage_ms = {n: statistics.mean(v) for n, v in stage.items()}
    if w.dtype == "bf16":
        # Both expert GEMMs run in one launch: their events bracket it together.
        stage_ms = {("gemms" if n == "gemm1" else n): (v + stage_ms["gemm2"] if n == "gemm1" else v)
                    for n, v in stage_ms.items() if n != "gemm2"}
    res = dict(w=w, inp=inp, T=T, K=K, ms_max=ms_max, ms_step=ms_max / K, ms_eager=statistics.mean(eager_steps),
               stage=stage_ms, kept=kept, touched=touched,
               n_dropped=int(out["n_dropped"].item()), launches_per_step=launches_per_step, clocks=clk,
               value=world * T * K / (ms_max / 1e3))

    # End to end through the public API with host buffers: binding.HostPipeline
    # uploads each step's inputs from pinned host memory, runs the forward and
    # statistics, and downloads y and the statistics, overlapping the copies of
    # one step with the neighbouring steps' compute (two device slots).
    res["e2e"] = None
    if headline and not args.no_e2e:
        x_h = x.cpu().pin_memory()
        noise_h = noise.cpu().pin_memory() if noise is not None else None
        tl_h = tl.cpu().pin_memory() if tl is not None else None
        y_h = [torch.empty_like(out["y"], device="cpu").pin_memory() for _ in range(2)]
        st_h = [{k: torch.empty_like(out[k], device="cpu").pin_memory() for k in binding.HostPipeline.STAT_KEYS}
                for _ in range(2)]
        pipe = binding.HostPipeline(layer, T, with_noise=noise is not None, with_loss=tl is not None)
        for i in range(2):
            pipe.submit(x_h, y_h[i % 2], noise_h, tl_h, st_h[i % 2])
        pipe.synchronize()
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        Ke = max(3, K)  # the same steps as the device timing; one upload and one download are not overlapped
        s2.record(pipe.up)
        for i in range(Ke):
            pipe.submit(x_h, y_h[i % 2], noise_h, tl_h, st_h[i % 2])
        e2.record(pipe.down)
        pipe.synchronize()
        t2 = torch.tensor([s2.elapsed_time(e2)], device=dev)
        if world > 1:
            dist.all_reduce(t2, op=dist.ReduceOp.MAX)
        h2d = x_h.numel() * x_h.element_size() + (noise_h.numel() * 4 if noise_h is not None else 0) + \
            (tl_h.numel() * 4 if tl_h is not None else 0)
        d2h = y_h[0].numel() * y_h[0].element_size() + sum(v.numel() * v.element_size() for v in st_h[0].values())
        res["e2e"] = {"value": world * T * Ke / (float(t2.item()) / 1e3), "unit": UNIT,
                      "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": Ke,
                      "how": "binding.HostPipeline: pinned-host inputs uploaded, forward + statistics, y and "
                             "statistics downloaded every step; copies of one step overlap the neighbouring "
                             "steps' compute"}
        del pipe
    del graph, layer, out, flush
    return res


def gemm_roofline(r, peaks):
    """The expert GEMMs (both launches) between their own stage events. A
    tensor-bound layer: the algorithmic FLOPs of the kept and shared rows over
    their mean duration, against the bf16 tensor peak. An HBM-bound layer
    (decode-sized batches): the weight bytes of the experts with a kept row
    (the bytes the two GEMMs must stream) over the same duration, against the
    HBM peak."""
    w = r["w"]
    rows = r["kept"] + w.S * w.T
    ms = r["stage"]["gemms"] if "gemms" in r["stage"] else r["stage"]["gemm1"] + r["stage"]["gemm2"]
    lr = layer_roofline(w, r["kept"], r["touched"], r["ms_step"], peaks)
    if lr["bound"] == "hbm":
        es = 2 if w.dtype == "bf16" else 4
        wbytes = r["touched"] * (w.F * w.d + w.O * w.F) * es
        achieved = wbytes / (ms / 1e3) / 1e9
        return {"kernel": "grouped_gemm_pair (expert GEMM 1 + 2)", "bound": "hbm", "achieved": achieved,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "peak_kind": f"HBM copy ({peaks['source']})", "algorithmic_bytes": wbytes}
    achieved = 2.0 * rows * w.F * (w.d + w.O) / (ms / 1e3) / 1e12
    return {"kernel": "grouped_gemm_pair (expert GEMM 1 + 2)", "bound": "tensor", "achieved": achieved,
            "peak": peaks["bf16"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16"],
            "frac_sustained": achieved / peaks["bf16_sustained"],
            "peak_kind": f"bf16 burst ({peaks['source']}); frac_sustained against the sustained peak"}


def config_summary(r, peaks):
    """The sub-object of one non-headline configuration."""
    w = r["w"]
    d = {"T": w.T, "d": w.d, "d_ff": w.F, "out": w.O, "E": w.E, "k": w.k, "S": w.S, "dtype": w.dtype,
         "ms_per_step": r["ms_step"], "value": r["value"], "unit": UNIT, "steps": r["K"],
         "ms_per_step_eager": r["ms_eager"], "stage_ms": r["stage"], "kept_rows": r["kept"],
         "n_dropped": r["n_dropped"], "gpu_launches": r["launches_per_step"] * r["K"], "clocks": r["clocks"],
         "l2": l2_note(w)}
    if w.dtype == "bf16":
        d.update(layer_roofline(w, r["kept"], r["touched"], r["ms_step"], peaks))
        d["roofline"] = gemm_roofline(r, peaks)
    else:
        d["bound"] = "latency"
        d["note"] = "fp32 layer on CUDA cores at T=4: launch-latency bound, no roofline"
    return d


EXTRA_CONFIGS = ("tiny", "default", "e64", "decode")


def run_ours(args):
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_gate_b200.workloads import WORKLOADS

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_(T=args.tokens)
    if args.experts:
        w = w.with_(E=args.experts)
    if args.dff:
        w = w.with_(F=args.dff)
    head = measure(w, args, dev, rank, world, headline=True)
    inp = head.pop("inp")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # A first sample calibrates; the reported one is sized to about 12 s of
        # oracle work (at most 512 tokens).
        T_s = min(w.T, 64, max(8, 2 * oracle_threads()))
        secs, n = cpu_sample_from_device(w, inp, T_s)
        if secs < 8.0 and T_s < min(w.T, 512):
            T_s = int(min(w.T, 512, max(T_s + 1, T_s * 12.0 / max(secs, 1e-3))))
            secs, n = cpu_sample_from_device(w, inp, T_s)
        cpu = {"value": n / secs, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
               "sample": f"{n} tokens of {w.name} through the whole fp64 oracle forward (capacity at T={n}), "
                         f"{secs:.1f} s"}
    del inp
    torch.cuda.empty_cache()
    extras = {}
    if args.workload == "e256" and not (args.tokens or args.experts or args.dff or args.no_extras):
        for name in EXTRA_CONFIGS:
            r = measure(WORKLOADS[name], args, dev, rank, world, headline=False)
            del r["inp"]
            torch.cuda.empty_cache()
            extras[name] = config_summary(r, measured_peaks())

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peaks = measured_peaks()
    lr = layer_roofline(w, head["kept"], head["touched"], head["ms_step"], peaks)
    roof = gemm_roofline(head, peaks)
    roof["traffic"] = committed_traffic(w, head["kept"] + w.S * w.T)

    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": head["K"],
        "warmup": args.warmup, "ms_per_step": head["ms_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded; x ~ N(0,1), weights ~ N(0,1/fan_in))",
        "config": {"workload": w.name, "T": w.T, "d": w.d, "d_ff": w.F, "out": w.O, "E": w.E, "k": w.k, "S": w.S,
                   "activation": w.activation, "capacity_factor": w.capacity_factor,
                   "tokens_per_rank": w.T, "parallelism": f"replicas x{world}", "l2": l2_note(w)},
        "expert_gemm_tflops": lr["expert_gemm_tflops"],
        "layer_roofline_frac": lr["layer_roofline_frac"],
        "layer_roofline_frac_sustained": lr["layer_roofline_frac_sustained"],
        "layer_roofline_frac_spec_sheet": lr["layer_roofline_frac_spec_sheet"],
        "layer_bound": lr["bound"],
        "roofline": roof,
        "stage_ms": head["stage"],
        "launch": "cuda_graph (one graph per step); stage_ms from an instrumented eager loop; router planes "
                  "split once per run (moe_prepare_router)",
        "ms_per_step_eager": head["ms_eager"],
        "kept_rows": head["kept"], "n_dropped": head["n_dropped"],
        "gpu_launches": head["launches_per_step"] * head["K"],
        "e2e": head["e2e"], "cpu_baseline": cpu, "clocks": head["clocks"],
        "peaks": {k: peaks[k] for k in ("bf16", "bf16_sustained", "hbm_gbs", "source")},
    }
    if extras:
        line["configs"] = extras
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


L2_BYTES = 126e6


def _input_bytes(w):
    es = 2 if w.dtype == "bf16" else 4
    return w.T * w.d * es, (w.E + w.S) * w.F * (w.d + w.O) * es


def inputs_exceed_l2(w) -> bool:
    """True when the expert weights alone are larger than L2, so that no step
    finds the previous step's data there."""
    return _input_bytes(w)[1] > L2_BYTES


def l2_note(w):
    xb, wb = _input_bytes(w)
    size = (lambda b: f"{b / 1e9:.1f} GB" if b >= 1e9 else f"{b / 1e6:.0f} MB")
    return (f"x {size(xb)}, expert weights {size(wb)}: "
            + ("inputs larger than L2 (126 MB); no flush" if inputs_exceed_l2(w)
               else "inputs fit in L2 (126 MB): a 256 MB write before every timed step, outside its events"))


def committed_traffic(w, rows):
    """DRAM bytes per expert-GEMM launch pair for workload `w` with `rows` kept
    plus shared rows, from the committed ncu summary of a scaled case of the same
    per-expert shape (fewer experts and tokens, a few GB on the device), scaled
    by the rows processed. None when the kernel source changed since the capture
    or the workload was resized on the command line."""
    import hashlib
    from sparse_mixture_experts_gate_b200.workloads import WORKLOADS
    if WORKLOADS.get(w.name) != w:
        return None
    path = os.path.join(ROOT, "profiles", f"grouped_gemm_pair_{w.name}_traffic.txt")
    src = os.path.join(ROOT, "sparse_mixture_experts_gate_b200", "csrc", "gemm_pair.cu")
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256") != sha:
        return None
    try:
        return float(vals["dram_bytes_per_launch_pair"]) * rows / float(vals["capture_rows"])
    except (KeyError, ValueError, ZeroDivisionError):
        return None


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    import numpy as np
    import torch
    from sparse_mixture_experts_gate_b200.workloads import WORKLOADS, make_expert_weights, make_tokens, \
        make_router

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_(T=args.tokens)
    if args.experts:
        w = w.with_(E=args.experts)
    threads = oracle_threads()
    # Calibrate: a step is a T_s-token sample sized to about 2 s of oracle work.
    router = make_router(w, "cpu")
    toks = make_tokens(w.with_(T=max(1, min(w.T, 256))), "cpu")
    cache = {}

    def experts(es):
        need = [e for e in es if e not in cache]
        if need:
            got = make_expert_weights(w, need, "cpu")
            for e in need:
                cache[e] = {k: got[k][e] for k in got}
        return {k: {e: cache[e][k] for e in es} for k in ("w1", "b1", "w2", "b2")}

    def sample(n):
        sl = slice(0, n)
        return oracle_sample(w, toks["x"][sl], router["w_gate"], router.get("b_gate"), router.get("sel_bias"),
                             None if toks.get("noise") is None else toks["noise"][sl],
                             None if toks.get("token_loss") is None else toks["token_loss"][sl], experts)

    t1, _ = sample(1)
    budget_s = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    T_s = int(max(1, min(toks["x"].shape[0], budget_s / max(t1, 1e-3) * min(threads, 8))))
    for _ in range(args.warmup):
        sample(T_s)
    tot, n_tok = 0.0, 0
    for _ in range(args.steps):
        s, n = sample(T_s)
        tot += s
        n_tok += n
    value = n_tok / tot
    desc = f"{T_s} tokens of {w.name} per step through the whole fp64 oracle forward (capacity at T={T_s})"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, CPU generator)",
            "config": {"workload": w.name, "T": w.T, "d": w.d, "d_ff": w.F, "out": w.O, "E": w.E, "k": w.k,
                       "S": w.S, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def torchrun_argv(argv, n: int, port: int, limit_s: int = 1800):
    """The command that runs this script as n ranks of one node (one process
    per GPU, rendezvous on 127.0.0.1), bounded from outside by `timeout`."""
    return ["timeout", "-k", "60", str(limit_s), sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.join(ROOT, "bench.py")] + list(argv)


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # Not started by a launcher: start the N ranks here; rank 0 prints the line.
        sys.exit(subprocess.call(torchrun_argv(sys.argv[1:], args.gpus, free_port())))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

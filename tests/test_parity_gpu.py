"""CUDA path vs the CPU oracle, element by element, through the C ABI (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import (check_end_to_end, check_expert_loss, check_same_logits_routing, expert_table,
                         run_gpu, stratified_tokens)
from sparse_mixture_experts_gate_b200.binding import MoEError, MoELayer
from sparse_mixture_experts_gate_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def full_check(w, inp):
    g, layer = run_gpu(w, inp)
    check_same_logits_routing(w, inp, g)
    info = check_end_to_end(w, inp, g)
    if inp.get("token_loss") is not None:
        check_expert_loss(w, inp, g)
    return g, info


# ---------------------------------------------------------------- small cases

def test_tiny_fp32_minimal_example():
    """The walkthrough's minimal example: 4 experts, 2 active, 8/16/8, T=4, fp32."""
    w = WORKLOADS["tiny"]
    full_check(w, make_inputs(w, "cpu"))


def test_tiny_fp32_random_biases():
    w = WORKLOADS["tiny"].with_(T=37)
    full_check(w, make_inputs(w, "cpu", seed=5, random_biases=True))


@pytest.mark.parametrize("act", ["relu", "gelu", "swish"])
def test_default_shape_ragged(act):
    """Default SER shape, ragged T spanning several tiles, every activation,
    random biases to exercise the fused epilogues."""
    w = WORKLOADS["default"].with_(T=1000, activation=act)
    full_check(w, make_inputs(w, "cpu", seed=11, random_biases=True))


def test_default_full():
    w = WORKLOADS["default"]
    inp = make_inputs(w, "cpu")
    g, info = full_check(w, inp)
    assert g["n_dropped"][0] >= 0


def test_e64_shape_small():
    """Fine-grained experts (F=1408: five 256-column N tiles and a 128-column one),
    a shared expert, selection bias."""
    w = WORKLOADS["e64"].with_(T=700)
    g, _ = full_check(w, make_inputs(w, "cpu", seed=3))
    assert g["n_dropped"][0] > 0  # C_f = 1.25 at T=700 binds for some experts


def test_decode_shape_noisy():
    w = WORKLOADS["decode"]
    full_check(w, make_inputs(w, "cpu"))


def test_e256_shape_small():
    w = WORKLOADS["e256"].with_(T=300)
    full_check(w, make_inputs(w, "cpu", seed=9))


# ---------------------------------------------------------------- edge cases

def test_single_token():
    w = WORKLOADS["e64"].with_(T=1)
    full_check(w, make_inputs(w, "cpu"))


def test_dense_reduction_E1_k1():
    w = WORKLOADS["default"].with_(T=300, E=1, k=1, S=0, capacity_factor=0.0)
    g, _ = full_check(w, make_inputs(w, "cpu", random_biases=True))
    assert (g["topk_idx"] == 0).all() and np.allclose(g["gates"], 1.0)


def test_k_equals_E_two_shared():
    w = WORKLOADS["default"].with_(T=260, E=4, k=4, S=2, capacity_factor=0.0, activation="swish")
    full_check(w, make_inputs(w, "cpu", seed=2, random_biases=True))


def test_all_tokens_one_expert_heavy_drops():
    """A large router bias on expert 0: every token selects it, and the cap
    C = ceil(C_f k T / E) keeps only the earliest C tokens."""
    w = WORKLOADS["default"].with_(T=900, capacity_factor=1.0, router_bias=True)
    inp = make_inputs(w, "cpu", seed=4)
    inp["b_gate"][0] = 50.0
    g, _ = full_check(w, inp)
    C = oracle.capacity(1.0, w.k, w.T, w.E)
    assert g["count_pre"][0] == w.T and g["count_kept"][0] == C
    assert g["n_dropped"][0] >= w.T - C
    assert (g["slot"][:C, 0] == np.arange(C)).all() and (g["slot"][C:, 0] == -1).all()


def test_tiny_capacity():
    w = WORKLOADS["e64"].with_(T=200, capacity_factor=0.05)
    g, _ = full_check(w, make_inputs(w, "cpu", seed=6))
    assert (g["count_kept"] <= 1).all()


def test_zero_tokens_is_a_noop():
    w = WORKLOADS["default"]
    inp = make_inputs(w.with_(T=4), "cpu")
    layer = MoELayer(w, inp)
    x = torch.empty(0, w.d, dtype=torch.bfloat16, device="cuda")
    out = layer.forward(x)
    layer.aux_stats(out)
    torch.cuda.synchronize()
    assert layer.device_status() == 0


def test_determinism_bit_identical():
    w = WORKLOADS["e64"].with_(T=1500)
    inp = make_inputs(w, "cpu", seed=8)
    g1, layer = run_gpu(w, inp)
    g2, _ = run_gpu(w, inp, layer=layer)
    for k in ("y", "logits", "gates", "topk_idx", "slot", "count_pre", "f", "p_mean", "l_aux", "l_z", "credit"):
        assert np.array_equal(g1[k], g2[k], equal_nan=True), k


@pytest.mark.parametrize("name,T", [("e64", 8192), ("default", 100), ("decode", 128)])
def test_repeated_forwards_bit_identical(name, T):
    """Both expert GEMM layers share one launch, GEMM 2's units of a token
    tile waiting on a per-tile counter that GEMM 1's epilogues release once
    their stores are complete. A missed or early release would let a unit
    read hidden rows that are not written yet, so repeated forwards of the
    same batch (full-size e64 with wide tiles, narrow-tile batches) must give
    the same bits every time."""
    w = WORKLOADS[name].with_(T=T)
    inp = make_inputs(w, "cuda", seed=19)
    layer = MoELayer(w, inp)
    ref = None
    for _ in range(12):
        out = layer.forward(inp["x"], noise=inp.get("noise"))
        torch.cuda.synchronize()
        y = out["y"].view(torch.int16).cpu().numpy()
        if ref is None:
            ref = y.copy()
        else:
            assert np.array_equal(ref, y)
    assert layer.device_status() == 0


def test_forward_argument_errors_on_host():
    w = WORKLOADS["default"]
    inp = make_inputs(w.with_(T=8), "cpu")
    layer = MoELayer(w, inp, max_tokens=8)
    x = inp["x"].cuda()
    with pytest.raises(MoEError):  # T > max_tokens
        layer.forward(torch.empty(9, w.d, dtype=torch.bfloat16, device="cuda"))
    ws, need = layer.workspace(8)
    from sparse_mixture_experts_gate_b200 import binding
    y = torch.empty(8, w.O, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    with pytest.raises(MoEError) as ei:
        binding.moe_forward(layer.handle, x.data_ptr(), 8, None, ws.data_ptr(), need - 1, y.data_ptr(), None, s)
    assert ei.value.code == binding.MOE_ERR_WORKSPACE
    with pytest.raises(MoEError) as ei:
        binding.moe_forward(layer.handle, x.data_ptr(), 8, None, ws.data_ptr() + 16, need, y.data_ptr(), None, s)
    assert ei.value.code == binding.MOE_ERR_WORKSPACE
    noisy = MoELayer(w.with_(top_k_method="noisy"), inp)
    with pytest.raises(MoEError) as ei:
        noisy.forward(x)  # NOISY without noise
    assert ei.value.code == binding.MOE_ERR_INVALID_ARG
    fresh = MoELayer(w, inp)
    with pytest.raises(MoEError) as ei:
        fresh.aux_stats(fresh.alloc_outputs(8))
    assert ei.value.code == binding.MOE_ERR_STATE


# ---------------------------------------------------------------- full sizes

def _sampled_full(name, min_tokens):
    """The full-size workload in the launch configuration the benchmark times:
    routing, dispatch and statistics over every token (same-logits mode); y and
    credit on a stratified sample of tokens that reaches every token tile of
    every expert (both GEMMs, every feature tile), the last kept row of every
    expert, every shared-expert tile and the last token."""
    w = WORKLOADS[name]
    inp = make_inputs(w, "cuda")
    g, _ = run_gpu(w, inp, poison=False)
    check_same_logits_routing(w, {k: (v.cpu() if v is not None else None) for k, v in inp.items()
                                  if k in ("noise", "sel_bias")}, g)
    toks, n_items = stratified_tokens(g, w, tile_rows=256, min_tokens=min_tokens)
    experts = g["topk_idx"][toks].ravel()
    table = expert_table(w, inp, experts)
    info = check_end_to_end(w, inp, g, tokens=toks, table=table)
    if inp.get("token_loss") is not None:
        check_expert_loss(w, {"token_loss": inp["token_loss"]}, g)
    # Properties that hold at any size.
    assert int(g["count_kept"].sum()) == w.k * w.T - int(g["n_dropped"][0])
    assert int(g["count_pre"].sum()) == w.k * w.T
    assert np.allclose(g["gates"].sum(1), 1.0, atol=1e-5)
    print(f"{name}: {len(toks)} sampled tokens cover {n_items} GEMM tiles and last rows; y_err {info['y_err']:.2e}, "
          f"logit_err {info['logit_err']:.2e}")
    return g, info


def test_e64_full_size_sampled():
    _sampled_full("e64", 128)


def test_e256_full_size_sampled():
    _sampled_full("e256", 512)


# ------------------------------------------------- data-parallel statistics

def test_dp_stats_two_shards_through_kernels():
    """Two shards of one batch run in turn through the same layer; their
    partial sums (moe_stat_partials), added, give through
    moe_stats_from_partials the statistics of the whole batch: f, P, L_aux and
    L_z of the concatenated routing, drops and attributed loss of each shard's
    own dispatch divided by the whole batch size."""
    from sparse_mixture_experts_gate_b200.binding import (MoeStats, moe_stat_partials, moe_stats_from_partials,
                                                          stat_partials_size)
    w = WORKLOADS["e64"].with_(T=1100, token_loss=True)
    inp = make_inputs(w, "cpu", seed=21)
    cuts = [0, 389, w.T]
    layer = MoELayer(w, inp)
    total = torch.zeros(stat_partials_size(w.E), dtype=torch.float32, device="cuda")
    shards = []
    s = torch.cuda.current_stream().cuda_stream
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        sub = {k: (v[lo:hi] if (v is not None and k in ("x", "noise", "token_loss")) else v) for k, v in inp.items()}
        g, _ = run_gpu(w.with_(T=hi - lo), sub, layer=layer)
        part = torch.full((stat_partials_size(w.E),), float("nan"), device="cuda")
        tl = sub["token_loss"].cuda().contiguous()
        moe_stat_partials(layer.handle, tl.data_ptr(), part.data_ptr(), s)
        total += part
        shards.append(g)
    out = layer.alloc_outputs(1)
    for v in out.values():
        v.fill_(-7)
    st = MoELayer._stats_struct(out, True, False)
    moe_stats_from_partials(layer.handle, total.data_ptr(), True, st, s)
    torch.cuda.synchronize()
    dp = {k: out[k].cpu().numpy().astype(np.float64) for k in ("f", "p_mean", "l_aux", "l_z", "n_dropped",
                                                               "expert_loss", "importance", "cv_load",
                                                               "cv_importance")}

    # Same-logits oracle routing of the whole batch from the GPU's logits.
    logits = np.concatenate([g["logits"] for g in shards]).astype(np.float32)
    r = oracle.routing_from_logits(logits, w, noise=None, sel_bias=inp["sel_bias"])
    f, pm, la, lz = oracle.balance_stats(r["P"], r["lse"], r["count_pre"], w.k, w.alpha, w.beta)
    assert np.abs(dp["f"] - f).max() <= 1e-4
    assert np.abs(dp["p_mean"] - pm).max() <= 1e-4
    assert abs(dp["l_aux"][0] - la) <= 1e-4
    assert abs(dp["l_z"][0] - lz) <= 1e-4
    assert int(dp["n_dropped"][0]) == sum(int(g["n_dropped"][0]) for g in shards)
    imp = oracle.importance(np.concatenate([g["topk_idx"] for g in shards]),
                            np.concatenate([g["gates"] for g in shards]), w.E)
    assert np.abs(dp["importance"] - imp).max() <= 1e-4 * (1 + imp.max())
    assert abs(dp["cv_load"][0] - oracle.cv_squared(r["count_pre"])) <= 1e-4
    assert abs(dp["cv_importance"][0] - oracle.cv_squared(imp)) <= 1e-4
    el = oracle.expert_loss(np.concatenate([g["topk_idx"] for g in shards]),
                            np.concatenate([g["slot"] for g in shards]),
                            np.concatenate([g["credit"] for g in shards]), inp["token_loss"], w.E)
    assert (np.abs(dp["expert_loss"] - el) / (1 + np.abs(el))).max() <= 1e-4
    # The one-rank helper equals moe_aux_stats on the last shard alone.
    g_last = shards[-1]
    out1 = layer.alloc_outputs(cuts[2] - cuts[1])
    layer.forward(inp["x"][cuts[1]:].cuda().contiguous(), out=out1)
    layer.dp_aux_stats(out1, token_loss=inp["token_loss"][cuts[1]:].cuda().contiguous())
    torch.cuda.synchronize()
    assert np.array_equal(out1["f"].cpu().numpy(), g_last["f"].astype(np.float32))
    assert np.array_equal(out1["l_aux"].cpu().numpy(), g_last["l_aux"].astype(np.float32))
    assert np.array_equal(out1["expert_loss"].cpu().numpy(), g_last["expert_loss"].astype(np.float32))


@pytest.mark.parametrize("F,O", [(1088, 320), (704, 384)])
def test_ragged_n_tiles_both_layers(F, O):
    """Expert widths that are not multiples of the 256-feature tile. A last
    tile of at most 128 features runs as a transposed unit (tokens on the
    MMA's M side): 64 features (F = 1088, O = 320) or 128 (O = 384); a last
    tile of 192 features (F = 704) runs as an ordinary unit with a partly idle
    M side."""
    w = WORKLOADS["default"].with_(T=777, F=F, O=O, S=1, activation="swish")
    full_check(w, make_inputs(w, "cpu", seed=13, random_biases=True))


def test_selection_bias_update_bit_exact():
    """Aux-loss-free balancing ("Balancing": b_i with update rate gamma): the
    update from this forward's loads and the one from summed partials of two
    shards match the oracle's update on the same loads bit for bit, and the
    next forward selects with the updated bias."""
    from sparse_mixture_experts_gate_b200.binding import moe_stat_partials, stat_partials_size
    w = WORKLOADS["e64"].with_(T=900)
    inp = make_inputs(w, "cpu", seed=31)
    g, layer = run_gpu(w, inp)
    b0 = layer.weights["sel_bias"].cpu().numpy().copy()
    layer.update_selection_bias(1e-3)
    torch.cuda.synchronize()
    want = oracle.selection_bias_update(b0, g["count_pre"], w.k, w.T, 1e-3)
    assert np.array_equal(layer.weights["sel_bias"].cpu().numpy(), want)
    # From the partial sums of two shards (the data-parallel path).
    b1 = layer.weights["sel_bias"].cpu().numpy().copy()
    total = torch.zeros(stat_partials_size(w.E), device="cuda")
    loads = np.zeros(w.E, np.int64)
    s = torch.cuda.current_stream().cuda_stream
    for lo, hi in ((0, 500), (500, w.T)):
        sub = {k: (v[lo:hi] if (v is not None and k in ("x", "noise", "token_loss")) else v) for k, v in inp.items()}
        gs, _ = run_gpu(w.with_(T=hi - lo), sub, layer=layer)
        part = torch.empty(stat_partials_size(w.E), device="cuda")
        moe_stat_partials(layer.handle, None, part.data_ptr(), s)
        total += part
        loads += gs["count_pre"]
    layer.update_selection_bias(-2e-3, partials=total)
    torch.cuda.synchronize()
    want = oracle.selection_bias_update(b1, loads, w.k, w.T, -2e-3)
    assert np.array_equal(layer.weights["sel_bias"].cpu().numpy(), want)
    # The next forward routes with the updated bias (same-logits check).
    inp2 = dict(inp, sel_bias=layer.weights["sel_bias"].cpu())
    g2, _ = run_gpu(w, inp2, layer=layer)
    check_same_logits_routing(w, inp2, g2)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_credit_hidden_activation_norm(dtype):
    """Credit with ||h|| read as the hidden activation's norm ("Sparse MoE
    Expert-Credit Loss Reweighting Diagram", panel (b)), and the attributed
    loss built from it."""
    w = WORKLOADS["default"].with_(T=333, E=6, k=2, S=1, F=1088 if dtype == "bf16" else 96,
                                   d=256 if dtype == "bf16" else 64, O=320 if dtype == "bf16" else 48,
                                   activation="swish", dtype=dtype, credit_norm="hidden", token_loss=True,
                                   capacity_factor=1.0)
    full_check(w, make_inputs(w, "cpu", seed=17, random_biases=True))


def test_dro_update_matches_oracle():
    """Panel (c) bookkeeping: EMA of the expert losses, mu <- softmax(mu + eta lhat)
    and the objective sum mu l, fp32 on the GPU against the fp64 oracle."""
    from sparse_mixture_experts_gate_b200.binding import moe_dro_update
    w = WORKLOADS["default"].with_(T=64, d=64, F=64, O=64, E=200, k=4)
    layer = MoELayer(w, make_inputs(w, "cpu", seed=3))
    rng = np.random.default_rng(9)
    l = rng.gamma(2.0, 0.5, w.E)
    lhat = rng.gamma(2.0, 0.5, w.E)
    mu = rng.dirichlet(np.ones(w.E))
    dl, dlh, dmu = (torch.tensor(v, dtype=torch.float32, device="cuda") for v in (l, lhat, mu))
    obj = torch.empty(1, device="cuda")
    for ema, eta in ((0.9, 0.5), (0.0, 3.0), (1.0, 0.0)):
        lh0, mu0 = dlh.cpu().numpy().astype(np.float64), dmu.cpu().numpy().astype(np.float64)
        moe_dro_update(layer.handle, dl.data_ptr(), ema, eta, dlh.data_ptr(), dmu.data_ptr(), obj.data_ptr(),
                       torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        want_lh, want_mu, want_obj = oracle.dro_update(dl.cpu().numpy(), lh0, mu0, ema, eta)
        assert np.abs(dlh.cpu().numpy() - want_lh).max() <= 1e-6 * (1 + np.abs(want_lh).max())
        assert np.abs(dmu.cpu().numpy() - want_mu).max() <= 1e-6
        assert abs(obj.item() - want_obj) <= 1e-6 * (1 + abs(want_obj))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_rank_major_capacity_priority(dtype):
    """GShard-style capacity priority (every first choice before any second
    choice): bit-exact slots and drops on the same logits, with heavy drops."""
    w = WORKLOADS["default"].with_(T=1500, E=16, k=4, S=0, capacity_factor=0.6, capacity_priority="rank",
                                   dtype=dtype, d=128 if dtype == "bf16" else 64,
                                   F=256 if dtype == "bf16" else 64, O=128 if dtype == "bf16" else 64)
    inp = make_inputs(w, "cpu", seed=23)
    g, layer = run_gpu(w, inp)
    # C_f = 0.6 is stored as fp32 (0.600000024): C = ceil(fl32(C_f) k T / E).
    from sparse_mixture_experts_gate_b200.binding import moe_capacity
    assert moe_capacity(layer.handle, w.T) == oracle.capacity(oracle.layer_capacity_factor(w), w.k, w.T, w.E)
    check_same_logits_routing(w, inp, g)
    check_end_to_end(w, inp, g)
    assert g["n_dropped"][0] > 0
    # The priority changes which assignments drop, not how many per expert.
    r_tok = oracle.routing_from_logits(g["logits"].astype(np.float32), w.with_(capacity_priority="token"))
    assert np.array_equal(g["count_kept"], r_tok["count_kept"])
    assert not np.array_equal(g["slot"], r_tok["slot"])


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_mlp_gate_router(dtype):
    """The optional MLP gate (use_mlp_gater, hidden 128): logits against the
    oracle's h = W_2 relu(W_1 x + b_1) + b_2, routing and outputs as usual."""
    w = WORKLOADS["default"].with_(T=700, E=24, k=3, S=1, mlp_gater=True, router_bias=True, dtype=dtype,
                                   d=256 if dtype == "bf16" else 64, F=256 if dtype == "bf16" else 64,
                                   O=128 if dtype == "bf16" else 32, use_selection_bias=True)
    full_check(w, make_inputs(w, "cpu", seed=29, random_biases=True))


def test_host_pipeline_matches_serial_forward():
    """binding.HostPipeline (pinned host inputs and outputs, copies overlapped
    with the neighbouring steps' compute) gives bit-for-bit the results of the
    plain device forward, for several different batches in flight."""
    from sparse_mixture_experts_gate_b200.binding import HostPipeline
    from sparse_mixture_experts_gate_b200.workloads import make_tokens
    w = WORKLOADS["e64"].with_(T=640, token_loss=True)
    inp = make_inputs(w, "cpu", seed=41)
    layer = MoELayer(w, inp)
    batches = [make_tokens(w, "cpu", seed=100 + i) for i in range(4)]
    want = []
    for b in batches:
        out = layer.forward(b["x"].cuda(), out=None)
        layer.aux_stats(out, token_loss=b["token_loss"].cuda())
        torch.cuda.synchronize()
        want.append({k: v.cpu().clone() for k, v in out.items()})
    pipe = HostPipeline(layer, w.T, with_loss=True)
    ys = [torch.empty(w.T, w.O, dtype=torch.bfloat16).pin_memory() for _ in batches]
    sts = [{k: torch.empty_like(want[0][k]).pin_memory() for k in HostPipeline.STAT_KEYS} for _ in batches]
    xs = [b["x"].pin_memory() for b in batches]
    ls = [b["token_loss"].pin_memory() for b in batches]
    for i in range(len(batches)):
        pipe.submit(xs[i], ys[i], loss_h=ls[i], stats_h=sts[i])
    pipe.synchronize()
    for i in range(len(batches)):
        assert torch.equal(ys[i], want[i]["y"]), f"batch {i}: y differs"
        for k in HostPipeline.STAT_KEYS:
            assert torch.equal(sts[i][k], want[i][k]), f"batch {i}: {k} differs"


def test_bounded_wait_times_out_and_context_survives():
    """Failure detection without a GPU fault: a wait on a barrier nothing
    arrives on gives up after its limit and reports the timeout; afterwards the
    context still runs a forward that matches the oracle."""
    from sparse_mixture_experts_gate_b200.binding import moe_selftest_bounded_wait
    assert moe_selftest_bounded_wait(torch.cuda.current_stream().cuda_stream) == 0
    w = WORKLOADS["default"].with_(T=300)
    full_check(w, make_inputs(w, "cpu", seed=2))


@pytest.mark.parametrize("T", [600, 100])
def test_expert_gemm_timeout_drains_and_context_survives(T):
    """Failure detection inside the real expert GEMM: GEMM 1's leader CTAs skip
    one stage's loads (a test-only launch argument) and the launch's waits give
    up after 20 ms. The MMA role's wait runs out, every role drains and the
    kernel returns; the device status reports the timeout; the same layer and
    context then run a forward that matches the oracle. T = 100 is a
    decode-sized batch (narrow token tiles), whose two GEMMs share one launch:
    there the GEMM 2 units waiting for GEMM 1's rows give up as well."""
    from sparse_mixture_experts_gate_b200 import binding
    w = WORKLOADS["default"].with_(T=T)
    inp = make_inputs(w, "cpu", seed=2)
    layer = MoELayer(w, inp)
    x = inp["x"].cuda()
    ws, need = layer.workspace(w.T)
    y = torch.empty(w.T, w.O, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert binding.moe_selftest_gemm_timeout(layer.handle, x.data_ptr(), w.T, ws.data_ptr(), ws.numel(),
                                             y.data_ptr(), s) == 0
    assert layer.device_status() == binding.MOE_ERR_TIMEOUT
    g, _ = run_gpu(w, inp, layer=layer)  # asserts a clean status itself
    check_same_logits_routing(w, inp, g)
    check_end_to_end(w, inp, g)


def test_router_timeout_drains_and_context_survives():
    """Failure detection inside the fused router: every CTA pair's leader skips
    one stage's loads (a test-only launch argument) and the launch's waits give
    up after 20 ms. The MMA role's wait runs out, every role stops, the CTAs
    pass the grid barrier without routing and the kernel returns; the status
    word reports the timeout; the same layer and context then run a forward that
    matches the oracle."""
    from sparse_mixture_experts_gate_b200 import binding
    w = WORKLOADS["default"].with_(T=600)
    inp = make_inputs(w, "cpu", seed=3)
    layer = MoELayer(w, inp)
    x = inp["x"].cuda()
    ws, need = layer.workspace(w.T)
    s = torch.cuda.current_stream().cuda_stream
    assert binding.moe_selftest_router_timeout(layer.handle, x.data_ptr(), w.T, ws.data_ptr(), ws.numel(), s) == 0
    g, _ = run_gpu(w, inp, layer=layer)  # asserts a clean status itself
    check_same_logits_routing(w, inp, g)
    check_end_to_end(w, inp, g)


def _emulated_all_to_all(inputs, splits):
    """What all_to_all_single delivers to each rank q: from every rank r, in
    rank order, the rows r sends to q (splits[r][q] rows after the earlier ones)."""
    G = len(inputs)
    outs = []
    for q in range(G):
        parts = []
        for r in range(G):
            off = sum(splits[r][:q])
            parts.append(inputs[r][off:off + splits[r][q]])
        outs.append(torch.cat(parts))
    return outs


def test_expert_parallel_two_ranks_emulated_on_one_gpu():
    """Expert parallelism ("Capacity & communication": E/G experts per device,
    all-to-all dispatch and combine) with G = 2 ranks emulated in one process:
    each rank routes its own tokens with its own capacity, its rows go to the
    owner of each expert, the owners run their experts, the results come back,
    each rank adds its shared expert and combines. Each rank's y and credit
    match the oracle on that rank's tokens with all experts."""
    from sparse_mixture_experts_gate_b200.binding import ep_send_splits
    from sparse_mixture_experts_gate_b200.workloads import make_tokens
    G = 2
    w = WORKLOADS["e64"].with_(T=500, E=16, k=4, S=1, d=256, F=384, O=320, capacity_factor=1.0)
    inp = make_inputs(w, "cpu", seed=51, random_biases=True)
    El = w.E // G
    layers, batches = [], []
    for r in range(G):
        local = dict(inp)
        for key in ("w1", "b1", "w2", "b2"):
            local[key] = torch.cat([inp[key][r * El:(r + 1) * El], inp[key][w.E:]])
        layers.append(MoELayer(w, local, ep_size=G, ep_rank=r))
        batches.append(make_tokens(w, "cpu", seed=300 + r))
    xs = [b["x"].cuda() for b in batches]  # x must stay valid until ep_combine (shared experts read it)
    phase1 = [layers[r].ep_dispatch(xs[r]) for r in range(G)]
    splits = [ep_send_splits(ph[3], G) for ph in phase1]
    recv = _emulated_all_to_all([ph[1] for ph in phase1], splits)
    counts = [torch.tensor([phase1[r][3][q * El:(q + 1) * El] for r in range(G)], dtype=torch.int32).cuda()
              for q in range(G)]
    outs = [layers[q].ep_experts(recv[q], counts[q]) for q in range(G)]
    # Back: rank q returns to rank r the rows r sent it, in the same order.
    back_splits = [[sum(phase1[r][3][q * El:(q + 1) * El]) for r in range(G)] for q in range(G)]
    returned = _emulated_all_to_all(outs, back_splits)
    for r in range(G):
        phase1[r][2][:returned[r].shape[0]].copy_(returned[r])
        layers[r].ep_combine(phase1[r][0])
        layers[r].aux_stats(phase1[r][0])
    torch.cuda.synchronize()
    table = expert_table(w, inp)
    for r in range(G):
        assert layers[r].device_status() == 0
        out = phase1[r][0]
        g = {k: (v.float().cpu().numpy().astype(np.float64) if v.is_floating_point() else v.cpu().numpy())
             for k, v in out.items()}
        binp = dict(inp, x=batches[r]["x"], token_loss=None, noise=None)
        check_same_logits_routing(w, binp, g)
        check_end_to_end(w, binp, g, table=table)


def test_cuda_graph_step_matches_eager():
    """binding.StepGraph: the forward + statistics captured once and replayed
    (inputs refilled in place) gives bit-for-bit the eager results."""
    from sparse_mixture_experts_gate_b200.binding import StepGraph
    from sparse_mixture_experts_gate_b200.workloads import make_tokens
    w = WORKLOADS["e64"].with_(T=512, token_loss=True)
    inp = make_inputs(w, "cpu", seed=61)
    layer = MoELayer(w, inp)
    b0, b1 = make_tokens(w, "cpu", seed=70), make_tokens(w, "cpu", seed=71)
    x = b0["x"].cuda()
    tl = b0["token_loss"].cuda()
    graph = StepGraph(layer, x, token_loss=tl)
    for b in (b1, b0, b1):
        x.copy_(b["x"].cuda())
        tl.copy_(b["token_loss"].cuda())
        got = {k: v.clone() for k, v in graph.replay().items()}
        torch.cuda.synchronize()
        want = layer.forward(b["x"].cuda())
        layer.aux_stats(want, token_loss=b["token_loss"].cuda())
        torch.cuda.synchronize()
        for k in want:
            assert torch.equal(got[k], want[k]), f"{k} differs between graph replay and eager"


def test_nan_tokens_route_to_valid_experts():
    """NaN inputs are outside the contract, but they must not make the layer
    fault or hang: a NaN token's keys select like -inf (the lowest free expert
    indices), so routing stays valid, and tokens without NaNs keep finite outputs."""
    w = WORKLOADS["default"].with_(T=300, E=8, k=2, capacity_factor=0.0)
    inp = make_inputs(w, "cpu", seed=81)
    x = inp["x"].clone()
    bad = [3, 77, 150]
    x[bad] = float("nan")
    g, layer = run_gpu(w, dict(inp, x=x))
    idx = g["topk_idx"]
    assert ((idx >= 0) & (idx < w.E)).all()
    assert all(len(set(r)) == w.k for r in idx.tolist())
    for t in bad:  # every key ties at -inf: the lowest indices, in ascending order
        assert idx[t].tolist() == list(range(w.k))
    good = np.setdiff1d(np.arange(w.T), bad)
    assert np.isfinite(g["y"][good]).all()


@pytest.mark.parametrize("T", [200, 1500])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_many_active_experts_k16(dtype, T):
    """k = 16 of E = 40 (the largest k the layer takes): the combine's second
    batch of routed terms, top-k over two expert lanes per warp lane group.
    T = 200 runs the combine with a block per token, T = 1500 (more than
    eight tokens per SM) with a warp per token."""
    w = WORKLOADS["default"].with_(T=T, E=40, k=16, S=1, capacity_factor=1.0, dtype=dtype,
                                   d=128 if dtype == "bf16" else 32, F=128 if dtype == "bf16" else 32,
                                   O=128 if dtype == "bf16" else 32, token_loss=True)
    full_check(w, make_inputs(w, "cpu", seed=91, random_biases=True))


@pytest.mark.parametrize("E,d,mode", [(24, 256, "greedy"), (24, 256, "selection_bias"), (24, 256, "noisy"),
                                      (160, 2048, "greedy")])
def test_exact_ties_go_to_the_lower_index(E, d, mode):
    """Finite keys that tie exactly: duplicated router rows give bit-identical
    logits (same operands, same accumulation order, on the tensor cores too, in
    different N tiles and K splits at E = 160, d = 2048), and equal selection
    bias or equal noise keeps the keys equal. The top-k must list the same
    experts in the same order as the oracle's (key descending, lower index
    first on ties), both where a tie straddles the k-th place and where several
    tied experts are all selected."""
    w = WORKLOADS["default"].with_(T=700, E=E, k=4, S=0, d=d, F=256, O=256, capacity_factor=1.0,
                                   top_k_method="noisy" if mode == "noisy" else "greedy", noise=mode == "noisy",
                                   use_selection_bias=mode == "selection_bias")
    inp = make_inputs(w, "cpu", seed=37)
    groups = [[3, 10, 17], [6, 21]] if E == 24 else [[5, 70, 150], [20, 140]]
    wg = inp["w_gate"]
    for grp in groups:
        wg[grp[0]] *= 2.0  # selected often, so that ties decide many tokens
        for e in grp[1:]:
            wg[e] = wg[grp[0]]
            if mode == "selection_bias":
                inp["sel_bias"][e] = inp["sel_bias"][grp[0]]
            if mode == "noisy":
                inp["noise"][:, e] = inp["noise"][:, grp[0]]
    g, _ = full_check(w, inp)
    idx = g["topk_idx"]
    straddle = together = 0
    for grp in groups:
        for e in grp[1:]:
            assert np.array_equal(g["logits"][:, e], g["logits"][:, grp[0]]), "duplicated rows, different logits"
        for t in range(w.T):
            sel = [e for e in idx[t].tolist() if e in grp]
            if 0 < len(sel) < len(grp):  # the tie straddles the k-th place: the lowest indices win
                straddle += 1
                assert sel == grp[:len(sel)], (t, sel, grp)
            if len(sel) >= 2:  # tied experts listed next to each other, lower index first
                together += 1
                pos = [idx[t].tolist().index(e) for e in sel]
                assert pos == list(range(pos[0], pos[0] + len(sel))), (t, idx[t])
    assert straddle > 0 and together > 0, (straddle, together)


def test_prepared_router_planes():
    """moe_prepare_router: the router matrix split once into persistent planes
    gives bit-for-bit the results of the per-forward split with one launch
    fewer, and after the weights change, a new prepare makes the next forward
    follow the new matrix."""
    w = WORKLOADS["e64"].with_(T=900, token_loss=True)
    inp = make_inputs(w, "cpu", seed=44)
    g1, layer = run_gpu(w, inp)
    layer.prepare_router()
    g2, _ = run_gpu(w, inp, layer=layer)
    assert g2["launches"] == g1["launches"] - 1
    for k in ("y", "logits", "gates", "topk_idx", "slot", "count_pre", "f", "p_mean", "l_aux", "l_z", "credit",
              "expert_loss"):
        assert np.array_equal(g1[k], g2[k]), k
    layer.weights["w_gate"].mul_(-0.5)
    layer.prepare_router()
    inp2 = dict(inp, w_gate=layer.weights["w_gate"].cpu())
    g3, _ = run_gpu(w, inp2, layer=layer)
    check_same_logits_routing(w, inp2, g3)
    check_end_to_end(w, inp2, g3)

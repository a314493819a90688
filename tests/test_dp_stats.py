"""Data-parallel balancing statistics on CPU: two gloo ranks each take a ragged
shard of one batch, form the additive partial sums of their shard, sum them
with the package's all-reduce helper, and turn the sums into f_i, P_i, L_aux,
L_z and the attributed loss. The result must equal the oracle's statistics of
the whole, unsharded batch ("Appendix C - Acronyms & Symbols", table
"Balancing": f_i and P_i are fractions and means over the batch, the z-loss a
batch mean; "Sparse MoE Expert-Credit Loss Reweighting Diagram", panel (b): the
attributed loss divides by the batch size N).

The partial-sum layout and the closing step are the ones the C ABI documents
for moe_stat_partials / moe_stats_from_partials; the GPU test of the same
decomposition runs the kernels (test_parity_gpu.py).
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _workload():
    from sparse_mixture_experts_gate_b200.workloads import WORKLOADS
    return WORKLOADS["default"].with_(T=97, d=64, F=128, O=64, E=8, k=2, S=1, capacity_factor=1.0,
                                      dtype="fp32", token_loss=True, router_bias=True)


def _bounds(T: int, world: int):
    cuts = [0, 41, T] if world == 2 else [T * r // world for r in range(world + 1)]
    return cuts


def shard_partials(w, inp, lo: int, hi: int) -> np.ndarray:
    """This shard's sums, laid out as moe_stat_partials writes them."""
    import oracle
    shard = {k: (v[lo:hi] if (v is not None and k in ("x", "noise", "token_loss")) else v) for k, v in inp.items()}
    o = oracle.forward(w, shard)
    E = w.E
    p = np.zeros(4 * E + 3, np.float64)
    p[:E] = o["P"].sum(axis=0)
    p[E:2 * E] = o["count_pre"]
    p[2 * E] = float((o["lse"] ** 2).sum())
    p[2 * E + 1] = hi - lo
    p[2 * E + 2] = o["n_dropped"]
    p[3 * E + 3:] = oracle.importance(o["idx"], o["gates"], E)
    tl = shard["token_loss"].double().numpy()
    for t in range(hi - lo):
        for r in range(w.k):
            if o["slot"][t, r] >= 0:
                p[2 * E + 3 + o["idx"][t, r]] += o["credit"][t, r] * tl[t]
    return p, o


def stats_from_partials(p: np.ndarray, E: int, k: int, alpha: float, beta: float):
    T = p[2 * E + 1]
    pm = p[:E] / T
    f = p[E:2 * E] / (k * T)
    import oracle
    l_aux, l_z = alpha * E * float((f * pm).sum()), beta * p[2 * E] / T
    imp = p[3 * E + 3:]
    return dict(f=f, p_mean=pm, l_aux=l_aux, l_z=l_z, l_total=alpha * oracle.cv_squared(p[E:2 * E]) + l_z,
                n_dropped=int(p[2 * E + 2]),
                expert_loss=p[2 * E + 3:3 * E + 3] / T, importance=imp,
                cv_load=oracle.cv_squared(p[E:2 * E]), cv_importance=oracle.cv_squared(imp))


def _rank_main(rank: int, port: int, result_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        from sparse_mixture_experts_gate_b200.binding import allreduce_partials
        from sparse_mixture_experts_gate_b200.workloads import make_inputs
        w = _workload()
        inp = make_inputs(w)
        cuts = _bounds(w.T, WORLD)
        p, _ = shard_partials(w, inp, cuts[rank], cuts[rank + 1])
        t = torch.from_numpy(p.copy())
        allreduce_partials(t)
        np.save(os.path.join(result_dir, f"rank{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_dp_stats_two_gloo_ranks(tmp_path):
    import oracle
    from sparse_mixture_experts_gate_b200.workloads import make_inputs
    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    sums = [np.load(tmp_path / f"rank{r}.npy") for r in range(WORLD)]
    assert np.array_equal(sums[0], sums[1]), "ranks disagree after the all-reduce"

    w = _workload()
    inp = make_inputs(w)
    dp = stats_from_partials(sums[0], w.E, w.k, w.alpha, w.beta)
    whole = oracle.forward(w, inp)
    # Sharding leaves every per-token quantity unchanged, so these are the
    # whole batch's statistics.
    assert np.allclose(dp["f"], whole["f"], rtol=0, atol=1e-12)
    assert np.allclose(dp["p_mean"], whole["p_mean"], rtol=0, atol=1e-12)
    assert abs(dp["l_aux"] - whole["l_aux"]) <= 1e-12
    assert abs(dp["l_z"] - whole["l_z"]) <= 1e-12
    imp_whole = oracle.importance(whole["idx"], whole["gates"], w.E)
    assert np.allclose(dp["importance"], imp_whole, rtol=1e-12, atol=1e-12)
    assert abs(dp["cv_load"] - oracle.cv_squared(whole["count_pre"])) <= 1e-12
    assert abs(dp["cv_importance"] - oracle.cv_squared(imp_whole)) <= 1e-12
    assert abs(dp["l_total"] - whole["aux_loss"]) <= 1e-12
    # Capacity is per shard, so drops and the attributed loss follow each
    # shard's own dispatch, divided by the whole batch's size.
    cuts = _bounds(w.T, WORLD)
    idx, slot, credit, nd = [], [], [], 0
    for r in range(WORLD):
        _, o = shard_partials(w, inp, cuts[r], cuts[r + 1])
        idx.append(o["idx"]), slot.append(o["slot"]), credit.append(o["credit"])
        nd += o["n_dropped"]
    assert dp["n_dropped"] == nd
    el = oracle.expert_loss(np.concatenate(idx), np.concatenate(slot), np.concatenate(credit),
                            inp["token_loss"], w.E)
    assert np.allclose(dp["expert_loss"], el, rtol=1e-12, atol=1e-12)
    assert nd > 0, "the shard capacity should drop some assignments in this case"


def test_allreduce_partials_without_group_is_identity():
    from sparse_mixture_experts_gate_b200.binding import allreduce_partials
    assert not dist.is_initialized()
    t = torch.arange(9, dtype=torch.float32)
    assert torch.equal(allreduce_partials(t.clone()), t)


def test_stats_from_partials_matches_unsharded_oracle_on_one_shard():
    import oracle
    from sparse_mixture_experts_gate_b200.workloads import make_inputs
    w = _workload()
    inp = make_inputs(w)
    p, o = shard_partials(w, inp, 0, w.T)
    dp = stats_from_partials(p, w.E, w.k, w.alpha, w.beta)
    assert np.allclose(dp["f"], o["f"], atol=1e-12) and np.allclose(dp["p_mean"], o["p_mean"], atol=1e-12)
    assert abs(dp["l_aux"] - o["l_aux"]) <= 1e-12 and abs(dp["l_z"] - o["l_z"]) <= 1e-12
    assert abs(dp["l_total"] - o["aux_loss"]) <= 1e-12
    assert np.allclose(dp["expert_loss"], o["expert_loss"], atol=1e-12)
    assert dp["n_dropped"] == o["n_dropped"]

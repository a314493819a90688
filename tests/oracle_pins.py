"""Pins that tie the CPU oracle to what the pages and the mathematics fix.

Each check_* function raises AssertionError when the oracle disagrees with a
value printed or implied by the pages, a closed form, an invariant, a library
routine for a special case, or brute force on tiny inputs. None of them re-types
the oracle's own formula. They run against whatever oracle library is loaded, so
the mutant test can point them at a deliberately broken build.

Sources:
  [C] "Appendix C - Acronyms & Symbols": "Core MoE symbols", "Balancing",
      "Capacity & communication", "Parameter accounting".
  [D] "Sparse MoE Expert-Credit Loss Reweighting Diagram", panel (b).
  [W] "Code Walkthrough - SER (Sparse Expert Routing)": "Configuration",
      "The gating / routing path", "Load balancing", "Minimal example".
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle
from sparse_mixture_experts_gate_b200.workloads import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sections(path):
    out, cur = {}, None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("["):
            cur = line.strip("[]")
            out[cur] = []
            continue
        out[cur].append([float(v) for v in line.split()])
    return {k: np.array(v) for k, v in out.items()}


def _kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        out[key] = [float(v) for v in vals]
    return out


# ------------------------------------------------------------------ capacity

def check_capacity_golden():
    """[C] "Capacity & communication": C = ceil(C_f k T / E), hand-worked table."""
    for line in open(os.path.join(GOLDEN, "capacity.txt")):
        if line.startswith("#") or not line.strip():
            continue
        cf, k, T, E, C = line.split()
        got = oracle.capacity(float(cf), int(k), int(T), int(E))
        assert got == int(C), (cf, k, T, E, C, got)


# ------------------------------------------------------------------ router

def check_hand_router():
    """[C] "Core MoE symbols": hand-worked h, P, top-k, gates, capacity, ranks."""
    g = _sections(os.path.join(GOLDEN, "hand_router.txt"))
    x = g["x"].astype(np.float32)
    wg = g["w_gate"].astype(np.float32)
    h = oracle.router_logits(x, wg)
    P, lse = oracle.softmax_lse(h)
    assert np.allclose(lse, g["lse"].ravel(), rtol=0, atol=1e-14), lse
    assert np.allclose(P[0], g["P0"].ravel(), rtol=0, atol=1e-10), P[0]
    idx = oracle.topk(h.astype(np.float32), 2)
    assert (idx == g["idx"].astype(np.int32)).all(), idx
    gt = oracle.gates(P, idx)
    assert np.allclose(gt, g["gates"], rtol=0, atol=1e-15), gt
    C = oracle.capacity(1.0, 2, 2, 3)
    slot, cpre, ckept, nd = oracle.dispatch(idx, 3, C)
    assert (slot == g["slot"].astype(np.int32)).all(), slot
    assert (cpre == g["count_pre"].ravel().astype(np.int32)).all(), cpre
    assert nd == 0


def check_logits_vs_matmul():
    """h = W_g x + b against numpy's fp64 matrix product (a library routine)."""
    rng = np.random.default_rng(7)
    for T, d, E in ((5, 3, 4), (17, 33, 9), (3, 64, 16)):
        x = rng.standard_normal((T, d)).astype(np.float32)
        wg = rng.standard_normal((E, d)).astype(np.float32)
        b = rng.standard_normal(E).astype(np.float32)
        h = oracle.router_logits(x, wg, b)
        ref = x.astype(np.float64) @ wg.astype(np.float64).T + b.astype(np.float64)
        assert np.allclose(h, ref, rtol=1e-13, atol=1e-13)
        # bf16 storage of x widens exactly: same logits as the fp32 copy of its values.
        xb = torch.from_numpy(x).to(torch.bfloat16)
        hb = oracle.router_logits(xb, wg, b)
        refb = xb.double().numpy() @ wg.astype(np.float64).T + b
        assert np.allclose(hb, refb, rtol=1e-13, atol=1e-13)


def check_softmax_lse():
    """P = softmax(h), lse = log sum e^h against scipy, plus closed forms."""
    from scipy.special import logsumexp, softmax, expit
    rng = np.random.default_rng(3)
    h = rng.standard_normal((11, 7)) * 5
    P, lse = oracle.softmax_lse(h)
    assert np.allclose(P, softmax(h, axis=1), rtol=1e-13, atol=1e-15)
    assert np.allclose(lse, logsumexp(h, axis=1), rtol=1e-14, atol=1e-14)
    assert np.allclose(P.sum(1), 1.0, rtol=0, atol=1e-12)
    # Two experts: P_0 = sigmoid(h_0 - h_1).
    h2 = rng.standard_normal((9, 2)) * 3
    P2, _ = oracle.softmax_lse(h2)
    assert np.allclose(P2[:, 0], expit(h2[:, 0] - h2[:, 1]), rtol=1e-13, atol=1e-15)
    # Large logits do not overflow: lse(h + c) = lse(h) + c, P unchanged.
    P3, lse3 = oracle.softmax_lse(h + 800.0)
    assert np.allclose(P3, P, rtol=1e-12, atol=1e-15)
    assert np.allclose(lse3, lse + 800.0, rtol=1e-14, atol=1e-10)
    # All-equal logits: P = 1/E exactly, lse = c + log E.
    for E in (1, 2, 4, 8, 64, 256):
        Pz, lz = oracle.softmax_lse(np.full((3, E), 0.25))
        assert (Pz == 1.0 / E).all()
        assert np.allclose(lz, 0.25 + math.log(E), rtol=1e-15, atol=1e-15)


# ------------------------------------------------------------------ selection

def check_selection_keys():
    """[W] noisy top-k and [C] selection bias b_i: one fp32 add (numpy float32)."""
    rng = np.random.default_rng(11)
    h = rng.standard_normal((6, 10)).astype(np.float32)
    n = (rng.standard_normal((6, 10)) / 10).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, 10).astype(np.float32)
    assert (oracle.selection_keys(h) == h).all()
    assert (oracle.selection_keys(h, noise=n) == (h + n)).all()
    assert (oracle.selection_keys(h, sel_bias=b) == (h + b[None, :])).all()
    # A selection bias equal for every expert selects the same experts as none.
    k0 = oracle.topk(oracle.selection_keys(h), 3)
    k1 = oracle.topk(oracle.selection_keys(h, sel_bias=np.full(10, 0.03125, np.float32)), 3)
    assert (k0 == k1).all()


def _brute_topk(keys, k):
    return [i for i, _ in sorted(enumerate(keys), key=lambda p: (-p[1], p[0]))[:k]]


def check_topk_bruteforce():
    """[C] T_k(x): full sort of (-key, index) on tiny inputs, every k, with ties."""
    rng = np.random.default_rng(5)
    for T, E in ((64, 1), (64, 2), (64, 5), (32, 16), (16, 13)):
        key = rng.standard_normal((T, E)).astype(np.float32)
        # Constructed exact ties: snap a third of the entries to a small grid.
        m = rng.random((T, E)) < 0.35
        key[m] = np.round(key[m] * 2) / 2
        for k in range(1, E + 1):
            idx = oracle.topk(key, k)
            for t in range(T):
                assert list(idx[t]) == _brute_topk(list(key[t]), k), (T, E, k, t)


def check_ties_golden():
    """Tie-break reading: lower expert index wins (hand-worked table)."""
    for line in open(os.path.join(GOLDEN, "ties.txt")):
        if line.startswith("#") or not line.strip():
            continue
        head, keys, want = line.split("|")
        E, k = map(int, head.split())
        key = np.array([keys.split()], dtype=np.float32)
        assert key.shape[1] == E
        got = oracle.topk(key, k)[0].tolist()
        assert got == [int(v) for v in want.split()], (line, got)


def check_gates():
    """[C] g_i: renormalised probabilities; sum to 1; k=1 gives 1; k=E gives P."""
    rng = np.random.default_rng(9)
    h = rng.standard_normal((20, 8)) * 2
    P, _ = oracle.softmax_lse(h)
    for k in range(1, 9):
        idx = oracle.topk(h.astype(np.float32), k)
        g = oracle.gates(P, idx)
        assert np.allclose(g.sum(1), 1.0, rtol=0, atol=1e-12)
        if k == 1:
            assert (g == 1.0).all()
        # Ratios of gates are ratios of probabilities.
        if k >= 2:
            ratio = g[:, 0] / g[:, 1]
            pr = P[np.arange(20), idx[:, 0]] / P[np.arange(20), idx[:, 1]]
            assert np.allclose(ratio, pr, rtol=1e-12)
    idx = oracle.topk(h.astype(np.float32), 8)
    g = oracle.gates(P, idx)
    assert np.allclose(g, np.take_along_axis(P, idx.astype(np.int64), 1), rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------------ dispatch

def _brute_dispatch(idx, E, C):
    queues = [[] for _ in range(E)]
    slot = np.full(idx.shape, -1, np.int32)
    for t in range(idx.shape[0]):
        for r in range(idx.shape[1]):
            q = queues[idx[t, r]]
            if len(q) < C:
                slot[t, r] = len(q)
            q.append(t)
    cpre = np.array([len(q) for q in queues], np.int32)
    return slot, cpre, np.minimum(cpre, C)


def check_dispatch_golden():
    """[C] capacity buffers and [W] hard cap with overflow drop: hand-worked case."""
    g = _kv(os.path.join(GOLDEN, "hand_dispatch.txt"))
    T, E, k = int(g["T"][0]), int(g["E"][0]), int(g["k"][0])
    C = oracle.capacity(g["capacity_factor"][0], k, T, E)
    assert C == int(g["C"][0])
    idx = np.array(g["idx"], np.int32).reshape(T, k)
    slot, cpre, ckept, nd = oracle.dispatch(idx, E, C)
    assert slot.ravel().tolist() == [int(v) for v in g["slot"]]
    assert cpre.tolist() == [int(v) for v in g["count_pre"]]
    assert ckept.tolist() == [int(v) for v in g["count_kept"]]
    assert nd == int(g["n_dropped"][0])


def check_dispatch_bruteforce():
    """Queue simulation on random tiny inputs; counts sum to kT - drops; a large
    C_f drops nothing; count_pre is numpy's bincount."""
    rng = np.random.default_rng(13)
    for T, E, k, cf in ((40, 4, 2, 1.0), (33, 8, 3, 1.25), (64, 16, 4, 0.5), (50, 5, 5, 1.0),
                        (20, 3, 1, 2.0), (64, 8, 2, 4.0)):
        key = rng.standard_normal((T, E)).astype(np.float32)
        key[:, 0] += 1.0  # skew toward expert 0 so that caps bind
        idx = oracle.topk(key, k)
        C = oracle.capacity(cf, k, T, E)
        slot, cpre, ckept, nd = oracle.dispatch(idx, E, C)
        bs, bc, bk = _brute_dispatch(idx, E, C)
        assert (slot == bs).all() and (cpre == bc).all() and (ckept == bk).all()
        assert (cpre == np.bincount(idx.ravel(), minlength=E)).all()
        assert int(ckept.sum()) == k * T - nd
        assert int((slot >= 0).sum()) == k * T - nd
        if cf >= E / k:
            assert nd == 0
    # Unlimited capacity never drops.
    idx = np.zeros((9, 1), np.int32)
    C = oracle.capacity(0.0, 1, 9, 4)
    _, _, _, nd = oracle.dispatch(idx, 4, C)
    assert nd == 0


# ------------------------------------------------------------------ experts

def _torch_ffn(x, w1, b1, w2, b2, act):
    f = {"relu": torch.nn.functional.relu,
         "gelu": lambda z: torch.nn.functional.gelu(z, approximate="none"),
         "swish": torch.nn.functional.silu}[act]
    z = torch.nn.functional.linear(x, w1, b1)
    return torch.nn.functional.linear(f(z), w2, b2)


def check_dense_ffn_reduction():
    """E=1, k=1, S=0 reduces the layer to one dense FFN; torch fp64
    linear -> activation -> linear is the reference for all three activations."""
    for act in ("relu", "gelu", "swish"):
        for dtype in ("fp32", "bf16"):
            w = WORKLOADS["tiny"].with_(T=7, d=24, F=40, O=16, E=1, k=1, S=0, activation=act,
                                        dtype=dtype, capacity_factor=0.0)
            inp = make_inputs(w, "cpu", seed=3, random_biases=True)
            out = oracle.forward(w, inp)
            assert (out["idx"] == 0).all() and (out["gates"] == 1.0).all()
            ref = _torch_ffn(inp["x"].double(), inp["w1"][0].double(), inp["b1"][0].double(),
                             inp["w2"][0].double(), inp["b2"][0].double(), act)
            assert np.allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-12), act
            # Credit with k=1, S=0: c = 1 * ||o||_2.
            assert np.allclose(out["credit"][:, 0], torch.linalg.vector_norm(ref, dim=1).numpy(),
                               rtol=1e-12, atol=1e-12)


def check_combine_against_torch():
    """[W] gate-weighted combine and [C] shared experts, rebuilt with torch fp64
    from the oracle's routing: y = sum_s FFN_s(x) + sum_kept g FFN_e(x)."""
    w = WORKLOADS["tiny"].with_(T=12, d=16, F=24, O=8, E=6, k=3, S=2, activation="swish",
                                dtype="bf16", capacity_factor=0.75)
    inp = make_inputs(w, "cpu", seed=5, random_biases=True)
    out = oracle.forward(w, inp)
    assert out["n_dropped"] > 0
    x = inp["x"].double()
    outs = [_torch_ffn(x, inp["w1"][e].double(), inp["b1"][e].double(), inp["w2"][e].double(),
                       inp["b2"][e].double(), w.activation) for e in range(w.E + w.S)]
    y = torch.zeros(w.T, w.O, dtype=torch.float64)
    for s in range(w.S):
        y += outs[w.E + s]
    for t in range(w.T):
        for r in range(w.k):
            if out["slot"][t, r] >= 0:
                y[t] += float(out["gates"][t, r]) * outs[int(out["idx"][t, r])][t]
    assert np.allclose(out["y"], y.numpy(), rtol=1e-12, atol=1e-12)


def check_shared_expert_linearity():
    """[C] "Parameter accounting": shared experts are always on, with weight 1, so
    adding one adds its dense FFN output to every token and changes nothing else."""
    w0 = WORKLOADS["tiny"].with_(T=9, d=16, F=20, O=12, E=4, k=2, S=1, activation="gelu",
                                 dtype="bf16", capacity_factor=1.0)
    inp = make_inputs(w0, "cpu", seed=8, random_biases=True)
    with_s = oracle.forward(w0, inp)
    w_no = w0.with_(S=0)
    inp_no = dict(inp)
    inp_no["w1"], inp_no["w2"] = inp["w1"][:4], inp["w2"][:4]
    inp_no["b1"], inp_no["b2"] = inp["b1"][:4], inp["b2"][:4]
    without = oracle.forward(w_no, inp_no)
    shared = _torch_ffn(inp["x"].double(), inp["w1"][4].double(), inp["b1"][4].double(),
                        inp["w2"][4].double(), inp["b2"][4].double(), "gelu").numpy()
    assert np.allclose(with_s["y"] - without["y"], shared, rtol=1e-10, atol=1e-12)
    assert (with_s["idx"] == without["idx"]).all()


# ------------------------------------------------------------------ statistics

def check_aux_uniform():
    """[C] "Balancing": f_i = P_i = 1/E gives L_aux = alpha E * E * (1/E^2) = alpha."""
    for E in (2, 4, 8, 64, 256):
        for k in (1, 2):
            T = 4 * E
            P = np.full((T, E), 1.0 / E)
            lse = np.zeros(T)
            cpre = np.full(E, k * T // E, np.int32)
            f, pm, la, lz = oracle.balance_stats(P, lse, cpre, k, 0.01, 1e-3)
            assert (f == 1.0 / E).all() and (pm == 1.0 / E).all()
            assert la == 0.01, la
            assert lz == 0.0


def check_aux_end_to_end():
    """k = E makes f_i = 1/E exactly and W_g = 0 makes P = 1/E exactly, so the whole
    layer gives L_aux = alpha and L_z = beta (log E)^2."""
    for E in (2, 4, 8):
        w = WORKLOADS["tiny"].with_(T=8, d=8, F=8, O=4, E=E, k=E, S=0, activation="relu",
                                    capacity_factor=0.0, alpha=0.01, beta=1e-3)
        inp = make_inputs(w, "cpu", seed=1)
        inp["w_gate"] = torch.zeros_like(inp["w_gate"])
        out = oracle.forward(w, inp)
        assert (out["P"] == 1.0 / E).all()
        assert (out["f"] == 1.0 / E).all()
        assert out["l_aux"] == 0.01, out["l_aux"]
        assert abs(out["l_z"] - 1e-3 * math.log(E) ** 2) <= 1e-18 + 1e-15 * out["l_z"]


def check_aux_skewed():
    """All tokens on expert 0 with P concentrated on it: f = e_0, P_0 = p, so
    L_aux = alpha E p (closed form); L_z is beta times the mean of squared lse."""
    E, T, k = 4, 6, 1
    p = 0.7
    P = np.tile(np.array([p] + [(1 - p) / 3] * 3), (T, 1))
    lse = np.arange(T, dtype=np.float64)
    cpre = np.array([T, 0, 0, 0], np.int32)
    f, pm, la, lz = oracle.balance_stats(P, lse, cpre, k, 0.5, 2.0)
    assert np.allclose(f, [1, 0, 0, 0])
    assert abs(la - 0.5 * E * p) < 1e-14
    assert abs(lz - 2.0 * (0 + 1 + 4 + 9 + 16 + 25) / 6) < 1e-13


def check_expert_loss():
    """[D] panel (b): with l = 1 and k = E every expert is selected by every token,
    so l_i is the mean over tokens of that expert's credit; dropped assignments add 0;
    a constant token loss c scales l_i by c."""
    rng = np.random.default_rng(2)
    T, E = 10, 4
    idx = np.array([rng.permutation(E) for _ in range(T)], np.int32)
    slot = np.zeros((T, E), np.int32)
    credit = rng.random((T, E))
    ones = np.ones(T, np.float32)
    el = oracle.expert_loss(idx, slot, credit, ones, E)
    want = np.zeros(E)
    for t in range(T):
        for r in range(E):
            want[idx[t, r]] += credit[t, r]
    assert np.allclose(el, want / T, rtol=1e-14)
    slot2 = slot.copy()
    slot2[0, :] = -1
    el2 = oracle.expert_loss(idx, slot2, credit, ones, E)
    assert np.allclose(el - el2, np.bincount(idx[0], weights=credit[0], minlength=E) / T, rtol=1e-12)
    el3 = oracle.expert_loss(idx, slot, credit, np.full(T, 2.5, np.float32), E)
    assert np.allclose(el3, 2.5 * el, rtol=1e-14)


def check_credit_is_gate_times_norm():
    """[D] panel (b): c = p ||h|| with p the applied gate and h the expert output;
    checked against torch fp64 FFNs on the oracle's routing."""
    w = WORKLOADS["tiny"].with_(T=10, d=16, F=16, O=8, E=5, k=2, S=1, activation="relu",
                                dtype="fp32", capacity_factor=0.8)
    inp = make_inputs(w, "cpu", seed=4, random_biases=True)
    out = oracle.forward(w, inp)
    x = inp["x"].double()
    for t in range(w.T):
        for r in range(w.k):
            e = int(out["idx"][t, r])
            o = _torch_ffn(x[t:t + 1], inp["w1"][e].double(), inp["b1"][e].double(),
                           inp["w2"][e].double(), inp["b2"][e].double(), "relu")[0]
            want = float(out["gates"][t, r]) * float(torch.linalg.vector_norm(o)) if out["slot"][t, r] >= 0 else 0.0
            assert abs(out["credit"][t, r] - want) <= 1e-12 * (1 + abs(want))


def check_cv_squared():
    """[W] "Load balancing" (coefficient-of-variation style balance): equal loads
    give 0; m equal non-zero loads out of n give n/m - 1; two loads a, b give
    ((a - b) / (a + b))^2; scaling every load leaves it unchanged."""
    assert oracle.cv_squared([7, 7, 7, 7, 7]) == 0.0
    for n, m in ((4, 1), (4, 2), (8, 3), (256, 8)):
        v = [5.0] * m + [0.0] * (n - m)
        assert abs(oracle.cv_squared(v) - (n / m - 1)) <= 1e-12 * (n / m)
    a, b = 3.0, 11.0
    assert abs(oracle.cv_squared([a, b]) - ((a - b) / (a + b)) ** 2) < 1e-15
    rng = np.random.default_rng(5)
    v = rng.random(13)
    assert abs(oracle.cv_squared(v) - oracle.cv_squared(4.0 * v)) < 1e-13
    assert oracle.cv_squared([0.0, 0.0, 0.0]) == 0.0


def check_aux_loss():
    """[W] "Load balancing": aux_loss = load_balance_coef * load_balance +
    z_loss_coef * z_loss, load_balance the coefficient-of-variation style loss of
    the selection counts. Closed forms: uniform routing (W_g = 0, k = E) leaves
    only beta (log E)^2; with z_loss_coef = 0, m equal non-zero loads of n give
    alpha (n/m - 1) and two loads a, b give alpha ((a - b) / (a + b))^2; a
    hand-worked log-partition vector; the value ignores the order of the experts."""
    w = WORKLOADS["tiny"].with_(T=12, d=8, F=8, O=8, E=4, k=4, S=0, dtype="fp32", capacity_factor=0.0)
    inp = make_inputs(w, "cpu", seed=3)
    inp["w_gate"] = torch.zeros_like(inp["w_gate"])
    inp["b_gate"] = None
    out = oracle.forward(w, inp)
    assert abs(oracle.aux_loss(out["count_pre"], out["lse"], 0.01, 1e-3) - 1e-3 * math.log(4) ** 2) <= 1e-15
    lse0 = np.zeros(5)
    for n, m in ((4, 1), (8, 3), (256, 8)):
        load = [9] * m + [0] * (n - m)
        assert abs(oracle.aux_loss(load, lse0, 0.25, 7.0) - 0.25 * (n / m - 1)) <= 1e-12 * (n / m)
    assert abs(oracle.aux_loss([3, 11], lse0, 0.5, 7.0) - 0.5 * (8 / 14) ** 2) <= 1e-15
    # lse = 1, 2, 3: mean square 14/3; equal loads: no balance term.
    assert abs(oracle.aux_loss([5, 5], [1.0, 2.0, 3.0], 0.5, 0.3) - 0.3 * 14 / 3) <= 1e-15
    rng = np.random.default_rng(12)
    load = rng.integers(0, 50, 16)
    lse = rng.normal(size=30)
    a = oracle.aux_loss(load, lse, 0.01, 1e-3)
    assert a == oracle.aux_loss(load[::-1].copy(), lse, 0.01, 1e-3)
    assert abs(oracle.aux_loss(load, lse, 0.01, 0.0) - 0.01 * oracle.cv_squared(load)) <= 1e-15


def check_importance():
    """[W] "Load balancing" (importance per expert): with k = 1 every gate is 1,
    so the importance is the selection count; the importances of a batch sum to
    T (each token's gates sum to 1); a hand-worked case."""
    rng = np.random.default_rng(6)
    T, E = 40, 6
    idx1 = rng.integers(0, E, size=(T, 1)).astype(np.int32)
    imp1 = oracle.importance(idx1, np.ones((T, 1)), E)
    assert np.array_equal(imp1, np.bincount(idx1[:, 0], minlength=E).astype(np.float64))
    idx = np.array([rng.permutation(E)[:3] for _ in range(T)], np.int32)
    g = rng.random((T, 3))
    g /= g.sum(1, keepdims=True)
    assert abs(oracle.importance(idx, g, E).sum() - T) < 1e-12
    hand = oracle.importance(np.array([[0, 1], [1, 2]]), np.array([[0.7, 0.3], [0.6, 0.4]]), 4)
    assert np.allclose(hand, [0.7, 0.9, 0.4, 0.0], atol=1e-15)


def check_selection_bias_update():
    """[C] "Balancing" (b_i, update rate gamma): experts above the mean load kT/E
    move down by gamma, those below move up, those at the mean stay; gamma = 0
    changes nothing; the result is the fp32 rounding of the exact sum."""
    # E=4, k=2, T=6: mean load 3.
    b = oracle.selection_bias_update([0.0, 0.0, 0.0, 0.0], [5, 3, 3, 1], 2, 6, 0.5)
    assert b.tolist() == [-0.5, 0.0, 0.0, 0.5]
    b0 = np.array([0.1, -0.2, 0.3, 0.05], np.float32)
    assert np.array_equal(oracle.selection_bias_update(b0, [9, 0, 1, 2], 3, 4, 0.0), b0)
    # Mean load 12 * 3 / 5 = 7.2 is not an integer: loads 7 and 8 straddle it.
    b1 = oracle.selection_bias_update(b0.tolist() + [0.0], [7, 8, 7, 8, 6], 3, 12, 1e-3)
    want = np.float32(np.array(b0.tolist() + [0.0], np.float64) + 1e-3 * np.array([1, -1, 1, -1, 1]))
    assert np.array_equal(b1, want.astype(np.float32))


def check_credit_hidden_dense():
    """[D] panel (b), hidden-activation reading: with E = 1, k = 1 the credit is
    g * ||act(w1 x + b1)||_2 of the one expert, checked against torch fp64 for
    every activation; a dropped assignment has credit 0."""
    for act in ("relu", "gelu", "swish"):
        w = WORKLOADS["tiny"].with_(T=6, d=12, F=20, O=8, E=1, k=1, S=0, activation=act, dtype="fp32")
        inp = make_inputs(w, "cpu", seed=8, random_biases=True)
        table = oracle.ExpertTable(1, inp["w1"], inp["b1"], inp["w2"], inp["b2"])
        idx = np.zeros((w.T, 1), np.int32)
        slot = np.zeros((w.T, 1), np.int32)
        slot[2, 0] = -1
        g = np.linspace(0.5, 1.0, w.T).reshape(w.T, 1)
        cr = oracle.experts_credit_hidden(range(w.T), inp["x"], table, idx, slot, g, w.d, w.F, w.E, act)
        x = inp["x"].double()
        z = x @ inp["w1"][0].double().T + inp["b1"][0].double()
        a = {"relu": torch.relu, "gelu": lambda v: torch.nn.functional.gelu(v), "swish": torch.nn.functional.silu}[act](z)
        want = g[:, 0] * torch.linalg.vector_norm(a, dim=1).numpy()
        want[2] = 0.0
        assert np.allclose(cr[:, 0], want, rtol=1e-12, atol=1e-14)


def check_dro_update():
    """[D] panel (c): ema = 0 tracks the loss, ema = 1 keeps the tracker; eta = 0
    with uniform weights keeps them uniform; two experts give the logistic
    closed form; the weights sum to 1 and the objective is sum mu_i l_i."""
    l = np.array([0.3, 1.2, 0.7, 0.1])
    lh0 = np.array([0.5, 0.5, 0.5, 0.5])
    lh, _, _ = oracle.dro_update(l, lh0, np.full(4, 0.25), 0.0, 1.0)
    assert np.allclose(lh, l, rtol=0, atol=0)
    lh, _, _ = oracle.dro_update(l, lh0, np.full(4, 0.25), 1.0, 1.0)
    assert np.array_equal(lh, lh0)
    _, mu, obj = oracle.dro_update(l, lh0, np.full(4, 0.25), 0.9, 0.0)
    assert np.allclose(mu, 0.25, rtol=0, atol=1e-15) and abs(obj - l.mean()) < 1e-15
    l2, lh2, mu2, ema, eta = np.array([2.0, 0.5]), np.array([1.0, 3.0]), np.array([0.4, 0.6]), 0.8, 1.7
    lh_new = ema * lh2 + (1 - ema) * l2
    p0 = 1.0 / (1.0 + math.exp(-((mu2[0] + eta * lh_new[0]) - (mu2[1] + eta * lh_new[1]))))
    lh_o, mu_o, obj = oracle.dro_update(l2, lh2, mu2, ema, eta)
    assert abs(mu_o[0] - p0) < 1e-14 and abs(mu_o.sum() - 1.0) < 1e-15
    assert abs(obj - (mu_o[0] * l2[0] + mu_o[1] * l2[1])) < 1e-15


def check_dispatch_rank_major():
    """GShard-style priority (capacity_priority = rank): a hand-worked case where
    it differs from token order; k = 1 makes the two orders equal; a queue
    simulation over (choice, token) order; per-expert counts and the number of
    drops do not depend on the order."""
    # T=3, k=2, E=2, C=2. Rank-major: choice 0: t0->e0 (rank 0), t1->e1 (0),
    # t2->e0 (1); choice 1: t0->e1 (1), t1->e0 (2: dropped), t2->e1 (2: dropped).
    # Token order instead: e0 sees t0, t1, t2 and e1 sees t0, t1, t2, so both of
    # t2's choices drop.
    idx = np.array([[0, 1], [1, 0], [0, 1]], np.int32)
    slot, cpre, ckept, nd = oracle.dispatch(idx, 2, 2, "rank")
    assert slot.tolist() == [[0, 1], [0, -1], [1, -1]] and nd == 2
    slot_t, _, _, nd_t = oracle.dispatch(idx, 2, 2, "token")
    assert slot_t.tolist() == [[0, 0], [1, 1], [-1, -1]] and nd_t == 2
    rng = np.random.default_rng(12)
    T, E = 50, 7
    idx1 = rng.integers(0, E, size=(T, 1)).astype(np.int32)
    assert np.array_equal(oracle.dispatch(idx1, E, 5, "rank")[0], oracle.dispatch(idx1, E, 5, "token")[0])
    k, C = 3, 12
    idx3 = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32)
    slot, cpre, ckept, nd = oracle.dispatch(idx3, E, C, "rank")
    fill = [0] * E
    want = np.empty((T, k), np.int32)
    for r in range(k):
        for t in range(T):
            e = idx3[t, r]
            want[t, r] = fill[e] if fill[e] < C else -1
            fill[e] += 1
    assert np.array_equal(slot, want)
    _, cpre_t, ckept_t, nd_t = oracle.dispatch(idx3, E, C, "token")
    assert np.array_equal(cpre, cpre_t) and np.array_equal(ckept, ckept_t) and nd == nd_t


def check_router_mlp():
    """[W] optional MLP gate: h = W_2 relu(W_1 x + b_1) + b_2 against numpy fp64;
    a hand-worked two-unit case (one hidden unit clipped by the ReLU)."""
    rng = np.random.default_rng(13)
    T, d, H, E = 9, 12, 7, 5
    x = rng.standard_normal((T, d)).astype(np.float32)
    w1 = rng.standard_normal((H, d)).astype(np.float32)
    b1 = rng.standard_normal(H).astype(np.float32)
    w2 = rng.standard_normal((E, H)).astype(np.float32)
    b2 = rng.standard_normal(E).astype(np.float32)
    h = oracle.router_mlp(x, w1, b1, w2, b2)
    z = np.maximum(x.astype(np.float64) @ w1.astype(np.float64).T + b1, 0.0)
    assert np.allclose(h, z @ w2.astype(np.float64).T + b2, rtol=1e-13, atol=1e-13)
    # x = (1, 2); unit 0 = x0 + x1 = 3, unit 1 = x0 - x1 - 1 = -2 -> 0;
    # h0 = 2*3 + 5*0 + 0.5 = 6.5, h1 = -1*3 + 1*0 = -3.
    hx = oracle.router_mlp(np.array([[1.0, 2.0]], np.float32), np.array([[1, 1], [1, -1]], np.float32),
                           np.array([0, -1], np.float32), np.array([[2, 5], [-1, 1]], np.float32),
                           np.array([0.5, 0.0], np.float32))
    assert hx.tolist() == [[6.5, -3.0]]


def check_minimal_example_shapes():
    """[W] "Minimal example": 4 experts, 2 active, dims 8/16/8, a (4, 8) input;
    the forward yields a (4, 8) output, 2 distinct experts per token, gates
    summing to 1 and, with no capacity limit, nothing dropped."""
    w = WORKLOADS["tiny"]
    assert (w.E, w.k, w.d, w.F, w.O, w.T, w.seed) == (4, 2, 8, 16, 8, 4, 42)
    inp = make_inputs(w, "cpu")
    out = oracle.forward(w, inp)
    assert out["y"].shape == (4, 8)
    assert all(len(set(r)) == 2 for r in out["idx"].tolist())
    assert np.allclose(out["gates"].sum(1), 1.0, atol=1e-12)
    assert out["n_dropped"] == 0


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]

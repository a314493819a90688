"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs.

Tolerances (bf16 operands with fp32 accumulation, fp32 routing and statistics):
  * routing indices, slots, drop flags, per-expert counts: bit-exact when the
    oracle routes from the GPU's own fp32 logits (same-logits mode);
  * logits vs the oracle's fp64 logits: 1e-4 absolute; in end-to-end index
    comparisons, tokens whose k-th vs (k+1)-th key margin is < 1e-5 are counted
    and excluded;
  * y: |gpu - oracle| <= 2e-2 (1 + |oracle|) per element for bf16 storage and
    1e-4 (1 + |oracle|) for fp32, with the oracle's expert and combine steps run
    on the GPU's routing so that one near-tie cannot cascade;
  * gates, P_i, f_i, L_aux, L_z (fp32 router arithmetic): 1e-4 absolute;
  * credit c = g ||o||: 2e-3 (1 + |c|) for bf16 layers, 1e-4 (1 + |c|) for fp32.
    The expert output o is a bf16-operand product: the hidden activations are
    stored in bf16 between the two expert GEMMs (unit roundoff 2^-9 ~ 1.95e-3),
    and that rounding, not the fp32 accumulation, sets the error of ||o||; a
    CPU recomputation with the hidden vector rounded to bf16 matches the GPU
    credit to ~1e-5 relative. 2e-3 is that unit roundoff, ten times tighter than
    the 2e-2 (1 + |y|) bound on the bf16-operand outputs themselves;
  * expert-attributed loss: reduced from the GPU's own credit, 1e-4 (1 + |value|);
    against the oracle's own l_i (from the oracle's credit on the same routing),
    the credit bound carried through the sum (check_expert_loss_vs_oracle).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_mixture_experts_gate_b200.binding import MoELayer

Y_TOL = {"bf16": 2e-2, "fp32": 1e-4}
CREDIT_TOL = {"bf16": 2e-3, "fp32": 1e-4}
STAT_TOL = 1e-4
LOGIT_TOL = 1e-4
TIE_MARGIN = 1e-5


def run_gpu(w, inp, layer: MoELayer = None, poison: bool = True):
    """One forward + aux stats through the C ABI; returns numpy copies."""
    dev = "cuda"
    if layer is None:
        layer = MoELayer(w, inp)
    x = inp["x"].to(dev).contiguous()
    noise = inp["noise"].to(dev).contiguous() if inp.get("noise") is not None else None
    tl = inp["token_loss"].to(dev).contiguous() if inp.get("token_loss") is not None else None
    T = x.shape[0]
    ws, _ = layer.workspace(T)
    if poison:
        ws.fill_(0xFF)  # NaN bit patterns: any read of an unwritten scratch word shows up
    out = layer.alloc_outputs(T)
    for v in out.values():
        if v.dtype.is_floating_point:
            v.fill_(float("nan"))
        else:
            v.fill_(-7)
    layer.forward(x, noise=noise, out=out)
    layer.aux_stats(out, token_loss=tl)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    res = {}
    for k, v in out.items():
        res[k] = v.float().cpu().numpy().astype(np.float64) if v.is_floating_point() else v.cpu().numpy()
    res["launches"] = layer.launch_count()
    return res, layer


def expert_table(w, inp, experts=None):
    """Oracle expert table; `experts` limits which experts are copied to the host."""
    G = w.E + w.S
    if experts is None:
        return oracle.ExpertTable(G, inp["w1"], inp["b1"], inp["w2"], inp["b2"])
    sel = sorted(set(int(e) for e in experts) | set(range(w.E, G)))
    return oracle.ExpertTable(G, {e: inp["w1"][e].cpu() for e in sel}, {e: inp["b1"][e].cpu() for e in sel},
                              {e: inp["w2"][e].cpu() for e in sel}, {e: inp["b2"][e].cpu() for e in sel})


def check_same_logits_routing(w, inp, g):
    """Bit-exact integer routing when the oracle consumes the GPU's fp32 logits."""
    noise = inp.get("noise") if w.top_k_method == "noisy" else None
    sb = inp.get("sel_bias") if w.use_selection_bias else None
    r = oracle.routing_from_logits(g["logits"].astype(np.float32), w, noise=noise, sel_bias=sb)
    assert np.array_equal(g["topk_idx"], r["idx"]), "top-k indices differ (same logits)"
    assert np.array_equal(g["slot"], r["slot"]), "slots / drop flags differ (same logits)"
    assert np.array_equal(g["count_pre"], r["count_pre"])
    assert np.array_equal(g["count_kept"], r["count_kept"])
    assert int(g["n_dropped"][0]) == r["n_dropped"]
    assert np.abs(g["gates"] - r["gates"]).max() <= STAT_TOL
    # Statistics that depend only on logits and counts, from the same logits.
    f, pm, la, lz = oracle.balance_stats(r["P"], r["lse"], r["count_pre"], w.k, w.alpha, w.beta)
    assert np.abs(g["f"] - f).max() <= STAT_TOL
    bad = np.flatnonzero(~(np.abs(g["p_mean"] - pm) <= STAT_TOL))
    assert bad.size == 0, f"p_mean differs at {bad[:8]}: gpu {g['p_mean'][bad[:4]]} oracle {pm[bad[:4]]}"
    assert abs(g["l_aux"][0] - la) <= STAT_TOL, (g["l_aux"][0], la)
    assert abs(g["l_z"][0] - lz) <= STAT_TOL, (g["l_z"][0], lz)
    # Load-balancing extras: importance from the GPU's own gates (fp32 sums of
    # fp32 gates), the CVs of counts and importances, the weighted aux loss.
    imp = oracle.importance(g["topk_idx"], g["gates"], w.E)
    assert np.abs(g["importance"] - imp).max() <= STAT_TOL * (1 + np.abs(imp).max()), "importance"
    cvl = oracle.cv_squared(r["count_pre"])
    assert abs(g["cv_load"][0] - cvl) <= STAT_TOL * (1 + cvl), "cv of the loads"
    cvi = oracle.cv_squared(imp)
    assert abs(g["cv_importance"][0] - cvi) <= STAT_TOL * (1 + cvi), "cv of the importances"
    lt = oracle.aux_loss(r["count_pre"], r["lse"], w.alpha, w.beta)
    assert abs(g["l_total"][0] - lt) <= STAT_TOL * (1 + abs(lt)), "weighted aux loss"
    return r


def near_tie_tokens(key: np.ndarray, k: int) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest keys are closer than TIE_MARGIN
    (or any two of the top k+1, which could reorder the listed indices)."""
    s = -np.sort(-key.astype(np.float64), axis=1)
    upto = min(k + 1, key.shape[1])
    gaps = s[:, :upto - 1] - s[:, 1:upto]
    if gaps.shape[1] == 0:
        return np.zeros(key.shape[0], bool)
    return (gaps < TIE_MARGIN).any(axis=1)


def check_end_to_end(w, inp, g, tokens=None, table=None):
    """GPU logits vs oracle fp64 logits, top-k away from near ties, and y /
    credit from the oracle's expert and combine steps on the GPU's routing."""
    T = inp["x"].shape[0]
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    x_rows = inp["x"][torch.as_tensor(toks)].cpu()
    bg = inp["b_gate"].cpu() if inp.get("b_gate") is not None else None
    if w.mlp_gater:
        g1 = inp["gater_b1"].cpu() if inp.get("gater_b1") is not None else None
        h = oracle.router_mlp(x_rows, inp["gater_w1"].cpu(), g1, inp["w_gate"].cpu(), bg)
    else:
        h = oracle.router_logits(x_rows, inp["w_gate"].cpu(), bg)
    logit_err = float(np.abs(g["logits"][toks] - h).max())
    assert logit_err <= LOGIT_TOL, logit_err
    noise = inp["noise"].cpu()[torch.as_tensor(toks)] if (w.top_k_method == "noisy") else None
    sb = inp.get("sel_bias").cpu() if w.use_selection_bias else None
    key = oracle.selection_keys(h.astype(np.float32), noise, sb)
    idx = oracle.topk(key, w.k)
    ties = near_tie_tokens(key, w.k)
    ok = ~ties
    assert np.array_equal(g["topk_idx"][toks][ok], idx[ok]), "end-to-end top-k differs away from near ties"
    # y and credit on the GPU's routing.
    if table is None:
        table = expert_table(w, inp)
    y, credit = oracle.experts_combine(toks, inp["x"].cpu(), table, g["topk_idx"], g["slot"], g["gates"],
                                       w.d, w.F, w.O, w.E, w.S, w.activation)
    tol = Y_TOL[w.dtype]
    err = np.abs(g["y"][toks] - y) / (1.0 + np.abs(y))
    assert err.max() <= tol, f"y: max scaled error {err.max():.3e} > {tol}"
    if w.credit_norm == "hidden":  # norm of act(w1 x + b1) instead of the output
        credit = oracle.experts_credit_hidden(toks, inp["x"].cpu(), table, g["topk_idx"], g["slot"], g["gates"],
                                              w.d, w.F, w.E, w.activation)
    cerr = np.abs(g["credit"][toks] - credit) / (1.0 + np.abs(credit))
    assert cerr.max() <= CREDIT_TOL[w.dtype], f"credit: max scaled error {cerr.max():.3e}"
    info = dict(n_near_ties=int(ties.sum()), y_err=float(err.max()), credit_err=float(cerr.max()), logit_err=logit_err)
    if tokens is None and inp.get("token_loss") is not None:
        info["expert_loss_err"] = check_expert_loss_vs_oracle(w, inp, g, credit)
    return info


def check_expert_loss_vs_oracle(w, inp, g, credit_oracle):
    """The GPU's expert-attributed loss against the oracle's own l_i, built from
    the oracle's credit on the same routing. The bound follows from the credit
    bound: l_i = (1/T) sum c l_t over i's kept assignments, so each credit's
    error CREDIT_TOL (1 + |c|) enters weighted by its token loss; the fp32 sum
    itself adds STAT_TOL (1 + |l_i|)."""
    tl = inp["token_loss"].cpu().double().numpy()
    T = tl.shape[0]
    el = oracle.expert_loss(g["topk_idx"], g["slot"], credit_oracle, inp["token_loss"].cpu(), w.E)
    kept = g["slot"] >= 0
    per = np.where(kept, CREDIT_TOL[w.dtype] * (1.0 + np.abs(credit_oracle)) * tl[:, None], 0.0)
    bound = np.bincount(g["topk_idx"][kept], weights=per[kept], minlength=w.E) / T + STAT_TOL * (1 + np.abs(el))
    diff = np.abs(g["expert_loss"] - el)
    assert (diff <= bound).all(), f"expert loss: max error {diff.max():.3e}, worst margin {(diff - bound).max():.3e}"
    return float((diff / bound).max())


def check_expert_loss(w, inp, g):
    """Attributed loss from the GPU's routing and credit, reduced by the oracle."""
    el = oracle.expert_loss(g["topk_idx"], g["slot"], g["credit"], inp["token_loss"].cpu(), w.E)
    err = np.abs(g["expert_loss"] - el) / (1.0 + np.abs(el))
    assert err.max() <= STAT_TOL, err.max()


def stratified_tokens(g, w, tile_rows: int, min_tokens: int = 0, seed: int = 1234, candidates: int = 32):
    """A sample of tokens that together reach every unit of work the expert
    GEMMs hand out: for every routed expert, a token in each of its token tiles
    (slots [j tile_rows, (j + 1) tile_rows) of its segment) and the token in its
    last kept slot; for every shared expert, a token in each tile of the token
    axis; and the batch's last token. A token covers its k experts' tiles at
    once, so the items are covered greedily (for each uncovered item, the
    candidate token that covers most uncovered items), then random tokens are
    added up to `min_tokens`. Every output column of a sampled token is compared,
    so every feature tile of both GEMMs is reached for each of those tiles."""
    rng = np.random.default_rng(seed)
    idx, slot = g["topk_idx"], g["slot"]
    T, k = idx.shape
    kept = g["count_kept"].astype(np.int64)
    n_tiles = (kept + tile_rows - 1) // tile_rows
    base = np.concatenate([[0], np.cumsum(n_tiles)])
    n_routed = int(base[-1])
    n_last = int((kept > 0).sum())
    last_id = np.full(w.E, -1, np.int64)
    last_id[kept > 0] = n_routed + np.arange(n_last)
    n_shared_tiles = (T + tile_rows - 1) // tile_rows if w.S > 0 else 0
    cover = [set() for _ in range(T)]
    holders = {}
    for t in range(T):
        for r in range(k):
            s_ = int(slot[t, r])
            if s_ < 0:
                continue
            e = int(idx[t, r])
            items = [int(base[e] + s_ // tile_rows)]
            if s_ == kept[e] - 1:
                items.append(int(last_id[e]))
            for it in items:
                cover[t].add(it)
                holders.setdefault(it, []).append(t)
        if n_shared_tiles:
            it = n_routed + n_last + t // tile_rows
            cover[t].add(it)
            holders.setdefault(it, []).append(t)
    uncovered = set(holders)
    chosen = {T - 1}
    uncovered -= cover[T - 1]
    for it in sorted(holders):
        if it not in uncovered:
            continue
        hs = holders[it]
        cands = hs if len(hs) <= candidates else [hs[i] for i in rng.choice(len(hs), candidates, replace=False)]
        best = max(cands, key=lambda t: len(cover[t] & uncovered))
        chosen.add(best)
        uncovered -= cover[best]
    assert not uncovered
    n_items = n_routed + n_last + n_shared_tiles
    if len(chosen) < min_tokens:
        rest = np.setdiff1d(np.arange(T), np.fromiter(chosen, np.int64))
        chosen.update(rng.choice(rest, min(len(rest), min_tokens - len(chosen)), replace=False).tolist())
    return np.array(sorted(chosen), np.int64), n_items

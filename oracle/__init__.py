"""CPU oracle for the sparse top-k MoE layer forward (test infrastructure).

A ctypes front end over liboracle.so, built from moe_oracle.c with gcc. Only the
tests, the smoke check and the benchmark's CPU-baseline leg import this package;
the CUDA path never does, and this package imports nothing from it.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_DIR, "moe_oracle.c")
_HDR = os.path.join(_DIR, "moe_oracle.h")
LIB_PATH = os.path.join(_DIR, "liboracle.so")

ACT = {"relu": 0, "gelu": 1, "swish": 2}
BF16, F32 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so (plain C99, fp64, no fast-math, OpenMP over tokens)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= newest:
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


class Expert(ctypes.Structure):
    _fields_ = [("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p)]


def _configure(L):
    i32, i64, dbl, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    L.orc_load.argtypes = [vp, i64, i32]
    L.orc_load.restype = dbl
    L.orc_router_logits.argtypes = [i32, i32, i32, vp, i32, vp, vp, vp]
    L.orc_softmax_lse.argtypes = [i32, i32, vp, vp, vp]
    L.orc_selection_keys.argtypes = [i32, i32, vp, vp, vp, vp]
    L.orc_topk.argtypes = [i32, i32, i32, vp, vp]
    L.orc_gates.argtypes = [i32, i32, i32, vp, vp, vp]
    L.orc_capacity.argtypes = [dbl, i32, i32, i32]
    L.orc_capacity.restype = i64
    L.orc_dispatch.argtypes = [i32, i32, i32, i64, vp, vp, vp, vp, vp]
    L.orc_expert_ffn.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(Expert), vp, vp]
    L.orc_experts_combine.argtypes = [i32, vp, i32, i32, i32, i32, i32, i32, i32, i32, i32,
                                      i32, vp, ctypes.POINTER(Expert), vp, vp, vp, vp, vp]
    L.orc_balance_stats.argtypes = [i32, i32, i32, vp, vp, vp, dbl, dbl, vp, vp, vp, vp]
    L.orc_expert_loss.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp]
    L.orc_importance.argtypes = [i32, i32, i32, vp, vp, vp]
    L.orc_dispatch_rank_major.argtypes = [i32, i32, i32, i64, vp, vp, vp, vp, vp]
    L.orc_router_mlp.argtypes = [i32, i32, i32, i32, vp, i32, vp, vp, vp, vp, vp]
    L.orc_experts_credit_hidden.argtypes = [i32, vp, i32, i32, i32, i32, i32, i32, i32, vp,
                                            ctypes.POINTER(Expert), vp, vp, vp, vp]
    L.orc_dro_update.argtypes = [i32, dbl, dbl, vp, vp, vp]
    L.orc_dro_update.restype = dbl
    L.orc_cv_squared.argtypes = [i32, vp]
    L.orc_cv_squared.restype = dbl
    L.orc_aux_loss.argtypes = [i32, i32, vp, vp, dbl, dbl]
    L.orc_aux_loss.restype = dbl
    L.orc_selection_bias_update.argtypes = [i32, i32, i64, vp, ctypes.c_float, vp]
    L.orc_max_threads.restype = i32
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(LIB_PATH))
    return _lib


@contextlib.contextmanager
def using_library(path: str):
    """Run the wrappers against another build of moe_oracle.c (the mutant test
    uses this to check that the pins catch planted mistakes)."""
    global _lib
    old = _lib
    _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = old


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def as_storage(t) -> tuple:
    """torch tensor or numpy array -> (contiguous numpy storage, oracle dtype code).
    bf16 tensors become their raw uint16 bit patterns."""
    import torch
    if isinstance(t, torch.Tensor):
        t = t.detach().contiguous().cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), BF16
        return np.ascontiguousarray(t.float().numpy()), F32
    a = np.ascontiguousarray(t)
    if a.dtype == np.uint16:
        return a, BF16
    return np.ascontiguousarray(a, dtype=np.float32), F32


def _f32(t) -> Optional[np.ndarray]:
    if t is None:
        return None
    import torch
    if isinstance(t, torch.Tensor):
        return np.ascontiguousarray(t.detach().cpu().float().numpy())
    return np.ascontiguousarray(t, dtype=np.float32)


def max_threads() -> int:
    return lib().orc_max_threads()


# ---------------------------------------------------------------- single steps

def router_logits(x, w_gate, b_gate=None) -> np.ndarray:
    xs, xd = as_storage(x)
    wg = _f32(w_gate)
    T, d = xs.shape
    E = wg.shape[0]
    h = np.empty((T, E), np.float64)
    lib().orc_router_logits(T, d, E, _p(xs), xd, _p(wg), _p(_f32(b_gate)), _p(h))
    return h


def softmax_lse(h: np.ndarray):
    h = np.ascontiguousarray(h, dtype=np.float64)
    T, E = h.shape
    P = np.empty_like(h)
    lse = np.empty(T, np.float64)
    lib().orc_softmax_lse(T, E, _p(h), _p(P), _p(lse))
    return P, lse


def selection_keys(h32, noise=None, sel_bias=None) -> np.ndarray:
    h32 = _f32(h32)
    T, E = h32.shape
    key = np.empty_like(h32)
    lib().orc_selection_keys(T, E, _p(h32), _p(_f32(noise)), _p(_f32(sel_bias)), _p(key))
    return key


def topk(key, k: int) -> np.ndarray:
    key = _f32(key)
    T, E = key.shape
    idx = np.empty((T, k), np.int32)
    lib().orc_topk(T, E, k, _p(key), _p(idx))
    return idx


def gates(P: np.ndarray, idx: np.ndarray) -> np.ndarray:
    P = np.ascontiguousarray(P, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, E = P.shape
    k = idx.shape[1]
    g = np.empty((T, k), np.float64)
    lib().orc_gates(T, E, k, _p(P), _p(idx), _p(g))
    return g


def capacity(capacity_factor: float, k: int, T: int, E: int) -> int:
    return int(lib().orc_capacity(float(capacity_factor), k, T, E))


def dispatch(idx: np.ndarray, E: int, C: int, priority: str = "token"):
    """Capacity-capped ranks; priority "token" (ascending token index) or "rank"
    (first choices of all tokens, then second choices, ...)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    slot = np.empty((T, k), np.int32)
    cpre = np.empty(E, np.int32)
    ckept = np.empty(E, np.int32)
    nd = np.zeros(1, np.int32)
    fn = lib().orc_dispatch if priority == "token" else lib().orc_dispatch_rank_major
    fn(T, E, k, int(C), _p(idx), _p(slot), _p(cpre), _p(ckept), _p(nd))
    return slot, cpre, ckept, int(nd[0])


def router_mlp(x, w1, b1, w2, b2) -> np.ndarray:
    """MLP gate logits h = W_2 relu(W_1 x + b_1) + b_2 in double."""
    xs, xd = as_storage(x)
    T, d = xs.shape
    w1 = _f32(w1)
    w2 = _f32(w2)
    H, E = w1.shape[0], w2.shape[0]
    b1 = _f32(b1) if b1 is not None else None
    b2 = _f32(b2) if b2 is not None else None
    h = np.empty((T, E), np.float64)
    lib().orc_router_mlp(T, d, H, E, _p(xs), xd, _p(w1), _p(b1) if b1 is not None else None, _p(w2),
                         _p(b2) if b2 is not None else None, _p(h))
    return h


class ExpertTable:
    """Per-expert weight pointers for the oracle. `w1`, `w2` are stacks
    [G][F][d] / [G][O][F] (torch or numpy; bf16 or fp32), or dicts {e: array}
    holding only the experts a check needs."""

    def __init__(self, G: int, w1, b1, w2, b2):
        self.G = G
        self._keep = []
        self.arr = (Expert * G)()
        self.w_dtype = None
        for e in range(G):
            parts = []
            for src, is_w in ((w1, True), (b1, False), (w2, True), (b2, False)):
                if src is None:
                    parts.append(None)
                    continue
                if isinstance(src, dict):
                    if e not in src:
                        parts.append(None)
                        continue
                    a = src[e]
                else:
                    a = src[e]
                if is_w:
                    s, dt = as_storage(a)
                    if self.w_dtype is None:
                        self.w_dtype = dt
                    assert dt == self.w_dtype
                else:
                    s = _f32(a)
                self._keep.append(s)
                parts.append(_p(s))
            self.arr[e] = Expert(*parts)


def expert_ffn(x_row: np.ndarray, table: ExpertTable, e: int, d: int, F: int, O: int, act: str) -> np.ndarray:
    x_row = np.ascontiguousarray(x_row, dtype=np.float64)
    o = np.empty(O, np.float64)
    lib().orc_expert_ffn(d, F, O, ACT[act], table.w_dtype, ctypes.byref(table.arr[e]), _p(x_row), _p(o))
    return o


def experts_combine(tokens: Sequence[int], x, table: ExpertTable, idx, slot, g,
                    d: int, F: int, O: int, E: int, S: int, act: str, want_credit: bool = True):
    xs, xd = as_storage(x)
    T = xs.shape[0]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    g = np.ascontiguousarray(g, dtype=np.float64)
    k = idx.shape[1]
    tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
    n = tok.shape[0]
    y = np.empty((n, O), np.float64)
    cr = np.empty((n, k), np.float64) if want_credit else None
    lib().orc_experts_combine(n, _p(tok), T, d, F, O, E, S, k, ACT[act], xd, table.w_dtype,
                              _p(xs), table.arr, _p(idx), _p(slot), _p(g), _p(y), _p(cr))
    return y, cr


def experts_credit_hidden(tokens: Sequence[int], x, table: ExpertTable, idx, slot, g, d: int, F: int, E: int,
                          act: str) -> np.ndarray:
    """Credit g * ||act(w1 x + b1)|| of each kept assignment (the hidden-activation reading)."""
    xs, xd = as_storage(x)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    g = np.ascontiguousarray(g, dtype=np.float64)
    k = idx.shape[1]
    tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
    cr = np.empty((tok.shape[0], k), np.float64)
    lib().orc_experts_credit_hidden(tok.shape[0], _p(tok), d, F, E, k, ACT[act], xd, table.w_dtype, _p(xs),
                                    table.arr, _p(idx), _p(slot), _p(g), _p(cr))
    return cr


def dro_update(l, lhat, mu, ema: float, eta: float):
    """EMA of the expert losses, mu <- softmax(mu + eta lhat), and sum_i mu_i l_i."""
    l = np.ascontiguousarray(l, dtype=np.float64)
    lh = np.ascontiguousarray(np.array(lhat, dtype=np.float64).copy())
    m = np.ascontiguousarray(np.array(mu, dtype=np.float64).copy())
    obj = lib().orc_dro_update(int(l.size), float(ema), float(eta), _p(l), _p(lh), _p(m))
    return lh, m, float(obj)


def balance_stats(P, lse, count_pre, k: int, alpha: float, beta: float):
    P = np.ascontiguousarray(P, dtype=np.float64)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    cpre = np.ascontiguousarray(count_pre, dtype=np.int32)
    T, E = P.shape
    f = np.empty(E, np.float64)
    pm = np.empty(E, np.float64)
    la = np.zeros(1, np.float64)
    lz = np.zeros(1, np.float64)
    lib().orc_balance_stats(T, E, k, _p(P), _p(lse), _p(cpre), float(alpha), float(beta),
                            _p(f), _p(pm), _p(la), _p(lz))
    return f, pm, float(la[0]), float(lz[0])


def expert_loss(idx, slot, credit, token_loss, E: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    credit = np.ascontiguousarray(credit, dtype=np.float64)
    tl = _f32(token_loss)
    T, k = idx.shape
    out = np.empty(E, np.float64)
    lib().orc_expert_loss(T, E, k, _p(idx), _p(slot), _p(credit), _p(tl), _p(out))
    return out


def importance(idx, g, E: int) -> np.ndarray:
    """Sum of the routed gate weights per expert ("Load balancing")."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    g = np.ascontiguousarray(g, dtype=np.float64)
    T, k = idx.shape
    out = np.empty(E, np.float64)
    lib().orc_importance(T, E, k, _p(idx), _p(g), _p(out))
    return out


def cv_squared(v) -> float:
    """Squared coefficient of variation, population variance ("Load balancing")."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    return float(lib().orc_cv_squared(int(v.size), _p(v)))


def aux_loss(count_pre, lse, load_balance_coef: float, z_loss_coef: float) -> float:
    """The walkthrough's aux_loss ("Load balancing"): load_balance_coef times the
    coefficient-of-variation style balance loss of the selection counts, plus
    z_loss_coef times the mean squared log-partition."""
    cpre = np.ascontiguousarray(count_pre, dtype=np.int32)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    return float(lib().orc_aux_loss(int(lse.size), int(cpre.size), _p(cpre), _p(lse), float(load_balance_coef),
                                    float(z_loss_coef)))


def selection_bias_update(b, load, k: int, T: int, gamma: float) -> np.ndarray:
    """b_i + gamma sign(kT/E - load_i), rounded to fp32 ("Balancing")."""
    out = np.ascontiguousarray(np.array(b, dtype=np.float32).copy())
    ld = np.ascontiguousarray(np.asarray(load, dtype=np.int64))
    lib().orc_selection_bias_update(int(out.size), int(k), int(T), _p(ld), float(gamma), _p(out))
    return out


# ---------------------------------------------------------------- whole layer

def layer_capacity_factor(w) -> float:
    """The capacity factor as a layer holds it: the configuration stores C_f in
    fp32, so C = ceil(C_f k T / E) is formed (in double) from fl32(C_f). For C_f
    = 0.6, for instance, fl32(0.6) k T / E can exceed an integer that 0.6 k T / E
    equals exactly."""
    return float(np.float32(w.capacity_factor))


def routing_from_logits(h32, w, noise=None, sel_bias=None) -> Dict[str, object]:
    """Selection, top-k and dispatch from given fp32 logits (the integer
    decisions), with P, lse and gates formed in double from those logits."""
    h32 = _f32(h32)
    T, E = h32.shape
    key = selection_keys(h32, noise, sel_bias)
    idx = topk(key, w.k)
    P, lse = softmax_lse(h32.astype(np.float64))
    g = gates(P, idx)
    C = capacity(layer_capacity_factor(w), w.k, T, E)
    slot, cpre, ckept, nd = dispatch(idx, E, C, getattr(w, "capacity_priority", "token"))
    return dict(key=key, idx=idx, P=P, lse=lse, gates=g, C=C, slot=slot,
                count_pre=cpre, count_kept=ckept, n_dropped=nd)


def forward(w, inp: Dict[str, object], tokens: Optional[Sequence[int]] = None,
            routing: Optional[Dict[str, object]] = None) -> Dict[str, object]:
    """The whole layer forward in double.

    Without `routing`, the oracle routes from its own logits (rounded to fp32 to
    form the selection key). With `routing` (idx, slot, gates), the expert and
    combine steps run on that routing instead. `tokens` restricts y and credit to
    a subset of tokens; the statistics that need every token's credit are then
    skipped."""
    x = inp["x"]
    if getattr(w, "mlp_gater", False):
        h = router_mlp(x, inp["gater_w1"], inp.get("gater_b1"), inp["w_gate"], inp.get("b_gate"))
    else:
        h = router_logits(x, inp["w_gate"], inp.get("b_gate"))
    T, E = h.shape
    P, lse = softmax_lse(h)
    out: Dict[str, object] = dict(h=h, P=P, lse=lse)
    h32 = h.astype(np.float32)
    key = selection_keys(h32, inp.get("noise"), inp.get("sel_bias"))
    idx = topk(key, w.k)
    g = gates(P, idx)
    C = capacity(layer_capacity_factor(w), w.k, T, E)
    slot, cpre, ckept, nd = dispatch(idx, E, C, getattr(w, "capacity_priority", "token"))
    out.update(h32=h32, key=key, idx=idx, gates=g, C=C, slot=slot, count_pre=cpre,
               count_kept=ckept, n_dropped=nd)
    f, pm, la, lz = balance_stats(P, lse, cpre, w.k, w.alpha, w.beta)
    out.update(f=f, p_mean=pm, l_aux=la, l_z=lz, aux_loss=aux_loss(cpre, lse, w.alpha, w.beta))
    r_idx, r_slot, r_g = idx, slot, g
    if routing is not None:
        r_idx, r_slot, r_g = routing["idx"], routing["slot"], routing["gates"]
    toks = list(range(T)) if tokens is None else list(tokens)
    table = ExpertTable(w.E + w.S, inp["w1"], inp["b1"], inp["w2"], inp["b2"])
    y, credit = experts_combine(toks, x, table, r_idx, r_slot, r_g, w.d, w.F, w.O, w.E, w.S,
                                w.activation)
    out.update(y=y, credit=credit, tokens=np.asarray(toks, dtype=np.int64))
    if tokens is None and inp.get("token_loss") is not None:
        out["expert_loss"] = expert_loss(r_idx, r_slot, credit, inp["token_loss"], E)
    return out

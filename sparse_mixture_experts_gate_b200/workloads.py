"""Seeded synthetic workloads for the sparse top-k MoE layer forward.

This module only draws random numbers and lays them out in memory. It holds none
of the layer's arithmetic: no router product, softmax, top-k, dispatch, expert
FFN, combine or statistic. The CUDA path's tests and benchmark and the CPU
oracle's tests all take their inputs from here, so both sides always consume the
same arrays.

The five named workloads follow the configuration sizes printed on the pages:
  * "tiny"    - the minimal example of "Code Walkthrough - SER", section
                "Minimal example" (4 experts, 2 active, dims 8/16/8, seed 42,
                a (4, 8) token tensor);
  * "default" - the defaults of the same page, section "Configuration"
                (8 experts, 2 active, 512/1024/512, aux weight 0.01);
  * "e64", "decode", "e256" - fine-grained, decode-shaped and large
                training-shaped layers that use the symbols of "Appendix C -
                Acronyms & Symbols" (shared experts S, capacity factor C_f,
                per-expert selection bias b_i) and the expert credit of
                "Sparse MoE Expert-Credit Loss Reweighting Diagram", panel (b).

Distributions: x ~ N(0, 1); every weight matrix ~ N(0, 1/fan_in); expert biases
zero unless `random_biases` (then N(0, 1/fan_in)); selection bias ~ U(-0.1, 0.1);
logit noise n = sigma * N(0, 1) with sigma = 1/E; per-token loss ~ Gamma(2, 1),
drawn as the sum of two Exp(1) variates. Each tensor has its own generator,
seeded from (seed, tensor tag), so a tensor does not depend on which others were
drawn before it.
"""
from __future__ import annotations

import dataclasses
import os
from typing import Dict, Optional

import torch

ACTIVATIONS = {"relu": 0, "gelu": 1, "swish": 2}
TOPK_METHODS = {"greedy": 0, "noisy": 1}
DTYPES = {"bf16": 0, "fp32": 1}

_GOLDEN_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests", "golden")
ZIPF_SCALES_FILE = os.path.join(_GOLDEN_DIR, "decode_zipf_router_row_scales.txt")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens in the batch
    d: int            # input_dim (model width)
    F: int            # expert_dim (d_ff, hidden width of an expert MLP)
    O: int            # output_dim
    E: int            # routed experts
    k: int            # experts active per token
    S: int = 0        # always-on shared experts
    activation: str = "gelu"
    top_k_method: str = "greedy"
    use_selection_bias: bool = False
    capacity_factor: float = 1.25     # <= 0 means no capacity limit
    alpha: float = 0.01               # aux-loss weight
    beta: float = 1e-3                # z-loss weight
    dtype: str = "bf16"               # x, w1, w2, y storage type
    router_bias: bool = False         # linear router carries a bias vector
    noise: bool = False               # draw [T][E] logit noise (noisy top-k)
    zipf: bool = False                # scale router rows for skewed popularity
    token_loss: bool = False          # draw per-token losses for the credit stats
    credit_norm: str = "output"       # credit ||h||: the expert's "output" or its "hidden" activation
    capacity_priority: str = "token"  # capacity queue order: "token" index, or "rank" (choice by choice)
    mlp_gater: bool = False           # router logits from an MLP gate (hidden width gater_hidden)
    gater_hidden: int = 128
    seed: int = 42

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def n_groups(self) -> int:
        return self.E + self.S


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", T=4, d=8, F=16, O=8, E=4, k=2, S=0, activation="relu",
                     capacity_factor=0.0, dtype="fp32", router_bias=True),
    "default": Workload("default", T=4096, d=512, F=1024, O=512, E=8, k=2, activation="gelu",
                        capacity_factor=1.25),
    "e64": Workload("e64", T=8192, d=2048, F=1408, O=2048, E=64, k=6, S=1, activation="swish",
                    capacity_factor=1.25, use_selection_bias=True),
    "decode": Workload("decode", T=128, d=4096, F=1536, O=4096, E=128, k=8, activation="gelu",
                       top_k_method="noisy", capacity_factor=1.0, noise=True, zipf=True),
    "e256": Workload("e256", T=32768, d=7168, F=2048, O=7168, E=256, k=8, S=1,
                     activation="swish", capacity_factor=1.25, token_loss=True),
}

_TAGS = {"x": 1, "w_gate": 2, "b_gate": 3, "sel_bias": 4, "w1": 5, "b1": 6, "w2": 7,
         "b2": 8, "noise": 9, "token_loss": 10, "gater_w1": 11, "gater_b1": 12}


def _gen(device: str, seed: int, tag: str, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + _TAGS[tag] + 100003 * sub)
    return g


def _normal(shape, std: float, device: str, seed: int, tag: str, out_dtype: torch.dtype) -> torch.Tensor:
    g = _gen(device, seed, tag)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    return t.to(out_dtype)


def _expert_normal(e: int, shape, std: float, device: str, seed: int, tag: str,
                   out_dtype: torch.dtype) -> torch.Tensor:
    """One expert's slice of an expert stack, from its own generator, so any
    subset of experts can be drawn without drawing the others."""
    g = _gen(device, seed, tag, sub=e + 1)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    return t.to(out_dtype)


def _expert_stack(G: int, shape, std: float, device: str, seed: int, tag: str,
                  out_dtype: torch.dtype) -> torch.Tensor:
    out = torch.empty((G,) + tuple(shape), device=device, dtype=out_dtype)
    for e in range(G):
        out[e].copy_(_expert_normal(e, shape, std, device, seed, tag, out_dtype))
    return out


def make_expert_weights(w: "Workload", experts, device: str = "cpu", seed: Optional[int] = None,
                        random_biases: bool = False) -> Dict[str, Dict[int, torch.Tensor]]:
    """The w1, b1, w2, b2 slices of the listed experts only (dicts keyed by
    expert index), identical to the same slices of make_inputs on that device."""
    seed = w.seed if seed is None else seed
    sdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out: Dict[str, Dict[int, torch.Tensor]] = {"w1": {}, "b1": {}, "w2": {}, "b2": {}}
    for e in sorted(set(int(v) for v in experts)):
        out["w1"][e] = _expert_normal(e, (w.F, w.d), (1.0 / w.d) ** 0.5, device, seed, "w1", sdt)
        out["w2"][e] = _expert_normal(e, (w.O, w.F), (1.0 / w.F) ** 0.5, device, seed, "w2", sdt)
        if random_biases:
            out["b1"][e] = _expert_normal(e, (w.F,), (1.0 / w.d) ** 0.5, device, seed, "b1", torch.float32)
            out["b2"][e] = _expert_normal(e, (w.O,), (1.0 / w.F) ** 0.5, device, seed, "b2", torch.float32)
        else:
            out["b1"][e] = torch.zeros(w.F, device=device)
            out["b2"][e] = torch.zeros(w.O, device=device)
    return out


def load_zipf_row_scales(E: int) -> Optional[torch.Tensor]:
    """Router row scales for the skewed decode workload, calibrated once by
    tests/golden/make_decode_zipf_scales.py and stored as text."""
    if not os.path.exists(ZIPF_SCALES_FILE):
        return None
    vals = []
    with open(ZIPF_SCALES_FILE) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(float(line))
    if len(vals) != E:
        raise ValueError(f"{ZIPF_SCALES_FILE}: expected {E} scales, found {len(vals)}")
    return torch.tensor(vals, dtype=torch.float32)


def make_tokens(w: Workload, device: str = "cpu", seed: Optional[int] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Per-batch inputs: x [T][d], noise [T][E] (noisy workloads), token_loss [T]."""
    seed = w.seed if seed is None else seed
    sdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out: Dict[str, Optional[torch.Tensor]] = {"x": _normal((w.T, w.d), 1.0, device, seed, "x", sdt)}
    out["noise"] = _normal((w.T, w.E), 1.0 / w.E, device, seed, "noise", torch.float32) if w.noise else None
    if w.token_loss:
        g = _gen(device, seed, "token_loss")
        u = torch.rand((2, w.T), generator=g, device=device, dtype=torch.float64)
        # Gamma(2, 1) is the sum of two independent Exp(1) variates; 1 - u lies in (0, 1].
        out["token_loss"] = (-torch.log1p(-u[0]) - torch.log1p(-u[1])).float()
    else:
        out["token_loss"] = None
    return out


def make_router(w: Workload, device: str = "cpu", seed: Optional[int] = None, random_biases: bool = False,
                apply_zipf: bool = True) -> Dict[str, Optional[torch.Tensor]]:
    """Router parameters: w_gate [E][d], b_gate [E] or None, sel_bias [E] or None.
    With an MLP gate: gater_w1 [H][d] ~ N(0, 1/d), gater_b1 [H] (zero, or
    N(0, 1/d) with random_biases), and w_gate [E][H] ~ N(0, 1/H) its output layer."""
    seed = w.seed if seed is None else seed
    fan = w.gater_hidden if w.mlp_gater else w.d
    wg = _normal((w.E, fan), (1.0 / fan) ** 0.5, device, seed, "w_gate", torch.float32)
    if w.zipf and apply_zipf:
        s = load_zipf_row_scales(w.E)
        if s is not None:
            wg.mul_(s.to(device)[:, None])
    out: Dict[str, Optional[torch.Tensor]] = {"w_gate": wg, "gater_w1": None, "gater_b1": None}
    if w.mlp_gater:
        H = w.gater_hidden
        out["gater_w1"] = _normal((H, w.d), (1.0 / w.d) ** 0.5, device, seed, "gater_w1", torch.float32)
        out["gater_b1"] = (_normal((H,), (1.0 / w.d) ** 0.5, device, seed, "gater_b1", torch.float32)
                           if random_biases else torch.zeros(H, device=device))
    if w.router_bias:
        out["b_gate"] = (_normal((w.E,), (1.0 / w.d) ** 0.5, device, seed, "b_gate", torch.float32)
                         if random_biases else torch.zeros(w.E, device=device))
    else:
        out["b_gate"] = None
    if w.use_selection_bias:
        g = _gen(device, seed, "sel_bias")
        out["sel_bias"] = (torch.rand(w.E, generator=g, device=device) * 0.2 - 0.1).float()
    else:
        out["sel_bias"] = None
    return out


def make_inputs(w: Workload, device: str = "cpu", seed: Optional[int] = None,
                random_biases: bool = False, apply_zipf: bool = True) -> Dict[str, Optional[torch.Tensor]]:
    """Draw every input of one layer forward for workload `w` on `device`.

    Returns a dict with
      x [T][d], w_gate [E][d] fp32, b_gate [E] fp32 or None, sel_bias [E] fp32 or None,
      w1 [E+S][F][d], b1 [E+S][F] fp32, w2 [E+S][O][F], b2 [E+S][O] fp32,
      noise [T][E] fp32 or None, token_loss [T] fp32 or None.
    x, w1 and w2 are bf16 for dtype "bf16" and fp32 for "fp32"; shared experts
    are the last S entries of the expert stacks.
    """
    seed = w.seed if seed is None else seed
    sdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    G = w.n_groups
    inp: Dict[str, Optional[torch.Tensor]] = {}
    inp.update(make_tokens(w, device, seed))
    inp.update(make_router(w, device, seed, random_biases, apply_zipf))
    inp["w1"] = _expert_stack(G, (w.F, w.d), (1.0 / w.d) ** 0.5, device, seed, "w1", sdt)
    inp["w2"] = _expert_stack(G, (w.O, w.F), (1.0 / w.F) ** 0.5, device, seed, "w2", sdt)
    if random_biases:
        inp["b1"] = _expert_stack(G, (w.F,), (1.0 / w.d) ** 0.5, device, seed, "b1", torch.float32)
        inp["b2"] = _expert_stack(G, (w.O,), (1.0 / w.F) ** 0.5, device, seed, "b2", torch.float32)
    else:
        inp["b1"] = torch.zeros(G, w.F, device=device)
        inp["b2"] = torch.zeros(G, w.O, device=device)
    return inp

"""Writes decode_zipf_router_row_scales.txt: per-expert router row scales that
skew the decode workload's expert popularity toward Zipf(1.2).

Recipe (input construction only; it calls nothing but the CPU oracle and the
seeded generator):
  * target popularity pi_i proportional to (rho(i) + 1)^-1.2, with rho a
    permutation seeded by 43, so popularity is unrelated to expert index (and to
    the lower-index tie-break);
  * with k = 8 distinct experts per token f_i <= 1/k, so the head of the Zipf
    target is infeasible: each target is capped at 1/k (the head saturates and
    only the tail follows Zipf);
  * scale row i of W_g by s_i; starting from s = 1, take 60 fixed
    multiplicative steps s_i <- clip(s_i * ((pi_i + 1e-4) / (f_i + 1e-4))^0.3,
    1/4, 4), where f_i is the oracle's selection fraction (counts before the
    cap / kT) on a 4096-token calibration batch drawn with seed 43, noise
    included. The clip keeps router logits in a realistic range (std <= 4);
  * freeze s. The achieved histogram is recorded in the header; it is a
    workload shape, not a parity target.

Run: python tests/golden/make_decode_zipf_scales.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sparse_mixture_experts_gate_b200.workloads import WORKLOADS, ZIPF_SCALES_FILE, make_router, make_tokens  # noqa: E402


def main():
    w = WORKLOADS["decode"]
    cal = w.with_(T=4096)
    router = make_router(w, "cpu", apply_zipf=False)
    toks = make_tokens(cal, "cpu", seed=43)
    h0 = oracle.router_logits(toks["x"], router["w_gate"])
    noise = toks["noise"].numpy()
    rng = np.random.default_rng(43)
    rho = rng.permutation(w.E)
    pi = (rho + 1.0) ** -1.2
    pi /= pi.sum()
    pi = np.minimum(pi, 1.0 / w.k)
    s = np.ones(w.E)
    C = oracle.capacity(w.capacity_factor, w.k, cal.T, w.E)
    for _ in range(60):
        key = oracle.selection_keys((h0 * s[None, :]).astype(np.float32), noise)
        idx = oracle.topk(key, w.k)
        _, cpre, _, _ = oracle.dispatch(idx, w.E, C)
        f = cpre / (w.k * cal.T)
        s = np.clip(s * ((pi + 1e-4) / (f + 1e-4)) ** 0.3, 0.25, 4.0)
    key = oracle.selection_keys((h0 * s[None, :]).astype(np.float32), noise)
    idx = oracle.topk(key, w.k)
    _, cpre, _, _ = oracle.dispatch(idx, w.E, C)
    f = cpre / (w.k * cal.T)
    order = np.argsort(-f)
    with open(ZIPF_SCALES_FILE, "w") as fh:
        fh.write("# Router row scales s_i (one per expert, index order) for the decode workload.\n")
        fh.write("# Written by tests/golden/make_decode_zipf_scales.py (calls only the CPU oracle and the\n")
        fh.write("# seeded generator); recipe in that script. Target pi_i ~ (rho(i)+1)^-1.2.\n")
        fh.write("# Achieved selection fractions on the calibration batch, largest 8: "
                 + " ".join(f"{v:.4f}" for v in f[order[:8]]) + "\n")
        fh.write("# smallest 8: " + " ".join(f"{v:.5f}" for v in f[order[-8:]]) + "\n")
        for v in s:
            fh.write(f"{v:.9g}\n")
    print(ZIPF_SCALES_FILE)


if __name__ == "__main__":
    main()

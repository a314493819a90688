"""Planted mistakes in the oracle must be caught by its pins (no GPU).

Each case copies moe_oracle.c to a temporary directory, replaces one expression
with a plausible mistake (a dropped term, a wrong sign, index or operand, an
off-by-one), builds it with gcc and runs every pin against that build. At least
one pin must fail. The committed oracle is never modified.
"""
import os
import shutil
import subprocess

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "lse_drops_max": ("lse[t] = m + log(z);", "lse[t] = log(z);"),
    "topk_ties_to_higher_index": ("kt[i] > kt[best]", "kt[i] >= kt[best]"),
    "gates_wrong_index": ("s += P[(int64_t)t * E + idx[(int64_t)t * k + r]];",
                          "s += P[(int64_t)t * E + r];"),
    "capacity_floor": ("(int64_t)ceil(capacity_factor", "(int64_t)floor(capacity_factor"),
    "dispatch_off_by_one": ("count_pre[e] = rank + 1;\n            slot[(int64_t)t * k + r] = (rank < C) ? rank : -1;\n        }\n    }\n    int32_t dropped = 0;\n    for (int e = 0; e < E; ++e) {\n        count_kept[e] = (count_pre[e] < C) ? count_pre[e] : (int32_t)C;\n        dropped += count_pre[e] - count_kept[e];\n    }\n    *n_dropped = dropped;\n}\n\n/* Capacity cap with rank-major",
                            "count_pre[e] = rank + 1;\n            slot[(int64_t)t * k + r] = (rank <= C) ? rank : -1;\n        }\n    }\n    int32_t dropped = 0;\n    for (int e = 0; e < E; ++e) {\n        count_kept[e] = (count_pre[e] < C) ? count_pre[e] : (int32_t)C;\n        dropped += count_pre[e] - count_kept[e];\n    }\n    *n_dropped = dropped;\n}\n\n/* Capacity cap with rank-major"),
    "ffn_w1_transposed": ("orc_load(ex->w1, (int64_t)f * d + j, w_dtype)",
                          "orc_load(ex->w1, (int64_t)j * F + f, w_dtype)"),
    "ffn_drops_b2": ("s += (double)ex->b2[n];", "s += 0.0;"),
    "ffn_drops_b1": ("z += (double)ex->b1[f];", "z += 0.0;"),
    "gelu_sign": ("(1.0 + erf(z / sqrt(2.0)))", "(1.0 - erf(z / sqrt(2.0)))"),
    "swish_sign": ("z / (1.0 + exp(-z))", "z / (1.0 + exp(z))"),
    "relu_identity": ("z > 0.0 ? z : 0.0", "z"),
    "shared_experts_skipped": ("for (int s = 0; s < S; ++s) {", "for (int s = 0; s < 0; ++s) {"),
    "credit_drops_gate": ("c = g[a] * sqrt(ss);", "c = sqrt(ss);"),
    "combine_ignores_gate": ("yj[n] += g[a] * o[n];", "yj[n] += o[n];"),
    "f_wrong_normaliser": ("((double)k * (double)T)", "((double)T)"),
    "aux_drops_E": ("*l_aux = alpha * (double)E * aux;", "*l_aux = alpha * aux;"),
    "zloss_not_squared": ("z += lse[t] * lse[t];", "z += lse[t];"),
    "expert_loss_no_mean": ("expert_loss[i] /= (double)T;", "expert_loss[i] /= 1.0;"),
    "router_drops_bias": ("s += (double)b_gate[i];", "s += 0.0;"),
    "noise_ignored": ("v = h32[a] + noise[a];", "v = h32[a];"),
    "selection_bias_sign": ("v = h32[a] + sel_bias[i];", "v = h32[a] - sel_bias[i];"),
    "cv_sample_variance": ("var /= (double)n;", "var /= (double)(n - 1);"),
    "cv_not_squared_mean": ("return var / (mean * mean);", "return var / mean;"),
    "importance_counts_only": ("imp[idx[(int64_t)t * k + r]] += g[(int64_t)t * k + r];",
                               "imp[idx[(int64_t)t * k + r]] += 1.0;"),
    "bias_update_sign": ("const double s = diff > 0 ? 1.0 : (diff < 0 ? -1.0 : 0.0);",
                         "const double s = diff > 0 ? -1.0 : (diff < 0 ? 1.0 : 0.0);"),
    "bias_update_mean_off": ("(int64_t)k * T - (int64_t)E * load[i]", "(int64_t)T - (int64_t)E * load[i]"),
    "hidden_credit_drops_gate": ("c = g[as] * sqrt(ss);", "c = sqrt(ss);"),
    "dro_ema_swapped": ("lhat[i] = ema * lhat[i] + (1.0 - ema) * l[i];", "lhat[i] = (1.0 - ema) * lhat[i] + ema * l[i];"),
    "dro_eta_dropped": ("s += exp(mu[i] + eta * lhat[i] - m);", "s += exp(mu[i] - m);"),
    "dro_objective_old_mu": ("obj += mu[i] * l[i];", "obj += lhat[i] * l[i];"),
    "rank_major_token_order": ("    for (int r = 0; r < k; ++r) {\n        for (int t = 0; t < T; ++t) {\n            int e = idx[(int64_t)t * k + r];",
                               "    for (int t = 0; t < T; ++t) {\n        for (int r = 0; r < k; ++r) {\n            int e = idx[(int64_t)t * k + r];"),
    "mlp_no_relu": ("z[u] = s > 0.0 ? s : 0.0;", "z[u] = s;"),
    "mlp_drops_b1": ("                s += (double)b1[u];", "                s += 0.0;"),
    "aux_loss_coefs_swapped": ("return load_balance_coef * balance + z_loss_coef * (z / (double)T);",
                               "return z_loss_coef * balance + load_balance_coef * (z / (double)T);"),
    "aux_loss_z_not_mean": ("return load_balance_coef * balance + z_loss_coef * (z / (double)T);",
                            "return load_balance_coef * balance + z_loss_coef * z;"),
    "aux_loss_lse_not_squared": ("z += v * v;", "z += v;"),
    "softmax_wrong_exponent": ("P[(int64_t)t * E + i] = exp(ht[i] - m) / z;",
                               "P[(int64_t)t * E + i] = exp(ht[i]) / z;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    shutil.copy(os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.h"), tmp_path)
    (tmp_path / "moe_oracle.c").write_text(src.replace(old, new))
    so = str(tmp_path / "libmutant.so")
    subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", so,
                    str(tmp_path / "moe_oracle.c"), "-lm"], check=True)
    failed = []
    with oracle.using_library(so):
        for check in oracle_pins.ALL_CHECKS:
            try:
                check()
            except AssertionError:
                failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake {name}"

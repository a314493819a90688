"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before touching a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

from sparse_mixture_experts_gate_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return binding.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(binding.EXPORTS)


def test_header_constants_match_the_binding():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    ev = int(re.search(r"#define MOE_TIMING_EVENTS (\d+)", src).group(1))
    assert ev == binding.MOE_TIMING_EVENTS == len(binding.STAGES) + 1
    m = re.search(r"#define MOE_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", src)
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == binding.MOE_NOALLOC_SCRATCH_BYTES


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_config_default_mirrors_ser_configuration(L):
    c = binding.moe_config_default()
    # "Code Walkthrough - SER", section "Configuration".
    assert (c.num_experts, c.num_active, c.input_dim, c.expert_dim, c.output_dim) == (8, 2, 512, 1024, 512)
    assert c.top_k_method == binding.MOE_TOPK["greedy"]
    assert abs(c.load_balance_coef - 0.01) < 1e-9
    assert c.temperature == 1.0 and c.dtype == binding.MOE_DTYPE["bf16"]


def test_status_strings(L):
    for code, name in ((0, "MOE_OK"), (-1, "MOE_ERR_INVALID_ARG"), (-2, "MOE_ERR_UNSUPPORTED"),
                       (-3, "MOE_ERR_CUDA"), (-4, "MOE_ERR_WORKSPACE"), (-5, "MOE_ERR_TIMEOUT"),
                       (-6, "MOE_ERR_STATE"), (-7, "MOE_ERR_INTERNAL")):
        assert binding.moe_status_string(code) == name


def _weights():
    # Fake, never-dereferenced addresses: validation happens before any CUDA call.
    return binding.MoeWeights(0x1000, None, None, 0x2000, 0x3000, None, None)


@pytest.mark.parametrize("field,value,code", [
    ("num_experts", 0, binding.MOE_ERR_INVALID_ARG),
    ("num_experts", 300, binding.MOE_ERR_UNSUPPORTED),
    ("num_active", 0, binding.MOE_ERR_INVALID_ARG),
    ("num_active", 9, binding.MOE_ERR_INVALID_ARG),       # k > E
    ("input_dim", 0, binding.MOE_ERR_INVALID_ARG),
    ("input_dim", 500, binding.MOE_ERR_UNSUPPORTED),      # bf16 needs multiples of 64
    ("expert_dim", 1000, binding.MOE_ERR_UNSUPPORTED),
    ("output_dim", 520, binding.MOE_ERR_UNSUPPORTED),     # bf16 stores 64-column boxes
    ("num_shared", -1, binding.MOE_ERR_INVALID_ARG),
    ("activation", 7, binding.MOE_ERR_INVALID_ARG),
    ("top_k_method", 5, binding.MOE_ERR_INVALID_ARG),
    ("dtype", 9, binding.MOE_ERR_INVALID_ARG),
    ("temperature", 0.5, binding.MOE_ERR_UNSUPPORTED),
    ("max_tokens", -3, binding.MOE_ERR_INVALID_ARG),
    ("credit_norm", 4, binding.MOE_ERR_INVALID_ARG),
    ("capacity_priority", 2, binding.MOE_ERR_INVALID_ARG),
    ("use_mlp_gater", 3, binding.MOE_ERR_INVALID_ARG),
])
def test_create_rejects_bad_config_on_host(L, field, value, code):
    c = binding.moe_config_default()
    setattr(c, field, value)
    h = ctypes.c_void_p(0xdead)
    rc = L.moe_layer_create(ctypes.byref(c), ctypes.byref(_weights()), ctypes.byref(h))
    assert rc == code, binding.moe_last_error()
    assert h.value is None
    assert binding.moe_last_error()


def test_create_rejects_missing_weights(L):
    c = binding.moe_config_default()
    h = ctypes.c_void_p()
    for name in ("w_gate", "w1", "w2"):
        w = _weights()
        setattr(w, name, None)
        assert L.moe_layer_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG
        assert name in binding.moe_last_error()
    c.use_selection_bias = 1
    assert L.moe_layer_create(ctypes.byref(c), ctypes.byref(_weights()), ctypes.byref(h)) == \
        binding.MOE_ERR_INVALID_ARG
    assert "sel_bias" in binding.moe_last_error()
    assert L.moe_layer_create(None, ctypes.byref(_weights()), ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_layer_create(ctypes.byref(c), None, ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG


def test_mlp_gate_config_checked_on_host(L):
    c = binding.moe_config_default()
    c.use_mlp_gater = 1
    h = ctypes.c_void_p()
    assert L.moe_layer_create(ctypes.byref(c), ctypes.byref(_weights()), ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG
    assert "gater_w1" in binding.moe_last_error()
    w = _weights()
    w.gater_w1 = 0x1000
    for H in (0, 257):
        c.gater_hidden_dim = H
        assert L.moe_layer_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_UNSUPPORTED


def test_null_layer_calls_fail_cleanly(L):
    assert binding.moe_workspace_bytes(None, 16) == 0
    assert binding.moe_capacity(None, 16) == -1
    assert L.moe_forward(None, None, 0, None, None, 0, None, None, None) == binding.MOE_ERR_INVALID_ARG
    st = binding.MoeStats()
    assert L.moe_aux_stats(None, None, ctypes.byref(st), None) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_device_status(None, None) == binding.MOE_ERR_INVALID_ARG
    assert binding.moe_launch_count(None) == 0
    assert L.moe_update_selection_bias(None, None, ctypes.c_float(0.1), None, None) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_dro_update(None, None, ctypes.c_float(0.9), ctypes.c_float(1.0), None, None, None, None) == \
        binding.MOE_ERR_INVALID_ARG
    assert L.moe_stat_partials(None, None, None, None) == binding.MOE_ERR_INVALID_ARG
    binding.moe_destroy(None)


def test_valid_config_without_gpu_reports_cuda_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    c = binding.moe_config_default()
    h = ctypes.c_void_p()
    assert L.moe_layer_create(ctypes.byref(c), ctypes.byref(_weights()), ctypes.byref(h)) == binding.MOE_ERR_CUDA

"""moe_forward_noalloc against moe_forward (GPU).

moe_forward_noalloc is for callers that cannot allocate device memory
themselves (a plugin whose host application owns all device memory through its
own pool, or a loop that must not call cudaMalloc/cudaFree); it runs the same
forward with the library's built-in 64 MiB device scratch instead of a caller
workspace. Both entry points launch the same kernels on the same inputs, and
those kernels are deterministic (every output has one fixed summation order),
so the results must be identical bit for bit on each of two calls in a row.
An oversized batch must be refused on the host.
"""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_gate_b200 import binding
from sparse_mixture_experts_gate_b200.binding import MoEError, MoELayer, MoeRouting
from sparse_mixture_experts_gate_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _routing(out):
    return MoeRouting(out["logits"].data_ptr(), out["gates"].data_ptr(), out["topk_idx"].data_ptr(),
                      out["slot"].data_ptr(), out["count_pre"].data_ptr(), out["count_kept"].data_ptr())


def _host(out):
    return {k: v.float().cpu().numpy().astype(np.float64) if v.is_floating_point() else v.cpu().numpy()
            for k, v in out.items()}


def test_noalloc_matches_workspace_forward_on_two_calls():
    w = WORKLOADS["default"]  # the SER default shape, T = 4096
    inp = make_inputs(w, "cpu", seed=21, random_biases=True)
    layer = MoELayer(w, inp)
    assert binding.moe_workspace_bytes(layer.handle, w.T) <= binding.MOE_NOALLOC_SCRATCH_BYTES
    x = inp["x"].cuda()
    ref = layer.forward(x)
    layer.aux_stats(ref)
    torch.cuda.synchronize()
    ref = _host(ref)
    s = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = layer.alloc_outputs(w.T)
        for v in out.values():
            v.fill_(float("nan")) if v.is_floating_point() else v.fill_(-7)
        binding.moe_forward_noalloc(layer.handle, x.data_ptr(), w.T, None, out["y"].data_ptr(), _routing(out), s)
        layer.aux_stats(out)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        got = _host(out)
        for k in ("y", "topk_idx", "slot", "count_pre", "count_kept", "n_dropped", "logits", "gates", "f",
                  "p_mean", "l_aux", "l_z", "credit", "importance", "cv_load", "cv_importance", "l_total"):
            assert np.array_equal(got[k], ref[k]), (call, k)


def test_noalloc_refuses_a_batch_beyond_its_scratch():
    w = WORKLOADS["default"].with_(T=20000)
    inp = make_inputs(w.with_(T=8), "cpu", seed=3)
    layer = MoELayer(w, inp)
    assert binding.moe_workspace_bytes(layer.handle, w.T) > binding.MOE_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(w.T, w.d, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(w.T, w.O, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(MoEError) as ei:
        binding.moe_forward_noalloc(layer.handle, x.data_ptr(), w.T, None, y.data_ptr(), None,
                                    torch.cuda.current_stream().cuda_stream)
    assert ei.value.code == binding.MOE_ERR_WORKSPACE
    assert "built-in" in str(ei.value)

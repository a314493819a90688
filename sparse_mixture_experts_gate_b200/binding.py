"""ctypes binding of libmoe.so (the C ABI of include/moe.h).

Argument marshalling only: every step of the layer forward runs in the CUDA
kernels behind the C ABI. PyTorch supplies device memory and streams. If the
library has not been built, loading it raises; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 0, -1, -2, -3
MOE_ERR_WORKSPACE, MOE_ERR_TIMEOUT, MOE_ERR_STATE, MOE_ERR_INTERNAL = -4, -5, -6, -7
MOE_ACT = {"relu": 0, "gelu": 1, "swish": 2}
MOE_TOPK = {"greedy": 0, "noisy": 1}
MOE_DTYPE = {"bf16": 0, "fp32": 1}
MOE_CREDIT = {"output": 0, "hidden": 1}
MOE_PRIORITY = {"token": 0, "rank": 1}

# Every symbol include/moe.h declares.
EXPORTS = ("moe_config_default", "moe_layer_create", "moe_workspace_bytes", "moe_capacity", "moe_forward",
           "moe_forward_noalloc", "moe_aux_stats", "moe_stat_partials", "moe_stats_from_partials",
           "moe_update_selection_bias", "moe_dro_update", "moe_selftest_bounded_wait", "moe_device_status", "moe_set_timing_events", "moe_launch_count", "moe_destroy", "moe_status_string",
           "moe_last_error")


class MoeConfig(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int32), ("num_active", ctypes.c_int32), ("input_dim", ctypes.c_int32),
                ("expert_dim", ctypes.c_int32), ("output_dim", ctypes.c_int32), ("num_shared", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("activation", ctypes.c_int32),
                ("top_k_method", ctypes.c_int32), ("use_selection_bias", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("load_balance_coef", ctypes.c_float),
                ("z_loss_coef", ctypes.c_float), ("temperature", ctypes.c_float), ("credit_norm", ctypes.c_int32),
                ("capacity_priority", ctypes.c_int32), ("use_mlp_gater", ctypes.c_int32),
                ("gater_hidden_dim", ctypes.c_int32)]


class MoeWeights(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("b_gate", ctypes.c_void_p), ("sel_bias", ctypes.c_void_p),
                ("w1", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("b2", ctypes.c_void_p), ("gater_w1", ctypes.c_void_p), ("gater_b1", ctypes.c_void_p)]


class MoeRouting(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("gates", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p),
                ("slot", ctypes.c_void_p), ("count_pre", ctypes.c_void_p), ("count_kept", ctypes.c_void_p)]


class MoeStats(ctypes.Structure):
    _fields_ = [("f", ctypes.c_void_p), ("p_mean", ctypes.c_void_p), ("l_aux", ctypes.c_void_p),
                ("l_z", ctypes.c_void_p), ("n_dropped", ctypes.c_void_p), ("credit", ctypes.c_void_p),
                ("expert_loss", ctypes.c_void_p), ("importance", ctypes.c_void_p), ("cv_load", ctypes.c_void_p),
                ("cv_importance", ctypes.c_void_p), ("l_total", ctypes.c_void_p)]


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str, message: str):
        super().__init__(f"{where}: {moe_status_string(code)} ({code}): {message}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_mixture_experts_gate_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.moe_config_default.restype = MoeConfig
        L.moe_config_default.argtypes = []
        L.moe_layer_create.restype = ctypes.c_int
        L.moe_layer_create.argtypes = [ctypes.POINTER(MoeConfig), ctypes.POINTER(MoeWeights), ctypes.POINTER(vp)]
        L.moe_workspace_bytes.restype = sz
        L.moe_workspace_bytes.argtypes = [vp, i32]
        L.moe_capacity.restype = i64
        L.moe_capacity.argtypes = [vp, i32]
        L.moe_forward.restype = ctypes.c_int
        L.moe_forward.argtypes = [vp, vp, i32, vp, vp, sz, vp, ctypes.POINTER(MoeRouting), vp]
        L.moe_forward_noalloc.restype = ctypes.c_int
        L.moe_forward_noalloc.argtypes = [vp, vp, i32, vp, vp, ctypes.POINTER(MoeRouting), vp]
        L.moe_aux_stats.restype = ctypes.c_int
        L.moe_aux_stats.argtypes = [vp, vp, ctypes.POINTER(MoeStats), vp]
        L.moe_stat_partials.restype = ctypes.c_int
        L.moe_stat_partials.argtypes = [vp, vp, vp, vp]
        L.moe_stats_from_partials.restype = ctypes.c_int
        L.moe_stats_from_partials.argtypes = [vp, vp, i32, ctypes.POINTER(MoeStats), vp]
        L.moe_update_selection_bias.restype = ctypes.c_int
        L.moe_update_selection_bias.argtypes = [vp, vp, ctypes.c_float, vp, vp]
        L.moe_dro_update.restype = ctypes.c_int
        L.moe_dro_update.argtypes = [vp, vp, ctypes.c_float, ctypes.c_float, vp, vp, vp, vp]
        L.moe_selftest_bounded_wait.restype = ctypes.c_int
        L.moe_selftest_bounded_wait.argtypes = [vp]
        L.moe_device_status.restype = ctypes.c_int
        L.moe_device_status.argtypes = [vp, vp]
        L.moe_set_timing_events.restype = ctypes.c_int
        L.moe_set_timing_events.argtypes = [vp, ctypes.POINTER(vp)]
        L.moe_launch_count.restype = i32
        L.moe_launch_count.argtypes = [vp]
        L.moe_destroy.restype = None
        L.moe_destroy.argtypes = [vp]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_last_error.argtypes = []
        _lib = L
    return _lib


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def _check(rc: int, where: str) -> int:
    if rc != MOE_OK:
        raise MoEError(rc, where, moe_last_error())
    return rc


def moe_config_default() -> MoeConfig:
    return lib().moe_config_default()


def moe_layer_create(cfg: MoeConfig, weights: MoeWeights) -> int:
    h = ctypes.c_void_p()
    _check(lib().moe_layer_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(h)), "moe_layer_create")
    return h.value


def moe_workspace_bytes(layer: int, T: int) -> int:
    return int(lib().moe_workspace_bytes(layer, T))


def moe_capacity(layer: int, T: int) -> int:
    return int(lib().moe_capacity(layer, T))


def moe_forward(layer: int, x: int, T: int, logit_noise: Optional[int], workspace: int, ws_bytes: int, y: int,
                routing: Optional[MoeRouting], stream: int) -> int:
    r = ctypes.byref(routing) if routing is not None else None
    return _check(lib().moe_forward(layer, x, T, logit_noise, workspace, ws_bytes, y, r, stream), "moe_forward")


MOE_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def moe_forward_noalloc(layer: int, x: int, T: int, logit_noise: Optional[int], y: int,
                        routing: Optional[MoeRouting], stream: int) -> int:
    """moe_forward with the library's built-in device scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    r = ctypes.byref(routing) if routing is not None else None
    return _check(lib().moe_forward_noalloc(layer, x, T, logit_noise, y, r, stream), "moe_forward_noalloc")


def moe_aux_stats(layer: int, token_loss: Optional[int], stats: MoeStats, stream: int) -> int:
    return _check(lib().moe_aux_stats(layer, token_loss, ctypes.byref(stats), stream), "moe_aux_stats")


def moe_stat_partials(layer: int, token_loss: Optional[int], partials: int, stream: int) -> int:
    return _check(lib().moe_stat_partials(layer, token_loss, partials, stream), "moe_stat_partials")


def moe_stats_from_partials(layer: int, partials: int, has_token_loss: bool, stats: MoeStats, stream: int) -> int:
    return _check(lib().moe_stats_from_partials(layer, partials, int(has_token_loss), ctypes.byref(stats), stream),
                  "moe_stats_from_partials")


def stat_partials_size(E: int) -> int:
    return 4 * E + 3


def moe_update_selection_bias(layer: int, partials: Optional[int], gamma: float, sel_bias: int, stream: int) -> int:
    return _check(lib().moe_update_selection_bias(layer, partials, float(gamma), sel_bias, stream),
                  "moe_update_selection_bias")


def allreduce_partials(partials, group=None):
    """Sums the statistics' partial sums over the ranks of `group` in place
    (a no-op without an initialised process group). Every rank must call it
    at the same step, like any collective."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(partials, op=dist.ReduceOp.SUM, group=group)
    return partials


def moe_dro_update(layer: int, expert_loss: int, ema: float, eta: float, lhat: int, mu: int,
                   objective: Optional[int], stream: int) -> int:
    return _check(lib().moe_dro_update(layer, expert_loss, float(ema), float(eta), lhat, mu, objective, stream),
                  "moe_dro_update")


def moe_selftest_bounded_wait(stream: int) -> int:
    return _check(lib().moe_selftest_bounded_wait(stream), "moe_selftest_bounded_wait")


def moe_device_status(layer: int, stream: int) -> int:
    return int(lib().moe_device_status(layer, stream))


MOE_TIMING_EVENTS = 7
STAGES = ("router", "dispatch", "gemm1", "gemm2", "combine", "stats")


def moe_set_timing_events(layer: int, events) -> int:
    """events: sequence of MOE_TIMING_EVENTS raw cudaEvent_t handles, or None."""
    if events is None:
        return _check(lib().moe_set_timing_events(layer, None), "moe_set_timing_events")
    arr = (ctypes.c_void_p * MOE_TIMING_EVENTS)(*events)
    return _check(lib().moe_set_timing_events(layer, arr), "moe_set_timing_events")


def moe_launch_count(layer: int) -> int:
    return int(lib().moe_launch_count(layer))


def moe_destroy(layer: int) -> None:
    lib().moe_destroy(layer)


# ------------------------------------------------------------------ torch helper

def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


class MoELayer:
    """Owns the device tensors around one C-ABI layer: borrowed weights, the
    workspace and the routing/statistics output buffers. Pointer marshalling
    only; the forward itself is moe_forward + moe_aux_stats."""

    def __init__(self, workload, weights: Dict[str, object], max_tokens: Optional[int] = None, device="cuda"):
        import torch
        w = workload
        self.w = w
        self.device = torch.device(device)
        cfg = moe_config_default()
        cfg.num_experts, cfg.num_active = w.E, w.k
        cfg.input_dim, cfg.expert_dim, cfg.output_dim = w.d, w.F, w.O
        cfg.num_shared = w.S
        cfg.capacity_factor = w.capacity_factor
        cfg.activation = MOE_ACT[w.activation]
        cfg.top_k_method = MOE_TOPK[w.top_k_method]
        cfg.use_selection_bias = int(w.use_selection_bias)
        cfg.dtype = MOE_DTYPE[w.dtype]
        cfg.max_tokens = max_tokens or 0
        cfg.load_balance_coef, cfg.z_loss_coef, cfg.temperature = w.alpha, w.beta, 1.0
        cfg.credit_norm = MOE_CREDIT[w.credit_norm]
        cfg.capacity_priority = MOE_PRIORITY[w.capacity_priority]
        cfg.use_mlp_gater = int(w.mlp_gater)
        cfg.gater_hidden_dim = w.gater_hidden
        self.cfg = cfg
        self.weights = {k: (v.to(self.device).contiguous() if v is not None else None)
                        for k, v in weights.items()
                        if k in ("w_gate", "b_gate", "sel_bias", "w1", "b1", "w2", "b2", "gater_w1", "gater_b1")}
        ww = self.weights
        self._cw = MoeWeights(_ptr(ww["w_gate"]), _ptr(ww.get("b_gate")), _ptr(ww.get("sel_bias")),
                              _ptr(ww["w1"]), _ptr(ww["w2"]), _ptr(ww.get("b1")), _ptr(ww.get("b2")),
                              _ptr(ww.get("gater_w1")), _ptr(ww.get("gater_b1")))
        self.handle = moe_layer_create(cfg, self._cw)
        self._ws = None
        self._ws_T = -1
        self._dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def close(self):
        if getattr(self, "handle", None):
            moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace(self, T: int):
        import torch
        need = moe_workspace_bytes(self.handle, T)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        return self._ws, need

    def alloc_outputs(self, T: int):
        import torch
        w, dev = self.w, self.device
        out = dict(
            y=torch.empty(T, w.O, dtype=self._dt, device=dev),
            logits=torch.empty(T, w.E, dtype=torch.float32, device=dev),
            gates=torch.empty(T, w.k, dtype=torch.float32, device=dev),
            topk_idx=torch.empty(T, w.k, dtype=torch.int32, device=dev),
            slot=torch.empty(T, w.k, dtype=torch.int32, device=dev),
            count_pre=torch.empty(w.E, dtype=torch.int32, device=dev),
            count_kept=torch.empty(w.E, dtype=torch.int32, device=dev),
            f=torch.empty(w.E, dtype=torch.float32, device=dev),
            p_mean=torch.empty(w.E, dtype=torch.float32, device=dev),
            l_aux=torch.empty(1, dtype=torch.float32, device=dev),
            l_z=torch.empty(1, dtype=torch.float32, device=dev),
            n_dropped=torch.empty(1, dtype=torch.int32, device=dev),
            credit=torch.empty(T, w.k, dtype=torch.float32, device=dev),
            expert_loss=torch.empty(w.E, dtype=torch.float32, device=dev),
            importance=torch.empty(w.E, dtype=torch.float32, device=dev),
            cv_load=torch.empty(1, dtype=torch.float32, device=dev),
            cv_importance=torch.empty(1, dtype=torch.float32, device=dev),
            l_total=torch.empty(1, dtype=torch.float32, device=dev),
        )
        return out

    def forward(self, x, noise=None, out=None, stream=None, with_routing=True):
        import torch
        T = int(x.shape[0])
        if out is None:
            out = self.alloc_outputs(T)
        ws, need = self.workspace(T)
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        routing = None
        if with_routing:
            routing = MoeRouting(_ptr(out["logits"]), _ptr(out["gates"]), _ptr(out["topk_idx"]), _ptr(out["slot"]),
                                 _ptr(out["count_pre"]), _ptr(out["count_kept"]))
        moe_forward(self.handle, _ptr(x), T, _ptr(noise), ws.data_ptr(), ws.numel(), _ptr(out["y"]), routing, s)
        return out

    def aux_stats(self, out, token_loss=None, stream=None):
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        moe_aux_stats(self.handle, _ptr(token_loss), self._stats_struct(out, token_loss is not None, True), s)
        return out

    @staticmethod
    def _stats_struct(out, with_loss: bool, with_credit: bool) -> "MoeStats":
        g = lambda k: _ptr(out.get(k))
        return MoeStats(g("f"), g("p_mean"), g("l_aux"), g("l_z"), g("n_dropped"),
                        g("credit") if with_credit else None, g("expert_loss") if with_loss else None,
                        g("importance"), g("cv_load"), g("cv_importance"), g("l_total"))

    def update_selection_bias(self, gamma: float, partials=None, stream=None):
        """sel_bias += gamma * sign(kT/E - load) in place on the layer's own selection
        bias, loads from `partials` (e.g. all-reduced) or from the last forward."""
        import torch
        if self.weights.get("sel_bias") is None:
            raise ValueError("the layer has no selection bias")
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        moe_update_selection_bias(self.handle, _ptr(partials), gamma, self.weights["sel_bias"].data_ptr(), s)

    def dp_aux_stats(self, out, token_loss=None, group=None, stream=None):
        """Statistics of the whole data-parallel batch: this rank's partial sums,
        a sum all-reduce over `group` (torch.distributed), then the statistics
        from the summed partials. out["credit"] stays this rank's."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        self.aux_stats(out, token_loss=token_loss, stream=stream)
        partials = torch.empty(stat_partials_size(self.w.E), dtype=torch.float32, device=self.device)
        moe_stat_partials(self.handle, _ptr(token_loss), partials.data_ptr(), s)
        allreduce_partials(partials, group)
        moe_stats_from_partials(self.handle, partials.data_ptr(), token_loss is not None,
                                self._stats_struct(out, token_loss is not None, False), s)
        return out, partials

    def device_status(self, stream=None) -> int:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        return moe_device_status(self.handle, s)

    def launch_count(self) -> int:
        return moe_launch_count(self.handle)


class HostPipeline:
    """Forwards whose inputs and outputs live in pinned host memory, pipelined:
    step i's host-to-device input copy (on an upload stream), its forward and
    statistics (compute stream) and its result copy back (download stream)
    overlap with the neighbouring steps'. Two device slots alternate; events
    order every reuse of a slot, so each step's result is exactly what a
    serial copy-forward-copy would give.

    submit() enqueues one step and returns at once; synchronize() waits for all
    submitted steps. The host tensors of a step must stay untouched until
    synchronize() (or until the step's download has completed)."""

    STAT_KEYS = ("l_aux", "l_z", "n_dropped", "f", "p_mean", "expert_loss", "importance", "cv_load",
                 "cv_importance", "l_total")

    def __init__(self, layer: "MoELayer", T: int, with_noise: bool = False, with_loss: bool = False):
        import torch
        self.layer, self.T = layer, T
        dev = layer.device
        w = layer.w
        self.up = torch.cuda.Stream(dev)
        self.comp = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        self.slots = []
        for _ in range(2):
            self.slots.append(dict(
                x=torch.empty(T, w.d, dtype=layer._dt, device=dev),
                noise=torch.empty(T, w.E, dtype=torch.float32, device=dev) if with_noise else None,
                loss=torch.empty(T, dtype=torch.float32, device=dev) if with_loss else None,
                out=layer.alloc_outputs(T),
                uploaded=torch.cuda.Event(), computed=torch.cuda.Event(), downloaded=torch.cuda.Event(),
                used=False))
        layer.workspace(T)
        self.n = 0

    def submit(self, x_h, y_h, noise_h=None, loss_h=None, stats_h=None):
        """One step: x_h [T][d] (pinned host, the layer's dtype) in, y_h [T][O] out;
        optional noise [T][E] and token losses [T] in, and a dict of pinned host
        tensors (keys of STAT_KEYS) that receive the step's statistics."""
        import torch
        sl = self.slots[self.n % 2]
        self.n += 1
        with torch.cuda.stream(self.up):
            if sl["used"]:
                self.up.wait_event(sl["computed"])  # the slot's previous forward has read its inputs
            sl["x"].copy_(x_h, non_blocking=True)
            if noise_h is not None:
                sl["noise"].copy_(noise_h, non_blocking=True)
            if loss_h is not None:
                sl["loss"].copy_(loss_h, non_blocking=True)
            sl["uploaded"].record(self.up)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(sl["uploaded"])
            if sl["used"]:
                self.comp.wait_event(sl["downloaded"])  # the slot's previous results have left
            s = self.comp.cuda_stream
            self.layer.forward(sl["x"], noise=sl["noise"] if noise_h is not None else None, out=sl["out"], stream=s)
            self.layer.aux_stats(sl["out"], token_loss=sl["loss"] if loss_h is not None else None, stream=s)
            sl["computed"].record(self.comp)
        with torch.cuda.stream(self.down):
            self.down.wait_event(sl["computed"])
            y_h.copy_(sl["out"]["y"], non_blocking=True)
            for k, v in (stats_h or {}).items():
                v.copy_(sl["out"][k], non_blocking=True)
            sl["downloaded"].record(self.down)
        sl["used"] = True

    def synchronize(self):
        self.down.synchronize()
        self.comp.synchronize()
        self.up.synchronize()

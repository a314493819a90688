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
           "moe_update_selection_bias", "moe_dro_update", "moe_selftest_bounded_wait", "moe_selftest_gemm_timeout",
           "moe_selftest_router_timeout", "moe_router_planes_bytes", "moe_prepare_router",
           "moe_ep_dispatch", "moe_ep_layout", "moe_ep_experts_workspace_bytes", "moe_ep_experts", "moe_ep_combine", "moe_device_status", "moe_set_timing_events", "moe_launch_count", "moe_destroy", "moe_status_string",
           "moe_last_error")


class MoeConfig(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int32), ("num_active", ctypes.c_int32), ("input_dim", ctypes.c_int32),
                ("expert_dim", ctypes.c_int32), ("output_dim", ctypes.c_int32), ("num_shared", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("activation", ctypes.c_int32),
                ("top_k_method", ctypes.c_int32), ("use_selection_bias", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("load_balance_coef", ctypes.c_float),
                ("z_loss_coef", ctypes.c_float), ("temperature", ctypes.c_float), ("credit_norm", ctypes.c_int32),
                ("capacity_priority", ctypes.c_int32), ("use_mlp_gater", ctypes.c_int32),
                ("gater_hidden_dim", ctypes.c_int32), ("ep_size", ctypes.c_int32), ("ep_rank", ctypes.c_int32)]


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
        L.moe_ep_dispatch.restype = ctypes.c_int
        L.moe_ep_dispatch.argtypes = [vp, vp, i32, vp, vp, sz, ctypes.POINTER(MoeRouting), vp]
        L.moe_ep_layout.restype = ctypes.c_int
        L.moe_ep_layout.argtypes = [vp, vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp]
        L.moe_ep_experts_workspace_bytes.restype = sz
        L.moe_ep_experts_workspace_bytes.argtypes = [vp, i32]
        L.moe_ep_experts.restype = ctypes.c_int
        L.moe_ep_experts.argtypes = [vp, vp, vp, i32, vp, vp, sz, vp]
        L.moe_ep_combine.restype = ctypes.c_int
        L.moe_ep_combine.argtypes = [vp, vp, vp]
        L.moe_selftest_bounded_wait.restype = ctypes.c_int
        L.moe_selftest_bounded_wait.argtypes = [vp]
        L.moe_router_planes_bytes.restype = sz
        L.moe_router_planes_bytes.argtypes = [vp]
        L.moe_prepare_router.restype = ctypes.c_int
        L.moe_prepare_router.argtypes = [vp, vp, sz, vp]
        L.moe_selftest_gemm_timeout.restype = ctypes.c_int
        L.moe_selftest_gemm_timeout.argtypes = [vp, vp, i32, vp, sz, vp, vp]
        L.moe_selftest_router_timeout.restype = ctypes.c_int
        L.moe_selftest_router_timeout.argtypes = [vp, vp, i32, vp, sz, vp]
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


def moe_router_planes_bytes(layer: int) -> int:
    return int(lib().moe_router_planes_bytes(layer))


def moe_prepare_router(layer: int, planes: Optional[int], nbytes: int, stream: int) -> int:
    return _check(lib().moe_prepare_router(layer, planes, nbytes, stream), "moe_prepare_router")


def moe_selftest_gemm_timeout(layer: int, x: int, T: int, workspace: int, ws_bytes: int, y: int, stream: int) -> int:
    return _check(lib().moe_selftest_gemm_timeout(layer, x, T, workspace, ws_bytes, y, stream),
                  "moe_selftest_gemm_timeout")


def moe_selftest_router_timeout(layer: int, x: int, T: int, workspace: int, ws_bytes: int, stream: int) -> int:
    return _check(lib().moe_selftest_router_timeout(layer, x, T, workspace, ws_bytes, stream),
                  "moe_selftest_router_timeout")


def moe_device_status(layer: int, stream: int) -> int:
    return int(lib().moe_device_status(layer, stream))


MOE_TIMING_EVENTS = 8
STAGES = ("router", "dispatch", "scatter", "gemm1", "gemm2", "combine", "stats")


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

    def __init__(self, workload, weights: Dict[str, object], max_tokens: Optional[int] = None, device="cuda",
                 ep_size: int = 1, ep_rank: int = 0):
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
        cfg.ep_size, cfg.ep_rank = ep_size, ep_rank
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

    def prepare_router(self, stream=None):
        """Split the router matrix into bf16 planes once (moe_prepare_router) into
        a buffer this object keeps; later forwards skip the per-forward split.
        Call again after changing the router weights."""
        import torch
        n = moe_router_planes_bytes(self.handle)
        if n == 0:
            return
        if getattr(self, "_planes", None) is None or self._planes.numel() < n:
            self._planes = torch.empty(n, dtype=torch.uint8, device=self.device)
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        moe_prepare_router(self.handle, self._planes.data_ptr(), self._planes.numel(), s)

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

    # ------------------------------------------------------ expert parallelism
    # A layer created with ep_size = G > 1 holds experts ep_rank*E/G .. of the
    # stacks it is given (then the shared experts). ep_forward runs the whole
    # forward over torch.distributed; the three phases below are the pieces.

    def ep_dispatch(self, x, noise=None, out=None, stream=None):
        """Phase 1: routing and dispatch of this rank's tokens. Returns (out,
        send rows [n][d], output rows [n][O] (the row space, views of the
        workspace), expert_rows: padded rows per expert, a host list)."""
        import torch
        T = int(x.shape[0])
        if out is None:
            out = self.alloc_outputs(T)
        ws, _ = self.workspace(T)
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        routing = MoeRouting(_ptr(out["logits"]), _ptr(out["gates"]), _ptr(out["topk_idx"]), _ptr(out["slot"]),
                             _ptr(out["count_pre"]), _ptr(out["count_kept"]))
        _check(lib().moe_ep_dispatch(self.handle, _ptr(x), T, _ptr(noise), ws.data_ptr(), ws.numel(),
                                     ctypes.byref(routing), s), "moe_ep_dispatch")
        rows = (ctypes.c_int32 * self.w.E)()
        rin, rout = ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib().moe_ep_layout(self.handle, rows, ctypes.byref(rin), ctypes.byref(rout), s), "moe_ep_layout")
        n = int(sum(rows))
        esz = 2 if self.w.dtype == "bf16" else 4
        oi, oo = rin.value - ws.data_ptr(), rout.value - ws.data_ptr()
        send = ws[oi:oi + n * self.w.d * esz].view(self._dt).view(n, self.w.d)
        back = ws[oo:oo + n * self.w.O * esz].view(self._dt).view(n, self.w.O)
        return out, send, back, list(rows)

    def ep_experts(self, recv_x, recv_rows, stream=None):
        """Phase 3: this rank's experts on the received rows (recv_rows: device
        int32 [G][E/G], padded rows per source and local expert). Returns [R][O]."""
        import torch
        R = int(recv_x.shape[0])
        recv_out = torch.empty(R, self.w.O, dtype=self._dt, device=self.device)
        need = lib().moe_ep_experts_workspace_bytes(self.handle, R)
        if getattr(self, "_ws2", None) is None or self._ws2.numel() < need:
            self._ws2 = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        rr = recv_rows.to(torch.int32).contiguous()
        _check(lib().moe_ep_experts(self.handle, _ptr(recv_x.contiguous()), rr.data_ptr(), R, recv_out.data_ptr(),
                                    self._ws2.data_ptr(), self._ws2.numel(), s), "moe_ep_experts")
        return recv_out

    def ep_combine(self, out, stream=None):
        """Phase 5: shared experts and the combine into out["y"]."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().moe_ep_combine(self.handle, _ptr(out["y"]), s), "moe_ep_combine")
        return out

    def ep_forward(self, x, noise=None, out=None, group=None):
        """The whole expert-parallel forward: dispatch, all-to-all of the rows
        (and of the per-expert row counts), this rank's experts, all-to-all
        back, combine. Every rank of `group` calls it at the same step."""
        G = self.cfg.ep_size
        out, send, back, rows = self.ep_dispatch(x, noise=noise, out=out)
        recv_x, recv_rows, send_splits, recv_splits = ep_exchange(send, rows, G, group)
        recv_out = self.ep_experts(recv_x, recv_rows)
        ep_return(recv_out, back, send_splits, recv_splits, group)
        return self.ep_combine(out)

    def device_status(self, stream=None) -> int:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        return moe_device_status(self.handle, s)

    def launch_count(self) -> int:
        return moe_launch_count(self.handle)


def ep_send_splits(expert_rows, G: int):
    """Rows this rank sends to each rank q: the padded segments of q's experts
    (experts q E/G .. (q+1) E/G - 1, contiguous in the row space)."""
    El = len(expert_rows) // G
    return [int(sum(expert_rows[q * El:(q + 1) * El])) for q in range(G)]


def ep_exchange(send_rows, expert_rows, G: int, group=None):
    """All-to-all dispatch: every rank sends each rank its E/G per-expert row
    counts and then its rows. Returns (received rows [R][d], received counts
    [G][E/G] (source-major, on the rows' device), send splits, receive splits)."""
    import torch
    import torch.distributed as dist
    El = len(expert_rows) // G
    dev = send_rows.device
    cnt_send = torch.tensor(expert_rows, dtype=torch.int32, device=dev)
    cnt_recv = torch.empty_like(cnt_send)
    dist.all_to_all_single(cnt_recv, cnt_send, group=group)
    send_splits = ep_send_splits(expert_rows, G)
    recv_counts = cnt_recv.view(G, El)
    recv_splits = [int(v) for v in recv_counts.sum(1).tolist()]
    recv = torch.empty(sum(recv_splits), send_rows.shape[1], dtype=send_rows.dtype, device=dev)
    dist.all_to_all_single(recv, send_rows[:sum(send_splits)].contiguous(), recv_splits, send_splits, group=group)
    return recv, recv_counts, send_splits, recv_splits


def ep_return(recv_out, back_rows, send_splits, recv_splits, group=None):
    """All-to-all combine: the expert outputs of the received rows go back to
    their sources, into the row positions their inputs left from."""
    import torch.distributed as dist
    n = sum(send_splits)
    if n == back_rows.shape[0] and back_rows.is_contiguous():
        dist.all_to_all_single(back_rows, recv_out, send_splits, recv_splits, group=group)
    else:
        tmp = back_rows.new_empty((n, back_rows.shape[1]))
        dist.all_to_all_single(tmp, recv_out, send_splits, recv_splits, group=group)
        back_rows[:n].copy_(tmp)


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

    def __init__(self, layer: "MoELayer", T: int, with_noise: bool = False, with_loss: bool = False,
                 use_graphs: bool = True):
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
                x=torch.zeros(T, w.d, dtype=layer._dt, device=dev),
                noise=torch.zeros(T, w.E, dtype=torch.float32, device=dev) if with_noise else None,
                loss=torch.zeros(T, dtype=torch.float32, device=dev) if with_loss else None,
                out=layer.alloc_outputs(T),
                uploaded=torch.cuda.Event(), computed=torch.cuda.Event(), downloaded=torch.cuda.Event(),
                used=False))
        layer.workspace(T)
        # Each slot's forward + statistics as one CUDA graph over its buffers.
        self.graphs = None
        if use_graphs:
            self.graphs = [StepGraph(layer, sl["x"], noise=sl["noise"], token_loss=sl["loss"], out=sl["out"])
                           for sl in self.slots]
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
            if self.graphs is not None:
                self.graphs[(self.n - 1) % 2].replay()
            else:
                s = self.comp.cuda_stream
                self.layer.forward(sl["x"], noise=sl["noise"], out=sl["out"], stream=s)
                self.layer.aux_stats(sl["out"], token_loss=sl["loss"], stream=s)
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


class StepGraph:
    """One forward + statistics captured as a CUDA graph over fixed device
    buffers (x, noise, token loss in; out's tensors written), so that a step
    replays as one graph launch instead of a dozen kernel launches. Refill the
    input tensors in place and call replay(); the layer's workspace and the
    output tensors are the ones the graph was captured with."""

    def __init__(self, layer: "MoELayer", x, noise=None, token_loss=None, out=None):
        import torch
        self.layer, self.x, self.noise, self.token_loss = layer, x, noise, token_loss
        T = int(x.shape[0])
        self.out = out if out is not None else layer.alloc_outputs(T)
        layer.workspace(T)  # allocate before capture
        side = torch.cuda.Stream(layer.device)
        side.wait_stream(torch.cuda.current_stream(layer.device))
        with torch.cuda.stream(side):  # one eager step: host-side set-up outside the capture
            self._step()
        torch.cuda.current_stream(layer.device).wait_stream(side)
        torch.cuda.synchronize(layer.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._step()

    def _step(self):
        self.layer.forward(self.x, noise=self.noise, out=self.out)
        self.layer.aux_stats(self.out, token_loss=self.token_loss)

    def replay(self):
        self.graph.replay()
        return self.out

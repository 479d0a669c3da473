"""ctypes binding of ``libbeam_moe.so`` (C ABI in ``include/beam_moe.h``).

Argument marshalling only: every step of the block runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If the
library is missing the first call raises; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np
import torch

from .build import LIB

BEAM_OK = 0
BEAM_ERR_INVALID_ARG = -1
BEAM_ERR_UNSUPPORTED = -2
BEAM_ERR_CUDA = -3
BEAM_ERR_OOM = -4
BEAM_ERR_TIMEOUT = -5
BEAM_ERR_CHECK = -6
BEAM_ERR_RANGE = -7

# every entry point declared in include/beam_moe.h
SYMBOLS = (
    "beam_moe_create", "beam_moe_create_dense", "beam_moe_create_nvfp4", "beam_nvfp4_dequant",
    "beam_moe_route", "beam_moe_route_static", "beam_moe_router_logits", "beam_moe_route_logits",
    "beam_moe_forward",
    "beam_moe_forward_host", "beam_moe_forward_host_async", "beam_moe_host_join",
    "beam_moe_host_fence",
    "beam_moe_dispatch_info", "beam_moe_router_stats", "beam_moe_launch_plan", "beam_moe_set_checks", "beam_moe_debug_corrupt_routing",
    "beam_moe_get_status",
    "beam_moe_set_wait_limit", "beam_moe_set_gemm_tuning", "beam_moe_set_gate_up_layout",
    "beam_moe_profile_begin",
    "beam_moe_profile_end", "beam_moe_check_wait_timeout", "beam_moe_last_error",
    "beam_moe_create_error", "beam_moe_destroy",
)

_lib = None


class BeamMoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"beam_moe error {code}: {msg}")
        self.code = code


def library() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing: build it with "
                               "`python -m group_limited_routing_sigmoid_b200.build`")
        lib = ctypes.CDLL(LIB)
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        lib.beam_moe_create.argtypes = [ctypes.POINTER(P), I, I, I, I, I, I, F, P, P, P, P, P, P, F, I]
        lib.beam_moe_route.argtypes = [P, P, P, I, P, P]
        lib.beam_moe_router_logits.argtypes = [P, P, P, I, P]
        lib.beam_moe_route_static.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P]
        lib.beam_moe_create_dense.argtypes = [P, I, I, P, P, P, P, ctypes.c_float, I]
        lib.beam_moe_create_nvfp4.argtypes = [ctypes.POINTER(P), I, I, I, I, I, I, F, P, P,
                                              P, P, F, P, P, F, P, P, F, P, F, I]
        lib.beam_nvfp4_dequant.argtypes = [P, P, P, ctypes.c_int64, I, P]
        lib.beam_moe_route_logits.argtypes = [P, P, P, I, P, P, P]
        lib.beam_moe_forward.argtypes = [P, P, P, I, P, P, I]
        lib.beam_moe_forward_host.argtypes = [P, P, P, I, P, P, I]
        lib.beam_moe_forward_host_async.argtypes = [P, P, P, I, P, P, I]
        lib.beam_moe_host_join.argtypes = [P, P]
        lib.beam_moe_host_fence.argtypes = [P, P]
        lib.beam_moe_dispatch_info.argtypes = [P, P, I, P, P, P]
        lib.beam_moe_get_status.argtypes = [P, P]
        lib.beam_moe_router_stats.argtypes = [P, P, P]
        lib.beam_moe_launch_plan.argtypes = [P, I, P]
        lib.beam_moe_set_checks.argtypes = [P, I]
        lib.beam_moe_debug_corrupt_routing.argtypes = [P, I]
        lib.beam_moe_set_wait_limit.argtypes = [P, ctypes.c_int64]
        lib.beam_moe_set_gemm_tuning.argtypes = [P, I, I, I, I, I, I, I]
        lib.beam_moe_set_gate_up_layout.argtypes = [P, I]
        lib.beam_moe_check_wait_timeout.argtypes = [P, P]
        lib.beam_moe_profile_begin.argtypes = [P, I]
        lib.beam_moe_profile_end.argtypes = [P, P, P]
        lib.beam_moe_last_error.argtypes = [P]
        lib.beam_moe_last_error.restype = ctypes.c_char_p
        lib.beam_moe_create_error.argtypes = []
        lib.beam_moe_create_error.restype = ctypes.c_char_p
        lib.beam_moe_destroy.argtypes = [P]
        for name in SYMBOLS:
            if name not in ("beam_moe_last_error", "beam_moe_create_error"):
                getattr(lib, name).restype = I
        _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev(t: torch.Tensor, dtype, name: str):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise TypeError(f"{name}: expected a contiguous CUDA {dtype} tensor, got "
                        f"{t.dtype} on {t.device} (contiguous={t.is_contiguous()})")
    return t


def route_static(x: torch.Tensor, router_w: torch.Tensor, expert_bias: torch.Tensor, n_group: int,
                 topk_group: int, top_k: int, idx: Optional[torch.Tensor] = None,
                 w: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Routing through beam_moe_route_static: no handle, no device allocation
    inside the library (its scratch is a fixed device array)."""
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.float32, "router_w")
    _dev(expert_bias, torch.float32, "expert_bias")
    T, H = x.shape
    E = router_w.shape[0]
    if idx is None:
        idx = torch.empty(T, top_k, dtype=torch.int32, device=x.device)
    if w is None:
        w = torch.empty(T, top_k, dtype=torch.float32, device=x.device)
    rc = library().beam_moe_route_static(_stream(stream), _ptr(x), T, H, E, n_group, topk_group,
                                         top_k, _ptr(router_w), _ptr(expert_bias), _ptr(idx), _ptr(w))
    if rc != BEAM_OK:
        raise BeamMoEError(rc, "beam_moe_route_static rejected the call")
    return idx, w


def nvfp4_dequant(codes: torch.Tensor, scales: torch.Tensor, stream=None) -> torch.Tensor:
    """beam_nvfp4_dequant: codes uint8 [..., K/2], scales uint8 [..., K/16] ->
    bf16 [..., K], each element times its block scale (no per-tensor scale)."""
    _dev(codes, torch.uint8, "codes")
    _dev(scales, torch.uint8, "scales")
    K = codes.shape[-1] * 2
    rows = codes.numel() // max(codes.shape[-1], 1)
    if scales.shape[:-1] != codes.shape[:-1] or scales.shape[-1] * 16 != K:
        raise ValueError("scales must be [..., K/16] for codes [..., K/2]")
    out = torch.empty(*codes.shape[:-1], K, dtype=torch.bfloat16, device=codes.device)
    rc = library().beam_nvfp4_dequant(_stream(stream), _ptr(codes), _ptr(scales), rows, K, _ptr(out))
    if rc != BEAM_OK:
        raise BeamMoEError(rc, "beam_nvfp4_dequant rejected the call")
    return out


class BeamMoE:
    """One MoE block on the current CUDA device (borrows the weight tensors)."""

    def __init__(self, hidden: int, n_experts: int, inter: int, n_group: int, topk_group: int,
                 top_k: int, routed_scaling: float, router_w: torch.Tensor, expert_bias: torch.Tensor,
                 w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                 post_norm_w: Optional[torch.Tensor] = None, norm_eps: float = 1e-6,
                 max_tokens: int = 64):
        lib = library()
        _dev(router_w, torch.float32, "router_w")
        _dev(expert_bias, torch.float32, "expert_bias")
        for n, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
            _dev(t, torch.bfloat16, n)
        if post_norm_w is not None:
            _dev(post_norm_w, torch.float32, "post_norm_w")
        self._keep = (router_w, expert_bias, w_gate, w_up, w_down, post_norm_w)
        self.hidden, self.n_experts, self.inter = hidden, n_experts, inter
        self.top_k = top_k
        self.max_tokens = max_tokens
        self.device = router_w.device
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            rc = lib.beam_moe_create(ctypes.byref(h), hidden, n_experts, inter, n_group, topk_group,
                                     top_k, float(routed_scaling), _ptr(router_w), _ptr(expert_bias),
                                     _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(post_norm_w),
                                     float(norm_eps), max_tokens)
        if rc != BEAM_OK:
            raise BeamMoEError(rc, lib.beam_moe_create_error().decode())
        self._h = h

    @classmethod
    def dense(cls, hidden: int, inter: int, w_gate: torch.Tensor, w_up: torch.Tensor,
              w_down: torch.Tensor, post_norm_w: Optional[torch.Tensor] = None,
              norm_eps: float = 1e-6, max_tokens: int = 64) -> "BeamMoE":
        """A dense SwiGLU MLP layer (beam_moe_create_dense): forward only."""
        lib = library()
        for n, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
            _dev(t, torch.bfloat16, n)
        if post_norm_w is not None:
            _dev(post_norm_w, torch.float32, "post_norm_w")
        self = cls.__new__(cls)
        self._keep = (w_gate, w_up, w_down, post_norm_w)
        self.hidden, self.n_experts, self.inter, self.top_k = hidden, 1, inter, 1
        self.max_tokens = max_tokens
        self.device = w_gate.device
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            rc = lib.beam_moe_create_dense(ctypes.byref(h), hidden, inter, _ptr(w_gate), _ptr(w_up),
                                           _ptr(w_down), _ptr(post_norm_w), float(norm_eps), max_tokens)
        if rc != BEAM_OK:
            raise BeamMoEError(rc, lib.beam_moe_create_error().decode())
        self._h = h
        return self

    @classmethod
    def nvfp4(cls, hidden: int, n_experts: int, inter: int, n_group: int, topk_group: int,
              top_k: int, routed_scaling: float, router_w: torch.Tensor, expert_bias: torch.Tensor,
              gate: Tuple[torch.Tensor, torch.Tensor, float], up: Tuple[torch.Tensor, torch.Tensor, float],
              down: Tuple[torch.Tensor, torch.Tensor, float],
              post_norm_w: Optional[torch.Tensor] = None, norm_eps: float = 1e-6,
              max_tokens: int = 64) -> "BeamMoE":
        """A block with NVFP4 expert weights (beam_moe_create_nvfp4): each of
        gate, up, down is (codes uint8 [E, R, K/2], scales uint8 [E, R, K/16],
        per-tensor scale).  The handle keeps its own copy of the weights."""
        lib = library()
        _dev(router_w, torch.float32, "router_w")
        _dev(expert_bias, torch.float32, "expert_bias")
        for n, (c, sc, _) in (("gate", gate), ("up", up), ("down", down)):
            _dev(c, torch.uint8, n + "_codes")
            _dev(sc, torch.uint8, n + "_scales")
        if post_norm_w is not None:
            _dev(post_norm_w, torch.float32, "post_norm_w")
        self = cls.__new__(cls)
        self._keep = (router_w, expert_bias, post_norm_w)
        self.hidden, self.n_experts, self.inter = hidden, n_experts, inter
        self.top_k = top_k
        self.max_tokens = max_tokens
        self.device = router_w.device
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            rc = lib.beam_moe_create_nvfp4(
                ctypes.byref(h), hidden, n_experts, inter, n_group, topk_group, top_k,
                float(routed_scaling), _ptr(router_w), _ptr(expert_bias),
                _ptr(gate[0]), _ptr(gate[1]), float(gate[2]), _ptr(up[0]), _ptr(up[1]), float(up[2]),
                _ptr(down[0]), _ptr(down[1]), float(down[2]), _ptr(post_norm_w), float(norm_eps),
                max_tokens)
        if rc != BEAM_OK:
            raise BeamMoEError(rc, lib.beam_moe_create_error().decode())
        self._h = h
        return self

    @classmethod
    def from_workload(cls, wl, weights, max_tokens: Optional[int] = None) -> "BeamMoE":
        if wl.n_experts == 1:
            return cls.dense(wl.hidden, wl.inter, weights["w_gate"][0], weights["w_up"][0],
                             weights["w_down"][0], weights.get("gamma"), wl.norm_eps,
                             max_tokens or wl.T)
        if getattr(wl, "weight_format", "bf16") == "nvfp4":
            t = lambda n: (weights[n + "_codes"], weights[n + "_scales"], weights[n + "_global"])
            return cls.nvfp4(wl.hidden, wl.n_experts, wl.inter, wl.n_group, wl.topk_group, wl.top_k,
                             wl.routed_scaling, weights["router_w"], weights["bias"], t("gate"),
                             t("up"), t("down"), weights.get("gamma"), wl.norm_eps,
                             max_tokens or wl.T)
        return cls(wl.hidden, wl.n_experts, wl.inter, wl.n_group, wl.topk_group, wl.top_k,
                   wl.routed_scaling, weights["router_w"], weights["bias"], weights["w_gate"],
                   weights["w_up"], weights["w_down"], weights.get("gamma"), wl.norm_eps,
                   max_tokens or wl.T)

    def _check(self, rc: int):
        if rc != BEAM_OK:
            raise BeamMoEError(rc, library().beam_moe_last_error(self._h).decode())

    def route(self, x: torch.Tensor, idx: Optional[torch.Tensor] = None,
              w: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
        _dev(x, torch.bfloat16, "x")
        T = x.shape[0]
        if idx is None:
            idx = torch.empty(T, self.top_k, dtype=torch.int32, device=x.device)
        if w is None:
            w = torch.empty(T, self.top_k, dtype=torch.float32, device=x.device)
        self._check(library().beam_moe_route(self._h, _stream(stream), _ptr(x), T, _ptr(idx), _ptr(w)))
        return idx, w

    def router_logits(self, x: torch.Tensor, logits: Optional[torch.Tensor] = None, stream=None):
        _dev(x, torch.bfloat16, "x")
        T = x.shape[0]
        if logits is None:
            logits = torch.empty(T, self.n_experts, dtype=torch.float32, device=x.device)
        self._check(library().beam_moe_router_logits(self._h, _stream(stream), _ptr(x), T, _ptr(logits)))
        return logits

    def route_logits(self, logits: torch.Tensor, expert_bias: Optional[torch.Tensor] = None,
                     idx: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Routing from given FP32 logits [T, E], under `expert_bias` (fp32 [E])
        or the handle's bias."""
        _dev(logits, torch.float32, "logits")
        if expert_bias is not None:
            _dev(expert_bias, torch.float32, "expert_bias")
        T = logits.shape[0]
        if idx is None:
            idx = torch.empty(T, self.top_k, dtype=torch.int32, device=logits.device)
        if w is None:
            w = torch.empty(T, self.top_k, dtype=torch.float32, device=logits.device)
        self._check(library().beam_moe_route_logits(
            self._h, _stream(stream), _ptr(logits), T,
            None if expert_bias is None else _ptr(expert_bias), _ptr(idx), _ptr(w)))
        return idx, w

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                residual: Optional[torch.Tensor] = None, k: int = 1, want_out: bool = True,
                stream=None) -> Optional[torch.Tensor]:
        _dev(x, torch.bfloat16, "x")
        T = x.shape[0]
        if out is None and want_out:
            out = torch.empty(T, self.hidden, dtype=torch.bfloat16, device=x.device)
        if residual is not None:
            _dev(residual, torch.float32, "residual")
        self._check(library().beam_moe_forward(self._h, _stream(stream), _ptr(x), T, _ptr(out),
                                                _ptr(residual), int(k)))
        return out

    def forward_host(self, x_host: torch.Tensor, out_host: Optional[torch.Tensor] = None,
                     residual_host: Optional[torch.Tensor] = None, k: int = 1, stream=None):
        """Host buffers in, host buffers out (copies inside the call)."""
        assert not x_host.is_cuda and x_host.dtype == torch.bfloat16 and x_host.is_contiguous()
        T = x_host.shape[0]
        self._check(library().beam_moe_forward_host(self._h, _stream(stream), _ptr(x_host), T,
                                                     _ptr(out_host), _ptr(residual_host), int(k)))
        return out_host

    def forward_host_async(self, x_host: torch.Tensor, out_host: Optional[torch.Tensor] = None,
                           residual_host: Optional[torch.Tensor] = None, k: int = 1, stream=None):
        """Pipelined host-buffer pass: returns at once; host_join + a stream
        synchronise before reading the results."""
        assert not x_host.is_cuda and x_host.dtype == torch.bfloat16 and x_host.is_contiguous()
        T = x_host.shape[0]
        self._check(library().beam_moe_forward_host_async(self._h, _stream(stream), _ptr(x_host), T,
                                                           _ptr(out_host), _ptr(residual_host), int(k)))
        return out_host

    def host_join(self, stream=None):
        self._check(library().beam_moe_host_join(self._h, _stream(stream)))

    def host_fence(self, stream=None):
        self._check(library().beam_moe_host_fence(self._h, _stream(stream)))

    def dispatch_info(self, T: int, stream=None):
        counts = np.empty(self.n_experts, np.int32)
        offsets = np.empty(self.n_experts + 1, np.int32)
        pair_row = np.empty(T * self.top_k, np.int32)
        self._check(library().beam_moe_dispatch_info(
            self._h, _stream(stream), T, counts.ctypes.data_as(ctypes.c_void_p),
            offsets.ctypes.data_as(ctypes.c_void_p), pair_row.ctypes.data_as(ctypes.c_void_p)))
        return counts, offsets, pair_row

    def router_stats(self, stream=None) -> int:
        """Tokens of the last call whose routing was re-derived on the exact path."""
        n = ctypes.c_int32()
        self._check(library().beam_moe_router_stats(self._h, _stream(stream),
                                                     ctypes.cast(ctypes.pointer(n), ctypes.c_void_p)))
        return n.value

    def launch_plan(self, T: int) -> dict:
        """The kernels and launch shapes a forward pass of T tokens uses."""
        p = (ctypes.c_int32 * 11)()
        self._check(library().beam_moe_launch_plan(self._h, int(T), ctypes.cast(p, ctypes.c_void_p)))
        keys = ("tile_rows", "cta_pairs", "grid", "down_paired", "router_tensor_cores", "router_slices",
                "gather_rows", "stream_k_gate_up", "stream_k_down", "y_f32", "gate_up_interleaved")
        return dict(zip(keys, (int(v) for v in p)))

    def set_checks(self, on: bool = True):
        """Checked mode: validate routing and dispatch tables on the device."""
        self._check(library().beam_moe_set_checks(self._h, int(bool(on))))

    def debug_corrupt_routing(self, passes: int = 1):
        """Test hook (checked mode only): corrupt the next passes' routing."""
        self._check(library().beam_moe_debug_corrupt_routing(self._h, int(passes)))

    def last_error(self) -> str:
        return library().beam_moe_last_error(self._h).decode()

    def get_status(self, stream=None) -> int:
        return library().beam_moe_get_status(self._h, _stream(stream))

    def set_wait_limit(self, limit_ns: int):
        self._check(library().beam_moe_set_wait_limit(self._h, int(limit_ns)))

    def set_gemm_tuning(self, ctas: int = 0, tile_rows: int = 0, down_pair: int = -1,
                        cta_pairs: int = 1, router_mode: int = -1, gather_rows: int = -1,
                        token_stages: int = 0):
        self._check(library().beam_moe_set_gemm_tuning(self._h, int(ctas), int(tile_rows),
                                                        int(down_pair), int(cta_pairs),
                                                        int(router_mode), int(gather_rows),
                                                        int(token_stages)))

    STAGES = ("router", "dispatch", "gate_up_gemm", "down_gemm", "combine")

    def set_gate_up_layout(self, layout: int = -1):
        """0: separate gate and up tiles, 1: interleaved, -1: automatic."""
        self._check(library().beam_moe_set_gate_up_layout(self._h, int(layout)))

    def profile_begin(self, max_calls: int):
        self._check(library().beam_moe_profile_begin(self._h, int(max_calls)))

    def profile_end(self):
        """-> (calls, {stage: total ms}) over the forward passes since profile_begin."""
        ms = (ctypes.c_float * 5)()
        calls = ctypes.c_int()
        self._check(library().beam_moe_profile_end(self._h, ctypes.cast(ms, ctypes.c_void_p),
                                                    ctypes.cast(ctypes.pointer(calls), ctypes.c_void_p)))
        return calls.value, dict(zip(self.STAGES, [float(v) for v in ms]))

    def check_wait_timeout(self, stream=None) -> int:
        return library().beam_moe_check_wait_timeout(self._h, _stream(stream))

    def close(self):
        if getattr(self, "_h", None):
            library().beam_moe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

"""Plain fp64 CPU oracle for the Beam sparse MoE block (forward pass).

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path (the
CUDA library and its Python binding) never imports this package, and this
package imports nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, double accumulation in index
order, OpenMP over independent tokens or rows only).  This module compiles
it with gcc, loads it with ctypes and marshals numpy arrays; it adds no
arithmetic of its own apart from composing the C steps in the order the
pages give them (route -> per-expert SwiGLU -> weighted combine x 2.5 ->
optional post-norm + depth-scaled residual).

Sources (the Beam pages):
  * launch blog "Introducing Beam", section "Mixture of Experts" (router
    recipe, 256 experts, 8 groups of 32, top-2 group score, 4 groups kept,
    top-8, normalised weights, x2.5) and section "Residual Stream"
    (depth-scaled residual, sandwich norms, FP32 sites);
  * transformers documentation page "Beam", section "Overview", bullets
    "Sparse MoE" and "Depth-scaled residual and sandwich norm", and the
    closing paragraph on FP32 router weights and expert bias.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Callable, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.oracle_route.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_route.restype = I
        lib.oracle_route_logits.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_route_logits.restype = I
        lib.oracle_expert_swiglu.argtypes = [I, I, I, P, P, P, P, P, P]
        lib.oracle_expert_swiglu.restype = None
        lib.oracle_expert_swiglu_nvfp4.argtypes = [I, I, I, P, P, P, P, P, P, P, D, D, D, P, P]
        lib.oracle_expert_swiglu_nvfp4.restype = None
        lib.oracle_e2m1_value.argtypes = [ctypes.c_uint]
        lib.oracle_e2m1_value.restype = D
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint]
        lib.oracle_e4m3_value.restype = D
        lib.oracle_combine.argtypes = [I, I, I, P, P, D, P, P]
        lib.oracle_combine.restype = None
        lib.oracle_post_norm_residual.argtypes = [I, I, P, P, D, I, P, P, P]
        lib.oracle_post_norm_residual.restype = None
        lib.oracle_double_to_bf16.argtypes = [D]
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = D
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, f"bf16 inputs are passed as their uint16 bit patterns, got {a.dtype}"
    return a


def _f32(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.float32, f"expected float32, got {a.dtype}"
    return a


# ---------------------------------------------------------------------------
# bf16 helpers (bit patterns as uint16)
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: bf16 is the top half of binary32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(values: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 (ties to even), via the C routine, element by element."""
    lib = _load()
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    flat_in, flat_out = v.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = lib.oracle_double_to_bf16(float(flat_in[i]))
    return out


# ---------------------------------------------------------------------------
# Steps
# ---------------------------------------------------------------------------

@dataclass
class Routing:
    idx: np.ndarray          # int32 [T, k]
    w: np.ndarray            # float64 [T, k], sums to 1 per token
    scores: np.ndarray       # float64 [T, E] sigmoid(logit)
    biased: np.ndarray       # float64 [T, E] sigmoid(logit) + bias
    gap_expert: np.ndarray   # float64 [T]
    gap_group: np.ndarray    # float64 [T]
    kept_mask: np.ndarray    # int32 [T], bit j = group j kept
    gap_order: np.ndarray    # float64 [T] smallest neighbour gap within the chosen sequence


def route(x_bits: np.ndarray, router_w: np.ndarray, bias: np.ndarray,
          n_group: int, topk_group: int, top_k: int) -> Routing:
    """Group-limited sigmoid routing (launch blog, "Mixture of Experts")."""
    lib = _load()
    x = _u16(x_bits)
    wr = _f32(router_w)
    b = _f32(bias)
    T, H = x.shape
    E = wr.shape[0]
    assert wr.shape == (E, H) and b.shape == (E,)
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    scores = np.empty((T, E), np.float64)
    biased = np.empty((T, E), np.float64)
    ge = np.empty((T,), np.float64)
    gg = np.empty((T,), np.float64)
    km = np.empty((T,), np.int32)
    go = np.empty((T,), np.float64)
    rc = lib.oracle_route(T, H, E, n_group, topk_group, top_k, _ptr(x), _ptr(wr), _ptr(b),
                          _ptr(idx), _ptr(w), _ptr(scores), _ptr(biased), _ptr(ge), _ptr(gg), _ptr(km),
                          _ptr(go))
    if rc != 0:
        raise ValueError("oracle_route: routing configuration not defined by the method")
    return Routing(idx, w, scores, biased, ge, gg, km, go)


def route_logits(logits: np.ndarray, bias: np.ndarray, n_group: int, topk_group: int,
                 top_k: int) -> Routing:
    """The same routing from given FP32 logits [T, E] (selection only): what a
    re-route under another expert bias computes.  scores/biased are left
    empty."""
    lib = _load()
    lg = _f32(logits)
    b = _f32(bias)
    T, E = lg.shape
    assert b.shape == (E,)
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    ge = np.empty((T,), np.float64)
    gg = np.empty((T,), np.float64)
    km = np.empty((T,), np.int32)
    go = np.empty((T,), np.float64)
    rc = lib.oracle_route_logits(T, E, n_group, topk_group, top_k, _ptr(lg), _ptr(b), _ptr(idx),
                                 _ptr(w), _ptr(ge), _ptr(gg), _ptr(km), _ptr(go))
    if rc != 0:
        raise ValueError("oracle_route_logits: routing configuration not defined by the method")
    empty = np.empty((T, 0), np.float64)
    return Routing(idx, w, empty, empty, ge, gg, km, go)


def expert_swiglu(x_bits: np.ndarray, w_gate_bits: np.ndarray, w_up_bits: np.ndarray,
                  w_down_bits: np.ndarray, want_h: bool = False):
    """One SwiGLU expert on n rows; returns y float64 [n, H] (and h bf16 bits [n, I])."""
    lib = _load()
    x = _u16(x_bits)
    wg, wu, wd = _u16(w_gate_bits), _u16(w_up_bits), _u16(w_down_bits)
    n, H = x.shape
    I = wg.shape[0]
    assert wg.shape == (I, H) and wu.shape == (I, H) and wd.shape == (H, I)
    y = np.empty((n, H), np.float64)
    h = np.empty((n, I), np.uint16) if want_h else None
    if n:
        lib.oracle_expert_swiglu(n, H, I, _ptr(x), _ptr(wg), _ptr(wu), _ptr(wd), _ptr(y), _ptr(h))
    return (y, h) if want_h else y


def e2m1_value(code: int) -> float:
    """An E2M1 code (4 bits) -> its value (the C decoder, from the format's definition)."""
    return _load().oracle_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    """An FP8 E4M3 byte -> its value (the C decoder)."""
    return _load().oracle_e4m3_value(int(byte))


@dataclass
class Nvfp4Matrix:
    """One NVFP4 weight tensor: codes uint8 [..., R, K/2] (element 2j in the low
    nibble of byte j), scales uint8 [..., R, K/16] (E4M3), a per-tensor scale."""
    codes: np.ndarray
    scales: np.ndarray
    global_scale: float


def expert_swiglu_nvfp4(x_bits: np.ndarray, gate: Nvfp4Matrix, up: Nvfp4Matrix,
                        down: Nvfp4Matrix, want_h: bool = False):
    """One SwiGLU expert with NVFP4 matrices (gate, up [I, H], down [H, I])."""
    lib = _load()
    x = _u16(x_bits)
    n, H = x.shape
    I = gate.codes.shape[0]
    u8 = lambda a: np.ascontiguousarray(a, dtype=np.uint8)
    gc, gs, uc, us, dc, ds = (u8(gate.codes), u8(gate.scales), u8(up.codes), u8(up.scales),
                              u8(down.codes), u8(down.scales))
    assert gc.shape == (I, H // 2) and gs.shape == (I, H // 16)
    assert uc.shape == (I, H // 2) and us.shape == (I, H // 16)
    assert dc.shape == (H, I // 2) and ds.shape == (H, I // 16)
    y = np.empty((n, H), np.float64)
    h = np.empty((n, I), np.uint16) if want_h else None
    if n:
        lib.oracle_expert_swiglu_nvfp4(n, H, I, _ptr(x), _ptr(gc), _ptr(gs), _ptr(uc), _ptr(us),
                                       _ptr(dc), _ptr(ds), float(gate.global_scale),
                                       float(up.global_scale), float(down.global_scale),
                                       _ptr(y), _ptr(h))
    return (y, h) if want_h else y


def combine(y: np.ndarray, w: np.ndarray, scale: float):
    """o = scale * sum_j w_j y_j in slot order; returns (o float64 [T,H], out bf16 bits [T,H])."""
    lib = _load()
    y = np.ascontiguousarray(y, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, k, H = y.shape
    assert w.shape == (T, k)
    o = np.empty((T, H), np.float64)
    out = np.empty((T, H), np.uint16)
    lib.oracle_combine(T, H, k, _ptr(y), _ptr(w), float(scale), _ptr(o), _ptr(out))
    return o, out


def post_norm_residual(o: np.ndarray, gamma: Optional[np.ndarray], eps: float, kstep: int,
                       stream: np.ndarray):
    """Post-MoE RMSNorm (optional) + depth-scaled residual at step ``kstep``.

    Returns (contrib float64 [T,H], stream_out float64 [T,H]).
    """
    lib = _load()
    o = np.ascontiguousarray(o, dtype=np.float64)
    T, H = o.shape
    g = None if gamma is None else _f32(gamma)
    s = _f32(stream)
    assert s.shape == (T, H)
    contrib = np.empty((T, H), np.float64)
    s_out = np.empty((T, H), np.float64)
    lib.oracle_post_norm_residual(T, H, _ptr(o), _ptr(g), float(eps), int(kstep), _ptr(s),
                                  _ptr(contrib), _ptr(s_out))
    return contrib, s_out


# ---------------------------------------------------------------------------
# Whole block
# ---------------------------------------------------------------------------

@dataclass
class BlockResult:
    routing: Routing
    y: np.ndarray            # float64 [T, k, H] per-slot expert outputs
    o: np.ndarray            # float64 [T, H] scaled combine (pre-rounding)
    out: np.ndarray          # bf16 bits [T, H]
    contrib: Optional[np.ndarray] = None
    stream_out: Optional[np.ndarray] = None


ExpertFetch = Callable[[int], "tuple[np.ndarray, np.ndarray, np.ndarray]"]


def moe_block(x_bits: np.ndarray, router_w: np.ndarray, bias: np.ndarray,
              fetch_expert: ExpertFetch, n_group: int, topk_group: int, top_k: int,
              routed_scaling: float, gamma: Optional[np.ndarray] = None, eps: float = 1e-6,
              stream: Optional[np.ndarray] = None, kstep: int = 0,
              on_expert: Optional[Callable[[int, int], None]] = None) -> BlockResult:
    """The block's forward pass on the tokens in ``x_bits``.

    ``fetch_expert(e)`` returns expert e's (w_gate [I,H], w_up [I,H],
    w_down [H,I]) as bf16 bit patterns or as three Nvfp4Matrix; it is called
    once per expert that the tokens route to, so that the caller can stream
    large weight sets.
    Steps: route; for every (token, slot) run the slot's expert; combine in
    slot order x routed_scaling; round to bf16; optionally post-norm and
    residual update at step ``kstep``.
    """
    x = _u16(x_bits)
    T, H = x.shape
    r = route(x, router_w, bias, n_group, topk_group, top_k)
    y = np.zeros((T, top_k, H), np.float64)
    experts = sorted(set(int(e) for e in r.idx.reshape(-1)))
    for e in experts:
        tt, jj = np.nonzero(r.idx == e)
        mats = fetch_expert(e)
        if isinstance(mats[0], Nvfp4Matrix):
            ye = expert_swiglu_nvfp4(np.ascontiguousarray(x[tt]), *mats)
        else:
            ye = expert_swiglu(np.ascontiguousarray(x[tt]), *mats)
        y[tt, jj, :] = ye
        if on_expert is not None:
            on_expert(e, len(tt))
    o, out = combine(y, r.w, routed_scaling)
    res = BlockResult(r, y, o, out)
    if stream is not None:
        res.contrib, res.stream_out = post_norm_residual(o, gamma, eps, kstep, stream)
    return res


def dense_block(x_bits: np.ndarray, w_gate_bits: np.ndarray, w_up_bits: np.ndarray,
                w_down_bits: np.ndarray, gamma: Optional[np.ndarray] = None, eps: float = 1e-6,
                stream: Optional[np.ndarray] = None, kstep: int = 0) -> BlockResult:
    """A dense SwiGLU MLP layer (the blog's first three layers) on the tokens
    in ``x_bits``: the one-expert SwiGLU, its output rounded to bf16, and the
    same optional post-norm and residual update as the sparse block.  It
    composes the steps above with one slot of weight 1 and no scaling; no
    routing."""
    x = _u16(x_bits)
    T = x.shape[0]
    y = expert_swiglu(x, w_gate_bits, w_up_bits, w_down_bits)
    o, out = combine(y.reshape(T, 1, -1), np.ones((T, 1)), 1.0)
    empty = np.empty((T, 0))
    routing = Routing(np.zeros((T, 1), np.int32), np.ones((T, 1)), empty, empty,
                      np.full(T, np.inf), np.full(T, np.inf), np.ones(T, np.int32), np.full(T, np.inf))
    res = BlockResult(routing, y.reshape(T, 1, -1), o, out)
    if stream is not None:
        res.contrib, res.stream_out = post_norm_residual(o, gamma, eps, kstep, stream)
    return res


def dense_fetch(w_gate_bits: np.ndarray, w_up_bits: np.ndarray, w_down_bits: np.ndarray) -> ExpertFetch:
    """fetch_expert over in-memory [E, ...] weight arrays."""
    return lambda e: (np.ascontiguousarray(w_gate_bits[e]), np.ascontiguousarray(w_up_bits[e]),
                      np.ascontiguousarray(w_down_bits[e]))


def threads() -> int:
    """Host threads the oracle's OpenMP loops may use."""
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else len(os.sched_getaffinity(0))

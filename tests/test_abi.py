"""The C ABI library: loads without a GPU, exports every entry point the
header declares, and rejects invalid arguments on the host (no GPU needed:
validation runs before any CUDA call)."""
import ctypes
import os
import re

import pytest

from group_limited_routing_sigmoid_b200 import binding
from group_limited_routing_sigmoid_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build(quiet=True)
    return binding.library()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(beam_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 10
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert names == set(binding.SYMBOLS)


def _create(lib, **kw):
    args = dict(hidden=5120, n_experts=256, inter=2560, n_group=8, topk_group=4, top_k=8,
                scaling=2.5, rw=16, b=16, wg=16, wu=16, wd=16, gamma=None, eps=1e-6, max_tokens=64)
    args.update(kw)
    h = ctypes.c_void_p()
    P = lambda v: None if v is None else ctypes.c_void_p(v)
    rc = lib.beam_moe_create(ctypes.byref(h), args["hidden"], args["n_experts"], args["inter"],
                             args["n_group"], args["topk_group"], args["top_k"], args["scaling"],
                             P(args["rw"]), P(args["b"]), P(args["wg"]), P(args["wu"]), P(args["wd"]),
                             P(args["gamma"]), args["eps"], args["max_tokens"])
    return rc, lib.beam_moe_create_error().decode()


@pytest.mark.parametrize("kw, code", [
    (dict(n_group=7), binding.BEAM_ERR_INVALID_ARG),          # 256 % 7
    (dict(n_group=256), binding.BEAM_ERR_INVALID_ARG),        # group size 1
    (dict(topk_group=0), binding.BEAM_ERR_INVALID_ARG),
    (dict(topk_group=9), binding.BEAM_ERR_INVALID_ARG),
    (dict(top_k=0), binding.BEAM_ERR_INVALID_ARG),
    (dict(top_k=129), binding.BEAM_ERR_INVALID_ARG),          # > 4 groups x 32
    (dict(max_tokens=0), binding.BEAM_ERR_INVALID_ARG),
    (dict(rw=None), binding.BEAM_ERR_INVALID_ARG),
    (dict(wg=24), binding.BEAM_ERR_INVALID_ARG),              # misaligned pointer
    (dict(hidden=5000), binding.BEAM_ERR_UNSUPPORTED),        # not a multiple of 128
    (dict(inter=2500), binding.BEAM_ERR_UNSUPPORTED),
    (dict(n_experts=96, n_group=3, topk_group=2), binding.BEAM_ERR_UNSUPPORTED),
    (dict(top_k=40, topk_group=8), binding.BEAM_ERR_UNSUPPORTED),
])
def test_create_rejects_invalid_arguments(lib, kw, code):
    rc, msg = _create(lib, **kw)
    assert rc == code, msg
    assert msg


def _create_nvfp4(lib, **kw):
    args = dict(hidden=5120, n_experts=256, inter=2560, n_group=8, topk_group=4, top_k=8,
                scaling=2.5, rw=16, b=16, gc=16, gs=16, gg=1.0, uc=16, us=16, ug=1.0, dc=16, ds=16,
                dg=1.0, gamma=None, eps=1e-6, max_tokens=64)
    args.update(kw)
    h = ctypes.c_void_p()
    P = lambda v: None if v is None else ctypes.c_void_p(v)
    rc = lib.beam_moe_create_nvfp4(
        ctypes.byref(h), args["hidden"], args["n_experts"], args["inter"], args["n_group"],
        args["topk_group"], args["top_k"], args["scaling"], P(args["rw"]), P(args["b"]),
        P(args["gc"]), P(args["gs"]), args["gg"], P(args["uc"]), P(args["us"]), args["ug"],
        P(args["dc"]), P(args["ds"]), args["dg"], P(args["gamma"]), args["eps"], args["max_tokens"])
    return rc, lib.beam_moe_create_error().decode()


@pytest.mark.parametrize("kw, code", [
    (dict(n_group=7), binding.BEAM_ERR_INVALID_ARG),
    (dict(top_k=0), binding.BEAM_ERR_INVALID_ARG),
    (dict(gc=None), binding.BEAM_ERR_INVALID_ARG),
    (dict(ds=None), binding.BEAM_ERR_INVALID_ARG),
    (dict(us=24), binding.BEAM_ERR_INVALID_ARG),              # misaligned pointer
    (dict(gg=float("inf")), binding.BEAM_ERR_INVALID_ARG),
    (dict(dg=float("nan")), binding.BEAM_ERR_INVALID_ARG),
    (dict(hidden=5000), binding.BEAM_ERR_UNSUPPORTED),
    (dict(inter=2500), binding.BEAM_ERR_UNSUPPORTED),
])
def test_create_nvfp4_rejects_invalid_arguments(lib, kw, code):
    rc, msg = _create_nvfp4(lib, **kw)
    assert rc == code, msg
    assert msg


def test_nvfp4_dequant_rejects_invalid_arguments(lib):
    P = ctypes.c_void_p
    assert lib.beam_nvfp4_dequant(None, P(16), P(16), 4, 24, P(16)) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_nvfp4_dequant(None, P(16), P(16), -1, 32, P(16)) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_nvfp4_dequant(None, None, P(16), 4, 32, P(16)) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_nvfp4_dequant(None, P(24), P(16), 4, 32, P(16)) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_nvfp4_dequant(None, None, None, 0, 32, None) == binding.BEAM_OK   # nothing to do


def test_calls_on_null_handle_fail_cleanly(lib):
    assert lib.beam_moe_route(None, None, None, 0, None, None) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_forward(None, None, None, 0, None, None, 1) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_destroy(None) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_get_status(None, None) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_launch_plan(None, 1, None) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_set_checks(None, 1) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_debug_corrupt_routing(None, 1) == binding.BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_route_logits(None, None, None, 1, None, None, None) == binding.BEAM_ERR_INVALID_ARG


def test_product_path_has_no_fallback(monkeypatch, tmp_path):
    """A missing CUDA library is an error, not a silent CPU path."""
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        binding.library()

"""The dense SwiGLU MLP layer (beam_moe_create_dense) against the oracle's
dense_block: stream-K and grouped-GEMM paths, ragged token counts, the post-norm and
residual update, and the Beam-shaped layer (H=5120, intermediate 20480)."""
import dataclasses
import json
import os

import pytest
import torch

from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import BEAM_ERR_UNSUPPORTED, BeamMoE, BeamMoEError
from group_limited_routing_sigmoid_b200.build import build

from parity import check_dense

pytestmark = pytest.mark.gpu


def setup_module(_):
    build(quiet=True)


def _inputs(wl, T=None):
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    return d


def _log(case, rep, plan):
    path = os.environ.get("BEAM_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, **rep.__dict__, "plan": plan}) + "\n")


# (T, GEMM CTAs, largest token tile (0 = auto), CTA pairs, post-norm + residual)
DENSE_CASES = [(1, 0, 0, 1, False), (3, 0, 0, 1, False), (37, 5, 0, 1, False), (64, 0, 0, 1, False),
               (100, 0, 0, 1, False), (300, 0, 0, 1, False), (1000, 3, 0, 1, False),
               (1000, 0, 0, 0, False), (64, 0, 256, 1, False), (300, 0, 16, 1, False),
               (64, 0, 0, 1, True), (300, 0, 0, 1, True), (300, 0, 16, 1, True),
               (64, 7, 0, 1, False), (37, 1, 0, 1, False), (64, 0, 32, 1, False),
               (200, 5, 16, 1, False)]


@pytest.mark.parametrize("T,ctas,tile,pairs,resid", DENSE_CASES)
def test_dense_layer(T, ctas, tile, pairs, resid):
    wl = W.WORKLOADS["dense_tiny"]
    if resid:
        wl = dataclasses.replace(wl, post_norm=True, residual_k=20)
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(ctas, tile, -1, pairs)
    plan = moe.launch_plan(T)
    rep = check_dense(wl, d, moe)
    _log(f"dense_T{T}_ctas{ctas}_tile{tile}_pairs{pairs}_resid{resid}", rep, plan)
    assert rep.ok(), rep
    if resid:
        assert rep.res_rel_fro is not None
    moe.close()


def test_dense_plan_streams_k_for_few_tokens():
    wl = W.WORKLOADS["dense_decode"]
    g = W.generator(wl, "cuda")
    # the plan depends on the shapes only: small stand-in weights of the right size are enough
    w = dict(w_gate=torch.zeros(1, wl.inter, wl.hidden, dtype=torch.bfloat16, device="cuda"),
             w_up=torch.zeros(1, wl.inter, wl.hidden, dtype=torch.bfloat16, device="cuda"),
             w_down=torch.zeros(1, wl.hidden, wl.inter, dtype=torch.bfloat16, device="cuda"))
    moe = BeamMoE.from_workload(wl, w, max_tokens=8192)
    p = moe.launch_plan(64)
    assert p["tile_rows"] == 64 and p["stream_k_gate_up"] == 1 and p["stream_k_down"] == 1
    assert p["router_tensor_cores"] == 0 and p["gather_rows"] == 0
    p = moe.launch_plan(8192)
    assert p["tile_rows"] == 256 and p["stream_k_gate_up"] == 0 and p["stream_k_down"] == 0
    x = torch.zeros(4, wl.hidden, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(BeamMoEError) as err:
        moe.route(x)
    assert err.value.code == BEAM_ERR_UNSUPPORTED
    moe.close()


@pytest.mark.parametrize("name", ["dense_decode", "dense_prefill"])
def test_dense_beam_shape(name):
    wl = W.WORKLOADS[name]
    d = _inputs(wl)
    moe = BeamMoE.from_workload(wl, d)
    sample = W.sample_tokens(dataclasses.replace(wl, sample=128 if wl.sample else 0))
    rep = check_dense(wl, d, moe, sample=sample)
    _log(f"beam_{name}", rep, moe.launch_plan(wl.T))
    assert rep.ok(), rep
    moe.close()

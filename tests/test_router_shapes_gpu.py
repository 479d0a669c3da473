"""Routing on the other expert layouts the selection kernel supports (1 to
16 experts per lane, groups of 2 to 64, one group, every group kept, top-1),
index for index against the oracle, and the whole block on two of them.
The degenerate cases are the method's own: n_group = topk_group = 1 is a
plain top-k; topk_group = n_group keeps every group; top_k = 1 gives weight 1."""
import dataclasses

import numpy as np
import pytest

import oracle
from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import BeamMoE
from group_limited_routing_sigmoid_b200.build import build

from parity import NEAR_TIE, W_ABS, check_block

pytestmark = pytest.mark.gpu

# (n_experts, n_group, topk_group, top_k)
SHAPES = [(32, 1, 1, 2), (32, 16, 3, 5), (64, 4, 2, 4), (64, 16, 5, 1), (128, 8, 3, 6),
          (256, 8, 8, 8), (256, 4, 1, 8), (512, 16, 4, 8), (512, 8, 2, 16)]


def setup_module(_):
    build(quiet=True)


def _wl(E, G, KG, K, T):
    return dataclasses.replace(W.WORKLOADS["tiny"], name=f"r{E}_{G}_{KG}_{K}", T=T, n_experts=E,
                               n_group=G, topk_group=KG, top_k=K, inter=128)


@pytest.mark.parametrize("E,G,KG,K", SHAPES)
def test_routing_layouts_match_oracle(E, G, KG, K):
    T = 600
    wl = _wl(E, G, KG, K, T)
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g))
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    idx, w = moe.route(d["x"])
    r = oracle.route(W.bf16_bits(d["x"]), d["router_w"].cpu().numpy(), d["bias"].cpu().numpy(),
                     G, KG, K)
    keep = (r.gap_expert >= NEAR_TIE) & (r.gap_group >= NEAR_TIE) & (r.gap_order >= NEAR_TIE)
    assert keep.mean() > 0.99
    np.testing.assert_array_equal(idx.cpu().numpy()[keep], r.idx[keep])
    assert np.abs(w.cpu().numpy()[keep] - r.w[keep]).max() <= W_ABS
    if K == 1:
        assert bool((w == 1.0).all())
    moe.close()


@pytest.mark.parametrize("E,G,KG,K", [(64, 4, 2, 4), (512, 8, 2, 16)])
def test_block_on_other_layouts(E, G, KG, K):
    wl = _wl(E, G, KG, K, 300)
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g))
    moe = BeamMoE.from_workload(wl, d, max_tokens=300)
    rep = check_block(wl, d, moe)
    assert rep.ok(), rep
    moe.close()


def test_largest_supported_shapes():
    """The kernels' size limits at once: hidden 8192, 1024 experts (32 per
    lane in the selection) in 16 groups of 64, top-32 (the largest top_k),
    every token through the whole block."""
    wl = dataclasses.replace(W.WORKLOADS["tiny"], name="max", T=48, hidden=8192, n_experts=1024,
                             n_group=16, topk_group=4, top_k=32, inter=128)
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g))
    moe = BeamMoE.from_workload(wl, d, max_tokens=wl.T)
    rep = check_block(wl, d, moe)
    assert rep.ok(), rep
    moe.close()


@pytest.mark.parametrize("hidden,T", [(384, 64), (384, 1), (128, 37), (1024, 64), (5120, 64),
                                      (5120, 1)])
def test_small_batch_router(hidden, T):
    """Batches of at most 64 tokens take the small-batch logits kernel with
    its cost-chosen K slices: 2 and 6 slices of 64 (hidden 128, 384), 8 of
    128 (hidden 1024), 8 of 640 (hidden 5120). Checked here: the logits
    against their exact value, the routing against the oracle, and a second
    call equal to the first bit for bit."""
    import torch
    wl = dataclasses.replace(W.WORKLOADS["decode"], name=f"small_router_{hidden}", T=T,
                             hidden=hidden, inter=128)
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g))
    moe = BeamMoE.from_workload(wl, d, max_tokens=64)
    got = moe.router_logits(d["x"]).cpu().double().numpy()
    ref = oracle.bf16_to_f64(W.bf16_bits(d["x"])) @ d["router_w"].cpu().double().numpy().T
    assert np.abs(got - ref).max() < 2e-6 * max(1.0, np.abs(ref).max())
    idx, w = moe.route(d["x"])
    idx2, w2 = moe.route(d["x"])
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    r = oracle.route(W.bf16_bits(d["x"]), d["router_w"].cpu().numpy(), d["bias"].cpu().numpy(),
                     wl.n_group, wl.topk_group, wl.top_k)
    keep = (r.gap_expert >= NEAR_TIE) & (r.gap_group >= NEAR_TIE) & (r.gap_order >= NEAR_TIE)
    np.testing.assert_array_equal(idx.cpu().numpy()[keep], r.idx[keep])
    assert np.abs(w.cpu().numpy()[keep] - r.w[keep]).max() <= W_ABS
    moe.close()

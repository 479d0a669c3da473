"""beam_moe_route_static: routing for callers that cannot allocate device
memory (an engine that owns all of the GPU's memory, or a path that must not
enter the CUDA allocator), with its scratch in a fixed array inside the
library.  Checked through the C ABI against beam_moe_route on the same
inputs, on two calls in a row (the second call reuses the scratch the first
one left behind).  Kept in a file that runs after the other tests.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import (BEAM_ERR_INVALID_ARG, BeamMoE,
                                                        BeamMoEError, route_static)
from group_limited_routing_sigmoid_b200.build import build

from parity import NEAR_TIE, W_ABS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("tiny", 1000), ("decode", 64), ("decode", 3000)])
def test_route_static_matches_route(name, T):
    build(quiet=True)
    wl = W.WORKLOADS[name]
    if name == "decode":
        wl = dataclasses.replace(wl, inter=128)   # routing does not depend on the experts' size
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    idx_ref, w_ref = moe.route(d["x"])
    # the two entry points may split the router's K range differently (the
    # static scratch caps the slices), so logits can differ by rounding:
    # near-ties (the oracle's expert or group gap below the parity tests'
    # threshold) are exempt from the index comparison, as in those tests
    r = oracle.route(W.bf16_bits(d["x"]), d["router_w"].cpu().numpy(), d["bias"].cpu().numpy(),
                     wl.n_group, wl.topk_group, wl.top_k)
    keep = (r.gap_expert >= NEAR_TIE) & (r.gap_group >= NEAR_TIE) & (r.gap_order >= NEAR_TIE)
    for _ in range(2):
        idx, w = route_static(d["x"], d["router_w"], d["bias"], wl.n_group, wl.topk_group, wl.top_k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy()[keep], idx_ref.cpu().numpy()[keep])
        assert float((w - w_ref).abs().max()) <= W_ABS
    assert keep.mean() > 0.99
    moe.close()


def test_route_static_rejects_batches_beyond_its_scratch():
    build(quiet=True)
    wl = W.WORKLOADS["decode"]
    g = W.generator(W.WORKLOADS["tiny"], "cuda")
    router_w = torch.randn(wl.n_experts, wl.hidden, generator=g, device="cuda")
    bias = torch.zeros(wl.n_experts, device="cuda")
    x = torch.zeros(8193, wl.hidden, dtype=torch.bfloat16, device="cuda")   # 8193 * 256 > 2**21
    with pytest.raises(BeamMoEError) as err:
        route_static(x, router_w, bias, wl.n_group, wl.topk_group, wl.top_k)
    assert err.value.code == BEAM_ERR_INVALID_ARG

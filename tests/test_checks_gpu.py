"""Checked mode (beam_moe_set_checks): device-side validation of the routing
and the dispatch tables in place of a memory checker.  A failed check records
BEAM_ERR_CHECK without trapping, the rest of the pass skips its work, and the
context stays usable.  The failure is made on the host's request, by the
library's corruption hook, never by a bad address."""
import dataclasses

import pytest
import torch

from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import (BEAM_ERR_CHECK, BEAM_ERR_INVALID_ARG,
                                                        BeamMoE, BeamMoEError)
from group_limited_routing_sigmoid_b200.build import build

from parity import check_block

pytestmark = pytest.mark.gpu


def setup_module(_):
    build(quiet=True)


def _inputs(wl, T=None):
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    return d


@pytest.mark.parametrize("name,T", [("tiny", 1000), ("small", 1024), ("small", 37)])
def test_checked_forward_passes_and_matches_oracle(name, T):
    wl = W.WORKLOADS[name]
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_checks(True)
    rep = check_block(wl, d, moe)
    assert rep.ok(), rep
    assert moe.get_status() == 0
    moe.close()


def test_corrupted_routing_is_caught_and_the_context_survives():
    wl = dataclasses.replace(W.WORKLOADS["tiny"], post_norm=True, residual_k=20)
    d = _inputs(wl, 300)
    moe = BeamMoE.from_workload(wl, d, max_tokens=300)
    with pytest.raises(BeamMoEError) as err:
        moe.debug_corrupt_routing(1)            # only in checked mode
    assert err.value.code == BEAM_ERR_INVALID_ARG
    moe.set_checks(True)
    moe.debug_corrupt_routing(1)
    out = torch.full((300, wl.hidden), 3.0, dtype=torch.bfloat16, device="cuda")
    stream = d["stream"][:300].clone()
    before = stream.clone()
    moe.forward(d["x"], out=out, residual=stream, k=20)
    assert moe.get_status() == BEAM_ERR_CHECK
    assert "index 0" in moe.last_error()         # token 0 failed the routing check
    # the pass skipped its work: the output buffer and the stream are untouched
    assert bool((out == 3.0).all())
    assert torch.equal(stream, before)
    assert moe.get_status() == 0                 # read-and-clear
    rep = check_block(wl, d, moe, T=300)         # the next pass is checked and correct
    assert rep.ok(), rep
    assert moe.get_status() == 0
    moe.close()

"""A forward pass captured in a CUDA graph (the launch path a serving loop
uses to drop per-kernel launch cost) replays to the same bits as eager
calls, for new inputs copied into the captured buffers.  The forward pass
makes no synchronising call, and its programmatic dependent launches become
graph edges."""
import dataclasses

import pytest
import torch

from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import BeamMoE
from group_limited_routing_sigmoid_b200.build import build

pytestmark = pytest.mark.gpu


def setup_module(_):
    build(quiet=True)


@pytest.mark.parametrize("name,T,resid", [("small", 64, False), ("small", 1024, False),
                                          ("tiny", 300, True)])
def test_graph_replay_matches_eager(name, T, resid):
    wl = W.WORKLOADS[name]
    if resid:
        wl = dataclasses.replace(wl, post_norm=True, residual_k=20)
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    x2 = torch.randn(T, wl.hidden, device="cuda").to(torch.bfloat16)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)

    def run(x, out, stream_buf):
        if resid:
            moe.forward(x, out=out, residual=stream_buf, k=wl.residual_k)
        else:
            moe.forward(x, out=out)

    # eager reference for the second batch
    ref_out = torch.empty(T, wl.hidden, dtype=torch.bfloat16, device="cuda")
    ref_stream = d["stream"].clone() if resid else None
    run(x2, ref_out, ref_stream)
    torch.cuda.synchronize()

    # capture with the first batch's buffers, then replay on the second batch
    x_buf = d["x"].clone()
    out_buf = torch.empty_like(ref_out)
    stream_buf = d["stream"].clone() if resid else None
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(x_buf, out_buf, stream_buf.clone() if resid else None)   # warm-up outside the graph
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(x_buf, out_buf, stream_buf)
    x_buf.copy_(x2)
    if resid:
        stream_buf.copy_(d["stream"])
    graph.replay()
    torch.cuda.synchronize()
    assert moe.get_status() == 0
    assert torch.equal(out_buf, ref_out)
    if resid:
        assert torch.equal(stream_buf, ref_stream)
    del graph
    moe.close()

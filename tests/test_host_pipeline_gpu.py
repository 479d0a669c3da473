"""Host-buffer passes: the synchronous call and the pipelined one (copies on
the handle's own streams, two staging slots, overlapping neighbouring
calls) give the same bits as the device-buffer forward pass, over more
calls than slots, with and without the residual stream."""
import dataclasses

import pytest
import torch

from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import BeamMoE
from group_limited_routing_sigmoid_b200.build import build

pytestmark = pytest.mark.gpu


def setup_module(_):
    build(quiet=True)


@pytest.mark.parametrize("name,T,resid", [("tiny", 300, True), ("small", 1024, False)])
def test_pipelined_host_passes_match_device_passes(name, T, resid):
    wl = W.WORKLOADS[name]
    if resid:
        wl = dataclasses.replace(wl, post_norm=True, residual_k=20)
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    n = 5
    xs = [torch.randn(T, wl.hidden, generator=torch.Generator().manual_seed(i)).to(torch.bfloat16)
          for i in range(n)]
    streams = [torch.randn(T, wl.hidden, generator=torch.Generator().manual_seed(100 + i))
               for i in range(n)] if resid else [None] * n
    k = wl.residual_k if resid else 1

    # device-buffer reference
    ref_out, ref_stream = [], []
    for i in range(n):
        st = streams[i].cuda() if resid else None
        ref_out.append(moe.forward(xs[i].cuda(), residual=st, k=k).cpu())
        ref_stream.append(st.cpu() if resid else None)
    torch.cuda.synchronize()

    # pipelined host passes, every call in flight before the join
    x_h = [x.pin_memory() for x in xs]
    out_h = [torch.empty(T, wl.hidden, dtype=torch.bfloat16).pin_memory() for _ in range(n)]
    st_h = [s.clone().pin_memory() for s in streams] if resid else [None] * n
    for i in range(n):
        moe.forward_host_async(x_h[i], out_host=out_h[i], residual_host=st_h[i], k=k)
    moe.host_join()
    torch.cuda.synchronize()
    assert moe.get_status() == 0
    for i in range(n):
        assert torch.equal(out_h[i], ref_out[i])
        if resid:
            assert torch.equal(st_h[i], ref_stream[i])

    # the synchronous call
    out1 = torch.empty(T, wl.hidden, dtype=torch.bfloat16).pin_memory()
    st1 = streams[0].clone().pin_memory() if resid else None
    moe.forward_host(x_h[0], out_host=out1, residual_host=st1, k=k)
    assert torch.equal(out1, ref_out[0])
    if resid:
        assert torch.equal(st1, ref_stream[0])
    moe.close()

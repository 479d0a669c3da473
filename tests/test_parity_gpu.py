"""CUDA path vs the CPU oracle, through the C ABI, on the seeded workloads.

Small block (H=256, 32 experts): every token, at several T (ragged tails,
T=1, tiles of 16..128 token rows) and GEMM grid sizes (many work items per
CTA).  Beam shape (H=5120, 256 experts, I=2560): the decode batch in full;
the 8192- and 32768-token workloads on a seeded sample of tokens (512 by
default; BEAM_PARITY_SAMPLE overrides).
"""
import dataclasses
import json
import os

import numpy as np
import pytest
import torch

import oracle
from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import BeamMoE, BeamMoEError, BEAM_ERR_TIMEOUT
from group_limited_routing_sigmoid_b200.build import build

from parity import NEAR_TIE, W_ABS, check_block

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build(quiet=True)
    oracle.build()


def _log(name, rep):
    path = os.environ.get("BEAM_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **dataclasses.asdict(rep)}) + "\n")


def _inputs(wl, T=None):
    g = W.generator(wl, "cuda")
    d = W.make_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    return d


# (T, GEMM CTAs (0 = one per SM), largest token tile (0 = auto), paired down tiles (-1 = auto),
#  gate|up token rows gathered from x: -1 auto, 1 always, 0 never (sorted copy))
TINY_CASES = [(64, 0, 0, -1, -1), (64, 1, 0, -1, -1), (1, 0, 0, -1, -1), (3, 0, 0, -1, -1),
              (37, 5, 0, -1, -1), (100, 0, 0, -1, -1), (200, 3, 0, -1, -1), (1000, 0, 0, -1, -1),
              (1000, 2, 0, -1, -1), (4096, 0, 0, -1, -1), (1000, 0, 16, 0, 1), (1000, 0, 32, 1, 1),
              (1000, 0, 64, 0, 1), (1000, 3, 128, 1, 1), (1000, 0, 256, 0, 1), (1000, 2, 256, 1, 1),
              (300, 0, 256, 1, 1), (4096, 7, 256, 1, 1),
              (37, 5, 0, -1, 0), (1000, 0, 0, -1, 0), (1000, 0, 32, 1, 0), (4096, 7, 256, 1, 0)]


@pytest.mark.parametrize("T,ctas,tile,pair,gather", TINY_CASES)
def test_tiny_block(T, ctas, tile, pair, gather):
    wl = W.WORKLOADS["tiny"]
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(ctas, tile, pair, gather_rows=gather)
    rep = check_block(wl, d, moe)
    _log(f"tiny_T{T}_ctas{ctas}_tile{tile}_pair{pair}_gather{gather}", rep)
    assert rep.ok(), rep
    moe.close()


# (T, GEMM CTAs, largest token tile, paired down tiles, CTA pairs, router mode, gathered
#  token rows): H=512, I=256
SMALL_CASES = [(1024, 0, 0, -1, 1, -1, -1), (1024, 0, 0, -1, 0, 0, 1), (1024, 0, 64, 0, 1, 1, 1),
               (1024, 4, 128, 1, 1, 1, 1), (1024, 0, 256, 0, 1, 0, 1), (3000, 0, 256, 1, 1, 1, 1),
               (3000, 6, 256, 1, 1, -1, -1), (777, 0, 128, -1, 1, 1, 1), (2048, 2, 64, 1, 1, 0, 1),
               (64, 0, 64, -1, 1, 1, 1), (1, 0, 0, -1, 1, 1, -1), (130, 0, 0, -1, 1, 1, -1),
               (1024, 0, 0, -1, 1, 2, 1), (3000, 0, 0, -1, 1, 2, 1),
               (1024, 0, 0, -1, 1, -1, 0), (1024, 0, 0, -1, 0, 0, 0), (777, 0, 128, -1, 1, 1, 0),
               (3000, 6, 256, 1, 1, -1, 0)]


@pytest.mark.parametrize("T,ctas,tile,pair,pairs,router,gather", SMALL_CASES)
def test_small_block(T, ctas, tile, pair, pairs, router, gather):
    wl = W.WORKLOADS["small"]
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(ctas, tile, pair, pairs, router, gather)
    rep = check_block(wl, d, moe)
    _log(f"small_T{T}_ctas{ctas}_tile{tile}_pair{pair}_pairs{pairs}_router{router}_gather{gather}", rep)
    assert rep.ok(), rep
    moe.close()


# (T, largest token tile, gathered rows, gate|up layout): CTA pairs; layout 0
# keeps separate gate and up tiles (the default), 1 interleaves them, at
# every pair tile size and with gathered rows too
LAYOUT_CASES = [(1024, 256, 0, 0), (1024, 256, 0, 1), (3000, 256, 0, 0), (3000, 256, 1, 1),
                (1024, 128, 0, 1), (777, 64, 0, 1), (130, 256, 0, 1)]


@pytest.mark.parametrize("T,tile,gather,layout", LAYOUT_CASES)
def test_small_block_gate_up_layouts(T, tile, gather, layout):
    wl = W.WORKLOADS["small"]
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(0, tile, -1, 1, -1, gather)
    moe.set_gate_up_layout(layout)
    assert moe.launch_plan(T)["gate_up_interleaved"] == layout
    rep = check_block(wl, d, moe)
    _log(f"small_layout_T{T}_tile{tile}_gather{gather}_layout{layout}", rep)
    assert rep.ok(), rep
    moe.close()


@pytest.mark.parametrize("norm", [True, False])
def test_tiny_residual(norm):
    wl = dataclasses.replace(W.WORKLOADS["tiny"], post_norm=norm, residual_k=20)
    d = _inputs(wl, 300)
    if not norm:
        d["gamma"] = None
    moe = BeamMoE.from_workload(wl, d, max_tokens=300)
    rep = check_block(wl, d, moe)
    _log(f"tiny_residual_norm{norm}", rep)
    assert rep.ok(), rep
    assert rep.res_rel_fro is not None
    moe.close()


# T=1000 takes the three-kernel dispatch; T of at most 128 (top-8: 1024
# pairs) with gathered token rows takes the one-block dispatch
@pytest.mark.parametrize("gather,T", [(-1, 1000), (1, 1000), (0, 1000), (1, 100), (1, 1), (0, 100)])
def test_tiny_dispatch_is_a_stable_counting_sort(gather, T):
    wl = W.WORKLOADS["tiny"]
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(gather_rows=gather)
    moe.forward(d["x"])
    idx, _ = moe.route(d["x"])
    counts, offsets, pair_row = moe.dispatch_info(T)
    flat = idx.cpu().numpy().reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=wl.n_experts))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    order = np.argsort(flat, kind="stable")          # rows: pairs sorted by (expert, pair index)
    expect = np.empty_like(order)
    expect[order] = np.arange(order.size)
    np.testing.assert_array_equal(pair_row, expect)
    moe.close()


def test_tiny_router_logits():
    wl = W.WORKLOADS["tiny"]
    d = _inputs(wl)
    moe = BeamMoE.from_workload(wl, d)
    got = moe.router_logits(d["x"]).cpu().double().numpy()
    ref = oracle.bf16_to_f64(W.bf16_bits(d["x"])) @ d["router_w"].cpu().double().numpy().T
    assert np.abs(got - ref).max() < 1e-5 * max(1.0, np.abs(ref).max())
    moe.close()


@pytest.mark.parametrize("mode,T", [(0, 1024), (1, 1024), (1, 8192), (1, 100)])
def test_router_logits_precision(mode, T):
    """FP32 logits of the Beam-shaped router (H=5120, 256 experts) against
    the exact value.  beam_moe_router_logits always takes the CUDA-core path
    (whatever the routing mode), whose error is far below the 1e-6 near-tie
    threshold of the routing comparison."""
    wl = dataclasses.replace(W.WORKLOADS["decode"], inter=128)
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(0, 0, -1, 1, mode)
    got = moe.router_logits(d["x"]).cpu().double().numpy()
    ref = oracle.bf16_to_f64(W.bf16_bits(d["x"])) @ d["router_w"].cpu().double().numpy().T
    err = float(np.abs(got - ref).max())
    path = os.environ.get("BEAM_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": f"router_logits_mode{mode}_T{T}", "max_abs_err": err}) + "\n")
    assert err < 2e-6, err
    moe.close()


@pytest.mark.parametrize("mode", [1, 2])
def test_tensor_core_routing_matches_oracle(mode):
    """Routing of 8192 tokens at the Beam router shape through the
    tensor-core path (mode 1: thin-margin tokens re-derived on CUDA cores;
    mode 2: every token re-derived) against the oracle on every token."""
    from parity import NEAR_TIE, W_ABS
    wl = dataclasses.replace(W.WORKLOADS["prefill"], inter=128)
    T = 8192
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(0, 0, -1, 1, mode)
    idx, w = moe.route(d["x"])
    rederived = moe.router_stats()
    if mode == 2:
        assert rederived == T
    r = oracle.route(W.bf16_bits(d["x"]), d["router_w"].cpu().numpy(), d["bias"].cpu().numpy(),
                     wl.n_group, wl.topk_group, wl.top_k)
    keep = (r.gap_expert >= NEAR_TIE) & (r.gap_group >= NEAR_TIE) & (r.gap_order >= NEAR_TIE)
    mism = int((idx.cpu().numpy()[keep] != r.idx[keep]).any(axis=1).sum())
    werr = float(np.abs(w.cpu().numpy()[keep] - r.w[keep]).max())
    path = os.environ.get("BEAM_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": f"tc_routing_mode{mode}", "tokens": T, "exempt": int((~keep).sum()),
                                "idx_mismatch": mism, "w_max_err": werr, "rederived": rederived}) + "\n")
    assert mism == 0 and werr <= W_ABS, (mism, werr)
    moe.close()


@pytest.mark.parametrize("name,T", [("tiny", 1000), ("decode", 512)])
def test_reroute_from_logits_under_a_new_bias(name, T):
    """Routing from the router's FP32 logits: with the handle's bias it
    matches beam_moe_route; under another bias it matches the oracle's
    selection from the same logits, index for index (near-ties exempt)."""
    wl = W.WORKLOADS[name]
    if name == "decode":
        wl = dataclasses.replace(wl, inter=128)   # routing does not depend on the experts' size
    d = _inputs(wl, T)
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(router_mode=0)             # CUDA-core logits for both calls
    logits = moe.router_logits(d["x"])
    idx0, w0 = moe.route(d["x"])
    idx1, w1 = moe.route_logits(logits)
    np.testing.assert_array_equal(idx1.cpu().numpy(), idx0.cpu().numpy())
    torch.testing.assert_close(w1, w0, rtol=0, atol=0)
    g = torch.Generator().manual_seed(11)
    bias2 = (torch.rand(wl.n_experts, generator=g) * 0.4 - 0.2).float()
    idx2, w2 = moe.route_logits(logits, bias2.cuda())
    r = oracle.route_logits(logits.cpu().numpy(), bias2.numpy(), wl.n_group, wl.topk_group, wl.top_k)
    keep = (r.gap_expert >= NEAR_TIE) & (r.gap_group >= NEAR_TIE) & (r.gap_order >= NEAR_TIE)
    np.testing.assert_array_equal(idx2.cpu().numpy()[keep], r.idx[keep])
    assert np.abs(w2.cpu().numpy()[keep] - r.w[keep]).max() <= W_ABS
    assert keep.mean() > 0.99
    assert (idx2.cpu().numpy() != idx0.cpu().numpy()).any()   # the new bias moved some tokens
    moe.close()


def test_empty_batch_is_a_no_op():
    wl = W.WORKLOADS["tiny"]
    d = _inputs(wl)
    moe = BeamMoE.from_workload(wl, d)
    x0 = d["x"][:0]
    out = torch.full((0, wl.hidden), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.forward(x0, out=out)
    moe.route(x0)
    assert moe.get_status() == 0
    moe.close()


def test_launch_plan_follows_tokens_per_expert_and_tuning():
    """The plan a forward pass follows: 16-row tiles on single CTAs and
    CUDA-core router logits for a few tokens per expert; 256-row tiles on CTA
    pairs with paired down blocks and tensor-core logits for many; tuning
    overrides apply; T outside [0, max_tokens] is rejected."""
    wl = W.WORKLOADS["small"]
    d = _inputs(wl)
    moe = BeamMoE.from_workload(wl, d)
    p = moe.launch_plan(8)
    assert (p["tile_rows"], p["cta_pairs"], p["down_paired"], p["router_tensor_cores"],
            p["gather_rows"]) == (16, 0, 0, 0, 1)
    assert p["grid"] == torch.cuda.get_device_properties(0).multi_processor_count
    assert p["y_f32"] == 1 and p["gate_up_interleaved"] == 0
    p = moe.launch_plan(wl.T)
    assert (p["tile_rows"], p["cta_pairs"], p["down_paired"], p["router_tensor_cores"]) == (256, 1, 1, 1)
    assert p["gate_up_interleaved"] == 0
    assert p["grid"] % 2 == 0 and p["router_slices"] >= 1
    assert p["gather_rows"] == 0
    moe.set_gemm_tuning(6, 64, 0, 0, 0, 1)
    p = moe.launch_plan(wl.T)
    assert (p["tile_rows"], p["cta_pairs"], p["grid"], p["down_paired"], p["router_tensor_cores"],
            p["gather_rows"]) == (64, 0, 6, 0, 0, 1)
    with pytest.raises(BeamMoEError):
        moe.launch_plan(wl.T + 1)
    moe.close()


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait on a barrier that nothing completes, and a wait on a global
    counter that nothing increments, each give up after the limit, record
    BEAM_ERR_TIMEOUT and return; the context stays usable."""
    wl = W.WORKLOADS["tiny"]
    d = _inputs(wl)
    moe = BeamMoE.from_workload(wl, d)
    moe.set_wait_limit(1_000_000)   # 1 ms
    assert moe.check_wait_timeout() == BEAM_ERR_TIMEOUT
    assert moe.get_status() == 0     # read-and-clear
    moe.set_wait_limit(2_000_000_000)
    rep = check_block(wl, d, moe)
    assert rep.ok(), rep
    moe.close()


def _sample(wl):
    s = W.sample_tokens(wl)
    n = int(os.environ.get("BEAM_PARITY_SAMPLE", "0") or 0)
    return s[:n] if n else s


@pytest.mark.parametrize("name", ["decode", "prefill", "skewed", "long"])
def test_beam_shape(name):
    wl = W.WORKLOADS[name]
    d = W.make_inputs(wl, "cuda")
    moe = BeamMoE.from_workload(wl, d)
    rep = check_block(wl, d, moe, sample=_sample(wl))
    _log(f"beam_{name}", rep)
    assert rep.ok(), rep
    moe.close()
    del d, moe
    torch.cuda.empty_cache()

"""NVFP4 expert weights (beam_moe_create_nvfp4) against the oracle's NVFP4
expert: the decode the GEMMs run, bit for bit, over every code byte and
every finite scale byte; the block over ragged token counts, every token
tile, fewer CTAs than work items, and the post-norm and residual update; and
the Beam decode shape (H=5120, 256 experts, I=2560, 64 tokens) in full; and
the status the GEMMs record for an activation beyond their f16 operands'
range (65504 x 2^8)."""
import dataclasses
import json
import os

import numpy as np
import pytest
import torch

import oracle
from group_limited_routing_sigmoid_b200 import workloads as W
from group_limited_routing_sigmoid_b200.binding import BEAM_ERR_RANGE, BeamMoE, nvfp4_dequant
from group_limited_routing_sigmoid_b200.build import build

from parity import check_block

pytestmark = pytest.mark.gpu


def setup_module(_):
    build(quiet=True)


def _log(case, rep, plan):
    path = os.environ.get("BEAM_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, **rep.__dict__, "plan": plan}) + "\n")


def test_dequant_is_exact_for_every_code_and_scale():
    # rows of 512 elements: every code byte twice per row; one scale byte per
    # 16-element block, cycling through the 254 finite E4M3 bytes
    finite = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)
    rows, K = 254, 512
    codes = np.tile(np.concatenate([np.arange(256, dtype=np.uint8)] * 1), (rows, 1))
    scales = finite[(np.arange(rows)[:, None] + np.arange(K // 16)[None, :] * 7) % len(finite)]
    got = nvfp4_dequant(torch.from_numpy(codes).cuda(), torch.from_numpy(scales.astype(np.uint8)).cuda())
    torch.cuda.synchronize()
    e2m1 = np.array([oracle.e2m1_value(c) for c in range(16)])
    e4m3 = np.array([oracle.e4m3_value(b) for b in range(256)])
    c = codes.astype(np.int64)
    nib = np.stack([c & 15, c >> 4], axis=-1).reshape(rows, K)
    ref = e2m1[nib] * np.repeat(e4m3[scales], 16, axis=1)
    # the products have at most 6 significant bits: exact in bf16
    ref_bits = W.bf16_bits(torch.from_numpy(ref).to(torch.bfloat16))
    assert np.array_equal(oracle.bf16_to_f64(ref_bits), ref)
    got_bits = W.bf16_bits(got.cpu())
    # equal as values (a zero may carry either sign)
    np.testing.assert_array_equal(oracle.bf16_to_f64(got_bits), ref)


# (T, GEMM CTAs (0 = one per SM), largest token tile (0 = auto), post-norm + residual)
CASES = [(1, 0, 0, False), (5, 0, 0, False), (64, 0, 0, False), (64, 7, 0, False),
         (300, 0, 0, False), (300, 0, 16, False), (300, 0, 32, False), (1000, 0, 64, False),
         (1000, 0, 128, False), (1000, 0, 256, False), (1000, 3, 0, False), (64, 0, 0, True),
         (300, 0, 0, True)]


@pytest.mark.parametrize("T,ctas,tile,resid", CASES)
def test_nvfp4_block(T, ctas, tile, resid):
    wl = W.WORKLOADS["tiny_nvfp4"]
    if resid:
        wl = dataclasses.replace(wl, post_norm=True, residual_k=20)
    g = W.generator(wl, "cuda")
    d = W.make_nvfp4_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(ctas, tile, -1, 1)
    plan = moe.launch_plan(T)
    assert plan["cta_pairs"] == 0 and plan["gather_rows"] == 0 and plan["tile_rows"] <= 128
    rep = check_block(wl, d, moe)
    _log(f"nvfp4_T{T}_ctas{ctas}_tile{tile}_resid{resid}", rep, plan)
    assert rep.ok(), rep
    if resid:
        assert rep.res_rel_fro is not None
    moe.close()


# inter 256: the down GEMM takes four K steps per stage (K/64 a multiple of
# four), at every token tile size; inter 640: five K steps per stage for
# tiles of 16 and 32 rows (K/64 a multiple of five), two for larger tiles
@pytest.mark.parametrize("T,tile,inter", [(300, 16, 256), (300, 32, 256), (1000, 64, 256),
                                          (1000, 128, 256), (300, 16, 640), (37, 32, 640),
                                          (300, 64, 640)])
def test_nvfp4_block_several_k_steps_per_stage(T, tile, inter):
    wl = dataclasses.replace(W.WORKLOADS["tiny_nvfp4"], inter=inter)
    g = W.generator(wl, "cuda")
    d = W.make_nvfp4_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=T))
    moe = BeamMoE.from_workload(wl, d, max_tokens=T)
    moe.set_gemm_tuning(0, tile, -1, 1)
    plan = moe.launch_plan(T)
    assert plan["tile_rows"] == tile
    rep = check_block(wl, d, moe)
    _log(f"nvfp4_inter{inter}_T{T}_tile{tile}", rep, plan)
    assert rep.ok(), rep
    moe.close()


def test_nvfp4_beam_decode():
    wl = W.WORKLOADS["decode_nvfp4"]
    g = W.generator(wl, "cuda")
    d = W.make_nvfp4_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g))
    moe = BeamMoE.from_workload(wl, d)
    rep = check_block(wl, d, moe)
    _log("beam_decode_nvfp4", rep, moe.launch_plan(wl.T))
    assert rep.ok(), rep
    moe.close()
    del d, moe
    torch.cuda.empty_cache()


def test_nvfp4_activation_beyond_f16_range_sets_status():
    wl = W.WORKLOADS["tiny_nvfp4"]
    g = W.generator(wl, "cuda")
    d = W.make_nvfp4_weights(wl, "cuda", g)
    d.update(W.make_tokens(wl, "cuda", g, T=8))
    moe = BeamMoE.from_workload(wl, d, max_tokens=8)
    x = d["x"].clone()
    x[3, 5] = 2.0 ** 25                    # exact in bf16, above 65504 x 2^8
    moe.forward(x)
    assert moe.get_status() == BEAM_ERR_RANGE
    # read and cleared above: an ordinary batch leaves it at zero
    moe.forward(d["x"])
    assert moe.get_status() == 0
    moe.close()

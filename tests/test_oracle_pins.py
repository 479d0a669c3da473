"""Pins for the CPU oracle: each test checks it against something other than
itself -- library routines, exhaustive search, closed forms and the numbers
the Beam pages print.  No GPU needed.

Each pin is chosen so that a plausible slip in the oracle fails it:
  * sign or form of the sigmoid, or the router matmul orientation
    -> test_router_scores_match_library;
  * group score = top-1 only, wrong group count, no tie rule
    -> test_route_bruteforce_tiny / test_route_bruteforce_beam_groups;
  * bias left out of selection, or put into the weights
    -> test_bias_selects_but_does_not_weigh;
  * group limiting not applied -> test_single_group_reduces_to_topk;
  * selection from given logits (re-route under another bias)
    -> test_route_from_logits_*;
  * weights not normalised, x2.5 missing, slot/expert mix-up
    -> test_identical_experts_closed_form / test_permutation_experts_closed_form;
  * a transposed expert matrix -> test_permutation_experts_closed_form;
  * residual coefficients -> test_residual_closed_form;
  * RMSNorm form -> test_post_norm_properties.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

from group_limited_routing_sigmoid_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def to_bits(t: torch.Tensor) -> np.ndarray:
    return W.bf16_bits(t.to(torch.bfloat16))


def tiny_inputs(seed=0, T=None):
    wl = W.WORKLOADS["tiny"]
    wl = W.Workload(**{**wl.__dict__, "seed": seed})
    d = W.make_inputs(wl, "cpu")
    if T is not None:
        d["x"] = d["x"][:T]
    return wl, d


# --------------------------------------------------------------------------
# bf16 conversion vs torch (library routine)
# --------------------------------------------------------------------------

def test_bf16_rounding_matches_torch(oracle_lib):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-30).astype(np.float32),
        (rng.standard_normal(1000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 1e-40, -1e-39, 3.0e38], np.float32),
    ])
    # exact halfway points between neighbouring bf16 values: ties to even
    base = (rng.integers(0x3000, 0x4f00, 500).astype(np.uint32) << 16)
    half = (base | 0x8000).view(np.float32)
    vals = np.concatenate([vals, half, -half])
    ours = oracle_lib.f64_to_bf16(vals.astype(np.float64))
    ref = W.bf16_bits(torch.from_numpy(vals).to(torch.bfloat16))
    np.testing.assert_array_equal(ours, ref)
    back = oracle_lib.bf16_to_f64(ref)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_bf16_rounding_from_double_is_single_rounding(oracle_lib):
    # 1 + 2^-8 + 2^-30 lies just above the bf16 midpoint 1 + 2^-8: a single
    # rounding goes up; rounding to binary32 first would land on the midpoint
    # and then round to even (down).
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle_lib.bf16_to_f64(oracle_lib.f64_to_bf16(np.array([v])))[0] == 1.0 + 2.0 ** -7


# --------------------------------------------------------------------------
# Router
# --------------------------------------------------------------------------

def test_router_scores_match_library(oracle_lib):
    wl, d = tiny_inputs()
    x = W.bf16_bits(d["x"])
    r = oracle_lib.route(x, d["router_w"].numpy(), d["bias"].numpy(), wl.n_group, wl.topk_group, wl.top_k)
    logits = oracle_lib.bf16_to_f64(x) @ d["router_w"].numpy().astype(np.float64).T
    np.testing.assert_allclose(r.scores, expit(logits), rtol=1e-13, atol=0)
    np.testing.assert_allclose(r.biased, expit(logits) + d["bias"].numpy().astype(np.float64), rtol=1e-13, atol=1e-15)


def _brute_force(b32: np.ndarray, n_group: int, topk_group: int, top_k: int):
    """Exhaustive search: the kept-group subset with the largest total group
    score (ties -> lexicographically smallest), then the candidate subset of
    size top_k with the largest total score (ties -> lexicographically
    smallest)."""
    E = b32.shape[0]
    gsz = E // n_group
    gs = np.empty(n_group, np.float32)
    for j in range(n_group):
        grp = np.sort(b32[j * gsz:(j + 1) * gsz])[::-1]
        gs[j] = np.float32(grp[0]) + np.float32(grp[1])
    best_g, best_val = None, -np.inf
    for sub in itertools.combinations(range(n_group), topk_group):
        v = sum(float(gs[j]) for j in sub)
        if v > best_val:
            best_g, best_val = sub, v
    cand = [e for e in range(E) if e // gsz in best_g]
    best_e, best_val = None, -np.inf
    for sub in itertools.combinations(cand, top_k):
        v = sum(float(b32[e]) for e in sub)
        if v > best_val:
            best_e, best_val = sub, v
    return set(best_g), set(best_e)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_route_bruteforce_tiny(oracle_lib, seed):
    wl, d = tiny_inputs(seed, T=24)
    x = W.bf16_bits(d["x"])
    r = oracle_lib.route(x, d["router_w"].numpy(), d["bias"].numpy(), wl.n_group, wl.topk_group, wl.top_k)
    for t in range(x.shape[0]):
        b32 = r.biased[t].astype(np.float32)
        groups, experts = _brute_force(b32, wl.n_group, wl.topk_group, wl.top_k)
        kept = {j for j in range(wl.n_group) if (r.kept_mask[t] >> j) & 1}
        assert kept == groups
        assert set(r.idx[t].tolist()) == experts
        # canonical order: descending score, ties to the lower index
        order = sorted(experts, key=lambda e: (-float(b32[e]), e))
        assert r.idx[t].tolist() == order


def test_route_bruteforce_beam_groups(oracle_lib):
    """Beam shape (256 experts, 8 groups of 32): all C(8,4)=70 group subsets,
    then the selected experts must be the 8 best candidates."""
    wl = W.WORKLOADS["decode"]
    g = W.generator(wl, "cpu")
    d = W.make_weights(W.Workload(**{**wl.__dict__, "n_experts": 256, "inter": 64}), "cpu", g)
    x = torch.randn(16, wl.hidden, generator=g).to(torch.bfloat16)
    r = oracle_lib.route(W.bf16_bits(x), d["router_w"].numpy(), d["bias"].numpy(), 8, 4, 8)
    assert len(list(itertools.combinations(range(8), 4))) == 70
    for t in range(16):
        b32 = r.biased[t].astype(np.float32)
        gs = np.array([np.float32(np.sort(b32[j * 32:(j + 1) * 32])[-1]) + np.float32(np.sort(b32[j * 32:(j + 1) * 32])[-2])
                       for j in range(8)], np.float32)
        best = max(itertools.combinations(range(8), 4), key=lambda s: sum(float(gs[j]) for j in s))
        kept = {j for j in range(8) if (r.kept_mask[t] >> j) & 1}
        assert kept == set(best)
        cand = np.array([e for e in range(256) if e // 32 in kept])
        top = cand[np.argsort(-b32[cand], kind="stable")][:8]
        assert r.idx[t].tolist() == top.tolist()


def test_route_invariants_beam_shape(oracle_lib):
    wl = W.WORKLOADS["decode"]
    g = W.generator(wl, "cpu")
    router_w = torch.randn(256, wl.hidden, generator=g) / math.sqrt(wl.hidden)
    bias = torch.rand(256, generator=g) * 0.2 - 0.1
    x = torch.randn(64, wl.hidden, generator=g).to(torch.bfloat16)
    r = oracle_lib.route(W.bf16_bits(x), router_w.numpy(), bias.numpy(), 8, 4, 8)
    for t in range(64):
        idx = r.idx[t]
        assert len(set(idx.tolist())) == 8
        groups = {int(e) // 32 for e in idx}
        assert len(groups) <= 4
        kept = {j for j in range(8) if (r.kept_mask[t] >> j) & 1}
        assert len(kept) == 4 and groups <= kept
        b32 = r.biased[t].astype(np.float32)
        others = [e for e in range(256) if e // 32 in kept and e not in set(idx.tolist())]
        assert b32[idx].min() >= b32[others].max()
        assert np.all(r.w[t] > 0)
        assert abs(r.w[t].sum() - 1.0) < 1e-12
        # the near-tie diagnostics: gaps at the set boundary and within the order
        bd = r.biased[t]
        assert r.gap_expert[t] == bd[idx].min() - bd[others].max()
        assert r.gap_order[t] == np.min(bd[idx][:-1] - bd[idx][1:])


def test_single_group_reduces_to_topk(oracle_lib):
    """n_group=1, topk_group=1 is a plain top-k of sigmoid(logit)+bias;
    keeping every group (topk_group = n_group) must give the same result."""
    wl, d = tiny_inputs(3)
    x = W.bf16_bits(d["x"])
    wr, b = d["router_w"].numpy(), d["bias"].numpy()
    r1 = oracle_lib.route(x, wr, b, 1, 1, 8)
    r8 = oracle_lib.route(x, wr, b, 8, 8, 8)
    np.testing.assert_array_equal(r1.idx, r8.idx)
    logits = torch.from_numpy(oracle_lib.bf16_to_f64(x)) @ torch.from_numpy(wr).double().T
    biased32 = (torch.sigmoid(logits) + torch.from_numpy(b).double()).float()
    vals, ref = torch.topk(biased32, 8, dim=1)
    # torch.topk's order among exact ties is unspecified: compare scores, then sets
    np.testing.assert_array_equal(biased32.gather(1, torch.from_numpy(r1.idx).long()).numpy(), vals.numpy())
    for t in range(x.shape[0]):
        if len(set(vals[t].tolist())) == 8:
            assert set(ref[t].tolist()) == set(r1.idx[t].tolist())
    s = torch.sigmoid(logits).numpy()
    for t in range(x.shape[0]):
        sel = s[t, r1.idx[t]]
        np.testing.assert_allclose(r1.w[t], sel / sel.sum(), rtol=1e-14)


def test_bias_selects_but_does_not_weigh(oracle_lib):
    """A +10 bias on eight experts spread over four groups forces exactly those
    experts; their weights are still the unbiased sigmoid scores, normalised."""
    wl, d = tiny_inputs(4)
    x = W.bf16_bits(d["x"])
    bias = np.zeros(32, np.float32)
    forced = [1, 2, 9, 11, 20, 21, 30, 31]       # groups 0, 2, 5, 7 (4 experts per group)
    bias[forced] = 10.0
    r = oracle_lib.route(x, d["router_w"].numpy(), bias, 8, 4, 8)
    logits = oracle_lib.bf16_to_f64(x) @ d["router_w"].numpy().astype(np.float64).T
    s = expit(logits)
    for t in range(x.shape[0]):
        assert set(r.idx[t].tolist()) == set(forced)
        assert r.kept_mask[t] == (1 << 0) | (1 << 2) | (1 << 5) | (1 << 7)
        sel = s[t, r.idx[t]]
        np.testing.assert_allclose(r.w[t], sel / sel.sum(), rtol=1e-14)
        biased_w = (sel + 10.0) / (sel + 10.0).sum()
        assert np.abs(r.w[t] - biased_w).max() > 1e-3


@pytest.mark.parametrize("seed", [0, 1])
def test_route_from_logits_bruteforce(oracle_lib, seed):
    """Selection from given FP32 logits (the re-route under another bias):
    exhaustive search over group subsets and expert subsets on the tiny
    layout, with logits and a bias drawn directly."""
    rng = np.random.default_rng(100 + seed)
    logits = rng.standard_normal((20, 32)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, 32).astype(np.float32)
    r = oracle_lib.route_logits(logits, bias, 8, 4, 8)
    s = expit(logits.astype(np.float64))
    for t in range(20):
        b32 = (s[t] + bias.astype(np.float64)).astype(np.float32)
        groups, experts = _brute_force(b32, 8, 4, 8)
        assert {j for j in range(8) if (r.kept_mask[t] >> j) & 1} == groups
        assert set(r.idx[t].tolist()) == experts
        assert r.idx[t].tolist() == sorted(experts, key=lambda e: (-float(b32[e]), e))
        sel = s[t, r.idx[t]]
        np.testing.assert_allclose(r.w[t], sel / sel.sum(), rtol=1e-14)


def test_route_from_logits_single_group_is_topk(oracle_lib):
    """One group kept of one: a plain top-k of FP32(sigmoid(logit) + bias)."""
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((50, 256)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, 256).astype(np.float32)
    r = oracle_lib.route_logits(logits, bias, 1, 1, 8)
    biased32 = (torch.sigmoid(torch.from_numpy(logits).double()) + torch.from_numpy(bias).double()).float()
    vals, ref = torch.topk(biased32, 8, dim=1)
    np.testing.assert_array_equal(biased32.gather(1, torch.from_numpy(r.idx).long()).numpy(), vals.numpy())


def test_route_from_logits_bias_steers_selection_only(oracle_lib):
    """Re-routing the same logits with a +10 bias on eight experts in four
    groups forces exactly those experts; the weights stay the unbiased
    sigmoid scores of the chosen experts, normalised."""
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((30, 256)).astype(np.float32)
    bias = np.zeros(256, np.float32)
    forced = [3, 40, 41, 100, 101, 102, 250, 255]      # groups 0, 1, 3, 7 of 32 experts
    bias[forced] = 10.0
    r = oracle_lib.route_logits(logits, bias, 8, 4, 8)
    s = expit(logits.astype(np.float64))
    for t in range(30):
        assert set(r.idx[t].tolist()) == set(forced)
        assert r.kept_mask[t] == (1 << 0) | (1 << 1) | (1 << 3) | (1 << 7)
        sel = s[t, r.idx[t]]
        np.testing.assert_allclose(r.w[t], sel / sel.sum(), rtol=1e-14)


# --------------------------------------------------------------------------
# Experts + combine
# --------------------------------------------------------------------------

def _silu(z):
    return z * expit(z)


def test_identical_experts_closed_form(oracle_lib):
    """All experts equal: whatever the routing, the weights sum to 1, so the
    block output is 2.5 x one expert's SwiGLU(x)."""
    wl, d = tiny_inputs(5)
    E = wl.n_experts
    wg = W.bf16_bits(d["w_gate"][0])
    wu = W.bf16_bits(d["w_up"][0])
    wd = W.bf16_bits(d["w_down"][0])
    fetch = lambda e: (wg, wu, wd)
    x = W.bf16_bits(d["x"])
    res = oracle_lib.moe_block(x, d["router_w"].numpy(), d["bias"].numpy(), fetch,
                               wl.n_group, wl.topk_group, wl.top_k, wl.routed_scaling)
    xf = oracle_lib.bf16_to_f64(x)
    g = xf @ oracle_lib.bf16_to_f64(wg).T
    u = xf @ oracle_lib.bf16_to_f64(wu).T
    p32 = (_silu(g) * u).astype(np.float32)
    h = W.bf16_bits(torch.from_numpy(p32).to(torch.bfloat16))
    y = oracle_lib.bf16_to_f64(h) @ oracle_lib.bf16_to_f64(wd).T
    np.testing.assert_allclose(res.o, 2.5 * y, rtol=1e-10, atol=1e-12)
    assert len(set(res.routing.idx.reshape(-1).tolist())) > 8  # the routing really varies


def test_dense_layer_vs_torch(oracle_lib):
    """The dense SwiGLU layer (one expert, weight 1, no scaling) against the
    textbook formula written with numpy matmuls, the SwiGLU product rounded
    to FP32 then bf16; and its residual update against the closed form with
    the post-norm."""
    wl = W.WORKLOADS["dense_tiny"]
    d = W.make_inputs(wl, "cpu")
    x = W.bf16_bits(d["x"][:16])
    wg, wu, wd = (W.bf16_bits(d[k][0]) for k in ("w_gate", "w_up", "w_down"))
    xf = oracle_lib.bf16_to_f64(x)
    g = xf @ oracle_lib.bf16_to_f64(wg).T
    u = xf @ oracle_lib.bf16_to_f64(wu).T
    h = W.bf16_bits(torch.from_numpy((_silu(g) * u).astype(np.float32)).to(torch.bfloat16))
    y = oracle_lib.bf16_to_f64(h) @ oracle_lib.bf16_to_f64(wd).T
    gamma = (1.0 + 0.02 * np.random.default_rng(3).standard_normal(wl.hidden)).astype(np.float32)
    stream = np.random.default_rng(4).standard_normal((16, wl.hidden)).astype(np.float32)
    res = oracle_lib.dense_block(x, wg, wu, wd, gamma=gamma, eps=1e-6, stream=stream, kstep=20)
    np.testing.assert_allclose(res.o, y, rtol=1e-10, atol=1e-14)
    n = y / np.sqrt((y * y).mean(axis=1, keepdims=True) + 1e-6) * gamma.astype(np.float64)
    np.testing.assert_allclose(res.stream_out, math.sqrt(19 / 20) * stream.astype(np.float64) + n / math.sqrt(20),
                               rtol=1e-10, atol=1e-12)


def test_permutation_experts_closed_form(oracle_lib):
    """Expert e = (a_e P_e, b_e Q_e, c_e R_e) with permutation matrices and
    power-of-two scales.  Then g_i = a_e x[p_e(i)], u_i = b_e x[q_e(i)],
    y_h = c_e h[r_e(h)]: a transposed matrix or a wrong expert/slot pairing
    gives a different answer."""
    wl, d = tiny_inputs(6)
    H = I = wl.hidden
    E = wl.n_experts
    rng = np.random.default_rng(6)
    perms = [(rng.permutation(I), rng.permutation(I), rng.permutation(H)) for _ in range(E)]
    scales = [(2.0 ** rng.integers(-1, 2), 2.0 ** rng.integers(-1, 2), 2.0 ** rng.integers(-3, 0)) for _ in range(E)]

    def mat(perm, scale, rows, cols):
        m = np.zeros((rows, cols), np.float32)
        m[np.arange(rows), perm] = scale          # row i picks column perm[i]
        return to_bits(torch.from_numpy(m))

    experts = [(mat(p, a, I, H), mat(q, b, I, H), mat(rp, c, H, I)) for (p, q, rp), (a, b, c) in zip(perms, scales)]
    x = W.bf16_bits(d["x"])
    res = oracle_lib.moe_block(x, d["router_w"].numpy(), d["bias"].numpy(), lambda e: experts[e],
                               wl.n_group, wl.topk_group, wl.top_k, wl.routed_scaling)
    xf = oracle_lib.bf16_to_f64(x)
    expect = np.zeros_like(res.o)
    for t in range(x.shape[0]):
        for j in range(wl.top_k):
            e = int(res.routing.idx[t, j])
            (p, q, rp), (a, b, c) = perms[e], scales[e]
            g = a * xf[t, p]
            u = b * xf[t, q]
            h = oracle_lib.bf16_to_f64(W.bf16_bits(torch.from_numpy((_silu(g) * u).astype(np.float32)).to(torch.bfloat16)))
            expect[t] += res.routing.w[t, j] * c * h[rp]
    np.testing.assert_allclose(res.o, 2.5 * expect, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(res.out, oracle_lib.f64_to_bf16(res.o))


def test_tiny_block_vs_torch_dense(oracle_lib):
    """Cross-check of the whole tiny block against torch fp64 matmuls (a
    second, independent implementation of the expert and combine)."""
    wl, d = tiny_inputs(7)
    x = W.bf16_bits(d["x"])
    res = oracle_lib.moe_block(x, d["router_w"].numpy(), d["bias"].numpy(),
                               oracle_lib.dense_fetch(W.bf16_bits(d["w_gate"]), W.bf16_bits(d["w_up"]), W.bf16_bits(d["w_down"])),
                               wl.n_group, wl.topk_group, wl.top_k, wl.routed_scaling)
    xd = d["x"].double()
    out = torch.zeros(x.shape[0], wl.hidden, dtype=torch.float64)
    for t in range(x.shape[0]):
        for j in range(wl.top_k):
            e = int(res.routing.idx[t, j])
            g = d["w_gate"][e].double() @ xd[t]
            u = d["w_up"][e].double() @ xd[t]
            h = (torch.nn.functional.silu(g) * u).float().to(torch.bfloat16).double()
            out[t] += float(res.routing.w[t, j]) * (d["w_down"][e].double() @ h)
    np.testing.assert_allclose(res.o, 2.5 * out.numpy(), rtol=1e-9, atol=1e-12)


# --------------------------------------------------------------------------
# Post-norm + depth-scaled residual
# --------------------------------------------------------------------------

def test_residual_closed_form(oracle_lib):
    """Iterating the update for steps 1..K (step 1 = the embedding) leaves the
    stream equal to the sum of the K contributions over sqrt(K)."""
    rng = np.random.default_rng(8)
    T, H, K = 3, 16, 20
    contribs = rng.standard_normal((K, T, H))
    s = np.zeros((T, H))
    keep = lambda k: math.sqrt((k - 1) / k)
    for k in range(1, K + 1):
        c, _ = oracle_lib.post_norm_residual(contribs[k - 1], None, 0.0, k, np.zeros((T, H), np.float32))
        s = keep(k) * s + c
    np.testing.assert_allclose(s, contribs.sum(0) / math.sqrt(K), rtol=1e-12, atol=1e-12)
    # and the oracle's own stream update for one step equals keep*stream + contrib
    st = rng.standard_normal((T, H)).astype(np.float32)
    c, so = oracle_lib.post_norm_residual(contribs[0], None, 0.0, 20, st)
    np.testing.assert_allclose(so, math.sqrt(19 / 20) * st.astype(np.float64) + contribs[0] / math.sqrt(20), rtol=1e-14)


def test_post_norm_properties(oracle_lib):
    rng = np.random.default_rng(9)
    T, H = 4, 512
    o = rng.standard_normal((T, H)) * 3.0
    ones = np.ones(H, np.float32)
    z = np.zeros((T, H), np.float32)
    c1, _ = oracle_lib.post_norm_residual(o, ones, 1e-6, 1, z)           # step 1: contrib = n
    # unit mean square after the norm (gamma = 1), up to eps
    np.testing.assert_allclose((c1 ** 2).mean(1), 1.0, rtol=1e-6)
    # scale invariance: the norm cancels the routed scaling, up to eps
    c2, _ = oracle_lib.post_norm_residual(2.5 * o, ones, 1e-6, 1, z)
    np.testing.assert_allclose(c2, c1, rtol=1e-6)
    # gamma multiplies element-wise
    gamma = (1 + 0.02 * rng.standard_normal(H)).astype(np.float32)
    c3, _ = oracle_lib.post_norm_residual(o, gamma, 1e-6, 1, z)
    np.testing.assert_allclose(c3, c1 * gamma.astype(np.float64), rtol=1e-12)
    # without a norm weight the contribution is o itself
    c4, _ = oracle_lib.post_norm_residual(o, None, 1e-6, 4, z)
    np.testing.assert_allclose(c4, o / 2.0, rtol=1e-15)


# --------------------------------------------------------------------------
# Shapes vs the numbers the pages print
# --------------------------------------------------------------------------

def test_block_shape_matches_published_counts():
    with open(os.path.join(GOLDEN, "beam_counts.json")) as f:
        g = json.load(f)
    wl = W.WORKLOADS["decode"]
    H, I, E = wl.hidden, wl.inter, wl.n_experts
    assert H == g["hidden_size"]["value"] and I == g["intermediate_size"]["value"] and E == g["n_experts"]["value"]
    assert wl.n_group == g["n_group"]["value"] and E // wl.n_group == g["group_size"]["value"]
    assert wl.topk_group == g["topk_group"]["value"] and wl.top_k == g["experts_per_token"]["value"]
    assert wl.routed_scaling == g["routed_scaling"]["value"]
    per_expert = 3 * H * I                               # gate, up, down
    assert abs(per_expert / g["params_per_expert_approx"]["value"] - 1) < g["params_per_expert_approx"]["rel_tol"]
    moe = g["moe_layers"]["value"]
    assert moe + g["dense_layers"]["value"] == g["n_layers"]["value"]
    share = moe * E * per_expert / g["total_params"]["value"]
    assert abs(share - g["expert_param_share"]["value"]) < g["expert_param_share"]["abs_tol"]
    active = moe * wl.top_k * per_expert + g["replicated_params"]["value"]
    assert abs(active / g["active_params_approx"]["value"] - 1) < g["active_params_approx"]["rel_tol"]
    # two matrices per expert (no gate) would miss the published share badly
    assert abs(moe * E * 2 * H * I / g["total_params"]["value"] - g["expert_param_share"]["value"]) > 0.1

"""Property pins for the oracle's routing on random layouts and logits
(hypothesis): whatever the group layout, the selection must satisfy what the
method fixes -- at most topk_group groups, distinct experts, each chosen
expert at least as good as every unchosen candidate of a kept group, kept
groups the best by the sum of their two best biased scores (exhaustive over
group subsets), canonical order, and weights that are the unbiased scores
normalised to 1.  No GPU."""
import itertools

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st
from scipy.special import expit

LAYOUTS = [(E, G) for E in (8, 16, 32, 64) for G in (1, 2, 4, 8) if E // G >= 2]


@st.composite
def routing_case(draw):
    E, G = draw(st.sampled_from(LAYOUTS))
    gs = E // G
    kg = draw(st.integers(1, G))
    k = draw(st.integers(1, min(kg * gs, 12)))
    T = draw(st.integers(1, 6))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    logits = (rng.standard_normal((T, E)) * draw(st.sampled_from([0.1, 1.0, 4.0]))).astype(np.float32)
    bias = rng.uniform(-0.2, 0.2, E).astype(np.float32)
    return E, G, kg, k, logits, bias


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(routing_case())
def test_routing_properties(oracle_lib, case):
    E, G, kg, k, logits, bias = case
    gs = E // G
    r = oracle_lib.route_logits(logits, bias, G, kg, k)
    s = expit(logits.astype(np.float64))
    b32 = (s + bias.astype(np.float64)).astype(np.float32)
    for t in range(logits.shape[0]):
        idx = r.idx[t].tolist()
        assert len(set(idx)) == k and all(0 <= e < E for e in idx)
        kept = [j for j in range(G) if (r.kept_mask[t] >> j) & 1]
        assert len(kept) == kg
        assert {e // gs for e in idx} <= set(kept)
        # kept groups: the best total group score (sum of two best, FP32), ties to lower index
        gscore = [float(np.float32(np.sort(b32[t, j * gs:(j + 1) * gs])[-1]) +
                        np.float32(np.sort(b32[t, j * gs:(j + 1) * gs])[-2])) for j in range(G)]
        best = max(itertools.combinations(range(G), kg), key=lambda c: (sum(gscore[j] for j in c),
                                                                       [-j for j in c]))
        if r.gap_group[t] > 1e-6:
            assert set(kept) == set(best)
        # chosen experts dominate the other candidates; canonical order
        others = [e for e in range(E) if e // gs in kept and e not in idx]
        if others:
            assert b32[t, idx].min() >= b32[t, others].max()
        assert idx == sorted(idx, key=lambda e: (-float(b32[t, e]), e))
        sel = s[t, idx]
        np.testing.assert_allclose(r.w[t], sel / sel.sum(), rtol=1e-13)
        assert abs(r.w[t].sum() - 1.0) < 1e-12

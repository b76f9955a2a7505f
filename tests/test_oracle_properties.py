"""Property checks of the oracle over many random small layers (hypothesis): the routing is the
brute-force top-k of the logits under (logit desc, index asc), its weights are the renormalised
softmax of the chosen experts, the dispatch keeps exactly the first `capacity` assignments of each
expert in (slot, token) order, and the layer output is the weighted sum of the kept experts'
FFN rows.  Sizes stay tiny so each example runs in milliseconds."""
import itertools
import math

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from test_oracle_pins import _check_dispatch_invariants

CFS = [math.inf, 0.5, 1.0, 1.25, 2.0]


@st.composite
def layers(draw):
    E = draw(st.integers(1, 6))
    k = draw(st.integers(1, min(E, 3)))
    T = draw(st.integers(0, 24))
    H = draw(st.integers(1, 6))
    F = draw(st.integers(1, 5))
    cf = draw(st.sampled_from(CFS))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    f32 = lambda *s: rng.standard_normal(s).astype(np.float32)  # noqa: E731
    return dict(T=T, H=H, E=E, k=k, F=F, cf=cf, x=f32(T, H), Wg=f32(H, E), bg=f32(E), W1=f32(E, H, F),
                b1=f32(E, F), W2=f32(E, F, H), b2=f32(E, H))


SETTINGS = settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@SETTINGS
@given(layers())
def test_route_is_brute_force_topk_with_renormalised_softmax(L):
    r = oracle.route(L["x"], L["Wg"], L["bg"], L["k"], "f32")
    E, k = L["E"], L["k"]
    logits = L["x"].astype(np.float64) @ L["Wg"].astype(np.float64) + L["bg"].astype(np.float64)
    assert np.allclose(r.logits, logits, rtol=1e-12, atol=1e-12)
    for t in range(L["T"]):
        best = max(itertools.combinations(range(E), k),
                   key=lambda c: sorted(((r.logits[t, e], -e) for e in c), reverse=True))
        order = sorted(best, key=lambda e: (-r.logits[t, e], e))
        assert r.topk_idx[t].tolist() == order
        p = np.exp(r.logits[t] - r.logits[t].max())
        p /= p.sum()
        assert np.allclose(r.topk_w[t], p[order] / p[order].sum(), rtol=1e-12, atol=0)


@SETTINGS
@given(layers())
def test_dispatch_keeps_the_first_capacity_assignments(L):
    r = oracle.route(L["x"], L["Wg"], L["bg"], L["k"], "f32")
    d = oracle.dispatch(r.topk_idx, L["E"], L["cf"])
    _check_dispatch_invariants(r.topk_idx, L["E"], d)


@SETTINGS
@given(layers())
def test_output_is_the_weighted_sum_of_kept_expert_rows(L):
    f = oracle.forward(L["x"], L["Wg"], L["bg"], L["W1"], L["b1"], L["W2"], L["b2"], L["k"], L["cf"], "f32")
    if L["T"] == 0:
        assert f.out.shape[0] == 0
        return
    want = np.zeros((L["T"], L["H"]))
    for t in range(L["T"]):
        for s in range(L["k"]):
            if f.disp.dropped[t, s]:
                continue
            e = f.routing.topk_idx[t, s]
            y = oracle.expert_rows(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], np.array([t], np.int32),
                                   np.array([e], np.int32), "f32")
            want[t] += f.routing.topk_w[t, s] * y[0]
    assert np.allclose(f.out, want, rtol=1e-12, atol=1e-12)

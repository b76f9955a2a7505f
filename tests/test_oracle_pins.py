"""Pins of the fp64 oracle against facts fixed outside the oracle itself (CPU only).

Each pin checks the oracle against something other than its own code: textbook constants, closed
forms that follow from the MoE definitions on the pages ("MoE Training: Mixture of Experts":
Quick Start MoELayer; Core Concepts 2 Routing, 3 Load Balancing, 4 Expert Parallelism; Best
Practices 2 Capacity Factor; Advanced Patterns Mixtral block), library routines (numpy fp64
matmul, scipy logsumexp / softmax / erf / normal CDF), invariants and brute force on tiny inputs.
Every pin is chosen so that a plausible slip in the oracle (a dropped bias, a transposed operand, a
wrong sign, a wrong order of drops) fails it; ``test_planted_mistakes_are_caught`` demonstrates this
on copies of the inputs.
"""
import itertools
import math

import numpy as np
import pytest
from scipy import special, stats

import oracle
import synth

RNG_SEED = 1234


def _rand_layer(T, H, E, F, seed, dtype="f32", bias_std=0.1):
    cfg = synth.LayerConfig("t", T=T, H=H, E=E, k=1, F=F, CF=math.inf, dtype=dtype, seed=seed, bias_std=bias_std)
    inp = synth.make_inputs(cfg)
    # non-zero gate bias so a dropped bias term is visible
    inp.bg = synth.normal(seed, 99, (E,), 0.0, 0.5, dtype)
    return inp


def _f64(a, dtype):
    return synth.as_f64(a, dtype)


# ---------------------------------------------------------------- GELU ---------------------------

def test_gelu_textbook_values():
    # GELU(u) = u * Phi(u); Phi at 0.5, 1, 2 from standard normal tables
    assert oracle.gelu(0.0) == 0.0
    assert oracle.gelu(1.0) == pytest.approx(0.8413447460685429, abs=1e-15)
    assert oracle.gelu(-1.0) == pytest.approx(-(1 - 0.8413447460685429), abs=1e-15)
    assert oracle.gelu(2.0) == pytest.approx(2 * 0.9772498680518208, abs=1e-15)
    assert oracle.gelu(0.5) == pytest.approx(0.5 * 0.6914624612740131, abs=1e-15)
    assert oracle.gelu(40.0) == 40.0
    assert oracle.gelu(-40.0) == pytest.approx(0.0, abs=1e-300)


def test_gelu_matches_normal_cdf():
    for u in np.linspace(-8, 8, 161):
        assert oracle.gelu(u) == pytest.approx(u * stats.norm.cdf(u), rel=1e-14, abs=1e-15)


# ---------------------------------------------------------------- SiLU ---------------------------

def test_silu_textbook_values():
    # SiLU(u) = u * sigmoid(u); sigmoid(1) = e/(1+e), sigmoid(2) = 1/(1+e^-2)
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(1.0) == pytest.approx(math.e / (1 + math.e), abs=1e-15)
    assert oracle.silu(2.0) == pytest.approx(2 / (1 + math.exp(-2.0)), abs=1e-15)
    assert oracle.silu(-1.0) == pytest.approx(-1 / (1 + math.e), abs=1e-15)
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-16)
    assert oracle.silu(-40.0) == pytest.approx(-40.0 * math.exp(-40.0), rel=1e-12)


def test_silu_matches_expit_and_odd_part():
    for u in np.linspace(-12, 12, 241):
        assert oracle.silu(u) == pytest.approx(u * special.expit(u), rel=1e-14, abs=1e-300)
        # sigmoid(u) + sigmoid(-u) = 1  =>  SiLU(u) - SiLU(-u) = u
        assert oracle.silu(u) - oracle.silu(-u) == pytest.approx(u, abs=1e-14)


# ---------------------------------------------------------------- router -------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_route_logits_lse_softmax_vs_library(dtype):
    inp = _rand_layer(T=37, H=24, E=7, F=8, seed=11, dtype=dtype)
    r = oracle.route(inp.x, inp.Wg, inp.bg, k=3, dtype=dtype)
    x, Wg, bg = _f64(inp.x, dtype), _f64(inp.Wg, dtype), _f64(inp.bg, dtype)
    logits = x @ Wg + bg
    np.testing.assert_allclose(r.logits, logits, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r.lse, special.logsumexp(logits, axis=1), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(r.p, special.softmax(logits, axis=1), rtol=1e-12, atol=1e-15)


def test_route_topk_brute_force_and_renorm():
    """Over every k-subset, the chosen set is the unique one whose worst member beats every
    non-member under (logit desc, index asc); slots are in that order; weights are p renormalised."""
    inp = _rand_layer(T=64, H=16, E=6, F=8, seed=5)
    for k in (1, 2, 3, 6):
        r = oracle.route(inp.x, inp.Wg, inp.bg, k=k, dtype="f32")
        for t in range(64):
            lg = r.logits[t]
            key = lambda e: (lg[e], -e)  # noqa: E731
            winners = [set(S) for S in itertools.combinations(range(6), k)
                       if all(key(a) > key(b) for a in S for b in set(range(6)) - set(S))]
            assert len(winners) == 1
            assert set(r.topk_idx[t].tolist()) == winners[0]
            ks = [key(e) for e in r.topk_idx[t]]
            assert ks == sorted(ks, reverse=True)
            psel = special.softmax(lg)[r.topk_idx[t]]
            np.testing.assert_allclose(r.topk_w[t], psel / psel.sum(), rtol=1e-13)
            assert r.topk_w[t].sum() == pytest.approx(1.0, abs=1e-14)


def test_route_tie_break_lower_index_and_uniform_closed_form():
    """Wg = 0, bg = 0: all logits equal -> p = 1/E, top-k = {0..k-1}, w = 1/k, lse = ln E."""
    T, H, E, k = 9, 5, 8, 3
    x = synth.normal(3, 1, (T, H))
    Wg = np.zeros((H, E), np.float32)
    bg = np.zeros(E, np.float32)
    r = oracle.route(x, Wg, bg, k, "f32")
    assert (r.topk_idx == np.arange(k)[None, :]).all()
    np.testing.assert_allclose(r.topk_w, 1.0 / k, rtol=1e-15)
    np.testing.assert_allclose(r.p, 1.0 / E, rtol=1e-15)
    np.testing.assert_allclose(r.lse, math.log(E), rtol=1e-15)
    assert (r.margin == 0).all()


def test_route_k1_weight_is_one():
    inp = _rand_layer(T=20, H=8, E=5, F=8, seed=8)
    r = oracle.route(inp.x, inp.Wg, inp.bg, 1, "f32")
    assert (r.topk_w == 1.0).all()
    assert (r.topk_idx[:, 0] == np.argmax(r.logits, axis=1)).all()  # Switch argmax routing


def test_route_margin():
    inp = _rand_layer(T=30, H=8, E=6, F=8, seed=9)
    k = 2
    r = oracle.route(inp.x, inp.Wg, inp.bg, k, "f32")
    s = -np.sort(-r.logits, axis=1)
    np.testing.assert_allclose(r.margin, np.min(s[:, :k] - s[:, 1:k + 1], axis=1), rtol=0, atol=1e-15)


# ---------------------------------------------------------------- losses -------------------------

def test_losses_uniform_closed_form():
    """Equal logits: f and P uniform -> aux = 1 exactly; z = (ln E)^2; constant c -> (c + ln E)^2."""
    T, H, E, k = 16, 4, 8, 2
    x = synth.normal(4, 1, (T, H))
    r = oracle.route(x, np.zeros((H, E), np.float32), np.zeros(E, np.float32), k, "f32")
    # with ties every token picks {0,1}: f is not uniform -- use k = E to get uniform f
    r8 = oracle.route(x, np.zeros((H, E), np.float32), np.zeros(E, np.float32), E, "f32")
    aux, z = oracle.losses(r8.p, r8.lse, r8.topk_idx)
    assert aux == pytest.approx(1.0, abs=1e-15)
    assert z == pytest.approx(math.log(E) ** 2, rel=1e-15)
    # f one-hot-ish on {0,1} (each 1/2), P uniform 1/E -> aux = E * (1/2*1/E + 1/2*1/E) = 1
    aux2, _ = oracle.losses(r.p, r.lse, r.topk_idx)
    assert aux2 == pytest.approx(1.0, abs=1e-15)
    c = 2.5
    rc = oracle.route(x, np.zeros((H, E), np.float32), np.full(E, c, np.float32), k, "f32")
    _, zc = oracle.losses(rc.p, rc.lse, rc.topk_idx)
    assert zc == pytest.approx((c + math.log(E)) ** 2, rel=1e-14)


def test_losses_worked_example_two_experts():
    """H=1, x=1, Wg=[[1,0]]: both tokens have logits (1,0) -> p=(e/(e+1), 1/(e+1)), both pick expert 0.
    f=(1,0), P=p -> aux = 2 e/(e+1); z = ln(e+1)^2."""
    x = np.ones((2, 1), np.float32)
    Wg = np.array([[1.0, 0.0]], np.float32)
    r = oracle.route(x, Wg, np.zeros(2, np.float32), 1, "f32")
    aux, z = oracle.losses(r.p, r.lse, r.topk_idx)
    e = math.e
    assert aux == pytest.approx(2 * e / (e + 1), rel=1e-15)
    assert z == pytest.approx(math.log(e + 1) ** 2, rel=1e-15)


def test_losses_one_hot_limit_equals_E():
    """f and P both concentrated on one expert -> aux -> E (upper bound)."""
    T, H, E, k = 10, 3, 6, 1
    x = synth.normal(6, 1, (T, H))
    bg = np.zeros(E, np.float32)
    bg[2] = 60.0
    r = oracle.route(x, np.zeros((H, E), np.float32), bg, k, "f32")
    aux, _ = oracle.losses(r.p, r.lse, r.topk_idx)
    assert aux == pytest.approx(E, rel=1e-20 + 1e-12)
    assert aux <= E


def test_losses_bound_and_permutation_invariance():
    inp = _rand_layer(T=50, H=12, E=5, F=8, seed=21)
    r = oracle.route(inp.x, inp.Wg, inp.bg, 2, "f32")
    aux, z = oracle.losses(r.p, r.lse, r.topk_idx)
    assert 0 < aux <= 5
    perm = np.random.default_rng(RNG_SEED).permutation(50)
    aux2, z2 = oracle.losses(r.p[perm], r.lse[perm], r.topk_idx[perm])
    assert aux2 == pytest.approx(aux, rel=1e-14) and z2 == pytest.approx(z, rel=1e-14)


def test_losses_empty_batch():
    aux, z = oracle.losses(np.zeros((0, 4)), np.zeros(0), np.zeros((0, 2), np.int32))
    assert aux == 0.0 and z == 0.0


# ---------------------------------------------------------------- capacity / dispatch ------------

def test_capacity_values():
    assert oracle.capacity(1.25, 8192, 1, 128) == 80
    assert oracle.capacity(math.inf, 8192, 1, 128) is None
    assert oracle.capacity(1.0, 10, 1, 3) == 4  # ceil(10/3)
    assert oracle.capacity(2.0, 256, 2, 4) == 256
    assert oracle.capacity(1.25, 4096, 2, 8) == 1280


def _check_dispatch_invariants(idx, E, d):
    T, k = idx.shape
    cap = d.cap
    drops = int(d.dropped.sum())
    assert d.expert_counts.sum() == T * k - drops
    assert (d.cnt_pre == np.bincount(idx.ravel(), minlength=E)).all()
    if cap is not None:
        assert (d.expert_counts <= cap).all()
        assert (d.expert_counts == np.minimum(d.cnt_pre, cap)).all()
    else:
        assert drops == 0
    assert (np.diff(d.offsets) == d.expert_counts).all() and d.offsets[0] == 0
    # rows are a bijection onto the kept assignments
    kept = [(t, s) for t in range(T) for s in range(k) if not d.dropped[t, s]]
    assert sorted(zip(d.row_token.tolist(), d.row_slot.tolist())) == sorted(kept)
    for t, s in kept:
        r = d.row_of[t, s]
        assert d.row_token[r] == t and d.row_slot[r] == s
        assert d.offsets[idx[t, s]] <= r < d.offsets[idx[t, s] + 1]
    assert (d.row_of[d.dropped == 1] == -1).all()
    # stability: inside each expert's segment rows go (slot, token) increasing
    for e in range(E):
        seg = list(zip(d.row_slot[d.offsets[e]:d.offsets[e + 1]], d.row_token[d.offsets[e]:d.offsets[e + 1]]))
        assert seg == sorted(seg)
    # the kept set of each expert is the first `cap` of its assignments in (slot, token) order
    for e in range(E):
        order = [(s, t) for s in range(k) for t in range(T) if idx[t, s] == e]
        keep = order if cap is None else order[:cap]
        assert sorted(keep) == sorted((s, t) for (s, t) in order if not d.dropped[t, s])


@pytest.mark.parametrize("k,cf", [(1, 1.25), (2, 1.25), (2, 1.0), (3, 0.5), (2, math.inf), (1, 100.0)])
def test_dispatch_invariants_random(k, cf):
    rng = np.random.default_rng(k * 100 + int(min(cf, 99) * 10))
    T, E = 97, 6
    # skewed assignments: distinct experts per token, expert 0 popular
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        p = np.array([6, 3, 2, 1, 1, 1], float)
        idx[t] = rng.choice(E, size=k, replace=False, p=p / p.sum())
    d = oracle.dispatch(idx, E, cf)
    _check_dispatch_invariants(idx, E, d)


def test_dispatch_closed_form_same_expert():
    """Wg = 0 with distinct bg: every token picks the same expert (k=1); with CF=1.25 exactly
    cap = ceil(1.25*T/E) tokens -- the first cap in token order -- are kept."""
    T, H, E = 40, 4, 8
    x = synth.normal(7, 1, (T, H))
    bg = np.linspace(-1, 1, E).astype(np.float32)  # expert E-1 wins
    r = oracle.route(x, np.zeros((H, E), np.float32), bg, 1, "f32")
    assert (r.topk_idx[:, 0] == E - 1).all()
    d = oracle.dispatch(r.topk_idx, E, 1.25)
    cap = math.ceil(1.25 * T / E)
    assert d.cap == cap == 7
    assert d.expert_counts[E - 1] == cap and d.expert_counts[:E - 1].sum() == 0
    assert (d.dropped[:cap, 0] == 0).all() and (d.dropped[cap:, 0] == 1).all()
    assert d.row_token.tolist() == list(range(cap))


def test_dispatch_slot_major_drop_order():
    """Slot 0 of every token is placed before any slot 1: with cap=2 and tokens (0:[a,b], 1:[b,a],
    2:[a,b]) expert a keeps t0s0, t2s0 and drops t1s1; expert b keeps t1s0, t0s1 and drops t2s1."""
    idx = np.array([[0, 1], [1, 0], [0, 1]], np.int32)
    d = oracle.dispatch(idx, 2, cf=2 * 2 / (3 * 2))  # ceil(CF*T*k/E) = ceil(0.6667*6/2) = 2
    assert d.cap == 2
    assert d.dropped.tolist() == [[0, 0], [0, 1], [0, 1]]
    assert d.row_token.tolist() == [0, 2, 1, 0]
    assert d.row_slot.tolist() == [0, 0, 0, 1]


def test_dispatch_empty():
    d = oracle.dispatch(np.zeros((0, 2), np.int32), 4, math.inf)
    assert d.kept == 0 and (d.expert_counts == 0).all()


# ---------------------------------------------------------------- FFN / combine -----------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_expert_rows_vs_numpy_matmul(dtype):
    inp = _rand_layer(T=11, H=24, E=3, F=40, seed=31, dtype=dtype)
    tokens = np.array([0, 3, 10, 3, 7], np.int32)
    experts = np.array([2, 0, 1, 1, 2], np.int32)
    y = oracle.expert_rows(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, tokens, experts, dtype)
    x, W1, b1, W2, b2 = (_f64(a, dtype) for a in (inp.x, inp.W1, inp.b1, inp.W2, inp.b2))
    for i, (t, e) in enumerate(zip(tokens, experts)):
        u = x[t] @ W1[e] + b1[e]
        g = u * stats.norm.cdf(u)
        ref = g @ W2[e] + b2[e]
        np.testing.assert_allclose(y[i], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_expert_rows_silu_bias_free_vs_numpy_matmul(dtype):
    """Mixtral block expert: Linear(bias=False) -> SiLU -> Linear(bias=False); None biases are zeros."""
    inp = _rand_layer(T=11, H=24, E=3, F=40, seed=33, dtype=dtype)
    tokens = np.array([1, 4, 9, 4, 0, 10], np.int32)
    experts = np.array([0, 2, 1, 0, 2, 1], np.int32)
    y = oracle.expert_rows(inp.x, inp.W1, None, inp.W2, None, tokens, experts, dtype, act="silu")
    x, W1, W2 = (_f64(a, dtype) for a in (inp.x, inp.W1, inp.W2))
    for i, (t, e) in enumerate(zip(tokens, experts)):
        u = x[t] @ W1[e]
        ref = (u * special.expit(u)) @ W2[e]
        np.testing.assert_allclose(y[i], ref, rtol=1e-12, atol=1e-13)
    # with the biases present the result changes (they are not silently ignored) ...
    yb = oracle.expert_rows(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, tokens, experts, dtype, act="silu")
    assert not np.allclose(yb, y)
    # ... and the activation selector is honoured
    yg = oracle.expert_rows(inp.x, inp.W1, None, inp.W2, None, tokens, experts, dtype, act="gelu")
    assert not np.allclose(yg, y)


def test_route_without_gate_bias_equals_zero_bias():
    inp = _rand_layer(T=29, H=16, E=8, F=8, seed=37)
    a = oracle.route(inp.x, inp.Wg, None, 2, "f32")
    b = oracle.route(inp.x, inp.Wg, np.zeros(8, np.float32), 2, "f32")
    np.testing.assert_array_equal(a.logits, b.logits)
    np.testing.assert_array_equal(a.topk_idx, b.topk_idx)
    np.testing.assert_allclose(a.logits, inp.x.astype(np.float64) @ inp.Wg.astype(np.float64), rtol=1e-13,
                               atol=1e-14)


def test_mixtral_block_k_equals_E_is_dense_softmax_silu_mixture():
    """Bias-free gate and SiLU experts with k = E: out = sum_e softmax(x Wg)_e * FFN_e(x)."""
    T, H, E, F = 17, 12, 4, 20
    inp = _rand_layer(T=T, H=H, E=E, F=F, seed=45)
    f = oracle.forward(inp.x, inp.Wg, None, inp.W1, None, inp.W2, None, E, math.inf, "f32", act="silu")
    x = inp.x.astype(np.float64)
    p = special.softmax(x @ inp.Wg.astype(np.float64), axis=1)
    ref = np.zeros((T, H))
    for e in range(E):
        u = x @ inp.W1[e].astype(np.float64)
        ref += p[:, e:e + 1] * ((u * special.expit(u)) @ inp.W2[e].astype(np.float64))
    np.testing.assert_allclose(f.out, ref, rtol=1e-11, atol=1e-12)


def test_identical_experts_equal_dense_ffn():
    """All experts share weights and the k weights sum to 1 -> layer output = one dense FFN."""
    T, H, E, F, k = 23, 16, 5, 32, 2
    inp = _rand_layer(T=T, H=H, E=1, F=F, seed=41)
    W1 = np.repeat(inp.W1, E, 0)
    b1 = np.repeat(inp.b1, E, 0)
    W2 = np.repeat(inp.W2, E, 0)
    b2 = np.repeat(inp.b2, E, 0)
    Wg = synth.normal(41, 50, (H, E), 0, 0.3)
    bg = synth.normal(41, 51, (E,), 0, 0.3)
    f = oracle.forward(inp.x, Wg, bg, W1, b1, W2, b2, k, math.inf, "f32")
    x = inp.x.astype(np.float64)
    u = x @ inp.W1[0].astype(np.float64) + inp.b1[0]
    dense = (u * stats.norm.cdf(u)) @ inp.W2[0].astype(np.float64) + inp.b2[0]
    np.testing.assert_allclose(f.out, dense, rtol=1e-11, atol=1e-12)


def test_k_equals_E_is_dense_softmax_mixture():
    T, H, E, F = 19, 12, 4, 20
    inp = _rand_layer(T=T, H=H, E=E, F=F, seed=43)
    f = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, E, math.inf, "f32")
    x = inp.x.astype(np.float64)
    p = special.softmax(x @ inp.Wg.astype(np.float64) + inp.bg, axis=1)
    ref = np.zeros((T, H))
    for e in range(E):
        u = x @ inp.W1[e].astype(np.float64) + inp.b1[e]
        ref += p[:, e:e + 1] * ((u * stats.norm.cdf(u)) @ inp.W2[e].astype(np.float64) + inp.b2[e])
    np.testing.assert_allclose(f.out, ref, rtol=1e-11, atol=1e-12)


def test_forward_drops_contribute_nothing():
    """CF small enough to drop: out[t] = sum over kept slots only; all-dropped tokens are zero."""
    T, H, E, F, k = 40, 8, 4, 16, 2
    inp = _rand_layer(T=T, H=H, E=E, F=F, seed=47)
    f = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, k, 0.25, "f32")
    assert f.disp.dropped.sum() > 0
    allk = oracle.forward_tokens(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, f.routing.topk_idx, f.routing.topk_w, None,
                                 np.arange(T), "f32")
    ys = {}
    for t in range(T):
        ys[t] = oracle.expert_rows(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, np.array([t, t]), f.routing.topk_idx[t],
                                   "f32")
        ref = sum(f.routing.topk_w[t, s] * ys[t][s] for s in range(k) if not f.disp.dropped[t, s])
        ref = np.zeros(H) if isinstance(ref, int) else ref
        np.testing.assert_allclose(f.out[t], ref, rtol=1e-13, atol=1e-14)
        full = sum(f.routing.topk_w[t, s] * ys[t][s] for s in range(k))
        np.testing.assert_allclose(allk[t], full, rtol=1e-13, atol=1e-14)
    all_dropped = np.where(f.disp.dropped.all(axis=1))[0]
    assert len(all_dropped) > 0
    assert (f.out[all_dropped] == 0).all()


def test_forward_token_subset_matches_full():
    T, H, E, F, k = 30, 8, 4, 12, 2
    inp = _rand_layer(T=T, H=H, E=E, F=F, seed=53)
    full = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, k, 1.0, "f32")
    sub = np.array([29, 0, 13], np.int32)
    part = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, k, 1.0, "f32", tokens=sub)
    np.testing.assert_array_equal(part.out, full.out[sub])


# ---------------------------------------------------------------- planted mistakes ---------------

def test_planted_mistakes_are_caught():
    """Mistakes planted in a Python restatement's inputs (not in the oracle) show the pins have teeth:
    a transposed gate, a dropped gate bias and a flipped drop order each change the checked values."""
    inp = _rand_layer(T=37, H=24, E=7, F=8, seed=11)
    r = oracle.route(inp.x, inp.Wg, inp.bg, 3, "f32")
    x, Wg, bg = inp.x.astype(np.float64), inp.Wg.astype(np.float64), inp.bg.astype(np.float64)
    assert not np.allclose(r.logits, x @ Wg)  # dropped bias is visible
    Wsq = synth.normal(2, 2, (7, 7))
    r2 = oracle.route(synth.normal(2, 3, (5, 7)), Wsq, np.zeros(7, np.float32), 2, "f32")
    xs = synth.normal(2, 3, (5, 7)).astype(np.float64)
    assert not np.allclose(r2.logits, xs @ Wsq.T.astype(np.float64))  # transposed gate is visible
    idx = np.array([[0, 1], [1, 0], [0, 1]], np.int32)
    d = oracle.dispatch(idx, 2, 2 * 2 / 6)
    token_major_drop = [[0, 0], [1, 0], [0, 1]]  # what token-major order would give
    assert d.dropped.tolist() != token_major_drop


# ---------------------------------------------------------------- expert-choice routing ---------

def test_ec_capacity_values():
    assert oracle.ec_capacity(1.0, 4096, 2, 8) == 1024
    assert oracle.ec_capacity(1.25, 8192, 1, 128) == 80
    assert oracle.ec_capacity(1.0, 10, 1, 3) == 4  # ceil(10/3)
    assert oracle.ec_capacity(math.inf, 77, 2, 5) == 77
    assert oracle.ec_capacity(50.0, 77, 2, 5) == 77  # never more than T


def test_ec_brute_force_topC_per_expert():
    """The chosen set of every expert is the unique C-subset whose worst member beats every other token
    under (logit, -token); listed in ascending token order."""
    rng = np.random.default_rng(5)
    T, E, C = 8, 3, 3
    logits = np.round(rng.normal(size=(T, E)), 1)  # rounding makes ties likely
    ec = oracle.expert_choice(logits, C)
    for e in range(E):
        key = lambda t: (logits[t, e], -t)  # noqa: E731
        winners = [S for S in itertools.combinations(range(T), C)
                   if min(key(t) for t in S) > max(key(t) for t in range(T) if t not in S)]
        assert len(winners) == 1
        assert ec.chosen[e].tolist() == sorted(winners[0])
        srt = sorted(range(T), key=key, reverse=True)
        assert ec.margin[e] == logits[srt[C - 1], e] - logits[srt[C], e]


def test_ec_perfect_balance_and_scalar_closed_form():
    """H = 1 and Wg[0] = (+1, -1): expert 0 takes the C largest x, expert 1 the C smallest (numpy
    argsort gives the closed form); every expert holds exactly C distinct tokens."""
    T, C = 50, 7
    x = synth.normal(7, 1, (T, 1))
    Wg = np.array([[1.0, -1.0]], np.float32)
    r = oracle.route(x, Wg, None, 1, "f32")
    ec = oracle.expert_choice(r.logits, C)
    xs = x[:, 0].astype(np.float64)
    assert ec.chosen[0].tolist() == sorted(np.argsort(-xs, kind="stable")[:C].tolist())
    assert ec.chosen[1].tolist() == sorted(np.argsort(xs, kind="stable")[:C].tolist())
    for e in range(2):
        assert len(set(ec.chosen[e].tolist())) == C and (np.diff(ec.chosen[e]) > 0).all()


def test_ec_equal_scores_take_the_first_tokens():
    """Wg = 0: every token has the same logit for a given expert, so each expert takes tokens 0..C-1."""
    T, H, E, C = 20, 8, 4, 6
    x = synth.normal(8, 1, (T, H))
    bg = np.array([0.3, -1.0, 2.0, 0.0], np.float32)
    r = oracle.route(x, np.zeros((H, E), np.float32), bg, 1, "f32")
    ec = oracle.expert_choice(r.logits, C)
    assert (ec.chosen == np.arange(C)).all()
    assert (ec.margin == 0).all()


def test_ec_losses_closed_form():
    """f_e = 1/E under expert choice, so aux = sum_e P_e = 1 (softmax rows sum to 1); z as for top-k."""
    inp = _rand_layer(T=31, H=16, E=6, F=8, seed=61)
    r = oracle.route(inp.x, inp.Wg, inp.bg, 1, "f32")
    aux, z = oracle.ec_losses(r.p, r.lse, 9)
    assert aux == pytest.approx(1.0, abs=1e-13)
    assert z == pytest.approx(float(np.mean(special.logsumexp(r.logits, axis=1) ** 2)), rel=1e-13)
    assert oracle.ec_losses(np.zeros((0, 6)), np.zeros(0), 1) == (0.0, 0.0)


def test_ec_full_capacity_is_dense_softmax_mixture():
    """C = T (CF = +inf): every expert processes every token, so out = sum_e p_e FFN_e(x), the same
    dense mixture as token choice with k = E."""
    T, H, E, F = 15, 12, 4, 20
    inp = _rand_layer(T=T, H=H, E=E, F=F, seed=63)
    f = oracle.forward_ec(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, 2, math.inf, "f32")
    assert f.ec.C == T
    x = inp.x.astype(np.float64)
    p = special.softmax(x @ inp.Wg.astype(np.float64) + inp.bg, axis=1)
    ref = np.zeros((T, H))
    for e in range(E):
        u = x @ inp.W1[e].astype(np.float64) + inp.b1[e]
        ref += p[:, e:e + 1] * ((u * stats.norm.cdf(u)) @ inp.W2[e].astype(np.float64) + inp.b2[e])
    np.testing.assert_allclose(f.out, ref, rtol=1e-11, atol=1e-12)


def test_ec_forward_per_token_sum_and_unchosen_tokens():
    """out[t] = sum over the experts that chose t of p[t,e] * FFN_e(x_t), checked row by row with
    expert_rows; tokens chosen by no expert are exactly zero."""
    T, H, E, F = 40, 8, 4, 16
    inp = _rand_layer(T=T, H=H, E=E, F=F, seed=65)
    f = oracle.forward_ec(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, 1, 0.5, "f32", act="silu")
    assert f.ec.C == 5
    member = f.ec.member(T)
    assert (member.sum(axis=0) == 5).all()
    for t in range(T):
        es = np.where(member[t])[0].astype(np.int32)
        if len(es) == 0:
            assert (f.out[t] == 0).all()
            continue
        ys = oracle.expert_rows(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, np.full(len(es), t, np.int32), es, "f32",
                                act="silu")
        ref = sum(f.routing.p[t, e] * ys[i] for i, e in enumerate(es))
        np.testing.assert_allclose(f.out[t], ref, rtol=1e-13, atol=1e-14)
    assert (~member.any(axis=1)).sum() > 0


def test_ec_selects_on_logits_not_probabilities():
    """The page's expert-choice scores are the router outputs themselves: token 1 has the larger logit
    for expert 0 (3 > 2) but the smaller probability (0.5 < 0.88), and it is the one chosen."""
    logits = np.array([[2.0, 0.0], [3.0, 3.0]])
    ec = oracle.expert_choice(logits, 1)
    assert ec.chosen[0].tolist() == [1]
    assert ec.chosen[1].tolist() == [1]
    assert special.softmax(logits, axis=1)[0, 0] > special.softmax(logits, axis=1)[1, 0]


# ---------------------------------------------------------------- backward pass -----------------

@pytest.mark.parametrize("act", ["gelu", "silu"])
def test_act_grad_closed_forms_and_numeric_derivative(act):
    f = oracle.gelu if act == "gelu" else oracle.silu
    assert oracle.act_grad(0.0, act) == pytest.approx(0.5, abs=1e-15)  # Phi(0) = s(0) = 1/2
    if act == "gelu":
        # GELU'(1) = Phi(1) + phi(1)
        assert oracle.act_grad(1.0, act) == pytest.approx(0.8413447460685429 + 0.24197072451914337, abs=1e-14)
    else:
        # SiLU'(1) = s(1) (1 + 1 - s(1)) with s(1) = e/(1+e)
        s1 = math.e / (1 + math.e)
        assert oracle.act_grad(1.0, act) == pytest.approx(s1 * (2 - s1), abs=1e-15)
    for u in np.linspace(-6, 6, 49):
        h = 1e-5
        num = (f(u + h) - f(u - h)) / (2 * h)
        assert oracle.act_grad(u, act) == pytest.approx(num, abs=1e-9)
    assert oracle.act_grad(30.0, act) == pytest.approx(1.0, abs=1e-10)  # SiLU'(30) = 1 + 30 e^-30 + ...
    assert oracle.act_grad(-40.0, act) == pytest.approx(0.0, abs=1e-12)


def _fd_layer(seed, T=7, H=6, E=3, F=5, k=2, cf=math.inf, act="gelu", bias=True):
    cfg = synth.LayerConfig("fd", T=T, H=H, E=E, k=k, F=F, CF=cf, dtype="f32", seed=seed, bias_std=0.3, act=act,
                            bias=bias)
    inp = synth.make_inputs(cfg)
    if bias:
        inp.bg = synth.normal(seed, 98, (E,), 0.0, 0.4)
    dout = synth.normal(seed, 97, (T, H)).astype(np.float64)
    return cfg, inp, dout


@pytest.mark.parametrize("case", [
    dict(seed=71),                                  # GELU, biases, top-2, dropless
    dict(seed=72, act="silu", bias=False),          # the Mixtral block: SiLU, no biases
    dict(seed=73, cf=0.75),                         # capacity drops
    dict(seed=74, k=1, E=4),                        # top-1: the weight is constant, only the losses reach the gate
], ids=["gelu_bias", "silu_nobias", "drops", "top1"])
def test_backward_matches_central_differences(case):
    """Every gradient of L = sum(dout*out) + d_aux*aux + d_z*z against central differences of the oracle's
    own forward pass (fp64), at a few entries of every input; the step is the actual fp32 difference."""
    case = dict(case)
    seed = case.pop("seed")
    cfg, inp, dout = _fd_layer(seed, **case)
    d_aux, d_z = 0.37, -0.21
    r = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, "f32")
    assert r.margin.min() > 2e-2  # the routing cannot flip under the steps below
    g = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, "f32", dout, d_aux, d_z,
                        act=cfg.act)
    if cfg.CF < math.inf:
        assert oracle.dispatch(r.topk_idx, cfg.E, cfg.CF).dropped.sum() > 0
    names = ["x", "Wg", "W1", "W2"] + (["bg", "b1", "b2"] if cfg.bias else [])
    grads = dict(x=g.dx, Wg=g.dWg, bg=g.dbg, W1=g.dW1, b1=g.db1, W2=g.dW2, b2=g.db2)
    rng = np.random.default_rng(seed)
    for name in names:
        base = getattr(inp, name)
        for flat in rng.choice(base.size, size=min(6, base.size), replace=False):
            idx = np.unravel_index(flat, base.shape)
            lo, hi = base.copy(), base.copy()
            lo[idx] = np.float32(base[idx] - 1e-3)
            hi[idx] = np.float32(base[idx] + 1e-3)
            step = float(hi[idx]) - float(lo[idx])
            args = {n: getattr(inp, n) for n in ("x", "Wg", "bg", "W1", "b1", "W2", "b2")}
            args[name] = hi
            Lp = oracle.loss_of(args["x"], args["Wg"], args["bg"], args["W1"], args["b1"], args["W2"], args["b2"],
                                cfg.k, cfg.CF, "f32", dout, d_aux, d_z, act=cfg.act)
            args[name] = lo
            Lm = oracle.loss_of(args["x"], args["Wg"], args["bg"], args["W1"], args["b1"], args["W2"], args["b2"],
                                cfg.k, cfg.CF, "f32", dout, d_aux, d_z, act=cfg.act)
            assert grads[name][idx] == pytest.approx((Lp - Lm) / step, rel=1e-5, abs=1e-7), (name, idx)


def test_backward_top1_weight_gradient_does_not_reach_the_gate():
    """k = 1: the renormalised weight is 1 whatever the logits, so without the two losses the gate gets
    exactly zero gradient, while dw itself is not zero."""
    cfg, inp, dout = _fd_layer(75, k=1, E=4)
    g = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, 1, math.inf, "f32", dout, 0.0, 0.0)
    assert np.abs(g.dw).max() > 0.1
    assert np.abs(g.dlogits).max() < 1e-15 and np.abs(g.dWg).max() < 1e-15


def test_backward_sampled_columns_match_full():
    """bwd_expert_weights at a subset of FFN columns gives the same entries as the full gradient."""
    cfg, inp, dout = _fd_layer(76, T=9, F=7)
    g = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, 2, math.inf, "f32", dout, 0.1, 0.1)
    r = oracle.route(inp.x, inp.Wg, inp.bg, 2, "f32")
    e = 1
    toks, slots = np.where(r.topk_idx == e)
    cols = np.array([6, 0, 3], np.int32)
    r2, c1, b1s, b2s = oracle.bwd_expert_weights(inp.x, inp.W1, inp.b1, inp.W2, e, toks.astype(np.int32),
                                                 r.topk_w[toks, slots], dout, cols, "f32")
    np.testing.assert_allclose(r2, g.dW2[e][cols], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(c1, g.dW1[e][:, cols].T, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b1s, g.db1[e][cols], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b2s, g.db2[e], rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("case", [
    dict(seed=81, cf=1.0),                          # C = T k / E: some tokens unchosen, some chosen twice
    dict(seed=82, cf=math.inf, act="silu", bias=False),  # C = T: every expert sees every token
], ids=["ec_partial", "ec_all_tokens"])
def test_backward_expert_choice_matches_central_differences(case):
    """Expert-choice gradients against central differences of the oracle's expert-choice forward pass; the
    per-expert selection margins exceed the steps, so the choice cannot change."""
    case = dict(case)
    seed, cf = case.pop("seed"), case.pop("cf")
    cfg, inp, dout = _fd_layer(seed, T=9, **case)
    d_aux, d_z = 0.37, -0.21
    r = oracle.route(inp.x, inp.Wg, inp.bg, 1, "f32")
    C = oracle.ec_capacity(cf, cfg.T, cfg.k, cfg.E)
    ec = oracle.expert_choice(r.logits, C)
    assert ec.margin.min() > 2e-2
    g = oracle.backward_ec(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cf, "f32", dout, d_aux, d_z,
                           act=cfg.act)
    names = ["x", "Wg", "W1", "W2"] + (["bg", "b1", "b2"] if cfg.bias else [])
    grads = dict(x=g.dx, Wg=g.dWg, bg=g.dbg, W1=g.dW1, b1=g.db1, W2=g.dW2, b2=g.db2)
    rng = np.random.default_rng(seed)
    for name in names:
        base = getattr(inp, name)
        for flat in rng.choice(base.size, size=min(6, base.size), replace=False):
            idx = np.unravel_index(flat, base.shape)
            lo, hi = base.copy(), base.copy()
            lo[idx] = np.float32(base[idx] - 1e-3)
            hi[idx] = np.float32(base[idx] + 1e-3)
            step = float(hi[idx]) - float(lo[idx])
            args = {n: getattr(inp, n) for n in ("x", "Wg", "bg", "W1", "b1", "W2", "b2")}
            args[name] = hi
            Lp = oracle.loss_of_ec(args["x"], args["Wg"], args["bg"], args["W1"], args["b1"], args["W2"], args["b2"],
                                   cfg.k, cf, "f32", dout, d_aux, d_z, act=cfg.act)
            args[name] = lo
            Lm = oracle.loss_of_ec(args["x"], args["Wg"], args["bg"], args["W1"], args["b1"], args["W2"], args["b2"],
                                   cfg.k, cf, "f32", dout, d_aux, d_z, act=cfg.act)
            assert grads[name][idx] == pytest.approx((Lp - Lm) / step, rel=1e-5, abs=1e-7), (name, idx)


def test_min_capacity_lower_bound():
    """Core Concepts 4's "min_capacity": the capacity never falls below it (0 = no bound); dispatch keeps
    exactly min(count, max(ceil(CF*T*k/E), min_capacity)) per expert, first in slot-major order."""
    assert oracle.capacity(0.25, 40, 1, 4) == 3 and oracle.capacity(0.25, 40, 1, 4, min_capacity=4) == 4
    assert oracle.capacity(2.0, 40, 1, 4, min_capacity=4) == 20  # the bound does not bind
    assert oracle.capacity(math.inf, 40, 1, 4, min_capacity=4) is None
    assert oracle.ec_capacity(0.02, 100, 1, 4, min_capacity=6) == 6
    assert oracle.ec_capacity(0.5, 10, 1, 1, min_capacity=50) == 10  # never more than T
    idx = np.zeros((40, 1), np.int32)  # every token picks expert 0
    d = oracle.dispatch(idx, 4, 0.25, min_capacity=4)
    assert d.cap == 4 and d.expert_counts.tolist() == [4, 0, 0, 0]
    assert d.dropped[:4].sum() == 0 and d.dropped[4:].all()


# ------------------------------------------------------------------ backward with a given routing -------------
def test_renorm_weights_closed_forms():
    """The Quick Start's renormalisation over a given selection: hand-computed values, the slot order kept,
    any selection (not only the top-k), and the sum-to-one and ratio invariants."""
    p = np.array([[0.5, 0.3, 0.2], [0.1, 0.6, 0.3]])
    w = oracle.renorm_weights(p, np.array([[2, 0], [0, 2]], np.int32))
    assert w[0, 0] == pytest.approx(0.2 / 0.7, abs=1e-16) and w[0, 1] == pytest.approx(0.5 / 0.7, abs=1e-16)
    assert w[1, 0] == pytest.approx(0.1 / 0.4, abs=1e-16) and w[1, 1] == pytest.approx(0.3 / 0.4, abs=1e-16)
    rng = np.random.default_rng(5)
    q = rng.dirichlet(np.ones(7), size=50)
    idx = np.array([rng.choice(7, size=3, replace=False) for _ in range(50)], np.int32)
    w = oracle.renorm_weights(q, idx)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    sel = np.take_along_axis(q, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(w[:, 0] / w[:, 1], sel[:, 0] / sel[:, 1], rtol=1e-13)
    # k = 1: the weight is exactly one whatever the selection
    assert (oracle.renorm_weights(q, idx[:, :1]) == 1.0).all()


def test_renorm_weights_equal_the_routers_own():
    """Fed the oracle's own top-k, the given-routing weights equal route()'s renormalised weights (two
    statements of the same division: numpy here, the C loop there)."""
    cfg = synth.LayerConfig("rw", T=64, H=16, E=6, k=3, F=8, CF=math.inf, dtype="f32", seed=31)
    inp = synth.make_inputs(cfg)
    r = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, "f32")
    np.testing.assert_allclose(oracle.renorm_weights(r.p, r.topk_idx), r.topk_w, rtol=1e-14, atol=1e-16)


@pytest.mark.parametrize("cf", [math.inf, 0.75], ids=["dropless", "drops"])
def test_backward_given_own_routing_equals_default(cf):
    """backward(..., topk_idx=, dropped=) fed the oracle's own routing and drops gives every gradient of the
    default call, to rounding."""
    cfg, inp, dout = _fd_layer(91, T=11, cf=cf)
    r = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, "f32")
    d = oracle.dispatch(r.topk_idx, cfg.E, cf)
    if cf < math.inf:
        assert d.dropped.sum() > 0
    a = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cf, "f32", dout, 0.3, 0.2)
    b = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cf, "f32", dout, 0.3, 0.2,
                        topk_idx=r.topk_idx, dropped=d.dropped)
    for n in ("dx", "dWg", "dbg", "dW1", "db1", "dW2", "db2", "dw", "dlogits"):
        np.testing.assert_allclose(getattr(b, n), getattr(a, n), rtol=1e-15, atol=1e-15, err_msg=n)


def test_backward_given_routing_matches_central_differences():
    """The branch the GPU parity tests take: a given selection that is NOT the top-k (slots reversed for some
    tokens, a lower-ranked expert for others) and a given drop mask that is not the capacity rule's.  Every
    gradient must equal central differences of the loss with that routing held fixed; renormalising over
    the wrong axis, using the top-k weights, or letting a dropped slot contribute each fails here."""
    cfg, inp, dout = _fd_layer(92, T=9, E=4)
    r = oracle.route(inp.x, inp.Wg, inp.bg, 3, "f32")  # top-3 order, to take a lower-ranked expert from
    idx = r.topk_idx[:, :2].copy()
    idx[0::3] = idx[0::3, ::-1]          # reversed slot order
    idx[1::3, 1] = r.topk_idx[1::3, 2]   # the third-best expert in slot 1
    dropped = np.zeros((cfg.T, 2), np.uint8)
    dropped[2, 0] = dropped[5, 1] = 1
    dropped[7] = 1                       # every slot of token 7 dropped
    d_aux, d_z = 0.37, -0.21
    g = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, 2, math.inf, "f32", dout, d_aux, d_z,
                        topk_idx=idx, dropped=dropped)
    assert (g.dw[dropped.astype(bool)] == 0).all()
    grads = dict(x=g.dx, Wg=g.dWg, bg=g.dbg, W1=g.dW1, b1=g.db1, W2=g.dW2, b2=g.db2)
    rng = np.random.default_rng(92)
    for name in ("x", "Wg", "bg", "W1", "b1", "W2", "b2"):
        base = getattr(inp, name)
        for flat in rng.choice(base.size, size=min(6, base.size), replace=False):
            at = np.unravel_index(flat, base.shape)
            lo, hi = base.copy(), base.copy()
            lo[at] = np.float32(base[at] - 1e-3)
            hi[at] = np.float32(base[at] + 1e-3)
            step = float(hi[at]) - float(lo[at])
            args = {n: getattr(inp, n) for n in ("x", "Wg", "bg", "W1", "b1", "W2", "b2")}
            vals = []
            for v in (hi, lo):
                args[name] = v
                vals.append(oracle.loss_of_given(args["x"], args["Wg"], args["bg"], args["W1"], args["b1"], args["W2"],
                                                 args["b2"], idx, dropped, "f32", dout, d_aux, d_z))
            assert grads[name][at] == pytest.approx((vals[0] - vals[1]) / step, rel=1e-5, abs=1e-7), (name, at)
    # the fixed-routing loss itself reduces to the oracle's forward when fed the oracle's own routing
    own = oracle.route(inp.x, inp.Wg, inp.bg, 2, "f32")
    dd = oracle.dispatch(own.topk_idx, cfg.E, math.inf)
    assert oracle.loss_of_given(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, own.topk_idx, dd.dropped,
                                "f32", dout, d_aux, d_z) == pytest.approx(
        oracle.loss_of(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, 2, math.inf, "f32", dout, d_aux, d_z),
        rel=1e-14)

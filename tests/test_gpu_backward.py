"""Parity of the backward pass on the GPU against the fp64 oracle's chain rule, through the C ABI.

The GPU's own routing (top-k, drops) is fed to the oracle, so a near-tie flip cannot move a
gradient.  Tolerance, per gradient tensor: max|d| <= 4e-2 * RMS(ref) and a relative Frobenius error
<= 1e-2 (the GPU keeps dout rows, du, h and u in bf16 between the GEMMs, so each weight-gradient
product carries two bf16 roundings; the oracle is fp64 throughout).

  small layers   every gradient in full: dx, dWg, dbg, dW1, db1, dW2, db2 and the per-slot dw
  Mixtral shape  dx and dw on tokens of every expert segment, dW1 / dW2 / db1 on one FFN column in
                 every 256-column tile of every expert plus the last tile's, db2 in full, dWg / dbg
                 in full from the oracle's router backward fed the GPU's dw (every token's dw
                 would need every token's expert output)
"""
import math

import numpy as np
import pytest

import oracle
import synth
from moe_testlib import TOL_BWD_FRO, TOL_BWD_MAX, fro_rel, rms_rel, shape_of, stratified_columns, upload

pytestmark = pytest.mark.gpu

D_AUX, D_Z = 0.01, 0.001  # the loss coefficients the pages quote (Core Concepts 3)


def _cfg(name, T, H, E, k, F, CF, seed, **kw):
    return synth.LayerConfig(name, T=T, H=H, E=E, k=k, F=F, CF=CF, dtype="bf16", seed=seed, **kw)


SMALL = [
    _cfg("bwd_single_tiles", 200, 128, 4, 2, 256, math.inf, 51),        # 128-row tiles, N = 128 / 256
    _cfg("bwd_ragged", 100, 128, 6, 3, 192, 1.0, 52),                    # N = 192 -> 64-wide tiles, drops
    _cfg("bwd_pair_tiles", 1500, 256, 4, 2, 512, 1.1, 53),               # CTA-pair dgrad, half tiles, drops
    _cfg("bwd_silu_nobias", 600, 256, 4, 2, 512, 1.25, 54, act="silu", bias=False),
    _cfg("bwd_top1", 300, 128, 8, 1, 256, 1.25, 55),
]


def _lib():
    import sparse_mixture_experts_23_b200 as moe
    from sparse_mixture_experts_23_b200 import build as moe_build

    moe_build.build()
    return moe


def _run(cfg, dout, inp=None):
    import torch

    moe = _lib()
    inp = inp or synth.make_inputs(cfg)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp), train=True)
    buf.forward_train()
    grads = buf.make_grads()
    dout_d = torch.from_numpy(dout.astype(np.float32)).cuda()
    buf.backward(dout_d, grads, D_AUX, D_Z)
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK
    res = {n: t.cpu().numpy().astype(np.float64) for n, t in grads.items()}
    res.update(inp=inp, topk_idx=buf.topk_idx.cpu().numpy(), dropped=buf.dropped.cpu().numpy(),
               topk_w=buf.topk_w.cpu().numpy().astype(np.float64), launches=moe.moe_last_launch_count(),
               out=buf.out.cpu().numpy())
    # the training forward gives the same out as the inference forward
    buf2 = moe.MoEBuffers(shape_of(cfg), upload(inp))
    buf2.forward()
    torch.cuda.synchronize()
    res["out_inference"] = buf2.out.cpu().numpy()
    del buf, buf2
    torch.cuda.empty_cache()
    return res


def _check(name, got, ref, per_expert: bool = False):
    """max|d| <= 4e-2 RMS(ref) (per leading index when per_expert) and Frobenius <= 1e-2 overall.  The
    error against one RMS over the whole tensor is printed beside the per-expert one."""
    glob = rms_rel(got, ref)
    if per_expert:
        err = max(rms_rel(got[e], ref[e]) for e in range(ref.shape[0]) if np.any(ref[e]))
    else:
        err = glob
    fro = fro_rel(got, ref)
    print(f"  {name}: max {err:.3e} x RMS{' (per expert)' if per_expert else ''}, global-RMS {glob:.3e}, "
          f"Frobenius {fro:.3e}")
    assert err <= TOL_BWD_MAX and fro <= TOL_BWD_FRO, (name, err, fro)


def _check_experts(name, gots, refs):
    """The per-expert rule over per-expert arrays of different sizes (each expert's own column set)."""
    err = max(rms_rel(g, r) for g, r in zip(gots, refs) if np.any(r))
    cat_g = np.concatenate([np.ravel(g) for g in gots])
    cat_r = np.concatenate([np.ravel(r) for r in refs])
    glob, fro = rms_rel(cat_g, cat_r), fro_rel(cat_g, cat_r)
    print(f"  {name}: max {err:.3e} x RMS (per expert), global-RMS {glob:.3e}, Frobenius {fro:.3e}")
    assert err <= TOL_BWD_MAX and fro <= TOL_BWD_FRO, (name, err, fro)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_backward_small_all_gradients(cfg):
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run(cfg, dout)
    inp = r["inp"]
    # same out as the inference forward: bit for bit when at most two fp32 adds meet in an element
    if cfg.k <= 2:
        assert np.array_equal(r["out"], r["out_inference"])
    else:
        np.testing.assert_allclose(r["out"], r["out_inference"], rtol=0, atol=1e-6 * np.abs(r["out"]).max())
    ref = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, dout,
                          D_AUX, D_Z, act=cfg.act, topk_idx=r["topk_idx"], dropped=r["dropped"])
    print(cfg.name)
    _check("dw", r["dw"], ref.dw)
    assert (r["dw"][r["dropped"].astype(bool)] == 0).all()
    _check("dx", r["dx"], ref.dx)
    _check("dW1", r["dW1"], ref.dW1, per_expert=True)
    _check("dW2", r["dW2"], ref.dW2, per_expert=True)
    _check("dWg", r["dWg"], ref.dWg)
    if cfg.bias:
        _check("db1", r["db1"], ref.db1, per_expert=True)
        _check("db2", r["db2"], ref.db2, per_expert=True)
        _check("dbg", r["dbg"], ref.dbg)
    else:
        assert "db1" not in r and "dbg" not in r
    assert r["launches"] == (8 if cfg.bias else 7)


def _slots_parallel(inp, cfg, pairs, dout, w):
    """oracle.bwd_slot over (token, slot, expert) triples on a thread pool (the ctypes calls release the
    GIL): returns {(t, s): (dx part, dw)}."""
    from concurrent.futures import ThreadPoolExecutor

    def one(p):
        t, s, e = p
        dxp, dws, _ = oracle.bwd_slot(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, t, e, dout[t], w[t, s], cfg.dtype, cfg.act)
        return (t, s), (dxp, dws)

    with ThreadPoolExecutor(max_workers=oracle.max_threads()) as ex:
        return dict(ex.map(one, pairs))


def test_backward_mixtral_shape_stratified():
    """Mixtral shape, every expert covered.  dx and dw on the tokens of the first, last and a random row of
    every expert segment; dW1 / dW2 / db1 on one FFN column in every 256-column tile of every expert (so
    every N tile of the dgrad GEMM, every M tile of dW2 and every N tile of dW1) plus the last tile's
    columns, each over all H; db2 in full; dWg / dbg in full from the oracle's router backward fed the
    GPU's dw (every token's dw would need every token's expert output)."""
    cfg = synth.CONFIGS["mixtral"]
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run(cfg, dout)
    inp = r["inp"]
    idx, drp, w = r["topk_idx"], r["dropped"], r["topk_w"]
    E, k = cfg.E, cfg.k
    print("mixtral")
    rng = np.random.default_rng(cfg.seed)
    toks = set()
    for e in range(E):
        tt, _ = np.where((idx == e) & (drp == 0))
        tt = np.sort(tt)  # the segment's rows are in (slot, token) order; any three of its tokens will do
        if tt.size:
            toks.update([int(tt[0]), int(tt[-1]), int(rng.choice(tt))])
    toks = np.array(sorted(toks), np.int32)
    pairs = [(int(t), s, int(idx[t, s])) for t in toks for s in range(k) if not drp[t, s]]
    assert {e for _, _, e in pairs} == set(range(E))
    parts = _slots_parallel(inp, cfg, pairs, dout, w)
    ex_dx = np.zeros((len(toks), cfg.H))
    ref_dw = np.zeros((len(toks), k))
    for i, t in enumerate(toks):
        for s in range(k):
            if (int(t), s) in parts:
                ex_dx[i] += parts[(int(t), s)][0]
                ref_dw[i, s] = parts[(int(t), s)][1]
    _check("dw (tokens of every expert)", r["dw"][toks], ref_dw)
    cnt_pre = np.bincount(idx.reshape(-1), minlength=E).astype(np.int32)
    dl, dWg, dbg, dxr = oracle.bwd_router(inp.x, inp.Wg, inp.bg, idx, cnt_pre, r["dw"], D_AUX, D_Z, cfg.dtype)
    _check("dWg (router fed the GPU's dw)", r["dWg"], dWg)
    _check("dbg (router fed the GPU's dw)", r["dbg"], dbg)
    _check("dx (tokens of every expert)", r["dx"][toks], ex_dx + dxr[toks])
    g2, g1, gb1, gb2 = [], [], [], []
    r2, r1, rb1, rb2 = [], [], [], []
    for e in range(E):
        cols = stratified_columns(cfg.F, seed=cfg.seed + e)
        tt, ss = np.where((idx == e) & (drp == 0))
        dW2r, dW1c, db1s, db2e = oracle.bwd_expert_weights(inp.x, inp.W1, inp.b1, inp.W2, e, tt.astype(np.int32),
                                                           w[tt, ss], dout, cols, cfg.dtype, cfg.act)
        r2.append(dW2r)
        r1.append(dW1c)
        rb1.append(db1s)
        rb2.append(db2e)
        g2.append(r["dW2"][e][cols])
        g1.append(r["dW1"][e][:, cols].T)
        gb1.append(r["db1"][e][cols])
        gb2.append(r["db2"][e])
    print(f"  {len(toks)} tokens, {sum(len(c) for c in r1)} FFN columns over {E} experts")
    _check_experts("dW2 (stratified columns)", g2, r2)
    _check_experts("dW1 (stratified columns)", g1, r1)
    _check_experts("db1 (stratified columns)", gb1, rb1)
    _check("db2", np.array(gb2), np.array(rb2), per_expert=True)


EC_SMALL = [
    _cfg("ec_bwd_small", 256, 128, 4, 2, 256, 1.0, 61, routing="expert_choice"),              # C = 128
    _cfg("ec_bwd_pair", 1500, 256, 4, 2, 512, 1.0, 62, routing="expert_choice"),              # C = 750: pair tiles
    _cfg("ec_bwd_silu_nobias", 300, 256, 8, 2, 512, 1.25, 63, routing="expert_choice", act="silu", bias=False),
    _cfg("ec_bwd_many_experts", 1024, 128, 64, 2, 128, 1.0, 64, routing="expert_choice"),     # C = 32, GEMM gate
]


@pytest.mark.parametrize("cfg", EC_SMALL, ids=lambda c: c.name)
def test_backward_expert_choice_all_gradients(cfg):
    """Expert choice: every gradient against the oracle's chain rule fed the GPU's choice; dw is [T,E]."""
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run(cfg, dout)
    inp = r["inp"]
    chosen = r["topk_idx"]  # [E, C] under expert choice
    ref = oracle.backward_ec(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, dout,
                             D_AUX, D_Z, act=cfg.act, chosen=chosen)
    print(cfg.name)
    member = np.zeros((cfg.T, cfg.E), bool)
    for e in range(cfg.E):
        member[chosen[e], e] = True
    # measured over the chosen pairs: the others are zero by definition (checked exactly) and would
    # deflate the RMS scale (E*C of T*E entries are live)
    _check("dw (chosen pairs)", r["dw"][member], ref.dw[member])
    assert (r["dw"][~member] == 0).all()
    _check("dx", r["dx"], ref.dx)
    _check("dW1", r["dW1"], ref.dW1, per_expert=True)
    _check("dW2", r["dW2"], ref.dW2, per_expert=True)
    _check("dWg", r["dWg"], ref.dWg)
    if cfg.bias:
        _check("db1", r["db1"], ref.db1, per_expert=True)
        _check("db2", r["db2"], ref.db2, per_expert=True)
        _check("dbg", r["dbg"], ref.dbg)
    assert r["launches"] == (9 if cfg.bias else 8)


def _run_bg(cfg, dout, bg_override=None):
    """_run with an optional gate-bias override (to force empty experts or drops)."""
    import torch

    moe = _lib()
    inp = synth.make_inputs(cfg)
    if bg_override is not None:
        inp.bg = synth.to_storage(bg_override, cfg.dtype)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp), train=True)
    buf.forward_train()
    grads = buf.make_grads()
    buf.backward(torch.from_numpy(dout.astype(np.float32)).cuda(), grads, D_AUX, D_Z)
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK
    res = {n: t.cpu().numpy().astype(np.float64) for n, t in grads.items()}
    res.update(inp=inp, topk_idx=buf.topk_idx.cpu().numpy(), dropped=buf.dropped.cpu().numpy(),
               counts=buf.expert_counts.cpu().numpy())
    return res


def _ref_tc(cfg, r, dout):
    inp = r["inp"]
    return oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, dout,
                           D_AUX, D_Z, act=cfg.act, topk_idx=r["topk_idx"], dropped=r["dropped"])


def test_backward_empty_experts_get_zero_weight_gradients():
    """Experts 4..7 are never chosen: their dW1, dW2, db1, db2 are exactly zero (the weight-gradient
    kernel's empty-segment path), the others match the oracle."""
    cfg = _cfg("bwd_empty", 200, 128, 8, 2, 256, math.inf, 71)
    bg = np.zeros(8)
    bg[4:] = -30.0
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run_bg(cfg, dout, bg)
    assert (r["counts"][4:] == 0).all()
    for n in ("dW1", "dW2", "db1", "db2"):
        assert (r[n][4:] == 0).all(), n
    ref = _ref_tc(cfg, r, dout)
    for n in ("dx", "dWg", "dbg"):
        _check(n, r[n], getattr(ref, n))
    for n in ("dW1", "dW2", "db1", "db2"):
        _check(n, r[n][:4], getattr(ref, n)[:4], per_expert=True)


def test_backward_heavy_drops():
    """cap = 16 with everyone wanting experts 0 and 1: most slots are dropped (dw = 0 there) and tokens with
    every slot dropped get only the router's part of dx."""
    cfg = _cfg("bwd_drops", 256, 64, 4, 2, 128, 0.125, 72)
    bg = np.array([3.0, 2.5, -5.0, -5.0])
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run_bg(cfg, dout, bg)
    assert r["dropped"].sum() > cfg.T
    assert (r["dw"][r["dropped"].astype(bool)] == 0).all()
    ref = _ref_tc(cfg, r, dout)
    live = ~r["dropped"].astype(bool)
    _check("dw (kept slots)", r["dw"][live], ref.dw[live])
    for n in ("dx", "dWg", "dbg"):
        _check(n, r[n], getattr(ref, n))
    for n in ("dW1", "dW2", "db1", "db2"):
        _check(n, r[n], getattr(ref, n), per_expert=True)


def test_backward_one_token():
    cfg = _cfg("bwd_one_token", 1, 64, 4, 2, 64, math.inf, 73)
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run_bg(cfg, dout)
    ref = _ref_tc(cfg, r, dout)
    for n in ("dx", "dWg", "dw"):
        _check(n, r[n], getattr(ref, n))
    used = sorted(set(r["topk_idx"][0].tolist()))
    for n in ("dW1", "dW2"):
        _check(n, r[n][used], getattr(ref, n)[used], per_expert=True)
        unused = [e for e in range(cfg.E) if e not in used]
        assert (r[n][unused] == 0).all()


def test_backward_deterministic_parts_repeat_bitwise():
    """dW1, dW2 (tensor-core accumulation in a fixed order), db1/db2 over one expert-major chunk order and
    the per-slot dw repeat bit for bit; dx, dWg and dbg use fp32 atomics and are compared within 1e-6."""
    import torch

    moe = _lib()
    cfg = _cfg("bwd_repeat", 600, 256, 4, 2, 512, 1.25, 74)
    inp = synth.make_inputs(cfg)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp), train=True)
    dout = torch.from_numpy(synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float32)).cuda()
    outs = []
    for _ in range(3):
        buf.forward_train()
        g = buf.make_grads()
        buf.backward(dout, g, D_AUX, D_Z)
        torch.cuda.synchronize()
        outs.append({n: t.cpu().numpy() for n, t in g.items()})
    for o in outs[1:]:
        for n in ("dW1", "dW2"):
            assert np.array_equal(o[n], outs[0][n]), n
        for n in ("dx", "dWg", "dbg", "db1", "db2", "dw"):
            scale = float(np.abs(outs[0][n]).max()) or 1.0
            assert np.max(np.abs(o[n] - outs[0][n])) <= 1e-6 * scale, n


F32_CASES = [
    synth.LayerConfig("bwd_f32_ragged", T=77, H=20, E=5, k=2, F=12, CF=math.inf, dtype="f32", seed=81),
    synth.LayerConfig("bwd_f32_drops", T=256, H=64, E=4, k=2, F=256, CF=1.0, dtype="f32", seed=82),
    synth.LayerConfig("bwd_f32_silu_nobias", T=100, H=32, E=4, k=1, F=64, CF=1.25, dtype="f32", seed=83, act="silu",
                      bias=False),
    synth.LayerConfig("bwd_f32_expert_choice", T=96, H=32, E=4, k=2, F=48, CF=1.0, dtype="f32", seed=84,
                      routing="expert_choice"),
]


@pytest.mark.parametrize("cfg", F32_CASES, ids=lambda c: c.name)
def test_backward_f32_all_gradients(cfg):
    """fp32 storage: every gradient on CUDA cores with fp32 intermediates, within the fp32 rule
    (max|d| <= 1e-4 max|ref| per tensor) of the oracle's chain rule fed the GPU's routing."""
    from moe_testlib import TOL_F32, normwise_rel

    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run(cfg, dout)
    inp = r["inp"]
    if cfg.routing == "expert_choice":
        ref = oracle.backward_ec(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype,
                                 dout, D_AUX, D_Z, act=cfg.act, chosen=r["topk_idx"])
    else:
        ref = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, dout,
                              D_AUX, D_Z, act=cfg.act, topk_idx=r["topk_idx"], dropped=r["dropped"])
    names = ["dx", "dWg", "dW1", "dW2", "dw"] + (["dbg", "db1", "db2"] if cfg.bias else [])
    for n in names:
        err = normwise_rel(r[n], getattr(ref, n))
        print(f"  {cfg.name} {n}: {err:.3e}")
        assert err <= TOL_F32, (n, err)


@pytest.mark.parametrize("T", [256, 272, 263, 300, 9])
def test_weight_gradient_segment_tails(T):
    """The weight-gradient GEMM's last stage of a segment: with a zero gate matrix every token picks the
    same two experts (the two largest gate biases), so both hold exactly T rows.  T = 256 leaves no ragged
    stage; 272 ends on a whole 16-row MMA step (nothing to zero); 263 and 300 zero 9 and 4 rows past the
    segment; 9 is a segment shorter than one MMA step.  dW1 and dW2 in full against the oracle, fed the
    GPU's routing."""
    cfg = _cfg(f"bwd_tail_{T}", T, 128, 4, 2, 256, math.inf, 57)
    inp = synth.make_inputs(cfg)
    inp.Wg = synth.to_storage(np.zeros((cfg.H, cfg.E)), cfg.dtype)
    inp.bg = synth.to_storage(np.array([0.5, 0.25, -0.25, -0.5]), cfg.dtype)
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    r = _run(cfg, dout, inp)
    assert (np.sort(r["topk_idx"], axis=1) == np.array([0, 1])).all()
    ref = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, dout,
                          D_AUX, D_Z, act=cfg.act, topk_idx=r["topk_idx"], dropped=r["dropped"])
    print(cfg.name)
    _check("dW1", r["dW1"], ref.dW1, per_expert=True)
    _check("dW2", r["dW2"], ref.dW2, per_expert=True)
    assert not r["dW1"][2:].any() and not r["dW2"][2:].any()  # experts without rows get zeros

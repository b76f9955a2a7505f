"""Loss sums for data-parallel replicas (moe_loss_sums, moe_losses_from_sums) against the oracle:
the additive sums of one batch, the losses rebuilt from them, and two replicas' summed sums giving
the losses of their concatenated batch.  Tolerances as in moe_testlib: counts exact, sums and
losses 1e-3 relative against the fp64 oracle, 1e-5 between two GPU reductions of the same data."""
import math

import numpy as np
import pytest

import oracle
import synth
from moe_testlib import TOL_LOSS, shape_of, upload

pytestmark = pytest.mark.gpu

TOL_SAME = 1e-5  # the layer's own loss reduction vs the loss-sum path (same partials, other order)

CFGS = [
    synth.LayerConfig("ls_f32", T=300, H=64, E=4, k=2, F=128, CF=math.inf, dtype="f32", seed=81),
    synth.LayerConfig("ls_bf16_drops", T=600, H=256, E=8, k=2, F=256, CF=1.0, dtype="bf16", seed=82),
    synth.LayerConfig("ls_ec", T=512, H=128, E=8, k=2, F=256, CF=1.0, dtype="bf16", seed=83,
                      routing="expert_choice"),
]


def _lib():
    import sparse_mixture_experts_23_b200 as moe
    from sparse_mixture_experts_23_b200 import build as moe_build

    moe_build.build()
    return moe


def _forward(cfg, dev):
    import torch

    moe = _lib()
    buf = moe.MoEBuffers(shape_of(cfg), dev)
    buf.forward()
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK
    return buf


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
def test_loss_sums_match_oracle(cfg):
    import torch

    moe = _lib()
    inp = synth.make_inputs(cfg)
    buf = _forward(cfg, upload(inp))
    sums = buf.loss_sums()
    torch.cuda.synchronize()
    s = sums.cpu().numpy().astype(np.float64)
    E = cfg.E
    assert s.shape == (moe.loss_sums_size(E),)
    ref = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, cfg.dtype)
    if cfg.routing == "expert_choice":
        C = moe.moe_capacity(shape_of(cfg))
        cnt = np.full(E, C, np.float64)
    else:
        cnt = np.bincount(buf.topk_idx.cpu().numpy().reshape(-1), minlength=E).astype(np.float64)
    assert np.array_equal(s[:E], cnt)  # pre-drop counts, exact
    assert np.allclose(s[E:2 * E], ref.p.sum(axis=0), rtol=TOL_LOSS, atol=0)
    assert s[2 * E] == pytest.approx(float((ref.lse ** 2).sum()), rel=TOL_LOSS)
    assert s[2 * E + 1] == cfg.T


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
def test_losses_from_sums_reproduce_the_layer_losses(cfg):
    import torch

    moe = _lib()
    buf = _forward(cfg, upload(synth.make_inputs(cfg)))
    got = moe.losses_from_sums(cfg.E, buf.loss_sums())
    single = buf.global_losses()  # no process group: this replica's own sums
    torch.cuda.synchronize()
    want = buf.losses.cpu().numpy()
    for g in (got.cpu().numpy(), single.cpu().numpy()):
        assert g[0] == pytest.approx(want[0], rel=TOL_SAME) and g[1] == pytest.approx(want[1], rel=TOL_SAME)


def test_two_replicas_give_the_whole_batch_losses():
    """Two replicas on disjoint halves of a batch: their summed sums give the oracle's losses of the
    whole batch (and the GPU's own losses of the whole batch), not the mean of their own losses."""
    import torch

    moe = _lib()
    cfg = synth.LayerConfig("ls_halves", T=1024, H=256, E=8, k=2, F=256, CF=math.inf, dtype="bf16", seed=84)
    inp = synth.make_inputs(cfg)
    dev = upload(inp)
    half = cfg.with_(T=cfg.T // 2)
    bufs = []
    for lo in (0, cfg.T // 2):
        d = dict(dev)
        d["x"] = dev["x"][lo:lo + half.T]
        bufs.append(_forward(half, d))
    total = bufs[0].loss_sums() + bufs[1].loss_sums()  # what an all-reduce over the two would hold
    got = moe.losses_from_sums(cfg.E, total).cpu().numpy()
    full = _forward(cfg, dev)
    torch.cuda.synchronize()
    idx = np.concatenate([b.topk_idx.cpu().numpy() for b in bufs])
    ref = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, cfg.dtype)
    aux, z = oracle.losses(ref.p, ref.lse, idx)
    assert abs(got[0] - aux) <= TOL_LOSS * aux and abs(got[1] - z) <= TOL_LOSS * z
    whole = full.losses.cpu().numpy()
    assert got[0] == pytest.approx(whole[0], rel=TOL_SAME) and got[1] == pytest.approx(whole[1], rel=TOL_SAME)
    own = [b.losses.cpu().numpy()[0] for b in bufs]
    assert abs(0.5 * (own[0] + own[1]) - aux) > 10 * TOL_SAME * aux


def test_empty_batch_gives_zero_sums_and_losses():
    import torch

    moe = _lib()
    cfg = synth.LayerConfig("ls_empty", T=0, H=64, E=4, k=2, F=64, CF=math.inf, dtype="bf16", seed=85)
    dev = {n: torch.zeros(1, dtype=torch.bfloat16, device="cuda") for n in ("x", "Wg", "bg", "W1", "b1", "W2", "b2")}
    buf = moe.MoEBuffers(shape_of(cfg), dev)
    buf.forward()
    sums = buf.loss_sums()
    losses = moe.losses_from_sums(cfg.E, sums)
    torch.cuda.synchronize()
    assert (sums.cpu().numpy() == 0).all() and (losses.cpu().numpy() == 0).all()

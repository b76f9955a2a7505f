"""moe_route_noalloc, the router entry point for callers that cannot allocate device memory.

Some callers cannot give the library a workspace: code that runs inside another runtime's fixed
device-memory pool, serving paths that forbid device allocation once they are up, or plugins whose
host framework owns every allocation.  moe_route_noalloc keeps the router's scratch in an array
built into the library instead.  This test calls it through the C ABI, twice in a row, and checks
each result against moe_route with a caller workspace and against the fp64 oracle, under the
tolerances of the other parity tests: top-k indices bit-exact except tokens whose oracle logit
margin is below 1e-4 (excluded and counted), weights 1e-4 relative, losses 1e-3 relative (against
the oracle's losses of the same selection).  It also checks the launch count, and that a shape too
large for the built-in array is refused before any launch.  This file is collected last so that a
run stopping at the first failure has run everything else.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from moe_testlib import NEAR_TIE, TOL_LOSS, TOL_W, reduce_launches, shape_of, upload

pytestmark = pytest.mark.gpu


def _check_routing(name, got_idx, got_w, got_l, ref_idx, ref_w, ref_l, near, E):
    """Indices equal outside near ties; weights within the rule on the agreeing tokens; losses within
    the rule, plus 2E/(T*k) of aux per token whose selection differs at a near tie (such a flip moves
    one count from one expert to another)."""
    mism = (got_idx != ref_idx).any(axis=1)
    assert not (mism & ~near).any(), (name, np.where(mism & ~near)[0][:10])
    ok = ~mism
    assert np.max(np.abs(got_w[ok] - ref_w[ok]) / np.abs(ref_w[ok])) <= TOL_W, name
    slack = np.array([2.0 * E / got_idx.size * int(mism.sum()), 0.0])
    assert np.all(np.abs(got_l - ref_l) <= TOL_LOSS * np.abs(ref_l) + slack), (name, got_l, ref_l)
    return int((mism & near).sum())


@pytest.mark.parametrize("name", ["tiny", "switch", "skew"])
def test_route_noalloc_matches_workspace_route_and_oracle(name):
    import torch

    import sparse_mixture_experts_23_b200 as moe
    from sparse_mixture_experts_23_b200 import build as moe_build

    moe_build.build()
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg, with_weights=False)
    dev = upload(synth.LayerInputs(cfg, inp.x, inp.Wg, inp.bg, np.zeros(1, inp.x.dtype), inp.b1,
                                   np.zeros(1, inp.x.dtype), inp.b2))
    shape = shape_of(cfg)
    buf = moe.MoEBuffers(shape, dev)
    buf.route()
    torch.cuda.synchronize()
    ws_idx = buf.topk_idx.cpu().numpy()
    ws_w = buf.topk_w.cpu().numpy().astype(np.float64)
    ws_l = buf.losses.cpu().numpy().astype(np.float64)
    ref = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, cfg.dtype)
    near = ref.margin < NEAR_TIE

    T, k = cfg.T, cfg.k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    losses = torch.empty(2, dtype=torch.float32, device="cuda")
    io = moe.IO(dev["x"].data_ptr(), dev["Wg"].data_ptr(), dev["bg"].data_ptr(), None, None, None, None, None,
                idx.data_ptr(), w.data_ptr(), None, None, losses.data_ptr(), losses.data_ptr() + 4)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        idx.fill_(-1)
        w.fill_(float("nan"))
        losses.fill_(float("nan"))
        assert moe.moe_route_noalloc(shape, io, stream) == moe.MOE_OK
        # one gate kernel (no [T,E] scratch here), plus a reduce only after the GEMM-epilogue gate
        assert moe.moe_last_launch_count() == 1 + reduce_launches(cfg)
        torch.cuda.synchronize()
        got_idx, got_w, got_l = idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), losses.cpu().numpy()
        # against the workspace router (the same kernels, or the tensor-core gate for 64 experts)
        n_ws = _check_routing(f"{name} vs moe_route", got_idx, got_w, got_l, ws_idx, ws_w, ws_l, near, cfg.E)
        # against the oracle: its losses taken on this call's own selection (a near-tie flip moves f)
        aux, z = oracle.losses(ref.p, ref.lse, got_idx)
        n_or = _check_routing(f"{name} vs oracle", got_idx, got_w, got_l, ref.topk_idx, ref.topk_w,
                              np.array([aux, z]), near, cfg.E)
        print(f"{name} call {call}: near-tie tokens {int(near.sum())}, differing from moe_route {n_ws}, "
              f"from the oracle {n_or}")

    big = moe.make_shape(1 << 20, 64, 256, 8, 64, math.inf, "bf16")  # needs far more than 1 MiB
    assert moe.moe_route_noalloc(big, io, stream) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_last_launch_count() == 0

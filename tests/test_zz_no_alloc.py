"""moe_route_noalloc, the router entry point for callers that cannot allocate device memory.

Some callers cannot give the library a workspace: code that runs inside another runtime's fixed
device-memory pool, serving paths that forbid device allocation once they are up, or plugins whose
host framework owns every allocation.  moe_route_noalloc keeps the router's scratch in an array
built into the library instead.  This test calls it through the C ABI, twice in a row, and checks
each result against moe_route with a caller workspace, within the tolerances of the other parity
tests; it also checks that a shape too large for the built-in array is refused before any launch.
This file is collected last so that a run stopping at the first failure has run everything else.
"""
import math

import numpy as np
import pytest

import synth
from moe_testlib import TOL_LOSS, TOL_W, shape_of, upload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "switch", "skew"])
def test_route_noalloc_matches_workspace_route(name):
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
    ref_idx = buf.topk_idx.cpu().numpy()
    ref_w = buf.topk_w.cpu().numpy().astype(np.float64)
    ref_l = buf.losses.cpu().numpy().astype(np.float64)

    T, k = cfg.T, cfg.k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    losses = torch.empty(2, dtype=torch.float32, device="cuda")
    io = moe.IO(dev["x"].data_ptr(), dev["Wg"].data_ptr(), dev["bg"].data_ptr(), None, None, None, None, None,
                idx.data_ptr(), w.data_ptr(), None, None, losses.data_ptr(), losses.data_ptr() + 4)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        idx.fill_(-1)
        w.fill_(float("nan"))
        losses.fill_(float("nan"))
        assert moe.moe_route_noalloc(shape, io, stream) == moe.MOE_OK
        torch.cuda.synchronize()
        got_idx, got_w, got_l = idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), losses.cpu().numpy()
        assert np.array_equal(got_idx, ref_idx)
        assert np.max(np.abs(got_w - ref_w) / np.abs(ref_w)) <= TOL_W
        assert np.all(np.abs(got_l - ref_l) <= TOL_LOSS * np.abs(ref_l))

    big = moe.make_shape(1 << 20, 64, 256, 8, 64, math.inf, "bf16")  # needs far more than 1 MiB
    assert moe.moe_route_noalloc(big, io, stream) == moe.MOE_ERR_WORKSPACE

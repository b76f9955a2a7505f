"""Expert parallelism on the GPU ("MoE Training: Mixture of Experts" page, Core Concepts 4, "Expert
Parallelism"), through the C ABI:

  moe_copy_row_segments  bit-exact copies of random segment tables; a misaligned segment is skipped and
                         reported, the others still copied
  moe_expert_ffn_rows    every row against the oracle's expert FFN (CTA-pair and single-CTA tiles, empty
                         experts, no biases / SiLU); offsets that break the contract are clamped and reported
  EmulatedExpertParallel R = 2 and 4 workers on one GPU, each with its own batch and workspace, exchanging
                         rows through moe_copy_row_segments: every worker's output against the oracle's
                         whole layer on its own batch (capacity per worker), and against the one-worker
                         moe_forward on the same batch
  ep_forward             the process-group path with the product's CudaExpertWorker on a one-rank NCCL group
"""
import math

import numpy as np
import pytest

import oracle
import synth
from moe_testlib import NEAR_TIE, out_error, rms_rel, shape_of, to_device, upload

pytestmark = pytest.mark.gpu


def _lib():
    import sparse_mixture_experts_23_b200 as moe
    from sparse_mixture_experts_23_b200 import build as moe_build

    moe_build.build()
    return moe


def test_copy_row_segments_bit_exact_and_misaligned_reported():
    import torch

    from sparse_mixture_experts_23_b200.expert_parallel import copy_segments

    moe = _lib()
    g = torch.Generator(device="cuda").manual_seed(5)
    src = torch.randint(-2 ** 31, 2 ** 31 - 1, (4000, 64), dtype=torch.int32, device="cuda", generator=g)
    dst = torch.zeros_like(src)
    rb = 64 * 4
    rng = np.random.default_rng(5)
    segs, expect = [], []
    d0 = 0
    for _ in range(40):
        n = int(rng.integers(0, 120))
        s0 = int(rng.integers(0, 4000 - n))
        segs.append((src.data_ptr() + s0 * rb, dst.data_ptr() + d0 * rb, n))
        expect.append((s0, d0, n))
        d0 += n
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    t = copy_segments(segs, rb, status.data_ptr())
    torch.cuda.synchronize()
    for s0, dd, n in expect:
        assert torch.equal(dst[dd:dd + n], src[s0:s0 + n])
    assert int(status.item()) == 0 and moe.moe_last_launch_count() == 1
    # a misaligned destination: that segment is skipped and reported, the next one is copied
    dst.zero_()
    bad = [(src.data_ptr(), dst.data_ptr() + 8, 3), (src.data_ptr() + 10 * rb, dst.data_ptr() + 100 * rb, 5)]
    t = copy_segments(bad, rb, status.data_ptr())
    torch.cuda.synchronize()
    assert int(status.item()) != 0
    assert torch.equal(dst[100:105], src[10:15]) and int(dst[:99].abs().sum().item()) == 0
    del t
    # host validation
    assert moe.moe_copy_row_segments(0, 1, 24, 10) == moe.MOE_ERR_INVALID_ARG  # row_bytes not a multiple of 16
    assert moe.moe_copy_row_segments(0, 3, 64, 10) == moe.MOE_ERR_INVALID_ARG  # NULL table
    assert moe.moe_copy_row_segments(0, 0, 64, 10) == moe.MOE_OK


def _rows_case(name, H, F, E, counts, dtype, act="gelu", bias=True, seed=0):
    cfg = synth.LayerConfig(name, T=int(sum(counts)), H=H, E=E, k=1, F=F, CF=math.inf, dtype=dtype, seed=seed,
                            act=act, bias=bias)
    return cfg, np.asarray(counts)


@pytest.mark.parametrize("case", [
    _rows_case("rows_pair", 256, 512, 4, [300, 0, 700, 77], "bf16", seed=61),          # CTA-pair tiles (269 rows per expert), empty expert
    _rows_case("rows_single", 128, 192, 5, [40, 3, 0, 90, 17], "bf16", seed=62),       # single-CTA, 64-wide N tiles
    _rows_case("rows_silu_nobias", 256, 256, 2, [200, 180], "bf16", "silu", False, 63),
    _rows_case("rows_f32", 20, 12, 3, [7, 0, 11], "f32", seed=64),
], ids=lambda c: c[0].name)
def test_expert_ffn_rows_vs_oracle(case):
    import torch

    moe = _lib()
    cfg, counts = case
    inp = synth.make_inputs(cfg)  # x has sum(counts) rows; rows are grouped by expert as they come
    n = cfg.T
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    experts = np.repeat(np.arange(cfg.E, dtype=np.int32), counts)
    dev = upload(inp)
    shape = shape_of(cfg)
    wsb = moe.moe_expert_ffn_rows_workspace_size(shape, n)
    ws = torch.zeros((wsb,), dtype=torch.uint8, device="cuda")
    y = torch.full((n + 5, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    offs = torch.from_numpy(offsets).cuda()
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    st = torch.cuda.current_stream().cuda_stream
    assert moe.moe_expert_ffn_rows(shape, n, offs.data_ptr(), dev["x"].data_ptr(), dev["W1"].data_ptr(),
                                   p(dev.get("b1")), dev["W2"].data_ptr(), p(dev.get("b2")), y.data_ptr(),
                                   ws.data_ptr(), wsb, st) == moe.MOE_OK
    assert moe.moe_last_launch_count() == 3
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws.data_ptr(), st) == moe.MOE_OK
    ref = oracle.expert_rows(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, np.arange(n, dtype=np.int32), experts, cfg.dtype,
                             act=cfg.act)
    got = y[:n].cpu().numpy().astype(np.float64)
    err, tol = out_error(got, ref, cfg.dtype)
    print(f"{cfg.name}: {err:.3e} (tol {tol:.0e})")
    assert err <= tol
    assert torch.isnan(y[n:]).all()  # rows past rows_cap untouched
    # offsets past rows_cap or decreasing: clamped on the device, nothing outside y written, error reported
    bad = offsets.copy()
    bad[-1] = n + 1000
    if cfg.E > 2:
        bad[2] = bad[1] - 1 if bad[1] > 0 else bad[2]
    offs.copy_(torch.from_numpy(bad))
    assert moe.moe_expert_ffn_rows(shape, n, offs.data_ptr(), dev["x"].data_ptr(), dev["W1"].data_ptr(),
                                   p(dev.get("b1")), dev["W2"].data_ptr(), p(dev.get("b2")), y.data_ptr(),
                                   ws.data_ptr(), wsb, st) == moe.MOE_OK
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws.data_ptr(), st) == moe.MOE_ERR_INVALID_ARG
    assert torch.isnan(y[n:]).all()


EP_CFG = synth.LayerConfig("ep_gpu", T=512, H=256, E=8, k=2, F=512, CF=1.25, dtype="bf16", seed=65)


@pytest.mark.parametrize("R", [2, 4])
def test_emulated_expert_parallel_matches_oracle_and_single_worker(R):
    import torch

    from sparse_mixture_experts_23_b200.expert_parallel import EmulatedExpertParallel

    moe = _lib()
    cfg = EP_CFG
    inp = synth.make_inputs(cfg)
    dev = upload(inp)
    batches = [synth.x_batch(cfg, r) if r > 0 else inp.x for r in range(R)]
    ep = EmulatedExpertParallel(shape_of(cfg), dev, [to_device(b, cfg.dtype) for b in batches])
    outs = ep.forward()
    torch.cuda.synchronize()
    assert int(ep.status.item()) == 0 and all(v == 0 for v in ep.ffn_status())
    crossed = sum(int(p.recv_rows[s]) for d, p in enumerate(ep.plans) for s in range(R) if s != d)
    assert crossed > 0
    for r in range(R):
        w = ep.workers[r]
        assert w.device_status() == moe.MOE_OK
        idx, drp = w.topk_idx.cpu().numpy(), w.dropped.cpu().numpy()
        ref_r = oracle.route(batches[r], inp.Wg, inp.bg, cfg.k, cfg.dtype)
        ok = ref_r.margin >= NEAR_TIE
        assert (idx[ok] == ref_r.topk_idx[ok]).all()
        d = oracle.dispatch(idx, cfg.E, cfg.CF)
        assert (drp == d.dropped).all()
        want = oracle.forward_tokens(batches[r], inp.W1, inp.b1, inp.W2, inp.b2, idx,
                                     w.topk_w.cpu().numpy().astype(np.float64), drp, np.arange(cfg.T, dtype=np.int32),
                                     cfg.dtype)
        got = outs[r].cpu().numpy().astype(np.float64)
        live = ~drp.astype(bool).all(axis=1)
        err, tol = out_error(got, want, cfg.dtype, rows=live)
        print(f"R={R} worker {r}: out error {err:.3e} (tol {tol:.0e}), drops {int(drp.sum())}")
        assert err <= tol
        # the same batch through one worker's moe_forward: the same rows, the same GEMMs per row
        one = moe.MoEBuffers(shape_of(cfg), dict(dev, x=to_device(batches[r], cfg.dtype)))
        one.forward()
        torch.cuda.synchronize()
        ref1 = one.out.cpu().numpy().astype(np.float64)
        assert rms_rel(got, ref1) <= 1e-5, rms_rel(got, ref1)


def test_ep_forward_one_rank_nccl_group_uses_the_cuda_worker():
    """ep_forward on a one-rank NCCL group: the process-group path end to end with the product worker
    (moe_route, moe_permute, moe_copy_row_segments regrouping, moe_expert_ffn_rows, moe_combine)."""
    import os
    import socket

    import torch
    import torch.distributed as dist

    from sparse_mixture_experts_23_b200.expert_parallel import CudaExpertWorker, ep_forward

    moe = _lib()
    cfg = EP_CFG
    inp = synth.make_inputs(cfg)
    dev = upload(inp)
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta

    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        buf = moe.MoEBuffers(shape_of(cfg), dev)
        worker = CudaExpertWorker(buf, dev["W1"], dev["b1"], dev["W2"], dev["b2"], cfg.E)
        out, plan = ep_forward(worker)
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        idx, drp = buf.topk_idx.cpu().numpy(), buf.dropped.cpu().numpy()
        want = oracle.forward_tokens(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, idx,
                                     buf.topk_w.cpu().numpy().astype(np.float64), drp, np.arange(cfg.T, dtype=np.int32),
                                     cfg.dtype)
        live = ~drp.astype(bool).all(axis=1)
        err, tol = out_error(got, want, cfg.dtype, rows=live)
        print(f"ep_forward (1 rank): {err:.3e}")
        assert err <= tol and plan.received == int(buf.expert_counts.sum().item())
    finally:
        dist.destroy_process_group()

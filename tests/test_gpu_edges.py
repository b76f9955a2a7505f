"""Edge cases of the CUDA path, each checked against the oracle: empty batch, ragged token counts,
odd expert counts, every N-tile width of the tensor-core kernel, empty experts, heavy capacity drops
(tokens with every slot dropped), maximum E and k, the unfused combine, the host-buffer entry point,
run-to-run determinism and the bounded device wait."""
import math

import numpy as np
import pytest

import oracle
import synth
from moe_testlib import NEAR_TIE, TOL_LOSS, out_error, shape_of, upload

pytestmark = pytest.mark.gpu


def _lib():
    import sparse_mixture_experts_23_b200 as moe
    from sparse_mixture_experts_23_b200 import build as moe_build

    moe_build.build()
    return moe


def _cfg(name, T, H, E, k, F, CF, dtype, seed, **kw):
    return synth.LayerConfig(name, T=T, H=H, E=E, k=k, F=F, CF=CF, dtype=dtype, seed=seed, **kw)


def _run_forward(cfg, inp=None, bg_override=None):
    import torch

    moe = _lib()
    inp = inp or synth.make_inputs(cfg)
    if bg_override is not None:
        inp.bg = synth.to_storage(bg_override, cfg.dtype)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp))
    buf.out.fill_(float("nan"))  # the forward must write (or clear) every element of out
    buf.forward()
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK
    r = dict(inp=inp, buf=buf, out=buf.out.cpu().numpy(), topk_idx=buf.topk_idx.cpu().numpy(),
             topk_w=buf.topk_w.cpu().numpy(), dropped=buf.dropped.cpu().numpy(),
             counts=buf.expert_counts.cpu().numpy(), losses=buf.losses.cpu().numpy())
    return r


def _check_against_oracle(cfg, r):
    inp = r["inp"]
    ref = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, cfg.dtype)
    ok = ref.margin >= NEAR_TIE
    assert (r["topk_idx"][ok] == ref.topk_idx[ok]).all()
    d = oracle.dispatch(r["topk_idx"], cfg.E, cfg.CF, cfg.min_capacity)
    assert (r["dropped"] == d.dropped).all()
    assert (r["counts"] == d.expert_counts).all()
    aux, z = oracle.losses(ref.p, ref.lse, r["topk_idx"])
    assert abs(r["losses"][0] - aux) <= TOL_LOSS * abs(aux)
    assert abs(r["losses"][1] - z) <= TOL_LOSS * abs(z)
    toks = np.arange(cfg.T, dtype=np.int32)
    want = oracle.forward_tokens(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, r["topk_idx"],
                                 r["topk_w"].astype(np.float64), r["dropped"], toks, cfg.dtype, act=cfg.act)
    live = ~r["dropped"].astype(bool).all(axis=1)
    err, tol = out_error(r["out"].astype(np.float64), want, cfg.dtype, rows=live)
    assert err <= tol, (err, tol)
    assert (r["out"][~live] == 0).all()
    return d


@pytest.mark.parametrize("cfg", [
    # ragged T (not a multiple of 32), odd E, k=3, F=192 -> 64-wide N tiles, H=128 -> 128-wide N tiles
    _cfg("ragged_bf16", 100, 128, 6, 3, 192, 1.0, "bf16", 21),
    # fp32 path with small odd sizes
    _cfg("ragged_f32", 77, 20, 5, 2, 12, math.inf, "f32", 22),
    # maximum E and k
    _cfg("maxE_bf16", 64, 64, 256, 8, 64, math.inf, "bf16", 23),
    # k = 1 Switch routing with drops, 256-wide N tiles
    _cfg("switch_small", 300, 256, 16, 1, 512, 1.25, "bf16", 24),
    # one token
    _cfg("one_token", 1, 64, 4, 2, 64, math.inf, "bf16", 25),
    # segments longer than one 128-row tile and a ragged tail in several experts
    _cfg("long_segments", 1000, 128, 3, 2, 256, math.inf, "bf16", 26),
    # CTA-pair tiles in both GEMMs (N divisible by 256, K by 128), ragged tails, capacity drops
    _cfg("pair_tiles", 1500, 256, 4, 2, 512, 1.1, "bf16", 27),
    # the Mixtral block's expert (SiLU, no bias anywhere) on the fp32 path, the single-CTA tiles
    # (N = 192 -> 64-wide, 128 -> 128-wide) and the CTA-pair tiles with half tiles and drops
    _cfg("silu_nobias_f32", 77, 20, 5, 2, 12, math.inf, "f32", 28, act="silu", bias=False),
    _cfg("silu_nobias_bf16", 100, 128, 6, 3, 192, 1.0, "bf16", 29, act="silu", bias=False),
    _cfg("silu_nobias_pair", 1500, 256, 4, 2, 512, 1.1, "bf16", 30, act="silu", bias=False),
    # SiLU with biases present, k = 1 with drops
    _cfg("silu_bias", 300, 256, 16, 1, 512, 1.25, "bf16", 33, act="silu"),
    # min_capacity binding: ceil(0.02 * 256 * 2 / 8) = 2 < 6
    _cfg("min_capacity", 256, 128, 8, 2, 128, 0.02, "bf16", 36, min_capacity=6),
], ids=lambda c: c.name)
def test_small_shapes_end_to_end(cfg):
    r = _run_forward(cfg)
    _check_against_oracle(cfg, r)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_some_biases_absent(dtype):
    """Each bias is optional on its own: no gate bias and no b2, but b1 present (GELU)."""
    cfg = _cfg("partial_bias", 260, 128, 4, 2, 256, math.inf, dtype, 34)
    inp = synth.make_inputs(cfg)
    inp.bg = None
    inp.b2 = None
    r = _run_forward(cfg, inp=inp)
    _check_against_oracle(cfg, r)


def test_empty_experts():
    cfg = _cfg("empty_experts", 200, 128, 8, 2, 128, math.inf, "bf16", 31)
    bg = np.zeros(8)
    bg[4:] = -30.0  # experts 4..7 are never chosen
    r = _run_forward(cfg, bg_override=bg)
    d = _check_against_oracle(cfg, r)
    assert (d.expert_counts[4:] == 0).all()


@pytest.mark.parametrize("T,H,F,CF,seed,cap", [
    (256, 64, 128, 0.125, 32, 16),    # cap = ceil(0.125*256*2/4); single-CTA GEMMs, the scatter clears out
    (1024, 128, 256, 0.15, 35, 77),   # T*k/E = 512 rows per expert on average: GEMM1 on CTA pairs zeroes out
], ids=["single_cta", "cta_pair"])
def test_heavy_drops_and_all_dropped_tokens(T, H, F, CF, seed, cap):
    cfg = _cfg("drops", T, H, 4, 2, F, CF, "bf16", seed)
    bg = np.array([3.0, 2.5, -5.0, -5.0])  # everyone wants experts 0 and 1
    r = _run_forward(cfg, bg_override=bg)  # out starts as NaN
    d = _check_against_oracle(cfg, r)
    assert d.cap == cap
    all_dropped = r["dropped"].all(axis=1)
    assert all_dropped.sum() > 100
    assert (r["out"][all_dropped] == 0).all()


def test_empty_batch():
    import torch

    moe = _lib()
    cfg = _cfg("empty", 0, 64, 4, 2, 64, math.inf, "bf16", 33)
    dev = {n: torch.zeros(1, dtype=torch.bfloat16, device="cuda") for n in ("x", "Wg", "bg", "W1", "b1", "W2", "b2")}
    buf = moe.MoEBuffers(shape_of(cfg), dev)
    buf.expert_counts.fill_(7)
    buf.losses.fill_(5.0)
    buf.forward()
    torch.cuda.synchronize()
    assert (buf.expert_counts.cpu().numpy() == 0).all()
    assert (buf.losses.cpu().numpy() == 0).all()
    for fn in (buf.route, buf.permute, buf.combine):
        fn()
    buf.expert_ffn(True)
    torch.cuda.synchronize()


@pytest.mark.parametrize("E", [8, 2])  # 83 rows per expert (single-CTA tiles) / 333 (CTA-pair tiles)
def test_unfused_combine_matches_fused(E):
    import torch

    moe = _lib()
    cfg = _cfg("unfused", 333, 256, E, 2, 512, 1.25, "bf16", 34)
    inp = synth.make_inputs(cfg)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp))
    buf.forward()
    torch.cuda.synchronize()
    fused = buf.out.cpu().numpy().copy()
    buf.out.fill_(float("nan"))
    buf.route()
    buf.permute()
    buf.expert_ffn(fuse_combine=False)
    buf.out.fill_(float("nan"))  # combine must overwrite every element
    buf.combine()
    torch.cuda.synchronize()
    unfused = buf.out.cpu().numpy()
    assert np.isfinite(unfused).all()
    np.testing.assert_allclose(unfused, fused, rtol=1e-5, atol=1e-6)
    toks = np.arange(cfg.T, dtype=np.int32)
    want = oracle.forward_tokens(inp.x, inp.W1, inp.b1, inp.W2, inp.b2, buf.topk_idx.cpu().numpy(),
                                 buf.topk_w.cpu().numpy().astype(np.float64), buf.dropped.cpu().numpy(), toks,
                                 cfg.dtype)
    err, tol = out_error(unfused.astype(np.float64), want, cfg.dtype)
    assert err <= tol


@pytest.mark.parametrize("dtype,E", [("f32", 8), ("bf16", 8), ("bf16", 2)])
def test_deterministic_bitwise(dtype, E):
    import torch

    moe = _lib()
    cfg = _cfg("det", 512, 128, E, 2, 256, math.inf, dtype, 35)
    buf = moe.MoEBuffers(shape_of(cfg), upload(synth.make_inputs(cfg)))
    outs = []
    for _ in range(3):
        buf.forward()
        torch.cuda.synchronize()
        outs.append((buf.out.cpu().numpy().copy(), buf.losses.cpu().numpy().copy()))
    for o, l in outs[1:]:
        assert np.array_equal(o, outs[0][0]) and np.array_equal(l, outs[0][1])


def test_k3_repeat_runs_agree_within_rounding():
    """k = 3: three fp32 atomic adds can reach one element of out, and fp32 addition is not associative,
    so repeat runs may differ in the last bits.  Routing, dispatch and the losses still repeat exactly;
    out agrees within a few ulps of its magnitude (and each run meets the oracle rule)."""
    import torch

    moe = _lib()
    cfg = _cfg("det_k3", 600, 128, 6, 3, 192, math.inf, "bf16", 39)
    buf = moe.MoEBuffers(shape_of(cfg), upload(synth.make_inputs(cfg)))
    outs = []
    for _ in range(3):
        buf.forward()
        torch.cuda.synchronize()
        outs.append((buf.out.cpu().numpy().copy(), buf.topk_idx.cpu().numpy().copy(), buf.losses.cpu().numpy().copy()))
    scale = float(np.abs(outs[0][0]).max())
    for o, i, l in outs[1:]:
        assert np.array_equal(i, outs[0][1]) and np.array_equal(l, outs[0][2])
        assert float(np.abs(o - outs[0][0]).max()) <= 1e-6 * scale


def test_forward_host_buffers():
    import torch

    moe = _lib()
    cfg = _cfg("host", 128, 128, 4, 2, 256, math.inf, "bf16", 36)
    inp = synth.make_inputs(cfg)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp))
    buf.forward()
    torch.cuda.synchronize()
    ref = buf.out.cpu().numpy().copy()
    x2 = synth.x_batch(cfg, 1)
    x_host = torch.from_numpy(x2.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_host = torch.empty((cfg.T, cfg.H), dtype=torch.float32).pin_memory()
    buf.inputs["x"].zero_()
    buf.forward_host(x_host, out_host)
    torch.cuda.synchronize()
    inp2 = synth.make_inputs(cfg)
    inp2.x = x2
    r = oracle.forward(inp2.x, inp2.Wg, inp2.bg, inp2.W1, inp2.b1, inp2.W2, inp2.b2, cfg.k, cfg.CF, cfg.dtype)
    err, tol = out_error(out_host.numpy().astype(np.float64), r.out, cfg.dtype)
    assert err <= tol
    assert not np.array_equal(out_host.numpy(), ref)


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch

    moe = _lib()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    moe.moe_set_wait_limit(2_000_000)  # ~1 ms
    try:
        assert moe.moe_debug_timeout_probe(ws.data_ptr(), 256, stream) == moe.MOE_OK
        assert moe.moe_get_device_status(ws.data_ptr(), stream) == moe.MOE_ERR_TIMEOUT
        assert moe.moe_get_device_status(ws.data_ptr(), stream) == moe.MOE_OK  # cleared
    finally:
        moe.moe_set_wait_limit(0)
    # the context is still usable
    cfg = _cfg("after_timeout", 64, 64, 4, 2, 64, math.inf, "bf16", 37)
    r = _run_forward(cfg)
    _check_against_oracle(cfg, r)


def test_stream_ordering_on_side_stream():
    import torch

    moe = _lib()
    cfg = _cfg("side", 256, 128, 8, 2, 256, math.inf, "bf16", 38)
    inp = synth.make_inputs(cfg)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        buf.forward()
    s.synchronize()
    r = dict(inp=inp, out=buf.out.cpu().numpy(), topk_idx=buf.topk_idx.cpu().numpy(),
             topk_w=buf.topk_w.cpu().numpy(), dropped=buf.dropped.cpu().numpy(),
             counts=buf.expert_counts.cpu().numpy(), losses=buf.losses.cpu().numpy())
    _check_against_oracle(cfg, r)


@pytest.mark.parametrize("T,H,E,k,F", [(640, 256, 8, 2, 256), (8192, 128, 128, 1, 128), (32, 512, 8, 2, 256)],
                         ids=["fused_gate_reduce", "multi_block_reduce", "decode_scatter_slices"])
def test_concurrent_calls_on_distinct_workspaces(T, H, E, k, F):
    """Calls on distinct workspaces may run concurrently on different streams: three layers (each with
    its own batch and workspace, so its own finished-block counters) are enqueued on three streams
    without waits between them, twice over, and every result must equal the same call run alone."""
    import torch

    moe = _lib()
    bufs, serial = [], []
    for i in range(3):
        cfg = _cfg(f"concurrent_{E}_{i}", T, H, E, k, F, 1.25, "bf16", 81 + i)
        buf = moe.MoEBuffers(shape_of(cfg), upload(synth.make_inputs(cfg)))
        buf.forward()
        torch.cuda.synchronize()
        serial.append((buf.out.clone(), buf.topk_idx.clone(), buf.losses.clone(), buf.expert_counts.clone()))
        bufs.append(buf)
    streams = [torch.cuda.Stream() for _ in bufs]
    for s_ in streams:
        s_.wait_stream(torch.cuda.current_stream())
    for _ in range(2):
        for buf, s_ in zip(bufs, streams):
            with torch.cuda.stream(s_):
                buf.forward()
    torch.cuda.synchronize()
    for buf, (out, idx, losses, counts) in zip(bufs, serial):
        assert buf.device_status() == moe.MOE_OK
        assert torch.equal(buf.topk_idx, idx) and torch.equal(buf.expert_counts, counts)
        assert torch.equal(buf.losses, losses)
        assert torch.equal(buf.out, out)  # k <= 2: the fp32 adds into out do not depend on their order


def test_out_of_range_indices_are_reported_not_followed():
    """A caller-supplied topk_idx with an expert outside [0, E) (token choice), or a chosen token outside
    [0, T) (expert choice): the kernels skip the entry, touch nothing outside the buffers, and the device
    status reports MOE_ERR_INVALID_ARG once; the next call on the same workspace is clean."""
    import torch

    moe = _lib()
    cfg = _cfg("bad_index", 96, 128, 4, 2, 128, math.inf, "bf16", 37)
    inp = synth.make_inputs(cfg)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp))
    buf.route()
    bad = buf.topk_idx.clone()
    buf.topk_idx[5, 1] = 1000
    buf.topk_idx[9, 0] = -3
    buf.permute()
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_ERR_INVALID_ARG
    dropped = buf.dropped.cpu().numpy()
    assert dropped[5, 1] == 1 and dropped[9, 0] == 1
    assert int(buf.expert_counts.sum().item()) == cfg.T * cfg.k - 2
    buf.topk_idx.copy_(bad)
    buf.forward()
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK

    ec = _cfg("bad_token_ec", 96, 128, 4, 2, 128, 1.0, "bf16", 38, routing="expert_choice")
    inp = synth.make_inputs(ec)
    buf = moe.MoEBuffers(shape_of(ec), upload(inp))
    buf.route()
    buf.topk_idx[2, 3] = ec.T + 7
    buf.permute()
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_ERR_INVALID_ARG
    buf.forward()
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK


@pytest.mark.parametrize("T,H,E,k,F,CF,extra", [
    (1000, 256, 16, 2, 512, math.inf, {}),
    (640, 128, 16, 1, 256, 1.25, {}),
    (777, 192, 8, 1, 384, 1.1, {"act": "silu", "bias": False}),
], ids=["avg125_dropless", "avg40_drops", "avg97_silu_nobias"])
def test_spread_rows_every_row_against_oracle(T, H, E, k, F, CF, extra):
    """32 to 127 rows per expert on average: the single-CTA GEMM tiles place each 8-row group of a
    segment in a different TMEM lane quarter.  Routing, dispatch and every output row against the
    oracle; then a training forward (u and h written through the same placement) and the backward."""
    import torch

    moe = _lib()
    cfg = _cfg(f"spread_{T}_{E}", T, H, E, k, F, CF, "bf16", 61 + E, **extra)
    inp = synth.make_inputs(cfg)
    r = _run_forward(cfg, inp)
    _check_against_oracle(cfg, r)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp), train=True)
    buf.forward_train()
    grads = buf.make_grads()
    dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
    buf.backward(torch.from_numpy(dout.astype(np.float32)).cuda(), grads, 0.01, 0.001)
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK
    assert np.array_equal(buf.out.cpu().numpy(), r["out"])  # the training forward gives the same out
    ref = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, dout,
                          0.01, 0.001, act=cfg.act, topk_idx=buf.topk_idx.cpu().numpy(),
                          dropped=buf.dropped.cpu().numpy())
    from moe_testlib import TOL_BWD_FRO, TOL_BWD_MAX, fro_rel, rms_rel
    for n in ("dx", "dWg", "dW1", "dW2"):
        got = grads[n].cpu().numpy().astype(np.float64)
        want = getattr(ref, n)
        per = [rms_rel(got[e], want[e]) for e in range(cfg.E) if np.any(want[e])] if n in ("dW1", "dW2") \
            else [rms_rel(got, want)]
        assert max(per) <= TOL_BWD_MAX and fro_rel(got, want) <= TOL_BWD_FRO, (n, max(per))


@pytest.mark.parametrize("T,H,E,k,CF", [(1536, 64, 256, 2, math.inf), (4096, 128, 200, 1, 1.25), (4096, 64, 96, 3, 1.1)],
                         ids=["E256", "E200_partial_block_drops", "E96_k3"])
def test_multi_block_reduction_against_oracle(T, H, E, k, CF):
    """k * ceil(T/32) * E past one 1024-thread batch: the loss / dispatch reduction runs over blocks of
    experts (up to 16 per block; 256 experts exercise the last offset, 200 a partial last block).  Forward
    and the standalone route + permute: routing, drops, counts, losses and every output row against the
    oracle."""
    import torch

    moe = _lib()
    cfg = _cfg(f"multi_reduce_{E}", T, H, E, k, 64, CF, "bf16", 71 + E)
    inp = synth.make_inputs(cfg)
    r = _run_forward(cfg, inp)
    _check_against_oracle(cfg, r)
    buf = moe.MoEBuffers(shape_of(cfg), upload(inp))
    buf.route()
    buf.permute()
    torch.cuda.synchronize()
    assert buf.device_status() == moe.MOE_OK
    idx = buf.topk_idx.cpu().numpy()
    d = oracle.dispatch(idx, cfg.E, cfg.CF, cfg.min_capacity)
    assert (buf.expert_counts.cpu().numpy() == d.expert_counts).all()
    assert (buf.dropped.cpu().numpy() == d.dropped).all()
    np.testing.assert_array_equal(buf.losses.cpu().numpy(), r["losses"])  # the same reduction, the same bits


@pytest.mark.parametrize("T,H,E,F,CF", [(4096, 256, 64, 2048, 1.25), (3000, 128, 16, 4096, math.inf)],
                         ids=["spread_drops", "ragged_dropless"])
def test_top1_split_k_every_row_and_bitwise_repeatable(T, H, E, F, CF):
    """Top-1 layers on single-CTA tiles with a long GEMM2 K split each GEMM2 tile into two K halves,
    each adding its partial product into out (the bias with the first).  Every output row against the
    oracle, and three runs give the same bits: with k = 1 each element receives exactly two adds."""
    import torch

    moe = _lib()
    cfg = _cfg(f"split_k_{E}_{F}", T, H, E, 1, F, CF, "bf16", 91 + E)
    inp = synth.make_inputs(cfg)
    r = _run_forward(cfg, inp)
    _check_against_oracle(cfg, r)
    buf = r["buf"]
    outs = []
    for _ in range(3):
        buf.forward()
        torch.cuda.synchronize()
        outs.append(buf.out.clone())
    assert buf.device_status() == moe.MOE_OK
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    assert np.array_equal(outs[0].cpu().numpy(), r["out"])


def test_epilogue_activations_match_their_definitions():
    """The bf16 epilogues' GELU and SiLU (and their derivatives), run on the device through
    moe_debug_activation, against the fp64 definitions on a dense grid of [-12, 12] and special values.
    GELU(u) = u Phi(u) with Phi from Abramowitz & Stegun 7.1.26, whose error in erfc is at most 1.5e-7,
    so |Phi error| <= 0.75e-7 plus fp32 evaluation (a few ulp of quantities <= 1): the bound used is
    |dGELU| <= 4e-7 |u| + 2^-22 |GELU| and |dGELU'| <= 6e-7 + 2^-20 |GELU'|.  SiLU uses the fast
    exponential and division: relative error <= 2^-20 + |u| 2^-22."""
    import torch
    from scipy.special import erf

    moe = _lib()
    grid = np.linspace(-12.0, 12.0, 1 << 20)
    special = np.array([0.0, -0.0, 1e-30, -1e-30, 1e-8, -1e-8, 0.5, -0.5, 1.0, -1.0, 3.0, -3.0, 6.0, -6.0])
    u = np.concatenate([grid, special]).astype(np.float32)
    n = u.size
    ud = torch.from_numpy(u).cuda()
    out = torch.empty(2 * n, dtype=torch.float32, device="cuda")
    u64 = u.astype(np.float64)
    phi = 0.5 * (1.0 + erf(u64 / np.sqrt(2.0)))
    dens = np.exp(-0.5 * u64 * u64) / np.sqrt(2.0 * np.pi)
    sig = 1.0 / (1.0 + np.exp(-u64))
    refs = {moe.MOE_ACT_GELU: (u64 * phi, phi + u64 * dens), moe.MOE_ACT_SILU: (u64 * sig, sig * (1.0 + u64 * (1.0 - sig)))}
    stream = torch.cuda.current_stream().cuda_stream
    for act, (f, df) in refs.items():
        assert moe.moe_debug_activation(act, ud.data_ptr(), out.data_ptr(), n, stream) == moe.MOE_OK
        assert moe.moe_last_launch_count() == 1
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        g, dg = got[:n], got[n:]
        if act == moe.MOE_ACT_GELU:
            tol_f = 4e-7 * np.abs(u64) + 2.0 ** -22 * np.abs(f) + 1e-37
            tol_d = 6e-7 + 2.0 ** -20 * np.abs(df)
        else:
            # the fast exponential's relative error grows with its argument (|u| log2 e rounded to
            # fp32 before the base-2 power); SiLU' crosses zero near u = -1.28, where its two terms of
            # size ~0.2 cancel, hence the error is bounded against |ref| + 1 there
            rel = 2.0 ** -20 + np.abs(u64) * 2.0 ** -22
            tol_f = rel * np.abs(f) + 1e-37
            tol_d = rel * (np.abs(df) + 1.0)
        ef, ed = np.abs(g - f), np.abs(dg - df)
        print(f"act {act}: max |d act| {ef.max():.3e} (worst ratio to bound {np.max(ef / tol_f):.3f}), "
              f"max |d act'| {ed.max():.3e} (ratio {np.max(ed / tol_d):.3f})")
        assert np.all(ef <= tol_f), (act, u[np.argmax(ef / tol_f)])
        assert np.all(ed <= tol_d), (act, u[np.argmax(ed / tol_d)])


@pytest.mark.parametrize("T,H,E,k", [(1000, 256, 8, 2), (77, 2304, 8, 2), (333, 1152, 16, 2), (4100, 4096, 8, 1),
                                     (32, 4096, 16, 2)],
                         ids=["one_stage_ragged", "nine_stages", "e16_nine_stages", "two_rounds_ragged", "decode_e16"])
def test_streamed_gate_stage_counts_and_ragged_chunks(T, H, E, k):
    """The bulk-copy gate (bf16, 8 or 16 experts) with stage counts below, at and past one per warp,
    a last chunk of fewer than 32 tokens, a single chunk, and its last block's fused loss / dispatch
    reduction: routing, dispatch and losses against the oracle, and the same results as the register-
    direct gate."""
    import torch

    moe = _lib()
    cfg = _cfg(f"stream_gate_{T}_{H}_{E}", T, H, E, k, 128, 1.25, "bf16", 51 + E)
    inp = synth.make_inputs(cfg)
    r = _run_forward(cfg, inp)
    _check_against_oracle(cfg, r)
    try:
        moe.moe_set_kernel_options(moe.MOE_KERNEL_NO_TMA_ROUTER)
        r2 = _run_forward(cfg, inp)
    finally:
        moe.moe_set_kernel_options(0)
    ref = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, cfg.dtype)
    ok = ref.margin >= NEAR_TIE
    assert (r["topk_idx"][ok] == r2["topk_idx"][ok]).all()
    np.testing.assert_allclose(r["topk_w"][ok], r2["topk_w"][ok], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(r["losses"], r2["losses"], rtol=1e-5)
    torch.cuda.synchronize()


@pytest.mark.parametrize("flags", [1, 2, 3, 4], ids=["no_cta_pair", "no_tc_gate", "both", "no_tma_router"])
def test_kernel_options_select_other_kernels_same_results(flags):
    """moe_set_kernel_options: the single-CTA GEMM tiles in place of CTA pairs, the CUDA-core gate in
    place of the tensor-core ones, and the register-direct gate in place of the bulk-copy stream give
    results that meet the same oracle rules (forward and backward)."""
    import torch

    moe = _lib()
    cfg = _cfg("options", 1500, 256, 8, 2, 512, 1.1, "bf16", 37)       # pair tiles and the E = 8 mma gate
    wide = _cfg("options_gemm_gate", 600, 128, 64, 2, 128, 1.0, "bf16", 38)  # the tcgen05 gate (E = 64)
    try:
        moe.moe_set_kernel_options(flags)
        for c in (cfg, wide):
            r = _run_forward(c)
            _check_against_oracle(c, r)
        # backward through the single-CTA dgrad / wgrad kernels as well
        inp = synth.make_inputs(cfg)
        buf = moe.MoEBuffers(shape_of(cfg), upload(inp), train=True)
        buf.forward_train()
        grads = buf.make_grads()
        dout = synth.normal(cfg.seed, 96, (cfg.T, cfg.H)).astype(np.float64)
        buf.backward(torch.from_numpy(dout.astype(np.float32)).cuda(), grads, 0.01, 0.001)
        torch.cuda.synchronize()
        assert buf.device_status() == moe.MOE_OK
        ref = oracle.backward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, dout,
                              0.01, 0.001, topk_idx=buf.topk_idx.cpu().numpy(), dropped=buf.dropped.cpu().numpy())
        from moe_testlib import TOL_BWD_FRO, TOL_BWD_MAX, fro_rel, rms_rel
        for n in ("dx", "dWg", "dW1", "dW2"):
            got = grads[n].cpu().numpy().astype(np.float64)
            want = getattr(ref, n)
            per = [rms_rel(got[e], want[e]) for e in range(cfg.E)] if n in ("dW1", "dW2") else [rms_rel(got, want)]
            assert max(per) <= TOL_BWD_MAX and fro_rel(got, want) <= TOL_BWD_FRO, (n, max(per))
    finally:
        moe.moe_set_kernel_options(0)

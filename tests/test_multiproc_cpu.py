"""The N>1 (replicas) host logic on CPU: two gloo ranks each route their own batch through the same
weights with the oracle, the timing is reduced as the max over ranks, and the whole-job rate counts
every rank's tokens.  No GPU is involved.  The one exchange replicas may want -- the losses of the
whole batch -- goes through the binding's all-reduce of the additive loss sums."""
import math
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth

CFG = synth.LayerConfig("mp", T=64, H=32, E=4, k=2, F=48, CF=math.inf, dtype="f32", seed=77)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import oracle

        inp = bench.replica_inputs(CFG, rank)
        f = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, CFG.k, CFG.CF, CFG.dtype)
        fake_ms = 10.0 * (rank + 1)  # rank 1 is the slow one
        slowest = bench.max_over_ranks(fake_ms, world, "cpu")
        rate = bench.aggregate_rate(world, CFG.T, 5, slowest)
        dist.barrier()
        q.put((rank, float(inp.x.sum()), float(f.out.sum()), slowest, rate, int(f.disp.kept)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, xs0, os0, slow0, rate0, kept0), (r1, xs1, os1, slow1, rate1, kept1) = res
    assert xs0 != xs1 and os0 != os1          # each replica routes its own batch
    assert slow0 == slow1 == 20.0              # max over ranks
    assert rate0 == rate1 == pytest.approx(2 * CFG.T * 5 / 0.020)
    assert kept0 == kept1 == CFG.T * CFG.k     # dropless, per-replica dispatch


def test_rank0_batch_is_the_single_gpu_batch():
    import bench

    a = bench.replica_inputs(CFG, 0)
    b = synth.make_inputs(CFG)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.W1, b.W1)
    c = bench.replica_inputs(CFG, 3)
    assert not np.array_equal(a.x, c.x) and np.array_equal(a.W2, c.W2)


def _sums_of(inp, k):
    """The 2E+2 loss sums of one batch, from the oracle's routing: [cnt_e][Psum_e][Zsum][T]."""
    import oracle

    r = oracle.route(inp.x, inp.Wg, inp.bg, k, CFG.dtype)
    E = inp.Wg.shape[1]
    cnt = np.bincount(r.topk_idx.reshape(-1), minlength=E).astype(np.float64)
    return np.concatenate([cnt, r.p.sum(axis=0), [float((r.lse ** 2).sum())], [float(inp.x.shape[0])]])


def _losses_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import sparse_mixture_experts_23_b200 as moe

        inp = bench.replica_inputs(CFG, rank)
        sums = torch.from_numpy(_sums_of(inp, CFG.k))
        moe.allreduce_sums(sums)
        q.put((rank, sums.numpy().tolist()))
    finally:
        dist.destroy_process_group()


def test_global_losses_from_allreduced_sums():
    """Summing the replicas' loss sums and applying the loss formulas gives the oracle's losses of
    the concatenated batch; the mean of the replicas' own aux values does not."""
    import bench
    import oracle

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_losses_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    tot0, tot1 = np.array(res[0][1]), np.array(res[1][1])
    assert np.array_equal(tot0, tot1)  # every rank holds the same totals
    E = CFG.E
    cnt, psum, zsum, T = tot0[:E], tot0[E:2 * E], tot0[2 * E], tot0[2 * E + 1]
    aux = E * float(np.sum((cnt / cnt.sum()) * (psum / T)))
    z = zsum / T
    a, b = bench.replica_inputs(CFG, 0), bench.replica_inputs(CFG, 1)
    x = np.concatenate([a.x, b.x])
    r = oracle.route(x, a.Wg, a.bg, CFG.k, CFG.dtype)
    aux_ref, z_ref = oracle.losses(r.p, r.lse, r.topk_idx)
    assert T == 2 * CFG.T and cnt.sum() == 2 * CFG.T * CFG.k
    assert aux == pytest.approx(aux_ref, rel=1e-12) and z == pytest.approx(z_ref, rel=1e-12)
    own = []
    for inp in (a, b):
        rr = oracle.route(inp.x, inp.Wg, inp.bg, CFG.k, CFG.dtype)
        own.append(oracle.losses(rr.p, rr.lse, rr.topk_idx)[0])
    assert abs(0.5 * (own[0] + own[1]) - aux_ref) > 1e-9  # a product of means is not a mean of products

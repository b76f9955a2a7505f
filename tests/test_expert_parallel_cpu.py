"""Expert parallelism ("MoE Training: Mixture of Experts" page, Core Concepts 4, "Expert Parallelism") on
CPU: the exchange bookkeeping on its own, then whole layer calls over gloo process groups of 2 and 4
ranks.  In the gloo runs each rank's arithmetic (routing, permutation, expert FFN rows, combine) comes
from the fp64 oracle through a test-side worker, so what is under test is the product's orchestration:
the counts all-gather, the plan, both all-to-alls and the regrouping between the source-major and the
expert-major layouts.  Every rank's output must equal the oracle's whole layer on that rank's own batch
(capacity per rank) -- the statement that expert placement changes where the arithmetic runs, not what
it computes."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth
from sparse_mixture_experts_23_b200.expert_parallel import ExpertPlacement, exchange_plan


def _random_counts(R, E, seed):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 9, size=(R, E))
    c[rng.random((R, E)) < 0.2] = 0  # some experts empty on some workers
    return c


@pytest.mark.parametrize("R,E", [(1, 4), (2, 8), (4, 8), (4, 16), (8, 8)])
def test_exchange_plan_is_consistent(R, E):
    counts = _random_counts(R, E, seed=R * 100 + E)
    pl = ExpertPlacement(E, R)
    plans = [exchange_plan(counts, r, pl) for r in range(R)]
    for r, p in enumerate(plans):
        # what r sends to d is what d receives from r
        for d in range(R):
            assert p.send_rows[d] == plans[d].recv_rows[r]
        # send ranges tile the rank's kept rows in worker order (its x_perm is expert-major)
        assert p.send_rows.sum() == counts[r].sum()
        assert p.send_start[0] == 0 and (np.diff(p.send_start) == p.send_rows[:-1]).all()
        # both layouts are tilings of [0, received), and the moves form a bijection between them
        moves = p.to_grouped()
        n = p.received
        src = np.zeros(n, int)
        dst = np.zeros(n, int)
        for s_, d_, m in moves:
            src[s_:s_ + m] += 1
            dst[d_:d_ + m] += 1
        assert (src == 1).all() and (dst == 1).all()
        # grouped segments: local expert j holds every worker's rows of expert r*L + j, in worker order
        L = pl.local
        assert p.grouped_offsets[-1] == n
        for j in range(L):
            e = r * L + j
            assert p.grouped_offsets[j + 1] - p.grouped_offsets[j] == counts[:, e].sum()
            starts = p.grouped_start[j]
            assert starts[0] == p.grouped_offsets[j]
            assert (np.diff(starts) == counts[:-1, e]).all()
        # the reverse moves undo the forward ones
        assert sorted((d_, s_, m) for s_, d_, m in moves) == sorted(p.to_source_major())


def test_placement_rejects_uneven_split():
    with pytest.raises(ValueError):
        ExpertPlacement(6, 4)
    pl = ExpertPlacement(8, 4)
    assert list(pl.experts_of(2)) == [4, 5] and pl.owner(5) == 2


# ---------------------------------------------------------------------------------------------------
CFG = synth.LayerConfig("ep", T=96, H=16, E=8, k=2, F=24, CF=1.25, dtype="f32", seed=83)


class OracleWorker:
    """A rank's arithmetic from the oracle (test infrastructure): the same interface as the product's
    CudaExpertWorker."""

    def __init__(self, inp, rank, R):
        self.inp, self.rank, self.R = inp, rank, R

    def route_permute(self):
        import torch

        import oracle

        cfg, inp = CFG, self.inp
        self.r = oracle.route(inp.x, inp.Wg, inp.bg, cfg.k, cfg.dtype)
        self.d = oracle.dispatch(self.r.topk_idx, cfg.E, cfg.CF)
        x = np.asarray(inp.x, np.float64)
        return self.d.expert_counts.copy(), torch.from_numpy(x[self.d.row_token].copy())

    def regroup(self, rows, moves, n_out):
        out = rows.new_zeros((n_out,) + tuple(rows.shape[1:]))
        for s_, d_, m in moves:
            out[d_:d_ + m] = rows[s_:s_ + m]
        return out

    def ffn_rows(self, rows, grouped_offsets):
        """This rank's experts on its grouped rows: the oracle's expert FFN of each row, with only this
        rank's block of the expert weights."""
        import torch

        import oracle

        inp = self.inp
        L = CFG.E // self.R
        e0 = self.rank * L
        sl = slice(e0, e0 + L)
        n = rows.shape[0]
        experts = np.zeros(n, np.int32)
        for j in range(L):
            experts[grouped_offsets[j]:grouped_offsets[j + 1]] = j
        x_rows = rows.numpy().astype(np.float32)  # the fp32 inputs, exact
        y = oracle.expert_rows(x_rows, inp.W1[sl], inp.b1[sl], inp.W2[sl], inp.b2[sl], np.arange(n, dtype=np.int32),
                               experts, CFG.dtype)
        return torch.from_numpy(y)

    def combine(self, y_perm):
        y = y_perm.numpy()
        T, k = CFG.T, CFG.k
        out = np.zeros((T, CFG.H))
        for t in range(T):
            for s in range(k):
                row = self.d.row_of[t, s]
                if row >= 0:
                    out[t] += self.r.topk_w[t, s] * y[row]
        return out


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _ep_rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import oracle
        from sparse_mixture_experts_23_b200.expert_parallel import ep_forward

        inp = bench.replica_inputs(CFG, rank)
        out, plan = ep_forward(OracleWorker(inp, rank, world))
        ref = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, CFG.k, CFG.CF, CFG.dtype)
        err = float(np.max(np.abs(out - ref.out)) / np.max(np.abs(ref.out)))
        drops = int(ref.disp.dropped.sum())
        dist.barrier()
        q.put((rank, err, int(plan.received), [int(v) for v in plan.recv_rows], drops))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_gloo_matches_oracle_per_rank(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, received, recv_rows, drops in res:
        assert err <= 1e-12, (rank, err)
        assert sum(recv_rows) == received
    # rows did cross ranks, and capacity dropped some assignments on some rank
    assert any(r[3][i] > 0 for r in res for i in range(world) if i != r[0])
    assert sum(r[4] for r in res) > 0

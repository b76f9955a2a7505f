"""Expert parallelism of the MoE layer ("MoE Training: Mixture of Experts" page, Core Concepts 4, "Expert
Parallelism"; the CSDN MoE explainer's section on expert parallelism): the E experts are spread over R
workers, every kept assignment's row travels to the worker that holds its expert, that worker runs its
experts on everything it received, and the outputs travel back to be combined where the token lives.

Each worker routes and permutes its own tokens over all E experts (moe_route, moe_permute; capacity is
per worker, from its own T).  The permuted rows of expert e are the segment [offsets[e], offsets[e+1])
of its x_perm, and worker d holds the contiguous block of experts [d*E/R, (d+1)*E/R), so the rows bound
for worker d are one contiguous range of x_perm, and the rows coming back land in the same range of y.

  ExpertPlacement  which experts each worker holds
  exchange_plan    from every worker's per-expert kept counts: the rows each worker sends to and
                   receives from each other worker, and the segment moves between the received layout
                   (source-major: all rows from worker 0, then worker 1, ...) and the grouped layout the
                   expert GEMMs take (expert-major: expert 0's rows from every worker, then expert 1's)
  ep_forward       one layer call on a process group (NCCL between GPUs, or gloo): counts all-gather,
                   dispatch all-to-all, grouped expert FFN, return all-to-all, combine; the arithmetic
                   runs in a backend (CudaExpertWorker: the CUDA library on this rank's GPU)
  EmulatedExpertParallel  R workers on one GPU, each with its own workspace; the dispatch and the
                   return are one moe_copy_row_segments launch each, reading the source workers'
                   buffers directly (with peer-mapped buffers the same launch would pull over NVLink)

Every number is computed by the CUDA library; this module holds integer bookkeeping and collectives.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


class ExpertPlacement:
    """Worker r holds experts [r*E/R, (r+1)*E/R) (E divisible by R)."""

    def __init__(self, E: int, R: int):
        if R < 1 or E % R != 0:
            raise ValueError(f"{E} experts cannot be split evenly over {R} workers")
        self.E, self.R, self.local = E, R, E // R

    def experts_of(self, r: int) -> range:
        return range(r * self.local, (r + 1) * self.local)

    def owner(self, e: int) -> int:
        return e // self.local


@dataclass
class ExchangePlan:
    rank: int
    R: int
    local: int                 # experts per worker
    counts: np.ndarray         # [R, E] kept rows of every expert on every worker
    send_rows: np.ndarray      # [R] rows this worker sends to each worker (x_perm ranges, in worker order)
    send_start: np.ndarray     # [R] first x_perm row of each range
    recv_rows: np.ndarray      # [R] rows this worker receives from each worker
    recv_start: np.ndarray     # [R, local] row of (source s, local expert j) in the source-major buffer
    grouped_start: np.ndarray  # [local, R] row of (local expert j, source s) in the grouped buffer
    grouped_offsets: np.ndarray  # [local + 1] expert segments of the grouped buffer

    @property
    def received(self) -> int:
        return int(self.recv_rows.sum())

    def to_grouped(self):
        """(source row, destination row, rows) moves from the source-major to the grouped layout."""
        return [(int(self.recv_start[s, j]), int(self.grouped_start[j, s]), int(self.counts[s, self.e0 + j]))
                for j in range(self.local) for s in range(self.R) if self.counts[s, self.e0 + j] > 0]

    def to_source_major(self):
        """The reverse moves: grouped layout back to the source-major one."""
        return [(d, s_, n) for (s_, d, n) in self.to_grouped()]

    @property
    def e0(self) -> int:
        return self.rank * self.local


def exchange_plan(counts: np.ndarray, rank: int, placement: ExpertPlacement) -> ExchangePlan:
    """The plan of worker `rank` from counts[s, e] = kept rows of expert e on worker s (every worker's
    expert_counts).  Pure integer bookkeeping; every worker computes the same counts matrix."""
    counts = np.asarray(counts, np.int64)
    R, E, L = placement.R, placement.E, placement.local
    if counts.shape != (R, E):
        raise ValueError(f"counts must be [{R}, {E}], got {counts.shape}")
    per_dest = counts.reshape(R, R, L)  # [source, destination worker, local expert]
    send_rows = per_dest[rank].sum(axis=1)
    send_start = np.concatenate([[0], np.cumsum(send_rows)[:-1]])
    mine = per_dest[:, rank, :]  # [source, local expert]: the rows this worker receives
    recv_rows = mine.sum(axis=1)
    base = np.concatenate([[0], np.cumsum(recv_rows)[:-1]])
    recv_start = base[:, None] + np.concatenate([np.zeros((R, 1), np.int64), np.cumsum(mine, axis=1)[:, :-1]], axis=1)
    per_expert = mine.sum(axis=0)  # [local]
    grouped_offsets = np.concatenate([[0], np.cumsum(per_expert)])
    grouped_start = grouped_offsets[:-1, None] + np.concatenate(
        [np.zeros((L, 1), np.int64), np.cumsum(mine.T, axis=1)[:, :-1]], axis=1)
    return ExchangePlan(rank, R, L, counts, send_rows, send_start, recv_rows, recv_start, grouped_start,
                        grouped_offsets)


def ep_forward(worker, group=None):
    """One expert-parallel layer call on the process group `group` (every rank calls it, in the same order:
    it runs one all-gather and two all-to-alls).  `worker` does this rank's arithmetic:

      worker.route_permute() -> (counts [E] ints, x_perm rows [kept, H])   routing + permutation, all E experts
      worker.regroup(rows, moves, n_out) -> rows [n_out, ...]              segment moves (see ExchangePlan)
      worker.ffn_rows(rows, grouped_offsets) -> y [n, H] fp32              this rank's experts on its rows
      worker.combine(y_perm) -> out [T, H]                                 weighted combine from y in x_perm order

    Returns (out, plan)."""
    import torch
    import torch.distributed as dist

    R = dist.get_world_size(group)
    rank = dist.get_rank(group)
    counts, x_perm = worker.route_permute()
    placement = ExpertPlacement(len(counts), R)
    c = torch.as_tensor(np.asarray(counts, np.int64), device=x_perm.device)
    gathered = [torch.empty_like(c) for _ in range(R)]
    dist.all_gather(gathered, c, group=group)
    plan = exchange_plan(torch.stack(gathered).cpu().numpy(), rank, placement)
    recv = x_perm.new_empty((plan.received,) + tuple(x_perm.shape[1:]))
    dist.all_to_all_single(recv, x_perm[:int(plan.send_rows.sum())].contiguous(), plan.recv_rows.tolist(),
                           plan.send_rows.tolist(), group=group)
    grouped = worker.regroup(recv, plan.to_grouped(), plan.received)
    y_grouped = worker.ffn_rows(grouped, plan.grouped_offsets)
    y_src = worker.regroup(y_grouped, plan.to_source_major(), plan.received)
    y_perm = y_src.new_empty((int(plan.send_rows.sum()),) + tuple(y_src.shape[1:]))
    dist.all_to_all_single(y_perm, y_src, plan.send_rows.tolist(), plan.recv_rows.tolist(), group=group)
    return worker.combine(y_perm), plan


def local_shape(shape, local_experts: int):
    """The layer's shape with E = the experts one worker holds (for moe_expert_ffn_rows)."""
    from . import Shape

    s = Shape.from_buffer_copy(shape)
    s.E = local_experts
    s.k = 1
    return s


def _segment_table(segs, device):
    """Device array of moe_row_segment_t for a list of (src pointer, dst pointer, rows)."""
    import torch

    from . import RowSegment

    arr = (RowSegment * max(len(segs), 1))()
    for i, (src, dst, n) in enumerate(segs):
        arr[i] = RowSegment(src, dst, n)
    host = torch.frombuffer(bytearray(bytes(arr)), dtype=torch.uint8)
    return host.to(device)


def copy_segments(segs, row_bytes: int, status_ptr=None, stream=None):
    """One moe_copy_row_segments launch over (src pointer, dst pointer, rows) triples; returns the device
    table (keep it alive until the stream has run the copy)."""
    import torch

    from . import _check, moe_copy_row_segments

    if not segs:
        return None
    table = _segment_table(segs, "cuda")
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    _check(moe_copy_row_segments(table.data_ptr(), len(segs), row_bytes, max(n for _, _, n in segs), status_ptr, st),
           "moe_copy_row_segments")
    return table


class CudaExpertWorker:
    """This rank's share of an expert-parallel layer on its GPU, for ep_forward: routing, permutation,
    regrouping and the combine on its own MoEBuffers; the expert FFN of its own experts (W1/b1/W2/b2 hold
    only those, [E/R, ...]) through moe_expert_ffn_rows."""

    def __init__(self, buffers, W1, b1, W2, b2, local_experts: int):
        import torch

        self.buf = buffers
        self.W1, self.b1, self.W2, self.b2 = W1, b1, W2, b2
        self.local_shape = local_shape(buffers.shape, local_experts)
        self._torch = torch
        self._tables = []

    def route_permute(self):
        self.buf.route()
        self.buf.permute()
        counts = self.buf.expert_counts.cpu().numpy()
        kept = int(counts.sum())
        v = self.buf.view()
        es = 2 if self.buf.shape.dtype == 1 else 4
        H = self.buf.shape.H
        off = v.x_perm - self.buf.ws_ptr
        raw = self.buf.ws[off:off + kept * H * es]
        rows = raw.view(self._torch.bfloat16 if es == 2 else self._torch.float32).view(kept, H)
        return counts, rows

    def regroup(self, rows, moves, n_out):
        out = rows.new_empty((n_out,) + tuple(rows.shape[1:]))
        rb = rows.shape[1] * rows.element_size()
        segs = [(rows.data_ptr() + s * rb, out.data_ptr() + d * rb, n) for s, d, n in moves]
        self._tables.append(copy_segments(segs, rb))
        return out

    def ffn_rows(self, rows, grouped_offsets):
        from . import _check, moe_expert_ffn_rows, moe_expert_ffn_rows_workspace_size

        torch = self._torch
        n, H = rows.shape
        y = torch.empty((n, H), dtype=torch.float32, device=rows.device)
        if n == 0:
            return y
        offs = torch.as_tensor(np.asarray(grouped_offsets, np.int32), device=rows.device)
        wsb = moe_expert_ffn_rows_workspace_size(self.local_shape, n)
        ws = torch.empty((wsb,), dtype=torch.uint8, device=rows.device)
        ws[:256].zero_()
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        _check(moe_expert_ffn_rows(self.local_shape, n, offs.data_ptr(), rows.data_ptr(), p(self.W1), p(self.b1),
                                   p(self.W2), p(self.b2), y.data_ptr(), ws.data_ptr(), wsb,
                                   torch.cuda.current_stream().cuda_stream), "moe_expert_ffn_rows")
        self._keep = (offs, ws)
        return y

    def combine(self, y_perm):
        torch = self._torch
        v = self.buf.view()
        n, H = y_perm.shape
        off = v.y - self.buf.ws_ptr
        self.buf.ws[off:off + n * H * 4].view(torch.float32).view(n, H).copy_(y_perm)
        self.buf.combine()
        return self.buf.out


class EmulatedExpertParallel:
    """R expert-parallel workers on one GPU, each with its own batch and workspace (MoEBuffers), the experts
    split in contiguous blocks.  One call of forward() runs, on the current stream:

      every worker's moe_route + moe_permute over all E experts;
      the dispatch: one moe_copy_row_segments launch moving every (source worker, expert) segment of x_perm
        straight into the owner's grouped (expert-major) receive buffer;
      every owner's moe_expert_ffn_rows over its received rows with its block of the expert weights;
      the return: one moe_copy_row_segments launch moving every output segment straight into the source
        worker's y, at the rows its x_perm had;
      every worker's moe_combine.

    The per-expert counts are read back to the host once to build the two segment tables."""

    def __init__(self, shape, inputs: dict, batches: list, device="cuda"):
        import torch

        from . import MoEBuffers

        self.R = len(batches)
        self.placement = ExpertPlacement(shape.E, self.R)
        self.shape = shape
        self.inputs = inputs
        self.workers = []
        for x in batches:
            d = dict(inputs)
            d["x"] = x
            self.workers.append(MoEBuffers(shape, d, device=device))
        self.local_shape = local_shape(shape, self.placement.local)
        self.es = 2 if shape.dtype == 1 else 4
        self._torch = torch
        self.status = torch.zeros((1,), dtype=torch.int32, device=device)

    def _expert_block(self, name, d):
        """Device pointer of worker d's block of expert tensor `name` (None stays None)."""
        t = self.inputs.get(name)
        if t is None:
            return None
        per_expert = t[0].numel() * t.element_size()
        return t.data_ptr() + d * self.placement.local * per_expert

    def forward(self):
        import torch

        from . import _check, moe_expert_ffn_rows, moe_expert_ffn_rows_workspace_size

        R, L, H, es = self.R, self.placement.local, self.shape.H, self.es
        for w in self.workers:
            w.route()
            w.permute()
        counts = np.stack([w.expert_counts.cpu().numpy() for w in self.workers]).astype(np.int64)
        views = [w.view() for w in self.workers]
        offsets = [np.concatenate([[0], np.cumsum(c)]) for c in counts]
        self.plans = [exchange_plan(counts, d, self.placement) for d in range(R)]
        self.recv = [torch.empty((max(p.received, 1), H), dtype=self.workers[0].inputs["x"].dtype,
                                 device=self.status.device) for p in self.plans]
        self.y_recv = [torch.empty((max(p.received, 1), H), dtype=torch.float32, device=self.status.device)
                       for p in self.plans]
        disp, ret = [], []
        for d, p in enumerate(self.plans):
            for j in range(L):
                e = d * L + j
                for s in range(R):
                    n = int(counts[s, e])
                    if n == 0:
                        continue
                    g = int(p.grouped_start[j, s])
                    disp.append((views[s].x_perm + int(offsets[s][e]) * H * es, self.recv[d].data_ptr() + g * H * es, n))
                    ret.append((self.y_recv[d].data_ptr() + g * H * 4, views[s].y + int(offsets[s][e]) * H * 4, n))
        st = self.status.data_ptr()
        self._t1 = copy_segments(disp, H * es, st)
        self._keep = []
        stream = torch.cuda.current_stream().cuda_stream
        for d, p in enumerate(self.plans):
            n = p.received
            if n == 0:
                continue
            offs = torch.as_tensor(p.grouped_offsets.astype(np.int32), device=self.status.device)
            wsb = moe_expert_ffn_rows_workspace_size(self.local_shape, n)
            ws = torch.empty((wsb,), dtype=torch.uint8, device=self.status.device)
            ws[:256].zero_()
            _check(moe_expert_ffn_rows(self.local_shape, n, offs.data_ptr(), self.recv[d].data_ptr(),
                                       self._expert_block("W1", d), self._expert_block("b1", d),
                                       self._expert_block("W2", d), self._expert_block("b2", d),
                                       self.y_recv[d].data_ptr(), ws.data_ptr(), wsb, stream), "moe_expert_ffn_rows")
            self._keep.append((offs, ws))
        self._t2 = copy_segments(ret, H * 4, st)
        for w in self.workers:
            w.combine()
        return [w.out for w in self.workers]

    def ffn_status(self) -> list:
        """Device error words of the per-worker expert FFN workspaces (0 = ok) after forward()."""
        return [int(ws[:4].view(self._torch.int32).item()) for _, ws in self._keep]



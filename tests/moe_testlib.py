"""Helpers shared by the GPU parity tests: upload seeded inputs, run the CUDA stages through the C ABI,
and the tolerance rules used against the oracle.

Tolerances (written here once, used by every parity test):
  * integer outputs (top-k indices, counts, drop flags, row maps): bit-exact, except tokens whose
    oracle logit margin (smallest gap among the top-(k+1) logits) is below NEAR_TIE; those are
    excluded from the index comparison and counted;
  * fp32 path: normwise relative error max|d| / max|ref| <= 1e-4 per output tensor;
  * bf16-input / fp32-accumulate path: max|d| <= 2e-2 * RMS(ref) per output tensor;
  * topk_w (fp32 from fp32 logits): max relative error 1e-4; losses: relative error 1e-3;
  * backward pass (bf16 path): max|d| <= 4e-2 * RMS(ref) and ||d||_F <= 1e-2 * ||ref||_F per gradient
    tensor.  Each product of a weight-gradient GEMM multiplies two bf16-rounded operands (h and the
    weighted dout rows, or x and du), where the forward GEMMs round one (h); a rounding of 2^-9
    relative on each operand gives a bulk (Frobenius) error of a few 1e-3, and the largest of ~1e5
    elements reaches 4-5 standard deviations of it.  A wrong or missing term moves the Frobenius
    error to O(1).  The per-expert weight and bias gradients are checked per expert (each is its
    own GEMM over its own rows, and the experts' scales differ): max|d_e| <= 4e-2 * RMS(ref_e).
"""
from __future__ import annotations

import math

import numpy as np

import synth

NEAR_TIE = 1e-4
TOL_F32 = 1e-4
TOL_BF16_RMS = 2e-2
TOL_W = 1e-4
TOL_LOSS = 1e-3
TOL_BWD_MAX = 4e-2
TOL_BWD_FRO = 1e-2


def torch_dtype(dtype: str):
    import torch

    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_device(arr: np.ndarray, dtype: str, device="cuda"):
    import torch

    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)


def upload(inp: synth.LayerInputs, device="cuda") -> dict:
    return {name: to_device(a, inp.cfg.dtype, device) for name, a in inp.arrays().items()}


def shape_of(cfg: synth.LayerConfig):
    import sparse_mixture_experts_23_b200 as moe

    return moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.k, cfg.F, cfg.CF, cfg.dtype, cfg.act, cfg.routing, cfg.min_capacity)


def from_device_bits(t, dtype: str) -> np.ndarray:
    """Storage-dtype tensor -> numpy in the oracle's input convention (bf16 as uint16 bits)."""
    import torch

    if dtype == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def normwise_rel(a: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    return float(np.max(np.abs(a - ref))) / den if den > 0 else float(np.max(np.abs(a - ref), initial=0.0))


def rms_rel(a: np.ndarray, ref: np.ndarray) -> float:
    rms = math.sqrt(float(np.mean(np.square(ref)))) if ref.size else 0.0
    d = float(np.max(np.abs(a - ref), initial=0.0))
    return d / rms if rms > 0 else d


def out_error(a: np.ndarray, ref: np.ndarray, dtype: str, rows=None) -> tuple[float, float]:
    """(error, tolerance) under the rule for the storage dtype.

    ``rows`` (boolean mask) restricts both the error and the reference scale to the output rows
    that received at least one expert output: rows whose every slot was dropped are zero by
    definition, are checked for exact zeros separately, and would otherwise shrink RMS(ref)."""
    if rows is not None:
        a, ref = a[rows], ref[rows]
    if dtype == "f32":
        return normwise_rel(a, ref), TOL_F32
    return rms_rel(a, ref), TOL_BF16_RMS


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    if T <= n:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    fixed = [0, 1, T // 2, T - 2, T - 1]
    rest = rng.choice(np.arange(2, T - 2), size=n - len(fixed), replace=False)
    return np.unique(np.concatenate([fixed, rest])).astype(np.int32)


def stratified_rows(offsets, tile: int = 128, seed: int = 0) -> np.ndarray:
    """Rows of the permuted layout chosen so that every GEMM tile of every expert segment is checked:
    the first and last row of each non-empty segment, one random row in each 128-row block (every
    128-row and 256-row m-tile starts on a block boundary inside its segment), and every row of each
    segment's last block (the expert's tail tile: a half pair tile when it holds <= 128 rows)."""
    rng = np.random.default_rng(seed)
    rows = []
    offsets = np.asarray(offsets)
    for e in range(len(offsets) - 1):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b <= a:
            continue
        rows += [a, b - 1]
        rows += [int(rng.integers(m0, min(b, m0 + tile))) for m0 in range(a, b, tile)]
        rows += range(a + ((b - a - 1) // tile) * tile, b)
    return np.unique(np.asarray(rows, np.int64))


def stratified_tokens(offsets, row_token, tile: int = 128, seed: int = 0) -> np.ndarray:
    """Tokens owning the stratified rows (each token's whole output row, every slot, is then checked)."""
    rows = stratified_rows(offsets, tile, seed)
    return np.unique(np.asarray(row_token)[rows]).astype(np.int32)


def stratified_columns(n: int, block: int = 256, extra_last: int = 8, seed: int = 0) -> np.ndarray:
    """One random column in every `block`-wide block of n columns (every N tile of the GEMMs that produce
    or consume them), plus `extra_last` more from the last block, whole or partial."""
    rng = np.random.default_rng(seed)
    cols = [int(rng.integers(c0, min(n, c0 + block))) for c0 in range(0, n, block)]
    last0 = ((n - 1) // block) * block
    cols += rng.choice(np.arange(last0, n), size=min(extra_last, n - last0), replace=False).tolist()
    cols.append(n - 1)
    return np.unique(np.asarray(cols, np.int32))


def fro_rel(a: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.linalg.norm(ref))
    num = float(np.linalg.norm(a - ref))
    return num / den if den > 0 else num


def gate_in_gemm_epilogue(cfg, sms: int = 148) -> bool:
    """Whether the gate is one tensor-core GEMM with the softmax / top-k in its epilogue: bf16 token
    choice with 64, 128 or 256 experts and at least sms/2 tiles of 128 tokens."""
    return (cfg.dtype == "bf16" and cfg.routing == "token_choice" and cfg.E in (64, 128, 256)
            and 2 * ((cfg.T + 127) // 128) >= sms)


def router_launches(cfg, sms: int = 148) -> int:
    """Kernels of the gate: one, or two (a tensor-core logits GEMM, then the per-chunk softmax / top-k
    kernel) for bf16 layers whose expert count is a multiple of 64 -- except when the softmax / top-k
    runs in the GEMM's epilogue (one kernel)."""
    if cfg.dtype != "bf16" or cfg.E % 64 != 0:
        return 1
    return 1 if gate_in_gemm_epilogue(cfg, sms) else 2


def reduce_launches(cfg, sms: int = 148) -> int:
    """Separate reduce kernels after the gate under token choice: none when the gate works chunk by
    chunk and the partials fit its last block (k * ceil(T/32) * E <= 16 * 256 values; that block then
    reduces the losses and the dispatch), else one (also after the GEMM-epilogue gate)."""
    fits = cfg.k * ((cfg.T + 31) // 32) * cfg.E <= 16 * 256
    return 1 if gate_in_gemm_epilogue(cfg, sms) or not fits else 0

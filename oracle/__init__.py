"""fp64 CPU oracle of the sparse top-k MoE layer forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of ``bench.py`` may
import this package.  The CUDA library and its Python binding never import it, and the two share no
code; the only thing both sides see is the seeded input generator (``synth``), which holds no MoE
arithmetic.

The arithmetic lives in ``moe_oracle.c`` (plain loops in double, each function citing the page and
section it follows).  This wrapper only marshals numpy arrays through ctypes and composes the
documented steps:

  route      -> logits, logsumexp, softmax, top-k (logit desc, index asc), renormalised weights
  losses     -> Switch aux loss E*sum f*P (pre-drop counts / (T*k)), z-loss mean(lse^2)
  dispatch   -> capacity ceil(CF*T*k/E) or unlimited; slot-major then token-order ranks; rows
  forward    -> out[t] = sum over kept slots of w * FFN_e(x_t)
  expert choice (ec_*) -> every expert takes its top-C tokens by logit; out[t] = sum over the
                experts that chose t of p[t,e] * FFN_e(x_t)
  backward (bwd_*) -> gradients of L = sum dout*out + d_aux*aux + d_z*z with respect to x and every
                weight, by the chain rule through the definitions above

Parity status of each function is recorded in the test-suite pins (``tests/test_oracle_pins.py``);
every function here is pinned there against closed forms, library routines or brute force.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

F32, BF16 = 0, 1
_DT = {"f32": F32, "bf16": BF16}
ACT = {"gelu": 0, "silu": 1}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, IEEE semantics kept: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, vp, c_int, dbl = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_double
    lib.oracle_gelu.argtypes = [dbl]
    lib.oracle_gelu.restype = dbl
    lib.oracle_silu.argtypes = [dbl]
    lib.oracle_silu.restype = dbl
    lib.oracle_capacity.argtypes = [dbl, i64, i64, i64, i64]
    lib.oracle_capacity.restype = i64
    lib.oracle_route.argtypes = [i64, i64, i64, i64, c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.oracle_route.restype = None
    lib.oracle_losses.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp]
    lib.oracle_losses.restype = None
    lib.oracle_dispatch.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.oracle_dispatch.restype = i64
    lib.oracle_expert_rows.argtypes = [i64, i64, c_int, c_int, vp, vp, vp, vp, vp, i64, vp, vp, vp, c_int]
    lib.oracle_expert_rows.restype = None
    lib.oracle_forward_tokens.argtypes = [i64, i64, i64, c_int, c_int, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp,
                                          vp, c_int]
    lib.oracle_forward_tokens.restype = None
    lib.oracle_ec_capacity.argtypes = [dbl, i64, i64, i64, i64]
    lib.oracle_ec_capacity.restype = i64
    lib.oracle_expert_choice.argtypes = [i64, i64, i64, vp, vp, vp]
    lib.oracle_expert_choice.restype = None
    lib.oracle_ec_losses.argtypes = [i64, i64, i64, vp, vp, vp, vp]
    lib.oracle_ec_losses.restype = None
    lib.oracle_act_grad.argtypes = [c_int, dbl]
    lib.oracle_act_grad.restype = dbl
    lib.oracle_bwd_slot.argtypes = [i64, i64, c_int, c_int, vp, i64, ctypes.c_int32, vp, vp, vp, vp, vp, dbl, vp,
                                    vp, vp]
    lib.oracle_bwd_slot.restype = None
    lib.oracle_bwd_expert_weights.argtypes = [i64, i64, c_int, c_int, vp, ctypes.c_int32, vp, vp, vp, i64, vp, vp,
                                              vp, i64, vp, vp, vp, vp, vp, c_int]
    lib.oracle_bwd_expert_weights.restype = None
    lib.oracle_bwd_router.argtypes = [i64, i64, i64, i64, c_int, vp, vp, vp, vp, vp, vp, dbl, dbl, vp, vp, vp, vp]
    lib.oracle_bwd_router.restype = None
    lib.oracle_bwd_router_ec.argtypes = [i64, i64, i64, c_int, vp, vp, vp, vp, dbl, dbl, vp, vp, vp, vp]
    lib.oracle_bwd_router_ec.restype = None
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = c_int
    lib.oracle_set_threads.argtypes = [c_int]
    lib.oracle_set_threads.restype = None
    _lib = lib
    return lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype=None):
    a = np.ascontiguousarray(a) if dtype is None else np.ascontiguousarray(a, dtype=dtype)
    return a


def max_threads() -> int:
    return _load().oracle_max_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def gelu(u: float) -> float:
    return _load().oracle_gelu(float(u))


def silu(u: float) -> float:
    return _load().oracle_silu(float(u))


def _opt(a):
    """Optional bias: None stays None (NULL pointer, i.e. zeros)."""
    return None if a is None else _c(a)


def capacity(cf: float, T: int, k: int, E: int, min_capacity: int = 0):
    """Per-expert capacity max(ceil(CF*T*k/E), min_capacity), or None when unlimited (CF = +inf)."""
    c = _load().oracle_capacity(float(cf), T, k, E, int(min_capacity))
    return None if c < 0 else int(c)


@dataclass
class Routing:
    logits: np.ndarray  # [T,E] f64
    lse: np.ndarray  # [T] f64
    p: np.ndarray  # [T,E] f64
    topk_idx: np.ndarray  # [T,k] int32
    topk_w: np.ndarray  # [T,k] f64
    margin: np.ndarray  # [T] f64: smallest adjacent gap among the top-(k+1) logits


def route(x, Wg, bg, k: int, dtype: str) -> Routing:
    x, Wg, bg = _c(x), _c(Wg), _opt(bg)
    T, H = x.shape
    E = Wg.shape[1]
    logits = np.empty((T, E), np.float64)
    lse = np.empty(T, np.float64)
    p = np.empty((T, E), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    margin = np.empty(T, np.float64)
    _load().oracle_route(T, H, E, k, _DT[dtype], _p(x), _p(Wg), _p(bg), _p(logits), _p(lse), _p(p), _p(idx),
                         _p(w), _p(margin))
    return Routing(logits, lse, p, idx, w, margin)


def losses(p, lse, topk_idx):
    p, lse, idx = _c(p, np.float64), _c(lse, np.float64), _c(topk_idx, np.int32)
    T, E = p.shape if p.ndim == 2 else (0, 0)
    k = idx.shape[1] if idx.ndim == 2 else 0
    aux = np.zeros(1, np.float64)
    z = np.zeros(1, np.float64)
    _load().oracle_losses(T, E, k, _p(p), _p(lse), _p(idx), _p(aux), _p(z))
    return float(aux[0]), float(z[0])


@dataclass
class Dispatch:
    cap: int | None
    cnt_pre: np.ndarray  # [E] int32
    expert_counts: np.ndarray  # [E] int32
    offsets: np.ndarray  # [E+1] int32
    dropped: np.ndarray  # [T,k] uint8
    row_of: np.ndarray  # [T,k] int32
    row_token: np.ndarray  # [kept] int32
    row_slot: np.ndarray  # [kept] int32

    @property
    def kept(self) -> int:
        return int(self.offsets[-1])


def dispatch(topk_idx, E: int, cf: float, min_capacity: int = 0) -> Dispatch:
    idx = _c(topk_idx, np.int32)
    T, k = idx.shape
    cap = capacity(cf, T, k, E, min_capacity)
    cnt_pre = np.empty(E, np.int32)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    dropped = np.empty((T, k), np.uint8)
    row_of = np.empty((T, k), np.int32)
    row_token = np.full(max(T * k, 1), -1, np.int32)
    row_slot = np.full(max(T * k, 1), -1, np.int32)
    kept = _load().oracle_dispatch(T, E, k, -1 if cap is None else cap, _p(idx), _p(cnt_pre), _p(counts),
                                   _p(offsets), _p(dropped), _p(row_of), _p(row_token), _p(row_slot))
    return Dispatch(cap, cnt_pre, counts, offsets, dropped, row_of, row_token[:kept].copy(),
                    row_slot[:kept].copy())


def expert_rows(x, W1, b1, W2, b2, tokens, experts, dtype: str, nthreads: int = 0, act: str = "gelu") -> np.ndarray:
    """y[i] = FFN_{experts[i]}(x[tokens[i]]) in double; b1/b2 may be None (no bias)."""
    x, W1, b1, W2, b2 = _c(x), _c(W1), _opt(b1), _c(W2), _opt(b2)
    tokens, experts = _c(tokens, np.int32), _c(experts, np.int32)
    E, H, F = W1.shape
    n = tokens.shape[0]
    y = np.empty((n, H), np.float64)
    _load().oracle_expert_rows(H, F, _DT[dtype], ACT[act], _p(x), _p(W1), _p(b1), _p(W2), _p(b2), n, _p(tokens),
                               _p(experts), _p(y), int(nthreads))
    return y


def forward_tokens(x, W1, b1, W2, b2, topk_idx, topk_w, dropped, tokens, dtype: str,
                   nthreads: int = 0, act: str = "gelu") -> np.ndarray:
    """out[i] = sum over kept slots of w * FFN(x[tokens[i]]) in double, for the listed tokens."""
    x, W1, b1, W2, b2 = _c(x), _c(W1), _opt(b1), _c(W2), _opt(b2)
    idx, w = _c(topk_idx, np.int32), _c(topk_w, np.float64)
    drp = None if dropped is None else _c(dropped, np.uint8)
    tokens = _c(tokens, np.int32)
    E, H, F = W1.shape
    k = idx.shape[1]
    n = tokens.shape[0]
    out = np.empty((n, H), np.float64)
    _load().oracle_forward_tokens(H, F, k, _DT[dtype], ACT[act], _p(x), _p(W1), _p(b1), _p(W2), _p(b2), _p(idx),
                                  _p(w), _p(drp), n, _p(tokens), _p(out), int(nthreads))
    return out


@dataclass
class Forward:
    routing: Routing
    aux: float
    z: float
    disp: Dispatch
    out: np.ndarray | None  # [len(tokens), H] f64
    tokens: np.ndarray


def forward(x, Wg, bg, W1, b1, W2, b2, k: int, cf: float, dtype: str, tokens=None, nthreads: int = 0,
            act: str = "gelu", min_capacity: int = 0) -> Forward:
    """Whole layer: routing and dispatch over all tokens, FFN + combine for ``tokens`` (default: all)."""
    r = route(x, Wg, bg, k, dtype)
    aux, z = losses(r.p, r.lse, r.topk_idx)
    d = dispatch(r.topk_idx, Wg.shape[1], cf, min_capacity)
    T = x.shape[0]
    tokens = np.arange(T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    out = forward_tokens(x, W1, b1, W2, b2, r.topk_idx, r.topk_w, d.dropped, tokens, dtype, nthreads, act)
    return Forward(r, aux, z, d, out, tokens)


# ------------------------------------------------------------------ expert-choice routing -------

def ec_capacity(cf: float, T: int, k: int, E: int, min_capacity: int = 0) -> int:
    """Tokens per expert under expert choice: min(T, max(ceil(CF*T*k/E), min_capacity)); T when CF = +inf."""
    return int(_load().oracle_ec_capacity(float(cf), T, k, E, int(min_capacity)))


@dataclass
class ExpertChoice:
    C: int
    chosen: np.ndarray  # [E, C] int32, ascending token order per expert
    margin: np.ndarray  # [E] f64: gap between the C-th and (C+1)-th logit of each expert

    def member(self, T: int) -> np.ndarray:
        """[T, E] bool: token t chosen by expert e."""
        E = self.chosen.shape[0]
        m = np.zeros((T, E), bool)
        for e in range(E):
            m[self.chosen[e], e] = True
        return m


def expert_choice(logits, C: int) -> ExpertChoice:
    lg = _c(logits, np.float64)
    T, E = lg.shape
    chosen = np.empty((E, max(C, 0)), np.int32)
    margin = np.empty(E, np.float64)
    _load().oracle_expert_choice(T, E, C, _p(lg), _p(chosen), _p(margin))
    return ExpertChoice(C, chosen, margin)


def ec_losses(p, lse, C: int):
    p, lse = _c(p, np.float64), _c(lse, np.float64)
    T, E = p.shape
    aux = np.zeros(1, np.float64)
    z = np.zeros(1, np.float64)
    _load().oracle_ec_losses(T, E, C, _p(p), _p(lse), _p(aux), _p(z))
    return float(aux[0]), float(z[0])


def ec_forward_tokens(x, W1, b1, W2, b2, p, member, tokens, dtype: str, nthreads: int = 0,
                      act: str = "gelu") -> np.ndarray:
    """out[i] = sum over experts e that chose token tokens[i] of p[t,e] * FFN_e(x_t), experts in
    ascending order: the token-choice combine with every expert as a slot and the unchosen ones
    dropped."""
    p = _c(p, np.float64)
    T, E = p.shape
    idx = np.tile(np.arange(E, dtype=np.int32), (T, 1))
    dropped = (~np.asarray(member, bool)).astype(np.uint8)
    return forward_tokens(x, W1, b1, W2, b2, idx, p, dropped, tokens, dtype, nthreads, act)


@dataclass
class ForwardEC:
    routing: Routing
    ec: ExpertChoice
    aux: float
    z: float
    out: np.ndarray
    tokens: np.ndarray


def forward_ec(x, Wg, bg, W1, b1, W2, b2, k: int, cf: float, dtype: str, tokens=None, nthreads: int = 0,
               act: str = "gelu") -> ForwardEC:
    """Whole layer under expert-choice routing (Core Concepts 2)."""
    T = x.shape[0]
    E = Wg.shape[1]
    r = route(x, Wg, bg, 1, dtype)
    C = ec_capacity(cf, T, k, E)
    ec = expert_choice(r.logits, C)
    aux, z = ec_losses(r.p, r.lse, C)
    tokens = np.arange(T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    out = ec_forward_tokens(x, W1, b1, W2, b2, r.p, ec.member(T), tokens, dtype, nthreads, act)
    return ForwardEC(r, ec, aux, z, out, tokens)


# ------------------------------------------------------------------ backward pass ----------------

def act_grad(u: float, act: str = "gelu") -> float:
    return _load().oracle_act_grad(ACT[act], float(u))


def bwd_slot(x, W1, b1, W2, b2, t: int, e: int, dout_t, w: float, dtype: str, act: str = "gelu"):
    """One kept slot: (dx_part[H] = W1[e] du, dw = dout_t . y, du[F])."""
    x, W1, b1, W2, b2 = _c(x), _c(W1), _opt(b1), _c(W2), _opt(b2)
    E, H, F = W1.shape
    d = _c(dout_t, np.float64)
    dx = np.empty(H, np.float64)
    du = np.empty(F, np.float64)
    dw = np.zeros(1, np.float64)
    _load().oracle_bwd_slot(H, F, _DT[dtype], ACT[act], _p(x), int(t), int(e), _p(W1), _p(b1), _p(W2), _p(b2), _p(d),
                            float(w), _p(dx), _p(dw), _p(du))
    return dx, float(dw[0]), du


def bwd_expert_weights(x, W1, b1, W2, e: int, tokens, w, dout, fcols, dtype: str, act: str = "gelu",
                       nthreads: int = 0):
    """Expert e's weight gradients from its kept rows, at FFN columns fcols:
    (dW2[e][fcols, :], dW1[e][:, fcols].T, db1[e][fcols], db2[e])."""
    x, W1, b1, W2 = _c(x), _c(W1), _opt(b1), _c(W2)
    E, H, F = W1.shape
    tokens, w = _c(tokens, np.int32), _c(w, np.float64)
    dout = _c(dout, np.float64)
    fcols = _c(fcols, np.int32)
    nf = fcols.shape[0]
    dW2r = np.empty((nf, H), np.float64)
    dW1c = np.empty((nf, H), np.float64)
    db1 = np.empty(nf, np.float64)
    db2 = np.empty(H, np.float64)
    _load().oracle_bwd_expert_weights(H, F, _DT[dtype], ACT[act], _p(x), int(e), _p(W1), _p(b1), _p(W2),
                                      tokens.shape[0], _p(tokens), _p(w), _p(dout), nf, _p(fcols), _p(dW2r), _p(dW1c),
                                      _p(db1), _p(db2), int(nthreads))
    return dW2r, dW1c, db1, db2


def bwd_router(x, Wg, bg, topk_idx, cnt_pre, dw, d_aux: float, d_z: float, dtype: str):
    """(dlogits[T,E], dWg[H,E], dbg[E], dx_router[T,H]) given dw[T,k] (0 on dropped slots)."""
    x, Wg, bg = _c(x), _c(Wg), _opt(bg)
    idx, cnt, dw = _c(topk_idx, np.int32), _c(cnt_pre, np.int32), _c(dw, np.float64)
    T, H = x.shape
    E = Wg.shape[1]
    k = idx.shape[1]
    dl = np.empty((T, E), np.float64)
    dWg = np.empty((H, E), np.float64)
    dbg = np.empty(E, np.float64)
    dxr = np.empty((T, H), np.float64)
    _load().oracle_bwd_router(T, H, E, k, _DT[dtype], _p(x), _p(Wg), _p(bg), _p(idx), _p(cnt), _p(dw), float(d_aux),
                              float(d_z), _p(dl), _p(dWg), _p(dbg), _p(dxr))
    return dl, dWg, dbg, dxr


@dataclass
class Grads:
    dx: np.ndarray    # [T,H]
    dWg: np.ndarray   # [H,E]
    dbg: np.ndarray   # [E]
    dW1: np.ndarray   # [E,H,F]
    db1: np.ndarray   # [E,F]
    dW2: np.ndarray   # [E,F,H]
    db2: np.ndarray   # [E,H]
    dw: np.ndarray    # [T,k] gradient of each slot's combine weight (0 when dropped)
    dlogits: np.ndarray  # [T,E]


def backward(x, Wg, bg, W1, b1, W2, b2, k: int, cf: float, dtype: str, dout, d_aux: float, d_z: float,
             act: str = "gelu", topk_idx=None, dropped=None) -> Grads:
    """All gradients of L = sum(dout*out) + d_aux*aux + d_z*z (small problems).  The routing is the
    oracle's own unless topk_idx / dropped are given (e.g. the GPU's, to avoid near-tie flips)."""
    T, H = x.shape
    E, _, F = W1.shape
    r = route(x, Wg, bg, k, dtype)
    idx = r.topk_idx if topk_idx is None else np.asarray(topk_idx, np.int32)
    w = r.topk_w if topk_idx is None else renorm_weights(r.p, idx)
    d = dispatch(idx, E, cf)
    drp = d.dropped if dropped is None else np.asarray(dropped, np.uint8)
    dout = _c(dout, np.float64)
    dx = np.zeros((T, H))
    dw = np.zeros((T, k))
    rows = {e: ([], []) for e in range(E)}
    for t in range(T):
        for s in range(k):
            if drp[t, s]:
                continue
            e = int(idx[t, s])
            dxp, dws, _ = bwd_slot(x, W1, b1, W2, b2, t, e, dout[t], w[t, s], dtype, act)
            dx[t] += dxp
            dw[t, s] = dws
            rows[e][0].append(t)
            rows[e][1].append(w[t, s])
    dW1 = np.zeros((E, H, F))
    dW2 = np.zeros((E, F, H))
    db1 = np.zeros((E, F))
    db2 = np.zeros((E, H))
    allf = np.arange(F, dtype=np.int32)
    for e in range(E):
        toks, ws = rows[e]
        r2, c1, b1s, b2s = bwd_expert_weights(x, W1, b1, W2, e, np.array(toks, np.int32), np.array(ws), dout, allf,
                                              dtype, act)
        dW2[e] = r2
        dW1[e] = c1.T
        db1[e] = b1s
        db2[e] = b2s
    dl, dWg, dbg, dxr = bwd_router(x, Wg, bg, idx, d.cnt_pre, dw, d_aux, d_z, dtype)
    return Grads(dx + dxr, dWg, dbg, dW1, db1, dW2, db2, dw, dl)


def renorm_weights(p, idx):
    """w[t,s] = p[t, idx[t,s]] / sum_s' p[t, idx[t,s']]: the Quick Start's division of the selected
    softmax scores by their sum, for a given selection (not necessarily the top-k of p).  The
    weights are pre-drop values: a dropped slot keeps its weight and contributes nothing."""
    sel = np.take_along_axis(np.asarray(p, np.float64), np.asarray(idx, np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def loss_of_given(x, Wg, bg, W1, b1, W2, b2, topk_idx, dropped, dtype: str, dout, d_aux: float, d_z: float,
                  act: str = "gelu") -> float:
    """L = sum(dout * out) + d_aux * aux + d_z * z with the routing held fixed at (topk_idx, dropped):
    p and lse from the gate as usual, the weights renormalised over the given selection, out from
    the kept slots only, aux from the given selection's pre-drop counts.  This is the function whose
    gradient backward(..., topk_idx=, dropped=) returns."""
    idx = np.asarray(topk_idx, np.int32)
    k = idx.shape[1]
    r = route(x, Wg, bg, k, dtype)
    w = renorm_weights(r.p, idx)
    aux, z = losses(r.p, r.lse, idx)
    T = x.shape[0]
    out = forward_tokens(x, W1, b1, W2, b2, idx, w, dropped, np.arange(T, dtype=np.int32), dtype, act=act)
    return float(np.sum(np.asarray(dout, np.float64) * out)) + d_aux * aux + d_z * z


def loss_of(x, Wg, bg, W1, b1, W2, b2, k: int, cf: float, dtype: str, dout, d_aux: float, d_z: float,
            act: str = "gelu") -> float:
    """L = sum(dout * out) + d_aux * aux + d_z * z of the oracle's forward pass."""
    f = forward(x, Wg, bg, W1, b1, W2, b2, k, cf, dtype, act=act)
    return float(np.sum(np.asarray(dout, np.float64) * f.out)) + d_aux * f.aux + d_z * f.z


def bwd_router_ec(x, Wg, bg, dw, d_aux: float, d_z: float, dtype: str):
    """Expert-choice router backward: (dlogits[T,E], dWg[H,E], dbg[E], dx_router[T,H]) given dw[T,E]
    (dout_t . y for the chosen pairs, 0 elsewhere)."""
    x, Wg, bg, dw = _c(x), _c(Wg), _opt(bg), _c(dw, np.float64)
    T, H = x.shape
    E = Wg.shape[1]
    dl = np.empty((T, E), np.float64)
    dWg = np.empty((H, E), np.float64)
    dbg = np.empty(E, np.float64)
    dxr = np.empty((T, H), np.float64)
    _load().oracle_bwd_router_ec(T, H, E, _DT[dtype], _p(x), _p(Wg), _p(bg), _p(dw), float(d_aux), float(d_z), _p(dl),
                                 _p(dWg), _p(dbg), _p(dxr))
    return dl, dWg, dbg, dxr


def backward_ec(x, Wg, bg, W1, b1, W2, b2, k: int, cf: float, dtype: str, dout, d_aux: float, d_z: float,
                act: str = "gelu", chosen=None) -> Grads:
    """All gradients of L = sum(dout*out) + d_aux*aux + d_z*z under expert choice (small problems).
    The selection is the oracle's own unless chosen[E,C] is given.  Grads.dw is [T,E] here."""
    T, H = x.shape
    E, _, F = W1.shape
    r = route(x, Wg, bg, 1, dtype)
    if chosen is None:
        chosen = expert_choice(r.logits, ec_capacity(cf, T, k, E)).chosen
    chosen = np.asarray(chosen, np.int32)
    dout = _c(dout, np.float64)
    dx = np.zeros((T, H))
    dw = np.zeros((T, E))
    dW1 = np.zeros((E, H, F))
    dW2 = np.zeros((E, F, H))
    db1 = np.zeros((E, F))
    db2 = np.zeros((E, H))
    allf = np.arange(F, dtype=np.int32)
    for e in range(E):
        toks = chosen[e]
        ws = r.p[toks, e]
        for t, w in zip(toks, ws):
            dxp, dws, _ = bwd_slot(x, W1, b1, W2, b2, int(t), e, dout[t], float(w), dtype, act)
            dx[t] += dxp
            dw[t, e] = dws
        r2, c1, b1s, b2s = bwd_expert_weights(x, W1, b1, W2, e, toks, ws, dout, allf, dtype, act)
        dW2[e] = r2
        dW1[e] = c1.T
        db1[e] = b1s
        db2[e] = b2s
    dl, dWg, dbg, dxr = bwd_router_ec(x, Wg, bg, dw, d_aux, d_z, dtype)
    return Grads(dx + dxr, dWg, dbg, dW1, db1, dW2, db2, dw, dl)


def loss_of_ec(x, Wg, bg, W1, b1, W2, b2, k: int, cf: float, dtype: str, dout, d_aux: float, d_z: float,
               act: str = "gelu") -> float:
    """L = sum(dout * out) + d_aux * aux + d_z * z of the oracle's expert-choice forward pass."""
    f = forward_ec(x, Wg, bg, W1, b1, W2, b2, k, cf, dtype, act=act)
    return float(np.sum(np.asarray(dout, np.float64) * f.out)) + d_aux * f.aux + d_z * f.z

"""Seeded synthetic inputs for the sparse top-k MoE layer (shared by tests, bench and oracle checks).

This module holds no MoE arithmetic.  It generates the layer's inputs -- activations x[T,H], gate
weights Wg[H,E], bg[E] and expert weights W1[E,H,F], b1[E,F], W2[E,F,H], b2[E,H] -- from a
counter-based generator (``synth.c`` states the exact definition) and rounds them to the storage
dtype.  Values are produced on the host so that the CUDA path and the oracle see the same bits.

The workload recipes (``CONFIGS``) restate the synthetic layer shapes used for parity and
measurement: a tiny fp32 layer, a decode-sized layer, a Switch-style training layer with a capacity
factor, a Mixtral-shaped layer, a skewed-load layer, the Mixtral block's own expert variant
(bias-free, SiLU) and expert-choice routing, both at the Mixtral shape.  Shapes follow the pages' DeepSpeed
launch examples ("MoE Training" skill page, Quick Start / Training Script sections) where they give
them.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        for name in ("synth_normal_f32", "synth_normal_bf16"):
            fn = getattr(lib, name)
            fn.argtypes = [u64, u64, u64, i64, dbl, dbl, vp]
            fn.restype = None
        lib.synth_words.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_words.restype = None
        lib.synth_f32_to_bf16.argtypes = [vp, i64, vp]
        lib.synth_f32_to_bf16.restype = None
        _lib = lib
    return _lib


def words(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().synth_words(seed, stream, offset, n, out.ctypes.data)
    return out


def normal(seed: int, stream: int, shape, mean: float = 0.0, std: float = 1.0, dtype: str = "f32",
           offset: int = 0) -> np.ndarray:
    """mean + std*N(0,1), shaped; ``dtype`` "f32" gives float32, "bf16" gives uint16 bf16 bit patterns."""
    n = int(np.prod(shape)) if len(shape) else 1
    lib = _load()
    if dtype == "f32":
        out = np.empty(n, dtype=np.float32)
        lib.synth_normal_f32(seed, stream, offset, n, float(mean), float(std), out.ctypes.data)
    elif dtype == "bf16":
        out = np.empty(n, dtype=np.uint16)
        lib.synth_normal_bf16(seed, stream, offset, n, float(mean), float(std), out.ctypes.data)
    else:
        raise ValueError(dtype)
    return out.reshape(shape)


def to_storage(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round a float array to the storage dtype (f32: float32; bf16: uint16 bit patterns, RNE from float32)."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return a32
    out = np.empty(a32.shape, dtype=np.uint16)
    _load().synth_f32_to_bf16(a32.ctypes.data, a32.size, out.ctypes.data)
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


def as_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to float64 (bf16 and f32 are both exact in double)."""
    return (bf16_bits_to_f32(a) if dtype == "bf16" else a).astype(np.float64)


# Stream ids of the seven layer inputs inside one seed.
STREAM = {"x": 1, "Wg": 2, "bg": 3, "W1": 4, "b1": 5, "W2": 6, "b2": 7}


@dataclass
class LayerConfig:
    """One synthetic MoE layer workload: shapes, storage dtype, seed and value distributions.

    Distribution notation follows the workload statements: ``N(0, 1/H)`` is read as variance 1/H
    (std 1/sqrt(H), the usual fan-in scaling), while the bias spread ``N(0, 0.02)`` is read as std
    0.02 (the usual transformer initialisation scale).  Gate bias is zero unless ``bg_rule`` says
    otherwise.
    """
    name: str
    T: int
    H: int
    E: int
    k: int
    F: int
    CF: float  # math.inf = dropless
    dtype: str  # "f32" or "bf16" storage of x and all weights
    seed: int
    bias_std: float = 0.02
    bg_rule: str = "zero"  # "zero" or "zipf"  (bg[e] = 1.5 * ln(1/(e+1)))
    note: str = ""
    act: str = "gelu"  # expert activation: "gelu" (Quick Start expert) or "silu" (Mixtral block)
    bias: bool = True  # False: gate and experts have no bias at all (bg = b1 = b2 = None)
    routing: str = "token_choice"  # or "expert_choice" (every expert takes its top-C tokens)
    min_capacity: int = 0  # lower bound on the per-expert capacity (0 = none)

    @property
    def x_std(self) -> float:
        return 1.0

    def shape_tuple(self):
        return (self.T, self.H, self.E, self.k, self.F, self.CF)

    def with_(self, **kw) -> "LayerConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return LayerConfig(**d)


CONFIGS = {
    "tiny": LayerConfig("tiny", T=256, H=64, E=4, k=2, F=256, CF=math.inf, dtype="f32", seed=1,
                        note="tiny fp32 layer, dropless"),
    "decode": LayerConfig("decode", T=32, H=4096, E=8, k=2, F=14336, CF=math.inf, dtype="bf16", seed=2,
                          note="decode-sized, weight-streaming-bound"),
    "switch": LayerConfig("switch", T=8192, H=1024, E=128, k=1, F=4096, CF=1.25, dtype="bf16", seed=3,
                          note="Switch-style training shape, capacity factor 1.25"),
    "mixtral": LayerConfig("mixtral", T=4096, H=4096, E=8, k=2, F=14336, CF=math.inf, dtype="bf16", seed=4,
                           note="Mixtral-shaped layer, dropless (headline)"),
    "skew": LayerConfig("skew", T=16384, H=2048, E=64, k=2, F=8192, CF=math.inf, dtype="bf16", seed=5,
                        bg_rule="zipf", note="skewed expert load, dropless"),
    "mixtral_block": LayerConfig("mixtral_block", T=4096, H=4096, E=8, k=2, F=14336, CF=math.inf, dtype="bf16",
                                 seed=6, act="silu", bias=False,
                                 note="the Mixtral block's own expert: bias-free gate and Linear layers, SiLU"),
    "mixtral_ec": LayerConfig("mixtral_ec", T=4096, H=4096, E=8, k=2, F=14336, CF=1.0, dtype="bf16", seed=7,
                              routing="expert_choice",
                              note="expert-choice routing at the Mixtral shape: C = T*k/E = 1024 tokens per expert"),
}


@dataclass
class LayerInputs:
    cfg: LayerConfig
    x: np.ndarray
    Wg: np.ndarray
    bg: np.ndarray | None
    W1: np.ndarray
    b1: np.ndarray | None
    W2: np.ndarray
    b2: np.ndarray | None
    extra: dict = field(default_factory=dict)

    def arrays(self):
        """The inputs that are present (a bias-free layer has no bg / b1 / b2 entries)."""
        d = dict(x=self.x, Wg=self.Wg, bg=self.bg, W1=self.W1, b1=self.b1, W2=self.W2, b2=self.b2)
        return {n: a for n, a in d.items() if a is not None}


def make_bg(cfg: LayerConfig) -> np.ndarray:
    if cfg.bg_rule == "zero":
        return to_storage(np.zeros(cfg.E, dtype=np.float64), cfg.dtype)
    if cfg.bg_rule == "zipf":
        e = np.arange(cfg.E, dtype=np.float64)
        return to_storage(1.5 * np.log(1.0 / (e + 1.0)), cfg.dtype)
    raise ValueError(cfg.bg_rule)


def make_inputs(cfg: LayerConfig, with_weights: bool = True) -> LayerInputs:
    """Generate all seven inputs of a layer workload on the host."""
    s, dt = cfg.seed, cfg.dtype
    T, H, E, F = cfg.T, cfg.H, cfg.E, cfg.F
    x = normal(s, STREAM["x"], (T, H), 0.0, cfg.x_std, dt)
    Wg = normal(s, STREAM["Wg"], (H, E), 0.0, 1.0 / math.sqrt(H), dt)
    bg = make_bg(cfg)
    if with_weights:
        W1 = normal(s, STREAM["W1"], (E, H, F), 0.0, 1.0 / math.sqrt(H), dt)
        W2 = normal(s, STREAM["W2"], (E, F, H), 0.0, 1.0 / math.sqrt(F), dt)
    else:
        W1 = W2 = None
    b1 = normal(s, STREAM["b1"], (E, F), 0.0, cfg.bias_std, dt)
    b2 = normal(s, STREAM["b2"], (E, H), 0.0, cfg.bias_std, dt)
    if not cfg.bias:
        bg = b1 = b2 = None
    return LayerInputs(cfg, x, Wg, bg, W1, b1, W2, b2)


def x_batch(cfg: LayerConfig, step: int) -> np.ndarray:
    """Activations for a later step of a stream of batches (same recipe, disjoint counter range)."""
    n = cfg.T * cfg.H
    return normal(cfg.seed, STREAM["x"], (cfg.T, cfg.H), 0.0, cfg.x_std, cfg.dtype, offset=step * n)

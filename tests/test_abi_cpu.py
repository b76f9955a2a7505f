"""The C-ABI library loads, exports every symbol its header declares, and validates arguments on the
host before touching the GPU (these calls return before any CUDA work, so they run without a GPU)."""
import ctypes
import math
import os
import re

import pytest

import sparse_mixture_experts_23_b200 as moe
from sparse_mixture_experts_23_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = header_symbols()
    for name in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward", "moe_workspace_size"):
        assert name in syms
    assert sorted(moe.ENTRY_POINTS) == syms


def test_library_exports_every_declared_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name


def test_no_torch_types_in_signatures():
    text = open(HEADER).read()
    assert "torch" not in text.lower().replace("pytorch", "") and "at::" not in text and "Tensor" not in text


def _shape(**kw):
    d = dict(T=256, H=64, E=4, k=2, F=256, capacity_factor=math.inf, dtype="f32")
    d.update(kw)
    return moe.make_shape(d["T"], d["H"], d["E"], d["k"], d["F"], d["capacity_factor"], d["dtype"])


FAKE = 1 << 20  # a 256-aligned non-null "device" address; never dereferenced by these calls


def _io(**over):
    io = moe.IO(*([FAKE] * 14))
    for k, v in over.items():
        setattr(io, k, v)
    return io


@pytest.mark.parametrize("bad,code", [
    (dict(T=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(H=0), moe.MOE_ERR_INVALID_ARG),
    (dict(E=0), moe.MOE_ERR_INVALID_ARG),
    (dict(k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(k=5), moe.MOE_ERR_INVALID_ARG),        # k > E
    (dict(E=300, k=2), moe.MOE_ERR_INVALID_ARG),  # E > 256
    (dict(E=16, k=9), moe.MOE_ERR_INVALID_ARG),   # k > 8
    (dict(capacity_factor=0.0), moe.MOE_ERR_INVALID_ARG),
    (dict(capacity_factor=-1.0), moe.MOE_ERR_INVALID_ARG),
    (dict(capacity_factor=float("nan")), moe.MOE_ERR_INVALID_ARG),
    (dict(dtype="bf16", H=96), moe.MOE_ERR_UNSUPPORTED),
    (dict(dtype="bf16", F=100), moe.MOE_ERR_UNSUPPORTED),
    (dict(H=66), moe.MOE_ERR_UNSUPPORTED),
])
def test_shape_validation(lib, bad, code):
    s = _shape(**bad)
    assert moe.moe_workspace_size(s) == 0
    for fn in (moe.moe_route, moe.moe_permute, moe.moe_combine, moe.moe_forward):
        assert fn(s, _io(), FAKE, 1 << 40) == code
    assert moe.moe_expert_ffn(s, _io(), FAKE, 1 << 40, 1) == code


def test_bad_dtype_enum(lib):
    s = _shape()
    s.dtype = 7
    assert moe.moe_forward(s, _io(), FAKE, 1 << 40) == moe.MOE_ERR_INVALID_ARG


def test_activation_field(lib):
    """The activation sits right after dtype, and a zero-initialised shape means GELU; unknown
    activations are rejected before any launch."""
    assert ctypes.sizeof(moe.Shape) == 48 and moe.Shape.activation.offset == 36 and moe.Shape.min_capacity.offset == 44
    assert moe.Shape().activation == moe.MOE_ACT_GELU
    s = _shape()
    assert moe.moe_workspace_size(s) > 0
    s.activation = moe.MOE_ACT_SILU
    assert moe.moe_workspace_size(s) > 0
    s.activation = 2
    assert moe.moe_workspace_size(s) == 0
    for fn in (moe.moe_route, moe.moe_permute, moe.moe_combine, moe.moe_forward):
        assert fn(s, _io(), FAKE, 1 << 40) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_expert_ffn(s, _io(), FAKE, 1 << 40, 1) == moe.MOE_ERR_INVALID_ARG
    text = open(HEADER).read()
    assert "MOE_ACT_GELU = 0" in text and "MOE_ACT_SILU = 1" in text


def test_workspace_errors(lib):
    s = _shape()
    n = moe.moe_workspace_size(s)
    assert n > 0 and n % 256 == 0
    assert moe.moe_forward(s, _io(), FAKE, n - 1) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_forward(s, _io(), None, n) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward(s, _io(), FAKE + 16, n) == moe.MOE_ERR_INVALID_ARG  # not 256-aligned


@pytest.mark.parametrize("field", ["x", "Wg", "W1", "W2", "out", "topk_idx", "topk_w",
                                   "expert_counts", "dropped", "aux_loss", "z_loss"])
def test_null_pointers_rejected(lib, field):
    s = _shape()
    n = moe.moe_workspace_size(s)
    assert moe.moe_forward(s, _io(**{field: None}), FAKE, n) == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("field", ["x", "Wg", "W1", "W2", "out", "b1", "b2"])
def test_misaligned_pointers_rejected(lib, field):
    s = _shape()
    n = moe.moe_workspace_size(s)
    assert moe.moe_forward(s, _io(**{field: FAKE + 4}), FAKE, n) == moe.MOE_ERR_INVALID_ARG


def test_null_shape_and_io(lib):
    s = _shape()
    L = moe.load_library()
    assert L.moe_forward(None, ctypes.byref(_io()), FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward(ctypes.byref(s), None, FAKE, 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_size(None) == 0


def test_workspace_layout_is_pure_and_ordered(lib):
    s = _shape(T=100, H=128, E=8, k=2, F=512, dtype="bf16")
    n = moe.moe_workspace_size(s)
    v = moe.moe_workspace_layout(s, FAKE)
    assert v.bytes == n
    ptrs = [v.status, v.offsets, v.cnt_pre, v.row_of, v.row_token, v.row_slot, v.x_perm, v.h, v.y]
    assert ptrs == sorted(ptrs) and all(p % 256 == 0 for p in ptrs)
    assert v.status == FAKE
    rows = 100 * 2
    assert v.h - v.x_perm >= rows * 128 * 2 and v.y - v.h >= rows * 512 * 2
    assert FAKE + n - v.y >= rows * 128 * 4


def test_status_strings(lib):
    assert moe.status_string(moe.MOE_OK) == "ok"
    assert "workspace" in moe.status_string(moe.MOE_ERR_WORKSPACE)
    assert "timed out" in moe.status_string(moe.MOE_ERR_TIMEOUT)


def test_missing_library_fails_loudly(tmp_path):
    import sparse_mixture_experts_23_b200 as m
    saved = m._lib
    try:
        m._lib = None
        with pytest.raises(RuntimeError, match="not built"):
            m.load_library(str(tmp_path / "nope.so"))
    finally:
        m._lib = saved


def test_routing_field_and_capacity(lib):
    """moe_shape_t.routing follows activation; zero means token choice.  moe_capacity gives the
    per-expert capacity of either rule; unknown rules are rejected before any launch."""
    assert moe.Shape.routing.offset == 40 and moe.Shape().routing == moe.MOE_ROUTING_TOKEN_CHOICE
    s = _shape(T=4096, H=64, E=8, k=2, F=64, capacity_factor=1.0)
    assert moe.moe_capacity(s) == 1024
    s.routing = moe.MOE_ROUTING_EXPERT_CHOICE
    assert moe.moe_capacity(s) == 1024
    s.capacity_factor = math.inf
    assert moe.moe_capacity(s) == 4096  # every expert sees every token
    s.routing = moe.MOE_ROUTING_TOKEN_CHOICE
    assert moe.moe_capacity(s) == -1  # no limit
    s.capacity_factor = 100.0
    s.routing = moe.MOE_ROUTING_EXPERT_CHOICE
    assert moe.moe_capacity(s) == 4096  # never more than T
    s.routing = 2
    assert moe.moe_capacity(s) == -2 and moe.moe_workspace_size(s) == 0
    for fn in (moe.moe_route, moe.moe_permute, moe.moe_combine, moe.moe_forward):
        assert fn(s, _io(), FAKE, 1 << 40) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_route_noalloc(s, _io()) == moe.MOE_ERR_INVALID_ARG


def test_expert_choice_workspace_and_layout(lib):
    """Under expert choice the row buffers hold E*C rows and the workspace gains the [E,T] score
    matrix; the view publishes it (NULL under token choice)."""
    tc = _shape(T=100, H=128, E=8, k=2, F=512, dtype="bf16", capacity_factor=2.0)
    ec = _shape(T=100, H=128, E=8, k=2, F=512, dtype="bf16", capacity_factor=2.0)
    ec.routing = moe.MOE_ROUTING_EXPERT_CHOICE
    C = moe.moe_capacity(ec)
    assert C == 50
    v_tc = moe.moe_workspace_layout(tc, FAKE)
    v_ec = moe.moe_workspace_layout(ec, FAKE)
    assert v_tc.scores is None and v_ec.scores is not None
    assert v_ec.h - v_ec.x_perm >= 8 * C * 128 * 2 and v_ec.y - v_ec.h >= 8 * C * 512 * 2
    assert v_ec.scores - v_ec.y >= 8 * C * 128 * 4
    assert FAKE + v_ec.bytes - v_ec.scores >= 8 * 100 * 4 + 100 * 4
    # the no-workspace router does not take expert choice
    assert moe.moe_route_noalloc(ec, _io()) == moe.MOE_ERR_UNSUPPORTED


def _grad(**over):
    g = moe.Grad(FAKE, 0.0, 0.0, *([FAKE] * 8))
    for k, v in over.items():
        setattr(g, k, v)
    return g


def test_training_entry_points_validate_before_launch(lib):
    """moe_forward_train / moe_backward: a training-sized workspace and bias gradients exactly where the
    layer has biases; every refusal happens before any launch (no call here reaches a kernel)."""
    L = moe.load_library()
    s = _shape(T=64, H=64, E=4, k=2, F=128, dtype="bf16")
    n_inf, n_train = moe.moe_workspace_size(s), moe.moe_train_workspace_size(s)
    assert n_train > n_inf > 0
    assert moe.moe_forward_train(s, _io(), FAKE, n_inf) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_backward(s, _io(), _grad(), FAKE, n_inf) == moe.MOE_ERR_WORKSPACE
    f32 = _shape(T=64, H=64, E=4, k=2, F=128, dtype="f32")  # fp32 is trained too: refused here only for its size
    assert moe.moe_forward_train(f32, _io(), FAKE, 100) == moe.MOE_ERR_WORKSPACE
    ec = _shape(T=64, H=64, E=4, k=2, F=128, dtype="bf16")
    ec.routing = moe.MOE_ROUTING_EXPERT_CHOICE
    assert moe.moe_backward(ec, _io(), _grad(), FAKE, 100) == moe.MOE_ERR_WORKSPACE  # expert choice is trained too
    # bias gradient present without the bias, or missing with it
    assert moe.moe_backward(s, _io(bg=None), _grad(), FAKE, n_train) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_backward(s, _io(), _grad(db1=None), FAKE, n_train) == moe.MOE_ERR_INVALID_ARG
    for f in ("dout", "dx", "dWg", "dW1", "dW2"):
        assert moe.moe_backward(s, _io(), _grad(**{f: None}), FAKE, n_train) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_backward(ctypes.byref(s), ctypes.byref(_io()), None, FAKE, n_train, None) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_train_workspace_size(_shape(T=-1)) == 0


def test_min_capacity_field(lib):
    s = _shape(T=40, H=64, E=4, k=1, F=64, capacity_factor=0.25)
    assert moe.moe_capacity(s) == 3
    s.min_capacity = 4
    assert moe.moe_capacity(s) == 4
    s.routing = moe.MOE_ROUTING_EXPERT_CHOICE
    assert moe.moe_capacity(s) == 4
    s.min_capacity = 100
    assert moe.moe_capacity(s) == 40  # expert choice never takes more than T
    s.min_capacity = -1
    assert moe.moe_capacity(s) == -2 and moe.moe_workspace_size(s) == 0
    assert moe.moe_forward(s, _io(), FAKE, 1 << 40) == moe.MOE_ERR_INVALID_ARG
    # the no-workspace router applies the same shape rules as moe_route, and launches nothing
    s.routing = moe.MOE_ROUTING_TOKEN_CHOICE
    assert moe.moe_route(s, _io(), FAKE, 1 << 40) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_route_noalloc(s, _io()) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_last_launch_count() == 0


def test_debug_activation_validates_before_launch(lib):
    """moe_debug_activation refuses an unknown activation, a negative count and null buffers without
    launching, and does nothing for n = 0."""
    assert moe.moe_debug_activation(7, FAKE, FAKE, 4) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_debug_activation(moe.MOE_ACT_GELU, FAKE, FAKE, -1) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_debug_activation(moe.MOE_ACT_SILU, None, FAKE, 4) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_debug_activation(moe.MOE_ACT_GELU, FAKE, None, 4) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_last_launch_count() == 0
    assert moe.moe_debug_activation(moe.MOE_ACT_GELU, None, None, 0) == moe.MOE_OK
    assert moe.moe_last_launch_count() == 0


def test_kernel_options_round_trip(lib):
    """moe_set_kernel_options keeps the known flags, drops unknown bits, and 0 restores the default."""
    assert moe.moe_get_kernel_options() == moe.MOE_KERNEL_DEFAULT
    try:
        known = moe.MOE_KERNEL_NO_CTA_PAIR | moe.MOE_KERNEL_NO_TC_GATE | moe.MOE_KERNEL_NO_TMA_ROUTER
        moe.moe_set_kernel_options(known | 0x40)
        assert moe.moe_get_kernel_options() == known
    finally:
        moe.moe_set_kernel_options(moe.MOE_KERNEL_DEFAULT)
    assert moe.moe_get_kernel_options() == 0


def test_loss_sum_entry_points_validate_before_launch(lib):
    s = _shape()
    need = moe.moe_workspace_size(s)
    E = s.E
    # moe_loss_sums: null or misaligned sums, missing or short workspace, bad shape
    assert moe.moe_loss_sums(s, FAKE, need, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_loss_sums(s, FAKE, need, FAKE + 2) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_loss_sums(s, 0, need, FAKE) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_loss_sums(s, FAKE, need - 1, FAKE) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_loss_sums(_shape(k=5), FAKE, need, FAKE) == moe.MOE_ERR_INVALID_ARG
    # moe_losses_from_sums: expert count outside [1, 256], null pointers
    for bad_e in (0, -1, 257):
        assert moe.moe_losses_from_sums(bad_e, FAKE, FAKE, FAKE) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_losses_from_sums(E, 0, FAKE, FAKE) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_losses_from_sums(E, FAKE, 0, FAKE) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_losses_from_sums(E, FAKE, FAKE, 0) == moe.MOE_ERR_INVALID_ARG
    assert moe.loss_sums_size(E) == 2 * E + 2

"""Python binding of the B200 sparse top-k MoE layer library (``libmoe.so``, C ABI in include/moe.h):
the forward pass, the backward pass and the losses across data-parallel replicas.

This module only marshals arguments: it mirrors the C structs with ctypes and calls the entry
points by the same names.  Every step of the layer runs in the CUDA kernels of ``libmoe.so``;
there is no Python or CPU fallback, and loading fails loudly when the library is missing.
PyTorch is used by ``MoEBuffers`` only to allocate device memory and to hand over its stream.
"""
from __future__ import annotations

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(6)
MOE_DTYPE_F32, MOE_DTYPE_BF16 = 0, 1
DTYPES = {"f32": MOE_DTYPE_F32, "bf16": MOE_DTYPE_BF16}
MOE_ACT_GELU, MOE_ACT_SILU = 0, 1
ACTIVATIONS = {"gelu": MOE_ACT_GELU, "silu": MOE_ACT_SILU}
MOE_ROUTING_TOKEN_CHOICE, MOE_ROUTING_EXPERT_CHOICE = 0, 1
ROUTINGS = {"token_choice": MOE_ROUTING_TOKEN_CHOICE, "expert_choice": MOE_ROUTING_EXPERT_CHOICE}

ENTRY_POINTS = (
    "moe_workspace_size", "moe_workspace_layout", "moe_route", "moe_permute", "moe_expert_ffn", "moe_combine",
    "moe_forward", "moe_forward_host", "moe_get_device_status", "moe_set_wait_limit", "moe_debug_timeout_probe",
    "moe_last_launch_count", "moe_status_string", "moe_route_noalloc", "moe_capacity",
    "moe_train_workspace_size", "moe_forward_train", "moe_backward", "moe_loss_sums", "moe_losses_from_sums",
    "moe_set_kernel_options", "moe_get_kernel_options", "moe_copy_row_segments", "moe_expert_ffn_rows",
    "moe_expert_ffn_rows_workspace_size", "moe_debug_activation",
)
MOE_KERNEL_DEFAULT, MOE_KERNEL_NO_CTA_PAIR, MOE_KERNEL_NO_TC_GATE, MOE_KERNEL_NO_TMA_ROUTER = 0, 1, 2, 4


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32), ("F", ctypes.c_int32),
                ("k", ctypes.c_int32), ("capacity_factor", ctypes.c_double), ("dtype", ctypes.c_int),
                ("activation", ctypes.c_int), ("routing", ctypes.c_int), ("min_capacity", ctypes.c_int32)]


class IO(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("x", "Wg", "bg", "W1", "b1", "W2", "b2", "out", "topk_idx", "topk_w",
                                               "expert_counts", "dropped", "aux_loss", "z_loss")]


class Grad(ctypes.Structure):
    _fields_ = [("dout", ctypes.c_void_p), ("d_aux", ctypes.c_float), ("d_z", ctypes.c_float)] + [
        (n, ctypes.c_void_p) for n in ("dx", "dWg", "dbg", "dW1", "db1", "dW2", "db2", "dw")]


class WsView(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("status", "offsets", "cnt_pre", "row_of", "row_token", "row_slot",
                                               "x_perm", "h", "y")] + [("bytes", ctypes.c_size_t),
                                                                        ("scores", ctypes.c_void_p)]


class RowSegment(ctypes.Structure):
    """moe_row_segment_t: `rows` rows from device pointer src to device pointer dst."""
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("rows", ctypes.c_int64)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load ``libmoe.so``; raises if it has not been built (run ``sparse_mixture_experts_23_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing (python -m sparse_mixture_experts_23_b200.build)")
    lib = ctypes.CDLL(path)
    P, vp, sz, st = ctypes.POINTER, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    lib.moe_workspace_size.argtypes = [P(Shape)]
    lib.moe_workspace_size.restype = sz
    lib.moe_capacity.argtypes = [P(Shape)]
    lib.moe_capacity.restype = ctypes.c_int64
    lib.moe_workspace_layout.argtypes = [P(Shape), vp, P(WsView)]
    lib.moe_workspace_layout.restype = st
    for name in ("moe_route", "moe_permute", "moe_combine", "moe_forward"):
        fn = getattr(lib, name)
        fn.argtypes = [P(Shape), P(IO), vp, sz, vp]
        fn.restype = st
    lib.moe_route_noalloc.argtypes = [P(Shape), P(IO), vp]
    lib.moe_route_noalloc.restype = st
    lib.moe_expert_ffn.argtypes = [P(Shape), P(IO), vp, sz, ctypes.c_int, vp]
    lib.moe_expert_ffn.restype = st
    lib.moe_forward_host.argtypes = [P(Shape), P(IO), vp, vp, vp, sz, vp]
    lib.moe_train_workspace_size.argtypes = [P(Shape)]
    lib.moe_train_workspace_size.restype = sz
    lib.moe_forward_train.argtypes = [P(Shape), P(IO), vp, sz, vp]
    lib.moe_forward_train.restype = st
    lib.moe_backward.argtypes = [P(Shape), P(IO), P(Grad), vp, sz, vp]
    lib.moe_backward.restype = st
    lib.moe_forward_host.restype = st
    lib.moe_loss_sums.argtypes = [P(Shape), vp, sz, vp, vp]
    lib.moe_loss_sums.restype = st
    lib.moe_losses_from_sums.argtypes = [ctypes.c_int, vp, vp, vp, vp]
    lib.moe_losses_from_sums.restype = st
    lib.moe_get_device_status.argtypes = [vp, vp]
    lib.moe_get_device_status.restype = st
    lib.moe_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.moe_set_wait_limit.restype = None
    lib.moe_set_kernel_options.argtypes = [ctypes.c_int]
    lib.moe_set_kernel_options.restype = None
    lib.moe_get_kernel_options.argtypes = []
    lib.moe_get_kernel_options.restype = ctypes.c_int
    lib.moe_copy_row_segments.argtypes = [vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, vp, vp]
    lib.moe_copy_row_segments.restype = st
    lib.moe_expert_ffn_rows_workspace_size.argtypes = [P(Shape), ctypes.c_int64]
    lib.moe_expert_ffn_rows_workspace_size.restype = sz
    lib.moe_expert_ffn_rows.argtypes = [P(Shape), ctypes.c_int64, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_expert_ffn_rows.restype = st
    lib.moe_debug_activation.argtypes = [ctypes.c_int, vp, vp, ctypes.c_int64, vp]
    lib.moe_debug_activation.restype = st
    lib.moe_debug_timeout_probe.argtypes = [vp, sz, vp]
    lib.moe_debug_timeout_probe.restype = st
    lib.moe_last_launch_count.argtypes = []
    lib.moe_last_launch_count.restype = ctypes.c_int
    lib.moe_status_string.argtypes = [st]
    lib.moe_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().moe_status_string(status).decode()


def make_shape(T: int, H: int, E: int, k: int, F: int, capacity_factor: float = math.inf, dtype: str = "bf16",
               activation: str = "gelu", routing: str = "token_choice", min_capacity: int = 0) -> Shape:
    return Shape(T, H, E, F, k, float(capacity_factor), DTYPES[dtype], ACTIVATIONS[activation], ROUTINGS[routing],
                 int(min_capacity))


def moe_capacity(shape: Shape) -> int:
    return load_library().moe_capacity(ctypes.byref(shape))


def _check(status: int, where: str) -> int:
    if status != MOE_OK:
        raise MoEError(status, where)
    return status


# ---- thin wrappers, same names as the C ABI; pointers are ints, streams are cudaStream_t ints ----

def moe_workspace_size(shape: Shape) -> int:
    return load_library().moe_workspace_size(ctypes.byref(shape))


def moe_workspace_layout(shape: Shape, ws: int) -> WsView:
    v = WsView()
    _check(load_library().moe_workspace_layout(ctypes.byref(shape), ws, ctypes.byref(v)), "moe_workspace_layout")
    return v


def moe_route(shape, io, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_route(ctypes.byref(shape), ctypes.byref(io), ws, ws_bytes, stream)


def moe_route_noalloc(shape, io, stream=0) -> int:
    return load_library().moe_route_noalloc(ctypes.byref(shape), ctypes.byref(io), stream)


def moe_permute(shape, io, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_permute(ctypes.byref(shape), ctypes.byref(io), ws, ws_bytes, stream)


def moe_expert_ffn(shape, io, ws, ws_bytes, fuse_combine=1, stream=0) -> int:
    return load_library().moe_expert_ffn(ctypes.byref(shape), ctypes.byref(io), ws, ws_bytes, int(fuse_combine), stream)


def moe_combine(shape, io, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_combine(ctypes.byref(shape), ctypes.byref(io), ws, ws_bytes, stream)


def moe_forward(shape, io, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_forward(ctypes.byref(shape), ctypes.byref(io), ws, ws_bytes, stream)


def moe_train_workspace_size(shape: Shape) -> int:
    return load_library().moe_train_workspace_size(ctypes.byref(shape))


def moe_forward_train(shape, io, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_forward_train(ctypes.byref(shape), ctypes.byref(io), ws, ws_bytes, stream)


def moe_backward(shape, io, grad, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_backward(ctypes.byref(shape), ctypes.byref(io), ctypes.byref(grad), ws, ws_bytes, stream)


def moe_forward_host(shape, io, x_host, out_host, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_forward_host(ctypes.byref(shape), ctypes.byref(io), x_host, out_host, ws, ws_bytes,
                                           stream)


def moe_loss_sums(shape, ws, ws_bytes, sums, stream=0) -> int:
    return load_library().moe_loss_sums(ctypes.byref(shape), ws, ws_bytes, sums, stream)


def moe_losses_from_sums(E, sums, aux_loss, z_loss, stream=0) -> int:
    return load_library().moe_losses_from_sums(int(E), sums, aux_loss, z_loss, stream)


def loss_sums_size(E: int) -> int:
    """Length of the loss-sum vector: [cnt_e (E)][Psum_e (E)][Zsum][T]."""
    return 2 * E + 2


def allreduce_sums(sums, group=None):
    """Element-wise total of every replica's loss sums (in place) over the torch.distributed process
    group, when one is initialised; a single process keeps its own.  Host plumbing only: the sums
    and the losses are computed by moe_loss_sums / moe_losses_from_sums."""
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
    return sums


def losses_from_sums(E: int, sums):
    """[aux_loss, z_loss] (fp32 CUDA tensor) from a CUDA tensor of 2E+2 loss sums."""
    import torch

    out = torch.empty((2,), dtype=torch.float32, device=sums.device)
    _check(moe_losses_from_sums(E, sums.data_ptr(), out.data_ptr(), out.data_ptr() + 4,
                                torch.cuda.current_stream().cuda_stream), "moe_losses_from_sums")
    return out


def moe_get_device_status(ws, stream=0) -> int:
    return load_library().moe_get_device_status(ws, stream)


def moe_set_wait_limit(cycles: int) -> None:
    load_library().moe_set_wait_limit(int(cycles))


def moe_set_kernel_options(flags: int) -> None:
    load_library().moe_set_kernel_options(int(flags))


def moe_get_kernel_options() -> int:
    return load_library().moe_get_kernel_options()


def moe_copy_row_segments(segs, nsegs: int, row_bytes: int, max_rows: int, status=None, stream=0) -> int:
    """segs: device address of a moe_row_segment_t array (see RowSegment)."""
    return load_library().moe_copy_row_segments(segs, nsegs, row_bytes, max_rows, status, stream)


def moe_expert_ffn_rows_workspace_size(shape, rows_cap: int) -> int:
    return load_library().moe_expert_ffn_rows_workspace_size(ctypes.byref(shape), rows_cap)


def moe_expert_ffn_rows(shape, rows_cap, offsets, x_rows, W1, b1, W2, b2, y, ws, ws_bytes, stream=0) -> int:
    return load_library().moe_expert_ffn_rows(ctypes.byref(shape), rows_cap, offsets, x_rows, W1, b1, W2, b2, y, ws,
                                              ws_bytes, stream)


def moe_debug_activation(activation: int, u, out, n: int, stream=0) -> int:
    return load_library().moe_debug_activation(int(activation), u, out, int(n), stream)


def moe_debug_timeout_probe(ws, ws_bytes, stream=0) -> int:
    return load_library().moe_debug_timeout_probe(ws, ws_bytes, stream)


def moe_last_launch_count() -> int:
    return load_library().moe_last_launch_count()


class MoEBuffers:
    """Device buffers of one layer invocation, allocated with PyTorch (plumbing only).

    ``inputs`` maps x, Wg, bg, W1, b1, W2, b2 to device tensors of the storage dtype (bf16 as
    torch.bfloat16, f32 as torch.float32); a bias that is missing or None is passed as NULL (no
    bias).  Outputs and the workspace are allocated here.
    """

    def __init__(self, shape: Shape, inputs: dict, device="cuda", train: bool = False):
        import torch

        self.shape = shape
        T, H, E, k = shape.T, shape.H, shape.E, shape.k
        self.inputs = inputs
        self.out = torch.empty((T, H), dtype=torch.float32, device=device)
        if shape.routing == MOE_ROUTING_EXPERT_CHOICE:
            # expert choice: chosen tokens [E, C], softmax over all experts [T, E], per-token flags [T]
            C = moe_capacity(shape)
            if C < 0:
                raise MoEError(MOE_ERR_INVALID_ARG, "moe_capacity")
            idx_shape, w_shape, drop_shape = (E, C), (T, E), (T,)
        else:
            idx_shape, w_shape, drop_shape = (T, k), (T, k), (T, k)
        self.topk_idx = torch.empty(idx_shape, dtype=torch.int32, device=device)
        self.topk_w = torch.empty(w_shape, dtype=torch.float32, device=device)
        self.expert_counts = torch.empty((E,), dtype=torch.int32, device=device)
        self.dropped = torch.empty(drop_shape, dtype=torch.uint8, device=device)
        self.losses = torch.empty((2,), dtype=torch.float32, device=device)
        self.ws_bytes = moe_train_workspace_size(shape) if train else moe_workspace_size(shape)
        if self.ws_bytes == 0:
            raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
        self.ws = torch.empty((self.ws_bytes,), dtype=torch.uint8, device=device)
        self.ws[:256].zero_()  # the device error word starts cleared
        self.io = self.make_io()

    def make_io(self) -> IO:
        p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        i = self.inputs
        return IO(p(i.get("x")), p(i.get("Wg")), p(i.get("bg")), p(i.get("W1")), p(i.get("b1")), p(i.get("W2")),
                  p(i.get("b2")), p(self.out), p(self.topk_idx), p(self.topk_w), p(self.expert_counts),
                  p(self.dropped), self.losses.data_ptr(), self.losses.data_ptr() + 4)

    def set_input(self, name: str, tensor) -> None:
        self.inputs[name] = tensor
        self.io = self.make_io()

    @property
    def ws_ptr(self) -> int:
        return self.ws.data_ptr()

    def view(self) -> WsView:
        return moe_workspace_layout(self.shape, self.ws_ptr)

    @staticmethod
    def stream() -> int:
        import torch

        return torch.cuda.current_stream().cuda_stream

    def route(self):
        return _check(moe_route(self.shape, self.io, self.ws_ptr, self.ws_bytes, self.stream()), "moe_route")

    def permute(self):
        return _check(moe_permute(self.shape, self.io, self.ws_ptr, self.ws_bytes, self.stream()), "moe_permute")

    def expert_ffn(self, fuse_combine=True):
        return _check(moe_expert_ffn(self.shape, self.io, self.ws_ptr, self.ws_bytes, int(fuse_combine), self.stream()),
                      "moe_expert_ffn")

    def combine(self):
        return _check(moe_combine(self.shape, self.io, self.ws_ptr, self.ws_bytes, self.stream()), "moe_combine")

    def forward(self):
        return _check(moe_forward(self.shape, self.io, self.ws_ptr, self.ws_bytes, self.stream()), "moe_forward")

    def forward_host(self, x_host, out_host):
        """x_host / out_host: pinned CPU tensors (storage dtype / float32)."""
        return _check(moe_forward_host(self.shape, self.io, x_host.data_ptr(), out_host.data_ptr(), self.ws_ptr,
                                       self.ws_bytes, self.stream()), "moe_forward_host")

    def device_status(self) -> int:
        return moe_get_device_status(self.ws_ptr, self.stream())

    def loss_sums(self):
        """The 2E+2 additive loss sums of the last routed batch (fp32 CUDA tensor)."""
        import torch

        sums = torch.empty((loss_sums_size(self.shape.E),), dtype=torch.float32, device=self.out.device)
        _check(moe_loss_sums(self.shape, self.ws_ptr, self.ws_bytes, sums.data_ptr(), self.stream()), "moe_loss_sums")
        return sums

    def global_losses(self, group=None):
        """[aux_loss, z_loss] of the whole batch across data-parallel replicas: every rank's loss sums
        all-reduced over `group`, then the losses from the totals.  Call on every rank after the
        forward pass, in the same order (it is a collective)."""
        return losses_from_sums(self.shape.E, allreduce_sums(self.loss_sums(), group))

    # ---- training (buffers built with train=True) ----
    def forward_train(self):
        return _check(moe_forward_train(self.shape, self.io, self.ws_ptr, self.ws_bytes, self.stream()),
                      "moe_forward_train")

    def make_grads(self, with_dw: bool = True) -> dict:
        """fp32 gradient buffers for every input the layer has (bias gradients only where the bias exists)."""
        import torch

        s, dev = self.shape, self.out.device
        T, H, E, F, k = s.T, s.H, s.E, s.F, s.k
        g = {"dx": torch.empty((T, H), dtype=torch.float32, device=dev),
             "dWg": torch.empty((H, E), dtype=torch.float32, device=dev),
             "dW1": torch.empty((E, H, F), dtype=torch.float32, device=dev),
             "dW2": torch.empty((E, F, H), dtype=torch.float32, device=dev)}
        if self.inputs.get("bg") is not None:
            g["dbg"] = torch.empty((E,), dtype=torch.float32, device=dev)
        if self.inputs.get("b1") is not None:
            g["db1"] = torch.empty((E, F), dtype=torch.float32, device=dev)
        if self.inputs.get("b2") is not None:
            g["db2"] = torch.empty((E, H), dtype=torch.float32, device=dev)
        if with_dw:
            ec = s.routing == MOE_ROUTING_EXPERT_CHOICE
            g["dw"] = torch.empty((T, E if ec else k), dtype=torch.float32, device=dev)
        return g

    def backward(self, dout, grads: dict, d_aux: float = 0.0, d_z: float = 0.0):
        p = lambda n: None if grads.get(n) is None else grads[n].data_ptr()  # noqa: E731
        g = Grad(dout.data_ptr(), float(d_aux), float(d_z), p("dx"), p("dWg"), p("dbg"), p("dW1"), p("db1"), p("dW2"),
                 p("db2"), p("dw"))
        return _check(moe_backward(self.shape, self.io, g, self.ws_ptr, self.ws_bytes, self.stream()), "moe_backward")

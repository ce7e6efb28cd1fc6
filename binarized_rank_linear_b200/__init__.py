"""LittleBit factored linear layer on NVIDIA B200: Python binding of ``liblb.so``.

The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
method actually computes", Proposition 1) is
``y = h (.) (sign(U) (l (.) (sign(V)^T (g (.) x))))`` per path, with an optional
residual path added on top.  Every step runs in the library's CUDA kernels;
this module only marshals arguments through the C ABI declared in
``include/lb.h``.  PyTorch provides device memory and streams.  There is no
CPU fallback: if ``liblb.so`` is missing or the device is not an sm_100 part,
the calls raise.

Build the library with ``python -m binarized_rank_linear_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblb.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lb.h")

# lb_status
LB_OK = 0
LB_ERR_INVALID_ARGUMENT = 1
LB_ERR_UNSUPPORTED_SHAPE = 2
LB_ERR_MISALIGNED = 3
LB_ERR_CUDA = 4
LB_ERR_DEVICE_TIMEOUT = 5
LB_ERR_NOT_SUPPORTED_DEVICE = 6
LB_ERR_WORKSPACE_TOO_SMALL = 7
LB_ERR_RANGE = 8
# lb_dtype
LB_F32, LB_F16, LB_BF16, LB_I8 = 0, 1, 2, 3
# lb_factor
LB_FACTOR_U, LB_FACTOR_V = 0, 1


class LbPath(ctypes.Structure):
    """``lb_path`` of include/lb.h."""
    _fields_ = [
        ("u_bits", ctypes.c_void_p),
        ("vt_bits", ctypes.c_void_p),
        ("h", ctypes.c_void_p),
        ("g", ctypes.c_void_p),
        ("l", ctypes.c_void_p),
        ("rank", ctypes.c_int64),
        ("u_ld", ctypes.c_int64),
        ("vt_ld", ctypes.c_int64),
    ]


class LbError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}" if what else status_string(status))


_lock = threading.Lock()
_lib = None


class LbProjection(ctypes.Structure):
    """``lb_projection`` (include/lb.h): one layer of a group that shares x."""
    _fields_ = [("n_out", ctypes.c_int64), ("main", ctypes.POINTER(LbPath)), ("residual", ctypes.POINTER(LbPath)),
                ("y", ctypes.c_void_p), ("ldy", ctypes.c_int64)]


MAX_SIBLINGS = 4


def lib() -> ctypes.CDLL:
    """Load ``liblb.so`` (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m binarized_rank_linear_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            i64, vp, sz, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
            L.lb_status_string.restype = ctypes.c_char_p
            L.lb_status_string.argtypes = [i32]
            L.lb_packed_ld_words.restype = i64
            L.lb_packed_ld_words.argtypes = [i64]
            L.lb_packed_bytes.restype = sz
            L.lb_packed_bytes.argtypes = [i32, i64, i64]
            L.lb_rank_for_budget.restype = i32
            L.lb_rank_for_budget.argtypes = [i64, i64, i64, i64, i32, i32, ctypes.POINTER(i64)]
            L.lb_pack_signs.restype = i32
            L.lb_pack_signs.argtypes = [vp, i32, i32, i64, i64, i64, vp, i64, vp]
            L.lb_forward_workspace_bytes.restype = sz
            L.lb_forward_workspace_bytes.argtypes = [i64, i64, i64, i64, i64]
            L.lb_linear_forward.restype = i32
            L.lb_linear_forward.argtypes = [vp, i64, i64, i64, i64, ctypes.POINTER(LbPath),
                                            ctypes.POINTER(LbPath), vp, i64, vp, sz, vp]
            L.lb_latent_forward.restype = i32
            L.lb_latent_forward.argtypes = [vp, i64, i64, i64, ctypes.POINTER(LbPath), ctypes.POINTER(LbPath),
                                            vp, i64, vp]
            L.lb_expand_forward.restype = i32
            L.lb_expand_forward.argtypes = [vp, i64, i64, i64, ctypes.POINTER(LbPath), ctypes.POINTER(LbPath),
                                            vp, i64, vp]
            L.lb_linear_forward_fixed_scratch.restype = i32
            L.lb_linear_forward_fixed_scratch.argtypes = [vp, i64, i64, i64, i64, ctypes.POINTER(LbPath),
                                                          ctypes.POINTER(LbPath), vp, i64, vp]
            L.lb_siblings_workspace_bytes.restype = sz
            L.lb_siblings_workspace_bytes.argtypes = [i64, i64, i32, ctypes.POINTER(LbProjection)]
            L.lb_linear_forward_siblings.restype = i32
            L.lb_linear_forward_siblings.argtypes = [vp, i64, i64, i64, i32, ctypes.POINTER(LbProjection), vp, sz, vp]
            L.lb_linear_forward_host.restype = i32
            L.lb_linear_forward_host.argtypes = [vp, i64, i64, i64, ctypes.POINTER(LbPath), ctypes.POINTER(LbPath),
                                                 vp, vp, vp, vp, sz, vp]
            L.lb_backward_workspace_bytes.restype = sz
            L.lb_backward_workspace_bytes.argtypes = [i64, i64, i64, i64, i64]
            L.lb_linear_backward.restype = i32
            L.lb_linear_backward.argtypes = [vp, vp, i64, i64, i64, i64, i64, ctypes.POINTER(LbPath),
                                             ctypes.POINTER(LbPath), vp, i64, vp, vp, vp, vp, sz, vp]
            L.lb_device_status.restype = i32
            L.lb_device_status.argtypes = [vp, ctypes.POINTER(i32)]
            L.lb_debug_inject_stall.restype = i32
            L.lb_debug_inject_stall.argtypes = [i32, ctypes.c_uint64]
            L.lb_set_prefill_pairs.restype = i32
            L.lb_set_prefill_pairs.argtypes = [i32]
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().lb_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != LB_OK:
        raise LbError(status, what)


# ------------------------------------------------------------------ host-only queries

def packed_ld_words(cols: int) -> int:
    return int(lib().lb_packed_ld_words(cols))


def packed_bytes(kind: int, n_in_or_out: int, rank: int) -> int:
    return int(lib().lb_packed_bytes(kind, n_in_or_out, rank))


def rank_for_budget(n_in: int, n_out: int, eff_num: int, eff_den: int, paths: int = 1,
                    align: int = 32) -> int:
    r = ctypes.c_int64(0)
    _check(lib().lb_rank_for_budget(n_in, n_out, eff_num, eff_den, paths, align, ctypes.byref(r)),
           "lb_rank_for_budget")
    return int(r.value)


def forward_workspace_bytes(tokens: int, n_in: int, n_out: int, rank_main: int,
                            rank_residual: int = 0) -> int:
    return int(lib().lb_forward_workspace_bytes(tokens, n_in, n_out, rank_main, rank_residual))


# ------------------------------------------------------------------ device calls

def _torch():
    import torch
    return torch


def _stream_handle(stream) -> ctypes.c_void_p:
    torch = _torch()
    if stream is None:
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:  # the current stream of the current device, without a Stream object
            return ctypes.c_void_p(raw(torch.cuda.current_device()))
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t) -> int:
    torch = _torch()
    codes = {torch.float32: LB_F32, torch.float16: LB_F16, torch.bfloat16: LB_BF16, torch.int8: LB_I8}
    if t.dtype not in codes:
        raise TypeError(f"unsupported factor dtype {t.dtype}")
    return codes[t.dtype]


def _require(t, name: str, dtype, device: str = "cuda", contiguous: bool = False) -> None:
    """Checks an activation tensor before its pointer crosses the C ABI: the
    library reads the bits as the element type and layout its header states,
    so a tensor of another dtype or with a non-unit inner stride would be read
    as wrong data without an error."""
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    if t.stride(1) != 1 and t.shape[1] > 1:
        raise ValueError(f"{name} must have unit inner stride, got strides {t.stride()}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (rows of exactly {t.shape[1]} elements)")
    if (device == "cuda") != bool(t.is_cuda):
        raise ValueError(f"{name} must be in {'device' if device == 'cuda' else 'host'} memory")


def _require_workspace(ws) -> None:
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous device tensor")


def pack_signs(src, kind: str, ld_words: int | None = None, stream=None):
    """Pack a device factor (f32 / f16 / bf16 / int8, 2-D, unit column stride)
    with ``lb_pack_signs``.  ``kind`` is ``"U"`` (src = U [n_out, r]) or
    ``"V"`` (src = V [n_in, r], packed as V^T).  Returns an int32 tensor of
    packed words (bit patterns)."""
    torch = _torch()
    if src.dim() != 2 or src.stride(1) != 1 or not src.is_cuda:
        raise ValueError("src must be a 2-D CUDA tensor with unit column stride")
    rows, cols = src.shape
    packed_rows, packed_cols = (rows, cols) if kind == "U" else (cols, rows)
    ld = packed_ld_words(packed_cols) if ld_words is None else int(ld_words)
    dst = torch.empty((packed_rows, ld), dtype=torch.int32, device=src.device)
    code = LB_FACTOR_U if kind == "U" else LB_FACTOR_V
    _check(lib().lb_pack_signs(src.data_ptr(), _dtype_code(src), code, rows, cols, src.stride(0),
                               dst.data_ptr(), ld, _stream_handle(stream)), "lb_pack_signs")
    return dst


@dataclass(frozen=True)
class PackedPath:
    """One binarized path on the device: packed sign(U) [n_out, u_ld] and
    sign(V)^T [rank, vt_ld] (int32 words) and fp16 scales h [n_out], g [n_in],
    l [rank]."""
    u_bits: object
    vt_bits: object
    h: object
    g: object
    l: object
    rank: int

    @classmethod
    def from_factors(cls, su, sv, h, g, l, stream=None) -> "PackedPath":
        """Pack U [n_out, r] and V [n_in, r] (any supported dtype, on the
        device) and keep the fp16 scales."""
        torch = _torch()
        f16 = lambda t: t.to(device=su.device, dtype=torch.float16).contiguous()
        return cls(pack_signs(su, "U", stream=stream), pack_signs(sv, "V", stream=stream),
                   f16(h), f16(g), f16(l), int(su.shape[1]))

    def as_c(self) -> LbPath:
        """The lb_path struct of this path, built once (the fields are frozen
        and a tensor's storage does not move)."""
        c = self.__dict__.get("_c")
        if c is None:
            torch = _torch()
            for name in ("u_bits", "vt_bits"):
                t = getattr(self, name)
                if t.dtype != torch.int32 or t.dim() != 2 or t.stride(1) != 1 or not t.is_cuda:
                    raise ValueError(f"{name} must be a 2-D int32 device tensor of packed words with unit "
                                     f"inner stride")
            for name in ("h", "g", "l"):
                t = getattr(self, name)
                if t.dtype != torch.float16 or t.dim() != 1 or not t.is_contiguous() or not t.is_cuda:
                    raise ValueError(f"{name} must be a contiguous 1-D float16 device tensor")
            c = LbPath(self.u_bits.data_ptr(), self.vt_bits.data_ptr(), self.h.data_ptr(),
                       self.g.data_ptr(), self.l.data_ptr(), self.rank, self.u_bits.shape[1],
                       self.vt_bits.shape[1])
            object.__setattr__(self, "_c", c)
        return c


def linear_forward(x, main: PackedPath, residual: PackedPath | None = None, y=None,
                   workspace=None, stream=None):
    """``lb_linear_forward``: x bf16 [tokens, n_in] (row stride a multiple of 8)
    -> y bf16 [tokens, n_out].  Allocates y and the workspace with torch when
    not given."""
    torch = _torch()
    _require(x, "x", torch.bfloat16)
    tokens, n_in = x.shape
    n_out = main.h.shape[0]
    if y is None:
        y = torch.empty((tokens, n_out), dtype=torch.bfloat16, device=x.device)
    _require(y, "y", torch.bfloat16)
    if workspace is None:  # a caller's workspace size is checked by the library itself
        need = forward_workspace_bytes(tokens, n_in, n_out, main.rank, residual.rank if residual else 0)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    _require_workspace(workspace)
    cm = main.as_c()
    cr = residual.as_c() if residual is not None else None
    _check(lib().lb_linear_forward(
        x.data_ptr(), tokens, n_in, n_out, x.stride(0), ctypes.byref(cm),
        ctypes.byref(cr) if cr is not None else None, y.data_ptr(), y.stride(0),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream)),
        "lb_linear_forward")
    return y


def _projections(layers, ys):
    """ctypes array of lb_projection for [(main, residual or None), ...] and
    their outputs; the LbPath structs are returned too, to keep them alive."""
    keep = []
    arr = (LbProjection * len(layers))()
    for j, ((main, residual), y) in enumerate(zip(layers, ys)):
        cm = main.as_c()
        cr = residual.as_c() if residual is not None else None
        keep += [cm, cr]
        arr[j].n_out = main.h.shape[0]
        arr[j].main = ctypes.pointer(cm)
        arr[j].residual = ctypes.pointer(cr) if cr is not None else None
        arr[j].y = y.data_ptr() if y is not None else None
        arr[j].ldy = y.stride(0) if y is not None else main.h.shape[0]
    return arr, keep


def siblings_workspace_bytes(tokens: int, n_in: int, layers) -> int:
    arr, _keep = _projections(layers, [None] * len(layers))
    return int(lib().lb_siblings_workspace_bytes(tokens, n_in, len(layers), arr))


def linear_forward_siblings(x, layers, ys=None, workspace=None, stream=None):
    """``lb_linear_forward_siblings``: several layers that read the same x,
    given as [(main, residual or None), ...]; returns their outputs (bf16
    [tokens, n_out_j]), allocated with torch when not given."""
    torch = _torch()
    _require(x, "x", torch.bfloat16)
    tokens, n_in = x.shape
    if ys is None:
        ys = [torch.empty((tokens, main.h.shape[0]), dtype=torch.bfloat16, device=x.device) for main, _ in layers]
    for j, y in enumerate(ys):
        _require(y, f"ys[{j}]", torch.bfloat16)
    arr, _keep = _projections(layers, ys)
    need = int(lib().lb_siblings_workspace_bytes(tokens, n_in, len(layers), arr))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    _require_workspace(workspace)
    _check(lib().lb_linear_forward_siblings(
        x.data_ptr(), tokens, n_in, x.stride(0), len(layers), arr, workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_handle(stream)), "lb_linear_forward_siblings")
    return ys


def linear_forward_host(x_host, main: PackedPath, residual: PackedPath | None, y_host, x_dev, y_dev, workspace,
                        stream=None):
    """``lb_linear_forward_host``: x from pinned host memory (bf16 [tokens,
    n_in], contiguous) through the caller's device buffers x_dev and y_dev to
    y in pinned host memory (bf16 [tokens, n_out]), all on one stream; y_host
    is valid once the stream is synchronised.  For 1-128 tokens on pinned
    buffers x comes in through a gather kernel and y is written to y_host by
    the last kernel (y_dev is then not touched)."""
    torch = _torch()
    _require(x_host, "x_host", torch.bfloat16, device="cpu", contiguous=True)
    _require(y_host, "y_host", torch.bfloat16, device="cpu", contiguous=True)
    _require(x_dev, "x_dev", torch.bfloat16, contiguous=True)
    _require(y_dev, "y_dev", torch.bfloat16, contiguous=True)
    _require_workspace(workspace)
    tokens, n_in = x_host.shape
    n_out = main.h.shape[0]
    if tuple(y_host.shape) != (tokens, n_out) or tuple(x_dev.shape) != (tokens, n_in) \
            or tuple(y_dev.shape) != (tokens, n_out):
        raise ValueError("x_host / x_dev must be [tokens, n_in] and y_host / y_dev [tokens, n_out]")
    cm = main.as_c()
    cr = residual.as_c() if residual is not None else None
    _check(lib().lb_linear_forward_host(
        x_host.data_ptr(), tokens, n_in, n_out, ctypes.byref(cm), ctypes.byref(cr) if cr is not None else None,
        y_host.data_ptr(), x_dev.data_ptr(), y_dev.data_ptr(), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_handle(stream)), "lb_linear_forward_host")
    return y_host


def latent_forward(x, main: PackedPath, residual: PackedPath | None = None, z=None, stream=None):
    """``lb_latent_forward``: x bf16 [tokens, n_in] -> z fp16 [tokens, r_main
    + r_residual] (the latent of both paths, main first).  Allocates z with
    torch when not given (the C call allocates nothing)."""
    torch = _torch()
    _require(x, "x", torch.bfloat16)
    tokens, n_in = x.shape
    R = main.rank + (residual.rank if residual is not None else 0)
    if z is None:
        z = torch.empty((tokens, R), dtype=torch.float16, device=x.device)
    _require(z, "z", torch.float16)
    cm = main.as_c()
    cr = residual.as_c() if residual is not None else None
    _check(lib().lb_latent_forward(
        x.data_ptr(), tokens, n_in, x.stride(0), ctypes.byref(cm), ctypes.byref(cr) if cr is not None else None,
        z.data_ptr(), z.stride(0), _stream_handle(stream)), "lb_latent_forward")
    return z


def expand_forward(z, main: PackedPath, residual: PackedPath | None = None, y=None, stream=None):
    """``lb_expand_forward``: z fp16 [tokens, r_main + r_residual] -> y bf16
    [tokens, n_out].  Allocates y with torch when not given."""
    torch = _torch()
    _require(z, "z", torch.float16)
    tokens = z.shape[0]
    n_out = main.h.shape[0]
    if y is None:
        y = torch.empty((tokens, n_out), dtype=torch.bfloat16, device=z.device)
    _require(y, "y", torch.bfloat16)
    cm = main.as_c()
    cr = residual.as_c() if residual is not None else None
    _check(lib().lb_expand_forward(
        z.data_ptr(), tokens, n_out, z.stride(0), ctypes.byref(cm), ctypes.byref(cr) if cr is not None else None,
        y.data_ptr(), y.stride(0), _stream_handle(stream)), "lb_expand_forward")
    return y


def linear_forward_fixed_scratch(x, main: PackedPath, residual: PackedPath | None = None, y=None,
                                 stream=None):
    """``lb_linear_forward_fixed_scratch``: as :func:`linear_forward` for
    1..32 tokens, with the library's fixed device scratch instead of a
    workspace.  Allocates y with torch when not given (the C call itself
    allocates nothing)."""
    torch = _torch()
    _require(x, "x", torch.bfloat16)
    tokens, n_in = x.shape
    n_out = main.h.shape[0]
    if y is None:
        y = torch.empty((tokens, n_out), dtype=torch.bfloat16, device=x.device)
    _require(y, "y", torch.bfloat16)
    cm = main.as_c()
    cr = residual.as_c() if residual is not None else None
    _check(lib().lb_linear_forward_fixed_scratch(
        x.data_ptr(), tokens, n_in, n_out, x.stride(0), ctypes.byref(cm),
        ctypes.byref(cr) if cr is not None else None, y.data_ptr(), y.stride(0), _stream_handle(stream)),
        "lb_linear_forward_fixed_scratch")
    return y


def backward_workspace_bytes(tokens: int, n_in: int, n_out: int, rank_main: int, rank_residual: int = 0) -> int:
    return int(lib().lb_backward_workspace_bytes(tokens, n_in, n_out, rank_main, rank_residual))


def linear_backward(x, dy, main: PackedPath, residual: PackedPath | None = None, dx=None, want_dx: bool = True,
                    workspace=None, stream=None) -> dict:
    """``lb_linear_backward``: the gradients of a loss with respect to the
    layer's input and scale vectors, given ``dy`` = dL/dy (bf16 [tokens,
    n_out]) and the forward input ``x`` (bf16 [tokens, n_in]).  Returns
    ``{"dx": bf16 [tokens, n_in] or None, "dh": fp32 [paths, n_out], "dg":
    fp32 [paths, n_in], "dl": fp32 [r_main + r_residual]}``; outputs and the
    workspace are allocated with torch when not given."""
    torch = _torch()
    _require(x, "x", torch.bfloat16)
    _require(dy, "dy", torch.bfloat16)
    tokens, n_in = x.shape
    n_out = main.h.shape[0]
    if tuple(dy.shape) != (tokens, n_out):
        raise ValueError(f"dy must be [{tokens}, {n_out}], got {tuple(dy.shape)}")
    npaths = 2 if residual is not None else 1
    if dx is None and want_dx:
        dx = torch.empty((tokens, n_in), dtype=torch.bfloat16, device=x.device)
    if dx is not None:
        _require(dx, "dx", torch.bfloat16)
    dh = torch.empty((npaths, n_out), dtype=torch.float32, device=x.device)
    dg = torch.empty((npaths, n_in), dtype=torch.float32, device=x.device)
    dl = torch.empty((main.rank + (residual.rank if residual is not None else 0),), dtype=torch.float32,
                     device=x.device)
    if workspace is None:
        need = backward_workspace_bytes(tokens, n_in, n_out, main.rank, residual.rank if residual else 0)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    _require_workspace(workspace)
    cm = main.as_c()
    cr = residual.as_c() if residual is not None else None
    _check(lib().lb_linear_backward(
        x.data_ptr(), dy.data_ptr(), tokens, n_in, n_out, x.stride(0), dy.stride(0), ctypes.byref(cm),
        ctypes.byref(cr) if cr is not None else None, dx.data_ptr() if dx is not None else None,
        dx.stride(0) if dx is not None else n_in, dh.data_ptr(), dg.data_ptr(), dl.data_ptr(),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream)),
        "lb_linear_backward")
    return {"dx": dx, "dh": dh, "dg": dg, "dl": dl}


def device_status(stream=None) -> int:
    """``lb_device_status``: synchronise the stream, return and clear the
    device status word (an lb_status code)."""
    out = ctypes.c_int(0)
    _check(lib().lb_device_status(_stream_handle(stream), ctypes.byref(out)), "lb_device_status")
    return int(out.value)


def debug_inject_stall(enable: bool, wait_limit_ns: int = 2_000_000_000) -> None:
    """``lb_debug_inject_stall`` (tests only): make the tcgen05 decode kernels
    enqueued afterwards give up their bounded waits after ``wait_limit_ns``
    and skip one stage-barrier arrival, so that they time out and record
    LB_ERR_DEVICE_TIMEOUT; ``enable=False`` restores the defaults."""
    _check(lib().lb_debug_inject_stall(1 if enable else 0, int(wait_limit_ns) if enable else 0),
           "lb_debug_inject_stall")


def set_prefill_pairs(enable: bool) -> None:
    """``lb_set_prefill_pairs``: let prefill contractions run on CTA pairs
    (the default) or keep them on single-CTA tiles."""
    _check(lib().lb_set_prefill_pairs(1 if enable else 0), "lb_set_prefill_pairs")


class LittleBitLinear:
    """A deployed LittleBit layer: one or two packed paths on the device.

    ``layer(x)`` runs ``lb_linear_forward`` on the current stream."""

    def __init__(self, main: PackedPath, residual: PackedPath | None = None):
        self.main, self.residual = main, residual
        self.n_out = int(main.h.shape[0])
        self.n_in = int(main.g.shape[0])
        self._ws = None

    @classmethod
    def from_factors(cls, paths: list[dict], device="cuda") -> "LittleBitLinear":
        """``paths``: one or two dicts of host or device arrays ``su`` [n_out, r],
        ``sv`` [n_in, r] (+-1, any supported dtype) and fp16 ``h``, ``g``, ``l``."""
        torch = _torch()
        dev = lambda a: torch.as_tensor(a).to(device)
        packed = [PackedPath.from_factors(dev(p["su"]), dev(p["sv"]), dev(p["h"]), dev(p["g"]),
                                          dev(p["l"])) for p in paths]
        return cls(packed[0], packed[1] if len(packed) > 1 else None)

    def workspace(self, tokens: int, device):
        torch = _torch()
        need = forward_workspace_bytes(tokens, self.n_in, self.n_out, self.main.rank,
                                       self.residual.rank if self.residual else 0)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
        return self._ws

    def __call__(self, x, y=None, stream=None):
        return linear_forward(x, self.main, self.residual, y=y,
                              workspace=self.workspace(x.shape[0], x.device), stream=stream)

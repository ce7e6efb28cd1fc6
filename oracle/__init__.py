"""fp64 CPU oracle for the LittleBit factored linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never imports, links or calls it, and this package never imports
the CUDA library: the two share no code.  Inputs come to both sides from the
seeded generator module, which holds none of the method's arithmetic.

Sources (web pages about LittleBit / LittleBit-2; cited by page and section):

* sesamedisk.com, "Samsung LittleBit 13B Model", section "What the method
  actually computes" (Proposition 1): the factored forward pass
  ``Y = ((((X (.) g) V_sign) (.) l) U_sign^T) (.) h``.
* same page, section "How low-rank binarization works": U and V are binarized
  to +-1 (one bit per factor entry), h is the row scale, g the column scale,
  l the latent (per-rank) scale, all FP16; a residual binary path is added on
  top of the primary one without raising the total bit budget; "the rank sets
  the bit budget".
* littlebitllm.com, section "How small": the budget counts linear-layer sign
  bits only; scale vectors are not counted.

Functions:

* :func:`forward` - the factored pass, in C (``lb_oracle.c``), plain loops.
* :func:`backward` - the gradients of a loss with respect to x and to every
  path's h, g and l, given dL/dy: the chain rule through the five steps of
  the factored pass, in C (``lb_oracle.c``), plain loops.
* :func:`dense_weight` - ``W = sum_p diag(h) S_U diag(l) S_V^T diag(g)``, the
  same layer as one dense matrix (a numpy matmul per path).
* :func:`pack_signs` - this oracle's own bit packer for the library's packed
  sign layout (documented in ``include/lb.h``).
* :func:`rank_for_budget` - the bit-budget rank rule in exact integer
  arithmetic.

Every function is pinned by ``tests/test_oracle_*.py`` against values that do
not come from the oracle itself (hand-worked examples under ``tests/golden/``,
closed forms, brute force on tiny inputs, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lb_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liblb_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``lb_oracle.c`` with gcc (OpenMP, no fast-math, no FMA
    contraction) into ``oracle/_build/liblb_oracle.so``; return its path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Path(ctypes.Structure):
    _fields_ = [
        ("rank", ctypes.c_int64),
        ("su", ctypes.c_void_p),
        ("sv", ctypes.c_void_p),
        ("h", ctypes.c_void_p),
        ("g", ctypes.c_void_p),
        ("l", ctypes.c_void_p),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_forward.restype = ctypes.c_int
            lib.oracle_forward.argtypes = [
                ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                ctypes.POINTER(_Path), ctypes.c_int, ctypes.c_void_p]
            lib.oracle_latent.restype = ctypes.c_int
            lib.oracle_latent.argtypes = [
                ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                ctypes.POINTER(_Path), ctypes.c_int, ctypes.c_void_p]
            lib.oracle_expand.restype = ctypes.c_int
            lib.oracle_expand.argtypes = [
                ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                ctypes.POINTER(_Path), ctypes.c_int, ctypes.c_void_p]
            lib.oracle_backward.restype = ctypes.c_int
            lib.oracle_backward.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                ctypes.POINTER(_Path), ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p]
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_num_threads.argtypes = []
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the C oracle uses (``OMP_NUM_THREADS`` or all cores)."""
    return int(_load().oracle_num_threads())


# --------------------------------------------------------------------------
# exact widening of the storage formats
# --------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of
    an IEEE binary32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_to_f64(v: np.ndarray) -> np.ndarray:
    """IEEE binary16 -> float64, exactly."""
    return np.asarray(v, dtype=np.float16).astype(np.float64)


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------

def _as_path_arrays(p: dict) -> dict:
    su = np.ascontiguousarray(p["su"], dtype=np.int8)
    sv = np.ascontiguousarray(p["sv"], dtype=np.int8)
    r = su.shape[1]
    if sv.shape[1] != r:
        raise ValueError("U_sign and V_sign must have the same rank")
    if not (np.all(np.abs(su) == 1) and np.all(np.abs(sv) == 1)):
        raise ValueError("sign factors must hold only +1 and -1")
    out = dict(su=su, sv=sv, rank=r)
    for name in ("h", "g", "l"):
        out[name] = np.ascontiguousarray(p[name], dtype=np.float64)
    if out["h"].shape != (su.shape[0],) or out["g"].shape != (sv.shape[0],) \
            or out["l"].shape != (r,):
        raise ValueError("scale vector shapes do not match the factors")
    return out


def forward(x: np.ndarray, paths: list[dict]) -> np.ndarray:
    """fp64 factored forward pass.

    ``x``: float64 ``[tokens, n_in]`` (widen bf16 with :func:`bf16_bits_to_f64`).
    ``paths``: one or two dicts with ``su`` (int8 ``[n_out, r]``), ``sv`` (int8
    ``[n_in, r]``), ``h`` ``[n_out]``, ``g`` ``[n_in]``, ``l`` ``[r]`` (float64
    or float16; widened exactly).  Returns float64 ``[tokens, n_out]``.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    if x.ndim != 2:
        raise ValueError("x must be [tokens, n_in]")
    P = [_as_path_arrays(p) for p in paths]
    n_in = x.shape[1]
    n_out = P[0]["su"].shape[0]
    for p in P:
        if p["sv"].shape[0] != n_in or p["su"].shape[0] != n_out:
            raise ValueError("factor shapes do not match x / each other")
    arr = (_Path * len(P))()
    for j, p in enumerate(P):
        arr[j] = _Path(p["rank"], p["su"].ctypes.data, p["sv"].ctypes.data,
                       p["h"].ctypes.data, p["g"].ctypes.data, p["l"].ctypes.data)
    y = np.empty((x.shape[0], n_out), dtype=np.float64)
    rc = _load().oracle_forward(x.ctypes.data, x.shape[0], n_in, n_out, arr,
                                len(P), y.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_forward failed ({rc})")
    return y


def _c_paths(P):
    arr = (_Path * len(P))()
    for j, p in enumerate(P):
        arr[j] = _Path(p["rank"], p["su"].ctypes.data, p["sv"].ctypes.data,
                       p["h"].ctypes.data, p["g"].ctypes.data, p["l"].ctypes.data)
    return arr


def latent(x: np.ndarray, paths: list[dict]) -> np.ndarray:
    """fp64 first half of the forward pass (input scale, contraction 1,
    latent scale): ``z[m, off_p + k] = l_k sum_i sv[i, k] g_i x[m, i]``, the
    paths side by side (path 0 first).  Returns float64 ``[tokens, sum r_p]``.
    Same arguments as :func:`forward`."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    if x.ndim != 2:
        raise ValueError("x must be [tokens, n_in]")
    P = [_as_path_arrays(p) for p in paths]
    for p in P:
        if p["sv"].shape[0] != x.shape[1]:
            raise ValueError("V_sign does not match x")
    z = np.empty((x.shape[0], sum(p["rank"] for p in P)), dtype=np.float64)
    rc = _load().oracle_latent(x.ctypes.data, x.shape[0], x.shape[1], _c_paths(P), len(P), z.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_latent failed ({rc})")
    return z


def expand(z: np.ndarray, paths: list[dict]) -> np.ndarray:
    """fp64 second half of the forward pass (contraction 2, row scale, sum of
    the paths) from a latent laid out as :func:`latent` returns it.
    ``expand(latent(x, P), P)`` equals ``forward(x, P)`` exactly.  Returns
    float64 ``[tokens, n_out]``."""
    z = np.ascontiguousarray(z, dtype=np.float64)
    P = [_as_path_arrays(p) for p in paths]
    if z.ndim != 2 or z.shape[1] != sum(p["rank"] for p in P):
        raise ValueError("z must be [tokens, sum of the ranks]")
    n_out = P[0]["su"].shape[0]
    y = np.empty((z.shape[0], n_out), dtype=np.float64)
    rc = _load().oracle_expand(z.ctypes.data, z.shape[0], n_out, _c_paths(P), len(P), y.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_expand failed ({rc})")
    return y


def backward(x: np.ndarray, dy: np.ndarray, paths: list[dict]) -> dict:
    """fp64 backward pass of the layer for a loss L with ``dL/dy = dy``.

    The pages give the forward pass (sesamedisk.com, "What the method actually
    computes", Proposition 1) and train through it (littlebitllm.com,
    "Pipeline": quantization-aware training with a smooth surrogate for the
    gradient of sign); these are the chain-rule gradients of its five steps,
    with the signs held fixed: ``dx`` [tokens, n_in] and, per path, ``dh``
    [n_out], ``dg`` [n_in], ``dl`` [r] (lists, path order).  ``x`` and ``dy``
    are float64 [tokens, n_in] and [tokens, n_out]; ``paths`` as for
    :func:`forward`."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    P = [_as_path_arrays(p) for p in paths]
    n_in = x.shape[1]
    n_out = P[0]["su"].shape[0]
    if x.ndim != 2 or dy.shape != (x.shape[0], n_out):
        raise ValueError("x must be [tokens, n_in] and dy [tokens, n_out]")
    for p in P:
        if p["sv"].shape[0] != n_in or p["su"].shape[0] != n_out:
            raise ValueError("factor shapes do not match x / each other")
    R = sum(p["rank"] for p in P)
    dx = np.empty_like(x)
    dh = np.empty((len(P), n_out))
    dg = np.empty((len(P), n_in))
    dl = np.empty(R)
    rc = _load().oracle_backward(x.ctypes.data, dy.ctypes.data, x.shape[0], n_in, n_out, _c_paths(P), len(P),
                                 dx.ctypes.data, dh.ctypes.data, dg.ctypes.data, dl.ctypes.data)
    if rc != 0:
        raise RuntimeError(f"oracle_backward failed ({rc})")
    offs = np.cumsum([0] + [p["rank"] for p in P])
    return {"dx": dx, "dh": [dh[j] for j in range(len(P))], "dg": [dg[j] for j in range(len(P))],
            "dl": [dl[offs[j]:offs[j + 1]] for j in range(len(P))]}


def dense_weight(paths: list[dict]) -> np.ndarray:
    """The layer as one dense fp64 matrix ``W [n_out, n_in]`` with
    ``y = x W^T``:  ``W = sum_p diag(h_p) S_U,p diag(l_p) S_V,p^T diag(g_p)``
    (littlebitllm.com, "The method": W ~ sign(U) h.g.l sign(V)^T with h on the
    rows, g on the columns, l on the latent dimension)."""
    W = None
    for p in (_as_path_arrays(q) for q in paths):
        left = p["h"][:, None] * p["su"].astype(np.float64) * p["l"][None, :]
        right = p["sv"].astype(np.float64).T * p["g"][None, :]
        term = left @ right
        W = term if W is None else W + term
    return W


# --------------------------------------------------------------------------
# packed sign layout (this oracle's own packer)
# --------------------------------------------------------------------------

def packed_ld_words(cols: int) -> int:
    """Smallest packed row stride: ceil(cols / 32) words (rows are dense)."""
    return -(-int(cols) // 32)


def _negative_mask(src: np.ndarray, dtype: str) -> np.ndarray:
    """True where the element is strictly negative.  Zero, -0.0 and NaN are
    not negative; -inf is.  The pages only say each entry is +1 or -1; this
    reading (sign bit set AND value < 0) is the one the library documents."""
    if dtype == "bf16":
        v = (np.asarray(src, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
        return v < 0
    if dtype == "f16":
        return np.asarray(src, dtype=np.float16) < 0
    if dtype == "f32":
        return np.asarray(src, dtype=np.float32) < 0
    if dtype == "i8":
        return np.asarray(src, dtype=np.int8) < 0
    raise ValueError(f"unknown dtype {dtype!r}")


def pack_rows(neg: np.ndarray, ld_words: int | None = None) -> np.ndarray:
    """Pack a boolean ``[rows, cols]`` matrix along its columns: word ``w`` of a
    row holds columns ``32w .. 32w+31``, bit ``j`` (value ``1 << j``) set iff
    column ``32w + j`` is negative.  Padding bits and words are zero."""
    neg = np.asarray(neg, dtype=bool)
    rows, cols = neg.shape
    ld = packed_ld_words(cols) if ld_words is None else int(ld_words)
    if ld * 32 < cols:
        raise ValueError("ld_words too small")
    out = np.zeros((rows, ld), dtype=np.uint32)
    for j in range(32):
        colj = neg[:, j::32]                         # columns 32w + j
        out[:, : colj.shape[1]] |= colj.astype(np.uint32) << np.uint32(j)
    return out


def pack_signs(src: np.ndarray, kind: str, dtype: str = "i8",
               ld_words: int | None = None) -> np.ndarray:
    """Pack a factor the way ``lb_pack_signs`` documents it.

    ``kind == "U"``: ``src`` is U ``[n_out, r]``; row ``o`` of the result packs
    ``U[o, :]`` along r.  ``kind == "V"``: ``src`` is V ``[n_in, r]``; the
    result is V^T packed: row ``k`` packs ``V[:, k]`` along n_in.
    """
    neg = _negative_mask(src, dtype)
    if kind == "U":
        return pack_rows(neg, ld_words)
    if kind == "V":
        return pack_rows(neg.T, ld_words)
    raise ValueError("kind must be 'U' or 'V'")


def unpack_rows(words: np.ndarray, cols: int) -> np.ndarray:
    """Inverse of :func:`pack_rows`: int8 +-1 ``[rows, cols]``."""
    words = np.asarray(words, dtype=np.uint32)
    rows = words.shape[0]
    out = np.empty((rows, cols), dtype=np.int8)
    for c in range(cols):
        bit = (words[:, c // 32] >> np.uint32(c % 32)) & np.uint32(1)
        out[:, c] = 1 - 2 * bit.astype(np.int8)
    return out


# --------------------------------------------------------------------------
# bit budget
# --------------------------------------------------------------------------

def rank_for_budget(n_in: int, n_out: int, eff_num: int, eff_den: int,
                    paths: int = 1, align: int = 1) -> int:
    """Rank per path from the bit budget.

    The budget is ``eff * n_in * n_out`` sign bits for the layer (scale vectors
    not counted); a path of rank r stores ``r * (n_in + n_out)`` sign bits, and
    with residual compensation the paths share the budget.  So the largest
    admissible rank per path is ``floor(eff * n_in * n_out / (paths * (n_in +
    n_out)))``, then rounded down to a multiple of ``align``.  Exact integer
    arithmetic: ``eff`` is the fraction ``eff_num / eff_den``.
    """
    num = int(eff_num) * int(n_in) * int(n_out)
    den = int(eff_den) * int(paths) * (int(n_in) + int(n_out))
    r = num // den
    return (r // int(align)) * int(align)

"""Float64 CPU oracle for exact scaled dot-product attention.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or runs anything here, and nothing here imports the CUDA
library: the two share only the seeded input arrays that a test hands to both.

Contents
--------
``fwd`` / ``bwd``
    The plain definition (``fa_oracle.c``), float64, every S and P row
    materialised: the SDPA formula of the FlashAttention case-study slides
    (nmj0.github.io, "Attention is where tokens meet") with the safe softmax of
    "Problem: softmax needs the whole row".  Backward by the analytic gradient
    of that definition (the pages only state that the backward recomputes the
    scores; the formulas are derived, and pinned by finite differences).
``online``
    The tiled running-state form of "Online softmax: divide once, at the end"
    and the associative merge of the "twisted monoid" digest (setupai.cc,
    "Mastering FlashAttention: The Algebraic Foundation"), in float64.

Array layout everywhere: ``[B, H, N, D]`` with D fastest; key bias ``[B, Nk]``;
general additive mask ``[B or 1, H or 1, Nq, Nk]`` (or ``[Nq, Nk]``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ``fa_oracle.c`` with gcc (OpenMP, IEEE semantics kept)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    lib.oracle_fwd.argtypes = [dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_double, ip,
                               ctypes.c_int, dp, dp]
    lib.oracle_fwd.restype = None
    lib.oracle_bwd.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int,
                               ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_int, ctypes.c_double,
                               ip, ctypes.c_int, ip, ctypes.c_int, dp, dp, dp]
    lib.oracle_bwd.restype = None
    L = ctypes.c_long
    lib.oracle_fwd_mask.argtypes = [dp, dp, dp, dp, dp, L, L, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_double, ip,
                                    ctypes.c_int, dp, dp]
    lib.oracle_fwd_mask.restype = None
    lib.oracle_bwd_mask.argtypes = [dp, dp, dp, dp, dp, L, L, dp, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                    ip, ctypes.c_int, ip, ctypes.c_int, dp, dp, dp]
    lib.oracle_bwd_mask.restype = None
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def build_variant(src_text: str, tag: str) -> "Oracle":
    """Compile a modified copy of the oracle source (used by the tests that
    plant a mistake in the oracle and check that the pins catch it)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    c_path = os.path.join(_BUILD_DIR, f"variant_{tag}.c")
    so_path = os.path.join(_BUILD_DIR, f"libvariant_{tag}.so")
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                    "-std=c11", c_path, "-o", so_path, "-lm"], check=True)
    return Oracle(_bind(ctypes.CDLL(so_path)))


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def default_scale(D: int) -> float:
    """1/sqrt(d_k), the scale in the slides' SDPA formula."""
    return 1.0 / np.sqrt(D)


def _mask_arg(mask, B, H, Nq, Nk):
    """(array, batch stride, head stride) for the C oracle; strides in
    elements, 0 where the mask broadcasts over that axis."""
    if mask is None:
        return None, 0, 0
    m = _f64(mask)
    if m.ndim == 2:
        m = m[None, None]
    assert m.ndim == 4 and m.shape[2:] == (Nq, Nk), m.shape
    assert m.shape[0] in (1, B) and m.shape[1] in (1, H), m.shape
    assert not np.any(np.isposinf(m)) and not np.any(np.isnan(m)), "mask entries: finite or -inf"
    hs = Nq * Nk if m.shape[1] == H and H > 1 else 0
    bs = m.shape[1] * Nq * Nk if m.shape[0] == B and B > 1 else 0
    return m, bs, hs


class Oracle:
    """The oracle bound to one compiled copy of ``fa_oracle.c``."""

    def __init__(self, lib):
        self._lib = lib

    def fwd(self, q, k, v, key_bias=None, causal=False, scale=None, rows=None, mask=None):
        """Exact attention forward in float64.

        q: [B,H,Nq,D]; k, v: [B,H,Nk,D]; key_bias: [B,Nk] or None (additive, after
        scaling); mask: general additive mask [B or 1, H or 1, Nq, Nk] or
        [Nq, Nk] (finite or -inf, added after scaling), or None.  ``rows``:
        optional 1-D list of query-row indices evaluated for every (b, h); None
        means all rows.  Returns ``(o, lse)`` with o [B,H,R,D] and lse [B,H,R]
        (R = Nq or len(rows)).
        """
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, Nq, D = q.shape
        Nk = k.shape[2]
        assert k.shape == (B, H, Nk, D) and v.shape == (B, H, Nk, D)
        bias = None if key_bias is None else _f64(key_bias)
        if bias is not None:
            assert bias.shape == (B, Nk)
        if scale is None:
            scale = default_scale(D)
        rows_arr = None
        if rows is not None:
            rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
            assert rows_arr.ndim == 1 and (rows_arr.size == 0 or
                                           (rows_arr.min() >= 0 and rows_arr.max() < Nq))
        R = Nq if rows_arr is None else rows_arr.size
        o = np.zeros((B, H, R, D), dtype=np.float64)
        lse = np.zeros((B, H, R), dtype=np.float64)
        if B * H * R == 0:
            return o, lse
        if mask is None:
            self._lib.oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), B, H, Nq, Nk, D,
                               int(bool(causal)), float(scale),
                               _ptr(rows_arr, ctypes.c_int), 0 if rows_arr is None else R,
                               _ptr(o), _ptr(lse))
        else:
            m, bs, hs = _mask_arg(mask, B, H, Nq, Nk)
            self._lib.oracle_fwd_mask(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(m), bs, hs,
                                    B, H, Nq, Nk, D, int(bool(causal)), float(scale),
                                    _ptr(rows_arr, ctypes.c_int), 0 if rows_arr is None else R,
                                    _ptr(o), _ptr(lse))
        return o, lse


    def bwd(self, q, k, v, dO, key_bias=None, causal=False, scale=None, bh_list=None,
            rows=None, mask=None):
        """Exact gradients of L = sum(O * dO) w.r.t. q, k, v in float64.

        ``bh_list``: flat (b*H + h) indices to evaluate (None = all).  Returns
        ``(dq, dk, dv)`` of shapes [n, Nq, D], [n, Nk, D], [n, Nk, D].
        ``rows``: optional query-row subset; only those rows contribute (a
        bounded sample of the work for timing; None = the full gradient).
        ``mask``: as in ``fwd``; it receives no gradient.
        """
        q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
        B, H, Nq, D = q.shape
        Nk = k.shape[2]
        assert dO.shape == q.shape
        bias = None if key_bias is None else _f64(key_bias)
        if scale is None:
            scale = default_scale(D)
        if bh_list is None:
            bh_list = np.arange(B * H)
        bh = np.ascontiguousarray(np.asarray(bh_list, dtype=np.int32))
        n = bh.size
        rows_arr = None
        if rows is not None:
            rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
            assert rows_arr.size == 0 or (rows_arr.min() >= 0 and rows_arr.max() < Nq)
        dq = np.zeros((n, Nq, D))
        dk = np.zeros((n, Nk, D))
        dv = np.zeros((n, Nk, D))
        if n == 0:
            return dq, dk, dv
        if mask is None:
            self._lib.oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(dO), B, H, Nq,
                               Nk, D, int(bool(causal)), float(scale),
                               _ptr(bh, ctypes.c_int), n, _ptr(rows_arr, ctypes.c_int),
                               0 if rows_arr is None else rows_arr.size,
                               _ptr(dq), _ptr(dk), _ptr(dv))
        else:
            m, bs, hs = _mask_arg(mask, B, H, Nq, Nk)
            self._lib.oracle_bwd_mask(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(m), bs, hs,
                                    _ptr(dO), B, H, Nq, Nk, D, int(bool(causal)),
                                    float(scale), _ptr(bh, ctypes.c_int), n,
                                    _ptr(rows_arr, ctypes.c_int),
                                    0 if rows_arr is None else rows_arr.size,
                                    _ptr(dq), _ptr(dk), _ptr(dv))
        return dq, dk, dv


def fwd(*args, **kwargs):
    """See ``Oracle.fwd``; uses the oracle built from ``fa_oracle.c``."""
    return Oracle(_load()).fwd(*args, **kwargs)


def bwd(*args, **kwargs):
    """See ``Oracle.bwd``; uses the oracle built from ``fa_oracle.c``."""
    return Oracle(_load()).bwd(*args, **kwargs)

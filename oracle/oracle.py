"""ctypes binding of the float64 C oracle (``rra_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Arrays are taken as numpy arrays or
CPU torch tensors; 16-bit inputs are passed as raw bit patterns and widened exactly by the C
code.  Each wrapper follows the C function of the same name, which cites the passage of
"Dispatch-Aware Ragged Attention for Pruned Vision Transformers" that it restates.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rra_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "librra_oracle.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODES = {"f16": 0, "bf16": 1, "f32": 2, "f64": 3}


def library_path() -> str:
    return _LIB_PATH


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle with gcc (plain -O2, strict IEEE double: no -ffast-math)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src) and not extra_flags):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           *extra_flags, src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _declare(lib):
    i32p = ctypes.POINTER(ctypes.c_int32)
    i64p = ctypes.POINTER(ctypes.c_int64)
    u8p = ctypes.c_void_p
    vp = ctypes.c_void_p
    lib.rra_oracle_cu_seqlens.argtypes = [u8p, ctypes.c_int, ctypes.c_int, i32p]
    lib.rra_oracle_cu_seqlens.restype = ctypes.c_int64
    lib.rra_oracle_rank.argtypes = [u8p, ctypes.c_int, ctypes.c_int, i32p]
    lib.rra_oracle_rank.restype = None
    lib.rra_oracle_pack.argtypes = [u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int64, vp, vp,
                                    ctypes.c_int64, i32p]
    lib.rra_oracle_pack.restype = ctypes.c_int64
    lib.rra_oracle_attend.argtypes = [vp, vp, vp, ctypes.c_int, i32p, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_double, vp]
    lib.rra_oracle_attend.restype = ctypes.c_int
    lib.rra_oracle_attend_rows.argtypes = [vp, vp, vp, ctypes.c_int, i32p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_double, ctypes.c_int64, i64p, i32p, vp]
    lib.rra_oracle_attend_rows.restype = ctypes.c_int
    lib.rra_oracle_unpack.argtypes = [vp, i32p, u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_int, ctypes.c_int64, vp]
    lib.rra_oracle_unpack.restype = ctypes.c_int
    lib.rra_oracle_l2_mask.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, i32p,
                                       ctypes.c_double, u8p, u8p]
    lib.rra_oracle_l2_mask.restype = ctypes.c_int
    lib.rra_oracle_l2_score.argtypes = [vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                        ctypes.POINTER(ctypes.c_uint32)]
    lib.rra_oracle_l2_score.restype = ctypes.c_int
    lib.rra_oracle_l2_score_words.argtypes = []
    lib.rra_oracle_l2_score_words.restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library; `path` loads another build of it."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


# ----------------------------------------------------------------------------------------------
# array helpers (marshalling only)

def _np(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype in (torch.float16, torch.bfloat16):
                return x.view(torch.int16).numpy().view(np.uint16)
            return x.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x)


def _dtype_code(x, dtype: str | None) -> int:
    if dtype is not None:
        return DTYPE_CODES[dtype]
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2, torch.float64: 3}[x.dtype]
    except ImportError:  # pragma: no cover
        pass
    arr = np.asarray(x)
    return {np.dtype(np.float16): 0, np.dtype(np.float32): 2, np.dtype(np.float64): 3}[arr.dtype]


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


# ----------------------------------------------------------------------------------------------
# public wrappers

def cu_seqlens(mask, lib=None) -> np.ndarray:
    """int32 [B+1]: running sum of kept tokens per image (packer phase 1)."""
    lib = lib or load()
    m = np.ascontiguousarray(_np(mask).astype(np.uint8, copy=False))
    B, N = m.shape
    cu = np.zeros(B + 1, dtype=np.int32)
    lib.rra_oracle_cu_seqlens(_ptr(m), B, N, _i32p(cu))
    return cu


def rank(mask, lib=None) -> np.ndarray:
    """int32 [B, N]: position of each kept token among its image's kept tokens, -1 if pruned."""
    lib = lib or load()
    m = np.ascontiguousarray(_np(mask).astype(np.uint8, copy=False))
    B, N = m.shape
    r = np.zeros((B, N), dtype=np.int32)
    lib.rra_oracle_rank(_ptr(m), B, N, _i32p(r))
    return r


def pack(mask, src, capacity: int | None = None, lib=None):
    """Gather kept rows of padded src [B, N, ...] into [capacity, ...]; returns (packed, cu).

    Rows of the packed buffer past T keep the value of `fill` (zero bytes)."""
    lib = lib or load()
    m = np.ascontiguousarray(_np(mask).astype(np.uint8, copy=False))
    s = np.ascontiguousarray(_np(src))
    B, N = m.shape
    assert s.shape[:2] == (B, N)
    row_shape = s.shape[2:]
    row_bytes = int(s.itemsize * int(np.prod(row_shape, dtype=np.int64)))
    if capacity is None:
        capacity = B * N
    dst = np.zeros((capacity,) + row_shape, dtype=s.dtype)
    cu = np.zeros(B + 1, dtype=np.int32)
    lib.rra_oracle_pack(_ptr(m), B, N, row_bytes, _ptr(s), _ptr(dst), capacity, _i32p(cu))
    return dst, cu


def attend(q, k, v, cu, H: int, d: int, scale: float = 0.0, dtype: str | None = None, lib=None) -> np.ndarray:
    """float64 [T, H, d] ragged attention of packed q/k/v [>=T, H, d] over cu_seqlens."""
    lib = lib or load()
    code = _dtype_code(q, dtype)
    qa, ka, va = _np(q), _np(k), _np(v)
    cua = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    B = cua.shape[0] - 1
    T = int(cua[-1]) if B >= 0 else 0
    out = np.zeros((max(T, 0), H, d), dtype=np.float64)
    rc = lib.rra_oracle_attend(_ptr(qa), _ptr(ka), _ptr(va), code, _i32p(cua), B, H, d,
                               float(scale), _ptr(out))
    if rc != 0:
        raise ValueError("malformed cu_seqlens")
    return out


def attend_rows(q, k, v, cu, H: int, d: int, rows_t, rows_h, scale: float = 0.0,
                dtype: str | None = None, lib=None) -> np.ndarray:
    """float64 [n, d]: attention rows for the (packed token, head) pairs given."""
    lib = lib or load()
    code = _dtype_code(q, dtype)
    qa, ka, va = _np(q), _np(k), _np(v)
    cua = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    t = np.ascontiguousarray(np.asarray(rows_t, dtype=np.int64))
    h = np.ascontiguousarray(np.asarray(rows_h, dtype=np.int32))
    out = np.zeros((t.shape[0], d), dtype=np.float64)
    rc = lib.rra_oracle_attend_rows(_ptr(qa), _ptr(ka), _ptr(va), code, _i32p(cua), cua.shape[0] - 1,
                                    H, d, float(scale), t.shape[0],
                                    t.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _i32p(h), _ptr(out))
    if rc != 0:
        raise ValueError("row outside every sequence")
    return out


def unpack(packed, cu, mask, fill_mode: int = 0, dst=None, capacity: int | None = None, lib=None) -> np.ndarray:
    """Scatter packed rows back to padded [B, N, ...]; pruned rows zero (mode 0) or untouched (1)."""
    lib = lib or load()
    p = np.ascontiguousarray(_np(packed))
    m = np.ascontiguousarray(_np(mask).astype(np.uint8, copy=False))
    cua = np.ascontiguousarray(np.asarray(cu, dtype=np.int32))
    B, N = m.shape
    row_shape = p.shape[1:]
    row_bytes = int(p.itemsize * int(np.prod(row_shape, dtype=np.int64)))
    if dst is None:
        out = np.zeros((B, N) + row_shape, dtype=p.dtype)
    else:
        out = np.ascontiguousarray(_np(dst)).copy()
    if capacity is None:
        capacity = p.shape[0]
    lib.rra_oracle_unpack(_ptr(p), _i32p(cua), _ptr(m), B, N, row_bytes, int(fill_mode), int(capacity), _ptr(out))
    return out


def l2_mask(x, k_keep=None, threshold_sq: float = 0.0, prev=None, dtype: str | None = None, lib=None) -> np.ndarray:
    """Threshold-l2 selection: embeddings x [B, N, C] (16-bit or float) -> keep mask uint8 [B, N].

    With k_keep ([B] ints) each image keeps CLS and its k_b highest-norm candidates (lower
    index first among ties); otherwise CLS and every candidate whose squared norm reaches
    threshold_sq.  Candidates are tokens n >= 1 kept in `prev` (all of them without it)."""
    lib = lib or load()
    xa = _np(x)
    code = _dtype_code(x, dtype)
    B, N, C = xa.shape
    out = np.zeros((B, N), dtype=np.uint8)
    kk = None if k_keep is None else np.ascontiguousarray(np.asarray(k_keep, dtype=np.int32))
    pv = None if prev is None else np.ascontiguousarray(_np(prev).astype(np.uint8))
    rc = lib.rra_oracle_l2_mask(_ptr(xa), code, B, N, C, None if kk is None else _i32p(kk), float(threshold_sq),
                                None if pv is None else _ptr(pv), _ptr(out))
    if rc != 0:
        raise ValueError("rra_oracle_l2_mask: bad arguments")
    return out


SCORE_NAN, SCORE_FINITE, SCORE_INF = 0, 1, 2
SCORE_EMIN = -298  # weight of the last bit of the oracle's fixed-point squared norm


def l2_score(x, dtype: str | None = None, lib=None):
    """Exact squared l2 norm of every row of x [..., C] as computed by the oracle: a list of
    (class, value) with class SCORE_NAN / SCORE_FINITE / SCORE_INF and, for a finite score, the
    exact value as a fractions.Fraction (None otherwise)."""
    from fractions import Fraction
    lib = lib or load()
    xa = _np(x)
    code = _dtype_code(x, dtype)
    C = xa.shape[-1]
    rows = int(np.prod(xa.shape[:-1], dtype=np.int64))
    xa = np.ascontiguousarray(xa.reshape(rows, C))
    nw = lib.rra_oracle_l2_score_words()
    words = (ctypes.c_uint32 * nw)()
    out = []
    for r in range(rows):
        cls = lib.rra_oracle_l2_score(_ptr(xa), code, r, C, words)
        if cls < 0:
            raise ValueError("rra_oracle_l2_score: unsupported dtype")
        if cls == SCORE_FINITE:
            v = 0
            for i in reversed(range(nw)):
                v = (v << 32) | int(words[i])
            out.append((cls, Fraction(v, 1 << -SCORE_EMIN)))
        else:
            out.append((cls, None))
    return out

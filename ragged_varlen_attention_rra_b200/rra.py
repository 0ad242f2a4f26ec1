"""Thin Python binding of librra.so (the C ABI in include/rra.h).

Argument marshalling only: every step of the path runs in the library's CUDA kernels.  PyTorch
supplies device memory and the current stream.  If librra.so is missing or cannot be loaded,
every function here raises -- there is no fallback.

Names follow the C ABI: :func:`rra_pack`, :func:`rra_attend`, :func:`rra_unpack`,
:func:`rra_pack_attend_unpack`, :func:`rra_l2_mask`, :func:`rra_get_device_error`,
:func:`rra_status_string`, :func:`rra_attend_workspace_size`, :func:`rra_set_wait_timeout_ns`.
:func:`forward` runs the whole pack-attend-unpack call of one pruning stage, as three calls or
as the single launch.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("RRA_LIBRARY", os.path.join(_HERE, "librra.so"))

RRA_OK, RRA_ERR_INVALID_ARG, RRA_ERR_UNSUPPORTED, RRA_ERR_CUDA = 0, 1, 2, 3
RRA_ERR_CAPACITY, RRA_ERR_TIMEOUT, RRA_ERR_BAD_SEQLENS = 4, 5, 6
RRA_F16, RRA_BF16, RRA_F32 = 0, 1, 2

_DT = {torch.float16: RRA_F16, torch.bfloat16: RRA_BF16, torch.float32: RRA_F32}

_lock = threading.Lock()
_lib = None


class RRAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {rra_status_string(status)} ({status})")


def _declare(lib):
    c = ctypes
    vp, i32p = c.c_void_p, c.c_void_p
    lib.rra_pack.argtypes = [vp, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                             c.POINTER(c.c_void_p), c.POINTER(c.c_void_p), c.c_int64, i32p, i32p, vp]
    lib.rra_pack.restype = c.c_int
    lib.rra_attend.argtypes = [vp, vp, vp, vp, i32p, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int64,
                               c.c_float, c.c_int, c.c_int, vp, c.c_size_t, i32p, vp]
    lib.rra_attend.restype = c.c_int
    lib.rra_attend_workspace_size.argtypes = [c.c_int, c.c_int, c.c_int]
    lib.rra_attend_workspace_size.restype = c.c_size_t
    lib.rra_unpack.argtypes = [vp, i32p, vp, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                               c.c_int64, vp, i32p, vp]
    lib.rra_unpack.restype = c.c_int
    lib.rra_pack_attend_unpack.argtypes = [vp, vp, vp, vp, vp, i32p, c.c_int, c.c_int, c.c_int, c.c_int,
                                           c.c_float, c.c_int, c.c_int, i32p, vp]
    lib.rra_pack_attend_unpack.restype = c.c_int
    lib.rra_l2_mask.argtypes = [vp, c.c_int, c.c_int, c.c_int, c.c_int, i32p, c.c_double, vp, vp, vp]
    lib.rra_l2_mask.restype = c.c_int
    lib.rra_linear.argtypes = [vp, vp, vp, vp, c.POINTER(c.c_void_p), c.c_int, c.c_int64, i32p, c.c_int, c.c_int,
                               c.c_int, i32p, vp]
    lib.rra_linear.restype = c.c_int
    lib.rra_layernorm.argtypes = [vp, vp, vp, vp, c.c_int64, i32p, c.c_int, c.c_float, vp]
    lib.rra_layernorm.restype = c.c_int
    lib.rra_get_device_error.argtypes = [i32p, vp, c.POINTER(c.c_int32)]
    lib.rra_get_device_error.restype = c.c_int
    lib.rra_status_string.argtypes = [c.c_int]
    lib.rra_status_string.restype = c.c_char_p
    lib.rra_set_wait_timeout_ns.argtypes = [c.c_uint64]
    lib.rra_set_wait_timeout_ns.restype = None
    lib.rra_version.argtypes = []
    lib.rra_version.restype = c.c_int
    return lib


def lib():
    """The loaded librra.so (ctypes handle).  Raises if the library is missing."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise ImportError(
                        f"librra.so not found at {LIB_PATH}; build it with "
                        "`python -m ragged_varlen_attention_rra_b200.build` (no CPU fallback exists)")
                _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, what: str):
    if status != RRA_OK:
        raise RRAError(status, what)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("rra calls take contiguous CUDA tensors")


def _expect(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _is_mask(t: torch.Tensor) -> bool:
    return t.dtype in (torch.uint8, torch.bool)


def _span(t: torch.Tensor):
    a = t.data_ptr()
    return a, a + t.numel() * t.element_size()


def _disjoint(outs, ins, what: str):
    """Each output's bytes must not overlap any input's: the kernels read inputs of an image while
    other blocks write outputs of the same image, so an in-place call would race."""
    for o in outs:
        if o is None or o.numel() == 0:
            continue
        o0, o1 = _span(o)
        for i in ins:
            if i is None or i.numel() == 0:
                continue
            i0, i1 = _span(i)
            _expect(o1 <= i0 or i1 <= o0, f"{what}: an output overlaps an input")


def _check_cu(cu: Optional[torch.Tensor], B: int, what: str):
    if cu is None:
        return
    _expect(cu.dtype == torch.int32 and cu.dim() == 1 and cu.numel() >= B + 1,
            f"{what}: cu_seqlens must be int32 [B+1] (B = {B}), got {cu.dtype} {tuple(cu.shape)}")


def _check_err(err: Optional[torch.Tensor], what: str):
    if err is not None:
        _expect(err.dtype == torch.int32 and err.numel() >= 1, f"{what}: dev_error must be an int32 word")


# ------------------------------------------------------------------------------------ calls

def rra_status_string(status: int) -> str:
    return lib().rra_status_string(int(status)).decode()


def rra_attend_workspace_size(B: int, H: int, max_seqlen: int) -> int:
    return int(lib().rra_attend_workspace_size(B, H, max_seqlen))


def rra_set_wait_timeout_ns(ns: int) -> None:
    lib().rra_set_wait_timeout_ns(int(ns))


def rra_get_device_error(dev_error: torch.Tensor, stream=None) -> int:
    """Read the device error word (synchronises the stream)."""
    out = ctypes.c_int32(0)
    _check(lib().rra_get_device_error(_ptr(dev_error), _stream(stream), ctypes.byref(out)), "rra_get_device_error")
    return int(out.value)


def rra_pack(mask: torch.Tensor, srcs: Sequence[torch.Tensor], dsts: Sequence[torch.Tensor],
             cu_seqlens: torch.Tensor, capacity: Optional[int] = None,
             dev_error: Optional[torch.Tensor] = None, stream=None) -> None:
    """Keep mask [B, N] + padded srcs [B, N, H, d] -> packed dsts [capacity, H, d] and cu_seqlens [B+1]."""
    what = "rra_pack"
    _expect(1 <= len(srcs) <= 3 and len(srcs) == len(dsts), f"{what}: 1..3 sources and as many destinations")
    _expect(_is_mask(mask) and mask.dim() == 2, f"{what}: mask must be uint8/bool [B, N]")
    B, N = mask.shape
    s0 = srcs[0]
    _expect(s0.dim() == 4 and tuple(s0.shape[:2]) == (B, N) and s0.dtype in _DT,
            f"{what}: sources must be [B, N, H, d] = [{B}, {N}, H, d] fp16/bf16/fp32")
    H, d = s0.shape[2], s0.shape[3]
    for t in srcs:
        _expect(t.shape == s0.shape and t.dtype == s0.dtype, f"{what}: sources differ in shape or dtype")
    for t in dsts:
        _expect(t.dim() == 3 and tuple(t.shape[1:]) == (H, d) and t.dtype == s0.dtype,
                f"{what}: destinations must be [capacity, {H}, {d}] of the sources' dtype")
    rows = min(t.shape[0] for t in dsts)
    cap = rows if capacity is None else int(capacity)
    _expect(1 <= cap <= rows, f"{what}: capacity {cap} outside [1, {rows}] (rows of the destinations)")
    _check_cu(cu_seqlens, B, what)
    _check_err(dev_error, what)
    _disjoint([*dsts, cu_seqlens], [mask, *srcs], what)
    _disjoint(list(dsts), [cu_seqlens], what)
    _require_cuda(mask, cu_seqlens, dev_error, *srcs, *dsts)
    n = len(srcs)
    src_arr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in srcs])
    dst_arr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in dsts])
    st = lib().rra_pack(_ptr(mask), B, N, H, d, _DT[s0.dtype], n, src_arr, dst_arr, cap,
                        _ptr(cu_seqlens), _ptr(dev_error), _stream(stream))
    _check(st, what)


def rra_attend(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, cu_seqlens: torch.Tensor,
               max_seqlen: int, softmax_scale: float = 0.0, dev_error: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Packed q/k/v [capacity, H, 64] + cu_seqlens [B+1] -> packed o (o's dtype selects the output type)."""
    what = "rra_attend"
    _expect(q.dim() == 3 and q.dtype in (torch.float16, torch.bfloat16), f"{what}: q must be fp16/bf16 [capacity, H, d]")
    for t in (k, v):
        _expect(t.shape == q.shape and t.dtype == q.dtype, f"{what}: k and v must match q's shape and dtype")
    _expect(o.shape == q.shape and o.dtype in (q.dtype, torch.float32),
            f"{what}: o must be {tuple(q.shape)} in q's dtype or fp32")
    _expect(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 1,
            f"{what}: cu_seqlens must be int32 [B+1]")
    _check_err(dev_error, what)
    _disjoint([o], [q, k, v, cu_seqlens, workspace], what)
    _require_cuda(q, k, v, o, cu_seqlens, dev_error, workspace)
    B = cu_seqlens.shape[0] - 1
    cap, H, d = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().rra_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu_seqlens), B, H, d, int(max_seqlen), cap,
                          float(softmax_scale), _DT[q.dtype], _DT[o.dtype], _ptr(workspace), ws_bytes,
                          _ptr(dev_error), _stream(stream))
    _check(st, what)


def rra_unpack(packed: torch.Tensor, cu_seqlens: torch.Tensor, mask: torch.Tensor, dst: torch.Tensor,
               fill_mode: int = 0, capacity: Optional[int] = None, dev_error: Optional[torch.Tensor] = None,
               stream=None) -> None:
    """Packed [capacity, H, d] -> padded dst [B, N, H, d]; pruned rows zero (fill_mode 0) or untouched (1)."""
    what = "rra_unpack"
    _expect(packed.dim() == 3 and packed.dtype in _DT, f"{what}: packed must be [capacity, H, d]")
    _expect(_is_mask(mask) and mask.dim() == 2, f"{what}: mask must be uint8/bool [B, N]")
    B, N = mask.shape
    cap = packed.shape[0] if capacity is None else int(capacity)
    _expect(1 <= cap <= packed.shape[0], f"{what}: capacity {cap} outside [1, {packed.shape[0]}] (rows of packed)")
    H, d = packed.shape[1], packed.shape[2]
    _expect(tuple(dst.shape) == (B, N, H, d) and dst.dtype == packed.dtype,
            f"{what}: dst must be [{B}, {N}, {H}, {d}] in packed's dtype")
    _check_cu(cu_seqlens, B, what)
    _check_err(dev_error, what)
    _disjoint([dst], [packed, cu_seqlens, mask], what)
    _require_cuda(packed, cu_seqlens, mask, dst, dev_error)
    st = lib().rra_unpack(_ptr(packed), _ptr(cu_seqlens), _ptr(mask), B, N, H, d, _DT[packed.dtype],
                          int(fill_mode), cap, _ptr(dst), _ptr(dev_error), _stream(stream))
    _check(st, what)


def rra_pack_attend_unpack(mask: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, y: torch.Tensor,
                           cu_seqlens: Optional[torch.Tensor] = None, softmax_scale: float = 0.0,
                           dev_error: Optional[torch.Tensor] = None, stream=None) -> None:
    """The whole call in one launch: padded q/k/v [B, N, H, 64] + mask [B, N] -> padded y (pruned rows zero)."""
    what = "rra_pack_attend_unpack"
    _expect(_is_mask(mask) and mask.dim() == 2, f"{what}: mask must be uint8/bool [B, N]")
    B, N = mask.shape
    _expect(q.dim() == 4 and tuple(q.shape[:2]) == (B, N) and q.dtype in (torch.float16, torch.bfloat16),
            f"{what}: q must be fp16/bf16 [{B}, {N}, H, d]")
    for t in (k, v):
        _expect(t.shape == q.shape and t.dtype == q.dtype, f"{what}: k and v must match q's shape and dtype")
    _expect(y.shape == q.shape and y.dtype in (q.dtype, torch.float32),
            f"{what}: y must be {tuple(q.shape)} in q's dtype or fp32")
    _check_cu(cu_seqlens, B, what)
    _check_err(dev_error, what)
    _disjoint([y, cu_seqlens], [mask, q, k, v], what)
    _disjoint([y], [cu_seqlens], what)
    _require_cuda(mask, q, k, v, y, cu_seqlens, dev_error)
    H, d = q.shape[2], q.shape[3]
    st = lib().rra_pack_attend_unpack(_ptr(mask), _ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(cu_seqlens), B, N, H, d,
                                      float(softmax_scale), _DT[q.dtype], _DT[y.dtype], _ptr(dev_error),
                                      _stream(stream))
    _check(st, what)


def rra_l2_mask(x: torch.Tensor, keep_mask: torch.Tensor, k_keep: Optional[torch.Tensor] = None,
                threshold_sq: float = 0.0, prev_mask: Optional[torch.Tensor] = None, stream=None) -> None:
    """Threshold-l2 selection: embeddings x [B, N, C] (fp16/bf16) -> keep_mask uint8 [B, N] (CLS kept).

    With k_keep (int32 [B]) image b keeps its k_b highest-norm candidates; otherwise every
    candidate whose squared norm reaches threshold_sq.  Candidates: n >= 1 kept in prev_mask
    (which may be keep_mask itself)."""
    what = "rra_l2_mask"
    _expect(x.dim() == 3 and x.dtype in (torch.float16, torch.bfloat16), f"{what}: x must be fp16/bf16 [B, N, C]")
    B, N, C = x.shape
    _expect(keep_mask.dtype == torch.uint8 and tuple(keep_mask.shape) == (B, N),
            f"{what}: keep_mask must be uint8 [{B}, {N}]")
    if k_keep is not None:
        _expect(k_keep.dtype == torch.int32 and k_keep.numel() >= B, f"{what}: k_keep must be int32 [{B}]")
    if prev_mask is not None:
        _expect(_is_mask(prev_mask) and tuple(prev_mask.shape) == (B, N), f"{what}: prev_mask must be uint8 [{B}, {N}]")
    _disjoint([keep_mask], [x, k_keep], what)
    if prev_mask is not None and prev_mask.data_ptr() != keep_mask.data_ptr():
        _disjoint([keep_mask], [prev_mask], what)
    _require_cuda(x, keep_mask, k_keep, prev_mask)
    st = lib().rra_l2_mask(_ptr(x), B, N, C, _DT[x.dtype], _ptr(k_keep), float(threshold_sq), _ptr(prev_mask),
                           _ptr(keep_mask), _stream(stream))
    _check(st, what)


RRA_ACT_NONE, RRA_ACT_GELU = 0, 1


def rra_linear(x: torch.Tensor, w: torch.Tensor, outs: Sequence[torch.Tensor], bias: Optional[torch.Tensor] = None,
               residual: Optional[torch.Tensor] = None, act: int = RRA_ACT_NONE, m_dev: Optional[torch.Tensor] = None,
               dev_error: Optional[torch.Tensor] = None, stream=None) -> None:
    """outs = split(act(x w^T + bias) + residual): x bf16 [M, K], w bf16 [N, K], bias [N], residual
    [M, N], outs n_outs tensors bf16 [M, N / n_outs].  With m_dev (int32 device word) only rows
    [0, min(M, m_dev)) are computed."""
    what = "rra_linear"
    bf = torch.bfloat16
    _expect(x.dim() == 2 and x.dtype == bf and w.dim() == 2 and w.dtype == bf, f"{what}: x, w must be bf16 2-D")
    M, K = x.shape
    N = w.shape[0]
    _expect(w.shape[1] == K, f"{what}: w must be [N, {K}]")
    outs = list(outs)
    _expect(1 <= len(outs) <= 4 and N % len(outs) == 0, f"{what}: 1..4 outputs splitting N = {N}")
    for o in outs:
        _expect(o.dtype == bf and tuple(o.shape) == (M, N // len(outs)), f"{what}: outs must be bf16 [{M}, {N // len(outs)}]")
    if bias is not None:
        _expect(bias.dtype == bf and bias.numel() == N, f"{what}: bias must be bf16 [{N}]")
    if residual is not None:
        _expect(residual.dtype == bf and tuple(residual.shape) == (M, N), f"{what}: residual must be bf16 [{M}, {N}]")
    if m_dev is not None:
        _expect(m_dev.dtype == torch.int32 and m_dev.numel() >= 1, f"{what}: m_dev must be an int32 word")
    _check_err(dev_error, what)
    _disjoint(outs, [x, w, bias], what)
    if residual is not None and not (len(outs) == 1 and outs[0].data_ptr() == residual.data_ptr()):
        _disjoint(outs, [residual], what)
    for i, o in enumerate(outs):
        _disjoint([o], outs[:i], what)
    _require_cuda(x, w, bias, residual, m_dev, dev_error, *outs)
    arr = (ctypes.c_void_p * len(outs))(*[o.data_ptr() for o in outs])
    st = lib().rra_linear(_ptr(x), _ptr(w), _ptr(bias), _ptr(residual), arr, len(outs), M, _ptr(m_dev), N, K, act,
                          _ptr(dev_error), _stream(stream))
    _check(st, what)


def rra_layernorm(x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor, y: torch.Tensor, eps: float = 1e-6,
                  m_dev: Optional[torch.Tensor] = None, stream=None) -> None:
    """y = LayerNorm(x) * gamma + beta per row: x, y bf16 [M, C]; with m_dev only rows [0, min(M, m_dev))."""
    what = "rra_layernorm"
    bf = torch.bfloat16
    _expect(x.dim() == 2 and x.dtype == bf, f"{what}: x must be bf16 [M, C]")
    M, C = x.shape
    _expect(y.dtype == bf and tuple(y.shape) == (M, C), f"{what}: y must be bf16 [{M}, {C}]")
    _expect(gamma.dtype == bf and beta.dtype == bf and gamma.numel() == C and beta.numel() == C,
            f"{what}: gamma, beta must be bf16 [{C}]")
    if m_dev is not None:
        _expect(m_dev.dtype == torch.int32 and m_dev.numel() >= 1, f"{what}: m_dev must be an int32 word")
    _disjoint([y], [x, gamma, beta], what)
    _require_cuda(x, gamma, beta, y, m_dev)
    st = lib().rra_layernorm(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(y), M, _ptr(m_dev), C, float(eps), _stream(stream))
    _check(st, what)


class DeitBlock:
    """A transformer block on packed token rows (weights and activation buffers): LN1, the fused
    QKV projection split into packed Q, K, V, the ragged attention, the output projection with its
    residual, LN2, FC1 with GELU and FC2 with its residual.  `weights` maps the nn.Linear /
    nn.LayerNorm names (qkv_w [3C, C], qkv_b, proj_w [C, C], proj_b, fc1_w [4C, C], fc1_b, fc2_w
    [C, 4C], fc2_b, ln1_g, ln1_b, ln2_g, ln2_b) to bf16 device tensors."""

    STAGES = ("ln1", "qkv", "attend", "proj", "ln2", "fc1", "fc2")

    def __init__(self, weights, capacity: int, H: int, eps: float = 1e-6, device="cuda"):
        C = H * 64
        self.w, self.C, self.H, self.cap, self.eps = weights, C, H, capacity, eps
        e = lambda n: torch.empty(capacity, n, dtype=torch.bfloat16, device=device)
        self.h, self.q, self.k, self.v, self.a, self.x1, self.h2 = (e(C) for _ in range(7))
        self.m = e(4 * C)
        self.y = e(C)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def stage(self, name: str, x: torch.Tensor, cu: torch.Tensor, B: int, max_seqlen: int, stream=None):
        """Enqueue one of STAGES on `stream` (rows [0, cu[B]) of the capacity-row buffers)."""
        w, T = self.w, cu[B:B + 1]
        if name == "ln1":
            rra_layernorm(x, w["ln1_g"], w["ln1_b"], self.h, self.eps, m_dev=T, stream=stream)
        elif name == "qkv":
            rra_linear(self.h, w["qkv_w"], [self.q, self.k, self.v], bias=w["qkv_b"], m_dev=T, dev_error=self.err,
                       stream=stream)
        elif name == "attend":
            sh = (self.cap, self.H, 64)
            rra_attend(self.q.view(sh), self.k.view(sh), self.v.view(sh), self.a.view(sh), cu, max_seqlen=max_seqlen,
                       dev_error=self.err, stream=stream)
        elif name == "proj":
            rra_linear(self.a, w["proj_w"], [self.x1], bias=w["proj_b"], residual=x, m_dev=T, dev_error=self.err,
                       stream=stream)
        elif name == "ln2":
            rra_layernorm(self.x1, w["ln2_g"], w["ln2_b"], self.h2, self.eps, m_dev=T, stream=stream)
        elif name == "fc1":
            rra_linear(self.h2, w["fc1_w"], [self.m], bias=w["fc1_b"], act=RRA_ACT_GELU, m_dev=T, dev_error=self.err,
                       stream=stream)
        elif name == "fc2":
            rra_linear(self.m, w["fc2_w"], [self.y], bias=w["fc2_b"], residual=self.x1, m_dev=T, dev_error=self.err,
                       stream=stream)
        else:
            raise ValueError(name)

    def __call__(self, x: torch.Tensor, cu: torch.Tensor, B: int, max_seqlen: int, stream=None) -> torch.Tensor:
        """The block on packed rows x [capacity, C] whose first cu[B] rows are the kept tokens of B
        images (cu_seqlens of the pack); returns self.y (rows past cu[B] are not written)."""
        _expect(x.dtype == torch.bfloat16 and tuple(x.shape) == (self.cap, self.C),
                f"DeitBlock: x must be bf16 [{self.cap}, {self.C}]")
        for name in self.STAGES:
            self.stage(name, x, cu, B, max_seqlen, stream)
        return self.y


# ------------------------------------------------------------------------------------ whole call

class Buffers:
    """Device buffers for one pack-attend-unpack call at capacity B*N (reused across calls)."""

    def __init__(self, B: int, N: int, H: int, dtype: torch.dtype, out_dtype: Optional[torch.dtype] = None,
                 device="cuda"):
        cap = max(1, B * N)
        self.B, self.N, self.H, self.capacity = B, N, H, cap
        self.packed = [torch.empty(cap, H, 64, dtype=dtype, device=device) for _ in range(3)]
        od = out_dtype or dtype
        self.o = torch.empty(cap, H, 64, dtype=od, device=device)
        self.y = torch.empty(B, N, H, 64, dtype=od, device=device)
        self.cu = torch.empty(B + 1, dtype=torch.int32, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)


def forward(mask: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, bufs: Buffers,
            softmax_scale: float = 0.0, stream=None, fused: bool = False) -> torch.Tensor:
    """One pruning stage: pack the kept tokens of q/k/v, attend per image and head, unpack to padded.

    Enqueued on `stream` without any host synchronisation; the padded result is bufs.y (pruned
    rows zero).  fused=True runs the same call as the single launch rra_pack_attend_unpack
    (bufs.cu is written, the packed buffers are not used)."""
    _expect(tuple(mask.shape) == (bufs.B, bufs.N), f"forward: mask {tuple(mask.shape)} != buffers' [{bufs.B}, {bufs.N}]")
    for t in (q, k, v):
        _expect(tuple(t.shape) == (bufs.B, bufs.N, bufs.H, 64) and t.dtype == bufs.packed[0].dtype,
                f"forward: q/k/v must be [{bufs.B}, {bufs.N}, {bufs.H}, 64] {bufs.packed[0].dtype}")
    if fused:
        rra_pack_attend_unpack(mask, q, k, v, bufs.y, bufs.cu, softmax_scale=softmax_scale, dev_error=bufs.err,
                               stream=stream)
        return bufs.y
    rra_pack(mask, [q, k, v], bufs.packed, bufs.cu, dev_error=bufs.err, stream=stream)
    rra_attend(bufs.packed[0], bufs.packed[1], bufs.packed[2], bufs.o, bufs.cu, max_seqlen=mask.shape[1],
               softmax_scale=softmax_scale, dev_error=bufs.err, stream=stream)
    rra_unpack(bufs.o, bufs.cu, mask, bufs.y, fill_mode=0, dev_error=bufs.err, stream=stream)
    return bufs.y


class HostStream:
    """Pack-attend-unpack of a batch held in pinned host memory, streamed through the GPU in chunks
    of images (images are independent, so a chunk is a complete call of its own).

    Per chunk: its Q, K, V and masks go host -> device on one stream, the chunk's calls (one per
    pruning stage, through the same kernels as `forward`) run on a second, and each stage's padded
    output goes device -> host on a third.  Two sets of device buffers alternate, so the copies of
    chunk j+1 in, chunk j's kernels and chunk j-1's results out overlap: PCIe carries both
    directions at once and the kernels hide behind the copies.  Only copies, events and stream
    waits are issued here; every step of the path runs in the library's kernels.
    """

    def __init__(self, B: int, N: int, H: int, dtype: torch.dtype, stages: int = 1, chunk: int = 128,
                 out_dtype: Optional[torch.dtype] = None, fused: bool = True, device="cuda"):
        _expect(B >= 1 and N >= 1 and H >= 1 and stages >= 1 and chunk >= 1, "HostStream: sizes must be positive")
        self.B, self.N, self.H, self.stages, self.fused = B, N, H, stages, fused
        self.chunk = min(chunk, B)
        od = out_dtype or dtype
        self.dtype, self.out_dtype = dtype, od
        c = self.chunk
        self.sets = []
        for _ in range(2):
            st = {"qkv": [torch.empty(c, N, H, 64, dtype=dtype, device=device) for _ in range(3)],
                  "masks": [torch.empty(c, N, dtype=torch.uint8, device=device) for _ in range(stages)],
                  "ys": [torch.empty(c, N, H, 64, dtype=od, device=device) for _ in range(stages)],
                  "cu": torch.empty(c + 1, dtype=torch.int32, device=device),
                  "in_done": torch.cuda.Event(), "run_done": torch.cuda.Event(), "out_done": torch.cuda.Event()}
            if not fused:
                cap = c * N
                st["packed"] = [torch.empty(cap, H, 64, dtype=dtype, device=device) for _ in range(3)]
                st["o"] = torch.empty(cap, H, 64, dtype=od, device=device)
            self.sets.append(st)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(device=device) for _ in range(3))
        self.start = torch.cuda.Event()

    def __call__(self, masks: Sequence[torch.Tensor], q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 outs: Sequence[torch.Tensor], softmax_scale: float = 0.0, stream=None) -> None:
        """masks: `stages` uint8 [B', N]; q, k, v: [B', N, H, 64]; outs: `stages` [B', N, H, 64] in the
        output dtype (all pinned host tensors, B' <= B).  The work starts after what is already on
        `stream`, and `stream` waits for the last copy back, so an event or a synchronisation on
        `stream` covers the whole call.  Device errors land in self.err."""
        stream = stream or torch.cuda.current_stream()
        Bp = q.shape[0]
        _expect(len(masks) == self.stages and len(outs) == self.stages, f"HostStream: {self.stages} masks and outputs expected")
        _expect(1 <= Bp <= self.B, f"HostStream: batch {Bp} outside [1, {self.B}]")
        for t in (q, k, v):
            _expect(t.device.type == "cpu" and t.is_pinned() and t.is_contiguous() and t.dtype == self.dtype
                    and tuple(t.shape) == (Bp, self.N, self.H, 64), "HostStream: q/k/v must be pinned host [B', N, H, 64]")
        for m in masks:
            _expect(m.device.type == "cpu" and m.is_pinned() and m.is_contiguous() and m.dtype == torch.uint8
                    and tuple(m.shape) == (Bp, self.N), "HostStream: masks must be pinned host uint8 [B', N]")
        for o in outs:
            _expect(o.device.type == "cpu" and o.is_pinned() and o.is_contiguous() and o.dtype == self.out_dtype
                    and tuple(o.shape) == (Bp, self.N, self.H, 64), "HostStream: outputs must be pinned host [B', N, H, 64]")
        self.start.record(stream)
        for s in (self.s_in, self.s_run, self.s_out):
            s.wait_event(self.start)
        chunks = list(range(0, Bp, self.chunk))
        for j, b0 in enumerate(chunks):
            st = self.sets[j % 2]
            b1 = min(Bp, b0 + self.chunk)
            n = b1 - b0
            if j >= 2:
                self.s_in.wait_event(st["run_done"])   # chunk j-2's kernels are done with these inputs
            with torch.cuda.stream(self.s_in):
                for d, h in zip(st["qkv"], (q, k, v)):
                    d[:n].copy_(h[b0:b1], non_blocking=True)
                for d, h in zip(st["masks"], masks):
                    d[:n].copy_(h[b0:b1], non_blocking=True)
                st["in_done"].record(self.s_in)
            self.s_run.wait_event(st["in_done"])
            if j >= 2:
                self.s_run.wait_event(st["out_done"])  # chunk j-2's results have left these outputs
            qd, kd, vd = (t[:n] for t in st["qkv"])
            for s in range(self.stages):
                m, y = st["masks"][s][:n], st["ys"][s][:n]
                if self.fused:
                    rra_pack_attend_unpack(m, qd, kd, vd, y, st["cu"][:n + 1], softmax_scale=softmax_scale,
                                           dev_error=self.err, stream=self.s_run)
                else:
                    pk = [t[:n * self.N] for t in st["packed"]]
                    o = st["o"][:n * self.N]
                    rra_pack(m, [qd, kd, vd], pk, st["cu"][:n + 1], dev_error=self.err, stream=self.s_run)
                    rra_attend(pk[0], pk[1], pk[2], o, st["cu"][:n + 1], max_seqlen=self.N,
                               softmax_scale=softmax_scale, dev_error=self.err, stream=self.s_run)
                    rra_unpack(o, st["cu"][:n + 1], m, y, fill_mode=0, dev_error=self.err, stream=self.s_run)
            st["run_done"].record(self.s_run)
            self.s_out.wait_event(st["run_done"])
            with torch.cuda.stream(self.s_out):
                for s in range(self.stages):
                    outs[s][b0:b1].copy_(st["ys"][s][:n], non_blocking=True)
                st["out_done"].record(self.s_out)
        for st in self.sets[:min(2, len(chunks))]:
            stream.wait_event(st["out_done"])

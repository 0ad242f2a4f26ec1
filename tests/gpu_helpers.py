"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and the float64
oracle on the same seeded inputs, and compare them."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O
from ragged_varlen_attention_rra_b200 import rra

ATOL = 2e-3  # absolute bound on |O_gpu - O_oracle| with fp32 accumulation


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def raw(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.float16, torch.bfloat16):
        return bits16(t)
    return t.numpy()


def half_ulp(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Half a unit in the last place of |x| in a 16-bit output type (rounding bound of the store)."""
    mant = {torch.bfloat16: 7, torch.float16: 10}[dtype]
    min_exp = {torch.bfloat16: -126, torch.float16: -14}[dtype]
    ax = np.maximum(np.abs(x), np.finfo(np.float64).tiny)
    e = np.maximum(np.floor(np.log2(ax)), min_exp)
    return 0.5 * np.exp2(e - mant)


def tolerance(oracle: np.ndarray, out_dtype: torch.dtype) -> np.ndarray:
    if out_dtype == torch.float32:
        return np.full(oracle.shape, ATOL)
    return ATOL + 2.0 * half_ulp(oracle, out_dtype)  # both binades around a boundary


class GpuRun:
    """Device copies of one workload stage and the outputs of pack / attend / unpack."""

    def __init__(self, w, stage: int = 0, out_dtype: torch.dtype | None = None, capacity: int | None = None,
                 fill_packed: float | None = None, fill_out: float | None = None, guard: int = 0):
        dev = "cuda"
        self.w = w
        self.mask = w.masks[stage].to(dev)
        self.q, self.k, self.v = (t.to(dev) for t in (w.q, w.k, w.v))
        B, N, H = w.B, w.N, w.H
        cap = capacity if capacity is not None else max(1, B * N)
        self.capacity = cap
        od = out_dtype or w.q.dtype
        self.out_dtype = od
        self.guard = guard

        def alloc(shape, dtype, fill):
            t = torch.empty((shape[0] + guard,) + tuple(shape[1:]), dtype=dtype, device=dev)
            if fill is None:
                t.zero_()
            else:
                t.fill_(fill)
            return t

        self.packed_full = [alloc((cap, H, 64), w.q.dtype, fill_packed) for _ in range(3)]
        self.packed = [t[:cap] for t in self.packed_full]
        self.o_full = alloc((cap, H, 64), od, fill_out)
        self.o = self.o_full[:cap]
        self.y_full = alloc((B * N, H, 64), od, fill_out)
        self.y = self.y_full[:B * N].view(B, N, H, 64)
        self.cu = torch.full((B + 2,), -7, dtype=torch.int32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def pack(self):
        rra.rra_pack(self.mask, [self.q, self.k, self.v], self.packed, self.cu[:-1], capacity=self.capacity,
                     dev_error=self.err)

    def attend(self):
        rra.rra_attend(self.packed[0], self.packed[1], self.packed[2], self.o, self.cu[:-1],
                       max_seqlen=self.w.N, dev_error=self.err)

    def unpack(self, fill_mode=0):
        rra.rra_unpack(self.o, self.cu[:-1], self.mask, self.y, fill_mode=fill_mode, dev_error=self.err)

    def run(self):
        self.pack()
        self.attend()
        self.unpack()
        torch.cuda.synchronize()
        return self

    def error(self) -> int:
        return rra.rra_get_device_error(self.err)


def oracle_stage(w, stage: int = 0, full_attention: bool = True):
    """Oracle pack (+ attention when full_attention) of one stage."""
    mask = w.masks[stage]
    qp, cu = O.pack(mask, w.q)
    kp, _ = O.pack(mask, w.k)
    vp, _ = O.pack(mask, w.v)
    res = {"cu": cu, "qp": qp, "kp": kp, "vp": vp, "T": int(cu[-1])}
    if full_attention:
        res["o"] = O.attend(qp, kp, vp, cu, w.H, 64, dtype=w.dtype)
    return res


def compare_attention(gpu_o: torch.Tensor, oracle_o: np.ndarray, out_dtype: torch.dtype):
    g = gpu_o.detach().cpu().double().numpy()
    err = np.abs(g - oracle_o)
    tol = tolerance(oracle_o, out_dtype)
    bad = err > tol
    return float(err.max()) if err.size else 0.0, int(bad.sum()), np.isfinite(g).all()


def oracle_attention_threaded(w, stage: int = 0, threads: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """The oracle's float64 attention over every kept row of one stage, one image per task on a
    thread pool (the oracle's C calls release the GIL), reassembled in packed order: (O [T, H, d],
    cu_seqlens)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    mask = w.masks[stage]
    cu = O.cu_seqlens(mask)
    T = int(cu[-1])
    out = np.zeros((T, w.H, 64), dtype=np.float64)

    def one(b):
        m = mask[b:b + 1]
        qp, c = O.pack(m, w.q[b:b + 1])
        kp, _ = O.pack(m, w.k[b:b + 1])
        vp, _ = O.pack(m, w.v[b:b + 1])
        out[cu[b]:cu[b + 1]] = O.attend(qp, kp, vp, c, w.H, 64, dtype=w.dtype)

    n = threads or max(1, len(os.sched_getaffinity(0)))
    with ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(one, range(w.B)))
    return out, cu

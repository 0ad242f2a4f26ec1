"""The C-ABI library without a GPU: it loads, exports every symbol include/rra.h declares, and
its host-side argument validation answers before any CUDA call is made."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

from ragged_varlen_attention_rra_b200 import build as rra_build
from ragged_varlen_attention_rra_b200 import rra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rra.h")


@pytest.fixture(scope="module")
def L():
    rra_build.build()
    return rra.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rra_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for required in ("rra_pack", "rra_attend", "rra_unpack", "rra_pack_attend_unpack", "rra_attend_workspace_size",
                     "rra_get_device_error", "rra_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", rra.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (rra_\w+)", out.stdout))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(L, n)


def test_status_strings(L):
    for code, name in [(0, "RRA_OK"), (1, "RRA_ERR_INVALID_ARG"), (2, "RRA_ERR_UNSUPPORTED"), (3, "RRA_ERR_CUDA"),
                       (4, "RRA_ERR_CAPACITY"), (5, "RRA_ERR_TIMEOUT"), (6, "RRA_ERR_BAD_SEQLENS")]:
        assert rra.rra_status_string(code) == name
    assert rra.rra_status_string(99) == "RRA_ERR_UNKNOWN"
    assert L.rra_version() >= 100


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails before any use


def _pack(L, mask=FAKE, B=2, N=8, H=1, d=64, dt=1, n=3, src=True, dst=True, cap=16, cu=FAKE, srcp=FAKE, dstp=FAKE):
    sa = (ctypes.c_void_p * 3)(srcp, srcp, srcp) if src else None
    da = (ctypes.c_void_p * 3)(dstp, dstp, dstp) if dst else None
    return L.rra_pack(mask, B, N, H, d, dt, n, sa, da, cap, cu, None, None)


def test_pack_validation(L):
    assert _pack(L, mask=None) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, cu=None) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, src=False) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, B=-1) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, N=0) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, n=0) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, n=4) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, cap=0) == rra.RRA_ERR_INVALID_ARG
    assert _pack(L, dt=7) == rra.RRA_ERR_UNSUPPORTED
    assert _pack(L, d=3) == rra.RRA_ERR_UNSUPPORTED          # 6-byte rows cannot move as 16-byte vectors
    assert _pack(L, srcp=FAKE + 8) == rra.RRA_ERR_INVALID_ARG  # misaligned
    assert _pack(L, B=70000) == rra.RRA_ERR_UNSUPPORTED


def _attend(L, q=FAKE, o=FAKE, cu=FAKE, B=2, H=1, d=64, ms=8, cap=16, scale=0.0, idt=1, odt=1, ws=0):
    return L.rra_attend(q, q, q, o, cu, B, H, d, ms, cap, scale, idt, odt, None, ws, None, None)


def test_attend_validation(L):
    assert _attend(L, q=None) == rra.RRA_ERR_INVALID_ARG
    assert _attend(L, cu=None) == rra.RRA_ERR_INVALID_ARG
    assert _attend(L, B=-1) == rra.RRA_ERR_INVALID_ARG
    assert _attend(L, cap=0) == rra.RRA_ERR_INVALID_ARG
    assert _attend(L, ms=-1) == rra.RRA_ERR_INVALID_ARG
    assert _attend(L, q=FAKE + 4) == rra.RRA_ERR_INVALID_ARG
    assert _attend(L, d=128) == rra.RRA_ERR_UNSUPPORTED
    assert _attend(L, idt=2, odt=2) == rra.RRA_ERR_UNSUPPORTED   # fp32 inputs are not a tensor-core type here
    assert _attend(L, idt=0, odt=1) == rra.RRA_ERR_UNSUPPORTED   # output fp16 in or fp32 only
    assert _attend(L, B=100000) == rra.RRA_ERR_UNSUPPORTED
    assert _attend(L, B=8193) == rra.RRA_ERR_UNSUPPORTED
    assert _attend(L, scale=float("nan")) == rra.RRA_ERR_INVALID_ARG
    assert L.rra_attend_workspace_size(64, 12, 197) == 0


def test_unpack_validation(L):
    f = L.rra_unpack
    assert f(None, FAKE, FAKE, 2, 8, 1, 64, 1, 0, 16, FAKE, None, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 2, 8, 1, 64, 1, 2, 16, FAKE, None, None) == rra.RRA_ERR_INVALID_ARG  # fill_mode
    assert f(FAKE, FAKE, FAKE, 2, 8, 1, 64, 9, 0, 16, FAKE, None, None) == rra.RRA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 2, 8, 1, 64, 1, 0, 16, FAKE + 2, None, None) == rra.RRA_ERR_INVALID_ARG


def test_fused_validation(L):
    f = L.rra_pack_attend_unpack
    assert f(None, FAKE, FAKE, FAKE, FAKE, None, 2, 8, 1, 64, 0.0, 1, 1, None, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE + 8, None, 2, 8, 1, 64, 0.0, 1, 1, None, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 8, 1, 32, 0.0, 1, 1, None, None) == rra.RRA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 1025, 1, 64, 0.0, 1, 1, None, None) == rra.RRA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 4097, 8, 1, 64, 0.0, 1, 1, None, None) == rra.RRA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 8, 1, 64, 0.0, 2, 2, None, None) == rra.RRA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 1024, 16384, 64, 0.0, 1, 1, None, None) == rra.RRA_ERR_UNSUPPORTED


def test_l2_mask_validation(L):
    f = L.rra_l2_mask
    assert f(None, 2, 8, 16, 1, None, 1.0, None, FAKE, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, 2, 8, 16, 1, None, 1.0, None, None, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE + 8, 2, 8, 16, 1, None, 1.0, None, FAKE, None) == rra.RRA_ERR_INVALID_ARG  # misaligned
    assert f(FAKE, -1, 8, 16, 1, None, 1.0, None, FAKE, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, 2, 0, 16, 1, None, 1.0, None, FAKE, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, 2, 8, 12, 1, None, 1.0, None, FAKE, None) == rra.RRA_ERR_UNSUPPORTED  # C not a multiple of 8
    assert f(FAKE, 2, 8, 16, 2, None, 1.0, None, FAKE, None) == rra.RRA_ERR_UNSUPPORTED  # fp32 embeddings
    assert f(FAKE, 2, 4097, 16, 1, None, 1.0, None, FAKE, None) == rra.RRA_ERR_UNSUPPORTED
    assert f(FAKE, 2, 8, 16, 1, None, float("nan"), None, FAKE, None) == rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, 0, 8, 16, 1, None, 1.0, None, FAKE, None) == rra.RRA_OK  # nothing to do, no launch


def test_get_device_error_validation(L):
    out = ctypes.c_int32(0)
    assert L.rra_get_device_error(None, None, ctypes.byref(out)) == rra.RRA_ERR_INVALID_ARG
    assert L.rra_get_device_error(FAKE, None, None) == rra.RRA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    code = ("import os, sys; os.environ['RRA_LIBRARY'] = %r\n"
            "sys.path.insert(0, %r)\n"
            "from ragged_varlen_attention_rra_b200 import rra\n"
            "try:\n    rra.rra_status_string(0)\nexcept ImportError as e:\n    print('RAISED', e); sys.exit(0)\n"
            "sys.exit(1)\n") % (str(tmp_path / "nope.so"), ROOT)
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert p.returncode == 0 and "RAISED" in p.stdout, p.stdout + p.stderr


def test_binding_matches_header_arity(L):
    """Every declared call is bound in Python with as many arguments as the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    for name, params in re.findall(r"\b(rra_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text):
        params = params.strip()
        arity = 0 if params in ("", "void") else params.count(",") + 1
        fn = getattr(L, name)
        assert fn.argtypes is not None and len(fn.argtypes) == arity, (name, arity, fn.argtypes)


try:
    from hypothesis import given, settings, strategies as st

    bad_field = st.sampled_from(["B", "H", "d", "cap", "ms", "align", "idt", "odt", "scale", "null"])

    @settings(max_examples=200, deadline=None)
    @given(bad=bad_field, B=st.integers(0, 8192), H=st.integers(1, 64), ms=st.integers(0, 4096),
           cap=st.integers(1, 1 << 20), odt_same=st.booleans(), idt=st.sampled_from([0, 1]))
    def test_attend_rejects_any_invalid_field_before_launch(L, bad, B, H, ms, cap, odt_same, idt):
        """Whatever else the arguments are, one invalid field makes rra_attend return an error code
        without touching a device (these calls never reach a launch, on any machine)."""
        args = dict(q=FAKE, o=FAKE, cu=FAKE, B=B, H=H, d=64, ms=ms, cap=cap, scale=0.0, idt=idt,
                    odt=idt if odt_same else 2)
        if bad == "B":
            args["B"] = -1 - B
        elif bad == "H":
            args["H"] = -H
        elif bad == "d":
            args["d"] = 64 + H
        elif bad == "cap":
            args["cap"] = -cap
        elif bad == "ms":
            args["ms"] = -1 - ms
        elif bad == "align":
            args["q"] = FAKE + 2 * (1 + H % 7)
        elif bad == "idt":
            args["idt"] = 2 + H % 3
        elif bad == "odt":
            args["odt"] = 1 - idt  # the other 16-bit type
        elif bad == "scale":
            args["scale"] = float("nan")
        else:
            args["cu"] = None
        st_code = _attend(L, **args)
        assert st_code in (rra.RRA_ERR_INVALID_ARG, rra.RRA_ERR_UNSUPPORTED), (bad, args, st_code)
except ImportError:  # pragma: no cover
    pass


def test_overlapping_output_is_rejected_before_launch(L):
    """An output whose bytes intersect an input's is refused with RRA_ERR_INVALID_ARG before any
    CUDA call (every other argument here is valid, so only the overlap check can answer)."""
    # rra_attend, o == q
    assert _attend(L, q=FAKE, o=FAKE) == rra.RRA_ERR_INVALID_ARG
    # o starts inside q (capacity 16 rows x 128 bytes of bf16 = 2048 bytes)
    assert _attend(L, q=FAKE, o=FAKE + 1024) == rra.RRA_ERR_INVALID_ARG
    # single launch: y overlaps v, or cu_seqlens overlaps q
    f = L.rra_pack_attend_unpack
    assert f(FAKE, 0x100000, 0x200000, 0x300000, 0x300000, None, 2, 8, 1, 64, 0.0, 1, 1, None, None) == \
        rra.RRA_ERR_INVALID_ARG
    assert f(FAKE, 0x100000, 0x200000, 0x300000, 0x400000, 0x100010, 2, 8, 1, 64, 0.0, 1, 1, None, None) == \
        rra.RRA_ERR_INVALID_ARG
    # unpack: dst overlaps the mask
    assert L.rra_unpack(0x100000, 0x200000, 0x300000, 2, 8, 1, 64, 1, 0, 16, 0x300000, None, None) == \
        rra.RRA_ERR_INVALID_ARG
    # pack: a destination overlaps a source
    assert _pack(L, srcp=0x100000, dstp=0x100000, cu=0x900000) == rra.RRA_ERR_INVALID_ARG
    # l2 mask: keep_mask overlaps the embeddings; keep_mask partially overlapping prev_mask
    g = L.rra_l2_mask
    assert g(0x100000, 2, 8, 16, 1, None, 1.0, None, 0x100000, None) == rra.RRA_ERR_INVALID_ARG
    assert g(0x100000, 2, 8, 16, 1, None, 1.0, 0x200008, 0x200000, None) == rra.RRA_ERR_INVALID_ARG


class _T:
    """CPU tensors with the shapes of a call: the binding's shape and dtype checks run before its
    device check, so every mismatch below is reported without a GPU."""

    def __init__(self, B=2, N=8, H=2, dt=None):
        import torch
        dt = dt or torch.bfloat16
        self.torch = torch
        self.mask = torch.ones(B, N, dtype=torch.uint8)
        self.q, self.k, self.v = (torch.zeros(B, N, H, 64, dtype=dt) for _ in range(3))
        self.y = torch.zeros(B, N, H, 64, dtype=dt)
        self.cu = torch.zeros(B + 1, dtype=torch.int32)
        self.packed = [torch.zeros(B * N, H, 64, dtype=dt) for _ in range(3)]
        self.o = torch.zeros(B * N, H, 64, dtype=dt)


def _raises(fn, match):
    with pytest.raises(ValueError, match=match):
        fn()


def test_binding_checks_shapes_and_dtypes():
    t = _T()
    torch = t.torch
    # a well-formed call on CPU tensors reaches the device check
    _raises(lambda: rra.rra_pack_attend_unpack(t.mask, t.q, t.k, t.v, t.y, t.cu), "CUDA")
    _raises(lambda: rra.rra_attend(*t.packed, t.o, t.cu, max_seqlen=8), "CUDA")
    # rra_attend: k/v/o shape or dtype different from q, cu_seqlens of the wrong type
    _raises(lambda: rra.rra_attend(t.packed[0], t.packed[1][:5], t.packed[2], t.o, t.cu, 8), "k and v")
    _raises(lambda: rra.rra_attend(t.packed[0], t.packed[1].half(), t.packed[2], t.o, t.cu, 8), "k and v")
    _raises(lambda: rra.rra_attend(*t.packed, t.o[:, :1], t.cu, 8), "o must be")
    _raises(lambda: rra.rra_attend(*t.packed, t.o.half(), t.cu, 8), "o must be")
    _raises(lambda: rra.rra_attend(*t.packed, t.o, t.cu.long(), 8), "cu_seqlens")
    _raises(lambda: rra.rra_attend(t.packed[0], t.packed[1], t.packed[2], t.packed[0], t.cu, 8), "overlaps")
    # rra_unpack: capacity beyond packed rows, dst shape or dtype, mask dtype, short cu_seqlens
    _raises(lambda: rra.rra_unpack(t.o, t.cu, t.mask, t.y, capacity=t.o.shape[0] + 1), "capacity")
    _raises(lambda: rra.rra_unpack(t.o, t.cu, t.mask, t.y[:1]), "dst must be")
    _raises(lambda: rra.rra_unpack(t.o, t.cu, t.mask, t.y.float()), "dst must be")
    _raises(lambda: rra.rra_unpack(t.o, t.cu, t.mask.int(), t.y), "mask")
    _raises(lambda: rra.rra_unpack(t.o, t.cu[:2], t.mask, t.y), "cu_seqlens")
    # rra_pack: destination row size, destination dtype, capacity, source shapes
    _raises(lambda: rra.rra_pack(t.mask, [t.q], [t.o[:, :1]], t.cu), "destinations")
    _raises(lambda: rra.rra_pack(t.mask, [t.q], [t.o.half()], t.cu), "destinations")
    _raises(lambda: rra.rra_pack(t.mask, [t.q], [t.o], t.cu, capacity=t.o.shape[0] + 1), "capacity")
    _raises(lambda: rra.rra_pack(t.mask, [t.q, t.k[:1]], t.packed[:2], t.cu), "sources")
    _raises(lambda: rra.rra_pack(t.mask[:1], [t.q], [t.o], t.cu), "sources")
    _raises(lambda: rra.rra_pack(t.mask, [t.q], [t.o, t.o], t.cu), "destinations")
    # single launch: y shape/dtype, k/v dtype, mask vs q, cu_seqlens length
    _raises(lambda: rra.rra_pack_attend_unpack(t.mask, t.q, t.k, t.v, t.y[:1]), "y must be")
    _raises(lambda: rra.rra_pack_attend_unpack(t.mask, t.q, t.k, t.v, t.y.half()), "y must be")
    _raises(lambda: rra.rra_pack_attend_unpack(t.mask, t.q, t.k.half(), t.v, t.y), "k and v")
    _raises(lambda: rra.rra_pack_attend_unpack(t.mask[:, :4], t.q, t.k, t.v, t.y), "q must be")
    _raises(lambda: rra.rra_pack_attend_unpack(t.mask, t.q, t.k, t.v, t.y, t.cu[:1]), "cu_seqlens")
    _raises(lambda: rra.rra_pack_attend_unpack(t.mask, t.q, t.k, t.v, t.q), "overlaps")
    # rra_l2_mask: mask shape, k_keep dtype, prev_mask shape
    x = torch.zeros(2, 8, 16, dtype=torch.bfloat16)
    _raises(lambda: rra.rra_l2_mask(x, torch.zeros(2, 7, dtype=torch.uint8)), "keep_mask")
    _raises(lambda: rra.rra_l2_mask(x, t.mask, k_keep=torch.zeros(2, dtype=torch.int64)), "k_keep")
    _raises(lambda: rra.rra_l2_mask(x, t.mask, prev_mask=t.mask[:1]), "prev_mask")
    _raises(lambda: rra.rra_l2_mask(x, t.mask, prev_mask=t.mask), "CUDA")  # in place is allowed
    # forward: mask or q/k/v that do not match the buffers
    bufs = type("Bufs", (), {"B": 2, "N": 8, "H": 2, "packed": t.packed, "y": t.y, "cu": t.cu, "err": None,
                             "o": t.o})()
    _raises(lambda: rra.forward(t.mask[:1], t.q, t.k, t.v, bufs), "mask")
    _raises(lambda: rra.forward(t.mask, t.q[:, :, :1], t.k, t.v, bufs), "q/k/v")


def test_microbench_library_exports_and_validates():
    """The exponential-unit microbenchmark bench.py times builds, exports its two calls, and
    refuses bad arguments before any CUDA call."""
    path = rra_build.build_microbench()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (rra_mb_\w+)", out.stdout))
    assert {"rra_mb_ex2_launch", "rra_mb_ex2_per_block_iter"} <= exported
    mb = ctypes.CDLL(path)
    mb.rra_mb_ex2_launch.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    assert mb.rra_mb_ex2_per_block_iter() == 256 * 8
    assert mb.rra_mb_ex2_launch(None, 4, 16, None) != 0
    assert mb.rra_mb_ex2_launch(FAKE, 0, 16, None) != 0
    assert mb.rra_mb_ex2_launch(FAKE, 4, 0, None) != 0


def _linear(L, x=FAKE, w=FAKE, bias=None, res=None, outs=(FAKE,), M=256, m_dev=None, N=256, K=64, act=0):
    arr = (ctypes.c_void_p * len(outs))(*outs) if outs is not None else None
    return L.rra_linear(x, w, bias, res, arr, len(outs) if outs is not None else 0, M, m_dev, N, K, act, None, None)


def test_linear_validation_before_any_launch(L):
    """rra_linear refuses bad arguments before touching the device (these pointers are never
    dereferenced): every case below is refused, or has M = 0 and succeeds without a launch."""
    big = 1 << 30
    assert _linear(L, M=0) == rra.RRA_OK
    assert _linear(L, x=None) == rra.RRA_ERR_INVALID_ARG
    assert _linear(L, outs=None) == rra.RRA_ERR_INVALID_ARG
    assert _linear(L, act=7) == rra.RRA_ERR_INVALID_ARG
    assert _linear(L, x=FAKE + 8) == rra.RRA_ERR_INVALID_ARG            # misaligned
    assert _linear(L, K=96) == rra.RRA_ERR_UNSUPPORTED                  # K not a multiple of 64
    assert _linear(L, N=192) == rra.RRA_ERR_UNSUPPORTED                 # width not a multiple of 128
    assert _linear(L, N=192, outs=(FAKE + big, FAKE + 2 * big, FAKE + 3 * big)) == rra.RRA_ERR_UNSUPPORTED
    # outputs overlapping an input or each other
    assert _linear(L, outs=(FAKE,)) == rra.RRA_ERR_INVALID_ARG          # out == x
    assert _linear(L, x=FAKE, w=FAKE + big, outs=(FAKE + 2 * big, FAKE + 2 * big + 4096), N=512, M=64) \
        == rra.RRA_ERR_INVALID_ARG
    # the residual may be the single output itself, but must not partly overlap it
    assert _linear(L, M=0, res=FAKE + 2 * big, outs=(FAKE + 2 * big,)) == rra.RRA_OK
    assert _linear(L, M=4, x=FAKE, w=FAKE + big, res=FAKE + 2 * big + 16, outs=(FAKE + 2 * big,)) == rra.RRA_ERR_INVALID_ARG


def test_layernorm_validation_before_any_launch(L):
    f = ctypes.c_float
    big = 1 << 30
    ok = dict(x=FAKE, g=FAKE + big, b=FAKE + 2 * big, y=FAKE + 3 * big)

    def ln(x=ok["x"], g=ok["g"], b=ok["b"], y=ok["y"], M=8, C=768, eps=1e-6):
        return L.rra_layernorm(x, g, b, y, M, None, C, f(eps), None)
    assert ln(M=0) == rra.RRA_OK
    assert ln(x=None) == rra.RRA_ERR_INVALID_ARG
    assert ln(eps=0.0) == rra.RRA_ERR_INVALID_ARG
    assert ln(C=12) == rra.RRA_ERR_UNSUPPORTED
    assert ln(C=4096) == rra.RRA_ERR_UNSUPPORTED
    assert ln(y=FAKE) == rra.RRA_ERR_INVALID_ARG                        # y over x

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

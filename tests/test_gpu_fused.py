"""The single-launch call rra_pack_attend_unpack against the three-call path (bit-exact: same
arithmetic) and against the float64 oracle (pruned rows zero, kept rows within tolerance)."""
import numpy as np
import pytest
import torch

from gpu_helpers import ATOL, GpuRun, compare_attention, oracle_stage, raw, tolerance
from oracle import oracle as O
from ragged_varlen_attention_rra_b200 import rra
from ragged_varlen_attention_rra_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    rra.lib()


def run_fused(w, stage=0, out_dtype=None, guard=0, fill=None, dirty=False):
    mask = w.masks[stage].cuda()
    q, k, v = (t.cuda() for t in (w.q, w.k, w.v))
    od = out_dtype or w.q.dtype
    rows = w.B * w.N
    y_full = torch.empty((rows + guard, w.H, 64), dtype=od, device="cuda")
    y_full.fill_(float("nan") if fill is None else fill)
    y = y_full[:rows].view(w.B, w.N, w.H, 64)
    cu = torch.full((w.B + 2,), -7, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rra.rra_pack_attend_unpack(mask, q, k, v, y, cu[:-1], dev_error=err)
    torch.cuda.synchronize()
    assert rra.rra_get_device_error(err) == 0
    return y, y_full, cu


def check(w, stage=0, out_dtype=None, full_oracle=True, n_rows=256):
    y, _, cu = run_fused(w, stage, out_dtype)
    three = GpuRun(w, stage, out_dtype=out_dtype).run()
    assert three.error() == 0
    # identical to the three-call path, byte for byte (pruned rows zero in both)
    assert np.array_equal(raw(y), raw(three.y)), "fused output differs from pack+attend+unpack"
    ref_cu = O.cu_seqlens(w.masks[stage])
    assert np.array_equal(cu[:-1].cpu().numpy(), ref_cu)
    assert int(cu[-1]) == -7
    keep = w.masks[stage].bool()
    yc = y.cpu()
    assert np.all(raw(yc[~keep]).view(np.uint8) == 0)
    if full_oracle:
        ref = oracle_stage(w, stage)
        err, nbad, finite = compare_attention(yc[keep], ref["o"], y.dtype)
        assert finite and nbad == 0, err
        return err
    qp, c = O.pack(w.masks[stage], w.q)
    kp, _ = O.pack(w.masks[stage], w.k)
    vp, _ = O.pack(w.masks[stage], w.v)
    T = int(c[-1])
    rng = np.random.default_rng(1)
    ts = rng.integers(0, T, n_rows)
    hs = rng.integers(0, w.H, n_rows)
    want = O.attend_rows(qp, kp, vp, c, w.H, 64, ts, hs, dtype=w.dtype)
    got = yc[keep][torch.from_numpy(ts), torch.from_numpy(hs)].double().numpy()
    e = np.abs(got - want)
    assert np.all(e <= tolerance(want, y.dtype)), float(e.max())
    return float(e.max())


@pytest.mark.parametrize("name", ["c1", "c2", "c3:1", "c3:4", "c3:64", "c5:1.0:4", "c5:0.1:16", "c5:0.5:16"])
@pytest.mark.parametrize("out", ["native", "f32"])
def test_fused_small(name, out):
    err = check(W.by_name(name), out_dtype=torch.float32 if out == "f32" else None)
    if out == "f32":
        assert err <= ATOL


@pytest.mark.parametrize("name", ["c4", "c3:256", "c5:1.0:512", "c5:0.1:512"])
def test_fused_full_size(name):
    w = W.by_name(name)
    assert check(w, out_dtype=torch.float32, full_oracle=False) <= ATOL
    check(w, full_oracle=False)


def test_fused_staged():
    w = W.config5_staged(4)
    for s in range(3):
        assert check(w, stage=s, out_dtype=torch.float32) <= ATOL


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_fused_edge_lengths(dtype):
    w = W.from_lengths([0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 256, 257, 577], 577, 2, dtype=dtype,
                       seed=3)
    assert check(w, out_dtype=torch.float32) <= ATOL
    check(w)


@pytest.mark.parametrize("lengths,N", [([0, 0, 0], 197), ([197] * 5, 197), ([1] * 7, 33), ([0, 40, 0], 197),
                                        ([3, 0, 5], 10)])
def test_fused_degenerate(lengths, N):
    w = W.from_lengths(lengths, N, 3, seed=4)
    check(w, out_dtype=torch.float32)
    check(w)


def test_fused_guard_and_nan_at_pruned():
    w = W.config2()
    keep = w.masks[0].bool()
    clean, _, _ = run_fused(w)
    for t in (w.q, w.k, w.v):
        t[~keep] = float("nan")
    dirty, y_full, _ = run_fused(w, guard=64, fill=321.0)
    assert torch.equal(dirty.view(torch.int16), clean.view(torch.int16))
    assert torch.all(y_full[w.B * w.N:] == 321.0)
    assert torch.isfinite(dirty.float()).all()


def test_fused_graph_replay():
    ws = [W.config2(seed=s) for s in (0, 1)]
    w0 = ws[0]
    bufs = rra.Buffers(w0.B, w0.N, w0.H, torch.bfloat16, out_dtype=torch.float32)
    mask = w0.masks[0].cuda()
    q, k, v = w0.q.cuda(), w0.k.cuda(), w0.v.cuda()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        rra.forward(mask, q, k, v, bufs, stream=s, fused=True)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        rra.forward(mask, q, k, v, bufs, stream=s, fused=True)
    for w in ws:
        mask.copy_(w.masks[0])
        q.copy_(w.q)
        k.copy_(w.k)
        v.copy_(w.v)
        g.replay()
        torch.cuda.synchronize()
        ref = oracle_stage(w)
        keep = w.masks[0].bool()
        err, nbad, _ = compare_attention(bufs.y.cpu()[keep], ref["o"], torch.float32)
        assert nbad == 0, err
        assert torch.all(bufs.y.cpu()[~keep] == 0)

"""Parity of the CUDA path (through the C ABI) with the float64 oracle on the same seeded inputs.

pack / unpack / cu_seqlens: bit-exact.  attention: max |O_gpu - O_oracle| <= 2e-3 with fp32
output; with 16-bit output the bound adds the store's rounding (half an ulp of the output type,
taken over both neighbouring binades).
"""
import numpy as np
import pytest
import torch

from gpu_helpers import ATOL, GpuRun, bits16, compare_attention, oracle_stage, raw, tolerance
from oracle import oracle as O
from ragged_varlen_attention_rra_b200 import rra
from ragged_varlen_attention_rra_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    rra.lib()
    yield


def check_full(w, stage=0, out_dtype=None):
    """Whole path on one stage: pack bit-exact, attention within tolerance, unpacked result exact."""
    ref = oracle_stage(w, stage)
    T = ref["T"]
    g = GpuRun(w, stage, out_dtype=out_dtype).run()
    assert g.error() == 0
    assert np.array_equal(g.cu[:-1].cpu().numpy(), ref["cu"])
    for got, want in zip(g.packed, (ref["qp"], ref["kp"], ref["vp"])):
        assert np.array_equal(raw(got[:T]), want[:T])
    err, nbad, finite = compare_attention(g.o[:T], ref["o"], g.out_dtype)
    assert finite and nbad == 0, f"max err {err}"
    # unpacked: kept rows are the packed outputs, pruned rows zero bytes
    keep = w.masks[stage].bool()
    y = g.y.cpu()
    assert np.array_equal(raw(y[keep]), raw(g.o[:T]))
    assert np.all(raw(y[~keep]).view(np.uint8) == 0)
    return err


SMALL = ["c1", "c2", "c3:1", "c3:2", "c3:4", "c3:64"] + \
        [f"c5:{r}:{B}" for r in (1.0, 0.7, 0.5, 0.3, 0.2, 0.1) for B in (1, 4, 16)]


@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("out", ["native", "f32"])
def test_full_path(name, out):
    w = W.by_name(name)
    err = check_full(w, out_dtype=torch.float32 if out == "f32" else None)
    if out == "f32":
        assert err <= ATOL


def test_config4_small_batch_full():
    """DeiT-B 384 shape (L up to 404: several q-tiles and key chunks with ragged tails)."""
    w = W.config4(B=4)
    assert check_full(w, out_dtype=torch.float32) <= ATOL
    check_full(w)


def test_config5_staged_small():
    w = W.config5_staged(4)
    for s in range(3):
        assert check_full(w, stage=s, out_dtype=torch.float32) <= ATOL


def sampled_check(w, stage=0, n_rows=384, out_dtype=None, seed=0):
    """Full-size launch; pack/unpack exact everywhere, attention on sampled oracle rows."""
    mask = w.masks[stage]
    qp, cu = O.pack(mask, w.q)
    T = int(cu[-1])
    g = GpuRun(w, stage, out_dtype=out_dtype).run()
    assert g.error() == 0
    assert np.array_equal(g.cu[:-1].cpu().numpy(), cu)
    assert np.array_equal(raw(g.packed[0][:T]), qp[:T])
    del qp
    kp, _ = O.pack(mask, w.k)
    assert np.array_equal(raw(g.packed[1][:T]), kp[:T])
    vp, _ = O.pack(mask, w.v)
    assert np.array_equal(raw(g.packed[2][:T]), vp[:T])
    qp, _ = O.pack(mask, w.q)
    rng = np.random.default_rng(seed)
    ts = rng.integers(0, T, n_rows)
    hs = rng.integers(0, w.H, n_rows)
    # always include the first and last row of the batch and of a long image
    ts[:2] = [0, T - 1]
    want = O.attend_rows(qp, kp, vp, cu, w.H, 64, ts, hs, dtype=w.dtype)
    got = g.o[torch.from_numpy(ts).cuda(), torch.from_numpy(hs).cuda()].double().cpu().numpy()
    err = np.abs(got - want)
    assert np.all(err <= tolerance(want, g.out_dtype)), float(err.max())
    keep = mask.bool()
    assert np.all(raw(g.y.cpu()[~keep]).view(np.uint8) == 0)
    assert np.array_equal(raw(g.y.cpu()[keep]), raw(g.o[:T]))
    return float(err.max())


@pytest.mark.parametrize("name", ["c3:256", "c4"] + [f"c5:{r}:{B}" for r in (1.0, 0.5, 0.1) for B in (64, 256, 512)])
def test_full_size_sampled(name):
    w = W.by_name(name)
    assert sampled_check(w, out_dtype=torch.float32) <= ATOL
    sampled_check(w)


@pytest.mark.parametrize("B", [64, 512])
def test_staged_full_size_sampled(B):
    w = W.config5_staged(B)
    for s in range(3):
        assert sampled_check(w, stage=s, out_dtype=torch.float32, seed=s) <= ATOL


EDGE_LENGTHS = [0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 256, 257, 577]


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_edge_lengths(dtype):
    w = W.from_lengths(EDGE_LENGTHS, 577, 2, dtype=dtype, seed=3)
    assert check_full(w, out_dtype=torch.float32) <= ATOL
    check_full(w)


@pytest.mark.parametrize("lengths,N", [([197], 197), ([0, 0, 0], 197), ([197] * 5, 197), ([1] * 7, 33),
                                        ([40], 197), ([577, 1], 577)])
def test_degenerate_masks(lengths, N):
    w = W.from_lengths(lengths, N, 3, seed=4)
    check_full(w, out_dtype=torch.float32)
    check_full(w)


def test_scale_override():
    w = W.config1()
    ref = oracle_stage(w, full_attention=False)
    want = O.attend(ref["qp"], ref["kp"], ref["vp"], ref["cu"], w.H, 64, scale=0.3, dtype=w.dtype)
    g = GpuRun(w, out_dtype=torch.float32)
    g.pack()
    rra.rra_attend(g.packed[0], g.packed[1], g.packed[2], g.o, g.cu[:-1], max_seqlen=w.N, softmax_scale=0.3,
                   dev_error=g.err)
    torch.cuda.synchronize()
    assert g.error() == 0
    err = np.abs(g.o[:ref["T"]].double().cpu().numpy() - want).max()
    assert err <= ATOL


def test_nan_at_pruned_positions_and_garbage_capacity():
    """NaN/Inf at pruned padded positions and in unused capacity rows never reach the outputs."""
    w = W.config2()
    clean = GpuRun(w).run()
    keep = w.masks[0].bool()
    dirty_w = W.config2()
    for t, bad in ((dirty_w.q, float("nan")), (dirty_w.k, float("inf")), (dirty_w.v, float("nan"))):
        t[~keep] = bad
    dirty = GpuRun(dirty_w, fill_packed=float("nan"), fill_out=float("nan")).run()
    assert dirty.error() == 0
    T = int(clean.cu[-2])
    assert torch.equal(bits16_t(dirty.o[:T]), bits16_t(clean.o[:T]))
    assert torch.equal(bits16_t(dirty.y), bits16_t(clean.y))
    assert torch.isfinite(dirty.y.float()).all()


def bits16_t(t):
    return t.contiguous().view(torch.int16)


def test_guard_bands_untouched():
    w = W.config1()
    sentinel = 1234.5
    g = GpuRun(w, guard=64, fill_packed=sentinel, fill_out=sentinel).run()
    assert g.error() == 0
    cap = g.capacity
    for t in g.packed_full:
        assert torch.all(t[cap:] == sentinel)
    assert torch.all(g.o_full[cap:] == sentinel)
    assert torch.all(g.y_full[w.B * w.N:] == sentinel)
    assert int(g.cu[-1]) == -7  # one int past cu_seqlens[B]


def test_capacity_overflow_reports_and_stays_in_bounds():
    w = W.config2()
    ref = oracle_stage(w, full_attention=False)
    T = ref["T"]
    cap = T - 37
    sentinel = -77.0
    g = GpuRun(w, capacity=cap, guard=128, fill_packed=sentinel, fill_out=sentinel)
    g.pack()
    torch.cuda.synchronize()
    assert g.error() == rra.RRA_ERR_CAPACITY
    assert np.array_equal(g.cu[:-1].cpu().numpy(), ref["cu"])  # true counts still reported
    for got, want, full in zip(g.packed, (ref["qp"], ref["kp"], ref["vp"]), g.packed_full):
        assert np.array_equal(raw(got), want[:cap])
        assert torch.all(full[cap:] == sentinel)
    # attention over a cu_seqlens that runs past capacity: offending images skipped, flagged
    g.err.zero_()
    g.attend()
    torch.cuda.synchronize()
    assert g.error() == rra.RRA_ERR_BAD_SEQLENS
    assert torch.all(g.o_full[cap:] == sentinel)


def test_bad_seqlens_rejected_on_device():
    w = W.config1()
    g = GpuRun(w, fill_out=5.0)
    g.pack()
    torch.cuda.synchronize()
    good = g.cu[:-1].clone()
    bad = good.clone()
    bad[2] = g.capacity + 5  # image 1 ends past capacity, image 2 ends before it starts
    g.err.zero_()
    rra.rra_attend(g.packed[0], g.packed[1], g.packed[2], g.o, bad, max_seqlen=w.N, dev_error=g.err)
    torch.cuda.synchronize()
    assert g.error() == rra.RRA_ERR_BAD_SEQLENS
    assert torch.all(g.o[int(good[1]):int(good[3])] == 5.0)   # images 1 and 2 skipped
    assert not torch.all(g.o[int(good[0]):int(good[1])] == 5.0)  # image 0 computed
    g.err.zero_()
    rra.rra_unpack(g.o, bad, g.mask, g.y, dev_error=g.err)
    torch.cuda.synchronize()
    assert g.error() == rra.RRA_ERR_BAD_SEQLENS


def test_bounded_wait_timeout_reports_and_recovers():
    """A zero wait budget makes the first wait give up: the kernel reports RRA_ERR_TIMEOUT,
    drains its own copies, frees TMEM and returns; the context stays usable."""
    w = W.config2()
    g = GpuRun(w, out_dtype=torch.float32)
    g.pack()
    torch.cuda.synchronize()
    try:
        rra.rra_set_wait_timeout_ns(0)
        g.attend()
        torch.cuda.synchronize()
    finally:
        rra.rra_set_wait_timeout_ns(2_000_000_000)
    assert g.error() == rra.RRA_ERR_TIMEOUT
    g.err.zero_()
    g.attend()
    torch.cuda.synchronize()
    assert g.error() == 0
    ref = oracle_stage(w)
    err, nbad, _ = compare_attention(g.o[:ref["T"]], ref["o"], torch.float32)
    assert nbad == 0


def test_graph_replay_with_new_masks():
    """Capture pack/attend/unpack once; replay with new masks and values in the same buffers."""
    ws = [W.config2(seed=s) for s in (0, 1, 2)]
    w0 = ws[0]
    bufs = rra.Buffers(w0.B, w0.N, w0.H, torch.bfloat16, out_dtype=torch.float32)
    mask = w0.masks[0].cuda()
    q, k, v = w0.q.cuda(), w0.k.cuda(), w0.v.cuda()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        rra.forward(mask, q, k, v, bufs, stream=s)  # warm-up outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        rra.forward(mask, q, k, v, bufs, stream=s)
    for w in ws:
        mask.copy_(w.masks[0])
        q.copy_(w.q)
        k.copy_(w.k)
        v.copy_(w.v)
        bufs.err.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert rra.rra_get_device_error(bufs.err) == 0
        ref = oracle_stage(w)
        assert np.array_equal(bufs.cu.cpu().numpy(), ref["cu"])
        err, nbad, _ = compare_attention(bufs.o[:ref["T"]], ref["o"], torch.float32)
        assert nbad == 0, err
        keep = w.masks[0].bool()
        y = bufs.y.cpu()
        assert torch.all(y[~keep] == 0)


def test_unpack_bitexact_from_oracle_packed():
    """unpack alone, fed the oracle's packed rows: identical to the oracle's unpack (both modes)."""
    w = W.config3(64)
    mask = w.masks[0]
    qp, cu = O.pack(mask, w.q)
    dev_qp = torch.from_numpy(qp.view(np.int16)).view(torch.bfloat16).cuda()
    dev_cu = torch.from_numpy(cu).cuda()
    dmask = mask.cuda()
    for mode in (0, 1):
        init = torch.full((w.B, w.N, w.H, 64), 3.0, dtype=torch.bfloat16)
        dst = init.cuda()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        rra.rra_unpack(dev_qp, dev_cu, dmask, dst, fill_mode=mode, dev_error=err)
        torch.cuda.synchronize()
        assert rra.rra_get_device_error(err) == 0
        want = O.unpack(qp, cu, mask, fill_mode=mode, dst=init)
        assert np.array_equal(bits16(dst), want)


def test_pack_single_tensor_and_f32():
    """n_tensors = 1 and a 4-byte element type: still a bitwise gather."""
    w = W.config1()
    x = torch.randn(w.B, w.N, w.H, 64, generator=torch.Generator().manual_seed(9))
    mask = w.masks[0]
    want, cu = O.pack(mask, x)
    out = torch.full((w.B * w.N, w.H, 64), float("nan"), device="cuda")
    dcu = torch.zeros(w.B + 1, dtype=torch.int32, device="cuda")
    rra.rra_pack(mask.cuda(), [x.cuda()], [out], dcu)
    torch.cuda.synchronize()
    T = int(cu[-1])
    assert np.array_equal(dcu.cpu().numpy(), cu)
    assert np.array_equal(out[:T].cpu().numpy().view(np.uint32), want[:T].view(np.uint32))


@pytest.mark.parametrize("name", ["c4", "c5:1.0:64", "c2"])
def test_full_size_every_row(name):
    """Full-size workloads compared with the float64 oracle on EVERY kept row and head (the oracle
    runs one image per thread), both output types; the single launch is byte-identical to the
    three calls."""
    from gpu_helpers import oracle_attention_threaded
    w = W.by_name(name)
    want, cu = oracle_attention_threaded(w)
    T = int(cu[-1])
    for od in (torch.float32, None):
        g = GpuRun(w, out_dtype=od).run()
        assert g.error() == 0
        assert np.array_equal(g.cu[:-1].cpu().numpy(), cu)
        err, nbad, finite = compare_attention(g.o[:T], want, g.out_dtype)
        assert finite and nbad == 0, err
        if od == torch.float32:
            assert err <= ATOL
        y = torch.empty_like(g.y)
        rra.rra_pack_attend_unpack(g.mask, g.q, g.k, g.v, y)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.uint8), g.y.view(torch.uint8))


@pytest.mark.parametrize("B", [1024, 1025, 3000])
def test_large_batch_pack_and_path(B):
    """From 1025 images on, rra_pack writes cu_seqlens in a separate one-block launch and the
    gather blocks read their image start from it: bit-exact either side of the switch, with the
    whole path checked against the oracle."""
    rng = np.random.default_rng(B)
    lengths = rng.integers(0, 34, size=B)
    w = W.from_lengths(lengths.tolist(), 33, 1, seed=B)
    assert check_full(w, out_dtype=torch.float32) <= ATOL


@pytest.mark.parametrize("bad", [70000.0, float("inf")])
@pytest.mark.parametrize("fused", [False, True])
def test_v_tile_beyond_fp16_range(bad, fused):
    """A V tile holding a value beyond fp16's range (or an infinity) is not converted to fp16: it is
    restored to its bf16 bytes and meets a bf16 P.  That (image, head) keeps bf16-P precision
    (relative 2^-9 of the largest |v| it attends); every other one keeps the usual tolerance, and
    non-finite outputs sit exactly where the oracle's are."""
    lengths = [150, 100, 197, 130]  # one image per tile: the fallback stays inside its image
    w = W.from_lengths(lengths, 197, 2, seed=31)
    b, h = 2, 1
    kept = np.nonzero(w.masks[0][b].numpy())[0]
    w.v[b, kept[57], h, 5] = bad  # in the first 128-key chunk of image 2, head 1
    ref = oracle_stage(w)
    T, cu = ref["T"], ref["cu"]
    if fused:
        y = torch.empty(w.B, w.N, w.H, 64, dtype=torch.float32, device="cuda")
        rra.rra_pack_attend_unpack(w.masks[0].cuda(), w.q.cuda(), w.k.cuda(), w.v.cuda(), y)
        torch.cuda.synchronize()
        got = y.cpu()[w.masks[0].bool()].double().numpy()
    else:
        g = GpuRun(w, out_dtype=torch.float32).run()
        assert g.error() == 0
        got = g.o[:T].cpu().double().numpy()
    want = ref["o"]
    assert np.array_equal(np.isfinite(got), np.isfinite(want))
    assert np.array_equal(np.isnan(got), np.isnan(want))
    fin = np.isfinite(want)
    tol = np.full(want.shape, ATOL)
    vb = w.v[b][w.masks[0][b].bool(), h].double().abs()
    vmax = float(torch.where(torch.isfinite(vb), vb, torch.zeros_like(vb)).max())
    tol[cu[b]:cu[b + 1], h] = ATOL + 2.0 ** -8 * vmax
    assert np.all(np.abs(got[fin] - want[fin]) <= tol[fin])

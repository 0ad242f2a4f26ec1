"""Threshold-l2 token selection on the GPU (rra_l2_mask) against the exact oracle (whose squared
norms are exact rational sums): the masks must be identical, bit for bit, on the same seeded
embeddings -- top-k and threshold modes, nested stages, exact ties, NaN tokens, scores that a
rounded accumulation cannot tell apart, fp16 and bf16, and the configs' sizes."""
import numpy as np
import pytest
import torch

from gpu_helpers import compare_attention
from oracle import oracle as O
from ragged_varlen_attention_rra_b200 import rra
from ragged_varlen_attention_rra_b200 import workloads as W

pytestmark = pytest.mark.gpu


def gpu_mask(x, k=None, thr=0.0, prev=None, inplace=False):
    B, N, _ = x.shape
    xd = x.cuda()
    kd = None if k is None else torch.as_tensor(k, dtype=torch.int32).cuda()
    pd = None if prev is None else torch.as_tensor(prev, dtype=torch.uint8).cuda().contiguous()
    out = pd if inplace else torch.full((B, N), 7, dtype=torch.uint8, device="cuda")  # garbage to overwrite
    rra.rra_l2_mask(xd, out, k_keep=kd, threshold_sq=thr, prev_mask=pd)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("kind", ["normal", "ties", "nan"])
def test_topk_matches_oracle(dtype, kind):
    B, N, C = 64, 197, 384
    x = W.embeddings(B, N, C, dtype, seed=3, kind=kind)
    k = W.keep_counts(B, N, seed=3)
    want = O.l2_mask(x, k_keep=k)
    got = gpu_mask(x, k)
    assert np.array_equal(got, want)
    assert np.array_equal(got.sum(1), 1 + np.minimum(k, N - 1))  # CLS + k_b


@pytest.mark.parametrize("kind", ["normal", "ties", "nan"])
def test_threshold_matches_oracle(kind):
    B, N, C = 16, 197, 384
    x = W.embeddings(B, N, C, "bf16", seed=5, kind=kind)
    for thr in (0.0, 350.0, 384.0, 420.0, float("inf")):
        assert np.array_equal(gpu_mask(x, thr=thr), O.l2_mask(x, threshold_sq=thr)), thr


def test_exact_where_rounding_ties():
    """Tokens whose squared norms differ only below double precision (1 + k * 2^-60 and the like,
    the tiny terms before or after the 1): the kernel's double-double sums order them exactly as
    the oracle's exact sums, in top-k and threshold mode."""
    C = 128
    t = 2.0 ** -30
    rows = [[0.0] * C, [1.0] + [0.0] * (C - 1), [1.0] + [t] * 100 + [0.0] * 27, [t] * 100 + [1.0] + [0.0] * 27,
            [1.0] + [t] * 99 + [0.0] * 28, [1.0] + [2.0 ** -27] * 5 + [0.0] * 122,
            [1.0, 2.0 ** -26] + [0.0] * 126]
    for dt in (torch.bfloat16, torch.float16):
        r = [[v if dt == torch.bfloat16 or v == 0.0 or abs(v) >= 2.0 ** -24 else 0.0 for v in row] for row in rows]
        x = torch.tensor([r, r[::-1]], dtype=torch.float32).to(dt)
        for k in range(0, 8):
            kk = np.array([k, k], np.int32)
            assert np.array_equal(gpu_mask(x, kk), O.l2_mask(x, k_keep=kk)), (dt, k)
        for thr in (0.0, 1.0, 1.0 + 2.0 ** -52, 1.0 + 2.0 ** -51, float("inf"), -1.0):
            assert np.array_equal(gpu_mask(x, thr=thr), O.l2_mask(x, threshold_sq=thr)), (dt, thr)


def test_wide_range_and_special_values():
    """Embeddings spanning 2^-20 .. 2^20 in magnitude, plus rows with +-inf, NaN and zeros."""
    rng = np.random.default_rng(17)
    B, N, C = 8, 197, 384
    z = (rng.standard_normal((B, N, C)) * np.exp2(rng.integers(-20, 21, size=(B, N, C)))).astype(np.float32)
    z[0, 5, 3] = np.inf
    z[0, 6, 0] = -np.inf
    z[1, 7, 9] = np.nan
    z[1, 8, :] = 0.0
    z[2, 9, 1] = np.inf
    z[2, 9, 2] = np.nan
    x = torch.from_numpy(z).to(torch.bfloat16)
    k = np.random.default_rng(3).integers(0, N, size=B).astype(np.int32)
    assert np.array_equal(gpu_mask(x, k), O.l2_mask(x, k_keep=k))
    for thr in (0.0, 1e6, float("inf")):
        assert np.array_equal(gpu_mask(x, thr=thr), O.l2_mask(x, threshold_sq=thr)), thr


def test_nested_stages_match_oracle():
    """EViT-like schedule: three stages each keeping 0.7 of the previous survivors, chained on the
    device through prev_mask (the last stage in place)."""
    B, N, C = 64, 197, 384
    x = W.embeddings(B, N, C, "bf16", seed=9)
    prev_gpu = prev_cpu = None
    kk = N - 1
    for stage in range(3):
        kk = W.keep_count(0.7, kk)
        k = np.full(B, kk, np.int32)
        want = O.l2_mask(x, k_keep=k, prev=prev_cpu)
        got = gpu_mask(x, k, prev=prev_gpu, inplace=stage == 2)
        assert np.array_equal(got, want), stage
        if prev_cpu is not None:
            assert np.all(want <= prev_cpu | (np.arange(N) == 0))  # nested
        prev_gpu = prev_cpu = want


@pytest.mark.parametrize("B,N,C", [(1, 1, 8), (3, 2, 8), (64, 577, 768), (512, 197, 384), (4, 4096, 64)])
def test_sizes_match_oracle(B, N, C):
    x = W.embeddings(B, N, C, "bf16", seed=B + N, kind="ties" if N % 2 else "normal")
    k = np.random.default_rng(N).integers(-2, N + 2, size=B).astype(np.int32)  # incl. k < 0 and k > N-1
    assert np.array_equal(gpu_mask(x, k), O.l2_mask(x, k_keep=k))


def test_mask_feeds_the_pipeline():
    """The device-made mask drives the single-launch call exactly as the same mask from the host."""
    B, N, H = 8, 197, 6
    x = W.embeddings(B, N, 384, "bf16", seed=11)
    k = W.keep_counts(B, N, seed=11)
    w = W.from_lengths([1] * B, N, H, seed=11)  # only its Q/K/V are used
    q, kk, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    dmask = torch.empty(B, N, dtype=torch.uint8, device="cuda")
    rra.rra_l2_mask(x.cuda(), dmask, k_keep=torch.as_tensor(k).cuda())
    hmask = torch.from_numpy(O.l2_mask(x, k_keep=k)).cuda()
    y1 = torch.empty(B, N, H, 64, dtype=q.dtype, device="cuda")
    y2 = torch.empty_like(y1)
    rra.rra_pack_attend_unpack(dmask, q, kk, v, y1)
    rra.rra_pack_attend_unpack(hmask, q, kk, v, y2)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_three_stage_schedule_in_one_graph():
    """EViT-like schedule entirely on the device inside one CUDA graph: for each of three stages,
    select (nested in the previous stage's mask) then run the single-launch call; replayed with
    new embeddings in the same buffers, every stage's mask equals the oracle's selection and its
    output the oracle's attention on that mask (within the attention tolerance, pruned rows zero)."""
    B, N, H = 16, 197, 6
    w = W.from_lengths([1] * B, N, H, seed=21)
    q, kk, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    ks = []
    kprev = N - 1
    for _ in range(3):
        kprev = W.keep_count(0.7, kprev)
        ks.append(torch.full((B,), kprev, dtype=torch.int32, device="cuda"))
    x = torch.empty(B, N, 384, dtype=torch.bfloat16, device="cuda")
    masks = [torch.empty(B, N, dtype=torch.uint8, device="cuda") for _ in range(3)]
    ys = [torch.empty(B, N, H, 64, dtype=q.dtype, device="cuda") for _ in range(3)]
    s = torch.cuda.Stream()

    def enqueue():
        for i in range(3):
            rra.rra_l2_mask(x, masks[i], k_keep=ks[i], prev_mask=masks[i - 1] if i else None, stream=s)
            rra.rra_pack_attend_unpack(masks[i], q, kk, v, ys[i], stream=s)

    x.copy_(W.embeddings(B, N, 384, "bf16", seed=1).cuda())
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        enqueue()  # eager once (sets function attributes outside capture)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        enqueue()
    for seed in (2, 3):
        xe = W.embeddings(B, N, 384, "bf16", seed=seed)
        x.copy_(xe.cuda())
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        prev = None
        for i in range(3):
            want = O.l2_mask(xe, k_keep=ks[i].cpu().numpy(), prev=prev)
            assert np.array_equal(masks[i].cpu().numpy(), want), (seed, i)
            # the stage's attention output against the oracle on the oracle's own mask
            qp, cu = O.pack(want, w.q)
            kp, _ = O.pack(want, w.k)
            vp, _ = O.pack(want, w.v)
            T = int(cu[-1])
            ref = O.attend(qp, kp, vp, cu, H, 64, dtype=w.dtype)
            keep = torch.from_numpy(want).bool()
            y = ys[i].cpu()
            err, nbad, finite = compare_attention(y[keep], ref[:T], q.dtype)
            assert finite and nbad == 0, (seed, i, err)
            assert torch.all(y[~keep].view(torch.int16) == 0), (seed, i)
            prev = want

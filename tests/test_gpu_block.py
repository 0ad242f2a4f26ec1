"""The dense parts of a transformer block on packed rows (rra_layernorm, rra_linear, and the
whole block around rra_attend) against the float64 block oracle.

Tolerances come from the arithmetic.  A GPU output is one rounding to bf16 of an fp32 value;
the oracle rounds the exact value.  The two can differ by the fp32 error before rounding, plus
one bf16 unit in the last place where the exact value lies next to a rounding boundary.  For a
linear layer the fp32 error of a K-term dot product is at most about K 2^-24 sum |x_k w_k|
(doubled here for margin); for LayerNorm it is the fp32 error of the row statistics (see
layernorm_tol) plus a few fp32 roundings."""
import numpy as np
import pytest
import torch

from oracle import block as OB
from oracle import oracle as O
from ragged_varlen_attention_rra_b200 import rra
from ragged_varlen_attention_rra_b200 import workloads as W

pytestmark = pytest.mark.gpu
bf = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    rra.lib()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def ulp_bf16(a: np.ndarray) -> np.ndarray:
    """Spacing of the bf16 grid at |a| (8 significant bits; subnormal spacing 2^-133)."""
    a = np.abs(np.asarray(a, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def layernorm_tol(x, g, b, ref, eps=1e-6):
    """One bf16 ulp of the rounded exact value, plus the fp32 error before rounding: the row mean
    and variance are C-term fp32 sums (error up to about C 2^-24 of the sums of magnitudes; doubled
    here), which shift (x - mean) rstd gamma by |gamma| rstd C 2^-23 (mean|x| + |x - mean|), and a
    few roundings of the elementwise products.  Near-zero outputs, where gamma (x - mean) rstd and
    beta cancel, are where the statistics' error exceeds the output's own ulp."""
    xd, gd, bd = f64(x), f64(g), f64(b)
    C = xd.shape[1]
    mean = xd.mean(1, keepdims=True)
    rstd = 1.0 / np.sqrt(((xd - mean) ** 2).mean(1, keepdims=True) + eps)
    d = np.abs(xd - mean)
    stats = np.abs(gd) * rstd * C * 2.0 ** -23 * (np.abs(xd).mean(1, keepdims=True) + d)
    elem = 8 * 2.0 ** -24 * (np.abs(gd) * d * rstd + np.abs(bd))
    return ulp_bf16(ref) + stats + elem


def rand_bf16(shape, scale=1.0, shift=0.0, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale + shift).to(bf)


# ------------------------------------------------------------------------------ LayerNorm

@pytest.mark.parametrize("M,C", [(1, 768), (37, 384), (1000, 768), (300, 2048), (5, 8), (7, 256), (9, 1024), (11, 1280)])
def test_layernorm_matches_oracle(M, C):
    x = rand_bf16((M, C), 2.0, 0.5, seed=M)
    g = rand_bf16((C,), 0.1, 1.0, seed=1)
    b = rand_bf16((C,), 0.1, 0.0, seed=2)
    y = torch.empty(M, C, dtype=bf, device="cuda")
    rra.rra_layernorm(x.cuda(), g.cuda(), b.cuda(), y, eps=1e-6)
    torch.cuda.synchronize()
    ref = OB.bf16_round(OB.layernorm(f64(x), f64(g), f64(b), 1e-6))
    err = np.abs(f64(y) - ref)
    bad = err > layernorm_tol(x, g, b, ref)
    assert not bad.any(), (int(bad.sum()), float(err[bad].max()))


def test_layernorm_row_count_from_device():
    M, C = 40, 768
    x = rand_bf16((M, C), seed=3).cuda()
    g, b = torch.ones(C, dtype=bf, device="cuda"), torch.zeros(C, dtype=bf, device="cuda")
    y = torch.full((M, C), 7.0, dtype=bf, device="cuda")
    rra.rra_layernorm(x, g, b, y, m_dev=torch.tensor([13], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert (y[13:] == 7.0).all()
    one, zero = torch.ones(C, dtype=bf), torch.zeros(C, dtype=bf)
    ref = OB.bf16_round(OB.layernorm(f64(x[:13]), np.ones(C), np.zeros(C), 1e-6))
    assert (np.abs(f64(y[:13]) - ref) <= layernorm_tol(x[:13], one, zero, ref)).all()


# ------------------------------------------------------------------------------ linear

def linear_ref(x, w, bias, residual, act):
    """(reference output rounded to bf16, its tolerance) for rra_linear on the same bf16 inputs."""
    xd, wd = f64(x), f64(w)
    z = OB.linear(xd, wd, None if bias is None else f64(bias))
    acc_bound = 2.0 * xd.shape[1] * 2.0 ** -24 * (np.abs(xd) @ np.abs(wd).T)
    if act == rra.RRA_ACT_GELU:
        z = OB.gelu(z)  # GELU's slope is at most 1.13, so the bound carries over
        acc_bound = acc_bound * 1.13 + 2.0 ** -20 * np.abs(z)
    if residual is not None:
        z = z + f64(residual)
    ref = OB.bf16_round(z)
    return ref, ulp_bf16(ref) + acc_bound


CASES = [
    # M, N, K, n_outs, act, bias, residual
    (1, 256, 64, 1, rra.RRA_ACT_NONE, False, False),
    (300, 768, 768, 1, rra.RRA_ACT_NONE, True, False),
    (1000, 2304, 768, 3, rra.RRA_ACT_NONE, True, False),
    (517, 3072, 768, 1, rra.RRA_ACT_GELU, True, False),
    (300, 768, 3072, 1, rra.RRA_ACT_NONE, True, True),
    (129, 512, 128, 2, rra.RRA_ACT_GELU, False, True),
    (4097, 1024, 256, 4, rra.RRA_ACT_NONE, True, True),
    # 128-column tiles: DeiT-S widths (odd multiples of 128)
    (777, 1152, 384, 3, rra.RRA_ACT_NONE, True, False),
    (300, 1536, 384, 1, rra.RRA_ACT_GELU, True, False),
    (300, 384, 1536, 1, rra.RRA_ACT_NONE, True, True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"M{c[0]}N{c[1]}K{c[2]}o{c[3]}a{c[4]}" for c in CASES])
def test_linear_matches_oracle(case):
    M, N, K, n_outs, act, has_bias, has_res = case
    x = rand_bf16((M, K), seed=M + K)
    w = rand_bf16((N, K), 0.05, seed=N)
    bias = rand_bf16((N,), 0.5, seed=5) if has_bias else None
    res = rand_bf16((M, N), seed=6) if has_res else None
    outs = [torch.full((M, N // n_outs), 3.0, dtype=bf, device="cuda") for _ in range(n_outs)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rra.rra_linear(x.cuda(), w.cuda(), outs, bias=None if bias is None else bias.cuda(),
                   residual=None if res is None else res.cuda(), act=act, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = np.concatenate([f64(o) for o in outs], axis=1)
    ref, tol = linear_ref(x, w, bias, res, act)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (int(bad.sum()), float(np.abs(got - ref).max()))


def test_gelu_epilogue_across_its_range():
    """The GELU epilogue alone: an identity weight makes each output GELU of one bf16 input
    (the single-term dot product is exact in fp32).  Every bf16 value in [-16, 16] -- the far
    negative tail, where the output is tiny and 1 + erf cancels, included -- must round to the
    bf16 value of the exact GELU, up to one unit in the last place and the approximation's own
    error (below 5e-6 |x|; Abramowitz and Stegun 7.1.28 for erfc)."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 16.0)]
    K = N = 128
    M = -(-vals.size // K)
    flat = np.zeros(M * K, np.float32)
    flat[:vals.size] = vals
    x = torch.from_numpy(flat.reshape(M, K)).to(bf)
    w = torch.eye(N, K, dtype=bf)
    y = torch.empty(M, N, dtype=bf, device="cuda")
    rra.rra_linear(x.cuda(), w.cuda(), [y], act=rra.RRA_ACT_GELU)
    torch.cuda.synchronize()
    z = f64(x)
    ref = OB.bf16_round(OB.gelu(z))
    err = np.abs(f64(y) - ref)
    tol = ulp_bf16(ref) + 5e-6 * np.abs(z)
    assert (err <= tol).all(), (float(err.max()), float(z.ravel()[np.argmax((err - tol).ravel())]))
    # the tail is really formed: large negative inputs give tiny negative outputs, not zero
    tail = (z < -4) & (z > -8)
    assert (f64(y)[tail] < 0).all()


def test_linear_residual_in_place_and_row_count_from_device():
    M, N, K = 600, 768, 768
    x = rand_bf16((M, K), seed=11).cuda()
    w = rand_bf16((N, K), 0.05, seed=12).cuda()
    res = rand_bf16((M, N), seed=13)
    y = res.clone().cuda()
    rra.rra_linear(x, w, [y], residual=y, m_dev=torch.tensor([257], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(y[257:].cpu(), res[257:])
    ref, tol = linear_ref(x[:257].cpu(), w.cpu(), None, res[:257], rra.RRA_ACT_NONE)
    assert (np.abs(f64(y[:257]) - ref) <= tol).all()


def test_linear_full_size_sampled_rows():
    """DeiT-B FC1 at the size of config 5 at B = 512, r = 1 (M = 100,864 rows, GELU): 256 rows
    spread over the tiles compared in full."""
    M, N, K = 100864, 3072, 768
    g = torch.Generator(device="cuda").manual_seed(21)
    x = torch.randn(M, K, generator=g, device="cuda").to(bf)
    w = (torch.randn(N, K, generator=g, device="cuda") * 0.03).to(bf)
    bias = (torch.randn(N, generator=g, device="cuda") * 0.1).to(bf)
    y = torch.empty(M, N, dtype=bf, device="cuda")
    rra.rra_linear(x, w, [y], bias=bias, act=rra.RRA_ACT_GELU)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(3).integers(0, M, 250), [0, 127, 128, M - 1, M - 128]]))
    ref, tol = linear_ref(x[rows].cpu(), w.cpu(), bias.cpu(), None, rra.RRA_ACT_GELU)
    assert (np.abs(f64(y[rows]) - ref) <= tol).all()


# ------------------------------------------------------------------------------ the block

def _block_case(lengths, N=197, H=12, seed=0):
    C = 64 * H
    B = len(lengths)
    cap = B * N
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    x = torch.full((cap, C), float("nan"), dtype=bf)  # rows past T must never matter
    x[:T] = W.block_input(T, C, seed=seed)
    wts = W.block_weights(C, seed=seed)
    blk = rra.DeitBlock({k: v.cuda() for k, v in wts.items()}, cap, H)
    return B, N, H, C, T, cu, x, wts, blk


ATT_TOL = 2e-3  # the path's attention tolerance (fp32 accumulation, 16-bit inputs)


def test_block_stagewise_and_end_to_end():
    lengths = [197, 0, 61, 1, 130, 197]
    B, N, H, C, T, cu_np, x, wts, blk = _block_case(lengths)
    xd, cu = x.cuda(), torch.from_numpy(cu_np).cuda()
    y = blk(xd, cu, B, N)
    torch.cuda.synchronize()
    assert int(blk.err.item()) == 0
    w = {k: v for k, v in wts.items()}
    g = lambda t: t[:T].cpu()
    # every stage against the oracle on the GPU's own inputs to that stage
    ln1 = OB.bf16_round(OB.layernorm(f64(x[:T]), f64(w["ln1_g"]), f64(w["ln1_b"]), 1e-6))
    assert (np.abs(f64(g(blk.h)) - ln1) <= layernorm_tol(x[:T], w["ln1_g"], w["ln1_b"], ln1)).all()
    ref, tol = linear_ref(g(blk.h), w["qkv_w"], w["qkv_b"], None, rra.RRA_ACT_NONE)
    got = np.concatenate([f64(g(blk.q)), f64(g(blk.k)), f64(g(blk.v))], axis=1)
    assert (np.abs(got - ref) <= tol).all()
    sh = (T, H, 64)
    att = O.attend(g(blk.q).reshape(sh), g(blk.k).reshape(sh), g(blk.v).reshape(sh), cu_np, H, 64).reshape(T, C)
    assert (np.abs(f64(g(blk.a)) - att) <= ATT_TOL + ulp_bf16(att)).all()
    ref, tol = linear_ref(g(blk.a), w["proj_w"], w["proj_b"], x[:T], rra.RRA_ACT_NONE)
    assert (np.abs(f64(g(blk.x1)) - ref) <= tol).all()
    ln2 = OB.bf16_round(OB.layernorm(f64(g(blk.x1)), f64(w["ln2_g"]), f64(w["ln2_b"]), 1e-6))
    assert (np.abs(f64(g(blk.h2)) - ln2) <= layernorm_tol(g(blk.x1), w["ln2_g"], w["ln2_b"], ln2)).all()
    ref, tol = linear_ref(g(blk.h2), w["fc1_w"], w["fc1_b"], None, rra.RRA_ACT_GELU)
    assert (np.abs(f64(g(blk.m)) - ref) <= tol).all()
    ref, tol = linear_ref(g(blk.m), w["fc2_w"], w["fc2_b"], g(blk.x1), rra.RRA_ACT_NONE)
    assert (np.abs(f64(g(y)) - ref) <= tol).all()
    # end to end against the oracle's own chain (bf16 at the same stored points): the stages' one-ulp
    # rounding differences propagate through the layers, so this bound is looser; it catches a
    # wrong wiring (a missing residual or a swapped buffer moves values by O(1))
    want = OB.block(f64(x[:T]), cu_np, {k: f64(v) for k, v in w.items()}, H)["y"]
    err = np.abs(f64(g(y)) - want)
    assert float(err.max()) <= 0.0625 and float(err.mean()) <= 2e-3, (float(err.max()), float(err.mean()))


def test_deit_s_block_stagewise():
    """The DeiT-S width (C = 384, H = 6): every GEMM on 128-column tiles; each stage against the
    oracle on the GPU's own inputs, and the block end to end."""
    lengths = [197, 40, 0, 150]
    B, N, H, C, T, cu_np, x, wts, blk = _block_case(lengths, H=6, seed=3)
    xd, cu = x.cuda(), torch.from_numpy(cu_np).cuda()
    y = blk(xd, cu, B, N)
    torch.cuda.synchronize()
    assert int(blk.err.item()) == 0
    w = wts
    g = lambda t: t[:T].cpu()
    ref, tol = linear_ref(g(blk.h), w["qkv_w"], w["qkv_b"], None, rra.RRA_ACT_NONE)
    got = np.concatenate([f64(g(blk.q)), f64(g(blk.k)), f64(g(blk.v))], axis=1)
    assert (np.abs(got - ref) <= tol).all()
    ref, tol = linear_ref(g(blk.h2), w["fc1_w"], w["fc1_b"], None, rra.RRA_ACT_GELU)
    assert (np.abs(f64(g(blk.m)) - ref) <= tol).all()
    ref, tol = linear_ref(g(blk.m), w["fc2_w"], w["fc2_b"], g(blk.x1), rra.RRA_ACT_NONE)
    assert (np.abs(f64(g(y)) - ref) <= tol).all()
    want = OB.block(f64(x[:T]), cu_np, {k: f64(v) for k, v in w.items()}, H)["y"]
    err = np.abs(f64(g(y)) - want)
    assert float(err.max()) <= 0.0625 and float(err.mean()) <= 2e-3, (float(err.max()), float(err.mean()))


def test_block_graph_replay_with_new_rows():
    """The whole block (7 launches, no host synchronisation) captured once and replayed on new
    rows and new lengths gives the same bytes as the eager calls."""
    B, N, H, C, T, cu_np, x, wts, blk = _block_case([150, 197, 20, 88], seed=4)
    xd, cu = x.cuda(), torch.from_numpy(cu_np).cuda()
    s = torch.cuda.Stream()
    blk(xd, cu, B, N, stream=s)  # warm up (library load, attributes)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        blk(xd, cu, B, N, stream=s)
    cu2 = np.concatenate([[0], np.cumsum([197, 3, 64, 197])]).astype(np.int32)
    T2 = int(cu2[-1])
    x2 = W.block_input(T2, C, seed=9)
    xd[:T2].copy_(x2.cuda())
    cu.copy_(torch.from_numpy(cu2).cuda())
    graph.replay()
    torch.cuda.synchronize()
    y_graph = blk.y[:T2].clone()
    blk(xd, cu, B, N)
    torch.cuda.synchronize()
    assert torch.equal(y_graph.view(torch.int16), blk.y[:T2].view(torch.int16))
    del graph

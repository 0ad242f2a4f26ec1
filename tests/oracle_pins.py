"""Pins of the float64 oracle against facts fixed by mathematics and by library routines.

Each check takes an oracle library handle (the real build, or a build with a planted mistake)
and raises AssertionError when the oracle disagrees.  The checks are chosen so that a dropped
term, a wrong sign, a wrong index or a transposed operand anywhere in the oracle fails at least
one of them (``test_oracle_mutants.py`` plants such mistakes and checks exactly that).

What is computed follows "Dispatch-Aware Ragged Attention for Pruned Vision Transformers"
(sota2.com card, Abstract: bidirectional attention over the kept tokens of each image of a
token-pruned ViT, inside a pack-attend-unpack pipeline; aissential.tech summary, Method: a
two-phase packer -- index computation, then a gather).
"""
from __future__ import annotations

import math
import os
from decimal import Decimal, getcontext

import numpy as np
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_mask(rng, B, N, p=0.5, cls=True):
    m = (rng.random((B, N)) < p).astype(np.uint8)
    if cls:
        m[:, 0] = 1
    return m


# ------------------------------------------------------------------------------------ indexing

def pin_cu_seqlens_matches_cumsum(lib):
    """cu_seqlens equals torch.cumsum of per-image kept counts, with a leading zero."""
    rng = np.random.default_rng(11)
    for B, N, p in [(1, 7, 0.5), (5, 197, 0.3), (17, 577, 0.7), (3, 33, 0.0), (4, 16, 1.0)]:
        m = _rand_mask(rng, B, N, p, cls=False)
        # non-0/1 nonzero bytes also mean "keep"
        m = m * rng.integers(1, 256, size=m.shape).astype(np.uint8)
        cu = O.cu_seqlens(m, lib=lib)
        ref = torch.cat([torch.zeros(1, dtype=torch.int64),
                         torch.cumsum(torch.from_numpy(m != 0).sum(1), 0)]).numpy()
        assert np.array_equal(cu.astype(np.int64), ref), (B, N, p)
        assert cu[-1] == int(np.count_nonzero(m))


def pin_rank_matches_nonzero(lib):
    """rank(b, n) is the index of n in torch.nonzero(mask[b]); pruned positions are -1."""
    rng = np.random.default_rng(12)
    m = _rand_mask(rng, 6, 197, 0.4)
    r = O.rank(m, lib=lib)
    for b in range(m.shape[0]):
        nz = torch.nonzero(torch.from_numpy(m[b])).flatten().numpy()
        want = np.full(m.shape[1], -1, dtype=np.int32)
        want[nz] = np.arange(nz.shape[0], dtype=np.int32)
        assert np.array_equal(r[b], want), b


def pin_pack_matches_boolean_index(lib):
    """Packed rows [0, T) equal torch's row-major boolean indexing X[mask] byte for byte."""
    rng = np.random.default_rng(13)
    for dt in (torch.float16, torch.bfloat16, torch.float32):
        B, N, H, d = 5, 41, 3, 8
        m = _rand_mask(rng, B, N, 0.45)
        x = torch.randn(B, N, H, d, generator=torch.Generator().manual_seed(3)).to(dt)
        packed, cu = O.pack(m, x, lib=lib)
        T = int(cu[-1])
        want = x[torch.from_numpy(m).bool()]
        got = torch.from_numpy(packed[:T].view(np.int16) if dt != torch.float32 else packed[:T])
        if dt != torch.float32:
            assert torch.equal(got, want.view(torch.int16)), dt
        else:
            assert torch.equal(got, want), dt
        assert np.all(packed[T:].view(np.uint8) == 0)


def pin_pack_identity_and_roundtrip(lib):
    """All-ones mask: pack is the identity reshape.  unpack(pack(X)) == X * mask (fill 0), and
    fill_mode 1 keeps the destination's pruned rows."""
    rng = np.random.default_rng(14)
    B, N, H, d = 3, 29, 2, 4
    x = torch.randn(B, N, H, d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    ones = np.ones((B, N), np.uint8)
    packed, cu = O.pack(ones, x, lib=lib)
    assert np.array_equal(packed.reshape(B, N, H, d), x.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(cu, np.arange(B + 1, dtype=np.int32) * N)
    m = _rand_mask(rng, B, N, 0.5)
    packed, cu = O.pack(m, x, lib=lib)
    back = O.unpack(packed, cu, m, fill_mode=0, lib=lib)
    keep4 = torch.from_numpy(m).bool()[:, :, None, None].expand_as(x)
    want = torch.where(keep4, x, torch.zeros_like(x))  # +0.0 bytes at pruned rows
    assert np.array_equal(back, want.view(torch.int16).numpy().view(np.uint16))
    sentinel = np.full((B, N, H, d), 0x7FC1, dtype=np.uint16)
    back1 = O.unpack(packed, cu, m, fill_mode=1, dst=sentinel, lib=lib)
    keep = m.astype(bool)
    assert np.all(back1[~keep] == 0x7FC1)
    assert np.array_equal(back1[keep], back[keep])


def pin_pack_capacity_and_empty(lib):
    """No row at or past capacity is written; T is still reported.  Empty masks give T = 0."""
    rng = np.random.default_rng(15)
    B, N = 4, 20
    m = _rand_mask(rng, B, N, 0.9)
    x = np.arange(B * N * 4, dtype=np.float32).reshape(B, N, 4)
    full, cu = O.pack(m, x, lib=lib)
    T = int(cu[-1])
    cap = T - 5
    part, cu2 = O.pack(m, x, capacity=cap, lib=lib)
    assert np.array_equal(cu2, cu)
    assert part.shape[0] == cap and np.array_equal(part, full[:cap])
    zero = np.zeros((B, N), np.uint8)
    p0, cu0 = O.pack(zero, x, lib=lib)
    assert np.all(cu0 == 0) and np.all(p0 == 0)
    y = O.unpack(p0, cu0, zero, fill_mode=0, lib=lib)
    assert np.all(y == 0)


# ------------------------------------------------------------------------------------ attention

def _padded_sdpa_reference(q, k, v, mask, scale=None):
    """torch float64 SDPA on the padded batch with a boolean key mask (a library routine)."""
    B, N, H, d = q.shape
    out = torch.zeros(B, N, H, d, dtype=torch.float64)
    for b in range(B):
        keep = torch.from_numpy(mask[b].astype(bool))
        if not keep.any():
            continue
        qb = q[b].permute(1, 0, 2)[None].double()
        kb = k[b].permute(1, 0, 2)[None].double()
        vb = v[b].permute(1, 0, 2)[None].double()
        am = keep[None, None, None, :].expand(1, H, N, N)
        ob = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=am, scale=scale)
        out[b] = ob[0].permute(1, 0, 2)
    return out


def pin_attend_matches_padded_sdpa(lib):
    """Ragged attention on the kept tokens equals padded SDPA with a key mask, kept query rows."""
    rng = np.random.default_rng(21)
    g = torch.Generator().manual_seed(21)
    for B, N, H, d, dt in [(3, 23, 2, 8, torch.float64), (4, 37, 3, 64, torch.bfloat16),
                           (2, 50, 2, 16, torch.float16), (2, 9, 1, 64, torch.float32)]:
        q = torch.randn(B, N, H, d, generator=g).to(dt)
        k = torch.randn(B, N, H, d, generator=g).to(dt)
        v = torch.randn(B, N, H, d, generator=g).to(dt)
        m = _rand_mask(rng, B, N, 0.5)
        qp, cu = O.pack(m, q, lib=lib)
        kp, _ = O.pack(m, k, lib=lib)
        vp, _ = O.pack(m, v, lib=lib)
        dtn = {torch.float64: "f64", torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[dt]
        got = O.attend(qp, kp, vp, cu, H, d, dtype=dtn, lib=lib)
        ref = _padded_sdpa_reference(q, k, v, m)[torch.from_numpy(m).bool()].numpy()
        assert got.shape == ref.shape
        assert np.max(np.abs(got - ref)) < 1e-12, (B, N, H, d, dt, np.max(np.abs(got - ref)))
    # explicit scale is honoured
    q = torch.randn(1, 11, 2, 4, generator=g, dtype=torch.float64)
    m = np.ones((1, 11), np.uint8)
    qp = q.reshape(11, 2, 4).numpy()
    got = O.attend(qp, qp, qp, np.array([0, 11], np.int32), 2, 4, scale=0.37, dtype="f64", lib=lib)
    ref = _padded_sdpa_reference(q, q, q, m, scale=0.37)[0].numpy()
    assert np.max(np.abs(got - ref)) < 1e-12


def pin_attend_length_one_returns_v(lib):
    """A sequence of one token attends only to itself: o = v exactly."""
    rng = np.random.default_rng(22)
    H, d = 3, 64
    lens = [1, 5, 1, 1]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = rng.standard_normal((T, H, d))
    k = rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    got = O.attend(q, k, v, cu, H, d, dtype="f64", lib=lib)
    for b, L in enumerate(lens):
        if L == 1:
            assert np.array_equal(got[cu[b]], v[cu[b]])


def pin_attend_permutation_equivariant(lib):
    """Permuting the kept tokens of one image permutes its output rows the same way."""
    rng = np.random.default_rng(23)
    H, d, L = 2, 16, 13
    q = rng.standard_normal((L, H, d))
    k = rng.standard_normal((L, H, d))
    v = rng.standard_normal((L, H, d))
    cu = np.array([0, L], np.int32)
    base = O.attend(q, k, v, cu, H, d, dtype="f64", lib=lib)
    perm = rng.permutation(L)
    got = O.attend(q[perm], k[perm], v[perm], cu, H, d, dtype="f64", lib=lib)
    assert np.max(np.abs(got - base[perm])) < 1e-13
    # heads are independent: swapping heads swaps outputs
    got_h = O.attend(q[:, ::-1].copy(), k[:, ::-1].copy(), v[:, ::-1].copy(), cu, H, d, dtype="f64", lib=lib)
    assert np.max(np.abs(got_h - base[:, ::-1])) < 1e-13


def pin_attend_uniform_cases(lib):
    """Identical keys, or q = 0, give the mean of V; a constant V gives that constant."""
    rng = np.random.default_rng(24)
    H, d = 2, 8
    lens = [7, 3, 11]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    kk = np.empty((T, H, d))
    for b, L in enumerate(lens):
        kk[cu[b]:cu[b + 1]] = rng.standard_normal((1, H, d))
    got = O.attend(q, kk, v, cu, H, d, dtype="f64", lib=lib)
    got0 = O.attend(np.zeros_like(q), rng.standard_normal((T, H, d)), v, cu, H, d, dtype="f64", lib=lib)
    for b in range(len(lens)):
        mean = v[cu[b]:cu[b + 1]].mean(axis=0)
        assert np.max(np.abs(got[cu[b]:cu[b + 1]] - mean[None])) < 1e-13
        assert np.max(np.abs(got0[cu[b]:cu[b + 1]] - mean[None])) < 1e-13
    const = np.broadcast_to(rng.standard_normal((1, H, d)), (T, H, d)).copy()
    gotc = O.attend(q, rng.standard_normal((T, H, d)), const, cu, H, d, dtype="f64", lib=lib)
    assert np.max(np.abs(gotc - const)) < 1e-13


def pin_attend_two_token_closed_form(lib):
    """L = 2, d = 1: o_i = sigma(s_i1 - s_i2) v_1 + sigma(s_i2 - s_i1) v_2 with s_ij = q_i k_j."""
    rng = np.random.default_rng(25)
    for _ in range(5):
        q = rng.standard_normal((2, 1, 1)) * 3
        k = rng.standard_normal((2, 1, 1)) * 3
        v = rng.standard_normal((2, 1, 1))
        got = O.attend(q, k, v, np.array([0, 2], np.int32), 1, 1, dtype="f64", lib=lib)
        for i in range(2):
            s1, s2 = q[i, 0, 0] * k[0, 0, 0], q[i, 0, 0] * k[1, 0, 0]
            sig = 1.0 / (1.0 + math.exp(-(s1 - s2)))
            want = sig * v[0, 0, 0] + (1.0 - sig) * v[1, 0, 0]
            assert abs(got[i, 0, 0] - want) < 1e-14


def _decimal_attention(q, k, v, scale):
    """Brute-force softmax attention of one sequence with 50-digit decimals (independent loop)."""
    getcontext().prec = 50
    L, d = q.shape
    out = []
    for i in range(L):
        s = []
        for j in range(L):
            acc = Decimal(0)
            for c in range(d):
                acc += Decimal(float(q[i, c])) * Decimal(float(k[j, c]))
            s.append(acc * Decimal(repr(scale)) if not isinstance(scale, Decimal) else acc * scale)
        w = [x.exp() for x in s]
        z = sum(w)
        row = []
        for c in range(d):
            row.append(float(sum(w[j] * Decimal(float(v[j, c])) for j in range(L)) / z))
        out.append(row)
    return np.array(out)


def pin_attend_decimal_bruteforce(lib):
    """Hand-sized cases recomputed with 50-digit decimal arithmetic."""
    rng = np.random.default_rng(26)
    for L, d in [(1, 1), (2, 3), (3, 4), (4, 2), (4, 4)]:
        q = rng.standard_normal((L, 1, d))
        k = rng.standard_normal((L, 1, d))
        v = rng.standard_normal((L, 1, d))
        scale = 1.0 / math.sqrt(d)
        got = O.attend(q, k, v, np.array([0, L], np.int32), 1, d, dtype="f64", lib=lib)
        want = _decimal_attention(q[:, 0], k[:, 0], v[:, 0], Decimal(1) / Decimal(d).sqrt())
        assert np.max(np.abs(got[:, 0] - want)) < 1e-14, (L, d)


def pin_attend_rows_agree(lib):
    """The sampled-row entry point returns exactly the rows of the full computation."""
    rng = np.random.default_rng(27)
    H, d = 3, 16
    lens = [4, 9, 1, 6]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v = (rng.standard_normal((T, H, d)) for _ in range(3))
    full = O.attend(q, k, v, cu, H, d, dtype="f64", lib=lib)
    ts = rng.integers(0, T, 12)
    hs = rng.integers(0, H, 12)
    rows = O.attend_rows(q, k, v, cu, H, d, ts, hs, dtype="f64", lib=lib)
    assert np.array_equal(rows, full[ts, hs])


def _read_golden(name):
    cases, cur = [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, _, val = line.partition("=")
            key = key.strip()
            if key == "case":
                cur = {}
                cases.append(cur)
            else:
                cur[key] = [float(eval(x, {"log": math.log, "sqrt": math.sqrt, "exp": math.exp})) for x in val.split()]
    return cases


def pin_attend_golden_hand_cases(lib):
    """Hand-worked cases (tests/golden/attention_hand.txt) with exact softmax weights."""
    for c in _read_golden("attention_hand.txt"):
        L, d = int(c["L"][0]), int(c["d"][0])
        q = np.array(c["q"]).reshape(L, 1, d)
        k = np.array(c["k"]).reshape(L, 1, d)
        v = np.array(c["v"]).reshape(L, 1, d)
        want = np.array(c["o"]).reshape(L, d)
        got = O.attend(q, k, v, np.array([0, L], np.int32), 1, d, scale=c["scale"][0], dtype="f64", lib=lib)
        assert np.max(np.abs(got[:, 0] - want)) < 1e-13, c


def pin_widening_exact(lib):
    """16-bit inputs are widened exactly: every finite fp16/bf16 bit pattern, passed as a length-1
    sequence, comes back as its exact value (o = v for L = 1)."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    for name, tdt in (("f16", torch.float16), ("bf16", torch.bfloat16)):
        vals = torch.from_numpy(bits.view(np.int16).copy()).view(tdt).double().numpy()
        finite = np.isfinite(vals)
        v = bits[finite]
        n = v.shape[0]
        cu = np.arange(n + 1, dtype=np.int32)
        z = np.zeros(n, np.uint16)
        got = O.attend(z.reshape(n, 1, 1), z.reshape(n, 1, 1), v.reshape(n, 1, 1), cu, 1, 1, dtype=name, lib=lib)
        assert np.array_equal(got[:, 0, 0], vals[finite]), name


def pin_unpack_ranks_and_fill(lib):
    """unpack places packed row cu[b] + rank(b, n) at (b, n); pruned rows become zero bytes."""
    rng = np.random.default_rng(28)
    B, N = 4, 31
    m = _rand_mask(rng, B, N, 0.5)
    cu = O.cu_seqlens(m, lib=lib)
    T = int(cu[-1])
    packed = np.arange(T * 2, dtype=np.float32).reshape(T, 2) + 1.0
    # the destination starts as NaN garbage: fill mode 0 must overwrite every pruned row
    y = O.unpack(packed, cu, m, fill_mode=0, dst=np.full((B, N, 2), np.nan, np.float32), lib=lib)
    for b in range(B):
        r = 0
        for n in range(N):
            if m[b, n]:
                assert np.array_equal(y[b, n], packed[cu[b] + r])
                r += 1
            else:
                assert np.all(y[b, n].view(np.uint32) == 0)


# ------------------------------------------------------------------------------------ token selection

def _int_bf16(rng, shape, lo=-6, hi=7):
    """Small integers stored as bf16: every square and every sum of squares is exact, so ties are
    real ties and the accumulation order cannot change a score."""
    return torch.from_numpy(rng.integers(lo, hi, size=shape).astype(np.float32)).to(torch.bfloat16)


def _scores(x):
    return x.float().double().pow(2).sum(-1).numpy()  # exact for small-integer inputs


def pin_l2_mask_topk_matches_sorted(lib):
    """Top-k Threshold-l2 selection: CLS plus the k_b candidates of highest squared norm, the lower
    index first among equal norms; candidates restricted by the previous stage's mask."""
    rng = np.random.default_rng(41)
    B, N, C = 6, 37, 8
    x = _int_bf16(rng, (B, N, C), -3, 4)  # few distinct norms: many exact ties
    prev = _rand_mask(rng, B, N, 0.7)
    prev[1, 0] = 0  # CLS is kept even when the previous stage dropped it
    k = rng.integers(0, 30, size=B).astype(np.int32)
    sc = _scores(x)
    for use_prev in (False, True):
        got = O.l2_mask(x, k_keep=k, prev=prev if use_prev else None, lib=lib)
        for b in range(B):
            cand = [n for n in range(1, N) if (not use_prev or prev[b, n])]
            order = sorted(cand, key=lambda n: (-sc[b, n], n))
            want = np.zeros(N, np.uint8)
            want[0] = 1
            want[order[:max(0, min(int(k[b]), len(cand)))]] = 1
            assert np.array_equal(got[b], want), (use_prev, b)


def pin_l2_mask_threshold_and_extremes(lib):
    """Threshold mode keeps exactly the candidates with squared norm >= threshold (equality kept);
    k = 0 keeps only CLS, k >= #candidates keeps every candidate."""
    rng = np.random.default_rng(42)
    B, N, C = 3, 21, 4
    x = _int_bf16(rng, (B, N, C))
    sc = _scores(x)
    thr = float(np.median(sc[:, 1:]))  # an attained value: the >= boundary is exercised
    got = O.l2_mask(x, threshold_sq=thr, lib=lib)
    want = (sc >= thr).astype(np.uint8)
    want[:, 0] = 1
    assert np.array_equal(got, want)
    assert np.array_equal(O.l2_mask(x, threshold_sq=0.0, lib=lib), np.ones((B, N), np.uint8))
    only_cls = np.zeros((B, N), np.uint8)
    only_cls[:, 0] = 1
    assert np.array_equal(O.l2_mask(x, threshold_sq=math.inf, lib=lib), only_cls)
    assert np.array_equal(O.l2_mask(x, k_keep=np.zeros(B, np.int32), lib=lib), only_cls)
    assert np.array_equal(O.l2_mask(x, k_keep=np.full(B, 10 * N, np.int32), lib=lib), np.ones((B, N), np.uint8))


def pin_l2_mask_norm_not_l1(lib):
    """The score is the l2 norm: (3, 0, 0, 0) (|.|_2 = 3, |.|_1 = 3) must beat (1, 1, 1, 1) and
    (2, 2, 0, 0) (|.|_2 = 2, 2.83; |.|_1 = 4); a NaN row ranks last and never passes a threshold."""
    x = torch.tensor([[[0, 0, 0, 0], [1, 1, 1, 1], [2, 2, 0, 0], [3, 0, 0, 0], [float("nan"), 0, 0, 0]]],
                     dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(O.l2_mask(x, k_keep=[1], lib=lib)[0], [1, 0, 0, 1, 0])
    assert np.array_equal(O.l2_mask(x, k_keep=[2], lib=lib)[0], [1, 0, 1, 1, 0])
    assert np.array_equal(O.l2_mask(x, k_keep=[4], lib=lib)[0], [1, 1, 1, 1, 1])
    assert np.array_equal(O.l2_mask(x, threshold_sq=4.0, lib=lib)[0], [1, 1, 1, 1, 0])
    assert np.array_equal(O.l2_mask(x, threshold_sq=8.5, lib=lib)[0], [1, 0, 0, 1, 0])


def _exact_sq(row):
    """(class, Fraction) of the exact squared norm of a list of Python floats (each the exact
    value of a 16-bit or single-precision input)."""
    from fractions import Fraction
    if any(math.isnan(v) for v in row):
        return (O.SCORE_NAN, None)
    if any(math.isinf(v) for v in row):
        return (O.SCORE_INF, None)
    return (O.SCORE_FINITE, sum((Fraction(v) ** 2 for v in row), Fraction(0)))


def pin_l2_score_is_exact_sum(lib):
    """The oracle's squared norm is the exact rational sum of the squares (fractions.Fraction):
    on N(0,1) rows of C = 384 and 768 in bf16 and fp16 (where a single-precision chain already
    rounds), on rows mixing magnitudes from 2^-60 to 2^60 (where a double-precision chain rounds
    too, in an order-dependent way), on subnormal and zero entries, and with inf / NaN entries."""
    rng = np.random.default_rng(43)
    cases = []
    for dt in (torch.bfloat16, torch.float16):
        for C in (384, 768):
            cases.append(torch.from_numpy(rng.standard_normal((4, C), dtype=np.float32)).to(dt))
    wide = (rng.standard_normal((6, 64)) * np.exp2(rng.integers(-60, 61, size=(6, 64)))).astype(np.float32)
    cases.append(torch.from_numpy(wide).to(torch.bfloat16))
    cases.append(torch.from_numpy(wide))  # single precision input
    cases.append(torch.tensor([[2.0 ** -133, -(2.0 ** -126), 1.0, 3.0, 0.0, -0.0, 2.0 ** 100, 2.0 ** -100]],
                              dtype=torch.float32).to(torch.bfloat16))
    cases.append(torch.tensor([[2.0 ** -24, 2.0 ** -14, 0.5, 65504.0, 0.0, -3.0, 1.0 / 3.0, 1e-5]],
                              dtype=torch.float32).to(torch.float16))
    cases.append(torch.tensor([[1.0, float("inf"), 2.0], [float("nan"), float("inf"), 1.0], [3.0, 4.0, 0.0]],
                              dtype=torch.float32).to(torch.bfloat16))
    for x in cases:
        got = O.l2_score(x, lib=lib)
        for r, row in enumerate(x.reshape(-1, x.shape[-1]).tolist()):
            assert got[r] == _exact_sq(row), (x.dtype, r)


def pin_l2_mask_exact_where_rounding_ties(lib):
    """Selection follows the exact sums where a rounded accumulation, in either order, sees a
    tie: token 1 is exactly 1; tokens 2 and 3 are 1 + 100 * 2^-60 (the tiny terms after the 1,
    or before it); token 4 is 1 + 99 * 2^-60; token 5 is 1 + 5 * 2^-54.  In double precision
    every one of them sums to 1.  Exactly, 5 > 2 = 3 > 4 > 1; token 6 (= 1 + 2^-52) beats them
    all, and of the others only 5 reaches the threshold 1 + 2^-52 that 6 attains."""
    C = 128
    t = 2.0 ** -30
    rows = [[0.0] * C, [1.0] + [0.0] * (C - 1), [1.0] + [t] * 100 + [0.0] * 27, [t] * 100 + [1.0] + [0.0] * 27,
            [1.0] + [t] * 99 + [0.0] * 28, [1.0] + [2.0 ** -27] * 5 + [0.0] * 122,
            [1.0, 2.0 ** -26] + [0.0] * 126]
    x = torch.tensor([rows], dtype=torch.float32).to(torch.bfloat16)
    assert x.float().tolist() == [rows]  # every entry is a bf16 value
    want = {1: [5], 2: [5, 2], 3: [5, 2, 3], 4: [5, 2, 3, 4], 5: [5, 2, 3, 4, 1]}
    for k, keep in want.items():
        # token 6 competes too: 1 + 2^-52 > 1 + 5 * 2^-54 (token 5), so it is always first
        got = O.l2_mask(x, k_keep=[k + 1], lib=lib)[0]
        exp = np.zeros(7, np.uint8)
        exp[[0, 6] + keep[:k]] = 1
        assert np.array_equal(got, exp), (k, got)
    got = O.l2_mask(x, threshold_sq=1.0 + 2.0 ** -52, lib=lib)[0]
    assert np.array_equal(got, [1, 0, 0, 0, 0, 1, 1]), got
    got = O.l2_mask(x, threshold_sq=1.0, lib=lib)[0]
    assert np.array_equal(got, [1, 1, 1, 1, 1, 1, 1]), got


ALL_PINS = [
    pin_cu_seqlens_matches_cumsum,
    pin_rank_matches_nonzero,
    pin_pack_matches_boolean_index,
    pin_pack_identity_and_roundtrip,
    pin_pack_capacity_and_empty,
    pin_attend_matches_padded_sdpa,
    pin_attend_length_one_returns_v,
    pin_attend_permutation_equivariant,
    pin_attend_uniform_cases,
    pin_attend_two_token_closed_form,
    pin_attend_decimal_bruteforce,
    pin_attend_rows_agree,
    pin_attend_golden_hand_cases,
    pin_widening_exact,
    pin_unpack_ranks_and_fill,
    pin_l2_mask_topk_matches_sorted,
    pin_l2_mask_threshold_and_extremes,
    pin_l2_mask_norm_not_l1,
    pin_l2_score_is_exact_sum,
    pin_l2_mask_exact_where_rounding_ties,
]

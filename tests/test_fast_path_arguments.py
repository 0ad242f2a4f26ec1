"""CPU checks of two arguments the kernels rest on, restated in numpy (no GPU):

* the Threshold-l2 fast path: when the smallest fp32 square of a row's (exactly squared) 16-bit
  inputs gives q = twice the last-bit exponent of the smallest input, and the double sum of the
  squares stays below 2^(q+52), the sum is exact -- whatever the order of the additions;
* the Threshold-l2 ranking: counting on fp32-rounded keys, with the tokens whose fp32 key is
  shared settled on the full keys, gives every token the rank of the full-key order (index
  breaking ties);
* the GEMM epilogue's GELU: erfc from Abramowitz and Stegun 7.1.28, evaluated in fp32 as the
  kernel does, stays within 5e-6 |x| of the exact GELU over every bf16 input in [-16, 16].

Each check compares against a value computed independently (exact rationals, scipy's erf)."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import erf


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _fast_sum_ok_bf16(row32):
    """The kernel's test for a bf16 row: fp32 squares, their minimum's exponent, double sum."""
    sq = (row32.astype(np.float32) * row32.astype(np.float32)).astype(np.float32)
    sqmin = sq.min()
    e2 = int(np.frombuffer(np.float32(sqmin).tobytes(), np.uint32)[0] >> 23)
    if e2 == 0:
        return False, None
    e = (e2 - 127) >> 1
    q = 2 * (e - 7)
    acc = 0.0
    for s in sq.astype(np.float64):
        acc = acc + s
    return acc < 2.0 ** (q + 52), sq


def _exact(sq):
    return sum((Fraction(float(s)) for s in sq), Fraction(0))


def _sums_in_orders(sq, rng):
    s = sq.astype(np.float64)
    orders = [s, s[::-1], np.sort(s), np.sort(s)[::-1], rng.permutation(s)]
    out = []
    for o in orders:
        acc = 0.0
        for v in o:
            acc = acc + v
        out.append(acc)
    # a pairwise tree, as a warp reduction adds lane partials
    t = list(s)
    while len(t) > 1:
        t = [t[i] + t[i + 1] if i + 1 < len(t) else t[i] for i in range(0, len(t), 2)]
    out.append(t[0])
    return out


@pytest.mark.parametrize("kind", ["normal", "scaled", "mixed"])
def test_threshold_l2_fast_path_is_exact_in_any_order(kind):
    rng = np.random.default_rng({"normal": 1, "scaled": 2, "mixed": 3}[kind])
    passed = 0
    for _ in range(300):
        C = int(rng.choice([64, 384, 768]))
        x = rng.standard_normal(C)
        if kind == "scaled":
            x = x * 2.0 ** rng.integers(-40, 40)
        elif kind == "mixed":
            x[rng.integers(0, C, 4)] *= 2.0 ** rng.integers(-12, -3, 4)
        row = _bf16(x)
        ok, sq = _fast_sum_ok_bf16(row)
        if not ok:
            continue
        passed += 1
        exact = _exact(sq)
        for v in _sums_in_orders(sq, rng):
            assert Fraction(v) == exact
    assert passed > (30 if kind == "mixed" else 100)  # the fast path is the common case on these rows


def test_threshold_l2_fast_path_refuses_a_rounding_sum():
    # 1 plus many squares of 2^-30 (each 2^-60): a double sum rounds them away, so the test must fail
    row = _bf16(np.concatenate([[1.0], np.full(300, 2.0 ** -30)]))
    ok, sq = _fast_sum_ok_bf16(row)
    assert not ok
    # and a zero input is refused (the slow path handles it)
    ok0, _ = _fast_sum_ok_bf16(_bf16([1.0, 0.0, 2.0]))
    assert not ok0


def _gelu_as_fp32(x):
    x = x.astype(np.float32)
    z = (np.abs(x) * np.float32(0.70710678118654752)).astype(np.float32)
    q = (z * np.float32(4.30638e-5) + np.float32(2.765672e-4)).astype(np.float32)
    for c in (1.520143e-4, 9.2705272e-3, 4.22820123e-2, 7.05230784e-2, 1.0):
        q = (q * z + np.float32(c)).astype(np.float32)
    for _ in range(4):
        q = (q * q).astype(np.float32)
    with np.errstate(over="ignore", divide="ignore"):
        h = (np.float32(0.5) / q).astype(np.float32)
    return np.where(x < 0, x * h, x * (np.float32(1) - h)).astype(np.float64)


def test_gelu_erfc_approximation_bound():
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (bits << 16).view(np.float32)
    x = vals[np.isfinite(vals) & (np.abs(vals) <= 16.0)].astype(np.float64)
    exact = 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))
    err = np.abs(_gelu_as_fp32(x) - exact)
    assert (err <= 5e-6 * np.abs(x) + 1e-300).all(), float((err / np.maximum(np.abs(x), 1e-300)).max())
    # the negative tail is formed, not cancelled to zero
    tail = (x < -4) & (x > -8)
    assert (_gelu_as_fp32(x)[tail] < 0).all()


def test_fast_path_bound_needs_the_last_bit_term():
    """A row with a large and a small input whose double sum rounds: the kernel's bound (q from the
    smallest input's last bit, 2^(e-7)) refuses it; a bound that forgot the 7 mantissa bits
    (q = 2e) would accept it although the sum is not exact -- the planted mistake this pins."""
    row = _bf16([2.0 ** 10, (1.0 + 1.0 / 128) * 2.0 ** -12])
    ok, sq = _fast_sum_ok_bf16(row)
    assert not ok
    sq = (row.astype(np.float32) ** 2).astype(np.float32)
    e = -12
    acc = float(sq[0]) + float(sq[1])
    assert acc < 2.0 ** (2 * e + 52)           # the mistaken bound passes ...
    assert Fraction(acc) != _exact(sq)         # ... an inexact sum


def _rank_by_fp32_counts(hi, lo):
    """The kernel's ranking, restated: fp32-rounded keys counted (greater, equal); a token whose
    fp32 key another token shares is settled on the full (hi, lo) keys, index breaking ties."""
    f = hi.astype(np.float32)  # a monotone rounding of the high part
    n = len(hi)
    ranks = np.zeros(n, np.int64)
    for i in range(n):
        gt = int((f > f[i]).sum())
        eq = int((f == f[i]).sum())
        r = gt
        if eq > 1:
            for m in np.nonzero(f == f[i])[0]:
                if m == i:
                    continue
                if hi[m] > hi[i] or (hi[m] == hi[i] and (lo[m] > lo[i] or (lo[m] == lo[i] and m < i))):
                    r += 1
        ranks[i] = r
    return ranks


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fp32_key_ranking_equals_the_full_key_order(seed):
    rng = np.random.default_rng(seed)
    n = 197
    # scores with many near-ties: equal in fp32, different in double, some fully equal
    base = rng.choice([1.0, 3.0, 768.0, 1e6], size=n)
    hi = base * (1.0 + rng.integers(0, 5, n) * 2.0 ** -40)
    lo = rng.integers(-2, 3, n) * 2.0 ** -80
    lo[rng.random(n) < 0.3] = 0.0
    ranks = _rank_by_fp32_counts(hi, lo)
    order = sorted(range(n), key=lambda i: (-hi[i], -lo[i], i))
    want = np.empty(n, np.int64)
    want[order] = np.arange(n)
    assert np.array_equal(ranks, want)

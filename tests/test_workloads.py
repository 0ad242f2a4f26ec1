"""The seeded input recipes (CPU only): shapes, determinism and mask structure."""
import numpy as np
import pytest
import torch

from ragged_varlen_attention_rra_b200 import workloads as W


def _check_common(w, dtype):
    assert w.q.shape == (w.B, w.N, w.H, 64) and w.q.dtype == dtype
    assert w.k.shape == w.q.shape and w.v.shape == w.q.shape
    for m in w.masks:
        assert m.dtype == torch.uint8 and m.shape == (w.B, w.N)
        assert torch.all(m[:, 0] == 1), "CLS always kept"


def test_config1_recipe():
    w = W.config1()
    _check_common(w, torch.float16)
    L = w.lengths[0]
    assert w.B == 4 and w.H == 3 and w.N == 197
    assert np.all((L >= 20) & (L <= 197))
    w2 = W.config1()
    assert torch.equal(w.q.view(torch.int16), w2.q.view(torch.int16))
    assert torch.equal(w.masks[0], w2.masks[0])
    w3 = W.config1(seed=1)
    assert not torch.equal(w.masks[0], w3.masks[0])


def test_config2_recipe():
    w = W.config2()
    _check_common(w, torch.bfloat16)
    L = w.lengths[0]
    assert w.B == 64 and w.H == 6
    # k = floor(196 r + 0.5) with r in [0.3, 0.7] -> L in [60, 138]
    assert np.all((L >= 60) & (L <= 138))
    assert 5000 < L.sum() < 7500
    # values ~ N(0, 1)
    assert abs(float(w.q.float().std()) - 1.0) < 0.02


@pytest.mark.parametrize("B", [1, 2, 4, 64])
def test_config3_recipe(B):
    w = W.config3(B)
    _check_common(w, torch.bfloat16)
    L = w.lengths[0]
    assert np.all((L >= 36) & (L <= 44)) and w.H == 12


def test_config4_recipe():
    w = W.config4(B=8)
    _check_common(w, torch.bfloat16)
    L = w.lengths[0]
    assert w.N == 577 and np.all((L >= 1 + 173) & (L <= 1 + 403))
    assert abs(float(w.q.float().std()) - 0.5) < 0.01


@pytest.mark.parametrize("r,L", [(1.0, 197), (0.7, 138), (0.5, 99), (0.3, 60), (0.2, 40), (0.1, 21)])
def test_config5_lengths(r, L):
    w = W.config5(r, 4)
    _check_common(w, torch.bfloat16)
    assert np.all(w.lengths[0] == L)


def test_config5_staged_nested():
    w = W.config5_staged(4)
    assert len(w.masks) == 3
    assert [int(l[0]) for l in w.lengths] == [138, 97, 68]
    for a, b in zip(w.masks, w.masks[1:]):
        assert torch.all(b <= a), "each stage keeps a subset of the previous survivors"
    assert w.total_tokens == 4 * (138 + 97 + 68)


def test_from_lengths():
    w = W.from_lengths([0, 1, 17, 197], 197, 2)
    assert list(w.lengths[0]) == [0, 1, 17, 197]


def test_embeddings_and_keep_counts_are_seeded():
    a = W.embeddings(3, 17, 16, "bf16", seed=4)
    b = W.embeddings(3, 17, 16, "bf16", seed=4)
    assert a.shape == (3, 17, 16) and a.dtype == torch.bfloat16 and torch.equal(a, b)
    t = W.embeddings(2, 9, 8, "f16", seed=1, kind="ties")
    assert t.dtype == torch.float16 and torch.all(t == t.round()) and t.abs().max() <= 3
    n = W.embeddings(2, 9, 8, "bf16", seed=1, kind="nan")
    assert torch.isnan(n.float()).any() and not torch.isnan(n[:, 0].float()).any()
    k = W.keep_counts(64, 197, seed=2)
    assert k.dtype == np.int32 and k.min() >= W.keep_count(0.3, 196) and k.max() <= W.keep_count(0.7, 196)

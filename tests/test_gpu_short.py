"""Short-sequence tiling of the attention kernel (both the packed call and the single launch):
when no image keeps more than 64 tokens, each 128-row tile of the packed token space holds the
rows of several images and every query row attends only to its own image's keys.  Checked against
the float64 oracle on every row, and the two paths against each other byte for byte: images that
straddle tile boundaries, empty images between them, the 64 / 65 boundary between the two tilings,
and NaN planted at pruned positions and past the last packed row."""
import numpy as np
import pytest
import torch

from gpu_helpers import ATOL, GpuRun, oracle_attention_threaded
from ragged_varlen_attention_rra_b200 import rra
from ragged_varlen_attention_rra_b200 import workloads as W
from test_gpu_fused import check as check_fused
from test_gpu_parity import check_full

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    rra.lib()


MIXED = [0, 1, 64, 0, 63, 17, 0, 0, 40, 33, 64, 64, 2, 1, 0, 50, 31, 32, 33, 7, 0, 64, 9, 48]


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("lengths", [MIXED, MIXED * 3, [64] * 9, [1] * 300, [5, 0] * 100])
def test_short_tiles_match_oracle(dtype, lengths):
    N = 197
    w = W.from_lengths(lengths, N, 3, dtype=dtype, seed=len(lengths))
    assert max(lengths) <= 64 and sum(lengths) > 128  # several tiles, images across tile edges
    assert check_full(w, out_dtype=torch.float32) <= ATOL
    check_full(w)
    assert check_fused(w, out_dtype=torch.float32) <= ATOL
    check_fused(w)


@pytest.mark.parametrize("longest", [64, 65])
def test_boundary_between_tilings(longest):
    """All images at most 64 long (short tiles), or one of them 65 (one image per tile): both exact."""
    lengths = [40, 64, 3, 0, longest, 21, 64, 1]
    w = W.from_lengths(lengths, 197, 12, seed=longest)
    assert check_full(w, out_dtype=torch.float32) <= ATOL
    assert check_fused(w, out_dtype=torch.float32) <= ATOL


def test_many_empty_images_between_short_ones():
    lengths = [0] * 300 + [5] + [0] * 257 + [64] + [0] * 31 + [13, 60, 0, 1] + [0] * 400 + [64, 64, 64]
    w = W.from_lengths(lengths, 65, 2, seed=8)
    assert check_full(w, out_dtype=torch.float32) <= ATOL
    assert check_fused(w, out_dtype=torch.float32) <= ATOL


def bits16_t(t):
    return t.contiguous().view(torch.int16)


def test_short_tiles_nan_at_pruned_positions_and_capacity_rows():
    """config 3 at B = 64 (L_b = 36..44): NaN/Inf at pruned padded positions and NaN in every packed
    row past T change nothing, on both paths."""
    w = W.config3(64)
    clean = GpuRun(w).run()
    keep = w.masks[0].bool()
    dirty_w = W.config3(64)
    for t, bad in ((dirty_w.q, float("nan")), (dirty_w.k, float("inf")), (dirty_w.v, float("nan"))):
        t[~keep] = bad
    dirty = GpuRun(dirty_w, fill_packed=float("nan"), fill_out=float("nan")).run()
    assert dirty.error() == 0
    T = int(clean.cu[-2])
    assert torch.equal(bits16_t(dirty.o[:T]), bits16_t(clean.o[:T]))
    assert torch.equal(bits16_t(dirty.y), bits16_t(clean.y))
    assert torch.isfinite(dirty.y.float()).all()
    y = torch.empty_like(clean.y)
    rra.rra_pack_attend_unpack(dirty_w.masks[0].cuda(), dirty_w.q.cuda(), dirty_w.k.cuda(), dirty_w.v.cuda(), y)
    torch.cuda.synchronize()
    assert torch.equal(bits16_t(y), bits16_t(clean.y))


@pytest.mark.parametrize("name", ["c3:256", "c5:0.1:512", "c5:0.2:256"])
def test_short_tiles_full_size_every_row(name):
    """Full-size short-sequence workloads compared with the oracle on every kept row and head."""
    w = W.by_name(name)
    g = GpuRun(w, out_dtype=torch.float32).run()
    assert g.error() == 0
    want, cu = oracle_attention_threaded(w)
    T = int(cu[-1])
    err = np.abs(g.o[:T].double().cpu().numpy() - want)
    assert float(err.max()) <= ATOL

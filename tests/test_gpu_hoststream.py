"""rra.HostStream: a batch in pinned host memory streamed through the GPU in chunks of images,
copies in both directions overlapping the kernels.  Every stage's padded output must match the
float64 oracle (kept rows within the path's tolerance, pruned rows zero), for chunk sizes that
leave a partial last chunk, for a batch smaller than the one the buffers were sized for, and on
both the single-launch and the three-call path."""
import numpy as np
import pytest
import torch

from gpu_helpers import compare_attention, raw
from oracle import oracle as O
from ragged_varlen_attention_rra_b200 import rra
from ragged_varlen_attention_rra_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    rra.lib()


def _workload():
    w = W.from_lengths([197, 0, 5, 64, 130, 1, 77], N=197, H=3, seed=7)
    rng = np.random.default_rng(3)
    m1 = w.masks[0].numpy()
    m2 = (m1 & (rng.random(m1.shape) < 0.5)).astype(np.uint8)
    m2[:, 0] = m1[:, 0]
    return w, [w.masks[0], torch.from_numpy(m2)]


def _check(w, masks, outs, Bp):
    for s, (m, y) in enumerate(zip(masks, outs)):
        m = m[:Bp]
        keep = m.bool()
        assert np.all(raw(y[~keep]).view(np.uint8) == 0), f"stage {s}: pruned rows not zero"
        qp, cu = O.pack(m, w.q[:Bp])
        kp, _ = O.pack(m, w.k[:Bp])
        vp, _ = O.pack(m, w.v[:Bp])
        ref = O.attend(qp, kp, vp, cu, w.H, 64, dtype=w.dtype)
        err, nbad, finite = compare_attention(y[keep], ref, y.dtype)
        assert finite and nbad == 0, (s, err)


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("chunk", [3, 1, 16])
def test_host_stream_matches_oracle(fused, chunk):
    w, masks = _workload()
    hs = rra.HostStream(w.B, w.N, w.H, w.q.dtype, stages=2, chunk=chunk, fused=fused)
    q, k, v = (t.contiguous().pin_memory() for t in (w.q, w.k, w.v))
    mh = [m.contiguous().pin_memory() for m in masks]
    outs = [torch.full((w.B, w.N, w.H, 64), float("nan"), dtype=w.q.dtype).pin_memory() for _ in masks]
    stream = torch.cuda.Stream()
    hs(mh, q, k, v, outs, stream=stream)
    stream.synchronize()
    assert rra.rra_get_device_error(hs.err) == 0
    _check(w, masks, outs, w.B)
    # a smaller batch through the same object, twice in a row (buffers reused)
    Bp = 4
    outs2 = [torch.full((Bp, w.N, w.H, 64), float("nan"), dtype=w.q.dtype).pin_memory() for _ in masks]
    for _ in range(2):
        hs([m[:Bp].contiguous().pin_memory() for m in masks], q[:Bp].contiguous().pin_memory(),
           k[:Bp].contiguous().pin_memory(), v[:Bp].contiguous().pin_memory(), outs2, stream=stream)
    stream.synchronize()
    assert rra.rra_get_device_error(hs.err) == 0
    _check(w, masks, outs2, Bp)


def test_host_stream_rejects_device_or_unpinned_tensors():
    w, masks = _workload()
    hs = rra.HostStream(w.B, w.N, w.H, w.q.dtype, stages=1, chunk=4)
    outs = [torch.empty((w.B, w.N, w.H, 64), dtype=w.q.dtype).pin_memory()]
    q, k, v = (t.contiguous().pin_memory() for t in (w.q, w.k, w.v))
    with pytest.raises(ValueError):
        hs([masks[0]], q, k, v, outs)  # mask not pinned
    with pytest.raises(ValueError):
        hs([masks[0].pin_memory()], w.q.cuda(), k, v, outs)  # q on the device

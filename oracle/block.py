"""Float64 oracle of a transformer block on packed token rows: the dense layers around the path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and by ``bench.py``'s CPU leg; never by the
product package, with which it shares no code.  It serves the attention-vs-MLP split of a
token-pruned ViT block ("Dispatch-Aware Ragged Attention for Pruned Vision Transformers",
aissential.tech summary, "In practice": decompose attention vs. MLP latency contributions).
The pages name the block (a DeiT block) but print none of its layers; each layer here is its
textbook definition, in float64, and the block is the pre-norm ViT block, on the packed rows
x [T, C] of B images (cu_seqlens cu):

    h  = LN1(x)                          LN(z) = (z - mean) / sqrt(var + eps) * gamma + beta,
                                          mean and var (biased) over the row
    q | k | v = h Wqkv^T + bqkv           a linear layer: z W^T + b, W [out, in]
    a  = attention of q, k, v per image and head over cu (the path's oracle, ``oracle.attend``)
    x1 = x + a Wo^T + bo
    h2 = LN2(x1)
    m  = GELU(h2 W1^T + b1)              GELU(z) = z Phi(z) = z (1 + erf(z / sqrt 2)) / 2
    y  = x1 + m W2^T + b2

With ``round_bf16`` every stored activation (h, q, k, v, a, x1, h2, m, y) is rounded to the
nearest bf16 (ties to even), where a bf16 model stores it; the arithmetic in between stays
float64.  Parity unpinned: none -- the pins are in ``tests/test_oracle_block.py``.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

from .oracle import attend

STORED = ("h", "q", "k", "v", "a", "x1", "h2", "m", "y")


def bf16_round(a) -> np.ndarray:
    """Nearest bf16 value (8 significant bits, ties to even) of each float64, as float64.

    a = f 2^e with 0.5 <= |f| < 1: scaled by 2^(8-e) it lies in [128, 256), and np.rint rounds
    it to an integer with ties to even; below 2^-126 the grid is bf16's subnormal spacing 2^-133
    (the exponent is held at -125).  Finite values at or past (2 - 2^-8) 2^127 become infinite;
    infinities and NaN pass through."""
    a = np.asarray(a, dtype=np.float64)
    out = a.copy()
    fin = np.isfinite(a)
    f, e = np.frexp(a[fin])
    e = np.maximum(e, -125)
    r = np.ldexp(np.rint(np.ldexp(a[fin], 8 - e)), e - 8)
    r[np.abs(r) >= 2.0 ** 128] = np.inf * np.sign(r[np.abs(r) >= 2.0 ** 128])
    out[fin] = r
    return out


def layernorm(x, gamma, beta, eps: float) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    mean = x.mean(axis=1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def linear(x, w, b=None) -> np.ndarray:
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)
    return y


def gelu(z) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def block(x, cu, weights, H: int, eps: float = 1e-6, round_bf16: bool = True, scale: float = 0.0, lib=None):
    """The block on packed rows x [T, C] (T = cu[-1]); returns a dict of every stored activation
    (float64, rounded to bf16 when ``round_bf16``).  ``weights`` maps qkv_w [3C, C], qkv_b, proj_w
    [C, C], proj_b, fc1_w [4C, C], fc1_b, fc2_w [C, 4C], fc2_b, ln1_g, ln1_b, ln2_g, ln2_b to
    float64 arrays."""
    R = bf16_round if round_bf16 else (lambda z: np.asarray(z, dtype=np.float64))
    W = {k: np.asarray(v, dtype=np.float64) for k, v in weights.items()}
    x = np.asarray(x, dtype=np.float64)
    T, C = x.shape
    cu = np.asarray(cu, dtype=np.int64)
    assert cu[-1] == T and C == 64 * H
    out = {}
    out["h"] = R(layernorm(x, W["ln1_g"], W["ln1_b"], eps))
    qkv = linear(out["h"], W["qkv_w"], W["qkv_b"])
    for i, name in enumerate("qkv"):
        out[name] = R(qkv[:, i * C:(i + 1) * C])
    a = attend(out["q"].reshape(T, H, 64), out["k"].reshape(T, H, 64), out["v"].reshape(T, H, 64), cu, H, 64,
               scale=scale, dtype="f64", lib=lib)
    out["a"] = R(np.asarray(a, dtype=np.float64).reshape(T, C))
    out["x1"] = R(x + linear(out["a"], W["proj_w"], W["proj_b"]))
    out["h2"] = R(layernorm(out["x1"], W["ln2_g"], W["ln2_b"], eps))
    out["m"] = R(gelu(linear(out["h2"], W["fc1_w"], W["fc1_b"])))
    out["y"] = R(out["x1"] + linear(out["m"], W["fc2_w"], W["fc2_b"]))
    return out

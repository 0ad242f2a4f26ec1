"""Pins of the block oracle (oracle/block.py) against what mathematics fixes, and planted
mistakes each pin must catch.  CPU only."""
import math

import numpy as np
import pytest
import torch

from oracle import block as OB

rng = np.random.default_rng(5)


# ------------------------------------------------------------------------------ bf16 rounding

def test_bf16_round_fixed_points_are_every_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (bits << 16).view(np.float32).astype(np.float64)
    fin = np.isfinite(vals)
    assert np.array_equal(OB.bf16_round(vals[fin]), vals[fin])


def test_bf16_round_ties_to_even_and_matches_an_independent_conversion():
    # midpoints between consecutive positive bf16 values go to the one with an even last bit
    b = np.arange(0x3F80, 0x3FA0, dtype=np.uint32)
    lo = (b << 16).view(np.float32).astype(np.float64)
    hi = ((b + 1) << 16).view(np.float32).astype(np.float64)
    mid = (lo + hi) / 2
    want = np.where(b % 2 == 0, lo, hi)
    assert np.array_equal(OB.bf16_round(mid), want)
    # fp32 values (so a conversion through fp32 rounds once): torch's bf16 conversion agrees
    x = np.concatenate([rng.standard_normal(20000), rng.standard_normal(2000) * 1e-39, rng.standard_normal(2000) * 1e37])
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(OB.bf16_round(x32.astype(np.float64)), ref)


# ------------------------------------------------------------------------------ layers

def test_layernorm_hand_case_and_invariants():
    y = OB.layernorm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.ones(4), np.zeros(4), eps=0.0)
    # mean 2.5, biased variance 1.25
    want = (np.array([1.0, 2.0, 3.0, 4.0]) - 2.5) / math.sqrt(1.25)
    assert np.allclose(y[0], want, rtol=0, atol=1e-15)
    x = rng.standard_normal((7, 96)) * 3 + 2
    z = OB.layernorm(x, np.ones(96), np.zeros(96), eps=1e-12)
    assert np.allclose(z.mean(1), 0, atol=1e-12) and np.allclose(z.var(1), 1, atol=1e-9)
    # affine in gamma, beta; unchanged by a positive scale and a shift of the row
    g, bb = rng.standard_normal(96), rng.standard_normal(96)
    assert np.allclose(OB.layernorm(x, g, bb, 1e-12), z * g + bb, atol=1e-12)
    assert np.allclose(OB.layernorm(4 * x - 7, g, bb, 1e-12), z * g + bb, atol=1e-9)


def test_gelu_closed_forms():
    # GELU(z) = z Phi(z): Phi(1) = 0.8413447460685429, Phi(2) = 0.9772498680518208 (normal tables)
    assert abs(OB.gelu(1.0) - 0.8413447460685429) < 1e-15
    assert abs(OB.gelu(-1.0) - (-(1 - 0.8413447460685429))) < 1e-15
    assert abs(OB.gelu(2.0) - 2 * 0.9772498680518208) < 1e-15
    assert OB.gelu(0.0) == 0.0
    z = rng.standard_normal(1000) * 4
    assert np.allclose(OB.gelu(z) - OB.gelu(-z), z, atol=1e-13)  # Phi(z) + Phi(-z) = 1


def test_linear_identity_and_bias():
    x = rng.standard_normal((5, 64))
    b = rng.standard_normal(64)
    assert np.array_equal(OB.linear(x, np.eye(64), b), x + b)


# ------------------------------------------------------------------------------ block

def _weights(C, scale=0.02, zero=False):
    w = {
        "qkv_w": rng.standard_normal((3 * C, C)) * scale, "qkv_b": rng.standard_normal(3 * C) * scale,
        "proj_w": rng.standard_normal((C, C)) * scale, "proj_b": rng.standard_normal(C) * scale,
        "fc1_w": rng.standard_normal((4 * C, C)) * scale, "fc1_b": rng.standard_normal(4 * C) * scale,
        "fc2_w": rng.standard_normal((C, 4 * C)) * scale, "fc2_b": rng.standard_normal(C) * scale,
        "ln1_g": np.ones(C), "ln1_b": np.zeros(C), "ln2_g": np.ones(C), "ln2_b": np.zeros(C),
    }
    if zero:
        for k in w:
            if not k.startswith("ln"):
                w[k] = np.zeros_like(w[k])
    return w


def pin_zero_weights_block_is_identity():
    """All linear weights and biases zero: q = k = v = 0, so a = 0, x1 = x; GELU(0) = 0, so y = x."""
    H, C = 2, 128
    cu = np.array([0, 3, 3, 10, 11])
    x = OB.bf16_round(rng.standard_normal((11, C)))
    out = OB.block(x, cu, _weights(C, zero=True), H)
    return np.array_equal(out["a"], np.zeros_like(x)) and np.array_equal(out["y"], x)


def pin_uniform_attention_block_is_image_mean():
    """q = k = 0 gives uniform weights over the image: with v = h and an identity projection,
    x1 = x + (mean of h over the row's image); with a zero MLP, y = x1."""
    H, C = 2, 128
    cu = np.array([0, 4, 9, 16])
    x = rng.standard_normal((16, C))
    w = _weights(C, zero=True)
    w["qkv_w"][2 * C:] = np.eye(C)
    w["proj_w"] = np.eye(C)
    out = OB.block(x, cu, w, H, round_bf16=False)
    h = OB.layernorm(x, w["ln1_g"], w["ln1_b"], 1e-6)
    want = x.copy()
    for b in range(3):
        want[cu[b]:cu[b + 1]] += h[cu[b]:cu[b + 1]].mean(0)
    return np.allclose(out["y"], want, rtol=0, atol=1e-12)


def test_block_pins():
    assert pin_zero_weights_block_is_identity()
    assert pin_uniform_attention_block_is_image_mean()


# ------------------------------------------------------------------------------ planted mistakes

def _pins_pass():
    try:
        test_layernorm_hand_case_and_invariants()
        test_gelu_closed_forms()
        test_linear_identity_and_bias()
        return pin_zero_weights_block_is_identity() and pin_uniform_attention_block_is_image_mean()
    except AssertionError:
        return False


MUTANTS = {
    "gelu_tanh": ("gelu", lambda z: 0.5 * np.asarray(z, np.float64) * (
        1 + np.tanh(math.sqrt(2 / math.pi) * (np.asarray(z, np.float64) + 0.044715 * np.asarray(z, np.float64) ** 3)))),
    "layernorm_unbiased_var": ("layernorm", lambda x, g, b, eps: (np.asarray(x) - np.asarray(x).mean(1, keepdims=True))
                               / np.sqrt(np.asarray(x).var(1, ddof=1, keepdims=True) + eps) * g + b),
    "layernorm_no_mean": ("layernorm", lambda x, g, b, eps: np.asarray(x) / np.sqrt(
        (np.asarray(x) ** 2).mean(1, keepdims=True) + eps) * g + b),
    "linear_no_bias": ("linear", lambda x, w, b=None: np.asarray(x, np.float64) @ np.asarray(w, np.float64).T),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(OB, attr, fn)
    assert not _pins_pass(), f"mutant {name} passed every pin"


def test_dropped_residual_is_caught(monkeypatch):
    """A block whose x1 forgets the residual x (x1 = a Wo^T + bo) fails the identity pin."""
    def block_no_residual(x, cu, weights, H, eps=1e-6, round_bf16=True, scale=0.0, lib=None):
        R = OB.bf16_round
        W = {k: np.asarray(v, np.float64) for k, v in weights.items()}
        x = np.asarray(x, np.float64)
        T, C = x.shape
        h = R(OB.layernorm(x, W["ln1_g"], W["ln1_b"], eps))
        qkv = OB.linear(h, W["qkv_w"], W["qkv_b"])
        q, k, v = (R(qkv[:, i * C:(i + 1) * C]).reshape(T, H, 64) for i in range(3))
        a = R(OB.attend(q, k, v, cu, H, 64, dtype="f64").reshape(T, C))
        x1 = R(OB.linear(a, W["proj_w"], W["proj_b"]))  # the mistake: no "x +"
        m = R(OB.gelu(OB.linear(R(OB.layernorm(x1, W["ln2_g"], W["ln2_b"], eps)), W["fc1_w"], W["fc1_b"])))
        return {"a": a, "y": R(x1 + OB.linear(m, W["fc2_w"], W["fc2_b"]))}
    monkeypatch.setattr(OB, "block", block_no_residual)
    assert not pin_zero_weights_block_is_identity()

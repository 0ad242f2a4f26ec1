"""Seeded synthetic inputs for the pack -> attend -> unpack path.

This module only draws random numbers: per-image keep masks (the pruning
decision, an *input* of the path) and padded Q/K/V tensors.  It holds none of
the path's arithmetic, so both the CUDA path and the CPU oracle can be fed
from it without sharing any computation.

The shapes follow the token-pruned DeiT workloads of "Dispatch-Aware Ragged
Attention for Pruned Vision Transformers" (sota2.com card, Abstract: ViT
sequences of at most 197 tokens at 224x224 and 577 at 384x384; aissential.tech
summary, Summary: DeiT-T/S/B with Threshold-l2, EViT and other pruning
methods).  The pages' own workloads are ImageNet-1k activations of trained
DeiT models; neither weights nor data are available, so seeded Gaussian
activations and synthetic pruning scores stand in for them.

Recipe (all draws from ``numpy.random.default_rng`` seeded through
``SeedSequence([seed, config_id, B, round(1000*r), stage_count])``, in the
order Q, K, V, then scores, then masks/lengths):

* values: fp32 normal with the config's standard deviation, rounded to
  fp16/bf16 with round-to-nearest-even (numpy / torch conversions);
* index 0 of every image is the CLS token and is always kept;
* keep-ratio r over the N-1 patches keeps k = floor(r*(N-1) + 0.5) patches,
  so L = k + 1 tokens survive;
* top-k selection orders by higher score, ties broken by lower index.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Sequence

import numpy as np
import torch

D_HEAD = 64

_TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@dataclass
class Workload:
    """One synthetic call: padded Q/K/V [B, N, H, d] plus one keep mask per stage."""

    name: str
    B: int
    N: int
    H: int
    d: int
    dtype: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    masks: List[torch.Tensor]          # uint8 [B, N], nonzero = keep
    seed: int
    recipe: str
    params: dict = field(default_factory=dict)

    @property
    def lengths(self) -> List[np.ndarray]:
        return [m.numpy().astype(bool).sum(axis=1) for m in self.masks]

    @property
    def total_tokens(self) -> int:
        """Sum over stages of the packed token count T."""
        return int(sum(int(l.sum()) for l in self.lengths))


def _rng(seed: int, config_id: int, B: int, r: float = 0.0, stages: int = 1) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed), int(config_id), int(B), int(round(1000 * r)), int(stages)])
    return np.random.default_rng(ss)


def _values(rng: np.random.Generator, B: int, N: int, H: int, d: int, std: float, dtype: str):
    out = []
    for _ in range(3):  # Q, K, V in that order
        x = rng.standard_normal((B, N, H, d), dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        t = torch.from_numpy(x).to(_TORCH_DTYPES[dtype])
        del x
        out.append(t.contiguous())
    return out


def keep_count(r: float, n_patches: int) -> int:
    """Number of patches kept at ratio r (CLS excluded)."""
    return int(np.floor(r * n_patches + 0.5))


def _topk_mask_row(score: np.ndarray, k: int, N: int, candidates: np.ndarray | None = None) -> np.ndarray:
    """Keep CLS plus the k highest-scoring patches (ties: lower index first)."""
    row = np.zeros(N, dtype=np.uint8)
    row[0] = 1
    if candidates is None:
        candidates = np.arange(1, N)
    s = score[candidates]
    order = np.argsort(-s, kind="stable")
    row[candidates[order[:k]]] = 1
    return row


def _random_subset_row(rng: np.random.Generator, L: int, N: int) -> np.ndarray:
    row = np.zeros(N, dtype=np.uint8)
    row[0] = 1
    if L > 1:
        row[rng.choice(N - 1, L - 1, replace=False) + 1] = 1
    return row


def _mk(name, B, N, H, dtype, qkv, masks, seed, recipe, **params) -> Workload:
    q, k, v = qkv
    return Workload(name=name, B=B, N=N, H=H, d=D_HEAD, dtype=dtype, q=q, k=k, v=v,
                    masks=[torch.from_numpy(np.ascontiguousarray(m)) for m in masks],
                    seed=seed, recipe=recipe, params=params)


def config1(seed: int = 0) -> Workload:
    """Tiny DeiT-T shape: B=4, H=3, N=197, L_b ~ U{20..197}, random subset, fp16 N(0,1)."""
    B, N, H = 4, 197, 3
    rng = _rng(seed, 1, B)
    qkv = _values(rng, B, N, H, D_HEAD, 1.0, "f16")
    lengths = rng.integers(20, N + 1, size=B)
    mask = np.stack([_random_subset_row(rng, int(L), N) for L in lengths])
    return _mk("config1_deit_t_tiny", B, N, H, "f16", qkv, [mask], seed,
               "L_b ~ U{20..197}; CLS + uniform random subset; fp16 N(0,1)")


def config2(seed: int = 0) -> Workload:
    """DeiT-S shape: B=64, H=6, N=197; l2-norm scores of N(0, I_384) embeddings, r_b ~ U[0.3,0.7]."""
    B, N, H = 64, 197, 6
    rng = _rng(seed, 2, B)
    qkv = _values(rng, B, N, H, D_HEAD, 1.0, "bf16")
    z = rng.standard_normal((B, N - 1, 384), dtype=np.float32)
    score = np.concatenate([np.zeros((B, 1), np.float64), np.linalg.norm(z.astype(np.float64), axis=-1)], axis=1)
    ratios = rng.uniform(0.3, 0.7, size=B)
    mask = np.stack([_topk_mask_row(score[b], keep_count(ratios[b], N - 1), N) for b in range(B)])
    return _mk("config2_deit_s_l2topk", B, N, H, "bf16", qkv, [mask], seed,
               "score = ||z||_2, z ~ N(0, I_384); r_b ~ U[0.3,0.7]; top-k + CLS; bf16 N(0,1)")


def config3(B: int, seed: int = 0) -> Workload:
    """DeiT-B shape at 80% pruning: H=12, N=197, L_b = 40 + U{-4..4}, bf16 N(0,1)."""
    N, H = 197, 12
    rng = _rng(seed, 3, B)
    qkv = _values(rng, B, N, H, D_HEAD, 1.0, "bf16")
    lengths = 40 + rng.integers(-4, 5, size=B)
    mask = np.stack([_random_subset_row(rng, int(L), N) for L in lengths])
    return _mk(f"config3_deit_b_keep0.2_B{B}", B, N, H, "bf16", qkv, [mask], seed,
               "L_b = 40 + U{-4..4} incl. CLS; random subset; bf16 N(0,1)", batch=B)


def config4(seed: int = 0, B: int = 64) -> Workload:
    """DeiT-B at 384x384: B=64, H=12, N=577; top-k of U(0,1) scores, r_b ~ U[0.3,0.7]; bf16 N(0, 0.5^2)."""
    N, H = 577, 12
    rng = _rng(seed, 4, B)
    qkv = _values(rng, B, N, H, D_HEAD, 0.5, "bf16")
    score = np.concatenate([np.zeros((B, 1)), rng.uniform(0.0, 1.0, size=(B, N - 1))], axis=1)
    ratios = rng.uniform(0.3, 0.7, size=B)
    mask = np.stack([_topk_mask_row(score[b], keep_count(ratios[b], N - 1), N) for b in range(B)])
    return _mk(f"config4_deit_b384_B{B}", B, N, H, "bf16", qkv, [mask], seed,
               "top-k of U(0,1) scores, r_b ~ U[0.3,0.7]; bf16 N(0, 0.5^2)")


def config5(r: float, B: int, seed: int = 0) -> Workload:
    """Sweep cell: H=12, N=197, fixed keep ratio r (top-k of U(0,1) scores), bf16 N(0,1)."""
    N, H = 197, 12
    rng = _rng(seed, 5, B, r)
    qkv = _values(rng, B, N, H, D_HEAD, 1.0, "bf16")
    score = np.concatenate([np.zeros((B, 1)), rng.uniform(0.0, 1.0, size=(B, N - 1))], axis=1)
    k = keep_count(r, N - 1)
    mask = np.stack([_topk_mask_row(score[b], k, N) for b in range(B)])
    return _mk(f"config5_deit_b_r{r}_B{B}", B, N, H, "bf16", qkv, [mask], seed,
               "fixed r; top-k of U(0,1) scores + CLS; bf16 N(0,1)", ratio=r, batch=B)


def config5_staged(B: int, seed: int = 0, ratio: float = 0.7, stages: int = 3) -> Workload:
    """EViT-like three-stage row: nested masks, each stage keeping `ratio` of the surviving patches.

    All stages read the same padded Q/K/V; stage s keeps floor(ratio*k_{s-1}+0.5) patches of
    the previous stage's survivors (k_0 = N-1), ranked by a fresh U(0,1) score per stage.
    """
    N, H = 197, 12
    rng = _rng(seed, 5, B, ratio, stages)
    qkv = _values(rng, B, N, H, D_HEAD, 1.0, "bf16")
    masks = []
    prev = np.ones((B, N), dtype=np.uint8)
    k = N - 1
    for _ in range(stages):
        k = keep_count(ratio, k)
        score = np.concatenate([np.zeros((B, 1)), rng.uniform(0.0, 1.0, size=(B, N - 1))], axis=1)
        cur = np.stack([_topk_mask_row(score[b], k, N, candidates=np.nonzero(prev[b, 1:])[0] + 1)
                        for b in range(B)])
        masks.append(cur)
        prev = cur
    return _mk(f"config5_deit_b_3stage{ratio}_B{B}", B, N, H, "bf16", qkv, masks, seed,
               f"{stages} nested stages keeping {ratio} of survivors; bf16 N(0,1)",
               ratio=ratio, batch=B, stages=stages)


def embeddings(B: int, N: int, C: int = 384, dtype: str = "bf16", seed: int = 0, kind: str = "normal") -> torch.Tensor:
    """Token embeddings [B, N, C] for the token-selection step (DeiT-S width 384 by default).

    kind "normal": N(0, 1) rounded to the 16-bit type; kind "ties": small integers in [-3, 3]
    (many tokens share a norm); kind "nan": normal with the embedding of a few tokens set to NaN."""
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), 77, int(B), int(N), int(C)]))
    if kind == "ties":
        x = rng.integers(-3, 4, size=(B, N, C)).astype(np.float32)
    else:
        x = rng.standard_normal((B, N, C), dtype=np.float32)
        if kind == "nan":
            bad = rng.integers(1, N, size=(B, 3))
            for b in range(B):
                x[b, bad[b], 0] = np.nan
    return torch.from_numpy(x).to(_TORCH_DTYPES[dtype]).contiguous()


def block_weights(C: int, seed: int = 0, std: float = 0.02) -> dict:
    """Synthetic weights of one DeiT block of width C (there are no trained weights): the linear
    layers N(0, std^2) as a truncated-normal init draws them (nn.Linear layout [out, in]), biases
    N(0, std^2), LayerNorm gamma 1 + N(0, 0.1^2) and beta N(0, 0.1^2) (so the affine part is
    exercised); all rounded to bf16, on the CPU."""
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), 91, int(C)]))
    shapes = {"qkv_w": (3 * C, C), "qkv_b": (3 * C,), "proj_w": (C, C), "proj_b": (C,), "fc1_w": (4 * C, C),
              "fc1_b": (4 * C,), "fc2_w": (C, 4 * C), "fc2_b": (C,)}
    w = {k: np.clip(rng.standard_normal(sh), -2, 2) * std for k, sh in shapes.items()}
    for ln in ("ln1", "ln2"):
        w[ln + "_g"] = 1 + 0.1 * rng.standard_normal(C)
        w[ln + "_b"] = 0.1 * rng.standard_normal(C)
    return {k: torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16) for k, v in w.items()}


def block_input(T: int, C: int, seed: int = 0) -> torch.Tensor:
    """Packed token rows [T, C] entering a block: N(0, 1) in bf16, on the CPU."""
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), 92, int(T), int(C)]))
    return torch.from_numpy(rng.standard_normal((T, C), dtype=np.float32)).to(torch.bfloat16)


def keep_counts(B: int, N: int, lo: float = 0.3, hi: float = 0.7, seed: int = 0) -> np.ndarray:
    """Patches kept per image at ratios r_b ~ U[lo, hi] (the configs' recipe), int32 [B]."""
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), 78, int(B), int(N)]))
    return np.array([keep_count(r, N - 1) for r in rng.uniform(lo, hi, size=B)], dtype=np.int32)


def from_lengths(lengths: Sequence[int], N: int, H: int, dtype: str = "bf16", seed: int = 0,
                 std: float = 1.0, contiguous_prefix: bool = False) -> Workload:
    """Edge-case workload with given per-image kept lengths (0 <= L_b <= N)."""
    B = len(lengths)
    rng = _rng(seed, 99, B, 0.0, int(sum(lengths)) % 100003)
    qkv = _values(rng, B, N, H, D_HEAD, std, dtype)
    rows = []
    for L in lengths:
        L = int(L)
        row = np.zeros(N, dtype=np.uint8)
        if L > 0:
            if contiguous_prefix:
                row[:L] = 1
            else:
                row = _random_subset_row(rng, L, N)
        rows.append(row)
    mask = np.stack(rows) if B else np.zeros((0, N), np.uint8)
    return _mk(f"lengths_{B}x{N}", B, N, H, dtype, qkv, [mask], seed,
               "explicit lengths; random subset incl. CLS", lengths=list(map(int, lengths)))


def by_name(name: str, seed: int = 0) -> Workload:
    """Resolve a workload by short name: c1, c2, c3:B, c4, c5:r:B, c5s:B."""
    parts = name.split(":")
    if parts[0] == "c1":
        return config1(seed)
    if parts[0] == "c2":
        return config2(seed)
    if parts[0] == "c3":
        return config3(int(parts[1]), seed)
    if parts[0] == "c4":
        return config4(seed)
    if parts[0] == "c5":
        return config5(float(parts[1]), int(parts[2]), seed)
    if parts[0] == "c5s":
        return config5_staged(int(parts[1]), seed)
    raise ValueError(f"unknown workload {name!r}")


# ------------------------------------------------------------------------------------ sweep inputs

def device_values(B: int, N: int, H: int, dtype: str = "bf16", seed: int = 0, std: float = 1.0,
                  device="cuda") -> List[torch.Tensor]:
    """Padded Q, K, V [B, N, H, 64] drawn directly on the device (torch's seeded generator there),
    for timing-only sweeps whose cells are never compared with the oracle: N(0, std^2) rounded to
    the 16-bit type, the same distribution as the named configs' host draws."""
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([int(seed), 55, int(B), int(N), int(H)]).generate_state(1)[0]))
    out = []
    for _ in range(3):
        x = torch.randn(B, N, H, D_HEAD, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out.append(x.to(_TORCH_DTYPES[dtype]).contiguous())
    return out


def sweep_masks(name: str, seed: int = 0) -> List[np.ndarray]:
    """Keep masks of a named workload (same recipes and seeds as ``by_name``) without drawing its
    Q/K/V: for c1/c3/c5 cells the lengths and kept positions come from a mask-only stream, so they
    follow the config's recipe but are not the same draws as the full workload's."""
    parts = name.split(":")
    kind = parts[0]
    if kind == "c1":
        B, N = 4, 197
        rng = np.random.default_rng(np.random.SeedSequence([seed, 1, B, 0, 1, 66]))
        lengths = rng.integers(20, N + 1, size=B)
        return [np.stack([_random_subset_row(rng, int(L), N) for L in lengths])]
    if kind == "c2":
        return [m.numpy() for m in config2(seed).masks]
    if kind == "c3":
        B, N = int(parts[1]), 197
        rng = np.random.default_rng(np.random.SeedSequence([seed, 3, B, 0, 1, 66]))
        lengths = 40 + rng.integers(-4, 5, size=B)
        return [np.stack([_random_subset_row(rng, int(L), N) for L in lengths])]
    if kind == "c4":
        B, N = 64, 577
        rng = np.random.default_rng(np.random.SeedSequence([seed, 4, B, 0, 1, 66]))
        score = np.concatenate([np.zeros((B, 1)), rng.uniform(0.0, 1.0, size=(B, N - 1))], axis=1)
        ratios = rng.uniform(0.3, 0.7, size=B)
        return [np.stack([_topk_mask_row(score[b], keep_count(ratios[b], N - 1), N) for b in range(B)])]
    if kind == "c5":
        r, B, N = float(parts[1]), int(parts[2]), 197
        rng = np.random.default_rng(np.random.SeedSequence([seed, 5, B, int(round(1000 * r)), 1, 66]))
        score = np.concatenate([np.zeros((B, 1)), rng.uniform(0.0, 1.0, size=(B, N - 1))], axis=1)
        k = keep_count(r, N - 1)
        return [np.stack([_topk_mask_row(score[b], k, N) for b in range(B)])]
    if kind == "c5s":
        B, N, ratio = int(parts[1]), 197, 0.7
        rng = np.random.default_rng(np.random.SeedSequence([seed, 5, B, 700, 3, 66]))
        masks, prev, k = [], np.ones((B, N), dtype=np.uint8), N - 1
        for _ in range(3):
            k = keep_count(ratio, k)
            score = np.concatenate([np.zeros((B, 1)), rng.uniform(0.0, 1.0, size=(B, N - 1))], axis=1)
            cur = np.stack([_topk_mask_row(score[b], k, N, candidates=np.nonzero(prev[b, 1:])[0] + 1)
                            for b in range(B)])
            masks.append(cur)
            prev = cur
        return masks
    raise ValueError(f"unknown workload {name!r}")


def shape_of(name: str):
    """(B, N, H, dtype, std) of a named workload."""
    parts = name.split(":")
    kind = parts[0]
    if kind == "c1":
        return 4, 197, 3, "f16", 1.0
    if kind == "c2":
        return 64, 197, 6, "bf16", 1.0
    if kind == "c3":
        return int(parts[1]), 197, 12, "bf16", 1.0
    if kind == "c4":
        return 64, 577, 12, "bf16", 0.5
    if kind == "c5":
        return int(parts[2]), 197, 12, "bf16", 1.0
    if kind == "c5s":
        return int(parts[1]), 197, 12, "bf16", 1.0
    raise ValueError(f"unknown workload {name!r}")


def sweep_names() -> List[str]:
    """Every cell the configs name: config 5's keep-ratio x batch grid and its three-stage row per
    batch, config 1, config 2, config 3's batch sweep and config 4."""
    names = [f"c5:{r}:{B}" for r in (1.0, 0.7, 0.5, 0.3, 0.2, 0.1) for B in (1, 4, 16, 64, 256, 512)]
    names += [f"c5s:{B}" for B in (1, 4, 16, 64, 256, 512)]
    names += ["c1", "c2"] + [f"c3:{B}" for B in (1, 2, 4, 64, 256)] + ["c4"]
    return names

"""Seeded synthetic inputs for the attention workloads.

This module generates inputs only; it holds none of the method's arithmetic.
Both the CUDA path and the float64 oracle consume what it produces, so they see
bit-identical bf16 inputs.

Recipe (shared by all workloads): float32 draws from numpy's PCG64, modified
per workload as described below, then rounded to bf16 with round-to-nearest-
even.  Every (tensor, b, h) head has its own stream, seeded with
``[20260 + workload index, tensor index, b, h]`` (tensor index: Q=0, K=1, V=2,
dO=3), so a single head can be regenerated without the rest.  Choices that a
recipe makes per head (outlier channels, scales, outlier tokens) come from a
separate stream ``[20260 + workload index, 100 + tensor index, b, h]``.

The shapes stand in for the pages' workload (Wan2.1 DiT attention: 12 heads of
dimension 128, and the 6-head, 31200-token shape the fastvideo-kernel commit
times); no dataset or model weights are involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

TENSORS = ("q", "k", "v", "do")


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    H: int
    Lq: int
    Lk: int
    D: int
    sm_scale: float
    recipe: str
    description: str

    @property
    def seed(self) -> int:
        return 20260 + self.index

    def nominal_flops(self) -> dict:
        """Nominal matmul flops: forward 4*B*H*Lq*Lk*D, backward 2.5x that."""
        fwd = 4.0 * self.B * self.H * self.Lq * self.Lk * self.D
        return dict(fwd=fwd, bwd=2.5 * fwd, total=3.5 * fwd)


WORKLOADS = [
    Workload("tiny", 0, 1, 2, 256, 256, 64, 1.0 / 8.0, "normal",
             "B1 H2 L256 D64, N(0,1)"),
    Workload("outlier_channels_4096", 1, 1, 12, 4096, 4096, 128, 1.0 / math.sqrt(128.0),
             "outlier_channels",
             "B1 H12 L4096 D128; Q,K N(0,1) with the same 4 random channels per head x20"),
    Workload("wan_6h_31200", 2, 1, 6, 31200, 31200, 128, 1.0 / math.sqrt(128.0), "normal",
             "B1 H6 L31200 D128, N(0,1) (tail KV tile of 96 keys)"),
    Workload("scaled_heads_16384", 3, 2, 12, 16384, 16384, 128, 1.0 / math.sqrt(128.0),
             "per_head_scale",
             "B2 H12 L16384 D128, N(0,1) x per-head U[0.5,2] scale per tensor"),
    Workload("large_40h_75600", 4, 1, 40, 75600, 75600, 128, 1.0 / math.sqrt(128.0),
             "token_outliers",
             "B1 H40 L75600 D128, N(0,1) with 1% of token rows x8 in Q, K, V"),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def get(name: str) -> Workload:
    return BY_NAME[name]


def custom(B, H, Lq, Lk, D, sm_scale=None, recipe="normal", seed_index=99, name="custom"):
    """A workload of arbitrary shape (for ragged/edge-case tests)."""
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    return Workload(name, seed_index, B, H, Lq, Lk, D, float(sm_scale), recipe,
                    "custom %dx%dx%dx%dx%d" % (B, H, Lq, Lk, D))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest, ties to even); returns the
    uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def head_f32(w: Workload, tensor: str, b: int, h: int) -> np.ndarray:
    """float32 values of one head of one tensor, before bf16 rounding."""
    t = TENSORS.index(tensor)
    L = w.Lq if tensor in ("q", "do") else w.Lk
    rng = np.random.default_rng([w.seed, t, b, h])
    x = rng.standard_normal((L, w.D), dtype=np.float32)
    meta = np.random.default_rng([w.seed, 100 + t, b, h])
    if w.recipe == "normal":
        pass
    elif w.recipe == "outlier_channels":
        if tensor in ("q", "k"):
            # the same 4 channels for Q and K of a head: drawn from the Q-side stream
            chan_rng = np.random.default_rng([w.seed, 100, b, h])
            ch = chan_rng.choice(w.D, size=4, replace=False)
            x[:, ch] *= np.float32(20.0)
    elif w.recipe == "per_head_scale":
        x *= np.float32(meta.uniform(0.5, 2.0))
    elif w.recipe == "token_outliers":
        if tensor in ("q", "k", "v"):
            n = max(1, int(round(0.01 * L)))
            rows = meta.choice(L, size=n, replace=False)
            x[rows] *= np.float32(8.0)
    else:
        raise ValueError("unknown recipe %r" % w.recipe)
    return x


def head_bits(w: Workload, tensor: str, b: int, h: int) -> np.ndarray:
    """bf16 bit patterns (uint16 [L, D]) of one head of one tensor."""
    return f32_to_bf16_bits(head_f32(w, tensor, b, h))


def tensor_bits(w: Workload, tensor: str) -> np.ndarray:
    """bf16 bit patterns of a whole [B, H, L, D] tensor."""
    L = w.Lq if tensor in ("q", "do") else w.Lk
    out = np.empty((w.B, w.H, L, w.D), np.uint16)
    for b in range(w.B):
        for h in range(w.H):
            out[b, h] = head_bits(w, tensor, b, h)
    return out


def inputs(w: Workload, with_grad: bool = True) -> dict:
    """All inputs of a workload as uint16 bf16 bit patterns, drawn in the order
    Q, K, V, dO."""
    out = {t: tensor_bits(w, t) for t in ("q", "k", "v")}
    if with_grad:
        out["do"] = tensor_bits(w, "do")
    return out


# ----------------------------------------------------- block-sparse masks ----
# Tile masks for the block-sparse (VSA fine attention) entry points:
# uint8 [B, H, ceil(Lq/128), ceil(Lk/128)], nonzero = the 128-query tile
# attends the 128-key tile.  The pages' selection keeps, per query cube, the
# top-k key cubes of a coarse attention with k = max(1, min(ceil((1 -
# sparsity) * n), n)) and sparsity 0.9 (vsqa-test-1.3b metadata.json,
# attention.selection); with no trained model the k tiles are drawn here
# uniformly without replacement, each (b, h) from its own stream
# [20260 + workload index, 200, b, h].

SPARSE_TILE = 128


def topk_tiles(n_tiles: int, sparsity: float) -> int:
    """Key tiles kept per query tile at the given sparsity."""
    return max(1, min(math.ceil((1.0 - sparsity) * n_tiles), n_tiles))


def tile_mask(w: Workload, sparsity: float = 0.9) -> np.ndarray:
    """VSA-style selection: topk_tiles(nk, sparsity) distinct key tiles per
    query tile."""
    nq, nk = -(-w.Lq // SPARSE_TILE), -(-w.Lk // SPARSE_TILE)
    k = topk_tiles(nk, sparsity)
    out = np.zeros((w.B, w.H, nq, nk), np.uint8)
    for b in range(w.B):
        for h in range(w.H):
            rng = np.random.default_rng([w.seed, 200, b, h])
            for i in range(nq):
                out[b, h, i, rng.choice(nk, size=k, replace=False)] = 1
    return out


def random_tile_mask(w: Workload, p: float) -> np.ndarray:
    """Each (query tile, key tile) pair selected independently with
    probability p (empty rows and columns happen), stream
    [20260 + workload index, 201]."""
    nq, nk = -(-w.Lq // SPARSE_TILE), -(-w.Lk // SPARSE_TILE)
    rng = np.random.default_rng([w.seed, 201])
    return (rng.random((w.B, w.H, nq, nk)) < p).astype(np.uint8)

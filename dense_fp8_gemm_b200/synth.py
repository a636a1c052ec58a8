"""Seeded synthetic inputs for the Spense GEMM: weights, activations, scales,
masks and dense index sets.

This module holds none of the Spense arithmetic (no packing, no decoding, no
GEMM). It draws Gaussian tensors, quantizes them to FP8 e4m3 with absmax
scales, and builds masks and index sets. Both the CUDA path's tests and the CPU
oracle's tests take their inputs from here, so the two sides see identical
bytes.

Every tensor comes from its own PCG64 stream keyed by (seed, tensor id), so a
tensor does not depend on which other tensors were drawn before it.
"""
from __future__ import annotations

import numpy as np
import torch

E4M3_MAX = 448.0


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(tensor_id)]))


def normal(seed: int, tensor_id: int, shape, std: float) -> np.ndarray:
    g = rng(seed, tensor_id)
    return (g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def quantize_rows(x: np.ndarray):
    """Per-row absmax FP8 e4m3 quantization: s = absmax / 448 over the whole row
    (an all-zero row gets s = 1), q = e4m3(round-to-nearest-even(x / s)),
    saturated to +-448. Returns (q as uint8 bytes, s as float32)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    t = torch.from_numpy(x) / torch.from_numpy(s)[:, None]
    t = t.clamp_(-E4M3_MAX, E4M3_MAX)
    q = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    return q, s


def device_fp8_rows(seed: int, tensor_id: int, shape, std: float, device, outliers: bool = False):
    """The recipe of ``normal`` (+ ``weight_outliers`` when `outliers`) +
    ``quantize_rows`` drawn on the GPU, for weights too large to draw on the
    host in reasonable time (a 64-layer decoder stack): N(0, std) from torch's
    counter-based Philox generator on `device`, seeded from (seed, tensor_id);
    with `outliers`, a Bernoulli(0.01) subset of the entries (a second draw of
    the same generator) multiplied by 20; then per-row absmax FP8 e4m3
    quantisation (s = absmax / 448, 1 for an all-zero row; round to nearest
    even, saturated to +-448). Same distribution as the host recipe, not the
    same values. Returns (q uint8 [rows, cols], s float32 [rows]) on `device`."""
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) << 32) ^ int(tensor_id))
    w = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    w.mul_(std)
    if outliers:
        hit = torch.rand(tuple(shape), generator=g, device=device, dtype=torch.float32) < 0.01
        w[hit] *= 20.0
        del hit
    amax = w.abs().amax(dim=1)
    s = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    w.div_(s[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    q = w.to(torch.float8_e4m3fn).view(torch.uint8)
    del w
    return q, s.to(torch.float32)


def weight_outliers(seed: int, tensor_id: int, w: np.ndarray, frac: float = 0.01,
                    factor: float = 20.0) -> np.ndarray:
    """Multiply a Bernoulli(frac) subset of the entries by `factor`."""
    g = rng(seed, tensor_id)
    hit = g.random(size=w.shape, dtype=np.float32) < np.float32(frac)
    out = w.copy()
    out[hit] *= np.float32(factor)
    return out


def activation_outliers(seed: int, tensor_id: int, x: np.ndarray, channels: int = 4,
                        factor: float = 50.0) -> np.ndarray:
    """Multiply `channels` seeded input channels (columns) by `factor`."""
    g = rng(seed, tensor_id)
    cols = g.choice(x.shape[1], size=channels, replace=False)
    out = x.copy()
    out[:, cols] *= np.float32(factor)
    return out


def scored_dense_idx(seed: int, tensor_id: int, K: int, Kd: int) -> np.ndarray:
    """Top-Kd columns of a seeded U(0,1) score, ascending (an arbitrary
    score-selected dense set, as SpenseGPT+ produces)."""
    g = rng(seed, tensor_id)
    score = g.random(size=K)
    idx = np.argsort(-score, kind="stable")[:Kd]
    return np.sort(idx).astype(np.int32)


def random_mask(seed: int, tensor_id: int, N: int, K: int, keep_per_group=(2,),
                sparse_cols=None) -> np.ndarray:
    """A 0/1 mask [N, K] whose groups of four (over `sparse_cols`, default all
    columns) keep a number of entries drawn from `keep_per_group`. Columns
    outside `sparse_cols` are set to 1."""
    g = rng(seed, tensor_id)
    mask = np.ones((N, K), np.uint8)
    cols = np.arange(K) if sparse_cols is None else np.asarray(sparse_cols)
    G = cols.shape[0] // 4
    grp = cols[: 4 * G].reshape(G, 4)
    counts = g.choice(np.asarray(keep_per_group), size=(N, G))
    pri = g.random(size=(N, G, 4))
    order = np.argsort(pri, axis=2)
    rank = np.argsort(order, axis=2)
    keep = rank < counts[:, :, None]
    rows = np.arange(N)[:, None, None]
    mask[rows, grp[None, :, :]] = keep.astype(np.uint8)
    return mask

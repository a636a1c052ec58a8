"""The synthetic workloads the Spense GEMM is checked and measured on.

Shapes follow the linear layers of 32B- and 36B-class decoder models (hidden
5120) at decode-sized token batches, the setting of the pages' experiments
(Qwen3-32B / Seed-OSS-36B, FP8, B200). No model weights or datasets are used;
every tensor is drawn by ``synth`` from the seeds below.

Tensor ids: weight of shape i -> 100 + 10 i; its outlier stream -> 101 + 10 i;
its dense-index score -> 102 + 10 i; activations for (shape i, batch M) ->
10000 + 1000 i + M, their outlier stream -> 10000 + 1000 i + M + 500. Layer L
of a multi-layer workload adds 1000000 L to its weight ids (layer 0 is the
single-layer weight).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    shapes: tuple  # ((label, N, K), ...)
    batches: tuple  # token counts M
    dense_fracs: tuple = (0.25,)
    w_std: float = 0.02
    x_std: float = 1.0
    outliers: bool = False
    scattered: bool = False  # SpenseGPT+: dense set = top-scoring columns
    layers: int = 1
    note: str = ""


TINY = Workload("tiny", 0, (("w", 256, 512),), (8,),
                note="first 384 columns 2:4 by top-2 magnitude, last 128 dense")
ATTN32B = Workload("attn32b", 1, (("q_proj", 8192, 5120), ("k_proj", 1024, 5120),
                                  ("v_proj", 1024, 5120), ("o_proj", 5120, 8192)), (1, 8, 16))
FFN32B = Workload("ffn32b", 2, (("gate_up", 51200, 5120), ("down", 5120, 25600)), (1, 16, 64),
                  outliers=True)
SPENSE_PLUS = Workload("spensegpt_plus", 3, (("down", 5120, 25600),), (32,),
                       dense_fracs=(0.0, 0.125, 0.25, 0.5, 1.0), scattered=True)
CHAIN36B = Workload("chain36b", 4, (("q_proj", 10240, 5120), ("k_proj", 1024, 5120),
                                    ("v_proj", 1024, 5120), ("o_proj", 5120, 10240),
                                    ("gate_up", 55296, 5120), ("down", 5120, 27648)),
                    (1, 4, 16, 64, 256), layers=64)

ALL = (TINY, ATTN32B, FFN32B, SPENSE_PLUS, CHAIN36B)
BY_NAME = {w.name: w for w in ALL}


def dense_count(K: int, dense_frac: float) -> int:
    """Kd = round(dense_frac * K)."""
    return int(round(dense_frac * K))


@dataclass
class Weight:
    label: str
    W: np.ndarray  # uint8 [N, K] e4m3 bytes
    s_w: np.ndarray  # float32 [N]
    dense_idx: object  # int32 [Kd] ascending, or None for the tail
    Kd: int

    @property
    def N(self):
        return self.W.shape[0]

    @property
    def K(self):
        return self.W.shape[1]


def weight_id(i: int, layer: int = 0) -> int:
    """Tensor id of the weight of shape i in layer `layer`."""
    return 100 + 10 * i + 1000000 * layer


def make_weight(wl: Workload, i: int, dense_frac: float | None = None, layer: int = 0, rows=None) -> Weight:
    """The weight of shape i (layer `layer`), quantised per row. `rows`: draw a
    matrix of only that many rows (a sample with the shape's columns and
    distribution, from its own stream)."""
    label, N, K = wl.shapes[i]
    df = wl.dense_fracs[0] if dense_frac is None else dense_frac
    Kd = dense_count(K, df)
    tid = weight_id(i, layer) + (500000 if rows is not None else 0)
    w = synth.normal(wl.seed, tid, (N if rows is None else rows, K), wl.w_std)
    if wl.outliers:
        w = synth.weight_outliers(wl.seed, tid + 1, w)
    q, s = synth.quantize_rows(w)
    del w
    idx = synth.scored_dense_idx(wl.seed, 102 + 10 * i, K, Kd) if wl.scattered else None
    return Weight(label, q, s, idx, Kd)


def make_activations(wl: Workload, i: int, M: int):
    _, _, K = wl.shapes[i]
    x = synth.normal(wl.seed, 10000 + 1000 * i + M, (M, K), wl.x_std)
    if wl.outliers:
        x = synth.activation_outliers(wl.seed, 10000 + 1000 * i + M + 500, x)
    return synth.quantize_rows(x)


def algorithmic_bytes(N: int, K: int, Kd: int, M: int) -> int:
    """Bytes the method itself must move for one GEMM: packed values, 2-bit
    metadata, dense columns, weight scales, activations, activation scales and
    the bf16 output (split-K partials are not counted)."""
    Ks = K - Kd
    return N * Ks // 2 + N * Ks // 8 + N * Kd + 4 * N + M * K + 4 * M + 2 * M * N


def weight_bytes(N: int, K: int, Kd: int) -> int:
    Ks = K - Kd
    return N * Ks // 2 + N * Ks // 8 + N * Kd


def useful_flops(N: int, K: int, Kd: int, M: int) -> int:
    """2 * M * N * (nonzero weights per row)."""
    Ks = K - Kd
    return 2 * M * N * (Ks // 2 + Kd)


def group_algorithmic_bytes(members, M: int) -> int:
    """Algorithmic bytes of one launch over weights (N_i, K, Kd) sharing one
    activation tensor: every member's packed weights, scales and output, and the
    shared activations once."""
    K = members[0][1]
    total = M * K + 4 * M
    for N, k, Kd in members:
        assert k == K
        total += weight_bytes(N, K, Kd) + 4 * N + 2 * M * N
    return total


"""Seeded synthetic inputs for shared-QK LSH attention workloads.

This module only draws random numbers; it holds none of the method's
arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle (tests)
take their inputs from here, so that the two sides see identical values.

Streams are independent per (batch, head, tensor): ``default_rng([seed, b, h,
tid])`` with tid 0 for the shared QK rows and 1 for V, 2 for the cluster
structure of the skewed workload.  The random projection of round r comes
from ``default_rng([seed, r, 99])`` and has shape [D, n_buckets // 2].
Values are drawn in float32 and then rounded to the workload dtype (bf16
round-to-nearest-even through torch), so any slice can be regenerated alone.
"""

from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    D: int
    dtype: str  # "f32" | "bf16"
    n_buckets: int
    chunk: int
    n_rounds: int
    qk_kind: str = "normal"  # "normal" | "clusters"
    n_clusters: int = 64
    zipf_s: float = 1.1
    noise_sigma: float = 0.2

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.L


WORKLOADS = {
    # 1 x 1 x 1024 x 64 fp32, 16 buckets, chunk 64, one round
    "tiny": Workload("tiny", 1, 1, 1024, 64, "f32", 16, 64, 1),
    # 8 x 8 x 4096 x 128 bf16 (d_model 1024, 8 heads), 64 buckets, 2 rounds
    "4k": Workload("4k", 8, 8, 4096, 128, "bf16", 64, 64, 2),
    # 8 x 8 x 16384 x 128 bf16, Zipf(1.1) mixture of 64 directions, 256 buckets, 4 rounds
    "skewed16k": Workload("skewed16k", 8, 8, 16384, 128, "bf16", 256, 64, 4, qk_kind="clusters"),
    # 8 x 8 x 65536 x 128 bf16, 1024 buckets, 8 rounds (64K char-LM shaped)
    "64k": Workload("64k", 8, 8, 65536, 128, "bf16", 1024, 64, 8),
    # 1 x 8 x 65536 x 128 bf16, 1024 buckets, 8 rounds: the 64K workload at batch 1
    # (profiling captures at the real per-slice shape; QK 128 MB, still larger than L2)
    "64k_b1": Workload("64k_b1", 1, 8, 65536, 128, "bf16", 1024, 64, 8),
    # 8 x 8 x 16384 x 128 bf16, 256 buckets, 8 rounds: the 64K workload at a quarter of the
    # length (profiling captures: inputs still larger than L2, a few GB on the device)
    "16k": Workload("16k", 8, 8, 16384, 128, "bf16", 256, 64, 8),
    # 1 x 8 x 1048576 x 64 bf16, 16384 buckets, 4 rounds
    "1m": Workload("1m", 1, 8, 1048576, 64, "bf16", 16384, 64, 4),
}


def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t if dtype == "f32" else t.to(torch.bfloat16)


def slice_qk_v(w: Workload, b: int, h: int, seed: int = 0):
    """QK and V rows of one (b, h) slice as float32 numpy arrays [L, D]."""
    g_qk = np.random.default_rng([seed, b, h, 0])
    g_v = np.random.default_rng([seed, b, h, 1])
    if w.qk_kind == "normal":
        qk = g_qk.standard_normal((w.L, w.D), dtype=np.float32)
    elif w.qk_kind == "clusters":
        g_c = np.random.default_rng([seed, b, h, 2])
        centers = g_c.standard_normal((w.n_clusters, w.D))
        centers /= np.linalg.norm(centers, axis=1, keepdims=True)
        ranks = np.arange(1, w.n_clusters + 1, dtype=np.float64)
        p = ranks ** (-w.zipf_s)
        p /= p.sum()
        member = g_c.choice(w.n_clusters, size=w.L, p=p)
        eps = g_qk.standard_normal((w.L, w.D))
        qk = (centers[member] + (w.noise_sigma / np.sqrt(w.D)) * eps).astype(np.float32)
    else:
        raise ValueError(w.qk_kind)
    v = g_v.standard_normal((w.L, w.D), dtype=np.float32)
    return qk, v


def projections(w: Workload, seed: int = 0) -> torch.Tensor:
    """R: [n_rounds, D, n_buckets // 2] in the workload dtype (CPU tensor)."""
    R = np.stack([
        np.random.default_rng([seed, r, 99]).standard_normal((w.D, w.n_buckets // 2), dtype=np.float32)
        for r in range(w.n_rounds)
    ])
    return _round(R, w.dtype)


def slice_inputs(w: Workload, b: int, h: int, seed: int = 0):
    """(qk [L, D], v [L, D]) of one slice, rounded to the workload dtype (CPU tensors)."""
    qk, v = slice_qk_v(w, b, h, seed)
    return _round(qk, w.dtype), _round(v, w.dtype)


def make_inputs(w: Workload, seed: int = 0, threads: int = 8, pin: bool = False):
    """Full (qk [B,H,L,D], v [B,H,L,D], R) CPU tensors in the workload dtype."""
    qk = torch.empty((w.B, w.H, w.L, w.D), dtype=w.torch_dtype, pin_memory=pin)
    v = torch.empty_like(qk, pin_memory=pin)

    def fill(bh):
        b, h = divmod(bh, w.H)
        q_s, v_s = slice_inputs(w, b, h, seed)
        qk[b, h].copy_(q_s)
        v[b, h].copy_(v_s)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, range(w.B * w.H)))
    return qk, v, projections(w, seed)


def small_workload(name: str, B: int, H: int, L: int, D: int, dtype: str, n_buckets: int,
                   chunk: int, n_rounds: int, **kw) -> Workload:
    """A workload of arbitrary size for tests (same generator, any shape)."""
    return Workload(name, B, H, L, D, dtype, n_buckets, chunk, n_rounds, **kw)


def make_shard_inputs(w: Workload, slices, seed: int = 0, threads: int = 8, pin: bool = False):
    """(qk [1,n,L,D], v [1,n,L,D], R) of the given (b, h) slices of one batch (the strong-scaling
    split of a batch over ranks: every slice is generated from its own (b, h) stream, so the shards
    of all ranks together are exactly the batch of ``make_inputs``)."""
    n = len(slices)
    qk = torch.empty((1, n, w.L, w.D), dtype=w.torch_dtype, pin_memory=pin)
    v = torch.empty_like(qk, pin_memory=pin)

    def fill(i):
        b, h = slices[i]
        q_s, v_s = slice_inputs(w, b, h, seed)
        qk[0, i].copy_(q_s)
        v[0, i].copy_(v_s)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, range(n)))
    return qk, v, projections(w, seed)

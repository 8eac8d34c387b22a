"""Seeded synthetic inputs shaped like video-DiT attention activations.

This module holds no arithmetic of the attention method itself: it only draws
Q, K, V tensors.  It is shared by the tests, the benchmark and the oracle
checks, so that the GPU path and the CPU oracle see identical inputs.

Recipe (AB-Attention news write-up, section "how it was measured": Wan2.1 at
81 frames and HunyuanVideo at 129 frames, 720p latents; the sweep shape is the
75,600-token x 10-head x d128 workload of the Splash-attention page, Table 2):

* Q, K, V are drawn as float32 N(0, 1), one PCG64 stream per (seed, batch,
  head, tensor), so that any single head can be rebuilt on its own.
* Token n is the frame-major (F, H, W) position n = (f * Hg + y) * Wg + x.
  A shared 3D sinusoidal code p[n] is added, scaled by 0.8, to Q, K and V of
  every batch and head.  p concatenates, for each axis a in (f, y, x),
  [sin(pos_a * w_i), cos(pos_a * w_i)] for i < da / 2 with da = 2 * floor(d / 6)
  and w_i = 10000 ** (-2 i / da); the rest of the d channels are zero.
* Optionally a fraction of tokens (chosen by a seeded permutation) has its
  Q, K and V rows multiplied by a factor (the 14B-like layer uses 1% x 8).
* The result is rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention layer's shape plus the method's knobs."""

    name: str
    B: int
    H: int
    grid: tuple  # (frames, height, width) in latent tokens
    d: int
    kv_block: int
    budget: float
    seed: int
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    n_clusters: int = 8
    kmeans_iters: int = 10
    q_block: int = 128
    forwards_per_plan: int = 1

    @property
    def N(self) -> int:
        f, y, x = self.grid
        return f * y * x


# The workloads: a tiny case the oracle runs in full, three video layers and
# the sweep shape.
TINY = Workload("tiny", 1, 2, (4, 32, 32), 64, 4, 0.125, 0)
WAN_1_3B = Workload("wan1.3b-480p", 1, 12, (21, 30, 52), 128, 4, 0.10, 1)
WAN_14B = Workload("wan14b-720p", 1, 40, (21, 45, 80), 128, 4, 0.08, 2,
                   outlier_frac=0.01, outlier_scale=8.0)
HUNYUAN = Workload("hunyuan-720p", 1, 24, (33, 45, 80), 128, 4, 0.11, 3,
                   forwards_per_plan=4)
SWEEP = Workload("sweep-75k", 1, 10, (21, 45, 80), 128, 4, 0.08, 4)

WORKLOADS = {w.name: w for w in (TINY, WAN_1_3B, WAN_14B, HUNYUAN, SWEEP)}


def position_code(grid, d: int) -> torch.Tensor:
    """3D sinusoidal code, float32 [N, d] (frame-major token order)."""
    F, Hg, Wg = grid
    da = 2 * (d // 6)
    half = da // 2
    i = torch.arange(half, dtype=torch.float64)
    omega = torch.pow(torch.tensor(10000.0, dtype=torch.float64), -2.0 * i / da)
    f = torch.arange(F, dtype=torch.float64).repeat_interleave(Hg * Wg)
    y = torch.arange(Hg, dtype=torch.float64).repeat_interleave(Wg).repeat(F)
    x = torch.arange(Wg, dtype=torch.float64).repeat(F * Hg)
    parts = []
    for pos in (f, y, x):
        ang = pos[:, None] * omega[None, :]
        parts += [torch.sin(ang), torch.cos(ang)]
    p = torch.cat(parts, dim=1)
    out = torch.zeros(F * Hg * Wg, d, dtype=torch.float64)
    out[:, : p.shape[1]] = p
    return out.to(torch.float32)


def _stream(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


def outlier_rows(w: Workload, seed: int | None = None) -> np.ndarray:
    """Token rows whose Q, K, V are scaled by the outlier factor."""
    seed = w.seed if seed is None else seed
    if w.outlier_frac <= 0:
        return np.zeros(0, dtype=np.int64)
    n_out = int(round(w.outlier_frac * w.N))
    return np.sort(_stream(seed, 0x0071E5).permutation(w.N)[:n_out])


def make_head(w: Workload, b: int, h: int, seed: int | None = None, pos=None, rows=None):
    """Q, K, V of one (batch, head) as bf16 [N, d] CPU tensors.

    Each of the three tensors of each head has its own PCG64 stream keyed
    by (seed, b, h, tensor), so any head can be rebuilt alone."""
    seed = w.seed if seed is None else seed
    pos = (0.8 * position_code(w.grid, w.d)).numpy() if pos is None else pos
    rows = outlier_rows(w, seed) if rows is None else rows
    out = []
    for t in range(3):
        x = _stream(seed, b, h, t).standard_normal((w.N, w.d), dtype=np.float32)
        x += pos
        if rows.size:
            x[rows] *= np.float32(w.outlier_scale)
        out.append(torch.from_numpy(x).to(torch.bfloat16))
    return tuple(out)


def make_qkv(w: Workload, device: str = "cpu", seed: int | None = None, threads: int | None = None):
    """Return bf16 Q, K, V of shape [B, H, N, d] on `device` (drawn on the
    host, one head per task in a thread pool; identical on every machine)."""
    seed = w.seed if seed is None else seed
    pos = (0.8 * position_code(w.grid, w.d)).numpy()
    rows = outlier_rows(w, seed)
    Q, K, V = (torch.empty(w.B, w.H, w.N, w.d, dtype=torch.bfloat16) for _ in range(3))

    def one(bh):
        b, h = divmod(bh, w.H)
        q, k, v = make_head(w, b, h, seed, pos, rows)
        Q[b, h], K[b, h], V[b, h] = q, k, v

    threads = threads or min(32, os.cpu_count() or 1)
    with concurrent.futures.ThreadPoolExecutor(threads) as ex:
        list(ex.map(one, range(w.B * w.H)))
    if device != "cpu":
        Q, K, V = (t.to(device) for t in (Q, K, V))
    return Q, K, V


def make_qkv_heads(w: Workload, heads: range, device: str = "cpu", seed: int | None = None):
    """Q, K, V of the heads `heads` of batch 0 only, [1, len(heads), N, d] bf16:
    the same values as those heads of make_qkv (each head has its own streams)."""
    seed = w.seed if seed is None else seed
    pos = (0.8 * position_code(w.grid, w.d)).numpy()
    rows = outlier_rows(w, seed)
    Q, K, V = (torch.empty(1, len(heads), w.N, w.d, dtype=torch.bfloat16) for _ in range(3))
    for i, h in enumerate(heads):
        Q[0, i], K[0, i], V[0, i] = make_head(w, 0, h, seed, pos, rows)
    if device != "cpu":
        Q, K, V = (t.to(device) for t in (Q, K, V))
    return Q, K, V


def row_sample(w: Workload, n_rows: int, seed: int = 1234):
    """A seeded sample of (b, h, qb) rows, used to check large layers."""
    nqb = math.ceil(w.N / w.q_block)
    g = torch.Generator().manual_seed(seed)
    total = w.B * w.H * nqb
    flat = torch.randperm(total, generator=g)[:n_rows].tolist()
    # always include the ragged last q-block of some head
    flat.append(nqb - 1)
    rows = []
    for r in sorted(set(flat)):
        b, rem = divmod(r, w.H * nqb)
        h, qb = divmod(rem, nqb)
        rows.append((b, h, qb))
    return rows

"""Seeded synthetic Q/K/V generator for the SageSLA attention forward.

This module is the one piece shared by the fp64 CPU oracle's tests and the
CUDA path's tests and benchmark.  It holds none of the attention method's
arithmetic: it only draws tensors.  Every tensor is returned as raw bfloat16
bits (``numpy.uint16``, layout ``[B, H, N, d]``, token order ``(t, y, x)``
row-major), which both sides consume unchanged.

Recipe (stand-in for attention activations of a Wan2.1 video DiT at its
latent token grids; the pages give no activations, only the grid sizes implied
by 81 frames at 480p / 720p, see "TurboDiffusion技术架构解析" §3.2 example
call):

* For every (b, h, channel) of each X in {Q, K, V} a smooth field over the
  (t, y, x) grid is built as a sum of 8 random Fourier modes
  ``a_m cos(2 pi (kt t/T + ky y/Hg + kx x/Wg) + phase_m)`` with integer
  wave vectors in [0,4]^3 minus the origin, ``a_m ~ N(0,1)`` and
  ``phase_m ~ U[0, 2 pi)``.  The field is normalised to zero mean and unit
  standard deviation over the grid.
* ``X = 0.5 * field + 0.5 * N(0, 1)`` per element.
* K additionally gets a per-(b, h, channel) offset drawn from N(0, 2)
  (variance 2).
* Q and K are multiplied by one common factor alpha chosen so that
  ``q.k / sqrt(d)`` over 65 536 seeded (b, h, i, j) pairs has standard
  deviation ``logit_std`` (3.0 by default).
* Values are rounded fp64 -> fp32 -> bf16, each step round-to-nearest-even.

Optional adversarial edits (used by the invariant/edge sweep):

* ``"ties"``: in batch 0, head 0 every key block is a copy of key block 0;
  head 1 has K == 0; head 2 has every odd key block a copy of the even block
  before it, so that an odd selection count always splits a tied pair.
* ``"outliers"``: in batch 1 (or batch 0 if B == 1), 4 seeded K channels of
  every head are replaced by 4 * Student-t(nu = 3) samples before scaling.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "make_qkv",
    "bf16_bits_to_f64",
    "f64_to_bf16_bits",
    "sample_rows",
]


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload (shape + method parameters)."""

    name: str
    B: int
    H: int
    grid: Tuple[int, int, int]  # (T, Hg, Wg); N = T * Hg * Wg
    d: int = 128
    blk_q: int = 128
    blk_k: int = 64
    topk: float = 0.10
    phi: int = 0  # 0 = elu+1, 1 = relu
    quant: int = 1
    seed: int = 0
    extra: Tuple[str, ...] = field(default_factory=tuple)

    @property
    def N(self) -> int:
        t, y, x = self.grid
        return t * y * x


# The five workload families of the method's measurement plan.  Seeds differ per
# family so that no two families share tensors.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, (8, 16, 16), blk_q=64, blk_k=64, topk=0.10, seed=1),
    "wan1.3b-480p": Workload("wan1.3b-480p", 1, 12, (21, 30, 52), seed=2),
    "wan14b-480p": Workload("wan14b-480p", 1, 40, (21, 30, 52), seed=3),
    "wan14b-720p": Workload("wan14b-720p", 1, 40, (21, 45, 80), seed=4),
    "sweep": Workload("sweep", 2, 40, (16, 32, 32), seed=5),
}


# ---------------------------------------------------------------------------
# bf16 bit helpers (pure representation changes, no method arithmetic)
# ---------------------------------------------------------------------------

def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 -> fp32 (RNE) -> bf16 (RNE); return the 16-bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the low 16 bits; NaN does not occur here
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# generator
# ---------------------------------------------------------------------------

_WAVES = np.array(
    [(a, b, c) for a in range(5) for b in range(5) for c in range(5) if (a, b, c) != (0, 0, 0)],
    dtype=np.float64,
)  # 124 integer wave vectors in [0,4]^3 \ {0}


def _basis(grid: Tuple[int, int, int]) -> np.ndarray:
    """[N, 2*124] cos/sin of every admissible wave vector over the grid."""
    T, Hg, Wg = grid
    t = np.arange(T, dtype=np.float64) / T
    y = np.arange(Hg, dtype=np.float64) / Hg
    x = np.arange(Wg, dtype=np.float64) / Wg
    tt, yy, xx = np.meshgrid(t, y, x, indexing="ij")
    pos = np.stack([tt.ravel(), yy.ravel(), xx.ravel()], axis=1)  # [N,3], t-major
    theta = 2.0 * np.pi * (pos @ _WAVES.T)  # [N,124]
    return np.concatenate([np.cos(theta), np.sin(theta)], axis=1)


def _field_coeffs(rng: np.random.Generator, d: int, n_modes: int = 8) -> np.ndarray:
    """Coefficients [248, d] so that basis @ coeffs = sum of n_modes cosines per channel."""
    coef = np.zeros((2 * len(_WAVES), d), dtype=np.float64)
    idx = rng.integers(0, len(_WAVES), size=(n_modes, d))
    amp = rng.standard_normal((n_modes, d))
    phase = rng.uniform(0.0, 2.0 * np.pi, size=(n_modes, d))
    cols = np.arange(d)
    for m in range(n_modes):
        # a cos(theta + p) = a cos p cos theta - a sin p sin theta
        np.add.at(coef, (idx[m], cols), amp[m] * np.cos(phase[m]))
        np.add.at(coef, (idx[m] + len(_WAVES), cols), -amp[m] * np.sin(phase[m]))
    return coef


def _one_head(basis, seed_seq: np.random.SeedSequence, d: int, with_offset: bool,
              outlier_channels: Optional[np.ndarray]) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed_seq))
    coef = _field_coeffs(rng, d)
    f = basis @ coef  # [N, d]
    f -= f.mean(axis=0, keepdims=True)
    sd = f.std(axis=0, keepdims=True)
    sd[sd == 0] = 1.0
    f /= sd
    x = 0.5 * f + 0.5 * rng.standard_normal(f.shape)
    if with_offset:
        x += rng.normal(0.0, math.sqrt(2.0), size=(1, d))
    if outlier_channels is not None:
        for c in outlier_channels:
            x[:, c] = 4.0 * rng.standard_t(3.0, size=x.shape[0])
    return x


def make_qkv(
    B: int,
    H: int,
    grid: Tuple[int, int, int],
    d: int = 128,
    seed: int = 0,
    logit_std: float = 3.0,
    adversarial: Sequence[str] = (),
    threads: Optional[int] = None,
    blk_k: int = 64,
):
    """Return (q, k, v) as bf16 bit arrays ``uint16[B, H, N, d]``.

    ``blk_k`` only matters for the ``"ties"`` edit (which copies whole key
    blocks).  The result is a pure function of the arguments.
    """
    T, Hg, Wg = grid
    N = T * Hg * Wg
    basis = _basis(grid)
    root = np.random.SeedSequence([20251223, seed, B, H, N, d])
    kids = root.spawn(3 * B * H + 2)
    pair_seq, out_seq = kids[-2], kids[-1]
    out_rng = np.random.Generator(np.random.PCG64(out_seq))
    outl_b = (1 if B > 1 else 0) if "outliers" in adversarial else -1
    outl_ch = out_rng.choice(d, size=4, replace=False) if outl_b >= 0 else None

    # pairs used to calibrate the logit scale: (b, h, i, j)
    prng = np.random.Generator(np.random.PCG64(pair_seq))
    n_pairs = 65536
    pb = prng.integers(0, B, n_pairs)
    ph = prng.integers(0, H, n_pairs)
    pi = prng.integers(0, N, n_pairs)
    pj = prng.integers(0, N, n_pairs)

    q32 = np.empty((B, H, N, d), dtype=np.float32)
    k32 = np.empty((B, H, N, d), dtype=np.float32)
    v16 = np.empty((B, H, N, d), dtype=np.uint16)
    dots = np.zeros(n_pairs, dtype=np.float64)

    def work(bh):
        b, h = divmod(bh, H)
        base = 3 * bh
        q = _one_head(basis, kids[base + 0], d, False, None)
        kk = _one_head(basis, kids[base + 1], d, True, outl_ch if b == outl_b else None)
        v = _one_head(basis, kids[base + 2], d, False, None)
        sel = np.nonzero((pb == b) & (ph == h))[0]
        dots[sel] = np.einsum("nd,nd->n", q[pi[sel]], kk[pj[sel]]) / math.sqrt(d)
        q32[b, h] = q
        k32[b, h] = kk
        v16[b, h] = f64_to_bf16_bits(v)

    nthreads = threads or min(8, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        list(ex.map(work, range(B * H)))

    sd = float(dots.std())
    alpha = math.sqrt(logit_std / sd) if sd > 0 else 1.0
    q16 = f64_to_bf16_bits(q32.astype(np.float64) * alpha)
    k16 = f64_to_bf16_bits(k32.astype(np.float64) * alpha)
    del q32, k32

    if "ties" in adversarial:
        nkb = (N + blk_k - 1) // blk_k
        full = N // blk_k
        if H >= 1:  # every key block identical to block 0 (partial tail copies a prefix)
            blk0 = k16[0, 0, :blk_k].copy()
            for J in range(1, nkb):
                n = min(blk_k, N - J * blk_k)
                k16[0, 0, J * blk_k:J * blk_k + n] = blk0[:n]
        if H >= 2:
            k16[0, 1] = 0
        if H >= 3:  # odd full blocks duplicate the even block before them
            for J in range(1, full, 2):
                k16[0, 2, J * blk_k:(J + 1) * blk_k] = k16[0, 2, (J - 1) * blk_k:J * blk_k]
    return q16, k16, v16


def sample_rows(B: int, H: int, N: int, n_heads: int, rows_per_head: int, seed: int = 7,
                must_include_last: bool = True) -> np.ndarray:
    """Seeded (bh, i) pairs used for sampled full-size parity checks.

    Always includes the first and (optionally) the last token of each chosen
    head so the ragged tail block is exercised.
    """
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, B, H, N])))
    heads = rng.choice(B * H, size=min(n_heads, B * H), replace=False)
    out = []
    for bh in sorted(heads.tolist()):
        rows = set(rng.choice(N, size=min(rows_per_head, N), replace=False).tolist())
        rows.add(0)
        if must_include_last:
            rows.add(N - 1)
        out.extend((bh, i) for i in sorted(rows))
    return np.asarray(out, dtype=np.int64)

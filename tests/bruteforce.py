"""Independent dense brute force used to pin the fp64 oracle (tests only).

It shares no code with ``oracle/``: it expands the block selection to a dense
token mask, materialises all N x N logits, and computes the linear branch in
*attention form* -- sum over unselected tokens of (phi(q).phi(k)) v divided by
sum of phi(q).phi(k) -- instead of the oracle's per-block *state form*.  It is
meant for N of a few hundred to a few thousand.
"""
from __future__ import annotations

import itertools

import numpy as np

from synth import bf16_bits_to_f64


def phi(x: np.ndarray, kind: int) -> np.ndarray:
    if kind == 1:
        return np.maximum(x, 0.0)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def token_mask(idx_head: np.ndarray, N: int, blk_q: int, blk_k: int) -> np.ndarray:
    """Boolean [N, N]: True where query token i attends key token j exactly."""
    m = np.zeros((N, N), dtype=bool)
    for I in range(idx_head.shape[0]):
        rows = slice(I * blk_q, min(N, (I + 1) * blk_q))
        for J in idx_head[I]:
            m[rows, J * blk_k:min(N, (J + 1) * blk_k)] = True
    return m


def sla_dense(qb, kb, vb, idx, blk_q, blk_k, phi_kind, logits=None):
    """Dense SLA for one head.

    qb, kb, vb: bf16 bits [N, d].  idx: [n_qb, k_sel].  ``logits`` overrides
    q k^T / sqrt(d) (used for the quantised path).  Returns (o, o_sparse,
    o_linear) in fp64.
    """
    q, k, v = bf16_bits_to_f64(qb), bf16_bits_to_f64(kb), bf16_bits_to_f64(vb)
    N, d = q.shape
    m = token_mask(idx, N, blk_q, blk_k)
    L = q @ k.T / np.sqrt(d) if logits is None else logits
    Lm = np.where(m, L, -np.inf)
    mx = Lm.max(axis=1, keepdims=True)
    has = np.isfinite(mx)
    P = np.where(m, np.exp(Lm - np.where(has, mx, 0.0)), 0.0)
    den = P.sum(axis=1, keepdims=True)
    os_ = np.where(has, (P @ v) / np.where(den > 0, den, 1.0), 0.0)
    A = phi(q, phi_kind) @ phi(k, phi_kind).T
    A = np.where(m, 0.0, A)
    lden = A.sum(axis=1, keepdims=True)
    ol = np.where(lden != 0, (A @ v) / np.where(lden != 0, lden, 1.0), 0.0)
    return os_ + ol, os_, ol


def quant_logits(q8, k8, sq, sk, blk_q, blk_k):
    """Logits of the quantised path from integer codes and per-block scales."""
    N, d = q8.shape
    dots = q8.astype(np.int64) @ k8.astype(np.int64).T
    rs = np.repeat(sq.astype(np.float64), blk_q)[:N]
    cs = np.repeat(sk.astype(np.float64), blk_k)[:N]
    return dots.astype(np.float64) * rs[:, None] * cs[None, :] / np.sqrt(d)


def dominant_subset(scores_row: np.ndarray, k_sel: int):
    """Exhaustive search: the unique k-subset S such that every selected block
    beats every unselected one (higher score, or equal score and lower index)."""
    n = len(scores_row)
    found = []
    for S in itertools.combinations(range(n), k_sel):
        Sset = set(S)
        ok = True
        for a in S:
            for b in range(n):
                if b in Sset:
                    continue
                if not (scores_row[a] > scores_row[b] or (scores_row[a] == scores_row[b] and a < b)):
                    ok = False
                    break
            if not ok:
                break
        if ok:
            found.append(S)
    assert len(found) == 1, found
    return np.array(found[0], dtype=np.int32)

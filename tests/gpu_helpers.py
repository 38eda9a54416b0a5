"""Helpers shared by the GPU parity tests (host-side marshalling and metrics)."""
from __future__ import annotations

import numpy as np


def to_dev(x: np.ndarray, torch, dtype=None):
    """bf16 bit patterns (uint16) -> CUDA bfloat16 tensor; other dtypes as they are."""
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(x).cuda()


def bf16_to_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    nb = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / nb if nb > 0 else float(np.linalg.norm(a))


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    na, nb = float(np.linalg.norm(a)), float(np.linalg.norm(b))
    if na == 0 and nb == 0:
        return 1.0
    return float((a * b).sum()) / (na * nb)


def mask_mismatches(idx_gpu: np.ndarray, idx_orc: np.ndarray, scores: np.ndarray, rel: float = 1e-5):
    """Rows whose selected sets differ, split into (exempt near-ties, real mismatches).

    A difference is exempt only if every block in the symmetric difference has
    a score within ``rel`` (relative, with an absolute floor of 1e-6 * the row's
    largest |score|) of the oracle's k_sel-th largest score.
    """
    exempt, real = [], []
    ks = idx_orc.shape[-1]
    flat_g = idx_gpu.reshape(-1, ks)
    flat_o = idx_orc.reshape(-1, ks)
    flat_s = scores.reshape(flat_o.shape[0], -1)
    for r in range(flat_o.shape[0]):
        a, b = set(flat_g[r].tolist()), set(flat_o[r].tolist())
        if a == b:
            continue
        row = flat_s[r]
        thr = np.sort(row)[::-1][ks - 1]
        floor = 1e-6 * np.abs(row).max()
        ok = all(abs(row[J] - thr) <= max(rel * max(abs(row[J]), abs(thr)), floor) for J in (a ^ b))
        (exempt if ok else real).append(r)
    return exempt, real


_INPUT_CACHE: dict = {}


def workload_qkv(name: str, adversarial=(), seed_offset: int = 0):
    """(q, k, v) of a named workload from synth.WORKLOADS (bf16 bits), generated once per
    test process and shared by the test modules; at most the two most recent input sets
    are kept (a 720P set is 2.3 GB of host memory)."""
    import synth

    key = (name, tuple(adversarial), seed_offset)
    if key not in _INPUT_CACHE:
        while len(_INPUT_CACHE) >= 2:
            _INPUT_CACHE.pop(next(iter(_INPUT_CACHE)))
        w = synth.WORKLOADS[name]
        _INPUT_CACHE[key] = synth.make_qkv(w.B, w.H, w.grid, seed=w.seed + seed_offset, adversarial=adversarial)
    return _INPUT_CACHE[key]

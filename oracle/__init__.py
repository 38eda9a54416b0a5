"""fp64 CPU oracle of the SageSLA attention forward -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``sparse_linear_bit_b200``) never does, and the two share no code: the only
thing both consume is the seeded input generator in ``synth``.

The arithmetic lives in ``sla_oracle.c`` (plain C loops, fp64, OpenMP over
heads / blocks / rows); this module only builds it with gcc and marshals numpy
arrays.  See that file's header for the method, step by step, with citations.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):

* ``topk_count``  -- pinned (the selection counts stated for every workload).
* ``block_mask``  -- pinned (exhaustive subset search on tiny inputs,
  permutation / scaling / shift invariances, tie rules).
* ``quantize``    -- pinned (hand-worked golden block, range and error bounds,
  amax element maps to +-127, smoothing identity).
* ``forward``     -- pinned (topk=1 equals dense softmax attention from a
  library routine; topk=0 equals closed-form linear attention; an independent
  attention-form brute force with a dense token mask; constant-V identity;
  convex-hull bounds; a hand-worked golden case).
* ``backward_dq_rows``, ``backward_dkdv_blocks`` -- pinned (equal, bit for bit,
  to the corresponding rows of ``backward``).
* ``backward``  -- pinned (float64 autograd of an independent PyTorch
  statement of the unquantised forward, whose values are checked against
  ``forward``; topk=1 against the gradient of a library attention routine;
  central differences of ``forward`` along random directions).
* Which block-score criterion, combine rule and quantisation granularity the
  pages' own SageSLA uses cannot be pinned from the pages: parity unpinned for
  that question; this oracle implements the stated reading.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-Wall"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the C oracle with gcc (OpenMP, no FP contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


_lib = None


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle shared library and declare its ABI."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build())
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.orc_topk_count.argtypes = [i32, f64]
    lib.orc_topk_count.restype = i32
    lib.orc_num_threads.restype = i32
    lib.orc_set_threads.argtypes = [i32]
    lib.orc_pool.argtypes = [P, i32, i32, i32, i32, P]
    lib.orc_block_mask.argtypes = [P, P, i32, i32, i32, i32, i32, f64, P, P, P]
    lib.orc_quantize.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P]
    lib.orc_e4m3_array.argtypes = [P, P, P, i64]
    lib.orc_rowquant.argtypes = [P, i32, i32, i32, P, ctypes.c_float, P, P]
    lib.orc_w8a8_linear.argtypes = [P, P, P, P, P, i32, i32, i32, P]
    lib.orc_states.argtypes = [P, P, i32, i32, i32, i32, P, P]
    lib.orc_forward.argtypes = [P, P, P, i32, i32, i32, i32, i32, f64, i32, i32, P, P, i64, P, P, P]
    lib.orc_forward.restype = i32
    lib.orc_backward.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, f64, i32, P, P, P, P]
    lib.orc_backward.restype = i32
    lib.orc_backward_dq_rows.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, f64, i32, P, P, i64, P]
    lib.orc_backward_dq_rows.restype = i32
    lib.orc_backward_dkdv_blocks.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, f64, i32, P, P, i64, P, P]
    lib.orc_backward_dkdv_blocks.restype = i32
    if path is None:
        _lib = lib
    return lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return x


def _shape(q: np.ndarray) -> Tuple[int, int, int]:
    """(BH, N, d) of a [B, H, N, d] or [BH, N, d] array."""
    if q.ndim == 4:
        return q.shape[0] * q.shape[1], q.shape[2], q.shape[3]
    if q.ndim == 3:
        return q.shape
    raise ValueError("expected [B,H,N,d] or [BH,N,d]")


def set_threads(n: int) -> None:
    load().orc_set_threads(int(n))


def num_threads() -> int:
    return int(load().orc_num_threads())


def topk_count(n_kb: int, topk: float) -> int:
    """k_sel = floor(topk * n_kb + 1e-4) clamped to [0, n_kb] (topk taken as given, in fp64)."""
    return int(load().orc_topk_count(int(n_kb), float(topk)))


def pool(x: np.ndarray, blk: int, lib=None) -> np.ndarray:
    """fp64 block means [BH, n_blocks, d]."""
    x = _bits(x)
    BH, N, d = _shape(x)
    nb = -(-N // blk)
    out = np.empty((BH, nb, d), dtype=np.float64)
    (lib or load()).orc_pool(_ptr(x), BH, N, d, blk, _ptr(out))
    return out


def block_mask(q, k, blk_q: int, blk_k: int, topk: float, with_scores: bool = False, lib=None):
    """Selected key blocks per query block.

    Returns ``idx int32[BH, n_qb, k_sel]`` (ascending), ``bitmap
    uint32[BH, n_qb, ceil(n_kb/32)]`` and, if asked, the fp64 scores
    ``[BH, n_qb, n_kb]``.
    """
    lib = lib or load()
    q, k = _bits(q), _bits(k)
    BH, N, d = _shape(q)
    n_qb, n_kb = -(-N // blk_q), -(-N // blk_k)
    ks = int(lib.orc_topk_count(n_kb, float(topk)))
    idx = np.zeros((BH, n_qb, ks), dtype=np.int32)
    bm = np.zeros((BH, n_qb, -(-n_kb // 32)), dtype=np.uint32)
    sc = np.zeros((BH, n_qb, n_kb), dtype=np.float64) if with_scores else None
    lib.orc_block_mask(_ptr(q), _ptr(k), BH, N, d, blk_q, blk_k, float(topk), _ptr(idx), _ptr(bm), _ptr(sc))
    return (idx, bm, sc) if with_scores else (idx, bm)


def quantize(q, k, blk_q: int, blk_k: int, lib=None, fp8: bool = False):
    """Codes and fp32 scales: (q8, k8, s_q[BH,n_qb], s_k[BH,n_kb], k_mean[BH,d]).

    INT8 codes by default; with ``fp8`` the codes are FP8 e4m3 bit patterns
    (stored in int8 arrays; view them as uint8)."""
    lib = lib or load()
    q, k = _bits(q), _bits(k)
    BH, N, d = _shape(q)
    n_qb, n_kb = -(-N // blk_q), -(-N // blk_k)
    q8 = np.zeros(q.shape, dtype=np.int8)
    k8 = np.zeros(k.shape, dtype=np.int8)
    sq = np.zeros((BH, n_qb), dtype=np.float32)
    sk = np.zeros((BH, n_kb), dtype=np.float32)
    km = np.zeros((BH, d), dtype=np.float32)
    lib.orc_quantize(_ptr(q), _ptr(k), BH, N, d, blk_q, blk_k, int(bool(fp8)), _ptr(q8), _ptr(k8), _ptr(sq),
                     _ptr(sk), _ptr(km))
    return q8, k8, sq, sk, km


def e4m3(x, lib=None):
    """(value, bits): the fp8 e4m3 value nearest to each fp32 x (ties to even, saturated to
    +-448) and its bit pattern."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    value = np.zeros(x.shape, dtype=np.float32)
    bits = np.zeros(x.shape, dtype=np.uint8)
    lib.orc_e4m3_array(_ptr(x), _ptr(value), _ptr(bits), x.size)
    return value, bits


def states(k, v, blk_k: int, phi: int, lib=None):
    """Per-key-block states of ONE head [N, d]: h[n_kb, d, d], z[n_kb, d] (fp64)."""
    lib = lib or load()
    k, v = _bits(k), _bits(v)
    N, d = k.shape
    n_kb = -(-N // blk_k)
    h = np.zeros((n_kb, d, d), dtype=np.float64)
    z = np.zeros((n_kb, d), dtype=np.float64)
    lib.orc_states(_ptr(k), _ptr(v), N, d, blk_k, int(phi), _ptr(h), _ptr(z))
    return h, z


def forward(q, k, v, blk_q: int, blk_k: int, topk: float, phi: int = 0, quant: int = 1,
            idx: Optional[np.ndarray] = None, rows: Optional[np.ndarray] = None,
            branches: bool = False, lib=None):
    """fp64 SLA forward.

    ``rows`` (int64 [n, 2] of (bh, i)) limits the work to those output rows and
    returns ``[n, d]``; otherwise the result has the input's shape.  ``idx``
    replaces the oracle's own block selection.  With ``branches`` the sparse and
    linear parts are returned too: ``(out, out_sparse, out_linear)``.
    """
    lib = lib or load()
    q, k, v = _bits(q), _bits(k), _bits(v)
    BH, N, d = _shape(q)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
        n = rows.shape[0]
        shape = (n, d)
    else:
        n = BH * N
        shape = q.shape
    out = np.zeros(shape, dtype=np.float64)
    os_ = np.zeros(shape, dtype=np.float64) if branches else None
    ol_ = np.zeros(shape, dtype=np.float64) if branches else None
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    rc = lib.orc_forward(_ptr(q), _ptr(k), _ptr(v), BH, N, d, blk_q, blk_k, float(topk), int(phi),
                         int(quant), _ptr(idx), _ptr(rows), n, _ptr(out), _ptr(os_), _ptr(ol_))
    if rc != 0:
        raise MemoryError("oracle forward failed (out of memory or bad row index)")
    return (out, os_, ol_) if branches else out


def backward(q, k, v, dout, blk_q: int, blk_k: int, topk: float, phi: int = 0,
             idx: Optional[np.ndarray] = None, lib=None):
    """fp64 gradients (dq, dk, dv) of the unquantised SLA forward for the output
    gradient ``dout`` (bf16 bits, same shape as q), with the block selection held
    fixed (the oracle's own, or ``idx``).  Results have the input's shape."""
    lib = lib or load()
    q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
    BH, N, d = _shape(q)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(q.shape, dtype=np.float64)
    dv = np.zeros(q.shape, dtype=np.float64)
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    rc = lib.orc_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), BH, N, d, blk_q, blk_k, float(topk), int(phi),
                          _ptr(idx), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise MemoryError("oracle backward failed (out of memory)")
    return dq, dk, dv


def backward_dq_rows(q, k, v, dout, blk_q: int, blk_k: int, topk: float, rows, phi: int = 0,
                     idx: Optional[np.ndarray] = None, lib=None) -> np.ndarray:
    """fp64 dq of the rows ``rows`` (int64 [n, 2] of (bh, i)) only: the same
    steps as ``backward``'s dq, evaluable at sizes where the full backward is too
    slow.  Returns ``[n, d]``."""
    lib = lib or load()
    q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
    BH, N, d = _shape(q)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    out = np.zeros((rows.shape[0], d), dtype=np.float64)
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    rc = lib.orc_backward_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), BH, N, d, blk_q, blk_k, float(topk),
                                  int(phi), _ptr(idx), _ptr(rows), rows.shape[0], _ptr(out))
    if rc != 0:
        raise MemoryError("oracle backward_dq_rows failed (out of memory or bad row index)")
    return out


def backward_dkdv_blocks(q, k, v, dout, blk_q: int, blk_k: int, topk: float, blocks, phi: int = 0,
                         idx: Optional[np.ndarray] = None, lib=None):
    """fp64 dk and dv of the key blocks ``blocks`` (int64 [n, 2] of (bh, J)) only: the
    same steps, in the same order, as ``backward`` restricted to those blocks.
    Returns ``(dk, dv)``, each ``[n, blk_k, d]`` (rows past N are zero)."""
    lib = lib or load()
    q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
    BH, N, d = _shape(q)
    blocks = np.ascontiguousarray(blocks, dtype=np.int64).reshape(-1, 2)
    dk = np.zeros((blocks.shape[0], blk_k, d), dtype=np.float64)
    dv = np.zeros((blocks.shape[0], blk_k, d), dtype=np.float64)
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    rc = lib.orc_backward_dkdv_blocks(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), BH, N, d, blk_q, blk_k, float(topk),
                                      int(phi), _ptr(idx), _ptr(blocks), blocks.shape[0], _ptr(dk), _ptr(dv))
    if rc != 0:
        raise MemoryError("oracle backward_dkdv_blocks failed (out of memory or bad block index)")
    return dk, dv


# --------------------------------------------------------------------------
# W8A8 INT8 linear layer with FusedNorm
# --------------------------------------------------------------------------

def rowquant(x, norm: bool = False, gamma=None, eps: float = 1e-6, lib=None):
    """Per-row symmetric INT8 codes and fp32 scales of a bf16 matrix [rows, cols]
    (uint16 bits), optionally after the row's RMS normalisation times gamma."""
    lib = lib or load()
    x = _bits(x)
    rows, cols = x.shape
    q = np.zeros((rows, cols), dtype=np.int8)
    s = np.zeros(rows, dtype=np.float32)
    g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    lib.orc_rowquant(_ptr(x), rows, cols, int(bool(norm)), _ptr(g), float(np.float32(eps)), _ptr(q), _ptr(s))
    return q, s


def w8a8_linear(qx, sx, qw, sw, bias=None, lib=None):
    """out[m][n] = (sum_k qx[m][k] qw[n][k]) * sx[m] * sw[n] (+ bias[n]) in fp64."""
    lib = lib or load()
    qx, qw = np.ascontiguousarray(qx, dtype=np.int8), np.ascontiguousarray(qw, dtype=np.int8)
    sx, sw = np.ascontiguousarray(sx, dtype=np.float32), np.ascontiguousarray(sw, dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    M, K = qx.shape
    N = qw.shape[0]
    out = np.zeros((M, N), dtype=np.float64)
    lib.orc_w8a8_linear(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), _ptr(b), M, N, K, _ptr(out))
    return out

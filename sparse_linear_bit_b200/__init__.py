"""Python binding of libsla.so, the B200 (sm_100a) SageSLA attention forward.

Argument marshalling only: every step of the forward runs in the CUDA kernels
behind the C ABI declared in ``include/sla.h``; torch supplies device memory
and streams.  The functions carry the C names:

* ``sla_topk_count(n_kb, topk)``
* ``sla_workspace_bytes(B, H, N, d, blk_q, blk_k, topk, quant)``
* ``sla_block_mask(q, k, blk_q, blk_k, topk, idx, bitmap, ws)``
* ``sla_quantize_qk(q, k, blk_q, blk_k, q_i8, k_i8, q_scale, k_scale, k_mean, ws)``
* ``sla_forward(q, k, v, out, blk_q, blk_k, topk, phi, quant, ws)``
* ``sla_forward_profile(...)`` (per-stage device times), ``sla_check(ws)``,
  ``sla_status_string(code)``, ``sla_workspace_layout(...)``,
  ``sla_set_wait_budget(cycles)`` (diagnostics: the bounded waits' budget)

Tensors are CUDA tensors laid out as the header states ([B, H, N, d] bf16 for
q/k/v/out).  Calls enqueue on torch's current stream (or ``stream=``).  A
non-OK status raises :class:`SlaError`.  There is no CPU fallback: importing
this package without the built library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "SlaError", "lib", "sla_version", "sla_status_string", "sla_topk_count", "sla_workspace_bytes",
    "sla_workspace_layout", "sla_block_mask", "sla_quantize_qk", "sla_quantize_qk_fp8", "sla_forward", "sla_check", "workspace",
    "LAYOUT_REGIONS", "LIB_PATH", "sla_forward_profile", "PROFILE_STAGES", "sla_block_mask_noalloc",
    "sla_block_mask_noalloc_limit", "head_shard", "shard_heads", "sla_w8a8_quantize", "sla_w8a8_linear",
    "w8a8_workspace", "sla_backward_workspace_bytes", "sla_backward", "backward_workspace", "sla_set_wait_budget",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsla.so")
LAYOUT_REGIONS = ("status", "qbar", "kbar", "scores", "idx", "amask", "q8", "k8", "qscale", "kscale", "kmean",
                  "states", "partials", "htot", "hq", "v16", "kpart")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python sparse_linear_bit_b200/build.py` "
        "(the SageSLA forward has no CPU fallback)")

lib = ctypes.CDLL(LIB_PATH)
_P, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
lib.sla_version.restype = ctypes.c_char_p
lib.sla_status_string.argtypes = [_I]
lib.sla_status_string.restype = ctypes.c_char_p
lib.sla_topk_count.argtypes = [_I, _F]
lib.sla_topk_count.restype = _I
lib.sla_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _F, _I]
lib.sla_workspace_bytes.restype = _SZ
lib.sla_workspace_layout.argtypes = [_I, _I, _I, _I, _I, _I, _F, _I, ctypes.POINTER(_SZ), _I]
lib.sla_workspace_layout.restype = _I
lib.sla_block_mask.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _SZ, _P]
lib.sla_block_mask.restype = _I
lib.sla_quantize_qk.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]
lib.sla_quantize_qk.restype = _I
lib.sla_quantize_qk_fp8.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]
lib.sla_quantize_qk_fp8.restype = _I
lib.sla_forward.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _SZ, _P]
lib.sla_forward.restype = _I
lib.sla_forward_host_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _F, _I, _I]
lib.sla_forward_host_bytes.restype = _SZ
lib.sla_forward_host.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P, _SZ, _P]
lib.sla_forward_host.restype = _I
lib.sla_forward_profile.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P, _SZ, _P,
                                    ctypes.POINTER(ctypes.c_float)]
lib.sla_forward_profile.restype = _I
lib.sla_block_mask_noalloc.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P]
lib.sla_block_mask_noalloc.restype = _I
lib.sla_block_mask_noalloc_limit.restype = _SZ
lib.sla_w8a8_quantize.argtypes = [_P, _I, _I, _I, _P, _F, _P, _P, _P]
lib.sla_w8a8_quantize.restype = _I
lib.sla_w8a8_workspace_bytes.restype = _SZ
lib.sla_w8a8_linear.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _SZ, _P]
lib.sla_w8a8_linear.restype = _I
lib.sla_backward_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _F]
lib.sla_backward_workspace_bytes.restype = _SZ
lib.sla_backward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _P]
lib.sla_backward.restype = _I
lib.sla_check.argtypes = [_P, _P]
lib.sla_check.restype = _I
lib.sla_set_wait_budget.argtypes = [ctypes.c_longlong]
lib.sla_set_wait_budget.restype = _I


class SlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = int(code)
        super().__init__(f"{what}: {sla_status_string(code)} ({code})")


def head_shard(B: int, H: int, world: int, rank: int) -> tuple:
    """(first, count): the contiguous range of the B*H (batch, head) pairs that rank
    ``rank`` of ``world`` owns.  Every stage of the forward (mask, smoothing mean,
    scales, states, per-query-block states, output) depends only on its own
    (batch, head), so sharded ranks exchange nothing.  The first B*H % world ranks
    take one pair more; a rank may own none when world > B*H."""
    if world < 1 or not 0 <= rank < world or B < 1 or H < 1:
        raise ValueError("need B, H, world >= 1 and 0 <= rank < world")
    bh = B * H
    base, extra = divmod(bh, world)
    first = rank * base + min(rank, extra)
    return first, base + (1 if rank < extra else 0)


def shard_heads(x, world: int, rank: int):
    """This rank's (batch, head) pairs of a [B, H, N, d] tensor (torch or numpy) as a
    [1, count, N, d] view: the pairs are consecutive rows of [B*H, N, d], so the view
    is contiguous and can go straight to sla_forward."""
    B, H, N, d = x.shape
    first, count = head_shard(B, H, world, rank)
    return x.reshape(B * H, N, d)[first:first + count].reshape(1, count, N, d)


def sla_version() -> str:
    return lib.sla_version().decode()


def sla_status_string(code: int) -> str:
    return lib.sla_status_string(int(code)).decode()


def sla_topk_count(n_kb: int, topk: float) -> int:
    return int(lib.sla_topk_count(int(n_kb), float(topk)))


def sla_workspace_bytes(B, H, N, d, blk_q, blk_k, topk, quant) -> int:
    return int(lib.sla_workspace_bytes(B, H, N, d, blk_q, blk_k, float(topk), int(quant)))


def sla_workspace_layout(B, H, N, d, blk_q, blk_k, topk, quant) -> dict:
    arr = (_SZ * len(LAYOUT_REGIONS))()
    n = lib.sla_workspace_layout(B, H, N, d, blk_q, blk_k, float(topk), int(quant), arr, len(arr))
    none = (1 << (8 * ctypes.sizeof(_SZ))) - 1
    return {name: (None if arr[i] == none else int(arr[i])) for i, name in enumerate(LAYOUT_REGIONS[:n])}


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(getattr(stream, "cuda_stream", stream))


def _bhnd(q):
    if q.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    return tuple(int(x) for x in q.shape)


def _ok(code: int, what: str) -> None:
    if code != 0:
        raise SlaError(code, what)


def workspace(B, H, N, d, blk_q, blk_k, topk, quant, device=None):
    """Allocate a workspace (uint8 CUDA tensor) large enough for sla_forward."""
    import torch
    n = sla_workspace_bytes(B, H, N, d, blk_q, blk_k, topk, quant)
    if n == 0:
        raise SlaError(1, "sla_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def sla_block_mask(q, k, blk_q, blk_k, topk, idx, bitmap, ws, stream=None) -> None:
    B, H, N, d = _bhnd(q)
    _ok(lib.sla_block_mask(_ptr(q), _ptr(k), B, H, N, d, blk_q, blk_k, float(topk), _ptr(idx), _ptr(bitmap),
                           _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "sla_block_mask")


def sla_block_mask_noalloc(q, k, blk_q, blk_k, topk, idx, bitmap, stream=None) -> None:
    """sla_block_mask without a workspace (scratch in a fixed static device array)."""
    B, H, N, d = _bhnd(q)
    _ok(lib.sla_block_mask_noalloc(_ptr(q), _ptr(k), B, H, N, d, blk_q, blk_k, float(topk), _ptr(idx),
                                   _ptr(bitmap), _stream(stream)), "sla_block_mask_noalloc")


def sla_block_mask_noalloc_limit() -> int:
    return int(lib.sla_block_mask_noalloc_limit())


def sla_quantize_qk(q, k, blk_q, blk_k, q_i8, k_i8, q_scale, k_scale, k_mean, ws, stream=None) -> None:
    B, H, N, d = _bhnd(q)
    _ok(lib.sla_quantize_qk(_ptr(q), _ptr(k), B, H, N, d, blk_q, blk_k, _ptr(q_i8), _ptr(k_i8), _ptr(q_scale),
                            _ptr(k_scale), _ptr(k_mean), _ptr(ws), ws.numel() * ws.element_size(),
                            _stream(stream)), "sla_quantize_qk")


def sla_quantize_qk_fp8(q, k, blk_q, blk_k, q_fp8, k_fp8, q_scale, k_scale, k_mean, ws, stream=None) -> None:
    B, H, N, d = _bhnd(q)
    _ok(lib.sla_quantize_qk_fp8(_ptr(q), _ptr(k), B, H, N, d, blk_q, blk_k, _ptr(q_fp8), _ptr(k_fp8),
                                _ptr(q_scale), _ptr(k_scale), _ptr(k_mean), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)), "sla_quantize_qk_fp8")


def sla_forward(q, k, v, out, blk_q, blk_k, topk, phi, quant, ws, stream=None) -> None:
    B, H, N, d = _bhnd(q)
    _ok(lib.sla_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, blk_q, blk_k, float(topk), int(phi),
                        int(quant), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "sla_forward")


def sla_forward_host_bytes(B, H, N, d, blk_q, blk_k, topk, quant, chunk_heads) -> int:
    return int(lib.sla_forward_host_bytes(B, H, N, d, blk_q, blk_k, float(topk), quant, chunk_heads))


def host_workspace(B, H, N, d, blk_q, blk_k, topk, quant, chunk_heads, device=None):
    """Allocate the device memory (uint8 CUDA tensor) of sla_forward_host."""
    import torch
    n = sla_forward_host_bytes(B, H, N, d, blk_q, blk_k, topk, quant, chunk_heads)
    if n == 0:
        raise SlaError(1, "sla_forward_host_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def sla_forward_host(q, k, v, out, blk_q, blk_k, topk, phi, quant, chunk_heads, dev, stream=None) -> None:
    """sla_forward from and to host memory: q, k, v, out are contiguous bf16 CPU tensors (page-locked for
    overlap); the copies run inside the call, chunk_heads (batch, head) problems at a time."""
    B, H, N, d = _bhnd(q)
    for t in (q, k, v, out):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("sla_forward_host takes contiguous host tensors")
    _ok(lib.sla_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, blk_q, blk_k, float(topk), int(phi),
                             int(quant), int(chunk_heads), _ptr(dev), dev.numel() * dev.element_size(),
                             _stream(stream)), "sla_forward_host")


def sla_backward_workspace_bytes(B, H, N, d, blk_q, blk_k, topk) -> int:
    return int(lib.sla_backward_workspace_bytes(B, H, N, d, blk_q, blk_k, float(topk)))


def backward_workspace(B, H, N, d, blk_q, blk_k, topk, device=None):
    """Allocate a workspace (uint8 CUDA tensor) large enough for sla_backward."""
    import torch
    n = sla_backward_workspace_bytes(B, H, N, d, blk_q, blk_k, topk)
    if n == 0:
        raise SlaError(1, "sla_backward_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def sla_backward(q, k, v, dout, dq, dk, dv, blk_q, blk_k, topk, phi, ws, stream=None) -> None:
    """Gradients (fp32 dq, dk, dv) of the unquantised forward for the output gradient dout."""
    B, H, N, d = _bhnd(q)
    _ok(lib.sla_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, blk_q,
                         blk_k, float(topk), int(phi), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
        "sla_backward")


PROFILE_STAGES = ("quantize_q", "states", "scores_topk", "quantize_k", "state_reduce", "attention", "total")


def sla_forward_profile(q, k, v, out, blk_q, blk_k, topk, phi, quant, ws, stream=None) -> dict:
    """sla_forward with per-stage device times (ms) from CUDA events between stages."""
    B, H, N, d = _bhnd(q)
    arr = (ctypes.c_float * len(PROFILE_STAGES))()
    _ok(lib.sla_forward_profile(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, blk_q, blk_k, float(topk),
                                int(phi), int(quant), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream),
                                arr), "sla_forward_profile")
    return {name: float(arr[i]) for i, name in enumerate(PROFILE_STAGES)}


def sla_set_wait_budget(cycles: int) -> None:
    """Clock-cycle budget of every bounded wait in the kernels on the current device
    (0 restores the default, about 0.5 s): a diagnostic for the failure path."""
    _ok(lib.sla_set_wait_budget(int(cycles)), "sla_set_wait_budget")


def sla_check(ws, stream=None) -> None:
    """Synchronise the stream and raise if a kernel recorded a device-side failure."""
    _ok(lib.sla_check(_ptr(ws), _stream(stream)), "sla_check")


# --------------------------------------------------------------------------
# W8A8 INT8 linear layer with FusedNorm
# --------------------------------------------------------------------------

def sla_w8a8_quantize(x, q, scale, norm: bool = False, gamma=None, eps: float = 1e-6, stream=None) -> None:
    """Per-row INT8 codes of a bf16 [rows, cols] tensor into q (int8, same shape) and scale
    (fp32 [rows]); with ``norm`` the rows are RMS-normalised (times ``gamma``) first."""
    rows, cols = x.shape
    _ok(lib.sla_w8a8_quantize(_ptr(x), rows, cols, int(bool(norm)), _ptr(gamma), float(eps), _ptr(q), _ptr(scale),
                              _stream(stream)), "sla_w8a8_quantize")


def w8a8_workspace(device=None):
    import torch
    return torch.zeros(int(lib.sla_w8a8_workspace_bytes()), dtype=torch.uint8, device=device or "cuda")


def sla_w8a8_linear(qx, sx, qw, sw, bias, out, ws, stream=None) -> None:
    """out (bf16 [M, N]) = (qx [M, K] int8) (qw [N, K] int8)^T * sx[M] * sw[N] (+ bias[N])."""
    M, K = qx.shape
    N = qw.shape[0]
    _ok(lib.sla_w8a8_linear(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), _ptr(bias), M, N, K, _ptr(out), _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "sla_w8a8_linear")

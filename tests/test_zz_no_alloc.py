"""The allocation-free block-mask entry point (GPU).

sla_block_mask_noalloc serves callers that cannot allocate device memory: its
scratch lives in a fixed static device array instead of a caller-provided
workspace.  It must give exactly the index lists and bitmaps of
sla_block_mask (masks are compared bit-exactly, like every mask test), on two
calls in a row -- the second call reuses the array the first one left behind
-- and refuse problems whose scratch does not fit the array.

Kept in its own file, collected last, so a failure here never stops the rest
of the GPU suite from running first.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_linear_bit_b200 as sla  # noqa: E402
import synth  # noqa: E402


def _dev(x):
    return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()


def _mask_with_workspace(qd, kd, blk_q, topk):
    B, H, N, d = qd.shape
    n_qb, n_kb = -(-N // blk_q), -(-N // 64)
    ks = sla.sla_topk_count(n_kb, topk)
    idx = torch.full((B, H, n_qb, max(ks, 1)), -7, dtype=torch.int32, device="cuda")
    bm = torch.full((B, H, n_qb, -(-n_kb // 32)), -1, dtype=torch.int32, device="cuda")
    ws = sla.workspace(B, H, N, d, blk_q, 64, topk, 0)
    sla.sla_block_mask(qd, kd, blk_q, 64, topk, idx, bm, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), bm.cpu().numpy()


def _mask_noalloc(qd, kd, blk_q, topk):
    """Through the C ABI directly (plain pointers, stream 0 = torch's default stream)."""
    B, H, N, d = qd.shape
    n_qb, n_kb = -(-N // blk_q), -(-N // 64)
    ks = sla.sla_topk_count(n_kb, topk)
    idx = torch.full((B, H, n_qb, max(ks, 1)), -7, dtype=torch.int32, device="cuda")
    bm = torch.full((B, H, n_qb, -(-n_kb // 32)), -1, dtype=torch.int32, device="cuda")
    rc = sla.lib.sla_block_mask_noalloc(ctypes.c_void_p(qd.data_ptr()), ctypes.c_void_p(kd.data_ptr()), B, H, N, d,
                                        blk_q, 64, ctypes.c_float(topk), ctypes.c_void_p(idx.data_ptr()),
                                        ctypes.c_void_p(bm.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, sla.sla_status_string(rc)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), bm.cpu().numpy()


CASES = [
    # (B, H, grid, blk_q, topk, adversarial)
    (1, 2, (8, 16, 16), 64, 0.1, ()),
    (1, 3, (21, 30, 52), 128, 0.1, ()),      # one 480P-grid head set: 256 x 512 blocks per head
    (2, 2, (5, 9, 13), 128, 0.3, ("ties",)),
]


def test_noalloc_matches_workspace_mask_twice():
    for (B, H, grid, blk_q, topk, adv) in CASES:
        q, k, _ = synth.make_qkv(B, H, grid, seed=77, adversarial=adv)
        qd, kd = _dev(q), _dev(k)
        ref_idx, ref_bm = _mask_with_workspace(qd, kd, blk_q, topk)
        for call in range(2):  # the second call reuses whatever the first left in the static array
            idx, bm = _mask_noalloc(qd, kd, blk_q, topk)
            assert np.array_equal(idx, ref_idx), (grid, call)
            assert np.array_equal(bm, ref_bm), (grid, call)


def test_noalloc_rejects_problems_beyond_the_static_scratch():
    limit = sla.sla_block_mask_noalloc_limit()
    assert limit == 16 << 20
    # 40 heads of the 720P grid need far more than 16 MiB of scores
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    rc = sla.lib.sla_block_mask_noalloc(ctypes.c_void_p(dummy.data_ptr()), ctypes.c_void_p(dummy.data_ptr()), 1, 40,
                                        75600, 128, 128, 64, ctypes.c_float(0.1),
                                        ctypes.c_void_p(dummy.data_ptr()), None, None)
    assert sla.sla_status_string(rc) == "SLA_ERR_WORKSPACE"

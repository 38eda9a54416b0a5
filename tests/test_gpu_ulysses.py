"""Ulysses layout permutations (CUDA) and the context-parallel forward on one rank.

The four block permutations of sla_ulysses_permute are compared with torch views of
the same permutation; with a single rank (NCCL, world size 1) the Ulysses forward
must equal sla_forward bit for bit (the exchange is then the identity).  The
two-rank exchange itself is covered by the gloo tests in test_multirank.py.
"""
from __future__ import annotations

import datetime
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import torch.distributed as dist  # noqa: E402

import sparse_linear_bit_b200 as sla  # noqa: E402
import synth  # noqa: E402
from sparse_linear_bit_b200 import ulysses  # noqa: E402


def _ref(src, B, H, P, n, d, mode):
    Hp = H // P
    if mode == 0:
        return src.reshape(B, P, Hp, n, d).permute(1, 0, 2, 3, 4).contiguous()
    if mode == 1:
        return src.permute(1, 2, 0, 3, 4).reshape(B, Hp, P * n, d).contiguous()
    if mode == 2:
        return src.reshape(B, Hp, P, n, d).permute(2, 0, 1, 3, 4).contiguous()
    return src.permute(1, 0, 2, 3, 4).reshape(B, H, n, d).contiguous()


@pytest.mark.parametrize("B,H,P,n,d,dtype", [
    (1, 40, 8, 9450, 128, torch.bfloat16),   # 720P tokens over 8 ranks
    (2, 12, 4, 100, 128, torch.bfloat16),
    (3, 6, 3, 33, 16, torch.float32),
    (1, 4, 1, 64, 128, torch.bfloat16),
])
def test_permute_modes(B, H, P, n, d, dtype):
    g = torch.Generator(device="cuda").manual_seed(3)
    Hp = H // P
    shapes = {0: (B, H, n, d), 1: (P, B, Hp, n, d), 2: (B, Hp, P * n, d), 3: (P, B, Hp, n, d)}
    for mode, shp in shapes.items():
        src = torch.randn(shp, device="cuda", generator=g).to(dtype)
        ref = _ref(src, B, H, P, n, d, mode)
        dst = torch.empty_like(ref)
        ulysses.cuda_permute(src, dst, B, H, P, n, d, mode)
        torch.cuda.synchronize()
        assert torch.equal(dst, ref), mode


def test_single_rank_ulysses_equals_forward():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        q, k, v = synth.make_qkv(1, 2, (8, 16, 16), seed=31)
        qd, kd, vd = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (q, k, v))
        out = torch.empty_like(qd)
        ws = sla.workspace(1, 2, qd.shape[2], 128, 64, 64, 0.1, 1)
        sla.sla_forward(qd, kd, vd, out, 64, 64, 0.1, 0, 1, ws)
        got = ulysses.sla_forward_ulysses(qd, kd, vd, 64, 64, 0.1, 0, 1)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), out.view(torch.int16))
    finally:
        dist.destroy_process_group()

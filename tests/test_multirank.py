"""Multi-rank host logic on CPU (gloo, world size 2): head sharding and device-time reduction.

Every stage of the forward depends only on its own (batch, head), so the multi-GPU path
shards contiguous head ranges across ranks with no exchange.  Here each rank runs the fp64
oracle on its shard; the gathered shards must equal the unsharded oracle output exactly.
The bench's max-over-ranks reduction is checked on the same process group.
"""
from __future__ import annotations

import datetime
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, B, H, grid, blk_q, topk, quant, result_path):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import bench
        import oracle
        import sparse_linear_bit_b200 as sla
        import synth

        # the bench's device-time reduction: max over ranks
        assert bench.max_over_ranks(1.5 * (rank + 1), torch.device("cpu"), world) == 1.5 * world

        q, k, v = synth.make_qkv(B, H, grid, seed=23)
        first, count = sla.head_shard(B, H, world, rank)
        shard = [np.ascontiguousarray(sla.shard_heads(x, world, rank)) for x in (q, k, v)]
        assert shard[0].shape == (1, count) + q.shape[2:]
        out = oracle.forward(*shard, blk_q, 64, topk, phi=0, quant=quant) if count else np.zeros((1, 0) + q.shape[2:])
        parts = [None] * world
        dist.all_gather_object(parts, (first, count, out))
        if rank == 0:
            full = oracle.forward(q, k, v, blk_q, 64, topk, phi=0, quant=quant).reshape(B * H, *q.shape[2:])
            got = np.concatenate([p[2].reshape(p[1], *q.shape[2:]) for p in sorted(parts, key=lambda p: p[0])])
            ok = got.shape == full.shape and np.array_equal(got, full)
            with open(result_path, "w") as f:
                f.write("ok" if ok else f"mismatch {got.shape} {full.shape}")
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,H,grid,blk_q,topk,quant", [
    (1, 3, (4, 8, 8), 64, 0.25, 1),     # 3 heads over 2 ranks: 2 + 1
    (2, 2, (3, 5, 7), 128, 0.3, 0),     # ragged N = 105, heads of two batch elements
])
def test_sharded_oracle_matches_unsharded_gloo(tmp_path, B, H, grid, blk_q, topk, quant):
    import oracle
    oracle.build()
    result = tmp_path / "result.txt"
    mp.start_processes(_worker, args=(2, _free_port(), B, H, grid, blk_q, topk, quant, str(result)), nprocs=2,
                       join=True, start_method="spawn")
    assert result.read_text() == "ok"


def test_head_shard_partition():
    import sparse_linear_bit_b200 as sla
    for B, H in [(1, 40), (2, 12), (1, 3), (3, 5)]:
        for world in (1, 2, 3, 4, 8, 16):
            seen = []
            for r in range(world):
                first, count = sla.head_shard(B, H, world, r)
                assert count >= 0
                seen.extend(range(first, first + count))
            assert seen == list(range(B * H))  # every pair exactly once, in rank order
            counts = [sla.head_shard(B, H, world, r)[1] for r in range(world)]
            assert max(counts) - min(counts) <= 1
    with pytest.raises(ValueError):
        sla.head_shard(1, 4, 2, 2)


def test_shard_heads_view_is_contiguous_rows():
    import sparse_linear_bit_b200 as sla
    x = np.arange(2 * 3 * 4 * 5).reshape(2, 3, 4, 5)
    parts = [sla.shard_heads(x, 4, r) for r in range(4)]
    assert [p.shape[1] for p in parts] == [2, 2, 1, 1]
    assert np.array_equal(np.concatenate([p[0] for p in parts]), x.reshape(6, 4, 5))
    t = torch.arange(2 * 3 * 4 * 5).reshape(2, 3, 4, 5)
    assert sla.shard_heads(t, 4, 1).is_contiguous()

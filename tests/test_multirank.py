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


# --------------------------------------------------------------------------
# Ulysses context parallelism: token shards -> head shards -> token shards
# --------------------------------------------------------------------------

def torch_permute(src, dst, B, H, P, n, d, mode):
    """Reference of the four block permutations (torch views; the CUDA kernel is checked
    against this on the GPU)."""
    Hp = H // P
    if mode == 0:    # [B][H][n][d] -> [P][B][Hp][n][d]
        dst.copy_(src.reshape(B, P, Hp, n, d).permute(1, 0, 2, 3, 4))
    elif mode == 1:  # [P][B][Hp][n][d] -> [B][Hp][P*n][d]
        dst.copy_(src.permute(1, 2, 0, 3, 4).reshape(B, Hp, P * n, d))
    elif mode == 2:  # [B][Hp][P*n][d] -> [P][B][Hp][n][d]
        dst.copy_(src.reshape(B, Hp, P, n, d).permute(2, 0, 1, 3, 4))
    else:            # [P][B][Hp][n][d] -> [B][H][n][d]
        dst.copy_(src.permute(1, 0, 2, 3, 4).reshape(B, H, n, d))


def _ulysses_worker(rank, world, port, B, H, grid, blk_q, topk, result_path):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        import synth
        from sparse_linear_bit_b200 import ulysses

        q, k, v = synth.make_qkv(B, H, grid, seed=29)
        N = q.shape[2]
        n = N // world
        # bf16 bit patterns carried as int32 (gloo's all-to-all takes no 16-bit tensors)
        as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).astype(np.int32))
        shard = lambda a: as_t(a[:, :, rank * n:(rank + 1) * n])
        qh, kh, vh = (ulysses.seq_to_heads(shard(a), permute=torch_permute) for a in (q, k, v))
        Hp = H // world
        # the exchange hands this rank every token of its heads
        assert torch.equal(qh, as_t(q[:, rank * Hp:(rank + 1) * Hp]))
        out_h = oracle.forward(*(x.numpy().astype(np.uint16) for x in (qh, kh, vh)), blk_q, 64, topk, phi=0, quant=1)
        # back to the token sharding (fp64 values carried as int64 bit patterns)
        out_seq = ulysses.heads_to_seq(torch.from_numpy(out_h.view(np.int64)), permute=torch_permute)
        parts = [None] * world
        dist.all_gather_object(parts, out_seq.numpy().view(np.float64))
        if rank == 0:
            full = oracle.forward(q, k, v, blk_q, 64, topk, phi=0, quant=1)
            got = np.concatenate(parts, axis=2)
            ok = got.shape == full.shape and np.array_equal(got, full)
            with open(result_path, "w") as f:
                f.write("ok" if ok else f"mismatch {got.shape} {full.shape}")
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,H,grid,blk_q,topk", [
    (1, 4, (4, 8, 8), 64, 0.25),     # N = 256: 128 tokens per rank, 2 heads per rank
    (2, 2, (2, 8, 16), 128, 0.3),    # two batch elements, one head per rank
])
def test_ulysses_exchange_gloo(tmp_path, B, H, grid, blk_q, topk):
    import oracle
    oracle.build()
    result = tmp_path / "result.txt"
    mp.start_processes(_ulysses_worker, args=(2, _free_port(), B, H, grid, blk_q, topk, str(result)), nprocs=2,
                       join=True, start_method="spawn")
    assert result.read_text() == "ok"

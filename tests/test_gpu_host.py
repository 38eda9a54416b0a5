"""The forward from and to host memory (sla_forward_host), on the GPU.

Every (batch, head) problem is independent, so the chunked, pipelined call must give
the output of one sla_forward over the whole problem bit for bit, whatever the
chunking (one problem per chunk, a ragged last chunk, one chunk for all), with
page-locked or pageable host buffers; and it must match the fp64 oracle within the
forward's bar (quantised: cosine >= 0.999, relative L2 <= 2e-2; unquantised:
relative L2 <= 2e-3).  Its status word is the workspace's at the start of the device
memory: a one-cycle wait budget makes every chunk time out and sla_check report
SLA_ERR_TIMEOUT, and the next call on the same memory is clean and exact.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_to_f64, cosine, rel_l2, to_dev, workload_qkv

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_linear_bit_b200 as sla  # noqa: E402


def host(x: np.ndarray, pinned: bool):
    t = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16)
    return t.pin_memory() if pinned else t


def device_forward(q, k, v, blk_q, topk, phi, quant):
    B, H, N, d = q.shape
    qd, kd, vd = to_dev(q, torch), to_dev(k, torch), to_dev(v, torch)
    out = torch.empty_like(qd)
    ws = sla.workspace(B, H, N, d, blk_q, 64, topk, quant)
    sla.sla_forward(qd, kd, vd, out, blk_q, 64, topk, phi, quant, ws)
    sla.sla_check(ws)
    return out.cpu()


def host_forward(q, k, v, blk_q, topk, phi, quant, chunk, pinned=True, stream=None):
    B, H, N, d = q.shape
    hq, hk, hv = host(q, pinned), host(k, pinned), host(v, pinned)
    hout = torch.empty(hq.shape, dtype=torch.bfloat16)
    if pinned:
        hout = hout.pin_memory()
    dev = sla.host_workspace(B, H, N, d, blk_q, 64, topk, quant, chunk)
    sla.sla_forward_host(hq, hk, hv, hout, blk_q, 64, topk, phi, quant, chunk, dev, stream=stream)
    sla.sla_check(dev, stream=stream)
    return hout, dev


@pytest.mark.parametrize("chunk", [1, 4, 6, 64])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_forward_equals_device_forward(chunk, pinned):
    q, k, v = synth.make_qkv(2, 3, (4, 16, 32), seed=71)  # 6 problems of N = 2048
    ref = device_forward(q, k, v, 64, 0.1, 0, 1)
    got, _ = host_forward(q, k, v, 64, 0.1, 0, 1, chunk, pinned)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), (chunk, pinned)


@pytest.mark.parametrize("quant,phi,topk", [(1, 0, 0.1), (0, 1, 0.25), (2, 0, 0.5)])
def test_host_forward_matches_oracle(quant, phi, topk):
    q, k, v = synth.make_qkv(1, 3, (3, 10, 70), seed=72 + quant)  # N = 2100: ragged tails
    s = torch.cuda.Stream()
    got, _ = host_forward(q, k, v, 128, topk, phi, quant, 2, stream=s)
    ref = oracle.forward(q, k, v, 128, 64, float(np.float32(topk)), phi=phi, quant=quant)
    r, c = rel_l2(bf16_to_f64(got), ref), cosine(bf16_to_f64(got), ref)
    if quant:
        assert r <= 2e-2 and c >= 0.999, (r, c)
    else:
        assert r <= 2e-3, r


def test_host_forward_timeout_is_reported_and_the_memory_recovers():
    q, k, v = synth.make_qkv(1, 4, (8, 32, 32), seed=73)  # N = 8192, 2 chunks of 2 heads
    B, H, N, d = q.shape
    hq, hk, hv = host(q, True), host(k, True), host(v, True)
    hout = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    dev = sla.host_workspace(B, H, N, d, 128, 64, 0.25, 1, 2)
    sla.sla_set_wait_budget(1)
    try:
        sla.sla_forward_host(hq, hk, hv, hout, 128, 64, 0.25, 0, 1, 2, dev)
        with pytest.raises(sla.SlaError) as err:
            sla.sla_check(dev)
        assert sla.sla_status_string(err.value.code) == "SLA_ERR_TIMEOUT"
    finally:
        sla.sla_set_wait_budget(0)
    torch.cuda.synchronize()
    sla.sla_forward_host(hq, hk, hv, hout, 128, 64, 0.25, 0, 1, 2, dev)
    sla.sla_check(dev)
    ref = device_forward(q, k, v, 128, 0.25, 0, 1)
    assert torch.equal(hout.view(torch.int16), ref.view(torch.int16))


def test_host_forward_rejects_device_tensors():
    q, k, v = synth.make_qkv(1, 1, (2, 8, 16), seed=74)
    qd = to_dev(q, torch)
    dev = sla.host_workspace(1, 1, 256, 128, 64, 64, 0.1, 1, 1)
    with pytest.raises(ValueError):
        sla.sla_forward_host(qd, qd, qd, qd, 64, 64, 0.1, 0, 1, 1, dev)


def test_host_forward_at_480p_shape_equals_device_forward():
    """The 1.3B-480P workload (B=1, H=12, N=32760) in chunks of 5 heads (5 + 5 + 2), INT8: the same
    bytes as one device call."""
    w = synth.WORKLOADS["wan1.3b-480p"]
    q, k, v = workload_qkv("wan1.3b-480p")
    ref = device_forward(q, k, v, w.blk_q, w.topk, 0, 1)
    got, _ = host_forward(q, k, v, w.blk_q, w.topk, 0, 1, 5)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))

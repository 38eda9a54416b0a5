"""The failure path of the kernels' bounded waits, on the GPU, without a GPU fault.

Every wait of the tensor-core kernels (states, state reduction, attention) gives up
after a clock budget, records SLA_ERR_TIMEOUT in the workspace's status word and
unwinds: it stops issuing work, lets the copies and tensor-core operations it already
issued retire, frees its tensor memory and returns.  With the budget set to one clock
cycle through sla_set_wait_budget, every wait that is still pending when it is first
tested runs out at once -- the linear-branch issuer of the attention kernel, for one,
waits from its start until the last key block is done -- so the call must:

* return (no hang), with sla_check reporting SLA_ERR_TIMEOUT;
* leave the context usable: a following call on the SAME workspace with the default
  budget reports SLA_OK and matches the oracle (cosine >= 0.999, relative L2 <= 2e-2).

The same holds for the backward, whose tensor-core kernels (the forward's states and
state reduction, and the softmax branch's query and key sides) wait the same bounded
way: with a one-cycle budget sla_backward must report SLA_ERR_TIMEOUT and return, and a
following call on the same workspace must match the oracle's gradients (relative L2
<= 5e-3, the backward's bar).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_to_f64, cosine, rel_l2, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_linear_bit_b200 as sla  # noqa: E402


def test_short_wait_budget_times_out_cleanly_and_the_workspace_recovers():
    B, H, grid, blk_q, topk = 1, 2, (8, 32, 32), 128, 0.25  # N = 8192: 32 selected of 128 key blocks
    q, k, v = synth.make_qkv(B, H, grid, seed=91)
    N, d = q.shape[2], q.shape[3]
    qd, kd, vd = to_dev(q, torch), to_dev(k, torch), to_dev(v, torch)
    out = torch.zeros_like(qd)
    ws = sla.workspace(B, H, N, d, blk_q, 64, topk, 1)
    sla.sla_set_wait_budget(1)
    try:
        sla.sla_forward(qd, kd, vd, out, blk_q, 64, topk, 0, 1, ws)
        with pytest.raises(sla.SlaError) as err:
            sla.sla_check(ws)
        assert sla.sla_status_string(err.value.code) == "SLA_ERR_TIMEOUT"
    finally:
        sla.sla_set_wait_budget(0)
    torch.cuda.synchronize()

    # the same workspace, the default budget: a clean, correct call
    sla.sla_forward(qd, kd, vd, out, blk_q, 64, topk, 0, 1, ws)
    sla.sla_check(ws)
    got = bf16_to_f64(out)
    ref = oracle.forward(q, k, v, blk_q, 64, float(np.float32(topk)), phi=0, quant=1)
    r, c = rel_l2(got, ref), cosine(got, ref)
    assert r <= 2e-2 and c >= 0.999, (r, c)


def test_short_wait_budget_in_the_backward_times_out_cleanly_and_recovers():
    B, H, grid, blk_q, topk = 1, 2, (8, 16, 16), 128, 0.25  # N = 2048: 8 selected of 32 key blocks
    q, k, v = synth.make_qkv(B, H, grid, seed=93)
    dout = synth.make_qkv(B, H, grid, seed=94)[0]
    N, d = q.shape[2], q.shape[3]
    qd, kd, vd, dod = (to_dev(x, torch) for x in (q, k, v, dout))
    grads = [torch.zeros(B, H, N, d, dtype=torch.float32, device="cuda") for _ in range(3)]
    ws = sla.backward_workspace(B, H, N, d, blk_q, 64, topk)
    sla.sla_set_wait_budget(1)
    try:
        sla.sla_backward(qd, kd, vd, dod, *grads, blk_q, 64, topk, 0, ws)
        with pytest.raises(sla.SlaError) as err:
            sla.sla_check(ws)
        assert sla.sla_status_string(err.value.code) == "SLA_ERR_TIMEOUT"
    finally:
        sla.sla_set_wait_budget(0)
    torch.cuda.synchronize()

    sla.sla_backward(qd, kd, vd, dod, *grads, blk_q, 64, topk, 0, ws)
    sla.sla_check(ws)
    ref = oracle.backward(q, k, v, dout, blk_q, 64, float(np.float32(topk)), phi=0)
    for g, r in zip(grads, ref):
        err = rel_l2(g.cpu().numpy().astype(np.float64), r)
        assert err <= 5e-3, err


def test_wait_budget_argument_checks():
    with pytest.raises(sla.SlaError):
        sla.sla_set_wait_budget(-1)
    sla.sla_set_wait_budget(0)

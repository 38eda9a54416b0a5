"""GPU parity of the backward (sla_backward, through the C ABI) against the
fp64 CPU oracle's backward.

Tolerance (relative L2 over each of dq, dk, dv): 5e-3.  The sparse branch's
per-tile products take bf16 operands (the inputs themselves, and P and dS
rounded to bf16: relative 2^-9 per element, with fp32 accumulation, so the
error of a sum of many such terms stays near 2^-9 or below); the linear branch
uses the forward's own state: key-block states in bf16 (2^-9), H_I rounded to
tf32 (2^-11), and the state gradients entering G = A^T dH as bf16 (2^-9).  So
either branch's part of a gradient carries up to ~2 x 2^-9 ~ 4e-3 relative
error, and the whole gradient less.
Every element must also be finite, and two calls must give identical bytes.
At the full 14B-720P and 1.3B-480P sizes, dq of sampled rows and dk, dv of sampled key
blocks are compared with the oracle, which evaluates exactly those rows / blocks.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import rel_l2, to_dev, workload_qkv

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_linear_bit_b200 as sla  # noqa: E402

TOL = 5e-3

CASES = {
    # name: ((B, H, grid), blk_q, topk, phi)
    "ragged_subtract_elu": ((1, 2, (3, 10, 7)), 128, 0.3, 0),
    "ragged_complement_relu": ((1, 2, (5, 9, 13)), 64, 0.6, 1),
    "multi_tile_elu": ((1, 2, (8, 16, 16)), 128, 0.1, 0),
    "linear_only": ((1, 2, (5, 9, 13)), 128, 0.0, 0),
    "sparse_only_relu": ((1, 2, (5, 9, 13)), 128, 1.0, 1),
    "two_batches_q64": ((2, 1, (4, 10, 13)), 64, 0.25, 0),
    # n_kb = 144 > 128: the transposed state reduction spans two row tiles
    "n_kb_144": ((1, 1, (8, 32, 36)), 128, 0.1, 0),
}


def run_backward(q, k, v, dout, blk_q, topk, phi):
    B, H, N, d = q.shape
    qd, kd, vd, dod = (to_dev(x, torch) for x in (q, k, v, dout))
    dq, dk, dv = (torch.empty(B, H, N, d, dtype=torch.float32, device="cuda") for _ in range(3))
    ws = sla.backward_workspace(B, H, N, d, blk_q, 64, topk)
    sla.sla_backward(qd, kd, vd, dod, dq, dk, dv, blk_q, 64, topk, phi, ws)
    sla.sla_check(ws)
    return dq, dk, dv


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_parity(name):
    (B, H, grid), blk_q, topk, phi = CASES[name]
    q, k, v = synth.make_qkv(B, H, grid, seed=500 + len(name))
    dout = synth.make_qkv(B, H, grid, seed=600 + len(name))[0]
    got = [t.cpu().numpy().astype(np.float64) for t in run_backward(q, k, v, dout, blk_q, topk, phi)]
    ref = oracle.backward(q, k, v, dout, blk_q, 64, float(np.float32(topk)), phi=phi)
    for nm, g_, r_ in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(g_).all(), (name, nm)
        err = rel_l2(g_, r_)
        print(f"\n{name} {nm}: rel_l2={err:.3e}")
        assert err <= TOL, (name, nm, err)


def test_backward_deterministic():
    q, k, v = synth.make_qkv(1, 2, (8, 16, 16), seed=77)
    dout = synth.make_qkv(1, 2, (8, 16, 16), seed=78)[0]
    a = run_backward(q, k, v, dout, 128, 0.1, 0)
    b = run_backward(q, k, v, dout, 128, 0.1, 0)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32))


def test_backward_full_size_scaling():
    """14B-720P shape (B=1, H=40, N=75600): the gradients are linear in dout, and
    doubling dout doubles every fp32 operation exactly, so the results must be
    exactly twice those for dout; all finite."""
    w = synth.WORKLOADS["wan14b-720p"]
    q, k, v = workload_qkv("wan14b-720p")
    dout = workload_qkv("wan14b-720p", seed_offset=1)[0]
    qd, kd, vd, dod = (to_dev(x, torch) for x in (q, k, v, dout))
    del q, k, v, dout
    B, H, N, d = qd.shape
    ws = sla.backward_workspace(B, H, N, d, w.blk_q, w.blk_k, 0.1)
    outs = []
    for scale in (1.0, 2.0):
        g = [torch.empty(B, H, N, d, dtype=torch.float32, device="cuda") for _ in range(3)]
        do_s = (dod.float() * scale).bfloat16()
        sla.sla_backward(qd, kd, vd, do_s, *g, w.blk_q, w.blk_k, 0.1, 0, ws)
        sla.sla_check(ws)
        outs.append(g)
    for x, y in zip(*outs):
        assert torch.isfinite(x).all()
        assert torch.equal(x * 2.0, y)


def test_backward_full_size_sampled_dq():
    """14B-720P shape (B=1, H=40, N=75600), the launch configuration bench.py times: dq of sampled rows
    of 3 heads against the oracle, which computes them row by row.  An fp64 emulation of the
    kernel's bf16 roundings (dS, and P inside D = do.os) on such rows predicts about 2.2e-3."""
    w = synth.WORKLOADS["wan14b-720p"]
    q, k, v = workload_qkv("wan14b-720p")
    dout = workload_qkv("wan14b-720p", seed_offset=1)[0]
    dq, dk, dv = run_backward(q, k, v, dout, w.blk_q, 0.1, 0)
    del dk, dv
    rows = synth.sample_rows(w.B, w.H, w.N, n_heads=3, rows_per_head=48)
    got = dq.cpu().numpy().reshape(w.B * w.H, w.N, 128)[rows[:, 0], rows[:, 1]].astype(np.float64)
    ref = oracle.backward_dq_rows(q, k, v, dout, w.blk_q, w.blk_k, float(np.float32(0.1)), rows, phi=0)
    assert np.isfinite(got).all()
    err = rel_l2(got, ref)
    print(f"\nfull-size sampled rows: dq rel_l2={err:.3e}")
    assert err <= TOL, err


def test_backward_full_size_sampled_dkdv():
    """14B-720P shape (B=1, H=40, N=75600), the launch configuration bench.py times: dk and dv of three
    key blocks of three heads -- the first block, one in the middle and the ragged last block (16 keys)
    -- against the oracle, which evaluates exactly those blocks (their linear part needs the state
    gradients of every query block that did not select them, their softmax part every row that did)."""
    w = synth.WORKLOADS["wan14b-720p"]
    q, k, v = workload_qkv("wan14b-720p")
    dout = workload_qkv("wan14b-720p", seed_offset=1)[0]
    dq, dk, dv = run_backward(q, k, v, dout, w.blk_q, 0.1, 0)
    del dq
    n_kb = -(-w.N // w.blk_k)
    blocks = np.array([[0, 0], [17, n_kb // 2], [39, n_kb - 1]], dtype=np.int64)
    ref_k, ref_v = oracle.backward_dkdv_blocks(q, k, v, dout, w.blk_q, w.blk_k, float(np.float32(0.1)), blocks,
                                               phi=0)
    dk_h, dv_h = dk.view(w.B * w.H, w.N, 128), dv.view(w.B * w.H, w.N, 128)
    gk, gv, rk, rv = [], [], [], []
    for b, (bh, J) in enumerate(blocks.tolist()):
        n = min(64, w.N - 64 * J)
        gk.append(dk_h[bh, 64 * J:64 * J + n].cpu().numpy().astype(np.float64))
        gv.append(dv_h[bh, 64 * J:64 * J + n].cpu().numpy().astype(np.float64))
        rk.append(ref_k[b, :n])
        rv.append(ref_v[b, :n])
    gk, gv, rk, rv = (np.concatenate(x) for x in (gk, gv, rk, rv))
    assert np.isfinite(gk).all() and np.isfinite(gv).all()
    ek, ev = rel_l2(gk, rk), rel_l2(gv, rv)
    print(f"\nfull-size sampled key blocks: dk rel_l2={ek:.3e} dv rel_l2={ev:.3e}")
    assert ek <= TOL and ev <= TOL, (ek, ev)


def test_backward_480p_sampled():
    """1.3B-480P shape (B=1, H=12, N=32760: its last query block holds 120 rows and its last key block
    56 keys), one call: dq of sampled rows of 3 heads, and dk, dv of the first, a middle and the ragged
    last key block of 3 heads, against the oracle."""
    w = synth.WORKLOADS["wan1.3b-480p"]
    q, k, v = workload_qkv("wan1.3b-480p")
    dout = workload_qkv("wan1.3b-480p", seed_offset=1)[0]
    dq, dk, dv = run_backward(q, k, v, dout, w.blk_q, 0.1, 0)
    topk = float(np.float32(0.1))
    rows = synth.sample_rows(w.B, w.H, w.N, n_heads=3, rows_per_head=32)
    got = dq.cpu().numpy().reshape(w.B * w.H, w.N, 128)[rows[:, 0], rows[:, 1]].astype(np.float64)
    ref = oracle.backward_dq_rows(q, k, v, dout, w.blk_q, w.blk_k, topk, rows, phi=0)
    eq = rel_l2(got, ref)
    n_kb = -(-w.N // w.blk_k)
    blocks = np.array([[0, 0], [5, n_kb // 2], [11, n_kb - 1]], dtype=np.int64)
    ref_k, ref_v = oracle.backward_dkdv_blocks(q, k, v, dout, w.blk_q, w.blk_k, topk, blocks, phi=0)
    dk_h, dv_h = dk.view(w.B * w.H, w.N, 128), dv.view(w.B * w.H, w.N, 128)
    gk, gv, rk, rv = [], [], [], []
    for b, (bh, J) in enumerate(blocks.tolist()):
        n = min(64, w.N - 64 * J)
        gk.append(dk_h[bh, 64 * J:64 * J + n].cpu().numpy().astype(np.float64))
        gv.append(dv_h[bh, 64 * J:64 * J + n].cpu().numpy().astype(np.float64))
        rk.append(ref_k[b, :n])
        rv.append(ref_v[b, :n])
    gk, gv, rk, rv = (np.concatenate(x) for x in (gk, gv, rk, rv))
    assert np.isfinite(got).all() and np.isfinite(gk).all() and np.isfinite(gv).all()
    ek, ev = rel_l2(gk, rk), rel_l2(gv, rv)
    print(f"\n480P sampled: dq rel_l2={eq:.3e} dk rel_l2={ek:.3e} dv rel_l2={ev:.3e}")
    assert eq <= TOL and ek <= TOL and ev <= TOL, (eq, ek, ev)

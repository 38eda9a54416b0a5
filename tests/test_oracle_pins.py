"""Pins of the fp64 CPU oracle against things other than itself.

Each ``pin_*`` function takes the loaded oracle library (so that
``test_oracle_mutants.py`` can re-run them against deliberately broken builds
of the oracle) and raises AssertionError on a mismatch.  What pins what:

* selection count  -- the counts every workload states, and the pages' "about
  10 %" kept fraction ("清华开源TurboDiffusion加速框架", SageAttention与稀疏计算)
* block mask       -- exhaustive subset search (dominance order) on tiny inputs
  with forced ties; invariances under token permutation inside a block, key
  block permutation, positive power-of-two scaling of Q, a constant shift of K;
  all-identical and all-zero key blocks select the lowest indices
* quantisation     -- a block whose values are exact multiples of the scale;
  range, amax -> +-127 and half-step error bounds; zero block; smoothing
  invariance to a per-channel shift of K; Q is not smoothed
* FP8 e4m3         -- the encoder equals torch's float8_e4m3fn conversion (round to
  nearest even) below the saturation point and saturates at +-448 above it; per
  block the amax element maps to +-448 and every element lies within half an e4m3
  step of its code; with quant = 2, topk = 1 equals softmax attention on the
  decoded codes and general topk equals the dense brute force on them
* W8A8 linear      -- per-row codes: amax -> +-127, half-step bounds, zero rows; with
  FusedNorm the decoded rows equal torch's float32 rms_norm (eps and gamma included,
  rows small enough for eps to matter) within half a step; the linear layer equals
  numpy's int64 matmul of the codes times both scales plus bias, and the decoded
  product stays within the quantisation error bound of the fp64 x w^T
* forward          -- topk = 1 equals dense softmax attention from
  torch's float64 scaled_dot_product_attention; topk = 0 equals closed-form
  linear attention phi(Q)(phi(K)^T V) / phi(Q)(phi(K)^T 1) ("TurboDiffusion
  技术架构解析" §2.1); the attention-form dense brute force for general topk,
  with and without quantisation, with ragged tails; constant V gives 2c
  (c at topk 0 or 1); convex-hull bounds; ReLU rows with phi(q) = 0 give a
  zero linear part; the row-sampled API equals the full forward.
* backward         -- float64 autograd of an attention-form PyTorch statement of
  the unquantised forward (dense token mask; the linear branch as masked
  phi(Q) phi(K)^T weights, not the oracle's state form), whose values are first
  checked against ``forward``; topk = 1 against autograd of torch's
  scaled_dot_product_attention; topk = 0 against autograd of closed-form
  linear attention; ragged blocks, both phi, and ReLU rows with a zero
  denominator; the row-sampled dq equals the full backward's.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from bruteforce import dominant_subset, phi as bf_phi, quant_logits, sla_dense

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _qkv(grid, d=32, B=1, H=1, seed=0, **kw):
    return synth.make_qkv(B, H, grid, d=d, seed=seed, threads=1, **kw)


def _bits_from_f64(x):
    return synth.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


# --------------------------------------------------------------------------
# selection count
# --------------------------------------------------------------------------

def pin_topk_count(lib):
    with open(os.path.join(GOLDEN, "topk_counts.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        got = int(lib.orc_topk_count(case["n_kb"], float(np.float32(case["topk"]))))
        assert got == case["k_sel"], (case, got)
    # the pages' default keeps about 10 % of key blocks
    for n_kb in (32, 256, 512, 1182):
        ks = int(lib.orc_topk_count(n_kb, float(np.float32(0.1))))
        assert abs(ks - 0.1 * n_kb) < 1.0


# --------------------------------------------------------------------------
# block mask
# --------------------------------------------------------------------------

def _mask(lib, q, k, blk_q, blk_k, topk):
    return oracle.block_mask(q, k, blk_q, blk_k, topk, with_scores=True, lib=lib)


def pin_mask_exhaustive(lib):
    # values on a 1/4 grid and power-of-two token counts per block: every mean
    # and every score is exact in fp64, so ties are exact ties on both sides
    rng = np.random.default_rng(11)
    d, blk_k = 4, 2
    for trial in range(8):
        n_kb = 7 + trial % 4                      # 7..10 key blocks
        N = n_kb * blk_k - (trial % 2)            # odd N -> ragged last block
        blk_q = 4 if N % 4 in (0, 1, 2) else 2
        q = _bits_from_f64(rng.integers(-4, 5, size=(1, N, d)) / 4.0)
        kf = rng.integers(-4, 5, size=(N, d)) / 4.0
        # force ties: duplicate a couple of key blocks
        kf[2 * blk_k:3 * blk_k] = kf[0:blk_k]
        kf[4 * blk_k:5 * blk_k] = kf[1 * blk_k:2 * blk_k]
        k = _bits_from_f64(kf[None])
        qf, kfr = synth.bf16_bits_to_f64(q[0]), synth.bf16_bits_to_f64(k[0])
        n_qb = -(-N // blk_q)
        for topk in (0.0, 0.15, 0.3, 0.5, 1.0):
            idx, bm, sc = _mask(lib, q, k, blk_q, blk_k, topk)
            ks = idx.shape[2]
            for I in range(n_qb):
                qm = qf[I * blk_q:(I + 1) * blk_q].mean(axis=0)
                km = np.stack([kfr[J * blk_k:(J + 1) * blk_k].mean(axis=0) for J in range(n_kb)])
                s = km @ qm
                expect = dominant_subset(s, ks)
                assert np.array_equal(idx[0, I], expect), (trial, topk, I, idx[0, I], expect, s)
                bits = [J for J in range(n_kb) if (bm[0, I, J >> 5] >> (J & 31)) & 1]
                assert bits == list(expect)


def pin_mask_invariances(lib):
    # values on a 1/8 grid with |x| <= 16: block sums, means (blocks of 16/32
    # tokens) and shifted copies stay exact in bf16 and fp64
    rng = np.random.default_rng(3)
    N, d, blk_q, blk_k, topk = 256, 32, 32, 16, 0.25
    q = _bits_from_f64(rng.integers(-128, 129, size=(1, N, d)) / 8.0)
    k = _bits_from_f64(rng.integers(-64, 65, size=(1, N, d)) / 8.0)
    idx0, _, sc0 = _mask(lib, q, k, blk_q, blk_k, topk)
    n_kb, ks = N // blk_k, idx0.shape[2]
    srt = -np.sort(-sc0[0], axis=1)
    ok_rows = (srt[:, ks - 1] - srt[:, ks]) > 1e-6 * np.abs(srt).max()
    assert ok_rows.mean() > 0.7
    # (1) permuting tokens inside each key block leaves every mean unchanged
    perm = np.concatenate([J * blk_k + rng.permutation(blk_k) for J in range(n_kb)])
    idx1, _, sc1 = _mask(lib, q[:, perm], k[:, perm], blk_q, blk_k, topk)
    assert np.array_equal(idx0, idx1) and np.array_equal(sc0, sc1)
    # (2) permuting key blocks permutes scores and selection
    bperm = rng.permutation(n_kb)
    tok = np.concatenate([np.arange(J * blk_k, (J + 1) * blk_k) for J in bperm])
    idx2, _, sc2 = _mask(lib, q, k[:, tok], blk_q, blk_k, topk)
    assert np.array_equal(sc2[0][:, np.argsort(bperm)], sc0[0])
    for I in np.nonzero(ok_rows)[0]:
        assert np.array_equal(np.sort(bperm[idx2[0, I]]), idx0[0, I]), I
    # (3) Q scaled by 2 (exact): scores double, same selection
    q2 = _bits_from_f64(2.0 * synth.bf16_bits_to_f64(q))
    idx3, _, sc3 = _mask(lib, q2, k, blk_q, blk_k, topk)
    assert np.array_equal(idx0, idx3) and np.array_equal(sc3, 2.0 * sc0)
    # (4) K shifted by one constant vector: each score row shifts by q_I . c
    c = rng.integers(-64, 65, size=d) / 8.0
    kf = synth.bf16_bits_to_f64(k) + c
    k4 = _bits_from_f64(kf)
    assert np.array_equal(synth.bf16_bits_to_f64(k4), kf)
    idx4, _, sc4 = _mask(lib, q, k4, blk_q, blk_k, topk)
    diff = sc4[0] - sc0[0]
    assert np.allclose(diff, diff[:, :1], rtol=0, atol=1e-9 * np.abs(sc4).max())
    assert np.array_equal(idx4[0][ok_rows], idx0[0][ok_rows])


def pin_mask_degenerate(lib):
    q, k, _ = _qkv((2, 8, 8), d=16, seed=4)     # N = 128
    blk = 16
    n_kb = 8
    # all key blocks identical -> lowest indices win every tie
    kk = k.copy()
    for J in range(1, n_kb):
        kk[0, 0, J * blk:(J + 1) * blk] = k[0, 0, :blk]
    for topk in (0.25, 0.5, 0.875):
        idx, _, _ = _mask(lib, q, kk, blk, blk, topk)
        ks = idx.shape[2]
        assert (idx[0] == np.arange(ks)).all()
    # K == 0 -> all scores 0 -> lowest indices
    idx, _, sc = _mask(lib, q, np.zeros_like(k), blk, blk, 0.5)
    assert (sc == 0).all() and (idx[0] == np.arange(4)).all()
    # topk 0 selects nothing, topk 1 everything
    idx, _, _ = _mask(lib, q, k, blk, blk, 0.0)
    assert idx.shape[2] == 0
    idx, _, _ = _mask(lib, q, k, blk, blk, 1.0)
    assert (idx[0] == np.arange(n_kb)).all()


# --------------------------------------------------------------------------
# quantisation
# --------------------------------------------------------------------------

def pin_quant_exact_block(lib):
    # One block of 32 tokens x 16 channels with integer pattern j in [-127, 127]
    # (second half of the rows = minus the first half, so every channel of j has
    # zero mean).  Q = j/16: amax = 127/16, so the scale is exactly 1/16 and every
    # Q code equals j.  K = j/16 + 3: the smoothing mean is exactly 3, the
    # smoothed block is j/16 again, and every K code equals j too.
    d, N = 16, 32
    half = (np.arange(16 * d) % 255 - 127).reshape(16, d)
    j = np.concatenate([half, -half])
    q = _bits_from_f64((j / 16.0)[None])
    kf = j / 16.0 + 3.0
    k = _bits_from_f64(kf[None])
    assert np.array_equal(synth.bf16_bits_to_f64(k[0]), kf)      # exact in bf16
    q8, k8, sq, sk, km = oracle.quantize(q, k, N, N, lib=lib)
    assert sq[0, 0] == np.float32(1 / 16) and sk[0, 0] == np.float32(1 / 16)
    assert (km[0] == np.float32(3.0)).all()
    assert np.array_equal(q8[0].astype(np.int64), j)
    assert np.array_equal(k8[0].astype(np.int64), j)
    # halving the block size: the second block holds -half, same amax, same codes
    q8b, k8b, sqb, skb, _ = oracle.quantize(q, k, 16, 16, lib=lib)
    assert np.array_equal(q8b[0].astype(np.int64), j) and np.array_equal(k8b[0].astype(np.int64), j)
    assert (sqb == np.float32(1 / 16)).all() and (skb == np.float32(1 / 16)).all()


def pin_quant_bounds(lib):
    q, k, _ = _qkv((3, 10, 7), d=128, seed=6, adversarial=("outliers",))   # N = 210, ragged
    for blk_q, blk_k in ((128, 64), (64, 64)):
        q8, k8, sq, sk, km = oracle.quantize(q, k, blk_q, blk_k, lib=lib)
        N = q.shape[2]
        qf = synth.bf16_bits_to_f64(q[0, 0])
        kf = synth.bf16_bits_to_f64(k[0, 0]).astype(np.float32) - km[0].astype(np.float32)
        kf = kf.astype(np.float64)
        for name, x, codes, s, blk in (("q", qf, q8, sq, blk_q), ("k", kf, k8, sk, blk_k)):
            c = codes[0, 0].astype(np.int64)
            assert c.min() >= -127 and c.max() <= 127
            for I in range(-(-N // blk)):
                xb = x[I * blk:(I + 1) * blk]
                cb = c[I * blk:(I + 1) * blk]
                sc = float(s[0, I])
                assert np.abs(cb).max() == 127, (name, I)
                a = np.unravel_index(np.argmax(np.abs(xb)), xb.shape)
                assert abs(cb[a]) == 127 and np.sign(cb[a]) == np.sign(xb[a])
                assert (np.abs(xb - cb * sc) <= 0.5 * sc * (1 + 1e-5)).all(), (name, I)
        # the smoothing mean is the fp64 mean over all N tokens, rounded to fp32
        mu = synth.bf16_bits_to_f64(k[0, 0]).mean(axis=0)
        assert np.array_equal(km[0], mu.astype(np.float32))


def pin_quant_smoothing(lib):
    q, k, _ = _qkv((2, 8, 8), d=32, seed=8)    # N = 128
    q8a, k8a, sqa, ska, kma = oracle.quantize(q, k, 64, 64, lib=lib)
    # zero K block -> scale 0 and zero codes (after the mean is also zero)
    q8z, k8z, _, skz, _ = oracle.quantize(q, np.zeros_like(k), 64, 64, lib=lib)
    assert (skz == 0).all() and (k8z == 0).all()
    # a per-channel shift of K by multiples of 1/8 leaves the smoothed codes
    # equal up to one rounding step
    off = np.round(np.random.default_rng(1).standard_normal(32) * 8) / 8
    kf = synth.bf16_bits_to_f64(k) + off
    k2 = _bits_from_f64(kf)
    exact = np.array_equal(synth.bf16_bits_to_f64(k2), kf)
    _, k8b, _, skb, _ = oracle.quantize(q, k2, 64, 64, lib=lib)
    d = np.abs(k8b.astype(np.int64) - k8a.astype(np.int64))
    if exact:
        assert d.max() <= 1 and (d == 0).mean() > 0.99
        assert np.allclose(skb, ska, rtol=1e-5)
    # Q is not smoothed: shifting Q changes the Q codes but not K's
    q2 = _bits_from_f64(synth.bf16_bits_to_f64(q) + 4.0)
    q8c, k8c, _, _, _ = oracle.quantize(q2, k, 64, 64, lib=lib)
    assert np.array_equal(k8c, k8a) and not np.array_equal(q8c, q8a)


# --------------------------------------------------------------------------
# FP8 e4m3
# --------------------------------------------------------------------------

def _torch_e4m3(x):
    torch = pytest.importorskip("torch")
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.float().numpy(), t.view(torch.uint8).numpy()


def _e4m3_grid():
    """All finite e4m3 values (decoded from every bit pattern but the NaNs)."""
    torch = pytest.importorskip("torch")
    b = torch.arange(256, dtype=torch.uint8)
    v = b.view(torch.float8_e4m3fn).float().numpy()
    return np.unique(v[np.isfinite(v)])


def pin_fp8_encoder(lib):
    rng = np.random.default_rng(21)
    grid = _e4m3_grid()
    pos = grid[grid > 0]
    mids = ((pos[:-1].astype(np.float64) + pos[1:]) / 2).astype(np.float32)  # exact in fp32: ties
    xs = [rng.standard_normal(20000).astype(np.float32) * np.float32(sc) for sc in (1e-4, 3e-3, 0.1, 1, 30, 150)]
    xs += [grid, mids, -mids, np.array([447.9, 448.0, 455.0, 463.99, 0.0, -0.0], dtype=np.float32)]
    x = np.concatenate(xs).astype(np.float32)
    x = x[np.abs(x) < 464]
    val, bits = oracle.e4m3(x, lib=lib)
    tv, tb = _torch_e4m3(x)
    assert np.array_equal(val, tv)
    assert np.array_equal(bits, tb)
    # ties go to the even mantissa: both neighbours of a midpoint are taken, in turn
    mv, _ = oracle.e4m3(mids, lib=lib)
    assert 0.3 < np.mean(mv == pos[1:]) < 0.7
    # saturation (what the conversion to e4m3 with satfinite does)
    big = np.array([464.0, 480.0, 1000.0, 3e38, -464.0, -1e9], dtype=np.float32)
    bv, bb = oracle.e4m3(big, lib=lib)
    assert np.array_equal(bv, np.sign(big) * 448.0)
    assert np.array_equal(bb, np.where(big > 0, 0x7E, 0xFE).astype(np.uint8))


def pin_fp8_quant(lib):
    torch = pytest.importorskip("torch")
    q, k, _ = _qkv((3, 10, 7), d=128, seed=22, adversarial=("outliers",))   # N = 210, ragged
    dec = lambda c: torch.from_numpy(np.ascontiguousarray(c).view(np.uint8)).view(torch.float8_e4m3fn).float().numpy()
    for blk_q, blk_k in ((128, 64), (64, 64)):
        q8, k8, sq, sk, km = oracle.quantize(q, k, blk_q, blk_k, lib=lib, fp8=True)
        _, _, _, _, km_i8 = oracle.quantize(q, k, blk_q, blk_k, lib=lib)
        assert np.array_equal(km, km_i8)                      # same smoothing mean as INT8
        N = q.shape[2]
        qf = synth.bf16_bits_to_f64(q[0, 0]).astype(np.float32)
        kf = synth.bf16_bits_to_f64(k[0, 0]).astype(np.float32) - km[0]
        for name, x, codes, s, blk in (("q", qf, q8, sq, blk_q), ("k", kf, k8, sk, blk_k)):
            c = dec(codes[0, 0]).astype(np.float64)
            assert np.isfinite(c).all() and np.abs(c).max() <= 448
            for I in range(-(-N // blk)):
                xb = x[I * blk:(I + 1) * blk].astype(np.float64)
                cb = c[I * blk:(I + 1) * blk]
                sc = float(s[0, I])
                assert sc == np.float32(np.float32(np.abs(xb).max()) / np.float32(448.0))
                a = np.unravel_index(np.argmax(np.abs(xb)), xb.shape)
                assert abs(cb[a]) == 448 and np.sign(cb[a]) == np.sign(xb[a]), (name, I)
                # within half an e4m3 step: 2^-4 relative for normal codes, 2^-10 absolute below 2^-6
                step = np.where(np.abs(cb) >= 2.0 ** -6, np.abs(cb) * 2.0 ** -3, 2.0 ** -9)
                assert (np.abs(xb / sc - cb) <= 0.5 * step * (1 + 1e-6) + 1e-7).all(), (name, I)


def pin_fp8_forward(lib):
    torch = pytest.importorskip("torch")
    dec = lambda c: torch.from_numpy(np.ascontiguousarray(c).view(np.uint8)).view(torch.float8_e4m3fn).double().numpy()
    q, k, v = _qkv((3, 10, 7), d=64, H=2, seed=23)           # N = 210, ragged
    for blk_q, blk_k, topk, ph in ((64, 64, 1.0, 0), (128, 64, 0.5, 1), (64, 32, 0.3, 0)):
        out, os_, ol = oracle.forward(q, k, v, blk_q, blk_k, topk, phi=ph, quant=2, branches=True, lib=lib)
        idx, _ = oracle.block_mask(q, k, blk_q, blk_k, topk, lib=lib)
        q8, k8, sq, sk, _ = oracle.quantize(q, k, blk_q, blk_k, lib=lib, fp8=True)
        N, d = q.shape[2], q.shape[3]
        for h in range(2):
            rs = np.repeat(sq[h].astype(np.float64), blk_q)[:N]
            cs = np.repeat(sk[h].astype(np.float64), blk_k)[:N]
            lg = (dec(q8[0, h]) @ dec(k8[0, h]).T) * rs[:, None] * cs[None, :] / np.sqrt(d)
            ref, rs_, rl = sla_dense(q[0, h], k[0, h], v[0, h], idx[h], blk_q, blk_k, ph, logits=lg)
            for a, b in ((out[0, h], ref), (os_[0, h], rs_), (ol[0, h], rl)):
                err = np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)
                assert err < 1e-10, (blk_q, topk, h, err)
            if topk == 1.0:  # all selected: softmax attention on the decoded codes
                P = torch.softmax(torch.from_numpy(lg), dim=-1).numpy()
                dense = P @ synth.bf16_bits_to_f64(v[0, h])
                assert np.abs(out[0, h] - dense).max() / np.abs(dense).max() < 1e-12


# --------------------------------------------------------------------------
# W8A8 INT8 linear with FusedNorm
# --------------------------------------------------------------------------

def _w8a8_inputs(seed, rows, cols, tiny_rows=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * rng.uniform(0.2, 3.0, size=(rows, 1))
    if tiny_rows:  # RMS ~ 1e-3: eps = 1e-6 is no longer negligible against the mean square
        x[:tiny_rows] *= 1e-3
    x[rows // 2] = 0.0  # an all-zero row
    return _bits_from_f64(x)


def pin_w8a8_rowquant(lib):
    torch = pytest.importorskip("torch")
    rows, cols = 24, 96
    x = _w8a8_inputs(31, rows, cols, tiny_rows=4)
    xf = synth.bf16_bits_to_f64(x)
    gamma = np.random.default_rng(32).uniform(0.5, 1.5, cols).astype(np.float32)
    for norm, g in ((False, None), (True, None), (True, gamma)):
        q, s = oracle.rowquant(x, norm=norm, gamma=g, eps=1e-6, lib=lib)
        c = q.astype(np.int64)
        assert c.min() >= -127 and c.max() <= 127
        if norm:
            y = torch.nn.functional.rms_norm(torch.from_numpy(xf.astype(np.float32)), (cols,),
                                             weight=None if g is None else torch.from_numpy(g), eps=1e-6)
            y = y.double().numpy()
        else:
            y = xf
        for m in range(rows):
            if not np.any(xf[m]):
                assert s[m] == 0 and not np.any(c[m])
                continue
            a = np.argmax(np.abs(y[m]))
            assert abs(c[m, a]) == 127 and np.sign(c[m, a]) == np.sign(y[m, a]), (norm, m)
            tol = 0.5 * float(s[m]) * (1 + 1e-5) + 2e-6 * np.abs(y[m]).max()
            assert (np.abs(y[m] - c[m] * float(s[m])) <= tol).all(), (norm, m)


def pin_w8a8_linear(lib):
    M, N, K = 20, 12, 96
    x = _w8a8_inputs(33, M, K)
    w = _w8a8_inputs(34, N, K)
    bias = np.random.default_rng(35).standard_normal(N).astype(np.float32)
    qx, sx = oracle.rowquant(x, lib=lib)
    qw, sw = oracle.rowquant(w, lib=lib)
    out = oracle.w8a8_linear(qx, sx, qw, sw, bias, lib=lib)
    ref = (qx.astype(np.int64) @ qw.astype(np.int64).T).astype(np.float64) * sx.astype(np.float64)[:, None] \
        * sw.astype(np.float64)[None, :] + bias.astype(np.float64)[None, :]
    assert np.allclose(out, ref, rtol=1e-14, atol=1e-14)
    # the decoded product against the fp64 product, within the quantisation error bound
    xf, wf = synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(w)
    exact = xf @ wf.T + bias.astype(np.float64)[None, :]
    dx, dw = 0.5 * sx.astype(np.float64)[:, None], 0.5 * sw.astype(np.float64)[:, None]
    bound = (np.abs(xf).sum(1)[:, None] * dw.T + dx * np.abs(wf).sum(1)[None, :] + K * dx * dw.T) * (1 + 1e-6)
    assert (np.abs(out - exact) <= bound + 1e-12).all()
    assert not np.allclose(oracle.w8a8_linear(qx, sx, qw, sw, None, lib=lib), out)


# --------------------------------------------------------------------------
# forward
# --------------------------------------------------------------------------

def pin_forward_dense_limit(lib):
    torch = pytest.importorskip("torch")
    q, k, v = _qkv((3, 10, 7), d=64, H=2, seed=9)          # N = 210, ragged blocks
    out = oracle.forward(q, k, v, 64, 64, 1.0, phi=0, quant=0, lib=lib)
    qt = torch.from_numpy(synth.bf16_bits_to_f64(q))
    kt = torch.from_numpy(synth.bf16_bits_to_f64(k))
    vt = torch.from_numpy(synth.bf16_bits_to_f64(v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).numpy()
    err = np.abs(out - ref).max() / np.abs(ref).max()
    assert err < 1e-12, err


def pin_forward_linear_limit(lib):
    q, k, v = _qkv((3, 10, 7), d=64, H=2, seed=10)
    for ph in (0, 1):
        out = oracle.forward(q, k, v, 128, 64, 0.0, phi=ph, quant=1, lib=lib)
        for h in range(2):
            Q = bf_phi(synth.bf16_bits_to_f64(q[0, h]), ph)
            K = bf_phi(synth.bf16_bits_to_f64(k[0, h]), ph)
            V = synth.bf16_bits_to_f64(v[0, h])
            num = Q @ (K.T @ V)
            den = Q @ K.sum(axis=0)
            ref = np.where(den[:, None] != 0, num / np.where(den != 0, den, 1)[:, None], 0.0)
            err = np.abs(out[0, h] - ref).max() / np.abs(ref).max()
            assert err < 1e-12, (ph, h, err)


def pin_forward_bruteforce(lib):
    for (grid, d, blk_q, blk_k, topk, ph, quant, seed) in (
        ((3, 10, 7), 64, 64, 64, 0.34, 0, 0, 12),       # N=210: 4 x 4 blocks, ragged
        ((3, 10, 7), 64, 128, 64, 0.5, 1, 1, 13),
        ((2, 9, 9), 32, 32, 16, 0.2, 0, 1, 14),         # N=162: 6 q-blocks, 11 k-blocks
        ((2, 9, 9), 32, 32, 16, 0.7, 1, 0, 15),
    ):
        q, k, v = _qkv(grid, d=d, H=2, seed=seed)
        out, os_, ol = oracle.forward(q, k, v, blk_q, blk_k, topk, phi=ph, quant=quant,
                                      branches=True, lib=lib)
        idx, _ = oracle.block_mask(q, k, blk_q, blk_k, topk, lib=lib)
        if quant:
            q8, k8, sq, sk, _ = oracle.quantize(q, k, blk_q, blk_k, lib=lib)
        for h in range(2):
            lg = quant_logits(q8[0, h], k8[0, h], sq[h], sk[h], blk_q, blk_k) if quant else None
            ref, rs, rl = sla_dense(q[0, h], k[0, h], v[0, h], idx[h], blk_q, blk_k, ph, logits=lg)
            for a, b in ((out[0, h], ref), (os_[0, h], rs), (ol[0, h], rl)):
                err = np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)
                assert err < 1e-10, (grid, topk, ph, quant, h, err)


def pin_forward_constant_v(lib):
    q, k, _ = _qkv((2, 8, 8), d=32, H=1, seed=16)          # N = 128
    c = np.linspace(-1.5, 2.0, 32)
    v = _bits_from_f64(np.broadcast_to(c, (1, 1, 128, 32)))
    cv = synth.bf16_bits_to_f64(v[0, 0, 0])
    for topk, factor in ((0.0, 1.0), (0.25, 2.0), (0.5, 2.0), (1.0, 1.0)):
        for quant in (0, 1):
            out = oracle.forward(q, k, v, 32, 16, topk, phi=0, quant=quant, lib=lib)
            assert np.allclose(out[0, 0], factor * cv, rtol=0, atol=1e-12), (topk, quant)


def pin_forward_hull(lib):
    q, k, v = _qkv((3, 10, 7), d=64, H=1, seed=17, adversarial=("outliers",))
    V = synth.bf16_bits_to_f64(v[0, 0])
    lo, hi = V.min(axis=0), V.max(axis=0)
    for ph in (0, 1):
        out, os_, ol = oracle.forward(q, k, v, 64, 64, 0.25, phi=ph, quant=1, branches=True, lib=lib)
        for part in (os_[0, 0], ol[0, 0]):
            nz = np.any(part != 0, axis=1)
            assert (part[nz] >= lo - 1e-12).all() and (part[nz] <= hi + 1e-12).all()
        assert (np.abs(out) <= 2 * np.abs(V).max() + 1e-12).all()


def pin_forward_relu_zero(lib):
    q, k, v = _qkv((2, 8, 8), d=32, H=1, seed=18)
    qf = synth.bf16_bits_to_f64(q)
    qf[0, 0, 5] = -np.abs(qf[0, 0, 5]) - 0.5     # row 5: every channel negative
    q2 = _bits_from_f64(qf)
    out, os_, ol = oracle.forward(q2, k, v, 32, 16, 0.25, phi=1, quant=0, branches=True, lib=lib)
    assert (ol[0, 0, 5] == 0).all() and np.any(ol[0, 0, 4] != 0)


def pin_forward_rows(lib):
    q, k, v = _qkv((3, 10, 7), d=32, H=3, seed=19)
    full = oracle.forward(q, k, v, 64, 32, 0.3, phi=0, quant=1, lib=lib)
    rows = np.array([[2, 209], [0, 0], [1, 64], [2, 3], [0, 150], [1, 65]], dtype=np.int64)
    part = oracle.forward(q, k, v, 64, 32, 0.3, phi=0, quant=1, rows=rows, lib=lib)
    BH = full.reshape(-1, 210, 32)
    for r, (bh, i) in enumerate(rows):
        assert np.array_equal(part[r], BH[bh, i])


# --------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------

def _torch_phi(x, ph):
    torch = pytest.importorskip("torch")
    if ph == 1:
        return torch.relu(x)
    return torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))


def _torch_sla(qt, kt, vt, allowed, ph):
    """Attention-form statement of the unquantised forward of one head, for
    autograd: ``allowed[i, j]`` marks the tokens of the key blocks that row i's
    query block selected; the linear branch weighs the other tokens by
    phi(q_i).phi(k_j)."""
    torch = pytest.importorskip("torch")
    d = qt.shape[-1]
    any_row = allowed.any(dim=-1, keepdim=True)
    s = (qt @ kt.T) / math.sqrt(d)
    s = torch.where(any_row, s.masked_fill(~allowed, float("-inf")), torch.zeros_like(s))
    p = torch.where(any_row, torch.softmax(s, dim=-1), torch.zeros_like(s))
    w = (_torch_phi(qt, ph) @ _torch_phi(kt, ph).T) * (~allowed)
    den = w.sum(dim=-1, keepdim=True)
    ol = torch.where(den != 0, (w @ vt) / torch.where(den != 0, den, torch.ones_like(den)), torch.zeros_like(qt))
    return p @ vt + ol


def _grads(fn, q, k, v, dout):
    """float64 autograd of sum(fn(q, k, v) * dout) for bf16-bit inputs of one head."""
    torch = pytest.importorskip("torch")
    ts = [torch.from_numpy(synth.bf16_bits_to_f64(x)).requires_grad_(True) for x in (q, k, v)]
    out = fn(*ts)
    (out * torch.from_numpy(synth.bf16_bits_to_f64(dout))).sum().backward()
    return out.detach().numpy(), [t.grad.numpy() for t in ts]


def _rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


def pin_backward_autograd(lib):
    torch = pytest.importorskip("torch")
    blk_q, blk_k = 32, 16
    for (topk, ph, seed) in ((0.3, 0, 30), (0.6, 0, 31), (0.3, 1, 32), (0.0, 0, 33), (1.0, 1, 34)):
        q, k, v = _qkv((3, 5, 7), d=32, H=2, seed=seed)          # N = 105: 4 x 7 ragged blocks
        dout = _qkv((3, 5, 7), d=32, H=2, seed=seed + 100)[0]
        if ph == 1:  # a row whose phi(q) is zero: zero linear denominator
            qf = synth.bf16_bits_to_f64(q)
            qf[0, 1, 40] = -np.abs(qf[0, 1, 40]) - 0.25
            q = _bits_from_f64(qf)
        N = q.shape[2]
        idx, _ = oracle.block_mask(q, k, blk_q, blk_k, topk, lib=lib)
        out_o = oracle.forward(q, k, v, blk_q, blk_k, topk, phi=ph, quant=0, lib=lib)
        dq, dk, dv = oracle.backward(q, k, v, dout, blk_q, blk_k, topk, phi=ph, lib=lib)
        n_qb, n_kb = -(-N // blk_q), -(-N // blk_k)
        for h in range(2):
            sel = np.zeros((n_qb, n_kb), dtype=bool)
            for I in range(n_qb):
                sel[I, idx[h, I]] = True
            tok = np.arange(N)
            allowed = torch.from_numpy(sel[(tok // blk_q)[:, None], (tok // blk_k)[None, :]])
            out_t, (gq, gk, gv) = _grads(lambda a, b, c: _torch_sla(a, b, c, allowed, ph),
                                         q[0, h], k[0, h], v[0, h], dout[0, h])
            assert _rel(out_o[0, h], out_t) < 1e-12, (topk, ph, h, "forward statement")
            for name, mine, ref in (("dq", dq, gq), ("dk", dk, gk), ("dv", dv, gv)):
                assert _rel(mine[0, h], ref) < 1e-10, (topk, ph, h, name, _rel(mine[0, h], ref))


def pin_backward_dense_limit(lib):
    torch = pytest.importorskip("torch")
    q, k, v = _qkv((3, 10, 7), d=64, H=1, seed=40)          # N = 210, ragged blocks
    dout = _qkv((3, 10, 7), d=64, H=1, seed=41)[0]
    dq, dk, dv = oracle.backward(q, k, v, dout, 64, 64, 1.0, phi=0, lib=lib)
    _, ref = _grads(lambda a, b, c: torch.nn.functional.scaled_dot_product_attention(a[None], b[None], c[None])[0],
                    q[0, 0], k[0, 0], v[0, 0], dout[0, 0])
    for mine, r in zip((dq, dk, dv), ref):
        assert _rel(mine[0, 0], r) < 1e-12, _rel(mine[0, 0], r)


def pin_backward_linear_limit(lib):
    q, k, v = _qkv((3, 10, 7), d=32, H=1, seed=42)
    dout = _qkv((3, 10, 7), d=32, H=1, seed=43)[0]
    for ph in (0, 1):
        dq, dk, dv = oracle.backward(q, k, v, dout, 128, 64, 0.0, phi=ph, lib=lib)

        def lin(a, b, c):
            fq, fk = _torch_phi(a, ph), _torch_phi(b, ph)
            return (fq @ (fk.T @ c)) / (fq @ fk.sum(dim=0))[:, None]

        _, ref = _grads(lin, q[0, 0], k[0, 0], v[0, 0], dout[0, 0])
        for mine, r in zip((dq, dk, dv), ref):
            assert _rel(mine[0, 0], r) < 1e-11, (ph, _rel(mine[0, 0], r))


def pin_backward_rows(lib):
    """The row-sampled dq equals the full backward's dq, row for row."""
    q, k, v = _qkv((3, 10, 7), d=32, H=3, seed=44)
    dout = _qkv((3, 10, 7), d=32, H=3, seed=45)[0]
    for ph, topk, bq in ((0, 0.3, 64), (1, 0.7, 32)):
        dq, _, _ = oracle.backward(q, k, v, dout, bq, 32, topk, phi=ph, lib=lib)
        rows = np.array([[2, 209], [0, 0], [1, 64], [2, 3], [0, 150], [1, 65]], dtype=np.int64)
        part = oracle.backward_dq_rows(q, k, v, dout, bq, 32, topk, rows, phi=ph, lib=lib)
        full = dq.reshape(-1, 210, 32)
        for r, (bh, i) in enumerate(rows):
            assert np.array_equal(part[r], full[bh, i]), (ph, topk, bh, i)


def pin_backward_key_blocks(lib):
    """The key-block-sampled dk, dv equal the full backward's rows of those key blocks, bit for bit:
    subtract and complement selections, both phi, a ragged last key block (N = 210, blk_k = 32: 18 rows),
    blocks of several heads given out of order, and topk 0 (linear only) and 1 (softmax only)."""
    q, k, v = _qkv((3, 10, 7), d=32, H=3, seed=46)
    dout = _qkv((3, 10, 7), d=32, H=3, seed=47)[0]
    for ph, topk, bq in ((0, 0.3, 64), (1, 0.7, 32), (0, 0.0, 64), (1, 1.0, 32)):
        _, dk, dv = oracle.backward(q, k, v, dout, bq, 32, topk, phi=ph, lib=lib)
        blocks = np.array([[2, 6], [0, 0], [1, 3], [0, 5], [2, 0]], dtype=np.int64)
        pk, pv = oracle.backward_dkdv_blocks(q, k, v, dout, bq, 32, topk, blocks, phi=ph, lib=lib)
        fk, fv = dk.reshape(-1, 210, 32), dv.reshape(-1, 210, 32)
        for b, (bh, J) in enumerate(blocks):
            n = min(32, 210 - 32 * J)
            assert np.array_equal(pk[b, :n], fk[bh, 32 * J:32 * J + n]), (ph, topk, bh, J)
            assert np.array_equal(pv[b, :n], fv[bh, 32 * J:32 * J + n]), (ph, topk, bh, J)
            assert not pk[b, n:].any() and not pv[b, n:].any()


PINS = [pin_topk_count, pin_mask_exhaustive, pin_mask_invariances, pin_mask_degenerate,
        pin_quant_exact_block, pin_quant_bounds, pin_quant_smoothing, pin_forward_dense_limit,
        pin_forward_linear_limit, pin_forward_bruteforce, pin_forward_constant_v, pin_forward_hull,
        pin_forward_relu_zero, pin_forward_rows, pin_fp8_encoder, pin_fp8_quant, pin_fp8_forward, pin_w8a8_rowquant, pin_w8a8_linear,
        pin_backward_autograd, pin_backward_dense_limit, pin_backward_linear_limit, pin_backward_rows,
        pin_backward_key_blocks]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle.load())

"""GPU parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

* block mask: bit-exact (index lists and bitmaps); near-ties (relative score
  gap < 1e-5) would be exempt but none are expected since both sides evaluate
  the same fp64 definition;
* INT8 quantisation: codes, scales and the smoothing mean bit-exact;
* forward: cosine >= 0.999 and relative L2 <= 2e-2 with quantisation on,
  relative L2 <= 2e-3 with it off, over small workloads that span several
  tiles with ragged tails, phi in {elu+1, relu}, topk in {0, 0.1, ..., 1}
  (the workloads at their full sizes are in test_gpu_configs.py);
* determinism: two calls give identical bytes.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_to_f64, cosine, mask_mismatches, rel_l2, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_linear_bit_b200 as sla  # noqa: E402

QUANT_TOL = dict(cos=0.999, rel=2e-2)
FP_TOL = dict(rel=2e-3)


def f32(x):
    return float(np.float32(x))


def run_forward(q, k, v, blk_q, blk_k, topk, phi, quant):
    B, H, N, d = q.shape
    qd, kd, vd = to_dev(q, torch), to_dev(k, torch), to_dev(v, torch)
    out = torch.empty_like(qd)
    ws = sla.workspace(B, H, N, d, blk_q, blk_k, topk, quant)
    sla.sla_forward(qd, kd, vd, out, blk_q, blk_k, topk, phi, quant, ws)
    sla.sla_check(ws)
    return out, ws


MASK_CASES = {
    "tiny_64x64": ((1, 2, (8, 16, 16)), 64, 64, 0.1, ()),
    "ragged_210": ((1, 3, (3, 10, 7)), 128, 64, 0.3, ()),
    "ragged_q64": ((2, 2, (5, 9, 13)), 64, 64, 0.2, ()),
    "wan_480p_2heads": ((1, 2, (21, 30, 52)), 128, 64, 0.1, ()),
    "ties_sweep": ((1, 3, (16, 32, 32)), 128, 64, 0.1, ("ties",)),
    "outliers_topk0": ((2, 2, (16, 16, 16)), 128, 64, 0.0, ("outliers",)),
    "topk1": ((1, 2, (8, 16, 16)), 128, 64, 1.0, ()),
    "topk_half": ((1, 2, (8, 16, 16)), 128, 64, 0.5, ()),
    "block_topk_1313": ((1, 1, (21, 40, 100)), 128, 64, 0.1, ()),
}


@pytest.mark.parametrize("name", sorted(MASK_CASES))
def test_block_mask_bit_exact(name):
    (B, H, grid), blk_q, blk_k, topk, adv = MASK_CASES[name]
    q, k, _ = synth.make_qkv(B, H, grid, seed=100 + len(name), adversarial=adv)
    N = q.shape[2]
    n_qb, n_kb = -(-N // blk_q), -(-N // blk_k)
    ks = sla.sla_topk_count(n_kb, topk)
    assert ks == oracle.topk_count(n_kb, f32(topk))
    idx_o, bm_o, sc = oracle.block_mask(q, k, blk_q, blk_k, f32(topk), with_scores=True)
    qd, kd = to_dev(q, torch), to_dev(k, torch)
    idx = torch.full((B, H, n_qb, max(ks, 1)), -1, dtype=torch.int32, device="cuda")
    bm = torch.full((B, H, n_qb, -(-n_kb // 32)), 0xFFFF, dtype=torch.int32, device="cuda")
    ws = sla.workspace(B, H, N, 128, blk_q, blk_k, topk, 0)
    sla.sla_block_mask(qd, kd, blk_q, blk_k, topk, idx if ks > 0 else None, bm, ws)
    sla.sla_check(ws)
    idx_g = idx.cpu().numpy().reshape(B * H, n_qb, -1)[..., :ks]
    bm_g = bm.cpu().numpy().view(np.uint32).reshape(B * H, n_qb, -1)
    assert np.array_equal(bm_g, bm_o), "bitmap differs"
    if ks > 0:
        assert (np.diff(idx_g, axis=-1) > 0).all(), "index lists must be strictly ascending"
        exempt, real = mask_mismatches(idx_g, idx_o, sc)
        assert not real, f"{len(real)} rows differ beyond near-ties"
        assert np.array_equal(idx_g, idx_o), f"near-tie rows differ: {len(exempt)}"


@pytest.mark.parametrize("blk_q", [64, 128])
@pytest.mark.parametrize("grid,H,adv", [((3, 10, 7), 3, ()), ((16, 16, 16), 2, ("outliers",)),
                                        ((21, 30, 52), 1, ())])
def test_quantize_bit_exact(blk_q, grid, H, adv):
    q, k, _ = synth.make_qkv(1, H, grid, seed=7, adversarial=adv)
    B, _, N, d = q.shape
    n_qb, n_kb = -(-N // blk_q), -(-N // 64)
    q8o, k8o, sqo, sko, kmo = oracle.quantize(q, k, blk_q, 64)
    qd, kd = to_dev(q, torch), to_dev(k, torch)
    q8 = torch.empty(q.shape, dtype=torch.int8, device="cuda")
    k8 = torch.empty(q.shape, dtype=torch.int8, device="cuda")
    sq = torch.empty((B, H, n_qb), dtype=torch.float32, device="cuda")
    sk = torch.empty((B, H, n_kb), dtype=torch.float32, device="cuda")
    km = torch.empty((B, H, d), dtype=torch.float32, device="cuda")
    ws = sla.workspace(B, H, N, d, blk_q, 64, 0.0, 1)
    sla.sla_quantize_qk(qd, kd, blk_q, 64, q8, k8, sq, sk, km, ws)
    sla.sla_check(ws)
    assert np.array_equal(km.cpu().numpy().reshape(B * H, d), kmo)
    assert np.array_equal(sq.cpu().numpy().reshape(B * H, -1), sqo)
    assert np.array_equal(sk.cpu().numpy().reshape(B * H, -1), sko)
    assert np.array_equal(q8.cpu().numpy(), q8o)
    assert np.array_equal(k8.cpu().numpy(), k8o)


@pytest.mark.parametrize("N", [2048, 1000])
def test_quantize_half_integer_quotients(N):
    """Every quotient x/s an exact half-integer (s = 1): codes must round half to even, like
    the IEEE fp32 quotient followed by rint in the oracle.  K is built from +-pairs per channel
    so that its smoothing mean is exactly 0 and K - mean keeps the half-integers."""
    rng = np.random.default_rng(11)
    B, H, d = 1, 2, 128
    qv = rng.integers(-254, 255, size=(B, H, N, d)) / 2.0
    qv[:, :, ::64, 0] = 127.0  # every block of 64 or 128 rows reaches amax = 127, so s = 1
    half = rng.integers(-254, 255, size=(B, H, N // 2, d)) / 2.0
    half[:, :, ::32, 1] = 127.0
    kv = np.empty((B, H, N, d))
    kv[:, :, 0::2] = half
    kv[:, :, 1::2] = -half
    q = synth.f64_to_bf16_bits(qv)
    k = synth.f64_to_bf16_bits(kv)
    for blk_q in (64, 128):
        n_qb, n_kb = -(-N // blk_q), -(-N // 64)
        q8o, k8o, sqo, sko, kmo = oracle.quantize(q, k, blk_q, 64)
        assert np.all(kmo == 0.0) and np.all(sqo == 1.0) and np.all(sko == 1.0)
        qd, kd = to_dev(q, torch), to_dev(k, torch)
        q8 = torch.empty(q.shape, dtype=torch.int8, device="cuda")
        k8 = torch.empty(q.shape, dtype=torch.int8, device="cuda")
        sq = torch.empty((B, H, n_qb), dtype=torch.float32, device="cuda")
        sk = torch.empty((B, H, n_kb), dtype=torch.float32, device="cuda")
        ws = sla.workspace(B, H, N, d, blk_q, 64, 0.0, 1)
        sla.sla_quantize_qk(qd, kd, blk_q, 64, q8, k8, sq, sk, None, ws)
        sla.sla_check(ws)
        assert np.array_equal(q8.cpu().numpy(), q8o)
        assert np.array_equal(k8.cpu().numpy(), k8o)
        # the half-integers really were rounded half to even
        assert np.array_equal(q8o.astype(np.float64), np.clip(np.round(qv), -127, 127))


FWD_CASES = {
    # name: ((B, H, grid), blk_q, topk, phi, quant)
    "tiny_quant_elu": ((1, 2, (8, 16, 16)), 64, 0.1, 0, 1),
    "tiny_fp_elu": ((1, 2, (8, 16, 16)), 64, 0.1, 0, 0),
    "tiny_quant_relu": ((1, 2, (8, 16, 16)), 64, 0.1, 1, 1),
    "tiny_fp_relu": ((1, 2, (8, 16, 16)), 64, 0.1, 1, 0),
    "ragged_quant": ((1, 3, (3, 10, 7)), 128, 0.34, 0, 1),
    "ragged_fp": ((2, 2, (5, 9, 13)), 128, 0.2, 1, 0),
    "ragged_q64_quant": ((2, 2, (5, 9, 13)), 64, 0.25, 0, 1),
    "multi_tile_quant": ((1, 2, (8, 32, 32)), 128, 0.1, 0, 1),
    "multi_tile_fp": ((1, 2, (8, 32, 32)), 128, 0.1, 0, 0),
    "topk0_quant": ((1, 2, (8, 16, 16)), 128, 0.0, 0, 1),
    "topk0_fp_relu": ((1, 2, (8, 16, 16)), 128, 0.0, 1, 0),
    "topk1_quant": ((1, 2, (8, 16, 16)), 128, 1.0, 0, 1),
    "topk1_fp": ((1, 2, (8, 16, 16)), 128, 1.0, 0, 0),
    "topk_0p6_fp": ((1, 2, (8, 16, 16)), 128, 0.6, 0, 0),
    "ties_quant": ((1, 3, (8, 16, 16)), 128, 0.1, 0, 1),
    # FP8 e4m3 Q.K^T (quant = 2), against the FP8 oracle
    "tiny_fp8_elu": ((1, 2, (8, 16, 16)), 64, 0.1, 0, 2),
    "ragged_fp8_relu": ((2, 2, (5, 9, 13)), 128, 0.2, 1, 2),
    "multi_tile_fp8": ((1, 2, (8, 32, 32)), 128, 0.1, 0, 2),
    "topk1_fp8": ((1, 2, (8, 16, 16)), 128, 1.0, 0, 2),
}


@pytest.mark.parametrize("blk_q,grid,H,adv", [
    (128, (8, 16, 16), 2, ()),
    (64, (3, 10, 7), 3, ("outliers",)),     # ragged N = 210, heavy-tailed K channels
    (128, (5, 9, 13), 2, ("ties",)),
])
def test_quantize_fp8_bit_exact(blk_q, grid, H, adv):
    q, k, _ = synth.make_qkv(1, H, grid, seed=17, adversarial=adv)
    B, _, N, d = q.shape
    n_qb, n_kb = -(-N // blk_q), -(-N // 64)
    q8o, k8o, sqo, sko, kmo = oracle.quantize(q, k, blk_q, 64, fp8=True)
    qd, kd = to_dev(q, torch), to_dev(k, torch)
    q8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    k8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    sq = torch.empty((B, H, n_qb), dtype=torch.float32, device="cuda")
    sk = torch.empty((B, H, n_kb), dtype=torch.float32, device="cuda")
    km = torch.empty((B, H, d), dtype=torch.float32, device="cuda")
    ws = sla.workspace(B, H, N, d, blk_q, 64, 0.0, 2)
    sla.sla_quantize_qk_fp8(qd, kd, blk_q, 64, q8, k8, sq, sk, km, ws)
    sla.sla_check(ws)
    assert np.array_equal(km.cpu().numpy().reshape(B * H, d), kmo)
    assert np.array_equal(sq.cpu().numpy().reshape(B * H, -1), sqo)
    assert np.array_equal(sk.cpu().numpy().reshape(B * H, -1), sko)
    assert np.array_equal(q8.cpu().numpy(), q8o.view(np.uint8))
    assert np.array_equal(k8.cpu().numpy(), k8o.view(np.uint8))


@pytest.mark.parametrize("name", sorted(FWD_CASES))
def test_forward_parity(name):
    (B, H, grid), blk_q, topk, phi, quant = FWD_CASES[name]
    adv = ("ties",) if name.startswith("ties") else ()
    q, k, v = synth.make_qkv(B, H, grid, seed=200 + len(name), adversarial=adv)
    out, _ = run_forward(q, k, v, blk_q, 64, topk, phi, quant)
    got = bf16_to_f64(out)
    ref = oracle.forward(q, k, v, blk_q, 64, f32(topk), phi=phi, quant=quant)
    r, c = rel_l2(got, ref), cosine(got, ref)
    if quant:
        assert r <= QUANT_TOL["rel"] and c >= QUANT_TOL["cos"], (name, r, c)
    else:
        assert r <= FP_TOL["rel"], (name, r, c)
    # every row separately stays close (no single row may hide behind the average)
    rows = np.linalg.norm((got - ref).reshape(-1, 128), axis=1) / np.maximum(
        np.linalg.norm(ref.reshape(-1, 128), axis=1), 1e-30)
    assert np.percentile(rows, 99.9) < (0.1 if quant else 0.02), (name, rows.max())


def test_forward_deterministic():
    q, k, v = synth.make_qkv(1, 2, (8, 32, 32), seed=9)
    a, _ = run_forward(q, k, v, 128, 64, 0.1, 0, 1)
    b, _ = run_forward(q, k, v, 128, 64, 0.1, 0, 1)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


LINEAR_CASES = {
    # name: (grid, topk): subtract mode (H_total - selected), complement mode, several
    # query-block tiles and key-block steps with ragged tails
    "ragged_subtract": ((3, 10, 7), 0.3),
    "ragged_complement": ((3, 10, 7), 0.7),
    "multi_tile_subtract": ((16, 32, 36), 0.1),
}


@pytest.mark.parametrize("name", sorted(LINEAR_CASES))
def test_linear_states_match_oracle(name):
    """Intermediate check: per-key-block states and per-query-block states."""
    grid, topk = LINEAR_CASES[name]
    q, k, v = synth.make_qkv(1, 1, grid, seed=11 + len(name))
    N = q.shape[2]
    out, ws = run_forward(q, k, v, 128, 64, topk, 0, 1)
    lay = sla.sla_workspace_layout(1, 1, N, 128, 128, 64, topk, 1)
    n_kb, n_qb = -(-N // 64), -(-N // 128)
    wsn = ws.cpu().numpy()
    st = wsn[lay["states"]:lay["states"] + n_kb * 16512 * 2].view(np.uint16).reshape(n_kb, 16512)
    st = synth.bf16_bits_to_f64(st)
    h, z = oracle.states(k[0, 0], v[0, 0], 64, 0)
    hT = np.transpose(h, (0, 2, 1)).reshape(n_kb, -1)
    assert rel_l2(st[:, :16384], hT) < 5e-3
    assert rel_l2(st[:, 16384:], z) < 5e-3
    hq = wsn[lay["hq"]:lay["hq"] + n_qb * 16512 * 4].view(np.float32).reshape(n_qb, 16512).astype(np.float64)
    _, bm = oracle.block_mask(q, k, 128, 64, f32(topk))
    sel = np.unpackbits(bm[0].view(np.uint8), axis=-1, bitorder="little")[:, :n_kb].astype(np.float64)
    HI = (1.0 - sel) @ hT  # unselected key blocks of each query block
    ZI = (1.0 - sel) @ z
    for I in range(n_qb):
        assert rel_l2(hq[I, :16384], HI[I]) < 5e-3, I
        assert rel_l2(hq[I, 16384:], ZI[I]) < 5e-3, I


REDUCE_MASK_CASES = {
    # name: ((B, H, grid), blk_q, topk); n_kb = 1313 takes the block-wide top-k kernel
    "ragged_subtract": ((1, 2, (3, 10, 7)), 128, 0.3),
    "ragged_complement": ((1, 2, (3, 10, 7)), 64, 0.7),
    "multi_step": ((1, 1, (16, 32, 36)), 128, 0.1),
    "block_topk_1313": ((1, 1, (21, 40, 100)), 128, 0.1),
    "block_topk_1313_complement": ((1, 1, (21, 40, 100)), 128, 0.6),
}


@pytest.mark.parametrize("name", sorted(REDUCE_MASK_CASES))
def test_state_reduction_mask_bits(name):
    """The state-reduction mask rows in the workspace, bit-exact: bit J of row I is set for the
    selected key blocks when at most half of them are selected, else for the unselected ones;
    the bits past n_kb (to a whole 64-block step) are zero."""
    (B, H, grid), blk_q, topk = REDUCE_MASK_CASES[name]
    q, k, v = synth.make_qkv(B, H, grid, seed=300 + len(name))
    N = q.shape[2]
    n_qb, n_kb = -(-N // blk_q), -(-N // 64)
    n_aw = 2 * (-(-n_kb // 64))
    _, ws = run_forward(q, k, v, blk_q, 64, topk, 0, 1)
    lay = sla.sla_workspace_layout(B, H, N, 128, blk_q, 64, topk, 1)
    raw = ws[lay["amask"]:lay["amask"] + B * H * n_qb * n_aw * 4].cpu().numpy()
    bits = np.unpackbits(raw, bitorder="little").reshape(B * H, n_qb, 32 * n_aw)
    _, bm = oracle.block_mask(q, k, blk_q, 64, f32(topk))
    sel = np.unpackbits(np.ascontiguousarray(bm).view(np.uint8), axis=-1, bitorder="little")[..., :n_kb]
    ks = oracle.topk_count(n_kb, f32(topk))
    expect = sel if 2 * ks <= n_kb else 1 - sel
    assert np.array_equal(bits[..., :n_kb], expect)
    assert not bits[..., n_kb:].any()

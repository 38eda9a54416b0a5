"""W8A8 INT8 linear layer with FusedNorm on the GPU against the fp64 oracle.

Codes and scales of the per-row quantisation (with and without the RMS
normalisation) are compared bit for bit; the GEMM output (bf16) element by element
against the oracle's fp64 result of the same codes, within the bf16 rounding of
the output plus the fp32 dequantisation.
"""
from __future__ import annotations

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import sparse_linear_bit_b200 as sla  # noqa: E402
import synth  # noqa: E402


def _bf16(x):
    return synth.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def _dev_bits(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()


def _rows(seed, rows, cols, tiny=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * rng.uniform(0.1, 4.0, size=(rows, 1))
    x[:, : cols // 16] *= 8.0  # a few outlier channels
    if tiny:
        x[:tiny] *= 1e-3
    x[rows // 3] = 0.0
    return _bf16(x)


def _gpu_quant(xb, norm, gamma, eps=1e-6):
    rows, cols = xb.shape
    xd = _dev_bits(xb)
    q = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    g = None if gamma is None else torch.from_numpy(gamma).cuda()
    sla.sla_w8a8_quantize(xd, q, s, norm=norm, gamma=g, eps=eps)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("rows,cols,norm,with_gamma,tiny", [
    (37, 256, False, False, 0),
    (130, 1024, True, True, 5),
    (9, 5120, True, False, 2),
    (64, 16384, True, True, 0),     # the largest supported row
])
def test_rowquant_bit_exact(rows, cols, norm, with_gamma, tiny):
    xb = _rows(40 + rows, rows, cols, tiny)
    gamma = np.random.default_rng(7).uniform(0.5, 1.5, cols).astype(np.float32) if with_gamma else None
    qo, so = oracle.rowquant(xb, norm=norm, gamma=gamma, eps=1e-6)
    q, s = _gpu_quant(xb, norm, gamma)
    assert np.array_equal(s, so)
    assert np.array_equal(q, qo)


@pytest.mark.parametrize("M,N,K,with_bias", [
    (128, 256, 128, False),     # one tile, one K stage
    (300, 384, 512, True),      # ragged M, two N tiles (the second one half full)
    (200, 264, 1040, True),     # ragged N (not a multiple of 256) and a partial last K stage
    (1000, 1024, 768, False),   # several waves of tiles over the persistent CTAs
])
def test_linear_matches_oracle(M, N, K, with_bias):
    xb, wb = _rows(60 + M, M, K), _rows(70 + N, N, K)
    qx, sx = oracle.rowquant(xb, norm=True)
    qw, sw = oracle.rowquant(wb)
    bias = np.random.default_rng(3).standard_normal(N).astype(np.float32) if with_bias else None
    ref = oracle.w8a8_linear(qx, sx, qw, sw, bias)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = sla.w8a8_workspace()
    sla.sla_w8a8_linear(torch.from_numpy(qx).cuda(), torch.from_numpy(sx).cuda(), torch.from_numpy(qw).cuda(),
                        torch.from_numpy(sw).cuda(), None if bias is None else torch.from_numpy(bias).cuda(), out, ws)
    sla.sla_check(ws)
    got = out.float().cpu().numpy().astype(np.float64)
    # bf16 output rounding (2^-9 relative) plus fp32 dequantisation
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(ref).max()).all()


def test_dit_shape_sampled_rows():
    """A 14B DiT projection shape (K = N = 5120) over 4096 tokens with FusedNorm on the
    activations; rows sampled across the tiles are checked against the oracle."""
    M, N, K = 4096, 5120, 5120
    rng = np.random.default_rng(5)
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xd = torch.from_numpy(x).cuda().bfloat16()
    wd = torch.from_numpy(w).cuda().bfloat16()
    gamma = torch.from_numpy(rng.uniform(0.5, 1.5, K).astype(np.float32)).cuda()
    qx = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    qw = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    sla.sla_w8a8_quantize(xd, qx, sx, norm=True, gamma=gamma)
    sla.sla_w8a8_quantize(wd, qw, sw)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = sla.w8a8_workspace()
    sla.sla_w8a8_linear(qx, sx, qw, sw, None, out, ws)
    sla.sla_check(ws)
    rows = np.sort(rng.choice(M, 24, replace=False))
    xb = xd.view(torch.int16).cpu().numpy().view(np.uint16)
    wb = wd.view(torch.int16).cpu().numpy().view(np.uint16)
    qxo, sxo = oracle.rowquant(xb[rows], norm=True, gamma=gamma.cpu().numpy())
    qwo, swo = oracle.rowquant(wb)
    assert np.array_equal(qx.cpu().numpy()[rows], qxo) and np.array_equal(sx.cpu().numpy()[rows], sxo)
    assert np.array_equal(qw.cpu().numpy(), qwo) and np.array_equal(sw.cpu().numpy(), swo)
    ref = oracle.w8a8_linear(qxo, sxo, qwo, swo)
    got = out.float().cpu().numpy()[rows].astype(np.float64)
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(ref).max()).all()

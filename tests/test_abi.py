"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching a GPU.

No call here reaches a CUDA API: every call is one the library must refuse
during validation (null / misaligned pointers, unsupported shapes, small
workspaces), or a pure host function.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sla.h")

sla = pytest.importorskip("sparse_linear_bit_b200")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SLA_API\s+[\w\s\*]*?\b(sla_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 9
    lib = ctypes.CDLL(sla.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_every_exported_symbol_is_declared():
    # the library's dynamic symbol table (default visibility) holds the header's calls and nothing else
    import shutil
    import subprocess

    if shutil.which("nm") is None:
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-D", "--defined-only", sla.LIB_PATH], capture_output=True, text=True, check=True)
    exported = sorted({line.split()[-1] for line in out.stdout.splitlines() if line.split()[-1].startswith("sla_")})
    assert exported == declared_symbols()


def test_library_links_no_torch():
    with open(sla.LIB_PATH, "rb") as f:
        blob = f.read()
    assert b"libtorch" not in blob and b"libc10" not in blob


def test_version_and_status_strings():
    assert "sm_100a" in sla.sla_version()
    for code, name in enumerate(["SLA_OK", "SLA_ERR_INVALID_ARG", "SLA_ERR_UNSUPPORTED", "SLA_ERR_WORKSPACE",
                                 "SLA_ERR_CUDA", "SLA_ERR_TIMEOUT"]):
        assert sla.sla_status_string(code) == name
    assert sla.sla_status_string(99) == "SLA_ERR_UNKNOWN"


@pytest.mark.parametrize("n_kb", [0, 1, 3, 10, 20, 32, 256, 512, 1182, 4096])
@pytest.mark.parametrize("topk", [0.0, 0.05, 0.1, 0.15, 0.2, 0.3, 0.5, 0.7, 0.99, 1.0])
def test_topk_count_matches_oracle_rule(n_kb, topk):
    assert sla.sla_topk_count(n_kb, topk) == oracle.topk_count(n_kb, float(np.float32(topk)))


def test_topk_count_rejects():
    assert sla.sla_topk_count(-1, 0.1) == -1
    assert sla.sla_topk_count(10, 1.5) == -1
    assert sla.sla_topk_count(10, -0.1) == -1
    assert sla.sla_topk_count(10, float("nan")) == -1


def test_workspace_bytes():
    a = sla.sla_workspace_bytes(1, 40, 75600, 128, 128, 64, 0.1, 1)
    b = sla.sla_workspace_bytes(1, 40, 75600, 128, 128, 64, 0.1, 0)
    assert a > b > 0
    assert sla.sla_workspace_bytes(1, 40, 75600, 64, 128, 64, 0.1, 1) == 0      # d != 128
    assert sla.sla_workspace_bytes(1, 40, 75600, 128, 96, 64, 0.1, 1) == 0      # blk_q
    assert sla.sla_workspace_bytes(1, 40, 75600, 128, 128, 32, 0.1, 1) == 0     # blk_k
    assert sla.sla_workspace_bytes(1, 40, 75600, 128, 128, 64, 1.1, 1) == 0     # topk
    assert sla.sla_workspace_bytes(0, 40, 75600, 128, 128, 64, 0.1, 1) == 0     # B
    lay = sla.sla_workspace_layout(1, 2, 2048, 128, 64, 64, 0.1, 1)
    offs = [v for v in lay.values() if v is not None]
    assert len(set(offs)) == len(offs) and all(o % 256 == 0 for o in offs)
    assert set(lay) == set(sla.LAYOUT_REGIONS)
    assert sla.sla_workspace_layout(1, 2, 2048, 128, 64, 64, 0.1, 0)["q8"] is None


FAKE = 1 << 20  # an aligned non-null address; never dereferenced because validation fails first
L = sla.lib


def fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, H=2, N=2048, d=128, blk_q=64, blk_k=64, topk=0.1, phi=0,
             quant=1, ws=FAKE, ws_bytes=0, stream=None)
    a.update(kw)
    return L.sla_forward(a["q"], a["k"], a["v"], a["out"], a["B"], a["H"], a["N"], a["d"], a["blk_q"], a["blk_k"],
                         a["topk"], a["phi"], a["quant"], a["ws"], a["ws_bytes"], a["stream"])


def test_forward_host_validation():
    assert fwd(q=None) == 1
    assert fwd(out=FAKE + 8) == 1          # misaligned
    assert fwd(B=0) == 1 and fwd(N=-5) == 1
    assert fwd(topk=1.5) == 1 and fwd(topk=float("nan")) == 1
    assert fwd(phi=2) == 1 and fwd(quant=3) == 1
    assert fwd(d=64) == 2 and fwd(blk_q=32) == 2 and fwd(blk_k=128) == 2
    assert fwd(ws_bytes=0) == 3            # workspace too small (everything else valid)
    need = sla.sla_workspace_bytes(1, 2, 2048, 128, 64, 64, 0.1, 1)
    assert fwd(ws_bytes=need - 1) == 3


def fwd_host(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, H=3, N=2048, d=128, blk_q=64, blk_k=64, topk=0.1, phi=0,
             quant=1, chunk=2, dev=FAKE, dev_bytes=0, stream=None)
    a.update(kw)
    return L.sla_forward_host(a["q"], a["k"], a["v"], a["out"], a["B"], a["H"], a["N"], a["d"], a["blk_q"],
                              a["blk_k"], a["topk"], a["phi"], a["quant"], a["chunk"], a["dev"], a["dev_bytes"],
                              a["stream"])


def test_forward_from_host_buffers_validation():
    assert fwd_host(q=None) == 1 and fwd_host(out=None) == 1 and fwd_host(dev=None) == 1
    assert fwd_host(dev=FAKE + 8) == 1                 # misaligned device memory
    assert fwd_host(chunk=0) == 1 and fwd_host(chunk=-3) == 1
    assert fwd_host(B=0) == 1 and fwd_host(topk=2.0) == 1 and fwd_host(phi=5) == 1 and fwd_host(quant=3) == 1
    assert fwd_host(d=64) == 2 and fwd_host(blk_q=32) == 2
    assert fwd_host(dev_bytes=0) == 3                  # device memory too small (everything else valid)
    need = sla.sla_forward_host_bytes(1, 3, 2048, 128, 64, 64, 0.1, 1, 2)
    assert fwd_host(dev_bytes=need - 1) == 3


def test_forward_from_host_buffers_bytes():
    # the workspace of one chunk's forward, then two slots of Q, K, V and output of one chunk
    for (B, H, N, quant, chunk) in ((1, 40, 75600, 1, 5), (1, 3, 2048, 0, 2), (2, 3, 585, 2, 4), (1, 2, 210, 1, 9)):
        hc = min(chunk, B * H)
        ws = sla.sla_workspace_bytes(1, hc, N, 128, 64, 64, 0.1, quant)
        tensor = -(-hc * N * 128 * 2 // 256) * 256
        assert sla.sla_forward_host_bytes(B, H, N, 128, 64, 64, 0.1, quant, chunk) == -(-ws // 256) * 256 + 8 * tensor
    assert sla.sla_forward_host_bytes(1, 3, 2048, 128, 64, 64, 0.1, 1, 0) == 0     # chunk_heads
    assert sla.sla_forward_host_bytes(1, 3, 2048, 128, 64, 64, 0.1, 3, 2) == 0     # quant
    assert sla.sla_forward_host_bytes(1, 3, 2048, 64, 64, 64, 0.1, 1, 2) == 0      # d


def bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, H=2, N=2048, d=128, blk_q=64,
             blk_k=64, topk=0.1, phi=0, ws=FAKE, ws_bytes=0, stream=None)
    a.update(kw)
    return L.sla_backward(a["q"], a["k"], a["v"], a["dout"], a["dq"], a["dk"], a["dv"], a["B"], a["H"], a["N"],
                          a["d"], a["blk_q"], a["blk_k"], a["topk"], a["phi"], a["ws"], a["ws_bytes"], a["stream"])


def test_backward_host_validation():
    assert bwd(dout=None) == 1 and bwd(dq=None) == 1 and bwd(dv=None) == 1
    assert bwd(dk=FAKE + 4) == 1           # misaligned
    assert bwd(B=0) == 1 and bwd(topk=-0.5) == 1 and bwd(phi=3) == 1
    assert bwd(d=64) == 2 and bwd(blk_q=256) == 2 and bwd(blk_k=32) == 2
    assert bwd(ws_bytes=0) == 3            # workspace too small (everything else valid)
    need = sla.sla_backward_workspace_bytes(1, 2, 2048, 128, 64, 64, 0.1)
    assert bwd(ws_bytes=need - 1) == 3


def test_backward_workspace_bytes():
    # the backward's workspace starts with the forward's (quantisation off) and adds its own regions
    for (B, H, N, blk_q, topk) in ((1, 2, 2048, 64, 0.1), (1, 40, 75600, 128, 0.1), (2, 3, 585, 64, 0.6),
                                   (1, 1, 210, 128, 0.0), (1, 1, 210, 128, 1.0)):
        f = sla.sla_workspace_bytes(B, H, N, 128, blk_q, 64, topk, 0)
        b = sla.sla_backward_workspace_bytes(B, H, N, 128, blk_q, 64, topk)
        n_qb, n_kb = -(-N // blk_q), -(-N // 64)
        # at least: row statistics, dH in fp32 and bf16, and G, over the state columns
        extra = B * H * (3 * N * 4 + n_qb * 16512 * 6 + n_kb * 16512 * 4)
        assert b >= f + extra, (B, H, N, blk_q, topk)
    assert sla.sla_backward_workspace_bytes(1, 2, 2048, 64, 64, 64, 0.1) == 0     # d != 128
    assert sla.sla_backward_workspace_bytes(1, 2, 2048, 128, 96, 64, 0.1) == 0    # blk_q
    assert sla.sla_backward_workspace_bytes(1, 2, 2048, 128, 64, 64, 1.5) == 0    # topk


def test_block_mask_and_quant_host_validation():
    assert L.sla_block_mask(FAKE, FAKE, 1, 2, 2048, 128, 64, 64, 0.1, None, None, FAKE, 1 << 40, None) == 1
    assert L.sla_block_mask(FAKE, FAKE, 1, 2, 2048, 128, 64, 64, 0.1, FAKE + 2, None, FAKE, 1 << 40, None) == 1
    assert L.sla_block_mask(FAKE, FAKE, 1, 2, 2048, 128, 64, 64, 0.1, FAKE, None, FAKE, 16, None) == 3
    assert L.sla_block_mask(FAKE, FAKE, 1, 2, 2048, 96, 64, 64, 0.1, FAKE, None, FAKE, 1 << 40, None) == 2
    assert L.sla_quantize_qk(FAKE, FAKE, 1, 2, 2048, 128, 64, 64, None, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                             None) == 1
    assert L.sla_quantize_qk(FAKE, FAKE, 1, 2, 2048, 128, 64, 64, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16, None) == 3
    # the FP8 variant validates the same way
    assert L.sla_quantize_qk_fp8(FAKE, FAKE, 1, 2, 2048, 128, 64, 64, None, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                                 None) == 1
    assert L.sla_quantize_qk_fp8(FAKE, FAKE, 1, 2, 2048, 128, 64, 64, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16,
                                 None) == 3
    assert L.sla_quantize_qk_fp8(FAKE, FAKE, 1, 2, 2048, 128, 96, 64, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                                 None) == 2
    # quant = 2 (FP8) needs the same workspace as INT8
    assert sla.sla_workspace_bytes(1, 2, 2048, 128, 64, 64, 0.1, 2) == sla.sla_workspace_bytes(1, 2, 2048, 128, 64,
                                                                                              64, 0.1, 1)
    # W8A8: shapes the kernels do not cover, null or misaligned pointers, a small workspace
    assert L.sla_w8a8_quantize(FAKE, 4, 100, 0, None, ctypes.c_float(1e-6), FAKE, FAKE, None) == 2   # cols % 8
    assert L.sla_w8a8_quantize(FAKE, 4, 16392, 0, None, ctypes.c_float(1e-6), FAKE, FAKE, None) == 2
    assert L.sla_w8a8_quantize(None, 4, 128, 0, None, ctypes.c_float(1e-6), FAKE, FAKE, None) == 1
    assert L.sla_w8a8_quantize(FAKE, 4, 128, 2, None, ctypes.c_float(1e-6), FAKE, FAKE, None) == 1     # norm
    assert L.sla_w8a8_quantize(FAKE, 4, 128, 1, None, ctypes.c_float(-1.0), FAKE, FAKE, None) == 1    # eps
    assert L.sla_w8a8_linear(FAKE, FAKE, FAKE, FAKE, None, 4, 8, 24, FAKE, FAKE, 256, None) == 2      # K % 16
    assert L.sla_w8a8_linear(FAKE, FAKE, FAKE, FAKE, None, 4, 12, 32, FAKE, FAKE, 256, None) == 2     # N % 8
    assert L.sla_w8a8_linear(FAKE, FAKE, FAKE + 8, FAKE, None, 4, 8, 32, FAKE, FAKE, 256, None) == 1  # align
    assert L.sla_w8a8_linear(FAKE, FAKE, FAKE, FAKE, None, 4, 8, 32, FAKE, FAKE, 16, None) == 3       # ws
    assert L.sla_w8a8_linear(FAKE, FAKE, FAKE, FAKE, None, 0, 8, 32, FAKE, FAKE, 256, None) == 1
    assert sla.lib.sla_w8a8_workspace_bytes() == 256
    assert L.sla_check(None, None) == 1


def test_binding_raises():
    with pytest.raises(sla.SlaError) as e:
        sla._ok(2, "x")
    assert e.value.code == 2 and "UNSUPPORTED" in str(e.value)

#!/usr/bin/env python
"""Benchmark of the SageSLA attention forward (libsla.so, sm_100a).

One step = one sla_forward call over the whole workload (pooling, top-k block
selection, smoothing + INT8 quantisation, linear states, per-query-block state,
fused block-sparse attention + linear epilogue).  Default workload: the
14B-720P attention shape (B=1, H=40, N=75600 tokens on a 21x45x80 grid,
d=128, blk_q=128, blk_k=64, topk=0.1, phi=elu+1, INT8 on), synthetic seeded
inputs.  The inputs (2.3 GB of Q/K/V) exceed the 126 MB L2, so no flush is
needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--topk T] [--quant 0|1]
    python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

Multi-GPU (launched with torch.distributed.run, one rank per GPU), no data-path
collective since every (batch, head) is independent:
  --scaling weak   (default) every rank runs the whole workload as its own batch
                   element; the job grows with the number of GPUs.
  --scaling strong the workload's B*H heads are split into contiguous ranges, one
                   per rank (sparse_linear_bit_b200.head_shard).
  --scaling ulysses every rank holds N/P tokens of every head (context
                   parallelism); a step is the all-to-all to head shards, the
                   forward on H/P heads and the all-to-all back (NCCL).
Times are taken on the device and the max over ranks is reported.  Rank 0
prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SLA fwd ms & dense-equiv TOPS at N=75600,H=40,d=128; % of tensor peak"
ATTN_SRC = os.path.join(ROOT, "sparse_linear_bit_b200", "csrc", "sla_attention.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_kernel_traffic.json")
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = {2: 10, 1: 10, 0: 8}  # our launches per sla_forward call (fp8 / int8 / off)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan14b-720p")
    ap.add_argument("--topk", type=float, default=0.10)
    ap.add_argument("--quant", type=int, default=1, choices=[0, 1, 2], help="0 none, 1 INT8, 2 FP8 e4m3")
    ap.add_argument("--phi", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-w8a8", action="store_true", help="skip the W8A8 linear-layer measurement")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward (fine-tuning) measurement")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong", "ulysses"])
    ap.add_argument("--heads", type=int, default=0, help="override the workload's head count (profiling runs)")
    return ap.parse_args()


def max_over_ranks(x: float, device, world: int) -> float:
    """Max of a per-rank scalar (a device-timed duration) over all ranks."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dense_equiv_ops(B, H, N, d):
    """4 B H N^2 d: the multiply-adds of dense softmax attention (QK^T and PV), x2."""
    return 4.0 * B * H * float(N) * float(N) * d


def workload_config(w, a):
    nbytes = w.B * w.H * w.N * w.d * 2
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "grid_thw": list(w.grid),
            "blk_q": w.blk_q, "blk_k": w.blk_k, "topk": a.topk, "phi": ["elu+1", "relu"][a.phi],
            "quant": {1: "int8 Q/K, bf16 P.V", 2: "fp8 e4m3 Q/K, bf16 P.V"}.get(a.quant, "bf16 Q.K^T, fp16 P.V"),
            "l2": ("inputs (3 x %.2f GB) exceed the 126 MB L2; no flush between steps" if 3 * nbytes > 126e6 else
                   "inputs (3 x %.3f GB) fit in L2: steps run warm") % (nbytes / 1e9)}


# --------------------------------------------------------------------------
# CPU oracle leg (reference arm and cpu_baseline)
# --------------------------------------------------------------------------

def oracle_sample(q, k, v, w, a, n_qblocks, head=0):
    """Time the fp64 oracle on one head's first n_qblocks query blocks."""
    import oracle
    oracle.build()
    rows_i = np.arange(min(w.N, n_qblocks * w.blk_q), dtype=np.int64)
    rows = np.stack([np.full_like(rows_i, head), rows_i], axis=1)
    t0 = time.perf_counter()
    oracle.forward(q, k, v, w.blk_q, w.blk_k, float(np.float32(a.topk)), phi=a.phi, quant=a.quant, rows=rows)
    dt = time.perf_counter() - t0
    ops = 4.0 * len(rows_i) * float(w.N) * w.d  # dense-equivalent ops of the sampled rows
    return ops, dt, len(rows_i), oracle.num_threads()


def run_reference(a, w, rank, world):
    if rank != 0:
        return 0
    import synth
    q, k, v = synth.make_qkv(w.B, w.H, w.grid, seed=w.seed)
    n_qb = 16
    for _ in range(a.warmup):
        oracle_sample(q, k, v, w, a, n_qb)
    times, ops_total = [], 0.0
    for _ in range(a.steps):
        ops, dt, nrows, cores = oracle_sample(q, k, v, w, a, n_qb)
        times.append(dt)
        ops_total += ops
    tot = sum(times)
    value = ops_total / tot / 1e12
    sample = (f"one head, first {nrows} query rows ({n_qb} query blocks) of the {w.name} workload per step, "
              f"with that head's mask, quantisation and states; dense-equivalent ops of those rows")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * tot / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, a),
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------

def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def attn_source_sha():
    h = hashlib.sha256()
    for name in ("sla_attention.cu", "sla_ptx.cuh"):
        with open(os.path.join(ROOT, "sparse_linear_bit_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, topk, quant):
    """DRAM bytes per attention launch from a committed ncu capture, or None when
    the capture does not match the current kernel source or this workload."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except Exception:
        return None
    if t.get("kernel_source_sha") != attn_source_sha():
        return None
    key = f"{workload}|topk={topk:g}|quant={quant}"
    return t.get("bytes_per_launch", {}).get(key)


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def selected_work(idx, w, k_sel):
    """Exact multiply-adds of the sparse branch: rows x valid selected keys x d, per launch."""
    n_qb = -(-w.N // w.blk_q)
    rows = np.minimum(w.blk_q, w.N - np.arange(n_qb) * w.blk_q).astype(np.float64)
    keys_per_block = np.minimum(64, w.N - np.arange(-(-w.N // 64)) * 64).astype(np.float64)
    keys = keys_per_block[idx].sum(axis=-1)  # [BH, n_qb]
    return float((keys * rows[None, :]).sum()) * w.d


def run_ulysses(a, w, q, k, v, rank, world, dev, ops_job):
    """Context-parallel step: token-sharded inputs, all-to-all, forward on H/P heads, all-to-all back."""
    import torch
    import torch.distributed as dist
    from sparse_linear_bit_b200 import ulysses
    if w.H % world or w.N % world:
        raise SystemExit(f"--scaling ulysses needs H and N divisible by {world}")
    n = w.N // world
    to_dev = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, :, rank * n:(rank + 1) * n]).view(np.int16)).view(
        torch.bfloat16).to(dev)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    import sparse_linear_bit_b200 as sla
    ws = sla.workspace(w.B, w.H // world, w.N, w.d, w.blk_q, w.blk_k, a.topk, a.quant, device=dev)
    step = lambda: ulysses.sla_forward_ulysses(qd, kd, vd, w.blk_q, w.blk_k, a.topk, a.phi, a.quant, ws=ws)
    for _ in range(max(3, a.warmup)):
        step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.steps):
        step()
    e1.record()
    torch.cuda.synchronize(dev)
    dist.barrier()
    sla.sla_check(ws)
    ms = max_over_ranks(e0.elapsed_time(e1) / a.steps, dev, world)
    if rank == 0:
        line = {"metric": METRIC, "value": ops_job / (ms * 1e-3) / 1e12, "unit": "TOPS", "n_gpus": world,
                "steps": a.steps, "warmup": max(3, a.warmup), "ms_per_step": ms, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None,
                "dtype": {0: "bf16+fp16", 1: "i8+bf16", 2: "fp8e4m3+bf16"}[a.quant], "data": "synthetic",
                "config": dict(workload_config(w, a), parallelism=f"{world} ranks, Ulysses context parallelism: "
                               f"{n} tokens of every head per rank, all-to-all to {w.H // world} heads per rank"),
                "gpu_launches": None}
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def main():
    a = parse()
    import synth

    w0 = synth.WORKLOADS[a.workload]
    w = synth.Workload(w0.name if not a.heads else f"{w0.name}-h{a.heads}", w0.B, a.heads or w0.H, w0.grid,
                       blk_q=w0.blk_q, blk_k=w0.blk_k, topk=a.topk, phi=a.phi, quant=a.quant, seed=w0.seed)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        return run_reference(a, w, rank, world)

    import torch
    import torch.distributed as dist
    import sparse_linear_bit_b200 as sla

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    # ---- inputs: generated once (rank 0) and shared through /dev/shm
    shm = f"/dev/shm/sla_bench_{w.name}_{w.seed}_{os.getuid()}"
    if world == 1:
        q, k, v = synth.make_qkv(w.B, w.H, w.grid, seed=w.seed)
    else:
        if rank == 0:
            q, k, v = synth.make_qkv(w.B, w.H, w.grid, seed=w.seed)
            for nm, x in (("q", q), ("k", k), ("v", v)):
                np.save(shm + f"_{nm}.npy", x)
        dist.barrier()
        if rank != 0:
            q, k, v = (np.load(shm + f"_{nm}.npy") for nm in ("q", "k", "v"))
    # ---- this rank's share: the whole workload (weak) or a contiguous head range (strong)
    ops_job = dense_equiv_ops(w.B, w.H, w.N, w.d) * (world if a.scaling == "weak" else 1)
    wl = w
    if a.scaling == "ulysses" and world > 1:
        return run_ulysses(a, w, q, k, v, rank, world, dev, ops_job)
    if a.scaling == "strong" and world > 1:
        first, count = sla.head_shard(w.B, w.H, world, rank)
        q, k, v = (np.ascontiguousarray(sla.shard_heads(x, world, rank)) for x in (q, k, v))
        wl = synth.Workload(w.name, 1, count, w.grid, d=w.d, blk_q=w.blk_q, blk_k=w.blk_k, topk=a.topk, phi=a.phi,
                            quant=a.quant, seed=w.seed)
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out = torch.empty_like(qd)
    ws = sla.workspace(wl.B, wl.H, wl.N, wl.d, wl.blk_q, wl.blk_k, a.topk, a.quant, device=dev)
    stream = torch.cuda.current_stream(dev)
    fwd = lambda: sla.sla_forward(qd, kd, vd, out, wl.blk_q, wl.blk_k, a.topk, a.phi, a.quant, ws, stream=stream)

    for _ in range(max(3, a.warmup)):
        fwd()
    sla.sla_check(ws, stream=stream)

    # ---- per-stage device times (CUDA events between the stages, same stream)
    stage = {n: [] for n in sla.PROFILE_STAGES}
    for _ in range(min(5, max(1, a.steps))):
        r = sla.sla_forward_profile(qd, kd, vd, out, wl.blk_q, wl.blk_k, a.topk, a.phi, a.quant, ws, stream=stream)
        for n_, t_ in r.items():
            stage[n_].append(t_)
    stage_ms = {n_: float(np.median(t_)) for n_, t_ in stage.items()}

    # ---- timed region: K steps, inputs resident in HBM
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(vis.split(",")[local].strip() if vis else local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)  # let the sampler start
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(a.steps):
        fwd()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    sla.sla_check(ws, stream=stream)
    ms = max_over_ranks(e0.elapsed_time(e1) / a.steps, dev, world)
    ops = dense_equiv_ops(wl.B, wl.H, wl.N, wl.d)  # this rank's share
    value = ops_job / (ms * 1e-3) / 1e12

    # ---- end to end through the C-ABI call that takes HOST buffers (sla_forward_host): pinned host
    # Q/K/V in, bf16 output back to pinned host memory, every copy inside the timed region.  The call
    # runs the (batch, head) problems in chunks of consecutive heads on three streams of its own, so
    # that the copy-in of chunk c+1 and the copy-out of chunk c-1 overlap the forward of chunk c; its
    # result equals one device call over the whole workload.
    e2e = None
    if not a.no_e2e:
        hq_, hk_, hv_ = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (q, k, v))
        hout = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
        steps_e2e = max(2, min(a.steps, 5))
        n_chunks = min(8, wl.B * wl.H)
        chunk_heads = -(-(wl.B * wl.H) // n_chunks)
        dev_host = sla.host_workspace(wl.B, wl.H, wl.N, wl.d, wl.blk_q, wl.blk_k, a.topk, a.quant, chunk_heads,
                                      device=dev)
        s_e2e = torch.cuda.current_stream(dev)

        def e2e_step():
            sla.sla_forward_host(hq_, hk_, hv_, hout, wl.blk_q, wl.blk_k, a.topk, a.phi, a.quant, chunk_heads,
                                 dev_host, stream=s_e2e)

        def timed(nsteps):
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            f0.record(s_e2e)
            for _ in range(nsteps):
                e2e_step()
            f1.record(s_e2e)
            torch.cuda.synchronize(dev)
            return f0.elapsed_time(f1) / nsteps

        timed(1)
        sla.sla_check(dev_host, stream=s_e2e)
        # the chunked host call gives, bit for bit, the output of one device call over the workload
        fwd()
        torch.cuda.synchronize(dev)
        same = bool(torch.equal(hout.view(torch.int16), out.cpu().view(torch.int16)))
        if world > 1:
            dist.barrier()
        ms_e2e = max_over_ranks(timed(steps_e2e), dev, world)
        sla.sla_check(dev_host, stream=s_e2e)
        nbytes = qd.numel() * 2
        e2e = {"value": ops_job / (ms_e2e * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes, "chunks": -(-(wl.B * wl.H) // chunk_heads),
               "output_equals_single_call": same,
               "note": ("sla_forward_host: Q, K, V copied in from pinned host memory and the output copied back "
                        f"inside the call, {chunk_heads} heads per chunk pipelined over copy-in, compute and "
                        "copy-out streams")}
        del dev_host

    # ---- roofline of the dominant kernel (attention), against the measured peaks
    peaks, peak_kind = load_peaks()
    n_kb = -(-w.N // w.blk_k)
    k_sel = sla.sla_topk_count(n_kb, a.topk)
    lay = sla.sla_workspace_layout(wl.B, wl.H, wl.N, wl.d, wl.blk_q, wl.blk_k, a.topk, a.quant)
    n_qb = -(-w.N // w.blk_q)
    idx = ws[lay["idx"]:lay["idx"] + wl.B * wl.H * n_qb * max(k_sel, 1) * 4].cpu().numpy().view(np.int32)
    idx = idx.reshape(wl.B * wl.H, n_qb, max(k_sel, 1))[..., :k_sel]
    macs = selected_work(idx, w, k_sel) if k_sel > 0 else 0.0
    ops_qk, ops_pv = 2.0 * macs, 2.0 * macs
    ops_lin = 2.0 * wl.B * wl.H * n_qb * 128.0 * w.d * w.d  # phi(Q_I) H_I, tf32
    p_bf16 = float(peaks["bf16_tflops"]) * 1e12
    p_qk = 2.0 * p_bf16 if a.quant else p_bf16  # int8 and fp8 = 2x bf16 (nominal ratio)
    p_tf32 = 0.5 * p_bf16
    t_attn = stage_ms["attention"] * 1e-3
    ideal = ops_qk / p_qk + ops_pv / p_bf16 + ops_lin / p_tf32
    tot_ops = ops_qk + ops_pv + ops_lin
    achieved = tot_ops / t_attn / 1e12
    peak = tot_ops / ideal / 1e12
    traffic = recorded_traffic(w.name, a.topk, a.quant)
    roofline = {"bound": "tensor", "kernel": "attn_kernel", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peak_kind} bf16 {peaks['bf16_tflops']} TFLOP/s (burst); int8/fp8 = 2x, tf32 = 0.5x",
                "ops_per_launch": {{0: "qk_bf16", 1: "qk_int8", 2: "qk_fp8"}[a.quant]: ops_qk, "pv_bf16": ops_pv,
                                   "linear_tf32": ops_lin},
                "launch_ms": stage_ms["attention"],
                # the same ideal tensor time over the whole call (every stage of the step)
                "whole_call_frac": ideal / (ms * 1e-3)}

    # ---- W8A8 INT8 linear layer (+ FusedNorm) at the DiT projection shape of this workload:
    #      the N tokens of one sample x hidden 5120 -> 5120 (the 14B model's width)
    w8a8 = None
    if rank == 0 and not a.no_w8a8:
        M_, N_, K_ = w.N, 5120, 5120
        gen = torch.Generator(device=dev).manual_seed(7)
        xw = torch.randn(M_, K_, device=dev, generator=gen).bfloat16()
        ww = (torch.randn(N_, K_, device=dev, generator=gen) * 0.02).bfloat16()
        gam = torch.ones(K_, device=dev)
        qx_ = torch.empty((M_, K_), dtype=torch.int8, device=dev)
        sx_ = torch.empty(M_, dtype=torch.float32, device=dev)
        qw_ = torch.empty((N_, K_), dtype=torch.int8, device=dev)
        sw_ = torch.empty(N_, dtype=torch.float32, device=dev)
        yw = torch.empty((M_, N_), dtype=torch.bfloat16, device=dev)
        wsw = sla.w8a8_workspace(dev)
        sla.sla_w8a8_quantize(ww, qw_, sw_, stream=stream)
        layer = lambda: (sla.sla_w8a8_quantize(xw, qx_, sx_, norm=True, gamma=gam, stream=stream),
                         sla.sla_w8a8_linear(qx_, sx_, qw_, sw_, None, yw, wsw, stream=stream))
        for _ in range(3):
            layer()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        tq_, tg_ = [], []
        for _ in range(10):
            evs[0].record(stream)
            sla.sla_w8a8_quantize(xw, qx_, sx_, norm=True, gamma=gam, stream=stream)
            evs[1].record(stream)
            sla.sla_w8a8_linear(qx_, sx_, qw_, sw_, None, yw, wsw, stream=stream)
            evs[2].record(stream)
            torch.cuda.synchronize(dev)
            tq_.append(evs[0].elapsed_time(evs[1]))
            tg_.append(evs[1].elapsed_time(evs[2]))
        sla.sla_check(wsw, stream=stream)
        gq, gg = float(np.median(tq_)), float(np.median(tg_))
        ops_w = 2.0 * M_ * N_ * K_
        p_i8 = 2.0 * float(peaks["bf16_tflops"])
        w8a8 = {"shape": {"M_tokens": M_, "N": N_, "K": K_}, "fused_norm_quantize_ms": gq,
                "quantize_gbs": M_ * K_ * 3 / gq / 1e6, "gemm_ms": gg, "gemm_tops": ops_w / gg / 1e9,
                "gemm_frac_of_int8_peak": ops_w / gg / 1e9 / p_i8,
                "int8_peak_source": f"{peak_kind} bf16 {peaks['bf16_tflops']} TFLOP/s x 2 (nominal int8 ratio)"}
        del xw, ww, qx_, qw_, yw

    # ---- backward of the unquantised forward (gradients for SLA fine-tuning) on this rank's
    #      workload; a side measurement like the W8A8 one (not part of the timed step)
    bwd = None
    if rank == 0 and not a.no_backward:
        gen = torch.Generator(device=dev).manual_seed(11)
        dout = torch.randn(qd.shape, device=dev, generator=gen).bfloat16()
        grads = [torch.empty(qd.shape, dtype=torch.float32, device=dev) for _ in range(3)]
        wsb = sla.backward_workspace(*qd.shape, wl.blk_q, wl.blk_k, a.topk, device=dev)
        bcall = lambda: sla.sla_backward(qd, kd, vd, dout, *grads, wl.blk_q, wl.blk_k, a.topk, a.phi, wsb,
                                         stream=stream)
        bcall()
        torch.cuda.synchronize(dev)
        tb = []
        for _ in range(3):
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            bcall()
            b1.record(stream)
            torch.cuda.synchronize(dev)
            tb.append(b0.elapsed_time(b1))
        sla.sla_check(wsb, stream=stream)
        ms_b = float(np.median(tb))
        Bq, Hq, Nq, dq_ = qd.shape
        n_qb_b, n_kb_b = -(-Nq // wl.blk_q), -(-Nq // wl.blk_k)
        k_sel_b = sla.sla_topk_count(n_kb_b, a.topk)
        # algorithmic work: per (query block, selected key block) tile the five products of the
        # softmax backward (S, dP, dV, dQ, dK), 2 * 128 x 64 x d each; per query block the three
        # d x d products of the linear branch; per key block its two
        fl_sparse = Bq * Hq * n_qb_b * k_sel_b * 5 * 2.0 * wl.blk_q * wl.blk_k * dq_
        fl_lin = Bq * Hq * (n_qb_b * 3 * 2.0 * wl.blk_q * dq_ * dq_ + n_kb_b * 2 * 2.0 * wl.blk_k * dq_ * dq_)
        # the per-tile products run as bf16 tensor-core MMAs (fp32 accumulation): bf16 tensor peak
        ach = (fl_sparse + fl_lin) / (ms_b * 1e-3) / 1e12
        p_bf16 = float(peaks["bf16_tflops"])
        bwd = {"ms": ms_b, "what": "dq, dk, dv (fp32) of the unquantised forward for a random dout",
               "roofline": {"bound": "tensor", "achieved": ach, "peak": p_bf16, "unit": "TFLOP/s",
                            "frac": ach / p_bf16, "peak_source": f"{peak_kind} bf16 {p_bf16} TFLOP/s (burst)",
                            "note": "every product (softmax and linear branches) as tcgen05 bf16 MMAs with fp32 accumulation in tensor memory"},
               "flops_per_call": fl_sparse + fl_lin}
        del dout, grads, wsb

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, single GPU only)
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        n_qb_s = -(-w.N // w.blk_q)  # whole heads, two of them (about 10-15 s on 16 cores)
        ops_s = dt = 0.0
        n_heads_s = min(2, w.B * w.H)
        for hd in range(n_heads_s):
            o_, t_, nrows, cores = oracle_sample(q, k, v, w, a, n_qb_s, head=hd)
            ops_s += o_
            dt += t_
        cpu = {"value": ops_s / dt / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle",
               "sample": f"{n_heads_s} of {w.B * w.H} heads of {w.name} ({nrows} query rows, {n_qb_s} query blocks "
                         f"each), including those heads' masks, quantisation and states; {dt:.1f} s; "
                         f"dense-equivalent ops of those rows"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": a.steps,
                "warmup": max(3, a.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": a.scaling,
                "vs_baseline": None, "dtype": {0: "bf16+fp16", 1: "i8+bf16", 2: "fp8e4m3+bf16"}[a.quant],
                "data": "synthetic",
                "config": dict(workload_config(w, a), parallelism=(
                    f"{world} rank(s), one per GPU; " + ("each runs the whole workload" if a.scaling == "weak"
                                                         else "B*H heads split in contiguous ranges"))),
                "stages_ms": stage_ms, "roofline": roofline,
                "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "w8a8_linear": w8a8, "backward": bwd,
                "gpu_launches": KERNELS_PER_STEP[a.quant] * a.steps,
                "dense_equiv_ops_per_step_per_gpu": ops}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
        if rank == 0:
            for nm in ("q", "k", "v"):
                try:
                    os.unlink(shm + f"_{nm}.npy")
                except OSError:
                    pass
    return 0


if __name__ == "__main__":
    sys.exit(main())

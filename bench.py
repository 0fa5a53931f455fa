#!/usr/bin/env python3
"""Benchmark of the tile-sparse attention layer (Veda, head-aware tiles) on B200.

One step = one attention layer of the inference path on one GPU, all
through the C ABI, inputs resident in HBM.  With ``--layout tile``:
    permute Q, K, V -> TripPool Q, K -> estimator + softmax + top-k
    -> tile-skipping attention -> unpermute;
with ``--layout grid`` the permutation is folded into the attention kernel's
tile fetch (each tile is one box of the grid-order tensor) and its output
goes straight to grid rows:
    TripPool Q, K (read in grid order) -> estimator + softmax + top-k
    -> tile-skipping attention (grid order in and out).  Default workload: the
Wan2.1-14B 720p/81-frame shape (21x45x80 grid = 75,600 tokens, 40 heads,
d = 128, 128-token per-head tiles, keep 5% = 95% sparsity).

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload instead.

Multi-GPU: one process per GPU (torchrun); every rank runs its own layer
(a different seed) with no data-path collective -- the heads of a layer are
independent, so the work partitions -- and the reported time is the max over
ranks (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tile-sparse attn ms/layer & kept-tile TFLOP/s (% of B200 BF16 peak) at 95% sparsity"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD_NAMES = {"wan14b": "Wan2.1-14B-720p-81f 21x45x80 (75,600 tokens) 40 heads d128 keep 5%",
                  "wan14b-k10": "Wan2.1-14B-720p-81f 21x45x80 40 heads d128 keep 10%",
                  "wan14b-dense": "Wan2.1-14B-720p-81f 21x45x80 40 heads d128 keep 100% (dense reference)",
                  "wan1.3b": "Wan2.1-1.3B-480p 21x30x52 (32,760 tokens) 12 heads d128 keep 10%",
                  "long": "long video 31x45x80 (111,600 tokens) 24 heads d128 keep 5%",
                  "sweep61k": "sweep 15x64x64 (61,440 tokens) 24 heads (2,8,8) keep 5%",
                  "sweep123k": "sweep 30x64x64 (122,880 tokens) 24 heads (2,8,8) keep 5%",
                  "sweep246k": "sweep 60x64x64 (245,760 tokens) 24 heads (2,8,8) keep 5%",
                  "tiny": "tiny 4x8x8 2 heads d64"}


# DRAM bytes (read + write) of one attention launch, from a one-pass ncu
# capture of the benchmarked launch (summarised with the committed profiles),
# keyed by workload and layout and tied to the kernel source it was measured
# on: reported only while csrc/sparse_attn.cu still hashes to that version.
ATTN_TRAFFIC = {("wan14b", "tile"): {"bytes": 1.26e9 + 858.49e6, "src_sha256_16": "b5a8f826b6c7f91f"},
                ("wan14b", "grid"): {"bytes": 1139.90e6 + 740.74e6, "src_sha256_16": "6768221b7d236b48"}}


def attn_traffic(workload: str, layout: str):
    import hashlib
    rec = ATTN_TRAFFIC.get((workload, layout))
    if rec is None:
        return None
    path = os.path.join(ROOT, "tile_sparse_attention_head_b200", "csrc", "sparse_attn.cu")
    with open(path, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    return rec["bytes"] if digest == rec["src_sha256_16"] else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kept_flops(nts, ks, B, S, d):
    """Algorithmic FLOPs of the tile-skipping attention: 4*S^2*d per kept (Q tile, K tile) pair."""
    return float(B * sum(nt * k for nt, k in zip(nts, ks)) * 4 * S * S * d)


class Clocks:
    """nvidia-smi sampling of SM clocks, power and throttle reasons.  Every
    sample carries the host time it was read at, so the summary can be
    restricted to the timed region (``mark``/``window``)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    # Bits of clocks_event_reasons.active (NVML's clock event reasons).
    ACTIVE_BITS = ((0x1, "gpu_idle"), (0x2, "applications_clocks_setting"), (0x4, "sw_power_cap"),
                   (0x8, "hw_slowdown"), (0x10, "sync_boost"), (0x20, "sw_thermal_slowdown"),
                   (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
                   (0x100, "display_clock_setting"))

    def __init__(self, device_index: int, interval_ms: int = 20):
        self.dev = device_index
        self.interval_ms = interval_ms
        self.proc = None
        self.file = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def window(self, t0: float, t1: float):
        """Host times (time.time()) bracketing the region the summary describes."""
        self.t0, self.t1 = t0, t1

    @staticmethod
    def parse(lines):
        """Rows of (host time or None, sm MHz, max MHz, power W, set of active
        named reasons, set of every reason in the active bitmask)."""
        import datetime
        out = []
        for ln in lines:
            r = [x.strip() for x in ln.split(",")]
            try:
                try:
                    ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                sm, mx = float(r[2]), float(r[3])
                try:
                    pw = float(r[4])
                except ValueError:
                    pw = None
                reasons = {n for n, v in zip(Clocks.REASONS, r[6:10]) if v.lower() == "active"}
                try:
                    mask = int(r[5], 16)
                except ValueError:
                    mask = 0
                active = {n for b, n in Clocks.ACTIVE_BITS if mask & b}
                out.append((ts, sm, mx, pw, reasons, active))
            except (ValueError, IndexError):
                continue
        return out

    @staticmethod
    def summarize(rows, t0=None, t1=None):
        """Median SM clock, maximum clock, reasons and median power over the
        samples inside [t0, t1] (host time); if none falls inside (a region
        shorter than the sampling interval), the first sample after t0."""
        if not rows:
            return None
        inside = rows
        if t0 is not None and t1 is not None and all(r[0] is not None for r in rows):
            inside = [r for r in rows if t0 <= r[0] <= t1]
            if not inside:
                after = [r for r in rows if r[0] >= t0]
                inside = after[:1] if after else rows[-1:]
        sm = [r[1] for r in inside]
        pw = [r[3] for r in inside if r[3] is not None]
        reasons, active = set(), set()
        for r in inside:
            reasons |= r[4]
            active |= r[5]
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(r[2] for r in rows), "reasons": sorted(reasons),
                "reasons_active": sorted(active), "samples": len(inside),
                "sm_mhz_samples": [float(x) for x in sm][:64],
                "power_w": float(np.median(pw)) if pw else None,
                "window": "timed region" if t0 is not None else "whole run"}

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = self.parse([ln for ln in self.file.read().splitlines() if ln.strip()])
        os.unlink(self.file.name)
        return self.summarize(rows, self.t0, self.t1)


def choose_peak(peaks, clk, peak_src):
    """The tensor peak a kernel timed in this run is held against.  The burst
    figure (a GEMM timed alone, at full clock) applies unless the clock record
    of the timed region shows the board's power cap (or a thermal or hardware
    slowdown) holding the clock down -- a throttle reason present and the
    median SM clock below its maximum; then the sustained figure (a GEMM run
    for seconds at the power cap) applies.  Returns (peak, basis)."""
    if clk is not None and clk.get("sm_mhz") and clk.get("sm_max_mhz"):
        active = clk.get("reasons_active", [])
        basis = (f"median SM clock {clk['sm_mhz']:.0f} of {clk['sm_max_mhz']:.0f} MHz over "
                 f"{clk['samples']} sample(s) in the {clk.get('window', 'run')}, reasons {clk['reasons']}"
                 + (f", active {active}" if active else ""))
        throttles = set(clk["reasons"]) | (set(active) & {"sw_power_cap", "hw_power_brake_slowdown", "hw_slowdown",
                                                           "sw_thermal_slowdown", "hw_thermal_slowdown"})
        held_down = bool(throttles) and clk["sm_mhz"] < 0.97 * clk["sm_max_mhz"]
        if not held_down:
            return peaks["bf16_tflops"], f"{peak_src} bf16 burst: {basis}"
        return peaks["bf16_tflops_sustained"], f"{peak_src} bf16 sustained (power-capped GEMM): {basis}"
    return peaks["bf16_tflops"], f"{peak_src} bf16 burst (no clock record)"


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of every rank's x (each rank's device-timed milliseconds)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job TFLOP/s: every rank runs its own layer, the job takes the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def tiles_per_head(w):
    """Tiles of each head: the grid padded up to multiples of its tiling."""
    return [(-(-w.T // pt)) * (-(-w.H // ph)) * (-(-w.W // pw)) for pt, ph, pw in w.tilings]


def workload_for(args):
    """The preset, with the keep ratio overridden by --keep or --fixed-k."""
    import dataclasses
    from veda_synth import PRESETS
    w = PRESETS[args.workload]
    if args.keep is not None:
        w = dataclasses.replace(w, keep=float(args.keep))
    if args.fixed_k is not None:
        w = dataclasses.replace(w, keep=float(args.fixed_k) / max(tiles_per_head(w)))
    return w


def tile_token_counts(w):
    """[heads, NT_max] number of token slots of every tile (0 past NT_h)."""
    nts = tiles_per_head(w)
    out = np.zeros((w.heads, max(nts)), dtype=np.int64)
    for h, (pt, ph, pw) in enumerate(w.tilings):
        nT, nH, nW = -(-w.T // pt), -(-w.H // ph), -(-w.W // pw)
        j = np.arange(nts[h])
        jt, jh, jw = j // (nH * nW), (j // nW) % nH, j % nW
        out[h, :nts[h]] = (np.minimum(pt, w.T - jt * pt) * np.minimum(ph, w.H - jh * ph) *
                           np.minimum(pw, w.W - jw * pw))
    return out


def useful_flops(w, idx):
    """FLOPs of the kept (query, key) pairs that are both tokens (pad slots excluded)."""
    cnt = tile_token_counts(w)                        # [heads, NT_max]
    idx = idx.astype(np.int64)                        # [B, heads, NT_max, k_max]
    sel = np.where(idx >= 0, idx, 0)
    kv = np.take_along_axis(cnt[None, :, None, :].repeat(idx.shape[2], axis=2).repeat(idx.shape[0], axis=0),
                            sel, axis=3)
    kv = np.where(idx >= 0, kv, 0).sum(axis=3)        # valid keys per Q tile
    return float((kv * cnt[None]).sum() * 4 * w.d)


def tile_map_measure(V, w, p, qd, kd, args, rank, att=None):
    """Times the max-pooled tile map over a random 10% of Q tiles per head (the
    distillation target), with its tensor and exponential bounds: on the
    grid-order tensors (veda_tile_map_maxpool_grid) with --layout grid, on
    permuted copies (veda_tile_map_maxpool) with --layout tile."""
    from veda_synth import make_map_rows
    dev = qd.device
    if args.layout == "grid":
        qm, km, map_call = qd, kd, V.veda_tile_map_maxpool_grid
    else:
        ts = p.tile_shape()
        qm = torch.empty(ts, dtype=torch.bfloat16, device=dev)
        km = torch.empty(ts, dtype=torch.bfloat16, device=dev)
        V.veda_tile_permute(p, qd, qm)
        V.veda_tile_permute(p, kd, km)
        map_call = V.veda_tile_map_maxpool
    rows = make_map_rows(p.nt_per_head, w.B, 0.1, seed=2)
    R = rows.shape[1]
    counts = (rows >= 0).sum(dim=1).view(w.B, w.heads).numpy()
    rows = rows.to(dev)
    ws = torch.empty(V.veda_tile_map_workspace(p, R) // 4 + 64, dtype=torch.float32, device=dev)
    mp = torch.empty((w.B, w.heads, R, p.nt_max), dtype=torch.float32, device=dev)
    for _ in range(2):
        map_call(p, qm, km, rows, mp, ws)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.map_steps):
        map_call(p, qm, km, rows, mp, ws)
    e1.record()
    torch.cuda.synchronize()
    V.veda_sync_status()
    ms = e0.elapsed_time(e1) / args.map_steps
    # the estimator's distillation step against this map (forward estimator,
    # row-wise KL, gradients of both MLPs)
    dist = None
    if att is not None:
        wt = (att._wq, att._wk)
        grads = [tuple(torch.empty_like(t) for t in ws_) for ws_ in wt]
        gq, gk = V.make_mlp_grad(*grads[0]), V.make_mlp_grad(*grads[1])
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        dws = torch.empty(V.veda_distill_workspace(p, att.mlp_q.hidden, att.mlp_q.e, R) // 4 + 64,
                          dtype=torch.float32, device=dev)
        step = lambda: V.veda_distill_loss_grad(p, att.desc_q, att.desc_k, att.mlp_q, att.mlp_k, mp, rows, loss,
                                                gq, gk, dws)
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.map_steps):
            step()
        e1.record()
        torch.cuda.synchronize()
        V.veda_sync_status()
        dist = {"ms": e0.elapsed_time(e1) / args.map_steps, "loss": float(loss.item())}
    nts = np.asarray(p.nt_per_head)
    keys = (counts * nts[None, :] * w.S).astype(np.float64)     # subset rows x all key slots
    flops = float((2.0 * w.S * w.d * keys).sum())               # one Q K^T sweep
    exps = float((w.S * keys).sum())
    peaks, src = load_peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    mufu_peak = 16 * 148 * peaks.get("sm_max_mhz", 1965.0) * 1e6   # ex2 per second at the maximum clock
    return {"ms": ms, "layout": args.layout, "subset_rows": int(counts.sum()), "flops": flops, "exps": exps, "tflops": tflops,
            "distill_step": dist,
            "roofline": {"bound": "tensor+exp", "achieved": tflops, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
                         "frac_of_sustained": tflops / peaks["bf16_tflops_sustained"],
                         "exp_rate": exps / (ms * 1e-3), "exp_peak_mufu": mufu_peak,
                         "peak_source": f"{src} bf16 burst (a few launches at full clock); "
                                        "exp peak = 16 ex2/clk/SM at the maximum clock"}}


def bench_config(w, args, world, flops):
    """The workload description shared by both arms' JSON lines."""
    tensor_mb = w.B * w.heads * w.N * w.d * 2 / 1e6
    return {"workload": WORKLOAD_NAMES.get(args.workload, args.workload), "preset": args.workload,
            "grid": [w.T, w.H, w.W], "tokens": w.N, "heads": w.heads, "d": w.d, "S": w.S,
            "keep": w.keep, "tilings": "per head from " + ",".join(str(t) for t in sorted(set(w.tilings))),
            "global_batch": w.B * world, "seq_len": w.N, "parallelism": f"replicas x{world}",
            "kept_tile_flops_per_layer": flops, "layout": args.layout,
            "l2": "inputs (3 x %.0f MB) larger than L2; no flush" % tensor_mb}


def attention_sustained(V, p, att, qd, kd, vd, out, args, flops, local):
    """The attention kernel alone, back to back for args.attn_sustain seconds,
    with the SM clock and board power sampled meanwhile: shows the clock the
    kernel settles at under the power cap."""
    def launch():
        if args.layout == "grid":
            V.veda_tile_sparse_attn_grid(p, qd, kd, vd, att.idx, out)
        else:
            V.veda_tile_sparse_attn(p, att.qp, att.kp, att.vp, att.idx, att.op)
    clocks = Clocks(local)
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n = 0
    t0 = time.time()
    e0.record()
    while time.time() - t0 < args.attn_sustain:
        for _ in range(10):
            launch()
        n += 10
        torch.cuda.synchronize()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / n
    # Operand bytes each launch streams from L2 into shared memory: every kept
    # (Q tile, K tile) pair fetches its K and V tile, every Q tile is fetched
    # once (the kept pairs follow from the kept-tile FLOPs, 4 S^2 d per pair).
    tile_bytes = p.S * p.d * 2
    pairs = flops / (4.0 * p.S * p.S * p.d)
    q_tiles = p.B * sum(p.nt_per_head)
    l2_bytes = pairs * 2 * tile_bytes + q_tiles * tile_bytes
    return {"launches": n, "ms_per_launch": ms, "tflops": flops / (ms * 1e-3) / 1e12, "clocks": clk,
            "l2_to_smem_bytes_per_launch": l2_bytes, "l2_to_smem_tb_per_s": l2_bytes / (ms * 1e-3) / 1e12}


def overlap_measure(V, w, qd, kd, vd, mlp, out_ref, args, dev):
    """Prototype of selection overlapped with attention: the heads split into
    args.overlap_groups groups (one Problem and VedaAttention each, on head
    slices of the same tensors), groups alternating between two streams, so
    that group g+1's TripPool, estimator and top-k can run beside group g's
    attention.  Returns ms per layer (CUDA events around the whole layer,
    after both streams join) and whether the output matches the one-stream
    layer bit for bit."""
    if args.layout != "grid" or w.B != 1:
        return {"skipped": "grid layout with B = 1 only (head slices must be contiguous)"}
    G = args.overlap_groups
    bounds = [round(i * w.heads / G) for i in range(G + 1)]
    groups = []
    for g in range(G):
        h0, h1 = bounds[g], bounds[g + 1]
        pg = V.Problem(w.B, h1 - h0, w.d, w.S, (w.T, w.H, w.W), w.tilings[h0:h1])
        mg = tuple(t[h0:h1].contiguous() for t in mlp)
        att = V.VedaAttention(pg, mg, mg, w.keep, device=dev, layout="grid")
        sl = lambda t: t[:, h0:h1]
        groups.append((pg, att, sl(qd), sl(kd), sl(vd)))
    out = torch.empty_like(out_ref)
    streams = [torch.cuda.current_stream(), torch.cuda.Stream()]
    start, join = torch.cuda.Event(), torch.cuda.Event()

    def layer():
        start.record(streams[0])
        streams[1].wait_event(start)
        for g, (pg, att, qg, kg, vg) in enumerate(groups):
            st = streams[g % 2]
            with torch.cuda.stream(st):
                att(qg, kg, vg, out[:, bounds[g]:bounds[g + 1]], stream=st.cuda_stream)
        join.record(streams[1])
        streams[0].wait_event(join)

    for _ in range(3):
        layer()
    torch.cuda.synchronize()
    V.veda_sync_status()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n = max(3, args.steps // 2)
    e0.record(streams[0])
    for _ in range(n):
        layer()
    e1.record(streams[0])
    torch.cuda.synchronize()
    V.veda_sync_status()
    return {"groups": G, "streams": 2, "ms_per_layer": e0.elapsed_time(e1) / n, "steps": n,
            "output_identical": bool(torch.equal(out, out_ref))}


def backward_measure(V, w, p, att, qd, kd, vd, args, flops, rank, dev):
    """The attention backward (dQ, dK, dV over the selected tiles) after the
    layer's forward, timed over args.bwd_steps calls with CUDA events.  Its
    algorithmic work is the usual 2.5x the forward's kept-tile FLOPs (five
    S x S x d products per kept pair: S, dP, dV, dQ, dK); the kernels run
    seven (S and dP once for dQ and once for dK/dV)."""
    from veda_synth import make_grad_out
    if args.layout != "grid":
        return {"skipped": "the backward runs on grid-order tensors (--layout grid)"}
    o = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((p.B, p.heads, p.N), dtype=torch.float32, device=dev)
    V.veda_tile_sparse_attn_grid(p, qd, kd, vd, att.idx, o, lse)
    do = make_grad_out(w, seed=rank + 4).to(dev)
    grads = [torch.empty_like(qd) for _ in range(3)]
    ws = torch.empty(V.veda_attn_backward_workspace(p, int(att.idx.shape[-1])), dtype=torch.uint8, device=dev)
    step = lambda: V.veda_tile_sparse_attn_backward_grid(p, qd, kd, vd, o, lse, do, att.idx, *grads, ws)
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.bwd_steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    V.veda_sync_status()
    ms = e0.elapsed_time(e1) / args.bwd_steps
    peaks, src = load_peaks()
    alg = 2.5 * flops / (ms * 1e-3) / 1e12
    return {"ms": ms, "algorithmic_flops": 2.5 * flops, "tflops": alg,
            "executed_tflops": 3.5 * flops / (ms * 1e-3) / 1e12,
            "frac_of_burst_peak": alg / peaks["bf16_tflops"],
            "frac_of_sustained_peak": alg / peaks["bf16_tflops_sustained"], "peak_source": src,
            "ratio_to_forward_attention": None}


SWEEP = (("sweep61k", 61440), ("sweep123k", 122880), ("sweep246k", 245760))


def loglog_slope(xs, ys):
    """Least-squares slope of log(y) against log(x)."""
    lx, ly = np.log(np.asarray(xs, float)), np.log(np.asarray(ys, float))
    return float(np.polyfit(lx, ly, 1)[0])


def sweep_measure(V, args, dev):
    """The token sweep (15/30/60 x 64 x 64 grids, 24 heads, (2,8,8) tiles):
    one layer per point at keep 5% and at a fixed k = 26 selected tiles per Q
    tile (about 5% at 61,440 tokens), timed with CUDA events.  At a fixed
    ratio the kept work grows as N^2; at fixed k it grows as N, and the
    log-log slope of ms/layer against tokens shows how close to linear the
    layer is.  Inputs follow the synthetic recipe, drawn on the device."""
    import dataclasses
    from veda_synth import PRESETS, make_mlp, make_qkv_on_device
    points = []
    for mode in ("keep5", "k26"):
        for name, tokens in SWEEP:
            w = PRESETS[name]
            if mode == "k26":
                nt = max(tiles_per_head(w))
                w = dataclasses.replace(w, keep=26.0 / nt)
            p = V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)
            q, k, v = make_qkv_on_device(w, dev, seed=0)
            m = make_mlp(w, seed=1)
            mlp = tuple(t.to(dev) for t in (m.w1, m.b1, m.w2, m.b2))
            att = V.VedaAttention(p, mlp, mlp, w.keep, device=dev, layout="grid")
            out = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device=dev)
            ks, _ = p.keep_count(w.keep)
            flops = kept_flops(p.nt_per_head, ks, w.B, w.S, w.d)
            for _ in range(3):
                att(q, k, v, out)
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            sel_ms, attn_ms, layer_ms = [], [], []
            for _ in range(args.sweep_steps):
                ev[0].record()
                att.select(q, k, v)
                ev[1].record()
                V.veda_tile_sparse_attn_grid(p, q, k, v, att.idx, out)
                ev[2].record()
                torch.cuda.synchronize()
                sel_ms.append(ev[0].elapsed_time(ev[1]))
                attn_ms.append(ev[1].elapsed_time(ev[2]))
                layer_ms.append(ev[0].elapsed_time(ev[2]))
            V.veda_sync_status()
            lm, am = float(np.median(layer_ms)), float(np.median(attn_ms))
            points.append({"workload": name, "mode": mode, "tokens": tokens, "k": int(ks[0]),
                           "ms_per_layer": lm, "select_ms": float(np.median(sel_ms)), "attention_ms": am,
                           "kept_tile_flops": flops, "attn_tflops": flops / (am * 1e-3) / 1e12,
                           "layer_tflops": flops / (lm * 1e-3) / 1e12})
            del q, k, v, out, att
            torch.cuda.empty_cache()
    res = {"points": points, "steps": args.sweep_steps, "timing": "median of per-step CUDA events"}
    for mode in ("keep5", "k26"):
        pts = [x for x in points if x["mode"] == mode]
        res[f"loglog_slope_{mode}"] = loglog_slope([x["tokens"] for x in pts], [x["ms_per_layer"] for x in pts])
    return res


def run_ours(args, world, rank, local):
    import tile_sparse_attention_head_b200 as V
    from veda_synth import PRESETS, make_mlp, make_qkv

    w = workload_for(args)
    p = V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)
    q, k, v = make_qkv(w, seed=rank)
    m = make_mlp(w, seed=1)
    dev = torch.device("cuda", torch.cuda.current_device())
    mlp = tuple(t.to(dev) for t in (m.w1, m.b1, m.w2, m.b2))
    att = V.VedaAttention(p, mlp, mlp, w.keep, device=dev, layout=args.layout)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device=dev)
    ks, _ = p.keep_count(w.keep)
    flops = kept_flops(p.nt_per_head, ks, w.B, w.S, w.d)
    stream = torch.cuda.current_stream()

    # The step's stages, in order, for per-stage events on one instrumented
    # step (the same calls VedaAttention makes).
    def score():
        V.veda_tile_score_topk(p, att.desc_q, att.desc_k, att.mlp_q, att.mlp_k, att.keep, att.idx, None,
                               att.workspace)

    # Rows of more than 512 tiles (e <= 64) score through the score matrix in
    # the workspace: the score GEMM is one more launch.
    sel_extra = 1 if (w.e <= 64 and p.nt_max > 512) else 0
    if args.layout == "tile":
        stages = [("permute_tripool_qk", lambda: (V.veda_tile_permute_tripool(p, qd, att.qp, att.desc_q),
                                                  V.veda_tile_permute_tripool(p, kd, att.kp, att.desc_k))),
                  ("permute_v", lambda: V.veda_tile_permute(p, vd, att.vp)),
                  ("score_topk", score),
                  ("attention", lambda: V.veda_tile_sparse_attn(p, att.qp, att.kp, att.vp, att.idx, att.op)),
                  ("unpermute", lambda: V.veda_tile_unpermute(p, att.op, out))]
        launches_per_step = 7 + sel_extra   # 2 permute+TripPool, permute, estimator, top-k, attention, unpermute
    else:
        stages = [("tripool_qk", lambda: (V.veda_tripool_grid(p, qd, att.desc_q),
                                          V.veda_tripool_grid(p, kd, att.desc_k))),
                  ("score_topk", score),
                  ("attention", lambda: V.veda_tile_sparse_attn_grid(p, qd, kd, vd, att.idx, out))]
        n_tilings = len(set(w.tilings))
        # 2 TripPool, estimator, top-k (+ the score GEMM), attention per 8 tilings
        launches_per_step = 4 + sel_extra + (n_tilings + 7) // 8

    def step(ev=None):
        if ev is None:
            att(qd, kd, vd, out)
            return
        ev[0].record()
        for si, (_, fn) in enumerate(stages):
            fn()
            ev[si + 1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    V.veda_sync_status()

    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    t0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    h1 = time.time()
    barrier(world)
    time.sleep(0.15)
    clocks.window(h0, h1)
    clk = clocks.stop()
    V.veda_sync_status()
    ms_total = max_over_ranks(t0.elapsed_time(t1), world)
    ms_step = ms_total / args.steps
    stage_ms = {name: float(np.mean([ev[si].elapsed_time(ev[si + 1]) for ev in evs]))
                for si, (name, _) in enumerate(stages)}
    attn_ms = max_over_ranks(stage_ms["attention"], world)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.pin_memory() for t in (q, k, v))
        oh = torch.empty(p.grid_shape(), dtype=torch.bfloat16).pin_memory()
        host = V.VedaAttentionHost(p, mlp, mlp, w.keep, device=dev)
        for _ in range(2):
            host(qh, kh, vh, oh)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        n_e2e = max(3, args.steps // 4)
        for _ in range(n_e2e):
            host(qh, kh, vh, oh)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        nbytes = lambda t: t.numel() * t.element_size()
        e2e = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": nbytes(q) + nbytes(k) + nbytes(v), "d2h_bytes_per_step": nbytes(oh),
               "steps": n_e2e}

    peaks, peak_src = load_peaks()
    achieved = flops / (attn_ms * 1e-3) / 1e12
    kst, vst, _ = V.veda_attn_config(p, att.k_max)
    # The peak follows the clock record of the timed region: the burst GEMM
    # figure when the SM clock sat at its maximum, the sustained (power-capped)
    # one when the cap held it down.  Both fractions are reported.
    peak, basis = choose_peak(peaks, clk, peak_src)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "traffic": attn_traffic(args.workload, args.layout),
                "traffic_unit": "bytes per launch (DRAM read + write)",
                "kernel": f"sparse_attn_kernel<{w.d},{w.S},{kst},{vst},{'grid' if args.layout == 'grid' else 'tile'}>",
                "peak_source": basis,
                "frac_of_burst": achieved / peaks["bf16_tflops"],
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]}
    sustained = None
    if args.attn_sustain > 0:
        sustained = attention_sustained(V, p, att, qd, kd, vd, out, args, flops, local)
    useful = useful_flops(w, att.idx.cpu().numpy())
    tmap = tile_map_measure(V, w, p, qd, kd, args, rank, att) if args.map else None
    bwd = backward_measure(V, w, p, att, qd, kd, vd, args, flops, rank, dev) if args.bwd else None
    overlap = None
    if args.overlap_groups > 1:
        att(qd, kd, vd, out)
        overlap = overlap_measure(V, w, qd, kd, vd, mlp, out, args, dev)
        if "ms_per_layer" in overlap:
            overlap["one_stream_ms_per_layer"] = ms_step
    if bwd is not None and "ms" in bwd:
        bwd["ratio_to_forward_attention"] = bwd["ms"] / attn_ms
    res = {"metric": METRIC, "value": weak_scaling_value(flops, ms_step, world), "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": bench_config(w, args, world, flops),
           "ms_per_layer": ms_step, "stage_ms": stage_ms, "attn_tflops": achieved,
           "useful_flops_per_layer": useful, "attn_useful_tflops": useful / (attn_ms * 1e-3) / 1e12,
           "pct_of_bf16_peak": 100.0 * achieved / peaks["bf16_tflops"],
           "roofline": roofline, "gpu_launches": launches_per_step * args.steps, "clocks": clk, "e2e": e2e}
    if sustained is not None:
        res["attention_sustained"] = sustained
    if tmap is not None:
        res["tile_map"] = tmap
    if world == 1 and not args.no_sweep:
        res["sweep"] = sweep_measure(V, args, dev)
    if bwd is not None:
        res["backward"] = bwd
    if overlap is not None:
        res["overlap_prototype"] = overlap
    return res, (w, p, ks, flops)


def cpu_sample_oracle(w, p_nts, ks, heads=1, tiles=None, seed=0):
    """Oracle over a bounded sample: `heads` heads, full permute/pool/score/top-k, attention for
    `tiles` Q tiles per head (all if None).  Returns (seconds, kept FLOPs processed, description)."""
    from oracle import veda_oracle as O
    from veda_synth import make_mlp, make_qkv
    q, k, v = make_qkv(w, seed=seed, heads=heads)
    m = make_mlp(w, seed=1, heads=heads)
    mlp = tuple(t.numpy().astype(np.float64) for t in (m.w1, m.b1, m.w2, m.b2))
    grid = (w.T, w.H, w.W)
    tl = list(w.tilings[:heads])
    qd, kd, vd = (t.to(torch.float64).numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    qp, kp, vp = (O.tile_permute(a, grid, tl, w.S) for a in (qd, kd, vd))
    dq, dk = O.tripool(qp, grid, tl, w.S), O.tripool(kp, grid, tl, w.S)
    idx, _ = O.score_topk(dq, dk, grid, tl, w.S, mlp, mlp, float(np.float32(w.keep)))
    done = 0.0
    scale = 1 / math.sqrt(w.d)
    for h in range(heads):
        tab = O.slot_table(grid, tl[h])
        nt = p_nts[h]
        sel = range(nt) if tiles is None else range(min(tiles, nt))
        for i in sel:
            O.attention_tile(qp[0, h], kp[0, h], vp[0, h], tab, i, idx[0, h, i], w.S, scale)
            done += ks[h] * 4 * w.S * w.S * w.d
    secs = time.perf_counter() - t0
    desc = (f"{heads} head(s) of {w.name}: full permute+TripPool+score/top-k, attention for "
            f"{'all' if tiles is None else tiles} Q tiles per head")
    return secs, done, desc


def run_reference(args, world, rank):
    """The fp64 CPU oracle as the reference arm, timed on the host cores."""
    from oracle import veda_oracle as O
    w = workload_for(args)
    nts, _ = O.tile_layout((w.T, w.H, w.W), w.tilings)
    ks = [O.keep_count(n, float(np.float32(w.keep))) for n in nts]
    tiles = args.ref_tiles
    for _ in range(args.warmup):
        cpu_sample_oracle(w, nts, ks, heads=1, tiles=max(1, tiles // 8))
    secs, flops = 0.0, 0.0
    desc = ""
    for s in range(args.steps):
        t, f, desc = cpu_sample_oracle(w, nts, ks, heads=1, tiles=tiles, seed=s)
        secs += t
        flops += f
    value = flops / secs / 1e12
    cores = os.cpu_count()
    layer_flops = kept_flops(nts, ks, w.B, w.S, w.d)
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": bench_config(w, args, world, layer_flops),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan14b")
    ap.add_argument("--layout", choices=["tile", "grid"], default="grid",
                    help="tile-major copies (permute/unpermute steps) or grid order throughout")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--keep", type=float, default=None, help="override the preset's keep ratio")
    ap.add_argument("--fixed-k", type=int, default=None,
                    help="keep ratio k / NT_max, i.e. k selected tiles per Q tile (the fixed-k token sweep)")
    ap.add_argument("--map", action="store_true", help="also time the max-pooled tile map (10%% of Q tiles)")
    ap.add_argument("--map-steps", type=int, default=5)
    ap.add_argument("--bwd", action="store_true", help="also time the attention backward (dQ, dK, dV)")
    ap.add_argument("--bwd-steps", type=int, default=5)
    ap.add_argument("--attn-sustain", type=float, default=0.0,
                    help="also run the attention kernel back to back for this many seconds, sampling clock and power")
    ap.add_argument("--overlap-groups", type=int, default=0,
                    help="also time the layer as G head groups on two streams (selection beside attention)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the token sweep record (N = 1 only)")
    ap.add_argument("--sweep-steps", type=int, default=5)
    ap.add_argument("--ref-tiles", type=int, default=24, help="Q tiles per oracle sample (reference arm)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return

    world, rank, local = dist_setup(args.gpus)
    res, (w, p, ks, flops) = run_ours(args, world, rank, local)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            # bounded sample: 5 whole heads (~12-15 s of CPU work on the bench host)
            secs, done, desc = cpu_sample_oracle(w, p.nt_per_head, ks, heads=min(5, w.heads), tiles=None)
            res["cpu_baseline"] = {"value": done / secs / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
                                   "kind": "oracle", "sample": desc, "seconds": secs}
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

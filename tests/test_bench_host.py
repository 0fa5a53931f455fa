"""Host-side logic of bench.py, on the CPU: tile token counts, useful FLOPs,
the fixed-k sweep override, and the multi-rank timing reduction on two gloo
ranks (the path bench.py takes under torchrun, minus the GPUs)."""
import argparse
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import veda_oracle as O  # noqa: E402
from veda_synth import PRESETS  # noqa: E402

from parity import SMALL  # noqa: E402


@pytest.mark.parametrize("w", SMALL + [PRESETS["wan14b"]], ids=[w.name for w in SMALL] + ["wan14b"])
def test_tile_token_counts_match_the_oracle_layout(w):
    cnt = bench.tile_token_counts(w)
    nts, ntmax = O.tile_layout((w.T, w.H, w.W), w.tilings)
    assert cnt.shape == (w.heads, ntmax)
    assert bench.tiles_per_head(w) == list(nts)
    for h in range(w.heads):
        tab = O.slot_table((w.T, w.H, w.W), w.tilings[h])
        ref = (tab.reshape(nts[h], w.S) >= 0).sum(axis=1)
        np.testing.assert_array_equal(cnt[h, :nts[h]], ref)
        assert np.all(cnt[h, nts[h]:] == 0)


def test_useful_flops_of_a_dense_selection_is_n_squared():
    w = SMALL[1]
    nts, ntmax = O.tile_layout((w.T, w.H, w.W), w.tilings)
    idx = np.full((w.B, w.heads, ntmax, ntmax), -1, dtype=np.int32)
    for h in range(w.heads):
        idx[:, h, :nts[h], :nts[h]] = np.arange(nts[h])
    N = w.T * w.H * w.W
    assert bench.useful_flops(w, idx) == pytest.approx(w.B * w.heads * N * N * 4 * w.d)
    # with -1 padding and invalid Q rows nothing is counted
    idx[:, :, :, 1:] = -1
    cnt = bench.tile_token_counts(w)
    expect = sum(int((cnt[h, :nts[h]] * cnt[h, 0]).sum()) for h in range(w.heads)) * w.B * 4 * w.d
    assert bench.useful_flops(w, idx) == pytest.approx(expect)


@pytest.mark.parametrize("name", ["sweep61k", "sweep123k", "sweep246k"])
def test_fixed_k_override_keeps_k_tiles(name):
    args = argparse.Namespace(workload=name, keep=None, fixed_k=26)
    w = bench.workload_for(args)
    nts, _ = O.tile_layout((w.T, w.H, w.W), w.tilings)
    assert {O.keep_count(n, float(np.float32(w.keep))) for n in nts} == {26}


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        out[rank] = ms
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}
    assert bench.weak_scaling_value(7.8e12, 15.0, 2) == pytest.approx(2 * 7.8e12 / 15e-3 / 1e12)


def _smi_line(ts, sm, mx=1965, pw=500.0, cap="Not Active", mask="0x0000000000000000"):
    return (f"{ts}, 0, {sm}, {mx}, {pw}, {mask}, Not Active, Not Active, Not Active, {cap}")


def test_clock_active_mask_is_decoded():
    """Every bit of clocks_event_reasons.active is named in the record, and a
    hardware power brake holding the clock down selects the sustained peak
    like the software power cap does."""
    lines = [_smi_line("2026/12/02 12:00:00.000", 1600, mask="0x0000000000000080"),
             _smi_line("2026/12/02 12:00:00.020", 1610, mask="0x0000000000000084", cap="Active"),
             _smi_line("2026/12/02 12:00:00.040", 1620, mask="0x0000000000000001")]
    clk = bench.Clocks.summarize(bench.Clocks.parse(lines))
    assert clk["reasons"] == ["sw_power_cap"]
    assert clk["reasons_active"] == ["gpu_idle", "hw_power_brake_slowdown", "sw_power_cap"]
    assert clk["sm_mhz_samples"] == [1600.0, 1610.0, 1620.0]
    peaks = {"bf16_tflops": 1674.3, "bf16_tflops_sustained": 1409.4, "hbm_gbs": 6541.8}
    brake_only = {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "reasons": [], "reasons_active": ["hw_power_brake_slowdown"],
                  "samples": 3, "window": "timed region"}
    peak, basis = bench.choose_peak(peaks, brake_only, "measured")
    assert peak == 1409.4 and "hw_power_brake_slowdown" in basis
    idle_only = dict(brake_only, reasons_active=["gpu_idle"])
    assert bench.choose_peak(peaks, idle_only, "measured")[0] == 1674.3


def test_clock_summary_keeps_only_the_timed_region():
    import datetime
    base = datetime.datetime(2026, 12, 2, 12, 0, 0)
    lines = []
    for i in range(20):                       # one sample every 50 ms, 1 s in all
        t = base + datetime.timedelta(milliseconds=50 * i)
        sm = 1965 if 6 <= i <= 9 else 1400    # the region runs at full clock, the rest does not
        lines.append(_smi_line(t.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3], sm, cap="Active" if i > 15 else "Not Active"))
    rows = bench.Clocks.parse(lines)
    assert len(rows) == 20
    t0 = (base + datetime.timedelta(milliseconds=290)).timestamp()
    t1 = (base + datetime.timedelta(milliseconds=460)).timestamp()
    clk = bench.Clocks.summarize(rows, t0, t1)
    assert clk["samples"] == 4 and clk["sm_mhz"] == 1965 and clk["reasons"] == []
    # a region shorter than the sampling interval takes the first sample after its start
    t0 = (base + datetime.timedelta(milliseconds=810)).timestamp()
    clk = bench.Clocks.summarize(rows, t0, t0 + 0.01)
    assert clk["samples"] == 1 and clk["sm_mhz"] == 1400 and clk["reasons"] == ["sw_power_cap"]


def test_peak_follows_the_clock_record():
    peaks = {"bf16_tflops": 1674.3, "bf16_tflops_sustained": 1409.4, "hbm_gbs": 6541.8}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3, "window": "timed region"}
    capped = {"sm_mhz": 1597.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 30,
              "window": "timed region"}
    assert bench.choose_peak(peaks, at_max, "measured")[0] == 1674.3
    peak, basis = bench.choose_peak(peaks, capped, "measured")
    assert peak == 1409.4 and "sustained" in basis and "sw_power_cap" in basis
    assert bench.choose_peak(peaks, None, "measured")[0] == 1674.3
    # below the maximum with no reason recorded: the burst figure still applies
    low = dict(at_max, sm_mhz=1852.0)
    assert bench.choose_peak(peaks, low, "measured")[0] == 1674.3
    # the power cap flagged while the clock stays at its maximum: still burst
    flagged = dict(at_max, reasons=["sw_power_cap"])
    assert bench.choose_peak(peaks, flagged, "measured")[0] == 1674.3


def test_loglog_slope():
    xs = [61440, 122880, 245760]
    assert bench.loglog_slope(xs, [2.0 * x for x in xs]) == pytest.approx(1.0)
    assert bench.loglog_slope(xs, [3e-9 * x * x for x in xs]) == pytest.approx(2.0)

"""CPU-only checks of the C-ABI library: it loads, exports every entry point
declared in include/veda.h, and its host-side logic (layout, keep counts,
argument validation, workspace sizes) agrees with the oracle.  No call here
launches a kernel."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

from oracle import veda_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "veda.h")


@pytest.fixture(scope="module")
def V():
    import tile_sparse_attention_head_b200 as V
    return V


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(veda_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(V):
    syms = declared_symbols()
    assert len(syms) >= 15
    lib = ctypes.CDLL(V.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s


def test_library_is_built_for_sm100a(V):
    # The build command pins the architecture; the library must not carry a CPU path.
    from tile_sparse_attention_head_b200 import build
    cmd = " ".join(build.nvcc_command())
    assert "arch=compute_100a,code=sm_100a" in cmd


CASES = [((4, 8, 8), 64, [(1, 8, 8), (4, 4, 4)]),
         ((21, 30, 52), 128, [(2, 8, 8), (1, 8, 16), (8, 4, 4), (4, 4, 8)]),
         ((21, 45, 80), 128, [(2, 8, 8), (1, 8, 16), (8, 4, 4), (4, 4, 8)]),
         ((5, 13, 19), 64, [(1, 8, 8), (4, 4, 4), (2, 4, 8), (1, 1, 64)])]


@pytest.mark.parametrize("grid,S,tilings", CASES)
def test_layout_and_keep_counts_match_oracle(V, grid, S, tilings):
    p = V.Problem(1, len(tilings), 128, S, grid, tilings)
    nts, ntmax = O.tile_layout(grid, tilings)
    assert p.nt_per_head == nts and p.nt_max == ntmax
    for r in (0.01, 0.05, 0.1, 0.3, 0.5, 0.7, 1.0):
        ks, kmax = p.keep_count(r)
        rr = float(np.float32(r))
        assert ks == [O.keep_count(n, rr) for n in nts]
        assert kmax == max(ks)


def test_invalid_arguments_are_rejected_on_the_host(V):
    B = V.binding
    with pytest.raises(V.VedaError) as e:
        V.Problem(1, 1, 96, 128, (2, 2, 2), [(2, 8, 8)])
    assert e.value.status == B.VEDA_ERR_UNSUPPORTED
    with pytest.raises(V.VedaError) as e:
        V.Problem(1, 1, 128, 128, (2, 2, 2), [(2, 8, 4)])        # pt*ph*pw != S
    assert e.value.status == B.VEDA_ERR_INVALID_ARG
    with pytest.raises(V.VedaError) as e:
        V.Problem(1, 1, 128, 96, (2, 2, 2), [(2, 8, 6)])
    assert e.value.status == B.VEDA_ERR_UNSUPPORTED
    with pytest.raises(V.VedaError):
        V.Problem(0, 1, 128, 128, (2, 2, 2), [(2, 8, 8)])
    with pytest.raises(V.VedaError):
        V.Problem(1, 1, 128, 128, (0, 2, 2), [(2, 8, 8)])
    p = V.Problem(1, 1, 128, 128, (4, 8, 8), [(2, 8, 8)])
    with pytest.raises(V.VedaError) as e:
        p.keep_count(0.0)
    assert e.value.status == B.VEDA_ERR_INVALID_ARG
    with pytest.raises(V.VedaError):
        p.keep_count(1.5)
    lib = V.LIB
    # NULL tensors are refused before anything touches the GPU
    assert lib.veda_tile_permute(p.ref, None, None, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_tripool(p.ref, None, None, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_tile_sparse_attn(p.ref, None, None, None, None, 1, 0.0, None, None, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_tripool_grid(p.ref, None, None, None) == B.VEDA_ERR_INVALID_ARG
    assert (lib.veda_tile_sparse_attn_grid(p.ref, None, None, None, None, 1, 0.0, None, None, None)
            == B.VEDA_ERR_INVALID_ARG)
    assert b"non-NULL" in lib.veda_last_error() or b"NULL" in lib.veda_last_error()
    # k_max < 1 and misaligned grid-order pointers (never dereferenced on the host)
    assert lib.veda_tile_sparse_attn_grid(p.ref, 256, 256, 256, 256, 0, 0.0, 256, None, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_tile_sparse_attn_grid(p.ref, 8, 256, 256, 256, 1, 0.0, 256, None, None) == B.VEDA_ERR_INVALID_ARG
    # misaligned pointers are refused too
    assert lib.veda_tile_permute(p.ref, 8, 16, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_set_wait_timeout_ns(0) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_selftest_wait_timeout(10**12, None) == B.VEDA_ERR_INVALID_ARG


def test_workspace_sizes(V):
    p = V.Problem(2, 3, 64, 64, (5, 13, 19), [(1, 8, 8), (4, 4, 4), (2, 4, 8)])
    e = 32
    assert V.veda_score_topk_workspace(p, e) >= 4 * 2 * 2 * 3 * p.nt_max * e
    R = 7
    assert V.veda_tile_map_workspace(p, R) >= 4 * 2 * 3 * R * (p.nt_max * 64 + 64)
    with pytest.raises(V.VedaError):
        V.veda_score_topk_workspace(p, 3)


def test_score_workspace_holds_the_score_matrix_for_long_rows(V):
    """Rows of more than 512 tiles score through the fp32 score matrix in the
    workspace (e <= 64); shorter rows, and e = 128, keep their scores in shared
    memory and need only the estimator features."""
    r256 = lambda x: (x + 255) // 256 * 256
    def phi(p, e):
        return r256(4 * 2 * p.B * p.heads * p.nt_max * e)
    long = V.Problem(1, 4, 128, 128, (21, 45, 80), [(2, 8, 8), (8, 4, 4), (1, 8, 16), (4, 4, 8)])
    assert long.nt_max == 720
    pad = (long.nt_max + 3) // 4 * 4
    for e in (16, 32, 64):
        assert V.veda_score_topk_workspace(long, e) == phi(long, e) + r256(4 * long.B * long.heads * long.nt_max * pad)
    assert V.veda_score_topk_workspace(long, 128) == phi(long, 128)
    short = V.Problem(2, 3, 128, 128, (21, 30, 52), [(2, 8, 8), (8, 4, 4), (1, 8, 16)])
    assert short.nt_max <= 512
    for e in (16, 32, 64, 128):
        assert V.veda_score_topk_workspace(short, e) == phi(short, e)


def test_attention_config_query(V):
    """Ring depths and shared memory of the attention launch, computed on the host."""
    p = V.Problem(1, 2, 128, 128, (21, 45, 80), [(2, 8, 8), (8, 4, 4)])
    ks, vs, smem = V.veda_attn_config(p, 36)
    assert (ks, vs) == (3, 3) and smem <= 232448
    # a long selection list grows the bookkeeping past the 3/3 budget
    ks, vs, smem2 = V.veda_attn_config(p, 400)
    assert (ks, vs) == (3, 2) and smem2 <= 232448
    # 16 KB tiles (d = 64) take four stages of each
    p64 = V.Problem(1, 1, 64, 64, (4, 8, 8), [(1, 8, 8)])
    assert V.veda_attn_config(p64, 2)[:2] == (4, 4)
    with pytest.raises(V.VedaError):
        V.veda_attn_config(p, 0)


def test_distill_entry_points_validate_on_the_host(V):
    B = V.binding
    p = V.Problem(1, 2, 64, 64, (4, 8, 8), [(1, 8, 8), (4, 4, 4)])
    nt = p.nt_max
    # workspace: phi + hidden + dL/ds + row losses + dphi (+ count), each rounded to 256 bytes
    r256 = lambda x: (x + 255) // 256 * 256
    bh, hidden, e, R = 2, 128, 32, 3
    expect = (r256(4 * 2 * bh * nt * e) + r256(4 * 2 * bh * nt * hidden) + r256(4 * bh * R * nt) + r256(4 * bh * R)
              + r256(4 * 2 * bh * nt * e) + 256)
    assert V.veda_distill_workspace(p, hidden, e, R) == expect
    with pytest.raises(V.VedaError):
        V.veda_distill_workspace(p, hidden, 24, R)     # e not in {16, 32, 64, 128}
    with pytest.raises(V.VedaError):
        V.veda_distill_workspace(p, hidden, e, 0)
    lib = V.LIB
    m = B.veda_mlp(256, 256, 256, 256, hidden, e)
    g = B.veda_mlp_grad(256, 256, 256, 256)
    ok_ws = 4096
    # NULL tensors, a misaligned workspace and a short workspace are refused before any launch
    assert lib.veda_distill_loss_grad(p.ref, None, 256, ctypes.byref(m), ctypes.byref(m), 256, 256, R, 256,
                                      ctypes.byref(g), ctypes.byref(g), ok_ws, 1 << 30, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_distill_loss_grad(p.ref, 256, 256, ctypes.byref(m), ctypes.byref(m), 256, 256, R, 256,
                                      ctypes.byref(g), ctypes.byref(g), 4097, 1 << 30, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_distill_loss_grad(p.ref, 256, 256, ctypes.byref(m), ctypes.byref(m), 256, 256, R, 256,
                                      ctypes.byref(g), ctypes.byref(g), ok_ws, 16, None) == B.VEDA_ERR_INVALID_ARG
    bad = B.veda_mlp_grad(256, 0, 256, 256)
    assert lib.veda_distill_loss_grad(p.ref, 256, 256, ctypes.byref(m), ctypes.byref(m), 256, 256, R, 256,
                                      ctypes.byref(bad), ctypes.byref(g), ok_ws, 1 << 30, None) == B.VEDA_ERR_INVALID_ARG


def test_head_error_validates_on_the_host(V):
    B = V.binding
    p = V.Problem(1, 2, 64, 64, (4, 8, 8), [(1, 8, 8), (4, 4, 4)])
    lib = V.LIB
    assert lib.veda_head_error(p.ref, None, 256, 256, 256, 256, 4096, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_head_error(p.ref, 8, 256, 256, 256, 256, 4096, None) == B.VEDA_ERR_INVALID_ARG
    assert lib.veda_head_error(p.ref, 256, 256, 256, 256, 256, 16, None) == B.VEDA_ERR_INVALID_ARG   # short workspace


def test_attention_backward_validates_on_the_host(V):
    """Workspace size from its parts; NULL, misaligned and short-workspace calls
    are refused before any launch (pointers are never dereferenced)."""
    B = V.binding
    p = V.Problem(2, 3, 64, 64, (5, 13, 19), [(1, 8, 8), (4, 4, 4), (2, 4, 8)])
    nt, k_max = p.nt_max, 5
    r256 = lambda x: (x + 255) // 256 * 256
    bh, N, W = 6, 5 * 13 * 19, (p.nt_max + 31) // 32
    expect = r256(8 * bh * nt * 64) + r256(4 * bh * nt * W) + r256(4 * bh * (nt + 1)) + r256(4 * bh * nt * k_max)
    assert V.veda_attn_backward_workspace(p, k_max) == expect
    with pytest.raises(V.VedaError):
        V.veda_attn_backward_workspace(p, 0)
    lib = V.LIB
    f = lib.veda_tile_sparse_attn_backward_grid
    good = [256] * 7
    args = lambda ptrs, k=k_max, sc=0.0, outs=(256, 256, 256), ws=4096, nb=1 << 30: (
        p.ref, *ptrs, k, ctypes.c_float(sc), *outs, ws, nb, None)
    assert f(*args([None] + good[1:])) == B.VEDA_ERR_INVALID_ARG                 # NULL q
    assert f(*args(good[:4] + [None] + good[5:])) == B.VEDA_ERR_INVALID_ARG      # NULL lse
    assert f(*args(good, outs=(256, 256, None))) == B.VEDA_ERR_INVALID_ARG      # NULL dv
    assert f(*args(good[:5] + [8] + good[6:])) == B.VEDA_ERR_INVALID_ARG        # misaligned d_o
    assert f(*args(good, ws=4096 + 16)) == B.VEDA_ERR_INVALID_ARG               # workspace not 256-aligned
    assert f(*args(good, nb=expect - 1)) == B.VEDA_ERR_INVALID_ARG              # short workspace
    assert f(*args(good, k=0)) == B.VEDA_ERR_INVALID_ARG
    assert f(*args(good, sc=float("inf"))) == B.VEDA_ERR_INVALID_ARG


def test_host_tensors_are_refused_no_cpu_fallback(V):
    """The binding accepts device tensors only: a layer built on host memory
    fails loudly at construction instead of falling back to a CPU path."""
    import torch
    p = V.Problem(1, 1, 64, 64, (4, 8, 8), [(1, 8, 8)])
    hid, e = 128, 32
    mlp = (torch.zeros(1, hid, 192), torch.zeros(1, hid), torch.zeros(1, e, hid), torch.zeros(1, e))
    with pytest.raises(ValueError, match="CUDA tensor"):
        V.VedaAttention(p, mlp, mlp, 0.5, device="cpu", layout="tile")
    with pytest.raises(ValueError, match="CUDA tensor"):
        V.make_mlp(*mlp)

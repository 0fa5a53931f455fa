"""GPU test of veda_tile_score_topk_noalloc, the scoring entry point for
callers that cannot hand the library device scratch memory (for example a
plugin whose host framework owns all device memory, or a latency-critical
loop that must not call cudaMalloc).

The call goes straight through the C ABI (ctypes) and its results are
compared with the workspace-taking veda_tile_score_topk on the same inputs,
twice in a row on problems of different sizes, so the second call runs over
whatever the first one left in the library's built-in scratch array.  On
rows of more than 512 tiles the two entry points take different kernels (the
fused one without a workspace, the score-matrix one with it), and the
comparison checks that they select the same tiles.  The file is named to be
collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from veda_synth import PRESETS, Workload, make_mlp, make_qkv

from parity import PROBS_ABS, PROBS_REL, mlp_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import tile_sparse_attention_head_b200 as V
    return V


def _case(V, w, seed):
    p = V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)
    q, k, _ = make_qkv(w, seed=seed)
    m = make_mlp(w, seed=seed + 1)
    wts = mlp_device(m)
    mlp = V.make_mlp(*wts)
    dshape = (p.B, p.heads, p.nt_max, 3 * p.d)
    dq = torch.empty(dshape, dtype=torch.float32, device="cuda")
    dk = torch.empty_like(dq)
    xp = torch.empty(p.tile_shape(), dtype=torch.bfloat16, device="cuda")
    V.veda_tile_permute_tripool(p, q.cuda(), xp, dq)
    V.veda_tile_permute_tripool(p, k.cuda(), xp, dk)
    _, k_max = p.keep_count(w.keep)
    return p, dq, dk, mlp, wts, k_max


def _reference(V, p, dq, dk, mlp, keep, k_max):
    idx = torch.empty((p.B, p.heads, p.nt_max, k_max), dtype=torch.int32, device="cuda")
    probs = torch.empty((p.B, p.heads, p.nt_max, p.nt_max), dtype=torch.float32, device="cuda")
    ws = torch.empty(V.veda_score_topk_workspace(p, mlp.e) // 4 + 64, dtype=torch.float32, device="cuda")
    V.veda_tile_score_topk(p, dq, dk, mlp, mlp, keep, idx, probs, ws)
    return idx, probs


def _noalloc_c_call(V, p, dq, dk, mlp, keep, k_max):
    """Direct C-ABI call: no workspace argument exists."""
    idx = torch.full((p.B, p.heads, p.nt_max, k_max), -7, dtype=torch.int32, device="cuda")
    probs = torch.full((p.B, p.heads, p.nt_max, p.nt_max), float("nan"), dtype=torch.float32, device="cuda")
    status = V.LIB.veda_tile_score_topk_noalloc(
        p.ref, ctypes.c_void_p(dq.data_ptr()), ctypes.c_void_p(dk.data_ptr()), ctypes.byref(mlp),
        ctypes.byref(mlp), ctypes.c_float(keep), ctypes.c_void_p(idx.data_ptr()), k_max,
        ctypes.c_void_p(probs.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 0, V.LIB.veda_last_error().decode()
    return idx, probs


def test_noalloc_matches_workspace_entry_point_twice(V):
    big = Workload(name="odd128", T=5, H=19, W=27, B=2, heads=4, d=128, S=128,
                   tilings=((2, 8, 8), (1, 8, 16), (8, 4, 4), (4, 4, 8)), keep=0.2, hidden=256, e=64, bias="rff")
    small = PRESETS["tiny"]
    for w, seed in ((big, 0), (small, 3)):
        p, dq, dk, mlp, _wts, k_max = _case(V, w, seed)
        ref_idx, ref_probs = _reference(V, p, dq, dk, mlp, w.keep, k_max)
        idx, probs = _noalloc_c_call(V, p, dq, dk, mlp, w.keep, k_max)
        V.veda_sync_status()
        # Same kernels on the same inputs: the selection is identical, the
        # probabilities agree within the tolerance the parity tests use.
        assert torch.equal(idx, ref_idx)
        np.testing.assert_allclose(probs.cpu().numpy(), ref_probs.cpu().numpy(), rtol=PROBS_REL, atol=PROBS_ABS)


# Rows of more than 512 tiles: the workspace entry point scores through the
# fp32 score matrix it keeps in the workspace (tensor-core GEMM, then one warp
# per row), the no-alloc one through the fused kernel that keeps each CTA's
# scores in shared memory.  Both form the same tf32 products in the same order
# and select from the same fp32 scores, so the selections are identical.
LONG_ROWS = [
    Workload(name="rows720", T=24, H=40, W=44, B=1, heads=2, d=64, S=64, tilings=((4, 4, 4), (2, 4, 8)),
             keep=0.05, hidden=128, e=32, bias="rff"),
    Workload(name="rows770", T=26, H=42, W=40, B=1, heads=2, d=128, S=64, tilings=((4, 4, 4), (2, 4, 8)),
             keep=0.05, hidden=256, e=64, bias="rff"),
    Workload(name="rows1760", T=39, H=41, W=58, B=1, heads=2, d=64, S=64, tilings=((4, 4, 4), (2, 4, 8)),
             keep=0.05, hidden=128, e=32, bias="rff"),
    Workload(name="rows2200", T=50, H=44, W=60, B=1, heads=2, d=64, S=64, tilings=((4, 4, 4), (2, 4, 8)),
             keep=0.05, hidden=128, e=32, bias="rff"),
]


@pytest.mark.parametrize("w", LONG_ROWS, ids=[w.name for w in LONG_ROWS])
def test_noalloc_fused_kernel_matches_score_matrix_path(V, w):
    p, dq, dk, mlp, _wts, k_max = _case(V, w, 5)
    assert p.nt_max > 512
    ref_idx, ref_probs = _reference(V, p, dq, dk, mlp, w.keep, k_max)
    idx, probs = _noalloc_c_call(V, p, dq, dk, mlp, w.keep, k_max)
    V.veda_sync_status()
    assert torch.equal(idx, ref_idx)
    np.testing.assert_allclose(probs.cpu().numpy(), ref_probs.cpu().numpy(), rtol=PROBS_REL, atol=PROBS_ABS)


def test_noalloc_rejects_problems_beyond_its_scratch(V):
    w = PRESETS["sweep246k"]           # 2 * 24 heads * 1920 tiles * 64 floats > 16 MiB
    p = V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)
    dummy = torch.zeros(16, device="cuda")
    hid, e = 256, 64
    mlp = V.binding.veda_mlp(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), hid, e)
    status = V.LIB.veda_tile_score_topk_noalloc(
        p.ref, ctypes.c_void_p(dummy.data_ptr()), ctypes.c_void_p(dummy.data_ptr()), ctypes.byref(mlp),
        ctypes.byref(mlp), ctypes.c_float(0.05), ctypes.c_void_p(dummy.data_ptr()), 96, None, None)
    assert status == V.binding.VEDA_ERR_UNSUPPORTED
    assert b"exceeds the built-in" in V.LIB.veda_last_error()

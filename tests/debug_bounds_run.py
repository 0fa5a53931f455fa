"""Runs the inference path, the tile map and the attention backward on the
small parity workloads through whichever library the binding loads, checks
that veda_sync_status reports no error after each call, and saves the
results to a file.  tests/test_gpu_debug_bounds.py runs it once with the
bounds-checked debug library (VEDA_DEBUG_BOUNDS=1, in a child process) and
once with the release library, and compares the two."""
from __future__ import annotations

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import tile_sparse_attention_head_b200 as V  # noqa: E402
from veda_synth import make_grad_out, make_map_rows, make_mlp, make_qkv  # noqa: E402

from parity import MANY_TILINGS, SMALL, mlp_device  # noqa: E402


def run_all() -> dict:
    out = {}
    for w in SMALL + [MANY_TILINGS]:
        p = V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)
        q, k, v = (t.cuda() for t in make_qkv(w, seed=0))
        md = mlp_device(make_mlp(w, seed=1))
        for layout in ("tile", "grid"):
            att = V.VedaAttention(p, md, md, w.keep, want_probs=True, want_lse=True, layout=layout)
            o = att(q, k, v)
            V.veda_sync_status()
            out[f"{w.name}/{layout}/o"] = o.cpu()
            out[f"{w.name}/{layout}/idx"] = att.idx.cpu()
            out[f"{w.name}/{layout}/lse"] = att.lse.cpu()
            out[f"{w.name}/{layout}/probs"] = att.probs.cpu()
            out[f"{w.name}/{layout}/desc_q"] = att.desc_q.cpu()
            if layout == "tile":
                rows = make_map_rows(p.nt_per_head, w.B, 0.3, seed=2).cuda()
                R = rows.shape[1]
                ws = torch.empty(V.veda_tile_map_workspace(p, R) // 4 + 64, dtype=torch.float32, device="cuda")
                mp = torch.empty((p.B, p.heads, R, p.nt_max), dtype=torch.float32, device="cuda")
                V.veda_tile_map_maxpool(p, att.qp, att.kp, rows, mp, ws)
                V.veda_sync_status()
                out[f"{w.name}/map"] = mp.cpu()
            else:
                do = make_grad_out(w, seed=4).cuda()
                grads = [torch.empty_like(q) for _ in range(3)]
                ws = torch.empty(V.veda_attn_backward_workspace(p, att.k_max), dtype=torch.uint8, device="cuda")
                V.veda_tile_sparse_attn_backward_grid(p, q, k, v, o, att.lse, do, att.idx, *grads, ws)
                V.veda_sync_status()
                for name, g in zip(("dq", "dk", "dv"), grads):
                    out[f"{w.name}/{name}"] = g.cpu()
    return out


if __name__ == "__main__":
    want_debug = os.environ.get("VEDA_DEBUG_BOUNDS") == "1"
    assert V.veda_bounds_checked() == want_debug, "the binding loaded the wrong library"
    if want_debug:
        # the reporting path: a deliberate failed check, no memory touched
        V.veda_selftest_bounds()
        try:
            V.veda_sync_status()
            raise AssertionError("the bounds self-test was not reported")
        except V.VedaError as e:
            assert e.status == V.binding.VEDA_ERR_BOUNDS, e
            assert "tile_map.cu" in str(e), e
        V.veda_sync_status()          # cleared
    res = run_all()
    torch.save(res, sys.argv[1])
    print(f"ok: {len(res)} results, bounds checked: {want_debug}")

"""GPU test of the bounds-checked debug build (libveda_debug.so, compiled with
-DVEDA_DEBUG_BOUNDS).  Its kernels check every index they compute -- tile ids
against the head's tile count, rows against the tensor's rows, selection
entries against [0, NT_h) -- and report a failed check through
veda_sync_status instead of touching the memory.

The small parity workloads (every tile size, head dim, ragged faces, B = 2,
ten tilings) run through the inference path in both layouts, the tile map and
the attention backward, once with the debug library and once with the
release library, each in a child process.  No check may fire, and the results
must agree.  The debug child also runs the self-test: a deliberate failed
check, with no memory touched, must come back as VEDA_ERR_BOUNDS.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _run(tmp_path, debug: bool):
    env = dict(os.environ)
    env["VEDA_DEBUG_BOUNDS"] = "1" if debug else "0"
    out = tmp_path / ("debug.pt" if debug else "release.pt")
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_run.py"), str(out)], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    return torch.load(out)


def test_debug_build_finds_no_bad_index_and_matches_release(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("veda_build", os.path.join(ROOT, "tile_sparse_attention_head_b200",
                                                                            "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build(debug=True)           # no-op when libveda_debug.so is up to date
    dbg = _run(tmp_path, True)
    rel = _run(tmp_path, False)
    assert dbg.keys() == rel.keys()
    for key in rel:
        a, r = dbg[key], rel[key]
        if a.dtype in (torch.int32, torch.bfloat16):
            assert torch.equal(a, r), key
        else:
            assert torch.allclose(a, r, rtol=1e-6, atol=1e-7, equal_nan=True), key

"""ctypes binding of libveda.so (the C ABI in include/veda.h).

Argument marshalling only: every function here checks tensor devices, dtypes
and shapes, passes raw device pointers and the current CUDA stream to the
library function of the same name, and raises ``VedaError`` on a non-zero
status.  All computation runs in the library's CUDA kernels; there is no
fallback of any kind -- if the library is missing, importing this module
fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# VEDA_DEBUG_BOUNDS=1 loads the debug build (build.py --debug), whose kernels
# check every computed index and report a failed check as VEDA_ERR_BOUNDS.
LIB_PATH = os.path.join(_HERE, "libveda_debug.so" if os.environ.get("VEDA_DEBUG_BOUNDS") == "1" else "libveda.so")

VEDA_OK, VEDA_ERR_INVALID_ARG, VEDA_ERR_UNSUPPORTED, VEDA_ERR_CUDA, VEDA_ERR_TIMEOUT, VEDA_ERR_BOUNDS = range(6)
MAX_HEADS = 128
_STATUS_NAMES = {0: "VEDA_OK", 1: "VEDA_ERR_INVALID_ARG", 2: "VEDA_ERR_UNSUPPORTED", 3: "VEDA_ERR_CUDA",
                 4: "VEDA_ERR_TIMEOUT", 5: "VEDA_ERR_BOUNDS"}


class VedaError(RuntimeError):
    def __init__(self, status: int, func: str, message: str):
        super().__init__(f"{func}: {_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class veda_grid(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32)]


class veda_tiling(ctypes.Structure):
    _fields_ = [("pt", ctypes.c_int32), ("ph", ctypes.c_int32), ("pw", ctypes.c_int32)]


class veda_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("heads", ctypes.c_int32), ("d", ctypes.c_int32), ("S", ctypes.c_int32),
                ("grid", veda_grid), ("tilings", ctypes.POINTER(veda_tiling))]


class veda_mlp(ctypes.Structure):
    _fields_ = [("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p),
                ("hidden", ctypes.c_int32), ("e", ctypes.c_int32)]


class veda_mlp_grad(ctypes.Structure):
    _fields_ = [("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p)]


_P = ctypes.POINTER(veda_problem)
_V = ctypes.c_void_p
_I32P = ctypes.POINTER(ctypes.c_int32)
_SIG = {
    "veda_tile_layout": [_P, _I32P, _I32P],
    "veda_keep_count": [_P, ctypes.c_float, _I32P, _I32P],
    "veda_tile_permute": [_P, _V, _V, _V],
    "veda_tile_unpermute": [_P, _V, _V, _V],
    "veda_tile_permute_tripool": [_P, _V, _V, _V, _V],
    "veda_tripool": [_P, _V, _V, _V],
    "veda_tripool_grid": [_P, _V, _V, _V],
    "veda_score_topk_workspace": [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)],
    "veda_tile_score_topk": [_P, _V, _V, ctypes.POINTER(veda_mlp), ctypes.POINTER(veda_mlp), ctypes.c_float, _V,
                             ctypes.c_int32, _V, _V, ctypes.c_size_t, _V],
    "veda_tile_score_topk_noalloc": [_P, _V, _V, ctypes.POINTER(veda_mlp), ctypes.POINTER(veda_mlp), ctypes.c_float,
                                     _V, ctypes.c_int32, _V, _V],
    "veda_tile_sparse_attn": [_P, _V, _V, _V, _V, ctypes.c_int32, ctypes.c_float, _V, _V, _V],
    "veda_tile_sparse_attn_grid": [_P, _V, _V, _V, _V, ctypes.c_int32, ctypes.c_float, _V, _V, _V],
    "veda_attn_config": [_P, ctypes.c_int32, _I32P, _I32P, ctypes.POINTER(ctypes.c_size_t)],
    "veda_tile_map_workspace": [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)],
    "veda_tile_map_maxpool": [_P, _V, _V, _V, ctypes.c_int32, ctypes.c_float, _V, _V, ctypes.c_size_t, _V],
    "veda_tile_map_maxpool_grid": [_P, _V, _V, _V, ctypes.c_int32, ctypes.c_float, _V, _V, ctypes.c_size_t, _V],
    "veda_distill_workspace": [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)],
    "veda_distill_loss_grad": [_P, _V, _V, ctypes.POINTER(veda_mlp), ctypes.POINTER(veda_mlp), _V, _V, ctypes.c_int32,
                               _V, ctypes.POINTER(veda_mlp_grad), ctypes.POINTER(veda_mlp_grad), _V, ctypes.c_size_t,
                               _V],
    "veda_head_error": [_P, _V, _V, _V, _V, _V, ctypes.c_size_t, _V],
    "veda_attn_backward_workspace": [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)],
    "veda_tile_sparse_attn_backward_grid": [_P, _V, _V, _V, _V, _V, _V, _V, ctypes.c_int32, ctypes.c_float, _V, _V,
                                            _V, _V, ctypes.c_size_t, _V],
    "veda_sync_status": [_V],
    "veda_set_wait_timeout_ns": [ctypes.c_uint64],
    "veda_selftest_wait_timeout": [ctypes.c_uint64, _V],
    "veda_selftest_bounds": [_V],
    "veda_bounds_checked": [],
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); "
                          "run tile_sparse_attention_head_b200/build.py" +
                          (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
    lib = ctypes.CDLL(LIB_PATH)
    for name, args in _SIG.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.veda_last_error.restype = ctypes.c_char_p
    lib.veda_last_error.argtypes = []
    lib.veda_version.restype = ctypes.c_char_p
    lib.veda_version.argtypes = []
    return lib


LIB = _load()


def _check(status: int, func: str) -> None:
    if status != VEDA_OK:
        raise VedaError(status, func, LIB.veda_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, dtype: Optional[torch.dtype] = None,
         shape: Optional[Tuple[int, ...]] = None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    return t.data_ptr()


class Problem:
    """The problem statement (B, heads, d, S, grid, per-head tilings) as the C struct."""

    def __init__(self, B: int, heads: int, d: int, S: int, grid: Sequence[int],
                 tilings: Sequence[Sequence[int]]):
        self.B, self.heads, self.d, self.S = int(B), int(heads), int(d), int(S)
        self.grid = tuple(int(v) for v in grid)
        self.tilings = tuple(tuple(int(v) for v in t) for t in tilings)
        if len(self.tilings) != self.heads:
            raise ValueError("one tiling per head is required")
        self._tilings_arr = (veda_tiling * max(1, self.heads))(*[veda_tiling(*t) for t in self.tilings])
        self.c = veda_problem(self.B, self.heads, self.d, self.S, veda_grid(*self.grid),
                              ctypes.cast(self._tilings_arr, ctypes.POINTER(veda_tiling)))
        nts = (ctypes.c_int32 * self.heads)()
        ntmax = ctypes.c_int32()
        _check(LIB.veda_tile_layout(ctypes.byref(self.c), nts, ctypes.byref(ntmax)), "veda_tile_layout")
        self.nt_per_head = list(nts)
        self.nt_max = int(ntmax.value)

    @property
    def N(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def grid_shape(self) -> Tuple[int, int, int, int]:
        return (self.B, self.heads, self.N, self.d)

    def tile_shape(self) -> Tuple[int, int, int, int]:
        return (self.B, self.heads, self.nt_max * self.S, self.d)

    def keep_count(self, keep_ratio: float):
        ks = (ctypes.c_int32 * self.heads)()
        kmax = ctypes.c_int32()
        _check(LIB.veda_keep_count(self.ref, ctypes.c_float(keep_ratio), ks, ctypes.byref(kmax)), "veda_keep_count")
        return list(ks), int(kmax.value)


def veda_tile_permute(p: Problem, x: torch.Tensor, xp: torch.Tensor, stream=None) -> torch.Tensor:
    _check(LIB.veda_tile_permute(p.ref, _ptr(x, "x", torch.bfloat16, p.grid_shape()),
                                 _ptr(xp, "xp", torch.bfloat16, p.tile_shape()), _stream(stream)),
           "veda_tile_permute")
    return xp


def veda_tile_permute_tripool(p: Problem, x: torch.Tensor, xp: torch.Tensor, desc: torch.Tensor,
                              stream=None) -> torch.Tensor:
    _check(LIB.veda_tile_permute_tripool(p.ref, _ptr(x, "x", torch.bfloat16, p.grid_shape()),
                                         _ptr(xp, "xp", torch.bfloat16, p.tile_shape()),
                                         _ptr(desc, "desc", torch.float32, (p.B, p.heads, p.nt_max, 3 * p.d)),
                                         _stream(stream)), "veda_tile_permute_tripool")
    return xp


def veda_tile_unpermute(p: Problem, xp: torch.Tensor, x: torch.Tensor, stream=None) -> torch.Tensor:
    _check(LIB.veda_tile_unpermute(p.ref, _ptr(xp, "xp", torch.bfloat16, p.tile_shape()),
                                   _ptr(x, "x", torch.bfloat16, p.grid_shape()), _stream(stream)),
           "veda_tile_unpermute")
    return x


def veda_tripool(p: Problem, xp: torch.Tensor, desc: torch.Tensor, stream=None) -> torch.Tensor:
    _check(LIB.veda_tripool(p.ref, _ptr(xp, "xp", torch.bfloat16, p.tile_shape()),
                            _ptr(desc, "desc", torch.float32, (p.B, p.heads, p.nt_max, 3 * p.d)), _stream(stream)),
           "veda_tripool")
    return desc


def veda_tripool_grid(p: Problem, x: torch.Tensor, desc: torch.Tensor, stream=None) -> torch.Tensor:
    _check(LIB.veda_tripool_grid(p.ref, _ptr(x, "x", torch.bfloat16, p.grid_shape()),
                                 _ptr(desc, "desc", torch.float32, (p.B, p.heads, p.nt_max, 3 * p.d)),
                                 _stream(stream)),
           "veda_tripool_grid")
    return desc


def veda_score_topk_workspace(p: Problem, e: int) -> int:
    n = ctypes.c_size_t()
    _check(LIB.veda_score_topk_workspace(p.ref, int(e), ctypes.byref(n)), "veda_score_topk_workspace")
    return int(n.value)


def make_mlp(w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor, b2: torch.Tensor) -> veda_mlp:
    """C struct for one set of per-head estimator weights (fp32 device tensors)."""
    heads, hidden, _ = w1.shape
    e = w2.shape[1]
    for t, n in ((w1, "w1"), (b1, "b1"), (w2, "w2"), (b2, "b2")):
        _ptr(t, n, torch.float32)
    if tuple(b1.shape) != (heads, hidden) or tuple(w2.shape) != (heads, e, hidden) or tuple(b2.shape) != (heads, e):
        raise ValueError("estimator weight shapes must be w1 [h,hid,3d], b1 [h,hid], w2 [h,e,hid], b2 [h,e]")
    return veda_mlp(w1.data_ptr(), b1.data_ptr(), w2.data_ptr(), b2.data_ptr(), int(hidden), int(e))


def veda_tile_score_topk(p: Problem, desc_q: torch.Tensor, desc_k: torch.Tensor, mlp_q: veda_mlp, mlp_k: veda_mlp,
                         keep_ratio: float, idx: torch.Tensor, probs: Optional[torch.Tensor],
                         workspace: torch.Tensor, stream=None) -> torch.Tensor:
    dshape = (p.B, p.heads, p.nt_max, 3 * p.d)
    k_max = int(idx.shape[-1])
    _check(LIB.veda_tile_score_topk(
        p.ref, _ptr(desc_q, "desc_q", torch.float32, dshape), _ptr(desc_k, "desc_k", torch.float32, dshape),
        ctypes.byref(mlp_q), ctypes.byref(mlp_k), ctypes.c_float(keep_ratio),
        _ptr(idx, "idx", torch.int32, (p.B, p.heads, p.nt_max, k_max)), k_max,
        _ptr(probs, "probs", torch.float32, (p.B, p.heads, p.nt_max, p.nt_max)),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)),
        "veda_tile_score_topk")
    return idx


def veda_tile_score_topk_noalloc(p: Problem, desc_q: torch.Tensor, desc_k: torch.Tensor, mlp_q: veda_mlp,
                                 mlp_k: veda_mlp, keep_ratio: float, idx: torch.Tensor,
                                 probs: Optional[torch.Tensor], stream=None) -> torch.Tensor:
    """veda_tile_score_topk without a workspace, for callers that cannot allocate device scratch."""
    dshape = (p.B, p.heads, p.nt_max, 3 * p.d)
    k_max = int(idx.shape[-1])
    _check(LIB.veda_tile_score_topk_noalloc(
        p.ref, _ptr(desc_q, "desc_q", torch.float32, dshape), _ptr(desc_k, "desc_k", torch.float32, dshape),
        ctypes.byref(mlp_q), ctypes.byref(mlp_k), ctypes.c_float(keep_ratio),
        _ptr(idx, "idx", torch.int32, (p.B, p.heads, p.nt_max, k_max)), k_max,
        _ptr(probs, "probs", torch.float32, (p.B, p.heads, p.nt_max, p.nt_max)), _stream(stream)),
        "veda_tile_score_topk_noalloc")
    return idx


def veda_tile_sparse_attn(p: Problem, qp: torch.Tensor, kp: torch.Tensor, vp: torch.Tensor, idx: torch.Tensor,
                          op: torch.Tensor, lse: Optional[torch.Tensor] = None, scale: float = 0.0,
                          stream=None) -> torch.Tensor:
    ts = p.tile_shape()
    k_max = int(idx.shape[-1])
    _check(LIB.veda_tile_sparse_attn(
        p.ref, _ptr(qp, "qp", torch.bfloat16, ts), _ptr(kp, "kp", torch.bfloat16, ts),
        _ptr(vp, "vp", torch.bfloat16, ts), _ptr(idx, "idx", torch.int32, (p.B, p.heads, p.nt_max, k_max)), k_max,
        ctypes.c_float(scale), _ptr(op, "op", torch.bfloat16, ts),
        _ptr(lse, "lse", torch.float32, (p.B, p.heads, p.nt_max * p.S)), _stream(stream)),
        "veda_tile_sparse_attn")
    return op


def veda_tile_sparse_attn_grid(p: Problem, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                               o: torch.Tensor, lse: Optional[torch.Tensor] = None, scale: float = 0.0,
                               stream=None) -> torch.Tensor:
    gs = p.grid_shape()
    k_max = int(idx.shape[-1])
    _check(LIB.veda_tile_sparse_attn_grid(
        p.ref, _ptr(q, "q", torch.bfloat16, gs), _ptr(k, "k", torch.bfloat16, gs),
        _ptr(v, "v", torch.bfloat16, gs), _ptr(idx, "idx", torch.int32, (p.B, p.heads, p.nt_max, k_max)), k_max,
        ctypes.c_float(scale), _ptr(o, "o", torch.bfloat16, gs),
        _ptr(lse, "lse", torch.float32, (p.B, p.heads, p.N)), _stream(stream)),
        "veda_tile_sparse_attn_grid")
    return o


def veda_attn_backward_workspace(p: Problem, k_max: int) -> int:
    n = ctypes.c_size_t()
    _check(LIB.veda_attn_backward_workspace(p.ref, int(k_max), ctypes.byref(n)), "veda_attn_backward_workspace")
    return int(n.value)


def veda_tile_sparse_attn_backward_grid(p: Problem, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                        o: torch.Tensor, lse: torch.Tensor, d_o: torch.Tensor, idx: torch.Tensor,
                                        dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor,
                                        workspace: torch.Tensor, scale: float = 0.0, stream=None):
    """dq, dk, dv of veda_tile_sparse_attn_grid for the upstream gradient d_o (all grid order)."""
    gs = p.grid_shape()
    k_max = int(idx.shape[-1])
    _check(LIB.veda_tile_sparse_attn_backward_grid(
        p.ref, _ptr(q, "q", torch.bfloat16, gs), _ptr(k, "k", torch.bfloat16, gs), _ptr(v, "v", torch.bfloat16, gs),
        _ptr(o, "o", torch.bfloat16, gs), _ptr(lse, "lse", torch.float32, (p.B, p.heads, p.N)),
        _ptr(d_o, "d_o", torch.bfloat16, gs), _ptr(idx, "idx", torch.int32, (p.B, p.heads, p.nt_max, k_max)), k_max,
        ctypes.c_float(scale), _ptr(dq, "dq", torch.bfloat16, gs), _ptr(dk, "dk", torch.bfloat16, gs),
        _ptr(dv, "dv", torch.bfloat16, gs), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "veda_tile_sparse_attn_backward_grid")
    return dq, dk, dv


def veda_attn_config(p: Problem, k_max: int) -> Tuple[int, int, int]:
    """(K ring depth, V ring depth, dynamic shared memory bytes) of the attention launch."""
    ks, vs, nb = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_size_t()
    _check(LIB.veda_attn_config(p.ref, int(k_max), ctypes.byref(ks), ctypes.byref(vs), ctypes.byref(nb)),
           "veda_attn_config")
    return int(ks.value), int(vs.value), int(nb.value)


def veda_tile_map_workspace(p: Problem, R: int) -> int:
    n = ctypes.c_size_t()
    _check(LIB.veda_tile_map_workspace(p.ref, int(R), ctypes.byref(n)), "veda_tile_map_workspace")
    return int(n.value)


def veda_tile_map_maxpool(p: Problem, qp: torch.Tensor, kp: torch.Tensor, rows: torch.Tensor, out: torch.Tensor,
                          workspace: torch.Tensor, scale: float = 0.0, stream=None) -> torch.Tensor:
    ts = p.tile_shape()
    R = int(rows.shape[-1])
    _check(LIB.veda_tile_map_maxpool(
        p.ref, _ptr(qp, "qp", torch.bfloat16, ts), _ptr(kp, "kp", torch.bfloat16, ts),
        _ptr(rows, "rows", torch.int32, (p.B * p.heads, R)), R, ctypes.c_float(scale),
        _ptr(out, "map", torch.float32, (p.B, p.heads, R, p.nt_max)), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "veda_tile_map_maxpool")
    return out


def veda_tile_map_maxpool_grid(p: Problem, q: torch.Tensor, k: torch.Tensor, rows: torch.Tensor, out: torch.Tensor,
                               workspace: torch.Tensor, scale: float = 0.0, stream=None) -> torch.Tensor:
    """The max-pooled tile map from grid-order q, k [B, heads, N, d] bf16 (no tile-major copies)."""
    gs = p.grid_shape()
    R = int(rows.shape[-1])
    _check(LIB.veda_tile_map_maxpool_grid(
        p.ref, _ptr(q, "q", torch.bfloat16, gs), _ptr(k, "k", torch.bfloat16, gs),
        _ptr(rows, "rows", torch.int32, (p.B * p.heads, R)), R, ctypes.c_float(scale),
        _ptr(out, "map", torch.float32, (p.B, p.heads, R, p.nt_max)), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "veda_tile_map_maxpool_grid")
    return out


def veda_distill_workspace(p: Problem, hidden: int, e: int, R: int) -> int:
    n = ctypes.c_size_t()
    _check(LIB.veda_distill_workspace(p.ref, int(hidden), int(e), int(R), ctypes.byref(n)), "veda_distill_workspace")
    return int(n.value)


def make_mlp_grad(w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor, b2: torch.Tensor) -> veda_mlp_grad:
    """C struct of gradient outputs for one estimator (fp32 device tensors shaped like its weights)."""
    for t, n in ((w1, "w1"), (b1, "b1"), (w2, "w2"), (b2, "b2")):
        _ptr(t, n, torch.float32)
    return veda_mlp_grad(w1.data_ptr(), b1.data_ptr(), w2.data_ptr(), b2.data_ptr())


def veda_distill_loss_grad(p: Problem, desc_q: torch.Tensor, desc_k: torch.Tensor, mlp_q: veda_mlp, mlp_k: veda_mlp,
                           tile_map: torch.Tensor, rows: torch.Tensor, loss: torch.Tensor, grad_q: veda_mlp_grad,
                           grad_k: veda_mlp_grad, workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """Row-wise KL distillation loss of the estimator against the tile map, and its gradients."""
    dshape = (p.B, p.heads, p.nt_max, 3 * p.d)
    R = int(rows.shape[-1])
    _check(LIB.veda_distill_loss_grad(
        p.ref, _ptr(desc_q, "desc_q", torch.float32, dshape), _ptr(desc_k, "desc_k", torch.float32, dshape),
        ctypes.byref(mlp_q), ctypes.byref(mlp_k),
        _ptr(tile_map, "map", torch.float32, (p.B, p.heads, R, p.nt_max)),
        _ptr(rows, "rows", torch.int32, (p.B * p.heads, R)), R, _ptr(loss, "loss", torch.float32, (1,)),
        ctypes.byref(grad_q), ctypes.byref(grad_k), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "veda_distill_loss_grad")
    return loss


def veda_head_error(p: Problem, o: torch.Tensor, o_ref: torch.Tensor, err: torch.Tensor, ref_sq: torch.Tensor,
                    workspace: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-head sums of (o - o_ref)^2 and o_ref^2 over grid-order bf16 outputs."""
    gs = p.grid_shape()
    _check(LIB.veda_head_error(p.ref, _ptr(o, "o", torch.bfloat16, gs), _ptr(o_ref, "o_ref", torch.bfloat16, gs),
                               _ptr(err, "err", torch.float32, (p.heads,)),
                               _ptr(ref_sq, "ref_sq", torch.float32, (p.heads,)), _ptr(workspace, "workspace"),
                               workspace.numel() * workspace.element_size(), _stream(stream)), "veda_head_error")
    return err, ref_sq


def veda_sync_status(stream=None) -> None:
    _check(LIB.veda_sync_status(_stream(stream)), "veda_sync_status")


def veda_set_wait_timeout_ns(ns: int) -> None:
    _check(LIB.veda_set_wait_timeout_ns(int(ns)), "veda_set_wait_timeout_ns")


def veda_selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check(LIB.veda_selftest_wait_timeout(int(timeout_ns), _stream(stream)), "veda_selftest_wait_timeout")


def veda_bounds_checked() -> bool:
    """True when the loaded library is the debug build with device-side index checks."""
    return bool(LIB.veda_bounds_checked())


def veda_selftest_bounds(stream=None) -> None:
    """Debug builds: one kernel fails a bounds check on purpose (no memory is
    touched); the next veda_sync_status raises VEDA_ERR_BOUNDS."""
    _check(LIB.veda_selftest_bounds(_stream(stream)), "veda_selftest_bounds")


def veda_version() -> str:
    return LIB.veda_version().decode()

"""B200 (sm_100a) Attention-Matching KV compaction (AM-OMP).

Thin ctypes binding over the C ABI in include/am_b200.h: it only marshals
torch tensors to pointers and sizes; every step of the compaction runs in the
library's CUDA kernels.  The library is built in-tree by
``attention_matching_b200._build.build()`` (or ``__graft_entry__.build()``).
There is no CPU fallback: without the shared library or a CUDA device the
calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

__all__ = ["AmError", "AmOpts", "lib", "library_path", "workspace_size", "compact_heads",
           "get_status", "profile_enable", "profile_collect", "kernel_launches", "STAGES",
           "STATUS", "BF16", "FP32", "CORR_AUTO", "CORR_STORED_FP32", "CORR_STORED_BF16",
           "CORR_RECOMPUTE", "CORR_BOUNDED", "SELECT_OMP", "SELECT_HIGHEST", "attend_packed",
           "assign_budgets"]

BF16, FP32 = 0, 1
CORR_AUTO, CORR_STORED_FP32, CORR_STORED_BF16, CORR_RECOMPUTE, CORR_BOUNDED = 0, 1, 2, 3, 4
SELECT_OMP, SELECT_HIGHEST = 0, 1   # am_select_mode_t
STATUS = {
    0: "AM_OK", 1: "AM_ERR_INVALID_ARG", 2: "AM_ERR_BUDGET", 3: "AM_ERR_WORKSPACE",
    4: "AM_ERR_NONFINITE", 5: "AM_ERR_CUDA", 6: "AM_ERR_TIMEOUT", 7: "AM_ERR_UNSUPPORTED",
    8: "AM_WARN_NOT_CONVERGED", 9: "AM_ERR_NOT_SPD", 10: "AM_WARN_MASS_UNDERFLOW",
}
WARNINGS = (8, 10)   # results valid as documented

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "_lib", "libam_b200.so")


class AmError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class AmWorkspaceView(ctypes.Structure):
    """Mirror of am_workspace_view_t."""
    _fields_ = [("phiT", ctypes.c_size_t), ("mass", ctypes.c_size_t), ("target", ctypes.c_size_t),
                ("shift", ctypes.c_size_t), ("ldn", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("weights", ctypes.c_size_t), ("resid", ctypes.c_size_t),
                ("rows_evaluated", ctypes.c_size_t), ("column_norms", ctypes.c_size_t),
                ("nnls_refits", ctypes.c_size_t), ("nnls_solves", ctypes.c_size_t)]


class AmOpts(ctypes.Structure):
    """Mirror of am_opts_t (include/am_b200.h); field order and types match."""
    _fields_ = [
        ("in_dtype", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("refit_every", ctypes.c_int32),
        ("nnls_max_iter", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("ridge", ctypes.c_float),
        ("w_floor_rel", ctypes.c_float),
        ("corr_mode", ctypes.c_int32),
        ("shift", ctypes.c_void_p),
        ("key_bias", ctypes.c_void_p),
        ("pick_order", ctypes.c_void_p),
        ("pick_corr", ctypes.c_void_p),
        ("shift_out", ctypes.c_void_p),
        ("residual_out", ctypes.c_void_p),
        ("w_out", ctypes.c_void_p),
        ("select_mode", ctypes.c_int32),
        ("reserved0", ctypes.c_int32),
        ("key_offsets", ctypes.c_void_p),
        ("wait_cycles", ctypes.c_int64),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library once; raise loudly if it has not been built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with attention_matching_b200._build.build()")
        L = ctypes.CDLL(path)
        c_int, c_void_p, c_size_t = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
        P_i32 = ctypes.POINTER(ctypes.c_int32)
        P_i64 = ctypes.POINTER(ctypes.c_int64)
        L.am_default_opts.argtypes = [ctypes.POINTER(AmOpts)]
        L.am_default_opts.restype = c_int
        L.am_workspace_size.argtypes = [c_int, c_int, c_int, c_int, P_i32, ctypes.POINTER(AmOpts),
                                        ctypes.POINTER(c_size_t)]
        L.am_workspace_size.restype = c_int
        L.am_workspace_size_waves.argtypes = [c_int, c_int, c_int, c_int, P_i32, ctypes.POINTER(AmOpts), c_int,
                                              ctypes.POINTER(c_size_t)]
        L.am_workspace_size_waves.restype = c_int
        L.am_compact_heads.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, P_i32,
                                       ctypes.POINTER(AmOpts), c_void_p, c_size_t, P_i64,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
        L.am_compact_heads.restype = c_int
        L.am_get_status.argtypes = [c_void_p, c_int, P_i32, c_void_p]
        L.am_get_status.restype = c_int
        L.am_status_string.argtypes = [c_int]
        L.am_status_string.restype = ctypes.c_char_p
        L.am_version.argtypes = []
        L.am_version.restype = c_int
        L.am_workspace_view.argtypes = [c_int, c_int, c_int, c_int, P_i32, ctypes.POINTER(AmOpts),
                                        ctypes.POINTER(AmWorkspaceView)]
        L.am_workspace_view.restype = c_int
        L.am_profile_enable.argtypes = [c_int]
        L.am_profile_enable.restype = c_int
        L.am_profile_collect.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
        L.am_profile_collect.restype = c_int
        L.am_kernel_launches.argtypes = []
        L.am_kernel_launches.restype = ctypes.c_int64
        L.am_attend_packed.argtypes = [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_int, ctypes.c_float, c_void_p,
                                       c_void_p]
        L.am_attend_packed.restype = c_int
        L.am_assign_budgets.argtypes = [ctypes.POINTER(ctypes.c_double), c_int, c_int, c_int, c_int,
                                        ctypes.c_int64, c_int, P_i32, P_i32]
        L.am_assign_budgets.restype = c_int
        _lib = L
    return _lib


def _i32_array(vals: Sequence[int]):
    return (ctypes.c_int32 * len(vals))(*[int(v) for v in vals])


def make_opts(dtype: int = BF16, topk: int = 1, refit_every: int = 1, scale: float = 0.0,
              ridge: float = 1e-6, w_floor_rel: float = 1e-12, nnls_max_iter: int = 0,
              corr_mode: int = CORR_AUTO, select_mode: int = 0, wait_cycles: int = 0) -> AmOpts:
    o = AmOpts()
    rc = lib().am_default_opts(ctypes.byref(o))
    if rc:
        raise AmError(rc, "am_default_opts")
    o.in_dtype, o.topk, o.refit_every, o.nnls_max_iter = dtype, topk, refit_every, nnls_max_iter
    o.scale, o.ridge, o.w_floor_rel = scale, ridge, w_floor_rel
    o.corr_mode = corr_mode
    o.select_mode = select_mode
    o.wait_cycles = wait_cycles
    return o


def workspace_size(n: int, T: int, d: int, budgets: Sequence[int], opts: AmOpts,
                   wave_heads: Optional[int] = None) -> int:
    """Workspace bytes for one call: every head in one wave, or (wave_heads)
    waves of at most that many consecutive heads through the same memory."""
    out = ctypes.c_size_t(0)
    if wave_heads is None:
        rc = lib().am_workspace_size(n, T, d, len(budgets), _i32_array(budgets), ctypes.byref(opts),
                                     ctypes.byref(out))
    else:
        rc = lib().am_workspace_size_waves(n, T, d, len(budgets), _i32_array(budgets), ctypes.byref(opts),
                                           int(wave_heads), ctypes.byref(out))
    if rc:
        raise AmError(rc, "am_workspace_size")
    return int(out.value)


def features(out: Dict, n: int, T: int, d: int, budgets: Sequence[int], topk: int = 1,
             refit_every: int = 1, dtype: int = BF16, corr_mode: int = CORR_AUTO,
             select_mode: int = SELECT_OMP) -> Dict:
    """Views of the intermediate features a finished call left in its
    workspace: phiT [H, T, ldn] fp32, mass [H, ldn] fp64, target [H, n, d]
    fp32, shift [H] fp32, weights [Σt] fp64 (last NNLS refit, pick order)
    and resid [H, ldn] fp32 (torch tensors sharing the workspace memory)."""
    import torch
    H = len(budgets)
    opts = make_opts(dtype, topk, refit_every, corr_mode=corr_mode, select_mode=select_mode)
    v = AmWorkspaceView()
    rc = lib().am_workspace_view(n, T, d, H, _i32_array(budgets), ctypes.byref(opts), ctypes.byref(v))
    if rc:
        raise AmError(rc, "am_workspace_view")
    ws = out["workspace"]

    def view(off, count, dt):
        nbytes = count * torch.empty((), dtype=dt).element_size()
        return ws[off:off + nbytes].view(dt)

    return {
        "phiT": view(v.phiT, H * T * v.ldn, torch.float32).view(H, T, v.ldn),
        "mass": view(v.mass, H * v.ldn, torch.float64).view(H, v.ldn),
        "target": view(v.target, H * n * d, torch.float32).view(H, n, d),
        "shift": view(v.shift, H, torch.float32),
        "weights": view(v.weights, int(sum(budgets)), torch.float64),
        "resid": view(v.resid, H * v.ldn, torch.float32).view(H, v.ldn),
        "rows_evaluated": view(v.rows_evaluated, H, torch.int64),
        "column_norms": view(v.column_norms, H * T, torch.float64).view(H, T),
        "nnls_refits": view(v.nnls_refits, H, torch.int32),
        "nnls_solves": view(v.nnls_solves, H, torch.int32),
        "ldn": v.ldn,
    }


def call_stats(out: Dict, n: int, T: int, d: int, budgets: Sequence[int], topk: int = 1,
               refit_every: int = 1, dtype: int = BF16, corr_mode: int = CORR_AUTO,
               select_mode: int = SELECT_OMP) -> Dict:
    """Per-head statistics of a finished call, valid whether or not it ran in
    one wave: keys whose correlation was evaluated (int64 [H]), NNLS refits and
    their inner solves (int32 [H] each); views into the workspace's prefix."""
    import torch
    H = len(budgets)
    opts = make_opts(dtype, topk, refit_every, corr_mode=corr_mode, select_mode=select_mode)
    v = AmWorkspaceView()
    rc = lib().am_workspace_view(n, T, d, H, _i32_array(budgets), ctypes.byref(opts), ctypes.byref(v))
    if rc:
        raise AmError(rc, "am_workspace_view")
    ws = out["workspace"]
    return {"rows_evaluated": ws[v.rows_evaluated:v.rows_evaluated + 8 * H].view(torch.int64),
            "nnls_refits": ws[v.nnls_refits:v.nnls_refits + 4 * H].view(torch.int32),
            "nnls_solves": ws[v.nnls_solves:v.nnls_solves + 4 * H].view(torch.int32)}


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def compact_heads(Q, K, V, budgets: Sequence[int], topk: int = 1, refit_every: int = 1,
                  shift=None, key_bias=None, ridge: float = 1e-6, w_floor_rel: float = 1e-12,
                  scale: float = 0.0, nnls_max_iter: int = 0, workspace=None, trace: bool = False,
                  stream=None, check: bool = True, corr_mode: int = CORR_AUTO,
                  select_mode: int = SELECT_OMP, key_offsets: Optional[Sequence[int]] = None,
                  wave_heads: Optional[int] = None, wait_cycles: int = 0) -> Dict:
    """Compact H heads on the GPU.

    Q [H, n, d], K [H, T, d], V [H, T, d]: contiguous tensors, bf16 or fp32,
    all on the current CUDA device or all on the host (then copied in, and the
    outputs copied back to the host).  With ``key_offsets`` (H + 1 ints,
    starting at 0) head h has T_h = key_offsets[h+1] − key_offsets[h] keys and
    K, V are packed [Σ T_h, d] (key_bias packed [Σ T_h]).
    budgets: H ints in [1, T_h].  shift [H] fp32 and key_bias [H, T] fp32 are
    optional CUDA tensors.  select_mode SELECT_HIGHEST keeps each head's t
    keys of largest total attention instead of the OMP picks (topk,
    refit_every and corr_mode are then ignored).  ``wave_heads`` sizes an
    allocated workspace for waves of at most that many heads (a workspace
    passed in decides the waves by its own size).  Returns a dict of CUDA
    tensors in the packed varlen layout (C_k, beta, C_v, indices, cu_t) plus,
    with ``trace``, the pick order, pick correlations, shift used, mass
    residual and weights.
    """
    import torch
    host = not (Q.is_cuda or K.is_cuda or V.is_cuda)
    if host:
        # host inputs: copy in (asynchronously from pinned memory), run, copy out
        dev = torch.device("cuda", torch.cuda.current_device())
        Q, K, V = (x.to(dev, non_blocking=True) for x in (Q, K, V))
    if not (Q.is_cuda and K.is_cuda and V.is_cuda):
        raise ValueError("Q, K, V must all be CUDA tensors or all host tensors")
    H, n, d = Q.shape
    if key_offsets is None:
        T = K.shape[1]
        if K.shape != (H, T, d) or V.shape != (H, T, d) or len(budgets) != H:
            raise ValueError("shape mismatch")
        koffs = None
    else:
        ko = [int(x) for x in key_offsets]
        if len(ko) != H + 1 or ko[0] != 0 or len(budgets) != H:
            raise ValueError("key_offsets must hold H + 1 offsets starting at 0")
        T = max(ko[h + 1] - ko[h] for h in range(H))
        if K.shape != (ko[-1], d) or V.shape != (ko[-1], d):
            raise ValueError("with key_offsets, K and V are packed [sum T_h, d]")
        koffs = (ctypes.c_int64 * (H + 1))(*ko)
    if Q.dtype != K.dtype or Q.dtype != V.dtype or Q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("Q, K, V must share dtype bf16 or fp32")
    for t in (Q, K, V):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    dt = BF16 if Q.dtype == torch.bfloat16 else FP32
    dev = Q.device
    opts = make_opts(dt, topk, refit_every, scale, ridge, w_floor_rel, nnls_max_iter, corr_mode, select_mode,
                     wait_cycles)
    if koffs is not None:
        opts.key_offsets = ctypes.cast(koffs, ctypes.c_void_p)
    if shift is not None:
        shift = shift.to(device=dev, dtype=torch.float32).contiguous()
        opts.shift = shift.data_ptr()
    if key_bias is not None:
        key_bias = key_bias.to(device=dev, dtype=torch.float32).contiguous()
        opts.key_bias = key_bias.data_ptr()
    cu = [0]
    for t in budgets:
        cu.append(cu[-1] + int(t))
    tot = cu[-1]
    out = {
        "C_k": torch.empty((tot, d), dtype=Q.dtype, device=dev),
        "beta": torch.empty((tot,), dtype=torch.float32, device=dev),
        "C_v": torch.empty((tot, d), dtype=torch.float32, device=dev),
        "indices": torch.empty((tot,), dtype=torch.int32, device=dev),
        "cu_t": torch.tensor(cu, dtype=torch.int64),
    }
    if trace:
        out["pick_order"] = torch.empty((tot,), dtype=torch.int32, device=dev)
        out["pick_corr"] = torch.empty((tot,), dtype=torch.float32, device=dev)
        out["shift"] = torch.empty((H,), dtype=torch.float32, device=dev)
        out["residual"] = torch.empty((H,), dtype=torch.float64, device=dev)
        out["w"] = torch.empty((tot,), dtype=torch.float32, device=dev)
        opts.pick_order = out["pick_order"].data_ptr()
        opts.pick_corr = out["pick_corr"].data_ptr()
        opts.shift_out = out["shift"].data_ptr()
        opts.residual_out = out["residual"].data_ptr()
        opts.w_out = out["w"].data_ptr()
    if workspace is None:
        workspace = torch.empty((workspace_size(n, T, d, budgets, opts, wave_heads),), dtype=torch.uint8,
                                device=dev)
    offs = (ctypes.c_int64 * (H + 1))(*cu)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = lib().am_compact_heads(Q.data_ptr(), K.data_ptr(), V.data_ptr(), n, T, d, H,
                                _i32_array(budgets), ctypes.byref(opts), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), offs,
                                out["C_k"].data_ptr(), out["beta"].data_ptr(), out["C_v"].data_ptr(),
                                out["indices"].data_ptr(), ctypes.c_void_p(stream))
    if rc:
        raise AmError(rc, "am_compact_heads")
    out["workspace"] = workspace
    if host:
        for k in ("C_k", "beta", "C_v", "indices", "pick_order", "pick_corr", "shift", "residual", "w"):
            if k in out:
                out[k] = out[k].to("cpu")
    if check:
        per_head, worst = get_status(workspace, H, stream)
        out["status"] = per_head
        if worst != 0 and worst not in WARNINGS:
            raise AmError(worst, "am_compact_heads (device)")
    return out


STAGES = ["shift", "phi", "target", "init", "corr", "select", "gram", "nnls", "resid",
          "finalize", "design", "normal", "solve", "norms", "rows", "attend"]


def profile_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events (stage timing)."""
    lib().am_profile_enable(1 if on else 0)


def profile_collect() -> Dict[str, Dict[str, float]]:
    """Wait for the recorded events; per stage: device ms and launch count."""
    ms = (ctypes.c_double * len(STAGES))()
    n = (ctypes.c_int64 * len(STAGES))()
    rc = lib().am_profile_collect(ms, n)
    if rc:
        raise AmError(rc, "am_profile_collect")
    return {name: {"ms": ms[k], "launches": int(n[k])} for k, name in enumerate(STAGES)}


def kernel_launches() -> int:
    return int(lib().am_kernel_launches())


def attend_packed(Q, packed: Dict, K_new=None, V_new=None, scale: float = 0.0, stream=None):
    """Attention of Q [H, nq, d] over each head's compacted segment (the
    packed C_k, beta, C_v, cu_t that compact_heads returned) followed by
    fresh keys K_new, V_new [H, T_new, d] (optional).  Q, C_k, K_new and
    V_new share a dtype (bf16 or fp32), all on the GPU; returns out
    [H, nq, d] fp32."""
    import torch
    if not Q.is_cuda or Q.dim() != 3 or not Q.is_contiguous():
        raise ValueError("Q must be a contiguous CUDA tensor [H, nq, d]")
    H, nq, d = Q.shape
    dt = BF16 if Q.dtype == torch.bfloat16 else FP32
    C_k, beta, C_v = packed["C_k"], packed["beta"], packed["C_v"]
    if C_k.dtype != Q.dtype:
        raise ValueError("C_k and Q must share a dtype")
    cu = packed["cu_t"].to(device=Q.device, dtype=torch.int64).contiguous()
    Tn = 0
    if K_new is not None:
        if K_new.shape[:1] != (H,) or K_new.shape != V_new.shape or K_new.dtype != Q.dtype:
            raise ValueError("K_new and V_new must be [H, T_new, d] in Q's dtype")
        K_new, V_new = K_new.contiguous(), V_new.contiguous()
        Tn = K_new.shape[1]
    out = torch.empty((H, nq, d), dtype=torch.float32, device=Q.device)
    if stream is None:
        stream = torch.cuda.current_stream(Q.device).cuda_stream
    rc = lib().am_attend_packed(Q.data_ptr(), nq, d, H, dt, C_k.data_ptr(), beta.data_ptr(), C_v.data_ptr(),
                                cu.data_ptr(), _ptr(K_new), _ptr(V_new), Tn, scale, out.data_ptr(),
                                ctypes.c_void_p(stream))
    if rc:
        raise AmError(rc, "am_attend_packed")
    return out


def assign_budgets(loss, t_min: int, quantum: int, total: int, max_swaps: Optional[int] = None):
    """Per-head budgets from sensitivity curves loss [H, G] (head h's loss at
    budget t_min + g·quantum) by the library's greedy swaps (host code).
    Returns (budgets, swaps)."""
    import numpy as np
    L = np.ascontiguousarray(loss, dtype=np.float64)
    if L.ndim != 2:
        raise ValueError("loss must be [num_heads, levels]")
    H, G = L.shape
    out = (ctypes.c_int32 * H)()
    sw = ctypes.c_int32(0)
    rc = lib().am_assign_budgets(L.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), H, G, t_min, quantum,
                                 total, -1 if max_swaps is None else max_swaps, out, ctypes.byref(sw))
    if rc:
        raise AmError(rc, "am_assign_budgets")
    return list(out), sw.value


def get_status(workspace, H: int, stream=None):
    """Synchronise and read the per-head device status words."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device).cuda_stream
    arr = (ctypes.c_int32 * H)()
    worst = lib().am_get_status(workspace.data_ptr(), H, arr, ctypes.c_void_p(stream))
    return list(arr), int(worst)

"""ctypes binding of libhstu.so (include/hstu.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels.  Torch is
used for device memory (outputs, workspaces) and the current stream.  If the
library is missing this module raises at import time -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libhstu.so")
# HSTU_LIB names another build of the same library (the phase-traced one of
# `build --trace`); unset, the in-tree library above is loaded.
LIB_PATH = os.environ.get("HSTU_LIB") or LIB_PATH

HSTU_OK = 0
STATUS = {0: "HSTU_OK", 1: "HSTU_ERR_INVALID_ARG", 2: "HSTU_ERR_UNSUPPORTED",
          3: "HSTU_ERR_WORKSPACE", 4: "HSTU_ERR_CUDA", 5: "HSTU_ERR_DEVICE_TIMEOUT",
          6: "HSTU_ERR_DEVICE"}
F32, BF16 = 0, 1
MASK_CAUSAL, MASK_MFALCON = 0, 1
IMPL = {"auto": 0, "simt": 1}

EXPORTED = [
    "hstu_status_string", "hstu_version", "hstu_attn_workspace_size", "hstu_attn_fwd",
    "hstu_attn_bwd", "hstu_layer_workspace_size", "hstu_layer_fwd", "hstu_debug_buckets",
    "hstu_get_device_error", "hstu_set_wait_limit", "hstu_kernel_launch_count",
    "hstu_attn_fwd_noalloc", "hstu_debug_wait_probe", "hstu_partition_batch",
    "hstu_layer_bwd_workspace_size", "hstu_layer_bwd", "hstu_layer_fwd_keep_proj",
    "hstu_attn_candidates_workspace_size", "hstu_attn_fwd_candidates",
    "hstu_layer_candidates_workspace_size", "hstu_layer_fwd_candidates",
    "hstu_debug_trace_read", "hstu_debug_trace_clear", "hstu_debug_plan",
]


class HstuError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS.get(status, status)}")
        self.status = status


class AttnParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("d_qk", ctypes.c_int32),
        ("d_v", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
        ("num_pos_buckets", ctypes.c_int32), ("num_time_buckets", ctypes.c_int32),
        ("time_bucket_sub_bits", ctypes.c_int32), ("rab_per_head", ctypes.c_int32),
        ("mask", ctypes.c_int32), ("dtype", ctypes.c_int32), ("impl", ctypes.c_int32),
        ("q_row_stride", ctypes.c_int64), ("k_row_stride", ctypes.c_int64),
        ("v_row_stride", ctypes.c_int64), ("o_row_stride", ctypes.c_int64),
        ("do_row_stride", ctypes.c_int64), ("dq_row_stride", ctypes.c_int64),
        ("dk_row_stride", ctypes.c_int64), ("dv_row_stride", ctypes.c_int64),
        ("alpha", ctypes.c_float), ("silu_scale", ctypes.c_float),
    ]


class LayerParams(ctypes.Structure):
    _fields_ = [("attn", AttnParams), ("d_model", ctypes.c_int32),
                ("residual", ctypes.c_int32), ("ln_eps", ctypes.c_float),
                ("reserved", ctypes.c_int32)]


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"libhstu.so not found at {path}; build it with "
                           "`python -m hstu_pointwise_attention_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    P, LP = ctypes.POINTER(AttnParams), ctypes.POINTER(LayerParams)
    lib.hstu_status_string.argtypes = [ctypes.c_int]
    lib.hstu_status_string.restype = ctypes.c_char_p
    lib.hstu_version.restype = ctypes.c_char_p
    lib.hstu_attn_workspace_size.argtypes = [P, vp, i32, ctypes.POINTER(sz)]
    lib.hstu_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hstu_attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                  vp, sz, vp]
    lib.hstu_layer_workspace_size.argtypes = [LP, vp, ctypes.POINTER(sz)]
    lib.hstu_layer_fwd.argtypes = [LP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                   sz, vp]
    lib.hstu_debug_buckets.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hstu_get_device_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.hstu_set_wait_limit.argtypes = [ctypes.c_uint32]
    lib.hstu_set_wait_limit.restype = None
    lib.hstu_kernel_launch_count.argtypes = []
    lib.hstu_kernel_launch_count.restype = ctypes.c_uint64
    lib.hstu_attn_fwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.hstu_attn_fwd_noalloc.restype = ctypes.c_int
    lib.hstu_debug_wait_probe.argtypes = [vp, sz, ctypes.c_uint32, vp]
    lib.hstu_debug_wait_probe.restype = ctypes.c_int
    lib.hstu_layer_bwd_workspace_size.argtypes = [LP, vp, ctypes.POINTER(sz)]
    lib.hstu_layer_bwd.argtypes = [LP] + [vp] * 23 + [sz, vp]
    i64 = ctypes.c_int64
    lib.hstu_layer_fwd_keep_proj.argtypes = [LP] + [vp] * 15 + [sz, vp]
    lib.hstu_attn_candidates_workspace_size.argtypes = [P, vp, vp, ctypes.POINTER(sz)]
    lib.hstu_attn_fwd_candidates.argtypes = [P] + [vp] * 9 + [i64, i64] + [vp] * 4 + [sz, vp]
    lib.hstu_layer_candidates_workspace_size.argtypes = [LP, vp, vp, ctypes.POINTER(sz)]
    lib.hstu_layer_fwd_candidates.argtypes = [LP] + [vp] * 16 + [sz, vp]
    lib.hstu_partition_batch.argtypes = [vp, vp, i32, i32, vp, vp]
    lib.hstu_partition_batch.restype = ctypes.c_int
    lib.hstu_debug_trace_read.argtypes = [i32, vp, sz]
    lib.hstu_debug_trace_read.restype = ctypes.c_int
    lib.hstu_debug_trace_clear.argtypes = [i32]
    lib.hstu_debug_trace_clear.restype = ctypes.c_int
    lib.hstu_debug_plan.argtypes = [P, vp, vp, i32, vp, vp, vp, vp]
    lib.hstu_debug_plan.restype = ctypes.c_int
    for name in ("hstu_attn_workspace_size", "hstu_attn_fwd", "hstu_attn_bwd",
                 "hstu_layer_workspace_size", "hstu_layer_fwd", "hstu_debug_buckets",
                 "hstu_get_device_error", "hstu_layer_bwd_workspace_size", "hstu_layer_bwd",
                 "hstu_layer_fwd_keep_proj", "hstu_attn_candidates_workspace_size",
                 "hstu_attn_fwd_candidates", "hstu_layer_candidates_workspace_size",
                 "hstu_layer_fwd_candidates"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


LIB = load()


def _check(rc: int, what: str) -> None:
    if rc != HSTU_OK:
        raise HstuError(rc, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _host_i64(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _host_i32(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _row_stride(t: torch.Tensor, H: int, d: int, name: str) -> int:
    """t is [T, H, d] (or a [T, H*d] view) with contiguous heads."""
    if t.dim() == 3:
        if t.shape[1] != H or t.shape[2] != d or t.stride(2) != 1 or t.stride(1) != d:
            raise ValueError(f"{name}: expected [T, {H}, {d}] with contiguous heads")
    elif t.dim() == 2:
        if t.shape[1] != H * d or t.stride(1) != 1:
            raise ValueError(f"{name}: expected [T, {H * d}] with unit column stride")
    else:
        raise ValueError(f"{name}: expected 2 or 3 dims")
    return int(t.stride(0)) if t.shape[0] > 1 else H * d


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def make_params(q, k, v, seq_offsets, *, max_seq_len, num_pos_buckets, num_time_buckets,
                time_bucket_sub_bits, alpha=None, silu_scale=None, num_candidates=None,
                rab_per_head=False, impl="auto", out=None, dout=None, dq=None, dk=None,
                dv=None) -> AttnParams:
    H = q.shape[1] if q.dim() == 3 else None
    if H is None:
        raise ValueError("q must be [T, H, d_qk]")
    d_qk, d_v = q.shape[2], v.shape[-1] if v.dim() == 3 else v.shape[1] // H
    off = _host_i64(seq_offsets)
    p = AttnParams()
    p.batch = len(off) - 1
    p.num_heads = H
    p.d_qk, p.d_v = d_qk, d_v
    p.max_seq_len = int(max_seq_len)
    p.num_pos_buckets, p.num_time_buckets = int(num_pos_buckets), int(num_time_buckets)
    p.time_bucket_sub_bits = int(time_bucket_sub_bits)
    p.rab_per_head = int(bool(rab_per_head))
    p.mask = MASK_MFALCON if num_candidates is not None else MASK_CAUSAL
    if q.dtype == torch.float32:
        p.dtype = F32
    elif q.dtype == torch.bfloat16:
        p.dtype = BF16
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    for t, name in ((k, "k"), (v, "v")):
        if t.dtype != q.dtype:
            raise ValueError(f"{name} dtype {t.dtype} != q dtype {q.dtype}")
    p.impl = IMPL[impl]
    p.q_row_stride = _row_stride(q, H, d_qk, "q")
    p.k_row_stride = _row_stride(k, H, d_qk, "k")
    p.v_row_stride = _row_stride(v, H, d_v, "v")
    p.o_row_stride = _row_stride(out, H, d_v, "out") if out is not None else H * d_v
    p.do_row_stride = _row_stride(dout, H, d_v, "dout") if dout is not None else H * d_v
    p.dq_row_stride = _row_stride(dq, H, d_qk, "dq") if dq is not None else H * d_qk
    p.dk_row_stride = _row_stride(dk, H, d_qk, "dk") if dk is not None else H * d_qk
    p.dv_row_stride = _row_stride(dv, H, d_v, "dv") if dv is not None else H * d_v
    p.alpha = float(1.0 / math.sqrt(d_qk) if alpha is None else alpha)
    p.silu_scale = float(1.0 / max(1, int(max_seq_len)) if silu_scale is None else silu_scale)
    return p


def attn_workspace_size(p: AttnParams, seq_offsets, is_bwd: bool) -> int:
    off = _host_i64(seq_offsets)
    n = ctypes.c_size_t(0)
    _check(LIB.hstu_attn_workspace_size(ctypes.byref(p), off.ctypes.data, int(is_bwd),
                                        ctypes.byref(n)), "hstu_attn_workspace_size")
    return int(n.value)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small")
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def attn_fwd(q, k, v, seq_offsets, timestamps, rab_pos, rab_time, *, max_seq_len,
             time_bucket_sub_bits, alpha=None, silu_scale=None, num_candidates=None,
             rab_per_head=False, impl="auto", out=None, workspace=None, stream=None):
    """out[T, H, d_v] = HSTU pointwise attention (include/hstu.h)."""
    T, H = q.shape[0], q.shape[1]
    d_v = v.shape[-1] if v.dim() == 3 else v.shape[1] // H
    if out is None:
        out = torch.empty((T, H, d_v), dtype=q.dtype, device=q.device)
    nbp = rab_pos.shape[-1]
    nbt = rab_time.shape[-1]
    p = make_params(q, k, v, seq_offsets, max_seq_len=max_seq_len, num_pos_buckets=nbp,
                    num_time_buckets=nbt, time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                    silu_scale=silu_scale, num_candidates=num_candidates,
                    rab_per_head=rab_per_head, impl=impl, out=out)
    off = _host_i64(seq_offsets)
    nc = _host_i32(num_candidates)
    ws = _workspace(attn_workspace_size(p, off, False), q.device, workspace)
    _check(LIB.hstu_attn_fwd(ctypes.byref(p), off.ctypes.data,
                             None if nc is None else nc.ctypes.data, _ptr(timestamps), _ptr(q),
                             _ptr(k), _ptr(v), _ptr(rab_pos), _ptr(rab_time), _ptr(out),
                             _ptr(ws), ws.numel(), _stream(stream)), "hstu_attn_fwd")
    return out


def attn_bwd(q, k, v, seq_offsets, timestamps, rab_pos, rab_time, dout, *, max_seq_len,
             time_bucket_sub_bits, alpha=None, silu_scale=None, num_candidates=None,
             rab_per_head=False, impl="auto", dq=None, dk=None, dv=None, drab_pos=None,
             drab_time=None, workspace=None, stream=None):
    """(dq, dk, dv, drab_pos, drab_time); drab_* are accumulated into if given."""
    if dq is None:
        dq = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    if dk is None:
        dk = torch.empty(k.shape, dtype=k.dtype, device=k.device)
    if dv is None:
        dv = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if drab_pos is None:
        drab_pos = torch.zeros(rab_pos.shape, dtype=torch.float32, device=q.device)
    if drab_time is None:
        drab_time = torch.zeros(rab_time.shape, dtype=torch.float32, device=q.device)
    p = make_params(q, k, v, seq_offsets, max_seq_len=max_seq_len,
                    num_pos_buckets=rab_pos.shape[-1], num_time_buckets=rab_time.shape[-1],
                    time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                    silu_scale=silu_scale, num_candidates=num_candidates,
                    rab_per_head=rab_per_head, impl=impl, dout=dout, dq=dq, dk=dk, dv=dv)
    off = _host_i64(seq_offsets)
    nc = _host_i32(num_candidates)
    ws = _workspace(attn_workspace_size(p, off, True), q.device, workspace)
    _check(LIB.hstu_attn_bwd(ctypes.byref(p), off.ctypes.data,
                             None if nc is None else nc.ctypes.data, _ptr(timestamps), _ptr(q),
                             _ptr(k), _ptr(v), _ptr(rab_pos), _ptr(rab_time), _ptr(dout),
                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(drab_pos), _ptr(drab_time),
                             _ptr(ws), ws.numel(), _stream(stream)), "hstu_attn_bwd")
    return dq, dk, dv, drab_pos, drab_time


def _layer_params(x, rab_pos, rab_time, seq_offsets, num_candidates, *, num_heads, d_qk, d_v,
                  max_seq_len, time_bucket_sub_bits, alpha, silu_scale, ln_eps, residual):
    off = _host_i64(seq_offsets)
    nc = _host_i32(num_candidates)
    lp = LayerParams()
    a = lp.attn
    a.batch = len(off) - 1
    a.num_heads, a.d_qk, a.d_v = num_heads, d_qk, d_v
    a.max_seq_len = int(max_seq_len)
    a.num_pos_buckets, a.num_time_buckets = rab_pos.shape[-1], rab_time.shape[-1]
    a.time_bucket_sub_bits = int(time_bucket_sub_bits)
    a.rab_per_head = 0
    a.mask = MASK_MFALCON if nc is not None else MASK_CAUSAL
    a.dtype = BF16
    a.impl = 0
    a.alpha = float(1.0 / math.sqrt(d_qk) if alpha is None else alpha)
    a.silu_scale = float(1.0 / max(1, int(max_seq_len)) if silu_scale is None else silu_scale)
    lp.d_model = x.shape[1]
    lp.residual = int(bool(residual))
    lp.ln_eps = float(ln_eps)
    return lp, off, nc


def layer_fwd(x, w1, b1, ln_gamma, ln_beta, w2, b2, rab_pos, rab_time, seq_offsets, timestamps,
              *, num_heads, d_qk, d_v, max_seq_len, time_bucket_sub_bits, alpha=None,
              silu_scale=None, num_candidates=None, ln_eps=1e-5, residual=True, out=None,
              workspace=None, stream=None):
    """One HSTU layer forward, bf16 (include/hstu.h, hstu_layer_fwd)."""
    T, D = x.shape
    if out is None:
        out = torch.empty((T, D), dtype=torch.bfloat16, device=x.device)
    lp, off, nc = _layer_params(x, rab_pos, rab_time, seq_offsets, num_candidates,
                                num_heads=num_heads, d_qk=d_qk, d_v=d_v, max_seq_len=max_seq_len,
                                time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                                silu_scale=silu_scale, ln_eps=ln_eps, residual=residual)
    n = ctypes.c_size_t(0)
    _check(LIB.hstu_layer_workspace_size(ctypes.byref(lp), off.ctypes.data, ctypes.byref(n)),
           "hstu_layer_workspace_size")
    ws = _workspace(int(n.value), x.device, workspace)
    _check(LIB.hstu_layer_fwd(ctypes.byref(lp), off.ctypes.data,
                              None if nc is None else nc.ctypes.data, _ptr(timestamps), _ptr(x),
                              _ptr(w1), _ptr(b1), _ptr(ln_gamma), _ptr(ln_beta), _ptr(w2),
                              _ptr(b2), _ptr(rab_pos), _ptr(rab_time), _ptr(out), _ptr(ws),
                              ws.numel(), _stream(stream)), "hstu_layer_fwd")
    return out


def layer_fwd_keep_proj(x, w1, b1, ln_gamma, ln_beta, w2, b2, rab_pos, rab_time, seq_offsets,
                        timestamps, *, num_heads, d_qk, d_v, max_seq_len, time_bucket_sub_bits,
                        alpha=None, silu_scale=None, num_candidates=None, ln_eps=1e-5,
                        residual=True, out=None, proj_out=None, workspace=None, stream=None):
    """hstu_layer_fwd_keep_proj: (y, proj) with proj = [U|V|Q|K] [T, N1] bf16,
    the history K/V cache of the M-FALCON candidate path."""
    T, D = x.shape
    n1 = 2 * num_heads * (d_v + d_qk)
    if out is None:
        out = torch.empty((T, D), dtype=torch.bfloat16, device=x.device)
    if proj_out is None:
        proj_out = torch.empty((T, n1), dtype=torch.bfloat16, device=x.device)
    lp, off, nc = _layer_params(x, rab_pos, rab_time, seq_offsets, num_candidates,
                                num_heads=num_heads, d_qk=d_qk, d_v=d_v, max_seq_len=max_seq_len,
                                time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                                silu_scale=silu_scale, ln_eps=ln_eps, residual=residual)
    n = ctypes.c_size_t(0)
    _check(LIB.hstu_layer_workspace_size(ctypes.byref(lp), off.ctypes.data, ctypes.byref(n)),
           "hstu_layer_workspace_size")
    ws = _workspace(int(n.value), x.device, workspace)
    _check(LIB.hstu_layer_fwd_keep_proj(
        ctypes.byref(lp), off.ctypes.data, None if nc is None else nc.ctypes.data,
        _ptr(timestamps), _ptr(x), _ptr(w1), _ptr(b1), _ptr(ln_gamma), _ptr(ln_beta), _ptr(w2),
        _ptr(b2), _ptr(rab_pos), _ptr(rab_time), _ptr(out), _ptr(proj_out), _ptr(ws),
        ws.numel(), _stream(stream)), "hstu_layer_fwd_keep_proj")
    return out, proj_out


def attn_fwd_candidates(q, k, v, k_hist, v_hist, hist_offsets, cand_offsets, hist_timestamps,
                        cand_timestamps, rab_pos, rab_time, *, max_seq_len,
                        time_bucket_sub_bits, alpha=None, silu_scale=None, rab_per_head=False,
                        out=None, workspace=None, stream=None):
    """hstu_attn_fwd_candidates: out[Tc, H, d_v] for a candidate micro-batch
    against cached history keys / values k_hist, v_hist [Th, H, d]."""
    Tc, H = q.shape[0], q.shape[1]
    d_v = v.shape[-1] if v.dim() == 3 else v.shape[1] // H
    if out is None:
        out = torch.empty((Tc, H, d_v), dtype=q.dtype, device=q.device)
    hoff = _host_i64(hist_offsets)
    coff = _host_i64(cand_offsets)
    p = make_params(q, k, v, coff, max_seq_len=max_seq_len, num_pos_buckets=rab_pos.shape[-1],
                    num_time_buckets=rab_time.shape[-1],
                    time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                    silu_scale=silu_scale, rab_per_head=rab_per_head, out=out)
    kh_rs = _row_stride(k_hist, H, q.shape[2], "k_hist")
    vh_rs = _row_stride(v_hist, H, d_v, "v_hist")
    n = ctypes.c_size_t(0)
    _check(LIB.hstu_attn_candidates_workspace_size(ctypes.byref(p), hoff.ctypes.data,
                                                   coff.ctypes.data, ctypes.byref(n)),
           "hstu_attn_candidates_workspace_size")
    ws = _workspace(int(n.value), q.device, workspace)
    _check(LIB.hstu_attn_fwd_candidates(
        ctypes.byref(p), hoff.ctypes.data, coff.ctypes.data, _ptr(hist_timestamps),
        _ptr(cand_timestamps), _ptr(q), _ptr(k), _ptr(v), _ptr(k_hist), _ptr(v_hist), kh_rs,
        vh_rs, _ptr(rab_pos), _ptr(rab_time), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
        "hstu_attn_fwd_candidates")
    return out


def layer_fwd_candidates(x_cand, w1, b1, ln_gamma, ln_beta, w2, b2, rab_pos, rab_time,
                         hist_proj, hist_offsets, cand_offsets, hist_timestamps,
                         cand_timestamps, *, num_heads, d_qk, d_v, max_seq_len,
                         time_bucket_sub_bits, alpha=None, silu_scale=None, ln_eps=1e-5,
                         residual=True, out=None, workspace=None, stream=None):
    """hstu_layer_fwd_candidates: one layer on a candidate micro-batch against
    the history projection kept by layer_fwd_keep_proj."""
    Tc, D = x_cand.shape
    if out is None:
        out = torch.empty((Tc, D), dtype=torch.bfloat16, device=x_cand.device)
    hoff = _host_i64(hist_offsets)
    coff = _host_i64(cand_offsets)
    lp, _, _ = _layer_params(x_cand, rab_pos, rab_time, coff, None, num_heads=num_heads,
                             d_qk=d_qk, d_v=d_v, max_seq_len=max_seq_len,
                             time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                             silu_scale=silu_scale, ln_eps=ln_eps, residual=residual)
    lp.attn.mask = MASK_MFALCON
    n = ctypes.c_size_t(0)
    _check(LIB.hstu_layer_candidates_workspace_size(ctypes.byref(lp), hoff.ctypes.data,
                                                    coff.ctypes.data, ctypes.byref(n)),
           "hstu_layer_candidates_workspace_size")
    ws = _workspace(int(n.value), x_cand.device, workspace)
    _check(LIB.hstu_layer_fwd_candidates(
        ctypes.byref(lp), hoff.ctypes.data, coff.ctypes.data, _ptr(hist_timestamps),
        _ptr(cand_timestamps), _ptr(x_cand), _ptr(w1), _ptr(b1), _ptr(ln_gamma), _ptr(ln_beta),
        _ptr(w2), _ptr(b2), _ptr(rab_pos), _ptr(rab_time), _ptr(hist_proj), _ptr(out),
        _ptr(ws), ws.numel(), _stream(stream)), "hstu_layer_fwd_candidates")
    return out


def layer_bwd(x, w1, b1, ln_gamma, ln_beta, w2, b2, rab_pos, rab_time, seq_offsets, timestamps,
              dy, *, num_heads, d_qk, d_v, max_seq_len, time_bucket_sub_bits, alpha=None,
              silu_scale=None, num_candidates=None, ln_eps=1e-5, residual=True, dx=None,
              grads=None, workspace=None, stream=None):
    """One HSTU layer backward (include/hstu.h, hstu_layer_bwd).

    Returns (dx, grads) with grads a dict of float32 tensors dw1, db1,
    dgamma, dbeta, dw2, db2, drab_pos, drab_time; pass ``grads`` to
    accumulate into existing ones (the library adds to them)."""
    T, D = x.shape
    dev = x.device
    if dx is None:
        dx = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    if grads is None:
        z = lambda t: torch.zeros(t.shape, dtype=torch.float32, device=dev)
        grads = dict(dw1=z(w1), db1=z(b1), dgamma=z(ln_gamma), dbeta=z(ln_beta), dw2=z(w2),
                     db2=z(b2), drab_pos=z(rab_pos), drab_time=z(rab_time))
    lp, off, nc = _layer_params(x, rab_pos, rab_time, seq_offsets, num_candidates,
                                num_heads=num_heads, d_qk=d_qk, d_v=d_v, max_seq_len=max_seq_len,
                                time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                                silu_scale=silu_scale, ln_eps=ln_eps, residual=residual)
    n = ctypes.c_size_t(0)
    _check(LIB.hstu_layer_bwd_workspace_size(ctypes.byref(lp), off.ctypes.data,
                                             ctypes.byref(n)), "hstu_layer_bwd_workspace_size")
    ws = _workspace(int(n.value), dev, workspace)
    g = grads
    _check(LIB.hstu_layer_bwd(ctypes.byref(lp), off.ctypes.data,
                              None if nc is None else nc.ctypes.data, _ptr(timestamps), _ptr(x),
                              _ptr(w1), _ptr(b1), _ptr(ln_gamma), _ptr(ln_beta), _ptr(w2),
                              _ptr(b2), _ptr(rab_pos), _ptr(rab_time), _ptr(dy), _ptr(dx),
                              _ptr(g["dw1"]), _ptr(g["db1"]), _ptr(g["dgamma"]),
                              _ptr(g["dbeta"]), _ptr(g["dw2"]), _ptr(g["db2"]),
                              _ptr(g["drab_pos"]), _ptr(g["drab_time"]), _ptr(ws), ws.numel(),
                              _stream(stream)), "hstu_layer_bwd")
    return dx, grads


def debug_buckets(seq_offsets, timestamps, *, num_heads, d_qk, d_v, max_seq_len,
                  num_pos_buckets, num_time_buckets, time_bucket_sub_bits,
                  num_candidates=None, stream=None):
    """(bp, bt, bt_fast) int32 device tensors, dense L x L blocks per sequence."""
    off = _host_i64(seq_offsets)
    L = np.diff(off)
    n = int((L.astype(np.int64) ** 2).sum())
    dev = timestamps.device
    dummy = torch.empty((1, num_heads, d_qk), dtype=torch.bfloat16, device=dev)
    dummy_v = torch.empty((1, num_heads, d_v), dtype=torch.bfloat16, device=dev)
    p = make_params(dummy, dummy, dummy_v, off, max_seq_len=max_seq_len,
                    num_pos_buckets=num_pos_buckets, num_time_buckets=num_time_buckets,
                    time_bucket_sub_bits=time_bucket_sub_bits, num_candidates=num_candidates)
    nc = _host_i32(num_candidates)
    ws = _workspace(attn_workspace_size(p, off, False), dev, None)
    bp = torch.empty(max(n, 1), dtype=torch.int32, device=dev)
    bt = torch.empty(max(n, 1), dtype=torch.int32, device=dev)
    btf = torch.empty(max(n, 1), dtype=torch.int32, device=dev)
    _check(LIB.hstu_debug_buckets(ctypes.byref(p), off.ctypes.data,
                                  None if nc is None else nc.ctypes.data, _ptr(timestamps),
                                  _ptr(bp), _ptr(bt), _ptr(btf), _ptr(ws), ws.numel(),
                                  _stream(stream)), "hstu_debug_buckets")
    return bp[:n], bt[:n], btf[:n]


def get_device_error(workspace: torch.Tensor, stream=None):
    detail = ctypes.c_uint32(0)
    rc = LIB.hstu_get_device_error(_ptr(workspace), _stream(stream), ctypes.byref(detail))
    return rc, int(detail.value)


def debug_wait_probe(workspace: torch.Tensor, limit_us: int, stream=None) -> int:
    """hstu_debug_wait_probe: a device wait that runs out after limit_us."""
    return int(LIB.hstu_debug_wait_probe(_ptr(workspace), workspace.numel() *
                                         workspace.element_size(), int(limit_us),
                                         _stream(stream)))


def set_wait_limit(microseconds: int) -> None:
    LIB.hstu_set_wait_limit(int(microseconds))


def attn_fwd_noalloc(q, k, v, seq_offsets, timestamps, rab_pos, rab_time, *, max_seq_len,
                     time_bucket_sub_bits, alpha=None, silu_scale=None, num_candidates=None,
                     rab_per_head=False, impl="auto", out=None, stream=None):
    """hstu_attn_fwd_noalloc: the forward without a workspace, for callers that
    cannot allocate device memory; its scratch is a fixed device array inside
    the library (see include/hstu.h).  `out` must be given by such callers."""
    T, H = q.shape[0], q.shape[1]
    d_v = v.shape[-1] if v.dim() == 3 else v.shape[1] // H
    if out is None:
        out = torch.empty((T, H, d_v), dtype=q.dtype, device=q.device)
    p = make_params(q, k, v, seq_offsets, max_seq_len=max_seq_len,
                    num_pos_buckets=rab_pos.shape[-1], num_time_buckets=rab_time.shape[-1],
                    time_bucket_sub_bits=time_bucket_sub_bits, alpha=alpha,
                    silu_scale=silu_scale, num_candidates=num_candidates,
                    rab_per_head=rab_per_head, impl=impl, out=out)
    off = _host_i64(seq_offsets)
    nc = _host_i32(num_candidates)
    _check(LIB.hstu_attn_fwd_noalloc(ctypes.byref(p), off.ctypes.data,
                                     None if nc is None else nc.ctypes.data, _ptr(timestamps),
                                     _ptr(q), _ptr(k), _ptr(v), _ptr(rab_pos), _ptr(rab_time),
                                     _ptr(out), _stream(stream)), "hstu_attn_fwd_noalloc")
    return out


def partition_batch(seq_offsets, world: int, num_candidates=None):
    """hstu_partition_batch: (rank_of_seq int32 [B], pairs_per_rank int64 [world])."""
    off = _host_i64(seq_offsets)
    nc = _host_i32(num_candidates)
    B = len(off) - 1
    rank_of = np.zeros(max(B, 1), np.int32)
    pairs = np.zeros(max(int(world), 1), np.int64)
    _check(LIB.hstu_partition_batch(off.ctypes.data, None if nc is None else nc.ctypes.data,
                                    int(B), int(world), rank_of.ctypes.data, pairs.ctypes.data),
           "hstu_partition_batch")
    return rank_of[:B], pairs[:int(world)]


def version() -> str:
    return LIB.hstu_version().decode()


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(LIB.hstu_kernel_launch_count())


# Phase traces of the tensor-core kernels (library built with `build --trace`):
# three CTAs x one recorder per warp x entries (code << 56 | ordinal << 40 | clock).
TRACE_SHAPE = (3, 20, 1024)
TRACE_KERNEL = {"bwd": 0, "fwd": 1}


def trace_clear(kernel: str = "bwd") -> None:
    _check(LIB.hstu_debug_trace_clear(TRACE_KERNEL[kernel]), "hstu_debug_trace_clear")


def trace_read(kernel: str = "bwd") -> np.ndarray:
    buf = np.zeros(TRACE_SHAPE, dtype=np.uint64)
    _check(LIB.hstu_debug_trace_read(TRACE_KERNEL[kernel], buf.ctypes.data, buf.nbytes),
           "hstu_debug_trace_read")
    return buf


def debug_plan(p: "AttnParams", seq_offsets, num_candidates=None):
    """(forward items, backward items) as int32 [n, 4] arrays (include/hstu.h,
    hstu_debug_plan); host only."""
    off = _host_i64(seq_offsets)
    nc = _host_i32(num_candidates)
    nf, nb = ctypes.c_int32(0), ctypes.c_int32(0)
    cap = 16
    while True:
        fi = np.zeros((cap, 4), dtype=np.int32)
        bi = np.zeros((cap, 4), dtype=np.int32)
        rc = LIB.hstu_debug_plan(ctypes.byref(p), off.ctypes.data,
                                 None if nc is None else nc.ctypes.data, cap, fi.ctypes.data,
                                 ctypes.byref(nf), bi.ctypes.data, ctypes.byref(nb))
        if rc == HSTU_OK:
            return fi[:nf.value].copy(), bi[:nb.value].copy()
        if nf.value <= cap and nb.value <= cap:
            _check(rc, "hstu_debug_plan")
        cap = max(nf.value, nb.value)

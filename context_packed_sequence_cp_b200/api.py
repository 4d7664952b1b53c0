"""Python binding of libthdcp: the C ABI's entry points under the same names, with
torch tensors for device memory and the current torch stream.  Argument marshalling
only; every step runs in the library's CUDA kernels.  Arguments after the tensors
are keyword-only, so that no argument can land in the wrong position.

Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance".
"""
from __future__ import annotations

import ctypes
import math

import numpy as np
import torch

from ._lib import (EN_FIELDS, QT_FIELDS, THD_DTYPE_BF16, THD_DTYPE_FP32, PlanInfo, check, lib)

_DTYPES = {torch.bfloat16: THD_DTYPE_BF16, torch.float32: THD_DTYPE_FP32}


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class Plan:
    """thd_cp_plan: the symmetric partition and the cached tile metadata of one packed
    layout.  Host tables on construction; device tables after ``upload``."""

    def __init__(self, cu_seqlens, cp: int):
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        h = ctypes.c_void_p()
        check("thd_cp_plan", lib().thd_cp_plan(_i32p(cu), int(cu.size - 1), int(cp), ctypes.byref(h)))
        self._h = h
        self.cu_seqlens = cu
        info = PlanInfo()
        check("thd_cp_plan_info", lib().thd_cp_plan_info(self._h, ctypes.byref(info)))
        self.T, self.cp, self.n_docs = int(info.T), int(info.cp), int(info.n_docs)
        self.Tl, self.n_qtiles, self.n_entries = int(info.Tl), int(info.n_qtiles), int(info.n_entries)
        self.causal_pairs = int(info.causal_pairs)
        self.uploaded = False

    @property
    def handle(self):
        return self._h

    def export(self) -> dict:
        T, nq, ne = self.T, self.n_qtiles, self.n_entries
        out = dict(q_idx=np.empty(T, np.int32), rm_of_global=np.empty(T, np.int32),
                   qtiles=np.empty((nq, QT_FIELDS), np.int32), entries=np.empty((ne, EN_FIELDS), np.int32),
                   lpt=np.empty(nq, np.int32), kt_off=np.empty(nq + 1, np.int32),
                   kt_list=np.empty((ne, 2), np.int32), kt_lpt=np.empty(nq, np.int32))
        check("thd_cp_plan_export", lib().thd_cp_plan_export(
            self._h, *(_i32p(out[k]) for k in ("q_idx", "rm_of_global", "qtiles", "entries", "lpt",
                                                "kt_off", "kt_list", "kt_lpt"))))
        return out

    def upload(self, stream=None) -> "Plan":
        check("thd_cp_plan_upload", lib().thd_cp_plan_upload(self._h, _stream(stream)))
        self.uploaded = True
        return self

    def device_status(self, reset: bool = True) -> int:
        v = ctypes.c_int32()
        check("thd_cp_device_status", lib().thd_cp_device_status(self._h, int(reset), ctypes.byref(v)))
        return int(v.value)

    def close(self):
        if getattr(self, "_h", None):
            lib().thd_cp_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def thd_cu_seqlens_from_eod(tokens, eod_id: int) -> np.ndarray:
    """Document boundaries of an EOD-delimited packed sequence (host int32 token ids):
    a document ends with, and includes, each EOD token; the tokens after the last EOD
    form a final document.  Returns cu_seqlens as an int32 array."""
    tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).ravel())
    n = ctypes.c_int32(0)
    rc = lib().thd_cu_seqlens_from_eod(_i32p(tok), tok.size, int(eod_id), None, 0, ctypes.byref(n))
    if rc not in (0, -9):
        check("thd_cu_seqlens_from_eod", rc)
    cu = np.zeros(n.value + 1, dtype=np.int32)
    check("thd_cu_seqlens_from_eod", lib().thd_cu_seqlens_from_eod(
        _i32p(tok), tok.size, int(eod_id), _i32p(cu), cu.size, ctypes.byref(n)))
    return cu


def thd_position_ids(cu_seqlens) -> np.ndarray:
    """Per-document position ids: token t of document d gets t - cu_seqlens[d]."""
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    pos = np.zeros(int(cu[-1]) if cu.size else 0, dtype=np.int32)
    check("thd_position_ids", lib().thd_position_ids(_i32p(cu), cu.size - 1, _i32p(pos)))
    return pos


def thd_rope_apply(x: torch.Tensor, pos: torch.Tensor, *, rot_dim: int | None = None, base: float = 10000.0,
                   workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Rotary position embedding (half-split) in place on bf16 x [T, heads, dim] with
    per-row positions pos (device int32 [T]); returns x."""
    T, heads, dim = x.shape
    rot_dim = dim if rot_dim is None else int(rot_dim)
    n = ctypes.c_size_t()
    check("thd_rope_workspace", lib().thd_rope_workspace(T, rot_dim, ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=x.device)
    check("thd_rope_apply", lib().thd_rope_apply(
        _ptr(x), _ptr(pos), T, heads, dim, rot_dim, float(base), _DTYPES[x.dtype], _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return x


def thd_cp_plan(cu_seqlens, cp: int) -> Plan:
    return Plan(cu_seqlens, cp)


def thd_kv_gather(plan: Plan, k: torch.Tensor, v: torch.Tensor | None = None, *,
                  k_rm: torch.Tensor | None = None, v_rm: torch.Tensor | None = None, stream=None):
    """k_rm[j] = k[q_idx[j]] (and v): the rank-major all-gather layout."""
    k = k.contiguous()
    k_rm = torch.empty_like(k) if k_rm is None else k_rm
    if v is not None:
        v = v.contiguous()
        v_rm = torch.empty_like(v) if v_rm is None else v_rm
    rb_k = k.numel() // plan.T * k.element_size()
    rb_v = (v.numel() // plan.T * v.element_size()) if v is not None else 0
    check("thd_kv_gather", lib().thd_kv_gather(plan.handle, _ptr(k), _ptr(v), _ptr(k_rm), _ptr(v_rm),
                                               rb_k, rb_v, _stream(stream)))
    return (k_rm, v_rm) if v is not None else k_rm


def thd_rows_to_global(plan: Plan, src_rm: torch.Tensor, *, out: torch.Tensor | None = None, stream=None):
    """out[g] = src_rm[rm_of_global[g]]: rank-major rows back to packed order."""
    src_rm = src_rm.contiguous()
    out = torch.empty_like(src_rm) if out is None else out
    rb = src_rm.numel() // plan.T * src_rm.element_size()
    check("thd_rows_to_global", lib().thd_rows_to_global(plan.handle, _ptr(src_rm), _ptr(out), rb,
                                                         _stream(stream)))
    return out


def thd_cp_attn_fwd(plan: Plan, q_rm: torch.Tensor, k_rm: torch.Tensor, v_rm: torch.Tensor, *,
                    scale: float | None = None, out: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, stream=None):
    """Causal attention with EOD resets over rank-major Q/K/V; returns (o_rm, lse_rm [hq, T])."""
    T, hq, dqk = q_rm.shape
    hkv, dv = k_rm.shape[1], v_rm.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    dt = _DTYPES[q_rm.dtype]
    out = torch.empty((T, hq, dv), dtype=q_rm.dtype, device=q_rm.device) if out is None else out
    lse = torch.empty((hq, T), dtype=torch.float32, device=q_rm.device) if lse is None else lse
    check("thd_cp_attn_fwd", lib().thd_cp_attn_fwd(
        plan.handle, _ptr(q_rm), _ptr(k_rm), _ptr(v_rm), _ptr(out), _ptr(lse), hq, hkv, dqk, dv,
        float(scale), dt, _stream(stream)))
    return out, lse


def thd_cp_attn_fwd_mla(plan: Plan, q_rm: torch.Tensor, k_nope_rm: torch.Tensor, k_rope_rm: torch.Tensor,
                        v_rm: torch.Tensor, *, scale: float | None = None, out: torch.Tensor | None = None,
                        lse: torch.Tensor | None = None, stream=None):
    """thd_cp_attn_fwd with multi-head latent attention keys in compact form: k_nope_rm
    [T, hkv, d_nope] per head and k_rope_rm [T, d_rope] shared by every head; q_rm is
    [T, hq, d_nope + d_rope].  Returns (o_rm, lse_rm [hq, T])."""
    T, hq, dq = q_rm.shape
    hkv, d_nope = k_nope_rm.shape[1], k_nope_rm.shape[2]
    d_rope, dv = k_rope_rm.shape[-1], v_rm.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(dq)
    out = torch.empty((T, hq, dv), dtype=q_rm.dtype, device=q_rm.device) if out is None else out
    lse = torch.empty((hq, T), dtype=torch.float32, device=q_rm.device) if lse is None else lse
    check("thd_cp_attn_fwd_mla", lib().thd_cp_attn_fwd_mla(
        plan.handle, _ptr(q_rm), _ptr(k_nope_rm), _ptr(k_rope_rm), _ptr(v_rm), _ptr(out), _ptr(lse), hq, hkv,
        d_nope, d_rope, dv, float(scale), _DTYPES[q_rm.dtype], _stream(stream)))
    return out, lse


def thd_cp_attn_bwd_workspace(plan: Plan, *, hq: int, hkv: int, dqk: int, dv: int,
                              dtype: torch.dtype = torch.bfloat16) -> int:
    n = ctypes.c_size_t()
    check("thd_cp_attn_bwd_workspace", lib().thd_cp_attn_bwd_workspace(
        plan.handle, hq, hkv, dqk, dv, _DTYPES[dtype], ctypes.byref(n)))
    return int(n.value)


def thd_cp_attn_bwd(plan: Plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, *, scale: float | None = None,
                    dq: torch.Tensor | None = None, dk: torch.Tensor | None = None,
                    dv: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Gradients (dq_rm, dk_rm, dv_rm), fp32, rank-major."""
    T, hq, dqk = q_rm.shape
    hkv, dvd = k_rm.shape[1], v_rm.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    dev = q_rm.device
    dq = torch.empty((T, hq, dqk), dtype=torch.float32, device=dev) if dq is None else dq
    dk = torch.empty((T, hkv, dqk), dtype=torch.float32, device=dev) if dk is None else dk
    dv = torch.empty((T, hkv, dvd), dtype=torch.float32, device=dev) if dv is None else dv
    nbytes = thd_cp_attn_bwd_workspace(plan, hq=hq, hkv=hkv, dqk=dqk, dv=dvd, dtype=q_rm.dtype)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    check("thd_cp_attn_bwd", lib().thd_cp_attn_bwd(
        plan.handle, _ptr(q_rm), _ptr(k_rm), _ptr(v_rm), _ptr(o_rm), _ptr(lse_rm), _ptr(do_rm),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
        hq, hkv, dqk, dvd, float(scale), _DTYPES[q_rm.dtype], _stream(stream)))
    return dq, dk, dv


def thd_cp_attn_bwd_noalloc(plan: Plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, *, scale: float | None = None,
                            dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor, stream=None):
    """thd_cp_attn_bwd without a workspace, for callers that cannot allocate device
    memory: the library keeps the per-row statistic in a fixed device array
    (hq * T <= 8,388,608).  Outputs must be passed in (fp32, rank-major)."""
    T, hq, dqk = q_rm.shape
    hkv, dvd = k_rm.shape[1], v_rm.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    check("thd_cp_attn_bwd_noalloc", lib().thd_cp_attn_bwd_noalloc(
        plan.handle, _ptr(q_rm), _ptr(k_rm), _ptr(v_rm), _ptr(o_rm), _ptr(lse_rm), _ptr(do_rm),
        _ptr(dq), _ptr(dk), _ptr(dv), hq, hkv, dqk, dvd, float(scale), _DTYPES[q_rm.dtype], _stream(stream)))
    return dq, dk, dv

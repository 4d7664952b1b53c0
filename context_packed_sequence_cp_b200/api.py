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

from ._lib import (ERRORS, EN_FIELDS, QT_FIELDS, THD_DTYPE_BF16, THD_DTYPE_FP32, PlanInfo, ThdError, check,
                   lib)

_DTYPES = {torch.bfloat16: THD_DTYPE_BF16, torch.float32: THD_DTYPE_FP32}
_CODE = {kind: code for code, kind in ERRORS.items()}


# ---------------------------------------------------------------- argument checks
# The C ABI receives bare device pointers, so it cannot see a tensor's device, shape or
# layout; a tensor with the wrong row count or on the wrong device would be read out of
# bounds by the kernels.  These checks run before any call into the library.  Whether a
# dtype or width is supported, pointer alignment and row sizes stay the library's checks.

def _current_device() -> int:
    return torch.cuda.current_device()


def _on_device(t: torch.Tensor, dev: int) -> bool:
    return t.is_cuda and t.device.index == dev


def _bad(fn: str, text: str):
    raise ThdError(fn, _CODE["INVALID_ARG"], text)


def _ready(fn: str, plan: "Plan") -> int:
    """The library's first check (uploaded device tables), then the device: kernels run
    on the current device, which must hold the plan's tables.  Returns that device."""
    if not plan.uploaded:
        check(fn, _CODE["NOT_UPLOADED"])
    dev = _current_device()
    if dev != plan.device:
        _bad(fn, f"the plan's tables are on cuda:{plan.device}, the current device is cuda:{dev}")
    return dev


def _dims(fn: str, name: str, t, n: int) -> tuple:
    if not isinstance(t, torch.Tensor):
        _bad(fn, f"{name} must be a torch.Tensor")
    if t.dim() != n:
        _bad(fn, f"{name} must have {n} dimensions, got shape {tuple(t.shape)}")
    return tuple(t.shape)


def _want(fn: str, name: str, t, dev: int, shape=None, dtype=None) -> torch.Tensor:
    """A device argument: a contiguous tensor on `dev`, of exactly `shape` and `dtype`
    where given."""
    if not isinstance(t, torch.Tensor):
        _bad(fn, f"{name} must be a torch.Tensor")
    if not _on_device(t, dev):
        _bad(fn, f"{name} must be a CUDA tensor on cuda:{dev}, got {t.device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        _bad(fn, f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        _bad(fn, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        _bad(fn, f"{name} must be contiguous")
    return t


def _dtype_code(fn: str, t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise ThdError(fn, _CODE["UNSUPPORTED"], f"dtype {t.dtype} (bf16 and fp32 are built)")
    return _DTYPES[t.dtype]


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
        self._refresh(cu)
        self.uploaded = False
        self.device = None

    @property
    def handle(self):
        return self._h

    def export(self) -> dict:
        T, nq, ne = self.T, self.n_qtiles, self.n_entries
        out = dict(q_idx=np.empty(T, np.int32), rm_of_global=np.empty(T, np.int32),
                   qtiles=np.empty((nq, QT_FIELDS), np.int32), entries=np.empty((ne, EN_FIELDS), np.int32),
                   lpt=np.empty(nq, np.int32), kt_off=np.empty(nq + 1, np.int32),
                   kt_list=np.empty((ne, 2), np.int32), kt_lpt=np.empty(nq, np.int32),
                   kt_seg=np.empty(self.n_kseg + 1, np.int32))
        check("thd_cp_plan_export", lib().thd_cp_plan_export(
            self._h, *(_i32p(out[k]) for k in ("q_idx", "rm_of_global", "qtiles", "entries", "lpt",
                                                "kt_off", "kt_list", "kt_lpt", "kt_seg"))))
        return out

    def export_fwd(self) -> dict:
        """The forward tables (thd_cp_plan_export_fwd)."""
        nf, ne = self.n_fqtiles, self.n_fentries
        out = dict(fqtiles=np.empty((nf, QT_FIELDS), np.int32), fentries=np.empty((ne, EN_FIELDS), np.int32),
                   flpt=np.empty(nf, np.int32), fkt_off=np.empty(nf + 1, np.int32),
                   fkt_list=np.empty((ne, 2), np.int32), fkt_lpt=np.empty(nf, np.int32),
                   fkt_seg=np.empty(self.n_fkseg + 1, np.int32))
        check("thd_cp_plan_export_fwd", lib().thd_cp_plan_export_fwd(
            self._h, *(_i32p(out[k]) for k in ("fqtiles", "fentries", "flpt", "fkt_off", "fkt_list", "fkt_lpt",
                                                "fkt_seg"))))
        return out

    def upload(self, stream=None) -> "Plan":
        """Copies the tables to the current device; a second call is a no-op, as in the
        library, and the tables stay on the device of the first."""
        first = not self.uploaded
        check("thd_cp_plan_upload", lib().thd_cp_plan_upload(self._h, _stream(stream)))
        if first:
            self.uploaded = True
            self.device = _current_device()
        return self

    def update(self, cu_seqlens, cp: int | None = None, stream=None) -> "Plan":
        """thd_cp_plan_update: re-plan in place for a new layout (a new batch).  The host
        tables are rebuilt; if the plan was uploaded, the new tables are copied to its
        device on `stream` (the current stream by default), in stream order, without a
        device-wide synchronisation."""
        fn = "thd_cp_plan_update"
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        cp = self.cp if cp is None else int(cp)
        if self.uploaded:
            dev = _current_device()
            if dev != self.device:
                _bad(fn, f"the plan's tables are on cuda:{self.device}, the current device is cuda:{dev}")
            s = _stream(stream)
        else:
            s = ctypes.c_void_p(0)
        rc = lib().thd_cp_plan_update(self._h, _i32p(cu), int(cu.size - 1), cp, s)
        if rc != 0 and rc in (_CODE["CUDA"], _CODE["ALLOC"]):
            self.uploaded = False
        if rc == 0 or rc in (_CODE["CUDA"], _CODE["ALLOC"]):
            self._refresh(cu)
        check(fn, rc)
        return self

    def _refresh(self, cu):
        self.cu_seqlens = cu
        info = PlanInfo()
        check("thd_cp_plan_info", lib().thd_cp_plan_info(self._h, ctypes.byref(info)))
        self.T, self.cp, self.n_docs = int(info.T), int(info.cp), int(info.n_docs)
        self.Tl, self.n_qtiles, self.n_entries = int(info.Tl), int(info.n_qtiles), int(info.n_entries)
        self.causal_pairs = int(info.causal_pairs)
        self.n_kseg = int(info.n_kseg)
        self.n_fqtiles, self.n_fentries = int(info.n_fqtiles), int(info.n_fentries)
        self.n_fkseg = int(info.n_fkseg)

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
    fn = "thd_rope_apply"
    T, heads, dim = _dims(fn, "x", x, 3)
    dev = _current_device()
    _want(fn, "x", x, dev)
    _want(fn, "pos", pos, dev, (T,), torch.int32)
    rot_dim = dim if rot_dim is None else int(rot_dim)
    n = ctypes.c_size_t()
    check("thd_rope_workspace", lib().thd_rope_workspace(T, rot_dim, ctypes.byref(n)))
    if workspace is None:
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=x.device)
    _want(fn, "workspace", workspace, dev)
    check(fn, lib().thd_rope_apply(
        _ptr(x), _ptr(pos), T, heads, dim, rot_dim, float(base), _dtype_code(fn, x), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return x


def thd_cp_plan(cu_seqlens, cp: int) -> Plan:
    return Plan(cu_seqlens, cp)


def thd_kv_gather(plan: Plan, k: torch.Tensor, v: torch.Tensor | None = None, *,
                  k_rm: torch.Tensor | None = None, v_rm: torch.Tensor | None = None, stream=None):
    """k_rm[j] = k[q_idx[j]] (and v): the rank-major all-gather layout."""
    fn = "thd_kv_gather"
    dev = _ready(fn, plan)
    k = _want(fn, "k", k.contiguous() if isinstance(k, torch.Tensor) else k, dev)
    if k.dim() < 1 or k.shape[0] != plan.T:
        _bad(fn, f"k must have the plan's {plan.T} rows, got shape {tuple(k.shape)}")
    k_rm = torch.empty_like(k) if k_rm is None else _want(fn, "k_rm", k_rm, dev, k.shape, k.dtype)
    if v is not None:
        v = _want(fn, "v", v.contiguous() if isinstance(v, torch.Tensor) else v, dev)
        if v.dim() < 1 or v.shape[0] != plan.T:
            _bad(fn, f"v must have the plan's {plan.T} rows, got shape {tuple(v.shape)}")
        v_rm = torch.empty_like(v) if v_rm is None else _want(fn, "v_rm", v_rm, dev, v.shape, v.dtype)
    elif v_rm is not None:
        _bad(fn, "v_rm given without v")
    rb_k = k.numel() // plan.T * k.element_size()
    rb_v = (v.numel() // plan.T * v.element_size()) if v is not None else 0
    check(fn, lib().thd_kv_gather(plan.handle, _ptr(k), _ptr(v), _ptr(k_rm), _ptr(v_rm), rb_k, rb_v,
                                  _stream(stream)))
    return (k_rm, v_rm) if v is not None else k_rm


def thd_rows_to_global(plan: Plan, src_rm: torch.Tensor, *, out: torch.Tensor | None = None, stream=None):
    """out[g] = src_rm[rm_of_global[g]]: rank-major rows back to packed order."""
    fn = "thd_rows_to_global"
    dev = _ready(fn, plan)
    src_rm = _want(fn, "src_rm", src_rm.contiguous() if isinstance(src_rm, torch.Tensor) else src_rm, dev)
    if src_rm.dim() < 1 or src_rm.shape[0] != plan.T:
        _bad(fn, f"src_rm must have the plan's {plan.T} rows, got shape {tuple(src_rm.shape)}")
    out = torch.empty_like(src_rm) if out is None else _want(fn, "out", out, dev, src_rm.shape, src_rm.dtype)
    rb = src_rm.numel() // plan.T * src_rm.element_size()
    check(fn, lib().thd_rows_to_global(plan.handle, _ptr(src_rm), _ptr(out), rb, _stream(stream)))
    return out


def _qkv(fn: str, plan: Plan, dev: int, q_rm, k_rm, v_rm):
    """Q [T, hq, dqk], K [T, hkv, dqk], V [T, hkv, dv], one dtype; returns hq, hkv, dqk, dv."""
    T = plan.T
    _, hq, dqk = _dims(fn, "q_rm", q_rm, 3)
    _, hkv, _ = _dims(fn, "k_rm", k_rm, 3)
    dv = _dims(fn, "v_rm", v_rm, 3)[2]
    _want(fn, "q_rm", q_rm, dev, (T, hq, dqk))
    _want(fn, "k_rm", k_rm, dev, (T, hkv, dqk), q_rm.dtype)
    _want(fn, "v_rm", v_rm, dev, (T, hkv, dv), q_rm.dtype)
    return hq, hkv, dqk, dv


def thd_cp_attn_fwd(plan: Plan, q_rm: torch.Tensor, k_rm: torch.Tensor, v_rm: torch.Tensor, *,
                    scale: float | None = None, out: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, stream=None):
    """Causal attention with EOD resets over rank-major Q/K/V; returns (o_rm, lse_rm [hq, T])."""
    fn = "thd_cp_attn_fwd"
    dev = _ready(fn, plan)
    hq, hkv, dqk, dv = _qkv(fn, plan, dev, q_rm, k_rm, v_rm)
    T = plan.T
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    dt = _dtype_code(fn, q_rm)
    out = torch.empty((T, hq, dv), dtype=q_rm.dtype, device=q_rm.device) if out is None else out
    lse = torch.empty((hq, T), dtype=torch.float32, device=q_rm.device) if lse is None else lse
    _want(fn, "out", out, dev, (T, hq, dv), q_rm.dtype)
    _want(fn, "lse", lse, dev, (hq, T), torch.float32)
    check(fn, lib().thd_cp_attn_fwd(
        plan.handle, _ptr(q_rm), _ptr(k_rm), _ptr(v_rm), _ptr(out), _ptr(lse), hq, hkv, dqk, dv,
        float(scale), dt, _stream(stream)))
    return out, lse


def thd_cp_attn_fwd_fused_gather(plan: Plan, q_rm: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *,
                                 scale: float | None = None, out: torch.Tensor | None = None,
                                 lse: torch.Tensor | None = None, stream=None):
    """thd_cp_attn_fwd with K/V given in packed (global) order: the K/V all-gather is fused
    into the attention's loads.  q_rm is rank-major; returns (o_rm, lse_rm [hq, T])."""
    fn = "thd_cp_attn_fwd_fused_gather"
    dev = _ready(fn, plan)
    hq, hkv, dqk, dv = _qkv(fn, plan, dev, q_rm, k, v)
    T = plan.T
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    dt = _dtype_code(fn, q_rm)
    out = torch.empty((T, hq, dv), dtype=q_rm.dtype, device=q_rm.device) if out is None else out
    lse = torch.empty((hq, T), dtype=torch.float32, device=q_rm.device) if lse is None else lse
    _want(fn, "out", out, dev, (T, hq, dv), q_rm.dtype)
    _want(fn, "lse", lse, dev, (hq, T), torch.float32)
    check(fn, lib().thd_cp_attn_fwd_fused_gather(
        plan.handle, _ptr(q_rm), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), hq, hkv, dqk, dv, float(scale), dt,
        _stream(stream)))
    return out, lse


def thd_cp_attn_fwd_mla(plan: Plan, q_rm: torch.Tensor, k_nope_rm: torch.Tensor, k_rope_rm: torch.Tensor,
                        v_rm: torch.Tensor, *, scale: float | None = None, out: torch.Tensor | None = None,
                        lse: torch.Tensor | None = None, stream=None):
    """thd_cp_attn_fwd with multi-head latent attention keys in compact form: k_nope_rm
    [T, hkv, d_nope] per head and k_rope_rm [T, d_rope] shared by every head; q_rm is
    [T, hq, d_nope + d_rope].  Returns (o_rm, lse_rm [hq, T])."""
    fn = "thd_cp_attn_fwd_mla"
    dev = _ready(fn, plan)
    T = plan.T
    _, hq, dq = _dims(fn, "q_rm", q_rm, 3)
    _, hkv, d_nope = _dims(fn, "k_nope_rm", k_nope_rm, 3)
    dv = _dims(fn, "v_rm", v_rm, 3)[2]
    if not isinstance(k_rope_rm, torch.Tensor) or k_rope_rm.dim() not in (2, 3):
        _bad(fn, "k_rope_rm must be a [T, d_rope] tensor")
    d_rope = k_rope_rm.shape[-1]
    _want(fn, "q_rm", q_rm, dev, (T, hq, d_nope + d_rope))
    _want(fn, "k_nope_rm", k_nope_rm, dev, (T, hkv, d_nope), q_rm.dtype)
    _want(fn, "k_rope_rm", k_rope_rm, dev, (T, d_rope) if k_rope_rm.dim() == 2 else (T, 1, d_rope), q_rm.dtype)
    _want(fn, "v_rm", v_rm, dev, (T, hkv, dv), q_rm.dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(dq)
    dt = _dtype_code(fn, q_rm)
    out = torch.empty((T, hq, dv), dtype=q_rm.dtype, device=q_rm.device) if out is None else out
    lse = torch.empty((hq, T), dtype=torch.float32, device=q_rm.device) if lse is None else lse
    _want(fn, "out", out, dev, (T, hq, dv), q_rm.dtype)
    _want(fn, "lse", lse, dev, (hq, T), torch.float32)
    check(fn, lib().thd_cp_attn_fwd_mla(
        plan.handle, _ptr(q_rm), _ptr(k_nope_rm), _ptr(k_rope_rm), _ptr(v_rm), _ptr(out), _ptr(lse), hq, hkv,
        d_nope, d_rope, dv, float(scale), dt, _stream(stream)))
    return out, lse


def thd_cp_attn_bwd_workspace(plan: Plan, *, hq: int, hkv: int, dqk: int, dv: int,
                              dtype: torch.dtype = torch.bfloat16) -> int:
    fn = "thd_cp_attn_bwd_workspace"
    if dtype not in _DTYPES:
        raise ThdError(fn, _CODE["UNSUPPORTED"], f"dtype {dtype} (bf16 and fp32 are built)")
    n = ctypes.c_size_t()
    check(fn, lib().thd_cp_attn_bwd_workspace(plan.handle, hq, hkv, dqk, dv, _DTYPES[dtype], ctypes.byref(n)))
    return int(n.value)


def _bwd_args(fn: str, plan: Plan, dev: int, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq, dk, dv):
    """The backward's tensors: inputs as the forward's plus O, lse and dO, fp32 gradients
    in the shapes of Q, K and V (allocated when None).  Returns (hq, hkv, dqk, dvd, dq, dk, dv)."""
    T = plan.T
    hq, hkv, dqk, dvd = _qkv(fn, plan, dev, q_rm, k_rm, v_rm)
    _want(fn, "o_rm", o_rm, dev, (T, hq, dvd), q_rm.dtype)
    _want(fn, "lse_rm", lse_rm, dev, (hq, T), torch.float32)
    _want(fn, "do_rm", do_rm, dev, (T, hq, dvd), q_rm.dtype)
    f32 = dict(dtype=torch.float32, device=q_rm.device)
    dq = torch.empty((T, hq, dqk), **f32) if dq is None else dq
    dk = torch.empty((T, hkv, dqk), **f32) if dk is None else dk
    dv = torch.empty((T, hkv, dvd), **f32) if dv is None else dv
    _want(fn, "dq", dq, dev, (T, hq, dqk), torch.float32)
    _want(fn, "dk", dk, dev, (T, hkv, dqk), torch.float32)
    _want(fn, "dv", dv, dev, (T, hkv, dvd), torch.float32)
    return hq, hkv, dqk, dvd, dq, dk, dv


def thd_cp_attn_bwd(plan: Plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, *, scale: float | None = None,
                    dq: torch.Tensor | None = None, dk: torch.Tensor | None = None,
                    dv: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Gradients (dq_rm, dk_rm, dv_rm), fp32, rank-major."""
    fn = "thd_cp_attn_bwd"
    dev = _ready(fn, plan)
    hq, hkv, dqk, dvd, dq, dk, dv = _bwd_args(fn, plan, dev, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq, dk, dv)
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    dt = _dtype_code(fn, q_rm)
    nbytes = thd_cp_attn_bwd_workspace(plan, hq=hq, hkv=hkv, dqk=dqk, dv=dvd, dtype=q_rm.dtype)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q_rm.device)
    _want(fn, "workspace", workspace, dev)
    check(fn, lib().thd_cp_attn_bwd(
        plan.handle, _ptr(q_rm), _ptr(k_rm), _ptr(v_rm), _ptr(o_rm), _ptr(lse_rm), _ptr(do_rm),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
        hq, hkv, dqk, dvd, float(scale), dt, _stream(stream)))
    return dq, dk, dv


def thd_cp_attn_bwd_noalloc(plan: Plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, *, scale: float | None = None,
                            dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor, stream=None):
    """thd_cp_attn_bwd without a workspace, for callers that cannot allocate device
    memory: the library keeps the per-row statistic in a fixed device array
    (hq * T <= 8,388,608).  Outputs must be passed in (fp32, rank-major)."""
    fn = "thd_cp_attn_bwd_noalloc"
    dev = _ready(fn, plan)
    if dq is None or dk is None or dv is None:
        _bad(fn, "dq, dk and dv must be passed in")
    hq, hkv, dqk, dvd, dq, dk, dv = _bwd_args(fn, plan, dev, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq, dk, dv)
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    check(fn, lib().thd_cp_attn_bwd_noalloc(
        plan.handle, _ptr(q_rm), _ptr(k_rm), _ptr(v_rm), _ptr(o_rm), _ptr(lse_rm), _ptr(do_rm),
        _ptr(dq), _ptr(dk), _ptr(dv), hq, hkv, dqk, dvd, float(scale), _dtype_code(fn, q_rm), _stream(stream)))
    return dq, dk, dv

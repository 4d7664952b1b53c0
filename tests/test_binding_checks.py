"""The binding's argument checks, on the CPU.  Every call pattern that the GPU tests,
the smoke run and the benchmark make passes them and reaches the library; tensors with
the wrong rows, shape, dtype, layout or device are refused before any library call.
The library object is replaced by a recorder here, so no entry point ever receives a
host pointer."""
import ctypes

import pytest
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import _lib, api

HOST_CALLS = {"thd_cp_plan", "thd_cp_plan_info", "thd_cp_plan_export", "thd_cp_plan_destroy", "thd_cp_strerror"}


class Recorder:
    """Stands in for the loaded library: host planning calls go to the real library,
    every device entry point is recorded and reports success without running."""

    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in HOST_CALLS:
            return getattr(self.real, name)

        def call(*args):
            self.calls.append(name)
            return 0
        return call


@pytest.fixture
def rec(monkeypatch):
    r = Recorder(_lib.lib())
    monkeypatch.setattr(api, "lib", lambda: r)
    monkeypatch.setattr(api, "_current_device", lambda: 0)
    monkeypatch.setattr(api, "_on_device", lambda t, dev: True)
    monkeypatch.setattr(api, "_stream", lambda s: ctypes.c_void_p(0))
    return r


def _plan(lens=(64, 128), cp=2):
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    p = thd.Plan(cu, cp)
    p.uploaded, p.device = True, 0   # as after upload(); the recorder never reads the tables
    return p


def _t(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


def _kind(excinfo):
    return excinfo.value.kind


# ---------------------------------------------------------------- call patterns that must pass

@pytest.mark.parametrize("hq,hkv,dqk,dv,dtype", [(4, 4, 128, 128, torch.bfloat16), (8, 2, 128, 128, torch.bfloat16),
                                                 (4, 4, 192, 128, torch.bfloat16), (2, 2, 64, 64, torch.float32)])
def test_forward_and_backward_patterns_reach_the_library(rec, hq, hkv, dqk, dv, dtype):
    plan = _plan()
    T = plan.T
    q, k, v, do = _t(T, hq, dqk, dtype=dtype), _t(T, hkv, dqk, dtype=dtype), _t(T, hkv, dv, dtype=dtype), \
        _t(T, hq, dv, dtype=dtype)
    q_rm = thd.thd_kv_gather(plan, q)
    k_rm, v_rm = thd.thd_kv_gather(plan, k, v)
    do_rm = thd.thd_kv_gather(plan, do)
    o_rm, lse = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm, scale=0.1)
    assert o_rm.shape == (T, hq, dv) and lse.shape == (hq, T) and lse.dtype == torch.float32
    dq, dk, dvv = thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o_rm, lse, do_rm)
    assert dq.shape == (T, hq, dqk) and dk.shape == (T, hkv, dqk) and dvv.shape == (T, hkv, dv)
    for x in (o_rm, dq, dk, dvv):
        thd.thd_rows_to_global(plan, x)
    thd.thd_cp_attn_bwd_noalloc(plan, q_rm, k_rm, v_rm, o_rm, lse, do_rm, dq=dq, dk=dk, dv=dvv)
    assert rec.calls == ["thd_kv_gather"] * 3 + ["thd_cp_attn_fwd", "thd_cp_attn_bwd_workspace", "thd_cp_attn_bwd"] \
        + ["thd_rows_to_global"] * 4 + ["thd_cp_attn_bwd_noalloc"]


def test_benchmark_pattern_with_preallocated_buffers(rec):
    plan = _plan()
    T, hq, hkv, d = plan.T, 8, 2, 128
    q, k, v, do = _t(T, hq, d), _t(T, hkv, d), _t(T, hkv, d), _t(T, hq, d)
    q_rm, k_rm, v_rm, do_rm = (torch.empty_like(x) for x in (q, k, v, do))
    o_rm, lse_rm = _t(T, hq, d), _t(hq, T, dtype=torch.float32)
    dq, dk, dv = _t(T, hq, d, dtype=torch.float32), _t(T, hkv, d, dtype=torch.float32), \
        _t(T, hkv, d, dtype=torch.float32)
    ws = torch.empty(thd.thd_cp_attn_bwd_workspace(plan, hq=hq, hkv=hkv, dqk=d, dv=d) + 256, dtype=torch.uint8)
    thd.thd_kv_gather(plan, q, k_rm=q_rm)
    thd.thd_kv_gather(plan, k, v, k_rm=k_rm, v_rm=v_rm)
    thd.thd_kv_gather(plan, do, k_rm=do_rm)
    thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm, out=o_rm, lse=lse_rm)
    thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq=dq, dk=dk, dv=dv, workspace=ws)
    o_g = torch.empty_like(o_rm)
    thd.thd_rows_to_global(plan, o_rm, out=o_g)
    for s_, d_ in zip((dq, dk, dv), (torch.empty_like(dq), torch.empty_like(dk), torch.empty_like(dv))):
        thd.thd_rows_to_global(plan, s_, out=d_)
    pos = torch.zeros(T, dtype=torch.int32)
    thd.thd_rope_apply(q.clone(), pos, workspace=torch.empty(T * (d // 2) * 8, dtype=torch.uint8))
    assert rec.calls.count("thd_cp_attn_bwd") == 1 and rec.calls.count("thd_rope_apply") == 1


def test_compact_mla_pattern(rec):
    plan = _plan()
    T = plan.T
    q_rm = thd.thd_kv_gather(plan, _t(T, 4, 192))
    kn_rm, v_rm = thd.thd_kv_gather(plan, _t(T, 2, 128), _t(T, 2, 128))
    kr_rm = thd.thd_kv_gather(plan, _t(T, 64))
    o, lse = thd.thd_cp_attn_fwd_mla(plan, q_rm, kn_rm, kr_rm, v_rm)
    assert o.shape == (T, 4, 128) and lse.shape == (4, T)
    thd.thd_cp_attn_fwd_mla(plan, q_rm, kn_rm, kr_rm.view(T, 1, 64), v_rm)
    assert rec.calls[-2:] == ["thd_cp_attn_fwd_mla"] * 2


def test_calls_that_the_library_itself_refuses_still_reach_it(rec):
    """Unsupported widths, dtypes and misaligned rows are the library's checks: these
    calls pass the binding's and reach the library, which reports its own code."""
    p16, p32 = _plan((16,), 2), _plan((32,), 2)
    x = _t(16, 2, 96)
    thd.thd_cp_attn_fwd(p16, x, x, x)
    x, y = _t(32, 2, 192), _t(32, 2, 128)
    thd.thd_cp_attn_bwd(p32, x, x, y, y, _t(2, 32, dtype=torch.float32), y)
    thd.thd_cp_attn_fwd_mla(p16, _t(16, 2, 160), _t(16, 2, 128), _t(16, 32), _t(16, 2, 128))
    thd.thd_kv_gather(p16, _t(16, 3))
    thd.thd_rope_apply(_t(4, 1, 8, dtype=torch.float32), torch.zeros(4, dtype=torch.int32))
    assert rec.calls == ["thd_cp_attn_fwd", "thd_cp_attn_bwd_workspace", "thd_cp_attn_bwd", "thd_cp_attn_fwd_mla",
                         "thd_kv_gather", "thd_rope_workspace", "thd_rope_apply"]


# ---------------------------------------------------------------- mismatches refused before any call

def test_mismatched_tensors_are_refused(rec):
    plan = _plan()
    T = plan.T
    q, k, v = _t(T, 4, 128), _t(T, 2, 128), _t(T, 2, 128)
    lse = _t(4, T, dtype=torch.float32)
    bad = [
        lambda: thd.thd_kv_gather(plan, _t(T - 2, 2, 128)),                               # rows
        lambda: thd.thd_kv_gather(plan, k, k_rm=_t(T, 2, 64)),                            # output shape
        lambda: thd.thd_kv_gather(plan, k, k_rm=_t(T, 2, 128, dtype=torch.float32)),     # output dtype
        lambda: thd.thd_kv_gather(plan, k, v_rm=_t(T, 2, 128)),                           # v_rm without v
        lambda: thd.thd_rows_to_global(plan, _t(T + 2, 4)),                               # rows
        lambda: thd.thd_cp_attn_fwd(plan, q, _t(T, 2, 64), v),                            # K width
        lambda: thd.thd_cp_attn_fwd(plan, q, k, _t(T, 3, 128)),                           # V heads
        lambda: thd.thd_cp_attn_fwd(plan, q, k, v.to(torch.float32)),                     # mixed dtypes
        lambda: thd.thd_cp_attn_fwd(plan, q, k, v, lse=_t(T, 4, dtype=torch.float32)),    # lse layout
        lambda: thd.thd_cp_attn_fwd(plan, q, k, v, out=_t(T, 4, 128, dtype=torch.float32)),
        lambda: thd.thd_cp_attn_fwd(plan, _t(4, T, 128).transpose(0, 1), k, v),           # not contiguous
        lambda: thd.thd_cp_attn_fwd(plan, q[:, :, None], k, v),                           # 4-D
        lambda: thd.thd_cp_attn_fwd_mla(plan, _t(T, 4, 160), _t(T, 2, 128), _t(T, 64), v),  # Q width
        lambda: thd.thd_cp_attn_fwd_mla(plan, _t(T, 4, 192), _t(T, 2, 128), _t(T, 2, 64), v),  # rope per head
        lambda: thd.thd_cp_attn_bwd(plan, q, k, v, _t(T, 4, 128), lse, _t(T, 4, 128),
                                    dq=_t(T, 4, 128)),                                    # bf16 dq
        lambda: thd.thd_cp_attn_bwd(plan, q, k, v, _t(T, 4, 128), lse, _t(T - 2, 4, 128)),  # dO rows
        lambda: thd.thd_cp_attn_bwd_noalloc(plan, q, k, v, _t(T, 4, 128), lse, _t(T, 4, 128),
                                            dq=None, dk=None, dv=None),
        lambda: thd.thd_rope_apply(_t(T, 4, 128), torch.zeros(T - 1, dtype=torch.int32)),  # positions
        lambda: thd.thd_rope_apply(_t(T, 4, 128), torch.zeros(T, dtype=torch.int64)),
    ]
    for i, f in enumerate(bad):
        with pytest.raises(_lib.ThdError) as e:
            f()
        assert _kind(e) == "INVALID_ARG", i
    assert rec.calls == []


def test_unsupported_dtype_is_the_library_code(rec):
    plan = _plan()
    x = _t(plan.T, 2, 128, dtype=torch.float16)
    with pytest.raises(_lib.ThdError) as e:
        thd.thd_cp_attn_fwd(plan, x, x, x)
    assert _kind(e) == "UNSUPPORTED" and rec.calls == []


def test_host_tensors_and_other_devices_are_refused(monkeypatch):
    """With the real device check: a host tensor, and a current device other than the
    one holding the plan's tables."""
    r = Recorder(_lib.lib())
    monkeypatch.setattr(api, "lib", lambda: r)
    monkeypatch.setattr(api, "_current_device", lambda: 0)
    plan = _plan()
    with pytest.raises(_lib.ThdError) as e:
        thd.thd_kv_gather(plan, _t(plan.T, 2, 128))
    assert _kind(e) == "INVALID_ARG" and "CUDA tensor" in str(e.value)
    monkeypatch.setattr(api, "_current_device", lambda: 1)
    with pytest.raises(_lib.ThdError) as e:
        thd.thd_kv_gather(plan, _t(plan.T, 2, 128))
    assert _kind(e) == "INVALID_ARG" and "cuda:0" in str(e.value)
    assert r.calls == []


def test_not_uploaded_comes_first(rec):
    plan = _plan()
    plan.uploaded = False
    with pytest.raises(_lib.ThdError) as e:
        thd.thd_cp_attn_fwd(plan, None, None, None)
    assert _kind(e) == "NOT_UPLOADED" and rec.calls == []


def test_second_upload_keeps_the_first_device(rec, monkeypatch):
    cu = [0, 64]
    plan = thd.Plan(cu, 2)
    plan.upload()
    assert plan.uploaded and plan.device == 0 and rec.calls == ["thd_cp_plan_upload"]
    monkeypatch.setattr(api, "_current_device", lambda: 1)
    plan.upload()
    assert plan.device == 0

"""thd_cp_attn_bwd_noalloc, the backward for callers that cannot allocate device
memory (their device memory belongs to another allocator, or their hot path may not
call cudaMalloc): called through the C ABI, it must give what thd_cp_attn_bwd with a
caller-provided workspace gives, on two calls in a row (the second call reuses the
library's fixed scratch array, which holds the first call's contents), and refuse
problems larger than that array.  Kept in a file of its own that runs last."""
import ctypes

import numpy as np
import pytest
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import _lib
from context_packed_sequence_cp_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

MAX_ERR, MEAN_ERR = 2e-2, 2e-3   # the bf16 bar of the other parity tests


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc_call(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq, dk, dv):
    T, hq, d = q_rm.shape
    hkv = k_rm.shape[1]
    rc = _lib.lib().thd_cp_attn_bwd_noalloc(
        plan.handle, _vp(q_rm), _vp(k_rm), _vp(v_rm), _vp(o_rm), _vp(lse_rm), _vp(do_rm),
        _vp(dq), _vp(dk), _vp(dv), hq, hkv, d, d, float(d ** -0.5), _lib.THD_DTYPE_BF16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


def test_noalloc_backward_matches_workspace_backward_twice():
    cu = syn.cu_seqlens_of([512, 2048, 64, 1536])
    q, k, v, do = syn.make_tensors(int(cu[-1]), 8, 2, 128, 128, torch.bfloat16, seed=21, with_do=True,
                                   device="cuda")
    plan = thd.Plan(cu, 4).upload()
    q_rm = thd.thd_kv_gather(plan, q)
    k_rm, v_rm = thd.thd_kv_gather(plan, k, v)
    do_rm = thd.thd_kv_gather(plan, do)
    o_rm, lse_rm = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm)
    want = [x.cpu().numpy() for x in thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm)]
    for _ in range(2):
        dq = torch.full_like(q_rm, float("nan"), dtype=torch.float32)
        dk = torch.full_like(k_rm, float("nan"), dtype=torch.float32)
        dv = torch.full_like(v_rm, float("nan"), dtype=torch.float32)
        assert _noalloc_call(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq, dk, dv) == _lib.THD_OK
        torch.cuda.synchronize()
        for got, ref in zip((dq, dk, dv), want):
            err = np.abs(got.cpu().numpy() - ref)
            assert np.isfinite(err).all()
            assert err.max() <= MAX_ERR and err.mean() <= MEAN_ERR
    assert plan.device_status() == 0


def test_noalloc_backward_refuses_problems_beyond_its_scratch():
    T = 131072
    plan = thd.Plan([0, T], 1).upload()
    hq = _lib.NOALLOC_MAX_ROWS_X_HEADS // T + 1           # hq * T just over the fixed array
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")  # never read: the size check comes first
    f = torch.zeros(64, dtype=torch.float32, device="cuda")
    rc = _lib.lib().thd_cp_attn_bwd_noalloc(
        plan.handle, _vp(x), _vp(x), _vp(x), _vp(x), _vp(f), _vp(x), _vp(f), _vp(f), _vp(f),
        hq, 1, 128, 128, 0.088, _lib.THD_DTYPE_BF16, ctypes.c_void_p(0))
    assert rc == -9 and b"scratch" in _lib.lib().thd_cp_strerror(rc)

"""thd_cp_plan_update on the GPU: one uploaded plan re-planned for a sequence of new
layouts (its device allocation growing and shrinking) gives, for each layout, exactly
what a freshly built and uploaded plan gives, with no device-wide synchronisation in
between; and a call made with another device current is refused."""
import numpy as np
import pytest
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _fwd(plan, q, k, v):
    q_rm = thd.thd_kv_gather(plan, q)
    k_rm, v_rm = thd.thd_kv_gather(plan, k, v)
    o_rm, lse_rm = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm)
    return thd.thd_rows_to_global(plan, o_rm), lse_rm


def test_updated_plan_matches_fresh_plans():
    rng = np.random.default_rng(3)
    layouts = []
    for T, cp in ((1024, 4), (8192, 8), (512, 2), (16384, 16), (2048, 4)):
        lens = syn.random_lengths(rng, T, 2 * cp, max_docs=6)
        layouts.append((syn.cu_seqlens_of(lens), cp))
    plan = thd.Plan(layouts[0][0], layouts[0][1]).upload()
    results = []
    for cu, cp in layouts:
        plan.update(cu, cp)
        T = int(cu[-1])
        q, k, v = syn.make_tensors(T, 4, 2, 128, 128, torch.bfloat16, seed=T, device="cuda")
        got = _fwd(plan, q, k, v)
        fresh = thd.Plan(cu, cp).upload()
        want = _fwd(fresh, q, k, v)
        results.append((got, want, fresh))
    torch.cuda.synchronize()
    for (o, l), (wo, wl), fresh in results:
        assert torch.equal(o, wo) and torch.equal(l, wl)
        assert fresh.device_status() == 0
    assert plan.device_status() == 0


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_calls_with_another_device_current_are_refused():
    import ctypes
    from context_packed_sequence_cp_b200 import _lib
    with torch.cuda.device(0):
        plan = thd.Plan([0, 64], 2).upload()
        x = torch.zeros(64, 2, 128, dtype=torch.bfloat16, device="cuda:0")
        y = torch.empty_like(x)
    with torch.cuda.device(1):
        rc = _lib.lib().thd_kv_gather(plan.handle, ctypes.c_void_p(x.data_ptr()), None,
                                      ctypes.c_void_p(y.data_ptr()), None, 512, 0, None)
        assert rc == -1

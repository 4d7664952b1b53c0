"""thd_kv_gather / thd_rows_to_global on the GPU: bit-exact row copies against the
oracle partition's index tables."""
import numpy as np
import pytest
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import synthetic as syn
from oracle import partition as P

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_kv_gather_bit_exact(cfg):
    w = syn.WORKLOADS[cfg]
    cu = syn.cu_seqlens_of(syn.doc_lengths(cfg, 0))
    g = torch.Generator().manual_seed(cfg)
    k = torch.randn(w.T, w.hkv, w.dqk, generator=g).to(w.dtype)
    v = torch.randn(w.T, w.hkv, w.dv, generator=g).to(w.dtype)
    q_idx, rm = P.partition(cu, w.cp)
    plan = thd.Plan(cu, w.cp).upload()
    k_rm, v_rm = thd.thd_kv_gather(plan, k.cuda(), v.cuda())
    ti = torch.from_numpy(q_idx.astype(np.int64))
    assert torch.equal(k_rm.cpu(), k[ti])
    assert torch.equal(v_rm.cpu(), v[ti])
    back = thd.thd_rows_to_global(plan, k_rm)
    assert torch.equal(back.cpu(), k)
    # Q-shaped rows through the single-tensor form
    q = torch.randn(w.T, w.hq, w.dqk, generator=g).to(w.dtype)
    q_rm = thd.thd_kv_gather(plan, q.cuda())
    assert torch.equal(q_rm.cpu(), q[ti])
    torch.cuda.synchronize()


def test_gather_rejects_misaligned_rows():
    cu = syn.cu_seqlens_of([8, 8])
    plan = thd.Plan(cu, 2).upload()
    x = torch.zeros(16, 3, dtype=torch.bfloat16, device="cuda")  # 6-byte rows
    with pytest.raises(thd.ThdError) as e:
        thd.thd_kv_gather(plan, x)
    assert e.value.kind == "MISALIGNED"

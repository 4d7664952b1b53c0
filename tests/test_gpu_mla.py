"""Multi-head latent attention with compact keys (a per-head part and one rope key
per token shared by every head), through thd_cp_attn_fwd_mla: parity with the fp64
oracle, and identity with the expanded-key forward on the same values."""
import math

import numpy as np
import pytest
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import synthetic as syn
from oracle import attention as A
from gpu_util import LSE_MAX, assert_bf16_close, unpermute_rows

pytestmark = pytest.mark.gpu

D_NOPE, D_ROPE, DV = 128, 64, 128


def _inputs(T, hq, hkv, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn(T, hq, D_NOPE + D_ROPE, generator=g).to(torch.bfloat16)
    kn = torch.randn(T, hkv, D_NOPE, generator=g).to(torch.bfloat16)
    kr = torch.randn(T, D_ROPE, generator=g).to(torch.bfloat16)
    v = torch.randn(T, hkv, DV, generator=g).to(torch.bfloat16)
    return q, kn, kr, v


def _run_compact(cu, cp, q, kn, kr, v):
    plan = thd.Plan(cu, cp).upload()
    dev = torch.device("cuda:0")
    q_rm = thd.thd_kv_gather(plan, q.to(dev))
    kn_rm, v_rm = thd.thd_kv_gather(plan, kn.to(dev), v.to(dev))
    kr_rm = thd.thd_kv_gather(plan, kr.to(dev))
    o_rm, lse_rm = thd.thd_cp_attn_fwd_mla(plan, q_rm, kn_rm, kr_rm, v_rm)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    return plan, q_rm, kn_rm, kr_rm, v_rm, o_rm, lse_rm


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
@pytest.mark.parametrize("cp", [1, 4, 8])
def test_mla_compact_keys_match_oracle(hq, hkv, cp):
    rng = np.random.default_rng(7 * cp + hq)
    lens = syn.random_lengths(rng, 3000, 2 * cp, max_docs=6) + [2 * cp]
    cu = syn.cu_seqlens_of(lens)
    q, kn, kr, v = _inputs(int(cu[-1]), hq, hkv, seed=cp + hq)
    plan, *_, o_rm, lse_rm = _run_compact(cu, cp, q, kn, kr, v)
    o = thd.thd_rows_to_global(plan, o_rm).float().cpu().numpy()
    q_idx = plan.export()["q_idx"]
    lse = unpermute_rows(lse_rm.cpu().numpy().T, q_idx).T
    want_o, want_l = A.attention_fwd_mla(q, kn, kr, v, cu, 1 / math.sqrt(D_NOPE + D_ROPE))
    assert_bf16_close(o, want_o, "O")
    assert np.abs(lse - want_l).max() <= LSE_MAX


def test_mla_compact_keys_equal_expanded_keys_exactly():
    """The compact form feeds the tensor cores the same key tiles as the expanded form
    (its third 64-column box comes from the shared rope key), so the results agree
    bit for bit."""
    cu = syn.cu_seqlens_of([1024, 96, 2560, 384])
    q, kn, kr, v = _inputs(int(cu[-1]), 4, 2, seed=3)
    plan, q_rm, kn_rm, kr_rm, v_rm, o_rm, lse_rm = _run_compact(cu, 4, q, kn, kr, v)
    T, hkv = kn_rm.shape[0], kn_rm.shape[1]
    k_full = torch.cat([kn_rm, kr_rm.view(T, 1, D_ROPE).expand(T, hkv, D_ROPE)], dim=2).contiguous()
    o2, lse2 = thd.thd_cp_attn_fwd(plan, q_rm, k_full, v_rm)
    torch.cuda.synchronize()
    assert torch.equal(o_rm, o2)
    assert torch.equal(lse_rm, lse2)


def test_mla_rejects_other_widths():
    plan = thd.Plan([0, 16], 2).upload()
    q = torch.zeros(16, 2, 160, dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros(16, 2, 128, dtype=torch.bfloat16, device="cuda")
    kr = torch.zeros(16, 32, dtype=torch.bfloat16, device="cuda")   # rope width 32: not built
    with pytest.raises(thd.ThdError) as e:
        thd.thd_cp_attn_fwd_mla(plan, q, kn, kr, kn)
    assert e.value.kind == "UNSUPPORTED"

"""Helpers shared by the GPU parity tests: run the library through its binding and
bring rank-major results back to packed order on the host."""
import math

import numpy as np
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import synthetic as syn

BF16_MAX, BF16_MEAN, LSE_MAX, FP32_MAX = 2e-2, 2e-3, 1e-3, 1e-5


def unpermute_rows(x_rm: np.ndarray, q_idx: np.ndarray) -> np.ndarray:
    out = np.empty_like(x_rm)
    out[q_idx] = x_rm
    return out


def run_forward(cu, cp, q, k, v, scale=None):
    """Plan + gather + fwd on cuda:0.  Returns (o_global, lse_global [hq,T], plan, q_idx)."""
    dev = torch.device("cuda:0")
    plan = thd.Plan(cu, cp).upload()
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    q_rm = thd.thd_kv_gather(plan, qd)
    k_rm, v_rm = thd.thd_kv_gather(plan, kd, vd)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[2])
    o_rm, lse_rm = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm, scale=scale)
    o = thd.thd_rows_to_global(plan, o_rm)
    torch.cuda.synchronize()
    assert plan.device_status() == 0, "a bounded wait gave up"
    q_idx = plan.export()["q_idx"]
    lse = unpermute_rows(lse_rm.cpu().numpy().T, q_idx).T
    return o.float().cpu().numpy(), lse, plan, q_idx


def assert_bf16_close(got, want, what):
    err = np.abs(got.astype(np.float64) - want)
    assert err.max() <= BF16_MAX, f"{what}: max |err| {err.max():.3g}"
    assert err.mean() <= BF16_MEAN, f"{what}: mean |err| {err.mean():.3g}"


def workload(cfg, seed=0):
    return syn.workload_inputs(cfg, seed)

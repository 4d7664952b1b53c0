"""A reduced long-context workload for profiler captures: the same structure as the
benchmarked workload (one long document of T/2 tokens plus lognormal(512, 1)
documents in multiples of 32, GQA 64/8, head dim 128, cp=16) at a size whose
inputs still exceed L2 but fit a profiler's replay budget.

    python profile_case.py [--T 16384] [--iters 2]

Each iteration launches gather (Q, K/V, dO), forward and backward once.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import context_packed_sequence_cp_b200 as thd  # noqa: E402


def layout(T: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    lens = [T // 2]
    total = T // 2
    while total < T:
        L = int(np.clip(int(np.rint(rng.lognormal(np.log(512.0), 1.0) / 32)) * 32, 32, T))
        L = min(L, T - total)
        lens.append(L)
        total += L
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    return cu


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=16384)
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--seed", type=int, default=0)
    ns = ap.parse_args()
    hq, hkv, d, cp = 64, 8, 128, 16
    dev = torch.device("cuda:0")
    cu = layout(ns.T, ns.seed)
    plan = thd.Plan(cu, cp).upload()
    g = torch.Generator(device=dev).manual_seed(ns.seed + 1)
    q = torch.randn(ns.T, hq, d, device=dev, generator=g).to(torch.bfloat16)
    k = torch.randn(ns.T, hkv, d, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(ns.T, hkv, d, device=dev, generator=g).to(torch.bfloat16)
    do = torch.randn(ns.T, hq, d, device=dev, generator=g).to(torch.bfloat16)
    for _ in range(ns.iters):
        q_rm = thd.thd_kv_gather(plan, q)
        k_rm, v_rm = thd.thd_kv_gather(plan, k, v)
        do_rm = thd.thd_kv_gather(plan, do)
        o, lse = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm)
        thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o, lse, do_rm)
    torch.cuda.synchronize()
    status = plan.device_status()
    print(f"profile case T={ns.T} docs={len(cu) - 1} pairs={plan.causal_pairs} status={status}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())

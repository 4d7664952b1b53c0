"""Seeded synthetic workloads for packed-sequence (THD) context-parallel attention.

This module only draws random document lengths and random tensors.  It holds none
of the method's arithmetic (no partitioning, no masking, no softmax), so both the
CUDA path and the fp64 oracle can consume what it produces.

The five workloads follow the shapes the MindSpeed pull request #3820 ("feat:
kvallgather cp thd load balance") is used with: THD packed sequences whose
documents are delimited by EOD resets, every document length divisible by
2 * context_parallel_size (section "Does this PR introduce any user-facing
change?"), MHA, GQA and expanded MLA head layouts (section "What this PR does /
why we need it?").

Recipe (seeded, deterministic):
  * document lengths come from ``numpy.random.default_rng(seed)``;
  * Q, K, V (and dO) come from ``torch.Generator('cpu').manual_seed(seed + 1)``,
    drawn with ``randn`` in fp32 in the order q, k, v, do, scaled by the
    per-tensor standard deviation, then cast to the workload dtype.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cp: int
    T: int
    hq: int
    hkv: int
    dqk: int
    dv: int
    dtype: torch.dtype
    backward: bool
    v_std: float = 1.0
    description: str = ""


WORKLOADS = {
    1: Workload("tiny-fp32", 2, 512, 2, 2, 64, 64, torch.float32, False,
                description="cp=2, T=512, docs [128,256,128], MHA H=2, D=64, fp32"),
    2: Workload("mha-d128", 4, 8192, 16, 16, 128, 128, torch.bfloat16, False,
                description="cp=4, T=8192, MHA H=16, D=128, docs U{256..4096 step 8}"),
    3: Workload("gqa-32-8", 8, 32768, 32, 8, 128, 128, torch.bfloat16, False,
                description="cp=8, T=32768, GQA 32/8, D=128, docs lognormal(1024,1) step 16"),
    4: Workload("mla-192-128", 8, 65536, 16, 16, 192, 128, torch.bfloat16, False,
                v_std=0.5,
                description="cp=8, T=65536, H=16, Dqk=192 Dv=128, docs U{512..8192 step 16}"),
    5: Workload("long-gqa-64-8-fwdbwd", 16, 131072, 64, 8, 128, 128, torch.bfloat16, True,
                description="cp=16, T=131072, GQA 64/8, D=128, [65536]+lognormal(512,1) step 32, fwd+bwd"),
}


def _round_to(x: float, unit: int) -> int:
    return int(np.rint(x / unit)) * unit


def _fill_to(T: int, draw, unit: int) -> list[int]:
    """Draw lengths until they reach T, trimming the last one to land exactly on T."""
    out: list[int] = []
    total = 0
    while total < T:
        L = draw()
        if total + L > T:
            L = T - total
        if L > 0:
            out.append(L)
            total += L
    assert total == T and all(L % unit == 0 for L in out)
    return out


def doc_lengths(cfg: int, seed: int = 0) -> list[int]:
    """Document lengths of workload ``cfg`` (1..5) for ``seed``."""
    rng = np.random.default_rng(seed)
    w = WORKLOADS[cfg]
    if cfg == 1:
        return [128, 256, 128]
    if cfg == 2:
        return _fill_to(w.T, lambda: 8 * int(rng.integers(256 // 8, 4096 // 8 + 1)), 8)
    if cfg == 3:
        return _fill_to(
            w.T,
            lambda: int(np.clip(_round_to(rng.lognormal(np.log(1024.0), 1.0), 16), 16, 16384)),
            16)
    if cfg == 4:
        return _fill_to(w.T, lambda: 16 * int(rng.integers(512 // 16, 8192 // 16 + 1)), 16)
    if cfg == 5:
        rest = _fill_to(
            w.T - 65536,
            lambda: int(np.clip(_round_to(rng.lognormal(np.log(512.0), 1.0), 32), 32, 65536)),
            32)
        return [65536] + rest
    raise ValueError(f"unknown workload {cfg}")


def cu_seqlens_of(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def random_lengths(rng: np.random.Generator, T_max: int, unit: int, max_docs: int = 8) -> list[int]:
    """Random small layout: up to ``max_docs`` documents, each a positive multiple of ``unit``."""
    n = int(rng.integers(1, max_docs + 1))
    budget = max(1, T_max // unit)
    lens = [unit * int(rng.integers(1, max(2, budget // n + 1))) for _ in range(n)]
    return lens


def make_tensors(T: int, hq: int, hkv: int, dqk: int, dv: int, dtype: torch.dtype,
                 seed: int, v_std: float = 1.0, with_do: bool = False,
                 device: Optional[str] = None):
    """Q [T,hq,dqk], K [T,hkv,dqk], V [T,hkv,dv] (and dO [T,hq,dv]) in global THD order."""
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    q = torch.randn(T, hq, dqk, generator=g, dtype=torch.float32)
    k = torch.randn(T, hkv, dqk, generator=g, dtype=torch.float32)
    v = torch.randn(T, hkv, dv, generator=g, dtype=torch.float32) * v_std
    out = [q.to(dtype), k.to(dtype), v.to(dtype)]
    if with_do:
        do = torch.randn(T, hq, dv, generator=g, dtype=torch.float32)
        out.append(do.to(dtype))
    if device is not None:
        out = [t.to(device) for t in out]
    return tuple(out)


def workload_inputs(cfg: int, seed: int = 0, device: Optional[str] = None):
    """(cu_seqlens, tensors) of workload ``cfg`` for ``seed``."""
    w = WORKLOADS[cfg]
    cu = cu_seqlens_of(doc_lengths(cfg, seed))
    tens = make_tensors(w.T, w.hq, w.hkv, w.dqk, w.dv, w.dtype, seed, w.v_std,
                        with_do=w.backward, device=device)
    return cu, tens

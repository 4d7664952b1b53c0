"""thd_cp_attn_fwd on the GPU against the fp64 oracle: full comparison where the
oracle finishes in seconds, sampled rows at the full workload sizes, the
cp-independence and per-document invariants, and edge layouts."""
import math

import numpy as np
import pytest
import torch

from context_packed_sequence_cp_b200 import synthetic as syn
from oracle import attention as A
from tests.gpu_util import (FP32_MAX, LSE_MAX, assert_bf16_close, run_forward)

pytestmark = pytest.mark.gpu


def test_fwd_fp32_tiny_workload():
    cu, (q, k, v) = syn.workload_inputs(1, 0)
    o, lse, _, _ = run_forward(cu, 2, q, k, v, scale=1 / math.sqrt(64))
    want_o, want_l = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(64))
    assert np.abs(o - want_o).max() <= FP32_MAX
    assert np.abs(lse - want_l).max() <= FP32_MAX


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fwd_bf16_mha_workload_full(seed):
    """T=8192, cp=4, MHA 16 heads, D=128: every output compared."""
    cu, (q, k, v) = syn.workload_inputs(2, seed)
    o, lse, _, _ = run_forward(cu, 4, q, k, v)
    want_o, want_l = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(128))
    assert_bf16_close(o, want_o, "O")
    assert np.abs(lse - want_l).max() <= LSE_MAX


def _sample_rows(cu, rng, n_rand=24):
    rows = set()
    for d in range(len(cu) - 1):
        s, e = int(cu[d]), int(cu[d + 1])
        rows.update({s, e - 1, min(e - 1, s + 127), min(e - 1, s + 128)})
    rows.update(int(x) for x in rng.integers(0, int(cu[-1]), n_rand))
    return sorted(rows)


@pytest.mark.parametrize("cfg", [3, 4, 5])
def test_fwd_bf16_workload_sampled(cfg):
    """Full-size GQA (T=32768), expanded MLA (T=65536) and long-context (T=131072)
    workloads, checked on sampled rows x heads the oracle computes one by one."""
    w = syn.WORKLOADS[cfg]
    cu, tens = syn.workload_inputs(cfg, 0)
    q, k, v = tens[:3]
    o, lse, _, _ = run_forward(cu, w.cp, q, k, v)
    rng = np.random.default_rng(cfg)
    rows = _sample_rows(cu, rng)
    if cfg == 5:
        # Short documents: a subset of their sampled rows.  The 65536-token document:
        # rows whose walks are the longest of the launch (up to 512 key tiles, the lazy
        # rescale and the chunk seams deep inside them), its first tiles, the seam between
        # a rank's two chunks, and random rows.
        short = [r for r in rows if r >= 65536][:48]
        deep = [0, 127, 128, 2047, 2048, 4095, 32767, 32768, 49152, 63488, 65407, 65535]
        rows = sorted(set(short + deep + [int(x) for x in rng.integers(0, 65536, 16)]))
    heads = sorted({0, w.hq - 1, int(rng.integers(0, w.hq))})
    want_o, want_l = A.attention_fwd_rows(q, k, v, cu, 1 / math.sqrt(w.dqk), rows, heads)
    assert_bf16_close(o[rows][:, heads], want_o, "O")
    assert np.abs(lse[heads][:, rows].T - want_l).max() <= LSE_MAX


# MHA, GQA with groups of 4, 6, 2 and 3, and expanded MLA
@pytest.mark.parametrize("hq,hkv,dqk,dv", [(4, 4, 128, 128), (8, 2, 128, 128), (4, 4, 192, 128), (6, 1, 128, 128),
                                           (4, 2, 128, 128), (3, 1, 128, 128)])
@pytest.mark.parametrize("cp", [1, 2, 4, 8])
def test_fwd_bf16_small_layouts_full(hq, hkv, dqk, dv, cp):
    """Random layouts spanning several tiles with ragged tails, every output compared."""
    rng = np.random.default_rng(cp * 31 + hq + dqk)
    lens = syn.random_lengths(rng, 3000, 2 * cp, max_docs=6) + [2 * cp]   # plus a minimal document
    cu = syn.cu_seqlens_of(lens)
    q, k, v = syn.make_tensors(int(cu[-1]), hq, hkv, dqk, dv, torch.bfloat16, seed=cp + hq)
    o, lse, _, _ = run_forward(cu, cp, q, k, v)
    want_o, want_l = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(dqk))
    assert_bf16_close(o, want_o, "O")
    assert np.abs(lse - want_l).max() <= LSE_MAX


def test_fwd_bf16_output_independent_of_cp():
    lens = [512, 2048, 64, 1536]
    cu = syn.cu_seqlens_of(lens)
    q, k, v = syn.make_tensors(int(cu[-1]), 4, 2, 128, 128, torch.bfloat16, seed=5)
    outs = [run_forward(cu, cp, q, k, v)[:2] for cp in (1, 2, 4, 8, 16)]
    for o, l in outs[1:]:
        assert np.abs(o - outs[0][0]).max() <= 2e-2
        assert np.abs(l - outs[0][1]).max() <= LSE_MAX


def test_fwd_bf16_each_document_is_standalone_attention():
    lens = [256, 1024, 32]
    cu = syn.cu_seqlens_of(lens)
    q, k, v = syn.make_tensors(int(cu[-1]), 2, 2, 128, 128, torch.bfloat16, seed=8)
    o, lse, _, _ = run_forward(cu, 4, q, k, v)
    for d in range(3):
        s, e = int(cu[d]), int(cu[d + 1])
        od, ld, _, _ = run_forward(np.array([0, e - s]), 4, q[s:e], k[s:e], v[s:e])
        assert np.abs(o[s:e] - od).max() <= 2e-2
        assert np.abs(lse[:, s:e] - ld).max() <= LSE_MAX


@pytest.mark.parametrize("lens,cp", [([2] * 64, 1), ([16] * 40, 8), ([2], 1), ([32, 16, 32], 8)])
def test_fwd_bf16_degenerate_layouts(lens, cp):
    """Documents of the minimum length 2*cp only (one-row chunks, q-tiles of a few rows),
    and a single two-token sequence."""
    cu = syn.cu_seqlens_of(lens)
    q, k, v = syn.make_tensors(int(cu[-1]), 4, 2, 128, 128, torch.bfloat16, seed=len(lens) + cp)
    o, lse, _, _ = run_forward(cu, cp, q, k, v)
    want_o, want_l = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(128))
    assert_bf16_close(o, want_o, "O")
    assert np.abs(lse - want_l).max() <= LSE_MAX


def test_fwd_rejects_unsupported_dims():
    import context_packed_sequence_cp_b200 as thd
    plan = thd.Plan([0, 16], 2).upload()
    x = torch.zeros(16, 2, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(thd.ThdError) as e:
        thd.thd_cp_attn_fwd(plan, x, x, x)
    assert e.value.kind == "UNSUPPORTED"


@pytest.mark.parametrize("cp", [2, 4])
def test_fwd_bf16_position_tiles_around_the_chunk_threshold(cp):
    """Documents whose chunks are shorter than a tile are tiled in position order (their
    rows gathered through rm_of_global), the others rank-major: chunk sizes 1, 17, 64,
    127 (position tiles) and 128, 129, 300 (rank-major) in one packed sequence, GQA 8/2,
    every output compared."""
    chunks = [1, 17, 64, 127, 128, 129, 300, 3]
    lens = [2 * cp * c for c in chunks]
    cu = syn.cu_seqlens_of(lens)
    q, k, v = syn.make_tensors(int(cu[-1]), 8, 2, 128, 128, torch.bfloat16, seed=40 + cp)
    o, lse, plan, _ = run_forward(cu, cp, q, k, v)
    fwd = plan.export_fwd()
    assert (fwd["fqtiles"][:, 2] < 0).any() and (fwd["fqtiles"][:, 2] >= 0).any()
    want_o, want_l = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(128))
    assert_bf16_close(o, want_o, "O")
    assert np.abs(lse - want_l).max() <= LSE_MAX


@pytest.mark.parametrize("cp", [2, 8])
def test_fwd_bf16_position_tiles_run_boxes(cp):
    """A position tile's rows are runs of consecutive rank-major rows, one per chunk, loaded
    as the largest aligned boxes of 8 to 128 rows that lie inside one run, the rest gathered
    4 rows at a time.  Chunk sizes 8, 16, 24, 32, 40, 64, 96, 120 put every run boundary on
    an 8-row group boundary (boxes of every size); 9, 65, 127 put groups across chunk
    boundaries (gathers mixed with boxes).  Every output is compared with the oracle, and the
    fused-gather entry (K/V from the packed tensors) is bit-identical."""
    import context_packed_sequence_cp_b200 as thd
    from tests.gpu_util import unpermute_rows
    chunks = [8, 16, 24, 32, 40, 64, 96, 120, 9, 65, 127]
    cu = syn.cu_seqlens_of([2 * cp * c for c in chunks])
    q, k, v = syn.make_tensors(int(cu[-1]), 8, 2, 128, 128, torch.bfloat16, seed=80 + cp, device="cuda")
    plan = thd.Plan(cu, cp).upload()
    assert (plan.export_fwd()["fqtiles"][:, 2] < 0).all()   # position tiles only
    q_rm = thd.thd_kv_gather(plan, q)
    k_rm, v_rm = thd.thd_kv_gather(plan, k, v)
    o_rm, l_rm = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm)
    o_fg, l_fg = thd.thd_cp_attn_fwd_fused_gather(plan, q_rm, k, v)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    assert torch.equal(o_fg, o_rm) and torch.equal(l_fg, l_rm)
    q_idx = plan.export()["q_idx"]
    o = unpermute_rows(o_rm.float().cpu().numpy(), q_idx)
    lse = unpermute_rows(l_rm.cpu().numpy().T, q_idx).T
    want_o, want_l = A.attention_fwd(q.cpu(), k.cpu(), v.cpu(), cu, 1 / math.sqrt(128))
    assert_bf16_close(o, want_o, "O")
    assert np.abs(lse - want_l).max() <= LSE_MAX


@pytest.mark.parametrize("cp,chunks,heads", [(4, [1, 17, 64, 127, 128, 129, 300, 3], (8, 2)),
                                              (16, [160, 32, 200], (8, 1)), (1, [900, 5], (4, 4))])
def test_fwd_fused_gather_is_bit_identical(cp, chunks, heads):
    """K/V read straight from the packed tensors (the all-gather fused into the loads):
    boxes for runs of consecutive positions, gathers for runs with a seam; the outputs
    equal thd_cp_attn_fwd's on the rank-major copy bit for bit, and the oracle's."""
    import context_packed_sequence_cp_b200 as thd
    hq, hkv = heads
    cu = syn.cu_seqlens_of([2 * cp * c for c in chunks])
    q, k, v = syn.make_tensors(int(cu[-1]), hq, hkv, 128, 128, torch.bfloat16, seed=60 + cp, device="cuda")
    plan = thd.Plan(cu, cp).upload()
    q_rm = thd.thd_kv_gather(plan, q)
    k_rm, v_rm = thd.thd_kv_gather(plan, k, v)
    o_ref, l_ref = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm)
    o_fg, l_fg = thd.thd_cp_attn_fwd_fused_gather(plan, q_rm, k, v)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    assert torch.equal(o_fg, o_ref) and torch.equal(l_fg, l_ref)
    if int(cu[-1]) <= 8192:
        q_idx = plan.export()["q_idx"]
        from tests.gpu_util import unpermute_rows
        o = unpermute_rows(o_fg.float().cpu().numpy(), q_idx)
        want_o, _ = A.attention_fwd(q.cpu(), k.cpu(), v.cpu(), cu, 1 / math.sqrt(128))
        assert_bf16_close(o, want_o, "O")

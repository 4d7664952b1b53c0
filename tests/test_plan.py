"""The library's host planner (C ABI thd_cp_plan / thd_cp_plan_export) against the
brute-force oracle tables: bit-exact on every workload layout and on random layouts,
and the same error classes on invalid input.  CPU only."""
import numpy as np
import pytest

from context_packed_sequence_cp_b200 import Plan, ThdError
from context_packed_sequence_cp_b200 import synthetic as syn
from oracle import partition as P
from oracle import tiles as TT

KEYS = ("q_idx", "rm_of_global", "qtiles", "entries", "lpt", "kt_off", "kt_list", "kt_lpt", "kt_seg")
FWD_KEYS = ("fqtiles", "fentries", "flpt", "fkt_off", "fkt_list", "fkt_lpt", "fkt_seg")


def _compare(cu, cp):
    got = Plan(cu, cp)
    want = TT.tile_plan(cu, cp)
    ex = got.export()
    assert got.T == want["T"] and got.Tl == want["Tl"] and got.n_docs == want["n_docs"]
    assert got.causal_pairs == P.causal_pairs_total(cu)
    for k in KEYS:
        assert np.array_equal(ex[k], want[k].reshape(ex[k].shape)), k
    fx = got.export_fwd()
    for k in FWD_KEYS:
        assert np.array_equal(fx[k], want[k].reshape(fx[k].shape)), k
    got.close()


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_plan_bit_exact_workloads(cfg):
    w = syn.WORKLOADS[cfg]
    for seed in range(2):
        _compare(syn.cu_seqlens_of(syn.doc_lengths(cfg, seed)), w.cp)


@pytest.mark.slow
def test_plan_bit_exact_long_context_workload():
    _compare(syn.cu_seqlens_of(syn.doc_lengths(5, 0)), syn.WORKLOADS[5].cp)


@pytest.mark.parametrize("seed", range(4))
def test_plan_bit_exact_random_layouts(seed):
    rng = np.random.default_rng(1000 + seed)
    for _ in range(25):
        cp = int(rng.choice([1, 2, 3, 4, 5, 8, 16]))
        lens = syn.random_lengths(rng, 3000, 2 * cp, max_docs=7)
        _compare(syn.cu_seqlens_of(lens), cp)


@pytest.mark.parametrize("lens,cp", [
    ([2], 1),                 # one token pair, one rank
    ([4], 2),                 # chunk of one token
    ([2 * 16], 16),           # every chunk one token, 16 ranks
    ([256], 1),               # cp = 1: plain varlen causal attention
    ([128 * 16], 8),          # chunks exactly one tile
    ([130 * 16], 8),          # chunks one tile plus a ragged tail
    ([64, 2 * 128 * 4, 8], 4),  # tiny docs around a long one
])
def test_plan_bit_exact_edge_layouts(lens, cp):
    _compare(syn.cu_seqlens_of(lens), cp)


@pytest.mark.parametrize("cu,cp,kind", [
    ([0, 4, 12], 0, "INVALID_ARG"),
    ([1, 4, 12], 2, "BAD_SEQLENS"),
    ([0, 4, 4, 12], 2, "BAD_SEQLENS"),
    ([0, 8, 4], 2, "BAD_SEQLENS"),
    ([0, 6, 12], 2, "NOT_DIVISIBLE"),
    ([0, 12], 4, "NOT_DIVISIBLE"),
])
def test_plan_rejects_like_oracle(cu, cp, kind):
    with pytest.raises(ThdError) as e:
        Plan(cu, cp)
    assert e.value.kind == kind
    with pytest.raises(P.PartitionError) as e2:
        P.partition(np.array(cu), cp)
    assert e2.value.kind == kind


def test_device_entry_points_refuse_before_upload():
    import torch
    from context_packed_sequence_cp_b200 import thd_cp_attn_fwd, thd_kv_gather
    plan = Plan([0, 8], 2)
    x = torch.zeros(8, 1, 8)
    with pytest.raises(ThdError) as e:
        thd_kv_gather(plan, x, stream=type("S", (), {"cuda_stream": 0})())
    assert e.value.kind == "NOT_UPLOADED"
    with pytest.raises(ThdError) as e:
        thd_cp_attn_fwd(plan, x, x, x, stream=type("S", (), {"cuda_stream": 0})())
    assert e.value.kind == "NOT_UPLOADED"


def test_plan_update_equals_a_fresh_plan():
    """thd_cp_plan_update re-plans in place: after every update (larger, smaller, another
    cp) the exported tables are bit-identical to a freshly built plan's and to the
    oracle's; an invalid layout leaves the plan as it was."""
    rng = np.random.default_rng(77)
    plan = Plan([0, 16], 2)
    for i in range(12):
        cp = int(rng.choice([1, 2, 4, 8]))
        lens = syn.random_lengths(rng, 4000 if i % 3 else 400, 2 * cp, max_docs=7)
        cu = syn.cu_seqlens_of(lens)
        plan.update(cu, cp)
        fresh = Plan(cu, cp)
        ex, ref = plan.export(), fresh.export()
        want = TT.tile_plan(cu, cp)
        assert (plan.T, plan.cp, plan.n_qtiles, plan.n_entries) == (fresh.T, fresh.cp, fresh.n_qtiles,
                                                                     fresh.n_entries)
        for k in KEYS:
            assert np.array_equal(ex[k], ref[k]), k
            assert np.array_equal(ex[k], want[k].reshape(ex[k].shape)), k
        fx = plan.export_fwd()
        for k in FWD_KEYS:
            assert np.array_equal(fx[k], want[k].reshape(fx[k].shape)), k
        fresh.close()
    before = plan.export()
    with pytest.raises(ThdError) as e:
        plan.update([0, 6, 12], 2)          # 6 is not a multiple of 2 * cp = 4
    assert e.value.kind == "NOT_DIVISIBLE"
    after = plan.export()
    for k in KEYS:
        assert np.array_equal(before[k], after[k]), k
    plan.close()

"""thd_cp_attn_bwd on the GPU against the fp64 oracle: full comparison on small
layouts, sampled rows / keys at the full long-context workload (T=131072, GQA 64/8,
cp=16), identities that hold at any size, and run-to-run determinism of dK / dV."""
import math

import numpy as np
import pytest
import torch

import context_packed_sequence_cp_b200 as thd
from context_packed_sequence_cp_b200 import synthetic as syn
from oracle import attention as A
from tests.gpu_util import BF16_MAX, BF16_MEAN, assert_bf16_close, unpermute_rows

pytestmark = pytest.mark.gpu


def run_fwd_bwd(cu, cp, q, k, v, do, repeat=1):
    dev = torch.device("cuda:0")
    plan = thd.Plan(cu, cp).upload()
    q_rm = thd.thd_kv_gather(plan, q.to(dev))
    k_rm, v_rm = thd.thd_kv_gather(plan, k.to(dev), v.to(dev))
    do_rm = thd.thd_kv_gather(plan, do.to(dev))
    o_rm, lse_rm = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm)
    outs = []
    for _ in range(repeat):
        outs.append([x.cpu().numpy() for x in thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm)])
    torch.cuda.synchronize()
    assert plan.device_status() == 0, "a bounded wait gave up"
    q_idx = plan.export()["q_idx"]
    res = [[unpermute_rows(x, q_idx) for x in o] for o in outs]
    return (res if repeat > 1 else res[0]), plan


@pytest.mark.parametrize("hq,hkv", [(2, 2), (8, 2), (6, 1)])
@pytest.mark.parametrize("cp", [1, 2, 4, 8, 16])
def test_bwd_small_layouts_full(hq, hkv, cp):
    rng = np.random.default_rng(cp * 7 + hq)
    lens = syn.random_lengths(rng, 2500, 2 * cp, max_docs=5) + [2 * cp]
    cu = syn.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v, do = syn.make_tensors(T, hq, hkv, 128, 128, torch.bfloat16, seed=cp + hq, with_do=True)
    (dq, dk, dv), _ = run_fwd_bwd(cu, cp, q, k, v, do)
    o, lse = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(128))
    wq, wk, wv = A.attention_bwd(q, k, v, o, lse, do, cu, 1 / math.sqrt(128))
    assert_bf16_close(dq, wq, "dQ")
    assert_bf16_close(dk, wk, "dK")
    assert_bf16_close(dv, wv, "dV")


@pytest.mark.parametrize("lens,cp", [([2] * 64, 1), ([16] * 40, 8), ([2], 1), ([32, 16, 32], 8)])
def test_bwd_degenerate_layouts(lens, cp):
    """Documents of the minimum length 2*cp only, and a single two-token sequence."""
    cu = syn.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v, do = syn.make_tensors(T, 4, 2, 128, 128, torch.bfloat16, seed=len(lens) + cp, with_do=True)
    (dq, dk, dv), _ = run_fwd_bwd(cu, cp, q, k, v, do)
    o, lse = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(128))
    wq, wk, wv = A.attention_bwd(q, k, v, o, lse, do, cu, 1 / math.sqrt(128))
    assert_bf16_close(dq, wq, "dQ")
    assert_bf16_close(dk, wk, "dK")
    assert_bf16_close(dv, wv, "dV")


@pytest.fixture(scope="module")
def long_context_run():
    """The long-context workload (T=131072, cp=16, GQA 64/8) through fwd + bwd once."""
    w = syn.WORKLOADS[5]
    cu, (q, k, v, do) = syn.workload_inputs(5, 0)
    (dq, dk, dv), plan = run_fwd_bwd(cu, w.cp, q, k, v, do)
    return w, cu, (q, k, v, do), (dq, dk, dv)


def test_bwd_long_context_workload_sampled(long_context_run):
    """dQ at sampled rows (the deepest rows of the 65536-token document among them),
    dK/dV at sampled keys near the end of their document, and two identities over all
    keys: sum_j dV_j = sum_i sum_{h in g} dO_ih and sum_j dK_j = 0."""
    w, cu, (q, k, v, do), (dq, dk, dv) = long_context_run
    scale = 1 / math.sqrt(128)
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()
    rng = np.random.default_rng(5)
    # dQ rows: the long document's first and last tiles, its chunk seams and its deep
    # rows (walks of up to 512 key tiles), and rows of short documents
    rows = [0, 127, 128, 2047, 2048, 32768, 49152, 65400, 65534, 65535]
    rows += [int(x) for x in rng.integers(0, 65536, 6)] + [int(x) for x in rng.integers(65536, w.T, 18)]
    heads = [0, 9, 63]
    want = A.attention_bwd_rows(q, k, v, do, cu, scale, rows, heads)
    assert_bf16_close(dq[rows][:, heads], want, "dQ rows")
    # dK / dV keys: last keys of the long document, and keys of short documents
    keys = [65535, 65530]
    ends = cu[1:]
    for d in rng.integers(1, len(cu) - 1, 6):
        keys.append(int(ends[d]) - 1 - int(rng.integers(0, 4)))
    kvh = [0, 5]
    wk, wv = A.attention_bwd_keys(q, k, v, do, cu, scale, keys, kvh)
    assert_bf16_close(dk[keys][:, kvh], wk, "dK keys")
    assert_bf16_close(dv[keys][:, kvh], wv, "dV keys")
    # identities over every key of every document (fp64 host sums)
    # (a random-walk sum of the same terms would be ~ sqrt(sum of squares); the
    # identities must hold far below that: bf16 rounding of P, dS and O is the slack)
    do64 = do.double().numpy().reshape(w.T, w.hkv, w.hq // w.hkv, w.dv).sum(axis=2)
    dv64, dk64 = dv.astype(np.float64), dk.astype(np.float64)
    walk_v = np.sqrt((dv64 ** 2).sum(axis=0))
    walk_k = np.sqrt((dk64 ** 2).sum(axis=0))
    assert np.all(np.abs(dv64.sum(axis=0) - do64.sum(axis=0)) <= 0.02 * walk_v)
    assert np.all(np.abs(dk64.sum(axis=0)) <= 0.05 * walk_k)


def test_bwd_long_context_longest_key_tiles_full(long_context_run):
    """Element by element, the key tiles whose dK/dV walks are the longest of the
    launch: keys 0..127 of the 65536-token document (seen by all its 512 query tiles x 8
    query heads) and keys 32768..32895 (256 query tiles), for two key/value heads, with
    the oracle's blocked key form (every query row of the document that sees them)."""
    w, cu, (q, k, v, do), (dq, dk, dv) = long_context_run
    blocks = [(0, 128), (32768, 128)]
    kvh = [0, 5]
    wk, wv = A.attention_bwd_key_blocks(q, k, v, do, cu, 1 / math.sqrt(128), blocks, kvh)
    for (j0, n), gk, gv in zip(blocks, wk, wv):
        assert_bf16_close(dk[j0:j0 + n][:, kvh], gk, f"dK keys {j0}..{j0 + n - 1}")
        assert_bf16_close(dv[j0:j0 + n][:, kvh], gv, f"dV keys {j0}..{j0 + n - 1}")


def test_bwd_single_16k_document_full():
    """One 16384-token document, cp=16, GQA 16/2: walks of up to 128 query tiles per key
    tile and 128 key tiles per query tile, every output compared (O, lse, dQ, dK, dV)."""
    cu = np.array([0, 16384], dtype=np.int32)
    q, k, v, do = syn.make_tensors(16384, 16, 2, 128, 128, torch.bfloat16, seed=16, with_do=True)
    dev = torch.device("cuda:0")
    plan = thd.Plan(cu, 16).upload()
    q_rm = thd.thd_kv_gather(plan, q.to(dev))
    k_rm, v_rm = thd.thd_kv_gather(plan, k.to(dev), v.to(dev))
    do_rm = thd.thd_kv_gather(plan, do.to(dev))
    o_rm, lse_rm = thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm)
    grads = thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm)
    torch.cuda.synchronize()
    assert plan.device_status() == 0, "a bounded wait gave up"
    q_idx = plan.export()["q_idx"]
    o = unpermute_rows(o_rm.float().cpu().numpy(), q_idx)
    lse = unpermute_rows(lse_rm.cpu().numpy().T, q_idx).T
    dq, dk, dv = (unpermute_rows(x.cpu().numpy(), q_idx) for x in grads)
    scale = 1 / math.sqrt(128)
    wo, wl = A.attention_fwd(q, k, v, cu, scale)
    assert_bf16_close(o, wo, "O")
    assert np.abs(lse - wl).max() <= 1e-3
    wq, wk, wv = A.attention_bwd(q, k, v, wo, wl, do, cu, scale)
    assert_bf16_close(dq, wq, "dQ")
    assert_bf16_close(dk, wk, "dK")
    assert_bf16_close(dv, wv, "dV")


def test_bwd_key_gradients_are_deterministic():
    lens = [1024, 96, 3072]
    cu = syn.cu_seqlens_of(lens)
    q, k, v, do = syn.make_tensors(int(cu[-1]), 8, 2, 128, 128, torch.bfloat16, seed=3, with_do=True)
    runs, _ = run_fwd_bwd(cu, 4, q, k, v, do, repeat=2)
    (dq0, dk0, dv0), (dq1, dk1, dv1) = runs
    assert np.array_equal(dk0, dk1) and np.array_equal(dv0, dv1)
    assert np.abs(dq0 - dq1).max() <= 1e-4   # dQ sums partial products with fp32 reductions


def test_bwd_gradients_independent_of_cp():
    lens = [512, 2048, 64, 1536]
    cu = syn.cu_seqlens_of(lens)
    q, k, v, do = syn.make_tensors(int(cu[-1]), 4, 2, 128, 128, torch.bfloat16, seed=11, with_do=True)
    ref = run_fwd_bwd(cu, 1, q, k, v, do)[0]
    for cp in (2, 4, 8, 16):
        got = run_fwd_bwd(cu, cp, q, k, v, do)[0]
        for a, b in zip(got, ref):
            assert np.abs(a - b).max() <= BF16_MAX and np.abs(a - b).mean() <= BF16_MEAN


def test_bwd_rejects_unsupported():
    plan = thd.Plan([0, 32], 2).upload()
    x = torch.zeros(32, 2, 192, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(32, 2, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 32, device="cuda")
    with pytest.raises(thd.ThdError) as e:
        thd.thd_cp_attn_bwd(plan, x, x, y, y, lse, y)
    assert e.value.kind == "UNSUPPORTED"


@pytest.mark.parametrize("cp", [2, 4])
def test_bwd_position_tiles_around_the_chunk_threshold(cp):
    """The backward walks the forward tables: documents whose chunks are shorter than a
    tile as position tiles (keys, queries and their gradients gathered / added through
    rm_of_global), the others rank-major; chunk sizes 1, 17, 64, 127 and 128, 129, 300 in
    one packed sequence, GQA 8/2, every gradient compared."""
    chunks = [1, 17, 64, 127, 128, 129, 300, 3]
    cu = syn.cu_seqlens_of([2 * cp * c for c in chunks])
    T = int(cu[-1])
    q, k, v, do = syn.make_tensors(T, 8, 2, 128, 128, torch.bfloat16, seed=50 + cp, with_do=True)
    (dq, dk, dv), plan = run_fwd_bwd(cu, cp, q, k, v, do)
    assert (plan.export_fwd()["fqtiles"][:, 2] < 0).any()
    o, lse = A.attention_fwd(q, k, v, cu, 1 / math.sqrt(128))
    wq, wk, wv = A.attention_bwd(q, k, v, o, lse, do, cu, 1 / math.sqrt(128))
    assert_bf16_close(dq, wq, "dQ")
    assert_bf16_close(dk, wk, "dK")
    assert_bf16_close(dv, wv, "dV")

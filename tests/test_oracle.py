"""Pins of the fp64 oracle against things other than itself: a hand-derived worked
example, closed forms, brute force on tiny inputs, library routines for the special
cases that reduce to them, and finite differences.  CPU only."""
import os

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import partition as P
from oracle import tiles as TT
from context_packed_sequence_cp_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, *vals = line.split()
                out[key] = np.array([int(x) for x in vals])
    return out


def _layouts(n, cps=(1, 2, 4), T_max=256, seed=0):
    rng = np.random.default_rng(seed)
    for _ in range(n):
        cp = int(rng.choice(cps))
        lens = syn.random_lengths(rng, T_max, 2 * cp, max_docs=6)
        yield cp, syn.cu_seqlens_of(lens)


# ---------------------------------------------------------------- partition pins

def test_partition_worked_example():
    g = _read_golden("partition_cp2_docs4_8.txt")
    q_idx, rm = P.partition(g["cu_seqlens"], int(g["cp"][0]))
    assert np.array_equal(q_idx, g["q_idx"])
    assert np.array_equal(rm, g["rm_of_global"])
    assert np.array_equal(P.rank_causal_pairs(g["cu_seqlens"], 2), g["rank_pairs"])
    plan = TT.tile_plan(g["cu_seqlens"], 2)
    assert np.array_equal(plan["qtiles"][0], g["qtile0"])
    assert np.array_equal(plan["entries"][0], g["entry0"])
    assert np.array_equal(plan["entries"][1], g["entry1"])


@pytest.mark.parametrize("seed", range(3))
def test_partition_bijection_and_balance(seed):
    for cp, cu in _layouts(20, cps=(1, 2, 3, 4, 8), seed=seed):
        T = int(cu[-1])
        q_idx, rm = P.partition(cu, cp)
        assert np.array_equal(np.sort(q_idx), np.arange(T))
        assert np.array_equal(q_idx[rm], np.arange(T))
        assert np.all(P.rank_query_counts(cu, cp) == T // cp)
        pairs = P.rank_causal_pairs(cu, cp)
        # closed form per rank: sum_d (2cp-1) c^2 + c (c+1), identical for every rank
        c = np.diff(cu).astype(np.int64) // (2 * cp)
        closed = int(np.sum((2 * cp - 1) * c * c + c * (c + 1)))
        assert np.all(pairs == closed)
        assert int(pairs.sum()) == P.causal_pairs_total(cu)


def test_partition_rank_major_closed_form():
    """Closed form of a token's rank-major row, derived independently of the
    enumeration: offset o in a document of chunk size c lies in chunk k = o // c."""
    for cp, cu in _layouts(30, cps=(1, 2, 4, 8), seed=7):
        T = int(cu[-1])
        Tl = T // cp
        _, rm = P.partition(cu, cp)
        for d in range(cu.size - 1):
            s, L = int(cu[d]), int(cu[d + 1] - cu[d])
            c = L // (2 * cp)
            for o in range(L):
                k, i = divmod(o, c)
                rank = k if k < cp else 2 * cp - 1 - k
                row = rank * Tl + s // cp + (0 if k < cp else c) + i
                assert rm[s + o] == row


@pytest.mark.parametrize("cu,cp,kind", [
    ([0, 4, 12], 0, P.BAD_ARG),
    ([1, 4, 12], 2, P.BAD_SEQLENS),
    ([0, 4, 4, 12], 2, P.BAD_SEQLENS),
    ([0, 8, 4], 2, P.BAD_SEQLENS),
    ([0, 6, 12], 2, P.NOT_DIVISIBLE),
    ([0], 2, P.BAD_ARG),
])
def test_partition_rejects(cu, cp, kind):
    with pytest.raises(P.PartitionError) as e:
        P.partition(np.array(cu), cp)
    assert e.value.kind == kind


# ---------------------------------------------------------------- tile-table pins

@pytest.mark.parametrize("seed", range(3))
def test_tiles_cover_every_visible_pair_once(seed):
    for cp, cu in _layouts(12, cps=(1, 2, 4, 8), T_max=1200, seed=100 + seed):
        plan = TT.tile_plan(cu, cp)
        total = 0
        for qt, q in enumerate(plan["qtiles"]):
            r, d, row0, m, qpos0, qbrk, qjump, qmax, nk, e0, ds, de = (int(x) for x in q)
            qpos = plan["q_idx"][row0:row0 + m]
            assert np.array_equal(TT.decode_run(qpos0, qbrk, qjump, m), qpos)
            assert qmax == qpos[-1] and ds == cu[d] and de == cu[d + 1]
            for e in range(e0, e0 + nk):
                en = plan["entries"][e]
                kpos = plan["q_idx"][en[0]:en[0] + en[1]]
                assert np.array_equal(TT.decode_run(en[2], en[3], en[4], int(en[1])), kpos)
                cnt = TT.visible_pairs_of_entry(plan, qt, e)
                assert cnt > 0, "listed entries hold a visible pair"
                assert (en[5] == TT.UNMASKED) == (cnt == m * int(en[1]))
                total += cnt
        assert total == P.causal_pairs_total(cu)


@pytest.mark.parametrize("seed", range(3))
def test_forward_tables_cover_every_visible_pair_once(seed):
    """The forward tables (rank-major tiles, position tiles for short-chunk documents)
    list every visible (query, key) pair exactly once, every query row of the packed
    sequence in exactly one query tile, and classes that match the pairs."""
    for cp, cu in _layouts(12, cps=(1, 2, 4, 8), T_max=1500, seed=300 + seed):
        plan = TT.tile_plan(cu, cp)
        doc = P.doc_of_token(cu)
        seen_q = np.zeros(int(cu[-1]), dtype=np.int64)
        total = 0
        for q in plan["fqtiles"]:
            r, d, row0, m, qpos0, qbrk, qjump, qmax, nk, e0, ds, de = (int(x) for x in q)
            qpos = TT.decode_run(qpos0, qbrk, qjump, m)
            if row0 >= 0:
                assert np.array_equal(plan["q_idx"][row0:row0 + m], qpos)
            else:   # position tile of a short-chunk document
                assert (de - ds) // (2 * cp) < TT.BM and r == -1
                assert np.array_equal(qpos, np.arange(qpos0, qpos0 + m))
            assert np.all(doc[qpos] == d) and qmax == qpos[-1]
            seen_q[qpos] += 1
            for en in plan["fentries"][e0:e0 + nk]:
                kpos = TT.decode_run(int(en[2]), int(en[3]), int(en[4]), int(en[1]))
                if en[0] >= 0:
                    assert np.array_equal(plan["q_idx"][en[0]:en[0] + en[1]], kpos)
                # its key tile (a tile of the same tables) starts with the entry's first key
                kt = plan["fqtiles"][en[6]]
                assert kt[4] == kpos[0] and kt[1] == d and (kt[2] == en[0] or kt[2] < 0)
                assert np.all(doc[kpos] == d)
                vis = kpos[None, :] <= qpos[:, None]
                cnt = int(vis.sum())
                assert cnt > 0 and vis.any(axis=0).all()
                assert (en[5] == TT.UNMASKED) == bool(vis.all())
                total += cnt
        assert np.all(seen_q == 1)
        assert total == P.causal_pairs_total(cu)
        order = plan["flpt"]
        assert sorted(order.tolist()) == list(range(plan["fqtiles"].shape[0]))
        nk = plan["fqtiles"][:, 8]
        for a, b in zip(order[:-1], order[1:]):
            assert nk[a] > nk[b] or (nk[a] == nk[b] and a < b)


def test_tiles_pairwise_bruteforce_tiny():
    """Every visible (query, key) pair of the packed sequence lies in exactly one
    listed entry of its query's tile; checked pair by pair."""
    for cp, cu in _layouts(10, cps=(1, 2, 4), T_max=96, seed=5):
        plan = TT.tile_plan(cu, cp)
        q_idx = plan["q_idx"]
        doc = P.doc_of_token(cu)
        T = int(cu[-1])
        covered = np.zeros((T, T), dtype=np.int64)
        for qt, q in enumerate(plan["qtiles"]):
            row0, m, nk, e0 = int(q[2]), int(q[3]), int(q[8]), int(q[9])
            for e in range(e0, e0 + nk):
                k0, nv = int(plan["entries"][e, 0]), int(plan["entries"][e, 1])
                for a in range(row0, row0 + m):
                    for b in range(k0, k0 + nv):
                        gi, gj = q_idx[a], q_idx[b]
                        if doc[gi] == doc[gj] and gj <= gi:
                            covered[gi, gj] += 1
        idx = np.arange(T)
        want = ((doc[:, None] == doc[None, :]) & (idx[None, :] <= idx[:, None])).astype(np.int64)
        assert np.array_equal(covered, want)


def test_backward_transpose_and_lpt():
    for cp, cu in _layouts(8, cps=(1, 2, 4), T_max=2000, seed=11):
        plan = TT.tile_plan(cu, cp)
        n = plan["qtiles"].shape[0]
        seen = np.zeros(plan["entries"].shape[0], dtype=np.int64)
        for kt in range(n):
            lst = plan["kt_list"][plan["kt_off"][kt]:plan["kt_off"][kt + 1]]
            qmax = plan["qtiles"][lst[:, 0], 7]
            assert np.all(np.diff(qmax) < 0)   # descending last query position
            # the list is every q-tile of the key tile's document whose last row is at or
            # past the key tile's first key: a prefix of one per-document order
            kpos_min = int(plan["q_idx"][plan["qtiles"][kt, 2]])
            d = plan["qtiles"][kt, 1]
            want = [qt for qt in range(n) if plan["qtiles"][qt, 1] == d and plan["qtiles"][qt, 7] >= kpos_min]
            assert sorted(lst[:, 0].tolist()) == want
            for qt, e in lst:
                assert plan["entries"][e, 6] == kt
                assert plan["qtiles"][qt, 9] <= e < plan["qtiles"][qt, 9] + plan["qtiles"][qt, 8]
                assert plan["entries"][e, 0] == plan["qtiles"][kt, 2]
                seen[e] += 1
        assert np.all(seen == 1)
        # longest-first orders: permutations, lengths non-increasing, equal lengths in
        # ascending tile index (so that the order is unique)
        lengths = {"lpt": plan["qtiles"][:, 8], "kt_lpt": np.diff(plan["kt_off"])}
        for key, ln in lengths.items():
            order = plan[key]
            assert sorted(order.tolist()) == list(range(n)), key
            for a, b in zip(order[:-1], order[1:]):
                assert ln[a] > ln[b] or (ln[a] == ln[b] and a < b), (key, a, b)
        # each key tile's list length counts the q-tiles of its document that reach it
        for kt in range(n):
            d = plan["qtiles"][kt, 1]
            kpos_min = int(plan["q_idx"][plan["qtiles"][kt, 2]])
            reach = sum(1 for qt in range(n) if plan["qtiles"][qt, 1] == d and plan["qtiles"][qt, 7] >= kpos_min)
            assert lengths["kt_lpt"][kt] == reach


# ---------------------------------------------------------------- attention pins

def _rand(T, hq, hkv, dqk, dv, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(T, hq, dqk, generator=g, dtype=torch.float64),
            torch.randn(T, hkv, dqk, generator=g, dtype=torch.float64),
            torch.randn(T, hkv, dv, generator=g, dtype=torch.float64),
            torch.randn(T, hq, dv, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("hq,hkv,dqk,dv", [(2, 2, 16, 16), (4, 2, 24, 8), (4, 1, 12, 20)])
def test_fwd_matches_bruteforce_mask(hq, hkv, dqk, dv):
    for i, (cp, cu) in enumerate(_layouts(6, cps=(1, 2), T_max=160, seed=3)):
        T = int(cu[-1])
        q, k, v, _ = _rand(T, hq, hkv, dqk, dv, i)
        o1, l1 = A.attention_fwd(q, k, v, cu, 0.3)
        o2, l2 = A.bruteforce_fwd(q, k, v, cu, 0.3)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_fwd_single_document_is_library_causal_attention():
    """One document reduces to textbook causal attention (torch SDPA, float64)."""
    T, hq, hkv, d = 300, 4, 2, 32
    q, k, v, _ = _rand(T, hq, hkv, d, d, 1)
    o, lse = A.attention_fwd(q, k, v, [0, T], d ** -0.5)
    kk = k.repeat_interleave(hq // hkv, dim=1)
    vv = v.repeat_interleave(hq // hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1), kk.transpose(0, 1), vv.transpose(0, 1), is_causal=True,
        scale=d ** -0.5).transpose(0, 1)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    s = torch.einsum("ihd,jhd->hij", q, kk) * d ** -0.5
    s = s.masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_fwd_documents_are_independent():
    """Each document equals standalone causal attention on it."""
    cu = np.array([0, 64, 96, 224])
    q, k, v, _ = _rand(224, 2, 2, 16, 16, 9)
    o, lse = A.attention_fwd(q, k, v, cu, 0.25)
    for d in range(3):
        s, e = cu[d], cu[d + 1]
        od, ld = A.attention_fwd(q[s:e], k[s:e], v[s:e], [0, e - s], 0.25)
        np.testing.assert_allclose(o[s:e], od, atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse[:, s:e], ld, atol=1e-13, rtol=0)


@pytest.mark.parametrize("cp", [1, 2, 4, 8])
def test_fwd_cp_formulation_is_cp_independent(cp):
    """Rank-local attention over the all-gathered rank-major K/V, un-permuted, equals
    the per-document definition for every cp."""
    rng = np.random.default_rng(cp)
    lens = syn.random_lengths(rng, 256, 2 * 8, max_docs=5)
    cu = syn.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v, _ = _rand(T, 4, 2, 16, 8, cp)
    o, lse = A.attention_fwd(q, k, v, cu, 0.2)
    q_idx, _ = P.partition(cu, cp)
    o_rm, l_rm = A.cp_rank_fwd(q, k, v, cu, 0.2, q_idx, cp)
    o_g = np.empty_like(o_rm)
    o_g[q_idx] = o_rm
    l_g = np.empty_like(l_rm)
    l_g[:, q_idx] = l_rm
    np.testing.assert_allclose(o_g, o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l_g, lse, atol=1e-12, rtol=0)


def test_mla_compact_keys_split_the_score_into_two_dot_products():
    """Compact MLA keys: every score is the per-head dot product plus the dot product
    with the token's shared rope key, checked pair by pair with explicit loops."""
    cu = np.array([0, 6, 16])
    T, hq, hkv, dn, dr, dv = 16, 4, 2, 5, 3, 4
    g = np.random.default_rng(4)
    q = g.standard_normal((T, hq, dn + dr))
    kn = g.standard_normal((T, hkv, dn))
    kr = g.standard_normal((T, dr))
    v = g.standard_normal((T, hkv, dv))
    scale = 0.37
    o, lse = A.attention_fwd_mla(q, kn, kr, v, cu, scale)
    for d in range(2):
        s0, s1 = cu[d], cu[d + 1]
        for h in range(hq):
            gh = h // (hq // hkv)
            for i in range(s0, s1):
                sc = []
                for j in range(s0, i + 1):
                    a = sum(q[i, h, t] * kn[j, gh, t] for t in range(dn))
                    b = sum(q[i, h, dn + t] * kr[j, t] for t in range(dr))
                    sc.append(scale * (a + b))
                sc = np.array(sc)
                w = np.exp(sc - sc.max())
                assert abs(lse[h, i] - (sc.max() + np.log(w.sum()))) < 1e-12
                want = (w[:, None] * v[s0:i + 1, gh, :]).sum(0) / w.sum()
                assert np.allclose(o[i, h], want, atol=1e-12)


def test_gqa_with_equal_heads_is_mha():
    cu = np.array([0, 48, 128])
    q, k, v, _ = _rand(128, 4, 4, 16, 16, 4)
    o, _ = A.attention_fwd(q, k, v, cu, 0.25)
    for h in range(4):
        oh, _ = A.attention_fwd(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], cu, 0.25)
        np.testing.assert_allclose(o[:, h:h + 1], oh, atol=1e-13, rtol=0)


def test_bwd_matches_library_autograd_single_document():
    T, hq, hkv, d = 96, 4, 2, 16
    q, k, v, do = _rand(T, hq, hkv, d, d, 2)
    o, lse = A.attention_fwd(q, k, v, [0, T], 0.3)
    dq, dk, dv = A.attention_bwd(q, k, v, o, lse, do, [0, T], 0.3)
    qq, kk, vv = (x.clone().requires_grad_() for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qq.transpose(0, 1), kk.repeat_interleave(2, 1).transpose(0, 1),
        vv.repeat_interleave(2, 1).transpose(0, 1), is_causal=True, scale=0.3).transpose(0, 1)
    ref.backward(do)
    np.testing.assert_allclose(dq, qq.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, kk.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, vv.grad.numpy(), atol=1e-11, rtol=0)


def test_bwd_finite_differences_multi_document():
    cu = np.array([0, 8, 20, 32])
    T, hq, hkv, d = 32, 2, 1, 6
    q, k, v, do = (x.numpy() for x in _rand(T, hq, hkv, d, d, 5))

    def loss(q_, k_, v_):
        o_, _ = A.attention_fwd(q_, k_, v_, cu, 0.5)
        return float(np.sum(o_ * do))

    o, lse = A.attention_fwd(q, k, v, cu, 0.5)
    dq, dk, dv = A.attention_bwd(q, k, v, o, lse, do, cu, 0.5)
    rng = np.random.default_rng(0)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) < 1e-7, (name, idx, fd, g[idx])


def test_sampled_forms_match_full_forms():
    cu = np.array([0, 40, 136, 200])
    T, hq, hkv, d = 200, 4, 2, 8
    q, k, v, do = (x.numpy() for x in _rand(T, hq, hkv, d, d, 6))
    o, lse = A.attention_fwd(q, k, v, cu, 0.4)
    dq, dk, dv = A.attention_bwd(q, k, v, o, lse, do, cu, 0.4)
    rows = [0, 39, 40, 77, 135, 199]
    heads = [0, 3]
    Os, Ls = A.attention_fwd_rows(q, k, v, cu, 0.4, rows, heads)
    np.testing.assert_allclose(Os, o[rows][:, heads], atol=1e-13, rtol=0)
    np.testing.assert_allclose(Ls, lse[heads][:, rows].T, atol=1e-13, rtol=0)
    dQs = A.attention_bwd_rows(q, k, v, do, cu, 0.4, rows, heads)
    np.testing.assert_allclose(dQs, dq[rows][:, heads], atol=1e-12, rtol=0)
    keys = [0, 39, 130, 199]
    dKs, dVs = A.attention_bwd_keys(q, k, v, do, cu, 0.4, keys, [0, 1])
    np.testing.assert_allclose(dKs, dk[keys], atol=1e-12, rtol=0)
    np.testing.assert_allclose(dVs, dv[keys], atol=1e-12, rtol=0)


def test_key_block_form_matches_full_form():
    """The blocked key-block form (row blocks smaller than the document, blocks at the
    document's start, middle and end, ragged sizes) equals the full backward."""
    cu = np.array([0, 24, 1224, 1300])
    T, hq, hkv, d = 1300, 4, 2, 8
    q, k, v, do = (x.numpy() for x in _rand(T, hq, hkv, d, d, 9))
    o, lse = A.attention_fwd(q, k, v, cu, 0.3)
    dq, dk, dv = A.attention_bwd(q, k, v, o, lse, do, cu, 0.3)
    blocks = [(24, 128), (600, 77), (1100, 124)]
    dKs, dVs = A.attention_bwd_key_blocks(q, k, v, do, cu, 0.3, blocks, [1, 0])
    for (j0, n), gk, gv in zip(blocks, dKs, dVs):
        np.testing.assert_allclose(gk, dk[j0:j0 + n][:, [1, 0]], atol=1e-12, rtol=0)
        np.testing.assert_allclose(gv, dv[j0:j0 + n][:, [1, 0]], atol=1e-12, rtol=0)
    # a key block in a single-block document, and the last key of a document alone
    dKs, dVs = A.attention_bwd_key_blocks(q, k, v, do, cu, 0.3, [(0, 24)], [0])
    np.testing.assert_allclose(dKs[0], dk[0:24][:, [0]], atol=1e-12, rtol=0)
    dKs, dVs = A.attention_bwd_key_blocks(q, k, v, do, cu, 0.3, [(1299, 1)], [1])
    np.testing.assert_allclose(dVs[0], dv[1299:1300][:, [1]], atol=1e-12, rtol=0)


# ---------------------------------------------------------------- workloads

@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_workload_layouts_satisfy_contract(cfg):
    w = syn.WORKLOADS[cfg]
    for seed in range(3):
        lens = syn.doc_lengths(cfg, seed)
        assert sum(lens) == w.T
        assert all(L > 0 and L % (2 * w.cp) == 0 for L in lens)
        P.validate(syn.cu_seqlens_of(lens), w.cp)

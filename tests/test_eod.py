"""Document boundaries from EOD tokens and per-document position ids: the oracle
(oracle/eod.py) pinned by a hand-derived example and invariants, then the library's
host entry points compared with it bit for bit; and the rotary-embedding oracle
(oracle/rope.py) pinned by properties that fix the rotation.  CPU only."""
import os

import numpy as np
import pytest

from oracle import eod as E

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "eod_example.txt")


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, *v = line.split()
                out[k] = np.array([int(x) for x in v])
    return out


def test_oracle_worked_example():
    g = _golden()
    cu = E.cu_seqlens_from_eod(g["tokens"], int(g["eod"][0]))
    assert np.array_equal(cu, g["cu_seqlens"])
    assert np.array_equal(E.position_ids(cu), g["positions"])


@pytest.mark.parametrize("seed", range(5))
def test_oracle_invariants(seed):
    rng = np.random.default_rng(seed)
    tok = rng.integers(0, 6, size=int(rng.integers(1, 400))).astype(np.int32)
    cu = E.cu_seqlens_from_eod(tok, 0)
    T = tok.size
    assert cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) > 0)
    for d in range(cu.size - 1):
        s, e = cu[d], cu[d + 1]
        assert not np.any(tok[s:e - 1] == 0)               # no EOD inside a document
        assert tok[e - 1] == 0 or e == T                    # it ends with EOD, or at the end
    pos = E.position_ids(cu)
    assert pos.size == T
    for d in range(cu.size - 1):
        assert list(pos[cu[d]:cu[d + 1]]) == list(range(cu[d + 1] - cu[d]))


@pytest.mark.parametrize("tokens,want", [
    ([4, 4, 4], [0, 3]),              # no EOD: one document
    ([9, 9, 9], [0, 1, 2, 3]),        # only EODs: single-token documents
    ([9, 4, 4], [0, 1, 3]),           # EOD first
    ([4, 4, 9], [0, 3]),              # EOD last: no empty tail document
    ([9], [0, 1]),
])
def test_oracle_edge_cases(tokens, want):
    assert np.array_equal(E.cu_seqlens_from_eod(np.array(tokens), 9), want)


def test_library_matches_oracle():
    import context_packed_sequence_cp_b200 as thd
    g = _golden()
    assert np.array_equal(thd.thd_cu_seqlens_from_eod(g["tokens"], 9), g["cu_seqlens"])
    rng = np.random.default_rng(3)
    for _ in range(50):
        T = int(rng.integers(1, 3000))
        tok = rng.integers(0, int(rng.integers(2, 40)), size=T).astype(np.int32)
        eod = int(rng.integers(0, 3))
        cu = thd.thd_cu_seqlens_from_eod(tok, eod)
        assert np.array_equal(cu, E.cu_seqlens_from_eod(tok, eod))
        assert np.array_equal(thd.thd_position_ids(cu), E.position_ids(cu))
    for tokens, _ in [([4, 4, 4], 0), ([9, 9, 9], 0), ([9, 4, 4], 0), ([4, 4, 9], 0), ([9], 0)]:
        assert np.array_equal(thd.thd_cu_seqlens_from_eod(np.array(tokens), 9),
                              E.cu_seqlens_from_eod(np.array(tokens), 9))


def test_library_boundaries_feed_the_plan():
    """EOD-derived boundaries of documents whose lengths are multiples of 2*cp plan as
    the same layout given directly."""
    import context_packed_sequence_cp_b200 as thd
    lens, cp = [8, 24, 16], 4
    tok = np.concatenate([np.r_[np.full(L - 1, 3), 0] for L in lens]).astype(np.int32)
    cu = thd.thd_cu_seqlens_from_eod(tok, 0)
    assert np.array_equal(cu, [0, 8, 32, 48])
    a, b = thd.Plan(cu, cp).export(), thd.Plan([0, 8, 32, 48], cp).export()
    assert all(np.array_equal(a[k], b[k]) for k in a)


def test_library_errors():
    import ctypes
    import context_packed_sequence_cp_b200 as thd
    from context_packed_sequence_cp_b200 import _lib
    L = _lib.lib()
    tok = np.array([1, 0, 1], dtype=np.int32)
    n = ctypes.c_int32(-1)
    p = tok.ctypes.data_as(ctypes.c_void_p)
    assert L.thd_cu_seqlens_from_eod(p, 0, 0, None, 0, ctypes.byref(n)) == -1          # T < 1
    cu = np.zeros(2, dtype=np.int32)                                                     # needs 3
    assert L.thd_cu_seqlens_from_eod(p, 3, 0, cu.ctypes.data_as(ctypes.c_void_p), 2, ctypes.byref(n)) == -9
    assert n.value == 2
    with pytest.raises(thd.ThdError) as e:
        thd.thd_position_ids([0, 3, 3])                                                  # empty document
    assert e.value.kind == "BAD_SEQLENS"


# ---------------------------------------------------------------- rotary embedding oracle
from oracle import rope as R   # noqa: E402


def _rand_x(T, H, D, seed):
    return np.random.default_rng(seed).standard_normal((T, H, D))


def test_rope_is_complex_rotation():
    """Each pair (x_i, x_{i+R/2}) as the complex number x_i + j x_{i+R/2}, multiplied by
    exp(j * pos * base^(-2i/R)); dimensions past R untouched."""
    T, H, D, Rd = 7, 2, 10, 8
    x = _rand_x(T, H, D, 1)
    pos = np.array([0, 1, 5, 17, 300, 65535, 2])
    y = R.rope(x, pos, Rd, 500.0)
    for i in range(Rd // 2):
        z = (x[:, :, i] + 1j * x[:, :, i + Rd // 2]) * np.exp(1j * pos[:, None] * 500.0 ** (-2 * i / Rd))
        assert np.allclose(y[:, :, i], z.real, atol=1e-12) and np.allclose(y[:, :, i + Rd // 2], z.imag, atol=1e-12)
    assert np.array_equal(y[:, :, Rd:], x[:, :, Rd:])


def test_rope_position_zero_is_identity_and_norms_are_kept():
    x = _rand_x(5, 3, 16, 2)
    assert np.allclose(R.rope(x, np.zeros(5), 16), x, atol=0)
    y = R.rope(x, np.arange(5) * 1000, 16)
    h = 8
    assert np.allclose(x[:, :, :h] ** 2 + x[:, :, h:] ** 2, y[:, :, :h] ** 2 + y[:, :, h:] ** 2, atol=1e-12)


def test_rope_scores_depend_on_relative_position_only():
    q = _rand_x(1, 1, 16, 3)
    k = _rand_x(1, 1, 16, 4)
    def score(m, n):
        return float((R.rope(q, [m], 16) * R.rope(k, [n], 16)).sum())
    for m, n, d in [(5, 2, 100), (40000, 39000, 7), (9, 9, 123)]:
        assert abs(score(m, n) - score(m + d, n + d)) < 1e-9

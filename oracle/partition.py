"""Oracle: validation and EOD-aware symmetric partitioning.  TEST INFRASTRUCTURE ONLY.

Source: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance".
  * "Does this PR introduce any user-facing change?": every packed subsequence
    length must be divisible by 2 * context_parallel_size.
  * "What this PR does / why we need it?": EOD-aware symmetric sequence
    partitioning, load-balanced across context-parallel ranks.

Reading of "symmetric" (the page gives no formula): every document of length L is
cut into 2*cp equal chunks of c = L / (2*cp) tokens; virtual rank r owns chunk r
and its mirror chunk 2*cp-1-r.  Inside a rank, documents come in ascending order
and, per document, chunk r precedes chunk 2*cp-1-r, each in ascending position.
The rank-major buffer stacks rank 0's rows, then rank 1's, and so on: it is
exactly what an all-gather of the rank-local shards produces.

Everything here is built by explicit enumeration (``np.arange`` per chunk and an
``argsort`` for the inverse), not by a closed form.
"""
from __future__ import annotations

import numpy as np

# Error classes mirror the library's error codes by name only.
BAD_ARG = "INVALID_ARG"
BAD_SEQLENS = "BAD_SEQLENS"
NOT_DIVISIBLE = "NOT_DIVISIBLE"


class PartitionError(ValueError):
    def __init__(self, kind: str, msg: str):
        super().__init__(f"{kind}: {msg}")
        self.kind = kind


def validate(cu_seqlens, cp: int) -> np.ndarray:
    """Check the input contract and return cu_seqlens as int64.

    cp >= 1; cu_seqlens[0] == 0; every document non-empty (strictly increasing);
    every length divisible by 2*cp (the page's stated constraint)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if int(cp) < 1:
        raise PartitionError(BAD_ARG, f"cp={cp} < 1")
    if cu.ndim != 1 or cu.size < 2:
        raise PartitionError(BAD_ARG, "need at least one document")
    if cu[0] != 0:
        raise PartitionError(BAD_SEQLENS, "cu_seqlens[0] != 0")
    lengths = np.diff(cu)
    if np.any(lengths <= 0):
        raise PartitionError(BAD_SEQLENS, "document lengths must be positive")
    if np.any(lengths % (2 * cp) != 0):
        raise PartitionError(NOT_DIVISIBLE, f"a length is not divisible by 2*cp={2 * cp}")
    return cu


def doc_of_token(cu_seqlens) -> np.ndarray:
    """Document id of every global token (EOD-delimited documents)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    out = np.empty(T, dtype=np.int64)
    for d in range(cu.size - 1):
        out[cu[d]:cu[d + 1]] = d
    return out


def rank_token_lists(cu_seqlens, cp: int) -> list[np.ndarray]:
    """Global token indices owned by each virtual rank, in that rank's local order."""
    cu = validate(cu_seqlens, cp)
    ranks = []
    for r in range(cp):
        parts = []
        for d in range(cu.size - 1):
            s, L = int(cu[d]), int(cu[d + 1] - cu[d])
            c = L // (2 * cp)
            for chunk in (r, 2 * cp - 1 - r):
                parts.append(s + chunk * c + np.arange(c, dtype=np.int64))
        ranks.append(np.concatenate(parts) if parts else np.zeros(0, np.int64))
    return ranks


def partition(cu_seqlens, cp: int):
    """(q_idx, rm_of_global): q_idx[j] is the global token at rank-major row j;
    rm_of_global is its inverse permutation."""
    ranks = rank_token_lists(cu_seqlens, cp)
    q_idx = np.concatenate(ranks).astype(np.int32)
    rm_of_global = np.argsort(q_idx, kind="stable").astype(np.int32)
    return q_idx, rm_of_global


def rank_query_counts(cu_seqlens, cp: int) -> np.ndarray:
    return np.array([len(x) for x in rank_token_lists(cu_seqlens, cp)], dtype=np.int64)


def rank_causal_pairs(cu_seqlens, cp: int) -> np.ndarray:
    """Causal (query, key) pairs each rank's queries attend to, counted one query at a
    time: a query at offset o inside its document sees o + 1 keys (itself included)."""
    cu = validate(cu_seqlens, cp)
    doc = doc_of_token(cu)
    out = []
    for toks in rank_token_lists(cu, cp):
        offs = toks - cu[doc[toks]]
        out.append(int(np.sum(offs + 1)))
    return np.array(out, dtype=np.int64)


def causal_pairs_total(cu_seqlens) -> int:
    """All visible pairs of the packed sequence: sum over documents of L(L+1)/2."""
    L = np.diff(np.asarray(cu_seqlens, dtype=np.int64))
    return int(np.sum(L * (L + 1) // 2))

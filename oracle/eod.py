"""Oracle: document boundaries of an EOD-delimited packed sequence and per-document
position ids.  TEST INFRASTRUCTURE ONLY.

Source: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance",
section "Does this PR introduce any user-facing change?": THD packed sequences with
the attention mask reset at every EOD token.  Reading (the page gives no formula):
a document ends with, and includes, an EOD token; the tokens after the last EOD form
a final document; positions restart at 0 with every document.
"""
from __future__ import annotations

import numpy as np


def cu_seqlens_from_eod(tokens, eod_id: int) -> np.ndarray:
    """cu_seqlens [n_docs + 1]: 0, the index after every EOD token, and T if the
    sequence does not end with an EOD."""
    tok = np.asarray(tokens).ravel()
    T = tok.size
    ends = np.flatnonzero(tok == eod_id) + 1             # exclusive end of each EOD-closed document
    if T == 0 or tok[-1] != eod_id:
        ends = np.concatenate([ends, [T]])
    return np.concatenate([[0], ends]).astype(np.int32)


def position_ids(cu_seqlens) -> np.ndarray:
    """pos[t] = t - start of t's document."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lengths = np.diff(cu)
    starts = np.repeat(cu[:-1], lengths)
    return (np.arange(int(cu[-1])) - starts).astype(np.int32)

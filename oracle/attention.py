"""Oracle: fp64 causal softmax attention with EOD resets.  TEST INFRASTRUCTURE ONLY.

Source: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance".
  * "Does this PR introduce any user-facing change?": causal attention over THD
    packed sequences with EOD attention-mask reset, i.e. a query sees exactly the
    keys of its own document at positions <= its own.
  * "What this PR does / why we need it?": MHA, GQA and expanded MLA.  GQA maps
    query head h to key/value head h // (Hq / Hkv) (contiguous groups: the usual
    convention; the page does not spell it out).  Expanded MLA means a per-head
    key of width Dqk (192) and a value of width Dv (128).

The attention is exact: context-parallel reordering and tile skipping change no
value, so the oracle is the plain definition, evaluated per document and head in
float64:
    S = scale * Q K^T,  S[i, j] = -inf for j > i,
    lse_i = log sum_j exp(S_ij)   (natural log of the scaled scores),
    O = softmax(S) V.
Backward, with Delta_i = sum(dO_i * O_i) and P = exp(S - lse):
    dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),
    dQ = scale * dS K,  dK = scale * dS^T Q,
summed over the query heads that share a key/value head.

Inputs are global THD-ordered arrays [T, heads, dim]; they are upcast exactly to
float64.  Query rows are processed in blocks only to bound memory.

MLA keys may also be given in compact form (a per-head part and one rope key per
token shared by every head); attention_fwd_mla expands them and applies the same
definition.
"""
from __future__ import annotations

import numpy as np

from .partition import doc_of_token

ROW_BLOCK = 512


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _kv_head(h: int, hq: int, hkv: int) -> int:
    return h // (hq // hkv)


def attention_fwd(q, k, v, cu_seqlens, scale: float):
    """O [T, Hq, Dv] and lse [Hq, T] in global token order."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hq, _ = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    out = np.zeros((T, hq, dv))
    lse = np.zeros((hq, T))
    for d in range(cu.size - 1):
        s, e = int(cu[d]), int(cu[d + 1])
        for h in range(hq):
            g = _kv_head(h, hq, hkv)
            for i0 in range(s, e, ROW_BLOCK):
                i1 = min(e, i0 + ROW_BLOCK)
                S = scale * (q[i0:i1, h] @ k[s:i1, g].T)          # keys s .. i1-1
                rows = np.arange(i0, i1)[:, None]
                cols = np.arange(s, i1)[None, :]
                S = np.where(cols <= rows, S, -np.inf)
                mx = S.max(axis=1, keepdims=True)
                P = np.exp(S - mx)
                l = P.sum(axis=1, keepdims=True)
                out[i0:i1, h] = (P @ v[s:i1, g]) / l
                lse[h, i0:i1] = (mx + np.log(l))[:, 0]
    return out, lse


def attention_bwd(q, k, v, o, lse, do, cu_seqlens, scale: float):
    """dQ [T,Hq,Dqk], dK [T,Hkv,Dqk], dV [T,Hkv,Dv] given the forward's O and lse."""
    q, k, v, o, do = _f64(q), _f64(k), _f64(v), _f64(o), _f64(do)
    lse = _f64(lse)
    T, hq, _ = q.shape
    hkv = k.shape[1]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    delta = np.sum(do * o, axis=2)                                  # [T, Hq]
    for d in range(cu.size - 1):
        s, e = int(cu[d]), int(cu[d + 1])
        for h in range(hq):
            g = _kv_head(h, hq, hkv)
            for i0 in range(s, e, ROW_BLOCK):
                i1 = min(e, i0 + ROW_BLOCK)
                S = scale * (q[i0:i1, h] @ k[s:i1, g].T)
                rows = np.arange(i0, i1)[:, None]
                cols = np.arange(s, i1)[None, :]
                P = np.where(cols <= rows, np.exp(S - lse[h, i0:i1, None]), 0.0)
                dv[s:i1, g] += P.T @ do[i0:i1, h]
                dP = do[i0:i1, h] @ v[s:i1, g].T
                dS = P * (dP - delta[i0:i1, h, None])
                dq[i0:i1, h] = scale * (dS @ k[s:i1, g])
                dk[s:i1, g] += scale * (dS.T @ q[i0:i1, h])
    return dq, dk, dv


# ----------------------------------------------------------------------------
# Sampled forms: the same definition evaluated only where asked, so that outputs
# of the full-size workloads can be checked one row at a time.
# ----------------------------------------------------------------------------

def expand_mla_keys(k_nope, k_rope):
    """Expanded key of multi-head latent attention from its compact form: every
    key/value head g of token t gets k[t, g] = concat(k_nope[t, g], k_rope[t]), the
    rope key being one per token and shared by every head.  (The page serves MLA in
    expanded form; this is the reading of what the compact form stands for.)"""
    k_nope = _f64(k_nope)
    k_rope = _f64(k_rope)
    T, hkv, _ = k_nope.shape
    rope = np.broadcast_to(k_rope.reshape(T, 1, -1), (T, hkv, k_rope.shape[-1]))
    return np.concatenate([k_nope, rope], axis=2)


def attention_fwd_mla(q, k_nope, k_rope, v, cu_seqlens, scale: float):
    """Forward attention with MLA keys in compact form: the definition is the expanded
    one, so this is attention_fwd on expand_mla_keys(k_nope, k_rope)."""
    return attention_fwd(q, expand_mla_keys(k_nope, k_rope), v, cu_seqlens, scale)


def _row_forward(qrow, kdoc, vdoc, scale):
    """One query row against its visible keys: (o, lse, p)."""
    s = scale * (kdoc @ qrow)
    mx = s.max()
    p = np.exp(s - mx)
    l = p.sum()
    return (p @ vdoc) / l, mx + np.log(l), p / l


def attention_fwd_rows(q, k, v, cu_seqlens, scale, rows, heads):
    """O[len(rows), len(heads), Dv] and lse[len(rows), len(heads)] for global rows."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    doc = doc_of_token(cu)
    hq, hkv = q.shape[1], k.shape[1]
    O = np.zeros((len(rows), len(heads), v.shape[2]))
    L = np.zeros((len(rows), len(heads)))
    for a, i in enumerate(rows):
        s = int(cu[doc[i]])
        for b, h in enumerate(heads):
            g = _kv_head(h, hq, hkv)
            O[a, b], L[a, b], _ = _row_forward(_f64(q[i, h]), _f64(k[s:i + 1, g]),
                                               _f64(v[s:i + 1, g]), scale)
    return O, L


def attention_bwd_rows(q, k, v, do, cu_seqlens, scale, rows, heads):
    """dQ[len(rows), len(heads), Dqk] at global query rows (row-local computation)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    doc = doc_of_token(cu)
    hq, hkv = q.shape[1], k.shape[1]
    out = np.zeros((len(rows), len(heads), q.shape[2]))
    for a, i in enumerate(rows):
        s = int(cu[doc[i]])
        for b, h in enumerate(heads):
            g = _kv_head(h, hq, hkv)
            kd, vd = _f64(k[s:i + 1, g]), _f64(v[s:i + 1, g])
            o, _, p = _row_forward(_f64(q[i, h]), kd, vd, scale)
            dorow = _f64(do[i, h])
            delta = dorow @ o
            ds = p * (vd @ dorow - delta)
            out[a, b] = scale * (ds @ kd)
    return out


def attention_bwd_keys(q, k, v, do, cu_seqlens, scale, keys, kv_heads):
    """dK[len(keys), len(kv_heads), Dqk], dV[len(keys), len(kv_heads), Dv] at global
    key rows.  Every query row of the document at or after the key contributes, so
    this is cheap for keys near the end of their document."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    doc = doc_of_token(cu)
    hq, hkv = q.shape[1], k.shape[1]
    group = hq // hkv
    dK = np.zeros((len(keys), len(kv_heads), q.shape[2]))
    dV = np.zeros((len(keys), len(kv_heads), v.shape[2]))
    for a, j in enumerate(keys):
        s, e = int(cu[doc[j]]), int(cu[doc[j] + 1])
        for b, g in enumerate(kv_heads):
            kj, vj = _f64(k[j, g]), _f64(v[j, g])
            for h in range(g * group, (g + 1) * group):
                for i in range(j, e):
                    kd, vd = _f64(k[s:i + 1, g]), _f64(v[s:i + 1, g])
                    qrow, dorow = _f64(q[i, h]), _f64(do[i, h])
                    o, _, p = _row_forward(qrow, kd, vd, scale)
                    delta = dorow @ o
                    pij = p[j - s]
                    dV[a, b] += pij * dorow
                    dK[a, b] += scale * pij * (dorow @ vj - delta) * qrow
    return dK, dV


def attention_bwd_key_blocks(q, k, v, do, cu_seqlens, scale, blocks, kv_heads):
    """dK and dV of contiguous key blocks of one document, by a blocked pass over the
    query rows that can see them.  ``blocks`` is a list of (first key, number of keys),
    all inside one document; returns lists dK[b] [n, len(kv_heads), Dqk] and
    dV[b] [n, len(kv_heads), Dv].

    The same definition as attention_bwd, evaluated where asked: for each query head h
    of a key/value head's group and each block of query rows i (from the first key of
    the earliest block to the document's end), the full row of scores against keys
    s .. i gives lse_i, P_i and O_i = P_i V, hence Delta_i = dO_i . O_i; then, for the
    asked keys j only, dP_ij = dO_i . V_j, dS_ij = P_ij (dP_ij - Delta_i),
    dV_j += P_ij dO_i and dK_j += scale dS_ij Q_i.  Written with float64 torch CPU
    operations (multi-threaded), so that a 65536-token document takes seconds per
    head rather than minutes."""
    import torch

    def t64(x):
        return x.detach().to("cpu", torch.float64) if hasattr(x, "detach") else torch.from_numpy(_f64(x))

    cu = np.asarray(cu_seqlens, dtype=np.int64)
    doc = doc_of_token(cu)
    hq, hkv = q.shape[1], k.shape[1]
    group = hq // hkv
    d = int(doc[blocks[0][0]])
    s, e = int(cu[d]), int(cu[d + 1])
    for j0, n in blocks:
        assert n > 0 and doc[j0] == d and doc[j0 + n - 1] == d, "blocks lie inside one document"
    first = min(j0 for j0, _ in blocks)
    dK = [np.zeros((n, len(kv_heads), q.shape[2])) for _, n in blocks]
    dV = [np.zeros((n, len(kv_heads), v.shape[2])) for _, n in blocks]
    for b, g in enumerate(kv_heads):
        kd, vd = t64(k[s:e, g]), t64(v[s:e, g])
        for h in range(g * group, (g + 1) * group):
            qh, doh = t64(q[first:e, h]), t64(do[first:e, h])
            for i0 in range(first, e, ROW_BLOCK):
                i1 = min(e, i0 + ROW_BLOCK)
                qb, dob = qh[i0 - first:i1 - first], doh[i0 - first:i1 - first]
                S = qb @ kd[:i1 - s].T                                 # keys s .. i1-1
                S.mul_(scale)
                # the causal mask: key j > row i is invisible (only keys >= i0 can be)
                rows = torch.arange(i0, i1)[:, None]
                cols = torch.arange(i0, i1)[None, :]
                S[:, i0 - s:].masked_fill_(cols > rows, float("-inf"))
                mx = S.amax(dim=1, keepdim=True)
                S.sub_(mx).exp_()                                      # E = exp(S - max)
                l = S.sum(dim=1)                                       # P = E / l = exp(S - lse)
                delta = (dob * (S @ vd[:i1 - s])).sum(dim=1) / l       # dO_i . O_i, O = P V
                for a, (j0, n) in enumerate(blocks):
                    j1 = min(j0 + n, i1)
                    if j1 <= j0:
                        continue
                    Pb = S[:, j0 - s:j1 - s] / l[:, None]
                    dPb = dob @ vd[j0 - s:j1 - s].T
                    dSb = Pb * (dPb - delta[:, None])
                    dV[a][:j1 - j0, b] += (Pb.T @ dob).numpy()
                    dK[a][:j1 - j0, b] += scale * (dSb.T @ qb).numpy()
    return dK, dV


# ----------------------------------------------------------------------------
# Brute-force forms used only to pin the definition above on tiny inputs.
# ----------------------------------------------------------------------------

def bruteforce_fwd(q, k, v, cu_seqlens, scale):
    """Full T x T attention with an explicit mask built from document ids."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hq, _ = q.shape
    hkv = k.shape[1]
    doc = doc_of_token(cu_seqlens)
    idx = np.arange(T)
    mask = (doc[:, None] == doc[None, :]) & (idx[None, :] <= idx[:, None])
    out = np.zeros((T, hq, v.shape[2]))
    lse = np.zeros((hq, T))
    for h in range(hq):
        g = _kv_head(h, hq, hkv)
        S = scale * q[:, h] @ k[:, g].T
        S[~mask] = -np.inf
        mx = S.max(axis=1, keepdims=True)
        E = np.exp(S - mx)
        out[:, h] = E @ v[:, g] / E.sum(axis=1, keepdims=True)
        lse[h] = np.log(E.sum(axis=1)) + mx[:, 0]
    return out, lse


def cp_rank_fwd(q, k, v, cu_seqlens, scale, q_idx, cp):
    """The context-parallel formulation: every virtual rank attends its local queries
    (rank-major rows r*Tl .. (r+1)*Tl-1) to the all-gathered rank-major K/V, with the
    mask taken from global positions and document ids.  Returns rank-major O and
    lse [Hq, T]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hq, _ = q.shape
    hkv = k.shape[1]
    Tl = T // cp
    doc = doc_of_token(cu_seqlens)
    q_idx = np.asarray(q_idx, dtype=np.int64)
    k_rm, v_rm = k[q_idx], v[q_idx]                        # the all-gathered buffer
    kpos, kdoc = q_idx, doc[q_idx]
    out = np.zeros((T, hq, v.shape[2]))
    lse = np.zeros((hq, T))
    for r in range(cp):
        rows = np.arange(r * Tl, (r + 1) * Tl)
        qpos = q_idx[rows]
        qdoc = doc[qpos]
        mask = (qdoc[:, None] == kdoc[None, :]) & (kpos[None, :] <= qpos[:, None])
        for h in range(hq):
            g = _kv_head(h, hq, hkv)
            S = scale * q[qpos, h] @ k_rm[:, g].T
            S[~mask] = -np.inf
            mx = S.max(axis=1, keepdims=True)
            E = np.exp(S - mx)
            out[rows, h] = E @ v_rm[:, g] / E.sum(axis=1, keepdims=True)
            lse[h, rows] = np.log(E.sum(axis=1)) + mx[:, 0]
    return out, lse

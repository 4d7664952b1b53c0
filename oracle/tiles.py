"""Oracle: the cached per-tile metadata table, built by brute force.  TEST INFRASTRUCTURE ONLY.

Source: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance",
section "What this PR does / why we need it?": a THD attention path with direct
rank-major K/V indexing and a single fused-attention call, with metadata caching
to avoid repeated calculation.  The page does not print the table's format; the
format below is this library's reading and is the bit-exact contract between the
library's planner and this oracle.

Geometry (BM = BN = 128):
  * A *segment* is the contiguous run of rank-major rows that one rank holds for
    one document (its two chunks).  Q-tiles and key tiles are both the 128-row
    slices of every segment, enumerated rank-major: rank, then document, then
    slice.  The last slice of a segment may be short (m < 128 rows).
  * For a q-tile of document d, its k-tile *entries* walk the segments of d on
    every rank r' = 0..cp-1 (direct rank-major indexing: the gathered buffer is
    read in place).  In each segment the keys visible to at least one row of the
    q-tile form a prefix of v rows; that prefix is cut into ceil(v/128) entries
    starting at the segment's 128-row slices.  An entry whose keys are visible to
    every row of the q-tile is UNMASKED (2), otherwise PARTIAL (1).  Keys no row
    can see are never listed (FULLY MASKED tiles are skipped).
  * Positions are global token indices.  A run of rows holds at most one jump in
    position (the seam between a rank's two chunks), encoded as
    pos(t) = pos0 + t + (t >= brk ? jump : 0), brk = n and jump = 0 when the run
    has no seam.

Record layouts (int32):
  qtile[12] = r, d, row0 (rank-major), m, qpos0, qbrk, qjump, qpos_max,
              nk, entry_off, doc_start, doc_end
  entry[8]  = k0 (rank-major), nvalid, kpos0, kbrk, kjump, cls, ktile, key_rank
  ktiles are the q-tiles themselves (same row slices); the backward transpose is
  kt_off[n_tiles+1] / kt_list[n_entries][2] = (qtile, entry), each key tile's list
  in descending order of the q-tile's qpos_max (ties by q-tile index).
  lpt: q-tiles by descending nk (ties by index); kt_lpt: key tiles by descending
  number of listed q-tiles (ties by index); kt_seg[j+1] - kt_seg[j]: the number of key
  tiles whose list has more than j*KSEG entries (segments of KSEG = 32 entries are
  the backward's work items), kt_seg[0] = 0.

Everything is derived from the explicit partition (``partition.partition``) by
enumerating every (query row, key row) pair of a tile; nothing uses the closed-form
offsets of the library's planner.
"""
from __future__ import annotations

import numpy as np

from .partition import partition, doc_of_token, validate

BM = 128
BN = 128
KSEG = 32           # key-tile list entries per backward work item
PARTIAL = 1
UNMASKED = 2
QT_FIELDS = 12
EN_FIELDS = 8


def _encode_run(pos: np.ndarray):
    """(pos0, brk, jump) of a run of increasing positions with at most one seam."""
    n = pos.size
    steps = np.diff(pos)
    seams = np.nonzero(steps != 1)[0]
    assert seams.size <= 1, "a tile run holds at most one seam"
    if seams.size == 0:
        return int(pos[0]), n, 0
    b = int(seams[0]) + 1
    return int(pos[0]), b, int(pos[b] - pos[b - 1] - 1)


def _segments(q_idx: np.ndarray, doc: np.ndarray, cp: int, n_docs: int):
    """seg[r][d] = (first rank-major row, length), found by scanning the partition."""
    T = q_idx.size
    Tl = T // cp
    seg = [[None] * n_docs for _ in range(cp)]
    for r in range(cp):
        docs_local = doc[q_idx[r * Tl:(r + 1) * Tl]]
        for d in range(n_docs):
            rows = np.nonzero(docs_local == d)[0]
            assert rows.size > 0 and rows[-1] - rows[0] + 1 == rows.size, "segment is contiguous"
            seg[r][d] = (r * Tl + int(rows[0]), int(rows.size))
    return seg


def tile_plan(cu_seqlens, cp: int) -> dict:
    cu = validate(cu_seqlens, cp)
    n_docs = cu.size - 1
    q_idx, rm_of_global = partition(cu, cp)
    doc = doc_of_token(cu)
    seg = _segments(q_idx, doc, cp, n_docs)

    # q-tiles (== key tiles): rank, then doc, then 128-row slice
    tiles = []
    tile_index = {}
    for r in range(cp):
        for d in range(n_docs):
            row_start, n = seg[r][d]
            for i, off in enumerate(range(0, n, BM)):
                tile_index[(r, d, i)] = len(tiles)
                tiles.append((r, d, row_start + off, min(BM, n - off)))

    qtiles = np.zeros((len(tiles), QT_FIELDS), dtype=np.int32)
    entries = []
    for ti, (r, d, row0, m) in enumerate(tiles):
        qpos = q_idx[row0:row0 + m].astype(np.int64)
        qpos0, qbrk, qjump = _encode_run(qpos)
        first_entry = len(entries)
        for rk in range(cp):
            krow_start, n = seg[rk][d]
            kpos = q_idx[krow_start:krow_start + n].astype(np.int64)
            assert np.all(doc[kpos] == d) and np.all(doc[qpos] == d)
            vis = kpos[None, :] <= qpos[:, None]          # every (query row, key row) pair
            seen = vis.any(axis=0)
            v = int(seen.sum())
            assert seen[:v].all() and not seen[v:].any(), "visible keys form a prefix"
            for j, u0 in enumerate(range(0, v, BN)):
                nvalid = min(BN, v - u0)
                kpos0, kbrk, kjump = _encode_run(kpos[u0:u0 + nvalid])
                cls = UNMASKED if vis[:, u0:u0 + nvalid].all() else PARTIAL
                entries.append((krow_start + u0, nvalid, kpos0, kbrk, kjump, cls,
                                tile_index[(rk, d, j)], rk))
        qtiles[ti] = (r, d, row0, m, qpos0, qbrk, qjump, int(qpos[-1]),
                      len(entries) - first_entry, first_entry, int(cu[d]), int(cu[d + 1]))
    entries = np.array(entries, dtype=np.int32).reshape(-1, EN_FIELDS)

    n_tiles = len(tiles)
    lpt = np.array(sorted(range(n_tiles), key=lambda t: (-int(qtiles[t, 8]), t)), dtype=np.int32)

    kt_off, kt_list, kt_lpt, kt_seg = _transpose(qtiles, entries)

    fqtiles, fentries, flpt = _forward_tables(cu, cp, qtiles, entries)
    fkt_off, fkt_list, fkt_lpt, fkt_seg = _transpose(fqtiles, fentries)
    return dict(T=int(cu[-1]), cp=int(cp), Tl=int(cu[-1]) // cp, n_docs=n_docs,
                q_idx=q_idx, rm_of_global=rm_of_global, qtiles=qtiles, entries=entries,
                lpt=lpt, kt_off=kt_off, kt_list=kt_list, kt_lpt=kt_lpt, kt_seg=kt_seg,
                fqtiles=fqtiles, fentries=fentries, flpt=flpt,
                fkt_off=fkt_off, fkt_list=fkt_list, fkt_lpt=fkt_lpt, fkt_seg=fkt_seg)


def _transpose(qtiles, entries):
    """Per key tile (entry field 6 names it, an index into the same tile table) the
    list of (q-tile, entry) pairs, by descending last query position, then q-tile index;
    key tiles by descending list length; and the running count of backward work items
    per list segment (segment j of every key tile whose list has more than j*KSEG
    entries)."""
    n_tiles = qtiles.shape[0]
    lists = [[] for _ in range(n_tiles)]
    for qt in range(n_tiles):
        e0, nk = int(qtiles[qt, 9]), int(qtiles[qt, 8])
        for e in range(e0, e0 + nk):
            lists[int(entries[e, 6])].append((qt, e))
    kt_off = np.zeros(n_tiles + 1, dtype=np.int32)
    kt_off[1:] = np.cumsum([len(x) for x in lists])
    kt_list = np.array([p for x in lists for p in sorted(x, key=lambda pr: (-int(qtiles[pr[0], 7]), pr[0]))],
                       dtype=np.int32).reshape(-1, 2)
    kt_lpt = np.array(sorted(range(n_tiles), key=lambda t: (-len(lists[t]), t)), dtype=np.int32)
    n_seg = -(-max((len(x) for x in lists), default=0) // KSEG)
    kt_seg = np.zeros(n_seg + 1, dtype=np.int32)
    for j in range(n_seg):
        kt_seg[j + 1] = kt_seg[j] + sum(1 for x in lists if len(x) > j * KSEG)
    return kt_off, kt_list, kt_lpt, kt_seg


def _forward_tables(cu, cp, qtiles, entries):
    """The forward's tiles.  A document whose chunks are shorter than a tile
    (L / (2 cp) < 128) is tiled in position order: query tile u holds positions
    s + 128u .. (up to 128), and every key tile v (positions s + 128v ..) holding a key
    that some of its queries can see is listed, found by enumerating the (query, key)
    pairs; row0 / k0 / r / key_rank are -1 for these records (the rows are found
    through rm_of_global).  Other documents keep their rank-major tiles, in the order of
    the main table, first.  An entry's key tile (field 6) is the index, in these
    tables, of the tile that holds its keys."""
    n_docs = cu.size - 1
    short = {d for d in range(n_docs) if (int(cu[d + 1]) - int(cu[d])) // (2 * cp) < BM}
    kept = [t for t in range(qtiles.shape[0]) if int(qtiles[t, 1]) not in short]
    f_of_tile = {t: i for i, t in enumerate(kept)}      # forward index of a rank-major tile
    fq, fe = [], []
    for t in kept:
        rec = qtiles[t].copy()
        e0, nk = int(rec[9]), int(rec[8])
        rec[9] = len(fe)
        fq.append(rec)
        for en in entries[e0:e0 + nk].tolist():
            en[6] = f_of_tile[en[6]]                     # key tile: its forward index
            fe.append(en)
    for d in sorted(short):
        s, e = int(cu[d]), int(cu[d + 1])
        first_tile = len(fq)                             # position tile 0 of d
        for p0 in range(s, e, BM):
            qpos = np.arange(p0, min(p0 + BM, e))
            first = len(fe)
            for k0 in range(s, e, BN):
                kpos = np.arange(k0, min(k0 + BN, e))
                vis = kpos[None, :] <= qpos[:, None]
                seen = vis.any(axis=0)
                nv = int(seen.sum())
                if nv == 0:
                    continue
                assert seen[:nv].all(), "visible keys of a position tile form a prefix"
                cls = UNMASKED if vis[:, :nv].all() else PARTIAL
                fe.append([-1, nv, int(kpos[0]), nv, 0, cls, first_tile + (k0 - s) // BN, -1])
            fq.append(np.array([-1, d, -1, qpos.size, int(qpos[0]), qpos.size, 0, int(qpos[-1]),
                                len(fe) - first, first, s, e], dtype=np.int32))
    fqtiles = np.array(fq, dtype=np.int32).reshape(-1, QT_FIELDS)
    fentries = np.array(fe, dtype=np.int32).reshape(-1, EN_FIELDS)
    flpt = np.array(sorted(range(fqtiles.shape[0]), key=lambda t: (-int(fqtiles[t, 8]), t)), dtype=np.int32)
    return fqtiles, fentries, flpt


def decode_run(pos0: int, brk: int, jump: int, n: int) -> np.ndarray:
    t = np.arange(n, dtype=np.int64)
    return pos0 + t + np.where(t >= brk, jump, 0)


def visible_pairs_of_entry(plan: dict, qt: int, e: int) -> int:
    """Brute-force count of visible (query, key) pairs covered by one entry."""
    q = plan["qtiles"][qt]
    en = plan["entries"][e]
    qpos = plan["q_idx"][q[2]:q[2] + q[3]].astype(np.int64)
    kpos = plan["q_idx"][en[0]:en[0] + en[1]].astype(np.int64)
    return int(np.sum(kpos[None, :] <= qpos[:, None]))

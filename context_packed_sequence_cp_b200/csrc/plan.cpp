// Host planner of libthdcp: validation, the symmetric two-chunk partition and the
// cached per-tile metadata, built in closed form.
//
// Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance".
// Section "Does this PR introduce any user-facing change?" fixes the input
// contract (THD packed documents, causal attention with EOD reset, every length a
// multiple of 2 * cp); section "What this PR does / why we need it?" asks for an
// EOD-aware symmetric partition, direct rank-major K/V indexing and metadata that
// is computed once and cached.
//
// Partition: document d (start s, length L, chunk c = L / 2cp) is cut into 2cp
// chunks; rank r keeps chunk r then chunk 2cp-1-r.  Rank r's rows of document d
// form one contiguous "segment" of 2c rank-major rows starting at
// r*Tl + s/cp (documents before d contribute 2c' = L'/cp rows each).  Row u of
// that segment holds global position
//     u <  c:  s + r c + u
//     u >= c:  s + (2cp-1-r) c + (u - c).
// Positions grow with u, so the keys of a segment that a query at position P can
// see are a prefix; its length is the count of chunk-r keys <= P plus the count of
// mirror-chunk keys <= P.
#include "plan.h"

#include <algorithm>
#include <limits>
#include <vector>

namespace {

constexpr int BM = THD_BM;
constexpr int BN = THD_BN;

struct Layout {
    int32_t cp;
    int64_t Tl;
    const std::vector<int64_t>& s;
    const std::vector<int64_t>& L;
    int64_t chunk(int d) const { return L[d] / (2 * cp); }
    int64_t seg_row(int r, int d) const { return (int64_t)r * Tl + s[d] / cp; }
    int64_t pos(int r, int d, int64_t u) const {
        const int64_t c = chunk(d);
        return u < c ? s[d] + (int64_t)r * c + u : s[d] + (int64_t)(2 * cp - 1 - r) * c + (u - c);
    }
    // (pos0, brk, jump) of segment rows u0 .. u0+n-1: pos(t) = pos0 + t + (t >= brk ? jump : 0)
    void encode(int r, int d, int64_t u0, int64_t n, int32_t* out) const {
        const int64_t c = chunk(d);
        out[0] = (int32_t)pos(r, d, u0);
        out[1] = (int32_t)n;
        out[2] = 0;
        const int64_t jump = (int64_t)(2 * cp - 2 - 2 * r) * c;  // gap between chunk r and its mirror
        if (u0 < c && u0 + n > c && jump != 0) {
            out[1] = (int32_t)(c - u0);
            out[2] = (int32_t)jump;
        }
    }
    int64_t visible_prefix(int rk, int d, int64_t pmax) const {
        const int64_t c = chunk(d);
        const int64_t a0 = s[d] + (int64_t)rk * c;
        const int64_t b0 = s[d] + (int64_t)(2 * cp - 1 - rk) * c;
        const int64_t na = std::clamp<int64_t>(pmax - a0 + 1, 0, c);
        const int64_t nb = std::clamp<int64_t>(pmax - b0 + 1, 0, c);
        return na + nb;
    }
};

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Key-tile transpose of a tile table (entries name their key tile in field 6, an index
// into the same tile table): per key tile the (query tile, entry) pairs, in descending
// order of the query tile's last position, ties (which cannot occur within one
// document) by tile index.  A key tile sees exactly the query tiles of its document
// whose last position is at or past its first key, so every list is a prefix of one
// per-document order, and key tiles walked at the same time read the same query tiles.
// Walking the query tiles once in that order makes the counting-sort fill emit every
// list already sorted.  Also the longest-first order of key tiles and the work items
// per list segment (segment j of every key tile whose list reaches it: the first n_j
// key tiles of the longest-first order).
void build_transpose(const std::vector<int32_t>& qtiles, const std::vector<int32_t>& entries,
                     std::vector<int32_t>& kt_off, std::vector<int32_t>& kt_list, std::vector<int32_t>& kt_lpt,
                     std::vector<int32_t>& kt_seg) {
    const int64_t n_tiles = (int64_t)qtiles.size() / THD_QTILE_FIELDS;
    const int64_t ne = (int64_t)entries.size() / THD_ENTRY_FIELDS;
    kt_off.assign(n_tiles + 1, 0);
    for (int64_t e = 0; e < ne; ++e) kt_off[entries[(size_t)e * THD_ENTRY_FIELDS + 6] + 1]++;
    for (int64_t t = 0; t < n_tiles; ++t) kt_off[t + 1] += kt_off[t];
    std::vector<int32_t> by_last(n_tiles);
    for (int64_t t = 0; t < n_tiles; ++t) by_last[t] = (int32_t)t;
    std::sort(by_last.begin(), by_last.end(), [&](int32_t a, int32_t b) {
        const int32_t pa = qtiles[(size_t)a * THD_QTILE_FIELDS + 7];
        const int32_t pb = qtiles[(size_t)b * THD_QTILE_FIELDS + 7];
        return pa != pb ? pa > pb : a < b;
    });
    std::vector<int32_t> fill(kt_off.begin(), kt_off.end() - 1);
    kt_list.assign((size_t)ne * 2, 0);
    for (const int32_t qt : by_last) {
        const int32_t* q = &qtiles[(size_t)qt * THD_QTILE_FIELDS];
        for (int64_t e = q[9]; e < (int64_t)q[9] + q[8]; ++e) {
            const int32_t kt = entries[(size_t)e * THD_ENTRY_FIELDS + 6];
            const int32_t at = fill[kt]++;
            kt_list[(size_t)at * 2] = qt;
            kt_list[(size_t)at * 2 + 1] = (int32_t)e;
        }
    }
    kt_lpt.resize(n_tiles);
    for (int64_t t = 0; t < n_tiles; ++t) kt_lpt[t] = (int32_t)t;
    std::stable_sort(kt_lpt.begin(), kt_lpt.end(),
                     [&](int32_t a, int32_t b) { return kt_off[a + 1] - kt_off[a] > kt_off[b + 1] - kt_off[b]; });
    const int64_t max_len = n_tiles ? (int64_t)kt_off[kt_lpt[0] + 1] - kt_off[kt_lpt[0]] : 0;
    const int64_t n_seg = ceil_div(max_len, THD_KSEG);
    kt_seg.assign(n_seg + 1, 0);
    int64_t reach = n_tiles;  // key tiles whose list is longer than j * THD_KSEG
    for (int64_t j = 0; j < n_seg; ++j) {
        while (reach > 0 && (int64_t)kt_off[kt_lpt[reach - 1] + 1] - kt_off[kt_lpt[reach - 1]] <= j * THD_KSEG) --reach;
        kt_seg[j + 1] = (int32_t)(kt_seg[j] + reach);
    }
}

}  // namespace

int thd_build_plan(const int32_t* cu, int32_t n_docs, int32_t cp, thd_cp_plan_s* p) {
    if (!cu || !p || n_docs < 1 || cp < 1) return THD_ERR_INVALID_ARG;
    if (cu[0] != 0) return THD_ERR_BAD_SEQLENS;
    std::vector<int64_t> s(n_docs), L(n_docs);
    for (int d = 0; d < n_docs; ++d) {
        s[d] = cu[d];
        L[d] = (int64_t)cu[d + 1] - (int64_t)cu[d];
        if (L[d] <= 0) return THD_ERR_BAD_SEQLENS;
    }
    for (int d = 0; d < n_docs; ++d)
        if (L[d] % (2 * (int64_t)cp) != 0) return THD_ERR_NOT_DIVISIBLE;
    const int64_t T = cu[n_docs];
    const int64_t Tl = T / cp;
    const Layout lay{cp, Tl, s, L};

    try {
        p->T = T;
        p->Tl = Tl;
        p->cp = cp;
        p->n_docs = n_docs;
        p->doc_start = s;
        p->doc_len = L;
        p->causal_pairs = 0;
        for (int d = 0; d < n_docs; ++d) p->causal_pairs += L[d] * (L[d] + 1) / 2;

        // ---- partition ------------------------------------------------------
        p->q_idx.assign(T, 0);
        p->rm_of_global.assign(T, 0);
        for (int r = 0; r < cp; ++r)
            for (int d = 0; d < n_docs; ++d) {
                const int64_t base = lay.seg_row(r, d), n = 2 * lay.chunk(d);
                for (int64_t u = 0; u < n; ++u) {
                    const int64_t g = lay.pos(r, d, u);
                    p->q_idx[base + u] = (int32_t)g;
                    p->rm_of_global[g] = (int32_t)(base + u);
                }
            }

        // ---- tiles: the 128-row slices of every (rank, document) segment ------
        std::vector<int64_t> tile_base((size_t)cp * n_docs + 1, 0);
        for (int r = 0; r < cp; ++r)
            for (int d = 0; d < n_docs; ++d) {
                const size_t k = (size_t)r * n_docs + d;
                tile_base[k + 1] = tile_base[k] + ceil_div(2 * lay.chunk(d), BM);
            }
        const int64_t n_tiles = tile_base.back();
        if (n_tiles > std::numeric_limits<int32_t>::max()) return THD_ERR_INVALID_ARG;
        p->qtiles.assign((size_t)n_tiles * THD_QTILE_FIELDS, 0);

        // Entry count first, so that the entry table is sized once and filled in place.
        int64_t n_entries = 0;
        for (int r = 0; r < cp; ++r)
            for (int d = 0; d < n_docs; ++d) {
                const int64_t nseg = 2 * lay.chunk(d);
                for (int64_t u0 = 0; u0 < nseg; u0 += BM) {
                    const int64_t qmax = lay.pos(r, d, std::min<int64_t>(u0 + BM, nseg) - 1);
                    for (int rk = 0; rk < cp; ++rk) n_entries += ceil_div(lay.visible_prefix(rk, d, qmax), BN);
                }
            }
        if (n_entries > std::numeric_limits<int32_t>::max() / 2) return THD_ERR_INVALID_ARG;
        p->entries.assign((size_t)n_entries * THD_ENTRY_FIELDS, 0);
        int64_t ne_fill = 0;

        for (int r = 0; r < cp; ++r)
            for (int d = 0; d < n_docs; ++d) {
                const int64_t nseg = 2 * lay.chunk(d);
                for (int64_t i = 0; i * BM < nseg; ++i) {
                    const int64_t ti = tile_base[(size_t)r * n_docs + d] + i;
                    const int64_t u0 = i * BM, m = std::min<int64_t>(BM, nseg - u0);
                    const int64_t qmin = lay.pos(r, d, u0), qmax = lay.pos(r, d, u0 + m - 1);
                    int32_t* q = &p->qtiles[(size_t)ti * THD_QTILE_FIELDS];
                    const int64_t first = ne_fill;
                    for (int rk = 0; rk < cp; ++rk) {
                        const int64_t v = lay.visible_prefix(rk, d, qmax);
                        for (int64_t j = 0; j * BN < v; ++j) {
                            const int64_t k0u = j * BN, nv = std::min<int64_t>(BN, v - k0u);
                            int32_t* e = &p->entries[(size_t)ne_fill++ * THD_ENTRY_FIELDS];
                            e[0] = (int32_t)(lay.seg_row(rk, d) + k0u);
                            e[1] = (int32_t)nv;
                            int32_t enc[3];
                            lay.encode(rk, d, k0u, nv, enc);
                            e[2] = enc[0];
                            e[3] = enc[1];
                            e[4] = enc[2];
                            e[5] = lay.pos(rk, d, k0u + nv - 1) <= qmin ? THD_CLS_UNMASKED : THD_CLS_PARTIAL;
                            e[6] = (int32_t)(tile_base[(size_t)rk * n_docs + d] + j);
                            e[7] = rk;
                        }
                    }
                    int32_t enc[3];
                    lay.encode(r, d, u0, m, enc);
                    q[0] = r;
                    q[1] = d;
                    q[2] = (int32_t)(lay.seg_row(r, d) + u0);
                    q[3] = (int32_t)m;
                    q[4] = enc[0];
                    q[5] = enc[1];
                    q[6] = enc[2];
                    q[7] = (int32_t)qmax;
                    q[8] = (int32_t)(ne_fill - first);
                    q[9] = (int32_t)first;
                    q[10] = (int32_t)s[d];
                    q[11] = (int32_t)(s[d] + L[d]);
                }
            }

        // ---- longest-first order of query tiles ------------------------------
        p->lpt.resize(n_tiles);
        for (int64_t t = 0; t < n_tiles; ++t) p->lpt[t] = (int32_t)t;
        std::stable_sort(p->lpt.begin(), p->lpt.end(), [&](int32_t a, int32_t b) {
            return p->qtiles[(size_t)a * THD_QTILE_FIELDS + 8] > p->qtiles[(size_t)b * THD_QTILE_FIELDS + 8];
        });

        // ---- key-tile transpose for the backward ----------------------------
        build_transpose(p->qtiles, p->entries, p->kt_off, p->kt_list, p->kt_lpt, p->kt_seg);

        // ---- forward tables -------------------------------------------------
        // A document whose chunks are shorter than a tile (c < BM) puts two or more
        // chunks, far apart in position, into every rank-major tile, so that most of
        // each tile pair is masked.  The forward tiles such a document in position
        // order instead: query tile u and key tile v are positions s + u*BM .. and
        // s + v*BM .. (read in place from the rank-major buffers through rm_of_global),
        // key tiles 0 .. u listed for query tile u, the last one the diagonal.  Rank-major
        // records are marked by row0 / k0 >= 0; position records carry -1 there.
        // An entry's key tile (field 6) is the forward tile that holds its keys.  Sizes are
        // counted first, so that both tables are allocated once and filled in place.
        std::vector<int32_t> f_of_tile(n_tiles, -1);  // forward index of a rank-major tile
        int64_t nf = 0, nfe = 0;
        for (int64_t t = 0; t < n_tiles; ++t) {
            const int32_t* q = &p->qtiles[(size_t)t * THD_QTILE_FIELDS];
            if (lay.chunk(q[1]) < BM) continue;
            f_of_tile[t] = (int32_t)nf++;
            nfe += q[8];
        }
        for (int d = 0; d < n_docs; ++d)
            if (lay.chunk(d) < BM) {
                const int64_t n = ceil_div(L[d], BM);
                nf += n;
                nfe += n * (n + 1) / 2;
            }
        if (nfe > std::numeric_limits<int32_t>::max() / 2) return THD_ERR_INVALID_ARG;
        p->fqtiles.assign((size_t)nf * THD_QTILE_FIELDS, 0);
        p->fentries.assign((size_t)nfe * THD_ENTRY_FIELDS, 0);
        int32_t* fq = p->fqtiles.data();
        int32_t* fe = p->fentries.data();
        int64_t ft = 0, fn = 0;  // tiles and entries written
        for (int64_t t = 0; t < n_tiles; ++t) {
            if (f_of_tile[t] < 0) continue;
            const int32_t* q = &p->qtiles[(size_t)t * THD_QTILE_FIELDS];
            std::copy(q, q + THD_QTILE_FIELDS, fq + ft * THD_QTILE_FIELDS);
            fq[ft * THD_QTILE_FIELDS + 9] = (int32_t)fn;
            ++ft;
            const int32_t* src = &p->entries[(size_t)q[9] * THD_ENTRY_FIELDS];
            for (int32_t k = 0; k < q[8]; ++k, ++fn) {
                int32_t* e = fe + fn * THD_ENTRY_FIELDS;
                std::copy(src + (size_t)k * THD_ENTRY_FIELDS, src + (size_t)(k + 1) * THD_ENTRY_FIELDS, e);
                e[6] = f_of_tile[e[6]];
            }
        }
        for (int d = 0; d < n_docs; ++d) {
            if (lay.chunk(d) >= BM) continue;
            const int64_t n = ceil_div(L[d], BM);
            const int32_t first_tile = (int32_t)ft;  // position tile 0 of d
            for (int64_t u = 0; u < n; ++u, ++ft) {
                const int64_t p0 = s[d] + u * BM, m = std::min<int64_t>(BM, L[d] - u * BM), qmax = p0 + m - 1;
                int32_t* q = fq + ft * THD_QTILE_FIELDS;
                q[0] = -1;
                q[1] = d;
                q[2] = -1;
                q[3] = (int32_t)m;
                q[4] = (int32_t)p0;
                q[5] = (int32_t)m;
                q[6] = 0;
                q[7] = (int32_t)qmax;
                q[8] = (int32_t)(u + 1);
                q[9] = (int32_t)fn;
                q[10] = (int32_t)s[d];
                q[11] = (int32_t)(s[d] + L[d]);
                for (int64_t v = 0; v <= u; ++v, ++fn) {
                    const int64_t kp0 = s[d] + v * BM, nv = std::min<int64_t>(BM, qmax - kp0 + 1);
                    int32_t* e = fe + fn * THD_ENTRY_FIELDS;
                    e[0] = -1;
                    e[1] = (int32_t)nv;
                    e[2] = (int32_t)kp0;
                    e[3] = (int32_t)nv;
                    e[4] = 0;
                    e[5] = kp0 + nv - 1 <= p0 ? THD_CLS_UNMASKED : THD_CLS_PARTIAL;
                    e[6] = first_tile + (int32_t)v;
                    e[7] = -1;
                }
            }
        }
        p->flpt.resize(nf);
        for (int64_t t = 0; t < nf; ++t) p->flpt[t] = (int32_t)t;
        std::stable_sort(p->flpt.begin(), p->flpt.end(), [&](int32_t a, int32_t b) {
            return p->fqtiles[(size_t)a * THD_QTILE_FIELDS + 8] > p->fqtiles[(size_t)b * THD_QTILE_FIELDS + 8];
        });
        // the fused backward walks the forward tables, key tile by key tile
        build_transpose(p->fqtiles, p->fentries, p->fkt_off, p->fkt_list, p->fkt_lpt, p->fkt_seg);
    } catch (const std::bad_alloc&) {
        return THD_ERR_ALLOC;
    }
    return THD_OK;
}

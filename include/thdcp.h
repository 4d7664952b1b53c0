/*
 * thdcp.h -- C ABI of libthdcp: packed-sequence (THD) causal attention with EOD
 * document-mask resets under load-balanced KV-all-gather context parallelism,
 * for NVIDIA B200 (sm_100a).  Every context-parallel rank is a virtual rank on one
 * GPU.
 *
 * Source of the method: MindSpeed pull request #3820, "feat: kvallgather cp thd
 * load balance".
 *   [WHAT]  section "What this PR does / why we need it?": load-balanced
 *           KV-all-gather context parallelism for the THD format, EOD-aware
 *           symmetric sequence partitioning, a THD attention path with direct
 *           rank-major K/V indexing and one fused attention call, metadata
 *           caching, and MHA, GQA and expanded MLA head layouts.
 *   [USER]  section "Does this PR introduce any user-facing change?": THD packed
 *           sequences, causal attention, EOD attention-mask reset, and every packed
 *           subsequence length divisible by 2 * context_parallel_size.
 *
 * Conventions shared by every entry point
 *   - Return value: THD_OK (0) or a negative THD_ERR_* code.  On an argument or
 *     layout error nothing is launched and no output is touched.  A launching entry
 *     point that finds a CUDA error already pending from earlier, unrelated work
 *     returns THD_ERR_CUDA without launching and leaves that error pending for its
 *     owner; THD_ERR_CUDA after a launch is this library's own.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Device entry points only enqueue work: they never synchronise and
 *     never allocate device memory, except thd_cp_plan_upload and
 *     thd_cp_plan_update (see there).
 *   - Device buffers are owned by the caller; the library reads and writes them
 *     only inside the enqueued kernels.  Device pointers must be 16-byte aligned
 *     (THD_ERR_MISALIGNED otherwise).
 *   - Tensors are dense row-major.  "Rank-major" row j is local row j % Tl of
 *     virtual rank j / Tl, Tl = T / cp: the order an all-gather of the rank-local
 *     shards produces.  Global order is the packed THD token order.
 *   - Thread safety: a plan may be used from several host threads once uploaded;
 *     creating, uploading and destroying it must not race with its use.
 */
#ifndef THDCP_H
#define THDCP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ------------------------------------------------------- */
#define THD_OK                 0
#define THD_ERR_INVALID_ARG   -1  /* null pointer, cp < 1, bad head/dim counts     */
#define THD_ERR_BAD_SEQLENS   -2  /* cu_seqlens[0] != 0, or a document of length 0  */
#define THD_ERR_NOT_DIVISIBLE -3  /* a document length is not a multiple of 2*cp    */
#define THD_ERR_MISALIGNED    -4  /* pointer or row size not a multiple of 16 bytes */
#define THD_ERR_NOT_UPLOADED  -5  /* device entry point called before plan_upload   */
#define THD_ERR_CUDA          -6  /* a CUDA runtime call or a launch failed         */
#define THD_ERR_UNSUPPORTED   -7  /* dtype / head-dim combination not built         */
#define THD_ERR_ALLOC         -8  /* host or device allocation failed               */
#define THD_ERR_TOO_LARGE     -9  /* result does not fit: hq * T beyond the fixed scratch of
                                      thd_cp_attn_bwd_noalloc, or a caller's array too small */

/* ---- element types ----------------------------------------------------- */
#define THD_DTYPE_BF16 0   /* bf16 inputs, fp32 accumulation, tcgen05 tensor cores */
#define THD_DTYPE_FP32 1   /* fp32 inputs and arithmetic (exact-precision path)    */

/* Tile geometry of the cached metadata (fixed; part of the plan's contract). */
#define THD_BM 128
#define THD_BN 128
#define THD_QTILE_FIELDS 12
#define THD_ENTRY_FIELDS 8
#define THD_CLS_PARTIAL  1
#define THD_CLS_UNMASKED 2
/* Query tiles per backward work item: a key tile's list is walked in segments of this
 * many entries (part of the plan's contract, see kt_seg). */
#define THD_KSEG 32

typedef struct thd_cp_plan_s* thd_cp_plan_t;   /* opaque, library-owned */

typedef struct thd_cp_plan_info_s {
    int64_t T;          /* packed tokens                                        */
    int32_t cp;         /* virtual context-parallel ranks                        */
    int32_t n_docs;     /* documents                                             */
    int64_t Tl;         /* tokens per rank, T / cp                               */
    int64_t n_qtiles;   /* 128-row tiles (query tiles == key tiles)              */
    int64_t n_entries;  /* listed (query tile, key tile) pairs                   */
    int64_t causal_pairs; /* sum over documents of L (L + 1) / 2                 */
    int64_t n_kseg;     /* segments of the longest key-tile list (THD_KSEG entries each) */
    int64_t n_fqtiles;  /* query tiles of the forward tables (thd_cp_plan_export_fwd)   */
    int64_t n_fentries; /* entries of the forward tables                                */
    int64_t n_fkseg;    /* segments of the longest key-tile list of the forward tables  */
} thd_cp_plan_info_t;

/*
 * thd_cu_seqlens_from_eod -- document boundaries of an EOD-delimited packed
 * sequence ([USER] EOD attention-mask reset): a document ends with, and includes,
 * each token equal to eod_id; the tokens after the last EOD form a final document.
 *   tokens      host int32[T], T >= 1 (and T <= INT32_MAX).
 *   cu_seqlens  host int32[capacity]: receives n_docs + 1 offsets, cu_seqlens[0] = 0,
 *               cu_seqlens[n_docs] = T, strictly increasing.
 *   n_docs      receives the number of documents, also when capacity is too small,
 *               so that a caller may size the array with a first call.
 * Errors: THD_ERR_INVALID_ARG (null tokens/n_docs, T out of range, capacity < 0),
 * THD_ERR_TOO_LARGE (cu_seqlens null or capacity < n_docs + 1; *n_docs set).
 * Host only; the divisibility rule of thd_cp_plan is not checked here.
 */
int thd_cu_seqlens_from_eod(const int32_t* tokens, int64_t T, int32_t eod_id, int32_t* cu_seqlens,
                            int32_t capacity, int32_t* n_docs);

/*
 * thd_position_ids -- per-document position ids of the packed tokens ([USER]: the
 * position of a token restarts with its document): pos[t] = t - cu_seqlens[d] for
 * cu_seqlens[d] <= t < cu_seqlens[d+1].
 *   cu_seqlens  host int32[n_docs + 1], n_docs >= 1; pos host int32[cu_seqlens[n_docs]].
 * Errors: THD_ERR_INVALID_ARG, THD_ERR_BAD_SEQLENS (cu_seqlens[0] != 0 or not strictly
 * increasing).  Host only.
 */
int thd_position_ids(const int32_t* cu_seqlens, int32_t n_docs, int32_t* pos);

/*
 * thd_rope_workspace -- bytes of the cos/sin table thd_rope_apply needs:
 * T * (rot_dim / 2) * 8.  Errors: THD_ERR_INVALID_ARG.
 */
int thd_rope_workspace(int64_t T, int32_t rot_dim, size_t* bytes);

/*
 * thd_rope_apply -- rotary position embedding with per-document positions, in place
 * ([USER]: positions restart with every EOD-delimited document; the pages name no
 * rotary variant -- this is the half-split form).  For every row t and head h, and
 * i < rot_dim / 2, with angle = pos[t] * base^(-2 i / rot_dim):
 *   x[t,h,i]             <- x[t,h,i] cos - x[t,h,i + rot_dim/2] sin
 *   x[t,h,i + rot_dim/2] <- x[t,h,i + rot_dim/2] cos + x[t,h,i] sin
 * dimensions rot_dim .. dim-1 unchanged.  The angles are formed in double precision
 * into a fp32 cos/sin table (the workspace), then applied to every head.
 *   x          device bf16 [T, heads, dim] (any row order; pos gives each row's position).
 *   pos        device int32[T] (e.g. thd_position_ids copied to the device).
 *   rot_dim    even, 2 <= rot_dim <= dim, base > 0; built for rot_dim % 16 == 0 and
 *              dim % 8 == 0 (16-byte accesses), THD_ERR_UNSUPPORTED otherwise.
 *   workspace  device, >= thd_rope_workspace bytes, 16-byte aligned; caller-owned.
 * Errors: THD_ERR_INVALID_ARG, THD_ERR_UNSUPPORTED (dtype other than bf16),
 * THD_ERR_MISALIGNED, THD_ERR_CUDA.
 */
int thd_rope_apply(void* x, const int32_t* pos, int64_t T, int32_t heads, int32_t dim, int32_t rot_dim,
                   double base, int32_t dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * thd_cp_plan -- validate a packed layout and build the symmetric partition and
 * the per-tile metadata ([USER] divisibility rule; [WHAT] EOD-aware symmetric
 * partitioning and metadata caching).
 *
 *   cu_seqlens  host int32[n_docs + 1]: document d spans global tokens
 *               [cu_seqlens[d], cu_seqlens[d+1]).  Documents are EOD-delimited:
 *               attention never crosses a boundary.
 *   n_docs      >= 1.
 *   cp          virtual ranks, >= 1.  Document d (length L, chunk c = L / (2 cp))
 *               is cut into 2 cp chunks; rank r owns chunk r and chunk 2 cp-1-r,
 *               documents ascending, chunk r first.
 *   out         receives a new plan; *out is left untouched on error.
 *
 * Errors: THD_ERR_INVALID_ARG (null, n_docs < 1, cp < 1, T overflow),
 * THD_ERR_BAD_SEQLENS, THD_ERR_NOT_DIVISIBLE, THD_ERR_ALLOC.  Host only.
 */
int thd_cp_plan(const int32_t* cu_seqlens, int32_t n_docs, int32_t cp, thd_cp_plan_t* out);

/* Sizes of the plan's tables.  Host only. */
int thd_cp_plan_info(thd_cp_plan_t plan, thd_cp_plan_info_t* out);

/*
 * thd_cp_plan_export -- copy the host tables into caller-allocated host arrays;
 * any pointer may be NULL to skip that table.
 *   q_idx        int32[T]      global token at rank-major row j
 *   rm_of_global int32[T]      rank-major row of global token g (inverse)
 *   qtiles       int32[n_qtiles * 12]: r, d, row0, m, qpos0, qbrk, qjump,
 *                qpos_max, nk, entry_off, doc_start, doc_end.  Tile rows are
 *                rank-major rows row0 .. row0+m-1 of one (rank, document) segment;
 *                the global position of tile row t is
 *                qpos0 + t + (t >= qbrk ? qjump : 0).
 *   entries      int32[n_entries * 8]: k0, nvalid, kpos0, kbrk, kjump, cls,
 *                ktile, key_rank.  Key rows k0 .. k0+nvalid-1 (rank-major, read in
 *                place: [WHAT] direct rank-major K/V indexing) are the keys of
 *                one 128-row slice that some row of the query tile can see;
 *                cls = THD_CLS_UNMASKED when every row sees every key, else
 *                THD_CLS_PARTIAL.  Fully masked slices are not listed.
 *   lpt          int32[n_qtiles]   query tiles by descending nk (ties by index)
 *   kt_off       int32[n_qtiles+1] CSR offsets of the key-tile transpose
 *   kt_list      int32[n_entries*2] (qtile, entry) per key tile, by descending
 *                qpos_max of the query tile (ties by qtile index)
 *   kt_lpt       int32[n_qtiles]   key tiles by descending list length
 *   kt_seg       int32[n_kseg+1]   backward work items by segment: a key tile's list
 *                is cut into segments of THD_KSEG entries; kt_seg[j+1] - kt_seg[j] is the
 *                number of key tiles whose list reaches segment j (the first ones of
 *                kt_lpt), kt_seg[0] = 0.  Lists being prefixes of one order per
 *                document, segment j of every key tile of a document walks the same
 *                query tiles.
 */
int thd_cp_plan_export(thd_cp_plan_t plan, int32_t* q_idx, int32_t* rm_of_global,
                       int32_t* qtiles, int32_t* entries, int32_t* lpt,
                       int32_t* kt_off, int32_t* kt_list, int32_t* kt_lpt, int32_t* kt_seg);

/*
 * thd_cp_plan_export_fwd -- copy the forward tables into caller-allocated host arrays
 * (NULL skips a table).  Documents whose chunks are shorter than a tile
 * (L / (2 cp) < THD_BM) put two or more chunks, far apart in position, into every
 * rank-major tile, so that most of each tile pair is masked ([WHAT] one fused call
 * over all documents: short documents must not waste it).  The forward tiles them in
 * position order, reading the rank-major buffers in place through rm_of_global:
 *   fqtiles   int32[n_fqtiles * 12], qtile layout.  First the rank-major query tiles
 *             of the other documents (as in qtiles, entry_off into fentries), then, per
 *             short-chunk document d (ascending) and u = 0 .. ceil(L/128)-1, a position
 *             tile: r = -1, d, row0 = -1, m = min(128, L - 128u), qpos0 = s_d + 128u,
 *             qbrk = m, qjump = 0, qpos_max, nk = u + 1, entry_off, doc_start, doc_end.
 *   fentries  int32[n_fentries * 8], entry layout; ktile (field 6) is the index in
 *             fqtiles of the tile holding the entry's keys.  For a position tile, its key
 *             tiles v = 0 .. u: k0 = -1, nvalid (128, or m for v = u), kpos0 = s_d + 128v,
 *             kbrk = nvalid, kjump = 0, cls (UNMASKED below the diagonal), ktile = the
 *             position tile v of d, key_rank = -1.
 *   flpt      int32[n_fqtiles]  forward query tiles by descending nk (ties by index).
 *   fkt_off, fkt_list, fkt_lpt, fkt_seg  the key-tile transpose of these tables, laid
 *             out as kt_off / kt_list / kt_lpt / kt_seg (sizes n_fqtiles + 1,
 *             n_fentries * 2, n_fqtiles, n_fkseg + 1): the backward walks it.
 */
int thd_cp_plan_export_fwd(thd_cp_plan_t plan, int32_t* fqtiles, int32_t* fentries, int32_t* flpt,
                           int32_t* fkt_off, int32_t* fkt_list, int32_t* fkt_lpt, int32_t* fkt_seg);

/*
 * thd_cp_plan_upload -- copy the tables to the current device once and keep them
 * there ([WHAT] metadata caching).  The plan owns one stream-ordered device
 * allocation (cudaMallocAsync on `stream`) holding every table and its status word,
 * and two pinned host staging buffers; the tables reach the device by one
 * cudaMemcpyAsync on `stream`.  The host tables stay valid.  Calling it again is a
 * no-op.  The tables live on the device that is current here; every later call with
 * this plan must be made with that same device current, on buffers of that device
 * (a launching call made with another device current returns THD_ERR_INVALID_ARG).
 * Errors: THD_ERR_CUDA, THD_ERR_ALLOC.
 */
int thd_cp_plan_upload(thd_cp_plan_t plan, void* stream);

/*
 * thd_cp_plan_update -- re-plan in place for a new packed layout (a new batch):
 * rebuilds the partition and the tile tables for (cu_seqlens, n_docs, cp), with the
 * validation and errors of thd_cp_plan, and, if the plan was uploaded, copies them to
 * its device on `stream` ([WHAT] metadata caching: the cache is refreshed, not
 * rebuilt, when the layout changes).  No device-wide synchronisation: the copy goes
 * through one of the plan's two pinned staging buffers (the host waits only for the
 * copy issued two updates earlier, which normally finished long ago), into the
 * plan's device allocation, which grows in stream order (cudaMallocAsync /
 * cudaFreeAsync on `stream`) only when the new tables do not fit.
 * Ordering: the copy overwrites the tables in place, after all work enqueued on
 * `stream` before this call; work that uses the plan on other streams must be
 * ordered before this call's position on `stream` by the caller.  Calls made after
 * it read the new layout.  The device status word is kept.
 * On a validation error the plan is unchanged.  If the device copy fails
 * (THD_ERR_CUDA / THD_ERR_ALLOC), the host tables hold the new layout and the plan
 * is left not uploaded.  With the plan uploaded, its device must be current
 * (THD_ERR_INVALID_ARG otherwise).
 */
int thd_cp_plan_update(thd_cp_plan_t plan, const int32_t* cu_seqlens, int32_t n_docs,
                       int32_t cp, void* stream);

/* Release the plan and its device tables.  If tables were uploaded, the plan's device
 * is made current, synchronised (so that no kernel still reads the tables) and the
 * caller's current device restored.  NULL is ignored.  A training loop that re-plans
 * every batch calls thd_cp_plan_update instead and destroys once. */
void thd_cp_plan_destroy(thd_cp_plan_t plan);

/*
 * thd_kv_gather -- materialise the rank-major buffer an all-gather of the
 * rank-local K/V shards produces ([WHAT] KV-all-gather, rank-major indexing):
 *   k_rm[j] = k[q_idx[j]],  v_rm[j] = v[q_idx[j]]   (whole rows, bit copies).
 * The same call shards Q or dO (pass v = v_rm = NULL).  One launch.
 *   k, v         device, [T, row] in global order (row = k_row_bytes bytes)
 *   k_rm, v_rm   device, [T, row] rank-major; must not overlap the sources
 *   *_row_bytes  > 0 and multiples of 16
 * Errors: THD_ERR_INVALID_ARG, THD_ERR_MISALIGNED, THD_ERR_NOT_UPLOADED,
 * THD_ERR_CUDA.
 */
int thd_kv_gather(thd_cp_plan_t plan, const void* k, const void* v, void* k_rm, void* v_rm,
                  int64_t k_row_bytes, int64_t v_row_bytes, void* stream);

/*
 * thd_rows_to_global -- the inverse permutation: dst[g] = src_rm[rm_of_global[g]],
 * whole rows of row_bytes bytes (multiple of 16).  Used to return rank-major
 * outputs in packed order.  Same errors as thd_kv_gather.
 */
int thd_rows_to_global(thd_cp_plan_t plan, const void* src_rm, void* dst,
                       int64_t row_bytes, void* stream);

/*
 * thd_cp_attn_fwd -- causal attention with EOD resets over the rank-major buffers,
 * every virtual rank at once, in one launch ([WHAT] single fused attention call;
 * [USER] causal + EOD reset).  For each rank-major query row i of document d and
 * query head h (key/value head g = h / (hq / hkv)):
 *   S_ij = scale * q_rm[i,h,:] . k_rm[j,g,:] over rank-major key rows j of d with
 *          position(j) <= position(i);
 *   o_rm[i,h,:]  = sum_j softmax_j(S_ij) v_rm[j,g,:];
 *   lse_rm[h*T+i] = log sum_j exp(S_ij)   (natural log, fp32).
 * Tiles the metadata lists as fully masked are never computed; the mask is
 * applied only on PARTIAL tiles.
 *   q_rm  [T, hq, dqk], k_rm [T, hkv, dqk], v_rm [T, hkv, dv], o_rm [T, hq, dv]:
 *         element type `dtype`; lse_rm fp32 [hq, T].
 *   scale > 0 and finite.  hq % hkv == 0.
 *   THD_DTYPE_BF16: (dqk, dv) in {(128,128), (192,128)}.
 *   THD_DTYPE_FP32: (dqk, dv) in {(64,64), (128,128)}.
 * Errors: THD_ERR_INVALID_ARG, THD_ERR_UNSUPPORTED, THD_ERR_MISALIGNED,
 * THD_ERR_NOT_UPLOADED, THD_ERR_CUDA.
 */
int thd_cp_attn_fwd(thd_cp_plan_t plan, const void* q_rm, const void* k_rm, const void* v_rm,
                    void* o_rm, float* lse_rm, int32_t hq, int32_t hkv, int32_t dqk,
                    int32_t dv, float scale, int32_t dtype, void* stream);

/*
 * thd_cp_attn_fwd_fused_gather -- thd_cp_attn_fwd with the K/V all-gather fused into
 * the attention's loads ([WHAT] KV all-gather with direct rank-major indexing: the
 * key/value rows a rank-major tile needs are fetched straight from the packed
 * tensors by position, so the rank-major K/V copy of thd_kv_gather is not needed).
 * Same attention, outputs and errors as thd_cp_attn_fwd; the query side stays
 * rank-major (a rank's own rows).
 *   q_rm [T, hq, dqk] rank-major; k [T, hkv, dqk], v [T, hkv, dv] in packed (global)
 *   order; o_rm [T, hq, dv] rank-major; lse_rm fp32 [hq, T].
 *   A key tile whose positions are consecutive (every tile of a document with chunks of
 *   128 or more rows, and every position tile) is one TMA box at its first position; a
 *   rank-major tile holding the seam between a rank's two chunks gathers its rows
 *   (TMA tile::gather4).  The loaded tiles are the rows thd_cp_attn_fwd reads from the
 *   rank-major copy, in the same order, so the outputs are bit-identical to it.
 *   Supported: THD_DTYPE_BF16 with (dqk, dv) in {(128,128), (192,128)}.
 */
int thd_cp_attn_fwd_fused_gather(thd_cp_plan_t plan, const void* q_rm, const void* k,
                                 const void* v, void* o_rm, float* lse_rm, int32_t hq,
                                 int32_t hkv, int32_t dqk, int32_t dv, float scale,
                                 int32_t dtype, void* stream);

/*
 * thd_cp_attn_fwd_mla -- thd_cp_attn_fwd for multi-head latent attention whose keys
 * are given in compact form: a per-head part and one rotary-position ("rope") key
 * per token shared by every head.  [WHAT] lists MLA among the head layouts the path
 * serves, in its expanded form (every head's key materialised at full width); the
 * compact form computes the same attention with the expanded key
 *   k[j,g,:] = concat(k_nope_rm[j,g,:], k_rope_rm[j,:])
 * so that
 *   S_ij = scale * (q_rm[i,h,:d_nope] . k_nope_rm[j,g,:] + q_rm[i,h,d_nope:] . k_rope_rm[j,:])
 * with the same mask, outputs and error codes as thd_cp_attn_fwd.  The gather then
 * moves d_nope * hkv + d_rope key elements per token instead of (d_nope + d_rope) * hkv.
 *   q_rm [T, hq, d_nope + d_rope], k_nope_rm [T, hkv, d_nope], k_rope_rm [T, d_rope],
 *   v_rm [T, hkv, dv], o_rm [T, hq, dv], lse_rm fp32 [hq, T].
 *   Supported: THD_DTYPE_BF16 with (d_nope, d_rope, dv) = (128, 64, 128).
 */
int thd_cp_attn_fwd_mla(thd_cp_plan_t plan, const void* q_rm, const void* k_nope_rm,
                        const void* k_rope_rm, const void* v_rm, void* o_rm, float* lse_rm,
                        int32_t hq, int32_t hkv, int32_t d_nope, int32_t d_rope, int32_t dv,
                        float scale, int32_t dtype, void* stream);

/*
 * thd_cp_attn_bwd_workspace -- device workspace bytes thd_cp_attn_bwd needs for
 * these sizes (fp32 row statistics and the fp32 dQ accumulator).
 */
int thd_cp_attn_bwd_workspace(thd_cp_plan_t plan, int32_t hq, int32_t hkv, int32_t dqk,
                              int32_t dv, int32_t dtype, size_t* bytes);

/*
 * thd_cp_attn_bwd -- gradients of thd_cp_attn_fwd (the backward pass of the
 * training path the page's context parallelism serves):
 *   Delta_i = sum(do_i * o_i);  P_ij = exp(S_ij - lse_i) on visible pairs;
 *   dV_j = sum_{i,h in group} P_ij do_i;   dP_ij = do_i . v_j;
 *   dS_ij = P_ij (dP_ij - Delta_i);
 *   dQ_i = scale * sum_j dS_ij k_j;   dK_j = scale * sum_{i,h in group} dS_ij q_i.
 * Inputs as in the forward (bf16), lse_rm from the forward, do_rm [T, hq, dv]
 * rank-major.  Outputs dq_rm [T, hq, dqk], dk_rm [T, hkv, dqk], dv_rm [T, hkv, dv]
 * are fp32, rank-major; dK/dV already hold the sum over virtual ranks (what a
 * reduce-scatter would deliver).  `workspace` must hold
 * thd_cp_attn_bwd_workspace bytes, 256-byte aligned; its contents on entry do not
 * matter.  THD_DTYPE_BF16 with (dqk, dv) = (128, 128) is built.
 */
int thd_cp_attn_bwd(thd_cp_plan_t plan, const void* q_rm, const void* k_rm, const void* v_rm,
                    const void* o_rm, const float* lse_rm, const void* do_rm,
                    float* dq_rm, float* dk_rm, float* dv_rm,
                    void* workspace, size_t workspace_bytes,
                    int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, float scale,
                    int32_t dtype, void* stream);

/*
 * thd_cp_attn_bwd_noalloc -- thd_cp_attn_bwd for callers that cannot allocate
 * device memory.  (The source page has no counterpart: this is a deployment variant of
 * the same backward.)  thd_cp_attn_bwd wants a workspace for the per-row
 * statistic Delta; a caller whose device memory is owned entirely by another
 * allocator, or whose hot path may not call cudaMalloc (it can synchronise the
 * device), cannot provide one.  This entry point keeps Delta in a fixed device
 * array built into the library instead and allocates nothing itself.
 *   Arguments, layouts, outputs and errors as thd_cp_attn_bwd, without the
 *   workspace; the plan must already be uploaded.
 *   Limit: hq * T <= THD_NOALLOC_MAX_ROWS_X_HEADS (8,388,608, i.e. 32 MiB of
 *   fp32); larger problems return THD_ERR_TOO_LARGE without launching anything.
 *   Every GPU that loads the library holds the 32 MiB array until the process
 *   exits.  The first call on a device looks up the array's device address (with
 *   that device current) and caches it; make that first call before any stream
 *   capture.  All calls share the array: calls whose kernels overlap on the GPU
 *   (e.g. on different streams) race on it and must be serialised by the caller.
 *   The array is fully rewritten by each call before it is read.  The cached
 *   address belongs to the device's current context: after cudaDeviceReset on a
 *   device, this entry point must not be called on that device again in the same
 *   process (the array then has a new address the cache does not know).
 */
#define THD_NOALLOC_MAX_ROWS_X_HEADS 8388608
int thd_cp_attn_bwd_noalloc(thd_cp_plan_t plan, const void* q_rm, const void* k_rm, const void* v_rm,
                            const void* o_rm, const float* lse_rm, const void* do_rm,
                            float* dq_rm, float* dk_rm, float* dv_rm,
                            int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, float scale,
                            int32_t dtype, void* stream);

/*
 * thd_cp_device_status -- every wait inside this library's kernels is bounded
 * (1 s per wait); a kernel whose wait gives up drains, records a nonzero code in
 * a status word owned by the plan (allocated by thd_cp_plan_upload) and returns,
 * so the context stays usable.  This call copies the word into *status (0 = no
 * timeout since the last reset) and clears it when reset != 0.  It synchronises
 * the device.  Errors: THD_ERR_INVALID_ARG, THD_ERR_NOT_UPLOADED, THD_ERR_CUDA.
 */
int thd_cp_device_status(thd_cp_plan_t plan, int32_t reset, int32_t* status);

/* Static, human-readable text of an error code. */
const char* thd_cp_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* THDCP_H */

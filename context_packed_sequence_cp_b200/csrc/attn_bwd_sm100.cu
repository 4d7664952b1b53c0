// Backward of the causal attention over the rank-major buffers on sm_100a.
//
// Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance":
// the context-parallel attention of a training stack (section "What this PR does /
// why we need it?": KV-all-gather CP with rank-major K/V indexing, cached tile
// metadata, MHA / GQA); its backward returns dQ for every rank's queries and dK /
// dV summed over every rank that read a key (what a reduce-scatter of the gathered
// gradients delivers; on one GPU the shared buffer already holds the sum).
//
// Two kernels:
//   bwd_prep   Delta_i = sum_d dO_id O_id per (row, head); zeroes dQ, dK and dV.
//   bwd_fused  key-major: one CTA per (list segment of a key tile, key/value head g)
//              walks the (query tile, query head) steps the plan lists for it and
//              computes every gradient once per step (no tile is recomputed):
//                a  S^T  = K Q^T   -> TMEM X       b  dP^T = V dO^T -> TMEM Y
//                P^T = exp(S^T - lse), bf16 over S^T; dS^T = P^T (dP^T - Delta), bf16
//                into shared memory (128-byte swizzled)
//                c  dV += P^T dO   d  dK += dS^T Q   (accumulated in TMEM)
//                e  Y = dS K: the key tile's share of the step's dQ, added into the
//                   fp32 dQ by TMA tensor reductions (whole 128-byte row segments)
//              dK, dV of the segment are added the same way at the end.
// A query tile's dQ gathers shares from every key tile that sees it, so dQ is summed
// at L2 (fp32 additions); an earlier design without additions, a key-major dK/dV
// kernel plus a query-major dQ kernel, recomputed S and dP for dQ (3/5 more tensor
// work) and was 10-25% slower end to end.
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"
#include "thdcp.h"

namespace thd {
namespace {

constexpr int kD = 128;                 // head dim built (Dqk = Dv = 128)
constexpr uint32_t kTmemCols = 512;
constexpr int kBox = 128 * 128;         // one 64-column x 128-row bf16 box, 16 KB
constexpr int kTile = 2 * kBox;         // 128 x 128 bf16 tile, 32 KB
constexpr int kCompute = 256;           // two compute warpgroups
constexpr int kThreads = 64 + kCompute; // producer warp, MMA warp, compute

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Per-step metadata of the key-major walk: the listed (query tile, entry) pair.
struct StepMeta {
    int row0, m, qpos0, qbrk, qjump, nvalid, cls;
};
__device__ __forceinline__ StepMeta load_meta(const int32_t* kt_list, const int32_t* qtiles, const int32_t* entries,
                                              int list_pos) {
    const int2 pr = __ldg(reinterpret_cast<const int2*>(kt_list) + list_pos);
    const int4 q = __ldg(reinterpret_cast<const int4*>(qtiles + (size_t)pr.x * 12));      // r, d, row0, m
    const int4 q2 = __ldg(reinterpret_cast<const int4*>(qtiles + (size_t)pr.x * 12) + 1); // qpos0, qbrk, qjump, -
    const int4 e0 = __ldg(reinterpret_cast<const int4*>(entries + (size_t)pr.y * 8));     // k0, nvalid, -, -
    const int4 e1 = __ldg(reinterpret_cast<const int4*>(entries + (size_t)pr.y * 8) + 1); // kjump, cls, -, -
    StepMeta mt;
    mt.row0 = q.z;
    mt.m = q.w;
    mt.qpos0 = q2.x;
    mt.qbrk = q2.y;
    mt.qjump = q2.z;
    mt.nvalid = e0.y;
    mt.cls = e1.y;
    return mt;
}

// ---------------------------------------------------------------- prep
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       float* __restrict__ delta, float* __restrict__ dq_zero,
                                                       float* __restrict__ dk_zero, float* __restrict__ dv_zero,
                                                       int64_t kv_rows, int64_t rows, int hq, int64_t T) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * 8;
    for (int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); w < rows; w += nwarps) {
        // w = row * hq + h; a row holds kD bf16 values, 4 per lane
        const uint2 a = *reinterpret_cast<const uint2*>(o + w * kD + lane * 4);
        const uint2 b = *reinterpret_cast<const uint2*>(dout + w * kD + lane * 4);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const float2 x = __bfloat1622float2(a2[t]), y = __bfloat1622float2(b2[t]);
            s = fmaf(x.x, y.x, s);
            s = fmaf(x.y, y.y, s);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) delta[(int64_t)(w % hq) * T + w / hq] = s;
        // dQ, dK and dV are accumulated with reductions: they start at zero
        *reinterpret_cast<float4*>(dq_zero + w * kD + lane * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
        if (w < kv_rows) {
            *reinterpret_cast<float4*>(dk_zero + w * kD + lane * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(dv_zero + w * kD + lane * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

// ================================================================ fused dK / dV / dQ
// One CTA per (list segment of a key tile, key/value head g).  Warp 0 loads K and V
// once and then, per step (query tile outer, the group's query heads inner), Q, dO and
// the rows' lse / Delta; warp 1 owns TMEM and issues every MMA; warps 2-9 are two
// compute warpgroups (key row on the TMEM lane, 64 query columns per thread).  Per step:
//   a  S^T  = K Q^T          -> TMEM X        b  dP^T = V dO^T -> TMEM Y
//   P^T = exp(S^T - lse) as bf16 over S^T (X); dS^T = P^T (dP^T - Delta) as bf16 into
//   shared memory (128-byte swizzled, the layout of a [key][query] tile)
//   c  dV += P^T dO   (A from TMEM X)
//   d  dK += dS^T Q   (A = dS^T, also stored as bf16 over dP^T in TMEM Y)
//   e  Y   = dS K     (A = dS from the same bytes read MN-major: this CTA's share of
//                      the query tile's dQ), drained by the compute warps and added
//                      into the fp32 dQ at L2
// issued as c(i), a(i+1), d(i), e(i), b(i+1).  No tile is computed twice.
struct FusedLayout {
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kTile;
    static constexpr int kOffQ = kOffV + kTile;             // 2 stages
    static constexpr int kOffDO = kOffQ + 2 * kTile;        // 2 stages
    static constexpr int kOffDS = kOffDO + 2 * kTile;       // dS^T, bf16 [128 keys][128 queries]
    static constexpr int kOffStat = kOffDS + kTile;         // per dO stage: lse2[128], delta[128]
    static constexpr int kOffBar = kOffStat + 2 * 256 * 4;
    static constexpr int kBytes = kOffBar + 256;
    static_assert(kBytes <= 232448, "shared memory budget");
};

// Phases: every barrier is used once per step (or per stage use) and its next phase
// needs work that its waiter has not released yet, so parities are unambiguous:
//   s_full   commit after a(i)   (waited: compute P1(i); producer before dO(i+1): c(i-1) done)
//   dp_full  commit after b(i)   (compute P2(i))
//   dq_full  commit after e(i)   (compute drain of dQ(i); producer before Q(i+2): d(i) done)
//   p_ready / ds_ready / dq_free  arrivals of the 256 compute threads (issuer)
struct FusedBars {
    uint64_t kv_full, q_full[2], do_full[2], stat_free[2], s_full, dp_full, dq_full, p_ready, ds_ready, dq_free,
        acc_done;
    uint32_t tmem_base;
    int abort;
};

// Tensor maps of the fused kernel: q, k, v, dout with 64-column x 128-row boxes; the same
// with 8 << s rows (runs inside position tiles, s = 0..3); 2-D row maps with one-row boxes
// (tile::gather4); dq, dk, dv: fp32 32 x 32 boxes for the TMA reductions, dq8, dk8, dv8 the
// same 8 rows high.
struct BwdMaps {
    CUtensorMap q, k, v, dout, dq, dk, dv, qg, kg, vg, dog, dq8, dk8, dv8;
    CUtensorMap qs[kRunBoxes], ks[kRunBoxes], vs[kRunBoxes], dos[kRunBoxes];
};

__global__ void __launch_bounds__(kThreads, 1)
bwd_fused_kernel(const __grid_constant__ BwdMaps tm, BwdArgs a) {
    using L = FusedLayout;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    FusedBars* bars = reinterpret_cast<FusedBars*>(smem_raw + L::kOffBar);
    float* s_stat = reinterpret_cast<float*>(smem_raw + L::kOffStat);
    const uint32_t sK = base + L::kOffK, sV = base + L::kOffV, sQ = base + L::kOffQ, sDO = base + L::kOffDO;
    const uint32_t sDS = base + L::kOffDS;
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = a.hq / a.hkv;
    // Work item: segment j (list entries j*THD_KSEG ..) of a key tile, for key/value
    // group g.  Items run groups outermost, then segment, then key tiles longest-first:
    // the resident CTAs walk the same THD_KSEG query tiles of a document, so the dQ tiles
    // they add into stay in L2 while they are hot.
    // The forward tables: a tile (query or key) is rank-major (row0 >= 0: 128 consecutive
    // rank-major rows, TMA boxes) or a position tile of a short-chunk document (row0 < 0:
    // positions pos0 .., rows gathered through rm_of_global with tile::gather4, outputs
    // added row by row).
    const int32_t* qtiles = a.fqtiles;
    const int32_t* entries = a.fentries;
    const int32_t* kt_list = a.fkt_list;
    const int per_group = a.fkt_seg[a.n_fkseg];
    const int g = blockIdx.x / per_group;
    const int item = blockIdx.x - g * per_group;
    int seg = 0;
    {
        int hi = a.n_fkseg;  // fkt_seg[seg] <= item < fkt_seg[hi]
        while (hi - seg > 1) {
            const int mid = (seg + hi) >> 1;
            if (__ldg(a.fkt_seg + mid) <= item) seg = mid;
            else hi = mid;
        }
    }
    const int kt = a.fkt_lpt[item - a.fkt_seg[seg]];
    const int* KT = qtiles + (size_t)kt * 12;
    const int k0 = KT[2], kn = KT[3], kpos0 = KT[4];
    const int l0 = a.fkt_off[kt] + seg * THD_KSEG;
    const int llen = min(THD_KSEG, a.fkt_off[kt + 1] - l0);
    const int n_it = group * llen;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->kv_full), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&bars->q_full[s]), 1);
            mbar_init(smem_u32(&bars->do_full[s]), 1 + 32);      // expect_tx + the warp's lse/Delta stores
            mbar_init(smem_u32(&bars->stat_free[s]), kCompute);  // lse/Delta of the stage read by every thread
        }
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->dp_full), 1);
        mbar_init(smem_u32(&bars->dq_full), 1);
        mbar_init(smem_u32(&bars->p_ready), kCompute);
        mbar_init(smem_u32(&bars->ds_ready), kCompute);
        mbar_init(smem_u32(&bars->dq_free), kCompute);
        mbar_init(smem_u32(&bars->acc_done), 1);
        bars->abort = (base & 1023u) ? 1 : *reinterpret_cast<volatile int*>(a.status);
        if (base & 1023u) atomicCAS(a.status, 0, 99);
        fence_mbar_init();
    }
    __syncthreads();
    if (bars->abort || n_it == 0) return;  // misaligned, or an earlier CTA timed out: do nothing
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tX = tmem, tY = tmem + 128, tDK = tmem + 256, tDV = tmem + 384;

    if (warp == 0) {
        // ---------------------------------------------------- producer warp
        const float log2e = 1.4426950408889634f;
        // A position tile's rows (positions pos0 .. pos0+n-1, rows past n repeating row n-1)
        // are runs of consecutive rank-major rows, one per chunk.  Lane l takes the group of
        // 8 tile rows l % 16 and the 64-column box l / 16; an aligned block of 2^s groups
        // inside one run is one box of 8 << s rows issued by its first lane (landing at the
        // block's 1024-byte-aligned offset, the full box's swizzled layout), any other group
        // two 4-row gathers.
        auto group_index = [&](int pos0, int n, int (&rr)[8]) {
            const int g8 = (lane & 15) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) rr[i] = __ldg(a.rm_of_global + pos0 + min(g8 + i, n - 1));
        };
        auto load_groups = [&](const CUtensorMap* full, const CUtensorMap* runs, const CUtensorMap* rows,
                               uint32_t dst, uint32_t bar, const int (&rr)[8], int heads, int head) {
            const int gq = lane & 15;
            bool run = true;
#pragma unroll
            for (int i = 1; i < 8; ++i) run = run && rr[i] == rr[0] + i;
            const int next0 = __shfl_down_sync(0xffffffffu, rr[0], 1);
            const uint32_t is_run = __ballot_sync(0xffffffffu, run) & 0xffffu;
            const uint32_t link = __ballot_sync(0xffffffffu, run && next0 == rr[0] + 8) & (is_run >> 1) & 0x7fffu;
            int size = -1;  // log2 of the groups in this lane's box; -1: gathers; -2: covered by another lane
#pragma unroll
            for (int sz = 4; sz >= 0 && size == -1; --sz) {
                const int n = 1 << sz, b = gq & ~(n - 1);
                const uint32_t need_run = ((1u << n) - 1u) << b, need_link = ((1u << (n - 1)) - 1u) << b;
                if ((is_run & need_run) == need_run && (link & need_link) == need_link) size = (gq == b) ? sz : -2;
            }
            const int c = lane >> 4;
            const uint32_t d = dst + c * kBox + gq * 1024;
            if (size >= 0) {
                tma_load_3d(size == 4 ? full : runs + size, d, bar, c * 64, head, rr[0]);
            } else if (size == -1) {
                tma_gather4(rows, d, bar, c * 64, rr[0] * heads + head, rr[1] * heads + head, rr[2] * heads + head,
                            rr[3] * heads + head);
                tma_gather4(rows, d + 512, bar, c * 64, rr[4] * heads + head, rr[5] * heads + head,
                            rr[6] * heads + head, rr[7] * heads + head);
            }
        };
        if (lane == 0) {
            tma_prefetch_desc(&tm.q);
            tma_prefetch_desc(&tm.k);
            tma_prefetch_desc(&tm.v);
            tma_prefetch_desc(&tm.dout);
            tma_prefetch_desc(&tm.dq);
            tma_prefetch_desc(&tm.dk);
            tma_prefetch_desc(&tm.dv);
        }
        const uint32_t kvf = smem_u32(&bars->kv_full);
        if (lane == 0) mbar_arrive_expect_tx(kvf, 2 * kTile);
        __syncwarp();
        if (k0 >= 0) {
            if (lane == 0)
                for (int c = 0; c < 2; ++c) {
                    tma_load_3d(&tm.k, sK + c * kBox, kvf, c * 64, g, k0);
                    tma_load_3d(&tm.v, sV + c * kBox, kvf, c * 64, g, k0);
                }
        } else {
            int rk[8];
            group_index(kpos0, kn, rk);
            load_groups(&tm.k, tm.ks, &tm.kg, sK, kvf, rk, a.hkv, g);
            load_groups(&tm.v, tm.vs, &tm.vg, sV, kvf, rk, a.hkv, g);
        }
        StepMeta cur = load_meta(kt_list, qtiles, entries, l0), nxt = cur;
        if (llen > 1) nxt = load_meta(kt_list, qtiles, entries, l0 + 1);
        int rq[8] = {0, 0, 0, 0, 0, 0, 0, 0};   // this lane's rows of the current query tile (position tiles)
        int rs[4] = {0, 0, 0, 0};   // rank-major rows of lse / Delta entries lane + 32 u (-1: none)
        for (int it = 0; it < n_it; ++it) {
            const int pos = it / group, hh = it - pos * group;   // query tiles outer, heads inner
            if (hh == 0 && it > 0) {
                cur = nxt;
                if (pos + 1 < llen) nxt = load_meta(kt_list, qtiles, entries, l0 + pos + 1);
            }
            const int h = g * group + hh;
            const int row0 = cur.row0;
            if (hh == 0) {   // rows of a new query tile
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = lane + 32 * u;
                    rs[u] = row0 >= 0 ? (row0 + t < a.T ? row0 + t : -1)
                                      : (t < cur.m ? __ldg(a.rm_of_global + cur.qpos0 + t) : -1);
                }
                if (row0 < 0) group_index(cur.qpos0, cur.m, rq);
            }
            float lv[4], dv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                lv[u] = rs[u] >= 0 ? __ldg(a.lse + (int64_t)h * a.T + rs[u]) * log2e : 0.f;
                dv[u] = rs[u] >= 0 ? __ldg(a.delta + (int64_t)h * a.T + rs[u]) * a.scale : 0.f;
            }
            const int st = it & 1;
            // dO(it) refills the stage c(it-2) read: c(it-2) is issued before a(it-1).
            if (it >= 2) {
                mbar_wait(smem_u32(&bars->s_full), (it - 1) & 1, abort, a.status, 61);
                mbar_wait(smem_u32(&bars->stat_free[st]), ((it >> 1) - 1) & 1, abort, a.status, 62);
            }
            const uint32_t f = smem_u32(&bars->do_full[st]);
            if (lane == 0) mbar_arrive_expect_tx(f, kTile);
            __syncwarp();
            if (row0 >= 0) {
                if (lane == 0)
                    for (int c = 0; c < 2; ++c) tma_load_3d(&tm.dout, sDO + st * kTile + c * kBox, f, c * 64, h, row0);
            } else {
                load_groups(&tm.dout, tm.dos, &tm.dog, sDO + st * kTile, f, rq, a.hq, h);
            }
            float* stat = s_stat + st * 256;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                stat[lane + 32 * u] = lv[u];
                stat[128 + lane + 32 * u] = dv[u];
            }
            mbar_arrive(f);
            // Q(it) refills the stage d(it-2) read: d(it-2) is issued before e(it-2).
            if (it >= 2) mbar_wait(smem_u32(&bars->dq_full), (it - 2) & 1, abort, a.status, 63);
            const uint32_t qf = smem_u32(&bars->q_full[st]);
            if (lane == 0) mbar_arrive_expect_tx(qf, kTile);
            __syncwarp();
            if (row0 >= 0) {
                if (lane == 0)
                    for (int c = 0; c < 2; ++c) tma_load_3d(&tm.q, sQ + st * kTile + c * kBox, qf, c * 64, h, row0);
            } else {
                load_groups(&tm.q, tm.qs, &tm.qg, sQ + st * kTile, qf, rq, a.hq, h);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idKK = idesc_bf16_f32(128, 128, false, false);  // A, B K-major
            constexpr uint32_t idTM = idesc_bf16_f32(128, 128, false, true);   // A TMEM / K-major, B MN-major
            constexpr uint32_t idMM = idesc_bf16_f32(128, 128, true, true);    // A and B MN-major
            constexpr uint32_t dhi = smem_desc_hi_sw128(1024);
            const uint32_t klo = smem_desc_lo(sK, 16), vlo = smem_desc_lo(sV, 16);
            const uint32_t kmlo = smem_desc_lo(sK, kBox);   // K as the MN-major B of e
            const uint32_t dsmlo = smem_desc_lo(sDS, kBox); // dS, MN-major A of e
            auto issue_a = [&](int it) {  // S^T = K Q^T -> X
                const int st = it & 1;
                mbar_wait(smem_u32(&bars->q_full[st]), (it >> 1) & 1, abort, a.status, 64);
                tc_fence_after();
                const uint32_t qlo = smem_desc_lo(sQ + st * kTile, 16);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * kBox + (kk & 3) * 32) >> 4;
                    mma_ss(tX, smem_desc_of(klo + off, dhi), smem_desc_of(qlo + off, dhi), idKK, kk > 0);
                }
                mma_commit(smem_u32(&bars->s_full));
            };
            auto issue_b = [&](int it) {  // dP^T = V dO^T -> Y
                const int st = it & 1;
                mbar_wait(smem_u32(&bars->do_full[st]), (it >> 1) & 1, abort, a.status, 65);
                tc_fence_after();
                const uint32_t dlo = smem_desc_lo(sDO + st * kTile, 16);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * kBox + (kk & 3) * 32) >> 4;
                    mma_ss(tY, smem_desc_of(vlo + off, dhi), smem_desc_of(dlo + off, dhi), idKK, kk > 0);
                }
                mma_commit(smem_u32(&bars->dp_full));
            };
            mbar_wait(smem_u32(&bars->kv_full), 0, abort, a.status, 66);
            tc_fence_after();
            issue_a(0);
            issue_b(0);
            for (int it = 0; it < n_it; ++it) {
                const int st = it & 1;
                // c: dV += P^T dO, once P^T is in X
                mbar_wait(smem_u32(&bars->p_ready), it & 1, abort, a.status, 67);
                tc_fence_after();
                const uint32_t dlo = smem_desc_lo(sDO + st * kTile, kBox);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tDV, tX + kk * 8, smem_desc_of(dlo + kk * (2048 >> 4), dhi), idTM, (it > 0 || kk > 0));
                // a of the next step: X is rewritten only after c has read it (issue order)
                if (it + 1 < n_it) issue_a(it + 1);
                // d: dK += dS^T Q and e: Y = dS K, once dS^T is in shared memory
                mbar_wait(smem_u32(&bars->ds_ready), it & 1, abort, a.status, 68);
                tc_fence_after();
                const uint32_t qlo = smem_desc_lo(sQ + st * kTile, kBox);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_ts(tDK, tY + kk * 8, smem_desc_of(qlo + kk * (2048 >> 4), dhi), idTM, (it > 0 || kk > 0));
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tY, smem_desc_of(dsmlo + kk * (2048 >> 4), dhi), smem_desc_of(kmlo + kk * (2048 >> 4), dhi),
                           idMM, kk > 0);
                mma_commit(smem_u32(&bars->dq_full));
                // b of the next step: Y is rewritten only after dQ(it) has been read out
                if (it + 1 < n_it) {
                    mbar_wait(smem_u32(&bars->dq_free), it & 1, abort, a.status, 69);
                    issue_b(it + 1);
                }
            }
            mma_commit(smem_u32(&bars->acc_done));
        }
    } else {
        // ---------------------------------------------------- compute warpgroups
        const int ct = threadIdx.x - 64;         // 0..255
        const int hf = ct >> 7;                  // column half
        const int wq = warp & 3;
        const int r = wq * 32 + lane;            // TMEM lane: key row (X, Y as S^T / dP^T), query row (Y as dQ)
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const float sl2 = a.scale_log2;
        const float sc = a.scale;
        const int kpos_r = KT[4] + r + (r >= KT[5] ? KT[6] : 0);
        // this thread's 128-byte row of dS^T: box hf, row r, 16-byte chunks swizzled by r % 8
        const uint32_t ds_row = sDS + hf * kBox + r * 128;
        StepMeta cur = load_meta(kt_list, qtiles, entries, l0), nxt = cur;
        if (llen > 1) nxt = load_meta(kt_list, qtiles, entries, l0 + 1);
        StepMeta prev = cur;  // the step whose dQ is drained
        int prev_h = 0;
        // Partial sums leave the CTA through its warps: a warp holds 32 rows x 64 columns
        // of an fp32 TMEM accumulator (rows 32 wq .., columns hf*64 ..).  It writes them, 32
        // columns at a time, into its own 4 KB of the dS^T buffer (the rows only it writes)
        // in the 128-byte swizzled layout of a 32 x 32 fp32 box, and one lane adds the box
        // into global memory with a TMA tensor reduction (whole 128-byte row segments).  A
        // warp whose rows run past the tile's valid rows adds those with vector reductions.
        const uint32_t warp_stage = sDS + hf * kBox + wq * 32 * 128;
        auto stage = [&](const uint32_t (&v)[32]) {  // chunks swizzled by lane % 8
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_shared_v4(warp_stage + lane * 128 + ((c ^ (lane & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2],
                             v[4 * c + 3]);
        };
        // The staging rows are rewritten only after stage_free(): a box handed to the TMA unit
        // is waited for (read out of shared memory) there, as late as possible.
        auto stage_free = [&]() {
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
        };
        // adds the staged box at (row0 + 32 wq, head, col) of a [rows, heads, 128] fp32
        // tensor with `valid` rows from row0 on.  A position tile (row0 < 0; rows at positions
        // pos0 .., found through rm_of_global) or a short tile adds every aligned group of 8
        // rows that are 8 consecutive rows of the tensor as an 8-row sub-box (map8: its staged
        // rows start at a 1024-byte boundary, the box's swizzled layout), the other rows one by
        // one with vector reductions.  Only lane 0 issues bulk operations, so that its wait
        // covers every box of the warp.
        auto reduce = [&](const CUtensorMap* map, const CUtensorMap* map8, float* gbase, int heads, int head,
                          int row0, int pos0, int valid, int col) {
            if (row0 >= 0 && wq * 32 + 32 <= valid) {
                fence_proxy_async_smem();   // the staged rows, visible to the TMA unit
                __syncwarp();
                if (lane == 0) {
                    tma_reduce_add_3d(map, warp_stage, col, head, row0 + wq * 32);
                    bulk_commit_group();
                }
            } else {
                const int q_l = wq * 32 + lane;
                const int row_l = q_l < valid ? (row0 >= 0 ? row0 + q_l : __ldg(a.rm_of_global + pos0 + q_l)) : -1;
                const int lead = __shfl_sync(0xffffffffu, row_l, lane & ~7);
                const uint32_t ok = __ballot_sync(0xffffffffu, row_l >= 0 && row_l == lead + (lane & 7));
                uint32_t runs = 0;  // bit k: rows 8k .. 8k+7 go as one sub-box
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (((ok >> (8 * k)) & 0xffu) == 0xffu) runs |= 1u << k;
                if (runs) fence_proxy_async_smem();   // the staged rows, visible to the TMA unit
                __syncwarp();
                int r8[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) r8[k] = __shfl_sync(0xffffffffu, row_l, 8 * k);
                if (lane == 0 && runs) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if ((runs >> k) & 1u) tma_reduce_add_3d(map8, warp_stage + k * 1024, col, head, r8[k]);
                    bulk_commit_group();
                }
                const int sub = lane >> 3, chunk = lane & 7;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int rr = 4 * j + sub;
                    const int row = __shfl_sync(0xffffffffu, row_l, rr);
                    if (row >= 0 && !((runs >> (rr >> 3)) & 1u)) {
                        const float4 x = ld_shared_f4(warp_stage + rr * 128 + ((chunk ^ (rr & 7)) << 4));
                        red_add_v4(gbase + ((int64_t)row * heads + head) * kD + col + 4 * chunk, x.x, x.y, x.z, x.w);
                    }
                }
                __syncwarp();
            }
        };
        // dQ(it) = dS K of this key tile, rows = the step's query rows: read out of Y (which
        // is then released for b(it+1)) and added, times scale, into the fp32 dQ.
        auto drain = [&](int it, const StepMeta& mt, int h) {
            mbar_wait(smem_u32(&bars->dq_full), it & 1, abort, a.status, 70);
            tc_fence_after();
            uint32_t v[32];
            tmem_ld32(tY + lane_addr + hf * 64, v);
            tmem_wait_ld();
            stage(v);
            // the first half goes to the TMA unit while the second is read out of TMEM
            reduce(&tm.dq, &tm.dq8, a.dq_acc, a.hq, h, mt.row0, mt.qpos0, mt.m, hf * 64);
            tmem_ld32(tY + lane_addr + hf * 64 + 32, v);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->dq_free));   // Y read out: b(it+1) may overwrite it
            stage_free();
            stage(v);
            reduce(&tm.dq, &tm.dq8, a.dq_acc, a.hq, h, mt.row0, mt.qpos0, mt.m, hf * 64 + 32);
        };
        for (int it = 0; it < n_it; ++it) {
            const int st = it & 1;
            const int pos = it / group, hh = it - pos * group;
            if (hh == 0 && it > 0) {
                cur = nxt;
                if (pos + 1 < llen) nxt = load_meta(kt_list, qtiles, entries, l0 + pos + 1);
            }
            const int m = cur.m, qpos0 = cur.qpos0, qbrk = cur.qbrk, qjump = cur.qjump;
            // visible query columns of this key row: a suffix [lo, hi) of the tile
            int lo = 0, hi = m;
            if (r >= cur.nvalid) hi = 0;
            else if (cur.cls != 2) {
                const int n1 = min(qbrk, m);
                if (kpos_r <= qpos0) lo = 0;
                else if (kpos_r - qpos0 < n1) lo = kpos_r - qpos0;
                else {
                    const int p1 = qpos0 + qbrk + qjump;   // position of row qbrk
                    lo = (kpos_r <= p1) ? n1 : min(m, n1 + (kpos_r - p1));
                }
            }
            const float* stat = s_stat + st * 256;

            // ---- P1: P^T = exp(S^T - lse) on this thread's 64 query columns, bf16 over S^T
            mbar_wait(smem_u32(&bars->do_full[st]), (it >> 1) & 1, abort, a.status, 71);  // lse/Delta staged
            mbar_wait(smem_u32(&bars->s_full), it & 1, abort, a.status, 72);
            tc_fence_after();
            float p[64];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t sv[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(tX + lane_addr + c0, sv);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 32; t += 4) {
                    const float4 l4 = *reinterpret_cast<const float4*>(stat + c0 + t);
                    const float lq[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = c0 + t + u;
                        const float e = ex2(fmaf(__uint_as_float(sv[t + u]), sl2, -lq[u]));
                        p[ch * 32 + t + u] = (i >= lo && i < hi) ? e : 0.f;
                    }
                }
            }
            named_bar_sync(2 + wq, 64);  // both halves of these rows have read S^T before P^T overwrites it
            {
                uint32_t pk[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) pk[t] = pack_bf16x2(p[2 * t], p[2 * t + 1]);
                tmem_st32(tX + lane_addr + hf * 32, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->p_ready));

            // ---- drain dQ of the previous step (frees Y for b(it), and the dS^T buffer)
            if (it >= 1) drain(it - 1, prev, prev_h);
            prev = cur;
            prev_h = a.hq / a.hkv * g + hh;

            // ---- P2: dS^T = P^T (dP^T - Delta) -> shared memory
            mbar_wait(smem_u32(&bars->dp_full), it & 1, abort, a.status, 73);
            tc_fence_after();
            uint32_t dsk[32];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t dpv[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(tY + lane_addr + c0, dpv);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 4; ++j) {   // 16-byte chunk (8 queries) ch * 4 + j of this half-row
                    uint32_t w4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int t = j * 8 + 2 * u;
                        const float2 d2 = *reinterpret_cast<const float2*>(stat + 128 + c0 + t);
                        // scale folded in: scale * dS = P (scale * dP - scale * Delta)
                        w4[u] = pack_bf16x2(p[ch * 32 + t] * fmaf(__uint_as_float(dpv[t]), sc, -d2.x),
                                            p[ch * 32 + t + 1] * fmaf(__uint_as_float(dpv[t + 1]), sc, -d2.y));
                    }
                    dsk[ch * 16 + j * 4] = w4[0];
                    dsk[ch * 16 + j * 4 + 1] = w4[1];
                    dsk[ch * 16 + j * 4 + 2] = w4[2];
                    dsk[ch * 16 + j * 4 + 3] = w4[3];
                    const int chunk = ch * 4 + j;
                    if (ch == 0 && j == 0) stage_free();   // the drain's last box has been read
                    st_shared_v4(ds_row + ((chunk ^ (r & 7)) << 4), w4[0], w4[1], w4[2], w4[3]);
                }
            }
            named_bar_sync(2 + wq, 64);  // both halves have read dP^T before dS^T overwrites it
            tmem_st32(tY + lane_addr + hf * 32, dsk);
            tmem_wait_st();
            mbar_arrive(smem_u32(&bars->stat_free[st]));  // lse and Delta of this stage read
            fence_proxy_async_smem();                      // dS^T visible to the tensor pipe
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->ds_ready));
        }
        drain(n_it - 1, prev, prev_h);
        // ---------------------------------------------------- dK, dV epilogue
        // This item's share of dK and dV (its list segment) is added into the outputs.
        mbar_wait(smem_u32(&bars->acc_done), 0, abort, a.status, 74);
        tc_fence_after();
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const uint32_t src = which == 0 ? tDK : tDV;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t v[32];
                tmem_ld32(src + lane_addr + hf * 64 + ch * 32, v);
                tmem_wait_ld();
                stage_free();
                stage(v);
                reduce(which == 0 ? &tm.dk : &tm.dv, which == 0 ? &tm.dk8 : &tm.dv8, which == 0 ? a.dk : a.dv, a.hkv, g,
                       k0, kpos0, kn, hf * 64 + ch * 32);
            }
        }
        stage_free();   // every box read before the CTA's shared memory is released
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}
}  // namespace

int launch_bwd_sm100(int dqk, int dv, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                     const CUtensorMap& dout, const BwdArgs& a, int n_items_per_group, int num_sms,
                     cudaStream_t stream) {
    if (dqk != kD || dv != kD) return -2;
    static std::atomic<uint64_t> configured{0};
    if (!ensure_dynamic_smem(bwd_fused_kernel, FusedLayout::kBytes, configured)) return -1;
    BwdMaps m;
    m.q = q;
    m.k = k;
    m.v = v;
    m.dout = dout;
    if (!make_map_f32_box32(&m.dq, a.dq_acc, a.T, a.hq, kD) || !make_map_f32_box32(&m.dk, a.dk, a.T, a.hkv, kD) ||
        !make_map_f32_box32(&m.dv, a.dv, a.T, a.hkv, kD) || !make_map_f32_box32(&m.dq8, a.dq_acc, a.T, a.hq, kD, 8) ||
        !make_map_f32_box32(&m.dk8, a.dk, a.T, a.hkv, kD, 8) || !make_map_f32_box32(&m.dv8, a.dv, a.T, a.hkv, kD, 8) || !make_map_bf16_rows(&m.qg, a.q, a.T * a.hq, kD) ||
        !make_map_bf16_rows(&m.kg, a.k, a.T * a.hkv, kD) || !make_map_bf16_rows(&m.vg, a.v, a.T * a.hkv, kD) ||
        !make_map_bf16_rows(&m.dog, a.dout, a.T * a.hq, kD))
        return -1;
    for (int s = 0; s < kRunBoxes; ++s)
        if (!make_map_bf16(&m.qs[s], a.q, a.T, a.hq, kD, 8 << s) || !make_map_bf16(&m.ks[s], a.k, a.T, a.hkv, kD, 8 << s) ||
            !make_map_bf16(&m.vs[s], a.v, a.T, a.hkv, kD, 8 << s) ||
            !make_map_bf16(&m.dos[s], a.dout, a.T, a.hq, kD, 8 << s))
            return -1;
    bwd_prep_kernel<<<num_sms * 8, 256, 0, stream>>>(a.o, a.dout, a.delta, a.dq_acc, a.dk, a.dv, a.T * a.hkv,
                                                     a.T * a.hq, a.hq, a.T);
    if (cudaGetLastError() != cudaSuccess) return -1;
    const unsigned items = (unsigned)((int64_t)n_items_per_group * a.hkv);
    bwd_fused_kernel<<<items, kThreads, FusedLayout::kBytes, stream>>>(m, a);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace thd

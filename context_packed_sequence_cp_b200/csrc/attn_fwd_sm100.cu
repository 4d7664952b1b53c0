// Forward causal attention over the rank-major buffers on sm_100a tensor cores.
//
// Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance",
// section "What this PR does / why we need it?": one fused attention call covers
// every document and every context-parallel rank, reading K/V in place in the
// rank-major (all-gathered) layout, driven by cached per-tile metadata; MHA, GQA
// and expanded MLA.  Section "Does this PR introduce any user-facing change?":
// causal attention with EOD reset.
//
// A work item is one (query tile, query head); the grid has one CTA per item, in one of
// two orders (fwd_item).  Two instantiations: PERSIST, where a CTA takes over the items of
// CTAs that have not started yet (cluster launch control) and keeps its TMEM and pipelines
// (plans of short query tiles), and one CTA per item.  Warp roles (384 threads):
//   warp 0      TMA producer of the Q tile and of K of every listed entry (position
//               tiles: aligned boxes over runs of consecutive rows, 4-row gathers
//               across chunk boundaries);
//   warp 2      TMA producer of V (separate K and V rings, 128-byte swizzled
//               boxes of 64 columns); a stage is refilled once the MMA that read
//               it retired (K on the S signal, V on the PV signal).
//   warp 1      TMEM owner and issuer of S_j = Q K_j^T into one of three TMEM
//               score buffers, up to three tiles ahead of the softmax;
//   warp 11     issuer of O += P_j V_j (P read from TMEM).
//               The tensor pipe's queue is short: with one issuing thread every
//               barrier wait or commit between MMA groups let it run dry, and the
//               issuing thread competed for its SMSP with two softmax warps
//               (measured in place: ~95-140 cycles per 128x128x16 MMA against 64).
//               Two issuers on different SMSPs keep it fed (measured 64 cycles per
//               MMA under the same load).
//   warps 3-10  two softmax warpgroups; a thread owns half of one query row: it
//               reads its 64 columns of S_j from TMEM, masks PARTIAL entries only,
//               keeps the running max / sum in fp32 (base-2, scale folded in; the
//               two halves' maxima meet in shared memory once per tile), writes its
//               P_j columns as bf16 over S_j, and rescales its half of O in TMEM only
//               when the running max grows by more than 2^8 (lazy correction);
//               finally O / l (whole 128-byte half rows after a lane transpose) and lse
//               to global memory.
// TMEM columns: [0,128) S0/P0, [128,256) S1/P1, [256,384) S2/P2, [384,384+DV) O.
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace thd {
namespace {

constexpr int BM = 128, BN = 128, kMaxStages = 3;
constexpr int kSBuf = 3;                 // S/P buffers in TMEM
constexpr uint32_t kTmemO = kSBuf * 128; // first O column
constexpr int kSoftmax = 256;          // two softmax warpgroups
constexpr int kPvWarp = 3 + kSoftmax / 32;  // PV issuer, after the softmax warps
constexpr int kThreads = 96 + kSoftmax + 32; // K producer, S issuer, V producer, softmax, PV issuer
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kClc = 2;                     // response slots of cluster launch control
constexpr int kWarps = kThreads / 32;       // every warp reads each response
static_assert(kClc * 16 <= 64, "response slots");

template <int DQK, int DV>
struct FwdLayout {
    // Separate K and V rings: K_j is released as soon as S_j retires, V_j once PV_j
    // has; each ring has its own producer warp, so neither load waits on the other.
    static constexpr int NK = (DQK <= 128) ? 3 : 2;
    static constexpr int NV = (DQK <= 128) ? 3 : 2;
    static constexpr int kBox = BM * 128;  // one 64-column, 128-row swizzled box: 16 KB
    static constexpr int kQBytes = BM * DQK * 2;
    static constexpr int kKBytes = BN * DQK * 2;
    static constexpr int kVBytes = BN * DV * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + NK * kKBytes;
    static constexpr int kOffBar = kOffV + NV * kVBytes;
    static constexpr int kOffClc = kOffBar + 256;           // kClc 16-byte responses (cluster launch control)
    static constexpr int kOffXchg = kOffClc + 64;           // [2 buffers][2 halves][128 rows] fp32
    static constexpr int kBytes = kOffXchg + 2 * 2 * 128 * 4;
    static constexpr int kDynSmem = kBytes;                 // base is 1024-aligned by declaration (checked)
    static_assert(kDynSmem <= 232448, "shared memory budget");
};

struct Bars {
    uint64_t q_full, q_free, k_full[kMaxStages], v_full[kMaxStages], s_full[kSBuf], p_full[kSBuf], o_done[kSBuf];
    uint64_t o_free;                       // the epilogue has read O out of TMEM
    uint64_t clc_full[kClc], clc_empty[kClc];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// A work item: one query tile and one query head.  Items are numbered key/value group
// outermost, then query tiles longest-first, then the query heads of the group, so that
// the items in flight together walk the K/V tiles of one group (a working set that stays
// in L2) instead of all groups at once; or, when a group has too few items to fill the
// GPU (qtile_outer), query tiles longest-first outermost and every query head inner, so
// that the longest items of every group start first.  The grid has one CTA per item.
struct FwdItem {
    int h, g;
    int4 q0, q1, q2;  // the tile record: r, d, row0, m | qpos0, qbrk, qjump, qpos_max | nk, entry_off, ..
};

__device__ __forceinline__ FwdItem fwd_item(int it, const FwdArgs& a) {
    const int group = a.hq / a.hkv;
    FwdItem x;
    int qr;  // rank of the query tile in the longest-first order
    if (a.qtile_outer) {
        qr = it / a.hq;
        x.h = it - qr * a.hq;
        x.g = x.h / group;
    } else {
        const int per_group = (int)(gridDim.x / (unsigned)a.hkv);  // query tiles x group
        x.g = it / per_group;
        const int rem = it - x.g * per_group;
        x.h = x.g * group + rem % group;
        qr = rem / group;
    }
    const int4* Q = reinterpret_cast<const int4*>(a.qtiles + (size_t)__ldg(a.lpt + qr) * 12);
    x.q0 = __ldg(Q);
    x.q1 = __ldg(Q + 1);
    x.q2 = __ldg(Q + 2);
    return x;
}

// Number of leading key columns of an entry visible to a query at global position
// qpos: key t sits at kpos0 + t + (t >= kbrk ? kjump : 0), positions increase with
// t, so the visible keys are a prefix of the nvalid listed ones.
// Pair barriers: the two threads that hold the halves of a row sit in warps w and w+4
// (the same TMEM lane quarter), so every exchange between halves, and every overwrite
// of a half's TMEM columns read by its partner, needs only those two warps: barrier
// 2 + (w & 3), 64 threads.
__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ int visible_prefix(int qpos, int nvalid, int kpos0, int kbrk, int kjump) {
    if (qpos < kpos0) return 0;
    const int a = min(kbrk, qpos - kpos0 + 1);
    if (a < kbrk || kbrk >= nvalid) return min(a, nvalid);
    const int b0 = kpos0 + kbrk + kjump;
    if (qpos < b0) return kbrk;
    return min(nvalid, kbrk + (qpos - b0 + 1));
}

// SHARED_ROPE (DQK = 192 only): keys come in the compact form of multi-head latent
// attention, a per-head 128-wide part (tm.k) and one 64-wide rope key per token shared
// by every head (tm.kr); the third 64-column box of each key tile is read from tm.kr.
template <int DQK, int DV, bool SHARED_ROPE, bool PERSIST>
__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ FwdMaps tm, FwdArgs a) {
    static_assert(!SHARED_ROPE || DQK == 192, "the shared rope key is the third 64-column box");
    static_assert(DV == 128, "the epilogue stores 8 chunks of 8 columns per half row");
    using L = FwdLayout<DQK, DV>;
    constexpr int NK = L::NK, NV = L::NV;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    Bars* bars = reinterpret_cast<Bars*>(smem_raw + L::kOffBar);
    float* xch = reinterpret_cast<float*>(smem_raw + L::kOffXchg);
    const uint32_t sQ = base + L::kOffQ, sK = base + L::kOffK, sV = base + L::kOffV;
    const uint32_t clc_resp = base + L::kOffClc;
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->q_full), 1);
        mbar_init(smem_u32(&bars->q_free), 1);  // every S of the item that read Q retired
        for (int s = 0; s < NK; ++s) mbar_init(smem_u32(&bars->k_full[s]), 1);
        for (int s = 0; s < NV; ++s) mbar_init(smem_u32(&bars->v_full[s]), 1);
        for (int b = 0; b < kSBuf; ++b) {
            mbar_init(smem_u32(&bars->s_full[b]), 1);
            mbar_init(smem_u32(&bars->p_full[b]), kSoftmax);
            mbar_init(smem_u32(&bars->o_done[b]), 1);  // PV_J with J % kSBuf == b retired
        }
        mbar_init(smem_u32(&bars->o_free), kSoftmax);
        for (int s = 0; s < kClc; ++s) {
            mbar_init(smem_u32(&bars->clc_full[s]), 1);
            mbar_init(smem_u32(&bars->clc_empty[s]), kWarps);
        }
        // the swizzled layout needs the 1024-byte alignment the declaration asks for
        bars->abort = (base & 1023u) ? 1 : *reinterpret_cast<volatile int*>(a.status);
        if (base & 1023u) atomicCAS(a.status, 0, 99);
        fence_mbar_init();
    }
    __syncthreads();
    if (bars->abort) return;  // an earlier CTA timed out: do nothing (no TMEM, no copies)
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    // Persistent CTAs (PERSIST; otherwise a CTA computes its own item only).  After its own
    // item (blockIdx.x) a CTA takes over the item of a CTA that has not started yet, by
    // cancelling that CTA's launch (cluster launch control), until none is left.  Items are
    // still taken in launch order, so the item order of fwd_item holds,
    // and an SM keeps its CTA, TMEM and pipelines across items: the next item's loads and
    // first MMAs overlap the current item's last tiles and its epilogue.  Every barrier
    // phase below counts the tiles J of all the CTA's items so far.
    // Response r (the CTA's item r + 1) lands in slot r % kClc.  Warp 0 requests it; every
    // warp reads it (lane 0 alone in the MMA issuer warps) and releases the slot.
    auto take_next = [&](int r, bool whole_warp) -> int {
        if (!PERSIST) return -1;
        const int s = r % kClc;
        int x = -1;
        if (mbar_wait(smem_u32(&bars->clc_full[s]), (r / kClc) & 1, abort, a.status, 11) && !*abort)
            x = clc_cancelled_x(clc_resp + s * 16);
        if (x >= (int)gridDim.x) {  // not an index of this grid: stop, and say so
            atomicCAS(a.status, 0, 15);
            x = -1;
        }
        fence_proxy_async_smem();  // the read is ordered before the slot's next (async-proxy) write
        if (whole_warp) x = __shfl_sync(0xffffffffu, x, 0);
        if (lane == 0) mbar_arrive(smem_u32(&bars->clc_empty[s]));
        return x;
    };

    if (warp == 0 || warp == 2) {
        // ---------------------------------------------------- TMA producers: warp 0 Q and K, warp 2 V
        // A rank-major tile (row0 / k0 >= 0) is a box of 128 consecutive rank-major rows,
        // loaded by lane 0.  A position tile (row0 / k0 < 0; short-chunk documents) holds
        // positions pos0 .. pos0+n-1, read in place from the rank-major buffer through
        // rm_of_global, in groups of 8 rows: lane l takes group l % 16 and the 64-column
        // boxes l / 16, l / 16 + 2, ...  The rows of a position tile are runs of consecutive
        // rows of the buffer, one per chunk.  An aligned block of 2^s groups (s = 4 .. 0)
        // that lies inside one run is one box of 8 << s rows, issued by the block's first
        // lane and landing at the block's 1024-byte-aligned offset, so that the swizzled
        // layout is the full box's; a group in no such block (it crosses a chunk boundary or
        // the tile's end) is two 4-row gathers (tile::gather4).  Rows past n repeat row n-1
        // (they are masked).
        const bool is_k = warp == 0;
        // this lane's group of 8 rows of a position tile (the indices are loaded one tile
        // ahead, so that the load latency overlaps the wait for a free stage)
        auto group_index = [&](int pos0, int n, int (&rr)[8]) {
            const int g8 = (lane & 15) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) rr[i] = __ldg(a.rm_of_global + pos0 + min(g8 + i, n - 1));
        };
        // 64-column boxes c0 .. c1-1 of those rows; a row r of the buffer is (r, head) of the
        // 3-D maps (full: 128-row boxes, runs[s]: 8 << s rows) and row r * heads + head of the
        // row map.  Called by the whole warp.
        auto load_groups = [&](const CUtensorMap* full, const CUtensorMap* runs, const CUtensorMap* rows,
                               uint32_t dst, uint32_t bar, const int (&rr)[8], int heads, int head, int c0, int c1) {
            const int g = lane & 15;
            bool run = true;
#pragma unroll
            for (int i = 1; i < 8; ++i) run = run && rr[i] == rr[0] + i;
            // bit g: group g is a run; bit g of link: group g+1 continues it (both halves of
            // the warp hold the same groups, so the low 16 bits say it all)
            const int next0 = __shfl_down_sync(0xffffffffu, rr[0], 1);
            const uint32_t is_run = __ballot_sync(0xffffffffu, run) & 0xffffu;
            const uint32_t link = __ballot_sync(0xffffffffu, run && next0 == rr[0] + 8) & (is_run >> 1) & 0x7fffu;
            int size = -1;  // log2 of the groups in this lane's box; -1: gathers; -2: covered by another lane
#pragma unroll
            for (int s = 4; s >= 0 && size == -1; --s) {
                const int n = 1 << s, b = g & ~(n - 1);
                const uint32_t need_run = ((1u << n) - 1u) << b, need_link = ((1u << (n - 1)) - 1u) << b;
                if ((is_run & need_run) == need_run && (link & need_link) == need_link) size = (g == b) ? s : -2;
            }
            const uint32_t gdst = dst + g * 1024;
            for (int c = c0 + (lane >> 4); c < c1; c += 2) {
                const uint32_t d = gdst + c * L::kBox;
                if (size >= 0) {
                    tma_load_3d(size == 4 ? full : runs + size, d, bar, (c - c0) * 64, head, rr[0]);
                } else if (size == -1) {
                    tma_gather4(rows, d, bar, (c - c0) * 64, rr[0] * heads + head, rr[1] * heads + head,
                                rr[2] * heads + head, rr[3] * heads + head);
                    tma_gather4(rows, d + 512, bar, (c - c0) * 64, rr[4] * heads + head, rr[5] * heads + head,
                                rr[6] * heads + head, rr[7] * heads + head);
                }
            }
        };
        // Where entry j's K/V rows come from: box_row >= 0 is the first row of one box of
        // 128 consecutive rows; otherwise this lane's group of 8 rows (rr).
        //   rank-major K/V (kv_global == 0): rank-major tiles are boxes at k0; position
        //   tiles take rank-major rows through rm_of_global.
        //   packed K/V (kv_global != 0; the gather of K/V fused into the loads): a run of
        //   consecutive positions is a box at kpos0; a rank-major run with a seam takes its
        //   positions.
        auto locate = [&](const int* E, int j, int (&rr)[8]) {
            const int4 lo = __ldg(reinterpret_cast<const int4*>(E + j * 8));  // k0, nvalid, kpos0, kbrk
            if (!a.kv_global) {
                if (lo.x < 0) group_index(lo.z, lo.y, rr);
                return lo.x;
            }
            const int kjump = __ldg(E + j * 8 + 4);
            if (lo.w >= lo.y || kjump == 0) return lo.z;
            const int g8 = (lane & 15) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = min(g8 + i, lo.y - 1);
                rr[i] = lo.z + t + (t >= lo.w ? kjump : 0);
            }
            return -1;
        };
        // warp 0 asks for the CTA's next item (response r) before it starts item r
        auto request = [&](int r) {
            const int s = r % kClc;
            if (r >= kClc &&
                !mbar_wait(smem_u32(&bars->clc_empty[s]), ((r / kClc) - 1) & 1, abort, a.status, 12))
                return;
            if (*abort) return;
            mbar_arrive_expect_tx(smem_u32(&bars->clc_full[s]), 16);
            clc_try_cancel(clc_resp + s * 16, smem_u32(&bars->clc_full[s]));
        };
        if (lane == 0) {
            if (is_k) {
                tma_prefetch_desc(&tm.q);
                tma_prefetch_desc(&tm.k);
                if (SHARED_ROPE) tma_prefetch_desc(&tm.kr);
                if (PERSIST) request(0);
            } else {
                tma_prefetch_desc(&tm.v);
            }
        }
        const int ns = is_k ? NK : NV;
        uint32_t J = 0;  // tiles of the CTA's earlier items
        int kq = 0;      // the CTA's earlier items with tiles
        FwdItem x = fwd_item(blockIdx.x, a);
        for (int it = blockIdx.x, r = 0; it >= 0; ++r) {
            const int nk = x.q2.x;
            const int* E = a.entries + (size_t)x.q2.y * 8;
            // The rows of the item's Q (a position tile) and of its first K/V tile are looked
            // up before the waits for a free buffer, so that their loads overlap the wait.
            int rq[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (is_k && nk > 0 && x.q0.z < 0) group_index(x.q1.x, x.q0.w, rq);
            int rr_next[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            int box_next = nk > 0 ? locate(E, 0, rr_next) : 0;
            if (is_k && nk > 0) {
                // One Q buffer, refilled once every S of the previous item has retired
                // (q_free, committed after that item's last S).  A second buffer measured no
                // faster: the reload hides behind the softmax of the previous item's last tiles.
                if (kq > 0) mbar_wait(smem_u32(&bars->q_free), (kq - 1) & 1, abort, a.status, 13);
                const uint32_t qf = smem_u32(&bars->q_full);
                if (lane == 0) mbar_arrive_expect_tx(qf, L::kQBytes);
                __syncwarp();
                if (x.q0.z >= 0) {
                    if (lane == 0)
                        for (int c = 0; c < DQK / 64; ++c) tma_load_3d(&tm.q, sQ + c * L::kBox, qf, c * 64, x.h, x.q0.z);
                } else {
                    load_groups(&tm.q, tm.qs, &tm.qg, sQ, qf, rq, a.hq, x.h, 0, DQK / 64);
                }
            }
            for (int j = 0; j < nk; ++j) {
                const uint32_t Jj = J + j;
                const int st = Jj % ns;
                const int box_row = box_next;
                int rr[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) rr[i] = rr_next[i];
                if (j + 1 < nk) box_next = locate(E, j + 1, rr_next);
                // A stage is refilled once the MMA that read it has retired: K_{J-NK} is
                // read by S_{J-NK} (signalled on s_full), V_{J-NV} by PV_{J-NV} (o_done).
                // NK, NV <= kSBuf, so the next use of either barrier needs the tile
                // being loaded here: the awaited phase is never ambiguous.
                if (is_k) {
                    if (Jj >= NK)
                        mbar_wait(smem_u32(&bars->s_full[(Jj - NK) % kSBuf]), ((Jj - NK) / kSBuf) & 1, abort,
                                  a.status, 1);
                    const uint32_t kf = smem_u32(&bars->k_full[st]);
                    if (lane == 0) mbar_arrive_expect_tx(kf, L::kKBytes);
                    __syncwarp();
                    if (box_row >= 0) {
                        if (lane == 0)
                            for (int c = 0; c < DQK / 64; ++c) {
                                if (SHARED_ROPE && c == 2)
                                    tma_load_3d(&tm.kr, sK + st * L::kKBytes + c * L::kBox, kf, 0, 0, box_row);
                                else
                                    tma_load_3d(&tm.k, sK + st * L::kKBytes + c * L::kBox, kf, c * 64, x.g, box_row);
                            }
                    } else if (SHARED_ROPE) {  // per-head part, then the shared rope key (one row per token)
                        load_groups(&tm.k, tm.ks, &tm.kg, sK + st * L::kKBytes, kf, rr, a.hkv, x.g, 0, 2);
                        load_groups(&tm.kr, tm.krs, &tm.krg, sK + st * L::kKBytes, kf, rr, 1, 0, 2, 3);
                    } else {
                        load_groups(&tm.k, tm.ks, &tm.kg, sK + st * L::kKBytes, kf, rr, a.hkv, x.g, 0, DQK / 64);
                    }
                } else {
                    if (Jj >= NV)
                        mbar_wait(smem_u32(&bars->o_done[(Jj - NV) % kSBuf]), ((Jj - NV) / kSBuf) & 1, abort,
                                  a.status, 9);
                    const uint32_t vf = smem_u32(&bars->v_full[st]);
                    if (lane == 0) mbar_arrive_expect_tx(vf, L::kVBytes);
                    __syncwarp();
                    if (box_row >= 0) {
                        if (lane == 0)
                            for (int c = 0; c < DV / 64; ++c)
                                tma_load_3d(&tm.v, sV + st * L::kVBytes + c * L::kBox, vf, c * 64, x.g, box_row);
                    } else {
                        load_groups(&tm.v, tm.vs, &tm.vg, sV + st * L::kVBytes, vf, rr, a.hkv, x.g, 0, DV / 64);
                    }
                }
            }
            J += nk;
            kq += nk > 0;
            it = take_next(r, true);
            if (PERSIST && is_k && lane == 0 && it >= 0) request(r + 1);
            if (it >= 0) x = fwd_item(it, a);
        }
    } else if (warp == 1 || warp == kPvWarp) {
        // ---------------------------------------------------- MMA issuers
        // Two issuing threads on different SMSPs keep the tensor pipe's short queue fed
        // while either of them waits or commits: warp 1 issues every S_J, warp kPvWarp
        // every PV_J.  Each waits only for what its own MMAs need:
        //   S_J:  Q of the item landed, K_J landed, and PV_{J-3} retired (S_J's TMEM
        //         buffer held P_{J-3}).  The next use of that o_done barrier is PV_J,
        //         which needs S_J: the awaited phase is unambiguous.
        //   PV_J: P_J released (which implies S_J retired) and V_J landed; the first PV
        //         of an item (which overwrites O) also waits until the previous item's
        //         epilogue has read O.
        if (lane == 0) {
            constexpr uint32_t dhi = smem_desc_hi_sw128(1024);
            uint32_t J = 0;
            int kq = 0;  // the CTA's earlier items with tiles: phases of q_full and o_free
            if (warp == 1) {
                constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false, false);
                const uint32_t qlo = smem_desc_lo(sQ, 16);
                for (int it = blockIdx.x, r = 0; it >= 0; ++r) {
                    const int nk = fwd_item(it, a).q2.x;
                    if (nk > 0) {
                        mbar_wait(smem_u32(&bars->q_full), kq & 1, abort, a.status, 2);
                        for (int j = 0; j < nk; ++j) {
                            const uint32_t Jj = J + j;
                            const int st = Jj % NK, b = Jj % kSBuf;
                            if (Jj >= kSBuf)
                                mbar_wait(smem_u32(&bars->o_done[b]), ((Jj - kSBuf) / kSBuf) & 1, abort, a.status, 10);
                            mbar_wait(smem_u32(&bars->k_full[st]), (Jj / NK) & 1, abort, a.status, 3);
                            tc_fence_after();
                            const uint32_t klo = smem_desc_lo(sK + st * L::kKBytes, 16);
                            const uint32_t dst = tmem + b * 128;
#pragma unroll
                            for (int kk = 0; kk < DQK / 16; ++kk) {
                                const uint32_t off = ((kk >> 2) * L::kBox + (kk & 3) * 32) >> 4;
                                mma_ss(dst, smem_desc_of(qlo + off, dhi), smem_desc_of(klo + off, dhi), idS, kk > 0);
                            }
                            mma_commit(smem_u32(&bars->s_full[b]));
                        }
                        mma_commit(smem_u32(&bars->q_free));  // the item's S MMAs no longer need Q
                        J += nk;
                        ++kq;
                    }
                    it = take_next(r, false);
                }
            } else {
                constexpr uint32_t idPV = idesc_bf16_f32(BM, DV, false, true);
                for (int it = blockIdx.x, r = 0; it >= 0; ++r) {
                    const int nk = fwd_item(it, a).q2.x;
                    if (nk > 0) {
                        if (kq > 0) mbar_wait(smem_u32(&bars->o_free), (kq - 1) & 1, abort, a.status, 14);
                        for (int j = 0; j < nk; ++j) {
                            const uint32_t Jj = J + j;
                            const int st = Jj % NV, b = Jj % kSBuf;
                            mbar_wait(smem_u32(&bars->p_full[b]), (Jj / kSBuf) & 1, abort, a.status, 4);
                            mbar_wait(smem_u32(&bars->v_full[st]), (Jj / NV) & 1, abort, a.status, 5);
                            tc_fence_after();
                            const uint32_t vlo = smem_desc_lo(sV + st * L::kVBytes, L::kBox);
                            const uint32_t pa = tmem + b * 128;
#pragma unroll
                            for (int kk = 0; kk < BN / 16; ++kk)
                                mma_ts(tmem + kTmemO, pa + kk * 8, smem_desc_of(vlo + kk * (2048 >> 4), dhi), idPV,
                                       (j > 0 || kk > 0));
                            mma_commit(smem_u32(&bars->o_done[b]));
                        }
                        J += nk;
                        ++kq;
                    }
                    it = take_next(r, false);
                }
            }
        }
    } else if (warp >= 3 && warp < 3 + kSoftmax / 32) {
        // ---------------------------------------------------- softmax warpgroups
        // Two warpgroups; thread (row, half) owns 64 of the row's 128 score columns
        // and DV/2 of its output columns.  Row maxima are combined through shared
        // memory once per tile (double-buffered); row sums once per item; the two
        // halves of a row meet on their pair barrier only.
        const int ct = threadIdx.x - 96;
        const int hf = ct >> 7;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const float sl2 = a.scale_log2;
        uint32_t J = 0;
        int it = blockIdx.x;
        FwdItem x = fwd_item(it, a);
        for (int r = 0; it >= 0; ++r) {
            const int h = x.h, row0 = x.q0.z, m = x.q0.w, qpos0 = x.q1.x, nk = x.q2.x;
            const int* E = a.entries + (size_t)x.q2.y * 8;
            const int qpos = qpos0 + row + (row >= x.q1.y ? x.q1.z : 0);
            float m_run = -INFINITY, l_run = 0.f;
            // entry record j+1 is fetched while entry j is processed
            int4 e_lo = make_int4(0, 0, 0, 0), e_hi = make_int4(0, 0, 0, 0);
            if (nk > 0) {
                e_lo = __ldg(reinterpret_cast<const int4*>(E));
                e_hi = __ldg(reinterpret_cast<const int4*>(E) + 1);
            }
            for (int j = 0; j < nk; ++j) {
                const uint32_t Jj = J + j;
                const int b = Jj % kSBuf, xb = Jj & 1;
                const int4 c_lo = e_lo, c_hi = e_hi;
                if (j + 1 < nk) {
                    e_lo = __ldg(reinterpret_cast<const int4*>(E + (j + 1) * 8));
                    e_hi = __ldg(reinterpret_cast<const int4*>(E + (j + 1) * 8) + 1);
                }
                // record: k0, nvalid, kpos0, kbrk | kjump, cls, ktile, key_rank
                const int nvalid = c_lo.y;
                int cnt = nvalid;
                if (c_hi.y != 2) cnt = visible_prefix(qpos, nvalid, c_lo.z, c_lo.w, c_hi.x);
                cnt -= hf * 64;  // visible columns within this thread's half
                mbar_wait(smem_u32(&bars->s_full[b]), (Jj / kSBuf) & 1, abort, a.status, 6);
                tc_fence_after();

                uint32_t sr[2][32];
#pragma unroll
                for (int c = 0; c < 2; ++c) tmem_ld32(tmem + lane_addr + b * 128 + hf * 64 + c * 32, sr[c]);
                tmem_wait_ld();
                if (__any_sync(0xffffffffu, cnt < 64)) {  // PARTIAL entry or short key run: mask
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int t = 0; t < 32; ++t)
                            if (c * 32 + t >= cnt) sr[c][t] = __float_as_uint(-INFINITY);
                }
                // Exponentials against the running max, with the tile's row max taken in the
                // same pass (the max runs on the ALU while the exponentials hold the XU).
                // Only when the max grows by more than 2^8 is the tile recomputed (rare).
                const float m_ref = (m_run == -INFINITY) ? 0.f : m_run;
                float pm[8], ps[8];
                uint32_t pk[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    pm[u] = -INFINITY;
                    ps[u] = 0.f;
                }
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int t = 0; t < 32; t += 2) {
                        const float s0 = __uint_as_float(sr[c][t]), s1 = __uint_as_float(sr[c][t + 1]);
                        pm[(t >> 1) & 7] = fmaxf(pm[(t >> 1) & 7], fmaxf(s0, s1));
                        const float p0 = ex2(fmaf(s0, sl2, -m_ref));
                        const float p1 = ex2(fmaf(s1, sl2, -m_ref));
                        ps[(t >> 1) & 7] += p0 + p1;
                        pk[c * 16 + (t >> 1)] = pack_bf16x2(p0, p1);
                    }
                const float pmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                         fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
                xch[(xb * 2 + hf) * 128 + row] = pmax;
                named_bar_sync(2 + wq, 64);  // both halves' scores are read and their maxima posted
                const float mx = fmaxf(pmax, xch[(xb * 2 + (hf ^ 1)) * 128 + row]) * sl2;
                const float m_new = fmaxf(m_run, mx);
                const bool grow = m_new > m_run + kRescaleThreshold;
                const float m_use = grow ? m_new : m_run;
                const float m_safe = (m_use == -INFINITY) ? 0.f : m_use;
                const float alpha = grow ? ex2(m_run - m_safe) : 1.f;
                if (__any_sync(0xffffffffu, grow)) {  // rare: redo this row's tile against the new max
                    if (grow) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
                        for (int c = 0; c < 2; ++c)
#pragma unroll
                            for (int t = 0; t < 32; t += 2) {
                                const float p0 = ex2(fmaf(__uint_as_float(sr[c][t]), sl2, -m_safe));
                                const float p1 = ex2(fmaf(__uint_as_float(sr[c][t + 1]), sl2, -m_safe));
                                ps[(t >> 1) & 7] += p0 + p1;
                                pk[c * 16 + (t >> 1)] = pack_bf16x2(p0, p1);
                            }
                    }
                }
                tmem_st32(tmem + lane_addr + b * 128 + hf * 32, pk);  // P as bf16 over S (read above)
                const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                l_run = l_run * alpha + sum;
                m_run = m_use;
                if (j >= 1 && __any_sync(0xffffffffu, grow)) {
                    // O is rescaled only once PV_{J-1} has retired.  The signal of S_J covers
                    // PV_{J-3} (S_J waited for it), so o_done of PV_{J-1}'s buffer is at most
                    // one use behind and its parity identifies the phase.
                    mbar_wait(smem_u32(&bars->o_done[(Jj - 1) % kSBuf]), ((Jj - 1) / kSBuf) & 1, abort, a.status, 7);
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < DV / 64; ++c) {
                        uint32_t o[32];
                        const uint32_t col = kTmemO + hf * (DV / 2) + c * 32;
                        tmem_ld32(tmem + lane_addr + col, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
                        tmem_st32(tmem + lane_addr + col, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&bars->p_full[b]));
            }
            // The next item's record is fetched while this item's last PV completes.
            it = take_next(r, true);
            if (it >= 0) x = fwd_item(it, a);
            // ---------------------------------------------------- epilogue
            // rank-major row of this query row (position tiles: through rm_of_global)
            const int orow_idx = row0 >= 0 ? row0 + row : (row < m ? __ldg(a.rm_of_global + qpos0 + row) : 0);
            __nv_bfloat16* orow = a.o + ((size_t)orow_idx * a.hq + h) * DV + hf * (DV / 2);
            if (nk == 0) {  // no key (never planned: every query sees itself)
                if (row < m) {
                    for (int c = 0; c < DV / 2; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
                    if (hf == 0) a.lse[(size_t)h * a.T + orow_idx] = -INFINITY;
                }
                continue;
            }
            const uint32_t Jl = J + nk - 1;  // the item's last tile
            J += nk;
            mbar_wait(smem_u32(&bars->o_done[Jl % kSBuf]), (Jl / kSBuf) & 1, abort, a.status, 8);
            tc_fence_after();
            // The sums go through the buffer of the last maxima: the next item's first tile
            // posts its maxima in the other one, and its second tile reaches this one only
            // after the pair barrier of the first, which both halves pass after reading here.
            const int xl = Jl & 1;
            named_bar_sync(2 + wq, 64);  // last maxima read before the buffer takes the sums
            xch[(xl * 2 + hf) * 128 + row] = l_run;
            named_bar_sync(2 + wq, 64);
            const float l_tot = l_run + xch[(xl * 2 + (hf ^ 1)) * 128 + row];
            const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
            uint32_t o[DV / 64][32];
#pragma unroll
            for (int c = 0; c < DV / 64; ++c) tmem_ld32(tmem + lane_addr + kTmemO + hf * (DV / 2) + c * 32, o[c]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->o_free));  // the next item's first PV may overwrite O
            // This thread's DV/2 = 64 output columns as bf16, in 16-byte chunks of 8 columns.
            uint4 ch[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t* s = o[q >> 2] + (q & 3) * 8;
                ch[q] = make_uint4(pack_bf16x2(__uint_as_float(s[0]) * inv_l, __uint_as_float(s[1]) * inv_l),
                                   pack_bf16x2(__uint_as_float(s[2]) * inv_l, __uint_as_float(s[3]) * inv_l),
                                   pack_bf16x2(__uint_as_float(s[4]) * inv_l, __uint_as_float(s[5]) * inv_l),
                                   pack_bf16x2(__uint_as_float(s[6]) * inv_l, __uint_as_float(s[7]) * inv_l));
            }
            // 8 x 8 transposes of the chunks within each group of 8 lanes (8 rows), by XOR
            // shuffles: afterwards lane i of a group holds chunk i of each of the group's rows,
            // so that one store instruction writes four whole 128-byte half rows instead of
            // 32 scattered 16-byte pieces (rows are hq * DV * 2 bytes apart).
            const int gi = lane & 7;
#pragma unroll
            for (int k = 4; k >= 1; k >>= 1) {
                const bool up = (gi & k) != 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j & k) continue;
                    uint4 x = up ? ch[j] : ch[j | k];
                    x.x = __shfl_xor_sync(0xffffffffu, x.x, k);
                    x.y = __shfl_xor_sync(0xffffffffu, x.y, k);
                    x.z = __shfl_xor_sync(0xffffffffu, x.z, k);
                    x.w = __shfl_xor_sync(0xffffffffu, x.w, k);
                    if (up)
                        ch[j] = x;
                    else
                        ch[j | k] = x;
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int src = (lane & ~7) + j;  // the lane of row 8 * group + j
                const unsigned long long p =
                    __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(orow), src);
                if (wq * 32 + src < m) *(reinterpret_cast<uint4*>(p) + gi) = ch[j];
            }
            if (row < m && hf == 0)
                a.lse[(size_t)h * a.T + orow_idx] = (m_run + __log2f(l_tot)) * 0.69314718055994530942f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int DQK, int DV, bool SHARED_ROPE, bool PERSIST>
int launch_as(const FwdMaps& m, const FwdArgs& a, int n_items, cudaStream_t stream) {
    using L = FwdLayout<DQK, DV>;
    static std::atomic<uint64_t> configured{0};
    if (!ensure_dynamic_smem(fwd_kernel<DQK, DV, SHARED_ROPE, PERSIST>, L::kDynSmem, configured)) return -1;
    fwd_kernel<DQK, DV, SHARED_ROPE, PERSIST><<<n_items, kThreads, L::kDynSmem, stream>>>(m, a);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int DQK, int DV, bool SHARED_ROPE>
int launch(const FwdMaps& m, const FwdArgs& a, int n_items, cudaStream_t stream) {
    return a.persistent ? launch_as<DQK, DV, SHARED_ROPE, true>(m, a, n_items, stream)
                        : launch_as<DQK, DV, SHARED_ROPE, false>(m, a, n_items, stream);
}

}  // namespace

int launch_fwd_sm100(int dqk, int dv, const FwdMaps& m, const FwdArgs& a, int n_items, cudaStream_t stream) {
    if (dqk == 128 && dv == 128) return launch<128, 128, false>(m, a, n_items, stream);
    if (dqk == 192 && dv == 128) return launch<192, 128, false>(m, a, n_items, stream);
    return -2;
}

int launch_fwd_mla_sm100(const FwdMaps& m, const FwdArgs& a, int n_items, cudaStream_t stream) {
    return launch<192, 128, true>(m, a, n_items, stream);
}

}  // namespace thd

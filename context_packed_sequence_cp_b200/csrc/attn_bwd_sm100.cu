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
//   bwd_prep   Delta_i = sum_d dO_id O_id per (row, head), and dQ := 0.
//   bwd_kernel one CTA per (key tile, key/value head g), key tiles in longest-first
//              order; it walks every query head of g's group and every query tile
//              that lists the key tile (the plan's key-tile transpose).  Per step,
//              with key rows on TMEM lanes:
//                a  S^T  = K Q^T            (tcgen05, smem x smem)  -> TMEM A
//                b  dP^T = V dO^T           (tcgen05, smem x smem)  -> TMEM B
//                   P^T = exp(S^T - lse), dS^T = P^T (dP^T - Delta), masked on
//                   PARTIAL entries and ragged tiles; P^T, dS^T as bf16 over dP^T
//                   in TMEM, dS (bf16) into shared memory
//                c  dV  += P^T dO           (A from TMEM)
//                d  dK  += dS^T Q           (A from TMEM)
//                e  dQp  = dS K             (smem x smem)            -> TMEM A
//              and dQp is added to the fp32 dQ in global memory with vector
//              reductions.  Query tiles are walked outer and the group's heads
//              inner, so CTAs of one group reach the same dQ tiles close together
//              in time and their reductions meet in L2.  dK, dV stay in TMEM for
//              the whole walk and are written once.
// Warp roles (320 threads): warp 0 producer (TMA of K, V once and of Q, dO per step
// into a two-stage ring; its lanes also stage the step's lse and Delta in shared
// memory), warp 1 TMEM owner and MMA issuer, warps 2-9 two compute warpgroups,
// each owning half of the 128 columns of every TMEM row.
// TMEM columns: A [0,128) S^T, then P^T (0..63) and dS^T (64..127) as packed bf16;
// B [128,256) dP^T, then dQp; dK [256,384); dV [384,512).
// Schedule per step: the compute warpgroups form P^T as soon as S^T is in TMEM
// (phase 1), and dS^T once dP^T is (phase 2); c, d, e follow; S^T of the next step
// is issued right behind c and d, dP^T of the next step as soon as dQp has been
// read out, so the exponentials of a step overlap the tensor work of the last.
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace thd {
namespace {

constexpr int kD = 128;                 // head dim built (Dqk = Dv = 128)
constexpr int kThreads = 320;
constexpr int kCompute = 256;           // threads of the two compute warpgroups
constexpr uint32_t kTmemCols = 512;
constexpr int kBox = 128 * 128;         // one 64-column x 128-row bf16 box, 16 KB
constexpr int kTile = 2 * kBox;         // 128 x 128 bf16 tile, 32 KB

struct BwdLayout {
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kTile;
    static constexpr int kOffQ = kOffV + kTile;       // 2 stages
    static constexpr int kOffDO = kOffQ + 2 * kTile;  // 2 stages
    static constexpr int kOffDS = kOffDO + 2 * kTile;
    static constexpr int kOffStat = kOffDS + kTile;   // 2 stages x (lse2[128], delta[128])
    static constexpr int kOffBar = kOffStat + 2 * 256 * 4;
    static constexpr int kBytes = kOffBar + 256;
    static constexpr int kDynSmem = kBytes;           // base is 1024-aligned by declaration (checked)
    static_assert(kDynSmem <= 232448, "shared memory budget");
};

struct BwdBars {
    uint64_t kv_full, qdo_full[2], qdo_empty[2], s_full, dp_full, ds_ready, dq_full, dq_free, acc_done;
    uint32_t tmem_base;
    int abort;
};

// Per-step metadata: the listed (query tile, entry) pair and the fields the step needs.
struct StepMeta {
    int row0, m, qpos0, qbrk, qjump, nvalid, cls;
};
__device__ __forceinline__ StepMeta load_meta(const BwdArgs& a, int list_pos) {
    const int2 pr = __ldg(reinterpret_cast<const int2*>(a.kt_list) + list_pos);
    const int4 q = __ldg(reinterpret_cast<const int4*>(a.qtiles + (size_t)pr.x * 12));      // r, d, row0, m
    const int4 q2 = __ldg(reinterpret_cast<const int4*>(a.qtiles + (size_t)pr.x * 12) + 1); // qpos0, qbrk, qjump, qmax
    const int4 e0 = __ldg(reinterpret_cast<const int4*>(a.entries + (size_t)pr.y * 8));     // k0, nvalid, ..
    const int4 e1 = __ldg(reinterpret_cast<const int4*>(a.entries + (size_t)pr.y * 8) + 1); // kjump, cls, ..
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

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// ---------------------------------------------------------------- prep
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       float* __restrict__ delta, float4* __restrict__ dq,
                                                       int64_t rows, int hq, int64_t T, int64_t dq_vec4) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * 8;
    for (int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); w < rows; w += nwarps) {
        // w = row * hq + h, rows of kD bf16 values: 4 per lane
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
        if (lane == 0) {
            const int64_t row = w / hq;
            const int h = (int)(w % hq);
            delta[(int64_t)h * T + row] = s;
        }
    }
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < dq_vec4; i += (int64_t)gridDim.x * blockDim.x)
        dq[i] = z;
}

// ---------------------------------------------------------------- main kernel
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, BwdArgs a) {
    using L = BwdLayout;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    BwdBars* bars = reinterpret_cast<BwdBars*>(smem_raw + L::kOffBar);
    float* s_stat = reinterpret_cast<float*>(smem_raw + L::kOffStat);  // [stage][lse2 128 | delta 128]
    const uint32_t sK = base + L::kOffK, sV = base + L::kOffV, sQ = base + L::kOffQ, sDO = base + L::kOffDO,
                   sDS = base + L::kOffDS;
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = a.hq / a.hkv;
    const int kt = a.kt_lpt[blockIdx.x / a.hkv];
    const int g = blockIdx.x % a.hkv;
    const int* KT = a.qtiles + (size_t)kt * 12;  // key tiles are the plan's row tiles
    const int k0 = KT[2], kn = KT[3];
    const int l0 = a.kt_off[kt], llen = a.kt_off[kt + 1] - l0;
    const int n_it = group * llen;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->kv_full), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&bars->qdo_full[s]), 1 + 32);  // expect_tx arrival + the warp's lse/Delta stores
            mbar_init(smem_u32(&bars->qdo_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->dp_full), 1);
        mbar_init(smem_u32(&bars->ds_ready), kCompute);
        mbar_init(smem_u32(&bars->dq_full), 1);
        mbar_init(smem_u32(&bars->dq_free), kCompute);
        mbar_init(smem_u32(&bars->acc_done), 1);
        // the layout needs the 1024-byte alignment the declaration asks for (swizzle atoms)
        bars->abort = (base & 1023u) ? 1 : *reinterpret_cast<volatile int*>(a.status);
        if (base & 1023u) atomicCAS(a.status, 0, 99);
        fence_mbar_init();
    }
    __syncthreads();
    if (bars->abort) return;  // misaligned, or an earlier CTA timed out: do nothing
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t tA = tmem, tB = tmem + 128, tDK = tmem + 256, tDV = tmem + 384;

    if (warp == 0) {
        // ---------------------------------------------------- producer warp
        // lane 0 issues the TMA copies; all 32 lanes stage lse (base 2) and Delta of
        // the step's 128 query rows, so no compute thread waits on global memory.
        const float log2e = 1.4426950408889634f;
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            const uint32_t kvf = smem_u32(&bars->kv_full);
            mbar_arrive_expect_tx(kvf, 2 * kTile);
            for (int c = 0; c < 2; ++c) {
                tma_load_3d(&tmK, sK + c * kBox, kvf, c * 64, g, k0);
                tma_load_3d(&tmV, sV + c * kBox, kvf, c * 64, g, k0);
            }
        }
        StepMeta cur = load_meta(a, l0), nxt = cur;
        if (llen > 1) nxt = load_meta(a, l0 + 1);
        for (int it = 0; it < n_it; ++it) {
            const int st = it & 1;
            const int pos = it / group, hh = it - pos * group;   // query tiles outer, heads inner
            if (hh == 0 && it > 0) {
                cur = nxt;
                if (pos + 1 < llen) nxt = load_meta(a, l0 + pos + 1);
            }
            const int h = g * group + hh;
            const int row0 = cur.row0;
            float lv[4], dv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t row = (int64_t)row0 + lane + 32 * u;
                lv[u] = row < a.T ? __ldg(a.lse + (int64_t)h * a.T + row) * log2e : 0.f;
                dv[u] = row < a.T ? __ldg(a.delta + (int64_t)h * a.T + row) : 0.f;
            }
            if (it >= 2) mbar_wait(smem_u32(&bars->qdo_empty[st]), ((it >> 1) - 1) & 1, abort, a.status, 11);
            const uint32_t f = smem_u32(&bars->qdo_full[st]);
            if (lane == 0) {
                mbar_arrive_expect_tx(f, 2 * kTile);
                for (int c = 0; c < 2; ++c) {
                    tma_load_3d(&tmQ, sQ + st * kTile + c * kBox, f, c * 64, h, row0);
                    tma_load_3d(&tmDO, sDO + st * kTile + c * kBox, f, c * 64, h, row0);
                }
            }
            float* stat = s_stat + st * 256;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                stat[lane + 32 * u] = lv[u];
                stat[128 + lane + 32 * u] = dv[u];
            }
            mbar_arrive(f);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idKK = idesc_bf16_f32(128, 128, false, false);  // A, B K-major
            constexpr uint32_t idTM = idesc_bf16_f32(128, 128, false, true);   // A TMEM, B MN-major
            constexpr uint32_t idMM = idesc_bf16_f32(128, 128, true, true);    // A, B MN-major
            auto issue_s = [&](int st) {  // a: S^T = K Q^T -> A
                const uint32_t q = sQ + st * kTile;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    mma_ss(tA, smem_desc_sw128(sK + off, 16, 1024), smem_desc_sw128(q + off, 16, 1024), idKK, kk > 0);
                }
                mma_commit(smem_u32(&bars->s_full));
            };
            auto issue_dp = [&](int st) {  // b: dP^T = V dO^T -> B
                const uint32_t d = sDO + st * kTile;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    mma_ss(tB, smem_desc_sw128(sV + off, 16, 1024), smem_desc_sw128(d + off, 16, 1024), idKK, kk > 0);
                }
                mma_commit(smem_u32(&bars->dp_full));
            };
            mbar_wait(smem_u32(&bars->kv_full), 0, abort, a.status, 12);
            mbar_wait(smem_u32(&bars->qdo_full[0]), 0, abort, a.status, 13);
            tc_fence_after();
            issue_s(0);
            issue_dp(0);
            for (int it = 0; it < n_it; ++it) {
                const int st = it & 1;
                const uint32_t q = sQ + st * kTile, d = sDO + st * kTile;
                mbar_wait(smem_u32(&bars->ds_ready), it & 1, abort, a.status, 15);
                tc_fence_after();
                // c: dV += P^T dO ; d: dK += dS^T Q  (A operands from region A)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tDV, tA + kk * 8, smem_desc_sw128(d + kk * 2048, kBox, 1024), idTM, (it > 0 || kk > 0));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tDK, tA + 64 + kk * 8, smem_desc_sw128(q + kk * 2048, kBox, 1024), idTM, (it > 0 || kk > 0));
                // e: dQp = dS K -> B (dP^T there was consumed before ds_ready)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tB, smem_desc_sw128(sDS + kk * 2048, kBox, 1024), smem_desc_sw128(sK + kk * 2048, kBox, 1024),
                           idMM, kk > 0);
                mma_commit(smem_u32(&bars->dq_full));
                if (it + 2 < n_it) mma_commit(smem_u32(&bars->qdo_empty[st]));
                if (it + 1 < n_it) {
                    const int sn = (it + 1) & 1;
                    mbar_wait(smem_u32(&bars->qdo_full[sn]), ((it + 1) >> 1) & 1, abort, a.status, 13);
                    tc_fence_after();
                    issue_s(sn);  // region A is rewritten only after c and d have read it (issue order)
                    mbar_wait(smem_u32(&bars->dq_free), it & 1, abort, a.status, 14);
                    tc_fence_after();
                    issue_dp(sn);
                }
            }
            mma_commit(smem_u32(&bars->acc_done));
        }
    } else {
        // ---------------------------------------------------- compute warpgroups
        const int ct = threadIdx.x - 64;         // 0..255
        const int hf = ct >> 7;                  // column half
        const int wq = warp & 3;
        const int r = wq * 32 + lane;            // TMEM lane: key row (phases 1-2), query row (dQ)
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const float sl2 = a.scale_log2;
        const int kbrk_t = KT[5], kjump_t = KT[6];
        const int kpos_r = KT[4] + r + (r >= kbrk_t ? kjump_t : 0);
        StepMeta cur = load_meta(a, l0), nxt = cur;
        if (llen > 1) nxt = load_meta(a, l0 + 1);
        for (int it = 0; it < n_it; ++it) {
            const int st = it & 1;
            const int pos = it / group, hh = it - pos * group;       // query tiles outer, heads inner
            if (hh == 0 && it > 0) {
                cur = nxt;
                if (pos + 1 < llen) nxt = load_meta(a, l0 + pos + 1);
            }
            const int h = g * group + hh;
            const int row0 = cur.row0, m = cur.m, qpos0 = cur.qpos0, qbrk = cur.qbrk, qjump = cur.qjump;

            // visible query columns of this key row: a suffix [lo, m) of the tile
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

            // ---- phase 1: P^T = exp(S^T - lse) on this thread's 64 query columns
            mbar_wait(smem_u32(&bars->qdo_full[st]), (it >> 1) & 1, abort, a.status, 16);  // lse/Delta staged
            mbar_wait(smem_u32(&bars->s_full), it & 1, abort, a.status, 16);
            tc_fence_after();
            float p[64];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t sv[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(tA + lane_addr + c0, sv);
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
            named_bar_sync(1, kCompute);  // every S^T read of region A is done before P^T overwrites it
            {
                uint32_t pk[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) pk[t] = pack_bf16x2(p[2 * t], p[2 * t + 1]);
                tmem_st32(tA + lane_addr + hf * 32, pk);
            }

            // ---- phase 2: dS^T = P^T (dP^T - Delta)
            mbar_wait(smem_u32(&bars->dp_full), it & 1, abort, a.status, 17);
            tc_fence_after();
            uint32_t dk[32];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t dpv[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(tB + lane_addr + c0, dpv);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 32; t += 4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(stat + 128 + c0 + t);
                    const float dq4[4] = {d4.x, d4.y, d4.z, d4.w};
                    float ds[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) ds[u] = p[ch * 32 + t + u] * (__uint_as_float(dpv[t + u]) - dq4[u]);
                    dk[ch * 16 + t / 2] = pack_bf16x2(ds[0], ds[1]);
                    dk[ch * 16 + t / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
                }
            }
            tmem_st32(tA + lane_addr + 64 + hf * 32, dk);
            // dS (query-major for the dQ product): rows = key r, 128-byte swizzled
            {
                const uint32_t rowb = sDS + hf * kBox + r * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(rowb + ((c ^ (r & 7)) << 4), dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
            }
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->ds_ready));

            // ---- dQp rows (TMEM lane = query row r) into the fp32 dQ
            mbar_wait(smem_u32(&bars->dq_full), it & 1, abort, a.status, 18);
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t q[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(tB + lane_addr + c0, q);
                tmem_wait_ld();
                if (r < m) {
                    float* dst = a.dq_acc + ((int64_t)(row0 + r) * a.hq + h) * kD + c0;
#pragma unroll
                    for (int t = 0; t < 32; t += 4)
                        red_add_v4(dst + t, __uint_as_float(q[t]) * a.scale, __uint_as_float(q[t + 1]) * a.scale,
                                   __uint_as_float(q[t + 2]) * a.scale, __uint_as_float(q[t + 3]) * a.scale);
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&bars->dq_free));
        }
        // ---------------------------------------------------- dK, dV epilogue
        mbar_wait(smem_u32(&bars->acc_done), 0, abort, a.status, 19);
        tc_fence_after();
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const uint32_t src = which == 0 ? tDK : tDV;
            float* out = which == 0 ? a.dk : a.dv;
            const float mul = which == 0 ? a.scale : 1.f;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t v[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(src + lane_addr + c0, v);
                tmem_wait_ld();
                if (r < kn) {
                    float4* dst = reinterpret_cast<float4*>(out + ((int64_t)(k0 + r) * a.hkv + g) * kD + c0);
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        dst[t] = make_float4(__uint_as_float(v[4 * t]) * mul, __uint_as_float(v[4 * t + 1]) * mul,
                                             __uint_as_float(v[4 * t + 2]) * mul, __uint_as_float(v[4 * t + 3]) * mul);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

int launch_bwd_sm100(int dqk, int dv, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                     const CUtensorMap& dout, const BwdArgs& a, int n_ktiles, int num_sms, cudaStream_t stream) {
    if (dqk != kD || dv != kD) return -2;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdLayout::kDynSmem) !=
            cudaSuccess)
            return -1;
        configured = true;
    }
    const int64_t rows = a.T * a.hq;
    const int64_t dq_vec4 = a.T * a.hq * kD / 4;
    bwd_prep_kernel<<<num_sms * 8, 256, 0, stream>>>(a.o, a.dout, a.delta, reinterpret_cast<float4*>(a.dq_acc),
                                                     rows, a.hq, a.T, dq_vec4);
    if (cudaGetLastError() != cudaSuccess) return -1;
    const int64_t ctas = (int64_t)n_ktiles * a.hkv;
    bwd_kernel<<<(unsigned)ctas, kThreads, BwdLayout::kDynSmem, stream>>>(q, k, v, dout, a);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace thd

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
//              reductions.  dK, dV stay in TMEM for the whole walk and are written
//              once.
// Warp roles (320 threads): warp 0 TMA producer (K, V once; Q, dO per step in a
// two-stage ring), warp 1 TMEM owner and MMA issuer, warps 2-9 two compute
// warpgroups, each owning half of the 128 columns of every TMEM row.
// TMEM columns: A [0,128) S^T then dQp; B [128,256) dP^T then P^T (128..191) and
// dS^T (192..255) as packed bf16; dK [256,384); dV [384,512).
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
    static constexpr int kOffStat = kOffDS + kTile;   // lse2[128], delta[128]
    static constexpr int kOffBar = kOffStat + 1024;
    static constexpr int kBytes = kOffBar + 256;
    static constexpr int kDynSmem = kBytes + 1024;    // slack for 1024-byte alignment
    static_assert(kDynSmem <= 232448, "shared memory budget");
};

struct BwdBars {
    uint64_t kv_full, qdo_full[2], qdo_empty[2], s_full, dp_full, ds_ready, dq_full, dq_free, acc_done;
    uint32_t tmem_base;
    int abort;
};

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
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    BwdBars* bars = reinterpret_cast<BwdBars*>(gbase + L::kOffBar);
    float* s_lse = reinterpret_cast<float*>(gbase + L::kOffStat);
    float* s_delta = s_lse + 128;
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
            mbar_init(smem_u32(&bars->qdo_full[s]), 1);
            mbar_init(smem_u32(&bars->qdo_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->dp_full), 1);
        mbar_init(smem_u32(&bars->ds_ready), kCompute);
        mbar_init(smem_u32(&bars->dq_full), 1);
        mbar_init(smem_u32(&bars->dq_free), kCompute);
        mbar_init(smem_u32(&bars->acc_done), 1);
        bars->abort = *reinterpret_cast<volatile int*>(a.status);
        fence_mbar_init();
    }
    __syncthreads();
    if (bars->abort) return;  // an earlier CTA timed out: do nothing
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
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
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
            for (int it = 0; it < n_it; ++it) {
                const int st = it & 1;
                if (it >= 2) mbar_wait(smem_u32(&bars->qdo_empty[st]), ((it >> 1) - 1) & 1, abort, a.status, 11);
                const int h = g * group + it / llen;
                const int qt = a.kt_list[2 * (l0 + it % llen)];
                const int row0 = a.qtiles[(size_t)qt * 12 + 2];
                const uint32_t f = smem_u32(&bars->qdo_full[st]);
                mbar_arrive_expect_tx(f, 2 * kTile);
                for (int c = 0; c < 2; ++c) {
                    tma_load_3d(&tmQ, sQ + st * kTile + c * kBox, f, c * 64, h, row0);
                    tma_load_3d(&tmDO, sDO + st * kTile + c * kBox, f, c * 64, h, row0);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            constexpr uint32_t idKK = idesc_bf16_f32(128, 128, false, false);  // A, B K-major
            constexpr uint32_t idTM = idesc_bf16_f32(128, 128, false, true);   // A TMEM, B MN-major
            constexpr uint32_t idMM = idesc_bf16_f32(128, 128, true, true);    // A, B MN-major
            mbar_wait(smem_u32(&bars->kv_full), 0, abort, a.status, 12);
            tc_fence_after();
            for (int it = 0; it < n_it; ++it) {
                const int st = it & 1;
                const uint32_t q = sQ + st * kTile, d = sDO + st * kTile;
                mbar_wait(smem_u32(&bars->qdo_full[st]), (it >> 1) & 1, abort, a.status, 13);
                tc_fence_after();
                // b: dP^T = V dO^T  (region B held P^T / dS^T of the previous step, consumed in order)
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    mma_ss(tB, smem_desc_sw128(sV + off, 16, 1024), smem_desc_sw128(d + off, 16, 1024), idKK, kk > 0);
                }
                mma_commit(smem_u32(&bars->dp_full));
                // a: S^T = K Q^T into region A, once the previous dQp has been read out
                if (it >= 1) mbar_wait(smem_u32(&bars->dq_free), (it - 1) & 1, abort, a.status, 14);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    mma_ss(tA, smem_desc_sw128(sK + off, 16, 1024), smem_desc_sw128(q + off, 16, 1024), idKK, kk > 0);
                }
                mma_commit(smem_u32(&bars->s_full));
                mbar_wait(smem_u32(&bars->ds_ready), it & 1, abort, a.status, 15);
                tc_fence_after();
                // c: dV += P^T dO ; d: dK += dS^T Q ; e: dQp = dS K
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tDV, tB + kk * 8, smem_desc_sw128(d + kk * 2048, kBox, 1024), idTM, (it > 0 || kk > 0));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tDK, tB + 64 + kk * 8, smem_desc_sw128(q + kk * 2048, kBox, 1024), idTM, (it > 0 || kk > 0));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tA, smem_desc_sw128(sDS + kk * 2048, kBox, 1024), smem_desc_sw128(sK + kk * 2048, kBox, 1024),
                           idMM, kk > 0);
                mma_commit(smem_u32(&bars->dq_full));
                if (it + 2 < n_it) mma_commit(smem_u32(&bars->qdo_empty[st]));
            }
            mma_commit(smem_u32(&bars->acc_done));
        }
    } else {
        // ---------------------------------------------------- compute warpgroups
        const int ct = threadIdx.x - 64;         // 0..255
        const int hf = ct >> 7;                  // column half
        const int wq = warp & 3;
        const int r = wq * 32 + lane;            // TMEM lane: key row (softmax), query row (dQ)
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const float sl2 = a.scale_log2;
        const float log2e = 1.4426950408889634f;
        const int kbrk_t = KT[5], kjump_t = KT[6];
        const int kpos_r = KT[4] + r + (r >= kbrk_t ? kjump_t : 0);
        for (int it = 0; it < n_it; ++it) {
            const int h = g * group + it / llen;
            const int qt = a.kt_list[2 * (l0 + it % llen)];
            const int e = a.kt_list[2 * (l0 + it % llen) + 1];
            const int* QT = a.qtiles + (size_t)qt * 12;
            const int row0 = QT[2], m = QT[3], qpos0 = QT[4], qbrk = QT[5], qjump = QT[6];
            const int* E = a.entries + (size_t)e * 8;
            const int nvalid = E[1], cls = E[5];

            // stage lse (base 2) and Delta of the step's 128 query rows
            named_bar_sync(1, kCompute);
            {
                const int i = ct & 127;
                const int64_t row = row0 + i;
                float v = 0.f;
                if (row < a.T) v = (ct < 128) ? a.lse[(int64_t)h * a.T + row] * log2e : a.delta[(int64_t)h * a.T + row];
                if (ct < 128) s_lse[i] = v; else s_delta[i] = v;
            }
            named_bar_sync(1, kCompute);

            // visible query columns of this key row: a suffix [lo, m) of the tile
            int lo = 0, hi = m;
            if (r >= nvalid) hi = 0;
            else if (cls != 2) {
                // first query row whose position reaches kpos_r
                const int n1 = min(qbrk, m);
                if (kpos_r <= qpos0) lo = 0;
                else if (kpos_r - qpos0 < n1) lo = kpos_r - qpos0;
                else {
                    const int p1 = qpos0 + qbrk + qjump;   // position of row qbrk
                    lo = (kpos_r <= p1) ? n1 : min(m, n1 + (kpos_r - p1));
                }
            }

            mbar_wait(smem_u32(&bars->s_full), it & 1, abort, a.status, 16);
            mbar_wait(smem_u32(&bars->dp_full), it & 1, abort, a.status, 17);
            tc_fence_after();
            uint32_t pk[32], dk[32];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t s[32], dp[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(tA + lane_addr + c0, s);
                tmem_ld32(tB + lane_addr + c0, dp);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 32; t += 2) {
                    const int i0 = c0 + t, i1 = c0 + t + 1;
                    float p0 = ex2(fmaf(__uint_as_float(s[t]), sl2, -s_lse[i0]));
                    float p1 = ex2(fmaf(__uint_as_float(s[t + 1]), sl2, -s_lse[i1]));
                    p0 = (i0 >= lo && i0 < hi) ? p0 : 0.f;
                    p1 = (i1 >= lo && i1 < hi) ? p1 : 0.f;
                    const float d0 = p0 * (__uint_as_float(dp[t]) - s_delta[i0]);
                    const float d1 = p1 * (__uint_as_float(dp[t + 1]) - s_delta[i1]);
                    pk[ch * 16 + t / 2] = pack_bf16x2(p0, p1);
                    dk[ch * 16 + t / 2] = pack_bf16x2(d0, d1);
                }
            }
            // both warpgroups have read dP^T before either overwrites region B
            named_bar_sync(1, kCompute);
            tmem_st32(tB + lane_addr + hf * 32, pk);
            tmem_st32(tB + lane_addr + 64 + hf * 32, dk);
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

            // dQp rows (TMEM lane = query row r) into the fp32 dQ
            mbar_wait(smem_u32(&bars->dq_full), it & 1, abort, a.status, 18);
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t q[32];
                const int c0 = hf * 64 + ch * 32;
                tmem_ld32(tA + lane_addr + c0, q);
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

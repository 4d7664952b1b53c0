// Forward causal attention in fp32 on the SIMT cores: the exact-precision path.
//
// Same method and metadata as the tensor-core forward (MindSpeed pull request
// #3820, "feat: kvallgather cp thd load balance", section "What this PR does /
// why we need it?": one call over every rank and document, K/V read in place in
// the rank-major layout, cached tile metadata; section "Does this PR introduce any
// user-facing change?": causal attention with EOD reset).  fp32 inputs rule out
// bf16/tf32 tensor-core products for a 1e-5 bound, so every product here is an
// fp32 FMA.
//
// One CTA per (query tile, query head) work item, one query row per thread; each
// listed K/V entry is staged in shared memory and every thread runs an online
// softmax over the prefix of keys its row can see (positions increase along an
// entry, so the visible keys are a prefix).
#include "kernels.h"

namespace thd {
namespace {

constexpr int BM = 128, BN = 128;

__device__ __forceinline__ int visible_prefix_f32(int qpos, int nvalid, int kpos0, int kbrk, int kjump) {
    if (qpos < kpos0) return 0;
    const int a = min(kbrk, qpos - kpos0 + 1);
    if (a < kbrk || kbrk >= nvalid) return min(a, nvalid);
    const int b0 = kpos0 + kbrk + kjump;
    if (qpos < b0) return kbrk;
    return min(nvalid, kbrk + (qpos - b0 + 1));
}

template <int DQK, int DV>
__global__ void __launch_bounds__(BM) fwd_f32_kernel(FwdF32Args a) {
    extern __shared__ float sm[];
    float* sk = sm;             // [BN][DQK]
    float* sv = sm + BN * DQK;  // [BN][DV]
    const int item = blockIdx.x;
    const int qt = a.lpt[item / a.hq];
    const int h = item % a.hq;
    const int g = h / (a.hq / a.hkv);
    const int* Q = a.qtiles + (size_t)qt * 12;
    const int row0 = Q[2], m = Q[3], qpos0 = Q[4], qbrk = Q[5], qjump = Q[6], nk = Q[8], e0 = Q[9];
    const int row = threadIdx.x;
    const int qpos = qpos0 + row + (row >= qbrk ? qjump : 0);
    const bool live = row < m;

    float q[DQK], o[DV];
    if (live) {
        const float* qr = a.q + ((size_t)(row0 + row) * a.hq + h) * DQK;
#pragma unroll
        for (int d = 0; d < DQK; ++d) q[d] = qr[d];
    }
#pragma unroll
    for (int d = 0; d < DV; ++d) o[d] = 0.f;
    float mrun = -INFINITY, l = 0.f;

    for (int j = 0; j < nk; ++j) {
        const int* e = a.entries + (size_t)(e0 + j) * 8;
        const int k0 = e[0], nvalid = e[1];
        __syncthreads();
        for (int i = threadIdx.x; i < nvalid * (DQK / 4); i += BM) {
            const int t = i / (DQK / 4), c = i % (DQK / 4);
            reinterpret_cast<float4*>(sk)[i] =
                reinterpret_cast<const float4*>(a.k + ((size_t)(k0 + t) * a.hkv + g) * DQK)[c];
        }
        for (int i = threadIdx.x; i < nvalid * (DV / 4); i += BM) {
            const int t = i / (DV / 4), c = i % (DV / 4);
            reinterpret_cast<float4*>(sv)[i] =
                reinterpret_cast<const float4*>(a.v + ((size_t)(k0 + t) * a.hkv + g) * DV)[c];
        }
        __syncthreads();
        if (!live) continue;
        const int cnt = (e[5] == 2) ? nvalid : visible_prefix_f32(qpos, nvalid, e[2], e[3], e[4]);
        for (int t = 0; t < cnt; ++t) {
            float s = 0.f;
#pragma unroll
            for (int d = 0; d < DQK; ++d) s = fmaf(q[d], sk[t * DQK + d], s);
            s *= a.scale;
            if (s > mrun) {
                const float corr = expf(mrun - s);
                l *= corr;
#pragma unroll
                for (int d = 0; d < DV; ++d) o[d] *= corr;
                mrun = s;
            }
            const float p = expf(s - mrun);
            l += p;
#pragma unroll
            for (int d = 0; d < DV; ++d) o[d] = fmaf(p, sv[t * DV + d], o[d]);
        }
    }
    if (!live) return;
    const float inv = 1.f / l;
    float* orow = a.o + ((size_t)(row0 + row) * a.hq + h) * DV;
#pragma unroll
    for (int d = 0; d < DV; ++d) orow[d] = o[d] * inv;
    a.lse[(size_t)h * a.T + row0 + row] = mrun + logf(l);
}

template <int DQK, int DV>
int launch(const FwdF32Args& a, int n_items, cudaStream_t stream) {
    const int smem = BN * (DQK + DV) * (int)sizeof(float);
    if (cudaFuncSetAttribute(fwd_f32_kernel<DQK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return -1;
    fwd_f32_kernel<DQK, DV><<<n_items, BM, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_fwd_f32(int dqk, int dv, const FwdF32Args& a, int n_items, cudaStream_t stream) {
    if (dqk == 64 && dv == 64) return launch<64, 64>(a, n_items, stream);
    if (dqk == 128 && dv == 128) return launch<128, 128>(a, n_items, stream);
    return -2;
}

}  // namespace thd

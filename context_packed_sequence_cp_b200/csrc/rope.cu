// Rotary position embedding with per-document positions, ahead of the attention.
//
// Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance",
// section "Does this PR introduce any user-facing change?": THD packed sequences whose
// attention resets at every EOD; the positions a rotary embedding sees restart with
// every document (thd_position_ids).  The pages name no rotary variant; this is the
// half-split form: for i < R/2 the pair (x[i], x[i + R/2]) of a head vector is rotated
// by the angle pos * base^(-2i/R); dimensions R..D-1 pass through unchanged.
//
// rope_table_kernel: cos/sin of every (token, i) in fp32, the angle formed in double
// precision (pos * base^(-2i/R) reaches tens of thousands of radians, where an fp32
// product alone would already be off by milliradians).
// rope_apply_kernel: 16-byte vectors, eight pairs per thread.
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

namespace thd {
namespace {

__global__ void __launch_bounds__(256) rope_table_kernel(const int32_t* __restrict__ pos, int64_t T, int half,
                                                         double log2_base, float2* __restrict__ table) {
    const int64_t n = T * half;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = k / half;
        const int i = (int)(k - t * half);
        const double inv_freq = exp2(-log2_base * (double)(2 * i) / (double)(2 * half));
        const double ang = (double)pos[t] * inv_freq;
        double s, c;
        sincos(ang, &s, &c);
        table[k] = make_float2((float)c, (float)s);
    }
}

// One thread per 8 consecutive pairs: a 16-byte load from each half of the rotated
// width and 64 bytes of the table row (shared by the token's heads, cache-resident).
// Requires rot_dim % 16 == 0 and dim % 8 == 0 (checked by the caller).
__global__ void __launch_bounds__(256) rope_apply_kernel(__nv_bfloat16* __restrict__ x, int64_t rows, int heads,
                                                         int dim, int half, const float2* __restrict__ table) {
    const int vpr = half >> 3;
    const int64_t items = rows * vpr;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < items; k += (int64_t)gridDim.x * blockDim.x) {
        const int64_t w = k / vpr;
        const int v = (int)(k - w * vpr);
        const int64_t t = w / heads;
        __nv_bfloat16* row = x + w * dim + v * 8;
        uint4 ua = *reinterpret_cast<const uint4*>(row);
        uint4 ub = *reinterpret_cast<const uint4*>(row + half);
        const float4* tab = reinterpret_cast<const float4*>(table + t * half + v * 8);
        __nv_bfloat162* pa = reinterpret_cast<__nv_bfloat162*>(&ua);
        __nv_bfloat162* pb = reinterpret_cast<__nv_bfloat162*>(&ub);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 cs = __ldg(tab + u);   // (cos, sin) of pairs 2u and 2u + 1
            const float2 a = __bfloat1622float2(pa[u]), b = __bfloat1622float2(pb[u]);
            pa[u] = __floats2bfloat162_rn(a.x * cs.x - b.x * cs.y, a.y * cs.z - b.y * cs.w);
            pb[u] = __floats2bfloat162_rn(b.x * cs.x + a.x * cs.y, b.y * cs.z + a.y * cs.w);
        }
        *reinterpret_cast<uint4*>(row) = ua;
        *reinterpret_cast<uint4*>(row + half) = ub;
    }
}

}  // namespace

int launch_rope(__nv_bfloat16* x, const int32_t* pos, int64_t T, int heads, int dim, int rot_dim, double base,
                float2* table, int num_sms, cudaStream_t stream) {
    const int half = rot_dim / 2;
    const int64_t n = T * half;
    const int tb = (int)((n + 255) / 256 < (int64_t)num_sms * 8 ? (n + 255) / 256 : (int64_t)num_sms * 8);
    rope_table_kernel<<<tb > 0 ? tb : 1, 256, 0, stream>>>(pos, T, half, log2(base), table);
    if (cudaGetLastError() != cudaSuccess) return -1;
    const int64_t items = T * heads * (half / 8);
    const int ab = (int)((items + 255) / 256 < (int64_t)num_sms * 8 ? (items + 255) / 256 : (int64_t)num_sms * 8);
    rope_apply_kernel<<<ab > 0 ? ab : 1, 256, 0, stream>>>(x, T * heads, heads, dim, half, table);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace thd

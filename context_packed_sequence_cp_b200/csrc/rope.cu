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
// rope_apply_kernel: one warp per (token, head) row of bf16; lane l rotates pairs
// l, l + 32, ... reading the table row once per token (L1/L2-resident across heads).
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

__global__ void __launch_bounds__(256) rope_apply_kernel(__nv_bfloat16* __restrict__ x, int64_t rows, int heads,
                                                         int dim, int half, const float2* __restrict__ table) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < rows; w += nwarps) {
        const int64_t t = w / heads;
        __nv_bfloat16* row = x + w * dim;
        const float2* tab = table + t * half;
        for (int i = lane; i < half; i += 32) {
            const float2 cs = tab[i];
            const float a = __bfloat162float(row[i]), b = __bfloat162float(row[i + half]);
            row[i] = __float2bfloat16_rn(a * cs.x - b * cs.y);
            row[i + half] = __float2bfloat16_rn(b * cs.x + a * cs.y);
        }
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
    const int64_t rows = T * heads;
    const int ab = (int)((rows + 7) / 8 < (int64_t)num_sms * 8 ? (rows + 7) / 8 : (int64_t)num_sms * 8);
    rope_apply_kernel<<<ab > 0 ? ab : 1, 256, 0, stream>>>(x, rows, heads, dim, half, table);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace thd

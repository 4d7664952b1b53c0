// Row gather: builds the rank-major buffer an all-gather of the rank-local shards
// would produce, and the inverse permutation back to packed order.
//
// Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance",
// section "What this PR does / why we need it?": KV-all-gather context
// parallelism with direct rank-major K/V indexing.  On one GPU the all-gather of
// every virtual rank's shard is a permuting copy, dst[j] = src[idx[j]].
//
// HBM-bound.  One warp moves one row at a time in 16-byte vectors (rows are whole
// multiples of 16 bytes, checked by the caller, so there is no scalar tail); every
// lane issues all of its loads for a row before its stores, to keep many requests
// in flight.  The grid is a whole number of waves over the SMs and strides over
// the rows.
#include "kernels.h"

namespace thd {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;  // 16-byte vectors per lane in flight per row pass

__device__ __forceinline__ uint4 ld_nc(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void st_cs(uint4* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, uint4* __restrict__ dst, int nvec,
                                         int lane) {
    for (int base = 0; base < nvec; base += 32 * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = base + u * 32 + lane;
            if (i < nvec) v[u] = ld_nc(src + i);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = base + u * 32 + lane;
            if (i < nvec) st_cs(dst + i, v[u]);
        }
    }
}

__global__ void __launch_bounds__(kThreads)
row_gather_kernel(const int32_t* __restrict__ idx, int64_t rows, const uint4* __restrict__ src0,
                  uint4* __restrict__ dst0, int nvec0, const uint4* __restrict__ src1, uint4* __restrict__ dst1,
                  int nvec1) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    for (int64_t j = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); j < rows; j += warps) {
        const int64_t s = __ldg(idx + j);
        copy_row(src0 + s * nvec0, dst0 + j * nvec0, nvec0, lane);
        if (nvec1 > 0) copy_row(src1 + s * nvec1, dst1 + j * nvec1, nvec1, lane);
    }
}

}  // namespace

int launch_row_gather(const int32_t* idx, int64_t rows, const void* src0, void* dst0, int64_t row_bytes0,
                      const void* src1, void* dst1, int64_t row_bytes1, int num_sms, cudaStream_t stream) {
    if (rows <= 0) return 0;
    const int64_t warps_needed = rows;
    const int64_t blocks_needed = (warps_needed + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t wave = (int64_t)num_sms * 8;  // 8 resident 256-thread blocks per SM
    const int grid = (int)(blocks_needed < wave ? blocks_needed : wave);
    row_gather_kernel<<<grid, kThreads, 0, stream>>>(
        idx, rows, static_cast<const uint4*>(src0), static_cast<uint4*>(dst0), (int)(row_bytes0 / 16),
        static_cast<const uint4*>(src1), static_cast<uint4*>(dst1), src1 ? (int)(row_bytes1 / 16) : 0);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace thd

// Launch interfaces between the C ABI layer (api.cu) and the device kernels.
#pragma once
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace thd {

// True once `fn` may use `bytes` of dynamic shared memory on the current device.  The
// attribute belongs to the device's context, so it is set once per device (devices
// 0-63 are remembered in `done`, others are set on every call); two host threads that
// race on the first call may both set it, which is harmless.
template <typename Kernel>
inline bool ensure_dynamic_smem(Kernel* fn, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    if (bit) done.fetch_or(bit, std::memory_order_release);
    return true;
}

// [rows, heads, dim] bf16 tensor viewed as a 3-D TMA map with 64-column x 1-head x
// box_rows-row boxes and 128-byte swizzle (the layout the tcgen05 descriptors expect).
// False when the driver's encoder is unavailable or rejects the map.
bool make_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int heads, int dim, int box_rows = 128);
// [rows, dim] bf16 tensor (a [T, heads, dim] tensor seen as T * heads rows) viewed as a
// 2-D TMA map with 64-column x 1-row boxes and 128-byte swizzle, for tile::gather4 loads.
bool make_map_bf16_rows(CUtensorMap* map, const void* base, int64_t rows, int dim);
// [rows, heads, dim] fp32 tensor viewed as a 3-D TMA map with 32-column x 1-head x 32-row
// boxes (128-byte rows) and 128-byte swizzle: the target of tiled reductions.
bool make_map_f32_box32(CUtensorMap* map, const void* base, int64_t rows, int heads, int dim, int box_rows = 32);

// ---- row gather (all-gather layout, and its inverse) -----------------------
// dst_t[j] = src_t[idx[j]] for whole rows of row_bytes_t bytes, t = 0, 1 (the second
// pair may be null).  Rows are copied with 16-byte vectors.
int launch_row_gather(const int32_t* idx, int64_t rows, const void* src0, void* dst0, int64_t row_bytes0,
                      const void* src1, void* dst1, int64_t row_bytes1, int num_sms, cudaStream_t stream);

// ---- forward, bf16 on tcgen05 ----------------------------------------------
struct FwdArgs {
    const int32_t* qtiles;
    const int32_t* entries;
    const int32_t* lpt;
    const int32_t* rm_of_global;  // rows of position tiles (row0 / k0 < 0)
    int32_t kv_global;            // K/V given in packed (global) order: rows are positions
    int32_t persistent;           // CTAs take over the items of CTAs that have not started
    int32_t qtile_outer;          // item order: query tiles longest-first outermost (else kv group)
    __nv_bfloat16* o;
    float* lse;
    int32_t hq, hkv;
    int64_t T;
    float scale_log2;  // scale * log2(e)
    int* status;       // device word: nonzero once a bounded wait gave up
};
// Tensor maps of the bf16 forward, over Q [T, hq, dqk], K [T, hkv, dqk], V [T, hkv, dv]
// (and K_rope [T, 1, 64] of the compact multi-head latent attention form, else K again):
//   q, k, v, kr          3-D {dim, heads, rows} maps, boxes of 64 columns x 128 rows;
//   qs, ks, vs, krs [s]  the same with boxes of 8 << s rows (runs inside position tiles);
//   qg, kg, vg, krg      2-D {dim, rows * heads} row maps, boxes of one row (tile::gather4).
constexpr int kRunBoxes = 4;  // 8, 16, 32 and 64 rows
struct FwdMaps {
    CUtensorMap q, k, v, kr;
    CUtensorMap qs[kRunBoxes], ks[kRunBoxes], vs[kRunBoxes], krs[kRunBoxes];
    CUtensorMap qg, kg, vg, krg;
};
int launch_fwd_sm100(int dqk, int dv, const FwdMaps& m, const FwdArgs& a, int n_items, cudaStream_t stream);
// Multi-head latent attention with a shared rope key: Q [T, hq, 192], K_nope [T, hkv, 128] (k),
// K_rope [T, 1, 64] (kr, one per token, every head), V [T, hkv, 128].
int launch_fwd_mla_sm100(const FwdMaps& m, const FwdArgs& a, int n_items, cudaStream_t stream);

// ---- forward, fp32 SIMT --------------------------------------------------------
struct FwdF32Args {
    const int32_t* qtiles;
    const int32_t* entries;
    const int32_t* lpt;
    const float* q;
    const float* k;
    const float* v;
    float* o;
    float* lse;
    int32_t hq, hkv;
    int64_t T;
    float scale;
};
int launch_fwd_f32(int dqk, int dv, const FwdF32Args& a, int n_items, cudaStream_t stream);

// ---- backward, bf16 on tcgen05 ---------------------------------------------------
struct BwdArgs {
    // the fused kernel walks the forward tables (rank-major and position tiles) and their
    // key-tile transpose; position rows are found through rm_of_global
    const int32_t* fqtiles;
    const int32_t* fentries;
    const int32_t* fkt_off;
    const int32_t* fkt_list;
    const int32_t* fkt_lpt;
    const int32_t* fkt_seg;  // work items by list segment (THD_KSEG entries each)
    int32_t n_fkseg;
    const int32_t* rm_of_global;
    const __nv_bfloat16* q;     // rank-major inputs (row maps of the position tiles)
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* o;
    const __nv_bfloat16* dout;
    const float* lse;
    float* delta;   // [hq, T] workspace
    float* dq_acc;  // [T, hq, dqk] fp32 output
    float* dk;      // [T, hkv, dqk]
    float* dv;      // [T, hkv, dv]
    int32_t hq, hkv;
    int64_t T;
    float scale;
    float scale_log2;
    int* status;
};
// n_items_per_group: backward work items per key/value head (fkt_seg[n_fkseg], the list
// segments of every key tile of the forward tables).
int launch_bwd_sm100(int dqk, int dv, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                     const CUtensorMap& dout, const BwdArgs& a, int n_items_per_group, int num_sms,
                     cudaStream_t stream);

// ---- rotary position embedding (half-split), per-document positions ---------------
int launch_rope(__nv_bfloat16* x, const int32_t* pos, int64_t T, int heads, int dim, int rot_dim, double base,
                float2* table, int num_sms, cudaStream_t stream);

}  // namespace thd

// thd_cp_attn_bwd_noalloc: the backward for callers that cannot allocate device
// memory.
//
// thd_cp_attn_bwd needs a caller-provided workspace for the per-row statistic
// Delta_i = sum(do_i * o_i).  Some callers cannot hand one over: their device
// memory is owned entirely by a framework allocator they may not call into from
// this code, or they run on a latency-critical path where cudaMalloc (which can
// synchronise the device) is not allowed.  This entry point keeps Delta in a
// fixed, file-scope device array instead, so it allocates nothing.
//
// The array is a static __device__ symbol of kScratchFloats floats (32 MiB); every
// GPU that loads the library holds it until the process exits.  In host code its
// name is only a stand-in, so the first call on each device resolves the device
// address with cudaGetSymbolAddress (with that device current) and caches it.
// The array is fully rewritten by every call before it is read, so nothing has to
// be cleared; because all calls share it, calls whose kernels overlap on the GPU
// (for example on different streams) race on it.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "kernels.h"
#include "plan.h"

namespace {

constexpr size_t kScratchFloats = size_t(1) << 23;  // 8,388,608 floats: Delta for hq * T up to this
static_assert(kScratchFloats == THD_NOALLOC_MAX_ROWS_X_HEADS, "header and array agree");

static __device__ __align__(256) float g_bwd_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
float* g_scratch_dev[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the array on the current device (set-up on first use).
int scratch_on_current_device(float** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return THD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_dev[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return THD_ERR_CUDA;
        g_scratch_dev[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_dev[dev];
    return THD_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace

extern "C" int thd_cp_attn_bwd_noalloc(thd_cp_plan_t plan, const void* q_rm, const void* k_rm, const void* v_rm,
                                       const void* o_rm, const float* lse_rm, const void* do_rm, float* dq_rm,
                                       float* dk_rm, float* dv_rm, int32_t hq, int32_t hkv, int32_t dqk, int32_t dv,
                                       float scale, int32_t dtype, void* stream) {
    int rc = thd_plan_ready(plan);
    if (rc != THD_OK) return rc;
    if (!q_rm || !k_rm || !v_rm || !o_rm || !lse_rm || !do_rm || !dq_rm || !dk_rm || !dv_rm ||
        !std::isfinite(scale) || !(scale > 0.f))
        return THD_ERR_INVALID_ARG;
    if (hq < 1 || hkv < 1 || hq % hkv != 0) return THD_ERR_INVALID_ARG;
    if (dtype != THD_DTYPE_BF16 || dqk != 128 || dv != 128) return THD_ERR_UNSUPPORTED;
    if ((size_t)hq * (size_t)plan->T > kScratchFloats) return THD_ERR_TOO_LARGE;
    const void* ptrs[] = {q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq_rm, dk_rm, dv_rm};
    for (const void* p : ptrs)
        if (!aligned16(p)) return THD_ERR_MISALIGNED;
    float* delta = nullptr;
    rc = scratch_on_current_device(&delta);
    if (rc != THD_OK) return rc;
    CUtensorMap mq, mk, mv, mdo;
    if (!thd::make_map_bf16(&mq, q_rm, plan->T, hq, dqk) || !thd::make_map_bf16(&mk, k_rm, plan->T, hkv, dqk) ||
        !thd::make_map_bf16(&mv, v_rm, plan->T, hkv, dv) || !thd::make_map_bf16(&mdo, do_rm, plan->T, hq, dv))
        return THD_ERR_CUDA;
    thd::BwdArgs a;
    a.fqtiles = plan->d_fqtiles;
    a.fentries = plan->d_fentries;
    a.fkt_off = plan->d_fkt_off;
    a.fkt_list = plan->d_fkt_list;
    a.fkt_lpt = plan->d_fkt_lpt;
    a.fkt_seg = plan->d_fkt_seg;
    a.n_fkseg = (int32_t)(plan->fkt_seg.size() - 1);
    a.rm_of_global = plan->d_rm_of_global;
    a.q = static_cast<const __nv_bfloat16*>(q_rm);
    a.k = static_cast<const __nv_bfloat16*>(k_rm);
    a.v = static_cast<const __nv_bfloat16*>(v_rm);
    a.o = static_cast<const __nv_bfloat16*>(o_rm);
    a.dout = static_cast<const __nv_bfloat16*>(do_rm);
    a.lse = lse_rm;
    a.delta = delta;
    a.dq_acc = dq_rm;
    a.dk = dk_rm;
    a.dv = dv_rm;
    a.hq = hq;
    a.hkv = hkv;
    a.T = plan->T;
    a.scale = scale;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.status = plan->d_status;
    if (plan->n_qtiles() == 0) return THD_OK;
    return thd::launch_bwd_sm100(dqk, dv, mq, mk, mv, mdo, a, plan->fkt_seg.back(), sm_count(),
                                 static_cast<cudaStream_t>(stream))
               ? THD_ERR_CUDA
               : THD_OK;
}

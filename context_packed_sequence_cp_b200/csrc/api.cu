// C ABI of libthdcp (declared in include/thdcp.h): argument validation, plan
// lifecycle with cached device tables, TMA descriptor encoding and kernel launches.
// No entry point falls back to another implementation: an unsupported shape is an
// error, and every computation runs in this library's kernels.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>

#include "kernels.h"
#include "plan.h"
#include "sm100.cuh"

namespace {

using thd_plan = thd_cp_plan_s;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms_current() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

int check_heads(int32_t hq, int32_t hkv) {
    if (hq < 1 || hkv < 1 || hq % hkv != 0) return THD_ERR_INVALID_ARG;
    return THD_OK;
}

// The plan's tables must be on the device, and that device must be current: the
// kernels launch on the current device and read the tables in place.  An error left
// pending by earlier, unrelated work is reported here (and not cleared), so that the
// launch checks after this point see only this library's launches.
int ready(thd_plan* p) {
    if (!p) return THD_ERR_INVALID_ARG;
    if (!p->uploaded) return THD_ERR_NOT_UPLOADED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    if (dev != p->device) return THD_ERR_INVALID_ARG;
    if (cudaPeekAtLastError() != cudaSuccess) return THD_ERR_CUDA;
    return THD_OK;
}

// Frees the device and pinned host memory of a plan.  The caller has made the plan's
// device current and waited for every kernel that reads the tables.
void free_device(thd_plan* p) {
    if (p->d_buf) cudaFree(p->d_buf);
    p->d_buf = nullptr;
    p->d_cap = 0;
    for (int i = 0; i < 2; ++i) {
        if (p->staged[i]) cudaEventDestroy(p->staged[i]);
        if (p->h_stage[i]) cudaFreeHost(p->h_stage[i]);
        p->staged[i] = nullptr;
        p->h_stage[i] = nullptr;
        p->h_cap[i] = 0;
    }
    p->d_q_idx = p->d_rm_of_global = p->d_qtiles = p->d_entries = p->d_lpt = nullptr;
    p->d_kt_off = p->d_kt_list = p->d_kt_lpt = p->d_kt_seg = p->d_status = nullptr;
    p->d_fqtiles = p->d_fentries = p->d_flpt = nullptr;
    p->d_fkt_off = p->d_fkt_list = p->d_fkt_lpt = p->d_fkt_seg = nullptr;
    p->uploaded = false;
}

constexpr size_t kAlign = 256;
size_t round_up(size_t n) { return (n + kAlign - 1) & ~(kAlign - 1); }

// Copies every host table into the plan's device allocation on `s`: through one of
// the two pinned staging buffers (waiting only for the copy that last used it) and
// one cudaMemcpyAsync.  The device allocation grows, in stream order, when the
// tables outgrow it; the status word at its start survives a re-plan.  Work on `s`
// enqueued earlier reads the previous tables before the copy overwrites them.
int copy_tables(thd_plan* p, cudaStream_t s, bool first) {
    constexpr int kTables = 16;
    const std::vector<int32_t>* src[kTables] = {&p->q_idx,    &p->rm_of_global, &p->qtiles,   &p->entries,
                                                &p->lpt,      &p->kt_off,       &p->kt_list,  &p->kt_lpt,
                                                &p->kt_seg,   &p->fqtiles,      &p->fentries, &p->flpt,
                                                &p->fkt_off,  &p->fkt_list,     &p->fkt_lpt,  &p->fkt_seg};
    int32_t** dst[kTables] = {&p->d_q_idx,   &p->d_rm_of_global, &p->d_qtiles,   &p->d_entries,
                              &p->d_lpt,     &p->d_kt_off,       &p->d_kt_list,  &p->d_kt_lpt,
                              &p->d_kt_seg,  &p->d_fqtiles,      &p->d_fentries, &p->d_flpt,
                              &p->d_fkt_off, &p->d_fkt_list,     &p->d_fkt_lpt,  &p->d_fkt_seg};
    size_t off[kTables];
    size_t total = kAlign;  // the status word (16 bytes) sits in the first 256
    for (int i = 0; i < kTables; ++i) {
        off[i] = total;
        total += round_up(std::max<size_t>(src[i]->size(), 4) * sizeof(int32_t));
    }
    const int st = p->next_stage;
    if (!p->staged[st] && cudaEventCreateWithFlags(&p->staged[st], cudaEventDisableTiming) != cudaSuccess)
        return THD_ERR_CUDA;
    if (cudaEventSynchronize(p->staged[st]) != cudaSuccess) return THD_ERR_CUDA;
    if (p->h_cap[st] < total) {
        if (p->h_stage[st]) cudaFreeHost(p->h_stage[st]);
        p->h_stage[st] = nullptr;
        p->h_cap[st] = 0;
        const size_t cap = total + total / 4;
        if (cudaHostAlloc(&p->h_stage[st], cap, cudaHostAllocDefault) != cudaSuccess) return THD_ERR_ALLOC;
        p->h_cap[st] = cap;
    }
    uint8_t* h = static_cast<uint8_t*>(p->h_stage[st]);
    for (int i = 0; i < kTables; ++i)
        if (!src[i]->empty()) std::memcpy(h + off[i], src[i]->data(), src[i]->size() * sizeof(int32_t));
    if (p->d_cap < total) {
        void* fresh = nullptr;
        const size_t cap = total + total / 4;
        if (cudaMallocAsync(&fresh, cap, s) != cudaSuccess) return THD_ERR_ALLOC;
        if (p->d_buf) {
            // the status word moves with the tables; the old buffer is released after
            // every earlier reader on this stream
            if (cudaMemcpyAsync(fresh, p->d_buf, 16, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
                cudaFreeAsync(p->d_buf, s) != cudaSuccess)
                return THD_ERR_CUDA;
        }
        p->d_buf = fresh;
        p->d_cap = cap;
    }
    uint8_t* d = static_cast<uint8_t*>(p->d_buf);
    if (first && cudaMemsetAsync(d, 0, 16, s) != cudaSuccess) return THD_ERR_CUDA;
    if (cudaMemcpyAsync(d + kAlign, h + kAlign, total - kAlign, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return THD_ERR_CUDA;
    if (cudaEventRecord(p->staged[st], s) != cudaSuccess) return THD_ERR_CUDA;
    p->next_stage = st ^ 1;
    p->d_status = reinterpret_cast<int32_t*>(d);
    for (int i = 0; i < kTables; ++i) *dst[i] = reinterpret_cast<int32_t*>(d + off[i]);
    return THD_OK;
}

}  // namespace

int thd_plan_ready(thd_cp_plan_s* p) { return ready(p); }

namespace thd {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link),
// resolved once (thread-safe initialisation of a function-local static).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return nullptr;
    }();
    return fn;
}

bool make_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int heads, int dim, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)dim * 2, (cuuint64_t)heads * dim * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_bf16_rows(CUtensorMap* map, const void* base, int64_t rows, int dim) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)dim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)dim * 2};
    const cuuint32_t box[2] = {64, 1};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The forward's maps of Q [T, hq, dqk], K [T, hkv, dk], V [T, hkv, dv] and the shared rope
// key K_rope [T, 1, dr] (kr; nullptr: K again): 128-row boxes, 8- to 64-row boxes, row maps.
bool make_fwd_maps(thd::FwdMaps* m, int64_t T, const void* q, int hq, int dqk, const void* k, int hkv, int dk,
                   const void* v, int dv, const void* kr, int dr) {
    if (!kr) {
        kr = k;
        dr = dk;
    }
    const int hr = kr == k ? hkv : 1;
    for (int s = 0; s < thd::kRunBoxes; ++s)
        if (!make_map_bf16(&m->qs[s], q, T, hq, dqk, 8 << s) || !make_map_bf16(&m->ks[s], k, T, hkv, dk, 8 << s) ||
            !make_map_bf16(&m->vs[s], v, T, hkv, dv, 8 << s) || !make_map_bf16(&m->krs[s], kr, T, hr, dr, 8 << s))
            return false;
    return make_map_bf16(&m->q, q, T, hq, dqk) && make_map_bf16(&m->k, k, T, hkv, dk) &&
           make_map_bf16(&m->v, v, T, hkv, dv) && make_map_bf16(&m->kr, kr, T, hr, dr) &&
           make_map_bf16_rows(&m->qg, q, T * hq, dqk) && make_map_bf16_rows(&m->kg, k, T * hkv, dk) &&
           make_map_bf16_rows(&m->vg, v, T * hkv, dv) && make_map_bf16_rows(&m->krg, kr, T * hr, dr);
}

bool make_map_f32_box32(CUtensorMap* map, const void* base, int64_t rows, int heads, int dim, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)dim * 4, (cuuint64_t)heads * dim * 4};
    const cuuint32_t box[3] = {32, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace thd

using thd::make_map_bf16;
using thd::make_map_bf16_rows;

extern "C" {

int thd_cp_plan(const int32_t* cu_seqlens, int32_t n_docs, int32_t cp, thd_cp_plan_t* out) {
    if (!out) return THD_ERR_INVALID_ARG;
    thd_plan* p = new (std::nothrow) thd_plan();
    if (!p) return THD_ERR_ALLOC;
    const int rc = thd_build_plan(cu_seqlens, n_docs, cp, p);
    if (rc != THD_OK) {
        delete p;
        return rc;
    }
    *out = p;
    return THD_OK;
}

int thd_cp_plan_info(thd_cp_plan_t plan, thd_cp_plan_info_t* out) {
    if (!plan || !out) return THD_ERR_INVALID_ARG;
    out->T = plan->T;
    out->cp = plan->cp;
    out->n_docs = plan->n_docs;
    out->Tl = plan->Tl;
    out->n_qtiles = plan->n_qtiles();
    out->n_entries = plan->n_entries();
    out->causal_pairs = plan->causal_pairs;
    out->n_kseg = plan->kt_seg.empty() ? 0 : (int64_t)plan->kt_seg.size() - 1;
    out->n_fqtiles = plan->n_fqtiles();
    out->n_fentries = plan->n_fentries();
    out->n_fkseg = plan->fkt_seg.empty() ? 0 : (int64_t)plan->fkt_seg.size() - 1;
    return THD_OK;
}

int thd_cp_plan_export(thd_cp_plan_t plan, int32_t* q_idx, int32_t* rm_of_global, int32_t* qtiles,
                       int32_t* entries, int32_t* lpt, int32_t* kt_off, int32_t* kt_list, int32_t* kt_lpt,
                       int32_t* kt_seg) {
    if (!plan) return THD_ERR_INVALID_ARG;
    auto cp = [](int32_t* dst, const std::vector<int32_t>& v) {
        if (dst && !v.empty()) std::memcpy(dst, v.data(), v.size() * sizeof(int32_t));
    };
    cp(q_idx, plan->q_idx);
    cp(rm_of_global, plan->rm_of_global);
    cp(qtiles, plan->qtiles);
    cp(entries, plan->entries);
    cp(lpt, plan->lpt);
    cp(kt_off, plan->kt_off);
    cp(kt_list, plan->kt_list);
    cp(kt_lpt, plan->kt_lpt);
    cp(kt_seg, plan->kt_seg);
    return THD_OK;
}

int thd_cp_plan_export_fwd(thd_cp_plan_t plan, int32_t* fqtiles, int32_t* fentries, int32_t* flpt,
                           int32_t* fkt_off, int32_t* fkt_list, int32_t* fkt_lpt, int32_t* fkt_seg) {
    if (!plan) return THD_ERR_INVALID_ARG;
    auto cp = [](int32_t* dst, const std::vector<int32_t>& v) {
        if (dst && !v.empty()) std::memcpy(dst, v.data(), v.size() * sizeof(int32_t));
    };
    cp(fqtiles, plan->fqtiles);
    cp(fentries, plan->fentries);
    cp(flpt, plan->flpt);
    cp(fkt_off, plan->fkt_off);
    cp(fkt_list, plan->fkt_list);
    cp(fkt_lpt, plan->fkt_lpt);
    cp(fkt_seg, plan->fkt_seg);
    return THD_OK;
}

int thd_cp_plan_upload(thd_cp_plan_t plan, void* stream) {
    if (!plan) return THD_ERR_INVALID_ARG;
    if (plan->uploaded) return THD_OK;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    const int rc = copy_tables(plan, static_cast<cudaStream_t>(stream), true);
    if (rc != THD_OK) {
        cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
        free_device(plan);
        return rc;
    }
    plan->device = dev;
    plan->uploaded = true;
    return THD_OK;
}

int thd_cp_plan_update(thd_cp_plan_t plan, const int32_t* cu_seqlens, int32_t n_docs, int32_t cp, void* stream) {
    if (!plan) return THD_ERR_INVALID_ARG;
    if (plan->uploaded) {
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
        if (dev != plan->device) return THD_ERR_INVALID_ARG;
    }
    thd_plan fresh;
    const int rc = thd_build_plan(cu_seqlens, n_docs, cp, &fresh);
    if (rc != THD_OK) return rc;
    plan->T = fresh.T;
    plan->Tl = fresh.Tl;
    plan->cp = fresh.cp;
    plan->n_docs = fresh.n_docs;
    plan->causal_pairs = fresh.causal_pairs;
    plan->doc_start.swap(fresh.doc_start);
    plan->doc_len.swap(fresh.doc_len);
    plan->q_idx.swap(fresh.q_idx);
    plan->rm_of_global.swap(fresh.rm_of_global);
    plan->qtiles.swap(fresh.qtiles);
    plan->entries.swap(fresh.entries);
    plan->lpt.swap(fresh.lpt);
    plan->kt_off.swap(fresh.kt_off);
    plan->kt_list.swap(fresh.kt_list);
    plan->kt_lpt.swap(fresh.kt_lpt);
    plan->kt_seg.swap(fresh.kt_seg);
    plan->fqtiles.swap(fresh.fqtiles);
    plan->fentries.swap(fresh.fentries);
    plan->flpt.swap(fresh.flpt);
    plan->fkt_off.swap(fresh.fkt_off);
    plan->fkt_list.swap(fresh.fkt_list);
    plan->fkt_lpt.swap(fresh.fkt_lpt);
    plan->fkt_seg.swap(fresh.fkt_seg);
    if (!plan->uploaded) return THD_OK;
    // On a failed copy the device tables no longer match the host tables: the plan
    // becomes not-uploaded, and a later thd_cp_plan_upload copies them afresh.
    const int cr = copy_tables(plan, static_cast<cudaStream_t>(stream), false);
    if (cr != THD_OK) {
        cudaDeviceSynchronize();
        free_device(plan);
    }
    return cr;
}

void thd_cp_plan_destroy(thd_cp_plan_t plan) {
    if (!plan) return;
    if (plan->uploaded || plan->d_buf || plan->h_stage[0] || plan->h_stage[1]) {
        // Free on the device that holds the tables, after every kernel there that may
        // still read them; the caller's current device is restored afterwards.
        int prev = -1;
        const bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
        const bool switched = plan->device >= 0 && (!have_prev || prev != plan->device) &&
                              cudaSetDevice(plan->device) == cudaSuccess;
        cudaDeviceSynchronize();
        free_device(plan);
        if (switched && have_prev) cudaSetDevice(prev);
    }
    delete plan;
}

int thd_kv_gather(thd_cp_plan_t plan, const void* k, const void* v, void* k_rm, void* v_rm, int64_t k_row_bytes,
                  int64_t v_row_bytes, void* stream) {
    int rc = ready(plan);
    if (rc) return rc;
    if (!k || !k_rm || k_row_bytes <= 0 || (!v) != (!v_rm) || (v && v_row_bytes <= 0)) return THD_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(k_rm) || (k_row_bytes & 15) || (v && (!aligned16(v) || !aligned16(v_rm))) ||
        (v && (v_row_bytes & 15)))
        return THD_ERR_MISALIGNED;
    if (k_row_bytes / 16 > INT32_MAX || (v && v_row_bytes / 16 > INT32_MAX)) return THD_ERR_INVALID_ARG;
    if (thd::launch_row_gather(plan->d_q_idx, plan->T, k, k_rm, k_row_bytes, v, v_rm, v_row_bytes,
                               num_sms_current(), static_cast<cudaStream_t>(stream)))
        return THD_ERR_CUDA;
    return THD_OK;
}

int thd_rope_workspace(int64_t T, int32_t rot_dim, size_t* bytes) {
    if (!bytes || T < 1 || rot_dim < 2 || (rot_dim & 1)) return THD_ERR_INVALID_ARG;
    *bytes = (size_t)T * (size_t)(rot_dim / 2) * sizeof(float2);
    return THD_OK;
}

int thd_rope_apply(void* x, const int32_t* pos, int64_t T, int32_t heads, int32_t dim, int32_t rot_dim,
                   double base, int32_t dtype, void* workspace, size_t ws_bytes, void* stream) {
    if (!x || !pos || !workspace || T < 1 || heads < 1 || dim < 2 || rot_dim < 2 || (rot_dim & 1) ||
        rot_dim > dim || !std::isfinite(base) || !(base > 0.0))
        return THD_ERR_INVALID_ARG;
    if (dtype != THD_DTYPE_BF16 || (rot_dim % 16) || (dim % 8)) return THD_ERR_UNSUPPORTED;
    size_t need = 0;
    thd_rope_workspace(T, rot_dim, &need);
    if (ws_bytes < need) return THD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(pos) || !aligned16(workspace)) return THD_ERR_MISALIGNED;
    return thd::launch_rope(static_cast<__nv_bfloat16*>(x), pos, T, heads, dim, rot_dim, base,
                            static_cast<float2*>(workspace), num_sms_current(), static_cast<cudaStream_t>(stream))
               ? THD_ERR_CUDA
               : THD_OK;
}

int thd_rows_to_global(thd_cp_plan_t plan, const void* src_rm, void* dst, int64_t row_bytes, void* stream) {
    int rc = ready(plan);
    if (rc) return rc;
    if (!src_rm || !dst || row_bytes <= 0) return THD_ERR_INVALID_ARG;
    if (!aligned16(src_rm) || !aligned16(dst) || (row_bytes & 15)) return THD_ERR_MISALIGNED;
    if (thd::launch_row_gather(plan->d_rm_of_global, plan->T, src_rm, dst, row_bytes, nullptr, nullptr, 0,
                               num_sms_current(), static_cast<cudaStream_t>(stream)))
        return THD_ERR_CUDA;
    return THD_OK;
}

namespace {
// Persistent CTAs (each taking over the items of CTAs that have not started) pay off when
// items are short: a CTA's fill and drain (Q load, first S, epilogue) is then a large share
// of an item and overlaps with the neighbouring items.  With long items one CTA per item
// measured as fast or faster, so the plan's mean key tiles per query tile decides.
constexpr int64_t kPersistMaxMeanTiles = 64;
// Item order.  Key/value group outermost keeps one group's K/V in L2 while its items run;
// query tiles outermost (longest first over every group) balances the SMs better, since no
// group's longest items start last, but its items in flight read one document's K/V for
// every key/value head at once.  That order is taken when that much K/V (the longest
// document's, all heads) fits in half of the 126 MB L2.
constexpr int64_t kQtileOuterMaxDocKvBytes = 64ll << 20;

// Arguments of the bf16 forward over the forward tables.
thd::FwdArgs fwd_args(thd_plan* plan, void* o_rm, float* lse_rm, int32_t hq, int32_t hkv, int32_t dk, int32_t dv,
                      float scale, int32_t kv_global) {
    thd::FwdArgs a;
    a.qtiles = plan->d_fqtiles;
    a.entries = plan->d_fentries;
    a.lpt = plan->d_flpt;
    a.rm_of_global = plan->d_rm_of_global;
    a.kv_global = kv_global;
    a.persistent = plan->n_fentries() < kPersistMaxMeanTiles * plan->n_fqtiles() ? 1 : 0;
    const int64_t max_doc = plan->doc_len.empty() ? 0 : *std::max_element(plan->doc_len.begin(), plan->doc_len.end());
    a.qtile_outer = max_doc * hkv * (dk + dv) * 2 <= kQtileOuterMaxDocKvBytes ? 1 : 0;
    a.o = static_cast<__nv_bfloat16*>(o_rm);
    a.lse = lse_rm;
    a.hq = hq;
    a.hkv = hkv;
    a.T = plan->T;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.status = plan->d_status;
    return a;
}
}  // namespace

int thd_cp_attn_fwd_mla(thd_cp_plan_t plan, const void* q_rm, const void* k_nope_rm, const void* k_rope_rm,
                        const void* v_rm, void* o_rm, float* lse_rm, int32_t hq, int32_t hkv, int32_t d_nope,
                        int32_t d_rope, int32_t dv, float scale, int32_t dtype, void* stream) {
    int rc = ready(plan);
    if (rc) return rc;
    if (!q_rm || !k_nope_rm || !k_rope_rm || !v_rm || !o_rm || !lse_rm || !std::isfinite(scale) || !(scale > 0.f))
        return THD_ERR_INVALID_ARG;
    if ((rc = check_heads(hq, hkv))) return rc;
    if (dtype != THD_DTYPE_BF16 || d_nope != 128 || d_rope != 64 || dv != 128) return THD_ERR_UNSUPPORTED;
    if (!aligned16(q_rm) || !aligned16(k_nope_rm) || !aligned16(k_rope_rm) || !aligned16(v_rm) || !aligned16(o_rm) ||
        !aligned16(lse_rm))
        return THD_ERR_MISALIGNED;
    const int64_t items = plan->n_fqtiles() * (int64_t)hq;
    if (items > INT32_MAX) return THD_ERR_INVALID_ARG;
    thd::FwdMaps maps;
    if (!make_fwd_maps(&maps, plan->T, q_rm, hq, d_nope + d_rope, k_nope_rm, hkv, d_nope, v_rm, dv, k_rope_rm, d_rope))
        return THD_ERR_CUDA;
    // the forward tables; K is the per-head part plus the shared rope key
    const thd::FwdArgs a = fwd_args(plan, o_rm, lse_rm, hq, hkv, d_nope + d_rope, dv, scale, 0);
    if (items == 0) return THD_OK;
    return thd::launch_fwd_mla_sm100(maps, a, (int)items, static_cast<cudaStream_t>(stream))
               ? THD_ERR_CUDA
               : THD_OK;
}

int thd_cp_attn_fwd(thd_cp_plan_t plan, const void* q_rm, const void* k_rm, const void* v_rm, void* o_rm,
                    float* lse_rm, int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, float scale, int32_t dtype,
                    void* stream) {
    int rc = ready(plan);
    if (rc) return rc;
    if (!q_rm || !k_rm || !v_rm || !o_rm || !lse_rm || !std::isfinite(scale) || !(scale > 0.f))
        return THD_ERR_INVALID_ARG;
    if ((rc = check_heads(hq, hkv))) return rc;
    if (!aligned16(q_rm) || !aligned16(k_rm) || !aligned16(v_rm) || !aligned16(o_rm) || !aligned16(lse_rm))
        return THD_ERR_MISALIGNED;
    const int64_t items = plan->n_qtiles() * (int64_t)hq;
    if (items > INT32_MAX || plan->n_fqtiles() * (int64_t)hq > INT32_MAX) return THD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == THD_DTYPE_BF16) {
        if (!((dqk == 128 && dv == 128) || (dqk == 192 && dv == 128))) return THD_ERR_UNSUPPORTED;
        thd::FwdMaps maps;
        if (!make_fwd_maps(&maps, plan->T, q_rm, hq, dqk, k_rm, hkv, dqk, v_rm, dv, nullptr, 0)) return THD_ERR_CUDA;
        // the forward tables: rank-major tiles, position tiles for short-chunk documents
        const thd::FwdArgs a = fwd_args(plan, o_rm, lse_rm, hq, hkv, dqk, dv, scale, 0);
        const int64_t fitems = plan->n_fqtiles() * (int64_t)hq;
        if (fitems == 0) return THD_OK;
        return thd::launch_fwd_sm100(dqk, dv, maps, a, (int)fitems, s) ? THD_ERR_CUDA : THD_OK;
    }
    if (dtype == THD_DTYPE_FP32) {
        if (!((dqk == 64 && dv == 64) || (dqk == 128 && dv == 128))) return THD_ERR_UNSUPPORTED;
        thd::FwdF32Args a;
        a.qtiles = plan->d_qtiles;
        a.entries = plan->d_entries;
        a.lpt = plan->d_lpt;
        a.q = static_cast<const float*>(q_rm);
        a.k = static_cast<const float*>(k_rm);
        a.v = static_cast<const float*>(v_rm);
        a.o = static_cast<float*>(o_rm);
        a.lse = lse_rm;
        a.hq = hq;
        a.hkv = hkv;
        a.T = plan->T;
        a.scale = scale;
        if (items == 0) return THD_OK;
        return thd::launch_fwd_f32(dqk, dv, a, (int)items, s) ? THD_ERR_CUDA : THD_OK;
    }
    return THD_ERR_UNSUPPORTED;
}

int thd_cp_attn_fwd_fused_gather(thd_cp_plan_t plan, const void* q_rm, const void* k, const void* v, void* o_rm,
                                 float* lse_rm, int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, float scale,
                                 int32_t dtype, void* stream) {
    int rc = ready(plan);
    if (rc) return rc;
    if (!q_rm || !k || !v || !o_rm || !lse_rm || !std::isfinite(scale) || !(scale > 0.f)) return THD_ERR_INVALID_ARG;
    if ((rc = check_heads(hq, hkv))) return rc;
    if (dtype != THD_DTYPE_BF16 || !((dqk == 128 && dv == 128) || (dqk == 192 && dv == 128))) return THD_ERR_UNSUPPORTED;
    if (!aligned16(q_rm) || !aligned16(k) || !aligned16(v) || !aligned16(o_rm) || !aligned16(lse_rm))
        return THD_ERR_MISALIGNED;
    const int64_t items = plan->n_fqtiles() * (int64_t)hq;
    if (items > INT32_MAX) return THD_ERR_INVALID_ARG;
    thd::FwdMaps maps;
    if (!make_fwd_maps(&maps, plan->T, q_rm, hq, dqk, k, hkv, dqk, v, dv, nullptr, 0)) return THD_ERR_CUDA;
    const thd::FwdArgs a = fwd_args(plan, o_rm, lse_rm, hq, hkv, dqk, dv, scale, 1);
    if (items == 0) return THD_OK;
    return thd::launch_fwd_sm100(dqk, dv, maps, a, (int)items, static_cast<cudaStream_t>(stream))
               ? THD_ERR_CUDA
               : THD_OK;
}

int thd_cp_attn_bwd_workspace(thd_cp_plan_t plan, int32_t hq, int32_t hkv, int32_t dqk, int32_t dv, int32_t dtype,
                              size_t* bytes) {
    if (!plan || !bytes) return THD_ERR_INVALID_ARG;
    int rc = check_heads(hq, hkv);
    if (rc) return rc;
    if (dtype != THD_DTYPE_BF16 || dqk != 128 || dv != 128) return THD_ERR_UNSUPPORTED;
    const size_t delta = ((size_t)hq * plan->T * sizeof(float) + 255) & ~(size_t)255;
    *bytes = delta;
    return THD_OK;
}

int thd_cp_attn_bwd(thd_cp_plan_t plan, const void* q_rm, const void* k_rm, const void* v_rm, const void* o_rm,
                    const float* lse_rm, const void* do_rm, float* dq_rm, float* dk_rm, float* dv_rm,
                    void* workspace, size_t workspace_bytes, int32_t hq, int32_t hkv, int32_t dqk, int32_t dv,
                    float scale, int32_t dtype, void* stream) {
    int rc = ready(plan);
    if (rc) return rc;
    if (!q_rm || !k_rm || !v_rm || !o_rm || !lse_rm || !do_rm || !dq_rm || !dk_rm || !dv_rm || !workspace ||
        !std::isfinite(scale) || !(scale > 0.f))
        return THD_ERR_INVALID_ARG;
    if ((rc = check_heads(hq, hkv))) return rc;
    if (dtype != THD_DTYPE_BF16 || dqk != 128 || dv != 128) return THD_ERR_UNSUPPORTED;
    size_t need = 0;
    thd_cp_attn_bwd_workspace(plan, hq, hkv, dqk, dv, dtype, &need);
    if (workspace_bytes < need) return THD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return THD_ERR_MISALIGNED;
    const void* ptrs[] = {q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq_rm, dk_rm, dv_rm};
    for (const void* p : ptrs)
        if (!aligned16(p)) return THD_ERR_MISALIGNED;
    CUtensorMap mq, mk, mv, mdo;
    if (!make_map_bf16(&mq, q_rm, plan->T, hq, dqk) || !make_map_bf16(&mk, k_rm, plan->T, hkv, dqk) ||
        !make_map_bf16(&mv, v_rm, plan->T, hkv, dv) || !make_map_bf16(&mdo, do_rm, plan->T, hq, dv))
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
    a.delta = static_cast<float*>(workspace);
    a.dq_acc = dq_rm;
    a.dk = dk_rm;
    a.dv = dv_rm;
    a.hq = hq;
    a.hkv = hkv;
    a.T = plan->T;
    a.scale = scale;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.status = plan->d_status;
    const int64_t nkt = plan->n_qtiles();
    if (nkt == 0) return THD_OK;
    return thd::launch_bwd_sm100(dqk, dv, mq, mk, mv, mdo, a, plan->fkt_seg.back(), num_sms_current(),
                                 static_cast<cudaStream_t>(stream))
               ? THD_ERR_CUDA
               : THD_OK;
}

int thd_cp_device_status(thd_cp_plan_t plan, int32_t reset, int32_t* status) {
    if (!plan || !status) return THD_ERR_INVALID_ARG;
    if (!plan->uploaded) return THD_ERR_NOT_UPLOADED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    if (dev != plan->device) return THD_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return THD_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, plan->d_status, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess) return THD_ERR_CUDA;
    *status = v;
    if (reset && (cudaMemset(plan->d_status, 0, sizeof(int32_t)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess))
        return THD_ERR_CUDA;
    return THD_OK;
}

const char* thd_cp_strerror(int code) {
    switch (code) {
        case THD_OK: return "ok";
        case THD_ERR_INVALID_ARG: return "invalid argument";
        case THD_ERR_BAD_SEQLENS: return "cu_seqlens must start at 0 and every document must be non-empty";
        case THD_ERR_NOT_DIVISIBLE: return "every document length must be divisible by 2 * cp";
        case THD_ERR_MISALIGNED: return "pointers and row sizes must be multiples of 16 bytes";
        case THD_ERR_NOT_UPLOADED: return "plan tables are not on the device: call thd_cp_plan_upload";
        case THD_ERR_CUDA: return "CUDA runtime or launch error";
        case THD_ERR_UNSUPPORTED: return "unsupported dtype / head dimension combination";
        case THD_ERR_ALLOC: return "allocation failed";
        case THD_ERR_TOO_LARGE:
            return "result does not fit: hq * T exceeds the fixed scratch of the no-allocation backward, "
                   "or the caller's output array is too small";
        default: return "unknown error";
    }
}

}  // extern "C"

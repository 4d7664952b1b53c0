// Internal plan object of libthdcp: host tables plus their cached device copies.
#pragma once
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/thdcp.h"

struct thd_cp_plan_s {
    // layout
    int64_t T = 0, Tl = 0;
    int32_t cp = 0, n_docs = 0;
    int64_t causal_pairs = 0;
    std::vector<int64_t> doc_start, doc_len;

    // host tables (see thd_cp_plan_export for the record layouts)
    std::vector<int32_t> q_idx, rm_of_global;
    std::vector<int32_t> qtiles, entries, lpt;
    std::vector<int32_t> kt_off, kt_list, kt_lpt, kt_seg;
    // forward tables: rank-major tiles of documents whose chunks span a tile or more,
    // position-ordered tiles of documents with shorter chunks
    std::vector<int32_t> fqtiles, fentries, flpt;
    std::vector<int32_t> fkt_off, fkt_list, fkt_lpt, fkt_seg;  // their key-tile transpose

    // Device side, valid after thd_cp_plan_upload.  Every table lives in one
    // stream-ordered allocation (d_buf, grown only when a layout needs more), and
    // reaches it by one copy from a pinned staging buffer.  Two staging buffers
    // alternate, so that a re-plan waits only for the copy issued two re-plans ago.
    bool uploaded = false;
    int device = -1;
    void* d_buf = nullptr;
    size_t d_cap = 0;
    void* h_stage[2] = {nullptr, nullptr};
    size_t h_cap[2] = {0, 0};
    cudaEvent_t staged[2] = {nullptr, nullptr};  // recorded after the copy out of h_stage[i]
    int next_stage = 0;
    int32_t *d_q_idx = nullptr, *d_rm_of_global = nullptr;
    int32_t *d_qtiles = nullptr, *d_entries = nullptr, *d_lpt = nullptr;
    int32_t *d_kt_off = nullptr, *d_kt_list = nullptr, *d_kt_lpt = nullptr, *d_kt_seg = nullptr;
    int32_t *d_fqtiles = nullptr, *d_fentries = nullptr, *d_flpt = nullptr;
    int32_t *d_fkt_off = nullptr, *d_fkt_list = nullptr, *d_fkt_lpt = nullptr, *d_fkt_seg = nullptr;
    int32_t* d_status = nullptr;  // set by kernels whose bounded waits gave up

    int64_t n_qtiles() const { return (int64_t)qtiles.size() / THD_QTILE_FIELDS; }
    int64_t n_entries() const { return (int64_t)entries.size() / THD_ENTRY_FIELDS; }
    int64_t n_fqtiles() const { return (int64_t)fqtiles.size() / THD_QTILE_FIELDS; }
    int64_t n_fentries() const { return (int64_t)fentries.size() / THD_ENTRY_FIELDS; }
};

// THD_OK when the plan's tables are on the device, that device is current and no
// earlier CUDA error is pending; else the code every launching entry point returns.
int thd_plan_ready(thd_cp_plan_s* p);

// Builds every host table; returns THD_OK or an error code (plan untouched on error).
int thd_build_plan(const int32_t* cu_seqlens, int32_t n_docs, int32_t cp, thd_cp_plan_s* p);

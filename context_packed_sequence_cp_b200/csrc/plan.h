// Internal plan object of libthdcp: host tables plus their cached device copies.
#pragma once
#include <cstdint>
#include <vector>

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
    std::vector<int32_t> kt_off, kt_list, kt_lpt;

    // device copies (owned), valid after thd_cp_plan_upload
    bool uploaded = false;
    int device = -1;
    int32_t *d_q_idx = nullptr, *d_rm_of_global = nullptr;
    int32_t *d_qtiles = nullptr, *d_entries = nullptr, *d_lpt = nullptr;
    int32_t *d_kt_off = nullptr, *d_kt_list = nullptr, *d_kt_lpt = nullptr;
    int32_t* d_status = nullptr;  // set by kernels whose bounded waits gave up

    int64_t n_qtiles() const { return (int64_t)qtiles.size() / THD_QTILE_FIELDS; }
    int64_t n_entries() const { return (int64_t)entries.size() / THD_ENTRY_FIELDS; }
};

// Builds every host table; returns THD_OK or an error code (plan untouched on error).
int thd_build_plan(const int32_t* cu_seqlens, int32_t n_docs, int32_t cp, thd_cp_plan_s* p);

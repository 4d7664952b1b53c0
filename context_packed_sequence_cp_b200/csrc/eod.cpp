// Document boundaries of an EOD-delimited packed sequence, ahead of thd_cp_plan.
//
// Method: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance",
// section "Does this PR introduce any user-facing change?": THD packed sequences
// whose attention mask resets at every EOD token.  A document ends with (and
// includes) an EOD token; tokens after the last EOD form a final document.  The
// cu_seqlens produced here feed thd_cp_plan, which applies the divisibility rule.
// Host only: the token ids and the tables are host memory, like the plan's input.
#include <cstdint>

#include "../../include/thdcp.h"

extern "C" int thd_cu_seqlens_from_eod(const int32_t* tokens, int64_t T, int32_t eod_id, int32_t* cu_seqlens,
                                       int32_t capacity, int32_t* n_docs) {
    if (!tokens || !n_docs || T < 1 || T > INT32_MAX || capacity < 0) return THD_ERR_INVALID_ARG;
    int64_t docs = 0;
    for (int64_t t = 0; t < T; ++t)
        if (tokens[t] == eod_id) ++docs;
    if (tokens[T - 1] != eod_id) ++docs;   // a final document without a closing EOD
    if (docs > INT32_MAX - 1) return THD_ERR_INVALID_ARG;
    *n_docs = static_cast<int32_t>(docs);
    if (!cu_seqlens || capacity < docs + 1) return THD_ERR_TOO_LARGE;
    int64_t d = 0;
    cu_seqlens[0] = 0;
    for (int64_t t = 0; t < T; ++t)
        if (tokens[t] == eod_id) cu_seqlens[++d] = static_cast<int32_t>(t + 1);
    if (tokens[T - 1] != eod_id) cu_seqlens[++d] = static_cast<int32_t>(T);
    return THD_OK;
}

extern "C" int thd_position_ids(const int32_t* cu_seqlens, int32_t n_docs, int32_t* pos) {
    if (!cu_seqlens || !pos || n_docs < 1) return THD_ERR_INVALID_ARG;
    if (cu_seqlens[0] != 0) return THD_ERR_BAD_SEQLENS;
    for (int32_t d = 0; d < n_docs; ++d)
        if (cu_seqlens[d + 1] <= cu_seqlens[d]) return THD_ERR_BAD_SEQLENS;
    for (int32_t d = 0; d < n_docs; ++d)
        for (int32_t t = cu_seqlens[d]; t < cu_seqlens[d + 1]; ++t) pos[t] = t - cu_seqlens[d];
    return THD_OK;
}

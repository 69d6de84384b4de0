// moe_internal.cuh -- forms of the MoE routing, combine and gather-sum steps
// with the shared expert optional (library-internal; the exported
// nvfp4_moe_* entry points are these with the shared expert present).
#pragma once

#include "common.cuh"

namespace nvfp4 {
namespace moe {

// Without `shared`, the shared expert's segment is empty, the combine and
// the gather-sum leave its term out, and combine_weights may be NULL (every
// routed row then has weight 1): the form an expert-parallel rank uses on the
// rows it received (one row per assignment, the combine done by the rows'
// home rank).
nvfp4_status route(const int32_t* expert_ids, const float* combine_weights, int tokens, int topk, int experts,
                   bool shared, int32_t* seg_len, int32_t* seg_off, int32_t* row_token, float* row_weight,
                   int32_t* slot_row, int64_t rows_cap, void* stream);
nvfp4_status combine(const void* y, int64_t cols, const int32_t* slot_row, const float* combine_weights, int tokens,
                     int topk, const int32_t* seg_off, int experts, bool shared, void* out, void* stream);
nvfp4_status gather_sum(const void* dxp, int64_t cols, const int32_t* slot_row, int tokens, int topk,
                        const int32_t* seg_off, int experts, bool shared, void* dx, void* stream);

}  // namespace moe
}  // namespace nvfp4

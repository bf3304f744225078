// sgmv_grouped_tc.cuh -- grouped tensor-core SGMV for long segments (placeholder).
#pragma once

#include "sgmv_common.cuh"

namespace sgmv {

constexpr int kGroupedMinSegment = 128;

inline bool grouped_tc_rank(int r) { return false && r; }

inline bool grouped_tc_supported(int r, int H1, int H2, lora_sgmv_dtype dt) {
    (void)H1; (void)H2; (void)dt;
    return grouped_tc_rank(r);
}

inline lora_sgmv_status launch_grouped_tc(void*, const void*, const void* const*, const void* const*,
                                          const int32_t*, const int32_t*, int, int, int, int, int, int,
                                          float, lora_sgmv_dtype, uint32_t*, cudaStream_t) {
    return LORA_SGMV_ERR_UNSUPPORTED;
}

}  // namespace sgmv

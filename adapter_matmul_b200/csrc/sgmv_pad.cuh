// sgmv_pad.cuh -- one adapter padded with zeros to a larger rank.
//
// Adapters of different ranks can share one SGMV call once every adapter is padded to one
// rank r: the authors' answer on different ranks (page "Punica: Serving multiple LoRA
// finetuned LLM as one", the Hacker News thread) is padding, because the kernels are bound by
// memory, not arithmetic. A_i [H1, r_src] becomes [H1, r] with zero columns r_src..r-1 and
// B_i [r_src, H2] becomes [r, H2] with zero rows r_src..r-1, so the extra entries of V are
// zero and the extra terms of the expand's sums are zero.
#pragma once

#include <cstdint>

namespace sgmv {

constexpr int kPadThreads = 256;

// dst [rows_dst, cols_dst] from src [rows_src, cols_src], both row-major 16-bit: the
// elements both cover are copied, every other element of dst is zero. Grid-stride over dst.
__global__ void __launch_bounds__(kPadThreads)
    sgmv_pad_kernel(uint16_t* __restrict__ dst, const uint16_t* __restrict__ src, int64_t rows_dst,
                    int64_t cols_dst, int64_t rows_src, int64_t cols_src) {
    const int64_t n = rows_dst * cols_dst;
    const int64_t step = int64_t(gridDim.x) * blockDim.x;
    for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += step) {
        const int64_t i = e / cols_dst;
        const int64_t j = e - i * cols_dst;
        dst[e] = (i < rows_src && j < cols_src) ? src[i * cols_src + j] : uint16_t(0);
    }
}

}  // namespace sgmv

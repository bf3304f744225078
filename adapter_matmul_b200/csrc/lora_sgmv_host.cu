// lora_sgmv_host.cu -- one serving step whose batch lives in host memory: the host grouping
// of the tokens' adapter ids into segments (the segmented batch of the multi-LoRA paragraph of
// page “Punica：多 LoRA 模型统一服务框架”, the Punica README), the copies in, one batched SGMV
// launch and the copies out, all enqueued on one stream. Host code only; it calls the
// library's own entry points.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/lora_sgmv.h"

namespace {

lora_sgmv_status copy_all(const lora_sgmv_copy* c, int32_t n, cudaMemcpyKind kind, cudaStream_t s) {
    for (int32_t k = 0; k < n; ++k) {
        if (c[k].bytes == 0) continue;
        if (cudaMemcpyAsync(c[k].dst, c[k].src, c[k].bytes, kind, s) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    }
    return LORA_SGMV_OK;
}

bool copies_valid(const lora_sgmv_copy* c, int32_t n) {
    if (n < 0 || (n > 0 && !c)) return false;
    for (int32_t k = 0; k < n; ++k)
        if (c[k].bytes > 0 && (!c[k].src || !c[k].dst)) return false;
    return true;
}

}  // namespace

extern "C" lora_sgmv_status lora_sgmv_step_host(const int32_t* ids, int32_t T, int32_t num_adapters,
                                                int32_t* meta_host, const int32_t* meta_dev, int32_t* perm,
                                                const lora_sgmv_copy* h2d, int32_t n_h2d,
                                                const lora_sgmv_problem* problems, int32_t n_problems, int32_t r,
                                                lora_sgmv_dtype dtype, uint32_t flags, const lora_sgmv_copy* d2h,
                                                int32_t n_d2h, uint32_t* dev_status, int32_t* n_segments_out,
                                                void* stream) {
    if (!meta_host || !meta_dev || !problems || (T > 0 && !ids)) return LORA_SGMV_ERR_NULL;
    if (T < 0 || num_adapters < 1 || n_problems < 1 || n_problems > LORA_SGMV_MAX_PROBLEMS) return LORA_SGMV_ERR_DIM;
    if (!copies_valid(h2d, n_h2d) || !copies_valid(d2h, n_d2h)) return LORA_SGMV_ERR_NULL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // 1. grouping, on the host: seg_starts straight into meta_host, lora_idx after them
    thread_local std::vector<int32_t> idx, perm_local;
    idx.resize(static_cast<size_t>(num_adapters));
    int32_t* pm = perm;
    if (!pm) {
        perm_local.resize(static_cast<size_t>(std::max(T, 1)));
        pm = perm_local.data();
    }
    int32_t n = 0;
    lora_sgmv_status st = lora_sgmv_group_segments(ids, T, num_adapters, meta_host, idx.data(), pm, &n);
    if (st != LORA_SGMV_OK) return st;
    std::memcpy(meta_host + n + 1, idx.data(), sizeof(int32_t) * static_cast<size_t>(n));
    int32_t max_len = 0;
    for (int32_t k = 0; k < n; ++k) max_len = std::max(max_len, meta_host[k + 1] - meta_host[k]);
    if (n_segments_out) *n_segments_out = n;

    // 2. copies in (one of them carries meta_host to meta_dev), 3. the launch, 4. copies out
    st = copy_all(h2d, n_h2d, cudaMemcpyHostToDevice, s);
    if (st != LORA_SGMV_OK) return st;
    if (n > 0) {
        st = lora_sgmv_apply_batched_flags(problems, n_problems, meta_dev, meta_dev + n + 1, n, T, r, dtype, max_len,
                                           flags, dev_status, stream);
        if (st != LORA_SGMV_OK) return st;
    }
    return copy_all(d2h, n_d2h, cudaMemcpyDeviceToHost, s);
}

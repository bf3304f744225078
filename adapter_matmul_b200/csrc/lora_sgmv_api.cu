// lora_sgmv_api.cu -- C ABI entry points: host-side validation, dispatch, launches.
//
// Every entry point validates its host-visible arguments first and returns an
// error code without launching anything when one is wrong. Arrays that live on
// the device (segments, adapter tables) are checked by the kernels per segment.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/lora_sgmv.h"
#include "sgmv_decode_tc.cuh"
#include "sgmv_fused.cuh"
#include "sgmv_gemm_tc2.cuh"
#include "sgmv_grouped_tc.cuh"
#include "sgmv_pad.cuh"
#include "sgmv_split.cuh"

namespace {

using sgmv::ExpandParams;
using sgmv::ShrinkParams;

constexpr int kVersion = 300;  // 0.3.0: early reads before the PDL wait only on request (flags)

// Number of kernels this library has launched successfully in this process.
std::atomic<uint64_t> g_launches{0};

// Last CUDA error a call of this thread ran into (cudaSuccess if none).
thread_local cudaError_t t_last_error = cudaSuccess;

cudaError_t record(cudaError_t e) {
    if (e != cudaSuccess) t_last_error = e;
    return e;
}

lora_sgmv_status counted(cudaError_t e) {
    if (record(e) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return LORA_SGMV_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool split_rank(int r) { return r == 8 || r == 16 || r == 32 || r == 64 || r == 128; }

// Lazily filled per-device facts, guarded by a mutex.
constexpr int kMaxDevices = 64;

struct DeviceFacts {
    int dev = 0;
    int sms = 0;
    int max_smem_optin = 0;
};
std::mutex g_mu;
std::vector<DeviceFacts> g_devices;

lora_sgmv_status device_facts(DeviceFacts& out) {
    int dev = 0;
    if (record(cudaGetDevice(&dev)) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (dev >= static_cast<int>(g_devices.size())) g_devices.resize(dev + 1);
    DeviceFacts& f = g_devices[dev];
    f.dev = dev;
    if (f.sms == 0) {
        if (cudaDeviceGetAttribute(&f.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&f.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess) {
            f.sms = 0;
            return LORA_SGMV_ERR_CUDA;
        }
    }
    out = f;
    return LORA_SGMV_OK;
}

// Opt a kernel into the dynamic shared memory a launch needs (above 48 KB), per device.
// `granted` holds, per device, the largest size already granted to this kernel.
template <typename K>
lora_sgmv_status ensure_smem(K kernel, size_t bytes, int* granted) {
    if (bytes <= 48 * 1024) return LORA_SGMV_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    if (dev < 0 || dev >= 64) return LORA_SGMV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (static_cast<size_t>(granted[dev]) >= bytes) return LORA_SGMV_OK;
    if (record(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes))) !=
        cudaSuccess)
        return LORA_SGMV_ERR_CUDA;
    granted[dev] = static_cast<int>(bytes);
    return LORA_SGMV_OK;
}

// ---- split path: launch plans ----------------------------------------------------------

int clamp_grid_y(int n) { return std::min(n, 65535); }

// token-chunk slots from a segment-length estimate
int chunk_slots(int max_len, int tokens_per_chunk, int cap) {
    const int chunks = (std::max(max_len, 1) + tokens_per_chunk - 1) / tokens_per_chunk;
    return std::max(1, std::min(chunks, cap));
}

int cluster_size_for(int H1) {
    // enough CTAs to split H1 into slices of at least 256 rows, at most 8 (portable cluster)
    int c = 1;
    while (c < 8 && H1 / (c * 2) >= 256) c *= 2;
    return c;
}

// Largest number of clusters of `cluster` CTAs with `smem` bytes each that can be resident at once.
template <typename K>
lora_sgmv_status max_active_clusters(K kernel, int cluster, size_t smem, int* out, int threads = sgmv::kFusedThreads) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (record(cudaOccupancyMaxActiveClusters(&n, kernel, &cfg)) != cudaSuccess || n <= 0) return LORA_SGMV_ERR_CUDA;
    *out = n;
    return LORA_SGMV_OK;
}

template <typename T, int R>
lora_sgmv_status launch_shrink(const ShrinkParams& p0, int max_len, cudaStream_t stream) {
    static int smem_granted[64] = {};
    ShrinkParams p = p0;
    DeviceFacts f;
    if (device_facts(f) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
    p.flat = p.n_segments <= sgmv::kShrinkFlatMaxSegments ? 1 : 0;
    // at most one chunk per token, and at most one partial chunk per segment
    const long long units = std::min<long long>(
        static_cast<long long>(p.n_segments) + (p.T + sgmv::kShrinkTokens - 1) / sgmv::kShrinkTokens, p.T);
    int C = cluster_size_for(p.H1);
    // Fewer, longer CTAs when clusters of 8 would fill the SMs several times over: each chunk's
    // fixed steps (the chunk list, the first copies, the cluster reduction) are then paid by
    // half as many CTAs. Measured on the 70B-shaped decode (106 chunks, H1 = 8192, three CTAs
    // per SM): 8 CTAs per chunk 44.4 us, 4 CTAs 37.5 us.
    if (p.flat && C == 8 && units * 8 > 4ll * f.sms) C = 4;
    p.ks = ((p.H1 + C - 1) / C + 7) / 8 * 8;
    const size_t smem = sgmv::shrink_smem_bytes(R, p.flat ? p.n_segments : 0);
    if (smem > static_cast<size_t>(f.max_smem_optin)) return LORA_SGMV_ERR_DIM;
    auto kernel = sgmv::sgmv_shrink_cluster_kernel<T, R>;
    if (ensure_smem(kernel, smem, smem_granted) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;

    // X [T, H1] as boxes of {XB columns, 8 rows}; rows past T read as zeros
    CUtensorMap xmap;
    {
        const uint64_t d[2] = {uint64_t(p.H1), uint64_t(p.T)};
        const uint64_t st[1] = {uint64_t(p.H1) * 2};
        const uint32_t b[2] = {uint32_t(sgmv::shrink_x_box(R)), uint32_t(sgmv::kShrinkTokens)};
        const lora_sgmv_dtype dt = std::is_same<T, __half>::value ? LORA_SGMV_F16 : LORA_SGMV_BF16;
        if (!sgmv::encode_map(&xmap, p.X, dt, 2, d, st, b, CU_TENSOR_MAP_SWIZZLE_NONE)) {
            t_last_error = cudaErrorInvalidValue;
            return LORA_SGMV_ERR_CUDA;
        }
    }

    cudaLaunchConfig_t cfg = {};
    if (p.flat) {
        // one cluster per chunk: clusters beyond those resident at once start as others end,
        // which evens out the chunks' unequal durations (measured on the 70B-shaped decode:
        // 37.5 us, against 47.8 us with the grid cut to the resident clusters walking the list)
        cfg.gridDim = dim3(C, static_cast<unsigned>(std::max<long long>(1, std::min<long long>(units, 65535))), 1);
    } else {
        cfg.gridDim = dim3(C, clamp_grid_y(p.n_segments), chunk_slots(max_len, sgmv::kShrinkTokens, 8));
    }
    cfg.blockDim = dim3(sgmv::kShrinkThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // a plain launch: with programmatic dependent launch, CTAs placed early while the previous
    // kernel drains made the call slower (70B-shaped decode: 39.0 -> 43.6 us for the shrink)
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return counted(cudaLaunchKernelEx(&cfg, kernel, xmap, p));
}

template <typename T, int R>
lora_sgmv_status launch_expand(const ExpandParams& p, int max_len, bool after_shrink, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    const int cols_per_cta = sgmv::kExpandThreads * 8;
    cfg.gridDim = dim3((p.H2 + cols_per_cta - 1) / cols_per_cta, clamp_grid_y(p.n_segments),
                       chunk_slots(max_len, sgmv::kExpandTokens, 8));
    cfg.blockDim = dim3(sgmv::kExpandThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_shrink ? 1 : 0;
    return counted(cudaLaunchKernelEx(&cfg, sgmv::sgmv_expand_kernel<T, R>, p));
}

template <typename T>
lora_sgmv_status shrink_dispatch_r(const ShrinkParams& p, int r, int max_len, cudaStream_t s) {
    switch (r) {
        case 8: return launch_shrink<T, 8>(p, max_len, s);
        case 16: return launch_shrink<T, 16>(p, max_len, s);
        case 32: return launch_shrink<T, 32>(p, max_len, s);
        case 64: return launch_shrink<T, 64>(p, max_len, s);
        case 128: return launch_shrink<T, 128>(p, max_len, s);
    }
    return LORA_SGMV_ERR_UNSUPPORTED;
}

template <typename T>
lora_sgmv_status expand_dispatch_r(const ExpandParams& p, int r, int max_len, bool chained, cudaStream_t s) {
    switch (r) {
        case 8: return launch_expand<T, 8>(p, max_len, chained, s);
        case 16: return launch_expand<T, 16>(p, max_len, chained, s);
        case 32: return launch_expand<T, 32>(p, max_len, chained, s);
        case 64: return launch_expand<T, 64>(p, max_len, chained, s);
        case 128: return launch_expand<T, 128>(p, max_len, chained, s);
    }
    return LORA_SGMV_ERR_UNSUPPORTED;
}

lora_sgmv_status shrink_dispatch(const ShrinkParams& p, int r, lora_sgmv_dtype dt, int max_len, cudaStream_t s) {
    return dt == LORA_SGMV_F16 ? shrink_dispatch_r<__half>(p, r, max_len, s)
                               : shrink_dispatch_r<__nv_bfloat16>(p, r, max_len, s);
}

lora_sgmv_status expand_dispatch(const ExpandParams& p, int r, lora_sgmv_dtype dt, int max_len, bool chained,
                                 cudaStream_t s) {
    return dt == LORA_SGMV_F16 ? expand_dispatch_r<__half>(p, r, max_len, chained, s)
                               : expand_dispatch_r<__nv_bfloat16>(p, r, max_len, chained, s);
}

// ---- grouped tensor-core path ------------------------------------------------------------------

template <bool V_OUT>
cudaError_t grouped_launch_r(int r, bool bf, const CUtensorMap& tmX, const CUtensorMap& tmY, const CUtensorMap& tmA,
                             const CUtensorMap& tmB, const sgmv::GroupedParams& P, int blocks, cudaStream_t stream) {
    switch (r) {
        case 16:
            return bf ? sgmv::launch_grouped_tc_kernel<__nv_bfloat16, 16, V_OUT>(tmX, tmY, tmA, tmB, P, blocks, stream)
                      : sgmv::launch_grouped_tc_kernel<__half, 16, V_OUT>(tmX, tmY, tmA, tmB, P, blocks, stream);
        case 32:
            return bf ? sgmv::launch_grouped_tc_kernel<__nv_bfloat16, 32, V_OUT>(tmX, tmY, tmA, tmB, P, blocks, stream)
                      : sgmv::launch_grouped_tc_kernel<__half, 32, V_OUT>(tmX, tmY, tmA, tmB, P, blocks, stream);
        case 64:
            return bf ? sgmv::launch_grouped_tc_kernel<__nv_bfloat16, 64, V_OUT>(tmX, tmY, tmA, tmB, P, blocks, stream)
                      : sgmv::launch_grouped_tc_kernel<__half, 64, V_OUT>(tmX, tmY, tmA, tmB, P, blocks, stream);
    }
    return cudaErrorInvalidValue;
}

// The grouped tensor-core kernel: the whole SGMV (v_out null), or only the shrink, V = X@A_i
// (fp32) into v_out, with Y unused (the whole-layer path).
lora_sgmv_status launch_grouped(void* Y, const void* X, const void* const* A_ptrs, const void* const* B_ptrs,
                                const int32_t* seg_starts, const int32_t* lora_idx, int n_segments, int num_adapters,
                                int T, int H1, int r, int H2, float scale, lora_sgmv_dtype dt, uint32_t* dev_status,
                                cudaStream_t stream, float* v_out = nullptr, const int32_t* ranks = nullptr) {
    if (r != 16 && r != 32 && r != 64) return LORA_SGMV_ERR_UNSUPPORTED;
    DeviceFacts f;
    if (device_facts(f) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
    // Rows per M-tile: the fewest that keep every tile in one wave (at most ceil(T/tm) + n tiles
    // for the SMs), not under 64; with more rows than 128 SMs can take, full 128-row tiles.
    // A CTA streams its tile's X and Y rows plus A_i and B_i, so smaller tiles spread the rows
    // over more SMs at the cost of more (L2-resident) adapter reads.
    const int sms_avail = std::max(1, f.sms - n_segments);
    int tm = static_cast<int>(std::min<long long>(sgmv::kGM, ((static_cast<long long>(T) + sms_avail - 1) / sms_avail + 7) / 8 * 8));
    tm = std::max(tm, 64);
    // X and Y as 3-D views {64 columns, T rows, blocks of 64 columns} when the width is a
    // multiple of 64, so that one copy brings two 64-column blocks; else row-major 2-D maps
    const bool x3d = H1 % 64 == 0;
    const bool y3d = !v_out && H2 % 64 == 0;
    auto view3d = [&](CUtensorMap* m, const void* base, int cols) {
        const uint64_t d[3] = {64, uint64_t(T), uint64_t(cols / 64)};
        const uint64_t st[2] = {uint64_t(cols) * 2, 128};
        const uint32_t b[3] = {64, uint32_t(tm), 2};
        return sgmv::encode_map(m, base, dt, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B);
    };
    CUtensorMap tmX, tmY;
    if (!(x3d ? view3d(&tmX, X, H1) : sgmv::make_tile_map(&tmX, X, T, H1, dt, tm)) ||
        !(y3d ? view3d(&tmY, Y, H2)
              : sgmv::make_tile_map(&tmY, v_out ? X : Y, T, v_out ? H1 : H2, dt, tm))) {  // (unused with v_out)
        t_last_error = cudaErrorInvalidValue;
        return LORA_SGMV_ERR_CUDA;
    }
    sgmv::GroupedParams P = {};
    P.x3d = x3d ? 1 : 0;
    P.y3d = y3d ? 1 : 0;
    P.Y = Y;
    P.A_ptrs = A_ptrs;
    P.B_ptrs = B_ptrs;
    P.seg_starts = seg_starts;
    P.lora_idx = lora_idx;
    P.dev_status = dev_status;
    P.n_segments = n_segments;
    P.num_adapters = num_adapters;
    P.T = T;
    P.H1 = H1;
    P.H2 = H2;
    P.scale = scale;
    P.v_out = v_out;
    P.ranks = ranks;
    // templates of the A_i and B_i maps; each CTA replaces the address with its adapter's
    CUtensorMap tmA, tmB;
    {
        // A_i boxes of r columns x 128 rows: both K-steps of a shrink stage in one copy
        const uint64_t da[2] = {uint64_t(r), uint64_t(H1)};
        const uint64_t sa[1] = {uint64_t(r) * 2};
        const uint32_t ba[2] = {uint32_t(r), uint32_t(2 * sgmv::kGK)};
        const CUtensorMapSwizzle swa =
            r == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : (r == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
        // B_i: {64 columns, r rows, blocks of 64 columns} with boxes of two blocks, or 2-D boxes
        // of r rows x 64 columns
        const uint64_t db3[3] = {64, uint64_t(r), uint64_t(H2 / 64)};
        const uint64_t sb3[2] = {uint64_t(H2) * 2, 128};
        const uint32_t bb3[3] = {64, uint32_t(r), 2};
        const uint64_t db[2] = {uint64_t(H2), uint64_t(r)};
        const uint64_t sb[1] = {uint64_t(H2) * 2};
        const uint32_t bb[2] = {64, uint32_t(r)};
        if (!sgmv::encode_map(&tmA, X, dt, 2, da, sa, ba, swa) ||
            !(y3d ? sgmv::encode_map(&tmB, X, dt, 3, db3, sb3, bb3, CU_TENSOR_MAP_SWIZZLE_128B)
                  : sgmv::encode_map(&tmB, X, dt, 2, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_128B))) {
            t_last_error = cudaErrorInvalidValue;
            return LORA_SGMV_ERR_CUDA;
        }
    }
    // M-tiles: at most ceil(T/128) + n (each segment adds at most one partial tile)
    P.tm = tm;
    const long long tiles_ub = (static_cast<long long>(T) + tm - 1) / tm + n_segments;
    const long long tiles_est = std::max<long long>(1, (static_cast<long long>(T) + tm - 1) / tm);
    const int max_split = (H2 + sgmv::kGN - 1) / sgmv::kGN;
    // N-slices per M-tile: every CTA of a tile streams the tile's X rows and A_i again and its
    // slice of Y and B_i, one CTA per SM at a time; pick the split with the least bytes on the
    // busiest SM (the slices of a tile run on different SMs)
    int nsplit = 1;
    {
        const double shrink = (double(tm) * H1 + double(H1) * r) * 2;
        const double expand = (2.0 * tm * H2 + double(r) * H2) * 2;
        const int sms = std::max(f.sms, 1);
        double best = 1e300;
        for (int ns = 1; ns <= std::min(max_split, 16); ++ns) {
            const double per_sm = double((tiles_est * ns + sms - 1) / sms) * (shrink + expand / ns);
            if (per_sm < best * (1 - 1e-9)) {
                best = per_sm;
                nsplit = ns;
            }
        }
    }
    if (v_out) nsplit = 1;  // the shrink alone: one CTA per M-tile
    const int span_tiles = ((H2 + sgmv::kGN - 1) / sgmv::kGN + nsplit - 1) / nsplit;
    P.nspan = span_tiles * sgmv::kGN;
    P.nsplit = (H2 + P.nspan - 1) / P.nspan;
    const long long blocks = tiles_ub * P.nsplit;
    if (blocks > (1ll << 31) - 1) return LORA_SGMV_ERR_DIM;
    const bool bf = dt == LORA_SGMV_BF16;
    const cudaError_t e = v_out ? grouped_launch_r<true>(r, bf, tmX, tmY, tmA, tmB, P, int(blocks), stream)
                                : grouped_launch_r<false>(r, bf, tmX, tmY, tmA, tmB, P, int(blocks), stream);
    return counted(e);
}

int estimate_max_len(int max_seg_len, int T, int n) {
    if (max_seg_len > 0) return std::min(max_seg_len, std::max(T, 1));
    return n > 0 ? (T + n - 1) / n : T;
}

// ---- fused path ---------------------------------------------------------------------------

int round8(int v) { return (v + 7) / 8 * 8; }

template <typename T, int R, int CH>
lora_sgmv_status launch_fused(sgmv::FusedParams P, int max_len, cudaStream_t stream) {
    static int smem_granted[64] = {};
    // resident clusters per (device, log2 cluster size, job-prefix size bucket)
    static int resident[64][4][9] = {};
    using G = sgmv::FusedGeom<R, CH>;
    if (P.n_segments > sgmv::kFusedMaxSegments) return LORA_SGMV_ERR_DIM;
    const int bucket = (P.n_segments + 1 + 1023) / 1024;  // 1..9
    const size_t smem = G::BASE + size_t(bucket) * 1024 * 4;
    auto kernel = sgmv::sgmv_fused_kernel<T, R, CH>;
    if (ensure_smem(kernel, smem, smem_granted) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
    int dev = 0;
    if (record(cudaGetDevice(&dev)) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    if (dev < 0 || dev >= 64) return LORA_SGMV_ERR_UNSUPPORTED;
    auto resident_for = [&](int lc, int* out) -> lora_sgmv_status {
        {
            std::lock_guard<std::mutex> lock(g_mu);
            if (resident[dev][lc][bucket - 1] > 0) {
                *out = resident[dev][lc][bucket - 1];
                return LORA_SGMV_OK;
            }
        }
        int n = 0;
        lora_sgmv_status st = max_active_clusters(kernel, 1 << lc, smem, &n);
        if (st != LORA_SGMV_OK) return st;
        std::lock_guard<std::mutex> lock(g_mu);
        resident[dev][lc][bucket - 1] = n;
        *out = n;
        return LORA_SGMV_OK;
    };
    // jobs: token chunks of <= CH over all segments and problems (upper bound from T and n)
    const long long chunks = std::min<long long>(P.n_segments + (P.T + CH - 1) / CH, std::max(P.T, 1));
    const long long jobs =
        std::max<long long>(1, (max_len <= CH ? static_cast<long long>(P.n_segments) : chunks) * P.n_problems);
    int ctas = 0;
    lora_sgmv_status st = resident_for(0, &ctas);
    if (st != LORA_SGMV_OK) return st;
    // cluster size: the largest C whose jobs*C CTAs are all resident at once, counting both the
    // CTA slots and the clusters of C the GPU places at once (clusters of 8 fit fewer times than
    // the CTA count suggests: a cluster's CTAs share a GPC); 1 if even that is too many
    int lc = 3;
    while (lc > 0) {
        int cm = 0;
        if (jobs * (1ll << lc) <= ctas && resident_for(lc, &cm) == LORA_SGMV_OK && jobs <= cm) break;
        --lc;
    }
    int clusters_max = 0;
    st = resident_for(lc, &clusters_max);
    if (st != LORA_SGMV_OK) return st;
    const int C = 1 << lc;
    P.one_chunk = max_len <= CH ? 1 : 0;
    for (int i = 0; i < P.n_problems; ++i) {
        P.prob[i].ks = round8((P.prob[i].H1 + C - 1) / C);
        P.prob[i].ns = round8((P.prob[i].H2 + C - 1) / C);
    }
    int clusters = static_cast<int>(std::min<long long>(jobs, clusters_max));
    const long long rounds = (jobs + clusters - 1) / clusters;  // balance jobs per cluster
    clusters = static_cast<int>((jobs + rounds - 1) / rounds);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(clusters * C, 1, 1);
    cfg.blockDim = dim3(sgmv::kFusedThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return counted(cudaLaunchKernelEx(&cfg, kernel, P));
}

// ---- tensor-core decode path -------------------------------------------------------------------

// Dispatch between the two fused decode kernels, from measurements on B200: the tensor-core
// kernel wins once segments hold several tokens and r is large enough that its expand
// (r x 16-token MMAs) replaces a long fp32 FMA loop; at r = 16 the CUDA-core kernel stays ahead.
bool decode_tc_preferred(int r, int max_len) { return max_len > 2 && r >= 32; }

// The split form of the tensor-core decode (V by the split-K shrink kernel, then an expand that
// spreads each job's N over independent CTAs) pays a second launch and a V round trip through
// the workspace, and wins when the fused form would leave SMs idle: fewer jobs than SMs, each
// with a large B_i to stream (measured on the 70B-shaped decode, 111 jobs: split 135 vs fused
// 177 us at 3.7 MB per B_i, 80 vs 83 us at 1 MB).
bool split_tc_preferred(int T, int n_segments, int max_len, int H2, int r, int sms) {
    const long long chunks = std::min<long long>(n_segments + (T + 15) / 16, std::max(T, 1));
    const long long jobs = max_len <= 16 ? n_segments : chunks;
    return jobs < sms && double(H2) * r * 2 >= 1e6;
}

bool decode_tc_supported(int r, int H1, int H2) {
    return (r == 16 || r == 32 || r == 64) && H1 >= 64 && H2 >= 64 && H1 % 64 == 0 && H2 % 64 == 0;
}

// The kernels AUTO runs for a call (host arithmetic only). max_len: the longest segment, as
// estimated by estimate_max_len; sms: the device's SM count.
lora_sgmv_variant auto_variant(int T, int n_segments, int max_len, int H1, int H2, int r, lora_sgmv_dtype dtype,
                               int sms) {
    if (max_len >= sgmv::kGroupedMinSegment && sgmv::grouped_tc_supported(r, H1, H2, dtype))
        return LORA_SGMV_VARIANT_GROUPED_TC;
    if (n_segments > sgmv::kFusedMaxSegments) return LORA_SGMV_VARIANT_SPLIT;
    if (decode_tc_preferred(r, max_len) && decode_tc_supported(r, H1, H2))
        return split_tc_preferred(T, n_segments, max_len, H2, r, sms) ? LORA_SGMV_VARIANT_SPLIT_TC
                                                                          : LORA_SGMV_VARIANT_FUSED_TC;
    return LORA_SGMV_VARIANT_FUSED;
}

// PRE_V: V comes from an earlier kernel (v_in); else the clusters compute it
template <typename T, int R, bool PRE_V>
lora_sgmv_status launch_decode_tc(sgmv::FusedParams P, const sgmv::DecodeMaps& maps, int max_len, cudaStream_t stream,
                                  const float* v_in) {
    static int smem_granted[64] = {};
    // resident clusters per (device, cluster size, job-prefix size bucket)
    static int resident[64][sgmv::kFusedMaxCluster + 1][9] = {};
    using G = sgmv::DecodeTCGeom<R, PRE_V>;
    constexpr int CH = sgmv::kDTokens;
    if (P.n_segments > sgmv::kFusedMaxSegments) return LORA_SGMV_ERR_DIM;
    const int bucket = (P.n_segments + 1 + 1023) / 1024;  // 1..9
    auto smem_for = [&](int C) {
        return G::BASE + size_t(C) * G::TILE + size_t(bucket) * 1024 * 4 + 1024 /* alignment slack */;
    };
    auto kernel = sgmv::sgmv_decode_tc_kernel<T, R, PRE_V>;
    DeviceFacts f;
    if (device_facts(f) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
    // the largest cluster whose shared memory (ring + one partial V tile per CTA of the cluster
    // + the job prefix) fits a CTA, leaving 4 KB for the kernel's static shared memory
    const size_t smem_cap = f.max_smem_optin > 4096 ? size_t(f.max_smem_optin) - 4096 : 0;
    int c_fit = sgmv::kFusedMaxCluster;
    while (c_fit > 0 && smem_for(c_fit) > smem_cap) --c_fit;
    if (c_fit == 0) return LORA_SGMV_ERR_DIM;
    if (ensure_smem(kernel, smem_for(c_fit), smem_granted) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
    int dev = 0;
    if (record(cudaGetDevice(&dev)) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    if (dev < 0 || dev >= 64) return LORA_SGMV_ERR_UNSUPPORTED;
    auto resident_for = [&](int C, int* out) -> lora_sgmv_status {
        {
            std::lock_guard<std::mutex> lock(g_mu);
            if (resident[dev][C][bucket - 1] > 0) {
                *out = resident[dev][C][bucket - 1];
                return LORA_SGMV_OK;
            }
        }
        int n = 0;
        lora_sgmv_status st = max_active_clusters(kernel, C, smem_for(C), &n, sgmv::kDThreads);
        if (st != LORA_SGMV_OK) return st;
        std::lock_guard<std::mutex> lock(g_mu);
        resident[dev][C][bucket - 1] = n;
        *out = n;
        return LORA_SGMV_OK;
    };
    const bool one_chunk = max_len <= CH;
    const long long chunks =
        std::min<long long>(P.n_segments + (P.T + CH - 1) / CH, std::max(P.T, 1));
    const long long jobs = std::max<long long>(1, (one_chunk ? static_cast<long long>(P.n_segments) : chunks) *
                                                      P.n_problems);
    if constexpr (PRE_V) {
        // V is precomputed: each job's N is cut into S slices and the jobs x S units are walked
        // by independent CTAs, all resident at once. Estimated time = rounds x (slice bytes at
        // the ~24 GB/s one CTA of this kernel streams + a fixed cost per unit).
        constexpr double kCtaBytesPerUs = 24e3;
        constexpr double kUnitFixedUs = 3.0;
        int resident1 = 0;
        lora_sgmv_status st1 = resident_for(1, &resident1);
        if (st1 != LORA_SGMV_OK) return st1;
        resident1 = std::max(resident1, 1);
        int s_cap = 16;
        double job_bytes = 0;
        for (int i = 0; i < P.n_problems; ++i) {
            s_cap = std::min(s_cap, (P.prob[i].H2 + G::NW - 1) / G::NW);
            job_bytes += double(P.prob[i].H2) * R * 2;
        }
        job_bytes /= P.n_problems;
        s_cap = std::max(s_cap, 1);
        int S = 1;
        long long rounds = 1;
        double best = 1e300;
        for (int sl = 1; sl <= s_cap; ++sl) {
            const long long units = jobs * sl;
            const long long rd = (units + resident1 - 1) / resident1;
            const double cost = double(rd) * (job_bytes / sl / kCtaBytesPerUs + kUnitFixedUs);
            if (cost < best - 1e-9) {
                best = cost;
                S = sl;
                rounds = rd;
            }
        }
        P.one_chunk = one_chunk ? 1 : 0;
        for (int i = 0; i < P.n_problems; ++i) {
            P.prob[i].ks = 0;  // no shrink
            P.prob[i].ns = (P.prob[i].H2 + S * G::NW - 1) / (S * G::NW) * G::NW;
        }
        const long long ctas = (jobs * S + rounds - 1) / rounds;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
        cfg.blockDim = dim3(sgmv::kDThreads, 1, 1);
        cfg.dynamicSmemBytes = smem_for(1);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return counted(cudaLaunchKernelEx(&cfg, kernel, maps, P, v_in, S));
    }
    // cluster size: a cluster runs its jobs one after another, each CTA streaming 1/C of the
    // job's adapter bytes; estimated time = rounds * (bytes per CTA / per-CTA bandwidth + a fixed
    // cost per job for metadata, map setup, pipeline fill and the V exchange). Every CTA keeps at
    // least one stage of A_i and of B_i.
    constexpr double kCtaBytesPerUs = 40e3;  // ~40 GB/s that one CTA streams with TMA
    constexpr double kJobFixedUs = 4.0;
    int c_cap = c_fit;
    double job_bytes = 0;
    for (int i = 0; i < P.n_problems; ++i) {
        c_cap = std::min(c_cap, (P.prob[i].H1 + G::KS - 1) / G::KS);
        c_cap = std::min(c_cap, (P.prob[i].H2 + G::NW - 1) / G::NW);
        job_bytes += (double(P.prob[i].H1) + double(P.prob[i].H2)) * R * 2;
    }
    job_bytes /= P.n_problems;
    c_cap = std::max(c_cap, 1);
    int C = 1, clusters_max = 0;
    double best = 1e300;
    for (int c = 1; c <= c_cap; ++c) {
        int cm = 0;
        lora_sgmv_status st = resident_for(c, &cm);
        if (st != LORA_SGMV_OK) {
            if (c == 1) return st;
            continue;  // this cluster size cannot be scheduled here
        }
        const long long rounds = (jobs + cm - 1) / cm;
        const double cost = double(rounds) * (job_bytes / c / kCtaBytesPerUs + kJobFixedUs);
        if (cost < best - 1e-9) {
            best = cost;
            C = c;
            clusters_max = cm;
        }
    }
    P.one_chunk = one_chunk ? 1 : 0;
    for (int i = 0; i < P.n_problems; ++i) {
        P.prob[i].ks = (P.prob[i].H1 + C * G::KS - 1) / (C * G::KS) * G::KS;
        P.prob[i].ns = (P.prob[i].H2 + C * G::NW - 1) / (C * G::NW) * G::NW;
    }
    int clusters = static_cast<int>(std::min<long long>(jobs, clusters_max));
    const long long rounds = (jobs + clusters - 1) / clusters;
    clusters = static_cast<int>((jobs + rounds - 1) / rounds);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(clusters * C, 1, 1);
    cfg.blockDim = dim3(sgmv::kDThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_for(C);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return counted(cudaLaunchKernelEx(&cfg, kernel, maps, P, static_cast<const float*>(nullptr), 1));
}

template <int R>
lora_sgmv_status decode_tc_maps_and_launch(sgmv::FusedParams& P, lora_sgmv_dtype dt, int max_len, cudaStream_t s,
                                           const float* v_in) {
    sgmv::DecodeMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    for (int i = 0; i < P.n_problems; ++i) {
        const bool ok = v_in ? sgmv::make_decode_maps<R, true>(maps, i, P.prob[i].X, P.prob[i].Y, P.T, P.prob[i].H1,
                                                               P.prob[i].H2, dt)
                             : sgmv::make_decode_maps<R, false>(maps, i, P.prob[i].X, P.prob[i].Y, P.T, P.prob[i].H1,
                                                                P.prob[i].H2, dt);
        if (!ok) {
            t_last_error = cudaErrorInvalidValue;
            return LORA_SGMV_ERR_CUDA;
        }
    }
    if (v_in)
        return dt == LORA_SGMV_BF16 ? launch_decode_tc<__nv_bfloat16, R, true>(P, maps, max_len, s, v_in)
                                    : launch_decode_tc<__half, R, true>(P, maps, max_len, s, v_in);
    return dt == LORA_SGMV_BF16 ? launch_decode_tc<__nv_bfloat16, R, false>(P, maps, max_len, s, v_in)
                                : launch_decode_tc<__half, R, false>(P, maps, max_len, s, v_in);
}

// v_in: V from an earlier kernel (the split form)
lora_sgmv_status decode_tc_dispatch(sgmv::FusedParams& P, int r, lora_sgmv_dtype dt, int max_len, cudaStream_t s,
                                    const float* v_in = nullptr) {
    switch (r) {
        case 16: return decode_tc_maps_and_launch<16>(P, dt, max_len, s, v_in);
        case 32: return decode_tc_maps_and_launch<32>(P, dt, max_len, s, v_in);
        case 64: return decode_tc_maps_and_launch<64>(P, dt, max_len, s, v_in);
    }
    return LORA_SGMV_ERR_UNSUPPORTED;
}

// Tokens per job of the fused kernel: 8, or 4 when segments reach 16 tokens, whose chunks would
// otherwise each stream 8 Y rows and do 8 tokens' fp32 expand on one cluster. Measured on the
// Skewed layer (H2 = 11008): 44.0 -> 26.9 us; Identical: 25.0 -> 16.4 us; the Uniform layer,
// whose segments hold 1-9 tokens, is better with 8 (25.4 vs 26.0 us).
constexpr int kFusedLongSegment = 16;

template <typename T, int CH>
lora_sgmv_status fused_dispatch_rc(const sgmv::FusedParams& P, int r, int max_len, cudaStream_t s) {
    switch (r) {
        case 8: return launch_fused<T, 8, CH>(P, max_len, s);
        case 16: return launch_fused<T, 16, CH>(P, max_len, s);
        case 32: return launch_fused<T, 32, CH>(P, max_len, s);
        case 64: return launch_fused<T, 64, CH>(P, max_len, s);
        case 128: return launch_fused<T, 128, CH>(P, max_len, s);
    }
    return LORA_SGMV_ERR_UNSUPPORTED;
}

template <typename T>
lora_sgmv_status fused_dispatch_r(const sgmv::FusedParams& P, int r, int max_len, cudaStream_t s) {
    return max_len >= kFusedLongSegment ? fused_dispatch_rc<T, 4>(P, r, max_len, s)
                                        : fused_dispatch_rc<T, sgmv::kFusedTokens>(P, r, max_len, s);
}

lora_sgmv_status fused_dispatch(const sgmv::FusedParams& P, int r, lora_sgmv_dtype dt, int max_len,
                                cudaStream_t s) {
    return dt == LORA_SGMV_F16 ? fused_dispatch_r<__half>(P, r, max_len, s)
                               : fused_dispatch_r<__nv_bfloat16>(P, r, max_len, s);
}

// One padding launch: dst [rows_dst, cols_dst] from src [rows_src, cols_src] (16-bit elements).
lora_sgmv_status launch_pad(void* dst, const void* src, int64_t rows_dst, int64_t cols_dst, int64_t rows_src,
                            int64_t cols_src, cudaStream_t stream) {
    DeviceFacts f;
    if (device_facts(f) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
    const int64_t n = rows_dst * cols_dst;
    const int64_t blocks = std::max<int64_t>(
        1, std::min<int64_t>((n + sgmv::kPadThreads - 1) / sgmv::kPadThreads, int64_t(f.sms) * 8));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(sgmv::kPadThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.numAttrs = 0;
    return counted(cudaLaunchKernelEx(&cfg, sgmv::sgmv_pad_kernel, static_cast<uint16_t*>(dst),
                                      static_cast<const uint16_t*>(src), rows_dst, cols_dst, rows_src, cols_src));
}

// Bytes of the fp32 V [T, r] a workspace holds (padded to 256 bytes).
size_t v_bytes_for(int32_t T, int32_t r) {
    const size_t v = static_cast<size_t>(T) * static_cast<size_t>(r) * sizeof(float);
    return (v + 255) / 256 * 256;
}

lora_sgmv_status check_common(int32_t n_segments, int32_t num_adapters, int32_t T, lora_sgmv_dtype dtype) {
    if (dtype != LORA_SGMV_F16 && dtype != LORA_SGMV_BF16) return LORA_SGMV_ERR_DTYPE;
    if (n_segments < 0 || T < 0 || num_adapters < 0) return LORA_SGMV_ERR_DIM;
    return LORA_SGMV_OK;
}

}  // namespace

extern "C" {

int32_t lora_sgmv_version(void) { return kVersion; }

lora_sgmv_variant lora_sgmv_auto_variant(int32_t T, int32_t n_segments, int32_t H1, int32_t r, int32_t H2,
                                         lora_sgmv_dtype dtype, int32_t max_seg_len, int32_t sm_count) {
    if (T <= 0 || n_segments <= 0 || H1 <= 0 || H2 <= 0 || r <= 0 || sm_count <= 0) return LORA_SGMV_VARIANT_AUTO;
    if (dtype != LORA_SGMV_F16 && dtype != LORA_SGMV_BF16) return LORA_SGMV_VARIANT_AUTO;
    return auto_variant(T, n_segments, estimate_max_len(max_seg_len, T, n_segments), H1, H2, r, dtype, sm_count);
}

uint64_t lora_sgmv_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* lora_sgmv_last_error(void) {
    return t_last_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(t_last_error);
}

int32_t lora_sgmv_rank_supported(int32_t r, lora_sgmv_variant variant) {
    switch (variant) {
        case LORA_SGMV_VARIANT_AUTO:
        case LORA_SGMV_VARIANT_SPLIT: return split_rank(r) ? 1 : 0;
        case LORA_SGMV_VARIANT_GROUPED_TC: return sgmv::grouped_tc_rank(r) ? 1 : 0;
        case LORA_SGMV_VARIANT_FUSED: return split_rank(r) ? 1 : 0;
        case LORA_SGMV_VARIANT_FUSED_TC:
        case LORA_SGMV_VARIANT_SPLIT_TC: return (r == 16 || r == 32 || r == 64) ? 1 : 0;
    }
    return 0;
}

const char* lora_sgmv_status_string(lora_sgmv_status status) {
    switch (status) {
        case LORA_SGMV_OK: return "ok";
        case LORA_SGMV_ERR_NULL: return "a required pointer is NULL";
        case LORA_SGMV_ERR_DIM: return "invalid size";
        case LORA_SGMV_ERR_ALIGN: return "pointer or row pitch not 16-byte aligned";
        case LORA_SGMV_ERR_DTYPE: return "unknown storage type";
        case LORA_SGMV_ERR_UNSUPPORTED: return "rank or variant not supported";
        case LORA_SGMV_ERR_CUDA: return "CUDA runtime error";
        case LORA_SGMV_ERR_WORKSPACE: return "workspace missing or too small";
        case LORA_SGMV_ERR_RANGE: return "value out of range";
    }
    return "unknown status";
}

lora_sgmv_status lora_sgmv_group_segments(const int32_t* ids, int32_t T, int32_t num_adapters,
                                          int32_t* seg_starts, int32_t* lora_idx, int32_t* perm,
                                          int32_t* n_segments) {
    if (!seg_starts || !lora_idx || !n_segments || (T > 0 && (!ids || !perm))) return LORA_SGMV_ERR_NULL;
    if (T < 0 || num_adapters < 1) return LORA_SGMV_ERR_DIM;
    for (int32_t t = 0; t < T; ++t)
        if (ids[t] < 0 || ids[t] >= num_adapters) return LORA_SGMV_ERR_RANGE;
    // counting sort: histogram, exclusive scan, stable scatter
    std::vector<int32_t> count(static_cast<size_t>(num_adapters) + 1, 0);
    for (int32_t t = 0; t < T; ++t) ++count[ids[t] + 1];
    int32_t n = 0;
    seg_starts[0] = 0;
    for (int32_t a = 0; a < num_adapters; ++a) {
        const int32_t c = count[a + 1];
        count[a + 1] += count[a];  // count[a] becomes the first row of adapter a
        if (c > 0) {
            lora_idx[n] = a;
            seg_starts[++n] = count[a + 1];
        }
    }
    for (int32_t t = 0; t < T; ++t) perm[count[ids[t]]++] = t;
    *n_segments = n;
    return LORA_SGMV_OK;
}

size_t lora_sgmv_workspace_bytes(int32_t T, int32_t r) {
    if (T <= 0 || r <= 0) return 0;
    return v_bytes_for(T, r);
}

lora_sgmv_status lora_sgmv_pad_rank(void* A_dst, const void* A_src, void* B_dst, const void* B_src, int32_t H1,
                                    int32_t H2, int32_t r_src, int32_t r, lora_sgmv_dtype dtype, void* stream) {
    if (dtype != LORA_SGMV_F16 && dtype != LORA_SGMV_BF16) return LORA_SGMV_ERR_DTYPE;
    const bool has_a = A_dst || A_src, has_b = B_dst || B_src;
    if (!has_a && !has_b) return LORA_SGMV_ERR_NULL;
    if ((has_a && (!A_dst || !A_src)) || (has_b && (!B_dst || !B_src))) return LORA_SGMV_ERR_NULL;
    if (r_src < 1 || r < r_src) return LORA_SGMV_ERR_DIM;
    if ((has_a && H1 < 1) || (has_b && H2 < 1)) return LORA_SGMV_ERR_DIM;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (has_a) {
        lora_sgmv_status st = launch_pad(A_dst, A_src, H1, r, H1, r_src, s);
        if (st != LORA_SGMV_OK) return st;
    }
    if (has_b) return launch_pad(B_dst, B_src, r, H2, r_src, H2, s);
    return LORA_SGMV_OK;
}

lora_sgmv_status lora_sgmv_shrink(float* V, const void* X, const void* const* A_ptrs,
                                  const int32_t* seg_starts, const int32_t* lora_idx,
                                  int32_t n_segments, int32_t num_adapters, int32_t T, int32_t H1,
                                  int32_t r, lora_sgmv_dtype dtype, uint32_t* dev_status, void* stream) {
    lora_sgmv_status st = check_common(n_segments, num_adapters, T, dtype);
    if (st != LORA_SGMV_OK) return st;
    if (H1 <= 0 || r <= 0) return LORA_SGMV_ERR_DIM;
    if (!split_rank(r)) return LORA_SGMV_ERR_UNSUPPORTED;
    if (n_segments == 0 || T == 0) return LORA_SGMV_OK;
    if (!V || !X || !A_ptrs || !seg_starts || !lora_idx) return LORA_SGMV_ERR_NULL;
    if (num_adapters < 1) return LORA_SGMV_ERR_DIM;
    if (!aligned16(V) || !aligned16(X) || H1 % 8) return LORA_SGMV_ERR_ALIGN;
    ShrinkParams p = {};
    p.V = V;
    p.X = X;
    p.A_ptrs = A_ptrs;
    p.B_check = nullptr;
    p.seg_starts = seg_starts;
    p.lora_idx = lora_idx;
    p.dev_status = dev_status;
    p.n_segments = n_segments;
    p.num_adapters = num_adapters;
    p.T = T;
    p.H1 = H1;
    const int max_len = estimate_max_len(0, T, n_segments);
    return shrink_dispatch(p, r, dtype, max_len, static_cast<cudaStream_t>(stream));
}

lora_sgmv_status lora_sgmv_expand(void* Y, const float* V, const void* const* B_ptrs,
                                  const int32_t* seg_starts, const int32_t* lora_idx,
                                  int32_t n_segments, int32_t num_adapters, int32_t T, int32_t r,
                                  int32_t H2, float scale, lora_sgmv_dtype dtype, uint32_t* dev_status,
                                  void* stream) {
    lora_sgmv_status st = check_common(n_segments, num_adapters, T, dtype);
    if (st != LORA_SGMV_OK) return st;
    if (H2 <= 0 || r <= 0) return LORA_SGMV_ERR_DIM;
    if (!split_rank(r)) return LORA_SGMV_ERR_UNSUPPORTED;
    if (n_segments == 0 || T == 0) return LORA_SGMV_OK;
    if (!Y || !V || !B_ptrs || !seg_starts || !lora_idx) return LORA_SGMV_ERR_NULL;
    if (num_adapters < 1) return LORA_SGMV_ERR_DIM;
    if (!aligned16(Y) || !aligned16(V) || H2 % 8) return LORA_SGMV_ERR_ALIGN;
    ExpandParams p = {};
    p.Y = Y;
    p.V = V;
    p.B_ptrs = B_ptrs;
    p.A_check = nullptr;
    p.seg_starts = seg_starts;
    p.lora_idx = lora_idx;
    p.dev_status = dev_status;
    p.n_segments = n_segments;
    p.num_adapters = num_adapters;
    p.T = T;
    p.H2 = H2;
    p.scale = scale;
    const int max_len = estimate_max_len(0, T, n_segments);
    return expand_dispatch(p, r, dtype, max_len, false, static_cast<cudaStream_t>(stream));
}

lora_sgmv_status lora_sgmv_apply_flags(void* Y, const void* X, const void* const* A_ptrs,
                                       const void* const* B_ptrs, const int32_t* seg_starts,
                                       const int32_t* lora_idx, int32_t n_segments, int32_t num_adapters,
                                       int32_t T, int32_t H1, int32_t r, int32_t H2, float scale,
                                       lora_sgmv_dtype dtype, int32_t max_seg_len, void* workspace,
                                       size_t workspace_bytes, uint32_t* dev_status, lora_sgmv_variant variant,
                                       uint32_t flags, void* stream) {
    if (flags & ~uint32_t(LORA_SGMV_FLAG_EARLY_READS)) return LORA_SGMV_ERR_UNSUPPORTED;
    lora_sgmv_status st = check_common(n_segments, num_adapters, T, dtype);
    if (st != LORA_SGMV_OK) return st;
    if (H1 <= 0 || H2 <= 0 || r <= 0) return LORA_SGMV_ERR_DIM;
    if (variant != LORA_SGMV_VARIANT_AUTO && variant != LORA_SGMV_VARIANT_SPLIT &&
        variant != LORA_SGMV_VARIANT_GROUPED_TC && variant != LORA_SGMV_VARIANT_FUSED &&
        variant != LORA_SGMV_VARIANT_FUSED_TC && variant != LORA_SGMV_VARIANT_SPLIT_TC)
        return LORA_SGMV_ERR_UNSUPPORTED;
    if (!lora_sgmv_rank_supported(r, variant)) return LORA_SGMV_ERR_UNSUPPORTED;
    if (n_segments == 0 || T == 0) return LORA_SGMV_OK;
    if (!Y || !X || !A_ptrs || !B_ptrs || !seg_starts || !lora_idx) return LORA_SGMV_ERR_NULL;
    if (num_adapters < 1) return LORA_SGMV_ERR_DIM;
    if (!aligned16(Y) || !aligned16(X) || H1 % 8 || H2 % 8) return LORA_SGMV_ERR_ALIGN;
    if (!workspace || workspace_bytes < lora_sgmv_workspace_bytes(T, r)) return LORA_SGMV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return LORA_SGMV_ERR_ALIGN;
    const int max_len = estimate_max_len(max_seg_len, T, n_segments);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    lora_sgmv_variant v = variant;
    if (v == LORA_SGMV_VARIANT_AUTO) {
        DeviceFacts f;
        if (device_facts(f) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
        v = auto_variant(T, n_segments, max_len, H1, H2, r, dtype, f.sms);
    }

    if (v == LORA_SGMV_VARIANT_FUSED || v == LORA_SGMV_VARIANT_FUSED_TC || v == LORA_SGMV_VARIANT_SPLIT_TC) {
        if ((v == LORA_SGMV_VARIANT_FUSED_TC || v == LORA_SGMV_VARIANT_SPLIT_TC) && !decode_tc_supported(r, H1, H2))
            return LORA_SGMV_ERR_UNSUPPORTED;
        sgmv::FusedParams P = {};
        P.prob[0].Y = Y;
        P.prob[0].X = X;
        P.prob[0].A_ptrs = A_ptrs;
        P.prob[0].B_ptrs = B_ptrs;
        P.prob[0].num_adapters = num_adapters;
        P.prob[0].H1 = H1;
        P.prob[0].H2 = H2;
        P.prob[0].scale = scale;
        P.seg_starts = seg_starts;
        P.lora_idx = lora_idx;
        P.dev_status = dev_status;
        P.n_problems = 1;
        P.n_segments = n_segments;
        P.T = T;
        P.early = (flags & LORA_SGMV_FLAG_EARLY_READS) ? 1 : 0;
        if (v == LORA_SGMV_VARIANT_FUSED_TC) return decode_tc_dispatch(P, r, dtype, max_len, s);
        if (v == LORA_SGMV_VARIANT_SPLIT_TC) {
            // V first (split-K shrink kernel, fp32 into the workspace), then the expand spread
            // over every SM, each job's N split among independent CTAs (its B_i stages stream
            // while the shrink finishes)
            float* V = static_cast<float*>(workspace);
            ShrinkParams sp = {};
            sp.V = V;
            sp.X = X;
            sp.A_ptrs = A_ptrs;
            sp.B_check = B_ptrs;
            sp.seg_starts = seg_starts;
            sp.lora_idx = lora_idx;
            sp.dev_status = dev_status;
            sp.n_segments = n_segments;
            sp.num_adapters = num_adapters;
            sp.T = T;
            sp.H1 = H1;
            st = shrink_dispatch(sp, r, dtype, max_len, s);
            if (st != LORA_SGMV_OK) return st;
            return decode_tc_dispatch(P, r, dtype, max_len, s, V);
        }
        return fused_dispatch(P, r, dtype, max_len, s);
    }

    if (v == LORA_SGMV_VARIANT_GROUPED_TC) {
        if (!sgmv::grouped_tc_supported(r, H1, H2, dtype)) return LORA_SGMV_ERR_UNSUPPORTED;
        return launch_grouped(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r, H2,
                              scale, dtype, dev_status, s);
    }

    float* V = static_cast<float*>(workspace);

    ShrinkParams sp = {};
    sp.V = V;
    sp.X = X;
    sp.A_ptrs = A_ptrs;
    sp.B_check = B_ptrs;
    sp.seg_starts = seg_starts;
    sp.lora_idx = lora_idx;
    sp.dev_status = dev_status;
    sp.n_segments = n_segments;
    sp.num_adapters = num_adapters;
    sp.T = T;
    sp.H1 = H1;
    st = shrink_dispatch(sp, r, dtype, max_len, s);
    if (st != LORA_SGMV_OK) return st;

    ExpandParams ep = {};
    ep.Y = Y;
    ep.V = V;
    ep.B_ptrs = B_ptrs;
    ep.A_check = A_ptrs;
    ep.seg_starts = seg_starts;
    ep.lora_idx = lora_idx;
    ep.dev_status = nullptr;  // the shrink already reported this call's bad segments
    ep.n_segments = n_segments;
    ep.num_adapters = num_adapters;
    ep.T = T;
    ep.H2 = H2;
    ep.scale = scale;
    return expand_dispatch(ep, r, dtype, max_len, true, s);
}

lora_sgmv_status lora_sgmv_apply_ex(void* Y, const void* X, const void* const* A_ptrs,
                                    const void* const* B_ptrs, const int32_t* seg_starts,
                                    const int32_t* lora_idx, int32_t n_segments, int32_t num_adapters,
                                    int32_t T, int32_t H1, int32_t r, int32_t H2, float scale,
                                    lora_sgmv_dtype dtype, int32_t max_seg_len, void* workspace,
                                    size_t workspace_bytes, uint32_t* dev_status, lora_sgmv_variant variant,
                                    void* stream) {
    return lora_sgmv_apply_flags(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r,
                                 H2, scale, dtype, max_seg_len, workspace, workspace_bytes, dev_status, variant, 0u,
                                 stream);
}

lora_sgmv_status lora_sgmv_apply(void* Y, const void* X, const void* const* A_ptrs,
                                 const void* const* B_ptrs, const int32_t* seg_starts,
                                 const int32_t* lora_idx, int32_t n_segments, int32_t num_adapters,
                                 int32_t T, int32_t H1, int32_t r, int32_t H2, float scale,
                                 lora_sgmv_dtype dtype, int32_t max_seg_len, void* workspace,
                                 size_t workspace_bytes, uint32_t* dev_status, void* stream) {
    return lora_sgmv_apply_ex(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r,
                              H2, scale, dtype, max_seg_len, workspace, workspace_bytes, dev_status,
                              LORA_SGMV_VARIANT_AUTO, stream);
}

}  // extern "C"

extern "C" lora_sgmv_status lora_sgmv_apply_batched_flags(const lora_sgmv_problem* problems, int32_t n_problems,
                                                          const int32_t* seg_starts, const int32_t* lora_idx,
                                                          int32_t n_segments, int32_t T, int32_t r,
                                                          lora_sgmv_dtype dtype, int32_t max_seg_len, uint32_t flags,
                                                          uint32_t* dev_status, void* stream) {
    if (flags & ~uint32_t(LORA_SGMV_FLAG_EARLY_READS)) return LORA_SGMV_ERR_UNSUPPORTED;
    if (dtype != LORA_SGMV_F16 && dtype != LORA_SGMV_BF16) return LORA_SGMV_ERR_DTYPE;
    if (!problems) return LORA_SGMV_ERR_NULL;
    if (n_problems < 1 || n_problems > LORA_SGMV_MAX_PROBLEMS || n_segments < 0 || T < 0 || r <= 0)
        return LORA_SGMV_ERR_DIM;
    if (!split_rank(r)) return LORA_SGMV_ERR_UNSUPPORTED;
    sgmv::FusedParams P = {};
    for (int i = 0; i < n_problems; ++i) {
        const lora_sgmv_problem& q = problems[i];
        if (q.H1 <= 0 || q.H2 <= 0 || q.num_adapters < 0) return LORA_SGMV_ERR_DIM;
        if (n_segments > 0 && T > 0) {
            if (!q.Y || !q.X || !q.A_ptrs || !q.B_ptrs) return LORA_SGMV_ERR_NULL;
            if (q.num_adapters < 1) return LORA_SGMV_ERR_DIM;
            if (!aligned16(q.Y) || !aligned16(q.X) || q.H1 % 8 || q.H2 % 8) return LORA_SGMV_ERR_ALIGN;
        }
        P.prob[i].Y = q.Y;
        P.prob[i].X = q.X;
        P.prob[i].A_ptrs = q.A_ptrs;
        P.prob[i].B_ptrs = q.B_ptrs;
        P.prob[i].num_adapters = q.num_adapters;
        P.prob[i].H1 = q.H1;
        P.prob[i].H2 = q.H2;
        P.prob[i].scale = q.scale;
    }
    if (n_segments == 0 || T == 0) return LORA_SGMV_OK;
    if (!seg_starts || !lora_idx) return LORA_SGMV_ERR_NULL;
    P.seg_starts = seg_starts;
    P.lora_idx = lora_idx;
    P.dev_status = dev_status;
    P.n_problems = n_problems;
    P.n_segments = n_segments;
    P.T = T;
    P.early = (flags & LORA_SGMV_FLAG_EARLY_READS) ? 1 : 0;
    const int max_len = estimate_max_len(max_seg_len, T, n_segments);
    bool tc = decode_tc_preferred(r, max_len);
    for (int i = 0; i < n_problems; ++i) tc = tc && decode_tc_supported(r, problems[i].H1, problems[i].H2);
    if (tc) return decode_tc_dispatch(P, r, dtype, max_len, static_cast<cudaStream_t>(stream));
    return fused_dispatch(P, r, dtype, max_len, static_cast<cudaStream_t>(stream));
}

extern "C" lora_sgmv_status lora_sgmv_apply_batched(const lora_sgmv_problem* problems, int32_t n_problems,
                                                    const int32_t* seg_starts, const int32_t* lora_idx,
                                                    int32_t n_segments, int32_t T, int32_t r, lora_sgmv_dtype dtype,
                                                    int32_t max_seg_len, uint32_t* dev_status, void* stream) {
    return lora_sgmv_apply_batched_flags(problems, n_problems, seg_starts, lora_idx, n_segments, T, r, dtype,
                                         max_seg_len, 0u, dev_status, stream);
}

// ---- adapters of different ranks, unpadded ------------------------------------------------------

extern "C" lora_sgmv_status lora_sgmv_apply_ranks(void* Y, const void* X, const void* const* A_ptrs,
                                                  const void* const* B_ptrs, const int32_t* ranks,
                                                  const int32_t* seg_starts, const int32_t* lora_idx,
                                                  int32_t n_segments, int32_t num_adapters, int32_t T, int32_t H1,
                                                  int32_t r_max, int32_t H2, float scale, lora_sgmv_dtype dtype,
                                                  uint32_t* dev_status, void* stream) {
    lora_sgmv_status st = check_common(n_segments, num_adapters, T, dtype);
    if (st != LORA_SGMV_OK) return st;
    if (H1 <= 0 || H2 <= 0 || r_max <= 0) return LORA_SGMV_ERR_DIM;
    if (!sgmv::grouped_tc_rank(r_max)) return LORA_SGMV_ERR_UNSUPPORTED;
    if (H1 < 64 || H2 < 64) return LORA_SGMV_ERR_UNSUPPORTED;
    if (n_segments == 0 || T == 0) return LORA_SGMV_OK;
    if (!Y || !X || !A_ptrs || !B_ptrs || !ranks || !seg_starts || !lora_idx) return LORA_SGMV_ERR_NULL;
    if (num_adapters < 1) return LORA_SGMV_ERR_DIM;
    if (!aligned16(Y) || !aligned16(X) || H1 % 8 || H2 % 8) return LORA_SGMV_ERR_ALIGN;
    return launch_grouped(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r_max, H2,
                          scale, dtype, dev_status, static_cast<cudaStream_t>(stream), nullptr, ranks);
}

// ---- the whole layer: Y = X@W + scale * (X@A_i)@B_i ------------------------------------------

namespace {

// Rows from which the layer runs on SM pairs (256 x 256 tiles) rather than single SMs (128 x 256).
#ifndef SGMV_GEMM_PAIR_MIN_T
#define SGMV_GEMM_PAIR_MIN_T 256
#endif

template <int R>
lora_sgmv_status launch_gemm_r(const CUtensorMap& tmX, const CUtensorMap& tmW, const CUtensorMap& tmB,
                               const sgmv::GemmParams& P, lora_sgmv_dtype dt, int grid, cudaStream_t s) {
    return counted(dt == LORA_SGMV_BF16 ? sgmv::launch_gemm_delta_kernel<__nv_bfloat16, R>(tmX, tmW, tmB, P, grid, s)
                                        : sgmv::launch_gemm_delta_kernel<__half, R>(tmX, tmW, tmB, P, grid, s));
}

// Pairs of SMs that can be resident at once for the pair kernel (cached per device).
template <typename T, int R>
lora_sgmv_status gemm_pairs_resident(int dev, int* out) {
    static int cached[kMaxDevices] = {};
    if (dev < 0 || dev >= kMaxDevices) return LORA_SGMV_ERR_UNSUPPORTED;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (cached[dev] > 0) {
            *out = cached[dev];
            return LORA_SGMV_OK;
        }
    }
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(sgmv::sgmv_gemm_delta_pair_kernel<T, R>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sgmv::kL2Smem));
    });
    if (record(attr_err) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    int n = 0;
    lora_sgmv_status st = max_active_clusters(sgmv::sgmv_gemm_delta_pair_kernel<T, R>, 2, sgmv::kL2Smem, &n,
                                              sgmv::kLThreads);
    if (st != LORA_SGMV_OK) return st;
    std::lock_guard<std::mutex> lock(g_mu);
    cached[dev] = n;
    *out = n;
    return LORA_SGMV_OK;
}

template <typename T, int R>
lora_sgmv_status launch_gemm_pair_t(const CUtensorMap& tmX, const CUtensorMap& tmW, const CUtensorMap& tmB,
                                    const sgmv::GemmParams& P, int dev, cudaStream_t s) {
    int resident = 0;
    lora_sgmv_status st = gemm_pairs_resident<T, R>(dev, &resident);
    if (st != LORA_SGMV_OK) return st;
    const long long units = static_cast<long long>(P.m_tiles) * P.n_tiles;
    const int pairs = static_cast<int>(std::max<long long>(1, std::min<long long>(units, resident)));
    return counted(sgmv::launch_gemm_delta_pair_kernel<T, R>(tmX, tmW, tmB, P, pairs, s));
}

template <int R>
lora_sgmv_status launch_gemm_pair_r(const CUtensorMap& tmX, const CUtensorMap& tmW, const CUtensorMap& tmB,
                                    const sgmv::GemmParams& P, lora_sgmv_dtype dt, int dev, cudaStream_t s) {
    return dt == LORA_SGMV_BF16 ? launch_gemm_pair_t<__nv_bfloat16, R>(tmX, tmW, tmB, P, dev, s)
                                : launch_gemm_pair_t<__half, R>(tmX, tmW, tmB, P, dev, s);
}

}  // namespace

extern "C" lora_sgmv_status lora_sgmv_gemm_apply(void* Y, const void* X, const void* W, const void* const* A_ptrs,
                                                 const void* const* B_ptrs, const int32_t* seg_starts,
                                                 const int32_t* lora_idx, int32_t n_segments, int32_t num_adapters,
                                                 int32_t T, int32_t H1, int32_t r, int32_t H2, float scale,
                                                 lora_sgmv_dtype dtype, int32_t max_seg_len, void* workspace,
                                                 size_t workspace_bytes, uint32_t* dev_status, void* stream) {
    lora_sgmv_status st = check_common(n_segments, num_adapters, T, dtype);
    if (st != LORA_SGMV_OK) return st;
    if (H1 <= 0 || H2 <= 0 || r <= 0) return LORA_SGMV_ERR_DIM;
    if (!sgmv::gemm_tc_supported(r, H1, H2)) return (H1 % 8 || H2 % 8) ? LORA_SGMV_ERR_ALIGN : LORA_SGMV_ERR_UNSUPPORTED;
    if (T == 0) return LORA_SGMV_OK;
    if (!Y || !X || !W) return LORA_SGMV_ERR_NULL;
    if (n_segments > 0 && (!A_ptrs || !B_ptrs || !seg_starts || !lora_idx)) return LORA_SGMV_ERR_NULL;
    if (n_segments > 0 && num_adapters < 1) return LORA_SGMV_ERR_DIM;
    if (!aligned16(Y) || !aligned16(X) || !aligned16(W)) return LORA_SGMV_ERR_ALIGN;
    const size_t need = lora_sgmv_workspace_bytes(T, r);
    if (n_segments > 0 && (!workspace || workspace_bytes < need)) return LORA_SGMV_ERR_WORKSPACE;
    if (n_segments > 0 && !aligned16(workspace)) return LORA_SGMV_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DeviceFacts f;
    if (device_facts(f) != LORA_SGMV_OK) return LORA_SGMV_ERR_CUDA;
    float* V = static_cast<float*>(workspace);
    const int max_len = estimate_max_len(max_seg_len, T, n_segments);
    if (n_segments > 0) {
        // V = X@A_i first: the grouped tensor-core kernel's shrink for long segments, else the
        // split-K shrink kernel
        if (max_len >= sgmv::kGroupedMinSegment && H1 >= 64 && H2 >= 64) {
            st = launch_grouped(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r, H2,
                                scale, dtype, dev_status, s, V);
        } else {
            ShrinkParams sp = {};
            sp.V = V;
            sp.X = X;
            sp.A_ptrs = A_ptrs;
            sp.B_check = B_ptrs;
            sp.seg_starts = seg_starts;
            sp.lora_idx = lora_idx;
            sp.dev_status = nullptr;  // the layer kernel reports this call's bad segments
            sp.n_segments = n_segments;
            sp.num_adapters = num_adapters;
            sp.T = T;
            sp.H1 = H1;
            st = shrink_dispatch(sp, r, dtype, max_len, s);
        }
        if (st != LORA_SGMV_OK) return st;
    }
    CUtensorMap tmX, tmW, tmB;
    {
        const uint64_t dw[2] = {uint64_t(H2), uint64_t(H1)};
        const uint64_t sw[1] = {uint64_t(H2) * 2};
        const uint32_t bw[2] = {64, uint32_t(sgmv::kLK)};
        const uint64_t db[2] = {uint64_t(H2), uint64_t(r)};
        const uint64_t sb[1] = {uint64_t(H2) * 2};
        const uint32_t bb[2] = {64, uint32_t(r)};
        if (!sgmv::make_tile_map(&tmX, X, T, H1, dtype, sgmv::kLM) ||
            !sgmv::encode_map(&tmW, W, dtype, 2, dw, sw, bw, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !sgmv::encode_map(&tmB, W, dtype, 2, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_128B)) {
            t_last_error = cudaErrorInvalidValue;
            return LORA_SGMV_ERR_CUDA;
        }
    }
    sgmv::GemmParams P = {};
    P.Y = Y;
    P.V = V;
    P.A_ptrs = n_segments > 0 ? A_ptrs : nullptr;
    P.B_ptrs = n_segments > 0 ? B_ptrs : nullptr;
    P.seg_starts = seg_starts;
    P.lora_idx = lora_idx;
    P.dev_status = dev_status;
    P.n_segments = n_segments;
    P.num_adapters = num_adapters;
    P.T = T;
    P.H1 = H1;
    P.H2 = H2;
    P.scale = scale;
    P.v_after_wait = n_segments > 0 ? 1 : 0;  // V from the shrink just launched
    if (T >= SGMV_GEMM_PAIR_MIN_T) {
        P.m_tiles = (T + sgmv::kL2M - 1) / sgmv::kL2M;
        P.n_tiles = (H2 + sgmv::kL2N - 1) / sgmv::kL2N;
        if (static_cast<long long>(P.m_tiles) * P.n_tiles > (1ll << 31) - 1) return LORA_SGMV_ERR_DIM;
        switch (r) {
            case 16: return launch_gemm_pair_r<16>(tmX, tmW, tmB, P, dtype, f.dev, s);
            case 32: return launch_gemm_pair_r<32>(tmX, tmW, tmB, P, dtype, f.dev, s);
            case 64: return launch_gemm_pair_r<64>(tmX, tmW, tmB, P, dtype, f.dev, s);
        }
        return LORA_SGMV_ERR_UNSUPPORTED;
    }
    P.m_tiles = (T + sgmv::kLM - 1) / sgmv::kLM;
    P.n_tiles = (H2 + sgmv::kLN - 1) / sgmv::kLN;
    const long long units = static_cast<long long>(P.m_tiles) * P.n_tiles;
    if (units > (1ll << 31) - 1) return LORA_SGMV_ERR_DIM;
    const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(units, f.sms)));
    switch (r) {
        case 16: return launch_gemm_r<16>(tmX, tmW, tmB, P, dtype, grid, s);
        case 32: return launch_gemm_r<32>(tmX, tmW, tmB, P, dtype, grid, s);
        case 64: return launch_gemm_r<64>(tmX, tmW, tmB, P, dtype, grid, s);
    }
    return LORA_SGMV_ERR_UNSUPPORTED;
}

// ---- apply for callers that cannot allocate device memory -----------------------------------
//
// Some callers cannot call cudaMalloc or any other allocator when they run
// SGMV: code that runs inside a region where allocation is forbidden (a
// real-time serving loop whose memory is fixed at start-up, a plugin whose
// host framework owns all device memory), or code with no allocator handle at
// all. lora_sgmv_apply_noalloc serves them: it runs the split kernels with
// their fp32 V scratch in the fixed array below instead of a caller workspace.

namespace {
constexpr size_t kNoAllocMaxFloats = size_t(1) << 20;  // T * r <= 1,048,576 (4 MiB of fp32 V)
constexpr int kNoAllocMaxDevices = 64;
}  // namespace

// Held on every device that loads this library, until the process exits.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxFloats];

namespace {
std::mutex g_noalloc_mu;
float* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. The name of a
// __device__ array in host code is only a host-side stand-in; the address a
// kernel may use comes from cudaGetSymbolAddress, once per device, with that
// device current.
lora_sgmv_status noalloc_scratch(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LORA_SGMV_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return LORA_SGMV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LORA_SGMV_ERR_CUDA;
        g_noalloc_addr[dev] = static_cast<float*>(p);
    }
    *out = g_noalloc_addr[dev];
    return LORA_SGMV_OK;
}
}  // namespace

extern "C" lora_sgmv_status lora_sgmv_apply_noalloc(void* Y, const void* X, const void* const* A_ptrs,
                                                    const void* const* B_ptrs, const int32_t* seg_starts,
                                                    const int32_t* lora_idx, int32_t n_segments,
                                                    int32_t num_adapters, int32_t T, int32_t H1, int32_t r,
                                                    int32_t H2, float scale, lora_sgmv_dtype dtype,
                                                    int32_t max_seg_len, uint32_t* dev_status, void* stream) {
    if (T > 0 && r > 0 && static_cast<size_t>(T) * static_cast<size_t>(r) > kNoAllocMaxFloats)
        return LORA_SGMV_ERR_WORKSPACE;
    lora_sgmv_status st = check_common(n_segments, num_adapters, T, dtype);
    if (st != LORA_SGMV_OK) return st;
    if (n_segments == 0 || T == 0) return LORA_SGMV_OK;
    float* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != LORA_SGMV_OK) return st;
    return lora_sgmv_apply_ex(Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r, H2,
                              scale, dtype, max_seg_len, scratch, kNoAllocMaxFloats * sizeof(float), dev_status,
                              LORA_SGMV_VARIANT_SPLIT, stream);
}

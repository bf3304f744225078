// sgmv_tmap.cuh -- tensor maps for adapter tiles, made on the device.
//
// A_i and B_i are reached through a device table of pointers, so the host cannot build a
// tensor map per adapter. Instead the host encodes one template map per problem (shape,
// strides, box and swizzle of A_i or B_i, with a placeholder address) and a kernel makes
// the map of adapter i by copying the template into shared memory, replacing its global
// address (tensormap.replace) and publishing it to a global slot with a release fence of
// the tensormap proxy; the thread that issues the TMA copies acquires it first.
//
// Slots. Every CTA that builds maps owns one slot table for its lifetime: a ring of
// kMapRing entries, each an (A, B) pair of maps. Tables live in a fixed array inside the
// library and are claimed with an atomic compare-and-swap, starting from the CTA's SM and
// probing onward; a CTA releases its table after all of its copies have landed. The array
// holds more tables than CTAs that can be resident at once (every kernel that claims one
// uses over 64 KB of shared memory, so at most three per SM), so a claim never waits and
// never fails on a GPU of up to 256 SMs; if it ever did, the CTA reports
// LORA_SGMV_DEV_TIMEOUT and does no work.
#pragma once

#include <cuda.h>

#include <cstdint>

namespace sgmv {

constexpr int kMapRing = 4;          // jobs whose maps may be in use at once, per CTA
constexpr int kMapTables = 1024;     // claimable tables (>= resident CTAs)

struct alignas(128) MapTable {
    CUtensorMap m[2 * kMapRing];  // entry e: A map at 2e, B map at 2e + 1
};

__device__ MapTable g_map_tables[kMapTables];
__device__ unsigned int g_map_owner[kMapTables];

__device__ __forceinline__ uint32_t sm_id() {
    uint32_t v;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(v));
    return v;
}

// Claim a table (one thread). Returns its index, or -1 if none is free.
__device__ __forceinline__ int claim_map_table() {
    const int start = static_cast<int>((sm_id() * 4u) % kMapTables);
    for (int i = 0; i < kMapTables; ++i) {
        const int t = (start + i) % kMapTables;
        if (atomicCAS(&g_map_owner[t], 0u, 1u) == 0u) {
            __threadfence();
            return t;
        }
    }
    return -1;
}

// Release a table (one thread), after every copy that used its maps has completed.
__device__ __forceinline__ void release_map_table(int t) {
    if (t < 0) return;
    __threadfence();
    atomicExch(&g_map_owner[t], 0u);
}

// Whole warp: copy a 128-byte template map from parameter space into shared memory.
__device__ __forceinline__ void map_template_to_smem(CUtensorMap* smem_map, const CUtensorMap* tmpl) {
    const int lane = threadIdx.x & 31;
    if (lane < 8) {
        const uint4 v = reinterpret_cast<const uint4*>(tmpl)[lane];
        reinterpret_cast<uint4*>(smem_map)[lane] = v;
    }
    __syncwarp();
}

// One thread: set the global address of a map held in shared memory.
__device__ __forceinline__ void map_set_address(CUtensorMap* smem_map, const void* addr) {
    asm volatile("tensormap.replace.tile.global_address.shared::cta.b1024.b64 [%0], %1;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem_map))),
                 "l"(reinterpret_cast<uint64_t>(addr))
                 : "memory");
}

// One thread: set the extent of dimension ORD (elements) of a map held in shared memory.
template <int ORD>
__device__ __forceinline__ void map_set_dim(CUtensorMap* smem_map, uint32_t extent) {
    asm volatile("tensormap.replace.tile.global_dim.shared::cta.b1024.b32 [%0], %1, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem_map))),
                 "n"(ORD), "r"(extent)
                 : "memory");
}

// One thread: set the byte stride of dimension ORD + 1 of a map held in shared memory (a
// multiple of 16).
template <int ORD>
__device__ __forceinline__ void map_set_stride(CUtensorMap* smem_map, uint64_t stride_bytes) {
    asm volatile("tensormap.replace.tile.global_stride.shared::cta.b1024.b64 [%0], %1, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(smem_map))),
                 "n"(ORD), "l"(stride_bytes)
                 : "memory");
}

// Whole warp: copy the map from shared memory to its global slot and release it to the
// tensormap proxy.
__device__ __forceinline__ void map_publish(CUtensorMap* gmem_map, const CUtensorMap* smem_map) {
    asm volatile(
        "tensormap.cp_fenceproxy.global.shared::cta.tensormap::generic.release.gpu.sync.aligned [%0], [%1], 128;" ::"l"(
            reinterpret_cast<uint64_t>(gmem_map)),
        "r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_map)))
        : "memory");
}

// The thread that will issue copies through the map: acquire it from the tensormap proxy.
__device__ __forceinline__ void map_acquire(const CUtensorMap* gmem_map) {
    asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(reinterpret_cast<uint64_t>(gmem_map))
                 : "memory");
}

}  // namespace sgmv

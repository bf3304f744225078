// sgmv_common.cuh -- device helpers shared by the SGMV kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lora_sgmv.h"

namespace sgmv {

// Per-segment metadata as seen by one CTA, validated against the contract in
// lora_sgmv.h: bounds inside [0, T], adapter id in range, table entries
// non-null and 16-byte aligned.
struct Segment {
    int begin;
    int end;
    const void* a;  // A_i or nullptr when the caller does not need it
    const void* b;  // B_i or nullptr when the caller does not need it
};

// Reads and checks segment s. Returns 0 when the segment may be processed,
// else the LORA_SGMV_DEV_* bits describing why it is skipped.
__device__ __forceinline__ uint32_t load_segment(const int32_t* __restrict__ seg_starts,
                                                 const int32_t* __restrict__ lora_idx,
                                                 const void* const* __restrict__ A_ptrs,
                                                 const void* const* __restrict__ B_ptrs, int s,
                                                 int T, int num_adapters, Segment& out) {
    const int b = __ldg(seg_starts + s);
    const int e = __ldg(seg_starts + s + 1);
    const int i = __ldg(lora_idx + s);
    out.begin = b;
    out.end = e;
    out.a = nullptr;
    out.b = nullptr;
    if (b < 0 || b > e || e > T) return LORA_SGMV_DEV_BAD_SEGMENT;
    if (i < 0 || i >= num_adapters) return LORA_SGMV_DEV_BAD_ADAPTER;
    uint32_t bad = 0;
    if (A_ptrs) {
        out.a = A_ptrs[i];
        if (out.a == nullptr || (reinterpret_cast<uintptr_t>(out.a) & 15u)) bad |= LORA_SGMV_DEV_BAD_POINTER;
    }
    if (B_ptrs) {
        out.b = B_ptrs[i];
        if (out.b == nullptr || (reinterpret_cast<uintptr_t>(out.b) & 15u)) bad |= LORA_SGMV_DEV_BAD_POINTER;
    }
    return bad;
}

__device__ __forceinline__ void report(uint32_t* dev_status, uint32_t bits) {
    if (dev_status && bits) atomicOr(dev_status, bits);
}

// ---- programmatic dependent launch (griddepcontrol, sm_90+) ------------------
// launch_dependents lets the next kernel on the stream (launched with the
// programmatic-serialization attribute) start its prologue; wait blocks until
// every prerequisite grid has completed and its memory is visible.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---- 16-byte vectors of eight 16-bit values --------------------------------------

// Streaming read-only load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_vec(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void st_vec(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

template <typename T>
struct Storage;

template <>
struct Storage<__half> {
    static __device__ __forceinline__ float2 to2(uint32_t w) {
        __half2 h = *reinterpret_cast<__half2*>(&w);
        return __half22float2(h);
    }
    static __device__ __forceinline__ uint32_t from2(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ float to1(__half v) { return __half2float(v); }
    // x rounded to the nearest fp16 value, returned as fp32
    static __device__ __forceinline__ float round(float x) { return __half2float(__float2half_rn(x)); }
    static __device__ __forceinline__ __half from1(float x) { return __float2half_rn(x); }
};

template <>
struct Storage<__nv_bfloat16> {
    static __device__ __forceinline__ float2 to2(uint32_t w) {
        // bf16 is the upper half of an fp32: widening is a shift, exact
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ uint32_t from2(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ float to1(__nv_bfloat16 v) { return __bfloat162float(v); }
    // x rounded to the nearest bf16 value, returned as fp32
    static __device__ __forceinline__ float round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
    static __device__ __forceinline__ __nv_bfloat16 from1(float x) { return __float2bfloat16_rn(x); }
};

template <typename T>
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    float2 p;
    p = Storage<T>::to2(v.x); f[0] = p.x; f[1] = p.y;
    p = Storage<T>::to2(v.y); f[2] = p.x; f[3] = p.y;
    p = Storage<T>::to2(v.z); f[4] = p.x; f[5] = p.y;
    p = Storage<T>::to2(v.w); f[6] = p.x; f[7] = p.y;
}

// Two fp32 lanes in one 64-bit register pair, for the paired fp32 arithmetic of sm_100
// (fma.rn.f32x2: each lane is one fused multiply-add rounded to nearest, the result fmaf gives).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f32x2_split(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
// a * b + c per lane
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

template <typename T>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 v;
    v.x = Storage<T>::from2(f[0], f[1]);
    v.y = Storage<T>::from2(f[2], f[3]);
    v.z = Storage<T>::from2(f[4], f[5]);
    v.w = Storage<T>::from2(f[6], f[7]);
    return v;
}

}  // namespace sgmv

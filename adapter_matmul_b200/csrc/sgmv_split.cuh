// sgmv_split.cuh -- the split SGMV path: a split-K shrink kernel (H1 -> r) and a
// streaming expand kernel (r -> H2) with the add onto Y fused in its epilogue.
//
// Shapes follow the LoRA paragraph of page “Punica：多 LoRA 模型统一服务框架” (the Punica README): A_i is [H1, r], B_i is
// [r, H2], rows are tokens; the batch form (multi-LoRA paragraph) maps each
// segment of rows to its own adapter.
//
// Shrink. One thread-block cluster of C CTAs per token chunk (8 tokens of one segment;
// the clusters walk a flat list of the chunks, or segment and chunk slots when there are
// too many segments for the list's prefix to fit in shared memory).
// CTA c of the cluster owns rows [c*KS, (c+1)*KS) of A_i; that slice of A_i is one
// contiguous run of KS*r*2 bytes. One thread streams it through a ring of shared-memory
// slots with 1-D bulk copies (16 KB each), and with each slot a tensor-map copy of the
// chunk's X columns for the same rows, so the copies run ahead of the arithmetic. All
// threads accumulate fp32 partial sums from the ring (paired FMAs, two columns per
// instruction), reduce them with warp shuffles and then across warps in shared memory. The
// C partial V tiles are summed in a fixed order through distributed shared memory (DSMEM),
// and each CTA stores its share of the reduced V with plain stores: no atomics, no
// zero-fill of V, bit-reproducible. 128 threads per CTA and three CTAs per SM.
//
// Expand. One CTA per (column block of 8*NT columns, segment, token-chunk
// slot). Each thread owns 8 consecutive columns: it streams B_i[j, cols] for
// j = 0..r-1 with 128-bit loads (each B_i byte is read once per token chunk),
// multiplies by V rows held in shared memory, and performs the read-add-round-
// write of Y in place. With programmatic dependent launch the expand grid is
// scheduled while the shrink grid drains; everything it does before
// griddepcontrol.wait (segment metadata, the first block of B_i) does not
// depend on V.
#pragma once

#include <cooperative_groups.h>

#include "sgmv_common.cuh"
#include "sgmv_grouped_tc.cuh"  // PTX wrappers (mbarriers, bulk and tensor-map copies)

namespace sgmv {

namespace cg = cooperative_groups;

struct ShrinkParams {
    float* V;
    const void* X;
    const void* const* A_ptrs;
    const void* const* B_check;  // non-null in apply: a segment whose B_i is bad is skipped here too
    const int32_t* seg_starts;
    const int32_t* lora_idx;
    uint32_t* dev_status;
    int n_segments;
    int num_adapters;
    int T;
    int H1;
    int ks;    // rows of A_i per CTA, multiple of 8
    int flat;  // 1: grid over the flat (segment, chunk) list (shared memory holds its prefix)
};

struct ExpandParams {
    void* Y;
    const float* V;
    const void* const* B_ptrs;
    const void* const* A_check;  // non-null in apply: a segment whose A_i is bad is skipped here too
    const int32_t* seg_starts;
    const int32_t* lora_idx;
    uint32_t* dev_status;
    int n_segments;
    int num_adapters;
    int T;
    int H2;
    float scale;
};

constexpr int kShrinkThreads = 128;
constexpr int kShrinkTokens = 8;     // tokens per chunk
constexpr int kShrinkSlotA = 16384;  // bytes of A_i per ring slot (one bulk copy)
constexpr int kShrinkSlots = 3;      // ring depth
constexpr int kExpandThreads = 128;
constexpr int kExpandTokens = 8;

constexpr int kShrinkFlatMaxSegments = 8192;  // flat grid: the chunk prefix fits in shared memory

// A ring slot: SR rows of A_i (16 KB), then the chunk's X columns for those rows, [8][SR]
// (16-bit), loaded by NXB tensor-map boxes of {XB columns, 8 rows}.
__host__ __device__ constexpr int shrink_slot_rows(int R) { return kShrinkSlotA / (R * 2); }
__host__ __device__ constexpr int shrink_x_box(int R) { return shrink_slot_rows(R) < 256 ? shrink_slot_rows(R) : 256; }
__host__ __device__ constexpr int shrink_slot_bytes(int R) {
    return kShrinkSlotA + kShrinkTokens * shrink_slot_rows(R) * 2;
}
__host__ __device__ constexpr size_t shrink_ring_bytes(int R) {
    // the ring, which after a chunk's last slot holds the per-warp partials [NW][TC*R]
    return size_t(kShrinkSlots) * shrink_slot_bytes(R) > size_t(kShrinkThreads / 32) * kShrinkTokens * R * 4
               ? size_t(kShrinkSlots) * shrink_slot_bytes(R)
               : size_t(kShrinkThreads / 32) * kShrinkTokens * R * 4;
}

__host__ __device__ constexpr size_t shrink_smem_bytes(int R, int flat_segments = 0) {
    // ring + CTA partial [TC*R] (+ flat grid: chunk prefix [n_segments + 1] and per-warp totals [NW])
    return shrink_ring_bytes(R) + size_t(kShrinkTokens) * R * 4 +
           (flat_segments > 0 ? size_t(flat_segments + 1 + kShrinkThreads / 32) * 4 : 0);
}

// One token chunk [t0, t0 + nt) of a segment, this CTA's rows [k0, k0 + nk) of its A_i:
// stream the rows, and the chunk's X columns beside them, through the ring, accumulate TCN
// token rows, reduce over the CTA, sum the C partial tiles across the cluster in rank order
// and store this CTA's share of V. X rows past nt (the next segment's tokens, or zeros past T)
// only reach sums that are never stored. Every CTA of the cluster calls it for the same
// chunk; `it` counts the ring slots this CTA has used.
template <typename T, int R, int TCN>
__device__ __forceinline__ void shrink_chunk(const CUtensorMap* xmap, const ShrinkParams& p, cg::cluster_group& cluster,
                                             const T* __restrict__ A, int t0, int nt, int k0, int nk,
                                             unsigned char* ring, uint64_t* full, uint32_t& it, bool& dead,
                                             float* part) {
    constexpr int NT = kShrinkThreads;
    constexpr int G = R / 8;                     // 16-byte vectors per row of A_i
    constexpr int RL = NT / G;                   // row lanes
    constexpr int NW = NT / 32;
    constexpr int SR = shrink_slot_rows(R);      // rows of A_i per slot
    constexpr int RPT = SR / RL;                 // rows per thread per slot
    constexpr int XB = shrink_x_box(R);
    constexpr int SLOT = shrink_slot_bytes(R);
    static_assert(SR % RL == 0 && SR % XB == 0, "a slot must hold whole rows for every row lane");
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int cgi = tid % G;
    const int rl = tid / G;
    const int c = static_cast<int>(cluster.block_rank());
    const int C = static_cast<int>(cluster.num_blocks());
    const int nslot = (nk + SR - 1) / SR;
    const unsigned char* Ab = reinterpret_cast<const unsigned char*>(A + size_t(k0) * R);
    auto issue = [&](int i) {  // slot i of this chunk
        const uint32_t a_bytes = static_cast<uint32_t>(min(SR, nk - i * SR)) * R * 2;
        const uint32_t b = (it + i) % kShrinkSlots;
        unsigned char* dst = ring + size_t(b) * SLOT;
        mbar_arrive_expect_tx(&full[b], a_bytes + kShrinkTokens * SR * 2);
        bulk_g2s(dst, Ab + size_t(i) * kShrinkSlotA, a_bytes, &full[b]);
#pragma unroll
        for (int xb = 0; xb < SR / XB; ++xb)
            tma_load_2d(dst + kShrinkSlotA + xb * kShrinkTokens * XB * 2, xmap, k0 + i * SR + xb * XB, t0, &full[b]);
    };
    if (tid == 0) {
        // the ring last held the previous chunk's partials, written by generic stores
        fence_proxy_async();
        for (int i = 0; i < min(nslot, kShrinkSlots); ++i) issue(i);
    }

    // column pairs (2q, 2q + 1) of the 8 sums per token row, updated by paired FMAs
    uint64_t acc2[TCN][4];
#pragma unroll
    for (int t = 0; t < TCN; ++t)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc2[t][q] = 0;

#pragma unroll 1
    for (int i = 0; i < nslot; ++i) {
        const uint32_t g = it + i;
        mbar_wait<false>(&full[g % kShrinkSlots], (g / kShrinkSlots) & 1u, p.dev_status, dead);
        const unsigned char* sl = ring + size_t(g % kShrinkSlots) * SLOT;
        const T* xs = reinterpret_cast<const T*>(sl + kShrinkSlotA);
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int row = rl + m * RL;
            if (i * SR + row < nk) {
                float a[8];
                unpack8<T>(ld_vec(sl + size_t(row) * (R * 2) + cgi * 16), a);
                uint64_t a2[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) a2[q] = f32x2(a[2 * q], a[2 * q + 1]);
                // X box xb holds columns [xb*XB, (xb+1)*XB) of the slot as [8][XB]
                const T* xr = xs + (row / XB) * (kShrinkTokens * XB) + (row % XB);
#pragma unroll
                for (int t = 0; t < TCN; ++t) {
                    const float x = Storage<T>::to1(xr[t * XB]);
                    const uint64_t x2 = f32x2(x, x);
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc2[t][q] = ffma2(x2, a2[q], acc2[t][q]);
                }
            }
        }
        __syncthreads();  // every thread is done with the slot before it is refilled
        if (tid == 0 && i + kShrinkSlots < nslot) issue(i + kShrinkSlots);
    }
    it += static_cast<uint32_t>(nslot);
    float acc[TCN][8];
#pragma unroll
    for (int t = 0; t < TCN; ++t)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 v = f32x2_split(acc2[t][q]);
            acc[t][2 * q] = v.x;
            acc[t][2 * q + 1] = v.y;
        }
    float* red = reinterpret_cast<float*>(ring);  // no copy is in flight after the last slot
    // reduce over the row lanes of this warp (lanes sharing cgi)
#pragma unroll
    for (int off = G; off < 32; off <<= 1)
#pragma unroll
        for (int t = 0; t < TCN; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[t][i] += __shfl_xor_sync(0xffffffffu, acc[t][i], off);
    if (lane < G) {
#pragma unroll
        for (int t = 0; t < TCN; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) red[(warp * TCN + t) * R + cgi * 8 + i] = acc[t][i];
    }
    __syncthreads();
    for (int e = tid; e < TCN * R; e += NT) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) sum += red[w * TCN * R + e];
        part[e] = sum;
    }
    // sum the C partial tiles across the cluster in rank order
    cluster.sync();
    const int per = (TCN * R + C - 1) / C;
    const int e0 = c * per;
    const int e1 = min(e0 + per, TCN * R);
    for (int e = e0 + tid; e < e1; e += NT) {
        float sum = 0.f;
        for (int qr = 0; qr < C; ++qr) sum += cluster.map_shared_rank(part, qr)[e];
        const int t = e / R;
        const int j = e - t * R;
        if (t < nt) p.V[size_t(t0 + t) * R + j] = sum;
    }
    cluster.sync();  // partial tiles and the X slice may be overwritten only after every read
}

// Two grids. p.flat == 0: x = C (one cluster along x), y = segment slots, z = token-chunk
// slots. p.flat == 1: x = C, y = slots over the flat list of (segment, chunk) units, z = 1;
// every CTA builds the list's prefix (chunks before each segment) in shared memory, so the
// grid holds no CTA without a chunk.
template <typename T, int R>
__global__ void __launch_bounds__(kShrinkThreads, 3)
    sgmv_shrink_cluster_kernel(const __grid_constant__ CUtensorMap xmap, const ShrinkParams p) {
    constexpr int NT = kShrinkThreads;
    constexpr int TC = kShrinkTokens;
    constexpr int G = R / 8;
    static_assert(R % 8 == 0 && G <= 32 && (32 % G) == 0, "rank must be 8..256, power of two");

    cg::cluster_group cluster = cg::this_cluster();
    const int c = static_cast<int>(cluster.block_rank());
    const int tid = threadIdx.x;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* ring = smem;
    float* part = reinterpret_cast<float*>(smem + shrink_ring_bytes(R));
    __shared__ __align__(8) uint64_t full[kShrinkSlots];
    if (tid == 0) {
        for (int i = 0; i < kShrinkSlots; ++i) mbar_init(&full[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    uint32_t it = 0;    // ring slots used
    bool dead = false;  // a wait on the ring gave up (reported; the results are invalid)

    // The expand kernel may be scheduled as soon as every shrink CTA is running.
    pdl_launch_dependents();

    const int k0 = c * p.ks;
    const int nk = max(0, min(k0 + p.ks, p.H1) - k0);
    auto run_chunk = [&](const T* A, int t0, int nt) {
        if (nt == 1)
            shrink_chunk<T, R, 1>(&xmap, p, cluster, A, t0, nt, k0, nk, ring, full, it, dead, part);
        else
            shrink_chunk<T, R, TC>(&xmap, p, cluster, A, t0, nt, k0, nk, ring, full, it, dead, part);
    };

    if (p.flat) {
        int* pref = reinterpret_cast<int*>(part + TC * R);  // n_segments + 1 entries
        int* wtot = pref + p.n_segments + 1;                // NW entries
        const int n = p.n_segments;
        const int per_thr = (n + NT - 1) / NT;
        const int s0 = min(n, tid * per_thr), s1 = min(n, s0 + per_thr);
        int local = 0;
        // chunk counts from the segment bounds alone (one round trip: the adapter id is read
        // beside them and its table entries are only prefetched), parked in the prefix slots; one
        // CTA reports each segment with invalid bounds while the list is built, and a segment
        // whose adapter or pointers fail is reported and skipped where its first chunk runs
        const bool reporter = blockIdx.y == 0 && c == 0;
        for (int s = s0; s < s1; ++s) {
            const int b = __ldg(p.seg_starts + s), e = __ldg(p.seg_starts + s + 1);
            const int i = __ldg(p.lora_idx + s);
            const bool ok = b >= 0 && b <= e && e <= p.T;
            if (reporter && !ok) report(p.dev_status, LORA_SGMV_DEV_BAD_SEGMENT);
            if (ok && i >= 0 && i < p.num_adapters) {
                asm volatile("prefetch.global.L1 [%0];" ::"l"(p.A_ptrs + i));
                if (p.B_check) asm volatile("prefetch.global.L1 [%0];" ::"l"(p.B_check + i));
            }
            const int k = ok ? (e - b + TC - 1) / TC : 0;
            pref[s + 1] = k;
            local += k;
        }
        const int lane = tid & 31, warp = tid >> 5;
        int v = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += y;
        }
        if (lane == 31) wtot[warp] = v;
        __syncthreads();
        int run = v - local;
        for (int w = 0; w < warp; ++w) run += wtot[w];
        if (tid == 0) pref[0] = 0;
        for (int s = s0; s < s1; ++s) {
            run += pref[s + 1];
            pref[s + 1] = run;
        }
        __syncthreads();
        const int total = pref[n];
        for (int u = blockIdx.y; u < total; u += gridDim.y) {
            int lo = 0, hi = n;  // largest s with pref[s] <= u
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (pref[mid] <= u)
                    lo = mid;
                else
                    hi = mid;
            }
            Segment seg;
            const uint32_t bad =
                load_segment(p.seg_starts, p.lora_idx, p.A_ptrs, p.B_check, lo, p.T, p.num_adapters, seg);
            if (bad) {  // uniform over the cluster: every CTA read the same words
                if (c == 0 && tid == 0 && u == pref[lo]) report(p.dev_status, bad);
                continue;
            }
            const int t0 = seg.begin + (u - pref[lo]) * TC;
            run_chunk(static_cast<const T*>(seg.a), t0, min(TC, seg.end - t0));
        }
        return;
    }

    for (int s = blockIdx.y; s < p.n_segments; s += gridDim.y) {
        Segment seg;
        const uint32_t bad = load_segment(p.seg_starts, p.lora_idx, p.A_ptrs, p.B_check, s, p.T,
                                          p.num_adapters, seg);
        if (bad) {  // uniform over the cluster: every CTA read the same words
            if (c == 0 && blockIdx.z == 0 && tid == 0) report(p.dev_status, bad);
            continue;
        }
        const int nchunks = (seg.end - seg.begin + TC - 1) / TC;
        for (int q = blockIdx.z; q < nchunks; q += gridDim.z) {
            const int t0 = seg.begin + q * TC;
            run_chunk(static_cast<const T*>(seg.a), t0, min(TC, seg.end - t0));
        }
    }
}

// grid: x = column blocks of 8*NT columns, y = segment slots, z = token-chunk slots.
template <typename T, int R>
__global__ void __launch_bounds__(kExpandThreads) sgmv_expand_kernel(const ExpandParams p) {
    constexpr int NT = kExpandThreads;
    constexpr int TC = kExpandTokens;
    constexpr int JB = R >= 128 ? 8 : (R < 16 ? R : 16);  // rows of B_i loaded per batch
    __shared__ float vs[TC][R];

    const int tid = threadIdx.x;
    const int col = (blockIdx.x * NT + tid) * 8;
    const bool active = col < p.H2;
    T* __restrict__ Y = static_cast<T*>(p.Y);
    bool waited = false;

    for (int s = blockIdx.y; s < p.n_segments; s += gridDim.y) {
        Segment seg;
        const uint32_t bad = load_segment(p.seg_starts, p.lora_idx, p.A_check, p.B_ptrs, s, p.T,
                                          p.num_adapters, seg);
        if (bad) {
            if (blockIdx.x == 0 && blockIdx.z == 0 && tid == 0) report(p.dev_status, bad);
            continue;
        }
        const T* __restrict__ B = static_cast<const T*>(seg.b);
        const int L = seg.end - seg.begin;
        const int nchunks = (L + TC - 1) / TC;
        for (int q = blockIdx.z; q < nchunks; q += gridDim.z) {
            const int t0 = seg.begin + q * TC;
            const int nt = min(TC, seg.end - t0);
            // first batch of B_i rows does not depend on V: issue it before the wait
            uint4 bv[JB];
#pragma unroll
            for (int u = 0; u < JB; ++u)
                bv[u] = active ? ld_stream(B + size_t(u) * p.H2 + col) : make_uint4(0, 0, 0, 0);
            if (!waited) {
                pdl_wait();
                waited = true;
            }
            for (int e = tid; e < TC * R; e += NT) {
                const int t = e / R;
                const int j = e - t * R;
                vs[t][j] = t < nt ? p.V[size_t(t0 + t) * R + j] : 0.f;
            }
            __syncthreads();

            float acc[TC][8];
#pragma unroll
            for (int t = 0; t < TC; ++t)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[t][i] = 0.f;
#pragma unroll 1
            for (int jb = 0; jb < R; jb += JB) {
                if (jb > 0) {
#pragma unroll
                    for (int u = 0; u < JB; ++u)
                        bv[u] = active ? ld_stream(B + size_t(jb + u) * p.H2 + col) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < JB; ++u) {
                    float b[8];
                    unpack8<T>(bv[u], b);
#pragma unroll
                    for (int t = 0; t < TC; ++t) {
                        if (t < nt) {
                            const float v = vs[t][jb + u];
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[t][i] = fmaf(v, b[i], acc[t][i]);
                        }
                    }
                }
            }
            if (active) {
#pragma unroll
                for (int t = 0; t < TC; ++t) {
                    if (t < nt) {
                        T* yp = Y + size_t(t0 + t) * p.H2 + col;
                        float y[8];
                        unpack8<T>(ld_vec(yp), y);
#pragma unroll
                        for (int i = 0; i < 8; ++i) y[i] = __fadd_rn(y[i], __fmul_rn(p.scale, acc[t][i]));
                        st_vec(yp, pack8<T>(y));
                    }
                }
            }
            __syncthreads();  // vs is rewritten by the next chunk
        }
    }
    if (!waited) pdl_wait();  // keep the dependency even when this CTA had no work
}

}  // namespace sgmv

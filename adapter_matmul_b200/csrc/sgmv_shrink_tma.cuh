// sgmv_shrink_tma.cuh -- split-K shrink V = X@A_i (H1 -> r, fp32) with every operand staged
// through a ring of shared-memory stages by the tensor memory accelerator.
//
// Maths (page "Punica：多 LoRA 模型统一服务框架", the Punica README, its LoRA and multi-LoRA
// paragraphs): for each segment s with adapter i and each row t of it, V[t, :] = X[t, :] @ A_i,
// the first half of x@A@B, with A_i [H1, r] row-major.
//
// Units. A unit is one chunk of up to 8 tokens of one segment; every CTA builds the exact list
// of units (a prefix over the segments' chunk counts, in shared memory) and the clusters walk it
// round-robin, persistent (as many clusters as are resident at once).
//
// Split over a cluster of C CTAs: CTA c owns rows [c*ks, (c+1)*ks) of A_i, which are one
// contiguous run of ks*r*2 bytes. Warp 0 streams the CTA's run through a ring of stages, each
// one bulk copy of KT rows of A_i (32 KB: the copy engine of an SM works through its copies
// one after another, with a fixed cost of a few hundred ns each from HBM, so a copy must be
// large to keep the SM's share of HBM bandwidth), and once per unit the chunk's X columns as
// one 3-D TMA box (8 rows of the CTA's ks columns, from a view of X whose third dimension steps
// 64 columns) into one of two X buffers. The producer runs ahead into the next unit while the
// consumers finish the current one, so the stream of A_i does not stop at unit boundaries.
//
// Compute: warps 1..8 multiply each stage in fp32 (one A_i row of 8 columns and the chunk's X
// values per step, specialised for 1, 2, 4 or 8 tokens), reduce over lanes by shuffles and
// over warps in shared memory. Reduction over the cluster: CTA q owns a share of the chunk's
// V tile; every CTA pushes that share of its partial tile into q's receive slot with
// st.async (completion counted on q's mbarrier); q sums the C slots in rank order and stores
// its share of V with plain stores (no atomics, no zero fill; bit-reproducible). Receive
// buffers alternate between two sets, so a sender waits for a set to be released only two
// units later.
//
// Every wait is bounded in time and reports LORA_SGMV_DEV_TIMEOUT. Requires H1 % 64 == 0 (the
// X view); the caller falls back to the per-thread-load shrink otherwise.
#pragma once

#include "sgmv_decode_tc.cuh"
#include "sgmv_split.cuh"

namespace sgmv {

constexpr int kSTThreads = 288;  // producer warp + 8 consumer warps
constexpr int kSTConsumers = 256;
constexpr int kSTWarps = 8;
constexpr int kSTTokens = 8;
constexpr int kSTMaxSegments = 8192;  // unit prefix held in shared memory
constexpr int kSTMaxKs = 2048;        // A_i rows per CTA (X buffer of 8 x 2048 values)

template <int R>
struct ShrinkTmaGeom {
    static constexpr int KT = 32768 / (2 * R);  // A_i rows per stage: 32 KB of A_i
    static constexpr int A_BYTES = KT * R * 2;
    static constexpr int STAGES = 4;
    static constexpr int G = R / 8;             // 16-byte column groups of an A_i row
    static constexpr int RL = kSTConsumers / G;  // row lanes
    static constexpr int TILE = kSTTokens * R;   // floats of one V tile
    static constexpr size_t RING = size_t(STAGES) * A_BYTES;
    static constexpr size_t RED = size_t(kSTWarps) * TILE * 4;
    static constexpr size_t RECV = 2 * size_t(TILE) * 4 + 2 * kFusedMaxCluster * 16;  // two sets of C shares
    // + two X buffers of 8 x ks values, then the unit prefix
    static constexpr size_t BASE = RING + RED + RECV;
    static __host__ __device__ constexpr size_t x_bytes(int ks) { return size_t(kSTTokens) * ks * 2; }
    static_assert(KT % 64 == 0, "a stage holds whole 64-row blocks of A_i");
};

struct ShrinkTmaParams {
    float* V;
    const void* const* A_ptrs;
    const void* const* B_check;
    const int32_t* seg_starts;
    const int32_t* lora_idx;
    uint32_t* dev_status;
    int n_segments;
    int num_adapters;
    int T;
    int H1;
    int ks;     // rows of A_i per CTA (multiple of 64)
    int share;  // floats of the V tile each CTA owns (multiple of 4)
};

__device__ __forceinline__ int st_segment_chunks(const ShrinkTmaParams& p, int s) {
    Segment seg;
    if (load_segment(p.seg_starts, p.lora_idx, p.A_ptrs, p.B_check, s, p.T, p.num_adapters, seg)) return 0;
    return (seg.end - seg.begin + kSTTokens - 1) / kSTTokens;
}

// unit u -> (segment, first token, tokens, A_i); false past the end
__device__ __forceinline__ bool st_unit(const ShrinkTmaParams& p, const int* pref, int u, int& t0, int& nt,
                                        const void*& a) {
    const int n = p.n_segments;
    if (u >= pref[n]) return false;
    int lo = 0, hi = n;  // largest s with pref[s] <= u
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pref[mid] <= u)
            lo = mid;
        else
            hi = mid;
    }
    Segment seg;
    load_segment(p.seg_starts, p.lora_idx, p.A_ptrs, p.B_check, lo, p.T, p.num_adapters, seg);
    t0 = seg.begin + (u - pref[lo]) * kSTTokens;
    nt = min(kSTTokens, seg.end - t0);
    a = seg.a;
    return true;
}

__device__ __forceinline__ void st_consumer_sync() {  // named barrier 1 over the consumer warps
    asm volatile("bar.sync 1, %0;" ::"n"(kSTConsumers) : "memory");
}

template <typename T, int R, int NTOK>
__device__ __forceinline__ void st_consume(const unsigned char* ring, uint64_t* full, uint64_t* empty, uint32_t& it,
                                           int nA, int nk, int nt, const T* xs, float* red, uint32_t* status,
                                           bool& dead) {
    using G = ShrinkTmaGeom<R>;
    const int ct = threadIdx.x - 32;
    const int lane = ct & 31, cw = ct >> 5;
    const int cg = ct % G::G, rl = ct / G::G;
    float acc[NTOK][8];
#pragma unroll
    for (int t = 0; t < NTOK; ++t)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[t][i] = 0.f;
    for (int ta = 0; ta < nA; ++ta, ++it) {
        const uint32_t st = it % G::STAGES;
        mbar_wait<false>(&full[st], (it / G::STAGES) & 1u, status, dead);
        const unsigned char* sa = ring + size_t(st) * G::A_BYTES;
        const int kt = min(G::KT, nk - ta * G::KT);
        for (int k = rl; k < kt; k += G::RL) {
            float a[8];
            unpack8<T>(*reinterpret_cast<const uint4*>(sa + (size_t(k) * R + cg * 8) * 2), a);
            const int kx = ta * G::KT + k;  // column of the CTA's slice of X
            const T* xk = xs + (kx >> 6) * (kSTTokens * 64) + (kx & 63);
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                if (t < nt) {
                    const float x = Storage<T>::to1(xk[t * 64]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[t][i] = fmaf(x, a[i], acc[t][i]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&empty[st]);
    }
#pragma unroll
    for (int off = G::G; off < 32; off <<= 1)
#pragma unroll
        for (int t = 0; t < NTOK; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[t][i] += __shfl_xor_sync(0xffffffffu, acc[t][i], off);
    if (lane < G::G) {
#pragma unroll
        for (int t = 0; t < kSTTokens; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) red[(cw * kSTTokens + t) * R + cg * 8 + i] = t < NTOK ? acc[t < NTOK ? t : 0][i] : 0.f;
    }
}

// grid.x = C * clusters, cluster (C,1,1). Warp 0 produces, warps 1..8 consume.
template <typename T, int R>
__global__ void __launch_bounds__(kSTThreads, 1)
    sgmv_shrink_tma_kernel(const __grid_constant__ CUtensorMap tmX, const ShrinkTmaParams p) {
    using G = ShrinkTmaGeom<R>;
    constexpr int S = G::STAGES;
    extern __shared__ __align__(128) unsigned char stsm[];
    unsigned char* ring = stsm;
    float* red = reinterpret_cast<float*>(stsm + G::RING);
    float* recv = reinterpret_cast<float*>(stsm + G::RING + G::RED);  // [2][C][share]
    const size_t xb = G::x_bytes(p.ks);
    unsigned char* xbuf = stsm + G::BASE;  // two X buffers [ks/64][8 rows][64 columns]
    int* pref = reinterpret_cast<int*>(stsm + G::BASE + 2 * xb);
    __shared__ __align__(8) uint64_t full[S], empty[S], vready[2], vfree[2], xfull[2], xempty[2];

    const int C = static_cast<int>(cluster_size());
    const int c = static_cast<int>(cluster_rank());
    const int cluster_id = blockIdx.x / C;
    const int n_clusters = gridDim.x / C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = c * p.ks;
    const int nk = max(0, min(k0 + p.ks, p.H1) - k0);
    const int nA = (nk + G::KT - 1) / G::KT;

    pdl_launch_dependents();  // the expand kernel may be scheduled as soon as every CTA runs
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kSTWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&vready[i], 1);  // own expect_tx; the C shares arrive as transaction bytes
            mbar_init(&vfree[i], C);   // one arrival per owner
            mbar_init(&xfull[i], 1);   // producer's expect_tx; the X box completes the bytes
            mbar_init(&xempty[i], kSTWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // unit prefix: pref[s] = chunks of segments before s
    {
        const int n = p.n_segments;
        __shared__ int wtot[kSTThreads / 32];
        const int per_thr = (n + kSTThreads - 1) / kSTThreads;
        const int s0 = min(n, int(threadIdx.x) * per_thr), s1 = min(n, s0 + per_thr);
        int local = 0;
        for (int s = s0; s < s1; ++s) {
            const int k = st_segment_chunks(p, s);
            pref[s + 1] = k;
            local += k;
        }
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
        if (threadIdx.x == 0) pref[0] = 0;
        for (int s = s0; s < s1; ++s) {
            run += pref[s + 1];
            pref[s + 1] = run;
        }
        __syncthreads();
    }
    if (C > 1) cluster_arrive();
    bool dead = false;
    const int share = p.share;
    const uint32_t share_bytes = uint32_t(share) * 4;

    if (warp == 0) {
        // ---------------------------------- producer ----------------------------------
        uint32_t it = 0, u_local = 0;
        int t0, nt;
        const void* av;
        for (int u = cluster_id; st_unit(p, pref, u, t0, nt, av); u += n_clusters, ++u_local) {
            const T* A = static_cast<const T*>(av);
            // the unit's X columns: one box into X buffer u_local & 1, once the consumers are done
            // with the unit two back
            const int b = u_local & 1;
            if (u_local >= 2) mbar_wait<false>(&xempty[b], ((u_local >> 1) - 1) & 1u, p.dev_status, dead);
            if (lane == 0 && nA > 0) {
                mbar_arrive_expect_tx(&xfull[b], uint32_t(xb));
                tma_load_3d(xbuf + b * xb, &tmX, 0, t0, k0 / 64, &xfull[b]);
            } else if (lane == 0) {
                mbar_arrive_local(&xfull[b]);
            }
            __syncwarp();
            for (int ta = 0; ta < nA; ++ta, ++it) {
                const uint32_t st = it % S;
                if (it >= S) mbar_wait<false>(&empty[st], ((it / S) - 1) & 1u, p.dev_status, dead);
                unsigned char* sa = ring + size_t(st) * G::A_BYTES;
                const int k = k0 + ta * G::KT;
                const int kt = min(G::KT, nk - ta * G::KT);
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[st], uint32_t(kt) * R * 2);
                    bulk_g2s(sa, A + size_t(k) * R, uint32_t(kt) * R * 2, &full[st]);
                }
                __syncwarp();
            }
        }
        if (lane == 0) {
            for (uint32_t i = it > uint32_t(S) ? it - S : 0u; i < it; ++i) drain_wait(&full[i % S], (i / S) & 1u);
            for (uint32_t v = u_local >= 2 ? u_local - 2 : 0u; v < u_local; ++v) drain_wait(&xfull[v & 1], (v >> 1) & 1u);
        }
        __syncwarp();
        if (C > 1) cluster_wait();
    } else {
        // ---------------------------------- consumers ----------------------------------
        if (C > 1) cluster_wait();
        const int ct = threadIdx.x - 32;
        uint32_t it = 0, u_local = 0;
        int t0, nt;
        const void* av;
        for (int u = cluster_id; st_unit(p, pref, u, t0, nt, av); u += n_clusters, ++u_local) {
            const int buf = u_local & 1;
            mbar_wait<false>(&xfull[buf], (u_local >> 1) & 1u, p.dev_status, dead);
            const T* xs = reinterpret_cast<const T*>(xbuf + buf * xb);
            if (nt == 1)
                st_consume<T, R, 1>(ring, full, empty, it, nA, nk, nt, xs, red, p.dev_status, dead);
            else if (nt <= 2)
                st_consume<T, R, 2>(ring, full, empty, it, nA, nk, nt, xs, red, p.dev_status, dead);
            else if (nt <= 4)
                st_consume<T, R, 4>(ring, full, empty, it, nA, nk, nt, xs, red, p.dev_status, dead);
            else
                st_consume<T, R, 8>(ring, full, empty, it, nA, nk, nt, xs, red, p.dev_status, dead);
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive_relaxed(&xempty[buf]);  // this unit's X is no longer read
            st_consumer_sync();
            // this CTA's partial tile (the warps' sums), then its C shares to their owners
            if (ct == 0) mbar_arrive_expect_tx(&vready[buf], share_bytes * C);
            if (u_local >= 2) mbar_wait<true>(&vfree[buf], ((u_local >> 1) - 1) & 1u, p.dev_status, dead);
            for (int e4 = ct; e4 < (share * C) / 4; e4 += kSTConsumers) {
                const int e = e4 * 4;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (e < G::TILE) {
#pragma unroll
                    for (int w = 0; w < kSTWarps; ++w) {
                        const float4 q = *reinterpret_cast<const float4*>(red + w * G::TILE + e);
                        v.x += q.x;
                        v.y += q.y;
                        v.z += q.z;
                        v.w += q.w;
                    }
                }
                const int q = e / share;  // owner
                st_async_v4(recv + (size_t(buf) * C + c) * share + (e - q * share), v, &vready[buf], uint32_t(q));
            }
            mbar_wait<true>(&vready[buf], (u_local >> 1) & 1u, p.dev_status, dead);
            for (int e = ct; e < share; e += kSTConsumers) {
                const int g = c * share + e;  // element of the tile
                const int t = g / R, j = g - t * R;
                if (t < nt) {
                    float sum = 0.f;
                    for (int q = 0; q < C; ++q) sum += recv[(size_t(buf) * C + q) * share + e];
                    p.V[size_t(t0 + t) * R + j] = sum;
                }
            }
            st_consumer_sync();  // every read of recv[buf] and red is done
            if (ct < C) mbar_arrive_remote(&vfree[buf], static_cast<uint32_t>(ct));
        }
        // every owner has consumed this CTA's last shares before its shared memory goes away
        for (uint32_t v = u_local >= 2 ? u_local - 2 : 0u; v < u_local; ++v)
            mbar_wait<true>(&vfree[v & 1], (v >> 1) & 1u, p.dev_status, dead);
        if (ct == 0 && c == 0)  // report each rejected segment once
            for (int s = cluster_id; s < p.n_segments; s += n_clusters) {
                Segment seg;
                report(p.dev_status, load_segment(p.seg_starts, p.lora_idx, p.A_ptrs, p.B_check, s, p.T,
                                                  p.num_adapters, seg));
            }
    }
}

// X view {64, T, H1/64} (element (k, t, b) at X + t*H1 + 64*b + k), box {64, 8, ks/64}, no swizzle.
inline bool make_shrink_x_map(CUtensorMap* m, const void* X, int T, int H1, int ks, lora_sgmv_dtype dt) {
    const uint64_t d[3] = {64, uint64_t(T), uint64_t(H1 / 64)};
    const uint64_t s[2] = {uint64_t(H1) * 2, 128};
    const uint32_t b[3] = {64, uint32_t(kSTTokens), uint32_t(ks / 64)};
    return encode_map(m, X, dt, 3, d, s, b, CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace sgmv

// sgmv_fused.cuh -- one-kernel SGMV for short segments (decode): shrink, V reduction
// and expand with the fused add, for one or several projections in one launch.
//
// Maths (Punica README, LoRA and multi-LoRA paragraphs): for each segment s
// with adapter i and each row t of it, Y[t,:] += scale * (X[t,:] @ A_i) @ B_i,
// A_i [H1, r], B_i [r, H2], row-major.
//
// Work decomposition. A job is (problem p, segment s, chunk of <= 8 tokens).
// One thread-block cluster of C CTAs runs a job; CTA c owns rows
// [c*KS, (c+1)*KS) of A_i for the shrink and columns [c*NS, (c+1)*NS) of B_i
// for the expand, so every adapter byte is read once per job by one CTA.
// Clusters are persistent (as many as fit on the GPU at once) and take jobs
// round-robin.
//
// Data movement. Warp 0 of each CTA is a producer: it streams the CTA's
// operands through a ring of shared-memory stages with TMA bulk copies
// (cp.async.bulk, completion counted on the stage's mbarrier). A shrink stage
// holds up to KT rows of A_i (one contiguous copy) and the same KT columns of
// the chunk's X rows; an expand stage holds the r rows of a column tile of
// B_i (one copy per row, rows padded by 16 bytes so that the
// consumers' 16-byte reads spread over all banks). B does not depend on V,
// so the producer runs ahead into the expand stages while the consumers wait
// for the cluster's reduction of V.
//
// Compute. Warps 1..4 consume. Shrink: fp32 FMA over the stage, specialised
// for 1, 2, 4 or 8 tokens; partial sums reduced across lanes by shuffles and
// across warps in shared memory. The C partial V tiles are exchanged through
// distributed shared memory: each CTA publishes its tile in its own shared
// memory and signals every CTA's "ready" mbarrier remotely; each CTA then
// sums all C tiles in rank order (so every CTA holds bit-identical V) and
// signals every owner's "free" mbarrier. Expand: each thread covers 8 columns
// and 8 of the r rows of a stage; lanes reduce over row groups by shuffles, and one
// lane per column group adds scale * acc to Y (read before waiting on the
// stage) and rounds once.
//
// Every mbarrier wait is bounded; a wait that gives up sets
// LORA_SGMV_DEV_TIMEOUT in the status word and the kernel runs to its end
// (results are then invalid, but nothing hangs). The kernel never traps.
#pragma once

#include <cooperative_groups.h>

#include "sgmv_common.cuh"

namespace sgmv {

constexpr int kFusedMaxProblems = 8;
constexpr int kFusedTokens = 8;       // tokens per job (chunk)
constexpr int kFusedStages = 4;       // ring depth
constexpr int kFusedStageData = 16384;  // payload bytes per stage
constexpr int kFusedConsumerWarps = 4;
constexpr int kFusedThreads = 32 * (1 + kFusedConsumerWarps);
constexpr int kFusedCluster = 8;
constexpr uint32_t kSpinLimit = 1u << 22;

struct FusedProblem {
    void* Y;
    const void* X;
    const void* const* A_ptrs;
    const void* const* B_ptrs;
    int num_adapters;
    int H1;
    int H2;
    float scale;
    int ks;  // rows of A_i per CTA (multiple of 8)
    int ns;  // columns of B_i per CTA (multiple of 8)
};

struct FusedParams {
    FusedProblem prob[kFusedMaxProblems];
    const int32_t* seg_starts;
    const int32_t* lora_idx;
    uint32_t* dev_status;
    int n_problems;
    int n_segments;
    int T;
    int chunk_slots;  // TY: token-chunk slots per segment
};

// compile-time geometry per rank
template <int R>
struct FusedGeom {
    static constexpr int KT = (kFusedStageData / (2 * (R + kFusedTokens))) / 8 * 8;  // A rows per stage
    static constexpr int NTC = kFusedStageData / (2 * R);                            // B columns per stage
    static constexpr int BPITCH = NTC * 2 + 16;                                      // bytes per B row in smem
    static constexpr int STAGE = (R * BPITCH > kFusedStageData ? R * BPITCH : kFusedStageData);
    static constexpr int CG = R / 8;                                                 // 8-column groups of A
    static constexpr int RLN = 128 / CG;                                             // shrink row lanes
    static constexpr int RG = R / 8;                                                 // expand row groups
    static constexpr int GC = 128 / RG;                                              // expand column groups
    static_assert(NTC == 8 * GC, "expand tile must give every consumer thread 8 columns");
    static constexpr size_t RING = size_t(kFusedStages) * STAGE;
    static constexpr size_t RED = size_t(kFusedConsumerWarps) * kFusedTokens * R * 4;
    static constexpr size_t SLOT = size_t(kFusedTokens) * R * 4;
    static constexpr size_t SMEM = RING + RED + 2 * SLOT + SLOT /* vs */;
};

// ---- PTX wrappers ------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive on the mbarrier at the same offset in CTA `rank` of this cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* bar, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded waits. A wait gives up after kWaitLimitNs (or kSpinLimit polls), records
// LORA_SGMV_DEV_TIMEOUT and marks the thread dead: every later wait of that thread
// returns at once, so a broken protocol ends the kernel quickly instead of hanging it.
constexpr uint64_t kWaitLimitNs = 200ull * 1000 * 1000;

template <bool kCluster>
__device__ __forceinline__ void mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t* status, bool& dead) {
    if (dead) return;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return;
        if ((i & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
    dead = true;
    report(status, LORA_SGMV_DEV_TIMEOUT);
}

__device__ __forceinline__ void mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status, bool& dead) {
    mbar_wait_bounded<false>(bar, parity, status, dead);
}

__device__ __forceinline__ void mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t* status, bool& dead) {
    mbar_wait_bounded<true>(bar, parity, status, dead);
}

// 1-D TMA bulk copy global -> this CTA's shared memory, completion on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

__device__ __forceinline__ void consumer_sync() {  // named barrier 1 over the 4 consumer warps
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kFusedConsumerWarps) : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// ---- job enumeration (identical in producer and consumers) ------------------------------

struct Job {
    int p;      // problem
    int t0;     // first token
    int nt;     // tokens (1..8)
    const void* a;
    const void* b;
    int k0, nk;  // this CTA's rows of A_i
    int c0, nc;  // this CTA's columns of B_i
};

// Returns false when job slot j holds no work; otherwise fills `job` (uniform over the cluster).
__device__ __forceinline__ bool job_at(const FusedParams& P, int j, int sub, int c, Job& job, uint32_t& bad) {
    const int TY = P.chunk_slots;
    const int qs = j % TY;
    const int s = (j / TY) % P.n_segments;
    const int p = j / (TY * P.n_segments);
    const FusedProblem& pr = P.prob[p];
    Segment seg;
    bad = load_segment(P.seg_starts, P.lora_idx, pr.A_ptrs, pr.B_ptrs, s, P.T, pr.num_adapters, seg);
    if (bad) return false;
    const int q = qs + sub * TY;
    const int t0 = seg.begin + q * kFusedTokens;
    if (t0 >= seg.end) return false;
    job.p = p;
    job.t0 = t0;
    job.nt = min(kFusedTokens, seg.end - t0);
    job.a = seg.a;
    job.b = seg.b;
    job.k0 = c * pr.ks;
    job.nk = max(0, min(pr.ks, pr.H1 - job.k0));
    job.c0 = c * pr.ns;
    job.nc = max(0, min(pr.ns, pr.H2 - job.c0));
    return true;
}

// Number of token chunks a job slot covers at most (sub-jobs); sub-job `sub` of slot j is chunk qs + sub*TY.
__device__ __forceinline__ int slot_subjobs(const FusedParams& P, int j) {
    const int TY = P.chunk_slots;
    const int qs = j % TY;
    const int s = (j / TY) % P.n_segments;
    const int b = __ldg(P.seg_starts + s), e = __ldg(P.seg_starts + s + 1);
    const int L = (b >= 0 && e >= b) ? e - b : 0;
    const int chunks = (L + kFusedTokens - 1) / kFusedTokens;
    return chunks > qs ? (chunks - qs + TY - 1) / TY : 0;
}

// ---- consumer bodies ---------------------------------------------------------------------

template <typename T, int R, int NTOK>
__device__ __forceinline__ void consume_job(const FusedParams& P, const Job& job, unsigned char* ring,
                                            uint64_t* full, uint64_t* empty, float* red, float* slot,
                                            float* vs, uint64_t* vready, uint64_t* vfree, uint32_t& it,
                                            uint32_t u, int C, int ct, bool& dead) {
    using G = FusedGeom<R>;
    const int lane = ct & 31;
    const int cw = ct >> 5;  // consumer warp 0..3
    const int nt = job.nt;
    const FusedProblem& pr = P.prob[job.p];

    // ---------------- shrink: partial V over this CTA's rows of A_i ----------------
    float acc[NTOK][8];
#pragma unroll
    for (int t = 0; t < NTOK; ++t)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[t][i] = 0.f;
    const int cg = ct % G::CG;
    const int rl = ct / G::CG;
    const int nA = (job.nk + G::KT - 1) / G::KT;
    for (int ta = 0; ta < nA; ++ta, ++it) {
        const uint32_t stage = it % kFusedStages;
        mbar_wait(&full[stage], (it / kFusedStages) & 1u, P.dev_status, dead);
        const unsigned char* st = ring + size_t(stage) * G::STAGE;
        const T* xs = reinterpret_cast<const T*>(st + size_t(G::KT) * R * 2);
        const int kt = min(G::KT, job.nk - ta * G::KT);
        for (int k = rl; k < kt; k += G::RLN) {
            float a[8];
            unpack8<T>(*reinterpret_cast<const uint4*>(st + (size_t(k) * R + cg * 8) * 2), a);
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                if (t < nt) {
                    const float x = Storage<T>::to1(xs[size_t(t) * G::KT + k]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[t][i] = fmaf(x, a[i], acc[t][i]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_local(&empty[stage]);
    }
    // reduce over the row lanes of each warp (lanes sharing cg), then across the 4 warps
#pragma unroll
    for (int off = G::CG; off < 32; off <<= 1)
#pragma unroll
        for (int t = 0; t < NTOK; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[t][i] += __shfl_xor_sync(0xffffffffu, acc[t][i], off);
    if (lane < G::CG) {
#pragma unroll
        for (int t = 0; t < NTOK; ++t)
            if (t < nt) {
#pragma unroll
                for (int i = 0; i < 8; ++i) red[(cw * kFusedTokens + t) * R + cg * 8 + i] = acc[t][i];
            }
    }
    const uint32_t ph = u & 1u;
    float* my_slot = slot + size_t(ph) * kFusedTokens * R;
    // the slot may still be read by the cluster for job u-2
    if (u >= 2) mbar_wait_cluster(&vfree[ph], ((u - 2) >> 1) & 1u, P.dev_status, dead);
    consumer_sync();
    for (int e = ct; e < nt * R; e += 128) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kFusedConsumerWarps; ++w) sum += red[w * kFusedTokens * R + e];
        my_slot[e] = sum;
    }
    fence_cluster();
    consumer_sync();
    if (ct < C) mbar_arrive_remote(&vready[ph], static_cast<uint32_t>(ct));
    // every CTA's tile of this job is published once vready completes
    mbar_wait_cluster(&vready[ph], (u >> 1) & 1u, P.dev_status, dead);
    {
        cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
        for (int e = ct; e < nt * R; e += 128) {
            float sum = 0.f;
            for (int q = 0; q < C; ++q) sum += cluster.map_shared_rank(my_slot, q)[e];
            vs[e] = sum;
        }
    }
    fence_cluster();
    consumer_sync();
    if (ct < C) mbar_arrive_remote(&vfree[ph], static_cast<uint32_t>(ct));

    // ---------------- expand: Y[t, cols] += scale * V[t,:] @ B_i[:, cols] ----------------
    const int rg = ct % G::RG;
    const int gc = ct / G::RG;
    T* __restrict__ Y = static_cast<T*>(pr.Y);
    const int nB = (job.nc + G::NTC - 1) / G::NTC;
    for (int tb = 0; tb < nB; ++tb, ++it) {
        const int col_in_tile = gc * 8;
        const int nct = min(G::NTC, job.nc - tb * G::NTC);
        const bool writer = (rg == 0) && (col_in_tile < nct);
        const int col = job.c0 + tb * G::NTC + col_in_tile;
        uint4 yv[NTOK];
        if (writer) {
#pragma unroll
            for (int t = 0; t < NTOK; ++t)
                if (t < nt) yv[t] = ld_vec(Y + size_t(job.t0 + t) * pr.H2 + col);
        }
        const uint32_t stage = it % kFusedStages;
        mbar_wait(&full[stage], (it / kFusedStages) & 1u, P.dev_status, dead);
        const unsigned char* st = ring + size_t(stage) * G::STAGE;
        float o[NTOK][8];
#pragma unroll
        for (int t = 0; t < NTOK; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) o[t][i] = 0.f;
        if (col_in_tile < nct) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int j = rg + G::RG * jj;
                float b[8];
                unpack8<T>(*reinterpret_cast<const uint4*>(st + size_t(j) * G::BPITCH + col_in_tile * 2), b);
#pragma unroll
                for (int t = 0; t < NTOK; ++t) {
                    if (t < nt) {
                        const float v = vs[t * R + j];
#pragma unroll
                        for (int i = 0; i < 8; ++i) o[t][i] = fmaf(v, b[i], o[t][i]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_local(&empty[stage]);
#pragma unroll
        for (int off = 1; off < G::RG; off <<= 1)
#pragma unroll
            for (int t = 0; t < NTOK; ++t)
#pragma unroll
                for (int i = 0; i < 8; ++i) o[t][i] += __shfl_xor_sync(0xffffffffu, o[t][i], off);
        if (writer) {
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                if (t < nt) {
                    float y[8];
                    unpack8<T>(yv[t], y);
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = __fadd_rn(y[i], __fmul_rn(pr.scale, o[t][i]));
                    st_vec(Y + size_t(job.t0 + t) * pr.H2 + col, pack8<T>(y));
                }
            }
        }
    }
}

// ---- the kernel ----------------------------------------------------------------------------

// grid.x = C * clusters, cluster (C,1,1). Block: warp 0 producer, warps 1..4 consumers.
template <typename T, int R>
__global__ void __launch_bounds__(kFusedThreads, 2) sgmv_fused_kernel(const FusedParams P) {
    using G = FusedGeom<R>;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kFusedStages];
    __shared__ __align__(8) uint64_t empty[kFusedStages];
    __shared__ __align__(8) uint64_t vready[2];
    __shared__ __align__(8) uint64_t vfree[2];

    unsigned char* ring = smem;
    float* red = reinterpret_cast<float*>(smem + G::RING);
    float* slot = red + kFusedConsumerWarps * kFusedTokens * R;
    float* vs = slot + 2 * kFusedTokens * R;

    const int C = kFusedCluster;
    const int c = static_cast<int>(cluster_rank());
    const int cluster_id = blockIdx.x / C;
    const int n_clusters = gridDim.x / C;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFusedStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kFusedConsumerWarps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&vready[s], C);
            mbar_init(&vfree[s], C);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // every CTA's barriers exist before any remote arrive
    cluster_sync_all();

    const int J = P.n_problems * P.n_segments * P.chunk_slots;
    bool dead = false;
    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        uint32_t it = 0;
        for (int j = cluster_id; j < J; j += n_clusters) {
            const int subs = slot_subjobs(P, j);
            for (int sub = 0; sub < subs; ++sub) {
                Job job;
                uint32_t bad;
                if (!job_at(P, j, sub, c, job, bad)) continue;
                const FusedProblem& pr = P.prob[job.p];
                const T* X = static_cast<const T*>(pr.X);
                const T* A = static_cast<const T*>(job.a);
                const T* B = static_cast<const T*>(job.b);
                const int nA = (job.nk + G::KT - 1) / G::KT;
                for (int ta = 0; ta < nA; ++ta, ++it) {
                    const uint32_t stage = it % kFusedStages;
                    if (it >= kFusedStages) mbar_wait(&empty[stage], ((it / kFusedStages) - 1) & 1u, P.dev_status, dead);
                    unsigned char* st = ring + size_t(stage) * G::STAGE;
                    const int k = job.k0 + ta * G::KT;
                    const int kt = min(G::KT, job.nk - ta * G::KT);
                    if (lane == 0) mbar_arrive_expect_tx(&full[stage], uint32_t(kt) * (R + job.nt) * 2);
                    __syncwarp();
                    if (lane == 0) bulk_g2s(st, A + size_t(k) * R, uint32_t(kt) * R * 2, &full[stage]);
                    else if (lane <= job.nt)
                        bulk_g2s(st + size_t(G::KT) * R * 2 + size_t(lane - 1) * G::KT * 2,
                                 X + size_t(job.t0 + lane - 1) * pr.H1 + k, uint32_t(kt) * 2, &full[stage]);
                }
                const int nB = (job.nc + G::NTC - 1) / G::NTC;
                for (int tb = 0; tb < nB; ++tb, ++it) {
                    const uint32_t stage = it % kFusedStages;
                    if (it >= kFusedStages) mbar_wait(&empty[stage], ((it / kFusedStages) - 1) & 1u, P.dev_status, dead);
                    unsigned char* st = ring + size_t(stage) * G::STAGE;
                    const int col = job.c0 + tb * G::NTC;
                    const int nct = min(G::NTC, job.nc - tb * G::NTC);
                    if (lane == 0) mbar_arrive_expect_tx(&full[stage], uint32_t(nct) * R * 2);
                    __syncwarp();
                    for (int row = lane; row < R; row += 32)
                        bulk_g2s(st + size_t(row) * G::BPITCH, B + size_t(row) * pr.H2 + col, uint32_t(nct) * 2,
                                 &full[stage]);
                }
            }
        }
    } else {
        // ------------------------------ consumers ------------------------------
        const int ct = threadIdx.x - 32;
        uint32_t it = 0, u = 0;
        for (int j = cluster_id; j < J; j += n_clusters) {
            const int subs = slot_subjobs(P, j);
            for (int sub = 0; sub < subs; ++sub) {
                Job job;
                uint32_t bad;
                if (!job_at(P, j, sub, c, job, bad)) continue;  // reported below
                if (job.nt == 1)
                    consume_job<T, R, 1>(P, job, ring, full, empty, red, slot, vs, vready, vfree, it, u, C, ct, dead);
                else if (job.nt <= 2)
                    consume_job<T, R, 2>(P, job, ring, full, empty, red, slot, vs, vready, vfree, it, u, C, ct, dead);
                else if (job.nt <= 4)
                    consume_job<T, R, 4>(P, job, ring, full, empty, red, slot, vs, vready, vfree, it, u, C, ct, dead);
                else
                    consume_job<T, R, 8>(P, job, ring, full, empty, red, slot, vs, vready, vfree, it, u, C, ct, dead);
                ++u;
            }
        }
        // the last two exchange slots may still be read by the cluster
        for (uint32_t v = (u >= 2 ? u - 2 : 0); v < u; ++v)
            mbar_wait_cluster(&vfree[v & 1u], (v >> 1) & 1u, P.dev_status, dead);
    }
    // report each rejected segment once (the job loops above skip them silently)
    if (threadIdx.x == 32 && c == 0) {
        for (int j = cluster_id; j < J; j += n_clusters) {
            if (j % P.chunk_slots) continue;
            const int s = (j / P.chunk_slots) % P.n_segments;
            const int p = j / (P.chunk_slots * P.n_segments);
            Segment seg;
            const uint32_t bad = load_segment(P.seg_starts, P.lora_idx, P.prob[p].A_ptrs, P.prob[p].B_ptrs, s,
                                              P.T, P.prob[p].num_adapters, seg);
            if (bad) report(P.dev_status, bad);
        }
    }
}

}  // namespace sgmv

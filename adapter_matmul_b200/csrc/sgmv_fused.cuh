// sgmv_fused.cuh -- one-kernel SGMV for short segments (decode): shrink, V reduction
// and expand with the fused add, for one or several projections in one launch.
//
// Maths (page “Punica：多 LoRA 模型统一服务框架”, the Punica README, its LoRA and multi-LoRA paragraphs): for each segment s
// with adapter i and each row t of it, Y[t,:] += scale * (X[t,:] @ A_i) @ B_i,
// A_i [H1, r], B_i [r, H2], row-major.
//
// Jobs. A job is (problem p, segment s, chunk of <= CH tokens of s), CH = 8, or 4 when the
// call's segments reach 16 tokens (the host's choice: a long segment's jobs then carry half the
// Y rows and expand work each and spread over twice as many clusters). At start
// every CTA reads seg_starts once and builds the exact job list (a prefix sum
// of the segments' chunk counts in shared memory), so long segments split
// into as many jobs as they have chunks and no slot is empty. Clusters are
// persistent (as many as are resident at once) and take jobs round-robin.
//
// Split of one job over a cluster of C CTAs (C = 1, 2, 4 or 8, chosen by the
// host so that all jobs run in one resident wave when they can): CTA c owns
// rows [c*KS, (c+1)*KS) of A_i for the shrink and columns [c*NS, (c+1)*NS) of
// B_i for the expand, so each adapter byte is read once per job.
//
// Data movement. Warp 0 of each CTA is a producer: it streams the CTA's
// operands through a ring of shared-memory stages with TMA bulk copies
// (cp.async.bulk; completion counted on the stage's mbarrier). A shrink stage
// holds KT rows of A_i (one contiguous copy) and the same KT columns of the
// chunk's X rows (KT shrinks as the chunk's token count grows). An expand
// stage holds r rows of a column tile of B_i (one copy per row, rows padded
// by 16 bytes so that 16-byte reads spread over the banks) and the matching
// tile of the chunk's Y rows. Nothing in an expand stage depends on V, so the
// producer streams ahead while the consumers reduce V.
//
// Compute. Warps 1..4 consume. Shrink: fp32 FMA over each stage, specialised
// for 1, 2, 4 or 8 tokens; partial sums reduced over lanes by shuffles and
// over warps in shared memory. Reduction of V over the cluster: each CTA
// pushes its partial tile into every CTA's receive buffer with st.async,
// whose completion is counted on the receiver's mbarrier; each CTA sums the
// C tiles in rank order (so all hold identical V) and then tells every sender
// that its slot may be reused. Expand: each thread covers 8 columns and 8 of
// the r rows of a stage; lanes reduce over row groups by shuffles, and one
// lane per column group adds scale * acc to the staged Y, rounds once and
// stores to global memory.
//
// Programmatic dependent launch: the kernel lets the next kernel on the stream
// launch at once. By default every thread waits (griddepcontrol.wait, which
// returns when the previous kernel has completed) before it reads anything the
// caller passed, so only the prologue overlaps the previous kernel. When the
// caller states that the segment arrays, pointer tables and adapters are not
// written by the kernel immediately before this one (P.early), those are read
// at once and the first A_i copies stream while that kernel finishes; X and Y
// are then read only after the wait.
//
// Every mbarrier wait is bounded in time; a wait that gives up sets
// LORA_SGMV_DEV_TIMEOUT in the status word and the thread's later waits
// return at once, so the kernel always ends. The kernel never traps.
#pragma once

#include "sgmv_common.cuh"

namespace sgmv {

constexpr int kFusedMaxProblems = 8;
#ifndef SGMV_FUSED_STAGES
#define SGMV_FUSED_STAGES 4
#endif
#ifndef SGMV_FUSED_MIN_BLOCKS
#define SGMV_FUSED_MIN_BLOCKS 2
#endif
constexpr int kFusedTokens = 8;                  // tokens per job (chunk); 4 for calls with long segments
constexpr int kFusedStages = SGMV_FUSED_STAGES;  // ring depth
constexpr int kFusedConsumerWarps = 4;
constexpr int kFusedConsumers = 32 * kFusedConsumerWarps;
constexpr int kFusedThreads = 32 + kFusedConsumers;
constexpr int kFusedMaxCluster = 8;
constexpr int kFusedMaxSegments = 8192;  // job list held in shared memory
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr uint64_t kWaitLimitNs = 200ull * 1000 * 1000;

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
    int one_chunk;  // host hint: every segment fits one chunk (job j is segment j; correct either way)
    int early;      // 1: segment arrays, tables and adapters may be read before griddepcontrol.wait
};

// compile-time geometry per rank and chunk size (tokens per job)
template <int R, int CH = kFusedTokens>
struct FusedGeom {
    static constexpr int RG = R / 8;                                   // expand row groups (8 rows each)
    static constexpr int NTC = (1024 / RG) < 512 ? (1024 / RG) : 512;  // B columns per stage
    static constexpr int GC = NTC / 8;                                 // expand column groups
    static_assert(RG * GC <= kFusedConsumers, "expand tile too wide");
    static constexpr int BPITCH = NTC * 2 + 16;                        // bytes per staged B row
    static constexpr int BSTAGE = R * BPITCH + CH * NTC * 2;          // B rows + Y rows
    static constexpr int STAGE = (BSTAGE > 16384 ? BSTAGE : 16384);
    static constexpr int CG = R / 8;                                   // 8-column groups of A
    static constexpr int RLN = kFusedConsumers / CG;                   // shrink row lanes
    static constexpr size_t RING = size_t(kFusedStages) * STAGE;
    static constexpr size_t RED = size_t(kFusedConsumerWarps) * CH * R * 4;
    static constexpr size_t TILE = size_t(CH) * R * 4;            // one partial V tile
    static constexpr size_t RECV = kFusedMaxCluster * TILE;
    static constexpr size_t BASE = RING + RED + RECV + TILE;      // + the job prefix (n+1 ints)
    // A rows per shrink stage for a chunk of nt tokens (A rows plus X columns fill a stage)
    static __host__ __device__ constexpr int kt_for(int nt) { return (STAGE / (2 * (R + nt))) / 8 * 8; }
};

// ---- PTX wrappers ------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t map_rank(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    return remote;
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

// Arrival without release semantics, for "this buffer has been read" signals: the reads it
// stands for have returned their values before it issues, and a release here would also wait
// for every global store still in flight from this thread (a round trip to L2 per stage).
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t* bar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive on the mbarrier at the same offset in CTA `rank` of this cluster (release, cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint64_t* bar, uint32_t rank) {
    const uint32_t remote = map_rank(smem_u32(bar), rank);
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

// Bounded wait: gives up after kWaitLimitNs (or kSpinLimit polls), records
// LORA_SGMV_DEV_TIMEOUT and marks the thread dead; a dead thread's later
// waits return at once, so a broken protocol ends the kernel quickly. The
// global timer is slow to read, so it is read only after 64 unsuccessful
// polls, and then every 64 polls.
template <bool kCluster>
__device__ __forceinline__ void mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status, bool& dead) {
    if (dead) return;
    uint64_t t0 = 0;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return;
        if ((i & 63u) == 63u) {
            const uint64_t now = globaltimer_ns();
            if (t0 == 0)
                t0 = now;
            else if (now - t0 > kWaitLimitNs)
                break;
        }
    }
    dead = true;
    report(status, LORA_SGMV_DEV_TIMEOUT);
}

// 1-D TMA bulk copy global -> this CTA's shared memory, completion on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 16-byte asynchronous store into CTA `rank`'s shared memory; completion counted on
// that CTA's mbarrier at the same offset as `bar`.
__device__ __forceinline__ void st_async_v4(float* dst_local, float4 v, uint64_t* bar, uint32_t rank) {
    const uint32_t dst = map_rank(smem_u32(dst_local), rank);
    const uint32_t mb = map_rank(smem_u32(bar), rank);
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(dst),
        "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(mb)
        : "memory");
}

__device__ __forceinline__ void consumer_sync() {  // named barrier 1 over the consumer warps
    asm volatile("bar.sync 1, %0;" ::"n"(kFusedConsumers) : "memory");
}

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Bulk prefetch of global memory into L2 (no shared memory, no completion to wait on).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// ---- job list --------------------------------------------------------------------------

// Warm L2 with the small arrays the first jobs read (segment bounds, adapter ids, pointer
// tables) while the previous kernel on the stream may still run. A prefetch reads no value into
// the kernel (L2 stays coherent with later writes), so it is safe under the default contract;
// the CTAs of the grid split the table lines between them.
__device__ __forceinline__ void prefetch_metadata(const FusedParams& P) {
    const int tid = threadIdx.x, nth = blockDim.x;
    const int n = P.n_segments;
    const int lines_seg = (n + 1 + 31) / 32;  // 128-byte lines of seg_starts (and of lora_idx)
    for (int l = tid; l < 2 * lines_seg; l += nth) {
        const int32_t* base = l < lines_seg ? P.seg_starts : P.lora_idx;
        const int off = (l < lines_seg ? l : l - lines_seg) * 32;
        if (off < n + 1) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + off));
    }
    for (int p = 0; p < P.n_problems; ++p) {
        const int lines_tab = (P.prob[p].num_adapters + 15) / 16;  // 16 pointers per line
        for (int l = blockIdx.x + gridDim.x * tid; l < 2 * lines_tab; l += gridDim.x * nth) {
            const void* const* tab = l < lines_tab ? P.prob[p].A_ptrs : P.prob[p].B_ptrs;
            asm volatile("prefetch.global.L2 [%0];" ::"l"(tab + (l < lines_tab ? l : l - lines_tab) * 16));
        }
    }
}

// LORA_SGMV_DEV_BAD_SEGMENT if the bounds of segment s break the contract, else 0.
__device__ __forceinline__ uint32_t segment_bounds_check(const FusedParams& P, int s) {
    const int b = __ldg(P.seg_starts + s), e = __ldg(P.seg_starts + s + 1);
    return (b < 0 || b > e || e > P.T) ? LORA_SGMV_DEV_BAD_SEGMENT : 0u;
}

// Number of CH-token chunks of segment s, or 0 if the segment is empty or invalid.
template <int CH = kFusedTokens>
__device__ __forceinline__ int segment_chunks(const FusedParams& P, int s) {
    const int b = __ldg(P.seg_starts + s), e = __ldg(P.seg_starts + s + 1);
    if (b < 0 || b > e || e > P.T) return 0;
    return (e - b + CH - 1) / CH;
}

// pref[s] = chunks of segments 0..s-1 (pref[0] = 0, pref[n] = chunks per problem), built by all
// threads of the block (at most 256).
template <int CH = kFusedTokens>
__device__ void build_job_prefix(const FusedParams& P, int* pref) {
    __shared__ int warp_tot[8];
    const int n = P.n_segments;
    const int nthreads = blockDim.x;
    const int per = (n + nthreads - 1) / nthreads;
    const int s0 = threadIdx.x * per;
    const int s1 = min(n, s0 + per);
    int local = 0;
    for (int s = s0; s < s1; ++s) {
        local += segment_chunks<CH>(P, s);
        // a segment with invalid bounds has no chunk, so no job reports it: CTA 0 does, here
        if (blockIdx.x == 0) report(P.dev_status, segment_bounds_check(P, s));
        // warm L1 for the lookups job_at() makes next: adapter id, then its table entries
        const int i = __ldg(P.lora_idx + s);
        for (int p = 0; p < P.n_problems; ++p) {
            if (i >= 0 && i < P.prob[p].num_adapters) {
                asm volatile("prefetch.global.L1 [%0];" ::"l"(P.prob[p].A_ptrs + i));
                asm volatile("prefetch.global.L1 [%0];" ::"l"(P.prob[p].B_ptrs + i));
            }
        }
    }
    // inclusive scan of `local` over the block
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int v = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += y;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    int run = before + v - local;  // exclusive prefix of this thread's first segment
    if (threadIdx.x == 0) pref[0] = 0;
    for (int s = s0; s < s1; ++s) {
        run += segment_chunks<CH>(P, s);
        pref[s + 1] = run;
    }
    __syncthreads();
}

struct Job {
    int p;   // problem
    int t0;  // first token
    int nt;  // tokens (1..8)
    const void* a;
    const void* b;
    int k0, nk;  // this CTA's rows of A_i
    int c0, nc;  // this CTA's columns of B_i
};

// Jobs of list entry j: (problem, segment, first chunk, number of chunks). With the
// prefix, an entry is one chunk; in one-chunk mode an entry is a whole segment, whose
// chunks the cluster then runs one after another.
template <int CH = kFusedTokens>
__device__ __forceinline__ void entry_at(const FusedParams& P, const int* pref, int j, int& p, int& s, int& q0,
                                         int& nq) {
    if (P.one_chunk) {
        p = j / P.n_segments;
        s = j - p * P.n_segments;
        q0 = 0;
        nq = segment_chunks<CH>(P, s);
        return;
    }
    const int per_problem = pref[P.n_segments];
    p = j / per_problem;
    const int r = j - p * per_problem;
    int lo = 0, hi = P.n_segments;  // largest s with pref[s] <= r
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pref[mid] <= r)
            lo = mid;
        else
            hi = mid;
    }
    s = lo;
    q0 = r - pref[s];
    nq = 1;
}

// Chunk q (of CH tokens) of segment s of problem p: 0, or the LORA_SGMV_DEV_* bits of the
// device-side checks the segment fails (then the job is not filled in).
template <int CH = kFusedTokens>
__device__ __forceinline__ uint32_t job_check(const FusedParams& P, int p, int s, int q, int c, Job& job) {
    const FusedProblem& pr = P.prob[p];
    Segment seg;
    const uint32_t bad = load_segment(P.seg_starts, P.lora_idx, pr.A_ptrs, pr.B_ptrs, s, P.T, pr.num_adapters, seg);
    if (bad) return bad;
    job.p = p;
    job.t0 = seg.begin + q * CH;
    job.nt = min(CH, seg.end - job.t0);
    job.a = seg.a;
    job.b = seg.b;
    job.k0 = c * pr.ks;
    job.nk = max(0, min(pr.ks, pr.H1 - job.k0));
    job.c0 = c * pr.ns;
    job.nc = max(0, min(pr.ns, pr.H2 - job.c0));
    return 0u;
}

template <int CH = kFusedTokens>
__device__ __forceinline__ bool job_at(const FusedParams& P, int p, int s, int q, int c, Job& job) {
    return job_check<CH>(P, p, s, q, c, job) == 0u;
}

// One-chunk mode, producer warp: the first chunk of segment s of problem p as a job, with the
// segment's metadata fetched by the lanes in parallel (its bounds and adapter id, and, when the
// problem has at most 32 adapters, every entry of both pointer tables), so the adapter's address
// is known after one round trip instead of three dependent ones. The checks are load_segment's.
// Returns the segment's chunks; 0 when it is empty or fails a check (the job is then not set).
template <int CH = kFusedTokens>
__device__ __forceinline__ int first_job_warp(const FusedParams& P, int p, int s, int c, int lane, Job& job) {
    const FusedProblem& pr = P.prob[p];
    int v = 0;
    if (lane == 0)
        v = __ldg(P.seg_starts + s);
    else if (lane == 1)
        v = __ldg(P.seg_starts + s + 1);
    else if (lane == 2)
        v = __ldg(P.lora_idx + s);
    const bool whole_table = pr.num_adapters <= 32;
    unsigned long long ta = 0, tb = 0;
    if (whole_table && lane < pr.num_adapters) {
        ta = __ldg(reinterpret_cast<const unsigned long long*>(pr.A_ptrs) + lane);
        tb = __ldg(reinterpret_cast<const unsigned long long*>(pr.B_ptrs) + lane);
    }
    const int b = __shfl_sync(0xffffffffu, v, 0);
    const int e = __shfl_sync(0xffffffffu, v, 1);
    const int i = __shfl_sync(0xffffffffu, v, 2);
    if (b < 0 || b > e || e > P.T || i < 0 || i >= pr.num_adapters) return 0;
    unsigned long long a, bb;
    if (whole_table) {
        a = __shfl_sync(0xffffffffu, ta, i);
        bb = __shfl_sync(0xffffffffu, tb, i);
    } else {
        a = __ldg(reinterpret_cast<const unsigned long long*>(pr.A_ptrs) + i);
        bb = __ldg(reinterpret_cast<const unsigned long long*>(pr.B_ptrs) + i);
    }
    if (a == 0 || bb == 0 || ((a | bb) & 15u)) return 0;
    job.p = p;
    job.t0 = b;
    job.nt = min(CH, e - b);
    job.a = reinterpret_cast<const void*>(a);
    job.b = reinterpret_cast<const void*>(bb);
    job.k0 = c * pr.ks;
    job.nk = max(0, min(pr.ks, pr.H1 - job.k0));
    job.c0 = c * pr.ns;
    job.nc = max(0, min(pr.ns, pr.H2 - job.c0));
    return (e - b + CH - 1) / CH;
}

// A rejected segment is reported by the one thread that meets it first as a job (`reporter`:
// one thread of the first CTA of the visiting cluster); a one-chunk-mode entry without chunks
// may be a segment with invalid bounds.
template <int CH = kFusedTokens>
__device__ __forceinline__ bool job_at_reporting(const FusedParams& P, int p, int s, int q, int c, Job& job,
                                                 bool reporter) {
    const uint32_t bad = job_check<CH>(P, p, s, q, c, job);
    if (bad && reporter) report(P.dev_status, bad);
    return bad == 0u;
}

// ---- consumer body ----------------------------------------------------------------------

struct FusedSmem {
    unsigned char* ring;
    uint64_t* full;
    uint64_t* empty;
    uint64_t* vready;
    uint64_t* vfree;
    float* red;
    float* recv;
    float* vs;
};

template <typename T, int R, int NTOK, int CH>
__device__ __forceinline__ void consume_job(const FusedParams& P, const Job& job, const FusedSmem& S, uint32_t& it,
                                            uint32_t u, int C, int c, int ct, bool& dead) {
    using G = FusedGeom<R, CH>;
    const int lane = ct & 31;
    const int cw = ct >> 5;
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
    const int KT = G::kt_for(nt);
    const int nA = (job.nk + KT - 1) / KT;
    for (int ta = 0; ta < nA; ++ta, ++it) {
        const uint32_t stage = it % kFusedStages;
        mbar_wait<false>(&S.full[stage], (it / kFusedStages) & 1u, P.dev_status, dead);
        const unsigned char* st = S.ring + size_t(stage) * G::STAGE;
        const T* xs = reinterpret_cast<const T*>(st + size_t(KT) * R * 2);
        const int kt = min(KT, job.nk - ta * KT);
        for (int k = rl; k < kt; k += G::RLN) {
            float a[8];
            unpack8<T>(*reinterpret_cast<const uint4*>(st + (size_t(k) * R + cg * 8) * 2), a);
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                if (t < nt) {
                    const float x = Storage<T>::to1(xs[size_t(t) * KT + k]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[t][i] = fmaf(x, a[i], acc[t][i]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&S.empty[stage]);
    }
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
                for (int i = 0; i < 8; ++i) S.red[(cw * CH + t) * R + cg * 8 + i] = acc[t][i];
            }
    }
    consumer_sync();

    // ---------------- V: push this CTA's tile to every CTA of the cluster ----------------
    const uint32_t tile_bytes = uint32_t(nt) * R * 4;
    if (ct == 0) mbar_arrive_expect_tx(S.vready, tile_bytes * C);
    // every receiver must have consumed this CTA's previous tile
    if (u >= 1) mbar_wait<true>(S.vfree, (u - 1) & 1u, P.dev_status, dead);
    for (int e4 = ct; e4 < nt * R / 4; e4 += kFusedConsumers) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kFusedConsumerWarps; ++w) {
            const float4 q = *reinterpret_cast<const float4*>(S.red + w * CH * R + e4 * 4);
            v.x += q.x;
            v.y += q.y;
            v.z += q.z;
            v.w += q.w;
        }
        for (int q = 0; q < C; ++q) st_async_v4(S.recv + size_t(c) * CH * R + e4 * 4, v, S.vready, q);
    }
    mbar_wait<true>(S.vready, u & 1u, P.dev_status, dead);
    for (int e = ct; e < nt * R; e += kFusedConsumers) {
        float sum = 0.f;
        for (int q = 0; q < C; ++q) sum += S.recv[size_t(q) * CH * R + e];
        S.vs[e] = sum;
    }
    consumer_sync();
    if (ct < C) mbar_arrive_remote(S.vfree, static_cast<uint32_t>(ct));  // sender ct may reuse my slot

    // ---------------- expand: Y[t, cols] += scale * V[t,:] @ B_i[:, cols] ----------------
    const int rg = ct % G::RG;
    const int gc = ct / G::RG;
    T* __restrict__ Y = static_cast<T*>(pr.Y);
    const int nB = (job.nc + G::NTC - 1) / G::NTC;
    for (int tb = 0; tb < nB; ++tb, ++it) {
        const int col_in_tile = gc * 8;
        const int nct = min(G::NTC, job.nc - tb * G::NTC);
        const bool active = gc < G::GC && col_in_tile < nct;
        const uint32_t stage = it % kFusedStages;
        mbar_wait<false>(&S.full[stage], (it / kFusedStages) & 1u, P.dev_status, dead);
        const unsigned char* st = S.ring + size_t(stage) * G::STAGE;
        float o[NTOK][8];
#pragma unroll
        for (int t = 0; t < NTOK; ++t)
#pragma unroll
            for (int i = 0; i < 8; ++i) o[t][i] = 0.f;
        if (active) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int j = rg + G::RG * jj;
                float b[8];
                unpack8<T>(*reinterpret_cast<const uint4*>(st + size_t(j) * G::BPITCH + col_in_tile * 2), b);
#pragma unroll
                for (int t = 0; t < NTOK; ++t) {
                    if (t < nt) {
                        const float v = S.vs[t * R + j];
#pragma unroll
                        for (int i = 0; i < 8; ++i) o[t][i] = fmaf(v, b[i], o[t][i]);
                    }
                }
            }
        }
#pragma unroll
        for (int off = 1; off < G::RG; off <<= 1)
#pragma unroll
            for (int t = 0; t < NTOK; ++t)
#pragma unroll
                for (int i = 0; i < 8; ++i) o[t][i] += __shfl_xor_sync(0xffffffffu, o[t][i], off);
        if (active && rg == 0) {
            const T* ys = reinterpret_cast<const T*>(st + size_t(R) * G::BPITCH);
            const int col = job.c0 + tb * G::NTC + col_in_tile;
#pragma unroll
            for (int t = 0; t < NTOK; ++t) {
                if (t < nt) {
                    float y[8];
                    unpack8<T>(*reinterpret_cast<const uint4*>(ys + size_t(t) * G::NTC + col_in_tile), y);
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = __fadd_rn(y[i], __fmul_rn(pr.scale, o[t][i]));
                    st_vec(Y + size_t(job.t0 + t) * pr.H2 + col, pack8<T>(y));
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&S.empty[stage]);
    }
}

// X columns of the first job's shrink stages (stages 0 .. tiles-1), requested once the
// previous kernel on the stream has completed.
template <typename T, int R, int CH>
__device__ __forceinline__ void issue_deferred_x(unsigned char* ring, uint64_t* full, const void* Xv, int H1, int t0,
                                                 int nt, int k0, int KT, int nk, int tiles, int lane) {
    using G = FusedGeom<R, CH>;
    const T* X = static_cast<const T*>(Xv);
    for (int ta = 0; ta < tiles; ++ta) {
        unsigned char* st = ring + size_t(ta) * G::STAGE;
        const int k = k0 + ta * KT;
        const int kt = min(KT, nk - ta * KT);
        if (lane >= 1 && lane <= nt)
            bulk_g2s(st + size_t(KT) * R * 2 + size_t(lane - 1) * KT * 2, X + size_t(t0 + lane - 1) * H1 + k,
                     uint32_t(kt) * 2, &full[ta]);
    }
}

// Producer side of one job: shrink stages (A rows + X columns), then expand stages (B rows + Y rows).
template <typename T, int R, int CH>
__device__ __forceinline__ void produce_job(const FusedParams& P, const Job& job, unsigned char* smem, uint64_t* full,
                                            uint64_t* empty, uint32_t& it, bool& waited, int lane, bool& dead) {
    using G = FusedGeom<R, CH>;
    const FusedProblem& pr = P.prob[job.p];
    const T* X = static_cast<const T*>(pr.X);
    const T* Yg = static_cast<const T*>(pr.Y);
    const T* A = static_cast<const T*>(job.a);
    const T* B = static_cast<const T*>(job.b);
    const int KT = G::kt_for(job.nt);
    const int nA = (job.nk + KT - 1) / KT;
    int deferred = 0;  // shrink stages of the first job whose X waits for the previous kernel
    for (int ta = 0; ta < nA; ++ta, ++it) {
        const uint32_t stage = it % kFusedStages;
        if (it >= kFusedStages) {
            if (!waited) {  // the ring is full: the deferred X must come first
                pdl_wait();
                waited = true;
                issue_deferred_x<T, R, CH>(smem, full, X, pr.H1, job.t0, job.nt, job.k0, KT, job.nk, deferred, lane);
            }
            mbar_wait<false>(&empty[stage], ((it / kFusedStages) - 1) & 1u, P.dev_status, dead);
        }
        unsigned char* st = smem + size_t(stage) * G::STAGE;
        const int k = job.k0 + ta * KT;
        const int kt = min(KT, job.nk - ta * KT);
        if (lane == 0) mbar_arrive_expect_tx(&full[stage], uint32_t(kt) * (R + job.nt) * 2);
        __syncwarp();
        if (lane == 0) bulk_g2s(st, A + size_t(k) * R, uint32_t(kt) * R * 2, &full[stage]);
        if (waited) {
            if (lane >= 1 && lane <= job.nt)
                bulk_g2s(st + size_t(KT) * R * 2 + size_t(lane - 1) * KT * 2,
                         X + size_t(job.t0 + lane - 1) * pr.H1 + k, uint32_t(kt) * 2, &full[stage]);
        } else {
            deferred = ta + 1;
        }
        if (ta == min(nA, kFusedStages) - 1 && job.nc > 0) {
            // start B on its way to L2 while the shrink runs, once the ring's first round of A
            // copies is queued ahead of the prefetches; the expand stages then hit L2
            for (int row = lane; row < R; row += 32)
                bulk_prefetch_l2(B + size_t(row) * pr.H2 + job.c0, uint32_t(job.nc) * 2);
        }
    }
    if (!waited) {
        pdl_wait();
        waited = true;
        issue_deferred_x<T, R, CH>(smem, full, X, pr.H1, job.t0, job.nt, job.k0, KT, job.nk, deferred, lane);
    }
    if (job.nc > 0 && lane < job.nt) bulk_prefetch_l2(Yg + size_t(job.t0 + lane) * pr.H2 + job.c0, uint32_t(job.nc) * 2);
    const int nB = (job.nc + G::NTC - 1) / G::NTC;
    for (int tb = 0; tb < nB; ++tb, ++it) {
        const uint32_t stage = it % kFusedStages;
        if (it >= kFusedStages) mbar_wait<false>(&empty[stage], ((it / kFusedStages) - 1) & 1u, P.dev_status, dead);
        unsigned char* st = smem + size_t(stage) * G::STAGE;
        const int col = job.c0 + tb * G::NTC;
        const int nct = min(G::NTC, job.nc - tb * G::NTC);
        if (lane == 0) mbar_arrive_expect_tx(&full[stage], uint32_t(nct) * (R + job.nt) * 2);
        __syncwarp();
        for (int row = lane; row < R + job.nt; row += 32) {
            if (row < R)
                bulk_g2s(st + size_t(row) * G::BPITCH, B + size_t(row) * pr.H2 + col, uint32_t(nct) * 2, &full[stage]);
            else
                bulk_g2s(st + size_t(R) * G::BPITCH + size_t(row - R) * G::NTC * 2,
                         Yg + size_t(job.t0 + row - R) * pr.H2 + col, uint32_t(nct) * 2, &full[stage]);
        }
    }
}

// ---- the kernel ----------------------------------------------------------------------------

// grid.x = C * clusters, cluster (C,1,1), C in {1,2,4,8}. Warp 0 produces, warps 1..4 consume.
// CH: tokens per job (8, or 4 for calls with long segments, whose jobs then carry half the Y
// rows and expand work each and spread over twice as many clusters).
template <typename T, int R, int CH = kFusedTokens>
__global__ void __launch_bounds__(kFusedThreads, SGMV_FUSED_MIN_BLOCKS) sgmv_fused_kernel(const FusedParams P) {
    using G = FusedGeom<R, CH>;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kFusedStages];
    __shared__ __align__(8) uint64_t empty[kFusedStages];
    __shared__ __align__(8) uint64_t vready[1];
    __shared__ __align__(8) uint64_t vfree[1];

    FusedSmem S;
    S.ring = smem;
    S.red = reinterpret_cast<float*>(smem + G::RING);
    S.recv = reinterpret_cast<float*>(smem + G::RING + G::RED);
    S.vs = reinterpret_cast<float*>(smem + G::RING + G::RED + G::RECV);
    int* pref = reinterpret_cast<int*>(smem + G::BASE);
    S.full = full;
    S.empty = empty;
    S.vready = vready;
    S.vfree = vfree;

    const int C = static_cast<int>(cluster_size());
    const int c = static_cast<int>(cluster_rank());
    const int cluster_id = blockIdx.x / C;
    const int n_clusters = gridDim.x / C;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // the next kernel on the stream may start its prologue now (programmatic dependent launch)
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kFusedStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kFusedConsumerWarps);
        }
        mbar_init(vready, 1);  // own expect_tx arrival; the C tiles arrive as transaction bytes
        mbar_init(vfree, C);   // one arrival per receiver
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // nothing the caller passed is read before the previous kernel completes, unless the
    // caller allows the early reads (the metadata is only prefetched into L2 before)
    if (!P.early) {
        prefetch_metadata(P);
        pdl_wait();
    }
    int entries;
    if (P.one_chunk) {
        __syncthreads();
        entries = P.n_problems * P.n_segments;
    } else {
        build_job_prefix<CH>(P, pref);  // ends with __syncthreads
        entries = P.n_problems * pref[P.n_segments];
    }
    // Barriers of every CTA exist before any remote operation: each CTA arrives here and
    // waits only before its first remote operation (consumers, below).
    if (C > 1) cluster_arrive();

    bool dead = false;
    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        // With early reads allowed, adapter weights and segment metadata are not written by the
        // previous kernel on the stream, so the first job's A rows are requested before
        // griddepcontrol.wait; X and Y (which the previous kernel may produce) only after it.
        uint32_t it = 0;
        bool waited = !P.early;
        for (int j = cluster_id; j < entries; j += n_clusters) {
            int p, s, q_begin, q_end;
            if (P.one_chunk) {
                p = j / P.n_segments;
                s = j - p * P.n_segments;
                Job job;
                q_end = first_job_warp<CH>(P, p, s, c, lane, job);
                if (q_end > 0) produce_job<T, R, CH>(P, job, smem, full, empty, it, waited, lane, dead);
                q_begin = 1;  // any further chunk (a longest-segment hint below the truth) as below
            } else {
                int q0, nq;
                entry_at<CH>(P, pref, j, p, s, q0, nq);
                q_begin = q0;
                q_end = q0 + nq;
            }
            for (int q = q_begin; q < q_end; ++q) {
                Job job;
                if (!job_at<CH>(P, p, s, q, c, job)) break;
                produce_job<T, R, CH>(P, job, smem, full, empty, it, waited, lane, dead);
            }
        }
        if (!waited) pdl_wait();
        if (C > 1) cluster_wait();
    } else {
        // ------------------------------ consumers ------------------------------
        if (C > 1) cluster_wait();
        const int ct = threadIdx.x - 32;
        // rejected segments are reported as the jobs meet them (no pass over the segments at
        // the end, which the next kernel on the stream would wait for)
        const bool reporter = c == 0 && ct == 0;
        uint32_t it = 0, u = 0;
        for (int j = cluster_id; j < entries; j += n_clusters) {
            int p, s, q0, nq;
            entry_at<CH>(P, pref, j, p, s, q0, nq);
            if (nq == 0 && reporter) report(P.dev_status, segment_bounds_check(P, s));
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at_reporting<CH>(P, p, s, q, c, job, reporter)) break;
                if (job.nt == 1)
                    consume_job<T, R, 1, CH>(P, job, S, it, u, C, c, ct, dead);
                else if (job.nt <= 2)
                    consume_job<T, R, 2, CH>(P, job, S, it, u, C, c, ct, dead);
                else if (CH == 4 || job.nt <= 4)
                    consume_job<T, R, 4, CH>(P, job, S, it, u, C, c, ct, dead);
                else
                    consume_job<T, R, (CH > 4 ? 8 : 4), CH>(P, job, S, it, u, C, c, ct, dead);
                ++u;
            }
        }
        // keep this grid behind its predecessor even when it had no work
        pdl_wait();
        // every receiver has consumed this CTA's last tile before its shared memory goes away
        if (u >= 1) mbar_wait<true>(vfree, (u - 1) & 1u, P.dev_status, dead);
    }
}

}  // namespace sgmv

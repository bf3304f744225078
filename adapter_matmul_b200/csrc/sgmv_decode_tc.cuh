// sgmv_decode_tc.cuh -- one-kernel SGMV on tcgen05 for decode batches, with every tile moved
// by the tensor memory accelerator in copies of 8-16 KB.
//
// Maths (page "Punica：多 LoRA 模型统一服务框架", the Punica README, its LoRA and
// multi-LoRA paragraphs): Y[t,:] += scale * (X[t,:] @ A_i) @ B_i for the rows t of each
// segment, A_i [H1, r], B_i [r, H2], row-major.
//
// Jobs and the cluster split are those of the fused kernel (sgmv_fused.cuh), with chunks of
// 16 tokens: a cluster of C CTAs runs a job (projection, segment, chunk); CTA c owns a
// K-slice of A_i and an N-slice of B_i.
//
//   shrink   D1[128 x r] (TMEM) = X_chunk[128 x K] @ A_i[K x r] over the CTA's K-slice, in
//            stages of KS rows of A_i; tcgen05.mma M=128 N=r. Only the chunk's first 16 rows
//            of X are loaded; the MMA's other rows read whatever follows in the same stage
//            and their results are never read back;
//   V        the partial D1 rows of the chunk leave TMEM (tcgen05.ld), are pushed to every
//            CTA of the cluster with st.async and summed in rank order; V (fp32) is written
//            as the two 16-bit operands V_hi + V_lo (about 16 significant bits of V);
//   expand   transposed, so that the MMA's N is the token count: for each 128-column group
//            of a stage, D2^T[128 cols x 32] = B_tile^T[128 x r] @ [V_hi^T | V_lo^T][r x 32],
//            M=128 N=32, the B tile as an MN-major operand, V_hi and V_lo side by side so one
//            MMA covers both; up to four D2 buffers in TMEM; the epilogue adds the two halves,
//            adds scale * D2 to the staged Y rows, rounds once and stores them.
//
// Copies. A TMA copy has a fixed cost per instruction that dominates until the copy is
// several KB long, so every stage is one or two instructions:
//   A_i  one box of KS rows x r (contiguous bytes; swizzle = the row width),
//   X    one 3-D box {64 columns, 16 rows, KS/64 column blocks} of a view of X whose third
//        dimension steps 128 bytes, landing as KS/64 swizzled K-major blocks of 16 rows,
//   B_i  one 3-D box {64 columns, r rows, NB column blocks}, landing as NB MN-major blocks,
//   Y    exact 2-D boxes of 16, 8, 4, 2 and 1 rows (the binary digits of the chunk length,
//        so no row of another segment is read or written).
// A_i and B_i come from a device table, so their tensor maps are made on the device from a
// template per problem (sgmv_tmap.cuh); X and Y maps are made on the host per call.
//
// Rings: X + A_i (shrink) and B_i (expand) stages share one ring that the MMA frees as soon
// as its reads are done; Y stages have their own ring, freed by the epilogue, so the stream of
// adapter bytes never waits on the epilogue's latency. D2 has up to four TMEM buffers.
//
// Warps: 0 producer of X, A_i and B_i, 1 TMEM owner and MMA issuer, 2..9 epilogue (two per
// TMEM lane quarter, each taking every other 128-column group of a stage; one of them also
// runs the V exchange), 10 producer of Y. Programmatic dependent launch: X and Y are read only after
// griddepcontrol.wait; so are the segment arrays, tables and adapters unless the caller allows
// reading them earlier (P.early) or the kernel runs in pre-V mode. Every wait is bounded in time.
//
// Pre-V mode (template flag PRE_V, the split form): V [T, r] (fp32) comes from an earlier
// kernel (the split-K shrink) through global memory. There is no shrink and no cluster: each
// job's H2 is cut into n_slices slices, every (job, slice) pair is a unit of work, and the
// CTAs (independent, one per SM) take the units round-robin, so that a few large adapters
// still spread over every SM. A unit reads its chunk's V rows after griddepcontrol.wait and
// runs the same expand pipeline over its slice.
#pragma once

#include "sgmv_grouped_tc.cuh"

namespace sgmv {

constexpr int kDTokens = 16;    // tokens per job = N of the expand MMA
constexpr int kDYStages = 4;    // Y ring, freed by the epilogue
constexpr int kDThreads = 352;  // producer, MMA issuer, 8 epilogue warps, Y producer
constexpr int kDEpiWarps = 8;   // two per TMEM lane quarter, splitting each stage's 128-column groups
constexpr int kDTmemCols = 512;  // D1 at [0, r), D2 buffers from column 64 (one CTA per SM)
constexpr int kDYMaps = 5;       // Y boxes of 1, 2, 4, 8 and 16 rows
constexpr int kDEpiBatch = 2;    // expand stages per epilogue pass

struct DecodeMaps {
    CUtensorMap x[kFusedMaxProblems];           // X view {64, T, H1/64}, box {64, 16, KS/64}, 128B swizzle
    CUtensorMap y[kFusedMaxProblems][kDYMaps];  // Y {H2, T}, box {YW, 2^i rows}, no swizzle
    CUtensorMap a[kFusedMaxProblems];           // template of A_i {r, H1}, box {r, KS}, swizzle = 2r bytes
    CUtensorMap b[kFusedMaxProblems];           // template of B_i view {64, r, H2/64}, box {64, r, NB}, 128B
};

__host__ __device__ constexpr int round1024(int v) { return (v + 1023) / 1024 * 1024; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int R, bool PRE_V = false>
struct DecodeTCGeom {
    static constexpr int KS = R == 16 ? 256 : 128;        // rows of A_i per shrink stage
    static constexpr int A_BYTES = KS * R * 2;            // 16, 8, 8 KB (r = 64, 32, 16)
    static constexpr int XB = KS / 64;                    // X column blocks per shrink stage
    static constexpr int X_BYTES = XB * kDTokens * 128;   // 16 rows per block
    // 64-column blocks of B_i per expand stage: a stage carries 32 KB of B_i at r = 64, 16 KB
    // otherwise (the per-stage costs of the MMA and the epilogue are paid per stage). With V
    // precomputed the ring holds B_i alone, and at r = 64 it takes two 64 KB stages of 512
    // columns: the same bytes in flight as four 32 KB stages, half the per-stage costs (the
    // fused form keeps 32 KB, since its shrink stages would leave most of a 64 KB slot unused).
    static constexpr bool WIDE = PRE_V && R == 64;
    static constexpr int NB = (WIDE ? 65536 : (R == 64 ? 32768 : 16384)) / (R * 128);
    static constexpr int NW = NB * 64;                    // columns per expand stage: 256 (512 wide), 256, 512
    static constexpr int B_BYTES = R * NW * 2;            // 32 (64 wide), 16, 16 KB
    static constexpr int STAGES = WIDE ? 2 : (R == 64 ? 4 : 6);  // main ring depth
    static constexpr int YW = NW < 256 ? NW : 256;        // Y box width
    static constexpr int YBOXES = NW / YW;
    static constexpr int Y_BYTES = round1024(kDTokens * NW * 2);  // one Y stage: [YBOXES][16 rows][YW]
    static constexpr int STAGE = round1024(cmax(X_BYTES + A_BYTES, B_BYTES));
    static constexpr int VT_BYTES = round1024(2 * kDTokens * R * 2);  // V^T: 16 rows of V_hi, then 16 of V_lo
    static constexpr int TILE = kDTokens * R * 4;                 // one partial V tile (fp32)
    static constexpr size_t BASE =
        size_t(STAGES) * STAGE + size_t(kDYStages) * Y_BYTES + size_t(VT_BYTES);  // + C tiles + prefix
    static constexpr int SW_BITS = R == 64 ? 3 : (R == 32 ? 2 : 1);
    static constexpr uint64_t SW_TYPE = R == 64 ? 2 : (R == 32 ? 4 : 6);
    static constexpr int ROW_BYTES = R * 2;
    static constexpr int D2_COLS = NB * 16;  // (NB / 2) groups x (16 tokens x hi, lo)
    static constexpr int ND2 = (kDTmemCols - 64) / D2_COLS < 4 ? (kDTmemCols - 64) / D2_COLS : 4;  // D2 buffers
    static_assert(ND2 >= 2, "TMEM holds fewer than two D2 buffers");
    // all 512 TMEM columns are allocated, so two CTAs must never share an SM: the shared
    // memory of one CTA rules out a second (an SM has 228 KB)
    static_assert(2 * BASE > 228 * 1024, "two CTAs could share an SM and wait on each other's TMEM");
    // the shrink MMA reads 128 rows (16 KB) from each X block (rows past the 16 loaded ones are
    // never used); from the last stage that span runs into the Y ring, still inside the allocation
    static_assert((XB - 1) * 2048 + 16384 <= STAGE + kDYStages * Y_BYTES, "X operand span leaves the allocation");
};

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// R consecutive fp32 columns of this thread's TMEM lane (R in 16, 32, 64).
template <int R>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&v)[R]) {
#pragma unroll
    for (int c0 = 0; c0 < R; c0 += 16) {
        float w[16];
        tmem_ld16(taddr + c0, w);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[c0 + i] = w[i];
    }
}

// TMA store of a 2-D box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N bulk groups of this thread still read their shared-memory source
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// wait until at most N bulk groups of this thread are still in flight (writes done)
template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// The rows [t0, t0 + nt) of a chunk are moved as boxes of 16, 8, 4, 2 and 1 rows (the binary
// digits of nt), so Y rows of other segments are never read or written. Box m (rows 2^m) of
// a chunk starts at row offset nt & ~(2^(m+1) - 1).


template <typename T, int R, bool PRE_V>
__global__ void __launch_bounds__(kDThreads, 1)
    sgmv_decode_tc_kernel(const __grid_constant__ DecodeMaps maps, const FusedParams P, const float* v_in,
                          int n_slices) {
    using G = DecodeTCGeom<R, PRE_V>;
    constexpr int S = G::STAGES;
    constexpr int SY = kDYStages;
    constexpr int ND2 = G::ND2;
    extern __shared__ __align__(1024) unsigned char dsm_raw[];
    unsigned char* dsm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    // PRE_V false: a cluster of C CTAs splits each job's K (shrink, V exchanged on chip) and
    // N, and the clusters walk the entries (v_in and n_slices unused). PRE_V true: V [T, r]
    // (fp32, v_in) was computed by an earlier kernel and the shrink is skipped; each entry's N is
    // cut into n_slices slices and every (entry, slice) pair is a unit of work, walked by
    // independent CTAs (no cluster).
    constexpr bool pre_v = PRE_V;
    const int C = pre_v ? 1 : static_cast<int>(cluster_size());
    const int c = pre_v ? 0 : static_cast<int>(cluster_rank());
    const int n_sl = pre_v ? n_slices : 1;
    unsigned char* ring = dsm;
    unsigned char* yring = ring + S * G::STAGE;
    unsigned char* vt = yring + SY * G::Y_BYTES;                  // V^T operand: [V_hi rows | V_lo rows]
    float* recv = reinterpret_cast<float*>(vt + G::VT_BYTES);  // C partial V tiles
    int* pref = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(recv) + size_t(C) * G::TILE);

    __shared__ __align__(8) uint64_t full[S], empty[S], yfull[SY], yempty[SY];
    __shared__ __align__(8) uint64_t d1_full, v_full, d2_full[ND2], d2_empty[ND2], vready, vfree;
    __shared__ __align__(128) CUtensorMap map_build[2];  // A and B maps of the next job
    __shared__ uint32_t tmem_base_s;
    __shared__ int table_s;

    const int cluster_id = blockIdx.x / C;  // in pre-V mode: the CTA
    const int n_clusters = gridDim.x / C;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);   // producer lane 0 (expect_tx); the copies complete the bytes
            mbar_init(&empty[i], 1);  // MMA commit
        }
        for (int i = 0; i < SY; ++i) {
            mbar_init(&yfull[i], 1);
            mbar_init(&yempty[i], kDEpiWarps);
        }
        mbar_init(&d1_full, 1);
        mbar_init(&v_full, 1);
        for (int i = 0; i < ND2; ++i) {
            mbar_init(&d2_full[i], 1);
            mbar_init(&d2_empty[i], kDEpiWarps);
        }
        mbar_init(&vready, 1);  // own expect_tx; the C tiles arrive as transaction bytes
        mbar_init(&vfree, C);   // one arrival per receiver
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        table_s = claim_map_table();
        if (table_s < 0) report(P.dev_status, LORA_SGMV_DEV_TIMEOUT);
    }
    // Early reads (segment arrays, tables, adapters before the previous kernel completes) only
    // where allowed: asked for by the caller, or in pre-V mode, whose previous kernel is this
    // library's shrink, which writes none of them.
    const bool early = pre_v || P.early;
    if (!early) {
        prefetch_metadata(P);  // L2 only: no value is read before the wait
        pdl_wait();
    }
    int entries;
    if (P.one_chunk) {
        __syncthreads();
        entries = P.n_problems * P.n_segments;
    } else {
        build_job_prefix<kDTokens>(P, pref);
        entries = P.n_problems * pref[P.n_segments];
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kDTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (C > 1) cluster_arrive();
    const uint32_t tmem = tmem_base_s;
    const int table = table_s;
    if (table < 0) entries = 0;
    bool dead = false;

    if (warp == 0) {
        // ---------------------------------- producer ----------------------------------
        MapTable* tab = g_map_tables + (table < 0 ? 0 : table);
        uint32_t it = 0;
        int last_use[kMapRing];
#pragma unroll
        for (int e = 0; e < kMapRing; ++e) last_use[e] = -1;
        int jc = 0;
        // X is read only after the wait; in pre-V mode there is no X to read, so the producer
        // never waits and B_i streams while the shrink kernel finishes
        bool waited = !early || pre_v;
        int deferred = 0;  // shrink stages of the first job still missing their X box
        int d_p = 0, d_t0 = 0, d_k0 = 0;
        auto flush_deferred = [&]() {
            if (lane == 0)
                for (int d = 0; d < deferred; ++d)
                    tma_load_3d(ring + d * G::STAGE, &maps.x[d_p], 0, d_t0, (d_k0 + d * G::KS) / 64, &full[d]);
            deferred = 0;
            __syncwarp();
        };
        for (int w = cluster_id; w < entries * n_sl; w += n_clusters) {
            const int j = pre_v ? w / n_sl : w;
            const int cw = pre_v ? w - j * n_sl : c;  // N slice (and K slice)
            int p, s, q0, nq;
            entry_at<kDTokens>(P, pref, j, p, s, q0, nq);
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at<kDTokens>(P, p, s, q, cw, job)) break;
                const int nA = (job.nk + G::KS - 1) / G::KS;
                const int nB = (job.nc + G::NW - 1) / G::NW;
                if (nA + nB == 0) continue;
                // maps of this job's adapter go to ring entry e; the copies of the entry's
                // previous job must have been consumed before it is rewritten
                const int e = jc % kMapRing;
                ++jc;
                const int lu = last_use[e];
                if (lu >= 0 && lu >= static_cast<int>(it) - S)
                    mbar_wait<false>(&empty[lu % S], (uint32_t(lu) / S) & 1u, P.dev_status, dead);
                CUtensorMap* gA = &tab->m[2 * e];
                CUtensorMap* gB = &tab->m[2 * e + 1];
                map_template_to_smem(&map_build[0], &maps.a[job.p]);
                map_template_to_smem(&map_build[1], &maps.b[job.p]);
                if (lane == 0) {
                    map_set_address(&map_build[0], job.a);
                    map_set_address(&map_build[1], job.b);
                }
                __syncwarp();
                map_publish(gA, &map_build[0]);
                map_publish(gB, &map_build[1]);
                if (lane == 0) {
                    map_acquire(gA);
                    map_acquire(gB);
                }
                __syncwarp();

                for (int ta = 0; ta < nA; ++ta, ++it) {
                    const uint32_t st = it % S;
                    if (it >= S) {
                        if (!waited) {
                            pdl_wait();
                            waited = true;
                            flush_deferred();
                        }
                        mbar_wait<false>(&empty[st], ((it / S) - 1) & 1u, P.dev_status, dead);
                    }
                    unsigned char* xs = ring + st * G::STAGE;
                    const int kbase = job.k0 + ta * G::KS;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[st], G::X_BYTES + G::A_BYTES);
                        tma_load_2d(xs + G::X_BYTES, gA, 0, kbase, &full[st]);
                        if (waited) tma_load_3d(xs, &maps.x[job.p], 0, job.t0, kbase / 64, &full[st]);
                    }
                    if (!waited) {
                        deferred = ta + 1;
                        d_p = job.p;
                        d_t0 = job.t0;
                        d_k0 = job.k0;
                    }
                    __syncwarp();
                }
                if (!waited) {
                    pdl_wait();
                    waited = true;
                    flush_deferred();
                }
                for (int tb = 0; tb < nB; ++tb, ++it) {
                    const uint32_t st = it % S;
                    if (it >= S) mbar_wait<false>(&empty[st], ((it / S) - 1) & 1u, P.dev_status, dead);
                    unsigned char* bs = ring + st * G::STAGE;
                    const int n0 = job.c0 + tb * G::NW;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[st], G::B_BYTES);
                        tma_load_3d(bs, gB, 0, 0, n0 / 64, &full[st]);
                    }
                    __syncwarp();
                }
                last_use[e] = static_cast<int>(it) - 1;
            }
        }
        if (!waited) pdl_wait();
        // every copy issued lands before the CTA may exit (pre-V mode: the epilogue's and the Y
        // producer's waits keep this grid behind the shrink)
        if (lane == 0)
            for (uint32_t i = it > uint32_t(S) ? it - S : 0u; i < it; ++i) drain_wait(&full[i % S], (i / S) & 1u);
        __syncwarp();
        if (C > 1) cluster_wait();
    } else if (warp == 10) {
        // --------------------------------- Y producer ---------------------------------
        // Y rows of each expand stage, through their own ring, so that the adapter stream
        // above never waits for the epilogue
        pdl_wait();
        uint32_t yit = 0;
        for (int w = cluster_id; w < entries * n_sl; w += n_clusters) {
            const int j = pre_v ? w / n_sl : w;
            const int cw = pre_v ? w - j * n_sl : c;  // N slice (and K slice)
            int p, s, q0, nq;
            entry_at<kDTokens>(P, pref, j, p, s, q0, nq);
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at<kDTokens>(P, p, s, q, cw, job)) break;
                const int nB = (job.nc + G::NW - 1) / G::NW;
                for (int tb = 0; tb < nB; ++tb, ++yit) {
                    const uint32_t sy = yit % SY;
                    if (yit >= SY) mbar_wait<false>(&yempty[sy], ((yit / SY) - 1) & 1u, P.dev_status, dead);
                    unsigned char* ys = yring + sy * G::Y_BYTES;
                    const int n0 = job.c0 + tb * G::NW;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&yfull[sy], G::YBOXES * job.nt * G::YW * 2);
                        for (int m = 4; m >= 0; --m) {
                            if (!(job.nt & (1 << m))) continue;
                            const int r0 = job.nt & ~((2 << m) - 1);
#pragma unroll
                            for (int k = 0; k < G::YBOXES; ++k)
                                tma_load_2d(ys + (k * kDTokens + r0) * G::YW * 2, &maps.y[job.p][m], n0 + k * G::YW,
                                            job.t0 + r0, &yfull[sy]);
                        }
                    }
                    __syncwarp();
                }
            }
        }
        if (lane == 0)
            for (uint32_t i = yit > uint32_t(SY) ? yit - SY : 0u; i < yit; ++i) drain_wait(&yfull[i % SY], (i / SY) & 1u);
        __syncwarp();
        if (C > 1) cluster_wait();
    } else if (warp == 1) {
        // ---------------------------------- MMA issuer ----------------------------------
        const uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
        const uint32_t idesc_s = instr_desc(fmt, 0, 1, R, kGM);         // X K-major, A_i MN-major, N = r
        // B tile MN-major, V^T K-major with N = 32: columns 0..15 of D2 take V_hi, 16..31 V_lo
        const uint32_t idesc_e = instr_desc(fmt, 1, 0, 2 * kDTokens, kGM);
        uint32_t it = 0, u = 0, g = 0;
        for (int w = cluster_id; w < entries * n_sl; w += n_clusters) {
            const int j = pre_v ? w / n_sl : w;
            const int cw = pre_v ? w - j * n_sl : c;  // N slice (and K slice)
            int p, s, q0, nq;
            entry_at<kDTokens>(P, pref, j, p, s, q0, nq);
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at<kDTokens>(P, p, s, q, cw, job)) break;
                const int nA = (job.nk + G::KS - 1) / G::KS;
                const int nB = (job.nc + G::NW - 1) / G::NW;
                for (int ta = 0; ta < nA; ++ta, ++it) {
                    const uint32_t st = it % S;
                    mbar_wait<false>(&full[st], (it / S) & 1u, P.dev_status, dead);
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t xa = smem_u32(ring + st * G::STAGE);
                        const uint32_t aa = xa + G::X_BYTES;
#pragma unroll
                        for (int kb = 0; kb < G::XB; ++kb)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t adesc = smem_desc(xa + kb * 2048 + kk * 32, 16, 1024, 2);
                                const uint64_t bdesc = smem_desc(aa + (kb * 64 + kk * 16) * G::ROW_BYTES,
                                                                 16 * G::ROW_BYTES, 8 * G::ROW_BYTES, G::SW_TYPE);
                                tc_mma(tmem, adesc, bdesc, idesc_s, (ta | kb | kk) ? 1u : 0u);
                            }
                        tc_commit(&empty[st]);
                    }
                    __syncwarp();
                }
                // (with no K rows here no shrink MMA ran; the epilogue then uses zeros for D1)
                if (lane == 0) tc_commit(&d1_full);
                __syncwarp();
                mbar_wait<false>(&v_full, u & 1u, P.dev_status, dead);
                tc_fence_after();
                for (int tb = 0; tb < nB; ++tb, ++it, ++g) {
                    const uint32_t st = it % S;
                    const uint32_t buf = g % ND2;
                    if (g >= uint32_t(ND2))
                        mbar_wait<false>(&d2_empty[buf], ((g / ND2) - 1) & 1u, P.dev_status, dead);
                    mbar_wait<false>(&full[st], (it / S) & 1u, P.dev_status, dead);
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t ba = smem_u32(ring + st * G::STAGE);
                        const uint32_t d2 = tmem + 64u + uint32_t(G::D2_COLS) * buf;
#pragma unroll
                        for (int gi = 0; gi < G::NB / 2; ++gi)
#pragma unroll
                            for (int kk = 0; kk < R / 16; ++kk) {
                                const uint64_t adesc = smem_desc(ba + 2 * gi * R * 128 + kk * 16 * 128, R * 128, 1024, 2);
                                const uint64_t bdesc =
                                    smem_desc(smem_u32(vt) + kk * 32, 16, 8 * G::ROW_BYTES, G::SW_TYPE);
                                tc_mma(d2 + 32u * gi, adesc, bdesc, idesc_e, kk ? 1u : 0u);
                            }
                        tc_commit(&d2_full[buf]);
                        tc_commit(&empty[st]);
                    }
                    __syncwarp();
                }
                ++u;
            }
        }
        if (C > 1) cluster_wait();
    } else {
        // ------------------------------ exchange and epilogue ------------------------------
        const int quarter = warp & 3;      // TMEM lanes [32*quarter, 32*quarter + 32)
        const int half = (warp - 2) >> 2;  // 128-column groups half, half + 2, ... of each stage
        const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
        if (C > 1) cluster_wait();
        uint32_t yit = 0, u = 0, g = 0;
        for (int w = cluster_id; w < entries * n_sl; w += n_clusters) {
            const int j = pre_v ? w / n_sl : w;
            const int cw = pre_v ? w - j * n_sl : c;  // N slice (and K slice)
            int p, s, q0, nq;
            entry_at<kDTokens>(P, pref, j, p, s, q0, nq);
            // rejected segments are reported as the jobs meet them: one thread of the first CTA
            // of the visiting cluster (of the first N slice in pre-V mode)
            const bool reporter = c == 0 && cw == 0 && warp == 9 && lane == 0;
            if (nq == 0 && reporter) report(P.dev_status, segment_bounds_check(P, s));
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at_reporting<kDTokens>(P, p, s, q, cw, job, reporter)) break;
                const FusedProblem& pr = P.prob[job.p];
                const int nA = (job.nk + G::KS - 1) / G::KS;
                const int nB = (job.nc + G::NW - 1) / G::NW;
                if (quarter == 0 && half == 0) {
                    // partial V of this CTA: D1 rows 0..nt-1 (lanes 0..15 of quarter 0)
                    mbar_wait<false>(&d1_full, u & 1u, P.dev_status, dead);
                    tc_fence_after();
                    // V^T operand rows: token `lane`, 8 values of chunk ch, K-major swizzled; hi + lo
                    auto put_v8 = [&](int ch, const float* x8) {
                        float hi[8], lo[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            hi[i] = Storage<T>::round(x8[i]);
                            lo[i] = x8[i] - hi[i];
                        }
                        st_vec(vt + swz(lane, ch, G::SW_BITS), pack8<T>(hi));
                        st_vec(vt + swz(kDTokens + lane, ch, G::SW_BITS), pack8<T>(lo));
                    };
                    if (pre_v) {
                        // V rows of the chunk from the earlier kernel (read once it has completed);
                        // rows past the chunk are V^T columns of zeros
                        pdl_wait();
                        if (lane < kDTokens) {
                            const float4* src = reinterpret_cast<const float4*>(v_in + size_t(job.t0 + lane) * R);
#pragma unroll
                            for (int ch = 0; ch < R / 8; ++ch) {
                                float x8[8];
                                const float4 a = lane < job.nt ? src[2 * ch] : make_float4(0.f, 0.f, 0.f, 0.f);
                                const float4 b = lane < job.nt ? src[2 * ch + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
                                x8[0] = a.x, x8[1] = a.y, x8[2] = a.z, x8[3] = a.w;
                                x8[4] = b.x, x8[5] = b.y, x8[6] = b.z, x8[7] = b.w;
                                put_v8(ch, x8);
                            }
                        }
                    } else {
                        float v[R];
                        tmem_ld_row<R>(lane_base, v);
                        if (nA == 0) {
#pragma unroll
                            for (int i = 0; i < R; ++i) v[i] = 0.f;
                        }
                        const uint32_t tile_bytes = uint32_t(job.nt) * R * 4;
                        if (lane == 0) mbar_arrive_expect_tx(&vready, tile_bytes * C);
                        if (u >= 1) mbar_wait<true>(&vfree, (u - 1) & 1u, P.dev_status, dead);
                        if (lane < job.nt) {
                            float* slot = recv + (size_t(c) * kDTokens + lane) * R;
                            for (int qr = 0; qr < C; ++qr)
#pragma unroll
                                for (int i = 0; i < R; i += 4)
                                    st_async_v4(slot + i, make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]), &vready,
                                                qr);
                        }
                        mbar_wait<true>(&vready, u & 1u, P.dev_status, dead);
#pragma unroll
                        for (int i = 0; i < R; ++i) v[i] = 0.f;  // rows past the chunk: V^T columns of zeros
                        if (lane < job.nt) {
                            for (int qr = 0; qr < C; ++qr) {
                                const float* src = recv + (size_t(qr) * kDTokens + lane) * R;
#pragma unroll
                                for (int i = 0; i < R; ++i) v[i] += src[i];
                            }
                        }
                        if (lane < kDTokens) {
#pragma unroll
                            for (int ch = 0; ch < R / 8; ++ch) {
                                float hi[8], lo[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    hi[i] = Storage<T>::round(v[ch * 8 + i]);
                                    lo[i] = v[ch * 8 + i] - hi[i];
                                }
                                st_vec(vt + swz(lane, ch, G::SW_BITS), pack8<T>(hi));
                                st_vec(vt + swz(kDTokens + lane, ch, G::SW_BITS), pack8<T>(lo));
                            }
                        }
                    }
                    fence_proxy_async();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_local(&v_full);
                    if (!pre_v && lane < C) mbar_arrive_remote(&vfree, static_cast<uint32_t>(lane));
                }
                // expand epilogue: this warp's 32 columns of each 128-column group, all tokens,
                // kDEpiBatch stages per pass: whatever a pass waits for after its Y stores is paid
                // once per batch rather than once per stage
                T* __restrict__ Y = static_cast<T*>(pr.Y);
                const int n_hi = job.c0 + job.nc;
                for (int tb = 0; tb < nB; tb += kDEpiBatch) {
                    const int nb = min(kDEpiBatch, nB - tb);
                    for (int e = 0; e < nb; ++e) {
                        mbar_wait<false>(&yfull[(yit + e) % SY], ((yit + e) / SY) & 1u, P.dev_status, dead);
                        mbar_wait<false>(&d2_full[(g + e) % ND2], ((g + e) / ND2) & 1u, P.dev_status, dead);
                    }
                    tc_fence_after();
                    for (int e = 0; e < nb; ++e) {
                        const unsigned char* ys = yring + ((yit + e) % SY) * G::Y_BYTES;
                        const uint32_t d2 = lane_base + 64u + uint32_t(G::D2_COLS) * ((g + e) % ND2);
                        const int n0 = job.c0 + (tb + e) * G::NW;
                        for (int gi = half; gi < G::NB / 2; gi += 2) {
                            float acc[16], acc_lo[16];
                            tmem_ld16(d2 + 32u * gi, acc);
                            tmem_ld16(d2 + 32u * gi + 16u, acc_lo);
#pragma unroll
                            for (int t = 0; t < kDTokens; ++t) acc[t] += acc_lo[t];
                            const int cw = gi * 128 + quarter * 32 + lane;  // column within the stage
                            const int col = n0 + cw;
                            if (col < n_hi) {
                                const int kbox = cw / G::YW;
                                const T* yk =
                                    reinterpret_cast<const T*>(ys + kbox * kDTokens * G::YW * 2) + (cw - kbox * G::YW);
#pragma unroll
                                for (int t = 0; t < kDTokens; ++t) {
                                    if (t < job.nt) {
                                        const float y = Storage<T>::to1(yk[t * G::YW]);
                                        const float o = __fadd_rn(y, __fmul_rn(pr.scale, acc[t]));
                                        Y[size_t(job.t0 + t) * pr.H2 + col] = Storage<T>::from1(o);
                                    }
                                }
                            }
                        }
                    }
                    // the TMEM reads completed at tcgen05.wait::ld and the Y rows were read: release
                    __syncwarp();
                    if (lane == 0)
                        for (int e = 0; e < nb; ++e) {
                            mbar_arrive_relaxed(&d2_empty[(g + e) % ND2]);
                            mbar_arrive_relaxed(&yempty[(yit + e) % SY]);
                        }
                    yit += nb;
                    g += nb;
                }
                ++u;
            }
        }
        if (quarter == 0 && half == 0) {
            pdl_wait();
            if (!pre_v && u >= 1) mbar_wait<true>(&vfree, (u - 1) & 1u, P.dev_status, dead);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kDTmemCols) : "memory");
    if (threadIdx.x == 0) release_map_table(table);
}

// ---- host side ---------------------------------------------------------------------------

// Tiled tensor map of rank 2 or 3 over 16-bit elements (dims in elements and strides in
// bytes, innermost first; the innermost stride is the element size and is not passed).
inline bool encode_map(CUtensorMap* map, const void* base, lora_sgmv_dtype dt, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc || rank < 2 || rank > 3) return false;
    cuuint64_t gdim[3];
    cuuint64_t gstride[2];
    cuuint32_t bx[3];
    cuuint32_t es[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bx[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
    const CUresult r = enc(map, dt == LORA_SGMV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                           static_cast<cuuint32_t>(rank), const_cast<void*>(base), gdim, gstride, bx, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// All maps of problem p for the tensor-core decode kernel at rank R (H1, H2 multiples of 64),
// for the kernel's form PRE_V.
template <int R, bool PRE_V>
inline bool make_decode_maps(DecodeMaps& m, int p, const void* X, void* Y, int T, int H1, int H2, lora_sgmv_dtype dt) {
    using G = DecodeTCGeom<R, PRE_V>;
    {  // X view {64, T, H1/64}: element (k, t, b) at X + t*H1 + 64*b + k
        const uint64_t d[3] = {64, uint64_t(T), uint64_t(H1 / 64)};
        const uint64_t s[2] = {uint64_t(H1) * 2, 128};
        const uint32_t b[3] = {64, uint32_t(kDTokens), uint32_t(G::XB)};
        if (!encode_map(&m.x[p], X, dt, 3, d, s, b, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
    }
    const uint32_t rows[kDYMaps] = {1, 2, 4, 8, 16};
    for (int i = 0; i < kDYMaps; ++i) {  // Y {H2, T}
        const uint64_t d[2] = {uint64_t(H2), uint64_t(T)};
        const uint64_t s[1] = {uint64_t(H2) * 2};
        const uint32_t b[2] = {uint32_t(G::YW), rows[i]};
        if (!encode_map(&m.y[p][i], Y, dt, 2, d, s, b, CU_TENSOR_MAP_SWIZZLE_NONE)) return false;
    }
    {  // A_i template {R, H1}; the address is replaced on the device
        const uint64_t d[2] = {uint64_t(R), uint64_t(H1)};
        const uint64_t s[1] = {uint64_t(R) * 2};
        const uint32_t b[2] = {uint32_t(R), uint32_t(G::KS)};
        const CUtensorMapSwizzle sw =
            R == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : (R == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
        if (!encode_map(&m.a[p], X, dt, 2, d, s, b, sw)) return false;
    }
    {  // B_i template view {64, R, H2/64}: element (n, k, b) at B + k*H2 + 64*b + n
        const uint64_t d[3] = {64, uint64_t(R), uint64_t(H2 / 64)};
        const uint64_t s[2] = {uint64_t(H2) * 2, 128};
        const uint32_t b[3] = {64, uint32_t(R), uint32_t(G::NB)};
        if (!encode_map(&m.b[p], X, dt, 3, d, s, b, CU_TENSOR_MAP_SWIZZLE_128B)) return false;
    }
    return true;
}

}  // namespace sgmv

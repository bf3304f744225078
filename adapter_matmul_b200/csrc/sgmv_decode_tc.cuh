// sgmv_decode_tc.cuh -- one-kernel SGMV on tcgen05 for decode batches whose segments hold
// several tokens (a few to a few dozen), where the fp32 CUDA-core expand of the fused
// kernel becomes the bottleneck.
//
// Maths (page "Punica：多 LoRA 模型统一服务框架", the Punica README, its LoRA and
// multi-LoRA paragraphs): Y[t,:] += scale * (X[t,:] @ A_i) @ B_i for the rows t of each
// segment, A_i [H1, r], B_i [r, H2], row-major.
//
// Jobs and the cluster split are those of the fused kernel (sgmv_fused.cuh), with chunks of
// 16 tokens: a cluster of C CTAs runs a job (projection, segment, chunk); CTA c owns a
// K-slice of A_i and an N-slice of B_i.
//
//   shrink   D1[128 x r] (TMEM) = X_chunk[128 x 64k] @ A_i[64k x r] over the CTA's K-slice,
//            tcgen05.mma M=128 N=r; only the chunk's first nt <= 16 rows are loaded (TMA,
//            16-row boxes) and used, the other rows of the operand are never read back;
//   V        the partial D1 rows of the chunk leave TMEM (tcgen05.ld), are pushed to every
//            CTA of the cluster with st.async and summed in rank order; V (fp32) is written
//            back as the two 16-bit operands V_hi + V_lo (about 16 significant bits of V);
//   expand   transposed, so that the MMA's N is the token count rather than 128 padded rows:
//            D2^T[128 cols x 16 tokens] = B_tile^T[128 x r] @ V^T[r x 16], M=128 N=16, the
//            B tile as an MN-major operand; double-buffered in TMEM; the epilogue adds
//            scale * D2 to the staged Y rows, rounds once and stores them.
//
// Data movement: X by TMA (tensor maps built per call), A_i and B_i tiles by cp.async into
// the swizzled canonical layouts, Y rows by bulk copies, all through one ring of shared
// memory stages. Warps: 0 producer, 1 TMEM owner and MMA issuer, 2..5 exchange and epilogue
// (one TMEM lane quarter each). Programmatic dependent launch as in the fused kernel: X and
// Y are read only after griddepcontrol.wait. Every wait is bounded in time.
#pragma once

#include "sgmv_grouped_tc.cuh"

namespace sgmv {

constexpr int kDTokens = 16;  // tokens per job = N of the expand MMA
constexpr int kDStages = 3;
constexpr int kDThreads = 192;
constexpr int kDTmemCols = 128;  // D1 at [0, r), D2 buffers at 64 and 80

struct XMaps {
    CUtensorMap m[kFusedMaxProblems];  // X of each problem: boxes of 16 rows x 64 columns, 128B swizzle
};

__host__ __device__ constexpr int round1024(int v) { return (v + 1023) / 1024 * 1024; }

template <int R>
struct DecodeTCGeom {
    static constexpr int X_BYTES = kGM * kGK * 2;  // 128-row operand tile; rows >= 16 never loaded
    static constexpr int A_BYTES = round1024(kGK * R * 2);
    static constexpr int SH_STAGE = X_BYTES + A_BYTES;
    static constexpr int B_BYTES = R * kGN * 2;  // two MN-major 64-column blocks
    static constexpr int Y_BYTES = kDTokens * kGN * 2;
    static constexpr int EX_STAGE = B_BYTES + Y_BYTES;
    static constexpr int STAGE = round1024(SH_STAGE > EX_STAGE ? SH_STAGE : EX_STAGE);
    static constexpr int VT_BYTES = round1024(kDTokens * R * 2);  // one of V_hi^T, V_lo^T
    static constexpr int RECV = kFusedMaxCluster * kDTokens * R * 4;
    static constexpr size_t BASE = size_t(kDStages) * STAGE + 2 * size_t(VT_BYTES) + RECV;
    static constexpr int SW_BITS = R == 64 ? 3 : (R == 32 ? 2 : 1);
    static constexpr uint64_t SW_TYPE = R == 64 ? 2 : (R == 32 ? 4 : 6);
    static constexpr int ROW_BYTES = R * 2;
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

template <typename T, int R>
__global__ void __launch_bounds__(kDThreads, 1)
    sgmv_decode_tc_kernel(const __grid_constant__ XMaps maps, const FusedParams P) {
    using G = DecodeTCGeom<R>;
    extern __shared__ __align__(1024) unsigned char dsm_raw[];
    unsigned char* dsm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* ring = dsm;
    unsigned char* vhi = ring + kDStages * G::STAGE;
    unsigned char* vlo = vhi + G::VT_BYTES;
    float* recv = reinterpret_cast<float*>(vlo + G::VT_BYTES);
    int* pref = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(recv) + G::RECV);

    __shared__ __align__(8) uint64_t full[kDStages], empty[kDStages];
    __shared__ __align__(8) uint64_t d1_full, v_full, d2_full[2], d2_empty[2], vready, vfree;
    __shared__ uint32_t tmem_base_s;

    const int C = static_cast<int>(cluster_size());
    const int c = static_cast<int>(cluster_rank());
    const int cluster_id = blockIdx.x / C;
    const int n_clusters = gridDim.x / C;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDStages; ++i) {
            mbar_init(&full[i], 1 + 32);  // producer lane 0 (expect_tx) + 32 cp.async arrivals
            mbar_init(&empty[i], 1 + 4);  // MMA commit + 4 arrivals (MMA thread or epilogue warps)
        }
        mbar_init(&d1_full, 1);
        mbar_init(&v_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&d2_full[i], 1);
            mbar_init(&d2_empty[i], 4);
        }
        mbar_init(&vready, 1);  // own expect_tx; the C tiles arrive as transaction bytes
        mbar_init(&vfree, C);   // one arrival per receiver
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
    bool dead = false;

    if (warp == 0) {
        // ---------------------------------- producer ----------------------------------
        uint32_t it = 0;
        bool waited = false;
        int deferred = 0;  // shrink stages of the first job still missing their X box
        int d_p = 0, d_t0 = 0, d_k0 = 0;
        for (int j = cluster_id; j < entries; j += n_clusters) {
            int p, s, q0, nq;
            entry_at<kDTokens>(P, pref, j, p, s, q0, nq);
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at<kDTokens>(P, p, s, q, c, job)) break;
                const FusedProblem& pr = P.prob[job.p];
                const T* A = static_cast<const T*>(job.a);
                const T* B = static_cast<const T*>(job.b);
                const T* Yg = static_cast<const T*>(pr.Y);
                const int nA = (job.nk + kGK - 1) / kGK;
                for (int ta = 0; ta < nA; ++ta, ++it) {
                    const uint32_t st = it % kDStages;
                    if (it >= kDStages) {
                        if (!waited) {
                            pdl_wait();
                            waited = true;
                            if (lane == 0)
                                for (int d = 0; d < deferred; ++d) {
                                    mbar_arrive_expect_tx(&full[d], kDTokens * kGK * 2);
                                    tma_load_2d(ring + d * G::STAGE, &maps.m[d_p], d_k0 + d * kGK, d_t0, &full[d]);
                                }
                        }
                        mbar_wait<false>(&empty[st], ((it / kDStages) - 1) & 1u, P.dev_status, dead);
                    }
                    unsigned char* xs = ring + st * G::STAGE;
                    unsigned char* as = xs + G::X_BYTES;
                    const int kbase = job.k0 + ta * kGK;
                    if (waited) {
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&full[st], kDTokens * kGK * 2);
                            tma_load_2d(xs, &maps.m[job.p], kbase, job.t0, &full[st]);
                        }
                    } else {
                        deferred = ta + 1;
                        d_p = job.p;
                        d_t0 = job.t0;
                        d_k0 = job.k0;
                    }
                    constexpr int CHUNKS = kGK * R / 8;
                    for (int qq = lane; qq < CHUNKS; qq += 32) {
                        const int k = qq / (R / 8), cc = qq % (R / 8);
                        const int gk = kbase + k;
                        const bool in = gk < job.k0 + job.nk;
                        cp_async16(as + swz(k, cc, G::SW_BITS), A + size_t(in ? gk : 0) * R + cc * 8, in ? 16u : 0u);
                    }
                    cp_async_arrive_noinc(&full[st]);
                }
                if (!waited) {
                    pdl_wait();
                    waited = true;
                    if (lane == 0)
                        for (int d = 0; d < deferred; ++d) {
                            mbar_arrive_expect_tx(&full[d], kDTokens * kGK * 2);
                            tma_load_2d(ring + d * G::STAGE, &maps.m[d_p], d_k0 + d * kGK, d_t0, &full[d]);
                        }
                }
                const int n_hi = job.c0 + job.nc;
                const int nB = (job.nc + kGN - 1) / kGN;
                for (int tb = 0; tb < nB; ++tb, ++it) {
                    const uint32_t st = it % kDStages;
                    if (it >= kDStages) mbar_wait<false>(&empty[st], ((it / kDStages) - 1) & 1u, P.dev_status, dead);
                    unsigned char* bs = ring + st * G::STAGE;
                    unsigned char* ys = bs + G::B_BYTES;
                    const int n0 = job.c0 + tb * kGN;
                    const int nct = min(kGN, n_hi - n0);
                    if (lane == 0) mbar_arrive_expect_tx(&full[st], uint32_t(job.nt) * nct * 2);
                    __syncwarp();
                    if (lane < job.nt)
                        bulk_g2s(ys + lane * kGN * 2, Yg + size_t(job.t0 + lane) * pr.H2 + n0, uint32_t(nct) * 2,
                                 &full[st]);
                    constexpr int CHUNKS = R * kGN / 8;
                    for (int qq = lane; qq < CHUNKS; qq += 32) {
                        const int k = qq / (kGN / 8), cc = qq % (kGN / 8);
                        const int blk = cc / 8, c8 = cc % 8;
                        const int gn = n0 + cc * 8;
                        const bool in = gn < n_hi;
                        cp_async16(bs + blk * (R * 128) + swz(k, c8, 3), B + size_t(k) * pr.H2 + (in ? gn : 0),
                                   in ? 16u : 0u);
                    }
                    cp_async_arrive_noinc(&full[st]);
                }
            }
        }
        if (!waited) pdl_wait();
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (C > 1) cluster_wait();
    } else if (warp == 1) {
        // ---------------------------------- MMA issuer ----------------------------------
        const uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
        const uint32_t idesc_s = instr_desc(fmt, 0, 1, R, kGM);         // X K-major, A_i MN-major, N = r
        const uint32_t idesc_e = instr_desc(fmt, 1, 0, kDTokens, kGM);  // B tile MN-major, V^T K-major, N = 16
        uint32_t it = 0, u = 0, g = 0;
        for (int j = cluster_id; j < entries; j += n_clusters) {
            int p, s, q0, nq;
            entry_at<kDTokens>(P, pref, j, p, s, q0, nq);
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at<kDTokens>(P, p, s, q, c, job)) break;
                const int nA = (job.nk + kGK - 1) / kGK;
                for (int ta = 0; ta < nA; ++ta, ++it) {
                    const uint32_t st = it % kDStages;
                    mbar_wait<false>(&full[st], (it / kDStages) & 1u, P.dev_status, dead);
                    fence_proxy_async();
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t xa = smem_u32(ring + st * G::STAGE);
                        const uint32_t aa = xa + G::X_BYTES;
#pragma unroll
                        for (int kk = 0; kk < kGK / 16; ++kk) {
                            const uint64_t adesc = smem_desc(xa + kk * 32, 16, 1024, 2);
                            const uint64_t bdesc =
                                smem_desc(aa + kk * 16 * G::ROW_BYTES, 16 * G::ROW_BYTES, 8 * G::ROW_BYTES, G::SW_TYPE);
                            tc_mma(tmem, adesc, bdesc, idesc_s, (ta | kk) ? 1u : 0u);
                        }
                        tc_commit(&empty[st]);
                        for (int i = 0; i < 4; ++i) mbar_arrive_local(&empty[st]);
                    }
                    __syncwarp();
                }
                // (with no K rows here no shrink MMA ran; the epilogue then uses zeros for D1)
                if (lane == 0) tc_commit(&d1_full);
                __syncwarp();
                mbar_wait<false>(&v_full, u & 1u, P.dev_status, dead);
                tc_fence_after();
                const int nB = (job.nc + kGN - 1) / kGN;
                for (int tb = 0; tb < nB; ++tb, ++it, ++g) {
                    const uint32_t st = it % kDStages;
                    const uint32_t buf = g & 1u;
                    if (g >= 2) mbar_wait<false>(&d2_empty[buf], ((g >> 1) - 1) & 1u, P.dev_status, dead);
                    mbar_wait<false>(&full[st], (it / kDStages) & 1u, P.dev_status, dead);
                    fence_proxy_async();
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t ba = smem_u32(ring + st * G::STAGE);
                        const uint32_t d2 = tmem + 64u + 16u * buf;
#pragma unroll
                        for (int kk = 0; kk < R / 16; ++kk) {
                            const uint64_t adesc = smem_desc(ba + kk * 16 * 128, R * 128, 1024, 2);
                            const uint64_t bhi = smem_desc(smem_u32(vhi) + kk * 32, 16, 8 * G::ROW_BYTES, G::SW_TYPE);
                            const uint64_t blo = smem_desc(smem_u32(vlo) + kk * 32, 16, 8 * G::ROW_BYTES, G::SW_TYPE);
                            tc_mma(d2, adesc, bhi, idesc_e, kk ? 1u : 0u);
                            tc_mma(d2, adesc, blo, idesc_e, 1u);
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
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
        const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
        if (C > 1) cluster_wait();
        uint32_t it = 0, u = 0, g = 0;
        for (int j = cluster_id; j < entries; j += n_clusters) {
            int p, s, q0, nq;
            entry_at<kDTokens>(P, pref, j, p, s, q0, nq);
            for (int q = q0; q < q0 + nq; ++q) {
                Job job;
                if (!job_at<kDTokens>(P, p, s, q, c, job)) break;
                const FusedProblem& pr = P.prob[job.p];
                const int nA = (job.nk + kGK - 1) / kGK;
                it += nA;
                if (quarter == 0) {
                    // partial V of this CTA: D1 rows 0..nt-1 (lanes 0..15 of quarter 0)
                    mbar_wait<false>(&d1_full, u & 1u, P.dev_status, dead);
                    tc_fence_after();
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
                                st_async_v4(slot + i, make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]), &vready, qr);
                    }
                    mbar_wait<true>(&vready, u & 1u, P.dev_status, dead);
                    if (lane < job.nt) {
#pragma unroll
                        for (int i = 0; i < R; ++i) v[i] = 0.f;
                        for (int qr = 0; qr < C; ++qr) {
                            const float* src = recv + (size_t(qr) * kDTokens + lane) * R;
#pragma unroll
                            for (int i = 0; i < R; ++i) v[i] += src[i];
                        }
                        // V^T operand rows: token `lane`, R values, K-major swizzled; hi + lo
#pragma unroll
                        for (int ch = 0; ch < R / 8; ++ch) {
                            float hi[8], lo[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                hi[i] = Storage<T>::round(v[ch * 8 + i]);
                                lo[i] = v[ch * 8 + i] - hi[i];
                            }
                            const uint32_t off = swz(lane, ch, G::SW_BITS);
                            st_vec(vhi + off, pack8<T>(hi));
                            st_vec(vlo + off, pack8<T>(lo));
                        }
                    }
                    fence_proxy_async();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_local(&v_full);
                    if (lane < C) mbar_arrive_remote(&vfree, static_cast<uint32_t>(lane));
                }
                // expand epilogue: this warp's 32 columns of each 128-column tile, all tokens
                T* __restrict__ Y = static_cast<T*>(pr.Y);
                const int n_hi = job.c0 + job.nc;
                const int nB = (job.nc + kGN - 1) / kGN;
                for (int tb = 0; tb < nB; ++tb, ++it, ++g) {
                    const uint32_t st = it % kDStages;
                    const uint32_t buf = g & 1u;
                    mbar_wait<false>(&full[st], (it / kDStages) & 1u, P.dev_status, dead);
                    mbar_wait<false>(&d2_full[buf], (g >> 1) & 1u, P.dev_status, dead);
                    tc_fence_after();
                    float acc[16];
                    tmem_ld16(lane_base + 64u + 16u * buf, acc);
                    const int col_in_tile = quarter * 32 + lane;
                    const int col = job.c0 + tb * kGN + col_in_tile;
                    if (col < n_hi) {
                        const T* ys = reinterpret_cast<const T*>(ring + st * G::STAGE + G::B_BYTES);
#pragma unroll
                        for (int t = 0; t < kDTokens; ++t) {
                            if (t < job.nt) {
                                const float y = Storage<T>::to1(ys[t * kGN + col_in_tile]);
                                const float o = __fadd_rn(y, __fmul_rn(pr.scale, acc[t]));
                                Y[size_t(job.t0 + t) * pr.H2 + col] = Storage<T>::from1(o);
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_local(&d2_empty[buf]);
                        mbar_arrive_local(&empty[st]);
                    }
                }
                ++u;
            }
        }
        if (quarter == 0) {
            pdl_wait();
            if (u >= 1) mbar_wait<true>(&vfree, (u - 1) & 1u, P.dev_status, dead);
            if (c == 0 && lane == 0) {  // report each rejected segment once
                for (int j = cluster_id; j < P.n_problems * P.n_segments; j += n_clusters) {
                    const int p2 = j / P.n_segments, s2 = j - p2 * P.n_segments;
                    Segment seg;
                    report(P.dev_status, load_segment(P.seg_starts, P.lora_idx, P.prob[p2].A_ptrs, P.prob[p2].B_ptrs,
                                                      s2, P.T, P.prob[p2].num_adapters, seg));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kDTmemCols) : "memory");
}

}  // namespace sgmv

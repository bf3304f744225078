// sgmv_gemm_tc2.cuh -- the whole LoRA layer, Y = X@W + scale * (X@A_i)@B_i, on pairs of SMs:
// tcgen05.mma with cta_group::2, 256 x 256 output tiles.
//
// Maths and the delta as extra K-steps: as in sgmv_gemm_tc.cuh (page "Punica：多 LoRA 模型统一服务
// 框架", the Punica README, LoRA and multi-LoRA paragraphs). What changes is the split of a tile
// over two SMs. The kernel runs in clusters of two CTAs (a pair). One MMA instruction, issued by
// one thread of the pair's first CTA, computes a 256 x 256 x 16 step: the first CTA's shared
// memory holds rows 0..127 of the A operand (X, or V' in a delta pass) and columns 0..127 of
// the B operand (W, or B_i), the second CTA's the other halves at the same offsets, and each
// CTA's tensor memory receives its own 128 rows of the accumulator. Per SM and K-step of 64 a
// stage is 32 KB (16 KB of X, 16 KB of W) for the same tensor-core work that takes 48 KB in
// the single-SM kernel: the operand traffic from L2 per unit of work drops by a third.
//
// Synchronisation across the pair:
//   full[s]      in the first CTA: its producer arms it with the bytes of both CTAs' copies;
//                both CTAs' copies complete on it (the second CTA addresses it by clearing the
//                pair bit of the barrier's shared-memory address);
//   empty[s]     in both CTAs: the MMA's commit arrives on both (multicast to the pair);
//   vfull        in the first CTA: 8 arrivals from each CTA's epilogue warps (V' rows written);
//   vempty       in both CTAs: the MMA's commit, multicast;
//   acc_full[b]  in both CTAs: the MMA's commit, multicast;
//   acc_empty[b] in the first CTA: 8 arrivals from each CTA's epilogue warps.
// Tensor memory is allocated and freed by both CTAs together (cta_group::2). Every wait is
// bounded in time and reports LORA_SGMV_DEV_TIMEOUT; the pair meets at a cluster barrier before
// it frees tensor memory and exits.
#pragma once

#include "sgmv_gemm_tc.cuh"

namespace sgmv {

constexpr int kL2M = 256;  // rows per pair tile (128 per CTA)
constexpr int kL2N = 256;  // columns per pair tile (128 per CTA for the B operand)
constexpr int kL2Stages = 6;
constexpr int kL2XBytes = 128 * kLK * 2;  // 16 KB: this CTA's 128 rows x 64
constexpr int kL2WBytes = kLK * 128 * 2;  // 16 KB: 64 x this CTA's 128 columns (two 8 KB boxes)
constexpr int kL2Stage = kL2XBytes + kL2WBytes;
constexpr size_t kL2Smem = size_t(kL2Stages) * kL2Stage + 2 * kLVBytes + 1024;

__device__ __forceinline__ uint32_t pair_rank() { return cluster_rank() & 1u; }

// shared::cluster address of the same object in the pair's first CTA
__device__ __forceinline__ uint32_t leader_addr(const void* p) { return map_rank(smem_u32(p), 0); }

// an int in the shared memory of CTA `rank` of the cluster, at the same offset as `p`
__device__ __forceinline__ int ld_cluster_int(const int* p, uint32_t rank) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(map_rank(smem_u32(p), rank)) : "memory");
    return v;
}

__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(leader_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on `bar` in both CTAs of the pair once every MMA issued so far has completed
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}\n" ::"r"(
            smem_u32(bar))
        : "memory");
}

// arrive on `bar` in the pair's first CTA (release, cluster scope)
__device__ __forceinline__ void mbar_arrive_leader(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(leader_addr(bar)) : "memory");
}

template <typename T, int R>
__global__ void __launch_bounds__(kLThreads, 1)
    sgmv_gemm_delta_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                                const __grid_constant__ CUtensorMap tmB, const GemmParams P) {
    extern __shared__ __align__(1024) unsigned char lsm_raw[];
    unsigned char* ring =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(lsm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[kL2Stages], empty[kL2Stages], vfull, vempty;
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ __align__(128) CUtensorMap map_build;
    __shared__ uint32_t tmem_base_s;
    __shared__ int table_s;
    unsigned char* vhi = ring + kL2Stages * kL2Stage;
    unsigned char* vlo = vhi + kLVBytes;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = pair_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int n_pairs = gridDim.x >> 1;
    const int units = P.m_tiles * P.n_tiles;  // pair tiles

    if (threadIdx.x == 0) {
        for (int i = 0; i < kL2Stages; ++i) {
            mbar_init(&full[i], 1);   // the first CTA's producer (expect_tx); both CTAs' copies complete it
            mbar_init(&empty[i], 1);  // the MMA's commit
        }
        mbar_init(&vfull, 2 * kLEpiWarps);
        mbar_init(&vempty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 2 * kLEpiWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        table_s = claim_map_table();
        if (table_s < 0) report(P.dev_status, LORA_SGMV_DEV_TIMEOUT);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kLTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    // the pair's barriers exist before either CTA touches the other's
    cluster_arrive();
    cluster_wait();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const int table = table_s;
    // a CTA that could not claim a map table does no work, and then neither does its pair
    const bool idle = table < 0 || ld_cluster_int(&table_s, rank ^ 1u) < 0;
    const int first_unit = idle ? units : pair;
    const int k_steps = (P.H1 + kLK - 1) / kLK;
    bool dead = false;

    if (warp == 0) {
        // ---------------------------------- producer ----------------------------------
        MapTable* tab = g_map_tables + (table < 0 ? 0 : table);
        uint32_t it = 0;
        int passes = 0;
        for (int u = first_unit; u < units; u += n_pairs) {
            const int m0 = (u / P.n_tiles) * kL2M, n0 = (u % P.n_tiles) * kL2N;
            const int mr = m0 + int(rank) * 128, nc = n0 + int(rank) * 128;  // this CTA's rows and columns
            for (int ks = 0; ks < k_steps; ++ks, ++it) {
                const uint32_t st = it % kL2Stages;
                if (it >= kL2Stages) mbar_wait<false>(&empty[st], ((it / kL2Stages) - 1) & 1u, P.dev_status, dead);
                unsigned char* xs = ring + st * kL2Stage;
                if (lane == 0) {
                    if (leader) mbar_arrive_expect_tx(&full[st], 2 * kL2Stage);
                    tma_load_2d_pair(xs, &tmX, ks * kLK, mr, &full[st]);
                    tma_load_2d_pair(xs + kL2XBytes, &tmW, nc, ks * kLK, &full[st]);
                    tma_load_2d_pair(xs + kL2XBytes + 8192, &tmW, nc + 64, ks * kLK, &full[st]);
                }
                __syncwarp();
            }
            Segment seg;
            for (int s = next_pass(P, 0, m0, m0 + kL2M, seg); s < P.n_segments;
                 s = next_pass(P, s + 1, m0, m0 + kL2M, seg)) {
                CUtensorMap* gB = &tab->m[passes % (2 * kMapRing)];
                ++passes;
                map_template_to_smem(&map_build, &tmB);
                if (lane == 0) map_set_address(&map_build, seg.b);
                __syncwarp();
                map_publish(gB, &map_build);
                if (lane == 0) map_acquire(gB);
                __syncwarp();
                const uint32_t st = it % kL2Stages;
                if (it >= kL2Stages) mbar_wait<false>(&empty[st], ((it / kL2Stages) - 1) & 1u, P.dev_status, dead);
                unsigned char* bs = ring + st * kL2Stage + kL2XBytes;
                if (lane == 0) {
                    if (leader) mbar_arrive_expect_tx(&full[st], 2 * 2 * R * 128);
                    tma_load_2d_pair(bs, gB, nc, 0, &full[st]);
                    tma_load_2d_pair(bs + R * 128, gB, nc + 64, 0, &full[st]);
                }
                __syncwarp();
                ++it;
            }
        }
        // Before the pair may exit: every copy of both CTAs has landed (they complete on the first
        // CTA's full barriers), and every commit of the pair's MMAs has arrived on this CTA's
        // empty barriers.
        if (lane == 0)
            for (uint32_t i = it > uint32_t(kL2Stages) ? it - kL2Stages : 0u; i < it; ++i) {
                if (leader) drain_wait(&full[i % kL2Stages], (i / kL2Stages) & 1u);
                drain_wait(&empty[i % kL2Stages], (i / kL2Stages) & 1u);
            }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------- MMA issuer (first CTA of the pair) -------------------------
        if (leader) {
            const uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
            const uint32_t idesc = instr_desc(fmt, 0, 1, kL2N, kL2M);  // M = 256 over the pair, N = 256
            uint32_t it = 0, pk = 0;
            int local = 0;
            for (int u = first_unit; u < units; u += n_pairs, ++local) {
                const int m0 = (u / P.n_tiles) * kL2M;
                const int buf = local & 1;
                if (local >= 2) mbar_wait<true>(&acc_empty[buf], ((local >> 1) - 1) & 1u, P.dev_status, dead);
                tc_fence_after();
                const uint32_t acc = tmem + uint32_t(buf * kLN);
                for (int ks = 0; ks < k_steps; ++ks, ++it) {
                    const uint32_t st = it % kL2Stages;
                    mbar_wait<false>(&full[st], (it / kL2Stages) & 1u, P.dev_status, dead);
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t xa = smem_u32(ring + st * kL2Stage);
                        const uint32_t wa = xa + kL2XBytes;
#pragma unroll
                        for (int kk = 0; kk < kLK / 16; ++kk) {
                            const uint64_t adesc = smem_desc(xa + kk * 32, 16, 1024, 2);
                            const uint64_t bdesc = smem_desc(wa + kk * 16 * 128, 8192, 1024, 2);
                            tc_mma_pair(acc, adesc, bdesc, idesc, (ks | kk) ? 1u : 0u);
                        }
                        tc_commit_pair(&empty[st]);
                    }
                    __syncwarp();
                }
                Segment seg;
                for (int s = next_pass(P, 0, m0, m0 + kL2M, seg); s < P.n_segments;
                     s = next_pass(P, s + 1, m0, m0 + kL2M, seg)) {
                    const uint32_t st = it % kL2Stages;
                    mbar_wait<false>(&full[st], (it / kL2Stages) & 1u, P.dev_status, dead);
                    mbar_wait<true>(&vfull, pk & 1u, P.dev_status, dead);
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t ba = smem_u32(ring + st * kL2Stage + kL2XBytes);
#pragma unroll
                        for (int kk = 0; kk < R / 16; ++kk) {
                            const uint64_t bdesc = smem_desc(ba + kk * 16 * 128, R * 128, 1024, 2);
                            tc_mma_pair(acc, smem_desc(smem_u32(vhi) + kk * 32, 16, 1024, 2), bdesc, idesc, 1u);
                            tc_mma_pair(acc, smem_desc(smem_u32(vlo) + kk * 32, 16, 1024, 2), bdesc, idesc, 1u);
                        }
                        tc_commit_pair(&empty[st]);
                        tc_commit_pair(&vempty);
                    }
                    __syncwarp();
                    ++it;
                    ++pk;
                }
                if (lane == 0) tc_commit_pair(&acc_full[buf]);
                __syncwarp();
            }
        }
    } else {
        // ------------------------- V' operands and the epilogue -------------------------
        const int ew = warp - 2;             // 0..7
        const int quarter = warp & 3;        // TMEM lanes [32*quarter, +32)
        const int half = ew >> 2;            // columns [128*half, +128) of the tile
        const int et = ew * 32 + lane;       // 0..255 over the epilogue warps
        const int vrow = et >> 1;            // V' operand: this CTA's row vrow, columns [vcol0, vcol0 + R/2)
        const int vcol0 = (et & 1) * (R / 2);
        T* __restrict__ Y = static_cast<T*>(P.Y);
        if (blockIdx.x == 0 && warp == 9)  // report every rejected segment once, one lane per segment
            for (int s = lane; s < P.n_segments; s += 32) {
                Segment seg;
                report(P.dev_status,
                       load_segment(P.seg_starts, P.lora_idx, P.A_ptrs, P.B_ptrs, s, P.T, P.num_adapters, seg));
            }
        uint32_t pk = 0;
        bool waited = !P.v_after_wait;
        int local = 0;
        for (int u = first_unit; u < units; u += n_pairs, ++local) {
            const int m0 = (u / P.n_tiles) * kL2M, n0 = (u % P.n_tiles) * kL2N;
            const int mr = m0 + int(rank) * 128;  // this CTA's 128 rows of the tile
            const int buf = local & 1;
            Segment seg;
            for (int s = next_pass(P, 0, m0, m0 + kL2M, seg); s < P.n_segments;
                 s = next_pass(P, s + 1, m0, m0 + kL2M, seg), ++pk) {
                const int g = mr + vrow;
                const bool in = g >= seg.begin && g < seg.end;
                if (!waited) {  // V is written by the kernel just before this one
                    pdl_wait();
                    waited = true;
                }
                float v[R / 2];
#pragma unroll
                for (int j = 0; j < R / 2; j += 4) {
                    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (in) q = *reinterpret_cast<const float4*>(P.V + size_t(g) * R + vcol0 + j);
                    v[j] = __fmul_rn(P.scale, q.x);
                    v[j + 1] = __fmul_rn(P.scale, q.y);
                    v[j + 2] = __fmul_rn(P.scale, q.z);
                    v[j + 3] = __fmul_rn(P.scale, q.w);
                }
                if (pk >= 1) mbar_wait<false>(&vempty, (pk - 1) & 1u, P.dev_status, dead);
#pragma unroll
                for (int c8 = 0; c8 < R / 16; ++c8) {
                    float hi[8], lo[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float x = v[c8 * 8 + i];
                        hi[i] = Storage<T>::round(x);
                        lo[i] = x - hi[i];
                    }
                    const uint32_t off = swz(vrow, (vcol0 / 8) + c8, 3);
                    st_vec(vhi + off, pack8<T>(hi));
                    st_vec(vlo + off, pack8<T>(lo));
                }
                fence_proxy_async();  // generic-proxy writes -> tensor-core reads
                __syncwarp();
                if (lane == 0) mbar_arrive_leader(&vfull);
            }
            // epilogue: this CTA's row m of the tile, this warp's 128 columns
            mbar_wait<true>(&acc_full[buf], (local >> 1) & 1u, P.dev_status, dead);
            tc_fence_after();
            const int m = quarter * 32 + lane;
            const int gr = mr + m;
            const uint32_t taddr = tmem + (uint32_t(quarter * 32) << 16) + uint32_t(buf * kLN + half * 128);
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 32) {
                float a[32];
                tmem_ld32(taddr + c0, a);
                const int col = n0 + half * 128 + c0;
                if (gr < P.T) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        if (col + ch * 8 < P.H2) {
                            float o[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) o[i] = a[ch * 8 + i];
                            st_vec(Y + size_t(gr) * P.H2 + col + ch * 8, pack8<T>(o));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_leader(&acc_empty[buf]);
        }
        if (!waited) pdl_wait();
    }
    tc_fence_before();
    __syncthreads();
    // neither CTA frees its tensor memory or shared memory while the pair may still use them
    cluster_arrive();
    cluster_wait();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kLTmemCols) : "memory");
    if (threadIdx.x == 0) release_map_table(table);
}

template <typename T, int R>
inline cudaError_t launch_gemm_delta_pair_kernel(const CUtensorMap& tmX, const CUtensorMap& tmW,
                                                 const CUtensorMap& tmB, const GemmParams& P, int pairs,
                                                 cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(sgmv_gemm_delta_pair_kernel<T, R>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kL2Smem));
    });
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kLThreads, 1, 1);
    cfg.dynamicSmemBytes = kL2Smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.v_after_wait ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, sgmv_gemm_delta_pair_kernel<T, R>, tmX, tmW, tmB, P);
}

}  // namespace sgmv

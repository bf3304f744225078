// sgmv_gemm_tc.cuh -- the whole LoRA layer on tcgen05: Y = X@W + scale * (X@A_i)@B_i, with the
// delta computed inside the base product's accumulator.
//
// Maths (page "Punica：多 LoRA 模型统一服务框架", the Punica README): its LoRA paragraph gives
// x@(W + A@B) = x@W + x@A@B for a frozen W [H1, H2] and an adapter A [H1, r], B [r, H2]; its
// multi-LoRA paragraph gives the batch form Y = X@W + (x_1@A_1@B_1, ..., x_n@A_n@B_n), each row
// with its own adapter. Here the rows of segment s use adapter i = lora_idx[s], and the delta
// carries the kernel contract's scale.
//
// The delta as extra K-steps. With V = X@A_i (fp32, [T, r], from a shrink kernel that runs
// first), the delta of a row is (scale * V[t, :]) @ B_i: a product with inner dimension r. So
// for an output tile the accumulator takes, after the H1 K-steps of X@W, 2r more K-steps per
// adapter that touches the tile's rows:
//     acc += V'_hi @ B_i[:, tile] + V'_lo @ B_i[:, tile],   V' = scale * V
// where V'_hi = round16(V') and V'_lo = round16(V' - V'_hi) are the two 16-bit operands that
// carry V' to about 16 significant bits (the MMA takes 16-bit operands; V is never rounded to
// one 16-bit value). Rows of the tile outside the adapter's segment are zero in that pass's
// V' operand, so a tile that spans several segments runs one pass per segment. The epilogue
// rounds the accumulator once to the storage type and writes Y (Y is an output here, not read).
//
// Tiles and pipeline. Output tiles of 128 rows x 256 columns; the kernel is persistent (one CTA
// per SM, tiles taken round-robin in row-major order so that the CTAs in flight share W and a
// few X panels in L2). One ring of four 48 KB stages: a base stage holds an X tile [128 x 64]
// (K-major, 128-byte swizzle) and a W tile [64 x 256] (four MN-major 64-column boxes); a delta
// stage holds the B_i tile [r x 256] in the W slot (TMA through a tensor map made on the device,
// as B_i is reached through a pointer table). The V'_hi and V'_lo operands [128 x r] of a pass
// have a buffer of their own, written by the epilogue warps as soon as the previous pass's MMAs
// have read it -- for a tile in one segment, during the main loop of the tile, well before its
// delta stage. The fp32 accumulator lives in TMEM, two buffers of 256 columns, so the epilogue of
// one tile overlaps the main loop of the next.
//
// The kernel that makes V runs just before this one on the stream; this kernel is launched with
// programmatic dependent launch after it, so its CTAs start on the SMs that kernel leaves free
// and stream X and W (which that kernel does not write) while it finishes; only the epilogue
// warps wait (griddepcontrol.wait) before they read V.
//
// Warps: 0 producer (TMA), 1 TMEM owner and MMA issuer (one thread), 2..9 epilogue (two per
// TMEM lane quarter, one per 128-column half of the tile), which also build the V' operands.
// Every wait is bounded in time and reports LORA_SGMV_DEV_TIMEOUT; TMEM is always freed.
#pragma once

#include "sgmv_grouped_tc.cuh"

namespace sgmv {

constexpr int kLM = 128;        // rows per tile (UMMA M)
constexpr int kLN = 256;        // columns per tile (UMMA N)
constexpr int kLK = 64;         // K per base stage
constexpr int kLStages = 4;
constexpr int kLThreads = 320;  // producer, MMA issuer, 8 epilogue warps
constexpr int kLEpiWarps = 8;
constexpr int kLTmemCols = 512;  // two accumulators of 256 columns
constexpr int kLXBytes = kLM * kLK * 2;         // 16 KB
constexpr int kLWBytes = kLK * kLN * 2;         // 32 KB (four 8 KB boxes)
constexpr int kLStage = kLXBytes + kLWBytes;    // 48 KB
constexpr int kLVBytes = kLM * 64 * 2;          // one V' operand [128 x r <= 64], 128-byte rows
constexpr size_t kLSmem = size_t(kLStages) * kLStage + 2 * kLVBytes + 1024;  // + alignment slack

inline bool gemm_tc_supported(int r, int H1, int H2) {
    return (r == 16 || r == 32 || r == 64) && H1 >= 8 && H2 >= 8 && H1 % 8 == 0 && H2 % 8 == 0;
}

struct GemmParams {
    void* Y;
    const float* V;  // [T, r] fp32, scale not applied
    const void* const* A_ptrs;  // only checked, as the shrink that made V checked it
    const void* const* B_ptrs;
    const int32_t* seg_starts;
    const int32_t* lora_idx;
    uint32_t* dev_status;
    int n_segments;
    int num_adapters;
    int T;
    int H1;
    int H2;
    float scale;
    int m_tiles;
    int n_tiles;
    int v_after_wait;  // 1: V comes from the kernel just before (read only after griddepcontrol.wait)
};

// Next valid segment at or after s that intersects rows [m0, m1); n_segments if none. The
// same walk runs in every warp role, so all roles agree on a tile's delta passes.
__device__ __forceinline__ int next_pass(const GemmParams& P, int s, int m0, int m1, Segment& seg) {
    for (; s < P.n_segments; ++s) {
        if (load_segment(P.seg_starts, P.lora_idx, P.A_ptrs, P.B_ptrs, s, P.T, P.num_adapters, seg)) continue;
        if (seg.begin < m1 && seg.end > m0 && seg.begin < seg.end) return s;
    }
    return P.n_segments;
}

template <typename T, int R>
__global__ void __launch_bounds__(kLThreads, 1)
    sgmv_gemm_delta_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                           const __grid_constant__ CUtensorMap tmB, const GemmParams P) {
    extern __shared__ __align__(1024) unsigned char lsm_raw[];
    unsigned char* ring =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(lsm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[kLStages], empty[kLStages], vfull, vempty;
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    unsigned char* vhi = ring + kLStages * kLStage;  // V' operands of the current delta pass
    unsigned char* vlo = vhi + kLVBytes;
    __shared__ __align__(128) CUtensorMap map_build;
    __shared__ uint32_t tmem_base_s;
    __shared__ int table_s;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int units = P.m_tiles * P.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kLStages; ++i) {
            mbar_init(&full[i], 1);    // producer's expect_tx; the copies complete the bytes
            mbar_init(&empty[i], 1);   // MMA commit
        }
        mbar_init(&vfull, kLEpiWarps);  // V' operands of the next pass written
        mbar_init(&vempty, 1);          // MMA commit: the pass's MMAs have read them
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kLEpiWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        table_s = claim_map_table();
        if (table_s < 0) report(P.dev_status, LORA_SGMV_DEV_TIMEOUT);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kLTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const int table = table_s;
    const int first_unit = table < 0 ? units : static_cast<int>(blockIdx.x);
    const int k_steps = (P.H1 + kLK - 1) / kLK;
    bool dead = false;

    if (warp == 0) {
        // ---------------------------------- producer ----------------------------------
        MapTable* tab = g_map_tables + (table < 0 ? 0 : table);
        uint32_t it = 0;
        int passes = 0;
        for (int u = first_unit; u < units; u += gridDim.x) {
            const int m0 = (u / P.n_tiles) * kLM, n0 = (u % P.n_tiles) * kLN;
            for (int ks = 0; ks < k_steps; ++ks, ++it) {
                const uint32_t st = it % kLStages;
                if (it >= kLStages) mbar_wait<false>(&empty[st], ((it / kLStages) - 1) & 1u, P.dev_status, dead);
                unsigned char* xs = ring + st * kLStage;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[st], kLStage);
                    tma_load_2d(xs, &tmX, ks * kLK, m0, &full[st]);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tma_load_2d(xs + kLXBytes + j * 8192, &tmW, n0 + j * 64, ks * kLK, &full[st]);
                }
                __syncwarp();
            }
            Segment seg;
            for (int s = next_pass(P, 0, m0, m0 + kLM, seg); s < P.n_segments;
                 s = next_pass(P, s + 1, m0, m0 + kLM, seg)) {
                // the B_i map of this pass goes to ring entry e; the stage that last used the
                // entry is at least eight stages back, so its copies have landed
                CUtensorMap* gB = &tab->m[passes % (2 * kMapRing)];
                ++passes;
                map_template_to_smem(&map_build, &tmB);
                if (lane == 0) map_set_address(&map_build, seg.b);
                __syncwarp();
                map_publish(gB, &map_build);
                if (lane == 0) map_acquire(gB);
                __syncwarp();
                {  // the delta stage: B_i's tile in the W slot
                    const uint32_t st = it % kLStages;
                    if (it >= kLStages) mbar_wait<false>(&empty[st], ((it / kLStages) - 1) & 1u, P.dev_status, dead);
                    unsigned char* bs = ring + st * kLStage + kLXBytes;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[st], 4 * R * 128);
#pragma unroll
                        for (int j = 0; j < 4; ++j) tma_load_2d(bs + j * (R * 128), gB, n0 + j * 64, 0, &full[st]);
                    }
                    __syncwarp();
                    ++it;
                }
            }
        }
        if (lane == 0)
            for (uint32_t i = it > uint32_t(kLStages) ? it - kLStages : 0u; i < it; ++i)
                drain_wait(&full[i % kLStages], (i / kLStages) & 1u);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------- MMA issuer ----------------------------------
        const uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
        const uint32_t idesc = instr_desc(fmt, 0, 1, kLN, kLM);  // A K-major, B MN-major, N = 256
        uint32_t it = 0, pk = 0;
        int local = 0;
        for (int u = first_unit; u < units; u += gridDim.x, ++local) {
            const int m0 = (u / P.n_tiles) * kLM;
            const int buf = local & 1;
            if (local >= 2) mbar_wait<false>(&acc_empty[buf], ((local >> 1) - 1) & 1u, P.dev_status, dead);
            tc_fence_after();
            const uint32_t acc = tmem + uint32_t(buf * kLN);
            for (int ks = 0; ks < k_steps; ++ks, ++it) {
                const uint32_t st = it % kLStages;
                mbar_wait<false>(&full[st], (it / kLStages) & 1u, P.dev_status, dead);
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t xa = smem_u32(ring + st * kLStage);
                    const uint32_t wa = xa + kLXBytes;
#pragma unroll
                    for (int kk = 0; kk < kLK / 16; ++kk) {
                        const uint64_t adesc = smem_desc(xa + kk * 32, 16, 1024, 2);
                        const uint64_t bdesc = smem_desc(wa + kk * 16 * 128, 8192, 1024, 2);
                        tc_mma(acc, adesc, bdesc, idesc, (ks | kk) ? 1u : 0u);
                    }
                    tc_commit(&empty[st]);
                }
                __syncwarp();
            }
            Segment seg;
            for (int s = next_pass(P, 0, m0, m0 + kLM, seg); s < P.n_segments;
                 s = next_pass(P, s + 1, m0, m0 + kLM, seg)) {
                {
                    const uint32_t st = it % kLStages;
                    mbar_wait<false>(&full[st], (it / kLStages) & 1u, P.dev_status, dead);
                    mbar_wait<false>(&vfull, pk & 1u, P.dev_status, dead);
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t ba = smem_u32(ring + st * kLStage + kLXBytes);
#pragma unroll
                        for (int kk = 0; kk < R / 16; ++kk) {
                            const uint64_t bdesc = smem_desc(ba + kk * 16 * 128, R * 128, 1024, 2);
                            tc_mma(acc, smem_desc(smem_u32(vhi) + kk * 32, 16, 1024, 2), bdesc, idesc, 1u);
                            tc_mma(acc, smem_desc(smem_u32(vlo) + kk * 32, 16, 1024, 2), bdesc, idesc, 1u);
                        }
                        tc_commit(&empty[st]);
                        tc_commit(&vempty);
                    }
                    __syncwarp();
                    ++it;
                    ++pk;
                }
            }
            if (lane == 0) tc_commit(&acc_full[buf]);
            __syncwarp();
        }
    } else {
        // ------------------------- V' operands and the epilogue -------------------------
        const int ew = warp - 2;             // 0..7
        const int quarter = warp & 3;        // TMEM lanes [32*quarter, +32)
        const int half = ew >> 2;            // columns [128*half, +128) of the tile
        const int et = ew * 32 + lane;       // 0..255 over the epilogue warps
        const int vrow = et >> 1;            // V' operand: row vrow, columns [vcol0, vcol0 + R/2)
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
        for (int u = first_unit; u < units; u += gridDim.x, ++local) {
            const int m0 = (u / P.n_tiles) * kLM, n0 = (u % P.n_tiles) * kLN;
            const int buf = local & 1;
            // the V' operands of this tile's delta passes, each written once the previous pass's
            // MMAs have read the buffer
            Segment seg;
            for (int s = next_pass(P, 0, m0, m0 + kLM, seg); s < P.n_segments;
                 s = next_pass(P, s + 1, m0, m0 + kLM, seg), ++pk) {
                const int g = m0 + vrow;
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
                if (lane == 0) mbar_arrive_local(&vfull);
            }
            // epilogue: row m of the tile, this warp's 128 columns
            mbar_wait<false>(&acc_full[buf], (local >> 1) & 1u, P.dev_status, dead);
            tc_fence_after();
            const int m = quarter * 32 + lane;
            const int g = m0 + m;
            const uint32_t taddr = tmem + (uint32_t(quarter * 32) << 16) + uint32_t(buf * kLN + half * 128);
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 32) {
                float a[32];
                tmem_ld32(taddr + c0, a);
                const int col = n0 + half * 128 + c0;
                if (g < P.T) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        if (col + ch * 8 < P.H2) {
                            float o[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) o[i] = a[ch * 8 + i];
                            st_vec(Y + size_t(g) * P.H2 + col + ch * 8, pack8<T>(o));
                        }
                    }
                }
            }
            // the TMEM reads completed at tcgen05.wait::ld: the buffer may take the next tile
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(&acc_empty[buf]);
        }
        if (!waited) pdl_wait();  // keep this grid behind its predecessor even without delta passes
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kLTmemCols) : "memory");
    if (threadIdx.x == 0) release_map_table(table);
}

template <typename T, int R>
inline cudaError_t launch_gemm_delta_kernel(const CUtensorMap& tmX, const CUtensorMap& tmW, const CUtensorMap& tmB,
                                            const GemmParams& P, int grid, cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(sgmv_gemm_delta_kernel<T, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kLSmem));
    });
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kLThreads, 1, 1);
    cfg.dynamicSmemBytes = kLSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.v_after_wait ? 1 : 0;  // overlap only the kernel that makes V
    return cudaLaunchKernelEx(&cfg, sgmv_gemm_delta_kernel<T, R>, tmX, tmW, tmB, P);
}

}  // namespace sgmv

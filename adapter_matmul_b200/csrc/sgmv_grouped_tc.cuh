// sgmv_grouped_tc.cuh -- grouped SGMV on the 5th-generation tensor cores (tcgen05, TMEM)
// for long segments (prefill).
//
// Maths (page “Punica：多 LoRA 模型统一服务框架”, the Punica README, its LoRA and multi-LoRA paragraphs): for each segment s with
// adapter i and every row t of it, Y[t,:] += scale * (X[t,:] @ A_i) @ B_i, A_i [H1, r],
// B_i [r, H2], row-major. With many rows per segment both halves are real matrix
// products: a [L, H1] x [H1, r] shrink and a [L, r] x [r, H2] expand per segment.
//
// One CTA computes one M-tile (128 rows of one segment) against one N-slice of H2:
//   shrink  D1[128 x r] (TMEM, fp32) = X[t0:t0+128, :] @ A_i, K-steps of 64;
//   V       the epilogue warps read D1 from TMEM and split it into two 16-bit
//           operands V_hi + V_lo (V_hi = round(D1), V_lo = round(D1 - V_hi)), so
//           the expand sees V to about 16 significant bits (the MMA takes 16-bit
//           operands; V itself is never rounded to one 16-bit value);
//   expand  D2[128 x 128] (TMEM, fp32) = V_hi @ B_tile + V_lo @ B_tile per N-tile,
//           in four TMEM buffers; the epilogue adds scale * D2 to the Y tile,
//           rounds once to the storage type and stores only rows inside the segment.
// Rows of a tile past the segment's end belong to the next segment (or past T, where
// TMA fills zeros); their results are discarded, so tiles never write across segments.
//
// Data movement. Every tile is a TMA load (cp.async.bulk.tensor) into the swizzled
// canonical layout the MMA descriptors describe: X and Y through tensor maps built per
// call, A_i and B_i (reached through a device table of pointers) through maps each CTA
// makes from a per-call template (sgmv_tmap.cuh). Warp roles: warp 0 producer, warp 1
// allocates TMEM and issues tcgen05.mma (one thread), warps 2..17 epilogue in two groups of
// eight (one TMEM lane quarter and one 64-column half of an N-tile per warp): group 0 makes
// V and takes the even N-tiles, group 1 the odd ones, so two tiles' epilogues (TMEM reads,
// the add onto the staged Y rows, the stores) overlap, and the MMAs run up to four N-tiles
// ahead of the epilogues (four D2 buffers). The host picks the number of N-slices per M-tile
// from the bytes the busiest SM streams (every slice re-reads its tile's X rows and A_i).
//
// Every mbarrier wait is bounded in time; a wait that gives up sets
// LORA_SGMV_DEV_TIMEOUT and the kernel runs to its end (TMEM is always freed).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "sgmv_common.cuh"
#include "sgmv_fused.cuh"  // PTX wrappers shared with the fused kernel (mbarriers, timers)
#include "sgmv_tmap.cuh"

namespace sgmv {

constexpr int kGroupedMinSegment = 128;  // dispatcher: longest segment at least one M-tile
constexpr int kGM = 128;                 // rows per M-tile (UMMA M)
constexpr int kGK = 64;                  // K per shrink stage (one 128-byte swizzle atom of 16-bit values)
constexpr int kGN = 128;                 // columns per expand N-tile
constexpr int kGMaxStages = 8;           // one ring for both phases: 2 K-steps or 1 N-tile per stage
constexpr int kGSmemMax = 225 * 1024;    // dynamic shared memory the ring and V may fill (+1 KB static)
constexpr int kGEpiWarps = 8;            // per group: two per TMEM lane quarter, one per 64-column half
constexpr int kGEpiGroups = 2;           // epilogue groups, taking alternate N-tiles
constexpr int kGThreads = 32 * (2 + kGEpiGroups * kGEpiWarps);  // producer, MMA issuer, epilogue groups
constexpr int kGD2Bufs = 4;              // D2 accumulators in TMEM (128 columns each; D1 shares buffer 0)
constexpr int kGTmemCols = 512;

inline bool grouped_tc_rank(int r) { return r == 16 || r == 32 || r == 64; }

inline bool grouped_tc_supported(int r, int H1, int H2, lora_sgmv_dtype dt) {
    (void)dt;
    return grouped_tc_rank(r) && H1 >= 64 && H2 >= 64 && H1 % 8 == 0 && H2 % 8 == 0;
}

struct GroupedParams {
    void* Y;
    const void* const* A_ptrs;
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
    int nsplit;  // N-slices of H2
    int nspan;   // columns per N-slice (multiple of kGN)
    int tm;      // rows per M-tile, 64..128, a multiple of 8 (the MMA's M stays 128; rows past tm are never used)
    float* v_out;  // V-only mode: V [T, r] fp32 written here, no expand
    const int32_t* ranks;  // rank of each adapter (device), or null: every adapter has rank R
    int x3d;       // tmX is the 3-D view {64, T, H1/64} (H1 a multiple of 64), box {64, tm, 2}
    int y3d;       // tmY {64, T, H2/64} and the B_i template {64, R, H2/64} are 3-D, boxes of 2 blocks
};

// Rank of the adapter of segment s when a rank table is given: 8 <= rank <= R, a multiple of 8
// (A_i rows of 16-byte multiples); 0 when it is not valid.
template <int R>
__device__ __forceinline__ int segment_rank(const GroupedParams& P, int s) {
    if (!P.ranks) return R;
    const int i = __ldg(P.lora_idx + s);
    if (i < 0 || i >= P.num_adapters) return 0;
    const int rs = __ldg(P.ranks + i);
    return (rs >= 8 && rs <= R && rs % 8 == 0) ? rs : 0;
}

// Ring stages are sized for the M-tile's tm rows (a multiple of 8), so short tiles give a
// deeper ring. Shrink stage: two K-steps, [X box 0][X box 1][A tile 0][A tile 1]: X boxes of
// tm rows x 64 columns (TMA, 128B swizzle, tm * 128 bytes each), A_i tiles [64 x R]
// (MN-major). Expand stage: [Y box 0][Y box 1][B_i tile]: the N-tile's Y rows as two boxes of
// tm rows x 64 columns, and B_i [R x 128] (MN-major). Every part starts on a 1024-byte
// boundary. The MMAs still read 128 rows (M = 128): an X operand spans 16 KB from its box,
// past the tm loaded rows into the rest of the ring or the V buffers after it, and the rows
// past tm only reach results that are discarded.
__host__ __device__ constexpr int grouped_a_slot(int r) { return (64 * r * 2 + 1023) / 1024 * 1024; }
__host__ __device__ constexpr int grouped_stage_bytes(int r, int tm) {
    return 2 * tm * 128 + (2 * grouped_a_slot(r) > r * kGN * 2 ? 2 * grouped_a_slot(r) : r * kGN * 2);
}
__host__ __device__ constexpr int grouped_stages(int r, int tm) {
    return (kGSmemMax - 1024 - 2 * kGM * r * 2) / grouped_stage_bytes(r, tm) < kGMaxStages
               ? (kGSmemMax - 1024 - 2 * kGM * r * 2) / grouped_stage_bytes(r, tm)
               : kGMaxStages;
}
__host__ __device__ constexpr size_t grouped_smem_bytes(int r, int tm) {
    return size_t(grouped_stages(r, tm)) * grouped_stage_bytes(r, tm) + 2 * size_t(kGM) * r * 2 +
           1024 /* alignment slack */;
}
static_assert(grouped_stages(64, 128) >= 4 && grouped_stages(16, 128) >= 4, "the ring holds at least four stages");
// the X operand read from box 1 of the last stage stays inside the allocation
static_assert(64 * 128 + kGM * 128 <= grouped_stage_bytes(16, 64) + 2 * kGM * 16 * 2, "X operand span");

template <int R>
struct GroupedGeom {
    static constexpr int A_BYTES = kGK * R * 2;
    static constexpr int A_SLOT = grouped_a_slot(R);
    static_assert(A_SLOT == A_BYTES, "one 128-row copy of A_i lands as the stage's two K-step tiles");
    static constexpr int B_BYTES = R * kGN * 2;
    static constexpr int V_BYTES = kGM * R * 2;  // one of V_hi, V_lo
    // swizzle of an MN-major A_i tile (rows of R 16-bit values) and of K-major V rows
    static constexpr int SW_BITS = R == 64 ? 3 : (R == 32 ? 2 : 1);           // 128B, 64B, 32B
    static constexpr uint64_t SW_TYPE = R == 64 ? 2 : (R == 32 ? 4 : 6);      // descriptor layout type
    static constexpr int ROW_BYTES = R * 2;                                   // bytes per row of R values
};

// ---- PTX wrappers specific to this kernel ---------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05): start, leading and stride byte offsets, layout.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint64_t layout) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3fff);
    d |= uint64_t((lbo >> 4) & 0x3fff) << 16;
    d |= uint64_t((sbo >> 4) & 0x3fff) << 32;
    d |= uint64_t(1) << 46;  // descriptor version for tcgen05
    d |= layout << 61;
    return d;
}

// Instruction descriptor, kind::f16: D fp32, A/B fp16 (0) or bf16 (1), majors, N, M.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t ab_format, uint32_t a_mn_major, uint32_t b_mn_major,
                                                   uint32_t N, uint32_t M) {
    return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
           ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// mbarrier arrives once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// byte offset of 16-byte chunk `chunk` of row `row` in a swizzled tile with rows of 16 << bits bytes
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk, int bits) {
    const uint32_t lin = row * (16u << bits) + chunk * 16u;
    return lin ^ (((lin >> 7) & ((1u << bits) - 1u)) << 4);
}

// Tile t (over all segments, 128 rows each) -> (segment, M-tile); false if t is past the last tile.
// Run by one whole warp.
__device__ bool find_tile(const GroupedParams& P, int tile, int& seg_out, int& mt_out) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int s0 = 0; s0 < P.n_segments; s0 += 32) {
        const int s = s0 + lane;
        int cnt = 0;
        if (s < P.n_segments) {
            const int b = __ldg(P.seg_starts + s), e = __ldg(P.seg_starts + s + 1);
            if (b >= 0 && b <= e && e <= P.T) cnt = (e - b + P.tm - 1) / P.tm;
        }
        int incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const int excl = base + incl - cnt;
        const unsigned hit = __ballot_sync(0xffffffffu, cnt > 0 && tile >= excl && tile < excl + cnt);
        if (hit) {
            const int src = __ffs(hit) - 1;
            seg_out = s0 + src;
            mt_out = tile - __shfl_sync(0xffffffffu, excl, src);
            return true;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    return false;
}

// Wait for a barrier phase without regard to earlier timeouts (lets copies land before the
// CTA exits); bounded like every other wait.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    uint64_t t0 = 0;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return;
        if ((i & 63u) == 63u) {
            const uint64_t now = globaltimer_ns();
            if (t0 == 0)
                t0 = now;
            else if (now - t0 > kWaitLimitNs)
                return;
        }
    }
}

// grid.x = tiles (upper bound) * nsplit; block kGThreads. tmA and tmB are templates of the
// A_i and B_i maps (shape, box, swizzle); each CTA makes its adapter's maps from them.
// V_OUT: the shrink alone -- V = X@A_i (fp32) of the tile's rows goes to P.v_out and there is
// no expand (nsplit must be 1); the whole-layer kernel (sgmv_gemm_tc.cuh) takes V from there.
template <typename T, int R, bool V_OUT = false>
__global__ void __launch_bounds__(kGThreads, 1)
    sgmv_grouped_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                           const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const GroupedParams P) {
    using G = GroupedGeom<R>;
    extern __shared__ __align__(1024) unsigned char gsmem_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char* gsmem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(gsmem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = grouped_stages(R, P.tm);           // ring stages
    const int SB = grouped_stage_bytes(R, P.tm);      // bytes per stage
    const int BOX = P.tm * 128;                       // one X or Y box of tm rows
    unsigned char* ring = gsmem;
    unsigned char* vhi = ring + size_t(NS) * SB;
    unsigned char* vlo = vhi + G::V_BYTES;

    __shared__ __align__(8) uint64_t full[kGMaxStages], empty[kGMaxStages];
    __shared__ __align__(8) uint64_t d1_full, v_full, d2_full[kGD2Bufs], d2_empty[kGD2Bufs];
    __shared__ __align__(128) CUtensorMap map_build[2];
    __shared__ uint32_t tmem_base_s;
    __shared__ int job_s[3];
    __shared__ int table_s;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tile = blockIdx.x / P.nsplit;
    if (V_OUT) pdl_launch_dependents();  // the whole-layer kernel may start on free SMs
    const int nsl = blockIdx.x - tile * P.nsplit;

    if (warp == 0) {
        int s = -1, mt = 0;
        const bool ok = find_tile(P, tile, s, mt);
        if (lane == 0) {
            job_s[0] = ok ? s : -1;
            job_s[1] = mt;
            Segment seg;
            if (ok && load_segment(P.seg_starts, P.lora_idx, P.A_ptrs, P.B_ptrs, s, P.T, P.num_adapters, seg))
                job_s[0] = -1;  // rejected segment: reported by CTA 0 below
            job_s[2] = job_s[0] >= 0 ? segment_rank<R>(P, s) : 0;
            if (job_s[2] == 0) job_s[0] = -1;  // a rank the kernel cannot take: reported below
        }
    }
    // every rejected segment reported once: by CTA 0's last epilogue warp, one lane per segment,
    // where that warp waits anyway (before its first expand tile, or on leaving without a tile)
    auto report_rejected = [&]() {
        if (blockIdx.x != 0 || warp != 9) return;
        for (int s2 = lane; s2 < P.n_segments; s2 += 32) {
            Segment seg;
            const uint32_t bad =
                load_segment(P.seg_starts, P.lora_idx, P.A_ptrs, P.B_ptrs, s2, P.T, P.num_adapters, seg);
            report(P.dev_status, bad ? bad : (segment_rank<R>(P, s2) ? 0u : LORA_SGMV_DEV_BAD_RANK));
        }
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);       // producer expect_tx; the TMA copies complete the bytes
            mbar_init(&empty[i], 1 + kGEpiWarps);  // MMA commit + 8 arrivals (the MMA thread for shrink
                                          // stages, the epilogue warps for expand stages)
        }
        mbar_init(&d1_full, 1);
        mbar_init(&v_full, kGEpiWarps);
        for (int i = 0; i < kGD2Bufs; ++i) {
            mbar_init(&d2_full[i], 1);
            mbar_init(&d2_empty[i], kGEpiWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        table_s = -1;
        if (job_s[0] >= 0) {
            table_s = claim_map_table();
            if (table_s < 0) {
                report(P.dev_status, LORA_SGMV_DEV_TIMEOUT);
                job_s[0] = -1;
            }
        }
    }
    __syncthreads();
    const int seg_id = job_s[0];
    if (seg_id < 0) {  // no tile here, or a rejected segment
        report_rejected();
        return;
    }
    const int mt = job_s[1];

    Segment seg;
    load_segment(P.seg_starts, P.lora_idx, P.A_ptrs, P.B_ptrs, seg_id, P.T, P.num_adapters, seg);
    const int t0 = seg.begin + mt * P.tm;
    const int rows = min(P.tm, seg.end - t0);  // valid rows of this tile
    const int n_lo = nsl * P.nspan;
    const int n_hi = min(P.H2, n_lo + P.nspan);
    const int n_tiles = (!V_OUT && n_lo < n_hi) ? (n_hi - n_lo + kGN - 1) / kGN : 0;
    const int k_steps = (P.H1 + kGK - 1) / kGK;
    const int s_stages = (k_steps + 1) / 2;  // shrink stages of two K-steps (the last may hold one)

    // TMEM: D2 buffers at columns 0, 128, 256 and 384; D1 at [0, R), inside buffer 0, which
    // the first expand MMA overwrites only after V has been read from it (v_full)
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kGTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    bool dead = false;

    if (warp == 0) {
        // ---------------------------------- producer ----------------------------------
        // this CTA's adapter maps, from the templates: A_i boxes of 64 rows x r, B_i boxes of
        // r rows x 64 columns; columns of B_i past this CTA's slice are loaded but never stored
        CUtensorMap* gA = &g_map_tables[table_s].m[0];
        CUtensorMap* gB = &g_map_tables[table_s].m[1];
        // the first stages' X tiles (through the host-made map) start before the adapter maps are
        // made; their A_i halves follow once the maps are published
        const int pre = min(NS, s_stages);
        auto issue_x = [&](int ss, unsigned char* xs) {  // lane 0: expect the stage's bytes, copy X
            const int nks = min(2, k_steps - 2 * ss);
            // X: one 3-D box of both K-steps when the view allows it (blocks past H1/64 read as
            // zeros), else one box per K-step; A_i (issued with the maps): one box of 128 rows
            const uint32_t xb = uint32_t(P.x3d ? 2 : nks) * uint32_t(BOX);
            mbar_arrive_expect_tx(&full[ss % NS], xb + 2u * G::A_BYTES);
            if (P.x3d) {
                tma_load_3d(xs, &tmX, 0, t0, 2 * ss, &full[ss % NS]);
            } else {
                for (int h = 0; h < nks; ++h) tma_load_2d(xs + h * BOX, &tmX, (2 * ss + h) * kGK, t0, &full[ss % NS]);
            }
        };
        if (lane == 0)
            for (int ss = 0; ss < pre; ++ss) issue_x(ss, ring + size_t(ss) * SB);
        __syncwarp();
        map_template_to_smem(&map_build[0], &tmA);
        map_template_to_smem(&map_build[1], &tmB);
        if (lane == 0) {
            map_set_address(&map_build[0], seg.a);
            map_set_address(&map_build[1], seg.b);
            if (P.ranks) {  // this adapter's own rank: columns (rows of B_i) past it read as zeros
                const int rs = job_s[2];
                map_set_dim<0>(&map_build[0], uint32_t(rs));
                map_set_stride<0>(&map_build[0], uint64_t(rs) * 2);
                map_set_dim<1>(&map_build[1], uint32_t(rs));
            }
        }
        __syncwarp();
        map_publish(gA, &map_build[0]);
        map_publish(gB, &map_build[1]);
        if (lane == 0) {
            map_acquire(gA);
            map_acquire(gB);
        }
        __syncwarp();
        uint32_t it = 0;
        for (int ss = 0; ss < s_stages; ++ss, ++it) {
            const uint32_t st = it % NS;
            if (it >= uint32_t(NS)) mbar_wait<false>(&empty[st], ((it / NS) - 1) & 1u, P.dev_status, dead);
            unsigned char* xs = ring + size_t(st) * SB;
            if (lane == 0) {
                if (ss >= pre) issue_x(ss, xs);
                tma_load_2d(xs + 2 * BOX, gA, 0, 2 * ss * kGK, &full[st]);  // rows past H1 read as zeros
            }
            __syncwarp();
        }
        for (int nt = 0; nt < n_tiles; ++nt, ++it) {
            const uint32_t st = it % NS;
            if (it >= uint32_t(NS)) mbar_wait<false>(&empty[st], ((it / NS) - 1) & 1u, P.dev_status, dead);
            unsigned char* ys = ring + size_t(st) * SB;
            unsigned char* bs = ys + 2 * BOX;
            const int n0 = n_lo + nt * kGN;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[st], 2u * P.tm * 64 * 2 + G::B_BYTES);
                if (P.y3d) {  // the N-tile's two 64-column blocks of Y and of B_i, one copy each
                    tma_load_3d(ys, &tmY, 0, t0, n0 / 64, &full[st]);
                    tma_load_3d(bs, gB, 0, 0, n0 / 64, &full[st]);
                } else {
                    tma_load_2d(ys, &tmY, n0, t0, &full[st]);
                    tma_load_2d(ys + BOX, &tmY, n0 + 64, t0, &full[st]);
                    tma_load_2d(bs, gB, n0, 0, &full[st]);
                    tma_load_2d(bs + R * 128, gB, n0 + 64, 0, &full[st]);
                }
            }
            __syncwarp();
        }
        // every copy issued lands before the CTA may exit
        if (lane == 0)
            for (uint32_t i = it > uint32_t(NS) ? it - NS : 0u; i < it; ++i)
                drain_wait(&full[i % NS], (i / NS) & 1u);
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------- MMA issuer ----------------------------------
        const uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
        const uint32_t idesc_s = instr_desc(fmt, 0, 1, R, kGM);    // X K-major, A_i MN-major, N = r
        const uint32_t idesc_e = instr_desc(fmt, 0, 1, kGN, kGM);  // V K-major, B_i MN-major, N = 128
        uint32_t it = 0;
        for (int ss = 0; ss < s_stages; ++ss, ++it) {
            const uint32_t st = it % NS;
            mbar_wait<false>(&full[st], (it / NS) & 1u, P.dev_status, dead);
            tc_fence_after();
            if (lane == 0) {
                const int nks = min(2, k_steps - 2 * ss);
                const uint32_t xa0 = smem_u32(ring + size_t(st) * SB);
                for (int h = 0; h < nks; ++h) {
                    const uint32_t xa = xa0 + h * BOX;
                    const uint32_t aa = xa0 + 2 * BOX + h * G::A_SLOT;
#pragma unroll
                    for (int kk = 0; kk < kGK / 16; ++kk) {
                        const uint64_t adesc = smem_desc(xa + kk * 32, 16, 1024, 2);
                        const uint64_t bdesc = smem_desc(aa + kk * 16 * G::ROW_BYTES, 16 * G::ROW_BYTES,
                                                         8 * G::ROW_BYTES, G::SW_TYPE);
                        tc_mma(tmem, adesc, bdesc, idesc_s, (ss | h | kk) ? 1u : 0u);
                    }
                }
                tc_commit(&empty[st]);
                for (int i = 0; i < kGEpiWarps; ++i) mbar_arrive_local(&empty[st]);
            }
            __syncwarp();
        }
        if (lane == 0) tc_commit(&d1_full);
        __syncwarp();
        mbar_wait<false>(&v_full, 0, P.dev_status, dead);
        tc_fence_after();
        for (int nt = 0; nt < n_tiles; ++nt, ++it) {
            const uint32_t st = it % NS;
            const int buf = nt % kGD2Bufs;
            if (nt >= kGD2Bufs) mbar_wait<false>(&d2_empty[buf], ((nt / kGD2Bufs) - 1) & 1u, P.dev_status, dead);
            mbar_wait<false>(&full[st], (it / NS) & 1u, P.dev_status, dead);
            tc_fence_after();
            if (lane == 0) {
                const uint32_t ba = smem_u32(ring + size_t(st) * SB + 2 * BOX);
                const uint32_t d2 = tmem + 128u * buf;
#pragma unroll
                for (int kk = 0; kk < R / 16; ++kk) {
                    const uint64_t bdesc = smem_desc(ba + kk * 16 * 128, R * 128, 1024, 2);
                    const uint64_t ahi = smem_desc(smem_u32(vhi) + kk * 32, 16, 8 * G::ROW_BYTES, G::SW_TYPE);
                    const uint64_t alo = smem_desc(smem_u32(vlo) + kk * 32, 16, 8 * G::ROW_BYTES, G::SW_TYPE);
                    tc_mma(d2, ahi, bdesc, idesc_e, kk ? 1u : 0u);
                    tc_mma(d2, alo, bdesc, idesc_e, 1u);
                }
                tc_commit(&d2_full[buf]);
                tc_commit(&empty[st]);
            }
            __syncwarp();
        }
    } else {
        // ---------------------------------- epilogue ----------------------------------
        report_rejected();
        const int grp = (warp - 2) / kGEpiWarps;         // this warp's group: N-tiles grp, grp + 2, ...
        const int quarter = warp & 3;                     // TMEM lanes [32*quarter, 32*quarter + 32)
        const int half = ((warp - 2) % kGEpiWarps) >> 2;  // columns [64*half, 64*half + 64) of its N-tiles
        const int m = quarter * 32 + lane;
        const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
        // V = D1 -> V_hi + V_lo (K-major, swizzled rows of R values), by group 0
        if (grp == 0) mbar_wait<false>(&d1_full, 0, P.dev_status, dead);
        tc_fence_after();
        for (int c0 = 32 * half; grp == 0 && c0 < R; c0 += 64) {  // the two halves share V's columns
            float v[32];
            tmem_ld32(lane_addr + c0, v);
            if (V_OUT) {
                if (m < rows) {
                    float* dst = P.v_out + size_t(t0 + m) * R + c0;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        if (c0 + i < R) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                }
            } else {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    if (c0 + ch * 8 >= R) break;
                    float hi[8], lo[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float x = v[ch * 8 + i];
                        const float h = Storage<T>::round(x);
                        hi[i] = h;
                        lo[i] = x - h;
                    }
                    const uint32_t off = swz(m, c0 / 8 + ch, G::SW_BITS);
                    st_vec(vhi + off, pack8<T>(hi));
                    st_vec(vlo + off, pack8<T>(lo));
                }
            }
        }
        if (grp == 0) {
            fence_proxy_async();  // generic-proxy writes of V -> tensor-core reads
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_local(&v_full);
        }

        T* __restrict__ Y = static_cast<T*>(P.Y);
        const bool row_ok = m < rows;
        for (int nt = grp; nt < n_tiles; nt += kGEpiGroups) {
            const uint32_t it = uint32_t(s_stages + nt);
            const uint32_t st = it % NS;
            const int buf = nt % kGD2Bufs;
            mbar_wait<false>(&full[st], (it / NS) & 1u, P.dev_status, dead);
            mbar_wait<false>(&d2_full[buf], (nt / kGD2Bufs) & 1u, P.dev_status, dead);
            tc_fence_after();
            unsigned char* ys = ring + size_t(st) * SB;
            const int n0 = n_lo + nt * kGN;
            // row m of the tile: y + scale * D2, written back over the staged Y row
#pragma unroll 1
            for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 32) {
                float acc[32];
                tmem_ld32(lane_addr + 128u * buf + c0, acc);
                if (row_ok) {
                    unsigned char* yb = ys + (c0 / 64) * BOX;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        if (n0 + c0 + ch * 8 < n_hi) {
                            unsigned char* yp = yb + swz(m, (c0 % 64) / 8 + ch, 3);
                            float y[8];
                            unpack8<T>(*reinterpret_cast<const uint4*>(yp), y);
#pragma unroll
                            for (int i = 0; i < 8; ++i) y[i] = __fadd_rn(y[i], __fmul_rn(P.scale, acc[ch * 8 + i]));
                            st_vec(yp, pack8<T>(y));
                        }
                    }
                }
            }
            __syncwarp();
            // this warp's 32 rows of its 64-column half leave row by row: 8 lanes per 128-byte
            // row segment, so each store instruction writes four whole segments
#pragma unroll
            for (int rq = 0; rq < 32; rq += 4) {
                const int rr = quarter * 32 + rq + (lane >> 3);
                const int c = lane & 7;
                const int col = n0 + half * 64 + c * 8;
                if (rr < rows && col < n_hi)
                    st_vec(Y + size_t(t0 + rr) * P.H2 + col,
                           *reinterpret_cast<const uint4*>(ys + half * BOX + swz(rr, c, 3)));
            }
            // the TMEM reads completed at tcgen05.wait::ld; no tcgen05 fence here (it would also
            // wait for the Y stores just issued)
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_relaxed(&d2_empty[buf]);
                mbar_arrive_relaxed(&empty[st]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGTmemCols) : "memory");
    if (threadIdx.x == 0) release_map_table(table_s);
}

// ---- host side ---------------------------------------------------------------------------

using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

// cuTensorMapEncodeTiled from the driver, looked up once (no link-time dependency on libcuda).
inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Row-major [rows, cols] 16-bit matrix, boxes of box_rows rows x 64 columns, 128-byte swizzle,
// zero fill outside the matrix.
inline bool make_tile_map(CUtensorMap* map, const void* base, int rows, int cols, lora_sgmv_dtype dt,
                          int box_rows = 128) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t gdim[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t gstride[1] = {cuuint64_t(cols) * 2};
    cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
    cuuint32_t estride[2] = {1, 1};
    const CUresult r = enc(map, dt == LORA_SGMV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                           2, const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename T, int R, bool V_OUT = false>
inline cudaError_t launch_grouped_tc_kernel(const CUtensorMap& tmX, const CUtensorMap& tmY, const CUtensorMap& tmA,
                                            const CUtensorMap& tmB, const GroupedParams& P, int blocks,
                                            cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(sgmv_grouped_tc_kernel<T, R, V_OUT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmemMax);
    });
    if (attr_err != cudaSuccess) return attr_err;
    if (P.tm < 64 || P.tm > kGM || P.tm % 8 != 0) return cudaErrorInvalidValue;  // the X span assumes tm >= 64
    // the V-only form has no expand: its second epilogue group would idle, so it is not launched
    const int threads = V_OUT ? 32 * (2 + kGEpiWarps) : kGThreads;
    sgmv_grouped_tc_kernel<T, R, V_OUT><<<blocks, threads, grouped_smem_bytes(R, P.tm), stream>>>(tmX, tmY, tmA, tmB,
                                                                                                  P);
    return cudaGetLastError();
}

}  // namespace sgmv

/*
 * lora_sgmv.h -- C ABI of the SGMV library for NVIDIA B200 (sm_100a).
 *
 * SGMV ("Segmented Gather Matrix-Vector multiplication", the Punica README
 * page "Punica：多 LoRA 模型统一服务框架", the paragraph that names the kernel) computes the LoRA term of a batch in which each token
 * uses its own adapter. The README's LoRA paragraph fixes the shapes: a
 * frozen weight W is [H1, H2]; an adapter adds A [H1, r] and B [r, H2];
 * y = x@(W + A@B) = x@W + x@A@B. Its multi-LoRA paragraph fixes the batch
 * form: Y = X@W + (x1@A1@B1, ..., xn@An@Bn). This library adds the second
 * term onto a Y that already holds X@W:
 *
 *     for every segment s, i = lora_idx[s], every row t in
 *     [seg_starts[s], seg_starts[s+1]):
 *         Y[t, :] += scale * (X[t, :] @ A_i) @ B_i
 *
 * computed as a shrink V = X@A_i (H1 -> r, fp32 result) and an expand
 * Y += scale * V@B_i (r -> H2) with the add fused in.
 *
 * Conventions shared by every entry point
 *   - Layout: all matrices row-major and dense. X is [T, H1], Y is [T, H2],
 *     V is [T, r] fp32, A_i is [H1, r], B_i is [r, H2]. Rows are tokens.
 *   - Storage type: fp16 or bf16 for X, Y, A_i, B_i (one type per call);
 *     products are accumulated in fp32; V is fp32 and never rounded; Y is
 *     rounded once, to nearest even, after the add.
 *   - Pointers marked "device" are CUDA device pointers on the current
 *     device; "host" pointers are ordinary CPU memory. The caller owns all
 *     memory. Nothing is retained after a call returns and the library never
 *     allocates device memory on the path of a call.
 *   - Adapter tables: A_ptrs and B_ptrs are device arrays of num_adapters
 *     device pointers; entry i points at A_i (resp. B_i). Adapters stay
 *     resident in device memory between calls; only the table is passed.
 *   - Segments: seg_starts is a device int32 array of n_segments+1 entries,
 *     lora_idx a device int32 array of n_segments entries. Segments may come
 *     in any order, may repeat an adapter, and may be empty (a no-op). Rows
 *     outside every segment are never written. Segments must not overlap
 *     (each row in at most one segment); overlapping rows give undefined
 *     results.
 *   - Asynchrony: every call only enqueues work on `stream` (a cudaStream_t
 *     passed as void*; NULL is the legacy default stream) and returns. The
 *     return value reports host-side validation and launch errors only; on
 *     any error nothing is launched.
 *   - Device-side checks: the segment arrays and pointer tables live on the
 *     device and are checked by the kernels, per segment. A segment with
 *     bounds outside 0 <= seg_starts[s] <= seg_starts[s+1] <= T, an adapter
 *     id outside [0, num_adapters), or a null or non-16-byte-aligned table
 *     entry is skipped and the matching LORA_SGMV_DEV_* bit is OR-ed into
 *     *dev_status (a device uint32; may be NULL). No kernel traps.
 *   - Alignment: X, Y, V and workspace must be 16-byte aligned; H1 and H2
 *     must be multiples of 8.
 *   - Overlap with the previous kernel: the fused kernels (variants FUSED
 *     and FUSED_TC, which AUTO picks for short segments, and the batched
 *     call) are launched with programmatic dependent launch, so their
 *     prologue (barriers, tensor memory, tables of tensor maps) overlaps the
 *     end of the kernel before them on the stream. By default they read
 *     nothing the caller passed until that kernel has completed, so any
 *     kernel may write any of a call's inputs right before it. With
 *     LORA_SGMV_FLAG_EARLY_READS (lora_sgmv_apply_flags,
 *     lora_sgmv_apply_batched_flags) the caller states that seg_starts,
 *     lora_idx, the pointer tables and the adapters are not written by the
 *     kernel launched immediately before the call on the same stream (copies
 *     and earlier kernels may write them); the kernels then start streaming
 *     adapter weights while that kernel still runs. X and Y are always read
 *     only after it has completed.
 *   - Thread safety: calls on different streams may run concurrently. The
 *     library keeps no mutable global state other than a lazily filled,
 *     mutex-guarded cache of device facts and kernel attributes, an atomic
 *     count of kernel launches, and, on every device that loads it, a fixed
 *     1 MiB array of tensor-map slots: the tensor-core kernels (GROUPED_TC,
 *     FUSED_TC) reach adapters through tensor maps they build on the device,
 *     and each of their CTAs claims a slot table with an atomic operation for
 *     its lifetime, so concurrent kernels never share a slot.
 */
#ifndef LORA_SGMV_H
#define LORA_SGMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LORA_SGMV_F16 = 0,
    LORA_SGMV_BF16 = 1
} lora_sgmv_dtype;

typedef enum {
    LORA_SGMV_OK = 0,
    LORA_SGMV_ERR_NULL = 1,        /* a required pointer is NULL */
    LORA_SGMV_ERR_DIM = 2,         /* a size is negative, zero where it must not be, or too large */
    LORA_SGMV_ERR_ALIGN = 3,       /* a pointer or a row pitch is not 16-byte aligned */
    LORA_SGMV_ERR_DTYPE = 4,       /* unknown storage type */
    LORA_SGMV_ERR_UNSUPPORTED = 5, /* rank r or variant not built into this library */
    LORA_SGMV_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed */
    LORA_SGMV_ERR_WORKSPACE = 7,   /* workspace missing or smaller than lora_sgmv_workspace_bytes() */
    LORA_SGMV_ERR_RANGE = 8        /* a host-side value is out of range (e.g. an adapter id) */
} lora_sgmv_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define LORA_SGMV_DEV_BAD_SEGMENT 0x1u  /* segment bounds invalid: segment skipped */
#define LORA_SGMV_DEV_BAD_ADAPTER 0x2u  /* lora_idx[s] outside [0, num_adapters): skipped */
#define LORA_SGMV_DEV_BAD_POINTER 0x4u  /* table entry NULL or not 16-byte aligned: skipped */
#define LORA_SGMV_DEV_TIMEOUT 0x8u      /* a bounded wait inside a kernel gave up: results invalid */
#define LORA_SGMV_DEV_BAD_RANK 0x10u    /* lora_sgmv_apply_ranks: the adapter's rank is not usable: skipped */

/* Flags of lora_sgmv_apply_flags and lora_sgmv_apply_batched_flags. */
#define LORA_SGMV_FLAG_EARLY_READS 0x1u /* segment arrays, tables and adapters are not written by the
                                           kernel launched right before the call: read them early */

/* Which kernels lora_sgmv_apply_ex runs. AUTO lets the dispatcher choose. */
typedef enum {
    LORA_SGMV_VARIANT_AUTO = 0,
    LORA_SGMV_VARIANT_SPLIT = 1,      /* split-K shrink kernel, then streaming expand kernel */
    LORA_SGMV_VARIANT_GROUPED_TC = 2, /* tcgen05/TMEM grouped kernel for long segments */
    LORA_SGMV_VARIANT_FUSED = 3,      /* one kernel: cluster shrink, V reduction on chip, expand (fp32 FMA) */
    LORA_SGMV_VARIANT_FUSED_TC = 4,   /* the same split on tcgen05, for segments of several tokens */
    LORA_SGMV_VARIANT_SPLIT_TC = 5    /* split-K shrink kernel (V into the workspace), then the
                                         tcgen05 expand with each segment's H2 split over
                                         independent CTAs: uses every SM when segments are few
                                         and B_i is large */
} lora_sgmv_variant;

/* Ranks r built into this library: 8, 16, 32, 64 and 128 for the split and
 * fused kernels; 16, 32 and 64 for the tensor-core kernels (GROUPED_TC,
 * FUSED_TC, SPLIT_TC). GROUPED_TC also needs H1 and H2 of at least 64;
 * FUSED_TC and SPLIT_TC need H1 and H2 to be multiples of 64 (at least 64),
 * and return LORA_SGMV_ERR_UNSUPPORTED otherwise. */
int32_t lora_sgmv_rank_supported(int32_t r, lora_sgmv_variant variant);

/* Human-readable name of a status code. Never NULL. */
const char* lora_sgmv_status_string(lora_sgmv_status status);

/* Text of the last CUDA error that a call made from this thread ran into
 * (the cause behind LORA_SGMV_ERR_CUDA), or "no CUDA error". Never NULL. */
const char* lora_sgmv_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int32_t lora_sgmv_version(void);

/* Number of kernels the library has launched successfully in this process
 * (all devices, all streams). For instrumentation: benchmarks read it before
 * and after a timed region. */
uint64_t lora_sgmv_launch_count(void);

/*
 * lora_sgmv_group_segments -- segment bookkeeping, on the host.
 *
 * Groups a batch of per-token adapter ids into contiguous segments (the
 * "segmented" part of SGMV): one segment per adapter that has tokens, in
 * ascending adapter id; tokens of one adapter keep their batch order.
 *
 *   ids          host, int32[T]: adapter id of each token, in batch order.
 *   T            number of tokens, >= 0.
 *   num_adapters ids must lie in [0, num_adapters); num_adapters >= 1.
 *   seg_starts   host, int32[num_adapters + 1] out: seg_starts[0] = 0,
 *                seg_starts[n] = T, strictly increasing.
 *   lora_idx     host, int32[num_adapters] out: adapter of each segment.
 *   perm         host, int32[T] out: perm[p] = batch index of the token that
 *                goes to row p of the grouped batch.
 *   n_segments   host, int32 out: n, the number of segments written.
 *
 * Returns LORA_SGMV_ERR_NULL, _DIM or _RANGE (an id out of range) without
 * writing the outputs, else LORA_SGMV_OK. Runs in O(T + num_adapters).
 */
lora_sgmv_status lora_sgmv_group_segments(const int32_t* ids, int32_t T, int32_t num_adapters,
                                          int32_t* seg_starts, int32_t* lora_idx, int32_t* perm,
                                          int32_t* n_segments);

/*
 * lora_sgmv_pad_rank -- one adapter of rank r_src, padded with zeros to rank r.
 *
 * Adapters of different ranks share one call once all are padded to one rank:
 * the authors' answer on different ranks (page "Punica: Serving multiple LoRA
 * finetuned LLM as one", the Hacker News thread) is padding, as the kernels
 * are bound by memory, not arithmetic. The padded adapter gives the original
 * adapter's result: the extra entries of V are zero and the extra terms of
 * each expand sum are zero (up to the sign of an exact zero sum).
 *   A_dst        device, [H1, r] out: A_dst[k, j] = A_src[k, j] for j < r_src,
 *                0 for r_src <= j < r.
 *   A_src        device, [H1, r_src].
 *   B_dst        device, [r, H2] out: B_dst[j, :] = B_src[j, :] for j < r_src,
 *                0 for r_src <= j < r.
 *   B_src        device, [r_src, H2].
 *   Either pair may be (NULL, NULL) to pad only the other matrix; H1 (H2) is
 *   then unused.
 *   H1, H2       sizes (>= 1 for each matrix given).
 *   r_src, r     1 <= r_src <= r; r_src == r copies.
 *   dtype        16-bit storage type of the four matrices.
 *   stream       cudaStream_t as void*; one kernel launch per matrix given.
 * A destination must not overlap its source. The padding kernel writes
 * adapters, so an SGMV call right after it on the same stream must not pass
 * LORA_SGMV_FLAG_EARLY_READS (the default calls wait for it to complete).
 * Returns LORA_SGMV_ERR_DTYPE,
 * _NULL (no pair given, or half a pair) or _DIM before any launch, _CUDA if a
 * launch fails, else LORA_SGMV_OK. Runs at adapter load time, not per call.
 */
lora_sgmv_status lora_sgmv_pad_rank(void* A_dst, const void* A_src, void* B_dst, const void* B_src,
                                    int32_t H1, int32_t H2, int32_t r_src, int32_t r,
                                    lora_sgmv_dtype dtype, void* stream);

/*
 * lora_sgmv_shrink -- V[t, :] = X[t, :] @ A_{lora_idx[s]} for rows t of each segment.
 *
 * The H1 -> r half of x@A@B (README LoRA paragraph), fp32 accumulation.
 *   V            device, fp32[T, r] out: rows of valid segments are
 *                overwritten; other rows are untouched.
 *   X            device, [T, H1] fp16/bf16.
 *   A_ptrs       device table of num_adapters device pointers to A_i [H1, r].
 *   seg_starts, lora_idx, n_segments, num_adapters: as in the conventions.
 *   T, H1, r     sizes; r must satisfy lora_sgmv_rank_supported(r, SPLIT).
 *   dtype        storage type of X and A_i.
 *   dev_status   device uint32 or NULL.
 *   stream       cudaStream_t as void*.
 */
lora_sgmv_status lora_sgmv_shrink(float* V, const void* X, const void* const* A_ptrs,
                                  const int32_t* seg_starts, const int32_t* lora_idx,
                                  int32_t n_segments, int32_t num_adapters, int32_t T, int32_t H1,
                                  int32_t r, lora_sgmv_dtype dtype, uint32_t* dev_status,
                                  void* stream);

/*
 * lora_sgmv_expand -- Y[t, :] = round(Y[t, :] + scale * V[t, :] @ B_{lora_idx[s]}).
 *
 * The r -> H2 half, with the add onto the base output fused in; one rounding
 * to the storage type per element.
 *   Y            device, [T, H2] fp16/bf16, in/out.
 *   V            device, fp32[T, r] (e.g. from lora_sgmv_shrink).
 *   B_ptrs       device table of num_adapters device pointers to B_i [r, H2].
 *   scale        multiplies the fp32 sum once, before the add.
 *   other arguments as for lora_sgmv_shrink.
 */
lora_sgmv_status lora_sgmv_expand(void* Y, const float* V, const void* const* B_ptrs,
                                  const int32_t* seg_starts, const int32_t* lora_idx,
                                  int32_t n_segments, int32_t num_adapters, int32_t T, int32_t r,
                                  int32_t H2, float scale, lora_sgmv_dtype dtype,
                                  uint32_t* dev_status, void* stream);

/* Bytes of workspace lora_sgmv_apply needs for T tokens at rank r (fp32 V,
 * padded to 256 bytes). 0 if T or r is not positive. */
size_t lora_sgmv_workspace_bytes(int32_t T, int32_t r);

/*
 * lora_sgmv_apply -- Y[t, :] += scale * (X[t, :] @ A_i) @ B_i, the whole SGMV.
 *
 *   Y, X, A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters,
 *   T, H1, r, H2, scale, dtype, dev_status, stream: as above.
 *   max_seg_len  host hint: an upper bound on any segment's length, used only
 *                to choose kernels and grid shapes; <= 0 means unknown (the
 *                dispatcher then assumes ceil(T / n_segments)). Results do
 *                not depend on it: a wrong hint costs speed, not correctness.
 *   workspace    device scratch of at least lora_sgmv_workspace_bytes(T, r)
 *                bytes, 16-byte aligned, owned by the caller; its contents
 *                on entry do not matter. Calls that share a workspace must be
 *                ordered on one stream.
 */
lora_sgmv_status lora_sgmv_apply(void* Y, const void* X, const void* const* A_ptrs,
                                 const void* const* B_ptrs, const int32_t* seg_starts,
                                 const int32_t* lora_idx, int32_t n_segments, int32_t num_adapters,
                                 int32_t T, int32_t H1, int32_t r, int32_t H2, float scale,
                                 lora_sgmv_dtype dtype, int32_t max_seg_len, void* workspace,
                                 size_t workspace_bytes, uint32_t* dev_status, void* stream);

/*
 * lora_sgmv_auto_variant -- the kernels lora_sgmv_apply (variant AUTO) runs for
 * a call of these sizes on a GPU with sm_count SMs. Host arithmetic only: no
 * CUDA call, no device needed.
 *   T, n_segments, H1, r, H2, dtype, max_seg_len: as for lora_sgmv_apply.
 *   sm_count     the device's multiprocessor count (148 on a B200).
 * The rule: the longest segment (max_seg_len, else ceil(T / n_segments)) of
 * at least 128 rows with r in {16, 32, 64} and H1, H2 >= 64 -> GROUPED_TC; else more than
 * 8192 segments -> SPLIT; else segments of more than 2 tokens, r >= 32 and
 * H1, H2 multiples of 64 -> SPLIT_TC when there are fewer jobs (16-token
 * chunks, or segments when none is longer than 16) than SMs and each B_i
 * holds at least 1,000,000 bytes (r * H2 * 2), else FUSED_TC; else FUSED.
 * Returns LORA_SGMV_VARIANT_AUTO when a size or sm_count is not positive or
 * dtype is unknown.
 */
lora_sgmv_variant lora_sgmv_auto_variant(int32_t T, int32_t n_segments, int32_t H1, int32_t r,
                                         int32_t H2, lora_sgmv_dtype dtype, int32_t max_seg_len,
                                         int32_t sm_count);

/* lora_sgmv_apply with the kernels chosen by the caller. GROUPED_TC returns
 * LORA_SGMV_ERR_UNSUPPORTED for ranks or types it does not cover. */
lora_sgmv_status lora_sgmv_apply_ex(void* Y, const void* X, const void* const* A_ptrs,
                                    const void* const* B_ptrs, const int32_t* seg_starts,
                                    const int32_t* lora_idx, int32_t n_segments,
                                    int32_t num_adapters, int32_t T, int32_t H1, int32_t r,
                                    int32_t H2, float scale, lora_sgmv_dtype dtype,
                                    int32_t max_seg_len, void* workspace, size_t workspace_bytes,
                                    uint32_t* dev_status, lora_sgmv_variant variant, void* stream);

/* lora_sgmv_apply_ex with flags: 0 or LORA_SGMV_FLAG_EARLY_READS (see
 * "Overlap with the previous kernel" above). Other bits return
 * LORA_SGMV_ERR_UNSUPPORTED. Flags change timing only, never results, as long
 * as the caller's statement holds. */
lora_sgmv_status lora_sgmv_apply_flags(void* Y, const void* X, const void* const* A_ptrs,
                                       const void* const* B_ptrs, const int32_t* seg_starts,
                                       const int32_t* lora_idx, int32_t n_segments,
                                       int32_t num_adapters, int32_t T, int32_t H1, int32_t r,
                                       int32_t H2, float scale, lora_sgmv_dtype dtype,
                                       int32_t max_seg_len, void* workspace, size_t workspace_bytes,
                                       uint32_t* dev_status, lora_sgmv_variant variant,
                                       uint32_t flags, void* stream);

/* One projection of a batched call (see lora_sgmv_apply_batched). */
typedef struct {
    void* Y;                      /* device, [T, H2], in/out */
    const void* X;                /* device, [T, H1] */
    const void* const* A_ptrs;    /* device table of num_adapters pointers to A_i [H1, r] */
    const void* const* B_ptrs;    /* device table of num_adapters pointers to B_i [r, H2] */
    int32_t num_adapters;
    int32_t H1;
    int32_t H2;
    float scale;
} lora_sgmv_problem;

/* Most problems lora_sgmv_apply_batched takes in one call. */
#define LORA_SGMV_MAX_PROBLEMS 8

/*
 * lora_sgmv_apply_batched -- several SGMV problems that share one token
 * grouping (e.g. the q, k, v and o projections of a decoder layer, whose
 * tokens map to the same adapters) in a single kernel launch.
 *
 * For every problem p and segment s, rows t of the segment:
 *     problems[p].Y[t, :] += problems[p].scale * (problems[p].X[t, :] @ A_i) @ B_i
 * with i = lora_idx[s] and A_i, B_i taken from problem p's tables. Each
 * problem may have its own H1, H2, tables and adapter count; r and dtype are
 * shared. Runs a fused kernel, which keeps V on chip and needs no
 * workspace: LORA_SGMV_VARIANT_FUSED_TC when max_seg_len > 2, r >= 32 and
 * every problem suits the tensor-core kernel, else LORA_SGMV_VARIANT_FUSED. It
 * takes at most 8192 segments (LORA_SGMV_ERR_DIM beyond).
 *   problems     host array of n_problems entries, 1 <= n_problems <= 8.
 *   other arguments as for lora_sgmv_apply.
 * Validation errors of any problem are returned before anything is launched.
 */
lora_sgmv_status lora_sgmv_apply_batched(const lora_sgmv_problem* problems, int32_t n_problems,
                                         const int32_t* seg_starts, const int32_t* lora_idx,
                                         int32_t n_segments, int32_t T, int32_t r,
                                         lora_sgmv_dtype dtype, int32_t max_seg_len,
                                         uint32_t* dev_status, void* stream);

/* lora_sgmv_apply_batched with flags, as for lora_sgmv_apply_flags. */
lora_sgmv_status lora_sgmv_apply_batched_flags(const lora_sgmv_problem* problems, int32_t n_problems,
                                               const int32_t* seg_starts, const int32_t* lora_idx,
                                               int32_t n_segments, int32_t T, int32_t r,
                                               lora_sgmv_dtype dtype, int32_t max_seg_len,
                                               uint32_t flags, uint32_t* dev_status, void* stream);

/*
 * lora_sgmv_apply_ranks -- lora_sgmv_apply for adapters of different ranks, unpadded.
 *
 * The authors' reply on adapters of different ranks (page "Punica: Serving
 * multiple LoRA finetuned LLM as one", the Hacker News thread) names a grouped
 * GEMM whose groups have their own sizes. Here adapter i keeps its own rank
 * r_i: A_i is [H1, r_i] and B_i is [r_i, H2], dense, no padded copy. The
 * grouped tensor-core kernel runs at rank r_max; each tile's tensor maps take
 * the adapter's own extent and row pitch, so the columns of A_i (rows of B_i)
 * past r_i are read as zeros by the copy engine and add nothing. The result is
 * the adapter's own product at its own rank.
 *   ranks        device, int32[num_adapters]: r_i, with 8 <= r_i <= r_max
 *                and r_i a multiple of 8 (rows of A_i in whole 16-byte units).
 *                A segment whose adapter has another rank is skipped and
 *                LORA_SGMV_DEV_BAD_RANK is set in *dev_status.
 *   r_max        16, 32 or 64 (LORA_SGMV_ERR_UNSUPPORTED otherwise).
 *   H1, H2       at least 64, multiples of 8.
 *   other arguments as for lora_sgmv_apply; no workspace (V stays on chip).
 * The grouped kernel is built for long segments (prefill); it is correct for
 * any segment length, but decode batches run faster padded to one rank
 * (lora_sgmv_pad_rank) through lora_sgmv_apply.
 */
lora_sgmv_status lora_sgmv_apply_ranks(void* Y, const void* X, const void* const* A_ptrs,
                                       const void* const* B_ptrs, const int32_t* ranks,
                                       const int32_t* seg_starts, const int32_t* lora_idx,
                                       int32_t n_segments, int32_t num_adapters, int32_t T, int32_t H1,
                                       int32_t r_max, int32_t H2, float scale, lora_sgmv_dtype dtype,
                                       uint32_t* dev_status, void* stream);

/*
 * lora_sgmv_gemm_apply -- the whole LoRA layer: Y = X@W + scale * (X@A_i)@B_i.
 *
 * The README's multi-LoRA paragraph writes the batch as Y = X@W plus the
 * per-row adapter terms, and its LoRA paragraph gives x@(W + A@B) = x@W +
 * x@A@B. This call computes both terms in one tensor-core accumulation: after
 * V = X@A_i (fp32, into the workspace, by the grouped kernel's shrink for
 * long segments or the split-K shrink), each output tile of X@W takes 2r more
 * K-steps per adapter whose segment touches the tile, with scale * V carried
 * as two 16-bit operands (about 16 significant bits). Y is rounded once to the
 * storage type and written; it is an output, not read. So the delta costs no
 * read and no write of Y beyond the base product's own write.
 *   Y            device, [T, H2] out: every row written; rows in no valid
 *                segment get round(X@W).
 *   X            device, [T, H1].
 *   W            device, [H1, H2] row-major, the frozen base weight.
 *   A_ptrs, B_ptrs, seg_starts, lora_idx, n_segments, num_adapters, T,
 *   scale, dtype, max_seg_len, dev_status, stream: as for lora_sgmv_apply.
 *   H1, H2       multiples of 8 (LORA_SGMV_ERR_ALIGN otherwise).
 *   r            16, 32 or 64 (LORA_SGMV_ERR_UNSUPPORTED otherwise).
 *   workspace    device scratch of lora_sgmv_workspace_bytes(T, r) bytes for V
 *                (may be NULL when n_segments is 0).
 * X, Y and W must be 16-byte aligned. Runs two kernels on `stream` (one when
 * n_segments is 0). Rejected segments are reported in *dev_status and their
 * rows get the base product alone.
 */
lora_sgmv_status lora_sgmv_gemm_apply(void* Y, const void* X, const void* W, const void* const* A_ptrs,
                                      const void* const* B_ptrs, const int32_t* seg_starts,
                                      const int32_t* lora_idx, int32_t n_segments, int32_t num_adapters,
                                      int32_t T, int32_t H1, int32_t r, int32_t H2, float scale,
                                      lora_sgmv_dtype dtype, int32_t max_seg_len, void* workspace,
                                      size_t workspace_bytes, uint32_t* dev_status, void* stream);

/*
 * lora_sgmv_apply_noalloc -- lora_sgmv_apply for callers that cannot allocate.
 *
 * The Punica README has no counterpart to this entry point; it exists for
 * callers that may not call cudaMalloc (or any allocator) where they run
 * SGMV -- for example a serving loop whose device memory is fixed at
 * start-up, or a plugin whose host framework owns all device memory -- and
 * so cannot supply the workspace lora_sgmv_apply needs.
 *
 * It runs the split kernels (LORA_SGMV_VARIANT_SPLIT) with their fp32 V
 * scratch in a fixed array inside the library: 1,048,576 floats (4 MiB),
 * which every GPU that loads the library holds until the process exits. It
 * allocates nothing. Arguments are those of lora_sgmv_apply without the
 * workspace; T * r above 1,048,576 is rejected with LORA_SGMV_ERR_WORKSPACE
 * before anything is launched.
 *
 * The first call on each device looks up the array's device address (once
 * per device, with that device current); make that first call before any
 * stream capture. The address is kept until the process exits: after a
 * cudaDeviceReset the array may move, so do not call this entry point again
 * on a device that was reset. Every call on a device shares the one array and leaves
 * its last contents there (nothing in it needs to start at zero: each call
 * writes every V row it reads). Calls whose kernels overlap on the GPU --
 * on different streams, or from different threads -- race on the array and
 * give wrong results: order them on one stream.
 */
lora_sgmv_status lora_sgmv_apply_noalloc(void* Y, const void* X, const void* const* A_ptrs,
                                         const void* const* B_ptrs, const int32_t* seg_starts,
                                         const int32_t* lora_idx, int32_t n_segments,
                                         int32_t num_adapters, int32_t T, int32_t H1, int32_t r,
                                         int32_t H2, float scale, lora_sgmv_dtype dtype,
                                         int32_t max_seg_len, uint32_t* dev_status, void* stream);

/* One copy for lora_sgmv_step_host: bytes from src to dst. */
typedef struct {
    const void* src;
    void* dst;
    size_t bytes;
} lora_sgmv_copy;

/*
 * lora_sgmv_step_host -- one serving step whose batch lives in host memory.
 *
 * The segmented batch of the multi-LoRA paragraph (page "Punica：多 LoRA
 * 模型统一服务框架", the Punica README) as one call a serving loop makes per
 * step, with every piece enqueued on `stream` and nothing waited for:
 *   1. groups ids (host, int32[T], the adapter of each batch token) as
 *      lora_sgmv_group_segments does, writing seg_starts (n + 1 entries)
 *      then lora_idx (n entries) to meta_host[0 .. 2n + 1), and perm to
 *      `perm` (host, int32[T]; NULL: not returned). Rows of every problem's
 *      X and Y are taken in grouped order: row p belongs to batch token
 *      perm[p];
 *   2. copies h2d[0 .. n_h2d) host -> device in order (cudaMemcpyAsync);
 *      one of them must carry meta_host to meta_dev, and they must fill the
 *      problems' X and Y;
 *   3. runs lora_sgmv_apply_batched_flags(problems, n_problems, meta_dev,
 *      meta_dev + n + 1, n, T, r, dtype, the longest segment, flags,
 *      dev_status) unless n == 0;
 *   4. copies d2h[0 .. n_d2h) device -> host in order.
 *   meta_host    host, int32[2 * num_adapters + 1]; pinned, so that its copy
 *                is asynchronous.
 *   meta_dev     device, int32[2 * num_adapters + 1].
 *   h2d, d2h     host arrays of copies (src, dst, bytes); the host side of
 *                each should be pinned memory.
 *   n_segments_out  host, int32 out (may be NULL): n.
 *   other arguments as for lora_sgmv_apply_batched_flags.
 * meta_host and every host range must not be written (nor, for d2h, read)
 * until the step's copies are done: record an event on `stream` after the
 * call and wait for it. Returns LORA_SGMV_ERR_NULL, _DIM or _RANGE (an id
 * out of range) before anything is enqueued; LORA_SGMV_ERR_CUDA when a copy
 * cannot be enqueued (cudaGetLastError holds the cause); a launch error of
 * step 3 after the copies in were enqueued (the copies out are then not
 * enqueued); else LORA_SGMV_OK.
 */
lora_sgmv_status lora_sgmv_step_host(const int32_t* ids, int32_t T, int32_t num_adapters,
                                     int32_t* meta_host, const int32_t* meta_dev, int32_t* perm,
                                     const lora_sgmv_copy* h2d, int32_t n_h2d,
                                     const lora_sgmv_problem* problems, int32_t n_problems, int32_t r,
                                     lora_sgmv_dtype dtype, uint32_t flags, const lora_sgmv_copy* d2h,
                                     int32_t n_d2h, uint32_t* dev_status, int32_t* n_segments_out,
                                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_SGMV_H */

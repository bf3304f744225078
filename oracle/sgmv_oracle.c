/*
 * sgmv_oracle.c -- CPU oracle for SGMV (Segmented Gather Matrix-Vector
 * multiplication), the multi-LoRA delta of Punica.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file. Only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark use it. It shares no code, header, table or
 * helper with the CUDA library: its storage-type conversions below are its
 * own, written from the IEEE 754 binary16 definition and from bfloat16 being
 * the upper half of an IEEE binary32.
 *
 * What it computes (the Punica README page, "Punica：多 LoRA 模型统一服务框架",
 * its LoRA paragraph and the multi-LoRA batch paragraph after it):
 *   - a frozen weight W of shape [H1, H2]; an adapter adds A of shape [H1, r]
 *     and B of shape [r, H2]; y = x @ (W + A@B) = x@W + x@A@B (row vectors);
 *   - with n adapters (A_1, B_1) ... (A_n, B_n) and a batch X whose input x_j
 *     maps to its own adapter, Y = X@W + (x_1@A_1@B_1, ..., x_n@A_n@B_n);
 *   - SGMV computes the right-hand term for a batch split into contiguous
 *     segments, segment s (rows seg_starts[s] .. seg_starts[s+1]-1) using
 *     adapter lora_idx[s], and adds it onto the base output already in Y.
 *
 * oracle_base_plus_delta_f32 computes the whole batch form, Y = X@W plus the
 * delta, for the layer that fuses the delta into the base product.
 *
 * The kernel contract adds a scale factor: Y[t,:] += scale * (X[t,:]@A_i)@B_i.
 * The product is taken as (x@A)@B -- shrink H1 -> r, then expand r -> H2 --
 * which is the association the README's identity writes.
 *
 * Precision. Two twins of the same loops:
 *   *_f32: fp16/bf16 storage in, fp32 accumulation, the r-wide intermediate V
 *          kept in fp32 (never rounded), scale applied once to the fp32 expand
 *          sum, one round-to-nearest-even to the storage type at the end;
 *          sums in ascending k (shrink) and ascending j (expand).
 *   *_f64: the same loops in binary64, for error analysis and for the
 *          algebraic pins (products of two fp16 or bf16 values are exact in
 *          binary64; only the sums round).
 * Build with -ffp-contract=off so that a*b+c is two roundings, as written.
 *
 * Segment rules (the library's contract, restated): a segment with
 * seg_starts[s] > seg_starts[s+1], bounds outside [0, T], or an adapter id
 * outside [0, num_adapters) is skipped and counted; zero-length segments are
 * no-ops; rows in no segment are never written; an adapter may appear in
 * several segments.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* ---------------------------------------------------------------------- */
/* Storage-type conversions                                                 */
/* ---------------------------------------------------------------------- */

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/2^10) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_to_double(uint16_t b)
{
    int sign = b >> 15;
    int e = (b >> 7) & 0xff;
    int m = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133);                /* subnormal: m * 2^-133 */
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), e - 134);     /* (1 + m/2^7) * 2^(e-127) */
    return sign ? -v : v;
}

/*
 * Round a binary64 value to a binary format with `frac_bits` stored fraction
 * bits and exponent bias `bias` (max biased exponent 2*bias+1 is inf/nan),
 * round-to-nearest, ties to even. Overflow gives +-inf like a cast.
 */
static uint16_t round_to_format(double v, int frac_bits, int bias)
{
    const int exp_all_ones = 2 * bias + 1;
    uint16_t sign = signbit(v) ? (uint16_t)0x8000u : (uint16_t)0; /* bit 15 in both formats */
    const int exp_shift = frac_bits;
    const uint16_t inf_bits = (uint16_t)(exp_all_ones << exp_shift);
    if (isnan(v))
        return (uint16_t)(sign | inf_bits | (1u << (frac_bits - 1)));
    double a = fabs(v);
    if (isinf(a))
        return (uint16_t)(sign | inf_bits);
    const double min_normal = ldexp(1.0, 1 - bias);
    if (a < min_normal) {
        /* subnormal grid: multiples of 2^(1 - bias - frac_bits); scaling is exact */
        double m = ldexp(a, bias - 1 + frac_bits);
        double r = nearbyint(m); /* default rounding mode: nearest, ties to even */
        return (uint16_t)(sign | (uint16_t)r); /* r == 2^frac_bits encodes the min normal */
    }
    int e;
    double f = frexp(a, &e);            /* a = f * 2^e, f in [0.5, 1) */
    double m = ldexp(f, frac_bits + 1); /* significand in [2^fb, 2^(fb+1)), exact */
    double r = nearbyint(m);
    int E = e - 1;
    if (r == ldexp(1.0, frac_bits + 1)) { /* rounded up to the next binade */
        r = ldexp(1.0, frac_bits);
        E += 1;
    }
    int biased = E + bias;
    if (biased >= exp_all_ones)
        return (uint16_t)(sign | inf_bits);
    return (uint16_t)(sign | (uint16_t)(biased << exp_shift) | (uint16_t)((int)r - (1 << frac_bits)));
}

uint16_t oracle_double_to_f16(double v) { return round_to_format(v, 10, 15); }
uint16_t oracle_double_to_bf16(double v) { return round_to_format(v, 7, 127); }

static double decode(uint16_t bits, int dtype)
{
    return dtype == ORACLE_F16 ? oracle_f16_to_double(bits) : oracle_bf16_to_double(bits);
}

static uint16_t encode(double v, int dtype)
{
    return dtype == ORACLE_F16 ? oracle_double_to_f16(v) : oracle_double_to_bf16(v);
}

/* Array forms, used by the Python wrapper and the pins. */
void oracle_decode_array(const uint16_t* in, double* out, int64_t n, int dtype)
{
    for (int64_t i = 0; i < n; ++i) out[i] = decode(in[i], dtype);
}

void oracle_encode_array(const double* in, uint16_t* out, int64_t n, int dtype)
{
    for (int64_t i = 0; i < n; ++i) out[i] = encode(in[i], dtype);
}

/* ---------------------------------------------------------------------- */
/* Segment bookkeeping                                                      */
/* ---------------------------------------------------------------------- */

/*
 * Group a batch of per-token adapter ids into contiguous segments, one per
 * adapter that has tokens, in ascending adapter id; tokens of one adapter keep
 * their batch order. Outputs: seg_starts[n+1] (seg_starts[0] = 0,
 * seg_starts[n] = T), lora_idx[n], perm[T] with perm[p] = the batch index of
 * the token placed at position p. Buffers must hold num_adapters+1,
 * num_adapters and T entries. Returns 0, or -1 if an id is out of range.
 * Written as the plain double loop (adapters outer, tokens inner).
 */
int oracle_group_segments(const int32_t* ids, int32_t T, int32_t num_adapters,
                          int32_t* seg_starts, int32_t* lora_idx, int32_t* perm,
                          int32_t* n_segments)
{
    for (int32_t t = 0; t < T; ++t)
        if (ids[t] < 0 || ids[t] >= num_adapters) return -1;
    int32_t pos = 0, n = 0;
    seg_starts[0] = 0;
    for (int32_t a = 0; a < num_adapters; ++a) {
        int32_t start = pos;
        for (int32_t t = 0; t < T; ++t)
            if (ids[t] == a) perm[pos++] = t;
        if (pos > start) {
            lora_idx[n] = a;
            seg_starts[++n] = pos;
        }
    }
    *n_segments = n;
    return 0;
}

static int segment_valid(const int32_t* seg_starts, const int32_t* lora_idx, int32_t s,
                         int32_t T, int32_t num_adapters)
{
    int32_t b = seg_starts[s], e = seg_starts[s + 1], i = lora_idx[s];
    return b >= 0 && b <= e && e <= T && i >= 0 && i < num_adapters;
}

/* ---------------------------------------------------------------------- */
/* fp32-accumulate twin                                                     */
/* ---------------------------------------------------------------------- */

/*
 * Shrink: V[t, j] = sum_k X[t, k] * A_i[k, j] for every row t of segment s,
 * i = lora_idx[s]; k ascending; fp32. X is [T, H1], A_i is [H1, r], V is
 * [T, r], all row-major. Rows of V outside every segment are not written.
 * Returns the number of skipped (invalid) segments.
 */
int oracle_shrink_f32(float* V, const uint16_t* X, const uint16_t* const* A,
                      const int32_t* seg_starts, const int32_t* lora_idx, int32_t n_segments,
                      int32_t num_adapters, int32_t T, int32_t H1, int32_t r, int dtype)
{
    int skipped = 0;
    float* xrow = (float*)malloc(sizeof(float) * (size_t)H1);
    for (int32_t s = 0; s < n_segments; ++s) {
        if (!segment_valid(seg_starts, lora_idx, s, T, num_adapters)) { ++skipped; continue; }
        const uint16_t* Ai = A[lora_idx[s]];
        for (int32_t t = seg_starts[s]; t < seg_starts[s + 1]; ++t) {
            float* v = V + (size_t)t * r;
            for (int32_t j = 0; j < r; ++j) v[j] = 0.0f;
            for (int32_t k = 0; k < H1; ++k) xrow[k] = (float)decode(X[(size_t)t * H1 + k], dtype);
            for (int32_t k = 0; k < H1; ++k) {
                const float xk = xrow[k];
                const uint16_t* arow = Ai + (size_t)k * r;
                for (int32_t j = 0; j < r; ++j) v[j] += xk * (float)decode(arow[j], dtype);
            }
        }
    }
    free(xrow);
    return skipped;
}

/*
 * Expand with the fused add: Y[t, c] = round(Y[t, c] + scale * sum_j V[t, j] * B_i[j, c])
 * for every row t of segment s; j ascending; fp32; one round-to-nearest-even to the
 * storage type. V is [T, r] fp32, B_i is [r, H2], Y is [T, H2], row-major.
 */
int oracle_expand_f32(uint16_t* Y, const float* V, const uint16_t* const* B,
                      const int32_t* seg_starts, const int32_t* lora_idx, int32_t n_segments,
                      int32_t num_adapters, int32_t T, int32_t r, int32_t H2, float scale, int dtype)
{
    int skipped = 0;
    for (int32_t s = 0; s < n_segments; ++s) {
        if (!segment_valid(seg_starts, lora_idx, s, T, num_adapters)) { ++skipped; continue; }
        const uint16_t* Bi = B[lora_idx[s]];
        for (int32_t t = seg_starts[s]; t < seg_starts[s + 1]; ++t) {
            const float* v = V + (size_t)t * r;
            uint16_t* y = Y + (size_t)t * H2;
            for (int32_t c = 0; c < H2; ++c) {
                float acc = 0.0f;
                for (int32_t j = 0; j < r; ++j) acc += v[j] * (float)decode(Bi[(size_t)j * H2 + c], dtype);
                const float delta = scale * acc;
                const float out = (float)decode(y[c], dtype) + delta;
                y[c] = encode((double)out, dtype);
            }
        }
    }
    return skipped;
}

/* apply = shrink then expand; V lives in a buffer of the oracle's own. */
int oracle_apply_f32(uint16_t* Y, const uint16_t* X, const uint16_t* const* A,
                     const uint16_t* const* B, const int32_t* seg_starts, const int32_t* lora_idx,
                     int32_t n_segments, int32_t num_adapters, int32_t T, int32_t H1, int32_t r,
                     int32_t H2, float scale, int dtype)
{
    float* V = (float*)calloc((size_t)T * (size_t)r + 1, sizeof(float));
    int skipped = oracle_shrink_f32(V, X, A, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r, dtype);
    oracle_expand_f32(Y, V, B, seg_starts, lora_idx, n_segments, num_adapters, T, r, H2, scale, dtype);
    free(V);
    return skipped;
}

/* ---------------------------------------------------------------------- */
/* binary64 twin                                                            */
/* ---------------------------------------------------------------------- */

/* Same loops as oracle_shrink_f32 in binary64; V is [T, r] double. */
int oracle_shrink_f64(double* V, const uint16_t* X, const uint16_t* const* A,
                      const int32_t* seg_starts, const int32_t* lora_idx, int32_t n_segments,
                      int32_t num_adapters, int32_t T, int32_t H1, int32_t r, int dtype)
{
    int skipped = 0;
    for (int32_t s = 0; s < n_segments; ++s) {
        if (!segment_valid(seg_starts, lora_idx, s, T, num_adapters)) { ++skipped; continue; }
        const uint16_t* Ai = A[lora_idx[s]];
        for (int32_t t = seg_starts[s]; t < seg_starts[s + 1]; ++t) {
            double* v = V + (size_t)t * r;
            for (int32_t j = 0; j < r; ++j) v[j] = 0.0;
            for (int32_t k = 0; k < H1; ++k) {
                const double xk = decode(X[(size_t)t * H1 + k], dtype);
                const uint16_t* arow = Ai + (size_t)k * r;
                for (int32_t j = 0; j < r; ++j) v[j] += xk * decode(arow[j], dtype);
            }
        }
    }
    return skipped;
}

/*
 * Same loops as oracle_expand_f32 in binary64, with Y held in binary64 and not
 * rounded: Y[t, c] += scale * sum_j V[t, j] * B_i[j, c]. The caller rounds with
 * oracle_encode_array when it wants storage values.
 */
int oracle_expand_f64(double* Y, const double* V, const uint16_t* const* B,
                      const int32_t* seg_starts, const int32_t* lora_idx, int32_t n_segments,
                      int32_t num_adapters, int32_t T, int32_t r, int32_t H2, double scale, int dtype)
{
    int skipped = 0;
    for (int32_t s = 0; s < n_segments; ++s) {
        if (!segment_valid(seg_starts, lora_idx, s, T, num_adapters)) { ++skipped; continue; }
        const uint16_t* Bi = B[lora_idx[s]];
        for (int32_t t = seg_starts[s]; t < seg_starts[s + 1]; ++t) {
            const double* v = V + (size_t)t * r;
            double* y = Y + (size_t)t * H2;
            for (int32_t c = 0; c < H2; ++c) {
                double acc = 0.0;
                for (int32_t j = 0; j < r; ++j) acc += v[j] * decode(Bi[(size_t)j * H2 + c], dtype);
                y[c] += scale * acc;
            }
        }
    }
    return skipped;
}

int oracle_apply_f64(double* Y, const uint16_t* X, const uint16_t* const* A, const uint16_t* const* B,
                     const int32_t* seg_starts, const int32_t* lora_idx, int32_t n_segments,
                     int32_t num_adapters, int32_t T, int32_t H1, int32_t r, int32_t H2,
                     double scale, int dtype)
{
    double* V = (double*)calloc((size_t)T * (size_t)r + 1, sizeof(double));
    int skipped = oracle_shrink_f64(V, X, A, seg_starts, lora_idx, n_segments, num_adapters, T, H1, r, dtype);
    oracle_expand_f64(Y, V, B, seg_starts, lora_idx, n_segments, num_adapters, T, r, H2, scale, dtype);
    free(V);
    return skipped;
}

/*
 * One output element of the fp32 twin, computed on its own: the value that
 * oracle_apply_f32 writes to Y[t, c] when row t lies in segment s. Used to
 * check sampled outputs of full-size problems without running the whole batch.
 * Returns the storage bits; y_in is the base value's bits.
 */
uint16_t oracle_apply_f32_element(const uint16_t* x_row, const uint16_t* Ai, const uint16_t* Bi,
                                  uint16_t y_in, int32_t H1, int32_t r, int32_t H2, int32_t c,
                                  float scale, int dtype)
{
    float v[512];
    if (r > 512) return 0xffff;
    for (int32_t j = 0; j < r; ++j) v[j] = 0.0f;
    for (int32_t k = 0; k < H1; ++k) {
        const float xk = (float)decode(x_row[k], dtype);
        for (int32_t j = 0; j < r; ++j) v[j] += xk * (float)decode(Ai[(size_t)k * r + j], dtype);
    }
    float acc = 0.0f;
    for (int32_t j = 0; j < r; ++j) acc += v[j] * (float)decode(Bi[(size_t)j * H2 + c], dtype);
    const float delta = scale * acc;
    const float out = (float)decode(y_in, dtype) + delta;
    return encode((double)out, dtype);
}

/* ---------------------------------------------------------------------- */
/* The whole layer: base product plus the delta                             */
/* ---------------------------------------------------------------------- */

/*
 * Y = X@W + (x_t@A_i@B_i)_t, the multi-LoRA batch of the README's multi-LoRA
 * paragraph with the kernel contract's scale: for every row t,
 *   base[c] = sum_k X[t, k] * W[k, c]               (fp32, k ascending)
 * and, when row t lies in a valid segment s with adapter i = lora_idx[s],
 *   v[j]    = sum_k X[t, k] * A_i[k, j]             (fp32, k ascending)
 *   acc[c]  = sum_j v[j] * B_i[j, c]                (fp32, j ascending)
 *   Y[t, c] = round(base[c] + scale * acc[c])
 * else Y[t, c] = round(base[c]). W is [H1, H2] row-major; Y is written, not
 * read. A row covered by several segments gets the delta of the last one
 * (segments must not overlap). Returns the number of skipped segments.
 */
int oracle_base_plus_delta_f32(uint16_t* Y, const uint16_t* X, const uint16_t* W,
                               const uint16_t* const* A, const uint16_t* const* B,
                               const int32_t* seg_starts, const int32_t* lora_idx,
                               int32_t n_segments, int32_t num_adapters, int32_t T, int32_t H1,
                               int32_t r, int32_t H2, float scale, int dtype)
{
    int skipped = 0;
    int32_t* owner = (int32_t*)malloc(sizeof(int32_t) * ((size_t)T + 1));
    float* base = (float*)malloc(sizeof(float) * ((size_t)H2 + 1));
    float* xrow = (float*)malloc(sizeof(float) * ((size_t)H1 + 1));
    float* v = (float*)malloc(sizeof(float) * ((size_t)r + 1));
    for (int32_t t = 0; t < T; ++t) owner[t] = -1;
    for (int32_t s = 0; s < n_segments; ++s) {
        if (!segment_valid(seg_starts, lora_idx, s, T, num_adapters)) { ++skipped; continue; }
        for (int32_t t = seg_starts[s]; t < seg_starts[s + 1]; ++t) owner[t] = lora_idx[s];
    }
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < H1; ++k) xrow[k] = (float)decode(X[(size_t)t * H1 + k], dtype);
        for (int32_t c = 0; c < H2; ++c) base[c] = 0.0f;
        for (int32_t k = 0; k < H1; ++k) {
            const float xk = xrow[k];
            const uint16_t* wrow = W + (size_t)k * H2;
            for (int32_t c = 0; c < H2; ++c) base[c] += xk * (float)decode(wrow[c], dtype);
        }
        uint16_t* y = Y + (size_t)t * H2;
        if (owner[t] < 0) {
            for (int32_t c = 0; c < H2; ++c) y[c] = encode((double)base[c], dtype);
            continue;
        }
        const uint16_t* Ai = A[owner[t]];
        const uint16_t* Bi = B[owner[t]];
        for (int32_t j = 0; j < r; ++j) v[j] = 0.0f;
        for (int32_t k = 0; k < H1; ++k) {
            const float xk = xrow[k];
            const uint16_t* arow = Ai + (size_t)k * r;
            for (int32_t j = 0; j < r; ++j) v[j] += xk * (float)decode(arow[j], dtype);
        }
        for (int32_t c = 0; c < H2; ++c) {
            float acc = 0.0f;
            for (int32_t j = 0; j < r; ++j) acc += v[j] * (float)decode(Bi[(size_t)j * H2 + c], dtype);
            const float delta = scale * acc;
            y[c] = encode((double)(base[c] + delta), dtype);
        }
    }
    free(owner);
    free(base);
    free(xrow);
    free(v);
    return skipped;
}

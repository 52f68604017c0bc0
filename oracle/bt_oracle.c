/*
 * CPU oracle for the ternary-weight FWHT-1024 path -- TEST INFRASTRUCTURE.
 *
 * Plain, slow, obviously correct FP64 C. Only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the CUDA library never does,
 * and this file shares no code, header, table or constant with it.
 *
 * What each function follows (pages cited by title and section):
 *
 *  - oracle_pack / oracle_unpack: the base-3 byte code of the Bonsai low-bit
 *    course (adenzhou1350.github.io/learn/bonsai-low-bit), section
 *    "先用五个数字理解 1.6bit": trit t in {-1,0,1} maps to digit t+1, five
 *    digits form code = sum_i (t_i + 1) * 3^i with i = 0 the first trit, and
 *    t_i = floor(code / 3^i) mod 3 - 1 restores them (example: [-1,0,1,-1,1]
 *    -> 183). Groups of 128 weights along K (one FP16 scale each, "g128",
 *    Ternary Bonsai 2 27B release summary, section 三值权重怎么压缩到 1.76
 *    bit) are packed as 26 bytes: 25 full bytes plus one byte holding the
 *    group's last 3 trits and two zero-valued pad trits (digit 1).
 *    The plain 2-bit layout stores digit t+1 in bits [2i, 2i+1] of byte
 *    i/4, 32 bytes per group; digit 3 is invalid.
 *    The continuous base-3 layout packs a row's trits five to a byte with no
 *    break at group boundaries (byte j holds trits 5j .. 5j+4 of the row, so
 *    a byte may hold trits of two groups): ceil(K/5) bytes, the last byte's
 *    trits past K are pads (digit 1), and the row is padded with zero bytes
 *    to a multiple of 16 bytes. This is the accounting behind the release
 *    summary's 1.72 bit for ternary + g128 (section 三值权重怎么压缩到 1.76
 *    bit): 8/5 bit per trit plus 16/128 for the scales, 1.725 bit at
 *    K = 5120; the per-group layout above spends 26 + 2 bytes per 128
 *    weights, 1.75 bit.
 *
 *  - oracle_hadamard: H[i][j] = (-1)^popcount(i & j), the closed form of the
 *    Sylvester recursion H_2n = [[H, H], [H, -H]] printed (with H4) in the
 *    TensorSharp blog (2kiu.com/news/5337570), section 3.2.
 *
 *  - oracle_rotate_matrix: x'_b = (1/sqrt(1024)) * H_1024 * (S . x_b) for every
 *    1024-long block b of each row, R = (1/sqrt n) H_n S from the release
 *    summary, section 三值权重怎么压缩到 1.76 bit ("f(x) = W(Rx)").
 *    Explicit matrix-vector product, O(n^2) per block.
 *
 *  - oracle_rotate_butterfly: the same rotation by the in-place butterfly
 *    (pairs (a, b) -> (a + b, a - b) at half-widths 1, 2, ..., n/2, then
 *    divide by sqrt n), as described in the TensorSharp blog, section 5.2.
 *    It exists so large inputs finish; tests tie it to the matrix form.
 *
 *  - oracle_ternarize: the offline weight path. Every row of a float W
 *    [N][K] is first rotated into the fixed basis block-wise, w'_b =
 *    (1/sqrt 1024) H_1024 (S . w_b) (release summary, section 三值权重怎么压缩到
 *    1.76 bit: the weights are transformed to R = (1/sqrt n) H_n S before
 *    ternarisation and the activation gets the same R at inference), so that
 *    W' R ~ W. Then every group of 128 rotated weights v gets a scale and a
 *    threshold by the rule of the TensorSharp blog (2kiu.com/news/5337570),
 *    section 2.1: t_i = 0 where |v_i / s| is below the threshold, sign(v_i)
 *    elsewhere, with s derived from the mean |v| and the threshold chosen by
 *    searching candidates for the smallest reconstruction error. Reading
 *    taken here: candidate thresholds tau_j = (j / 20) * mean|v|, j = 1..40;
 *    for each, the trits t_i = sign(v_i) where |v_i| >= tau_j, the scale the
 *    least-squares one for those trits (the mean |v| over the non-zero
 *    trits), rounded to FP16, and the error sum_i (v_i - s t_i)^2 with that
 *    FP16 scale; the smallest error wins, the smallest j on ties. A group of
 *    zeros gets s = 0 and zero trits. All in FP64, sums in index order.
 *
 *  - oracle_gemv: y[m][n] = sum_k w[n][k] * x'[m][k] with
 *    w[n][k] = scale[n][k/128] * t[n][k] (dense dequantisation, FP64), and the
 *    acceptance bound B[m][n] = 2e-3 * sum_k |w[n][k] x'[m][k]| + 1e-5.
 *    Naive triple loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_GROUP 128
#define ORACLE_BLOCK 1024

enum { ORACLE_LAYOUT_BASE3 = 0, ORACLE_LAYOUT_2BIT = 1, ORACLE_LAYOUT_BASE3_CONT = 2 };

enum {
    ORACLE_OK = 0,
    ORACLE_BAD_SHAPE = 1,
    ORACLE_BAD_TRIT = 2,
    ORACLE_BAD_CODE = 3,
    ORACLE_BAD_PAD = 4,
    ORACLE_BAD_LAYOUT = 5
};

int oracle_bytes_per_group(int layout)
{
    if (layout == ORACLE_LAYOUT_BASE3) return 26;
    if (layout == ORACLE_LAYOUT_2BIT) return 32;
    return -1;
}

/* ---- scalar conversions (bit patterns -> double) ---- */

double oracle_f16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)mant, -24);              /* subnormal: mant * 2^-24 */
    } else if (expo == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + mant), expo - 25); /* (1 + mant/1024) 2^(e-15) */
    }
    return sign ? -v : v;
}

double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void oracle_f16_array_to_double(const uint16_t* h, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_double(h[i]);
}

void oracle_bf16_array_to_double(const uint16_t* b, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_double(b[i]);
}

/* ---- packing ---- */

static int pow3(int i)
{
    int p = 1;
    while (i-- > 0) p *= 3;
    return p;
}

/* bytes of one packed row */
int64_t oracle_row_bytes(int layout, int64_t K)
{
    if (K % ORACLE_GROUP != 0 || K < 0) return -1;
    if (layout == ORACLE_LAYOUT_BASE3_CONT) {
        int64_t used = (K + 4) / 5;
        return (used + 15) / 16 * 16;
    }
    int bpg = oracle_bytes_per_group(layout);
    return bpg < 0 ? -1 : K / ORACLE_GROUP * bpg;
}

static int pack_cont(const int8_t* trits, int64_t N, int64_t K, uint8_t* codes)
{
    int64_t rb = oracle_row_bytes(ORACLE_LAYOUT_BASE3_CONT, K), used = (K + 4) / 5;
    for (int64_t i = 0; i < N * K; ++i)
        if (trits[i] < -1 || trits[i] > 1) return ORACLE_BAD_TRIT;
    for (int64_t n = 0; n < N; ++n) {
        const int8_t* t = trits + n * K;
        uint8_t* out = codes + n * rb;
        for (int64_t j = 0; j < rb; ++j) {
            int code = 0;
            if (j < used)
                for (int i = 0; i < 5; ++i) {
                    int64_t k = 5 * j + i;
                    int trit = k < K ? t[k] : 0;
                    code += (trit + 1) * pow3(i);
                }
            out[j] = (uint8_t)code;
        }
    }
    return ORACLE_OK;
}

static int unpack_cont(const uint8_t* codes, int64_t N, int64_t K, int8_t* trits)
{
    int64_t rb = oracle_row_bytes(ORACLE_LAYOUT_BASE3_CONT, K), used = (K + 4) / 5;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t* in = codes + n * rb;
        int8_t* t = trits + n * K;
        for (int64_t j = 0; j < rb; ++j) {
            int code = in[j];
            if (j >= used) {
                if (code != 0) return ORACLE_BAD_PAD;
                continue;
            }
            if (code >= 243) return ORACLE_BAD_CODE;
            for (int i = 0; i < 5; ++i) {
                int digit = (code / pow3(i)) % 3;
                int64_t k = 5 * j + i;
                if (k < K) t[k] = (int8_t)(digit - 1);
                else if (digit != 1) return ORACLE_BAD_PAD;
            }
        }
    }
    return ORACLE_OK;
}

int oracle_pack(int layout, const int8_t* trits, int64_t N, int64_t K, uint8_t* codes)
{
    if (K % ORACLE_GROUP != 0 || N < 0 || K < 0) return ORACLE_BAD_SHAPE;
    if (layout == ORACLE_LAYOUT_BASE3_CONT) return pack_cont(trits, N, K, codes);
    int bpg = oracle_bytes_per_group(layout);
    if (bpg < 0) return ORACLE_BAD_LAYOUT;
    int64_t groups = K / ORACLE_GROUP;
    for (int64_t i = 0; i < N * K; ++i)
        if (trits[i] < -1 || trits[i] > 1) return ORACLE_BAD_TRIT;

    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < groups; ++g) {
            const int8_t* t = trits + n * K + g * ORACLE_GROUP;
            uint8_t* out = codes + (n * groups + g) * bpg;
            if (layout == ORACLE_LAYOUT_BASE3) {
                /* byte b holds trits 5b .. 5b+4; positions past 127 are pads (trit 0) */
                for (int b = 0; b < 26; ++b) {
                    int code = 0;
                    for (int i = 0; i < 5; ++i) {
                        int k = 5 * b + i;
                        int trit = (k < ORACLE_GROUP) ? t[k] : 0;
                        code += (trit + 1) * pow3(i);
                    }
                    out[b] = (uint8_t)code;
                }
            } else {
                for (int b = 0; b < 32; ++b) {
                    int code = 0;
                    for (int i = 0; i < 4; ++i) code |= (t[4 * b + i] + 1) << (2 * i);
                    out[b] = (uint8_t)code;
                }
            }
        }
    }
    return ORACLE_OK;
}

int oracle_unpack(int layout, const uint8_t* codes, int64_t N, int64_t K, int8_t* trits)
{
    if (K % ORACLE_GROUP != 0 || N < 0 || K < 0) return ORACLE_BAD_SHAPE;
    if (layout == ORACLE_LAYOUT_BASE3_CONT) return unpack_cont(codes, N, K, trits);
    int bpg = oracle_bytes_per_group(layout);
    if (bpg < 0) return ORACLE_BAD_LAYOUT;
    int64_t groups = K / ORACLE_GROUP;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < groups; ++g) {
            const uint8_t* in = codes + (n * groups + g) * bpg;
            int8_t* t = trits + n * K + g * ORACLE_GROUP;
            if (layout == ORACLE_LAYOUT_BASE3) {
                for (int b = 0; b < 26; ++b) {
                    int code = in[b];
                    if (code >= 243) return ORACLE_BAD_CODE;
                    for (int i = 0; i < 5; ++i) {
                        int digit = (code / pow3(i)) % 3;
                        int k = 5 * b + i;
                        if (k < ORACLE_GROUP) t[k] = (int8_t)(digit - 1);
                        else if (digit != 1) return ORACLE_BAD_PAD;
                    }
                }
            } else {
                for (int b = 0; b < 32; ++b) {
                    for (int i = 0; i < 4; ++i) {
                        int digit = (in[b] >> (2 * i)) & 3;
                        if (digit == 3) return ORACLE_BAD_CODE;
                        t[4 * b + i] = (int8_t)(digit - 1);
                    }
                }
            }
        }
    }
    return ORACLE_OK;
}

/* ---- Hadamard and the rotation R = (1/sqrt n) H_n S ---- */

static int parity_of_and(int64_t i, int64_t j)
{
    uint64_t v = (uint64_t)(i & j);
    int p = 0;
    while (v) { p ^= 1; v &= v - 1; }
    return p;
}

/* H[i][j] = (-1)^popcount(i & j), n a power of two (n x n, int8, row-major). */
int oracle_hadamard(int64_t n, int8_t* H)
{
    if (n < 1 || (n & (n - 1)) != 0) return ORACLE_BAD_SHAPE;
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < n; ++j) H[i * n + j] = parity_of_and(i, j) ? -1 : 1;
    return ORACLE_OK;
}

/* Explicit matrix form: xr[m][b*n + i] = (1/sqrt n) sum_j H[i][j] S[j] x[m][b*n + j]. */
int oracle_rotate_matrix(const double* x, const int8_t* S, int64_t M, int64_t K, double* xr)
{
    const int64_t n = ORACLE_BLOCK;
    if (K % n != 0 || M < 0) return ORACLE_BAD_SHAPE;
    int8_t* H = (int8_t*)malloc((size_t)(n * n));
    if (!H) return ORACLE_BAD_SHAPE;
    oracle_hadamard(n, H);
    const double inv_sqrt_n = 1.0 / sqrt((double)n);
    int64_t nblocks = K / n;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < nblocks; ++b) {
            const double* xb = x + m * K + b * n;
            double* ob = xr + m * K + b * n;
            for (int64_t i = 0; i < n; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < n; ++j) acc += (double)H[i * n + j] * ((double)S[j] * xb[j]);
                ob[i] = acc * inv_sqrt_n;
            }
        }
    }
    free(H);
    return ORACLE_OK;
}

/* Butterfly form of the same rotation. */
int oracle_rotate_butterfly(const double* x, const int8_t* S, int64_t M, int64_t K, double* xr)
{
    const int64_t n = ORACLE_BLOCK;
    if (K % n != 0 || M < 0) return ORACLE_BAD_SHAPE;
    const double inv_sqrt_n = 1.0 / sqrt((double)n);
    int64_t nblocks = K / n;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < nblocks; ++b) {
            double v[ORACLE_BLOCK];
            const double* xb = x + m * K + b * n;
            for (int64_t j = 0; j < n; ++j) v[j] = (double)S[j] * xb[j];
            for (int64_t half = 1; half < n; half *= 2) {
                for (int64_t start = 0; start < n; start += 2 * half) {
                    for (int64_t j = start; j < start + half; ++j) {
                        double a = v[j], c = v[j + half];
                        v[j] = a + c;
                        v[j + half] = a - c;
                    }
                }
            }
            double* ob = xr + m * K + b * n;
            for (int64_t j = 0; j < n; ++j) ob[j] = v[j] * inv_sqrt_n;
        }
    }
    return ORACLE_OK;
}

/* ---- FP16 rounding and the offline ternarisation ---- */

/* double -> FP16 bit pattern, round to nearest, ties to even (overflow -> inf) */
uint16_t oracle_double_to_f16(double v)
{
    uint16_t sign = 0;
    if (v < 0 || (v == 0 && signbit(v))) { sign = 0x8000; v = -v; }
    if (isnan(v)) return 0x7E00;
    if (v == 0) return sign;
    /* the FP16 grid near v: exponent e with 2^e <= v < 2^(e+1), clamped to
     * the subnormal range; spacing 2^(e-10) */
    int e;
    frexp(v, &e);  /* v = f * 2^e, f in [0.5, 1) -> 2^(e-1) <= v < 2^e */
    e -= 1;
    if (e < -14) e = -14;
    double ulp = ldexp(1.0, e - 10);
    double q = v / ulp;                /* exact: a power-of-two division */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double rounded = r * ulp;          /* may carry into the next binade: fine */
    if (rounded >= 65520.0) return (uint16_t)(sign | 0x7C00);  /* beyond the largest finite half */
    /* encode */
    if (rounded < ldexp(1.0, -14)) {   /* subnormal (or the smallest normal after rounding) */
        int m = (int)(rounded / ldexp(1.0, -24));
        if (m >= 1024) return (uint16_t)(sign | 0x0400);
        return (uint16_t)(sign | m);
    }
    int ee;
    double ff = frexp(rounded, &ee);   /* rounded = ff * 2^ee, ff in [0.5, 1) */
    int m = (int)((ff * 2.0 - 1.0) * 1024.0 + 0.5);
    int biased = ee - 1 + 15;
    return (uint16_t)(sign | (biased << 10) | m);
}

int oracle_ternarize(const double* W, const int8_t* S, int64_t N, int64_t K, int8_t* trits, uint16_t* scales)
{
    if (K % ORACLE_BLOCK != 0 || N < 0) return ORACLE_BAD_SHAPE;
    double* Wr = (double*)malloc((size_t)(N * K) * sizeof(double));
    if (!Wr && N * K > 0) return ORACLE_BAD_SHAPE;
    int rc = oracle_rotate_butterfly(W, S, N, K, Wr);
    if (rc != ORACLE_OK) { free(Wr); return rc; }
    const int64_t groups = K / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (int64_t gi = 0; gi < N * groups; ++gi) {
        const int64_t n = gi / groups, g = gi % groups;
        const double* v = Wr + n * K + g * ORACLE_GROUP;
        int8_t* t = trits + n * K + g * ORACLE_GROUP;
        double mean = 0.0;
        for (int i = 0; i < ORACLE_GROUP; ++i) mean += fabs(v[i]);
        mean = mean / ORACLE_GROUP;
        int best_j = 0;
        double best_err = 0.0;
        uint16_t best_s = 0;
        for (int j = 1; j <= 40; ++j) {
            const double tau = ((double)j / 20.0) * mean;
            double sum = 0.0;
            int nnz = 0;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                if (fabs(v[i]) >= tau) { sum += fabs(v[i]); ++nnz; }
            }
            const uint16_t s16 = nnz ? oracle_double_to_f16(sum / nnz) : 0;
            const double s = oracle_f16_to_double(s16);
            double err = 0.0;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                const double q = fabs(v[i]) >= tau ? (v[i] < 0 ? -s : s) : 0.0;
                const double d = v[i] - q;
                err += d * d;
            }
            if (j == 1 || err < best_err) { best_err = err; best_j = j; best_s = s16; }
        }
        if (mean == 0.0) best_s = 0;   /* a group of zeros: no scale, zero trits */
        const double tau = ((double)best_j / 20.0) * mean;
        for (int i = 0; i < ORACLE_GROUP; ++i)
            t[i] = (mean != 0.0 && fabs(v[i]) >= tau) ? (v[i] < 0 ? -1 : 1) : 0;
        scales[n * groups + g] = best_s;
    }
    free(Wr);
    return ORACLE_OK;
}

/* ---- dequantisation and the product ---- */

int oracle_dequant(const int8_t* trits, const uint16_t* scales, int64_t N, int64_t K, double* W)
{
    if (K % ORACLE_GROUP != 0) return ORACLE_BAD_SHAPE;
    int64_t groups = K / ORACLE_GROUP;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            W[n * K + k] = oracle_f16_to_double(scales[n * groups + k / ORACLE_GROUP]) * (double)trits[n * K + k];
    return ORACLE_OK;
}

/*
 * y[m][n] = sum_k w[n][k] xr[m][k]; bound[m][n] = 2e-3 sum_k |w[n][k] xr[m][k]| + 1e-5.
 * trits int8 [N][K], scales fp16 bits [N][K/128], xr double [M][K], y/bound double [M][N].
 * bound may be NULL.
 */
int oracle_gemv(const int8_t* trits, const uint16_t* scales, const double* xr,
                int64_t M, int64_t N, int64_t K, double* y, double* bound)
{
    if (K % ORACLE_GROUP != 0) return ORACLE_BAD_SHAPE;
    int64_t groups = K / ORACLE_GROUP;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double w = oracle_f16_to_double(scales[n * groups + k / ORACLE_GROUP]) * (double)trits[n * K + k];
                double p = w * xr[m * K + k];
                acc += p;
                mag += fabs(p);
            }
            y[m * N + n] = acc;
            if (bound) bound[m * N + n] = 2e-3 * mag + 1e-5;
        }
    }
    return ORACLE_OK;
}

int oracle_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the parallel loops above use from now on (timing only). */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

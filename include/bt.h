/*
 * bt.h -- C ABI of libbt.so: ternary-weight GEMV/GEMM behind a block-wise
 * Walsh-Hadamard activation rotation, for NVIDIA B200 (sm_100a).
 *
 * The path computes y = W (R x). R = (1/sqrt(1024)) H_1024 S is applied to
 * every 1024-long block of each activation row: H_1024 is the Walsh-Hadamard
 * matrix in Sylvester (natural) order, S a fixed +-1 diagonal. W holds trits
 * t in {-1, 0, +1} and one FP16 scale per 128 consecutive weights of a row
 * (g128), w = s * t. Sources: the Ternary Bonsai 2 27B release summary
 * (linlog.top/article/1481), section 三值权重怎么压缩到 1.76 bit, for R,
 * g128 and f(x) = W(Rx); the Bonsai low-bit course
 * (adenzhou1350.github.io/learn/bonsai-low-bit), section
 * 先用五个数字理解 1.6bit, for the base-3 byte code; the TensorSharp blog
 * (2kiu.com/news/5337570), section 3.2, for the Hadamard ordering (H4).
 *
 * Conventions shared by every entry point
 *  - Pointers marked "device" are CUDA device memory owned by the caller.
 *    The library never allocates, frees or synchronises, and keeps no
 *    mutable global state.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *    the legacy default stream) and runs asynchronously.
 *  - Arguments are validated on the host before anything is launched; a
 *    non-zero bt_status means nothing was enqueued (except BT_ERR_CUDA,
 *    returned when a launch itself failed).
 *  - Errors found on the device are OR-ed into the caller's int32 word
 *    `dev_err` (device memory, nullable) as BT_DEVERR_* bits. Kernels never
 *    trap and never spin without a bound.
 *  - Row-major everywhere. Activations are [M][K], outputs [M][N], trits
 *    [N][K], codes [N][row bytes], scales [N][K/128] as FP16 bit patterns.
 *  - Reentrant; calls on one stream are ordered, calls on different streams
 *    must not share a workspace.
 */
#ifndef BT_H
#define BT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BT_OK = 0,
    BT_ERR_INVALID_ARG = 1,   /* NULL pointer, bad enum value            */
    BT_ERR_SHAPE = 2,         /* size constraint violated                */
    BT_ERR_ALIGN = 3,         /* pointer not aligned as required         */
    BT_ERR_WORKSPACE = 4,     /* workspace missing or too small          */
    BT_ERR_UNSUPPORTED = 5,   /* valid request the library does not serve */
    BT_ERR_CUDA = 6           /* a CUDA launch or query failed           */
} bt_status;

/* Bits OR-ed into *dev_err by kernels. */
#define BT_DEVERR_INVALID_TRIT 0x1   /* bt_pack: a trit outside {-1,0,1}           */
#define BT_DEVERR_INVALID_CODE 0x2   /* base-3 byte >= 243, or 2-bit field == 3    */
#define BT_DEVERR_INVALID_PAD  0x4   /* bt_unpack: a pad trit of a base-3 group != 0 */
#define BT_DEVERR_TIMEOUT      0x8   /* a bounded pipeline wait gave up            */

typedef enum {
    /* Base-3, 5 trits per byte, code = sum_i (t_i + 1) 3^i with trit i at the
     * lower k. Per row and per group of 128 weights: 25 full bytes, then one
     * byte with the group's last 3 trits and two pad trits of value 0
     * (digit 1), so the last byte is in [108, 134]. 26 bytes per group. */
    BT_LAYOUT_B3 = 0,
    /* Plain 2 bits per trit: digit t + 1 in bits [2i, 2i+1] of byte i/4 (4
     * trits per byte, lowest k in the low bits); 32 bytes per group. */
    BT_LAYOUT_2BIT = 1,
    /* Continuous base-3: the row's trits five to a byte with no break at
     * group boundaries (byte j holds trits 5j .. 5j+4, code as for
     * BT_LAYOUT_B3; a byte may hold trits of two groups); ceil(K/5) bytes,
     * the last byte's trits past K are pads of value 0, and the row is padded
     * with zero bytes to a multiple of 16. 1.725 bit per weight with the g128
     * scales at K = 5120, the release summary's 1.72-bit accounting (section
     * 三值权重怎么压缩到 1.76 bit). bt_pack, bt_unpack, and the single-row
     * products (bt_gemv at M = 1, bt_gemv_batched) take it; bt_gemm does not. */
    BT_LAYOUT_B3C = 2
} bt_layout;

typedef enum { BT_F32 = 0, BT_BF16 = 1 } bt_dtype;

const char* bt_status_string(int status);
int bt_version(void);

/* Bytes of one packed row: K/128 * 26 (base-3), K/128 * 32 (2-bit), or
 * ceil(K/5) rounded up to 16 (continuous base-3). -1 if K is not a positive
 * multiple of 128 or layout is unknown. */
int64_t bt_codes_row_bytes(int layout, int64_t K);

/*
 * bt_pack: trits (device, int8 [N][K]) -> codes (device, uint8
 * [N][bt_codes_row_bytes]). K % 128 == 0, N >= 0. Every byte of `codes` is
 * written. A trit outside {-1,0,1} is packed as 0 and sets
 * BT_DEVERR_INVALID_TRIT. Source: base-3 byte code, Bonsai low-bit course,
 * section 先用五个数字理解 1.6bit; group of 128 and FP16 scale, release
 * summary, section 三值权重怎么压缩到 1.76 bit.
 */
bt_status bt_pack(int layout, const int8_t* trits, int64_t N, int64_t K,
                  uint8_t* codes, int32_t* dev_err, void* stream);

/*
 * bt_unpack: inverse of bt_pack (device in, device out). Invalid codes set
 * BT_DEVERR_INVALID_CODE and decode as zeros; a non-zero base-3 pad trit
 * sets BT_DEVERR_INVALID_PAD. A test and debug helper.
 */
bt_status bt_unpack(int layout, const uint8_t* codes, int64_t N, int64_t K,
                    int8_t* trits, int32_t* dev_err, void* stream);

/*
 * bt_fwht1024: x_rot = R x block-wise, R = (1/32) H_1024 S.
 *  x_bf16    device, bf16 bit patterns [M][K], 16-byte aligned
 *  sign1024  device, int8 [1024], every entry +1 or -1 (other values are
 *            treated as +1 when >= 0 and -1 when < 0)
 *  K % 1024 == 0, M >= 0
 *  out_dtype BT_F32 (float [M][K]) or BT_BF16 (bf16 [M][K], round to
 *            nearest even); x_rot 16-byte aligned, must not overlap x
 * FP32 arithmetic; the 1/32 factor is exact. Source: release summary,
 * section 三值权重怎么压缩到 1.76 bit (R, blockwise, n = 1024); butterfly as
 * in the TensorSharp blog, section 5.2.
 */
bt_status bt_fwht1024(const uint16_t* x_bf16, const int8_t* sign1024, int64_t M, int64_t K,
                      int out_dtype, void* x_rot, void* stream);

/*
 * bt_gemv: decode path, y[m][n] = sum_g s[n][g] sum_{k in g} t[n][k] x'[m][k],
 * 1 <= M <= 16.
 *  layout    BT_LAYOUT_B3 or BT_LAYOUT_2BIT
 *  codes     device [N][bt_codes_row_bytes(layout, K)], 16-byte aligned
 *  scales    device fp16 bits [N][K/128], 4-byte aligned (16-byte aligned
 *            for the fastest kernels)
 *  x         device [M][K]. If sign1024 != NULL, x is the raw activation in
 *            bf16 (x_dtype must be BT_BF16) and the rotation is applied
 *            first (K % 1024 == 0). If sign1024 == NULL, x is already
 *            rotated, in x_dtype (BT_F32 or BT_BF16), K % 128 == 0.
 *  y         device [M][N] in y_dtype (BT_F32 or BT_BF16), 16-byte aligned
 *  workspace device, >= bt_gemv_workspace_bytes(...), 256-byte aligned;
 *            scratch (no call expects particular contents).
 *  dev_err   nullable. When given, the packed codes are validated on the
 *            fly and invalid ones set BT_DEVERR_INVALID_CODE (their
 *            contribution is then unspecified but finite); when NULL the
 *            check is skipped (it costs one ALU op per byte pair or word).
 *            A copy that does not arrive within a bounded wait sets
 *            BT_DEVERR_TIMEOUT and the affected outputs are unspecified.
 * Kernels: single rows that TMA can stream (M = 1, K % 1024 == 0, 16-byte
 * aligned codes and scales) run the table-lookup kernels of
 * bt_gemv_batched: per-chunk tables of the 5- or 4-trit partial dot products
 * of x', one lookup per packed byte, FP32 throughout, one partial per row and
 * 512-column chunk; a second kernel adds a row's partials in chunk order.
 * Other shapes run a prep
 * kernel (rotation, FP16 activation fragments) and an mma.sync kernel
 * (M <= 8 per launch; 9-16 rows take two launches).
 * Consecutive kernels of a call, and of consecutive calls, overlap through
 * programmatic dependent launch: a kernel may start reading codes and scales
 * before the preceding kernel in the stream has finished if that kernel
 * allows it, so codes and scales must not be written by a kernel that
 * triggers dependent launch early.
 * Numerics: single-row kernel: FP32 table entries, scale products and sums
 * in a fixed order; zero trits contribute exactly 0. Otherwise the rotated activation
 * feeds FP16 tensor-core products with FP32 accumulation (one power-of-two
 * exponent per 128 activations keeps it in range), and the digit offset is
 * taken out by the same tensor-core sum of an all-zero-trit row, so zero
 * trits contribute exactly 0 there too. Either way y satisfies
 * |y - y_exact| <= 2e-3 * sum_k |w x'| + 1e-5, and repeated calls give
 * bit-identical results.
 * Source: fused unpack and group scale inside the matrix product, release
 * summary, section 三值权重怎么压缩到 1.76 bit.
 */
size_t bt_gemv_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K);
bt_status bt_gemv(int layout, const uint8_t* codes, const uint16_t* scales,
                  const void* x, int x_dtype, const int8_t* sign1024,
                  int64_t M, int64_t N, int64_t K, int y_dtype, void* y,
                  void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream);

/*
 * bt_gemv_batched: the single-row (M = 1) product y_p = W_p (R x_p) for a list
 * of matrices: one persistent table-lookup kernel and one reduction kernel per
 * 12 matrices (fewer where a matrix reads an output of the current group:
 * it starts the next group). A matrix's activation is either given (x, x_dtype) or the output of
 * an earlier matrix of the list (x_from >= 0: the chained layers of a decode
 * step), so a whole token's stack of layers -- or matrices that share nothing
 * -- stream their weights without a gap between them. Every CTA takes an
 * equal contiguous share of the list's (matrix, 512-column chunk, row) items.
 * Source: release summary, sections 三值权重怎么压缩到 1.76 bit (R, g128,
 * fused unpack and scale) and 已知短板 (the activation transform is the
 * largest cost outside the product at batch 1).
 *  layout     BT_LAYOUT_B3 or BT_LAYOUT_2BIT (one layout per call)
 *  problems   host array of `count` descriptors (1 <= count <= 256):
 *    codes    device [N][bt_codes_row_bytes(layout, K)], 16-byte aligned
 *    scales   device fp16 bits [N][K/128], 16-byte aligned
 *    x        device [1][K], 16-byte aligned, in x_dtype (BT_BF16, or BT_F32
 *             when sign1024 is NULL); unused when x_from >= 0
 *    x_from   -1, or the index of an earlier problem whose y (N == this K,
 *             in y_dtype) is this activation; with sign1024 that y must be
 *             bf16 (y_dtype BT_BF16)
 *    y        device [1][N] in y_dtype, 16-byte aligned
 *    1 <= N <= 2^24; 1024 <= K <= 2^30, K % 1024 == 0
 *  sign1024   as for bt_gemv (NULL: every x is already rotated)
 *  workspace  device, >= bt_gemv_batched_workspace_bytes(...), 256-byte
 *             aligned; scratch for the chunk partials (N * K / 512 floats per
 *             matrix of the largest group).
 *  dev_err    as for bt_gemv; a dependency or copy that does not arrive
 *             within a bounded time sets BT_DEVERR_TIMEOUT.
 * Successive groups depend on one another through stream order.
 * Numerics and determinism as for single-row bt_gemv calls.
 */
typedef struct {
    const uint8_t* codes;
    const uint16_t* scales;
    const void* x;
    int32_t x_dtype;
    int32_t x_from;
    void* y;
    int64_t N;
    int64_t K;
} bt_gemv_problem;

size_t bt_gemv_batched_workspace_bytes(int layout, const bt_gemv_problem* problems, int count);
bt_status bt_gemv_batched(int layout, const bt_gemv_problem* problems, int count, const int8_t* sign1024,
                          int y_dtype, void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream);

/*
 * bt_gemv_noalloc: bt_gemv for callers that cannot allocate device memory --
 * code that runs where cudaMalloc is unavailable or not allowed (inside a
 * custom allocator or memory-pool callback, in a runtime that has handed all
 * device memory to its own arena, or under a fixed memory budget decided
 * before the call). The method has no counterpart; it is an interface
 * convenience of this library.
 * Arguments and results are those of bt_gemv without the workspace: the
 * scratch is an 8 MiB array in the library's own device memory, reserved on
 * every GPU that loads libbt.so until the process exits. Requests whose
 * bt_gemv_workspace_bytes exceeds 8 MiB return BT_ERR_WORKSPACE before
 * anything is launched. On the decode shapes, M <= 16 fits on 5120x5120,
 * M <= 11 on 5120x17408 and 17408x5120, M <= 3 on 17408x17408; single rows fit
 * up to N * K / 512 = 2^21 (N = K = 32768 fits, N = K = 33792 does not).
 * The first call in a CUDA context looks up the array's device address
 * (for the usual primary context: once per device, with that device
 * current) and caches it for that context; a context created later on the
 * same device -- after cudaDeviceReset, or a caller's own context -- gets a
 * lookup of its own. Make that first call before any stream capture. All calls share the one array and it keeps the last call's
 * contents (no call depends on them), so
 * calls that may overlap on the GPU -- on different streams, or from
 * different host threads -- race and must be serialised by the caller.
 * Never calls cudaMalloc, cudaFree or any allocating routine.
 */
bt_status bt_gemv_noalloc(int layout, const uint8_t* codes, const uint16_t* scales,
                          const void* x, int x_dtype, const int8_t* sign1024,
                          int64_t M, int64_t N, int64_t K, int y_dtype, void* y,
                          int32_t* dev_err, void* stream);

/*
 * bt_gemm: prefill path, Y = X' W^T with W = s * t decoded into FP16 tiles
 * in shared memory and multiplied on the tcgen05 tensor cores, FP32
 * accumulation, bf16 output [M][N] (round to nearest even).
 *  M % 128 == 0, N % 128 == 0, K % 128 == 0 (K % 1024 == 0 when rotating).
 *  Arguments as for bt_gemv (y is bf16). The rotated activation is rounded
 *  to FP16 after scaling each row by a power of two chosen from its largest
 *  magnitude.
 * Kernels: a prep kernel (rotation, row scaling, FP16 in the decoder's K
 *  order), then the tensor-core kernel, chained by programmatic dependent
 *  launch. With M % 256 == 0 the output tiles run as clusters of two CTAs
 *  that share each decoded weight tile (tcgen05 cta_group::2, M = 256 per
 *  instruction; with M % 512 == 0 a pair can take two 256-row tiles);
 *  otherwise one CTA per 128-row tile. Grids too small for the SMs split K:
 *  in two for pairs (the two pairs of a tile form a cluster of four CTAs and
 *  swap halves in shared memory), 2-4 ways for single CTAs (each split stores
 *  FP32 partial products in the workspace and the last to finish adds them
 *  in split order). The form is a function of
 *  (layout, M, N, K, SM count), so repeated calls give bit-identical results;
 *  different forms differ only in FP32 summation order.
 *  The workspace (>= bt_gemm_workspace_bytes, which includes the partials
 *  and arrival counters when K is split over single CTAs; the call zeroes
 *  the counters) is scratch, as for bt_gemv.
 *  Waits are bounded: one that runs out sets BT_DEVERR_TIMEOUT and the
 *  affected outputs are unspecified.
 * Source: pp512 prompt processing, release summary, section 实测吞吐.
 */
size_t bt_gemm_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K);
bt_status bt_gemm(int layout, const uint8_t* codes, const uint16_t* scales,
                  const void* x, int x_dtype, const int8_t* sign1024,
                  int64_t M, int64_t N, int64_t K, void* y_bf16,
                  void* workspace, size_t workspace_bytes, int32_t* dev_err, void* stream);

/*
 * bt_ternarize: the offline weight path, float W -> trits and g128 FP16
 * scales in the rotated basis, ready for bt_pack. Source: release summary,
 * section 三值权重怎么压缩到 1.76 bit (every weight tensor is transformed
 * block-wise to the fixed basis R = (1/sqrt 1024) H_1024 S before it is
 * ternarised, and the activation gets the same R, f(x) = W(Rx)); TensorSharp
 * blog, section 2.1 (per-block scale from the mean |w|, threshold chosen by
 * searching candidates for the smallest reconstruction error).
 *  W        device float [N][K], 16-byte aligned; K % 1024 == 0
 *  sign1024 device int8 [1024] (S), 16-byte aligned
 *  trits    device int8 [N][K] out: each row is R applied to the row of W,
 *           block-wise, then ternarised per 128 weights
 *  scales   device fp16 bits [N][K/128] out, 2-byte aligned
 *  workspace device, >= bt_ternarize_workspace_bytes(N, K) (the rotated
 *           weights in FP64), 256-byte aligned; scratch
 * Per group of 128 rotated weights v: candidate thresholds tau_j = (j / 20)
 * mean|v| for j = 1..40; trits sign(v_i) where |v_i| >= tau_j, else 0; scale
 * the mean |v_i| over the non-zero trits, rounded to nearest FP16; the
 * candidate with the smallest sum (v_i - s t_i)^2 wins (the smallest j on
 * ties); a group of zeros gets scale 0. All in FP64 in the plain order of
 * operations, so the result is that of the definition, bit for bit. An
 * offline step: one warp per (row, 1024-block) rotates, one thread per group
 * searches.
 */
size_t bt_ternarize_workspace_bytes(int64_t N, int64_t K);
bt_status bt_ternarize(const float* W, const int8_t* sign1024, int64_t N, int64_t K, int8_t* trits,
                       uint16_t* scales, void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BT_H */

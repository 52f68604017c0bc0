// Offline weight path: float W -> rotated basis -> g128 trits and FP16 scales.
//
// The release summary of Ternary Bonsai 2 27B (section 三值权重怎么压缩到
// 1.76 bit) transforms every weight tensor block-wise to the fixed basis
// R = (1/sqrt 1024) H_1024 S before ternarising, and applies the same R to
// the activation at inference (f(x) = W(Rx)). A row of the rotated weights is
// therefore w'_b = R w_b for each 1024-block b, so that W' R ~ W. The
// TensorSharp blog (2kiu.com/news/5337570), section 2.1, ternarises each
// block with a scale derived from the mean |w| and a threshold chosen by
// searching candidates for the smallest reconstruction error. Here, per
// 128-group of rotated weights v:
//   tau_j = (j / 20) mean|v|, j = 1..40; t_i = sign(v_i) where |v_i| >= tau_j;
//   s_j = FP16(mean of |v_i| over the non-zero t_i), the least-squares scale
//   for those trits; err_j = sum_i (v_i - s_j t_i)^2 with that FP16 scale;
// the smallest err_j wins (the smallest j on ties); a group of zeros gets
// s = 0 and zero trits.
//
// Everything is FP64, in the same order of operations as the plain
// definition (butterfly stages with half-widths 1, 2, ..., 512; sums in
// index order; no fused multiply-adds), so the integer result -- which trits
// and which FP16 scale -- is the same as the definition's, bit for bit.
// This is an offline step (once per weight tensor), not part of the decode
// path: one warp per (row, 1024-block) rotates, one thread per group searches.
#include "bt_internal.cuh"

namespace bt {

constexpr int kTernRotWarps = 8;   // rotation: warps per CTA, one (row, block) each
constexpr int kTernThreads = 128;  // search: one thread per 128-group

// Rotate one 1024-block of one row in FP64 into wr. Lane l holds elements
// 32 l + i; butterfly stages on index bits 0..4 run in registers, those on
// bits 5..9 between lanes, in the order of the definition.
__global__ void __launch_bounds__(kTernRotWarps * 32)
ternarize_rotate_kernel(const float* __restrict__ W, const int8_t* __restrict__ sign, int64_t N, int64_t K,
                        double* __restrict__ wr) {
    const int lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * kTernRotWarps + (threadIdx.x >> 5);
    const int64_t nb = K / kBlock;
    if (item >= N * nb) return;
    const int64_t row = item / nb, b = item % nb;
    const float4* src = reinterpret_cast<const float4*>(W + row * K + b * kBlock + 32 * lane);
    const uint4* sg = reinterpret_cast<const uint4*>(sign + 32 * lane);
    const uint4 s0 = __ldg(sg), s1 = __ldg(sg + 1);
    const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    double v[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 f = __ldg(src + q);
        v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int8_t sv = static_cast<int8_t>((sw[i >> 2] >> (8 * (i & 3))) & 0xFFu);
        if (sv < 0) v[i] = -v[i];  // S, exact
    }
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((i & h) == 0) {
                const double a = v[i], c = v[i + h];
                v[i] = __dadd_rn(a, c);
                v[i + h] = __dsub_rn(a, c);
            }
        }
    }
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {   // half-widths 32 h: partner lane l ^ h
        const bool upper = lane & h;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const double p = __shfl_xor_sync(0xffffffffu, v[i], h);
            // lower lane: a + b with b its partner's; upper lane: a - b with a the partner's
            v[i] = upper ? __dsub_rn(p, v[i]) : __dadd_rn(v[i], p);
        }
    }
    double* dst = wr + row * K + b * kBlock + 32 * lane;
#pragma unroll
    for (int i = 0; i < 32; ++i) dst[i] = __dmul_rn(v[i], 1.0 / 32.0);  // 1/sqrt(1024), exact
}

__global__ void __launch_bounds__(kTernThreads)
ternarize_search_kernel(const double* __restrict__ wr, int64_t N, int64_t K, int8_t* __restrict__ trits,
                        uint16_t* __restrict__ scales) {
    const int64_t G = K / kGroup;
    const int64_t gi = (int64_t)blockIdx.x * kTernThreads + threadIdx.x;
    if (gi >= N * G) return;
    const int64_t n = gi / G, g = gi % G;
    const double* v = wr + n * K + g * kGroup;
    double mean = 0.0;
    for (int i = 0; i < kGroup; ++i) mean = __dadd_rn(mean, fabs(v[i]));
    mean = __ddiv_rn(mean, (double)kGroup);
    int best_j = 0;
    double best_err = 0.0;
    uint16_t best_s = 0;
    for (int j = 1; j <= 40; ++j) {
        const double tau = __dmul_rn(__ddiv_rn((double)j, 20.0), mean);
        double sum = 0.0;
        int nnz = 0;
        for (int i = 0; i < kGroup; ++i) {
            const double a = fabs(v[i]);
            if (a >= tau) { sum = __dadd_rn(sum, a); ++nnz; }
        }
        const uint16_t s16 = nnz ? __half_as_ushort(__double2half(__ddiv_rn(sum, (double)nnz))) : uint16_t(0);
        const double s = (double)__half2float(__ushort_as_half(s16));
        double err = 0.0;
        for (int i = 0; i < kGroup; ++i) {
            const double q = fabs(v[i]) >= tau ? (v[i] < 0 ? -s : s) : 0.0;
            const double d = __dsub_rn(v[i], q);
            err = __dadd_rn(err, __dmul_rn(d, d));
        }
        if (j == 1 || err < best_err) {
            best_err = err;
            best_j = j;
            best_s = s16;
        }
    }
    if (mean == 0.0) best_s = 0;
    const double tau = __dmul_rn(__ddiv_rn((double)best_j, 20.0), mean);
    int8_t* t = trits + n * K + g * kGroup;
    for (int i = 0; i < kGroup; ++i) t[i] = (mean != 0.0 && fabs(v[i]) >= tau) ? (v[i] < 0 ? -1 : 1) : 0;
    scales[n * G + g] = best_s;
}

size_t ternarize_workspace_bytes(int64_t N, int64_t K) { return (size_t)N * (size_t)K * sizeof(double); }

cudaError_t launch_ternarize(const float* W, const int8_t* sign, int64_t N, int64_t K, int8_t* trits,
                             uint16_t* scales, void* workspace, cudaStream_t stream) {
    double* wr = static_cast<double*>(workspace);
    const int64_t items = N * (K / kBlock);
    ternarize_rotate_kernel<<<(unsigned)((items + kTernRotWarps - 1) / kTernRotWarps), kTernRotWarps * 32, 0,
                              stream>>>(W, sign, N, K, wr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t groups = N * (K / kGroup);
    ternarize_search_kernel<<<(unsigned)((groups + kTernThreads - 1) / kTernThreads), kTernThreads, 0, stream>>>(
        wr, N, K, trits, scales);
    return cudaGetLastError();
}

}  // namespace bt

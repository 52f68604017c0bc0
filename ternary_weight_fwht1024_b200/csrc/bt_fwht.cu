// Block-wise activation rotation x' = (1/32) H_1024 (S . x).
//
// The rotation R = (1/sqrt n) H_n S with n = 1024 is the fixed rotated basis
// of the Ternary Bonsai 2 27B release summary, section 三值权重怎么压缩到
// 1.76 bit (inference applies f(x) = W(Rx)). H is in Sylvester order (H4 as
// printed in the TensorSharp blog, section 3.2) and is applied by the fast
// butterfly (same blog, section 5.2), never as a matrix.
//
// One warp per (row, 1024-block): 32 values per lane, two register passes of
// five butterfly stages around one shared-memory transpose (bt_internal.cuh).
// HBM-bound at large M*K: 2 bytes in, 4 (or 2) bytes out per element.
#include "bt_internal.cuh"

namespace bt {

constexpr int kFwhtWarps = 4;

template <bool OUT_BF16>
__global__ void __launch_bounds__(kFwhtWarps * 32)
fwht1024_kernel(const uint16_t* __restrict__ x, const int8_t* __restrict__ sign, int64_t M,
                int64_t K, void* __restrict__ out) {
    __shared__ __align__(16) float tiles[kFwhtWarps][32 * kTileStride];
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t blocks_per_row = K / kBlock;
    const int64_t total = M * blocks_per_row;
    for (int64_t wb = (int64_t)blockIdx.x * kFwhtWarps + warp; wb < total;
         wb += (int64_t)gridDim.x * kFwhtWarps) {
        const int64_t m = wb / blocks_per_row, b = wb - m * blocks_per_row;
        const int64_t base = m * K + b * kBlock;
        float v[32];
        load_signed_bf16_block(x + base, sign, v);
        fwht1024_warp(v, tiles[warp]);
        if (OUT_BF16) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + base + lane;
#pragma unroll
            for (int j = 0; j < 32; ++j) o[32 * j] = __float2bfloat16_rn(v[j]);
        } else {
            float* o = reinterpret_cast<float*>(out) + base + lane;
#pragma unroll
            for (int j = 0; j < 32; ++j) o[32 * j] = v[j];
        }
    }
}

cudaError_t launch_fwht1024(const uint16_t* x, const int8_t* sign, int64_t M, int64_t K,
                            int out_dtype, void* out, int num_sms, cudaStream_t stream) {
    const int64_t warps = M * (K / kBlock);
    if (warps == 0) return cudaSuccess;
    int64_t blocks = (warps + kFwhtWarps - 1) / kFwhtWarps;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (out_dtype == BT_BF16)
        fwht1024_kernel<true><<<(unsigned)blocks, kFwhtWarps * 32, 0, stream>>>(x, sign, M, K, out);
    else
        fwht1024_kernel<false><<<(unsigned)blocks, kFwhtWarps * 32, 0, stream>>>(x, sign, M, K, out);
    return cudaGetLastError();
}

}  // namespace bt

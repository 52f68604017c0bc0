// Pack / unpack of ternary weights into the g128 byte layouts.
//
// Base-3 (Bonsai low-bit course, section 先用五个数字理解 1.6bit): five trits
// per byte, code = sum_i (t_i + 1) 3^i, trit i at the lower k. Each group of
// 128 weights of a row takes 26 bytes: 25 full bytes, then one byte with the
// last 3 trits and two pad trits of value 0 (digit 1).
// 2-bit: digit t + 1 in bits [2i, 2i+1] of byte i/4, 32 bytes per group.
// Continuous base-3: byte j of a row holds trits 5j .. 5j+4 across group
// boundaries, ceil(K/5) bytes (trits past K are pads of value 0), then zero
// bytes up to a multiple of 16 (the release summary's 1.72-bit accounting,
// section 三值权重怎么压缩到 1.76 bit).
//
// One thread per output byte; these run offline, not on the decode path.
#include "bt_internal.cuh"

namespace bt {

__global__ void pack_b3_kernel(const int8_t* __restrict__ trits, int64_t K, int64_t total_bytes,
                               uint8_t* __restrict__ codes, int32_t* dev_err) {
    const int64_t row_bytes = (K / kGroup) * kB3GroupBytes;
    int bad = 0;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_bytes;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = o / row_bytes;
        const int64_t r = o - n * row_bytes;
        const int64_t g = r / kB3GroupBytes;
        const int b = static_cast<int>(r - g * kB3GroupBytes);
        const int8_t* t = trits + n * K + g * kGroup + 5 * b;
        const int count = (b == kB3GroupBytes - 1) ? 3 : 5;  // last byte: 3 trits + 2 pads
        int code = 0, p3 = 1;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            int trit = 0;
            if (i < count) {
                trit = t[i];
                if (trit < -1 || trit > 1) {
                    bad = BT_DEVERR_INVALID_TRIT;
                    trit = 0;
                }
            }
            code += (trit + 1) * p3;
            p3 *= 3;
        }
        codes[o] = static_cast<uint8_t>(code);
    }
    report(dev_err, bad);
}

__global__ void pack_2b_kernel(const int8_t* __restrict__ trits, int64_t total_bytes,
                               uint8_t* __restrict__ codes, int32_t* dev_err) {
    // 4 trits per byte and 32 bytes per 128 trits: byte o holds trits 4o..4o+3
    int bad = 0;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_bytes;
         o += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(trits) + o);
        int code = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int trit = static_cast<int8_t>((w >> (8 * i)) & 0xFF);
            if (trit < -1 || trit > 1) {
                bad = BT_DEVERR_INVALID_TRIT;
                trit = 0;
            }
            code |= (trit + 1) << (2 * i);
        }
        codes[o] = static_cast<uint8_t>(code);
    }
    report(dev_err, bad);
}

__global__ void unpack_b3_kernel(const uint8_t* __restrict__ codes, int64_t K, int64_t total_bytes,
                                 int8_t* __restrict__ trits, int32_t* dev_err) {
    const int64_t row_bytes = (K / kGroup) * kB3GroupBytes;
    int bad = 0;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_bytes;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = o / row_bytes;
        const int64_t r = o - n * row_bytes;
        const int64_t g = r / kB3GroupBytes;
        const int b = static_cast<int>(r - g * kB3GroupBytes);
        int code = codes[o];
        if (code >= 243) {
            bad |= BT_DEVERR_INVALID_CODE;
            code = 121;  // all digits 1: decodes as five zero trits
        }
        int8_t* t = trits + n * K + g * kGroup + 5 * b;
        const int count = (b == kB3GroupBytes - 1) ? 3 : 5;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            const int digit = code % 3;
            code /= 3;
            if (i < count) t[i] = static_cast<int8_t>(digit - 1);
            else if (digit != 1) bad |= BT_DEVERR_INVALID_PAD;
        }
    }
    report(dev_err, bad);
}

__global__ void unpack_2b_kernel(const uint8_t* __restrict__ codes, int64_t total_bytes,
                                 int8_t* __restrict__ trits, int32_t* dev_err) {
    int bad = 0;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_bytes;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int code = codes[o];
        uint32_t w = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int digit = (code >> (2 * i)) & 3;
            if (digit == 3) {
                bad |= BT_DEVERR_INVALID_CODE;
                digit = 1;
            }
            w |= static_cast<uint32_t>(static_cast<uint8_t>(digit - 1)) << (8 * i);
        }
        reinterpret_cast<unsigned int*>(trits)[o] = w;
    }
    report(dev_err, bad);
}

__global__ void pack_b3c_kernel(const int8_t* __restrict__ trits, int64_t K, int64_t row_bytes, int64_t total_bytes,
                                uint8_t* __restrict__ codes, int32_t* dev_err) {
    const int64_t used = (K + 4) / 5;
    int bad = 0;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_bytes;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = o / row_bytes;
        const int64_t j = o - n * row_bytes;
        int code = 0;
        if (j < used) {
            const int8_t* t = trits + n * K + 5 * j;
            int p3 = 1;
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                int trit = 0;
                if (5 * j + i < K) {
                    trit = t[i];
                    if (trit < -1 || trit > 1) {
                        bad = BT_DEVERR_INVALID_TRIT;
                        trit = 0;
                    }
                }
                code += (trit + 1) * p3;
                p3 *= 3;
            }
        }
        codes[o] = static_cast<uint8_t>(code);
    }
    report(dev_err, bad);
}

__global__ void unpack_b3c_kernel(const uint8_t* __restrict__ codes, int64_t K, int64_t row_bytes,
                                  int64_t total_bytes, int8_t* __restrict__ trits, int32_t* dev_err) {
    const int64_t used = (K + 4) / 5;
    int bad = 0;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_bytes;
         o += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = o / row_bytes;
        const int64_t j = o - n * row_bytes;
        int code = codes[o];
        if (j >= used) {  // row padding
            if (code != 0) bad |= BT_DEVERR_INVALID_PAD;
            continue;
        }
        if (code >= 243) {
            bad |= BT_DEVERR_INVALID_CODE;
            code = 121;
        }
        int8_t* t = trits + n * K + 5 * j;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            const int digit = code % 3;
            code /= 3;
            if (5 * j + i < K) t[i] = static_cast<int8_t>(digit - 1);
            else if (digit != 1) bad |= BT_DEVERR_INVALID_PAD;
        }
    }
    report(dev_err, bad);
}

static int64_t b3c_row_bytes(int64_t K) { return ((K + 4) / 5 + 15) / 16 * 16; }

static int grid_for(int64_t work, int threads) {
    int64_t blocks = (work + threads - 1) / threads;
    const int64_t cap = 148 * 16;
    if (blocks > cap) blocks = cap;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

cudaError_t launch_pack(int layout, const int8_t* trits, int64_t N, int64_t K, uint8_t* codes,
                        int32_t* dev_err, cudaStream_t stream) {
    const int threads = 256;
    if (layout == BT_LAYOUT_B3C) {
        const int64_t rb = b3c_row_bytes(K), total = N * rb;
        if (total == 0) return cudaSuccess;
        pack_b3c_kernel<<<grid_for(total, threads), threads, 0, stream>>>(trits, K, rb, total, codes, dev_err);
    } else if (layout == BT_LAYOUT_B3) {
        const int64_t total = N * (K / kGroup) * kB3GroupBytes;
        if (total == 0) return cudaSuccess;
        pack_b3_kernel<<<grid_for(total, threads), threads, 0, stream>>>(trits, K, total, codes, dev_err);
    } else {
        const int64_t total = N * (K / kGroup) * k2bGroupBytes;
        if (total == 0) return cudaSuccess;
        pack_2b_kernel<<<grid_for(total, threads), threads, 0, stream>>>(trits, total, codes, dev_err);
    }
    return cudaGetLastError();
}

cudaError_t launch_unpack(int layout, const uint8_t* codes, int64_t N, int64_t K, int8_t* trits,
                          int32_t* dev_err, cudaStream_t stream) {
    const int threads = 256;
    if (layout == BT_LAYOUT_B3C) {
        const int64_t rb = b3c_row_bytes(K), total = N * rb;
        if (total == 0) return cudaSuccess;
        unpack_b3c_kernel<<<grid_for(total, threads), threads, 0, stream>>>(codes, K, rb, total, trits, dev_err);
    } else if (layout == BT_LAYOUT_B3) {
        const int64_t total = N * (K / kGroup) * kB3GroupBytes;
        if (total == 0) return cudaSuccess;
        unpack_b3_kernel<<<grid_for(total, threads), threads, 0, stream>>>(codes, K, total, trits, dev_err);
    } else {
        const int64_t total = N * (K / kGroup) * k2bGroupBytes;
        if (total == 0) return cudaSuccess;
        unpack_2b_kernel<<<grid_for(total, threads), threads, 0, stream>>>(codes, total, trits, dev_err);
    }
    return cudaGetLastError();
}

}  // namespace bt

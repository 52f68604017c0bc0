// Internal helpers shared by the libbt.so kernels (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/bt.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libbt is written for sm_100a (B200) only"
#endif

namespace bt {

constexpr int kGroup = 128;        // weights per FP16 scale
constexpr int kBlock = 1024;       // rotation block
constexpr int kB3GroupBytes = 26;  // base-3 bytes per group
constexpr int k2bGroupBytes = 32;  // 2-bit bytes per group

// MMA k16 steps per 128-weight group of one row, per layout (GEMV slot order).
constexpr int kB3Mmas = 9;
constexpr int k2bMmas = 8;

// One single-row product of a decode list, y = W (R x): x is either given or
// the output of an earlier entry of the same list (x_from >= 0).
struct DecodeProblem {
    const uint8_t* codes;
    const uint16_t* scales;
    const void* x;
    int x_bf16;
    int x_from;  // -1, or the index of the entry whose y is this x
    void* y;
    int64_t N, K;
};

// ---------------------------------------------------------------- PTX ----

__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t lop3_or_and(uint32_t a, uint32_t b, uint32_t m) {
    // (a | b) & m in one LOP3 (truth table: (0xF0 | 0xCC) & 0xAA = 0xA8)
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xA8;" : "=r"(r) : "r"(a), "r"(b), "r"(m));
    return r;
}

__device__ __forceinline__ uint32_t lop3_or3(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xFE;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// D = A(16x16 f16, row) * B(16x8 f16, col) + C, FP32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1,
                                              const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
    return __ldg(reinterpret_cast<const unsigned int*>(p));
}
__device__ __forceinline__ uint32_t ldg_u16(const void* p) {
    return __ldg(reinterpret_cast<const unsigned short*>(p));
}
__device__ __forceinline__ uint2 ldg_u64(const void* p) {
    return __ldg(reinterpret_cast<const uint2*>(p));
}

// Streaming loads: read once, do not allocate in L1 (keeps L1 for reused data).
__device__ __forceinline__ uint32_t ldg_stream_u32(const void* p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_stream_u16(const void* p) {
    uint16_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ldg_stream_u64(const void* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
// Asynchronous L2 prefetch of [p, p + bytes); p and bytes multiples of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_l1(const void* p) {
    asm volatile("prefetch.global.L1 [%0];" :: "l"(p));
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" :: "l"(p));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
    return __uint_as_float(b << 16);
}
__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

__device__ __forceinline__ void report(int32_t* dev_err, int bits) {
    if (dev_err && bits) atomicOr(dev_err, bits);
}

// ------------------------------------------------ 1024-point WHT in a warp ----
//
// The rotation of one 1024-block, (1/32) H_1024 (S . x), held by one warp.
// Entry: lane l holds elements 32 l + i in v[i] (i = 0..31), already signed.
// Exit:  lane l holds element 32 j + l of the result in v[j] (j = 0..31).
// Butterfly stages on index bits 0..4 run in registers, the warp exchanges
// the 32x32 tile through shared memory (rows padded to 36 floats: the
// column writes and the 16-byte row reads are both conflict-free), and the
// stages on bits 5..9 run in registers again. Stages commute, so this is
// H_1024 in natural (Sylvester) order.
__device__ __forceinline__ void butterfly32(float (&v)[32]) {
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
        }
    }
}

constexpr int kTileStride = 36;  // floats per padded row of the exchange tile

__device__ __forceinline__ void fwht1024_warp(float (&v)[32], float* tile /* 32*36 floats */) {
    const int lane = threadIdx.x & 31;
    butterfly32(v);
#pragma unroll
    for (int i = 0; i < 32; ++i) tile[i * kTileStride + lane] = v[i];
    __syncwarp();
    const float4* row = reinterpret_cast<const float4*>(tile + lane * kTileStride);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float4 f = row[q];
        v[4 * q + 0] = f.x;
        v[4 * q + 1] = f.y;
        v[4 * q + 2] = f.z;
        v[4 * q + 3] = f.w;
    }
    __syncwarp();
    butterfly32(v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= 0.03125f;  // 1/32, exact
}

// Load 32 contiguous bf16 activations of one block for this lane and apply S.
__device__ __forceinline__ void load_signed_bf16_block(const uint16_t* xb, const int8_t* sign,
                                                       float (&v)[32]) {
    const int lane = threadIdx.x & 31;
    const uint4* src = reinterpret_cast<const uint4*>(xb + 32 * lane);
    const uint4* sg = reinterpret_cast<const uint4*>(sign + 32 * lane);
    uint4 s0 = __ldg(sg), s1 = __ldg(sg + 1);
    uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w = __ldg(src + q);
        uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int i = 8 * q + 2 * h + half;
                uint32_t bits = (half ? (ww[h] & 0xFFFF0000u) : (ww[h] << 16));
                // sign byte i: bit 7 set for negative entries
                uint32_t sbyte = (sw[i >> 2] >> (8 * (i & 3))) & 0x80u;
                v[i] = __uint_as_float(bits ^ (sbyte << 24));
            }
        }
    }
}


// ------------------------------------------------ mbarriers and TMA ----

// Bound on every barrier wait (iterations of try_wait). The test-only build
// of the library lowers it so that a withheld copy times out quickly.
#ifndef BT_SPIN_LIMIT
#define BT_SPIN_LIMIT (1u << 26)
#endif
constexpr uint32_t kSpinLimit = BT_SPIN_LIMIT;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}
// Bounded wait on the given phase parity; false when the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
        if (ok) return true;
    }
    return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}


// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tensor_map_encoder() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}


}  // namespace bt

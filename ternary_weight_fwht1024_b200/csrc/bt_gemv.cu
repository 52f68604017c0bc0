// Decode-path GEMV for packed ternary weights, 1 <= M <= 16.
//
// y[m][n] = sum_g s[n][g] sum_{k in g} t[n][k] x'[m][k], x' = R x. The
// release summary of Ternary Bonsai 2 27B (section 三值权重怎么压缩到 1.76 bit)
// runs the product directly on packed ternary weights with unpack and group
// scale fused inside it, never materialising FP16 weights; decode is HBM
// bound (section 实测吞吐: tokens/s x model bytes = weight traffic).
//
// Two kernels, chained with programmatic dependent launch:
//
//  1. gemv_prep (one CTA per row m and 1024-block): rotates x (when a sign
//     vector is given) and writes, per row m and 128-group g, the
//     activations in the order the tensor-core fragments consume them
//     ("slots"), as FP16 scaled by 2^(24 - 2 i - e_g). e_g is a power-of-two
//     exponent chosen from the group's largest |x'|; i is the position of the
//     trit's 2-bit field inside a 16-bit half (see 2.). It also writes
//     corr_g = sum_k x~_k (the FP16-rounded activations, in real units) and
//     2^e_g.
//
//  2. gemv (persistent, one CTA per SM): each warp owns a contiguous run of
//     (32-row tile pair, group) units and streams the packed bytes straight
//     from HBM into registers (L2 bulk prefetch of the run, one group of
//     register double buffering). Base-3 bytes go through a 256-entry table
//     in shared memory, replicated per lane so the gathers are conflict-free,
//     that turns a byte into its five base-3 digits d = t + 1 as 2-bit fields;
//     2-bit bytes already are such fields. One LOP3 per two weights isolates
//     field i of two bytes into the two halves of a register; read as FP16,
//     each half is the subnormal d * 4^i * 2^-24, exactly. An m16n8k16
//     tensor-core MMA against the slot-ordered activations gives
//     D = 2^-e sum_k d_k x~_k in FP32, and the group adds
//     s * (2^e D - corr) = s * sum_k t_k x~_k. The MMA's A operand is 16 weight
//     rows; its 8 columns are activation rows m.
//     A tile split across warps leaves FP32 partials; the warp that finishes
//     it last (atomic counter) adds them in a fixed order, so results are
//     deterministic run to run.
#include "bt_internal.cuh"
#include "bt_slots.cuh"

#include <mutex>

namespace bt {

#ifndef BT_GEMV_WARPS
#define BT_GEMV_WARPS 16
#endif
#ifndef BT_GEMV_TILES
#define BT_GEMV_TILES 2
#endif
constexpr int kGemvWarps = BT_GEMV_WARPS;  // warps per CTA (one CTA per SM)
constexpr int kGemvTiles = BT_GEMV_TILES;  // 16-row tiles per unit (share the activation fragments)
constexpr int kPrepThreads = 256;    // 8 warps: one per group of a 1024-block
constexpr int kLutBytes = 256 * 256; // 256 codes x (128 B low table + 128 B high table)
constexpr int kZeroBytes = 512;      // zero fragment area (>= NT * 32)
constexpr size_t kBsmemMax = 128 * 1024;

// Bytes of the per-(row, group) constants (corr, 2^e) kept in shared memory,
// padded to 16 so that the activation fragments after them start on a
// 16-byte boundary (they are copied in with 16-byte stores).
__host__ __device__ constexpr uint32_t meta_area_bytes(int M, int G) {
    return (static_cast<uint32_t>(M * G * 8) + 15u) & ~15u;
}

// ----------------------------------------------------------- prep ----------

struct PrepArgs {
    const void* x;
    int x_bf16;
    const int8_t* sign;      // nullable: x already rotated
    int M, K, G;
    uint32_t* bslots;        // [M][G][NT][4][2] pairs of FP16
    float2* meta;            // [M][G] (corr, 2^e)
    int* counters;           // [P], zeroed here
    int P;
};

template <int LAYOUT>
__global__ void __launch_bounds__(kPrepThreads) gemv_prep_kernel(PrepArgs a) {
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    __shared__ __align__(16) float xs[32 * kTileStride];
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.P; i += blockDim.x) a.counters[i] = 0;

    const int nblocks = (a.G + 7) / 8;
    const int m = blockIdx.x / nblocks, b = blockIdx.x % nblocks;
    const int64_t k0 = (int64_t)b * kBlock;
    const int ng = min(8, a.G - 8 * b);
    if (warp == 0) {
        float v[32];
        if (a.sign) {
            load_signed_bf16_block(reinterpret_cast<const uint16_t*>(a.x) + (int64_t)m * a.K + k0, a.sign, v);
            fwht1024_warp(v, xs);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int64_t idx = k0 + 32 * j + lane;
                float val = 0.f;
                if (idx < a.K) {
                    const int64_t off = (int64_t)m * a.K + idx;
                    val = a.x_bf16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(a.x)[off])
                                   : reinterpret_cast<const float*>(a.x)[off];
                }
                v[j] = val;
            }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) xs[32 * j + lane] = v[j];  // element 32 j + lane
    }
    __syncthreads();
    const int q = warp;  // group within the block
    if (q >= ng) return;
    float v4[4];
    float amax = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        v4[r] = xs[128 * q + 32 * r + lane];
        amax = fmaxf(amax, fabsf(v4[r]));
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
    int E = amax > 0.f ? ilogbf(amax) + 1 : -100;  // amax < 2^E
    E = max(-100, min(100, E));
    const int e = 9 + E;
    // Lanes 0..3 (c) write their own fragment words -- (t, c) pairs of FP16
    // slots, as the MMA's B operand expects -- and keep them for the
    // correction below.
    const int64_t gidx = (int64_t)m * a.G + 8 * b + q;
    uint32_t* dst = a.bslots + gidx * (NT * 8);
    const float* xg = xs + 128 * q;
    uint32_t bf[NT][2];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
            uint32_t word = 0;
            if (lane < 4) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    int i = 0;
                    const int k = LAYOUT == BT_LAYOUT_B3 ? b3_slot(t, lane, 2 * hp + u, &i)
                                                         : tb_slot(t, lane, 2 * hp + u, &i);
                    if (k >= 0) {
                        const __half hv = __float2half_rn(xg[k] * exp2i(24 - 2 * i - e));
                        word |= static_cast<uint32_t>(__half_as_ushort(hv)) << (16 * u);
                    }
                }
                dst[t * 8 + lane * 2 + hp] = word;
            }
            bf[t][hp] = word;  // zero outside lanes 0..3: only column 0 is fed
        }
    }
    // corr = 2^e x (the group's tensor-core sum with every digit 1), by the
    // same MMA chain the GEMV kernels run: a row of zero trits decodes to
    // exactly these A registers, so its D equals this one bit for bit and
    // s * (2^e D - corr) is exactly 0.
    uint32_t Rg[16], Rh[16];
    float d[4];
    if constexpr (LAYOUT == BT_LAYOUT_B3) {
        uint32_t QG[3], QH[3];
        b3_ones_tile(lane & 3, Rg, Rh, QG, QH);
        b3_group_mma(Rg, Rh, QG, QH, bf, d);
    } else {
        tb_ones_tile(Rg, Rh);
        tb_group_mma(Rg, Rh, bf, d);
    }
    if (lane == 0) a.meta[gidx] = make_float2(d[0] * exp2i(e), exp2i(e));  // lane 0: D[0][0], column 0
}

// ----------------------------------------------------------- GEMV ----------

struct GemvArgs {
    const uint8_t* codes;
    const uint16_t* scales;
    const uint32_t* bslots;
    const float2* meta;
    float* partials;         // [warps][2][kGemvTiles*16][M]
    int* counters;           // [P]
    void* y;
    int y_bf16;
    int M, N, G;
    uint32_t row_bytes;
    int64_t U;               // P * G units
    int64_t chunk;           // units per warp
    int32_t* dev_err;
};

extern __shared__ __align__(1024) uint8_t gemv_smem[];

// Table lookup at byte offset `off` of the dynamic shared memory (the table
// sits at its start); indexing the symbol lets the compiler fold the base.
__device__ __forceinline__ uint32_t lut_u32(uint32_t off) {
    return *reinterpret_cast<const uint32_t*>(gemv_smem + off);
}

__device__ __forceinline__ uint32_t smem_u32addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
    return r;
}
__device__ __forceinline__ uint2 lds_u64(uint32_t addr) {
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
    return r;
}

// Registers a warp holds for one group: packed bytes and scales of its rows.
template <int LAYOUT>
struct CodeStage {
    uint32_t w[kGemvTiles][LAYOUT == BT_LAYOUT_B3 ? 5 : 4];
    uint32_t s[kGemvTiles][2];
};

// Byte offsets (from a.codes / a.scales) for one parity of groups j0, j0+2, ...
struct StagePtr {
    uint32_t og[kGemvTiles], oh[kGemvTiles];  // aligned windows (base-3) or 8-byte chunks (2-bit)
    uint32_t o12[kGemvTiles];                 // base-3 pair 12 (bytes 24, 25)
    uint32_t osg[kGemvTiles], osh[kGemvTiles];// scale element offsets
};

template <int LAYOUT>
__device__ __forceinline__ void load_stage(CodeStage<LAYOUT>& S, const GemvArgs& a, const StagePtr& P) {
#pragma unroll
    for (int tt = 0; tt < kGemvTiles; ++tt) {
        if constexpr (LAYOUT == BT_LAYOUT_B3) {
            S.w[tt][0] = ldg_stream_u32(a.codes + P.og[tt]);
            S.w[tt][1] = ldg_stream_u32(a.codes + P.og[tt] + 4);
            S.w[tt][2] = ldg_stream_u32(a.codes + P.oh[tt]);
            S.w[tt][3] = ldg_stream_u32(a.codes + P.oh[tt] + 4);
            S.w[tt][4] = ldg_stream_u16(a.codes + P.o12[tt]);
        } else {
            const uint2 x0 = ldg_stream_u64(a.codes + P.og[tt]);
            const uint2 x1 = ldg_stream_u64(a.codes + P.oh[tt]);
            S.w[tt][0] = x0.x; S.w[tt][1] = x0.y; S.w[tt][2] = x1.x; S.w[tt][3] = x1.y;
        }
        S.s[tt][0] = ldg_stream_u16(a.scales + P.osg[tt]);
        S.s[tt][1] = ldg_stream_u16(a.scales + P.osh[tt]);
    }
}

__device__ __forceinline__ void advance2(StagePtr& P, int group_bytes) {
#pragma unroll
    for (int tt = 0; tt < kGemvTiles; ++tt) {
        P.og[tt] += 2 * group_bytes;
        P.oh[tt] += 2 * group_bytes;
        P.o12[tt] += 2 * group_bytes;
        P.osg[tt] += 2;
        P.osh[tt] += 2;
    }
}

// Decode one row's bytes 6c..6c+5 of a base-3 group into 15 registers
// (CHECK: also OR the table entries into err, whose bit 31 flags codes >= 243).
template <bool CHECK = true>
__device__ __forceinline__ void b3_decode_pairs(uint32_t W0, uint32_t W1, uint32_t o8, uint32_t lane_addr,
                                                uint32_t (&R)[15], uint32_t& err) {
    const uint32_t lo = __funnelshift_r(W0, W1, o8);
    const uint32_t hi = W1 >> o8;
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        const uint32_t src = q == 2 ? hi : lo;
        const uint32_t b = q == 1 ? 2u : 0u;
        // address = table + code * 256 + lane * 4 (+128 for the high table)
        const uint32_t va = lut_u32(prmt(src, lane_addr, 0x5504u | (b << 4)));
        const uint32_t vb = lut_u32(prmt(src, lane_addr, 0x5504u | ((b + 1) << 4)) + 128);
        if (CHECK) err = lop3_or3(err, va, vb);
#pragma unroll
        for (int i = 0; i < 5; ++i) R[5 * q + i] = lop3_or_and(va, vb, fmask(i));
    }
}

struct LaneCtx {
    uint32_t lane_addr;          // lane * 4: byte offset of this lane's table column
    uint32_t mG[3], mH[3];       // pair-12 field masks for rows g and g+8
    uint32_t bbase[2], bstride[2];        // activation fragment base/stride per column tile (shared)
    uint32_t mbase[2][2], mstride[2][2];  // meta base/stride per column tile and column
};

// One group j for the warp's tiles: activation fragments, decode, MMA, scale.
template <int LAYOUT, int MT, bool BSMEM, bool M1>
__device__ __forceinline__ void process_group(const GemvArgs& a, const CodeStage<LAYOUT>& S, int j,
                                              uint32_t o8g, uint32_t o8h, const LaneCtx& cx,
                                              float (&acc)[kGemvTiles][MT][4], uint32_t& err) {
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    uint32_t bf[MT][NT][2];
    float pm[MT][2], cm[MT][2];
    if constexpr (BSMEM) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const uint32_t ba = cx.bbase[mt] + static_cast<uint32_t>(j) * cx.bstride[mt];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint2 v = lds_u64(ba + 32 * t);
                bf[mt][t][0] = v.x;
                bf[mt][t][1] = v.y;
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                if (M1 && r == 1) { cm[mt][1] = 0.f; pm[mt][1] = 0.f; continue; }
                const uint2 md = lds_u64(cx.mbase[mt][r] + static_cast<uint32_t>(j) * cx.mstride[mt][r]);
                cm[mt][r] = __uint_as_float(md.x);
                pm[mt][r] = __uint_as_float(md.y);
            }
        }
    } else {
        const int G = a.G;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int m = mt * 8 + g;
            const uint32_t* bp = a.bslots + (((int64_t)m * G + j) * NT) * 8 + c * 2;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                uint2 v = make_uint2(0u, 0u);
                if (m < a.M) v = ldg_u64(bp + t * 8);
                bf[mt][t][0] = v.x;
                bf[mt][t][1] = v.y;
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int mm = mt * 8 + 2 * c + r;
                float2 md = make_float2(0.f, 0.f);
                if (mm < a.M) md = __ldg(a.meta + (int64_t)mm * G + j);
                cm[mt][r] = md.x;
                pm[mt][r] = md.y;
            }
        }
        if (j + 1 < G) {
            // the next group's fragment lines and meta into L1
            constexpr int lines = (NT * 32 + 127) / 128;
            if (lane < a.M * (lines + 1)) {
                const int mm = lane / (lines + 1), l = lane % (lines + 1);
                if (l < lines)
                    prefetch_l1(reinterpret_cast<const uint8_t*>(a.bslots + (((int64_t)mm * G + j + 1) * NT) * 8) + 128 * l);
                else
                    prefetch_l1(a.meta + (int64_t)mm * G + j + 1);
            }
        }
    }
#pragma unroll
    for (int tt = 0; tt < kGemvTiles; ++tt) {
        const float sg = f16_bits_to_f32(S.s[tt][0]);
        const float sh = f16_bits_to_f32(S.s[tt][1]);
        uint32_t Rg[16], Rh[16], QG[3], QH[3];
        if constexpr (LAYOUT == BT_LAYOUT_B3) {
            uint32_t r15[15];
            b3_decode_pairs(S.w[tt][0], S.w[tt][1], o8g, cx.lane_addr, r15, err);
#pragma unroll
            for (int i = 0; i < 15; ++i) Rg[i] = r15[i];
            b3_decode_pairs(S.w[tt][2], S.w[tt][3], o8h, cx.lane_addr, r15, err);
#pragma unroll
            for (int i = 0; i < 15; ++i) Rh[i] = r15[i];
            Rg[15] = Rh[15] = 0u;
            const uint32_t w12 = S.w[tt][4];
            const uint32_t va = lut_u32(prmt(w12, cx.lane_addr, 0x5504u));
            const uint32_t vb = lut_u32(prmt(w12, cx.lane_addr, 0x5514u) + 128);
            err = lop3_or3(err, va, vb);
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                QG[i] = lop3_or_and(va, vb, cx.mG[i]);
                QH[i] = lop3_or_and(va, vb, cx.mH[i]);
            }
        } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const uint32_t w = S.w[tt][r];
                const uint32_t w12s = w >> 12;
                uint32_t* Rr = r < 2 ? Rg : Rh;
                const int base = (r & 1) * 8;
#pragma unroll
                for (int f = 0; f < 6; ++f) Rr[base + f] = w & fmask(f);
                Rr[base + 6] = w12s & fmask(0);
                Rr[base + 7] = w12s & fmask(1);
                err |= w & (w >> 1);
            }
#pragma unroll
            for (int i = 0; i < 3; ++i) QG[i] = QH[i] = 0u;
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float d[4];
            if constexpr (LAYOUT == BT_LAYOUT_B3) b3_group_mma(Rg, Rh, QG, QH, bf[mt], d);
            else tb_group_mma(Rg, Rh, bf[mt], d);
            acc[tt][mt][0] = fmaf(sg, fmaf(d[0], pm[mt][0], -cm[mt][0]), acc[tt][mt][0]);
            acc[tt][mt][2] = fmaf(sh, fmaf(d[2], pm[mt][0], -cm[mt][0]), acc[tt][mt][2]);
            if (!M1) {
                acc[tt][mt][1] = fmaf(sg, fmaf(d[1], pm[mt][1], -cm[mt][1]), acc[tt][mt][1]);
                acc[tt][mt][3] = fmaf(sh, fmaf(d[3], pm[mt][1], -cm[mt][1]), acc[tt][mt][3]);
            }
        }
    }
}

// L2 prefetch of one segment: lane l covers row l of the tile pair.
__device__ __forceinline__ void prefetch_segment(const GemvArgs& a, int p, int j0, int j1, int group_bytes) {
    const uintptr_t base = reinterpret_cast<uintptr_t>(a.codes);
    const uintptr_t lo_lim = (base + 15) & ~uintptr_t(15);
    const uintptr_t hi_lim = (base + (uintptr_t)a.N * a.row_bytes) & ~uintptr_t(15);
    for (int r = threadIdx.x & 31; r < kGemvTiles * 16; r += 32) {
        const int n = p * (kGemvTiles * 16) + r;
        if (n >= a.N) break;
        const uintptr_t row = base + (uintptr_t)n * a.row_bytes;
        uintptr_t s = (row + (uintptr_t)j0 * group_bytes) & ~uintptr_t(15);
        uintptr_t e = (row + (uintptr_t)j1 * group_bytes + 15) & ~uintptr_t(15);
        if (s < lo_lim) s = lo_lim;
        if (e > hi_lim) e = hi_lim;
        if (e > s) prefetch_l2_bulk(reinterpret_cast<const void*>(s), static_cast<uint32_t>(e - s));
        prefetch_l2(a.scales + (int64_t)n * a.G + j0);
        prefetch_l2(a.scales + (int64_t)n * a.G + (j1 - 1));
    }
}

// Block-wide copy global -> shared with eight loads in flight per thread.
template <typename T>
__device__ __forceinline__ void copy_to_smem(T* dst, const T* src, int n) {
    constexpr int U = 8;
    for (int base = 0; base < n; base += U * blockDim.x) {
        T v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x + threadIdx.x;
            if (i < n) v[u] = __ldcg(src + i);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x + threadIdx.x;
            if (i < n) dst[i] = v[u];
        }
    }
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ void store_y(void* y, int bf16, int64_t idx, float v) {
    if (bf16) reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(y)[idx] = v;
}

template <int LAYOUT, int MT, bool BSMEM, bool M1>
__global__ void __launch_bounds__(kGemvWarps * 32, 1) gemv_kernel(GemvArgs a) {
    constexpr int TL = kGemvTiles;
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    constexpr int GB = LAYOUT == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes;
    uint8_t* smem = gemv_smem;
    uint8_t* lut = smem;                                              // base-3 only
    uint8_t* sB = smem + (LAYOUT == BT_LAYOUT_B3 ? kLutBytes : 0);    // zero area, meta, slots
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int G = a.G;

    const int64_t wglobal = (int64_t)blockIdx.x * kGemvWarps + warp;
    const int64_t u_begin = wglobal * a.chunk;
    const int64_t u_end = min(a.U, u_begin + a.chunk);
    // The weights do not depend on the previous kernel: start streaming the
    // first segment into L2 before waiting for it.
    if (u_begin < u_end) {
        const int p0 = static_cast<int>(u_begin / G);
        const int j00 = static_cast<int>(u_begin - (int64_t)p0 * G);
        const int64_t j10 = (int64_t)j00 + (u_end - u_begin);
        prefetch_segment(a, p0, j00, static_cast<int>(j10 < G ? j10 : G), GB);
    }

    if constexpr (LAYOUT == BT_LAYOUT_B3) {
        // table row = code (256 B): [0,128) low table, [128,256) high table,
        // one 4-byte entry per lane. Entry: the five digits as 2-bit fields
        // at bits 2i (low) or 16 + 2i (high); bit 31 flags codes >= 243.
        // consecutive threads fill consecutive 16-byte chunks (conflict-free)
        for (int idx = threadIdx.x; idx < 256 * 16; idx += blockDim.x) {
            const int code = idx >> 4, v = idx & 15;
            uint32_t f = 0x80000000u;
            if (code < 243) {
                f = 0;
                int r = code;
#pragma unroll
                for (int i = 0; i < 5; ++i) { f |= static_cast<uint32_t>(r % 3) << (2 * i); r /= 3; }
                if (v >= 8) f <<= 16;
            }
            reinterpret_cast<uint4*>(lut)[idx] = make_uint4(f, f, f, f);
        }
    }
    const uint32_t zero_area = smem_u32addr(sB);
    const uint32_t meta_area = zero_area + kZeroBytes;
    const uint32_t slot_area = meta_area + meta_area_bytes(a.M, G);
    {
        uint4* z = reinterpret_cast<uint4*>(sB);
        for (int i = threadIdx.x; i < kZeroBytes / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    }
    pdl_wait();
    if constexpr (BSMEM) {
        // meta [M][G] float2, then slots [M][G][NT*32 B]
        const float2* gm = a.meta;
        float2* sm = reinterpret_cast<float2*>(sB + kZeroBytes);
        copy_to_smem<float2>(sm, gm, a.M * G);
        const uint4* gb = reinterpret_cast<const uint4*>(a.bslots);
        uint4* sb = reinterpret_cast<uint4*>(sB + kZeroBytes + meta_area_bytes(a.M, G));
        copy_to_smem<uint4>(sb, gb, a.M * G * NT * 2);  // NT * 32 bytes per (m, g)
    }
    __syncthreads();

    LaneCtx cx;
    cx.lane_addr = static_cast<uint32_t>(lane) * 4u;
    {
        // pair-12 field masks (base-3): even c -> fields 0,1,2; odd c -> 3,4,none.
        uint32_t mq[3];
        mq[0] = (c & 1) ? fmask(3) : fmask(0);
        mq[1] = (c & 1) ? fmask(4) : fmask(1);
        mq[2] = (c & 1) ? 0u : fmask(2);
#pragma unroll
        for (int i = 0; i < 3; ++i) { cx.mG[i] = c < 2 ? mq[i] : 0u; cx.mH[i] = c < 2 ? 0u : mq[i]; }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        const int m = mt * 8 + g;
        const bool okm = m < a.M;
        cx.bbase[mt] = okm ? slot_area + static_cast<uint32_t>(m * G * NT * 32 + c * 8) : zero_area + c * 8;
        cx.bstride[mt] = okm ? NT * 32 : 0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int mm = mt * 8 + 2 * c + r;
            const bool ok = mm < a.M;
            cx.mbase[mt][r] = ok ? meta_area + static_cast<uint32_t>(mm * G * 8) : zero_area;
            cx.mstride[mt][r] = ok ? 8 : 0;
        }
    }

    uint32_t err = 0;
    int64_t u = u_begin;
    bool first_segment = true;
    while (u < u_end) {
        const int p = static_cast<int>(u / G);
        const int j0 = static_cast<int>(u - (int64_t)p * G);
        const int64_t j1_64 = (int64_t)j0 + (u_end - u);
        const int j1 = static_cast<int>(j1_64 < G ? j1_64 : (int64_t)G);
        if (!first_segment) prefetch_segment(a, p, j0, j1, GB);

        // offsets of groups j0 (stage 0) and j0 + 1 (stage 1); base-3 window
        // shifts for each stage (a +26-byte step flips the 4-byte alignment)
        StagePtr P0, P1;
        uint32_t o8g0 = 0, o8h0 = 0, o8g1 = 0, o8h1 = 0;
#pragma unroll
        for (int tt = 0; tt < TL; ++tt) {
            const uint32_t ng = static_cast<uint32_t>(min(a.N - 1, (p * TL + tt) * 16 + g));
            const uint32_t nh = static_cast<uint32_t>(min(a.N - 1, (p * TL + tt) * 16 + g + 8));
            const uint32_t rg = ng * a.row_bytes, rh = nh * a.row_bytes;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                StagePtr& P = s ? P1 : P0;
                const uint32_t js = static_cast<uint32_t>(j0 + s) * GB;
                if constexpr (LAYOUT == BT_LAYOUT_B3) {
                    const uint32_t ug = rg + js + 6u * c, uh = rh + js + 6u * c;  // codes are 16-aligned
                    P.og[tt] = ug & ~3u;
                    P.oh[tt] = uh & ~3u;
                    P.o12[tt] = (c < 2 ? rg : rh) + js + 24u;
                    if (tt == 0) {
                        // rows 8 and 16 apart share their 4-byte alignment
                        // (8 * row_bytes is a multiple of 4), so tile 0's
                        // shifts hold for tile 1 as well
                        if (s == 0) { o8g0 = (ug & 3u) * 8u; o8h0 = (uh & 3u) * 8u; }
                        else { o8g1 = (ug & 3u) * 8u; o8h1 = (uh & 3u) * 8u; }
                    }
                } else {
                    P.og[tt] = rg + js + 8u * c;
                    P.oh[tt] = rh + js + 8u * c;
                    P.o12[tt] = 0;
                }
            }
            P0.osg[tt] = ng * G + j0;
            P0.osh[tt] = nh * G + j0;
            P1.osg[tt] = P0.osg[tt] + 1;
            P1.osh[tt] = P0.osh[tt] + 1;
        }
        float acc[TL][MT][4];
#pragma unroll
        for (int tt = 0; tt < TL; ++tt)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[tt][mt][r] = 0.f;

        // two register stages: the next group's bytes are in flight while
        // this one is decoded
        CodeStage<LAYOUT> S0, S1;
        load_stage(S0, a, P0);
        for (int j = j0; j < j1; j += 2) {
            if (j + 1 < j1) load_stage(S1, a, P1);
            advance2(P0, GB);
            process_group<LAYOUT, MT, BSMEM, M1>(a, S0, j, o8g0, o8h0, cx, acc, err);
            if (j + 1 >= j1) break;
            if (j + 2 < j1) load_stage(S0, a, P0);
            advance2(P1, GB);
            process_group<LAYOUT, MT, BSMEM, M1>(a, S1, j + 1, o8g1, o8h1, cx, acc, err);
        }

        // ---- write the segment: whole tile -> y, part of a tile -> partials + fixup
        const bool complete = (j0 == 0 && j1 == G);
        if (complete) {
#pragma unroll
            for (int tt = 0; tt < TL; ++tt)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int n = (p * TL + tt) * 16 + g + (r >> 1) * 8;
                        const int m = mt * 8 + 2 * c + (r & 1);
                        if (n < a.N && m < a.M) store_y(a.y, a.y_bf16, (int64_t)m * a.N + n, acc[tt][mt][r]);
                    }
        } else {
            const int slot = first_segment ? 0 : 1;
            float* part = a.partials + ((wglobal * 2 + slot) * (TL * 16)) * a.M;
#pragma unroll
            for (int tt = 0; tt < TL; ++tt)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int row = tt * 16 + g + (r >> 1) * 8;
                        const int m = mt * 8 + 2 * c + (r & 1);
                        if (m < a.M) __stcg(part + row * a.M + m, acc[tt][mt][r]);
                    }
            // release this warp's partials, then count the segment in
            fence_acq_rel_gpu();
            __syncwarp();
            const int64_t w_lo = ((int64_t)p * G) / a.chunk;
            const int64_t w_hi = ((int64_t)(p + 1) * G - 1) / a.chunk;
            int last = 0;
            if (lane == 0) {
                const int old = atomicAdd(a.counters + p, 1);
                last = (old == static_cast<int>(w_hi - w_lo));
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                // the last segment of the tile adds all partials in segment
                // order; lane l owns row l (loads of all segments in flight)
                fence_acq_rel_gpu();
                const int nseg = static_cast<int>(w_hi - w_lo) + 1;
                for (int row = lane; row < TL * 16; row += 32) {
                    const int n = p * TL * 16 + row;
                    for (int m = 0; m < a.M; ++m) {
                        float sum = 0.f;
                        for (int s0 = 0; s0 < nseg; s0 += 8) {
                            float v[8];
#pragma unroll
                            for (int s1 = 0; s1 < 8; ++s1) {
                                const int64_t w = w_lo + s0 + s1;
                                v[s1] = 0.f;
                                if (s0 + s1 < nseg) {
                                    const int ws = (w * a.chunk >= (int64_t)p * G) ? 0 : 1;  // w starts in p
                                    v[s1] = __ldcg(a.partials + ((w * 2 + ws) * (TL * 16) + row) * a.M + m);
                                }
                            }
#pragma unroll
                            for (int s1 = 0; s1 < 8; ++s1) sum += v[s1];
                        }
                        if (n < a.N) store_y(a.y, a.y_bf16, (int64_t)m * a.N + n, sum);
                    }
                }
                if (lane == 0) a.counters[p] = 0;
            }
        }
        u += j1 - j0;
        first_segment = false;
    }

    int bad = 0;
    if (LAYOUT == BT_LAYOUT_B3) bad = (err >> 31) ? BT_DEVERR_INVALID_CODE : 0;
    else bad = (err & 0x55555555u) ? BT_DEVERR_INVALID_CODE : 0;
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) report(a.dev_err, bad);
}

// ----------------------------------------------- GEMV, TMA-fed variant -----
//
// Used when K % 1024 == 0 and M <= 8. Work item = (64-row tile quad Q,
// 1024-block b). One producer warp streams each item's packed bytes
// ([64 rows][RB bytes], RB = 208 base-3 or 256 2-bit) and scales
// ([64 rows][8]) into a ring of shared-memory stages with 2D tensor copies,
// well ahead of use. Sixteen consumer warps split the item: warp w decodes
// group w % 8 of the block for the 32 rows of tile pair w / 8 (two 16-row
// tiles, two independent MMA chains sharing one set of activation
// fragments), so no warp waits on HBM. Each CTA owns a contiguous run of
// items; a tile quad's partial sums are reduced through shared memory in a
// fixed order, and a quad split across CTAs is finished by the CTA that
// completes it last (atomic counter), in segment order.

constexpr int kTmaConsumers = 16;
constexpr int kTmaThreads = (kTmaConsumers + 1) * 32;
constexpr int kTmaRows = 64;
constexpr int kRedBytes = kTmaConsumers * 32 * 8 * 4;   // [warp][32 rows][8 cols] floats

struct GemvTmaArgs {
    const uint32_t* bslots;
    const float2* meta;
    float* partials;         // [grid][2][64][M]
    int* counters;           // [quads]
    void* y;
    int y_bf16;
    int M, N, G, nb, stages;
    int64_t items;           // quads * nb
    int64_t chunk;           // items per CTA
    int32_t* dev_err;
};

template <int LAYOUT>
struct TmaGeom {
    static constexpr int RB = LAYOUT == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;  // 208 / 256
    static constexpr int kCodes = kTmaRows * RB;
    static constexpr int kScales = kTmaRows * 16;
    static constexpr int kStage = kCodes + kScales;
};

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t r;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(addr));
    return r;
}

__device__ __forceinline__ void consumer_bar() {
    asm volatile("bar.sync 1, %0;" :: "n"(kTmaConsumers * 32) : "memory");
}

template <int LAYOUT, bool BSMEM, bool M1, bool CHECK>
__global__ void __launch_bounds__(kTmaThreads, 1)
gemv_tma_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap smap, GemvTmaArgs a) {
    using GE = TmaGeom<LAYOUT>;
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    const int S = a.stages;
    uint8_t* smem = gemv_smem;
    uint8_t* lut = smem;
    uint8_t* sB = smem + (LAYOUT == BT_LAYOUT_B3 ? kLutBytes : 0);
    const int M = a.M, G = a.G, nb = a.nb;
    const uint32_t bbytes = BSMEM ? static_cast<uint32_t>(M * G * NT * 32) + meta_area_bytes(M, G) : 0u;
    uint8_t* stages = sB + ((kZeroBytes + bbytes + 1023) & ~1023u);
    float* red = reinterpret_cast<float*>(stages + S * GE::kStage);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + kRedBytes);
    uint64_t* empty = full + S;
    volatile int* flags = reinterpret_cast<volatile int*>(empty + S);   // [0] abort, [1] last-segment vote

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i0 = (int64_t)blockIdx.x * a.chunk;
    const int64_t i1 = min(a.items, i0 + a.chunk);
    const int nitems = static_cast<int>(i1 > i0 ? i1 - i0 : 0);
    const int Q0 = static_cast<int>(i0 / nb), b0 = static_cast<int>(i0 % nb);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(full + s), 1);
            mbar_init(smem_addr(empty + s), kTmaConsumers);
        }
        flags[0] = 0;
        flags[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if constexpr (LAYOUT == BT_LAYOUT_B3) {
        for (int idx = threadIdx.x; idx < 256 * 16; idx += blockDim.x) {
            const int code = idx >> 4, v = idx & 15;
            uint32_t f = c_b3_fields.v[code];
            if (v >= 8 && code < 243) f <<= 16;
            reinterpret_cast<uint4*>(lut)[idx] = make_uint4(f, f, f, f);
        }
    }
    for (int i = threadIdx.x; i < kZeroBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sB)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();

    int bad = 0;
    if (warp == kTmaConsumers) {
        // ---------------- producer: the weights do not depend on the previous
        // kernel, so streaming starts before the dependency wait
        if (lane == 0) {
            int Q = Q0, b = b0;
            int s = 0;
            uint32_t ph = 0;                 // parity of the current pass over the ring
            for (int it = 0; it < nitems; ++it) {
                if (it >= S && !mbar_wait(smem_addr(empty + s), ph ^ 1u)) {
                    bad = BT_DEVERR_TIMEOUT; flags[0] = 1; break;
                }
                if (flags[0]) break;
                const uint32_t dst = smem_addr(stages + s * GE::kStage);
                mbar_arrive_tx(smem_addr(full + s), GE::kStage);
                tma_load_2d(dst, &cmap, b * GE::RB, Q * kTmaRows, smem_addr(full + s));
                tma_load_2d(dst + GE::kCodes, &smap, b * 8, Q * kTmaRows, smem_addr(full + s));
                if (++b == nb) { b = 0; ++Q; }
                if (++s == S) { s = 0; ph ^= 1u; }
            }
        }
        pdl_wait();
    } else {
        // ---------------- consumers
        const int q = warp & 7, h = warp >> 3;
        const int g = lane >> 2, c = lane & 3;
        pdl_wait();
        if constexpr (BSMEM) {
            float2* smeta = reinterpret_cast<float2*>(sB + kZeroBytes);
            for (int i = threadIdx.x; i < M * G; i += kTmaConsumers * 32) smeta[i] = __ldcg(a.meta + i);
            const uint4* gb = reinterpret_cast<const uint4*>(a.bslots);
            uint4* sb = reinterpret_cast<uint4*>(sB + kZeroBytes + meta_area_bytes(M, G));
            const int n16 = M * G * NT * 2;
            for (int base = 0; base < n16; base += 8 * kTmaConsumers * 32) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = base + u * kTmaConsumers * 32 + threadIdx.x;
                    if (i < n16) v[u] = __ldcg(gb + i);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = base + u * kTmaConsumers * 32 + threadIdx.x;
                    if (i < n16) sb[i] = v[u];
                }
            }
            consumer_bar();
        }
        const uint32_t zero_area = smem_u32addr(sB);
        const uint32_t meta_area = zero_area + kZeroBytes;
        const uint32_t slot_area = meta_area + meta_area_bytes(M, G);
        const int m = g;                                  // activation row of this lane's fragment column
        const bool okm = m < M;
        const uint32_t bbase = okm ? slot_area + static_cast<uint32_t>(m * G * NT * 32 + c * 8) : zero_area + c * 8;
        const uint32_t bstride = okm ? NT * 32 : 0;
        uint32_t mbase[2], mstride[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int mm = 2 * c + r;
            const bool ok = mm < M;
            mbase[r] = ok ? meta_area + static_cast<uint32_t>(mm * G * 8) : zero_area;
            mstride[r] = ok ? 8 : 0;
        }
        uint32_t mq[3];
        mq[0] = (c & 1) ? fmask(3) : fmask(0);
        mq[1] = (c & 1) ? fmask(4) : fmask(1);
        mq[2] = (c & 1) ? 0u : fmask(2);
        uint32_t mG[3], mH[3];
#pragma unroll
        for (int i = 0; i < 3; ++i) { mG[i] = c < 2 ? mq[i] : 0u; mH[i] = c < 2 ? 0u : mq[i]; }
        const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
        // this warp's byte offset inside a stage row, and the base-3 window shift
        const uint32_t off = LAYOUT == BT_LAYOUT_B3 ? static_cast<uint32_t>(q * kB3GroupBytes + 6 * c)
                                                    : static_cast<uint32_t>(q * k2bGroupBytes + 8 * c);
        const uint32_t o8 = LAYOUT == BT_LAYOUT_B3 ? (off & 3u) * 8u : 0u;
        const uint32_t a4 = LAYOUT == BT_LAYOUT_B3 ? (off & ~3u) : off;

        uint32_t err = 0;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        int seg_start = 0;                                 // item index where the open segment began
        int Q = Q0, b = b0;
        int s = 0;
        uint32_t ph = 0;
        for (int it = 0; it < nitems; ++it) {
            const int j = 8 * b + q;
            // an aborted CTA keeps walking its items (no waits, no work) so that
            // every consumer warp still meets every barrier below
            bool ok = !flags[0];
            if (ok && !mbar_wait(smem_addr(full + s), ph)) { bad = BT_DEVERR_TIMEOUT; flags[0] = 1; ok = false; }
            if (ok) {
                const uint32_t st = smem_u32addr(stages + s * GE::kStage);
                const uint32_t sc = st + GE::kCodes;
                uint32_t w[2][5];
                float sgv[2], shv[2];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    const int rg = h * 32 + tt * 16 + g, rh = rg + 8;
                    sgv[tt] = f16_bits_to_f32(lds_u16(sc + rg * 16 + 2 * q));
                    shv[tt] = f16_bits_to_f32(lds_u16(sc + rh * 16 + 2 * q));
                    if constexpr (LAYOUT == BT_LAYOUT_B3) {
                        w[tt][0] = lds_u32(st + rg * GE::RB + a4);
                        w[tt][1] = lds_u32(st + rg * GE::RB + a4 + 4);
                        w[tt][2] = lds_u32(st + rh * GE::RB + a4);
                        w[tt][3] = lds_u32(st + rh * GE::RB + a4 + 4);
                        w[tt][4] = lds_u16(st + (c < 2 ? rg : rh) * GE::RB + q * kB3GroupBytes + 24);
                    } else {
                        const uint2 x0 = lds_u64(st + rg * GE::RB + a4);
                        const uint2 x1 = lds_u64(st + rh * GE::RB + a4);
                        w[tt][0] = x0.x; w[tt][1] = x0.y; w[tt][2] = x1.x; w[tt][3] = x1.y; w[tt][4] = 0;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(empty + s));   // the stage may be refilled

                // activation fragments and group constants
                uint32_t bf[NT][2];
                float pm[2], cm[2];
                if constexpr (BSMEM) {
                    const uint32_t ba = bbase + static_cast<uint32_t>(j) * bstride;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const uint2 v = lds_u64(ba + 32 * t);
                        bf[t][0] = v.x;
                        bf[t][1] = v.y;
                    }
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        if (M1 && r == 1) { cm[1] = 0.f; pm[1] = 0.f; continue; }
                        const uint2 md = lds_u64(mbase[r] + static_cast<uint32_t>(j) * mstride[r]);
                        cm[r] = __uint_as_float(md.x);
                        pm[r] = __uint_as_float(md.y);
                    }
                } else {
                    const uint32_t* bp = a.bslots + (((int64_t)m * G + j) * NT) * 8 + c * 2;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        uint2 v = make_uint2(0u, 0u);
                        if (okm) v = ldg_u64(bp + t * 8);
                        bf[t][0] = v.x;
                        bf[t][1] = v.y;
                    }
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int mm = 2 * c + r;
                        float2 md = make_float2(0.f, 0.f);
                        if (mm < M) md = __ldg(a.meta + (int64_t)mm * G + j);
                        cm[r] = md.x;
                        pm[r] = md.y;
                    }
                }
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    uint32_t Rg[16], Rh[16], QG[3], QH[3];
                    if constexpr (LAYOUT == BT_LAYOUT_B3) {
                        uint32_t r15[15];
                        b3_decode_pairs<CHECK>(w[tt][0], w[tt][1], o8, lane4, r15, err);
#pragma unroll
                        for (int k = 0; k < 15; ++k) Rg[k] = r15[k];
                        b3_decode_pairs<CHECK>(w[tt][2], w[tt][3], o8, lane4, r15, err);
#pragma unroll
                        for (int k = 0; k < 15; ++k) Rh[k] = r15[k];
                        Rg[15] = Rh[15] = 0u;
                        const uint32_t va = lut_u32(prmt(w[tt][4], lane4, 0x5504u));
                        const uint32_t vb = lut_u32(prmt(w[tt][4], lane4, 0x5514u) + 128);
                        if (CHECK) err = lop3_or3(err, va, vb);
#pragma unroll
                        for (int k = 0; k < 3; ++k) {
                            QG[k] = lop3_or_and(va, vb, mG[k]);
                            QH[k] = lop3_or_and(va, vb, mH[k]);
                        }
                    } else {
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const uint32_t x = w[tt][r];
                            const uint32_t x12 = x >> 12;
                            uint32_t* Rr = r < 2 ? Rg : Rh;
                            const int base = (r & 1) * 8;
#pragma unroll
                            for (int f = 0; f < 6; ++f) Rr[base + f] = x & fmask(f);
                            Rr[base + 6] = x12 & fmask(0);
                            Rr[base + 7] = x12 & fmask(1);
                            if (CHECK) err |= x & (x >> 1);
                        }
#pragma unroll
                        for (int k = 0; k < 3; ++k) QG[k] = QH[k] = 0u;
                    }
                    // two accumulator chains (even / odd MMA steps) halve the
                    // dependent MMA latency per tile
                    float d[4];
                    if constexpr (LAYOUT == BT_LAYOUT_B3) b3_group_mma(Rg, Rh, QG, QH, bf, d);
                    else tb_group_mma(Rg, Rh, bf, d);
                    acc[tt][0] = fmaf(sgv[tt], fmaf(d[0], pm[0], -cm[0]), acc[tt][0]);
                    acc[tt][2] = fmaf(shv[tt], fmaf(d[2], pm[0], -cm[0]), acc[tt][2]);
                    if (!M1) {
                        acc[tt][1] = fmaf(sgv[tt], fmaf(d[1], pm[1], -cm[1]), acc[tt][1]);
                        acc[tt][3] = fmaf(shv[tt], fmaf(d[3], pm[1], -cm[1]), acc[tt][3]);
                    }
                }
            }  // ok

            if (++s == S) { s = 0; ph ^= 1u; }

            // ---- close the quad's segment at a quad boundary or at the end
            const int Qcur = Q;
            const int bcur = b;
            if (++b == nb) { b = 0; ++Q; }
            const bool boundary = (it + 1 == nitems) || (Q != Qcur);
            if (boundary) {
                float* rw = red + warp * 32 * 8;                 // [32 rows][8 cols]
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int row = tt * 16 + g + (r >> 1) * 8, col = 2 * c + (r & 1);
                        rw[row * 8 + col] = acc[tt][r];
                    }
                consumer_bar();
                const int64_t seg_i0 = i0 + seg_start;
                const bool whole = (seg_i0 % nb == 0) && (bcur == nb - 1);
                const int tid = threadIdx.x;
                float* part = a.partials + (((int64_t)blockIdx.x * 2 + (seg_start == 0 ? 0 : 1)) * kTmaRows) * M;
                for (int e = tid; e < kTmaRows * M; e += kTmaConsumers * 32) {
                    const int row = e / M, col = e % M;
                    const int hh = row >> 5, lr = row & 31;
                    float sum = 0.f;
#pragma unroll
                    for (int qq = 0; qq < 8; ++qq) sum += red[((hh * 8 + qq) * 32 + lr) * 8 + col];
                    const int n = Qcur * kTmaRows + row;
                    if (whole) {
                        if (n < a.N) store_y(a.y, a.y_bf16, (int64_t)col * a.N + n, sum);
                    } else {
                        __stcg(part + row * M + col, sum);
                    }
                }
                if (!whole) {
                    fence_acq_rel_gpu();
                    consumer_bar();
                    const int64_t c_lo = ((int64_t)Qcur * nb) / a.chunk;
                    const int64_t c_hi = ((int64_t)(Qcur + 1) * nb - 1) / a.chunk;
                    if (tid == 0) {
                        const int old = atomicAdd(a.counters + Qcur, 1);
                        flags[1] = (old == static_cast<int>(c_hi - c_lo)) ? 1 : 0;
                    }
                    consumer_bar();
                    if (flags[1]) {
                        fence_acq_rel_gpu();
                        for (int e = tid; e < kTmaRows * M; e += kTmaConsumers * 32) {
                            const int row = e / M, col = e % M;
                            float sum = 0.f;
                            for (int64_t cc = c_lo; cc <= c_hi; ++cc) {
                                const int sl = (cc * a.chunk >= (int64_t)Qcur * nb) ? 0 : 1;   // cc starts in Q
                                sum += __ldcg(a.partials + ((cc * 2 + sl) * kTmaRows + row) * M + col);
                            }
                            const int n = Qcur * kTmaRows + row;
                            if (n < a.N) store_y(a.y, a.y_bf16, (int64_t)col * a.N + n, sum);
                        }
                        if (tid == 0) a.counters[Qcur] = 0;
                    }
                }
                consumer_bar();
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) acc[tt][0] = acc[tt][1] = acc[tt][2] = acc[tt][3] = 0.f;
                seg_start = it + 1;
            }
        }
        if (LAYOUT == BT_LAYOUT_B3) { if (err >> 31) bad |= BT_DEVERR_INVALID_CODE; }
        else if (err & 0x55555555u) bad |= BT_DEVERR_INVALID_CODE;
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) report(a.dev_err, bad);
}

// ------------------------------------------------------------ host ---------

struct GemvPlan {
    int NT, MT, P, grid, warps_total, prep_grid;
    int64_t G, U, chunk;
    bool bsmem;
    size_t smem;
    size_t off_bslots, off_meta, off_counters, off_partials, total;
};

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static GemvPlan make_gemv_plan(int layout, int64_t M, int64_t N, int64_t K, int num_sms) {
    GemvPlan pl{};
    pl.NT = layout == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    pl.MT = M > 8 ? 2 : 1;
    pl.G = K / kGroup;
    const int64_t tiles = (N + 15) / 16;
    pl.P = static_cast<int>((tiles + kGemvTiles - 1) / kGemvTiles);
    pl.U = (int64_t)pl.P * pl.G;
    const int64_t max_warps = (int64_t)num_sms * kGemvWarps;
    const int64_t min_chunk = 4;
    int64_t warps_needed = (pl.U + min_chunk - 1) / min_chunk;
    if (warps_needed < 1) warps_needed = 1;
    pl.grid = warps_needed >= max_warps ? num_sms
                                        : static_cast<int>((warps_needed + kGemvWarps - 1) / kGemvWarps);
    pl.warps_total = pl.grid * kGemvWarps;
    pl.chunk = (pl.U + pl.warps_total - 1) / pl.warps_total;
    if (pl.chunk < 1) pl.chunk = 1;
    pl.prep_grid = static_cast<int>(M * ((pl.G + 7) / 8));
    const size_t bbytes = (size_t)M * pl.G * pl.NT * 32 + meta_area_bytes((int)M, (int)pl.G);
    pl.bsmem = M <= 8 && bbytes <= kBsmemMax;
    pl.smem = (layout == BT_LAYOUT_B3 ? kLutBytes : 0) + kZeroBytes + (pl.bsmem ? bbytes : 0);
    size_t off = 0;
    pl.off_bslots = off;
    off = align_up(off + (size_t)M * pl.G * pl.NT * 32, 256);
    pl.off_meta = off;
    off = align_up(off + (size_t)M * pl.G * sizeof(float2), 256);
    pl.off_counters = off;
    off = align_up(off + (size_t)pl.P * sizeof(int), 256);
    pl.off_partials = off;
    // partials: enough for either kernel (the TMA-fed one needs grid x 2 x 32 x M)
    off = align_up(off + (size_t)pl.warps_total * 2 * kGemvTiles * 16 * M * sizeof(float), 256);
    pl.total = off;
    return pl;
}

// Products whose weights TMA can stream take the kernels of bt_gemv_lut.cu;
// a workspace sized here serves either path.
size_t gemv_lut_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K);

size_t gemv_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K, int num_sms) {
    // the continuous layout has the table-lookup kernel only
    if (layout == BT_LAYOUT_B3C) return gemv_lut_workspace_bytes(layout, M, N, K);
    size_t need = make_gemv_plan(layout, M, N, K, num_sms).total;
    if (K % 1024 == 0) {  // (alignment of the pointers is not known here)
        const size_t lut = gemv_lut_workspace_bytes(layout, M, N, K);
        if (lut > need) need = lut;
    }
    return need;
}

// TMA-fed variant: applies to M <= 8, K % 1024 == 0, 16-byte aligned scales,
// and activation fragments that fit next to the table and the stage ring.
struct TmaPlan {
    bool use, bsmem;
    int grid, nb, stages;
    int64_t items, chunk;
    size_t smem;
};

static TmaPlan make_tma_plan(int layout, int64_t M, int64_t N, int64_t K, const void* scales, int num_sms) {
    TmaPlan t{};
    const int NT = layout == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    const int G = static_cast<int>(K / kGroup);
    t.use = M <= 8 && K % kBlock == 0 && (reinterpret_cast<uintptr_t>(scales) & 15) == 0;
    if (!t.use) return t;
    t.nb = static_cast<int>(K / kBlock);
    const int64_t quads = (N + kTmaRows - 1) / kTmaRows;
    t.items = quads * t.nb;
    t.grid = static_cast<int>(t.items < num_sms ? t.items : num_sms);
    t.chunk = (t.items + t.grid - 1) / t.grid;
    const int RB = layout == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;
    const size_t stage = (size_t)kTmaRows * RB + kTmaRows * 16;
    const size_t limit = 227 * 1024;
    const size_t lutb = layout == BT_LAYOUT_B3 ? kLutBytes : 0;
    const size_t bbytes = align_up(kZeroBytes + (size_t)M * G * NT * 32 + meta_area_bytes((int)M, G), 1024);
    const size_t nob = align_up(kZeroBytes, 1024);
    t.use = false;
    for (int st : {6, 5, 4, 3}) {      // prefer activation fragments in shared memory, then more stages
        const size_t with_b = lutb + bbytes + (size_t)st * stage + kRedBytes + 256;
        if (with_b <= limit) { t.use = true; t.bsmem = true; t.stages = st; t.smem = with_b; break; }
    }
    if (!t.use) {
        for (int st : {6, 5, 4, 3}) {
            const size_t wo = lutb + nob + (size_t)st * stage + kRedBytes + 256;
            if (wo <= limit) { t.use = true; t.bsmem = false; t.stages = st; t.smem = wo; break; }
        }
    }
    return t;
}

template <int LAYOUT, bool BSMEM, bool M1, bool CHECK>
static cudaError_t launch_gemv_tma_t(const CUtensorMap& cmap, const CUtensorMap& smap, const GemvTmaArgs& ta,
                                     const TmaPlan& tp, cudaStream_t stream) {
    auto kern = gemv_tma_kernel<LAYOUT, BSMEM, M1, CHECK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tp.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(tp.grid);
    cfg.blockDim = dim3(kTmaThreads);
    cfg.dynamicSmemBytes = tp.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, cmap, smap, ta);
}

template <int LAYOUT, bool CHECK>
static cudaError_t dispatch_gemv_tma_c(const CUtensorMap& cmap, const CUtensorMap& smap, const GemvTmaArgs& ta,
                                       const TmaPlan& tp, cudaStream_t s) {
    // (single-row calls that qualify for this kernel take the table-lookup
    // kernel instead, so the M = 1 specialisation is not instantiated here)
    if (tp.bsmem) return launch_gemv_tma_t<LAYOUT, true, false, CHECK>(cmap, smap, ta, tp, s);
    return launch_gemv_tma_t<LAYOUT, false, false, CHECK>(cmap, smap, ta, tp, s);
}

// Code validation costs an ALU op per byte pair; it runs when the caller
// passes an error word to report into.
template <int LAYOUT>
static cudaError_t dispatch_gemv_tma(const CUtensorMap& cmap, const CUtensorMap& smap, const GemvTmaArgs& ta,
                                     const TmaPlan& tp, cudaStream_t s) {
    return ta.dev_err ? dispatch_gemv_tma_c<LAYOUT, true>(cmap, smap, ta, tp, s)
                      : dispatch_gemv_tma_c<LAYOUT, false>(cmap, smap, ta, tp, s);
}

template <int LAYOUT, int MT, bool BSMEM, bool M1>
static cudaError_t launch_gemv_t(const GemvArgs& ga, const GemvPlan& pl, cudaStream_t stream) {
    auto kern = gemv_kernel<LAYOUT, MT, BSMEM, M1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, ga);
}

template <int LAYOUT>
static cudaError_t dispatch_gemv(const GemvArgs& ga, const GemvPlan& pl, cudaStream_t s) {
    if (ga.M == 1 && pl.bsmem) return launch_gemv_t<LAYOUT, 1, true, true>(ga, pl, s);
    if (pl.MT == 1)
        return pl.bsmem ? launch_gemv_t<LAYOUT, 1, true, false>(ga, pl, s)
                        : launch_gemv_t<LAYOUT, 1, false, false>(ga, pl, s);
    return launch_gemv_t<LAYOUT, 2, false, false>(ga, pl, s);
}

cudaError_t launch_gemv(int layout, const uint8_t* codes, const uint16_t* scales, const void* x,
                        int x_dtype, const int8_t* sign, int64_t M, int64_t N, int64_t K, int y_dtype,
                        void* y, void* workspace, int32_t* dev_err, int num_sms,
                        cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const GemvPlan pl = make_gemv_plan(layout, M, N, K, num_sms);

    PrepArgs pa{};
    pa.x = x;
    pa.x_bf16 = x_dtype == BT_BF16;
    pa.sign = sign;
    pa.M = static_cast<int>(M);
    pa.K = static_cast<int>(K);
    pa.G = static_cast<int>(pl.G);
    pa.bslots = reinterpret_cast<uint32_t*>(ws + pl.off_bslots);
    pa.meta = reinterpret_cast<float2*>(ws + pl.off_meta);
    pa.counters = reinterpret_cast<int*>(ws + pl.off_counters);
    pa.P = pl.P;
    if (layout == BT_LAYOUT_B3)
        gemv_prep_kernel<BT_LAYOUT_B3><<<pl.prep_grid, kPrepThreads, 0, stream>>>(pa);
    else
        gemv_prep_kernel<BT_LAYOUT_2BIT><<<pl.prep_grid, kPrepThreads, 0, stream>>>(pa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // The TMA-fed kernel takes up to 8 activation rows (one n8 MMA column
    // block); 9-16 rows run as two launches over the same prepared
    // fragments, each streaming the weights once.
    const TmaPlan tp = make_tma_plan(layout, M < 8 ? M : 8, N, K, scales, num_sms);
    EncodeTiledFn enc = tp.use ? tensor_map_encoder() : nullptr;
    if (tp.use && enc) {
        const int RB = layout == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;
        const cuuint64_t row_bytes = (K / kGroup) * (layout == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes);
        CUtensorMap cmap, smap;
        const cuuint64_t cdim[2] = {row_bytes, static_cast<cuuint64_t>(N)};
        const cuuint64_t cstr[1] = {row_bytes};
        const cuuint32_t cbox[2] = {static_cast<cuuint32_t>(RB), kTmaRows};
        const cuuint64_t sdim[2] = {static_cast<cuuint64_t>(pl.G), static_cast<cuuint64_t>(N)};
        const cuuint64_t sstr[1] = {static_cast<cuuint64_t>(pl.G) * 2};
        const cuuint32_t sbox[2] = {8, kTmaRows};
        const cuuint32_t one[2] = {1, 1};
        const bool okc = enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), cdim, cstr, cbox,
                             one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        const bool oks = okc && enc(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(scales), sdim,
                                    sstr, sbox, one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        if (oks) {
            for (int64_t m0 = 0; m0 < M; m0 += 8) {
                // each launch waits for the previous one (programmatic
                // dependency) before it touches the partials; tile counters
                // are back at zero when a launch ends
                GemvTmaArgs ta{};
                ta.bslots = pa.bslots + m0 * pl.G * pl.NT * 8;
                ta.meta = pa.meta + m0 * pl.G;
                ta.partials = reinterpret_cast<float*>(ws + pl.off_partials);
                ta.counters = pa.counters;
                ta.y = static_cast<uint8_t*>(y) + m0 * N * (y_dtype == BT_BF16 ? 2 : 4);
                ta.y_bf16 = y_dtype == BT_BF16;
                ta.M = static_cast<int>(M - m0 < 8 ? M - m0 : 8);
                ta.N = static_cast<int>(N);
                ta.G = static_cast<int>(pl.G);
                ta.nb = tp.nb;
                ta.stages = tp.stages;
                ta.items = tp.items;
                ta.chunk = tp.chunk;
                ta.dev_err = dev_err;
                const cudaError_t e2 = layout == BT_LAYOUT_B3
                                           ? dispatch_gemv_tma<BT_LAYOUT_B3>(cmap, smap, ta, tp, stream)
                                           : dispatch_gemv_tma<BT_LAYOUT_2BIT>(cmap, smap, ta, tp, stream);
                if (e2 != cudaSuccess) return e2;
            }
            return cudaSuccess;
        }
    }

    GemvArgs ga{};
    ga.codes = codes;
    ga.scales = scales;
    ga.bslots = pa.bslots;
    ga.meta = pa.meta;
    ga.partials = reinterpret_cast<float*>(ws + pl.off_partials);
    ga.counters = pa.counters;
    ga.y = y;
    ga.y_bf16 = y_dtype == BT_BF16;
    ga.M = static_cast<int>(M);
    ga.N = static_cast<int>(N);
    ga.G = static_cast<int>(pl.G);
    ga.row_bytes = static_cast<uint32_t>((K / kGroup) * (layout == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes));
    ga.U = pl.U;
    ga.chunk = pl.chunk;
    ga.dev_err = dev_err;
    return layout == BT_LAYOUT_B3 ? dispatch_gemv<BT_LAYOUT_B3>(ga, pl, stream)
                                  : dispatch_gemv<BT_LAYOUT_2BIT>(ga, pl, stream);
}

// ------------------------------------------------ allocation-free variant ---
//
// Scratch for bt_gemv_noalloc: a fixed array in device memory, reserved by
// every GPU that loads the library for as long as the process lives. Host
// code only ever sees a stand-in for `noalloc_scratch`, so its device address
// is looked up with cudaGetSymbolAddress in the context that is current on the
// calling thread. The address belongs to that context's copy of the module,
// so it is cached per context (not per device ordinal): a context created
// later on the same device -- after cudaDeviceReset, or a caller's own
// non-primary context -- gets its own lookup, never a stale address.
// Every call uses it as plain scratch: no call expects particular contents.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxContexts = 64;
static std::mutex g_scratch_mutex;
static CUcontext g_scratch_ctx[kMaxContexts];
static void* g_scratch_ptr[kMaxContexts];
static int g_scratch_used = 0;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    return fn;
}

size_t gemv_noalloc_max_bytes() { return kNoAllocScratchBytes; }

cudaError_t gemv_noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    CtxGetCurrentFn get = ctx_get_current();
    CUcontext ctx = nullptr;
    if (get && get(&ctx) == CUDA_SUCCESS && ctx) {
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        for (int i = 0; i < g_scratch_used; ++i) {
            if (g_scratch_ctx[i] == ctx) {
                *out = g_scratch_ptr[i];
                return cudaSuccess;
            }
        }
    }
    // first call in this context (or no context yet: the runtime binds the
    // device's primary context here)
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, noalloc_scratch);
    if (e != cudaSuccess) return e;
    ctx = nullptr;
    if (get && get(&ctx) == CUDA_SUCCESS && ctx) {
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        bool known = false;
        for (int i = 0; i < g_scratch_used; ++i) known = known || g_scratch_ctx[i] == ctx;
        if (!known && g_scratch_used < kMaxContexts) {
            g_scratch_ctx[g_scratch_used] = ctx;
            g_scratch_ptr[g_scratch_used] = p;
            ++g_scratch_used;
        }
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace bt

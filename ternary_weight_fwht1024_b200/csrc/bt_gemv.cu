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
//  1. gemv_prep: rotates x (when a sign vector is given) and writes, per row m
//     and 128-group g, the activations in the order the tensor-core fragments
//     want them ("slots"), as FP16 scaled by 2^(24 - 2 i - e_g). e_g is a
//     power-of-two exponent chosen from the group's largest |x'|, i the
//     position of the trit's 2-bit field inside a 16-bit half (see 2.). It
//     also writes corr_g = sum_k x~_k (the FP16-rounded activations, back in
//     real units) and 2^e_g.
//
//  2. gemv: a persistent kernel. Each warp owns a contiguous run of (16-row
//     tile pair, group) units and streams the packed bytes straight from HBM
//     into registers. Base-3 bytes go through a 256-entry table in shared
//     memory, replicated per lane so the gathers are conflict-free, that
//     turns a byte into its five base-3 digits d = t + 1 as 2-bit fields;
//     2-bit bytes already are such fields. One LOP3 per two weights then
//     isolates field i of two bytes into the two halves of a register. Read
//     as FP16, the half is the subnormal d * 4^i * 2^-24, exact. An
//     m16n8k16 tensor-core MMA against the slot-ordered activations gives
//     D = 2^-e sum_k d_k x~_k in FP32, and the group contributes
//     s * (2^e D - corr) = s * sum_k t_k x~_k. The MMA's A operand is the
//     weights (16 rows); its 8 columns are the activation rows m.
//     Units that split a tile across warps leave FP32 partials; the warp
//     that finishes a tile last (atomic counter) adds them in a fixed order,
//     so results are deterministic.
#include "bt_internal.cuh"

namespace bt {

constexpr int kGemvWarps = 16;
constexpr int kGemvTiles = 2;        // 16-row tiles per unit (share the activation fragments)
constexpr int kPrepWarps = 4;
constexpr int kLutBytes = 256 * 256; // 256 codes x (128 B low table + 128 B high table)

// field mask: 2-bit field i of both 16-bit halves
__host__ __device__ constexpr uint32_t fmask(int i) {
    return (3u << (2 * i)) | (3u << (2 * i + 16));
}

// ---------------------------------------------------------- slot maps ----
// Slot (t, c, h): MMA step t of a group, lane c of a quad (threadID_in_group),
// half h: 0/1 = low/high half of fragment register a0, 2/3 = of a2.
// Returns the k (0..127) the slot carries, or -1 for an empty slot; *field is
// the 2-bit field index i of that trit inside its 16-bit half.

__device__ __forceinline__ int b3_slot(int t, int c, int h, int* field) {
    // lane c decodes byte pairs 3c, 3c+1, 3c+2 (bytes 6c..6c+5) into registers
    // rho = 5 q + i; pair 12 (bytes 24, 25) is shared by lanes c (fields
    // {0,1,2} for even c, {3,4} for odd c) and appears as registers Q0..Q2.
    const int which = h >> 1, hi = h & 1;
    int rho = -1, qi = -1;
    if (t < 7) rho = 2 * t + which;
    else if (t == 7) { if (which == 0) rho = 14; else qi = 0; }
    else qi = which == 0 ? 1 : 2;
    if (rho >= 0) {
        const int q = rho / 5, i = rho % 5, p = 3 * c + q;
        *field = i;
        return 10 * p + (hi ? 5 : 0) + i;
    }
    const int f = (c & 1) == 0 ? qi : (qi < 2 ? 3 + qi : -1);
    if (f < 0) return -1;
    const int k = (hi ? 125 : 120) + f;
    if (k >= kGroup) return -1;  // the two pad trits
    *field = f;
    return k;
}

__device__ __forceinline__ int tb_slot(int t, int c, int h, int* field) {
    // lane c holds bytes 8c..8c+7 = two words of 16 trits; register
    // rho = 8 w + f holds trits f and 8 + f of word w (f < 6 directly, f = 6, 7
    // after a 12-bit shift, then as field f - 6).
    const int rho = 2 * t + (h >> 1), hi = h & 1;
    const int w = rho >> 3, f = rho & 7;
    *field = f < 6 ? f : f - 6;
    return 32 * c + 16 * w + (hi ? 8 : 0) + f;
}

__device__ __forceinline__ int b3_field_of(int k) { return k % 5; }
__device__ __forceinline__ int tb_field_of(int k) { const int f = k & 7; return f < 6 ? f : f - 6; }

__device__ __forceinline__ float exp2i(int n) {  // 2^n for n in [-126, 127]
    return __int_as_float((n + 127) << 23);
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
__global__ void __launch_bounds__(kPrepWarps * 32) gemv_prep_kernel(PrepArgs a) {
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    __shared__ __align__(16) float tiles[kPrepWarps][32 * kTileStride];
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t i = gtid; i < a.P; i += (int64_t)gridDim.x * blockDim.x) a.counters[i] = 0;

    float* tile = tiles[warp];
    const int nblocks = (a.G + 7) / 8;
    const int64_t total = (int64_t)a.M * nblocks;
    for (int64_t wb = (int64_t)blockIdx.x * kPrepWarps + warp; wb < total;
         wb += (int64_t)gridDim.x * kPrepWarps) {
        const int m = static_cast<int>(wb / nblocks), b = static_cast<int>(wb % nblocks);
        const int64_t k0 = (int64_t)b * kBlock;
        const int ng = min(8, a.G - 8 * b);
        float v[32];
        if (a.sign) {
            load_signed_bf16_block(reinterpret_cast<const uint16_t*>(a.x) + (int64_t)m * a.K + k0, a.sign, v);
            fwht1024_warp(v, tile);
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
        for (int j = 0; j < 32; ++j) tile[32 * j + lane] = v[j];
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (q >= ng) break;
            float amax = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) amax = fmaxf(amax, fabsf(v[4 * q + r]));
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
            int E = amax > 0.f ? ilogbf(amax) + 1 : -100;  // amax < 2^E
            E = max(-100, min(100, E));
            const int e = 9 + E;
            float corr = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int k = 32 * r + lane;
                const int i = LAYOUT == BT_LAYOUT_B3 ? b3_field_of(k) : tb_field_of(k);
                const __half hv = __float2half_rn(v[4 * q + r] * exp2i(24 - 2 * i - e));
                corr += __half2float(hv) * exp2i(e + 2 * i - 24);
            }
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) corr += __shfl_xor_sync(0xffffffffu, corr, s);
            const int64_t gidx = (int64_t)m * a.G + 8 * b + q;
            if (lane == 0) a.meta[gidx] = make_float2(corr, exp2i(e));
            uint32_t* dst = a.bslots + gidx * (NT * 8);
            const float* xs = tile + 128 * q;
            for (int widx = lane; widx < NT * 8; widx += 32) {
                const int t = widx >> 3, c = (widx >> 1) & 3, hp = widx & 1;
                uint32_t word = 0;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    int i = 0;
                    const int k = LAYOUT == BT_LAYOUT_B3 ? b3_slot(t, c, 2 * hp + u, &i)
                                                         : tb_slot(t, c, 2 * hp + u, &i);
                    if (k >= 0) {
                        const __half hv = __float2half_rn(xs[k] * exp2i(24 - 2 * i - e));
                        word |= static_cast<uint32_t>(__half_as_ushort(hv)) << (16 * u);
                    }
                }
                dst[widx] = word;
            }
        }
        __syncwarp();
    }
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
    int64_t row_bytes;
    int64_t U;               // P * G units
    int64_t chunk;           // units per warp
    int32_t* dev_err;
};

__device__ __forceinline__ uint32_t lds_u32(const uint8_t* base, uint32_t off) {
    return *reinterpret_cast<const uint32_t*>(base + off);
}

// Decode one row's six bytes 6c..6c+5 of a base-3 group into 15 registers.
// W0, W1: the aligned 8-byte window holding them; o8 = 8 * (offset in window).
__device__ __forceinline__ void b3_decode_pairs(uint32_t W0, uint32_t W1, uint32_t o8, uint32_t lane4,
                                                const uint8_t* lut, uint32_t (&R)[15], uint32_t& err) {
    const uint32_t lo = __funnelshift_r(W0, W1, o8);
    const uint32_t hi = W1 >> o8;
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        const uint32_t src = q == 2 ? hi : lo;
        const uint32_t b = q == 1 ? 2u : 0u;
        const uint32_t aA = prmt(src, lane4, 0x5504u | (b << 4));
        const uint32_t aB = prmt(src, lane4, 0x5504u | ((b + 1) << 4));
        const uint32_t va = lds_u32(lut, aA);
        const uint32_t vb = lds_u32(lut, aB + 128);
        err = lop3_or3(err, va, vb);
#pragma unroll
        for (int i = 0; i < 5; ++i) R[5 * q + i] = lop3_or_and(va, vb, fmask(i));
    }
}

template <typename T>
__device__ __forceinline__ void store_y(void* y, int bf16, int64_t idx, float v) {
    if (bf16) reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(y)[idx] = v;
}

template <int LAYOUT, int MT>
__global__ void __launch_bounds__(kGemvWarps * 32, 1) gemv_kernel(GemvArgs a) {
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    constexpr int TL = kGemvTiles;
    extern __shared__ __align__(16) uint8_t lut[];
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;

    if (LAYOUT == BT_LAYOUT_B3) {
        // table row = code (256 B): [0,128) low table, [128,256) high table,
        // one 4-byte entry per lane. Entry: the five digits as 2-bit fields
        // at bits 2i (low) or 16 + 2i (high); bit 31 flags codes >= 243.
        uint32_t* lut32 = reinterpret_cast<uint32_t*>(lut);
        for (int idx = threadIdx.x; idx < 256 * 64; idx += blockDim.x) {
            const int code = idx >> 6, hi = (idx >> 5) & 1;
            uint32_t val = 0x80000000u;
            if (code < 243) {
                uint32_t f = 0;
                int r = code;
#pragma unroll
                for (int i = 0; i < 5; ++i) { f |= static_cast<uint32_t>(r % 3) << (2 * i); r /= 3; }
                val = hi ? (f << 16) : f;
            }
            lut32[idx] = val;
        }
        __syncthreads();
    }

    const int64_t wglobal = (int64_t)blockIdx.x * kGemvWarps + warp;
    const int64_t u_begin = wglobal * a.chunk;
    const int64_t u_end = min(a.U, u_begin + a.chunk);
    pdl_wait();

    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    // pair-12 field masks (base-3): even c -> fields 0,1,2; odd c -> 3,4,none.
    uint32_t mq[3];
    mq[0] = (c & 1) ? fmask(3) : fmask(0);
    mq[1] = (c & 1) ? fmask(4) : fmask(1);
    mq[2] = (c & 1) ? 0u : fmask(2);
    uint32_t mG[3], mH[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) { mG[i] = c < 2 ? mq[i] : 0u; mH[i] = c < 2 ? 0u : mq[i]; }

    uint32_t err = 0;
    const int G = a.G;
    int64_t u = u_begin;
    while (u < u_end) {
        const int p = static_cast<int>(u / G);
        const int j0 = static_cast<int>(u - (int64_t)p * G);
        const int64_t j1_64 = (int64_t)j0 + (u_end - u);
        const int j1 = static_cast<int>(j1_64 < G ? j1_64 : (int64_t)G);

        const uint8_t* rowg[TL];
        const uint8_t* rowh[TL];
        const uint16_t* scg[TL];
        const uint16_t* sch[TL];
#pragma unroll
        for (int tt = 0; tt < TL; ++tt) {
            const int ng = min(a.N - 1, (p * TL + tt) * 16 + g);
            const int nh = min(a.N - 1, (p * TL + tt) * 16 + g + 8);
            rowg[tt] = a.codes + (int64_t)ng * a.row_bytes;
            rowh[tt] = a.codes + (int64_t)nh * a.row_bytes;
            scg[tt] = a.scales + (int64_t)ng * G;
            sch[tt] = a.scales + (int64_t)nh * G;
        }
        float acc[TL][MT][4];
#pragma unroll
        for (int tt = 0; tt < TL; ++tt)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[tt][mt][r] = 0.f;

        for (int j = j0; j < j1; ++j) {
            // activation fragments and group constants, shared by the tiles
            uint32_t bf[MT][NT][2];
            float pm[MT][2], cm[MT][2];
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
#pragma unroll
            for (int tt = 0; tt < TL; ++tt) {
                const float sg = f16_bits_to_f32(__ldg(scg[tt] + j));
                const float sh = f16_bits_to_f32(__ldg(sch[tt] + j));
                uint32_t Rg[16], Rh[16];
                uint32_t QG[3], QH[3];
                if (LAYOUT == BT_LAYOUT_B3) {
                    // bytes 6c..6c+5 of the group lie in the aligned 8-byte window
                    // starting at (address & ~3); rows may differ in alignment
                    const int64_t off = (int64_t)j * kB3GroupBytes + 6 * c;
                    const uintptr_t ag = reinterpret_cast<uintptr_t>(rowg[tt] + off);
                    const uintptr_t ah = reinterpret_cast<uintptr_t>(rowh[tt] + off);
                    const uint32_t o8g = static_cast<uint32_t>(ag & 3) * 8u;
                    const uint32_t o8h = static_cast<uint32_t>(ah & 3) * 8u;
                    const uint8_t* pg = reinterpret_cast<const uint8_t*>(ag & ~uintptr_t(3));
                    const uint8_t* ph = reinterpret_cast<const uint8_t*>(ah & ~uintptr_t(3));
                    const uint32_t g0 = ldg_u32(pg), g1 = ldg_u32(pg + 4);
                    const uint32_t h0 = ldg_u32(ph), h1 = ldg_u32(ph + 4);
                    const uint8_t* pp = (c < 2 ? rowg[tt] : rowh[tt]) + (int64_t)j * kB3GroupBytes + 24;
                    const uint32_t w12 = ldg_u16(pp);
                    uint32_t r15[15];
                    b3_decode_pairs(g0, g1, o8g, lane4, lut, r15, err);
#pragma unroll
                    for (int i = 0; i < 15; ++i) Rg[i] = r15[i];
                    b3_decode_pairs(h0, h1, o8h, lane4, lut, r15, err);
#pragma unroll
                    for (int i = 0; i < 15; ++i) Rh[i] = r15[i];
                    Rg[15] = Rh[15] = 0u;
                    const uint32_t va = lds_u32(lut, prmt(w12, lane4, 0x5504u));
                    const uint32_t vb = lds_u32(lut, prmt(w12, lane4, 0x5514u) + 128);
                    err = lop3_or3(err, va, vb);
#pragma unroll
                    for (int i = 0; i < 3; ++i) {
                        QG[i] = lop3_or_and(va, vb, mG[i]);
                        QH[i] = lop3_or_and(va, vb, mH[i]);
                    }
                } else {
                    const int64_t off = (int64_t)j * k2bGroupBytes + 8 * c;
                    const uint2 wg = ldg_u64(rowg[tt] + off);
                    const uint2 wh = ldg_u64(rowh[tt] + off);
                    const uint32_t ws[4] = {wg.x, wg.y, wh.x, wh.y};
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const uint32_t w = ws[r];
                        const uint32_t w12s = w >> 12;
                        uint32_t* R = r < 2 ? Rg : Rh;
                        const int base = (r & 1) * 8;
#pragma unroll
                        for (int f = 0; f < 6; ++f) R[base + f] = w & fmask(f);
                        R[base + 6] = w12s & fmask(0);
                        R[base + 7] = w12s & fmask(1);
                        err |= w & (w >> 1);
                    }
#pragma unroll
                    for (int i = 0; i < 3; ++i) QG[i] = QH[i] = 0u;
                }
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
                    if (LAYOUT == BT_LAYOUT_B3) {
#pragma unroll
                        for (int t = 0; t < 7; ++t)
                            mma_f16_16816(d, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1],
                                          bf[mt][t][0], bf[mt][t][1], d);
                        mma_f16_16816(d, Rg[14], Rh[14], QG[0], QH[0], bf[mt][7][0], bf[mt][7][1], d);
                        mma_f16_16816(d, QG[1], QH[1], QG[2], QH[2], bf[mt][NT - 1][0], bf[mt][NT - 1][1], d);
                    } else {
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            mma_f16_16816(d, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1],
                                          bf[mt][t][0], bf[mt][t][1], d);
                    }
                    acc[tt][mt][0] = fmaf(sg, fmaf(d[0], pm[mt][0], -cm[mt][0]), acc[tt][mt][0]);
                    acc[tt][mt][1] = fmaf(sg, fmaf(d[1], pm[mt][1], -cm[mt][1]), acc[tt][mt][1]);
                    acc[tt][mt][2] = fmaf(sh, fmaf(d[2], pm[mt][0], -cm[mt][0]), acc[tt][mt][2]);
                    acc[tt][mt][3] = fmaf(sh, fmaf(d[3], pm[mt][1], -cm[mt][1]), acc[tt][mt][3]);
                }
            }
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
                        if (n < a.N && m < a.M) store_y<float>(a.y, a.y_bf16, (int64_t)m * a.N + n, acc[tt][mt][r]);
                    }
        } else {
            const int slot = (u == u_begin) ? 0 : 1;
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
            __threadfence();
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
                __threadfence();
                float sum[TL][MT][4];
#pragma unroll
                for (int tt = 0; tt < TL; ++tt)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) sum[tt][mt][r] = 0.f;
                for (int64_t w = w_lo; w <= w_hi; ++w) {
                    const int ws = ((w * a.chunk) / G == p) ? 0 : 1;
                    const float* pw = a.partials + ((w * 2 + ws) * (TL * 16)) * a.M;
#pragma unroll
                    for (int tt = 0; tt < TL; ++tt)
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const int row = tt * 16 + g + (r >> 1) * 8;
                                const int m = mt * 8 + 2 * c + (r & 1);
                                if (m < a.M) sum[tt][mt][r] += __ldcg(pw + row * a.M + m);
                            }
                }
#pragma unroll
                for (int tt = 0; tt < TL; ++tt)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int n = (p * TL + tt) * 16 + g + (r >> 1) * 8;
                            const int m = mt * 8 + 2 * c + (r & 1);
                            if (n < a.N && m < a.M) store_y<float>(a.y, a.y_bf16, (int64_t)m * a.N + n, sum[tt][mt][r]);
                        }
                if (lane == 0) a.counters[p] = 0;
            }
        }
        u += j1 - j0;
    }

    int bad = 0;
    if (LAYOUT == BT_LAYOUT_B3) bad = (err >> 31) ? BT_DEVERR_INVALID_CODE : 0;
    else bad = (err & 0x55555555u) ? BT_DEVERR_INVALID_CODE : 0;
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) report(a.dev_err, bad);
}

// ------------------------------------------------------------ host ---------

struct GemvPlan {
    int NT, MT, P, grid, warps_total, prep_grid;
    int64_t G, U, chunk;
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
    if (warps_needed >= max_warps) {
        pl.grid = num_sms;
    } else {
        pl.grid = static_cast<int>((warps_needed + kGemvWarps - 1) / kGemvWarps);
    }
    pl.warps_total = pl.grid * kGemvWarps;
    pl.chunk = (pl.U + pl.warps_total - 1) / pl.warps_total;
    if (pl.chunk < 1) pl.chunk = 1;
    const int64_t nblocks = (pl.G + 7) / 8;
    int64_t pg = (M * nblocks + kPrepWarps - 1) / kPrepWarps;
    if (pg < 1) pg = 1;
    if (pg > (int64_t)num_sms * 4) pg = (int64_t)num_sms * 4;
    pl.prep_grid = static_cast<int>(pg);
    size_t off = 0;
    pl.off_bslots = off;
    off = align_up(off + (size_t)M * pl.G * pl.NT * 32, 256);
    pl.off_meta = off;
    off = align_up(off + (size_t)M * pl.G * sizeof(float2), 256);
    pl.off_counters = off;
    off = align_up(off + (size_t)pl.P * sizeof(int), 256);
    pl.off_partials = off;
    off = align_up(off + (size_t)pl.warps_total * 2 * kGemvTiles * 16 * M * sizeof(float), 256);
    pl.total = off;
    return pl;
}

size_t gemv_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K, int num_sms) {
    return make_gemv_plan(layout, M, N, K, num_sms).total;
}

template <int LAYOUT, int MT>
static cudaError_t launch_gemv_t(const GemvArgs& ga, const GemvPlan& pl, cudaStream_t stream) {
    const size_t smem = LAYOUT == BT_LAYOUT_B3 ? kLutBytes : 0;
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<LAYOUT, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<LAYOUT, MT>, ga);
}

cudaError_t launch_gemv(int layout, const uint8_t* codes, const uint16_t* scales, const void* x,
                        int x_dtype, const int8_t* sign, int64_t M, int64_t N, int64_t K, int y_dtype,
                        void* y, void* workspace, int32_t* dev_err, int num_sms,
                        cudaStream_t stream) {
    const GemvPlan pl = make_gemv_plan(layout, M, N, K, num_sms);
    uint8_t* ws = static_cast<uint8_t*>(workspace);

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
        gemv_prep_kernel<BT_LAYOUT_B3><<<pl.prep_grid, kPrepWarps * 32, 0, stream>>>(pa);
    else
        gemv_prep_kernel<BT_LAYOUT_2BIT><<<pl.prep_grid, kPrepWarps * 32, 0, stream>>>(pa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

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
    ga.row_bytes = (K / kGroup) * (layout == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes);
    ga.U = pl.U;
    ga.chunk = pl.chunk;
    ga.dev_err = dev_err;
    if (layout == BT_LAYOUT_B3)
        return pl.MT == 1 ? launch_gemv_t<BT_LAYOUT_B3, 1>(ga, pl, stream)
                          : launch_gemv_t<BT_LAYOUT_B3, 2>(ga, pl, stream);
    return pl.MT == 1 ? launch_gemv_t<BT_LAYOUT_2BIT, 1>(ga, pl, stream)
                      : launch_gemv_t<BT_LAYOUT_2BIT, 2>(ga, pl, stream);
}

}  // namespace bt

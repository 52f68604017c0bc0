// Tensor-core slot maps and digit decoding shared by the decode GEMV kernels
// (sm_100a only).
//
// The products run as m16n8k16 MMAs with the packed weights as the A operand
// (16 weight rows x 16 k) and the rotated activations as B. A weight enters as
// its base-3 digit d = t + 1 in {0, 1, 2}, held as a 2-bit field at bits
// [2i, 2i+1] of a 16-bit half: read as FP16 that half is the subnormal
// d * 4^i * 2^-24, exactly. An activation that meets field i is stored as FP16
// of x' * 2^(24 - 2i - e), e a per-group exponent, so every product is
// d * x' * 2^-e. The group then adds s * (2^e D - corr), corr the same sum
// with every digit 1 (all trits zero), which takes out the +1 of the digits.
//
// Slot (t, c, h): MMA step t of a group (k16), lane c of a quad
// (threadID_in_group) and half h of that lane's A fragment registers (0/1 =
// low/high half of a0, 2/3 = of a2). The slot functions return the k (0..127)
// a slot carries, or -1 for an empty slot, and the field i of that trit.
#pragma once

#include "bt_internal.cuh"

namespace bt {

// field mask: 2-bit field i of both 16-bit halves
__host__ __device__ constexpr uint32_t fmask(int i) {
    return (3u << (2 * i)) | (3u << (2 * i + 16));
}

__host__ __device__ constexpr int b3_slot(int t, int c, int h, int* field) {
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

__host__ __device__ constexpr int tb_slot(int t, int c, int h, int* field) {
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

// The five base-3 digits of every byte value as 2-bit fields (bit 31 marks
// values >= 243), the source of the shared-memory decode table.
struct B3FieldTable {
    uint32_t v[256];
    constexpr B3FieldTable() : v() {
        for (int code = 0; code < 256; ++code) {
            uint32_t f = 0x80000000u;
            if (code < 243) {
                f = 0;
                int r = code;
                for (int i = 0; i < 5; ++i) { f |= static_cast<uint32_t>(r % 3) << (2 * i); r /= 3; }
            }
            v[code] = f;
        }
    }
};
static __constant__ B3FieldTable c_b3_fields = B3FieldTable();

constexpr int kB3LutBytes = 256 * 256;  // 256 codes x (128 B low table + 128 B high table)

// Fill the lane-replicated decode table at `lut` (64 KB): row = code (256 B),
// [0, 128) low table, [128, 256) high table, one 4-byte entry per lane, so the
// lookups of a warp never conflict. Entry: the digits as fields at bits 2i
// (low) or 16 + 2i (high); bit 31 flags codes >= 243.
__device__ __forceinline__ void b3_lut_fill(uint8_t* lut, int tid, int nthreads) {
    for (int idx = tid; idx < 256 * 16; idx += nthreads) {
        const int code = idx >> 4, v = idx & 15;
        uint32_t f = c_b3_fields.v[code];
        if (v >= 8 && code < 243) f <<= 16;
        reinterpret_cast<uint4*>(lut)[idx] = make_uint4(f, f, f, f);
    }
}

// Decode one row's bytes 6c..6c+5 of a base-3 group (window words W0, W1,
// shifted right by o8 bits) into 15 registers through the decode table; LUT
// reads the table entry at a byte offset (CHECK: OR the entries into err,
// whose bit 31 flags codes >= 243).
template <bool CHECK, class LUT>
__device__ __forceinline__ void b3_decode6(uint32_t W0, uint32_t W1, uint32_t o8, uint32_t lane4,
                                           uint32_t (&R)[15], uint32_t& err) {
    const uint32_t lo = __funnelshift_r(W0, W1, o8);
    const uint32_t hi = W1 >> o8;
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        const uint32_t src = q == 2 ? hi : lo;
        const uint32_t b = q == 1 ? 2u : 0u;
        // offset = code * 256 + lane * 4 (+128 for the high table)
        const uint32_t va = LUT::ld(prmt(src, lane4, 0x5504u | (b << 4)));
        const uint32_t vb = LUT::ld(prmt(src, lane4, 0x5504u | ((b + 1) << 4)) + 128);
        if (CHECK) err = lop3_or3(err, va, vb);
#pragma unroll
        for (int i = 0; i < 5; ++i) R[5 * q + i] = lop3_or_and(va, vb, fmask(i));
    }
}

// A fragments of one 16-row tile for one base-3 group: rows g (words wg0/1,
// shift o8) and g + 8 (wh0/1), and pair 12 (bytes 24, 25) of row g (c < 2) or
// g + 8 (c >= 2) in w12. mG / mH: the lane's pair-12 field masks.
template <bool CHECK, class LUT>
__device__ __forceinline__ void b3_decode_tile(uint32_t wg0, uint32_t wg1, uint32_t wh0, uint32_t wh1,
                                               uint32_t w12, uint32_t o8, uint32_t lane4, const uint32_t (&mG)[3],
                                               const uint32_t (&mH)[3], uint32_t (&Rg)[16], uint32_t (&Rh)[16],
                                               uint32_t (&QG)[3], uint32_t (&QH)[3], uint32_t& err) {
    uint32_t r15[15];
    b3_decode6<CHECK, LUT>(wg0, wg1, o8, lane4, r15, err);
#pragma unroll
    for (int k = 0; k < 15; ++k) Rg[k] = r15[k];
    b3_decode6<CHECK, LUT>(wh0, wh1, o8, lane4, r15, err);
#pragma unroll
    for (int k = 0; k < 15; ++k) Rh[k] = r15[k];
    Rg[15] = Rh[15] = 0u;
    const uint32_t va = LUT::ld(prmt(w12, lane4, 0x5504u));
    const uint32_t vb = LUT::ld(prmt(w12, lane4, 0x5514u) + 128);
    if (CHECK) err = lop3_or3(err, va, vb);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        QG[k] = lop3_or_and(va, vb, mG[k]);
        QH[k] = lop3_or_and(va, vb, mH[k]);
    }
}

// pair-12 field masks of lane c: even c -> fields 0, 1, 2; odd c -> 3, 4; the
// fields sit in row g's registers for c < 2 and in row g + 8's for c >= 2
__device__ __forceinline__ void b3_pair12_masks(int c, uint32_t (&mG)[3], uint32_t (&mH)[3]) {
    uint32_t mq[3];
    mq[0] = (c & 1) ? fmask(3) : fmask(0);
    mq[1] = (c & 1) ? fmask(4) : fmask(1);
    mq[2] = (c & 1) ? 0u : fmask(2);
#pragma unroll
    for (int i = 0; i < 3; ++i) { mG[i] = c < 2 ? mq[i] : 0u; mH[i] = c < 2 ? 0u : mq[i]; }
}

// A fragments of one 16-row tile for one 2-bit group: rows g (x0 = bytes
// 8c..8c+7) and g + 8 (x1). CHECK: OR the invalid-field bits into err.
template <bool CHECK>
__device__ __forceinline__ void tb_decode_tile(uint2 x0, uint2 x1, uint32_t (&Rg)[16], uint32_t (&Rh)[16],
                                               uint32_t& err) {
    const uint32_t w[4] = {x0.x, x0.y, x1.x, x1.y};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const uint32_t x = w[r];
        const uint32_t x12 = x >> 12;
        uint32_t* Rr = r < 2 ? Rg : Rh;
        const int base = (r & 1) * 8;
#pragma unroll
        for (int f = 0; f < 6; ++f) Rr[base + f] = x & fmask(f);
        Rr[base + 6] = x12 & fmask(0);
        Rr[base + 7] = x12 & fmask(1);
        if (CHECK) err |= x & (x >> 1);
    }
}

// D = sum over the group's MMA steps, as two accumulator chains (even / odd
// steps) added at the end. Every user of a group's D -- the tiles and the
// all-digits-1 correction -- goes through these, so equal A registers give
// bitwise equal D.
template <int NB>
__device__ __forceinline__ void b3_group_mma(const uint32_t (&Rg)[16], const uint32_t (&Rh)[16],
                                             const uint32_t (&QG)[3], const uint32_t (&QH)[3],
                                             const uint32_t (&bf)[NB][2], float (&d)[4]) {
    static_assert(NB >= 9, "nine MMA steps per base-3 group");
    float e4[4] = {0.f, 0.f, 0.f, 0.f};
    d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
    for (int t = 0; t < 7; ++t) {
        if (t & 1)
            mma_f16_16816(e4, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], bf[t][0], bf[t][1], e4);
        else
            mma_f16_16816(d, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], bf[t][0], bf[t][1], d);
    }
    mma_f16_16816(e4, Rg[14], Rh[14], QG[0], QH[0], bf[7][0], bf[7][1], e4);
    mma_f16_16816(d, QG[1], QH[1], QG[2], QH[2], bf[8][0], bf[8][1], d);
#pragma unroll
    for (int r = 0; r < 4; ++r) d[r] += e4[r];
}

// The same chains for two n8 blocks of B that share the A registers, issued
// interleaved so each block's MMA hides the other's latency; each block's D is
// bitwise what b3_group_mma / tb_group_mma would give it.
template <bool B3, int NB>
__device__ __forceinline__ void group_mma2(const uint32_t (&Rg)[16], const uint32_t (&Rh)[16],
                                           const uint32_t (&QG)[3], const uint32_t (&QH)[3],
                                           const uint32_t (&b0)[NB][2], const uint32_t (&b1)[NB][2], float (&d0)[4],
                                           float (&d1)[4]) {
    float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
    d0[0] = d0[1] = d0[2] = d0[3] = 0.f;
    d1[0] = d1[1] = d1[2] = d1[3] = 0.f;
    constexpr int T = B3 ? 7 : 8;
#pragma unroll
    for (int t = 0; t < T; ++t) {
        if (t & 1) {
            mma_f16_16816(e0, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], b0[t][0], b0[t][1], e0);
            mma_f16_16816(e1, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], b1[t][0], b1[t][1], e1);
        } else {
            mma_f16_16816(d0, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], b0[t][0], b0[t][1], d0);
            mma_f16_16816(d1, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], b1[t][0], b1[t][1], d1);
        }
    }
    if constexpr (B3) {
        mma_f16_16816(e0, Rg[14], Rh[14], QG[0], QH[0], b0[7][0], b0[7][1], e0);
        mma_f16_16816(e1, Rg[14], Rh[14], QG[0], QH[0], b1[7][0], b1[7][1], e1);
        mma_f16_16816(d0, QG[1], QH[1], QG[2], QH[2], b0[8][0], b0[8][1], d0);
        mma_f16_16816(d1, QG[1], QH[1], QG[2], QH[2], b1[8][0], b1[8][1], d1);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        d0[r] += e0[r];
        d1[r] += e1[r];
    }
}

template <int NB>
__device__ __forceinline__ void tb_group_mma(const uint32_t (&Rg)[16], const uint32_t (&Rh)[16],
                                             const uint32_t (&bf)[NB][2], float (&d)[4]) {
    static_assert(NB >= 8, "eight MMA steps per 2-bit group");
    float e4[4] = {0.f, 0.f, 0.f, 0.f};
    d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        if (t & 1)
            mma_f16_16816(e4, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], bf[t][0], bf[t][1], e4);
        else
            mma_f16_16816(d, Rg[2 * t], Rh[2 * t], Rg[2 * t + 1], Rh[2 * t + 1], bf[t][0], bf[t][1], d);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) d[r] += e4[r];
}

// A registers of a row whose trits are all zero (every digit 1): what the
// decoders produce for base-3 bytes of code 121 and 2-bit bytes 0x55.
__device__ __forceinline__ void b3_ones_tile(int c, uint32_t (&Rg)[16], uint32_t (&Rh)[16], uint32_t (&QG)[3],
                                             uint32_t (&QH)[3]) {
#pragma unroll
    for (int r = 0; r < 15; ++r) Rg[r] = Rh[r] = fmask(r % 5) & 0x55555555u;
    Rg[15] = Rh[15] = 0u;
    uint32_t mG[3], mH[3];
    b3_pair12_masks(c, mG, mH);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        QG[k] = mG[k] & 0x55555555u;
        QH[k] = mH[k] & 0x55555555u;
    }
}

__device__ __forceinline__ void tb_ones_tile(uint32_t (&Rg)[16], uint32_t (&Rh)[16]) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int f = r & 7;
        Rg[r] = Rh[r] = fmask(f < 6 ? f : f - 6) & 0x55555555u;
    }
}

}  // namespace bt

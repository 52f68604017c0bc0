// Decode GEMV for one activation row (M = 1), by table lookup of packed
// bytes, over a list of matrices in one persistent launch: y_p = W_p (R x_p).
//
// One base-3 byte holds five trits of a row of W (Bonsai low-bit course,
// section "先用五个数字理解 1.6bit"), a 2-bit byte four. Against a fixed
// activation vector the contribution of one byte, sum_i t_i x'_(5b+i), depends
// only on the byte's code, so for every byte position of a 512-wide K chunk
// the kernel tabulates that sum for all 256 codes once and then streams rows:
// one shared-memory lookup and one FP32 add per byte instead of decoding five
// trits. W is never decoded. The release summary of Ternary Bonsai 2 27B
// (section 三值权重怎么压缩到 1.76 bit) fuses unpack and group scale into the
// product; section 已知短板 names the activation transform as the largest
// cost outside the product at batch 1, and decode is bound by weight bytes
// (section 实测吞吐).
//
// Work. A launch's (matrix, 512-chunk, row) items, in that order, are cut
// into one contiguous range per CTA (one CTA per SM), balanced so that every
// CTA streams about the same number of row chunks once the chunk starts it
// takes on are counted (each costs about 256 rows of streaming). A range is a few segments (matrix p, chunk c,
// rows n0..n1); per segment the CTA rotates the 1024-block holding the chunk
// (the warp FWHT of the Sylvester H_1024, S applied first, 1/32; TensorSharp
// blog, sections 3.2 and 5.2) unless it already holds it, builds the chunk's
// tables, and its 16 warps stream the rows in sets of 16 (set k to warp
// k % 16), each warp with its own two-slot TMA ring ([16 rows][112 B] of codes,
// x rounded down to 16 B, and [16 rows][8 halves] of scales). Each row's chunk
// partial goes to the workspace with a plain store.
//
// Reduction. A second kernel, launched as a programmatic dependent, adds each
// row's partials in chunk order (one thread per row), so results do not
// depend on the schedule, and writes y. (A single kernel that counts finished
// rows and lets the last CTA of a row block add them was slower on B200: the
// fences and atomics of CTAs that finish early queue behind the other CTAs'
// weight stream, several microseconds each.) A list whose matrices read
// earlier outputs runs as one launch pair per dependency level; stream order
// carries the outputs from one to the next.
//
// Tables. Lane L of a warp reads code word L (bytes 4L..4L+3) of a row chunk,
// so byte position p = 4L + k is only ever looked up by lane L: its table
// lives in shared-memory bank L and a warp's 32 lookups never conflict. Two
// 64 KB regions [256 codes][64 slots] of FP32 hold the 128 tables; byte k of
// lane L sits in region k/2, slot L + 32 (k % 2). One PRMT turns the code byte
// and a lane constant into the byte offset code * 256 + slot * 4. Scales
// multiply per row: a base-3 chunk row has four groups of 26 bytes, so a
// lane's word lies in one group or (lanes 6 and 19) straddles two; the lane
// applies s_a to bytes 0-1 and s_b to bytes 2-3 of its word. Each warp keeps
// one FP32 partial per row of its set in every lane and reduces the 32 x 16
// block with a butterfly transpose (16 shuffles); lanes i and i + 16 then hold
// row i.
#include <algorithm>

#include "bt_internal.cuh"
#include "bt_slots.cuh"

namespace bt {

constexpr int kLutWarps = 16;                        // streaming warps
constexpr int kLutThreads = kLutWarps * 32;
constexpr int kLutChunk = 512;                      // k per table set (group-aligned layouts)
constexpr int kLutChunkC = 640;                     // k per table set, continuous base-3: 128 bytes, 5 groups
constexpr int kLutRegion = 256 * 64 * 4;            // [256 codes][64 slots] f32
constexpr int kLutTableBytes = 2 * kLutRegion;
constexpr int kLutSet = 16;                          // rows per set (one TMA box, one reduction)
constexpr int kLutDepth = 2;                         // sets in flight per warp
constexpr int kLutCBoxB3 = 112;                      // box bytes per row: 104 + up to 8 of alignment
constexpr int kLutCBox2b = 128;

// Continuous base-3 rows: the chunk's bytes 25, 51, 76 and 102 hold trits of
// two groups; their second-group parts come from four extra tables, looked
// up by lanes 6, 12, 19 and 25 (byte 1, 3, 0 and 2 of their word).
__host__ __device__ constexpr int split_byte(int s) { return s == 0 ? 25 : s == 1 ? 51 : s == 2 ? 76 : 102; }

// Shared memory of the table-lookup kernel, per layout: tables, [continuous:
// extra tables + a zero word], the chunk's rotated activations, the slot
// inputs, the signs of S, the ring barriers, a staging area for raw x
// (continuous: two blocks; f32 staging overlaps the FWHT tile, which only a
// bf16 rotation uses) and the per-warp TMA rings.
template <int LAYOUT>
struct LutGeom {
    static constexpr bool kCont = LAYOUT == BT_LAYOUT_B3C;
    static constexpr int kChunk = kCont ? kLutChunkC : kLutChunk;
    static constexpr int kCB = kCont ? 128 : (LAYOUT == BT_LAYOUT_B3 ? 4 * kB3GroupBytes : 4 * k2bGroupBytes);
    static constexpr int kCBox = LAYOUT == BT_LAYOUT_B3 ? kLutCBoxB3 : 128;
    static constexpr int kSBox = kCont ? 16 : 8;     // scale halves per row in a set's scale box
    static constexpr int kSlot = kLutSet * kCBox + kLutSet * kSBox * 2;
    static constexpr int kExtra = kLutTableBytes;
    static constexpr int kExtraBytes = kCont ? 256 * 16 + 16 : 0;
    static constexpr int kXr = kExtra + kExtraBytes;
    static constexpr int kXrBytes = (kCont ? kLutChunkC : kBlock) * 4;
    static constexpr int kXs = kXr + kXrBytes;       // [5][4][32] f32 slot inputs
    static constexpr int kSgn = kXs + 5 * 4 * 32 * 4;
    static constexpr int kBar = kSgn + kBlock;
    static constexpr int kStage = kBar + kLutWarps * kLutDepth * 8;
    static constexpr int kTile = kStage + kBlock * 4;  // FWHT exchange tile, 32 x 36 f32
    static constexpr int kRing = (kTile + 32 * kTileStride * 4 + 127) & ~127;
    static constexpr int kSmem = kRing + kLutWarps * kLutDepth * kSlot;
    static_assert(kRing % 128 == 0 && kSlot % 128 == 0 && (kLutSet * kCBox) % 128 == 0,
                  "ring slots and the scale boxes inside them are TMA destinations");
    static_assert(kStage % 16 == 0 && kSgn % 16 == 0, "16-byte asynchronous copies land there");
    static_assert(!kCont || kTile + 32 * kTileStride * 4 >= kStage + 2 * kBlock * 4, "two f32 blocks fit");
    static_assert(kSmem <= 227 * 1024, "one CTA per SM");
};

constexpr int kLutMaxProblems = 12;                  // per launch (kernel parameters < 4 KB)
constexpr int kLutReduceThreads = 256;

#ifndef BT_WAIT_NS
#define BT_WAIT_NS 2000000000ull
#endif
constexpr uint64_t kLutWaitNs = BT_WAIT_NS;

// Chunk partials: matrix p of a list keeps [nchunk][ld] floats (ld = N
// rounded up to 4, so every 4-row piece of a chunk is one 16-byte load).
struct LutProblem {
    const void* x;          // [1][K] bf16 or f32; unused when src != NULL
    const float* src;       // NULL, or the partials of the earlier matrix whose output is x
    int64_t rc_base;        // first (chunk, row) item of this matrix in the launch's order
    int64_t part_base;      // its own partials, from LutParams::part
    int32_t N, ld, nchunk, x_bf16;
    int32_t src_ld, src_nchunk;
    int32_t K;              // (the last continuous chunk may be partial)
};

struct LutParams {
    CUtensorMap cmap[kLutMaxProblems];
    CUtensorMap smap[kLutMaxProblems];
    LutProblem p[kLutMaxProblems];
    const int8_t* sign;                // NULL: x already rotated
    int32_t* dev_err;
    float* part;                       // chunk partials of every matrix of the list
    int64_t total_rc;
    int nprob, y_bf16;
    int M;                             // activation rows (1 for the table-lookup kernel)
    const void* frag;                  // M > 1: the prep kernel's fragment words and group constants
    const void* meta;
};
static_assert(sizeof(LutParams) <= 4096, "kernel parameters");

// Sums of chunk partials for up to kLutMaxProblems matrices and where they go.
// Partials of a matrix with M activation rows: [nchunk][ld][M] (a 16-row set
// of a chunk writes 16 M contiguous floats).
struct LutReduceParams {
    const float* part[kLutMaxProblems];
    void* y[kLutMaxProblems];
    int32_t N[kLutMaxProblems], ld[kLutMaxProblems], nchunk[kLutMaxProblems], M[kLutMaxProblems];
    int nprob, y_bf16;
};

extern __shared__ __align__(1024) uint8_t lut_smem[];

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint2 lds_u64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t r;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(addr) : "memory");
    return r;
}

// Table lookup at a shared-window byte address. The ring reads above carry a
// memory clobber (they must stay after the mbarrier wait that publishes the
// TMA bytes); the table is written before a CTA barrier, so lookups need none.
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Warp 0 starts copying the raw 1024-block `blk` of x (bf16: 2 KB, f32:
// 4 KB) into the staging buffer. Issued as soon as the block is known, so the
// copy overlaps the stream of the segment before; x may be an output of an
// earlier kernel, so only after the grid dependency is resolved.
__device__ __forceinline__ void lut_stage_block(const void* x, int x_bf16, int blk, uint32_t xst) {
    const int lane = threadIdx.x & 31;
    const int esz = x_bf16 ? 2 : 4;
    const uint8_t* src = static_cast<const uint8_t*>(x) + (size_t)blk * kBlock * esz;
    const int per_lane = esz * 2;  // 16-byte pieces per lane: 4 (bf16) or 8 (f32)
#pragma unroll 4
    for (int j = 0; j < per_lane; ++j) {
        const int off = (lane * per_lane + j) * 16;  // lane l's pieces hold elements 32 l .. 32 l + 31
        cp_async16(xst + off, src + off);
    }
    cp_async_commit();
}

// The staged block, rotated (or, without S, copied) into xr as FP32. Warp 0
// only, after every lane's staged copies have landed.
__device__ __forceinline__ void lut_rotate_block(const uint8_t* xst, int x_bf16, const int8_t* sgn, bool has_sign,
                                                 float* xr, float* tile) {
    const int lane = threadIdx.x & 31;
    float v[32];
    if (x_bf16) {
        const uint4* src = reinterpret_cast<const uint4*>(xst + 64 * lane);
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 t = src[q];
            w[4 * q] = t.x; w[4 * q + 1] = t.y; w[4 * q + 2] = t.z; w[4 * q + 3] = t.w;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = bf16_bits_to_f32((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu));
    } else {
        const float4* src = reinterpret_cast<const float4*>(xst + 128 * lane);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 t = src[q];
            v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
        }
    }
    if (has_sign) {  // the ABI accepts S with bf16 activations only
        const uint4* sg = reinterpret_cast<const uint4*>(sgn + 32 * lane);
        const uint4 s0 = sg[0], s1 = sg[1];
        const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            // sign byte i: bit 7 set for negative entries
            const uint32_t sbit = (sw[i >> 2] >> (8 * (i & 3))) & 0x80u;
            v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (sbit << 24));
        }
        fwht1024_warp(v, tile);
#pragma unroll
        for (int j = 0; j < 32; ++j) xr[32 * j + lane] = v[j];  // lane holds element 32 j + lane
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) xr[32 * lane + i] = v[i];
    }
}

// Slot inputs of chunk half `h` of the block in xr: xs[i][k][L] = x' of trit i
// of byte 4L + k (zero past the group's last trit and for unused lanes).
// Continuous base-3: xr holds the chunk's own x' (kvalid of them, zeros past
// K); a byte that holds trits of two groups keeps only its first group's here.
template <int LAYOUT>
__device__ __forceinline__ void lut_scatter(const float* xr, int h, float* xs, int kvalid = 0) {
    for (int t = threadIdx.x; t < 5 * 4 * 32; t += kLutThreads) {
        const int i = t >> 7, k = (t >> 5) & 3, L = t & 31;
        const int p = 4 * L + k;
        float v = 0.f;
        if (LAYOUT == BT_LAYOUT_B3C) {
            const int j = 5 * p + i;
            if (j < kvalid && j / kGroup == (5 * p) / kGroup) v = xr[j];
        } else if (LAYOUT == BT_LAYOUT_B3) {
            if (L < 26) {
                const int g = p / 26, b = p - 26 * g, j = 5 * b + i;
                if (j < kGroup) v = xr[h * kLutChunk + g * kGroup + j];
            }
        } else {
            if (i < 4) v = xr[h * kLutChunk + 4 * p + i];
        }
        xs[t] = v;
    }
}

// Entries for codes that are not valid (base-3 codes 243-255, 2-bit codes
// with a field of 3) read 0, so an invalid code contributes nothing (the
// checked kernel reports it). They never change: zeroed once per launch.
template <int LAYOUT>
__device__ __forceinline__ void lut_zero_invalid(float* table) {
    if (LAYOUT == BT_LAYOUT_B3C) {  // the extra tables' invalid codes and the zero word too
        float* extra = table + kLutTableBytes / 4;
        for (int t = threadIdx.x; t < 13 * 4 + 4; t += kLutThreads) extra[243 * 4 + t] = 0.f;
    }
    if (LAYOUT == BT_LAYOUT_B3 || LAYOUT == BT_LAYOUT_B3C) {
        for (int t = threadIdx.x; t < 2 * 13 * 64; t += kLutThreads) {
            const int r = t / (13 * 64), u = t - r * 13 * 64;
            table[r * (kLutRegion / 4) + 243 * 64 + u] = 0.f;
        }
    } else {
        for (int t = threadIdx.x; t < 2 * 256 * 64; t += kLutThreads) {
            const int c = (t >> 6) & 255;
            if (c & (c >> 1) & 0x55) table[t] = 0.f;
        }
    }
}

// Tables for the current chunk: entry(c) = sum_i (d_i(c) - 1) x'_i over the
// trits of byte slot (L, k). Warp w serves k = w % 4 for every lane and a
// quarter of the high digits. Base-3: c = a + 27 b (a: trits 0-2, b: trits
// 3-4), warp takes b = w / 4 + 4 j and writes the 27 entries of each b.
// 2-bit: c = lo + 16 hi (two 2-bit digits each), warp takes hi = w / 4 + 4 j
// and writes the entries whose digits are all valid.
template <int LAYOUT>
__device__ __forceinline__ void lut_build(const float* xs, float* table) {
    const int warp = threadIdx.x >> 5, L = threadIdx.x & 31;
    const int k = warp & 3, q = warp >> 2;
    const float x0 = xs[(0 * 4 + k) * 32 + L], x1 = xs[(1 * 4 + k) * 32 + L], x2 = xs[(2 * 4 + k) * 32 + L],
                x3 = xs[(3 * 4 + k) * 32 + L];
    float* col = table + (k >> 1) * (kLutRegion / 4) + L + 32 * (k & 1);
    if (LAYOUT == BT_LAYOUT_B3 || LAYOUT == BT_LAYOUT_B3C) {
        const float x4 = xs[(4 * 4 + k) * 32 + L];
        for (int b = q; b < 9; b += 4) {
            const float base = (float)(b % 3 - 1) * x3 + (float)(b / 3 - 1) * x4;
#pragma unroll
            for (int d2 = 0; d2 < 3; ++d2) {
                const float s2 = base + (float)(d2 - 1) * x2;
#pragma unroll
                for (int d1 = 0; d1 < 3; ++d1) {
                    const float s1 = s2 + (float)(d1 - 1) * x1;
                    const int c = 27 * b + 9 * d2 + 3 * d1;
                    col[(c + 0) * 64] = s1 - x0;
                    col[(c + 1) * 64] = s1;
                    col[(c + 2) * 64] = s1 + x0;
                }
            }
        }
    } else {
        for (int hi = q; hi < 16; hi += 4) {
            const int e2 = hi & 3, e3 = hi >> 2;
            if (e2 == 3 || e3 == 3) continue;
            const float base = (float)(e2 - 1) * x2 + (float)(e3 - 1) * x3;
#pragma unroll
            for (int e1 = 0; e1 < 3; ++e1) {
                const float s1 = base + (float)(e1 - 1) * x1;
                const int c = 16 * hi + 4 * e1;
                col[(c + 0) * 64] = s1 - x0;
                col[(c + 1) * 64] = s1;
                col[(c + 2) * 64] = s1 + x0;
            }
        }
    }
}

// Continuous base-3: the second-group parts of the four split bytes,
// extra[code][s] = sum_i (d_i(code) - 1) x'_i over the byte's trits in the
// later group (kvalid as for lut_scatter).
__device__ __forceinline__ void lut_build_extra(const float* xr, float* extra, int kvalid) {
    for (int t = threadIdx.x; t < 4 * 243; t += kLutThreads) {
        const int sidx = t / 243, code = t - 243 * sidx;
        const int p = split_byte(sidx);
        float v = 0.f;
        int c = code;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            const int d = c % 3;
            c /= 3;
            const int j = 5 * p + i;
            if (j < kvalid && j / kGroup != (5 * p) / kGroup) v += (float)(d - 1) * xr[j];
        }
        extra[code * 4 + sidx] = v;
    }
}

// acc[j] (j = 0..15, one row each) summed over the warp: halving exchanges on
// lane bits 3..0 leave lane L with row L % 16 summed over 16 lanes, and one
// more exchange adds the other half-warp. Lanes i and i + 16 return row i.
__device__ __forceinline__ float lut_transpose_reduce(float (&acc)[kLutSet]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) {
        const bool up = lane & w;
#pragma unroll
        for (int j = 0; j < w; ++j) {
            const float keep = up ? acc[j + w] : acc[j];
            const float send = up ? acc[j] : acc[j + w];
            acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 16);
}

// A base-3 byte >= 243, or a 2-bit field holding 3.
template <int LAYOUT>
__device__ __forceinline__ uint32_t lut_check(uint32_t w) {
    if (LAYOUT != BT_LAYOUT_2BIT) return __vcmpgeu4(w, 0xF3F3F3F3u) ? BT_DEVERR_INVALID_CODE : 0u;
    return (w & (w >> 1) & 0x55555555u) ? BT_DEVERR_INVALID_CODE : 0u;
}

// One warp's TMA ring: slot d holds [16 rows][box bytes] of codes followed by
// [16 rows][8 halves] of scales. Sets are numbered per warp across chunks;
// set n lives in slot n % 2 and completes phase (n / 2) % 2 of its mbarrier.
struct LutRing {
    uint32_t ring;  // shared address of slot 0
    uint32_t bar;   // shared address of slot 0's mbarrier
    int slot_bytes;
    int cbox;
};

// The test-only build of the library (BT_TEST_WITHHOLD_COPY, never the
// product) leaves out one copy -- the second set of CTA 0's warp 0 -- so that
// the bounded wait on it runs out: the kernel must then set
// BT_DEVERR_TIMEOUT, let its other copies land and return.
__device__ __forceinline__ bool lut_withheld(uint32_t n) {
#ifdef BT_TEST_WITHHOLD_COPY
    return blockIdx.x == 0 && (threadIdx.x >> 5) == 0 && n == 1;
#else
    (void)n;
    return false;
#endif
}

__device__ __forceinline__ void lut_issue_set(const LutRing& rg, const CUtensorMap* cmap, const CUtensorMap* smap,
                                              uint32_t n, int cx, int sx, int64_t r0) {
    if (lut_withheld(n)) return;
    const uint32_t d = n % kLutDepth;
    const uint32_t dst = rg.ring + d * rg.slot_bytes;
    const uint32_t bar = rg.bar + 8 * d;
    mbar_arrive_tx(bar, (uint32_t)rg.slot_bytes);  // codes box + scale box
    tma_load_2d(dst, cmap, cx, (int)r0, bar);
    tma_load_2d(dst + kLutSet * rg.cbox, smap, sx, (int)r0, bar);
}


// ------------------------------------------------------------ helpers ----

__device__ __forceinline__ uint64_t lut_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of the given parity, bounded in time.
__device__ __forceinline__ bool lut_wait(uint32_t bar, uint32_t parity) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
        if (ok) return true;
        if ((i & 63) == 63) {
            const uint64_t now = lut_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > kLutWaitNs) return false;
        }
    }
}

// One segment of a CTA's range: matrix p, chunk c, rows [n0, n1).
struct LutSeg {
    int p, c, n0, n1;
};

// A CTA's share of the launch's (matrix, chunk, row) items. Starting a chunk
// (rotation, scatter, table build) costs about kLutHead rows of streaming, so
// the items are laid on a cost line where every chunk start takes kLutHead
// units before its rows; CTA b takes the items of cost range
// [C b / G, C (b + 1) / G). A share that crosses a chunk start gets that many
// fewer rows; consecutive shares meet exactly.
constexpr int kLutHead = 256;

__device__ __forceinline__ int64_t lut_item_at_cost(const LutParams& P, int64_t x) {
    for (int p = 0; p < P.nprob; ++p) {
        const int64_t per = kLutHead + (int64_t)P.p[p].N;
        const int64_t span = per * P.p[p].nchunk;
        if (x < span) {
            const int64_t c = x / per, w = x - c * per;
            return P.p[p].rc_base + c * P.p[p].N + (w > kLutHead ? w - kLutHead : 0);
        }
        x -= span;
    }
    return P.total_rc;
}

__device__ __forceinline__ void lut_share(const LutParams& P, int64_t& rc0, int64_t& rc1) {
    int64_t C = 0;
    for (int p = 0; p < P.nprob; ++p) C += (kLutHead + (int64_t)P.p[p].N) * P.p[p].nchunk;
    rc0 = lut_item_at_cost(P, C * blockIdx.x / gridDim.x);
    rc1 = lut_item_at_cost(P, C * (blockIdx.x + 1) / gridDim.x);
}

__device__ __forceinline__ bool lut_next_seg(const LutParams& P, int64_t& rc, int64_t rc1, LutSeg& s) {
    if (rc >= rc1) return false;
    int p = 0;
    while (p + 1 < P.nprob && rc >= P.p[p + 1].rc_base) ++p;
    const int64_t local = rc - P.p[p].rc_base;
    const int N = P.p[p].N;
    s.p = p;
    s.c = static_cast<int>(local / N);
    s.n0 = static_cast<int>(local - (int64_t)s.c * N);
    const int64_t end = (int64_t)s.n0 + (rc1 - rc);
    s.n1 = static_cast<int>(end < N ? end : N);
    rc += s.n1 - s.n0;
    return true;
}

// Row n of matrix p of a group: its chunk partials added in chunk order, up
// to UNROLL loads in flight. The partials were written by an earlier kernel
// of the stream: read through L2.
__device__ __forceinline__ float4 ldcg_f4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

// Row n of a matrix whose partials ([nchunk][ld] floats) start at `part`:
// its chunk partials added in chunk order, RPT rows (n, n + step, ...) at a
// time with up to UNROLL loads of each row in flight together.
template <int RPT, int UNROLL>
__device__ __forceinline__ void lut_row_sums(const float* part, int64_t ld, int nchunk, int n, int step,
                                             float (&sum)[RPT]) {
#pragma unroll
    for (int j = 0; j < RPT; ++j) sum[j] = 0.f;
    for (int c0 = 0; c0 < nchunk; c0 += UNROLL) {
        float v[RPT][UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
#pragma unroll
            for (int j = 0; j < RPT; ++j)
                v[j][u] = c0 + u < nchunk ? __ldcg(part + (c0 + u) * ld + n + j * step) : 0.f;
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
#pragma unroll
            for (int j = 0; j < RPT; ++j)
                if (c0 + u < nchunk) sum[j] += v[j][u];
    }
}

// Block blk of the output of the matrix whose partials pr.src holds, as the
// stored output reads (bf16-rounded when outputs are bf16), into the staging
// buffer. All threads of the CTA, two rows each.
__device__ __forceinline__ void lut_gather_block(const LutProblem& pr, int y_bf16, int blk, uint8_t* xst) {
    static_assert(kBlock == 2 * kLutThreads, "two rows per thread");
    float v[2];
    lut_row_sums<2, 24>(pr.src, pr.src_ld, pr.src_nchunk, blk * kBlock + threadIdx.x, kLutThreads, v);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int i = threadIdx.x + kLutThreads * j;
        if (y_bf16) reinterpret_cast<__nv_bfloat16*>(xst)[i] = __float2bfloat16_rn(v[j]);
        else reinterpret_cast<float*>(xst)[i] = v[j];
    }
}

// ------------------------------------------------------------- kernel ----

// Continuous base-3: warp 0 rotates (or copies) the staged blocks b0 and b1
// (b1 < 0: one block) and keeps the chunk's kvalid values of x' in xr.
__device__ __forceinline__ void lut_rotate_chunk(const uint8_t* xst, int x_bf16, const int8_t* sgn, bool has_sign,
                                                 int64_t k0, int b0, int b1, int kvalid, float* xr, float* tile) {
    const int lane = threadIdx.x & 31;
    const int esz = x_bf16 ? 2 : 4;
    for (int u = 0; u < 2; ++u) {
        const int bb = u == 0 ? b0 : b1;
        if (bb < 0) break;
        float v[32];
        const uint8_t* raw = xst + u * kBlock * esz;
        if (x_bf16) {
            const uint4* src = reinterpret_cast<const uint4*>(raw + 64 * lane);
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 t = src[q];
                w[4 * q] = t.x; w[4 * q + 1] = t.y; w[4 * q + 2] = t.z; w[4 * q + 3] = t.w;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = bf16_bits_to_f32((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu));
        } else {
            const float4* src = reinterpret_cast<const float4*>(raw + 128 * lane);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 t = src[q];
                v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
            }
        }
        const int64_t e0 = (int64_t)bb * kBlock - k0;  // chunk position of the block's element 0
        if (has_sign) {
            const uint4* sg = reinterpret_cast<const uint4*>(sgn + 32 * lane);
            const uint4 s0 = sg[0], s1 = sg[1];
            const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t sbit = (sw[i >> 2] >> (8 * (i & 3))) & 0x80u;
                v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (sbit << 24));
            }
            fwht1024_warp(v, tile);
#pragma unroll
            for (int j = 0; j < 32; ++j) {  // lane holds element 32 j + lane
                const int64_t kk = e0 + 32 * j + lane;
                if (kk >= 0 && kk < kvalid) xr[kk] = v[j];
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int64_t kk = e0 + 32 * lane + i;
                if (kk >= 0 && kk < kvalid) xr[kk] = v[i];
            }
        }
    }
}

template <int LAYOUT, bool CHECK>
__global__ void __launch_bounds__(kLutThreads, 1) gemv_lut_kernel(const __grid_constant__ LutParams P) {
    using GE = LutGeom<LAYOUT>;
    constexpr bool CONT = GE::kCont;
    constexpr int CHUNK = GE::kChunk;
    float* table = reinterpret_cast<float*>(lut_smem);
    const uint32_t tab_s = smem_addr(lut_smem);
    float* xr = reinterpret_cast<float*>(lut_smem + GE::kXr);
    float* xs = reinterpret_cast<float*>(lut_smem + GE::kXs);
    const uint8_t* xst = lut_smem + GE::kStage;
    const uint32_t xst_s = smem_addr(xst);
    int8_t* sgn = reinterpret_cast<int8_t*>(lut_smem + GE::kSgn);
    float* tile = reinterpret_cast<float*>(lut_smem + GE::kTile);
    const uint32_t extra_s = smem_addr(lut_smem + GE::kExtra);
    const int warp = threadIdx.x >> 5, L = threadIdx.x & 31;
    const int CB = GE::kCB;  // bytes per chunk row
    const bool lane_on = LAYOUT == BT_LAYOUT_B3 ? L < 26 : true;
    LutRing rg;
    rg.cbox = GE::kCBox;
    rg.slot_bytes = GE::kSlot;
    rg.ring = smem_addr(lut_smem + GE::kRing) + warp * kLutDepth * rg.slot_bytes;
    rg.bar = smem_addr(lut_smem + GE::kBar) + warp * kLutDepth * 8;

    // lane constants: table byte offsets and scale selectors
    const uint32_t lanebytes = (uint32_t)(4 * L) | ((uint32_t)(4 * L + 128) << 8);
    uint32_t ga, gb;
    if (LAYOUT == BT_LAYOUT_B3) {
        ga = lane_on ? (4 * L) / 26 : 3;
        gb = lane_on ? (4 * L + 3) / 26 : 3;
    } else if (CONT) {
        ga = (20 * L) / kGroup;       // the groups of the lane's first and last trit
        gb = (20 * L + 19) / kGroup;
    } else {
        ga = gb = L >> 3;
    }
    const uint32_t ssel = (2 * ga) | ((2 * ga + 1) << 4) | ((2 * gb) << 8) | ((2 * gb + 1) << 12);
    // lanes past the 26 words of a base-3 chunk row read lane 25's word; their
    // table slots hold zeros
    const int wlane = LAYOUT == BT_LAYOUT_B3 ? (L < 26 ? L : 25) : L;
    // continuous base-3: which bytes of the lane's word count for its first
    // group (the split byte's first-group part among them), and where its
    // extra lookup goes (the zero word for lanes without a split byte)
    float wa[4] = {1.f, 1.f, 1.f, 1.f};
    uint32_t exsh = 0, exmul = 0, exadd = 256 * 16;
    if (CONT) {
        const int sidx = L == 6 ? 0 : L == 12 ? 1 : L == 19 ? 2 : L == 25 ? 3 : -1;
        if (sidx >= 0) {
            const int sb = split_byte(sidx) - 4 * L;
#pragma unroll
            for (int i = 0; i < 4; ++i) wa[i] = i <= sb ? 1.f : 0.f;
            exsh = 8u * sb;
            exmul = 16u;
            exadd = 4u * sidx;
        }
    }

    if (L == 0) {
        for (int d = 0; d < kLutDepth; ++d) mbar_init(rg.bar + 8 * d, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (P.sign && threadIdx.x < kBlock / 16)
        reinterpret_cast<uint4*>(sgn)[threadIdx.x] = __ldg(reinterpret_cast<const uint4*>(P.sign) + threadIdx.x);
    lut_zero_invalid<LAYOUT>(table);

    // This CTA's contiguous share of the launch's (matrix, chunk, row) items
    // (lut_share), cut into segments. Each warp requests its sets (warp, warp + 16, ... of
    // every segment) in order through its own cursor, up to kLutDepth ahead of
    // the set it works on, across segment boundaries. Weights, scales and S
    // are never written by the kernels this launch may overlap, so the first
    // sets go out before the grid dependency is resolved.
    int64_t rc0, rc1;
    lut_share(P, rc0, rc1);
    uint32_t issued = 0, done = 0;  // sets requested / consumed by this warp
    bool ok = true;
    LutSeg is;
    int64_t irc = rc0;
    int iq = 0;
    bool ihave = lut_next_seg(P, irc, rc1, is);
    auto warp_sets = [&](const LutSeg& g) {
        const int nsets = (g.n1 - g.n0 + kLutSet - 1) / kLutSet;
        return warp < nsets ? (nsets - warp + kLutWarps - 1) / kLutWarps : 0;
    };
    auto issue_next = [&]() {
        while (ihave && iq >= warp_sets(is)) {
            ihave = lut_next_seg(P, irc, rc1, is);
            iq = 0;
        }
        if (!ihave) return;
        if (L == 0) {
            const int cb = is.c * CB;
            const int sx = CONT ? (5 * is.c) & ~7 : (4 * is.c) & ~7;
            lut_issue_set(rg, &P.cmap[is.p], &P.smap[is.p], issued, cb & ~15, sx,
                          is.n0 + (int64_t)kLutSet * (warp + kLutWarps * iq));
        }
        ++iq;
        ++issued;
    };
    for (int d = 0; d < kLutDepth; ++d) issue_next();
    int64_t rc = rc0;
    LutSeg sg;
    bool have = lut_next_seg(P, rc, rc1, sg);

    // the raw blocks of x a segment needs (continuous: the one or two blocks
    // its 640 columns touch), staged by warp 0
    auto seg_blocks = [&](const LutSeg& g, int& b0, int& b1) {
        const int64_t k0 = (int64_t)g.c * CHUNK;
        b0 = (int)(k0 / kBlock);
        b1 = -1;
        if (CONT) {
            const int64_t K = (int64_t)P.p[g.p].K;
            const int64_t kend = min(k0 + CHUNK, K) - 1;
            if (kend / kBlock != b0) b1 = (int)(kend / kBlock);
        }
    };
    auto stage = [&](const LutSeg& g) {
        const LutProblem& q = P.p[g.p];
        int b0, b1;
        seg_blocks(g, b0, b1);
        lut_stage_block(q.x, q.x_bf16, b0, xst_s);
        if (b1 >= 0) lut_stage_block(q.x, q.x_bf16, b1, xst_s + kBlock * (q.x_bf16 ? 2 : 4));
    };

    pdl_wait();  // x may come from the preceding kernel, which may also still read the partials
    pdl_launch_dependents();

    int bad = 0;
    int cur_p = -1, cur_blk = -1;
    if (have && warp == 0 && !P.p[sg.p].src) stage(sg);
    while (have) {
        const LutProblem& pr = P.p[sg.p];
        const int n0 = sg.n0, n1 = sg.n1;
        float* part = P.part + pr.part_base + (int64_t)sg.c * pr.ld;
        const int coff = (sg.c * CB) & 15;
        const int soff = CONT ? 2 * ((5 * sg.c) & 7) : 2 * ((4 * sg.c) & 7);  // bytes into a scale row
        int b0, b1;
        seg_blocks(sg, b0, b1);
        const int blk = b0;
        // continuous chunks always rebuild xr from their own one or two blocks
        const bool new_blk = CONT || sg.p != cur_p || blk != cur_blk;
        const int kvalid = CONT ? (int)min((int64_t)CHUNK, (int64_t)pr.K - (int64_t)sg.c * CHUNK) : 0;
        const int my = warp_sets(sg);

        __syncthreads();  // the previous segment's lookups are done with table / xs
        if (new_blk) {
            if (pr.src) {  // x is an earlier matrix's output: add up its partials
                lut_gather_block(pr, P.y_bf16, b0, lut_smem + GE::kStage);
                if (b1 >= 0) lut_gather_block(pr, P.y_bf16, b1, lut_smem + GE::kStage + kBlock * (P.y_bf16 ? 2 : 4));
                __syncthreads();
            }
            if (warp == 0) {
                cp_async_wait_all();
                __syncwarp();
                if (CONT)
                    lut_rotate_chunk(xst, pr.x_bf16, sgn, P.sign != nullptr, (int64_t)sg.c * CHUNK, b0, b1, kvalid,
                                     xr, tile);
                else
                    lut_rotate_block(xst, pr.x_bf16, sgn, P.sign != nullptr, xr, tile);
            }
            cur_p = sg.p;
            cur_blk = blk;
            __syncthreads();
        }
        if (CONT) lut_scatter<LAYOUT>(xr, 0, xs, kvalid);
        else lut_scatter<LAYOUT>(xr, (sg.c * CHUNK - blk * kBlock) / CHUNK, xs);
        __syncthreads();
        lut_build<LAYOUT>(xs, table);
        if (CONT) lut_build_extra(xr, reinterpret_cast<float*>(lut_smem + GE::kExtra), kvalid);
        __syncthreads();

        // the next segment; its block(s) of x are staged now if needed
        LutSeg nx;
        int64_t nrc = rc;
        const bool nhave = lut_next_seg(P, nrc, rc1, nx);
        if (nhave && warp == 0) {
            const int nb = (int)(((int64_t)nx.c * CHUNK) / kBlock);
            if ((CONT || nx.p != sg.p || nb != blk) && !P.p[nx.p].src) stage(nx);
        }

        for (int q = 0; q < my && ok; ++q) {
            const uint32_t n = done;
            const uint32_t d = n % kLutDepth;
            if (!lut_wait(rg.bar + 8 * d, (n / kLutDepth) & 1u)) {
                ok = false;
                bad |= BT_DEVERR_TIMEOUT;
                break;
            }
            ++done;
            const uint32_t cslot = rg.ring + d * rg.slot_bytes + coff + 4 * wlane;
            const uint32_t sslot = rg.ring + d * rg.slot_bytes + kLutSet * rg.cbox + soff;
            float a16[kLutSet];
#pragma unroll
            for (int i = 0; i < kLutSet; ++i) {
                const uint32_t cw = lds_u32(cslot + i * rg.cbox);
                if (CHECK && lane_on) bad |= lut_check<LAYOUT>(cw);
                const uint32_t o0 = prmt(cw, lanebytes, 0x6604u);
                const uint32_t o1 = prmt(cw, lanebytes, 0x6615u);
                const uint32_t o2 = prmt(cw, lanebytes, 0x6624u);
                const uint32_t o3 = prmt(cw, lanebytes, 0x6635u);
                const float e0 = lds_f32(tab_s + o0);
                const float e1 = lds_f32(tab_s + o1);
                const float e2 = lds_f32(tab_s + kLutRegion + o2);
                const float e3 = lds_f32(tab_s + kLutRegion + o3);
                if (CONT) {
                    const float ex = lds_f32(extra_s + ((cw >> exsh) & 0xFFu) * exmul + exadd);
                    const float sa = f16_bits_to_f32(lds_u16(sslot + GE::kSBox * 2 * i + 2 * ga));
                    const float sbv = f16_bits_to_f32(lds_u16(sslot + GE::kSBox * 2 * i + 2 * gb));
                    const float A = fmaf(wa[3], e3, fmaf(wa[2], e2, fmaf(wa[1], e1, wa[0] * e0)));
                    const float B = fmaf(1.f - wa[3], e3, fmaf(1.f - wa[2], e2, fmaf(1.f - wa[1], e1,
                                                                                      fmaf(1.f - wa[0], e0, ex))));
                    a16[i] = fmaf(sbv, B, sa * A);
                } else {
                    const uint2 q4 = lds_u64(sslot + 16 * i);
                    const uint32_t sp = prmt(q4.x, q4.y, ssel);
                    const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sp));
                    a16[i] = fmaf(sf.y, e2 + e3, sf.x * (e0 + e1));
                }
            }
            const int r0 = n0 + kLutSet * (warp + kLutWarps * q);
            const float v = lut_transpose_reduce(a16);  // every value read from the slot is consumed here
            __syncwarp();
            issue_next();  // into the slot just freed
            if (L < kLutSet && r0 + L < n1) part[r0 + L] = v;  // the row's chunk partial
        }
        sg = nx;
        rc = nrc;
        have = nhave;
    }
    // after a timeout: let every copy still in flight land before exiting
    // (each wait is bounded; a set whose wait ran out does not stop the
    // waits on the sets requested after it)
    for (; done < issued; ++done) lut_wait(rg.bar + 8 * (done % kLutDepth), (done / kLutDepth) & 1u);
    cp_async_wait_all();
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (L == 0 && bad) report(P.dev_err, bad);
}

// y of up to 12 matrices, one thread per output: its chunk partials added in
// chunk order, up to UNROLL loads in flight together.
template <int UNROLL>
__global__ void __launch_bounds__(kLutReduceThreads, UNROLL >= 64 ? 1 : 4)
gemv_lut_reduce_kernel(const __grid_constant__ LutReduceParams R) {
    // the tile's matrix and first row, from the parameters, before the wait
    int q = 0, k = blockIdx.x;
    for (; q < R.nprob; ++q) {
        const int t = (int)(((int64_t)R.M[q] * R.N[q] + kLutReduceThreads - 1) / kLutReduceThreads);
        if (k < t) break;
        k -= t;
    }
    pdl_wait();
    pdl_launch_dependents();
    if (q >= R.nprob) return;
    const int64_t idx = (int64_t)k * kLutReduceThreads + threadIdx.x;  // n * M + m: partial (n, m) of a chunk
    if (idx >= (int64_t)R.M[q] * R.N[q]) return;
    const int n = (int)(idx / R.M[q]), m = (int)(idx - (int64_t)n * R.M[q]);
    float v[1];
    lut_row_sums<1, UNROLL>(R.part[q], (int64_t)R.M[q] * R.ld[q], R.nchunk[q], (int)idx, 0, v);
    const int64_t yi = (int64_t)m * R.N[q] + n;
    if (R.y_bf16) reinterpret_cast<__nv_bfloat16*>(R.y[q])[yi] = __float2bfloat16_rn(v[0]);
    else reinterpret_cast<float*>(R.y[q])[yi] = v[0];
}

// ------------------------------------------------- M = 2..16: tensor cores ----
//
// Several activation rows share every weight byte, so the bytes are decoded
// once into FP16 digit fields (bt_slots.cuh) and multiplied on the tensor
// cores (m16n8k16: 16 weight rows x 16 k by 8 activation rows, two n8 blocks
// for M > 8) instead of being looked up per row. A prep kernel rotates x and
// writes, per 128-group and activation row, the fragment words in slot order
// and the group constants; the main kernel keeps the table-lookup kernel's
// work split, TMA ring and chunk partials, and copies each segment's chunk of
// fragments into shared memory (the next one while it streams the current).

template <int LAYOUT>
struct MmaGeom {
    static constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    static constexpr int kCBox = LAYOUT == BT_LAYOUT_B3 ? kLutCBoxB3 : kLutCBox2b;
    static constexpr int kSlot = kLutSet * kCBox + kLutSet * 16;
    static constexpr int kLut = LAYOUT == BT_LAYOUT_B3 ? kB3LutBytes : 0;      // decode table
    static constexpr int kRing = kLut;
    // per chunk: fragment words [4 q][NT t][M m][4 c][2 hp] (the 32 lanes of a
    // load, m = lane / 4, c = lane % 4, read 256 contiguous bytes) and group
    // constants [4 q][M m] (corr, 2^e); two buffers
    static constexpr int kFragBytes = 4 * NT * 16 * 32;
    static constexpr int kMetaBytes = 4 * 16 * 8;
    static constexpr int kBuf = kRing + kLutWarps * kLutDepth * kSlot;
    static constexpr int kBufBytes = kFragBytes + kMetaBytes;
    static constexpr int kBar = kBuf + 2 * kBufBytes;
    static constexpr int kSmem = kBar + kLutWarps * kLutDepth * 8;
    static_assert(kRing % 128 == 0 && kSlot % 128 == 0, "ring slots are TMA destinations");
    static_assert(kBuf % 16 == 0 && kBufBytes % 16 == 0, "16-byte asynchronous copies land in the buffers");
    static_assert(kSmem <= 227 * 1024, "one CTA per SM");
};

struct MmaLut {  // the decode table at the start of dynamic shared memory
    __device__ __forceinline__ static uint32_t ld(uint32_t off) { return lds_u32(smem_addr(lut_smem) + off); }
};

// The k (0..127, or -1: empty) and digit field of every half of a group's
// activation fragment words, word w = 8 t + 2 c + hp, half u: the slot maps of
// bt_slots.cuh tabulated once at compile time.
struct SlotTable {
    int8_t k[2][kB3Mmas * 8 * 2];
    int8_t f[2][kB3Mmas * 8 * 2];
};
constexpr SlotTable make_slot_table() {
    SlotTable T{};
    for (int l = 0; l < 2; ++l)
        for (int w = 0; w < kB3Mmas * 8; ++w)
            for (int u = 0; u < 2; ++u) {
                const int t = w / 8, c = (w % 8) / 2, hp = w % 2;
                int field = 0, k = -1;
                if (l == 0) k = b3_slot(t, c, 2 * hp + u, &field);
                else if (t < k2bMmas) k = tb_slot(t, c, 2 * hp + u, &field);
                T.k[l][2 * w + u] = static_cast<int8_t>(k);
                T.f[l][2 * w + u] = static_cast<int8_t>(k >= 0 ? field : 0);
            }
    return T;
}
static __constant__ SlotTable c_slots = make_slot_table();

// Activation fragments and group constants of row m, group q of the chunk
// (the chunk's 128 x' values at xg), by one warp: per-group exponent e from
// the largest |x'|, fragment words FP16(x' 2^(24 - 2i - e)) in slot order
// (every lane writes some of the NT * 8 words), and corr = 2^e times the
// tensor-core sum with every digit 1, by the same MMA chain the stream runs,
// so zero trits give exactly 0.
// dst: the word (t = 0, c = 0, hp = 0) of this group and row; word (t, c, hp)
// at dst[t * tstride + c * 2 + hp]. tab: (k, field) pairs of the slot table.
template <int LAYOUT>
__device__ __forceinline__ void mma_build_group(const float* xg, uint32_t* dst, int tstride, float2* meta,
                                                const int8_t* tab) {
    constexpr int NT = MmaGeom<LAYOUT>::NT;
    const int lane = threadIdx.x & 31;
    float amax = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) amax = fmaxf(amax, fabsf(xg[32 * r + lane]));
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
    int E = amax > 0.f ? ilogbf(amax) + 1 : -100;  // amax < 2^E
    E = max(-100, min(100, E));
    const int e = 9 + E;
#pragma unroll
    for (int w = lane; w < NT * 8; w += 32) {  // w = 8 t + 2 c + hp
        uint32_t word = 0;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int k = tab[4 * w + 2 * u], i = tab[4 * w + 2 * u + 1];
            if (k >= 0) {
                const __half hv = __float2half_rn(xg[k] * exp2i(24 - 2 * i - e));
                word |= static_cast<uint32_t>(__half_as_ushort(hv)) << (16 * u);
            }
        }
        dst[(w >> 3) * tstride + (w & 7)] = word;
    }
    __syncwarp();
    uint32_t bf[NT][2];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) bf[t][hp] = lane < 4 ? dst[t * tstride + lane * 2 + hp] : 0u;  // column 0
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
    if (lane == 0) *meta = make_float2(d[0] * exp2i(e), exp2i(e));
}

// Prep: one CTA of 8 warps per (activation row m, 1024-block b). Warp 0
// rotates the block (S, then H_1024 / 32) or copies it when x is already
// rotated; warp q then writes group 8 b + q's fragment words and constants.
// Output layout, per 128-group g: words [g][NT][M][4][2], constants [g][M].
struct MmaPrepArgs {
    const void* x;
    const int8_t* sign;  // NULL: x already rotated
    uint32_t* frag;
    float2* meta;
    int x_bf16, M, K;
};

template <int LAYOUT>
__global__ void __launch_bounds__(256) gemv_mma_prep_kernel(const MmaPrepArgs a) {
    constexpr int NT = MmaGeom<LAYOUT>::NT;
    __shared__ __align__(16) float xs[32 * kTileStride];
    __shared__ int8_t tab[NT * 8 * 2 * 2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = a.K / kBlock;
    const int m = blockIdx.x / nblk, b = blockIdx.x % nblk;
    if (threadIdx.x < NT * 8 * 2) {
        constexpr int lt = LAYOUT == BT_LAYOUT_B3 ? 0 : 1;
        tab[2 * threadIdx.x] = c_slots.k[lt][threadIdx.x];
        tab[2 * threadIdx.x + 1] = c_slots.f[lt][threadIdx.x];
    }
    pdl_wait();  // x may be the previous kernel's output
    pdl_launch_dependents();
    if (warp == 0) {
        float v[32];
        const int64_t off = (int64_t)m * a.K + (int64_t)b * kBlock;
        if (a.sign) {
            load_signed_bf16_block(static_cast<const uint16_t*>(a.x) + off, a.sign, v);
            fwht1024_warp(v, xs);
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; ++j) xs[32 * j + lane] = v[j];  // lane holds element 32 j + lane
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int64_t i = off + 32 * j + lane;
                xs[32 * j + lane] = a.x_bf16 ? bf16_bits_to_f32(static_cast<const uint16_t*>(a.x)[i])
                                             : static_cast<const float*>(a.x)[i];
            }
        }
    }
    __syncthreads();
    const int g = 8 * b + warp;
    mma_build_group<LAYOUT>(xs + kGroup * warp, a.frag + ((int64_t)g * NT * a.M + m) * 8, a.M * 8,
                            a.meta + (int64_t)g * a.M + m, tab);
}

template <int LAYOUT, int NB, bool CHECK>
__global__ void __launch_bounds__(kLutThreads, 1) gemv_mma_kernel(const __grid_constant__ LutParams P) {
    using GE = MmaGeom<LAYOUT>;
    constexpr int NT = GE::NT;
    const int warp = threadIdx.x >> 5, L = threadIdx.x & 31;
    const int g = L >> 2, c = L & 3;
    const int M = P.M;
    const int CB = LAYOUT == BT_LAYOUT_B3 ? 4 * kB3GroupBytes : 4 * k2bGroupBytes;  // bytes per chunk row
    LutRing rg;
    rg.cbox = GE::kCBox;
    rg.slot_bytes = GE::kSlot;
    rg.ring = smem_addr(lut_smem + GE::kRing) + warp * kLutDepth * rg.slot_bytes;
    rg.bar = smem_addr(lut_smem + GE::kBar) + warp * kLutDepth * 8;
    const uint32_t buf_s = smem_addr(lut_smem + GE::kBuf);
    // words and constants of a chunk, in global memory: contiguous
    const int fwords = 4 * NT * M * 8, mbytes = 4 * M * 8;
    const uint32_t* frag = reinterpret_cast<const uint32_t*>(P.frag);
    const float2* gmeta = reinterpret_cast<const float2*>(P.meta);
    // all threads: the chunk c's fragments and constants into buffer `bi`
    auto fetch_chunk = [&](int chunk, int bi) {
        const uint32_t dst = buf_s + bi * GE::kBufBytes;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(frag + (int64_t)chunk * fwords);
        for (int i = threadIdx.x; i < fwords / 4; i += kLutThreads) cp_async16(dst + 16 * i, src + 16 * i);
        const uint8_t* msrc = reinterpret_cast<const uint8_t*>(gmeta + (int64_t)chunk * 4 * M);
        for (int i = threadIdx.x; i < mbytes / 16; i += kLutThreads)
            cp_async16(dst + GE::kFragBytes + 16 * i, msrc + 16 * i);
        cp_async_commit();
    };

    if (L == 0) {
        for (int d = 0; d < kLutDepth; ++d) mbar_init(rg.bar + 8 * d, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if constexpr (LAYOUT == BT_LAYOUT_B3) b3_lut_fill(lut_smem, threadIdx.x, kLutThreads);

    int64_t rc0, rc1;
    lut_share(P, rc0, rc1);
    uint32_t issued = 0, done = 0;
    bool ok = true;
    LutSeg is;
    int64_t irc = rc0;
    int iq = 0;
    bool ihave = lut_next_seg(P, irc, rc1, is);
    auto warp_sets = [&](const LutSeg& sgm) {
        const int nsets = (sgm.n1 - sgm.n0 + kLutSet - 1) / kLutSet;
        return warp < nsets ? (nsets - warp + kLutWarps - 1) / kLutWarps : 0;
    };
    auto issue_next = [&]() {
        while (ihave && iq >= warp_sets(is)) {
            ihave = lut_next_seg(P, irc, rc1, is);
            iq = 0;
        }
        if (!ihave) return;
        if (L == 0) {
            const int cb = is.c * CB;
            lut_issue_set(rg, &P.cmap[is.p], &P.smap[is.p], issued, cb & ~15, (4 * is.c) & ~7,
                          is.n0 + (int64_t)kLutSet * (warp + kLutWarps * iq));
        }
        ++iq;
        ++issued;
    };
    for (int d = 0; d < kLutDepth; ++d) issue_next();
    int64_t rc = rc0;
    LutSeg sg;
    bool have = lut_next_seg(P, rc, rc1, sg);
    uint32_t mG[3] = {0u, 0u, 0u}, mH[3] = {0u, 0u, 0u};
    if constexpr (LAYOUT == BT_LAYOUT_B3) b3_pair12_masks(c, mG, mH);
    const uint32_t lane4 = static_cast<uint32_t>(L) * 4u;

    pdl_wait();  // the prep kernel's fragments
    pdl_launch_dependents();

    uint32_t err = 0;
    int bad = 0;
    int bi = 0;
    if (have) fetch_chunk(sg.c, 0);
    while (have) {
        const LutProblem& pr = P.p[sg.p];
        const int n0 = sg.n0, n1 = sg.n1;
        float* part = P.part + pr.part_base + (int64_t)sg.c * M * pr.ld;
        const int coff = (sg.c * CB) & 15;
        const int soff = 2 * ((4 * sg.c) & 7);
        const int my = warp_sets(sg);
        cp_async_wait_all();
        __syncthreads();  // this chunk's fragments are in buffer bi; the other buffer is free
        LutSeg nx;
        int64_t nrc = rc;
        const bool nhave = lut_next_seg(P, nrc, rc1, nx);
        if (nhave) fetch_chunk(nx.c, bi ^ 1);  // overlaps this segment's stream
        const uint32_t slots_s = buf_s + bi * GE::kBufBytes, meta_s = slots_s + GE::kFragBytes;

        for (int qs = 0; qs < my && ok; ++qs) {
            const uint32_t n = done;
            const uint32_t d = n % kLutDepth;
            if (!lut_wait(rg.bar + 8 * d, (n / kLutDepth) & 1u)) {
                ok = false;
                bad |= BT_DEVERR_TIMEOUT;
                break;
            }
            ++done;
            const uint32_t cs = rg.ring + d * rg.slot_bytes + coff;       // row 0 of the chunk in the slot
            const uint32_t ss = rg.ring + d * rg.slot_bytes + kLutSet * rg.cbox + soff;
            const uint32_t rowg = cs + g * rg.cbox, rowh = cs + (g + 8) * rg.cbox;
            float acc[NB][4];
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t Rg[16], Rh[16], QG[3], QH[3];
                if constexpr (LAYOUT == BT_LAYOUT_B3) {
                    // the lane's bytes 6c .. 6c + 5 of group q, from the aligned word below them
                    const uint32_t Ag = rowg + q * kB3GroupBytes + 6 * c, Ah = rowh + q * kB3GroupBytes + 6 * c;
                    const uint32_t o8 = (Ag & 3u) * 8u;  // rows are 112 B apart: the same shift for both
                    const uint32_t w12 = lds_u16(cs + (c < 2 ? g : g + 8) * rg.cbox + q * kB3GroupBytes + 24);
                    b3_decode_tile<CHECK, MmaLut>(lds_u32(Ag & ~3u), lds_u32((Ag & ~3u) + 4), lds_u32(Ah & ~3u),
                                                  lds_u32((Ah & ~3u) + 4), w12, o8, lane4, mG, mH, Rg, Rh, QG, QH,
                                                  err);
                } else {
                    const uint2 x0 = lds_u64(rowg + q * k2bGroupBytes + 8 * c);
                    const uint2 x1 = lds_u64(rowh + q * k2bGroupBytes + 8 * c);
                    tb_decode_tile<CHECK>(x0, x1, Rg, Rh, err);
#pragma unroll
                    for (int k = 0; k < 3; ++k) QG[k] = QH[k] = 0u;
                }
                const float sgv = f16_bits_to_f32(lds_u16(ss + g * 16 + 2 * q));
                const float shv = f16_bits_to_f32(lds_u16(ss + (g + 8) * 16 + 2 * q));
                // B fragments of this lane's activation rows g (block 0) and 8 + g (block 1)
                uint32_t bf[NB][NT][2];
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    const int m = 8 * b + g;
                    const uint32_t ba = slots_s + (uint32_t)(((q * NT) * M + m) * 32 + c * 8);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        uint2 v = make_uint2(0u, 0u);
                        if (m < M) v = lds_u64(ba + (uint32_t)(t * M * 32));
                        bf[b][t][0] = v.x;
                        bf[b][t][1] = v.y;
                    }
                }
                float d4[NB][4];
                if constexpr (NB == 2) {
                    group_mma2<LAYOUT == BT_LAYOUT_B3>(Rg, Rh, QG, QH, bf[0], bf[1], d4[0], d4[1]);
                } else if constexpr (LAYOUT == BT_LAYOUT_B3) {
                    b3_group_mma(Rg, Rh, QG, QH, bf[0], d4[0]);
                } else {
                    tb_group_mma(Rg, Rh, bf[0], d4[0]);
                }
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    // D columns 2c, 2c + 1 of this block are activation rows 8 b + 2c (+1)
                    const int m0 = 8 * b + 2 * c;
                    const uint2 md0 = m0 < M ? lds_u64(meta_s + (uint32_t)((q * M + m0) * 8)) : make_uint2(0u, 0u);
                    const uint2 md1 = m0 + 1 < M ? lds_u64(meta_s + (uint32_t)((q * M + m0 + 1) * 8))
                                                 : make_uint2(0u, 0u);
                    const float c0 = __uint_as_float(md0.x), p0 = __uint_as_float(md0.y);
                    const float c1 = __uint_as_float(md1.x), p1 = __uint_as_float(md1.y);
                    acc[b][0] = fmaf(sgv, fmaf(d4[b][0], p0, -c0), acc[b][0]);
                    acc[b][1] = fmaf(sgv, fmaf(d4[b][1], p1, -c1), acc[b][1]);
                    acc[b][2] = fmaf(shv, fmaf(d4[b][2], p0, -c0), acc[b][2]);
                    acc[b][3] = fmaf(shv, fmaf(d4[b][3], p1, -c1), acc[b][3]);
                }
            }
            __syncwarp();
            issue_next();  // into the slot just freed
            const int r0 = n0 + kLutSet * (warp + kLutWarps * qs);
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                const int m0 = 8 * b + 2 * c;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int m = m0 + (r & 1), row = r0 + g + 8 * (r >> 1);
                    if (m < M && row < n1) part[(int64_t)row * M + m] = acc[b][r];
                }
            }
        }
        sg = nx;
        rc = nrc;
        have = nhave;
        bi ^= 1;
    }
    for (; done < issued; ++done) lut_wait(rg.bar + 8 * (done % kLutDepth), (done / kLutDepth) & 1u);
    cp_async_wait_all();
    if (CHECK) {
        if (LAYOUT == BT_LAYOUT_B3) { if (err >> 31) bad |= BT_DEVERR_INVALID_CODE; }
        else if (err & 0x55555555u) bad |= BT_DEVERR_INVALID_CODE;
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (L == 0 && bad) report(P.dev_err, bad);
}

// ---------------------------------------------------------------- host ----

static size_t lut_align(size_t v, size_t a) { return (v + a - 1) / a * a; }

// The launch pairs a list is cut into: at most kLutMaxProblems matrices each,
// and a new pair wherever a matrix reads the output of a matrix of the
// current pair.
template <class F>
static void lut_for_each_launch(const DecodeProblem* pr, int count, F&& f) {
    int first = 0;
    while (first < count) {
        int n = 1;
        while (first + n < count && n < kLutMaxProblems && pr[first + n].x_from < first) ++n;
        f(first, n);
        first += n;
    }
}

// Chunks of a row: 512 columns, or 640 (128 bytes) in the continuous layout
// (the last one may be partial).
static int64_t lut_nchunk(int layout, int64_t K) {
    return layout == BT_LAYOUT_B3C ? (K + kLutChunkC - 1) / kLutChunkC : K / kLutChunk;
}

// Bytes of one packed row.
static int64_t lut_row_bytes(int layout, int64_t K) {
    if (layout == BT_LAYOUT_B3C) return ((K + 4) / 5 + 15) / 16 * 16;
    return (K / kGroup) * (layout == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes);
}

// Partial floats of one matrix: [chunks][N rounded up to 4].
static int64_t lut_part_floats(int layout, const DecodeProblem& p) {
    return lut_nchunk(layout, p.K) * ((p.N + 3) & ~3);
}

// Every matrix of a list keeps its partials until the list's reductions at
// the end (a later group may read them as its input): their sum, each group
// starting on a 256-byte boundary.
size_t gemv1_workspace_bytes(int layout, const DecodeProblem* pr, int count) {
    size_t total = 0;
    lut_for_each_launch(pr, count, [&](int first, int n) {
        int64_t f = 0;
        for (int i = first; i < first + n; ++i) f += lut_part_floats(layout, pr[i]);
        total += lut_align((size_t)f * sizeof(float), 256);
    });
    return std::max(total, (size_t)256);
}

// Products whose weights TMA can stream: K a multiple of 1024 (so the scale
// rows are whole 16-byte units), 16-byte aligned codes and scales.
bool gemv_lut_applies(int layout, int64_t M, int64_t K, const void* codes, const void* scales) {
    return M >= 1 && M <= (layout == BT_LAYOUT_B3C ? 1 : 16) && K > 0 && K % kBlock == 0 &&
           (reinterpret_cast<uintptr_t>(scales) & 15) == 0 && (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
}

// Workspace of one product with M activation rows: for M > 1 the prep
// kernel's fragment words (M x K/128 x 9 x 32 bytes) and group constants
// (M x K/128 x 8 bytes) first, then the partials [K/512][N rounded up to 4][M].
static size_t mma_frag_bytes(int64_t M, int64_t K) { return lut_align((size_t)M * (K / kGroup) * kB3Mmas * 32, 256); }
static size_t mma_meta_bytes(int64_t M, int64_t K) { return lut_align((size_t)M * (K / kGroup) * 8, 256); }

size_t gemv_lut_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K) {
    const size_t part =
        lut_align((size_t)lut_nchunk(layout, K) * (size_t)M * (size_t)((N + 3) & ~3) * sizeof(float), 256);
    return std::max((M > 1 ? mma_frag_bytes(M, K) + mma_meta_bytes(M, K) : 0) + part, (size_t)256);
}

template <class Kern>
static cudaError_t lut_launch_k(Kern kern, int smem, const LutParams& P, int grid, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kLutThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, P);
}

// The partials and outputs of one group, as the reduction reads them.
template <int LAYOUT, bool CHECK>
static cudaError_t lut_launch_t(const LutParams& P, int grid, cudaStream_t stream) {
    if (P.M == 1) return lut_launch_k(gemv_lut_kernel<LAYOUT, CHECK>, LutGeom<LAYOUT>::kSmem, P, grid, stream);
    if constexpr (LAYOUT == BT_LAYOUT_B3C) {
        return cudaErrorInvalidValue;  // single rows only
    } else {
        if (P.M <= 8) return lut_launch_k(gemv_mma_kernel<LAYOUT, 1, CHECK>, MmaGeom<LAYOUT>::kSmem, P, grid, stream);
        return lut_launch_k(gemv_mma_kernel<LAYOUT, 2, CHECK>, MmaGeom<LAYOUT>::kSmem, P, grid, stream);
    }
}

// The main kernel of group [first, first + count), M activation rows (M > 1:
// one matrix). base[i]: offset in floats of matrix i's partials in the
// workspace `part`.
static cudaError_t lut_launch_group(int layout, const DecodeProblem* all, const int64_t* base, int first, int count,
                                    int M, const int8_t* sign, int y_bf16, float* part, int32_t* dev_err,
                                    int num_sms, cudaStream_t stream, const void* frag = nullptr,
                                    const void* meta = nullptr) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    LutParams P{};
    const bool cont = layout == BT_LAYOUT_B3C;
    int64_t rc = 0;
    for (int i = 0; i < count; ++i) {
        const DecodeProblem& s = all[first + i];
        LutProblem& d = P.p[i];
        const int64_t G = s.K / kGroup, RB = lut_row_bytes(layout, s.K);
        d.N = static_cast<int32_t>(s.N);
        d.K = static_cast<int32_t>(s.K);
        d.ld = static_cast<int32_t>((s.N + 3) & ~3);
        d.nchunk = static_cast<int32_t>(lut_nchunk(layout, s.K));
        d.rc_base = rc;
        d.part_base = base[first + i];
        if (s.x_from >= 0) {  // an earlier group's output: summed from its partials
            const DecodeProblem& q = all[s.x_from];
            d.src = part + base[s.x_from];
            d.src_ld = static_cast<int32_t>((q.N + 3) & ~3);
            d.src_nchunk = static_cast<int32_t>(lut_nchunk(layout, q.K));
            d.x = nullptr;
            d.x_bf16 = y_bf16;
        } else {
            d.src = nullptr;
            d.x = s.x;
            d.x_bf16 = s.x_bf16;
        }
        rc += (int64_t)d.nchunk * d.N;
        const cuuint64_t cdim[2] = {static_cast<cuuint64_t>(RB), static_cast<cuuint64_t>(s.N)};
        const cuuint64_t cstr[1] = {static_cast<cuuint64_t>(RB)};
        const cuuint32_t cbox[2] = {static_cast<cuuint32_t>(layout == BT_LAYOUT_B3 ? kLutCBoxB3 : kLutCBox2b), kLutSet};
        const cuuint64_t sdim[2] = {static_cast<cuuint64_t>(G), static_cast<cuuint64_t>(s.N)};
        const cuuint64_t sstr[1] = {static_cast<cuuint64_t>(G) * 2};
        const cuuint32_t sbox[2] = {cont ? 16u : 8u, kLutSet};
        const cuuint32_t one[2] = {1, 1};
        if (enc(&P.cmap[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(s.codes), cdim, cstr, cbox, one,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            enc(&P.smap[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(s.scales), sdim, sstr, sbox, one,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    P.sign = sign;
    P.dev_err = dev_err;
    P.part = part;
    P.total_rc = rc;
    P.nprob = count;
    P.y_bf16 = y_bf16;
    P.M = M;
    P.frag = frag;
    P.meta = meta;
    // one CTA per SM, never more CTAs than (chunk, row) items
    const int grid = (int)(rc < num_sms ? rc : num_sms);
    if (layout == BT_LAYOUT_B3)
        return dev_err ? lut_launch_t<BT_LAYOUT_B3, true>(P, grid, stream)
                       : lut_launch_t<BT_LAYOUT_B3, false>(P, grid, stream);
    if (layout == BT_LAYOUT_B3C)
        return dev_err ? lut_launch_t<BT_LAYOUT_B3C, true>(P, grid, stream)
                       : lut_launch_t<BT_LAYOUT_B3C, false>(P, grid, stream);
    return dev_err ? lut_launch_t<BT_LAYOUT_2BIT, true>(P, grid, stream)
                   : lut_launch_t<BT_LAYOUT_2BIT, false>(P, grid, stream);
}

// Outputs of matrices [first, first + count), count <= kLutMaxProblems.
static cudaError_t lut_launch_reduce(int layout, const DecodeProblem* all, const int64_t* base, int first, int count,
                                     int M, int y_bf16, float* part, cudaStream_t stream) {
    LutReduceParams R{};
    R.nprob = count;
    R.y_bf16 = y_bf16;
    int tiles = 0;
    for (int i = 0; i < count; ++i) {
        const DecodeProblem& s = all[first + i];
        R.part[i] = part + base[first + i];
        R.y[i] = s.y;
        R.N[i] = static_cast<int32_t>(s.N);
        R.ld[i] = static_cast<int32_t>((s.N + 3) & ~3);
        R.nchunk[i] = static_cast<int32_t>(lut_nchunk(layout, s.K));
        R.M[i] = M;
        tiles += (int)((M * s.N + kLutReduceThreads - 1) / kLutReduceThreads);
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)tiles);
    cfg.blockDim = dim3(kLutReduceThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // single rows: few outputs, every load of a row in flight at once; several
    // rows: many outputs, four CTAs per SM
    return M == 1 ? cudaLaunchKernelEx(&cfg, gemv_lut_reduce_kernel<64>, R)
                  : cudaLaunchKernelEx(&cfg, gemv_lut_reduce_kernel<16>, R);
}

// A list runs as one main kernel per group (a matrix that reads an output of
// the current group starts the next one) and, at the end, the reductions
// that write every output: a group reads its inputs from the partials of the
// groups before it, so between groups there is nothing else to wait for.
cudaError_t launch_gemv1(int layout, const DecodeProblem* problems, int count, const int8_t* sign, int y_dtype,
                         void* workspace, int32_t* dev_err, int num_sms, cudaStream_t stream) {
    const int y_bf16 = y_dtype == BT_BF16;
    float* part = static_cast<float*>(workspace);
    int64_t base[256];
    {
        int64_t off = 0;
        lut_for_each_launch(problems, count, [&](int first, int n) {
            for (int i = first; i < first + n; ++i) {
                base[i] = off;
                off += lut_part_floats(layout, problems[i]);
            }
            off = (int64_t)lut_align((size_t)off, 64);  // 256-byte boundary between groups
        });
    }
    cudaError_t err = cudaSuccess;
    lut_for_each_launch(problems, count, [&](int first, int n) {
        if (err == cudaSuccess)
            err = lut_launch_group(layout, problems, base, first, n, 1, sign, y_bf16, part, dev_err, num_sms, stream);
    });
    for (int first = 0; first < count && err == cudaSuccess; first += kLutMaxProblems)
        err = lut_launch_reduce(layout, problems, base, first, std::min(kLutMaxProblems, count - first), 1, y_bf16,
                                part, stream);
    return err;
}

// One product with 1 <= M <= 16 activation rows (x [M][K], y [M][N]): the
// table-lookup kernel for M = 1, the tensor-core kernel above it, then the
// reduction.
cudaError_t launch_gemv_lut(int layout, const uint8_t* codes, const uint16_t* scales, const void* x, int x_bf16,
                            const int8_t* sign, int M, int64_t N, int64_t K, int y_dtype, void* y, void* workspace,
                            int32_t* dev_err, int num_sms, cudaStream_t stream) {
    const DecodeProblem p{codes, scales, x, x_bf16, -1, y, N, K};
    const int64_t base[1] = {0};
    const int y_bf16 = y_dtype == BT_BF16;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void* frag = nullptr;
    void* meta = nullptr;
    if (M > 1) {
        frag = ws;
        meta = ws + mma_frag_bytes(M, K);
        ws += mma_frag_bytes(M, K) + mma_meta_bytes(M, K);
        MmaPrepArgs a{x, sign, static_cast<uint32_t*>(frag), static_cast<float2*>(meta), x_bf16, M, (int)K};
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(M * (K / kBlock)));
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = layout == BT_LAYOUT_B3 ? cudaLaunchKernelEx(&cfg, gemv_mma_prep_kernel<BT_LAYOUT_B3>, a)
                                                     : cudaLaunchKernelEx(&cfg, gemv_mma_prep_kernel<BT_LAYOUT_2BIT>, a);
        if (e != cudaSuccess) return e;
    }
    float* part = reinterpret_cast<float*>(ws);
    cudaError_t err = lut_launch_group(layout, &p, base, 0, 1, M, sign, y_bf16, part, dev_err, num_sms, stream,
                                       frag, meta);
    if (err != cudaSuccess) return err;
    return lut_launch_reduce(layout, &p, base, 0, 1, M, y_bf16, part, stream);
}

}  // namespace bt

// Decode GEMV for one activation row (M = 1): y = W x' with x' = R x, by table
// lookup of packed bytes.
//
// One base-3 byte holds five trits of a row of W (Bonsai low-bit course,
// section "先用五个数字理解 1.6bit"), a 2-bit byte four. Against a fixed
// activation vector the contribution of one byte, sum_i t_i x'_(5b+i), depends
// only on the byte's code, so for every byte position of a K chunk the kernel
// tabulates that sum for all 256 codes once and then streams the rows: one
// shared-memory lookup and one FP32 add per byte instead of decoding five
// trits. (The tables hold partial dot products of the rotated activations,
// so they are rebuilt per call; W is never decoded.)
//
// Work split. K is cut into 512-wide chunks (four g128 groups: 104 bytes of a
// base-3 row, 128 of a 2-bit row). Each CTA owns one chunk and an equal slice
// of the rows (with more chunks than SMs, a CTA walks chunks with all rows).
// It rotates the 1024-block that holds its chunk (the warp FWHT of the
// Sylvester H_1024, S applied first, scaled by 1/32; TensorSharp blog,
// sections 3.2 and 5.2), builds the tables and lets each warp stream its own
// contiguous rows in sets of 16. Each warp is its own producer: lane 0 moves a
// set's code bytes ([16 rows][112 B], x rounded down to 16 B so base-3 chunks
// at 8-byte offsets stay legal) and scales ([16 rows][8 halves]) with two TMA
// tensor copies into a two-slot ring, completing on the slot's mbarrier. The
// first sets are requested right after the activation loads, so the rotation
// and the table build run under their latency.
//
// Tables. Lane L of a warp reads code word L (bytes 4L..4L+3) of a row chunk,
// so byte position p = 4L + k is only ever looked up by lane L: its table
// lives in shared-memory bank L and a warp's 32 lookups never conflict. Two
// 64 KB regions [256 codes][64 slots] of FP32 hold the 128 tables; byte k of
// lane L sits in region k/2, slot L + 32 (k % 2). One PRMT turns the code byte
// and a lane constant into the byte offset code * 256 + slot * 4.
//
// Scales multiply per row: a base-3 chunk row has four groups of 26 bytes, so
// a lane's word lies in one group or (lanes 6 and 19) straddles two; the lane
// applies s_a to bytes 0-1 and s_b to bytes 2-3 of its word.
//
// Each warp keeps one FP32 partial per row of its set in every lane and
// reduces the 32 x 16 block with a butterfly transpose (16 shuffles); lanes i
// and i + 16 then hold row i. Partials per (chunk, row) go to the workspace
// and a second kernel, launched as a programmatic dependent, sums the chunks
// of each row in chunk order, so results are deterministic and the workspace
// needs no counters or clearing. (Having the last CTA of a row slice do that
// sum instead costs more on B200: its atomic arrival and the dependent L2
// reads are each about a microsecond, and one CTA per slice does the work.)
#include "bt_internal.cuh"

namespace bt {

constexpr int kLutWarps = 16;
constexpr int kLutThreads = kLutWarps * 32;
constexpr int kLutChunk = 512;                      // k per table set
constexpr int kLutRegion = 256 * 64 * 4;            // [256 codes][64 slots] f32
constexpr int kLutTableBytes = 2 * kLutRegion;
constexpr int kLutXrOffset = kLutTableBytes;         // rotated block, 1024 f32
constexpr int kLutXsOffset = kLutXrOffset + kBlock * 4;  // [5][4][32] f32 slot inputs
constexpr int kLutSet = 16;                          // rows per set (one TMA box, one reduction)
constexpr int kLutDepth = 2;                         // sets in flight per warp
constexpr int kLutCBoxB3 = 112;                      // box bytes per row: 104 + up to 8 of alignment
constexpr int kLutCBox2b = 128;
constexpr int kLutSlotMax = kLutSet * kLutCBox2b + kLutSet * 16;  // codes box + scale box (8 halves/row)
constexpr int kLutTileOffset = kLutXsOffset + 5 * 4 * 32 * 4;   // FWHT exchange tile, 32 x 36 f32
constexpr int kLutBarOffset = kLutTileOffset + 32 * kTileStride * 4;
constexpr int kLutRingOffset = kLutBarOffset + kLutWarps * kLutDepth * 8;
constexpr int kLutSmem = kLutRingOffset + kLutWarps * kLutDepth * kLutSlotMax;
constexpr int kLutMinRows = 64;                      // fewest rows worth a table build

struct LutArgs {
    const uint8_t* codes;
    const uint16_t* scales;
    const void* x;
    const int8_t* sign;  // NULL: x is already rotated
    float* partials;     // [nchunk][N]
    int32_t* dev_err;
    int64_t N;
    int64_t rows_per_part;  // rows of one CTA's slice (multiple of 16)
    int parts;              // CTAs per chunk (1: a CTA walks chunks)
    int K;
    int G;
    int RB;  // bytes per row of codes
    int nchunk;
    int x_bf16;
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

// Table lookup at a shared-window byte address. The ring reads above carry a
// memory clobber (they must stay after the mbarrier wait that publishes the
// TMA bytes); the table is written before a CTA barrier, so lookups need none.
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

struct LutReduceArgs {
    const float* partials;
    void* y;
    int64_t N;
    int nchunk;
    int y_bf16;
};

// Raw words of one lane's 32 bf16 activations of a 1024-block and of its 32
// sign bytes. Fetched before the first weight copies are requested, so that
// the rotation does not queue behind them. (FP32 activations are read when
// the block is rotated.)
struct XFetch {
    uint4 q[4];
    uint4 sg[2];
};

__device__ __forceinline__ void lut_fetch_block(const LutArgs& a, int blk, XFetch& f) {
    const int lane = threadIdx.x & 31;
    if (!a.x_bf16) return;
    const uint4* src =
        reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + (size_t)blk * kBlock + 32 * lane);
#pragma unroll
    for (int q = 0; q < 4; ++q) f.q[q] = __ldg(src + q);
    if (a.sign) {
        const uint4* sg = reinterpret_cast<const uint4*>(a.sign + 32 * lane);
        f.sg[0] = __ldg(sg);
        f.sg[1] = __ldg(sg + 1);
    }
}

// The rotated (or, without S, copied) block into xr as FP32. Warp 0 only.
__device__ __forceinline__ void lut_rotate_block(const LutArgs& a, int blk, const XFetch& f, float* xr,
                                                 float* tile) {
    const int lane = threadIdx.x & 31;
    float v[32];
    if (a.x_bf16) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(f.q);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = bf16_bits_to_f32((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu));
    } else {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + (size_t)blk * kBlock +
                                                            32 * lane);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 t = __ldg(src + q);
            v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
        }
    }
    if (a.sign) {  // the ABI accepts S with bf16 activations only
        const uint32_t* sw = reinterpret_cast<const uint32_t*>(f.sg);
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
template <int LAYOUT>
__device__ __forceinline__ void lut_scatter(const float* xr, int h, float* xs) {
    for (int t = threadIdx.x; t < 5 * 4 * 32; t += kLutThreads) {
        const int i = t >> 7, k = (t >> 5) & 3, L = t & 31;
        const int p = 4 * L + k;
        float v = 0.f;
        if (LAYOUT == BT_LAYOUT_B3) {
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
    if (LAYOUT == BT_LAYOUT_B3) {
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
    if (LAYOUT == BT_LAYOUT_B3) {
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
    if (LAYOUT == BT_LAYOUT_B3) return __vcmpgeu4(w, 0xF3F3F3F3u) ? BT_DEVERR_INVALID_CODE : 0u;
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
    mbar_arrive_tx(bar, (uint32_t)(kLutSet * rg.cbox + kLutSet * 16));
    tma_load_2d(dst, cmap, cx, (int)r0, bar);
    tma_load_2d(dst + kLutSet * rg.cbox, smap, sx, (int)r0, bar);
}

template <int LAYOUT, bool CHECK>
__global__ void __launch_bounds__(kLutThreads, 1)
gemv_lut_kernel(const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap smap, const LutArgs a) {
    float* table = reinterpret_cast<float*>(lut_smem);
    const uint32_t tab_s = smem_addr(lut_smem);
    float* xr = reinterpret_cast<float*>(lut_smem + kLutXrOffset);
    float* xs = reinterpret_cast<float*>(lut_smem + kLutXsOffset);

    const int warp = threadIdx.x >> 5, L = threadIdx.x & 31;
    const int CB = LAYOUT == BT_LAYOUT_B3 ? 4 * kB3GroupBytes : 4 * k2bGroupBytes;  // bytes per chunk row
    const bool lane_on = LAYOUT == BT_LAYOUT_B3 ? L < 26 : true;
    LutRing rg;
    rg.cbox = LAYOUT == BT_LAYOUT_B3 ? kLutCBoxB3 : kLutCBox2b;
    rg.slot_bytes = kLutSet * rg.cbox + kLutSet * 16;
    rg.ring = smem_addr(lut_smem + kLutRingOffset) + warp * kLutDepth * rg.slot_bytes;
    rg.bar = smem_addr(lut_smem + kLutBarOffset) + warp * kLutDepth * 8;

    // lane constants: table byte offsets and scale selectors
    const uint32_t lanebytes = (uint32_t)(4 * L) | ((uint32_t)(4 * L + 128) << 8);
    uint32_t ga, gb;
    if (LAYOUT == BT_LAYOUT_B3) {
        ga = lane_on ? (4 * L) / 26 : 3;
        gb = lane_on ? (4 * L + 3) / 26 : 3;
    } else {
        ga = gb = L >> 3;
    }
    const uint32_t ssel = (2 * ga) | ((2 * ga + 1) << 4) | ((2 * gb) << 8) | ((2 * gb + 1) << 12);
    // lanes past the 26 words of a base-3 chunk row read lane 25's word; their
    // table slots hold zeros
    const int wlane = LAYOUT == BT_LAYOUT_B3 ? (L < 26 ? L : 25) : L;

    // this CTA's chunks and rows
    int chunk = a.parts > 1 ? (int)(blockIdx.x / a.parts) : (int)blockIdx.x;
    const int cstep = a.parts > 1 ? a.nchunk : (int)gridDim.x;
    const int part = a.parts > 1 ? (int)(blockIdx.x % a.parts) : 0;
    const int64_t row_lo = (int64_t)part * a.rows_per_part;
    const int64_t row_hi = min(a.N, row_lo + a.rows_per_part);
    // each warp streams a contiguous share of the rows, in sets of 16
    const int64_t share = (((row_hi - row_lo) + kLutWarps * kLutSet - 1) / (kLutWarps * kLutSet)) * kLutSet;
    const int64_t w_lo = min(row_hi, row_lo + warp * share);
    const int64_t w_hi = min(row_hi, w_lo + share);
    const int nsets = (int)((w_hi - w_lo + kLutSet - 1) / kLutSet);

    if (L == 0) {
        for (int d = 0; d < kLutDepth; ++d) mbar_init(rg.bar + 8 * d, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();

    uint32_t issued = 0, done = 0;  // sets requested / consumed by this warp
    bool ok = true;

    auto box_x = [&](int c, int& cx, int& sx, int& coff, int& soff) {
        const int cb = c * CB;
        cx = cb & ~15;
        coff = cb - cx;
        sx = (4 * c) & ~7;
        soff = 2 * (4 * c - sx);
    };
    lut_zero_invalid<LAYOUT>(table);
    pdl_wait();
    pdl_launch_dependents();

    uint32_t bad = 0;
    int cur_blk = -1;
    for (; chunk < a.nchunk; chunk += cstep) {
        int cx, sx, coff, soff;
        box_x(chunk, cx, sx, coff, soff);
        float* pout = a.partials + (int64_t)chunk * a.N;

        const int blk = (chunk * kLutChunk) / kBlock;
        const bool new_blk = blk != cur_blk;
        XFetch xf;
        if (new_blk && warp == 0) lut_fetch_block(a, blk, xf);
        __syncthreads();  // previous chunk's lookups are done with table / xs
        // The first sets of this chunk's rows go out after warp 0 has issued
        // its activation loads, so those loads do not queue behind the
        // weight stream; the rotation and the table build run under the
        // copies' latency.
        if (L == 0 && ok)
            for (int d = 0; d < kLutDepth && d < nsets; ++d)
                lut_issue_set(rg, &cmap, &smap, issued + d, cx, sx, w_lo + (int64_t)d * kLutSet);
        if (ok) issued += min(kLutDepth, nsets);
        if (new_blk) {
            if (warp == 0) lut_rotate_block(a, blk, xf, xr, reinterpret_cast<float*>(lut_smem + kLutTileOffset));
            cur_blk = blk;
            __syncthreads();
        }
        lut_scatter<LAYOUT>(xr, (chunk * kLutChunk - blk * kBlock) / kLutChunk, xs);
        __syncthreads();
        lut_build<LAYOUT>(xs, table);
        __syncthreads();

        for (int q = 0; q < nsets && ok; ++q) {
            const uint32_t n = done;
            const uint32_t d = n % kLutDepth;
            if (!mbar_wait(rg.bar + 8 * d, (n / kLutDepth) & 1u)) {
                ok = false;
                bad |= BT_DEVERR_TIMEOUT;
                break;
            }
            ++done;
            const uint32_t cslot = rg.ring + d * rg.slot_bytes + coff + 4 * wlane;
            const uint32_t sslot = rg.ring + d * rg.slot_bytes + kLutSet * rg.cbox + soff;
            float acc[kLutSet];
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
                const uint2 q4 = lds_u64(sslot + 16 * i);
                const uint32_t sp = prmt(q4.x, q4.y, ssel);
                const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sp));
                acc[i] = fmaf(sf.y, e2 + e3, sf.x * (e0 + e1));
            }
            const int64_t r0 = w_lo + (int64_t)q * kLutSet;
            const float v = lut_transpose_reduce(acc);  // every value read from the slot is consumed here
            __syncwarp();
            if (L == 0 && q + kLutDepth < nsets) {
                lut_issue_set(rg, &cmap, &smap, issued, cx, sx, r0 + kLutDepth * kLutSet);
            }
            if (q + kLutDepth < nsets) ++issued;
            if (L < kLutSet && r0 + L < w_hi) pout[r0 + L] = v;
        }
    }
    // after a timeout: let every copy still in flight land before exiting
    // (each wait is bounded; a set whose wait ran out does not stop the
    // waits on the sets requested after it)
    for (; done < issued; ++done) mbar_wait(rg.bar + 8 * (done % kLutDepth), (done / kLutDepth) & 1u);

    if (bad) report(a.dev_err, (int)bad);
}

// y[r] = sum over chunks c, in order, of partials[c][r]. A CTA of 8 warps
// takes 32 rows: warp w sums chunks w, w + 8, ... and the eight warp sums
// are added in warp order.
__global__ void __launch_bounds__(256) gemv_lut_reduce_kernel(const LutReduceArgs a) {
    __shared__ float part[8][33];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 32 + lane;
    float s = 0.f;
    if (r < a.N) {
#pragma unroll 4
        for (int c = warp; c < a.nchunk; c += 8) s += a.partials[(int64_t)c * a.N + r];
    }
    part[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && r < a.N) {
        float t = part[0][lane];
#pragma unroll
        for (int w = 1; w < 8; ++w) t += part[w][lane];
        if (a.y_bf16)
            reinterpret_cast<__nv_bfloat16*>(a.y)[r] = __float2bfloat16_rn(t);
        else
            reinterpret_cast<float*>(a.y)[r] = t;
    }
}

// ------------------------------------------------------------------ host ----

bool gemv_lut_applies(int64_t M, int64_t K, const void* scales) {
    // tensor maps need 16-byte aligned bases (codes already are) and row pitches
    return M == 1 && K > 0 && K % kBlock == 0 && (reinterpret_cast<uintptr_t>(scales) & 15) == 0;
}

size_t gemv_lut_workspace_bytes(int64_t N, int64_t K) {
    return (size_t)(K / kLutChunk) * (size_t)N * sizeof(float);
}

template <int LAYOUT, bool CHECK>
static cudaError_t launch_lut_main(const CUtensorMap& cmap, const CUtensorMap& smap, const LutArgs& la, int grid,
                                   cudaStream_t stream) {
    auto kern = gemv_lut_kernel<LAYOUT, CHECK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kLutThreads);
    cfg.dynamicSmemBytes = kLutSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, cmap, smap, la);
}

cudaError_t launch_gemv_lut(int layout, const uint8_t* codes, const uint16_t* scales, const void* x, int x_dtype,
                            const int8_t* sign, int64_t N, int64_t K, int y_dtype, void* y, void* workspace,
                            int32_t* dev_err, int num_sms, cudaStream_t stream) {
    if (N <= 0) return cudaSuccess;
    LutArgs la{};
    la.codes = codes;
    la.scales = scales;
    la.x = x;
    la.sign = sign;
    la.partials = static_cast<float*>(workspace);
    la.dev_err = dev_err;
    la.N = N;
    la.K = static_cast<int>(K);
    la.G = static_cast<int>(K / kGroup);
    la.RB = static_cast<int>(la.G * (layout == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes));
    la.nchunk = static_cast<int>(K / kLutChunk);
    la.x_bf16 = x_dtype == BT_BF16;
    // one chunk per CTA, rows split into `parts` slices; more chunks than
    // SMs: a CTA per SM walks chunks with all rows
    int64_t grid;
    if (la.nchunk <= num_sms) {
        int64_t parts = num_sms / la.nchunk;
        const int64_t max_parts = (N + kLutMinRows - 1) / kLutMinRows;
        if (parts > max_parts) parts = max_parts;
        if (parts < 1) parts = 1;
        la.rows_per_part = ((N + parts - 1) / parts + kLutSet - 1) / kLutSet * kLutSet;
        la.parts = (int)((N + la.rows_per_part - 1) / la.rows_per_part);
        if (la.parts < 1) la.parts = 1;
        grid = (int64_t)la.nchunk * la.parts;  // parts == 1: CTA c takes chunk c
    } else {
        la.parts = 1;
        la.rows_per_part = N;
        grid = num_sms;
    }

    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap cmap, smap;
    const cuuint64_t cdim[2] = {static_cast<cuuint64_t>(la.RB), static_cast<cuuint64_t>(N)};
    const cuuint64_t cstr[1] = {static_cast<cuuint64_t>(la.RB)};
    const cuuint32_t cbox[2] = {static_cast<cuuint32_t>(layout == BT_LAYOUT_B3 ? kLutCBoxB3 : kLutCBox2b), kLutSet};
    const cuuint64_t sdim[2] = {static_cast<cuuint64_t>(la.G), static_cast<cuuint64_t>(N)};
    const cuuint64_t sstr[1] = {static_cast<cuuint64_t>(la.G) * 2};
    const cuuint32_t sbox[2] = {8, kLutSet};
    const cuuint32_t one[2] = {1, 1};
    if (enc(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), cdim, cstr, cbox, one,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        enc(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(scales), sdim, sstr, sbox, one,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    cudaError_t e;
    if (layout == BT_LAYOUT_B3)
        e = dev_err ? launch_lut_main<BT_LAYOUT_B3, true>(cmap, smap, la, (int)grid, stream)
                    : launch_lut_main<BT_LAYOUT_B3, false>(cmap, smap, la, (int)grid, stream);
    else
        e = dev_err ? launch_lut_main<BT_LAYOUT_2BIT, true>(cmap, smap, la, (int)grid, stream)
                    : launch_lut_main<BT_LAYOUT_2BIT, false>(cmap, smap, la, (int)grid, stream);
    if (e != cudaSuccess) return e;

    LutReduceArgs ra{};
    ra.partials = la.partials;
    ra.y = y;
    ra.N = N;
    ra.nchunk = la.nchunk;
    ra.y_bf16 = y_dtype == BT_BF16;
    cudaLaunchConfig_t cfg{};
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)((N + 31) / 32));
    cfg.blockDim = dim3(256);
    return cudaLaunchKernelEx(&cfg, gemv_lut_reduce_kernel, ra);
}

}  // namespace bt

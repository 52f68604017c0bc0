// Prefill GEMM on the tcgen05 tensor cores: Y = X' W^T, M % 128 == 0.
//
// pp512 prompt processing (release summary of Ternary Bonsai 2 27B, section
// 实测吞吐) is a dense contraction, so it runs on the 5th-generation tensor
// cores with the packed weights decoded to FP16 tiles in shared memory and
// never materialised in HBM (section 三值权重怎么压缩到 1.76 bit: unpack and
// group scale fused inside the matrix product).
//
// Two kernels:
//
//  1. gemm_prep (one CTA per activation row): rotates the row block-wise
//     (x' = H_1024 S x / 32, when a sign vector is given), picks a power of
//     two 2^e_m from the row's largest |x'|, and writes x' * 2^-e_m as FP16 in
//     the per-group slot order the weight decoder produces (below), plus
//     2^e_m.
//
//  2. gemm: one 128 x BN output tile per CTA, one 128-wide K group per
//     pipeline stage; a 2-stage ring of activation tiles (TMA) and a
//     3-stage ring of decoded weight tiles (2 at BN = 256; the CTA-pair
//     form below holds 3 and 3-4).
//       warp 0      TMA: the activation tile (two 64-column panels, 128-byte
//                   swizzle) into shared memory;
//       warp 1      allocates TMEM, one elected thread issues
//                   tcgen05.mma.cta_group::1.kind::f16 (M 128, N BN, K 16) x 8
//                   per stage into an FP32 accumulator in TMEM and commits
//                   each stage to its "empty" barrier;
//       warps 2..   decode the packed weights of the stage to FP16 s*t --
//                   exact -- and store them in the tensor cores' K-major
//                   128-byte-swizzled layout: BT_GEMM_TPR (4) threads per
//                   weight row, each one 128 / TPR-slot part of the group
//                   (BN TPR / 32 warps); then all of them read the
//                   accumulator back (tcgen05.ld) and write bf16 Y scaled by
//                   2^e_m (or, with K split, FP32 partials first).
//     A group's 128 trits are laid out in "slot" order: slot 2w + h holds
//     half h of decoded word w. For base-3, word w < 60 is digit w % 5 of
//     bytes (2p, 2p+1), p = w / 5; words 60-62 are digits 0-2 of bytes
//     (24, 25); word 63 is digits 3 and 4 of byte 24 (byte 25's digits 3
//     and 4 are the group's two pad trits). For 2-bit, word 8q + f is trits
//     f and 8 + f of the group's 32-bit word q. The activations are written
//     in the same order, so the contraction over each group is unchanged.
//     Decoding a word: OR the two digits' 2-bit fields into FP16 1024 + d 4^i
//     (exact), one HFMA2 makes it d - 1 = t (exact), one HMUL2 makes s t.
//
//     With M % 256 == 0 the tiles run as CTA pairs (clusters of two along
//     M): both CTAs decode half of a BN-row weight tile each, and the pair
//     leader issues tcgen05.mma.cta_group::2 (M 256) over both CTAs' shared
//     memory, so each decoded weight row serves 256 activation rows. With
//     M % 512 == 0 a pair can take two 256-row activation tiles (512 rows
//     per decoded weight row), and where that leaves too few CTAs the K
//     groups are split in two between two pairs of one cluster of four CTAs,
//     which swap halves through distributed shared memory at the end. Small
//     grids of single CTAs split K 2-4 ways through FP32 partials in the
//     workspace instead (the tile forms and their measurements are listed
//     above pick_tile).
// Base-3 digits are computed per byte pair (b3_pair_fields) rather than read
// from a table, which leaves shared memory for one more weight stage.
// Waits on barriers are bounded: a wait that runs out sets BT_DEVERR_TIMEOUT,
// the CTA skips the rest of its work and still releases its TMEM.
#include "bt_internal.cuh"

namespace bt {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;             // one weight group per stage
// decoder warps: TPR threads per weight row of the BN-row tile, each decoding
// 128 / TPR of a group's slots
#ifndef BT_GEMM_TPR
#define BT_GEMM_TPR 4
#endif
constexpr int kGemmTpr = BT_GEMM_TPR;
__host__ __device__ constexpr int gemm_dec_warps(int bn) { return bn * kGemmTpr / 32; }
__host__ __device__ constexpr int gemm_threads(int bn) { return (2 + gemm_dec_warps(bn)) * 32; }
// -DBT_GEMM_B3_LUT: base-3 digits from a decode table in shared memory
// instead of b3_pair_fields' arithmetic. Per code, one 32-bit word per lane
// (each lane reads only its own bank, so lookups never conflict) holding the
// code's five base-3 digits as 2-bit fields plus the FP16 exponent bits of
// 1024 (0x6400) in both halves; bit 31 marks codes 243-255. The 32 KB it
// takes cost a weight stage.
#ifdef BT_GEMM_B3_LUT
constexpr int kGemmLutRow = 32 * 4;                       // bytes per code
constexpr int kGemmLutBytes = 256 * kGemmLutRow;
#endif

// ---------------------------------------------------------------- helpers ----

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms
// 1024 bytes apart (SBO), version 1 (Blackwell).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;              // leading byte offset (unused for this layout) = 16 B
    d |= static_cast<uint64_t>(1024u >> 4) << 32;      // stride byte offset
    d |= static_cast<uint64_t>(1u) << 46;              // descriptor version
    d |= static_cast<uint64_t>(2u) << 61;              // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: FP16 A and B (both K-major), FP32 D.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
    return (1u << 4)                                   // D format F32
         | (0u << 7) | (0u << 10)                      // A, B format F16
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void gemm_cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void gemm_cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// NC accumulator columns of one row scaled by rs, rounded to bf16 and stored
template <int NC>
__device__ __forceinline__ void epi_store(const uint32_t (&r)[NC], float rs, __nv_bfloat16* dst) {
    uint32_t packed[NC / 2];
#pragma unroll
    for (int j = 0; j < NC / 2; ++j) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[2 * j]) * rs,
                                                        __uint_as_float(r[2 * j + 1]) * rs);
        packed[j] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    uint4* out = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int v = 0; v < NC / 8; ++v)
        out[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// ---- CTA pair (cta_group::2) helpers
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// all threads of both CTAs; hardware barrier (the pair is co-scheduled)
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory whose bytes complete on the pair
// leader's barrier (the peer bit of the barrier address cleared)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar & 0xFEFFFFFFu) : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// arrive once on the barrier at this offset in both CTAs of the pair when the
// pair's MMAs issued so far complete
// commit to the barrier at this offset in both CTAs of the pair (cluster
// ranks `pair_base` and pair_base + 1)
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint32_t pair_base) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 :: "r"(bar), "h"((uint16_t)(3u << pair_base)) : "memory");
}
// this CTA's shared-memory address `a` as seen from the cluster, in CTA `rank`
__device__ __forceinline__ uint32_t cluster_map(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}
// arrive on the barrier at this offset in CTA `rank` of the cluster
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar, uint32_t rank) {
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}"
        :: "r"(bar), "r"(rank) : "memory");
}
// bounded wait with cluster-scope acquire (arrivals may come from the peer)
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity) {
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
        if (ok) return true;
    }
    return false;
}

__host__ __device__ constexpr uint32_t gfmask(int i) { return (3u << (2 * i)) | (3u << (2 * i + 16)); }

// FP16 constants turning (1024 + d 4^i) into d - 1: multiply by 4^-i, add
// -(1024 4^-i + 1); both are exact in FP16 for i <= 5.
__device__ __forceinline__ uint32_t h2_mul_of(int i) {
    const uint32_t h = __half_as_ushort(__float2half_rn(ldexpf(1.f, -2 * i)));
    return h | (h << 16);
}
__device__ __forceinline__ uint32_t h2_add_of(int i) {
    const uint32_t h = __half_as_ushort(__float2half_rn(-(ldexpf(1024.f, -2 * i) + 1.f)));
    return h | (h << 16);
}

// Words per decoder thread and packed words it reads, per layout.
template <int LAYOUT>
struct GemmPart {
    static constexpr int WPT = 64 / kGemmTpr;
    static constexpr int NW = LAYOUT == BT_LAYOUT_B3 ? (kGemmTpr == 2 ? 7 : 4) : WPT / 8;
};

// Base-3 digits of a byte pair, computed: bytes 2p (low half) and 2p + 1
// (high half) of pr become the 2-bit digit fields of both codes with the FP16
// exponent bits of 1024 in each half. floor(c / 3) = (171 c) >> 9 for
// c < 256, and one 32-bit multiply serves both halves (171 c < 2^16, and the
// mask drops what the high half shifts down). Codes 243-255 set bit 8 or 24
// of err.
__device__ __forceinline__ uint32_t b3_pair_fields(uint32_t pr, uint32_t& err) {
    uint32_t x = prmt(pr, 0u, 0x4140u);                  // [byte 2p, 0, byte 2p+1, 0]
    err |= (x + 0x000D000Du) & 0x01000100u;
    uint32_t f = 0x64006400u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t q = ((x * 171u) >> 9) & 0x007F007Fu;
        f |= (x - 3u * q) << (2 * i);
        x = q;
    }
    return f | (x << 8);
}

// Decode part QQ of one group (WPT words of FP16 pairs s t, slot order) from
// the part's packed words. Base-3 word w < 60 is digit w % 5 of byte pair
// w / 5; words 60-62 are digits 0-2 of pair 12, word 63 digits 3-4 of byte
// 24. 2-bit: word 8 q + f holds fields f and 8 + f of the group's 32-bit
// word q.
template <int LAYOUT, int QQ>
__device__ __forceinline__ void gemm_decode_part(const uint32_t (&cw)[GemmPart<LAYOUT>::NW], uint32_t s2,
                                                 uint32_t (&words)[GemmPart<LAYOUT>::WPT], const uint8_t* lut_lane,
                                                 const uint32_t (&hm)[6], const uint32_t (&ha)[6], uint32_t hm34,
                                                 uint32_t ha34, uint32_t& err) {
    constexpr int WPT = GemmPart<LAYOUT>::WPT, NW = GemmPart<LAYOUT>::NW;
    constexpr int W0 = WPT * QQ, W1 = W0 + WPT, P0 = W0 / 5;
    if constexpr (LAYOUT == BT_LAYOUT_B3) {
#pragma unroll
        for (int j = 0; j < NW; ++j) {
            const int p = P0 + j;
            if (p > 12) continue;
            const uint32_t pr = cw[j];
#ifdef BT_GEMM_B3_LUT
            const uint32_t va = *reinterpret_cast<const uint32_t*>(lut_lane + (pr & 0xFFu) * kGemmLutRow);
            const uint32_t vb = *reinterpret_cast<const uint32_t*>(lut_lane + (pr >> 8) * kGemmLutRow);
            err |= (va | vb) & 0x80000000u;
            const uint32_t x = prmt(va, vb, 0x7610u);   // byte 2p's fields low, byte 2p+1's high
#else
            (void)lut_lane;
            const uint32_t x = b3_pair_fields(pr, err);
            const uint32_t va = x;                      // byte 2p's fields in the low half
#endif
            const int nw = p < 12 ? 5 : 3;
#pragma unroll
            for (int i = 0; i < nw; ++i) {
                const int w = 5 * p + i;
                if (w >= W0 && w < W1) {
                    const uint32_t f = x & (gfmask(i) | 0x64006400u);
                    words[w - W0] = hmul2_u32(hfma2_u32(f, hm[i], ha[i]), s2);
                }
            }
            if (p == 12 && W1 == 64) {
                const uint32_t f = (va & 0x64C0u) | ((va & 0x300u) << 16) | 0x64000000u;
                words[63 - W0] = hmul2_u32(hfma2_u32(f, hm34, ha34), s2);
            }
        }
    } else {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            // fields 0-4 of each half in place, fields 5-7 after a 10-bit
            // shift: a field at bits 10-11 would reach into the FP16
            // exponent of 1024 + d 4^i
            const uint32_t x = cw[w], x10 = x >> 10;
            err |= x & (x >> 1) & 0x55555555u;
#pragma unroll
            for (int f = 0; f < 8; ++f) {
                const uint32_t fl = (f < 5 ? (x & gfmask(f)) : (x10 & gfmask(f - 5))) | 0x64006400u;
                const int i = f < 5 ? f : f - 5;
                words[8 * w + f] = hmul2_u32(hfma2_u32(fl, hm[i], ha[i]), s2);
            }
        }
    }
}

// ------------------------------------------------------------------ prep ----

struct GemmPrepArgs {
    const void* x;
    int x_bf16;
    const int8_t* sign;   // nullable: x already rotated
    int M, K, G;
    int layout;
    __half* xt;           // [M][K] FP16, slot order within each group
    float* rowscale;      // [M] 2^e_m
    int32_t* tile_cnt;    // nullable: split-K arrival counters, zeroed here
    int n_cnt;
};

__device__ __forceinline__ int gemm_slot_k(int layout, int slot) {
    const int w = slot >> 1, h = slot & 1;
    if (layout == BT_LAYOUT_B3) {
        if (w < 60) return 10 * (w / 5) + 5 * h + (w % 5);
        if (w < 63) return 120 + 5 * h + (w - 60);
        return 123 + h;
    }
    return 16 * (w >> 3) + 8 * h + (w & 7);
}

constexpr int kGemmPrepWarps = 8;

__global__ void __launch_bounds__(kGemmPrepWarps * 32) gemm_prep_kernel(GemmPrepArgs a) {
    extern __shared__ __align__(16) float rowbuf[];   // K floats, then tiles
    float* tiles = rowbuf + a.K;                        // kGemmPrepWarps x 32 x 36
    __shared__ float red[kGemmPrepWarps];
    pdl_launch_dependents();
    pdl_wait();
    // the preceding GEMM of the stream is complete here, and the GEMM that
    // follows reads the counters only after this kernel has finished
    if (a.tile_cnt && blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.n_cnt; i += blockDim.x) a.tile_cnt[i] = 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m = blockIdx.x;
    const int nblocks = (a.K + kBlock - 1) / kBlock;
    float amax = 0.f;
    if (a.sign) {
        // bf16 blocks with S: the next block's raw words are loaded while the
        // current one is rotated, so the row's loads overlap
        const uint16_t* xrow = reinterpret_cast<const uint16_t*>(a.x) + (int64_t)m * a.K;
        const uint4* sg = reinterpret_cast<const uint4*>(a.sign + 32 * lane);
        const uint4 s0 = __ldg(sg), s1 = __ldg(sg + 1);
        const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        uint4 nxt[4];
        int b = warp;
        if (b < nblocks) {
            const uint4* src = reinterpret_cast<const uint4*>(xrow + (int64_t)b * kBlock + 32 * lane);
#pragma unroll
            for (int q = 0; q < 4; ++q) nxt[q] = __ldg(src + q);
        }
        for (; b < nblocks; b += kGemmPrepWarps) {
            uint4 cur[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
            if (b + kGemmPrepWarps < nblocks) {
                const uint4* src =
                    reinterpret_cast<const uint4*>(xrow + (int64_t)(b + kGemmPrepWarps) * kBlock + 32 * lane);
#pragma unroll
                for (int q = 0; q < 4; ++q) nxt[q] = __ldg(src + q);
            }
            float v[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t ww[4] = {cur[q].x, cur[q].y, cur[q].z, cur[q].w};
#pragma unroll
                for (int h = 0; h < 4; ++h)
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int i = 8 * q + 2 * h + half;
                        const uint32_t bits = half ? (ww[h] & 0xFFFF0000u) : (ww[h] << 16);
                        const uint32_t sbyte = (sw[i >> 2] >> (8 * (i & 3))) & 0x80u;  // bit 7: negative
                        v[i] = __uint_as_float(bits ^ (sbyte << 24));
                    }
            }
            fwht1024_warp(v, tiles + warp * 32 * kTileStride);
            const int64_t k0 = (int64_t)b * kBlock;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                rowbuf[k0 + 32 * j + lane] = v[j];
                amax = fmaxf(amax, fabsf(v[j]));
            }
        }
    } else {
        for (int b = warp; b < nblocks; b += kGemmPrepWarps) {
            const int64_t k0 = (int64_t)b * kBlock;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int64_t idx = k0 + 32 * j + lane;
                if (idx < a.K) {
                    const int64_t off = (int64_t)m * a.K + idx;
                    const float val = a.x_bf16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(a.x)[off])
                                               : reinterpret_cast<const float*>(a.x)[off];
                    rowbuf[idx] = val;
                    amax = fmaxf(amax, fabsf(val));
                }
            }
        }
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = 0.f;
    for (int w = 0; w < kGemmPrepWarps; ++w) amax = fmaxf(amax, red[w]);
    // 2^e with max |x'| 2^-e < 2^15 keeps FP16 finite with margin
    int e = amax > 0.f ? ilogbf(amax) + 1 - 15 : 0;
    e = max(-110, min(110, e));
    const float inv = __int_as_float((127 - e) << 23);
    if (threadIdx.x == 0) a.rowscale[m] = __int_as_float((127 + e) << 23);
    // eight consecutive slots per thread, one 16-byte store (K % 128 == 0)
    uint4* dst = reinterpret_cast<uint4*>(a.xt + (int64_t)m * a.K);
    for (int o = threadIdx.x; o < a.K / 8; o += blockDim.x) {
        const int idx = 8 * o, g = idx >> 7, slot0 = idx & 127;
        uint32_t w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __half lo = __float2half_rn(rowbuf[g * kGroup + gemm_slot_k(a.layout, slot0 + 2 * u)] * inv);
            const __half hi = __float2half_rn(rowbuf[g * kGroup + gemm_slot_k(a.layout, slot0 + 2 * u + 1)] * inv);
            w4[u] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
        }
        dst[o] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
}

// ------------------------------------------------------------------ GEMM ----

struct GemmArgs {
    const uint8_t* codes;
    const uint16_t* scales;
    const float* rowscale;
    __nv_bfloat16* y;
    int M, N, K, G;
    int64_t row_bytes;
    int32_t* dev_err;
    float* part;          // split-K: [2][M][N] FP32 partial products
    int32_t* tile_cnt;    // split-K: [tiles][decoder warps] arrivals
};

#ifndef BT_GEMM_ASTAGES
#define BT_GEMM_ASTAGES 2
#endif
#ifndef BT_GEMM_BSTAGES
#define BT_GEMM_BSTAGES 3
#endif

template <int LAYOUT, int BN, int STAGES, int ASTAGES = BT_GEMM_ASTAGES, int MT = 1>
struct GemmSmem {
    // activation ring (TMA; MT tiles of 128 rows per stage) and ring of
    // decoded weight tiles (BN rows each)
    static constexpr int kAStages = ASTAGES;
    static constexpr int kBStages = STAGES;
    static constexpr int kA1 = kGemmBM * kGemmBK * 2;  // 32 KB per 128-row tile: two 64-column panels
    static constexpr int kA = MT * kA1;
    static constexpr int kB = BN * kGemmBK * 2;
#ifdef BT_GEMM_B3_LUT
    static constexpr int kLut = LAYOUT == BT_LAYOUT_B3 ? kGemmLutBytes : 0;
#else
    static constexpr int kLut = 0;                      // base-3 digits are computed
#endif
    static constexpr int kBars = 1024;                  // barriers, TMEM address, flags
    static constexpr int kTotal = kAStages * kA + kBStages * kB + kLut + kBars + 1024;  // + alignment slack
};

// PAIR: the two CTAs of a cluster (M tiles 2j, 2j + 1) share one BN-column
// weight tile. Each decodes half of its rows (BL = BN / 2) into its own
// shared memory; the leader (rank 0) issues tcgen05.mma.cta_group::2 with
// M = 256, which reads A and B from both CTAs and accumulates each CTA's 128
// rows x BN columns in that CTA's TMEM. Activation copies complete on the
// leader's barrier; the peer's decoders arrive on their own barrier, which
// one relay thread forwards to the leader's; each commit arrives on the
// barrier pair in both CTAs.
//
// MT = 2 (pairs only): the pair takes two 256-row activation tiles against the
// same weight tile, so each decoded weight row serves 512 activation rows; the
// two accumulators sit side by side in TMEM (columns 0 .. BN - 1 and
// BN .. 2 BN - 1) and every stage issues the MMAs of both.
//
// SPLIT (split K): blockIdx.z takes 1 / gridDim.z of the K groups. Each
// epilogue warp stores its chunks' FP32 partial products, then counts itself
// in on its tile; the warp that arrives last adds the partials in split
// order, scales and writes the bf16 rows. Nobody waits for anybody.
template <int LAYOUT, int BN, int STAGES, int ASTAGES = BT_GEMM_ASTAGES, bool PAIR = false, int MT = 1,
          bool SPLIT = false>
__global__ void __launch_bounds__(gemm_threads(PAIR ? BN / 2 : BN), 1)
gemm_kernel(const __grid_constant__ CUtensorMap amap, GemmArgs a) {
    static_assert(MT == 1 || PAIR, "several activation tiles per CTA only in pairs");
    static_assert(!SPLIT || BN % 32 == 0, "K splits");
    static_assert(BN % 16 == 0 && (PAIR ? BN / 2 : BN) % 8 == 0, "tile width");
    constexpr int BL = PAIR ? BN / 2 : BN;             // weight rows decoded by this CTA
    using SM = GemmSmem<LAYOUT, BL, STAGES, ASTAGES, MT>;
    constexpr uint32_t kTmemCols = MT * BN <= 128 ? 128 : (MT * BN <= 256 ? 256 : 512);
    extern __shared__ uint8_t gsm_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~uintptr_t(1023));
    constexpr int SA = SM::kAStages, SB = SM::kBStages;
    uint8_t* a_ring = base;
    uint8_t* b_ring = base + SA * SM::kA;
    uint8_t* lut = b_ring + SB * SM::kB;
    uint8_t* ctl = lut + SM::kLut;
    uint64_t* fullA = reinterpret_cast<uint64_t*>(ctl);
    uint64_t* emptyA = fullA + SA;
    uint64_t* fullB = emptyA + SA;
    uint64_t* emptyB = fullB + SB;
    uint64_t* accf = emptyB + SB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a CTA pair sits along x, so that its two CTAs take the two halves of a
    // 256-row activation tile against the same weight tile
    // a pair's CTA of rank r holds rows r * 128 .. r * 128 + 127 of each of its
    // MT 256-row activation tiles; m0 is its first tile's
    const int m0 = PAIR ? ((int)(blockIdx.x >> 1) * MT * 2 + (int)(blockIdx.x & 1)) * kGemmBM
                        : (int)blockIdx.y * kGemmBM;
    const int n0 = (PAIR ? blockIdx.y : blockIdx.x) * BN;
    // K groups [kbase, kbase + ktiles) of this CTA
    const int ks = SPLIT ? (int)gridDim.z : 1;
    const int kbase = SPLIT ? (int)blockIdx.z * a.G / ks : 0;
    const int ktiles = SPLIT ? ((int)blockIdx.z + 1) * a.G / ks - kbase : a.G;
    // cluster ranks: pairs are (0, 1) and, when the two K halves of a split
    // share the cluster, (2, 3); the even rank of a pair leads
    const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
    const uint32_t rank = crank & 1u, pair_base = crank & ~1u;
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(smem_addr(fullA + s), 1);
            mbar_init(smem_addr(emptyA + s), 1);
        }
        for (int s = 0; s < SB; ++s) {
            // a pair leader also counts the one arrival relayed from the peer
            mbar_init(smem_addr(fullB + s), gemm_dec_warps(BL) + (PAIR && leader ? 1 : 0));
            mbar_init(smem_addr(emptyB + s), 1);
        }
        mbar_init(smem_addr(accf), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
#ifdef BT_GEMM_B3_LUT
    if (LAYOUT == BT_LAYOUT_B3) {
        // digits of each code as 2-bit fields with the FP16 exponent bits of
        // 1024 (0x6400), in both halves, so that field i masked out of a half
        // reads 1024 + d 4^i; one word per lane
        for (int idx = threadIdx.x; idx < 256 * 32; idx += blockDim.x) {
            const int code = idx >> 5;
            uint32_t f = 0x6400u;
            if (code < 243) {
                int r = code;
                for (int i = 0; i < 5; ++i) { f |= static_cast<uint32_t>(r % 3) << (2 * i); r /= 3; }
            }
            reinterpret_cast<uint32_t*>(lut)[idx] = f | (f << 16) | (code < 243 ? 0u : 0x80000000u);
        }
    }
#endif
    if (warp == 1) {
        if constexpr (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                         :: "r"(smem_addr(tmem_slot)), "r"(kTmemCols) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         :: "r"(smem_addr(tmem_slot)), "r"(kTmemCols) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();   // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the activations and row scales come from the prep kernel: the TMA and
    // MMA warps wait for it here, the decoders once their first weight loads
    // (never written by a kernel this one may overlap) are in flight
    if (warp < 2) pdl_wait();

    int bad = 0;
    if (warp == 0) {
        // ---------------- TMA producer: activation tiles
        if (lane == 0) {
            for (int kt = 0; kt < ktiles; ++kt) {
                const int s = kt % SA;
                if (kt >= SA && !mbar_wait(smem_addr(emptyA + s), ((kt / SA) - 1) & 1)) {
                    bad = BT_DEVERR_TIMEOUT; *abort_flag = 1; break;
                }
                if (*abort_flag) break;
                const uint32_t dst = smem_addr(a_ring + s * SM::kA);
                if constexpr (PAIR) {
                    // the leader's barrier counts both CTAs' activation bytes
                    if (leader) mbar_arrive_tx(smem_addr(fullA + s), 2 * SM::kA);
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint32_t dj = dst + j * SM::kA1;
                        const int mj = m0 + j * 2 * kGemmBM;
                        const int kx = (kbase + kt) * kGemmBK;
                        tma_load_2d_pair(dj, &amap, kx, mj, smem_addr(fullA + s));
                        tma_load_2d_pair(dj + SM::kA1 / 2, &amap, kx + 64, mj, smem_addr(fullA + s));
                    }
                } else {
                    mbar_arrive_tx(smem_addr(fullA + s), SM::kA);
                    tma_load_2d(dst, &amap, (kbase + kt) * kGemmBK, m0, smem_addr(fullA + s));
                    tma_load_2d(dst + SM::kA / 2, &amap, (kbase + kt) * kGemmBK + 64, m0, smem_addr(fullA + s));
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (the leader, for a pair)
        if (lane == 0 && leader) {
            constexpr uint32_t idesc = idesc_f16(PAIR ? 2 * kGemmBM : kGemmBM, BN);
            for (int kt = 0; kt < ktiles; ++kt) {
                const int s_a = kt % SA, s_b = kt % SB;
                const bool okb = PAIR ? mbar_wait_cluster(smem_addr(fullB + s_b), (kt / SB) & 1)
                                      : mbar_wait(smem_addr(fullB + s_b), (kt / SB) & 1);
                if (!mbar_wait(smem_addr(fullA + s_a), (kt / SA) & 1) || !okb) {
                    bad = BT_DEVERR_TIMEOUT; *abort_flag = 1; break;
                }
                if (*abort_flag) break;
                tc_fence_after();
                const uint32_t sa = smem_addr(a_ring + s_a * SM::kA);
                const uint32_t sb = smem_addr(b_ring + s_b * SM::kB);
#pragma unroll
                for (int k = 0; k < kGemmBK / 16; ++k) {
                    const uint32_t pb = sb + (k >> 2) * (SM::kB / 2) + (k & 3) * 32;
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint32_t pa = sa + j * SM::kA1 + (k >> 2) * (SM::kA1 / 2) + (k & 3) * 32;
                        if constexpr (PAIR)
                            tc_mma_pair(tmem + j * BN, smem_desc_sw128(pa), smem_desc_sw128(pb), idesc,
                                        (kt > 0 || k > 0) ? 1u : 0u);
                        else
                            tc_mma(tmem, smem_desc_sw128(pa), smem_desc_sw128(pb), idesc, (kt > 0 || k > 0) ? 1u : 0u);
                    }
                }
                if constexpr (PAIR) {
                    tc_commit_pair(smem_addr(emptyA + s_a), pair_base);
                    tc_commit_pair(smem_addr(emptyB + s_b), pair_base);
                } else {
                    tc_commit(smem_addr(emptyA + s_a));
                    tc_commit(smem_addr(emptyB + s_b));
                }
            }
            if constexpr (PAIR) tc_commit_pair(smem_addr(accf), pair_base);
            else tc_commit(smem_addr(accf));
        }
        if constexpr (PAIR) {
            // Relay (the peer's warp 1): once this CTA's decoders have filled
            // weight stage kt, one cluster-scope arrival tells the leader. The
            // decoders themselves arrive locally: a cluster-scope release in
            // their own code would wait for the code loads they keep in flight.
            if (lane == 0 && !leader) {
                for (int kt = 0; kt < ktiles; ++kt) {
                    const int s_b = kt % SB;
                    if (!mbar_wait(smem_addr(fullB + s_b), (kt / SB) & 1)) {
                        bad = BT_DEVERR_TIMEOUT; *abort_flag = 1; break;
                    }
                    if (*abort_flag) break;
                    mbar_arrive_cluster(smem_addr(fullB + s_b), pair_base);
                }
            }
        }
    } else {
        // ---------------- decoders: thread (part qq, row t) decodes the 128 /
        // TPR slots of weight row t with index 128 qq / TPR and up; they lie
        // in panel h (64-slot halves of the group)
        constexpr int WPT = GemmPart<LAYOUT>::WPT;      // 32-bit words per thread
        const int tt = threadIdx.x - 64;                // 0 .. TPR BL - 1
        const int qq = tt / BL, t = tt - qq * BL;
        const int h = qq * WPT / 32;                    // panel
        const int n = n0 + (int)rank * BL + t;
        const uint8_t* rowp = a.codes + (int64_t)n * a.row_bytes;
        const uint16_t* srow = a.scales + (int64_t)n * a.G;
        const uint8_t* lut_lane = lut + lane * 4;       // this lane's column (bank) of the table
        uint32_t hm[6], ha[6];
#pragma unroll
        for (int i = 0; i < 6; ++i) { hm[i] = h2_mul_of(i); ha[i] = h2_add_of(i); }
        const uint32_t hm34 = (hm[3] & 0xFFFFu) | (hm[4] & 0xFFFF0000u);
        const uint32_t ha34 = (ha[3] & 0xFFFFu) | (ha[4] & 0xFFFF0000u);
        uint32_t err = 0;
        // Base-3: word w < 60 is digit w % 5 of byte pair w / 5; words 60-63
        // come from pair 12. The words of part qq, [WPT qq, WPT qq + WPT), use
        // the pairs from WPT qq / 5 on: 7 pairs for TPR = 2, 4 for TPR = 4.
        // 2-bit: part qq is the group's 32-bit words WPT qq / 8 and on.
        constexpr int NW = GemmPart<LAYOUT>::NW;
        const int p_lo = (WPT * qq) / 5;
        auto load_group = [&](int kt, uint32_t (&dst)[NW], uint32_t& sc) {
            if (kt >= ktiles) return;
            kt += kbase;
            if constexpr (LAYOUT == BT_LAYOUT_B3) {
                // the 2 NW bytes from pair p_lo through the 8-byte aligned
                // window that holds them (alignment taken from the address:
                // rows are only 2-byte aligned when K % 512 != 0). A window
                // word is loaded only if it holds a needed byte, so no load
                // leaves the buffer's last aligned block.
                constexpr int NB = 2 * NW;                   // 14 or 8 bytes
                const uintptr_t sa = reinterpret_cast<uintptr_t>(rowp) + (uintptr_t)(kt * kB3GroupBytes + 2 * p_lo);
                const int sh = (int)(sa & 7);                // 0, 2, 4 or 6
                const uint2* wp = reinterpret_cast<const uint2*>(sa - (uintptr_t)sh);
                const uint2 x0 = __ldg(wp);
                const uint2 x1 = sh + NB > 8 ? __ldg(wp + 1) : make_uint2(0u, 0u);
                const uint2 x2 = sh + NB > 16 ? __ldg(wp + 2) : make_uint2(0u, 0u);
                const uint32_t w6[6] = {x0.x, x0.y, x1.x, x1.y, x2.x, x2.y};
                // 32-bit words at byte offsets sh, sh + 4, ...
                constexpr int NV = (NB + 3) / 4;
                uint32_t v[NV];
                const uint32_t bits = 8u * (uint32_t)(sh & 3);
                const bool up = sh >= 4;
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const uint32_t lo = up ? w6[i + 1] : w6[i];
                    const uint32_t hi = up ? w6[i + 2] : w6[i + 1];
                    v[i] = __funnelshift_r(lo, hi, bits);
                }
#pragma unroll
                for (int p = 0; p < NW; ++p) dst[p] = (p & 1) ? (v[p >> 1] >> 16) : (v[p >> 1] & 0xFFFFu);
            } else {
                const uint32_t* gp = reinterpret_cast<const uint32_t*>(rowp + (int64_t)kt * k2bGroupBytes) + NW * qq;
                if constexpr (NW == 4) {
                    const uint4 q = __ldg(reinterpret_cast<const uint4*>(gp));
                    dst[0] = q.x; dst[1] = q.y; dst[2] = q.z; dst[3] = q.w;
                } else {
                    const uint2 q = __ldg(reinterpret_cast<const uint2*>(gp));
                    dst[0] = q.x; dst[1] = q.y;
                }
            }
            sc = srow[kt];
        };
        // Stage kt decodes group kt from registers loaded two stages earlier:
        // the loop is unrolled by two over two named buffers, so no register
        // copy waits on a load in flight.
        auto stage = [&](int kt, const uint32_t (&cw)[NW], uint32_t scv) -> bool {
            const int s = kt % SB;
            if (kt >= SB && !mbar_wait(smem_addr(emptyB + s), ((kt / SB) - 1) & 1)) {
                bad = BT_DEVERR_TIMEOUT; *abort_flag = 1; return false;
            }
            if (*abort_flag) return false;
            {
                const uint32_t s1 = scv;
                const uint32_t s2 = s1 | (s1 << 16);
                uint8_t* bst = b_ring + s * SM::kB + h * (SM::kB / 2);
                // row t of panel h: 8-row atoms of 1024 bytes, 128 bytes per row
                const uint32_t row_off = static_cast<uint32_t>((t >> 3) * 1024 + (t & 7) * 128);
                uint32_t words[WPT];
                switch (qq) {
                    case 0: gemm_decode_part<LAYOUT, 0>(cw, s2, words, lut_lane, hm, ha, hm34, ha34, err); break;
                    case 1: gemm_decode_part<LAYOUT, 1>(cw, s2, words, lut_lane, hm, ha, hm34, ha34, err); break;
                    case 2: gemm_decode_part<LAYOUT, 2 % kGemmTpr>(cw, s2, words, lut_lane, hm, ha, hm34, ha34, err); break;
                    default: gemm_decode_part<LAYOUT, 3 % kGemmTpr>(cw, s2, words, lut_lane, hm, ha, hm34, ha34, err); break;
                }
                // 16-byte chunks of the panel row: chunk c0 + c, c0 = first chunk of this part
                const int c0 = (qq * WPT / 4) & 7;
#pragma unroll
                for (int c = 0; c < WPT / 4; ++c) {
                    uint8_t* dst = bst + row_off + (((c0 + c) ^ (t & 7)) << 4);
                    *reinterpret_cast<uint4*>(dst) =
                        make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_addr(fullB + s));
            }
            return true;
        };
        uint32_t bufA[NW], bufB[NW], sA = 0, sB = 0;
        load_group(0, bufA, sA);
        load_group(1, bufB, sB);
        pdl_wait();
        for (int kt = 0; kt < ktiles; kt += 2) {
            if (!stage(kt, bufA, sA)) break;
            load_group(kt + 2, bufA, sA);
            if (kt + 1 >= ktiles) break;
            if (!stage(kt + 1, bufB, sB)) break;
            load_group(kt + 3, bufB, sB);
        }
#ifdef BT_GEMM_B3_LUT
        if (LAYOUT == BT_LAYOUT_B3 ? (err >> 31) : (err != 0)) bad |= BT_DEVERR_INVALID_CODE;
#else
        if (err != 0) bad |= BT_DEVERR_INVALID_CODE;
#endif

        // ---------------- epilogue: TMEM -> bf16 Y. Every decoder warp takes
        // part: warp w reads TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31, i.e. rows
        // m0 + 256 j + 32 (w % 4) + lane, and the warps of one lane quarter
        // share its MT x NCH column chunks of 32 (16 for the last one when
        // BN % 32 == 16) round-robin
        if (!*abort_flag && !mbar_wait(smem_addr(accf), 0)) { bad |= BT_DEVERR_TIMEOUT; *abort_flag = 1; }
        tc_fence_after();
        constexpr int NDW = gemm_dec_warps(BL);
        static_assert(NDW >= 4, "a decoder warp for every TMEM lane quarter");
        constexpr int NCH = (BN + 31) / 32;
        const int quarter = warp & 3;
        const int w0 = 2 + ((quarter + 2) & 3);        // this quarter's first decoder warp
        const int slot = (warp - w0) >> 2;
        const int nslot = (NDW + 1 - w0) / 4 + 1;
        const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        // the decision is the whole warp's: TMEM loads and shuffles are warp-collective
        const bool do_epi = __all_sync(0xffffffffu, !*abort_flag);
        if constexpr (!SPLIT) {
#pragma unroll 1
            for (int u = slot; u < MT * NCH && do_epi; u += nslot) {
                const int j = u / NCH, c0 = (u - j * NCH) * 32;
                const int m = m0 + j * 2 * kGemmBM + quarter * 32 + lane;
                const float rs = a.rowscale[m];
                __nv_bfloat16* yrow = a.y + (int64_t)m * a.N + n0 + c0;
                if (BN % 32 == 16 && c0 + 32 > BN) {
                    uint32_t r[16];
                    tmem_ld16(tq + j * BN + c0, r);
                    epi_store<16>(r, rs, yrow);
                } else {
                    uint32_t r[32];
                    tmem_ld32(tq + j * BN + c0, r);
                    epi_store<32>(r, rs, yrow);
                }
            }
        } else if (PAIR) {
            // the pair's two K halves meet through the cluster, after the role branches
        } else if (do_epi) {
            // split K: store this split's FP32 partial products, count in; the
            // warp arriving last (the ks-th, for this warp's chunks of this
            // tile) adds the ks partials in split order, so the bits do not
            // depend on who finishes when. Partials move through a per-warp
            // 32 x 33 shared-memory transpose (the drained activation ring), so
            // that each global access of the warp covers four whole 128-byte
            // rows of a chunk instead of 16 bytes of 32 rows.
            static_assert(!SPLIT || NDW * 32 * 33 * 4 <= SA * SM::kA + SB * SM::kB, "transpose buffers");
            const size_t plane = (size_t)a.M * a.N;
            const int z = (int)blockIdx.z;
            float* tb = reinterpret_cast<float*>(a_ring) + (warp - 2) * (32 * 33);
            const int prow = lane >> 3, pcol = (lane & 7) * 4;   // coalesced role: rows 4 i + prow
#pragma unroll 1
            for (int u = slot; u < MT * NCH; u += nslot) {
                const int j = u / NCH, c0 = (u - j * NCH) * 32;
                float* base = a.part + z * plane + (int64_t)(m0 + j * 2 * kGemmBM + quarter * 32) * a.N + n0 + c0;
                uint32_t r[32];
                tmem_ld32(tq + j * BN + c0, r);
#pragma unroll
                for (int c = 0; c < 32; ++c) tb[lane * 33 + c] = __uint_as_float(r[c]);
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float* t = tb + (4 * i + prow) * 33 + pcol;
                    *reinterpret_cast<float4*>(base + (int64_t)(4 * i + prow) * a.N + pcol) =
                        make_float4(t[0], t[1], t[2], t[3]);
                }
                __syncwarp();
            }
            __threadfence();
            __syncwarp();
            int arrived = 0;
            if (lane == 0)
                arrived = atomicAdd(a.tile_cnt + ((int)blockIdx.y * (int)gridDim.x + (int)blockIdx.x) * NDW + (warp - 2), 1);
            arrived = __shfl_sync(0xffffffffu, arrived, 0);
            if (arrived == ks - 1) {
                __threadfence();   // the other splits' stores, made visible by their fences, are seen
                // The other splits' 32 x 32 chunks land in this warp's slots of the
                // drained rings by cp.async, a batch of whole units at a time, so
                // that a batch costs one round trip to L2. A slot is [32 rows][32 f32]
                // with row r's 16-byte pieces rotated by r % 8, so that the row-per-
                // lane reads below do not conflict.
                constexpr int kRingBytes = SA * SM::kA + SB * SM::kB;
                constexpr int kTbBytes = NDW * 32 * 33 * 4;
                constexpr int kSlots = (kRingBytes - kTbBytes) / NDW / 4096;
                const int per = ks - 1;
                const int upb = per <= kSlots ? kSlots / per : 0;   // units per batch
                const uint32_t land = smem_addr(a_ring) + kTbBytes + (warp - 2) * kSlots * 4096;
                const float* land_f = reinterpret_cast<const float*>(a_ring + kTbBytes + (warp - 2) * kSlots * 4096);
#pragma unroll 1
                for (int ub = slot; ub < MT * NCH; ub += (upb > 0 ? upb : 1) * nslot) {
                    if (upb > 0) {
                        int t = 0;
#pragma unroll 1
                        for (int u = ub; u < MT * NCH && t < upb; u += nslot, ++t) {
                            const int j = u / NCH, c0 = (u - j * NCH) * 32;
                            const int64_t off = (int64_t)(m0 + j * 2 * kGemmBM + quarter * 32) * a.N + n0 + c0;
                            int pz = 0;
#pragma unroll 1
                            for (int zz = 0; zz < ks; ++zz) {
                                if (zz == z) continue;
                                const float* src = a.part + zz * plane + off;
                                const uint32_t dst = land + (t * per + pz) * 4096;
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const int row = 4 * i + prow;
                                    gemm_cp_async16(dst + row * 128 + ((((pcol >> 2) ^ (row & 7))) << 4),
                                                    src + (int64_t)row * a.N + pcol);
                                }
                                ++pz;
                            }
                        }
                        gemm_cp_async_wait_all();
                        __syncwarp();
                    }
                    int t = 0;
#pragma unroll 1
                    for (int u = ub; u < MT * NCH && t < (upb > 0 ? upb : 1); u += nslot, ++t) {
                        const int j = u / NCH, c0 = (u - j * NCH) * 32;
                        const int mb = m0 + j * 2 * kGemmBM + quarter * 32;
                        const int64_t off = (int64_t)mb * a.N + n0 + c0;
                        float acc[32];
                        int pz = 0;
#pragma unroll 1
                        for (int zz = 0; zz < ks; ++zz) {
                            if (zz == z) {   // warp-uniform
                                uint32_t r[32];
                                tmem_ld32(tq + j * BN + c0, r);
#pragma unroll
                                for (int c = 0; c < 32; ++c)
                                    acc[c] = zz == 0 ? __uint_as_float(r[c]) : acc[c] + __uint_as_float(r[c]);
                            } else if (upb > 0) {
                                const float4* rowp = reinterpret_cast<const float4*>(land_f + (t * per + pz) * 1024 + lane * 32);
#pragma unroll
                                for (int c4 = 0; c4 < 8; ++c4) {
                                    const float4 v = rowp[c4 ^ (lane & 7)];
                                    acc[4 * c4] = zz == 0 ? v.x : acc[4 * c4] + v.x;
                                    acc[4 * c4 + 1] = zz == 0 ? v.y : acc[4 * c4 + 1] + v.y;
                                    acc[4 * c4 + 2] = zz == 0 ? v.z : acc[4 * c4 + 2] + v.z;
                                    acc[4 * c4 + 3] = zz == 0 ? v.w : acc[4 * c4 + 3] + v.w;
                                }
                                ++pz;
                            } else {
                                // no room for a unit's pieces: through the transpose
                                // buffer, one partial chunk at a time
                                const float* src = a.part + zz * plane + off;
#pragma unroll
                                for (int i0 = 0; i0 < 8; i0 += 4) {
                                    float4 q[4];
#pragma unroll
                                    for (int i = 0; i < 4; ++i)
                                        q[i] = __ldcg(reinterpret_cast<const float4*>(src + (int64_t)(4 * (i0 + i) + prow) * a.N + pcol));
#pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        float* tp = tb + (4 * (i0 + i) + prow) * 33 + pcol;
                                        tp[0] = q[i].x; tp[1] = q[i].y; tp[2] = q[i].z; tp[3] = q[i].w;
                                    }
                                }
                                __syncwarp();
#pragma unroll
                                for (int c = 0; c < 32; ++c)
                                    acc[c] = zz == 0 ? tb[lane * 33 + c] : acc[c] + tb[lane * 33 + c];
                                __syncwarp();
                            }
                        }
                        uint32_t r[32];
#pragma unroll
                        for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(acc[c]);
                        epi_store<32>(r, a.rowscale[mb + lane], a.y + off + (int64_t)lane * a.N);
                    }
                    __syncwarp();   // the batch's slots are read before the next batch lands
                }
            }
        }
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0) report(a.dev_err, bad);
    if constexpr (PAIR && SPLIT) {
        // K split in two across the cluster: the pair of cluster ranks (0, 1)
        // has the first half of the K groups, (2, 3) the second, for the same
        // rows and columns. Split z finishes activation tile j = z: it sends
        // its partial products of tile 1 - z to the CTA of rank crank ^ 2
        // (through distributed shared memory, into that CTA's drained
        // activation ring) and adds the partials it receives to its own,
        // split 0's first (a + b: the same bits either way round). Every
        // thread of the cluster passes both barriers.
        static_assert(MT == 2, "one activation tile per split");
        constexpr int kXs = BN + 4;   // row stride (floats) of the exchange buffer
        static_assert(kGemmBM * kXs * 4 <= SA * SM::kA, "exchange buffer in the activation ring");
        constexpr int NDW = gemm_dec_warps(BL);
        constexpr int NCH = BN / 32;
        const bool dec = warp >= 2;
        const int quarter = warp & 3;
        const int w0 = 2 + ((quarter + 2) & 3);
        const int slot = (warp - w0) >> 2;
        const int nslot = (NDW + 1 - w0) / 4 + 1;
        const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const int z = (int)blockIdx.z;
        const int row = quarter * 32 + lane;   // this lane's TMEM lane
        cluster_sync_all();                    // every MMA of the cluster is complete: the rings are free
        const bool go = dec && __all_sync(0xffffffffu, !*abort_flag);
        if (go) {
            const uint32_t rb = cluster_map(smem_addr(a_ring), crank ^ 2u) + (uint32_t)(row * kXs * 4);
#pragma unroll 1
            for (int u = slot; u < NCH; u += nslot) {
                uint32_t r[32];
                tmem_ld32(tq + (1 - z) * BN + u * 32, r);
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    st_cluster_v4(rb + (uint32_t)((u * 32 + 4 * v) * 4), r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            }
        }
        cluster_sync_all();                    // the other split's half is in this CTA's ring
        if (go) {
            const int m = m0 + z * 2 * kGemmBM + row;
            const float rs = a.rowscale[m];
            const float4* rp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a_ring) + row * kXs);
#pragma unroll 1
            for (int u = slot; u < NCH; u += nslot) {
                uint32_t r[32];
                tmem_ld32(tq + z * BN + u * 32, r);
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float4 o = rp[u * 8 + v];
                    r[4 * v] = __float_as_uint(__uint_as_float(r[4 * v]) + o.x);
                    r[4 * v + 1] = __float_as_uint(__uint_as_float(r[4 * v + 1]) + o.y);
                    r[4 * v + 2] = __float_as_uint(__uint_as_float(r[4 * v + 2]) + o.z);
                    r[4 * v + 3] = __float_as_uint(__uint_as_float(r[4 * v + 3]) + o.w);
                }
                epi_store<32>(r, rs, a.y + (int64_t)m * a.N + n0 + u * 32);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) {
        cluster_sync_all();   // both CTAs are done with the pair's TMEM and barriers
        if (warp == 1)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                         :: "r"(tmem), "r"(kTmemCols) : "memory");
    } else {
        if (warp == 1)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                         :: "r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ------------------------------------------------------------------ host ----

static size_t gemm_align(size_t v, size_t a) { return (v + a - 1) / a * a; }


static bool gemm_pairs(int64_t M) {
#ifdef BT_GEMM_NO_PAIR
    return false;
#else
    return M % (2 * kGemmBM) == 0;
#endif
}

static int pick_bn(int64_t M, int64_t N, int num_sms) {
#ifdef BT_GEMM_BN_FORCE
    if (N % BT_GEMM_BN_FORCE == 0) return BT_GEMM_BN_FORCE;
#endif
    const bool pair = gemm_pairs(M);
#ifdef BT_GEMM_NO_BN256
    const int cands[] = {160, 128};
#else
    // on equal wave efficiency the wider tile wins: fewer operand bytes per FLOP
    const int cands[] = {256, 160, 128};
#endif
    int best = 128;
    double best_eff = -1.0;
    for (int bn : cands) {
        if (N % bn) continue;
        if (gemm_threads(pair ? bn / 2 : bn) > 1024) continue;   // a CTA decodes BN (pair: BN / 2) rows
        const int64_t tiles = (M / kGemmBM) * (N / bn);
        const int64_t waves = (tiles + num_sms - 1) / num_sms;
        const double eff = (double)tiles / (double)(waves * num_sms);
        if (eff > best_eff + 1e-9) { best_eff = eff; best = bn; }
    }
    return best;
}

template <int LAYOUT, int BN, int STAGES, bool SPLIT = false>
static cudaError_t launch_gemm_t(const CUtensorMap& amap, const GemmArgs& ga, int ks, cudaStream_t stream) {
    using SM = GemmSmem<LAYOUT, BN, STAGES>;
    auto kern = gemm_kernel<LAYOUT, BN, STAGES, BT_GEMM_ASTAGES, false, 1, SPLIT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ga.N / BN, ga.M / kGemmBM, SPLIT ? ks : 1);
    cfg.blockDim = dim3(gemm_threads(BN));
    cfg.dynamicSmemBytes = SM::kTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, amap, ga);
}

// CTA-pair launch: clusters of two CTAs along M (M % 256 == 0). Each CTA
// decodes BN / 2 weight rows, so the rings hold 3 activation stages and 3-4
// weight stages. The pair has to lie along the grid's x axis: a kernel that
// uses cta_group::2 launched with clusters of (1, 2, 1) is refused with
// cudaErrorInvalidClusterSize. On B200 at M = 512 the pair gives the same bits
// as the single-CTA kernel at about 540 against 501 TFLOP/s over the three
// prefill layers (-DBT_GEMM_NO_PAIR builds without it).
// ring depths (weight, activation stages) of the pair kernel per tile width
#ifndef BT_GEMM_PAIR_SB160
#define BT_GEMM_PAIR_SB160 4
#endif
#ifndef BT_GEMM_PAIR_SA160
#define BT_GEMM_PAIR_SA160 3
#endif
#ifndef BT_GEMM_PAIR_SB256
#define BT_GEMM_PAIR_SB256 3
#endif
#ifndef BT_GEMM_PAIR_SA256
#define BT_GEMM_PAIR_SA256 3
#endif
template <int LAYOUT, int BN, int SB, int SA, int MT = 1, bool SPLIT = false>
static cudaError_t launch_gemm_pair_t(const CUtensorMap& amap, const GemmArgs& ga, int ks, cudaStream_t stream) {
    using SM = GemmSmem<LAYOUT, BN / 2, SB, SA, MT>;
    static_assert(SM::kTotal <= 227 * 1024, "shared memory");
    static_assert(MT * BN <= 512, "TMEM columns");
    auto kern = gemm_kernel<LAYOUT, BN, SB, SA, true, MT, SPLIT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kTotal);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(ga.M / (kGemmBM * MT), ga.N / BN, SPLIT ? ks : 1);
    cfg.blockDim = dim3(gemm_threads(BN / 2));
    cfg.dynamicSmemBytes = SM::kTotal;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = SPLIT ? ks : 1;   // the K halves of a tile share a cluster
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, amap, ga);
}

// Two 256-row activation tiles per pair (MT = 2) against one weight tile:
// each decoded weight row meets 512 activation rows, half the decode work per
// FLOP. The activation ring keeps two 64 KB stages; TMEM holds both
// accumulators side by side. Candidates, in order, each taken when its grid
// fills the SMs as well as the one-tile choice does:
//  - 256 wide (N = 17408 at M = 512: 136 CTAs). On B200 the 17408 x 5120
//    layer went from 830 to 950 TFLOP/s (base-3), 930 to 1210 (2-bit).
//  - 160 wide with K split in two (N = 5120 at M = 512: 2 x 64 CTAs, the
//    same grid as one tile per pair without the split). Half the K groups per
//    CTA and twice the MMAs per decoded group. The two pairs of a tile form
//    one cluster of four CTAs and swap halves through distributed shared
//    memory (each finishes one activation tile). 5120 x 17408 went from 546
//    to 771 TFLOP/s (base-3); 5120 x 5120 from 453 to 540. Exchanging FP32
//    partials through the workspace instead, with the CTA finishing second
//    adding them, left a 10-15 us tail per layer. Splitting K in three over
//    256-wide tiles (120 CTAs, fewer activation reads) lost the same way.
//  - 80 wide, 2-bit only, where K is too short to split.
struct GemmTile {
    int bn, mt, ks;   // weight tile width, activation tiles per CTA (pair), K splits
    bool pair;        // CTA pairs (cta_group::2) along M
};

#ifndef BT_GEMM_PAIR_SB80
#define BT_GEMM_PAIR_SB80 4
#endif

static double wave_eff(int64_t ctas, int num_sms) {
    const int64_t waves = (ctas + num_sms - 1) / num_sms;
    return (double)ctas / (double)(waves * num_sms);
}

// Small grids (M = 128 or 256 against N = 5120: 32-80 CTAs) split K over the
// single-CTA kernel, 2 to 4 ways, keeping at least 8 K groups per split; a
// split is taken when it fills the SMs clearly better (by 5 % of a wave).
static GemmTile pick_small_split(const GemmTile& one, int64_t M, int64_t N, int64_t K, int num_sms) {
    GemmTile best = one;
#ifndef BT_GEMM_NO_SPLITK
    double best_e = wave_eff((M / kGemmBM) * (N / one.bn), num_sms);
    for (int bn : {160, 128}) {
        if (N % bn) continue;
        const int64_t ctas = (M / kGemmBM) * (N / bn);
        for (int ks = 2; ks <= 4 && K / kGroup >= 8 * ks; ++ks) {
            const double e = wave_eff(ctas * ks, num_sms);
            if (e > best_e + 0.05) { best = GemmTile{bn, 1, ks, false}; best_e = e; }
        }
    }
#else
    (void)M; (void)N; (void)K; (void)num_sms;
#endif
    return best;
}

static GemmTile pick_tile(int layout, int64_t M, int64_t N, int64_t K, int num_sms) {
    const GemmTile one{pick_bn(M, N, num_sms), 1, 1, gemm_pairs(M)};
#if defined(BT_GEMM_NO_PAIR) || defined(BT_GEMM_NO_MT2)
    (void)layout;
    return pick_small_split(one, M, N, K, num_sms);
#else
    if (!gemm_pairs(M) || M % (4 * kGemmBM) != 0) return pick_small_split(one, M, N, K, num_sms);
    const double e1 = wave_eff((M / kGemmBM) * (N / one.bn), num_sms);
    const GemmTile cands[] = {{256, 2, 1, true}, {160, 2, 2, true}, {80, 2, 1, true}};
    for (const GemmTile& c : cands) {
        if (N % c.bn || (c.bn == 80 && layout != BT_LAYOUT_2BIT)) continue;
        if (c.ks > 1 && K / kGroup < 8 * c.ks) continue;   // each half keeps a pipeline's worth of K groups
#ifdef BT_GEMM_NO_SPLITK
        if (c.ks > 1) continue;
#endif
        if (wave_eff((M / (2 * kGemmBM)) * (N / c.bn) * c.ks, num_sms) >= e1 - 1e-9) return c;
    }
    return one;
#endif
}

// workspace: the rotated FP16 activations, the row scales and, for K split
// over single CTAs, the arrival counters and the splits' FP32 partial products
struct GemmWs {
    size_t xt, rowscale, cnt, part, total;
    int n_cnt;
};

static GemmWs gemm_ws_layout(const GemmTile& t, int64_t M, int64_t N, int64_t K) {
    GemmWs w{};
    w.xt = 0;
    w.rowscale = gemm_align((size_t)M * K * 2, 256);
    w.cnt = w.rowscale + gemm_align((size_t)M * 4, 256);
    // (split pairs exchange their halves inside the cluster and need neither)
    const bool global_split = t.ks > 1 && !t.pair;
    w.n_cnt = global_split ? (int)((M / kGemmBM) * (N / t.bn) * gemm_dec_warps(t.bn)) : 0;
    w.part = w.cnt + gemm_align((size_t)w.n_cnt * 4, 256);
    w.total = w.part + (global_split ? (size_t)t.ks * M * N * 4 : 0);
    return w;
}

size_t gemm_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K, int num_sms) {
    return gemm_ws_layout(pick_tile(layout, M, N, K, num_sms), M, N, K).total;
}

template <int LAYOUT>
static cudaError_t dispatch_gemm(GemmTile tile, const CUtensorMap& amap, const GemmArgs& ga, cudaStream_t s) {
    const int bn = tile.bn;
    // a decode table in shared memory leaves room for one weight stage less
    constexpr bool kTableLayout = GemmSmem<LAYOUT, 128, 1>::kLut > 0;
#ifndef BT_GEMM_NO_PAIR
    if (tile.pair) {
        if (tile.mt == 2 && bn == 256)
            return launch_gemm_pair_t<LAYOUT, 256, kTableLayout ? 2 : 3, 2, 2>(amap, ga, 1, s);
        if (tile.mt == 2 && bn == 160 && tile.ks == 2)   // the kernel pairs split z with cluster rank ^ 2
            return launch_gemm_pair_t<LAYOUT, 160, kTableLayout ? 3 : 4, 2, 2, true>(amap, ga, tile.ks, s);
        if constexpr (LAYOUT == BT_LAYOUT_2BIT) {
            if (tile.mt == 2 && bn == 80)
                return launch_gemm_pair_t<LAYOUT, 80, BT_GEMM_PAIR_SB80, 2, 2>(amap, ga, 1, s);
        }
        if (bn == 256) return launch_gemm_pair_t<LAYOUT, 256, BT_GEMM_PAIR_SB256, BT_GEMM_PAIR_SA256>(amap, ga, 1, s);
        if (bn == 160) return launch_gemm_pair_t<LAYOUT, 160, BT_GEMM_PAIR_SB160, BT_GEMM_PAIR_SA160>(amap, ga, 1, s);
        return launch_gemm_pair_t<LAYOUT, 128, 4, 3>(amap, ga, 1, s);
    }
#endif
    if (tile.ks > 1)
        return bn == 160 ? launch_gemm_t<LAYOUT, 160, BT_GEMM_BSTAGES, true>(amap, ga, tile.ks, s)
                         : launch_gemm_t<LAYOUT, 128, BT_GEMM_BSTAGES, true>(amap, ga, tile.ks, s);
    // BN = 256: two weight stages (64 KB each) fit beside the activation ring;
    // with four decoder threads per row its CTA would exceed 1024 threads, and
    // pick_bn does not choose it
    if constexpr (gemm_threads(256) <= 1024) {
        if (bn == 256) return launch_gemm_t<LAYOUT, 256, 2>(amap, ga, 1, s);
    }
    return bn == 160 ? launch_gemm_t<LAYOUT, 160, BT_GEMM_BSTAGES>(amap, ga, 1, s)
                     : launch_gemm_t<LAYOUT, 128, BT_GEMM_BSTAGES>(amap, ga, 1, s);
}

cudaError_t launch_gemm(int layout, const uint8_t* codes, const uint16_t* scales, const void* x, int x_dtype,
                        const int8_t* sign, int64_t M, int64_t N, int64_t K, void* y, void* workspace,
                        int32_t* dev_err, int num_sms, cudaStream_t stream) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const GemmTile tile = pick_tile(layout, M, N, K, num_sms);
    const GemmWs wl = gemm_ws_layout(tile, M, N, K);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    __half* xt = reinterpret_cast<__half*>(ws + wl.xt);
    float* rowscale = reinterpret_cast<float*>(ws + wl.rowscale);
    int32_t* tile_cnt = wl.n_cnt ? reinterpret_cast<int32_t*>(ws + wl.cnt) : nullptr;

    GemmPrepArgs pa{};
    pa.x = x;
    pa.x_bf16 = x_dtype == BT_BF16;
    pa.sign = sign;
    pa.M = static_cast<int>(M);
    pa.K = static_cast<int>(K);
    pa.G = static_cast<int>(K / kGroup);
    pa.layout = layout;
    pa.xt = xt;
    pa.rowscale = rowscale;
    pa.tile_cnt = tile_cnt;
    pa.n_cnt = wl.n_cnt;
    const size_t prep_smem = (size_t)K * 4 + (size_t)kGemmPrepWarps * 32 * kTileStride * 4;
    cudaError_t e = cudaFuncSetAttribute(gemm_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)prep_smem);
    if (e != cudaSuccess) return e;
    gemm_prep_kernel<<<static_cast<unsigned>(M), kGemmPrepWarps * 32, prep_smem, stream>>>(pa);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    CUtensorMap amap;
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {64, kGemmBM};
    const cuuint32_t estride[2] = {1, 1};
    if (enc(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xt, gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    GemmArgs ga{};
    ga.codes = codes;
    ga.scales = scales;
    ga.rowscale = rowscale;
    ga.y = static_cast<__nv_bfloat16*>(y);
    ga.M = static_cast<int>(M);
    ga.N = static_cast<int>(N);
    ga.K = static_cast<int>(K);
    ga.G = static_cast<int>(K / kGroup);
    ga.row_bytes = (K / kGroup) * (layout == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes);
    ga.dev_err = dev_err;
    ga.part = wl.n_cnt ? reinterpret_cast<float*>(ws + wl.part) : nullptr;
    ga.tile_cnt = tile_cnt;
    return layout == BT_LAYOUT_B3 ? dispatch_gemm<BT_LAYOUT_B3>(tile, amap, ga, stream)
                                  : dispatch_gemm<BT_LAYOUT_2BIT>(tile, amap, ga, stream);
}

}  // namespace bt

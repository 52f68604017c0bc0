// Decode GEMV for one activation row (M = 1) over a list of matrices, in one
// persistent launch: y_p = W_p (R x_p) for every matrix p of the list.
//
// The release summary of Ternary Bonsai 2 27B (section 三值权重怎么压缩到
// 1.76 bit) runs the product directly on the packed ternary weights, unpack
// and group scale fused, and names the activation-side Walsh-Hadamard
// transform as the largest cost outside the matrix product at batch 1
// (section 已知短板); decode is bound by weight bytes (section 实测吞吐). A
// decode step multiplies one activation row by many matrices, some of them
// in a chain (the output of one is the input of the next). This kernel takes
// the whole list at once so that the weight stream never stops between
// matrices, and rotates each activation block once for the whole GPU.
//
// Roles (one CTA of 19 warps per SM):
//  * rotation warp: takes rotation jobs (matrix p, 1024-block b) in a fixed
//    spread over the grid. It waits until the matrix whose output is x_p is
//    complete (when x_p comes from the list), rotates the block (the warp
//    FWHT of the Sylvester H_1024, S applied first, 1/32; TensorSharp blog,
//    sections 3.2 and 5.2), and writes, per 128-group, the activations as FP16
//    in the tensor-core slot order (x' * 2^(24 - 2i - e), e from the group's
//    largest |x'|) plus (corr, 2^e) to the workspace. corr is the tensor-core
//    sum of the group with every digit 1, by the MMA chain the tiles use, so a
//    row of zero trits cancels to exactly 0. It then counts the block done.
//  * two teams, each of 8 consumer warps and 1 producer warp, share nothing
//    but the decode table. A team takes 16-row tiles of the list (full K)
//    from a global ticket counter -- the first tile of every team is fixed,
//    so its weights are requested before the dependency wait -- and its
//    producer streams each tile as one TMA stage per 1024-block ([16 rows]
//    x 208 B of codes + [16 rows] x 8 scales) into a ring of stages. At a
//    change of matrix the team waits for that matrix's rotation and copies
//    its fragments (G x 320 B) and group constants into shared memory with
//    one bulk copy. Consumer warp q decodes group q of every block through the
//    lane-replicated base-3 table (or the 2-bit fields directly), runs the
//    group's 9 (8) MMAs and adds s * (2^e D - corr) for its two rows; the 8
//    partial sums of a row are added in warp order and y is written. A tile
//    is one CTA's from start to end, so no cross-CTA reduction is needed and
//    results do not depend on the schedule.
//
// The workspace holds, after 4096 bytes of counters, the fragments and group
// constants of every matrix of the launch. The counters must be zero when a
// launch starts; the last CTA to finish sets them back to zero, so a
// workspace that was zero-filled once stays usable.
//
// Every wait is bounded in time (global timer): one that runs out sets
// BT_DEVERR_TIMEOUT and the kernel winds down without touching the data
// again, so the context stays usable.
#include "bt_internal.cuh"
#include "bt_slots.cuh"

namespace bt {

constexpr int kDecMaxProblems = 12;            // per launch (kernel parameters < 4 KB)
constexpr int kDecTeams = 2;
constexpr int kDecTeamWarps = 8;              // one per 128-group of a 1024-block
constexpr int kDecConsumerWarps = kDecTeams * kDecTeamWarps;
constexpr int kDecRotWarp = kDecConsumerWarps + kDecTeams;  // warps 16, 17: producers
constexpr int kDecWarps = kDecRotWarp + 1;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecRows = 32;                  // rows per tile: two MMA row blocks of 16
constexpr int kDecQueue = 32;                 // tile ids per team in flight (more than stages)
constexpr int kDecMaxStages = 24;
constexpr int kDecFragBytes = 320;            // per group: 10 MMA steps (9 or 8 used) x 4 lanes x 8 B
constexpr int kDecMetaBytes = 8;              // per group: (corr, 2^e)
constexpr size_t kDecSyncBytes = 4096;        // counters at the start of the workspace
constexpr int kDecSyncTicket = 0, kDecSyncExit = 1, kDecSyncRot = 2, kDecSyncDone = 2 + kDecMaxProblems;
// rotation warp's scratch: the FWHT exchange tile (then the rotated block),
// the block's fragment words [8 groups][10 steps x 8], the slot table
constexpr int kDecRotTile = 32 * kTileStride * 4;
constexpr int kDecRotWords = 8 * 80 * 4;
constexpr int kDecSlotEntries = 10 * 4 * 4;  // (step, lane, half)
constexpr int kDecRotBytes = kDecRotTile + kDecRotWords + kDecSlotEntries * 2;

// Bound on every wait, in nanoseconds of the global timer. The test-only
// build of the library shortens it.
#ifndef BT_WAIT_NS
#define BT_WAIT_NS 2000000000ull
#endif
constexpr uint64_t kDecWaitNs = BT_WAIT_NS;

struct DecProblem {
    const void* x;        // [1][K] bf16 or f32 (the output of problem `dep` when dep >= 0)
    void* y;              // [1][N]
    int32_t N, K, G, nb;
    int32_t tiles, tile_base, job_base, frag_base;  // frag_base: first group in the workspace
    int32_t dep;          // problem whose output x is (-1: none)
    int32_t x_bf16;
    int32_t has_dependents;  // a later problem of the launch reads this y: count finished tiles
};

struct DecParams {
    CUtensorMap cmap[kDecMaxProblems];
    CUtensorMap smap[kDecMaxProblems];
    DecProblem p[kDecMaxProblems];
    const int8_t* sign;   // NULL: x already rotated
    int32_t* dev_err;
    int* sync;            // [ticket, exits, rotation blocks done[P], tiles done[P]]
    uint8_t* frag;        // [groups][320 B]
    float2* meta;         // [groups] (corr, 2^e)
    int nprob, total_tiles, total_jobs, y_bf16, stages, stage_bytes, gmax;
};

// Shared-memory layout (bytes), the same on host and device.
struct DecLayout {
    int team0, team_bytes;             // team blocks
    int frag, meta, ring, red, tq, bars;  // offsets inside a team block
    int rot;                           // rotation warp's FWHT tile
    int total;
};

__host__ __device__ inline DecLayout dec_layout(int layout, int gmax, int stages, int stage_bytes) {
    DecLayout L{};
    int t = 0;
    L.frag = t;
    t += gmax * kDecFragBytes;
    L.meta = t;
    t += gmax * kDecMetaBytes;
    t = (t + 127) & ~127;
    L.ring = t;
    t += stages * stage_bytes;
    L.red = t;
    t += 2 * kDecTeamWarps * kDecRows * 4;
    L.tq = t;
    t += kDecQueue * 4;
    L.bars = t;
    t += (2 * stages + 2) * 8;
    t = (t + 1023) & ~1023;
    L.team_bytes = t;
    L.team0 = layout == BT_LAYOUT_B3 ? kB3LutBytes : 0;
    L.rot = L.team0 + kDecTeams * t;
    L.total = L.rot + kDecRotBytes;
    return L;
}

// ------------------------------------------------------------ helpers ----

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for the phase of the given parity, bounded in time.
__device__ __forceinline__ bool mbar_wait_t(uint32_t bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 63) == 0 && global_ns() - t0 > kDecWaitNs) return false;
    }
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Wait until *p >= target (a counter other CTAs raise), bounded in time.
__device__ __forceinline__ bool poll_at_least(const int* p, int target) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        __nanosleep(100);
        if (ld_acquire(p) >= target) return true;
        if (global_ns() - t0 > kDecWaitNs) return false;
    }
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Shared-memory loads of data that TMA or bulk copies wrote: volatile, so they
// stay after the barrier wait (itself volatile, with a memory clobber) that
// publishes the bytes.
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ int find_problem(const DecParams& P, int tile) {
    int p = 0;
    while (p + 1 < P.nprob && tile >= P.p[p + 1].tile_base) ++p;
    return p;
}
__device__ __forceinline__ int find_job(const DecParams& P, int job) {
    int p = 0;
    while (p + 1 < P.nprob && job >= P.p[p + 1].job_base) ++p;
    return p;
}

// The test-only build of the library (BT_TEST_WITHHOLD_COPY, never the
// product) leaves out the second stage of CTA 0's first team, so that the
// bounded wait on it runs out.
__device__ __forceinline__ bool dec_withheld(int team, uint32_t sidx) {
#ifdef BT_TEST_WITHHOLD_COPY
    return blockIdx.x == 0 && team == 0 && sidx == 1;
#else
    (void)team;
    (void)sidx;
    return false;
#endif
}

// -------------------------------------------------------- rotation warp ----

// Slot table: entry (t, c, h) = k | field << 8 of the trit that slot carries
// (k = 0xFF: empty slot). Filled once per CTA.
template <int LAYOUT>
__device__ __forceinline__ void dec_slot_table(uint16_t* tab) {
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    for (int e = threadIdx.x; e < kDecSlotEntries; e += blockDim.x) {
        const int t = e >> 4, c = (e >> 2) & 3, h = e & 3;
        int i = 0, k = -1;
        if (t < NT) k = LAYOUT == BT_LAYOUT_B3 ? b3_slot(t, c, h, &i) : tb_slot(t, c, h, &i);
        tab[e] = k < 0 ? uint16_t(0xFF) : static_cast<uint16_t>(k | (i << 8));
    }
}

template <int LAYOUT>
__device__ void dec_rotate(const DecParams& P, uint8_t* scratch, int& bad) {
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    constexpr int WPG = NT * 8;  // fragment words per group: (step, lane c, b0/b1)
    const int lane = threadIdx.x & 31;
    float* xs = reinterpret_cast<float*>(scratch);
    uint32_t* words = reinterpret_cast<uint32_t*>(scratch + kDecRotTile);
    const uint16_t* tab = reinterpret_cast<const uint16_t*>(scratch + kDecRotTile + kDecRotWords);
    // A registers of an all-zero-trit row, for the correction term
    uint32_t Og[16], Oh[16], OQg[3], OQh[3];
    if constexpr (LAYOUT == BT_LAYOUT_B3) b3_ones_tile(lane & 3, Og, Oh, OQg, OQh);
    else tb_ones_tile(Og, Oh);

    for (int job = blockIdx.x; job < P.total_jobs; job += gridDim.x) {
        const int p = find_job(P, job);
        const DecProblem& pr = P.p[p];
        const int b = job - pr.job_base;
        if (pr.dep >= 0) {
            bool ok = true;
            if (lane == 0) ok = poll_at_least(P.sync + kDecSyncDone + pr.dep, P.p[pr.dep].tiles);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) bad |= BT_DEVERR_TIMEOUT;
        }
        // this lane's 32 consecutive activations of block b (L2 reads: x may
        // have been written by this kernel)
        float v[32];
        if (pr.x_bf16) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(pr.x) +
                                                              (size_t)b * kBlock + 32 * lane);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = __ldcg(src + q);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    v[8 * q + 2 * h] = bf16_bits_to_f32(ww[h] & 0xFFFFu);
                    v[8 * q + 2 * h + 1] = bf16_bits_to_f32(ww[h] >> 16);
                }
            }
        } else {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(pr.x) +
                                                                (size_t)b * kBlock + 32 * lane);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 f = __ldcg(src + q);
                v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
            }
        }
        __syncwarp();  // the previous job's readers of xs and words are done
        if (P.sign) {
            const uint4* sg = reinterpret_cast<const uint4*>(P.sign + 32 * lane);
            const uint4 s0 = __ldg(sg), s1 = __ldg(sg + 1);
            const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t sbit = (sw[i >> 2] >> (8 * (i & 3))) & 0x80u;  // bit 7: negative entry
                v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (sbit << 24));
            }
            fwht1024_warp(v, xs);  // lane l now holds element 32 j + l in v[j]
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; ++j) xs[32 * j + lane] = v[j];
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) xs[32 * lane + i] = v[i];
        }
        __syncwarp();

        // per group: e from the largest |x'| (every lane ends with all eight)
        int eg[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float amax = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) amax = fmaxf(amax, fabsf(xs[128 * q + 32 * r + lane]));
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
            int E = amax > 0.f ? ilogbf(amax) + 1 : -100;  // amax < 2^E
            E = max(-100, min(100, E));
            eg[q] = 9 + E;
        }
        // fragment words of the eight groups, spread over the lanes
        for (int f = lane; f < 8 * WPG; f += 32) {
            const int q = f / WPG, widx = f - q * WPG;
            const int t = widx >> 3, c = (widx >> 1) & 3, hp = widx & 1;
            int e = eg[0];
#pragma unroll
            for (int r = 1; r < 8; ++r) e = q == r ? eg[r] : e;
            uint32_t word = 0;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t en = tab[(t * 4 + c) * 4 + 2 * hp + u];
                const int k = en & 0xFF, i = en >> 8;
                if (k != 0xFF) {
                    const __half hv = __float2half_rn(xs[128 * q + k] * exp2i(24 - 2 * i - e));
                    word |= static_cast<uint32_t>(__half_as_ushort(hv)) << (16 * u);
                }
            }
            words[q * 80 + widx] = word;
        }
        __syncwarp();
        // to the workspace as [group][step pair s][lane c][b0(2s), b1(2s), b0(2s+1), b1(2s+1)]
        for (int f = lane; f < 8 * 20; f += 32) {
            const int q = f / 20, r = f - q * 20, s2 = r >> 2, c = r & 3;
            const int t0 = 2 * s2, t1 = 2 * s2 + 1;
            const uint32_t* wq = words + q * 80;
            const uint4 w = make_uint4(t0 < NT ? wq[t0 * 8 + 2 * c] : 0u, t0 < NT ? wq[t0 * 8 + 2 * c + 1] : 0u,
                                       t1 < NT ? wq[t1 * 8 + 2 * c] : 0u, t1 < NT ? wq[t1 * 8 + 2 * c + 1] : 0u);
            __stcg(reinterpret_cast<uint4*>(P.frag + (size_t)(pr.frag_base + 8 * b + q) * kDecFragBytes) + 4 * s2 + c, w);
        }
        // corr per group: the all-digits-1 tile through the tiles' MMA chain
#pragma unroll 1
        for (int q = 0; q < 8; ++q) {
            uint32_t bf[NT][2];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                bf[t][0] = lane < 4 ? words[q * 80 + t * 8 + 2 * lane] : 0u;  // only column 0 is fed
                bf[t][1] = lane < 4 ? words[q * 80 + t * 8 + 2 * lane + 1] : 0u;
            }
            float d[4];
            if constexpr (LAYOUT == BT_LAYOUT_B3) b3_group_mma(Og, Oh, OQg, OQh, bf, d);
            else tb_group_mma(Og, Oh, bf, d);
            if (lane == 0) __stcg(P.meta + pr.frag_base + 8 * b + q, make_float2(d[0] * exp2i(eg[q]), exp2i(eg[q])));
        }
        __syncwarp();
        if (lane == 0) {
            __threadfence();
            atomicAdd(P.sync + kDecSyncRot + p, 1);
        }
    }
}

// ------------------------------------------------------------- producer ----

template <int LAYOUT>
__device__ void dec_produce(const DecParams& P, const DecLayout& L, uint8_t* smem, int team, int& bad) {
    constexpr int RB = LAYOUT == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;
    const int S = P.stages;
    const uint32_t tb = smem_addr(smem) + L.team0 + team * L.team_bytes;
    const uint32_t full0 = tb + L.bars, empty0 = full0 + 8 * S;
    volatile int* tq = reinterpret_cast<volatile int*>(smem + L.team0 + team * L.team_bytes + L.tq);

    int tile = blockIdx.x + team * gridDim.x;  // fixed first ticket: its weights go out before the wait
    bool waited = false, ok = true;
    uint32_t sidx = 0;
    int k = 0, pending = 0;
    while (ok) {
        const bool end = tile >= P.total_tiles;
        // the next ticket is requested before this tile's stages go out, so
        // the atomic's round trip overlaps them
        if (!end && waited) pending = atomicAdd(P.sync + kDecSyncTicket, 1);
        int p = 0, t = 0, nb = 1;
        if (!end) {
            p = find_problem(P, tile);
            t = tile - P.p[p].tile_base;
            nb = P.p[p].nb;
        }
        for (int b = 0; b < nb; ++b) {
            const uint32_t slot = sidx % S;
            if (sidx >= (uint32_t)S && !mbar_wait_t(empty0 + 8 * slot, ((sidx / S) - 1) & 1u)) {
                bad |= BT_DEVERR_TIMEOUT;
                ok = false;
                break;
            }
            if (b == 0) tq[k % kDecQueue] = end ? -1 : tile;
            const uint32_t fb = full0 + 8 * slot;
            if (end) {
                mbar_arrive(fb);  // no data: the consumers read the end mark and stop
            } else if (!dec_withheld(team, sidx)) {
                mbar_arrive_tx(fb, (uint32_t)P.stage_bytes);
                const uint32_t dst = tb + L.ring + slot * P.stage_bytes;
                tma_load_2d(dst, &P.cmap[p], b * RB, t * kDecRows, fb);
                tma_load_2d(dst + kDecRows * RB, &P.smap[p], b * 8, t * kDecRows, fb);
            }
            ++sidx;
        }
        if (end) break;
        ++k;
        if (!waited) {
            pdl_wait();  // the ticket counter belongs to this launch only after the previous one ends
            waited = true;
            pending = atomicAdd(P.sync + kDecSyncTicket, 1);
        }
        tile = pending + kDecTeams * (int)gridDim.x;
    }
    // let every copy still in flight land before the CTA may exit
    const uint32_t first = sidx > (uint32_t)S ? sidx - S : 0u;
    for (uint32_t j = first; j < sidx; ++j) mbar_wait_t(full0 + 8 * (j % S), (j / S) & 1u);
}

// ------------------------------------------------------------- consumers ----

extern __shared__ __align__(1024) uint8_t dec_smem[];

// The decode table sits at the start of the dynamic shared memory.
struct DecLut {
    __device__ __forceinline__ static uint32_t ld(uint32_t off) {
        return *reinterpret_cast<const uint32_t*>(dec_smem + off);
    }
};

template <int LAYOUT, bool CHECK>
__device__ void dec_consume(const DecParams& P, const DecLayout& L, uint8_t* smem, int team, int& bad) {
    constexpr int RB = LAYOUT == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;
    constexpr int NT = LAYOUT == BT_LAYOUT_B3 ? kB3Mmas : k2bMmas;
    const int S = P.stages;
    const uint32_t stage_bytes = static_cast<uint32_t>(P.stage_bytes);
    const int y_bf16 = P.y_bf16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp % kDecTeamWarps;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t tb = smem_addr(smem) + L.team0 + team * L.team_bytes;
    const uint32_t full0 = tb + L.bars, empty0 = full0 + 8 * S;
    const uint32_t fbar = empty0 + 8 * S, tbar = fbar + 8;
    const uint32_t frag = tb + L.frag, meta = tb + L.meta, ring = tb + L.ring;
    float* red = reinterpret_cast<float*>(smem + L.team0 + team * L.team_bytes + L.red);
    volatile int* tq = reinterpret_cast<volatile int*>(smem + L.team0 + team * L.team_bytes + L.tq);

    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    uint32_t mG[3] = {0, 0, 0}, mH[3] = {0, 0, 0};
    if constexpr (LAYOUT == BT_LAYOUT_B3) b3_pair12_masks(c, mG, mH);
    // this lane's bytes inside a stage row, and the base-3 window shift
    const uint32_t off = LAYOUT == BT_LAYOUT_B3 ? static_cast<uint32_t>(q * kB3GroupBytes + 6 * c)
                                                : static_cast<uint32_t>(q * k2bGroupBytes + 8 * c);
    const uint32_t o8 = LAYOUT == BT_LAYOUT_B3 ? (off & 3u) * 8u : 0u;
    const uint32_t a4 = LAYOUT == BT_LAYOUT_B3 ? (off & ~3u) : off;
    const uint32_t o12 = static_cast<uint32_t>(q * kB3GroupBytes + 24 + (c < 2 ? 0 : 8 * RB));
    const uint32_t frag_lane = frag + c * 16;

    pdl_wait();  // x, y and the counters belong to this launch from here on

    auto team_bar = [&](uint32_t& ph) -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(tbar);
        const bool ok = mbar_wait_t(tbar, ph);
        ph ^= 1u;
        return ok;
    };

    uint32_t err = 0, sidx = 0, fph = 0, tph = 0;
    int k = 0, cur = -1;
    int nb = 0, N = 0, has_dep = 0, tile_base = 0;
    void* y = nullptr;
    for (;;) {
        uint32_t slot = sidx % S;
        if (!mbar_wait_t(full0 + 8 * slot, (sidx / S) & 1u)) { bad |= BT_DEVERR_TIMEOUT; break; }
        const int tile = tq[k % kDecQueue];
        if (tile < 0) break;
        const int p = find_problem(P, tile);
        if (p != cur) {
            nb = P.p[p].nb;
            N = P.p[p].N;
            has_dep = P.p[p].has_dependents;
            tile_base = P.p[p].tile_base;
            y = P.p[p].y;
            const int G = P.p[p].G, frag_base = P.p[p].frag_base;
            // every warp of the team is done with the previous fragments
            if (!team_bar(tph)) { bad |= BT_DEVERR_TIMEOUT; break; }
            if (q == 0 && lane == 0) {
                if (!poll_at_least(P.sync + kDecSyncRot + p, nb)) bad |= BT_DEVERR_TIMEOUT;
                asm volatile("fence.proxy.async;" ::: "memory");  // rotation results, read by the copy engine
                const uint32_t fbytes = G * kDecFragBytes, mbytes = G * kDecMetaBytes;
                mbar_arrive_tx(fbar, fbytes + mbytes);
                bulk_g2s(frag, P.frag + (size_t)frag_base * kDecFragBytes, fbytes, fbar);
                bulk_g2s(meta, P.meta + frag_base, mbytes, fbar);
            }
            const bool ok = mbar_wait_t(fbar, fph);
            fph ^= 1u;
            if (!ok) { bad |= BT_DEVERR_TIMEOUT; break; }
            cur = p;
        }
        const int t = tile - tile_base;
        // rows g, g + 8 (tt = 0) and 16 + g, 24 + g (tt = 1) of the tile
        float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        bool ok = true;
        for (int b = 0; b < nb; ++b) {
            if (b > 0) {
                slot = sidx % S;
                if (!mbar_wait_t(full0 + 8 * slot, (sidx / S) & 1u)) { ok = false; break; }
            }
            const uint32_t st = ring + slot * stage_bytes;
            const uint32_t sc = st + kDecRows * RB;
            float sgv[2], shv[2];
            uint32_t w[2][5];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const uint32_t rg = static_cast<uint32_t>((16 * tt + g) * RB), rh = rg + 8 * RB;
                sgv[tt] = f16_bits_to_f32(lds16(sc + (16 * tt + g) * 16 + 2 * q));
                shv[tt] = f16_bits_to_f32(lds16(sc + (16 * tt + g + 8) * 16 + 2 * q));
                if constexpr (LAYOUT == BT_LAYOUT_B3) {
                    w[tt][0] = lds32(st + rg + a4);
                    w[tt][1] = lds32(st + rg + a4 + 4);
                    w[tt][2] = lds32(st + rh + a4);
                    w[tt][3] = lds32(st + rh + a4 + 4);
                    w[tt][4] = lds16(st + 16 * tt * RB + g * RB + o12);
                } else {
                    const uint2 x0 = lds64(st + rg + a4), x1 = lds64(st + rh + a4);
                    w[tt][0] = x0.x; w[tt][1] = x0.y; w[tt][2] = x1.x; w[tt][3] = x1.y; w[tt][4] = 0;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * slot);  // the stage may be refilled
            ++sidx;
            // activation fragments of group 8 b + q (column 0: lanes with g == 0)
            const int j = 8 * b + q;
            uint32_t bf[NT][2];
#pragma unroll
            for (int s2 = 0; s2 < (NT + 1) / 2; ++s2) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (g == 0) v = lds128(frag_lane + j * kDecFragBytes + s2 * 64);
                bf[2 * s2][0] = v.x;
                bf[2 * s2][1] = v.y;
                if (2 * s2 + 1 < NT) {
                    bf[2 * s2 + 1][0] = v.z;
                    bf[2 * s2 + 1][1] = v.w;
                }
            }
            const uint2 md = lds64(meta + j * kDecMetaBytes);
            const float cm = __uint_as_float(md.x), pm = __uint_as_float(md.y);
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                uint32_t Rg[16], Rh[16], QG[3], QH[3];
                float d[4];
                if constexpr (LAYOUT == BT_LAYOUT_B3) {
                    b3_decode_tile<CHECK, DecLut>(w[tt][0], w[tt][1], w[tt][2], w[tt][3], w[tt][4], o8, lane4, mG,
                                                  mH, Rg, Rh, QG, QH, err);
                    b3_group_mma(Rg, Rh, QG, QH, bf, d);
                } else {
                    tb_decode_tile<CHECK>(make_uint2(w[tt][0], w[tt][1]), make_uint2(w[tt][2], w[tt][3]), Rg, Rh,
                                          err);
                    tb_group_mma(Rg, Rh, bf, d);
                }
                acc[tt][0] = fmaf(sgv[tt], fmaf(d[0], pm, -cm), acc[tt][0]);
                acc[tt][1] = fmaf(shv[tt], fmaf(d[2], pm, -cm), acc[tt][1]);
            }
        }
        if (!ok) { bad |= BT_DEVERR_TIMEOUT; break; }
        // the tile's rows: partial sums of the 8 warps, added in warp order
        float* rd = red + (k & 1) * (kDecTeamWarps * kDecRows);
        if (c == 0) {
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                rd[q * kDecRows + 16 * tt + g] = acc[tt][0];
                rd[q * kDecRows + 16 * tt + g + 8] = acc[tt][1];
            }
        }
        if (!team_bar(tph)) { bad |= BT_DEVERR_TIMEOUT; break; }
        if (q == 0) {
            float sum = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < kDecTeamWarps; ++w2) sum += rd[w2 * kDecRows + lane];
            const int n = t * kDecRows + lane;
            if (n < N) {
                if (y_bf16) reinterpret_cast<__nv_bfloat16*>(y)[n] = __float2bfloat16_rn(sum);
                else reinterpret_cast<float*>(y)[n] = sum;
            }
            __syncwarp();
            if (lane == 0 && has_dep) {
                __threadfence();
                atomicAdd(P.sync + kDecSyncDone + p, 1);
            }
        }
        ++k;
    }
    if (CHECK) {
        if (LAYOUT == BT_LAYOUT_B3) { if (err >> 31) bad |= BT_DEVERR_INVALID_CODE; }
        else if (err & 0x55555555u) bad |= BT_DEVERR_INVALID_CODE;
    }
}

// -------------------------------------------------------------- kernel ----

template <int LAYOUT, bool CHECK>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const __grid_constant__ DecParams P) {
    uint8_t* smem = dec_smem;
    const DecLayout L = dec_layout(LAYOUT, P.gmax, P.stages, P.stage_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if constexpr (LAYOUT == BT_LAYOUT_B3) b3_lut_fill(smem, threadIdx.x, blockDim.x);
    dec_slot_table<LAYOUT>(reinterpret_cast<uint16_t*>(smem + L.rot + kDecRotTile + kDecRotWords));
    if (threadIdx.x < kDecTeams) {
        const uint32_t tb = smem_addr(smem) + L.team0 + threadIdx.x * L.team_bytes;
        const uint32_t full0 = tb + L.bars, empty0 = full0 + 8 * P.stages;
        for (int s = 0; s < P.stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kDecTeamWarps);
        }
        mbar_init(empty0 + 8 * P.stages, 1);                  // fragment copy
        mbar_init(empty0 + 8 * P.stages + 8, kDecTeamWarps);  // team barrier
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    pdl_launch_dependents();

    int bad = 0;
    if (warp < kDecConsumerWarps) {
        dec_consume<LAYOUT, CHECK>(P, L, smem, warp / kDecTeamWarps, bad);
    } else if (warp < kDecRotWarp) {
        if (lane == 0) dec_produce<LAYOUT>(P, L, smem, warp - kDecConsumerWarps, bad);
    } else {
        pdl_wait();
        dec_rotate<LAYOUT>(P, smem + L.rot, bad);
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0 && bad) report(P.dev_err, bad);

    __syncthreads();
    if (threadIdx.x == 0) {
        pdl_wait();
        __threadfence();
        if (atomicAdd(P.sync + kDecSyncExit, 1) == (int)gridDim.x - 1) {
            // the last CTA: every other CTA is done with the counters
            __threadfence();
            P.sync[kDecSyncTicket] = 0;
            for (int i = 0; i < kDecMaxProblems; ++i) {
                P.sync[kDecSyncRot + i] = 0;
                P.sync[kDecSyncDone + i] = 0;
            }
            P.sync[kDecSyncExit] = 0;
            __threadfence();
        }
    }
}

// ---------------------------------------------------------------- host ----

struct DecodeProblem {
    const uint8_t* codes;
    const uint16_t* scales;
    const void* x;
    int x_bf16;
    int x_from;  // -1 or an earlier problem index
    void* y;
    int64_t N, K;
};

static size_t dec_align(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace of one launch over problems [first, last).
static size_t dec_ws_one(const DecodeProblem* pr, int count) {
    size_t groups = 0;
    for (int i = 0; i < count; ++i) groups += (size_t)(pr[i].K / kGroup);
    return kDecSyncBytes + dec_align(groups * kDecFragBytes, 256) + dec_align(groups * kDecMetaBytes, 256);
}

size_t decode_workspace_bytes(const int64_t* Ks, int count) {
    size_t need = kDecSyncBytes;
    for (int first = 0; first < count; first += kDecMaxProblems) {
        size_t groups = 0;
        for (int i = first; i < count && i < first + kDecMaxProblems; ++i) groups += (size_t)(Ks[i] / kGroup);
        const size_t w = kDecSyncBytes + dec_align(groups * kDecFragBytes, 256) + dec_align(groups * kDecMetaBytes, 256);
        if (w > need) need = w;
    }
    return need;
}

bool decode_applies(int64_t M, int64_t K, const void* codes, const void* scales) {
    return M == 1 && K > 0 && K % kBlock == 0 && (reinterpret_cast<uintptr_t>(scales) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
}

template <int LAYOUT, bool CHECK>
static cudaError_t dec_launch_t(const DecParams& P, int grid, size_t smem, cudaStream_t stream) {
    auto kern = decode_kernel<LAYOUT, CHECK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, P);
}

// One launch over problems[first, first + count); x_from indices refer to the
// whole list (dependencies on problems of earlier launches are met by stream
// order).
static cudaError_t dec_launch_group(int layout, const DecodeProblem* all, int first, int count, const int8_t* sign,
                                    int y_bf16, uint8_t* ws, int32_t* dev_err, int num_sms, cudaStream_t stream) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    DecParams P{};  // copied into the launch
    const int RB = layout == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;
    int tiles = 0, jobs = 0, groups = 0, gmax = 0;
    for (int i = 0; i < count; ++i) {
        const DecodeProblem& s = all[first + i];
        DecProblem& d = P.p[i];
        d.N = static_cast<int32_t>(s.N);
        d.K = static_cast<int32_t>(s.K);
        d.G = static_cast<int32_t>(s.K / kGroup);
        d.nb = static_cast<int32_t>(s.K / kBlock);
        d.tiles = static_cast<int32_t>((s.N + kDecRows - 1) / kDecRows);
        d.tile_base = tiles;
        d.job_base = jobs;
        d.frag_base = groups;
        d.y = s.y;
        if (s.x_from >= first) {
            d.dep = s.x_from - first;
            d.x = all[s.x_from].y;
            d.x_bf16 = y_bf16;
        } else {
            d.dep = -1;
            d.x = s.x_from >= 0 ? all[s.x_from].y : s.x;
            d.x_bf16 = s.x_from >= 0 ? y_bf16 : s.x_bf16;
        }
        d.has_dependents = 0;
        if (d.dep >= 0) P.p[d.dep].has_dependents = 1;
        tiles += d.tiles;
        jobs += d.nb;
        groups += d.G;
        if (d.G > gmax) gmax = d.G;
        const cuuint64_t row_bytes = static_cast<cuuint64_t>(d.G) * (layout == BT_LAYOUT_B3 ? kB3GroupBytes : k2bGroupBytes);
        const cuuint64_t cdim[2] = {row_bytes, static_cast<cuuint64_t>(s.N)};
        const cuuint64_t cstr[1] = {row_bytes};
        const cuuint32_t cbox[2] = {static_cast<cuuint32_t>(RB), kDecRows};
        const cuuint64_t sdim[2] = {static_cast<cuuint64_t>(d.G), static_cast<cuuint64_t>(s.N)};
        const cuuint64_t sstr[1] = {static_cast<cuuint64_t>(d.G) * 2};
        const cuuint32_t sbox[2] = {8, kDecRows};
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
    P.sync = reinterpret_cast<int*>(ws);
    P.frag = ws + kDecSyncBytes;
    P.meta = reinterpret_cast<float2*>(ws + kDecSyncBytes + dec_align((size_t)groups * kDecFragBytes, 256));
    P.nprob = count;
    P.total_tiles = tiles;
    P.total_jobs = jobs;
    P.y_bf16 = y_bf16;
    P.gmax = gmax;
    P.stage_bytes = kDecRows * RB + kDecRows * 16;
    // as many stages as fit next to the table, fragments and rotation tile
    const size_t limit = 227 * 1024;
    int stages = 0;
    for (int st = kDecMaxStages; st >= 2; --st) {
        if ((size_t)dec_layout(layout, gmax, st, P.stage_bytes).total <= limit) { stages = st; break; }
    }
    if (stages == 0) return cudaErrorInvalidValue;  // K too large for the fragment area
    P.stages = stages;
    const size_t smem = dec_layout(layout, gmax, stages, P.stage_bytes).total;
    const int grid = num_sms;
    if (layout == BT_LAYOUT_B3)
        return dev_err ? dec_launch_t<BT_LAYOUT_B3, true>(P, grid, smem, stream)
                       : dec_launch_t<BT_LAYOUT_B3, false>(P, grid, smem, stream);
    return dev_err ? dec_launch_t<BT_LAYOUT_2BIT, true>(P, grid, smem, stream)
                   : dec_launch_t<BT_LAYOUT_2BIT, false>(P, grid, smem, stream);
}

cudaError_t launch_decode(int layout, const DecodeProblem* problems, int count, const int8_t* sign, int y_dtype,
                          void* workspace, int32_t* dev_err, int num_sms, cudaStream_t stream) {
    for (int first = 0; first < count; first += kDecMaxProblems) {
        const int n = count - first < kDecMaxProblems ? count - first : kDecMaxProblems;
        const cudaError_t e = dec_launch_group(layout, problems, first, n, sign, y_dtype == BT_BF16,
                                               static_cast<uint8_t*>(workspace), dev_err, num_sms, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Largest K the decode kernel takes: the fragments of one matrix sit in each
// team's shared memory next to the decode table and at least two stages.
int64_t decode_max_k(int layout) {
    const int RB = layout == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;
    int64_t best = 0;
    for (int G = 8; G <= 4096; G += 8)
        if ((size_t)dec_layout(layout, G, 2, kDecRows * RB + kDecRows * 16).total <= 227 * 1024) best = (int64_t)G * kGroup;
    return best;
}

bool decode_k_fits(int layout, int64_t K) {
    const int G = static_cast<int>(K / kGroup);
    const int RB = layout == BT_LAYOUT_B3 ? 8 * kB3GroupBytes : 8 * k2bGroupBytes;
    return (size_t)dec_layout(layout, G, 2, kDecRows * RB + kDecRows * 16).total <= 227 * 1024;
}

}  // namespace bt

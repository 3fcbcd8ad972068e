// Paged decode attention for sm_100a.
//
// What it computes ("Walk through paged attention end to end", attention
// step): for each sequence b and query head g, softmax(scale * q K^T) V over
// the sequence's L tokens, where token p lives in block
// block_tables[b][p / bs] at row p % bs of the pool ("What is PagedAttention
// and how does it manage KV cache", How PagedAttention works: two-level
// indirection, tokens contiguous inside a block).
//
// How it runs on B200:
//  * One CTA per (kv head h, sequence b[, sequence partition]) serves all G
//    query heads of the group, so each K/V byte leaves HBM once.
//  * The sequence is cut into 16-token tiles.  A producer warp dereferences
//    the block table and stages each tile's K and V (16 rows x head_dim
//    bf16, contiguous in the pool) into shared memory with TMA tile loads
//    (128-byte swizzle, no multicast) through an 8-deep mbarrier ring
//    (16-deep for fp8 pools at head_dim 128, whose tiles are half the size).
//  * Four consumer warps take tiles round-robin.  Per tile a warp computes
//    S^T = K_tile Q^T with bf16 mma.sync (M = 16 tokens, N = 8 query-head
//    columns, K = head_dim), runs an online softmax in fp32 (log2 domain),
//    and accumulates O^T += V_tile^T P^T with a second mma (M = 16 dims,
//    N = 8 heads, K = 16 tokens).  P is split into bf16 hi + lo parts so the
//    PV product keeps ~16 mantissa bits (fp8 pools: one f16 part, 11 bits).
//  * Warps merge their (max, sum, O) states through shared memory.  In the
//    split variant each CTA writes its partition's state to the workspace
//    and a log-sum-exp reduce kernel, launched as a programmatic dependent,
//    combines the partitions.
//  * fp8 (E4M3) pools: K and V codes are widened to f16 in registers and run
//    through the same f16 mma.sync.  A tuning build (PA_DECODE_FP8_TCGEN05=1)
//    computes the scores on the 5th-generation tensor cores instead: a sixth
//    warp issues tcgen05.mma (kind::f8f6f4, M = 64 token rows = four ring
//    tiles, N = 8 query-head columns, K = 32 per step) straight from the
//    swizzled E4M3 K tiles, against q held as two E4M3 terms, with fp32
//    scores in tensor memory; each consumer warp reads its tile's 16 rows
//    back with tcgen05.ld, already in the mma.sync accumulator layout.  It is
//    correct but slower on B200, so the library keeps mma.sync.
//  * Shared-prefix variant: sequences that share their first tokens (n-way
//    sampling of one prompt) get one extra work item per group and kv head
//    that reads the shared tiles once and serves every member's query heads
//    as extra mma columns; each member's own work items start after the
//    shared tiles, and the reduce combines both.
//
// This header holds the device code (the decode kernel, the log-sum-exp
// reduce, their shared-memory layout and parameters).  decode.cu includes it
// and holds the host side, so a change there leaves the device code -- and
// any profile taken of it -- untouched.
#pragma once

#include "pa_common.cuh"

namespace pa {
namespace {

// Compile-time shape of the decode CTA (overridable for tuning builds).
#ifndef PA_DECODE_CONSUMER_WARPS
#define PA_DECODE_CONSUMER_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 8
#endif
#ifndef PA_DECODE_PRODUCER_LANES
#define PA_DECODE_PRODUCER_LANES 8
#endif
constexpr int kTileTokens = 16;
constexpr int kConsumerWarps = PA_DECODE_CONSUMER_WARPS;
constexpr int kDefaultStages = PA_DECODE_STAGES;
// fp8 pools at head_dim 128 compute the scores with mma.sync on K codes
// widened to f16 in registers (0) or with tcgen05.mma (1, a tuning build).
#ifndef PA_DECODE_FP8_TCGEN05
#define PA_DECODE_FP8_TCGEN05 0
#endif
// fp8 pools: P enters the PV mma as one f16 part (0) or as f16 hi + lo parts
// (1, a tuning build).  One part keeps 11 significant bits of each weight, for
// values that carry 4 (E4M3); measured on B200 it takes 3-5 % less time.
#ifndef PA_DECODE_FP8_P_LO
#define PA_DECODE_FP8_P_LO 0
#endif
// Ring depth of fp8 pools at head_dim 128 (their tiles are half the size).
#ifndef PA_DECODE_FP8_STAGES
#define PA_DECODE_FP8_STAGES (2 * PA_DECODE_STAGES)
#endif
// Producer lanes issue tiles round-robin; lane k owns ring slots k, k+P, ...
constexpr int kProducerLanes = PA_DECODE_PRODUCER_LANES;
static_assert(kProducerLanes >= 1 && kProducerLanes <= 8, "window indexing assumes <= 8 lanes");
// A 16-bit tile (bf16, or f16 expanded from fp8) is stored as HEAD_DIM/64
// boxes of 16 rows x 128 bytes with the TMA 128-byte swizzle.
constexpr int kBox16Bytes = kTileTokens * 128;
constexpr float kLog2e = 1.4426950408889634f;

template <int HEAD_DIM, bool FP8>
struct Cfg {
    // What TMA lands in the ring: bf16 tiles in 64-column swizzled boxes, or
    // fp8 tiles as one box of 16 rows x HEAD_DIM bytes (128-byte swizzle at
    // head_dim 128, none at 64).
    static constexpr int kBoxes = FP8 ? 1 : HEAD_DIM / 64;
    static constexpr int kBoxCols = FP8 ? HEAD_DIM : 64;
    static constexpr int kBoxRowBytes = FP8 ? HEAD_DIM : 128;
    static constexpr int kBoxBytes = kTileTokens * kBoxRowBytes;
    static constexpr int kTileBytes = kBoxes * kBoxBytes;  // K or V of one tile
    static constexpr int kStageBytes = 2 * kTileBytes;
    // fp8, head_dim 128: the ring tile carries the 128-byte swizzle; the K and V
    // mma fragments are built straight from it, in registers.
    // fp8, head_dim 64: the ring tile is unswizzled and both K and V are expanded
    // to per-warp 16-bit tiles.
    static constexpr bool kDirect = FP8 && HEAD_DIM == 128;
    // fp8, head_dim 128, tcgen05 scores: a sixth warp issues the MMAs.  Four
    // consecutive K tiles (a chunk) form one 64-row operand, so the ring keeps
    // all K tiles together and all V tiles after them (otherwise slot s holds
    // K then V).
    static constexpr bool kTc = kDirect && PA_DECODE_FP8_TCGEN05;
    static constexpr int kThreads = (kConsumerWarps + 1 + (kTc ? 1 : 0)) * 32;
    // Ring depth.  With K and V read from the ring, a slot stays busy until its
    // tile has gone through PV, and fp8 tiles are half the size: twice the
    // default depth keeps enough bytes in flight (measured on B200: 8-11 % less
    // time per call than the default depth).
    static constexpr int kStages = kDirect ? PA_DECODE_FP8_STAGES : kDefaultStages;
    // Ring slot s is filled by one producer lane and consumed by one consumer
    // warp, each in order: a parity wait can then never run a phase ahead.
    static constexpr int kLanes = kStages % kProducerLanes == 0 ? kProducerLanes : kStages % 6 == 0 ? 6 : 4;
    static_assert(kStages % kLanes == 0, "each producer lane owns whole ring slots");
    static_assert(kStages % kConsumerWarps == 0, "each consumer warp owns whole ring slots");
    static constexpr int kRingBytes = kStages * kStageBytes;
    __host__ __device__ static constexpr uint32_t k_off(int s) {
        return kTc ? (uint32_t)(s * kTileBytes) : (uint32_t)(s * kStageBytes);
    }
    __host__ __device__ static constexpr uint32_t v_off(int s) {
        return kTc ? (uint32_t)((kStages + s) * kTileBytes) : (uint32_t)(s * kStageBytes + kTileBytes);
    }
    // tcgen05 scores: q as two E4M3 terms, each 8 columns x 128 bytes (one swizzle atom)
    static constexpr int kQTerms = 2;
    static constexpr int kQOpBytes = kTc ? kQTerms * 1024 : 0;
    static constexpr int kScoreBufs = 4;  // TMEM score buffers (chunks in flight)
    static constexpr int kScoreBars = kTc ? 2 * kScoreBufs : 0;
    static constexpr int kTmemCols = 32;  // kScoreBufs x 8 fp32 columns
    static constexpr int kTile16Bytes = (HEAD_DIM / 64) * kBox16Bytes;
    static constexpr int kStagingBytes = FP8 && !kDirect ? kConsumerWarps * 2 * kTile16Bytes : 0;
    static constexpr int kDataBytes = kRingBytes + kStagingBytes + kQOpBytes;
    static constexpr int kMergeStride = HEAD_DIM + 4;  // padded row: conflict-free merge stores
    static constexpr int kMergeBytes = kConsumerWarps * 8 * (kMergeStride + 2) * 4;
    static_assert(kMergeBytes <= kDataBytes, "merge area reuses the ring");
    // + barriers, tile flags, the fused write's row (32 x 16 bytes), its block
    // id (twice: K and V halves with tcgen05 scores) and the TMEM address
    static constexpr int kSmemBytes =
        1024 /*align slack*/ + kDataBytes + 32 * 16 + kStages * 8 * 2 + kScoreBars * 8 + kStages * 4 + 16;
    static_assert(kDataBytes % 1024 == 0, "the tail (16-byte row, then 8-byte barriers) starts 1024-aligned");
};

struct DecodeParams {
    float *out;                 // [B, Hq, d]            (single pass)
    float *part_o;              // [B, Hq, P, d]         (split)
    float *part_ml;             // [B, Hq, P, 2]         (split)
    const uint16_t *q;          // [B, Hq, d] bf16
    const int32_t *block_tables;
    const int32_t *seq_lens;
    int32_t *err_flag;
    const uint16_t *k_new;      // [B, Hkv, d] bf16 (fused cache write only)
    const uint16_t *v_new;
    uint16_t *k_pool;           // pools, written by the fused cache write
    uint16_t *v_pool;
    int64_t num_blocks;
    int max_blocks;
    int max_seq_len;
    int num_q_heads;
    int num_kv_heads;
    int group;
    int block_size;
    int part_tokens;            // tokens per CTA along the sequence
    int num_parts;
    float scale_log2;           // softmax scale * log2(e)
    float k_scale;              // fp8 pools: dequantisation multipliers
    float v_scale;
    float k_inv_scale;          // fp8 pools: 1 / scale, for the fused cache write
    float v_inv_scale;
    int batch;
    int num_slots;              // split: partial-state slots per row: num_parts (x2 with prefix groups)
    // Shared-prefix groups: sequences [g*group_size, (g+1)*group_size) share prefix_lens[g] tokens.
    const int32_t *prefix_lens; // [num_groups]
    int group_size;
    int num_groups;
    int members_per_item;       // members one prefix item serves: 8 / G (the mma N columns)
    int items_per_group;        // ceil(group_size / members_per_item)
};

// Sequence length as every kernel of one call sees it: out-of-contract values
// are clamped (and reported once by the caller of this helper).
__device__ __forceinline__ int clamp_len(int L, const DecodeParams &p) {
    const int cap = min(p.max_seq_len, p.max_blocks * p.block_size);
    return L < 0 ? 0 : (L > cap ? cap : L);
}

// Partitions of `tokens` tokens at `part_tokens` per partition.
__device__ __forceinline__ int parts_of(int tokens, int part_tokens) {
    return tokens > 0 ? (tokens + part_tokens - 1) / part_tokens : 0;
}

// Tokens at the start of group g's sequences that are read once for the whole
// group: the group's prefix_lens entry, cut to every member's length minus one
// (the token appended in this step is never shared) and rounded down to whole
// 16-token tiles, so each member's own tiles start tile-aligned.  0 for groups
// of one sequence.
// Every lane of a warp loads members in parallel, so call it from whole warps.
__device__ __forceinline__ int group_shared_tokens(const DecodeParams &p, int g) {
    const int m0 = g * p.group_size;
    const int m1 = min(m0 + p.group_size, p.batch);
    if (m1 - m0 < 2) return 0;
    int s = __ldg(p.prefix_lens + g);
    for (int m = m0 + (int)(threadIdx.x & 31); m < m1; m += 32) s = min(s, clamp_len(__ldg(p.seq_lens + m), p) - 1);
#pragma unroll
    for (int off = 16; off; off >>= 1) s = min(s, __shfl_xor_sync(0xffffffffu, s, off));
    return s > 0 ? s / kTileTokens * kTileTokens : 0;
}

// Byte offset of 16-byte chunk c of token row r inside one swizzled 16-bit tile.
__device__ __forceinline__ uint32_t tile_offset(int r, int c) {
    return (uint32_t)((c >> 3) * kBox16Bytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Byte offset of byte `byte` of row r in a 128-byte-swizzled fp8 tile (128-byte rows).
__device__ __forceinline__ uint32_t fp8_tile_offset(int r, int byte) {
    return (uint32_t)(r * 128 + ((((byte >> 4) ^ (r & 7))) << 4) + (byte & 15));
}

// Eight E4M3 codes -> four f16x2 words (codes 0,1 | 2,3 | 4,5 | 6,7).
__device__ __forceinline__ uint4 e4m3x8_to_f16x8(uint32_t lo, uint32_t hi) {
    uint4 r;
    e4m3x4_to_f16x4(lo, r.x, r.y);
    e4m3x4_to_f16x4(hi, r.z, r.w);
    return r;
}

template <bool FP8>
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    if constexpr (FP8)
        mma_f16_16816(d, a0, a1, a2, a3, b0, b1);
    else
        mma_bf16_16816(d, a0, a1, a2, a3, b0, b1);
}

// Tuning builds only: PA_DECODE_SIMT_G1=1 computes the scores and PV of bf16
// groups of one query head on the CUDA cores (warp-shuffle dot products, fp32
// FMA) instead of mma.sync; =2 does the same with the mma path compiled out
// (bf16 groups of one query head only).  This is the comparison that keeps
// tensor cores on this path.  The library is built with 0.
#ifndef PA_DECODE_SIMT_G1
#define PA_DECODE_SIMT_G1 0
#endif

// CTAs per SM the register allocation must allow (bf16 is limited to 3 by shared memory).
#ifndef PA_DECODE_MIN_CTAS_FP8
#define PA_DECODE_MIN_CTAS_FP8 3
#endif
#ifndef PA_DECODE_MIN_CTAS_BF16
#define PA_DECODE_MIN_CTAS_BF16 3
#endif

template <int HEAD_DIM, bool SPLIT, bool APPEND, bool FP8, bool PREFIX>
__global__ void __launch_bounds__(Cfg<HEAD_DIM, FP8>::kThreads, FP8 ? PA_DECODE_MIN_CTAS_FP8 : PA_DECODE_MIN_CTAS_BF16)
    paged_decode_kernel(
    const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
    const DecodeParams p) {
    static_assert(SPLIT || !PREFIX, "shared-prefix items always merge through the split path");
    using C = Cfg<HEAD_DIM, FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // Fused write: the new token's bf16 K/V row (16 bytes per lane), fetched
    // asynchronously so no registers are held until the tile is reached.  It
    // comes first in the tail: kDataBytes is a multiple of 1024, so the row is
    // 16-byte aligned whatever the ring depth.
    uint4 *append_row = reinterpret_cast<uint4 *>(smem + C::kDataBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(append_row + 32);
    uint64_t *empty = full + C::kStages;
    // tcgen05 scores: chunk c's scores are in TMEM buffer c % kScoreBufs
    // (score_full: its MMAs completed; score_free: the four consumer warps read them)
    uint64_t *score_full = empty + C::kStages;
    uint64_t *score_free = score_full + C::kScoreBars / 2;
    int *tile_ok = reinterpret_cast<int *>(empty + C::kStages + C::kScoreBars);
    int *append_phys = tile_ok + C::kStages;  // the new row's block id: [0], and [1] for the V half (tcgen05)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(append_phys + 2);

    const int part = blockIdx.x;
    const int h = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- the work item ----
    // Normal item: sequence b = blockIdx.z, tokens [part * pt, ...) of it.
    // With prefix groups, z < num_groups * items_per_group names a prefix item
    // (group, member chunk): tokens [part * pt, ...) of the group's shared
    // range, read through the first member's table, for up to 8 / G members;
    // any other z names sequence b's own item: tokens from its group's shared
    // length on.
    bool pre = false;
    int b = blockIdx.z;  // the first member served
    int tb = b;          // the sequence whose block table is read
    int nmem = 1;        // members served (their query heads are the mma columns)
    int shared = 0;      // tokens of b's group read by the prefix items
    if constexpr (PREFIX) {
        const int n_pre_items = p.num_groups * p.items_per_group;
        if (b < n_pre_items) {
            pre = true;
            const int g = b / p.items_per_group;
            const int chunk = b - g * p.items_per_group;
            const int m_end = min((g + 1) * p.group_size, p.batch);
            tb = g * p.group_size;  // every member chunk reads the first member's blocks
            b = tb + chunk * p.members_per_item;
            nmem = min(p.members_per_item, m_end - b);
            if (nmem <= 0) return;  // member chunk past a short last group
            if (threadIdx.x == 0 && chunk == 0 && part == 0 && h == 0 && __ldg(p.prefix_lens + g) < 0)
                raise_flag(p.err_flag, PA_FLAG_BAD_LEN);
            shared = group_shared_tokens(p, g);
        } else {
            b -= n_pre_items;
            tb = b;
            shared = group_shared_tokens(p, b / p.group_size);
        }
    }
    const int L_raw = __ldg(p.seq_lens + b);
    const int L = clamp_len(L_raw, p);
    const int tok_begin = (pre ? 0 : shared) + part * p.part_tokens;
    const int tok_end = min(pre ? shared : L, tok_begin + p.part_tokens);
    const int n_tiles = tok_end > tok_begin ? (tok_end - tok_begin + kTileTokens - 1) / kTileTokens : 0;
    if (!pre && threadIdx.x == 0 && part == 0 && h == 0 && L != L_raw) raise_flag(p.err_flag, PA_FLAG_BAD_LEN);
    // Let the log-sum-exp reduce (launched as a programmatic dependent) get
    // scheduled while this grid's last wave runs; it waits for our results.
    if (SPLIT) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // Split: a sequence whose own tokens fit one partition (and share none) has
    // a single partial state -- that CTA writes the output itself, and the
    // reduce skips it.
    const bool direct = SPLIT && !pre && shared == 0 && L <= p.part_tokens;
    if (SPLIT && n_tiles == 0) {
        // Nothing to read.  An empty sequence has no partial states at all, so
        // its partition-0 CTA writes its zero rows; other empty partitions just end.
        if (!pre && part == 0 && L == 0)
            for (int x = threadIdx.x; x < p.group * HEAD_DIM; x += C::kThreads)
                p.out[((int64_t)b * p.num_q_heads + (int64_t)h * p.group) * HEAD_DIM + x] = 0.f;
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < C::kScoreBars / 2; ++s) {
            mbar_init(&score_full[s], 1);  // tcgen05.commit
            mbar_init(&score_free[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    if constexpr (C::kTc) {
        static_assert(kConsumerWarps == 4, "one 64-row MMA covers one tile per consumer warp");
        if (warp == kConsumerWarps + 1) {  // the MMA warp owns the TMEM columns
            tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
            tmem_relinquish();
            tc_fence_before();
        }
    }
    __syncthreads();
    uint32_t tmem = 0;
    if constexpr (C::kTc) {
        tc_fence_after();
        tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    }

    // Per consumer thread: softmax state of query-head columns 2t, 2t+1.
    const int gid = lane >> 2;  // mma group id
    const int tig = lane & 3;   // thread in group
#if PA_DECODE_SIMT_G1
    // CUDA-core state for a group of one query head (bf16): this lane's
    // HEAD_DIM/32 output dims, and the warp's running max and sum.
    float so[HEAD_DIM / 32];
#pragma unroll
    for (int k = 0; k < HEAD_DIM / 32; ++k) so[k] = 0.f;
    float sm = -INFINITY, sl = 0.f;
    // 2: CUDA cores only (the mma path compiled out; groups of one query head only)
    const bool simt = !FP8 && (PA_DECODE_SIMT_G1 == 2 || p.group == 1);
#endif
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float o[HEAD_DIM / 16][4];
#pragma unroll
    for (int mt = 0; mt < HEAD_DIM / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    // This CTA's query columns as mma B fragments (k = head dim, permuted; n =
    // column gid): column n is query head n % G of member b + n / G, zero from
    // nmem * G on.  Lane (gid, tig) holds dims 8 (4j + tig) .. +7, j < d / 32.
    auto load_q = [&](uint32_t (&qf)[HEAD_DIM / 16][2]) {
        const int G = p.group;
        if (gid < nmem * G) {
            const uint4 *qrow = reinterpret_cast<const uint4 *>(
                p.q + ((PREFIX ? (int64_t)(b + gid / G) * p.num_q_heads + (int64_t)h * G + gid % G
                               : (int64_t)b * p.num_q_heads + (int64_t)h * G + gid) *
                       HEAD_DIM));
#pragma unroll
            for (int j = 0; j < HEAD_DIM / 32; ++j) {
                const uint4 v = __ldg(qrow + 4 * j + tig);
                qf[2 * j][0] = v.x;
                qf[2 * j][1] = v.y;
                qf[2 * j + 1][0] = v.z;
                qf[2 * j + 1][1] = v.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < HEAD_DIM / 16; ++k) qf[k][0] = qf[k][1] = 0u;
        }
    };
    // fp8 pools: the power of two 2^qexp that puts the largest |q| of the CTA's
    // columns in [2^top, 2^(top+1)), clamped to [lo, hi] (0 for q = 0).  Every
    // warp that calls it gets the same value.
    auto fp8_q_exp = [&](const uint32_t (&qf)[HEAD_DIM / 16][2], int top, int lo, int hi) -> int {
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < HEAD_DIM / 16; ++k) {
            amax = fmaxf(amax, fmaxf(fabsf(bf16_lo_to_float(qf[k][0])), fabsf(bf16_hi_to_float(qf[k][0]))));
            amax = fmaxf(amax, fmaxf(fabsf(bf16_lo_to_float(qf[k][1])), fabsf(bf16_hi_to_float(qf[k][1]))));
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const int e = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xff) - 127 : top;
        return max(lo, min(hi, top - e));
    };

    if (warp == kConsumerWarps) {
        // ---------------- producer: block-table dereference + TMA ----------------
        // The whole warp walks the tiles so that block-table entries arrive 32 at a
        // time (one coalesced load per window, the next window loaded ahead).
        // P = kLanes lanes wait on the ring and issue copies in parallel:
        // lane k handles tiles k, k+P, k+2P, ... and therefore ring slots k, k+P, ...
        const int32_t *table = p.block_tables + (int64_t)tb * p.max_blocks;
        const int j_end = (tok_end + p.block_size - 1) / p.block_size;  // blocks this CTA reads
        int win = tok_begin / p.block_size;                             // first entry of the window
        int32_t cur = win + lane < j_end ? __ldg(table + win + lane) : -1;
        int32_t nxt = win + 32 + lane < j_end ? __ldg(table + win + 32 + lane) : -1;
        uint64_t policy = 0;
        if (lane < C::kLanes) {
            if (lane == 0) {
                prefetch_tensormap(&k_map);
                prefetch_tensormap(&v_map);
            }
            policy = l2_policy_evict_first();
        }
        int issued = 0;  // tiles issued by this lane's rounds (max over lanes below)
        bool stop = false;
        for (int i0 = 0; i0 < n_tiles; i0 += C::kLanes) {
            const int j0 = (tok_begin + i0 * kTileTokens) / p.block_size;
            if (j0 >= win + 32) {  // warp-uniform: slide the window
                win += 32;
                cur = nxt;
                nxt = win + 32 + lane < j_end ? __ldg(table + win + 32 + lane) : -1;
            }
            const int i = i0 + lane;
            const bool mine = lane < C::kLanes && i < n_tiles;
            const int tok0 = tok_begin + i * kTileTokens;
            const int j = mine ? tok0 / p.block_size : win;
            const int row = tok0 - j * p.block_size;
            // A tile is one slice of a block, or two whole 8-token blocks.
            const int idx = j - win;  // in [0, 32 + 2 * C::kLanes)
            const int32_t a_cur = __shfl_sync(0xffffffffu, cur, idx & 31);
            const int32_t a_nxt = __shfl_sync(0xffffffffu, nxt, idx & 31);
            const int32_t b_cur = __shfl_sync(0xffffffffu, cur, (idx + 1) & 31);
            const int32_t b_nxt = __shfl_sync(0xffffffffu, nxt, (idx + 1) & 31);
            const int64_t phys = idx < 32 ? a_cur : a_nxt;
            const int64_t phys2 = idx + 1 < 32 ? b_cur : b_nxt;
            const bool two_blocks = p.block_size < kTileTokens;
            const bool second = two_blocks && tok0 + p.block_size < tok_end;
            if (mine) {
                const int s = i % C::kStages;
                if (i >= C::kStages && !mbar_wait_bounded(&empty[s], ((i / C::kStages) - 1) & 1, p.err_flag)) {
                    stop = true;
                } else {
                    issued = i + 1;
                    if (phys < 0 || phys >= p.num_blocks || (second && (phys2 < 0 || phys2 >= p.num_blocks))) {
                        raise_flag(p.err_flag, PA_FLAG_BAD_BLOCK);
                        tile_ok[s] = 0;
                        mbar_arrive(&full[s]);
                    } else {
                        tile_ok[s] = 1;
                        const int y = (int)((phys * p.num_kv_heads + h) * p.block_size + row);
                        uint8_t *kdst = smem + C::k_off(s);
                        uint8_t *vdst = smem + C::v_off(s);
                        mbar_arrive_expect_tx(&full[s], two_blocks && !second ? C::kStageBytes / 2 : C::kStageBytes);
#pragma unroll
                        for (int bx = 0; bx < C::kBoxes; ++bx)
                            tma_load_2d(kdst + bx * C::kBoxBytes, &k_map, bx * C::kBoxCols, y, &full[s], policy);
#pragma unroll
                        for (int bx = 0; bx < C::kBoxes; ++bx)
                            tma_load_2d(vdst + bx * C::kBoxBytes, &v_map, bx * C::kBoxCols, y, &full[s], policy);
                        if (second) {  // rows 8..15 of the tile come from the next 8-token block
                            const int y2 = (int)((phys2 * p.num_kv_heads + h) * p.block_size);
#pragma unroll
                            for (int bx = 0; bx < C::kBoxes; ++bx)
                                tma_load_2d(kdst + bx * C::kBoxBytes + C::kBoxBytes / 2, &k_map, bx * C::kBoxCols, y2,
                                            &full[s], policy);
#pragma unroll
                            for (int bx = 0; bx < C::kBoxes; ++bx)
                                tma_load_2d(vdst + bx * C::kBoxBytes + C::kBoxBytes / 2, &v_map, bx * C::kBoxCols, y2,
                                            &full[s], policy);
                        }
                    }
                }
            }
            if (__any_sync(0xffffffffu, stop)) break;
        }
        // Drain: every issued tile has landed before the ring is reused or the CTA exits.
        // A tile is the last user of its slot when no tile one ring depth later was issued.
        const int issued_all = __reduce_max_sync(0xffffffffu, issued);
        if (lane < C::kLanes) {
            for (int i = lane; i < issued_all; i += C::kLanes)
                if (i + C::kStages >= issued_all && i < issued)
                    if (!mbar_wait_bounded(&full[i % C::kStages], (i / C::kStages) & 1, p.err_flag)) break;
        }
    } else if (C::kTc && warp == kConsumerWarps + 1) {
        if constexpr (C::kTc) {
            // ---------------- scores on the tensor cores (fp8 pools, head_dim 128) ----------------
            // q becomes the MMA's B operand: its 8 columns times 2^qexp (largest
            // |q| in [2^7, 2^8)) as two E4M3 terms, hi = E4M3(x) and lo =
            // E4M3(x - hi).  For a scaled bf16 element x with |x| >= 2^-2, x - hi
            // is a multiple of ulp_8(x) no larger than half ulp_4(x): at most 3
            // significant bits, an E4M3 normal, so hi + lo == x exactly.  Smaller
            // elements fall on the E4M3 subnormal grid (2^-9) and keep an error of
            // at most 2^-10, 2^-17 of the largest; a third term would be zero.
            uint32_t qf[HEAD_DIM / 16][2];
            load_q(qf);
            const int qexp = fp8_q_exp(qf, 7, -120, 126);
            const float up = __uint_as_float((uint32_t)(127 + qexp) << 23);
            const uint32_t qop = smem_addr(smem + C::kRingBytes + C::kStagingBytes);
#pragma unroll
            for (int j = 0; j < HEAD_DIM / 32; ++j) {
                const uint32_t w[4] = {qf[2 * j][0], qf[2 * j][1], qf[2 * j + 1][0], qf[2 * j + 1][1]};
                float x[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[2 * e] = bf16_lo_to_float(w[e]) * up;
                    x[2 * e + 1] = bf16_hi_to_float(w[e]) * up;
                }
                // dims 8 (4j + tig) .. +7 of column gid, in the 128-byte-swizzled row
                const uint32_t off = fp8_tile_offset(gid, 8 * (4 * j + tig));
#pragma unroll
                for (int t = 0; t < C::kQTerms; ++t) {
                    uint32_t codes[2] = {0u, 0u};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t pair = (uint32_t)__nv_cvt_float2_to_fp8x2(
                            make_float2(x[2 * e], x[2 * e + 1]), __NV_SATFINITE, __NV_E4M3);
                        codes[e >> 1] |= pair << ((e & 1) * 16);
                        const uint32_t back = e4m3x2_to_f16x2(pair);  // exact
                        x[2 * e] -= f16_lo_to_float(back);
                        x[2 * e + 1] -= f16_hi_to_float(back);
                    }
                    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(qop + t * 1024 + off), "r"(codes[0]),
                                 "r"(codes[1])
                                 : "memory");
                }
            }
            fence_proxy_async_smem();  // the MMAs read q through the async proxy
            __syncwarp();

            // Fused cache write, K half: the new token's K row is quantised into its
            // ring tile (and the pool) before the MMA of its chunk reads the tile.
            int i_new = -1;
            if (APPEND && !pre && L == L_raw && L > 0 && L - 1 >= tok_begin && L - 1 < tok_end) {
                i_new = (L - 1 - tok_begin) / kTileTokens;
                if (lane < HEAD_DIM / 8)
                    cp_async16(smem_addr(append_row + lane),
                               p.k_new + ((int64_t)b * p.num_kv_heads + h) * HEAD_DIM + lane * 8);
                if (lane == 0)
                    cp_async4(smem_addr(append_phys),
                              p.block_tables + (int64_t)b * p.max_blocks + (L - 1) / p.block_size);
                cp_async_commit();
            }

            // Instruction descriptor: fp32 scores, E4M3 A and B, both K-major, N = 8, M = 64.
            constexpr uint32_t kIdesc = (1u << 4) | ((8u >> 3) << 17) | ((64u >> 4) << 24);
            const uint32_t ring = smem_addr(smem);
            const int n_chunks = (n_tiles + kConsumerWarps - 1) / kConsumerWarps;
            int issued = 0;
            for (int c = 0; c < n_chunks; ++c) {
                const int buf = c % C::kScoreBufs;
                bool ok = true;
#pragma unroll
                for (int t = 0; t < kConsumerWarps; ++t) {
                    const int i = c * kConsumerWarps + t;
                    if (i < n_tiles) ok = ok && mbar_wait_bounded(&full[i % C::kStages], (i / C::kStages) & 1, p.err_flag);
                }
                if (c >= C::kScoreBufs)  // the consumers have read this buffer's previous chunk
                    ok = ok && mbar_wait_bounded(&score_free[buf], ((c / C::kScoreBufs) - 1) & 1, p.err_flag);
                if (!__all_sync(0xffffffffu, ok)) break;
                if (APPEND && i_new >= 0 && i_new / kConsumerWarps == c) {
                    cp_async_wait_all();
                    __syncwarp();
                    const int64_t phys = *reinterpret_cast<volatile int *>(append_phys);
                    if (lane < HEAD_DIM / 8) {
                        const uint2 q8 = bf16x8_to_e4m3x8(append_row[lane], p.k_inv_scale);
                        const int r = (L - 1 - tok_begin) - i_new * kTileTokens;
                        const uint32_t a = ring + C::k_off(i_new % C::kStages) + fp8_tile_offset(r, lane * 8);
                        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(q8.x), "r"(q8.y) : "memory");
                        if (phys >= 0 && phys < p.num_blocks)
                            reinterpret_cast<uint2 *>(p.k_pool)[((phys * p.num_kv_heads + h) * p.block_size +
                                                                 (L - 1) % p.block_size) *
                                                                    (HEAD_DIM / 8) +
                                                                lane] = q8;
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                }
                if (lane == 0) {
                    tc_fence_after();
                    // A: the chunk's four K tiles (64 token rows, contiguous in the ring);
                    // tile 4c + w is rows 16 w .. +15, in TMEM lane quarter w: warp w's.
                    const uint64_t a_desc = umma_desc_k_sw128(ring + C::k_off((c * kConsumerWarps) % C::kStages));
                    const uint64_t b_desc = umma_desc_k_sw128(qop);
                    const uint32_t d = tmem + 8 * buf;
#pragma unroll
                    for (int k = 0; k < HEAD_DIM / 32; ++k)
#pragma unroll
                        for (int t = 0; t < C::kQTerms; ++t)
                            umma_e4m3(d, a_desc + 2 * k, b_desc + (1024 >> 4) * t + 2 * k, kIdesc, k > 0 || t > 0);
                    umma_commit(&score_full[buf]);
                }
                __syncwarp();
                issued = c + 1;
            }
            // Every MMA has completed (a commit tracks all earlier MMAs of its thread)
            // before the ring is reused and TMEM is freed.
            if (issued > 0)
                mbar_wait_bounded(&score_full[(issued - 1) % C::kScoreBufs], ((issued - 1) / C::kScoreBufs) & 1,
                                  p.err_flag);
            if (APPEND && i_new >= 0) cp_async_wait_all();
        }
    } else {
        // ---------------- consumers ----------------
        uint32_t qf[HEAD_DIM / 16][2];
        load_q(qf);
        // fp8 pools run the mma in f16: q is scaled by a power of two 2^qexp so its
        // largest entry lands just below 2^14 (exact, well inside the f16 range);
        // 2^-qexp and the K dequantisation scale fold into the softmax scale.
        // (With tcgen05 scores the MMA warp scales q by its own 2^qexp, the same
        // value computed here.)
        float s_scale = p.scale_log2;
#if PA_DECODE_SIMT_G1
        // this lane's half of q (token lane/2 of a tile, dims of half lane & 1), bf16 pairs
        uint32_t sq[HEAD_DIM / 4];
        if (simt) {
            const uint4 *qh = reinterpret_cast<const uint4 *>(
                p.q + ((int64_t)b * p.num_q_heads + h) * HEAD_DIM + (lane & 1) * (HEAD_DIM / 2));
#pragma unroll
            for (int c = 0; c < HEAD_DIM / 16; ++c) {
                const uint4 v = __ldg(qh + c);
                sq[4 * c] = v.x;
                sq[4 * c + 1] = v.y;
                sq[4 * c + 2] = v.z;
                sq[4 * c + 3] = v.w;
            }
        }
#endif
        if constexpr (FP8) {
            const int qexp = C::kTc ? fp8_q_exp(qf, 7, -120, 126) : fp8_q_exp(qf, 13, -100, 100);
            const float down = __uint_as_float((uint32_t)(127 - qexp) << 23);
            if constexpr (!C::kTc) {
                const float up = __uint_as_float((uint32_t)(127 + qexp) << 23);
#pragma unroll
                for (int k = 0; k < HEAD_DIM / 16; ++k) {
                    qf[k][0] = pack_f16x2(bf16_lo_to_float(qf[k][0]) * up, bf16_hi_to_float(qf[k][0]) * up);
                    qf[k][1] = pack_f16x2(bf16_lo_to_float(qf[k][1]) * up, bf16_hi_to_float(qf[k][1]) * up);
                }
            }
            s_scale = p.scale_log2 * p.k_scale * down;
        }
        // Token row of mma row gid (gid+8 -> +8): this order keeps both the K
        // fragment loads and the V ldmatrix reads free of bank conflicts.
        // (fp8 with K read straight from the swizzled fp8 tile uses 0,2,4,6,1,3,5,7.)
        // (tcgen05 scores: TMEM row g is token g, so the order is the identity.)
        auto token_of = [](int g) {
            return C::kTc ? g : C::kDirect ? ((g & 3) << 1) | (g >> 2) : (g >> 1) | ((g & 1) << 2);
        };
        const int tau = token_of(gid);
        // ldmatrix row address pattern for V: matrix (lane>>3), row (lane&7).
        const int v_row = token_of(lane & 7) + (((lane >> 4) & 1) << 3);
        const int v_chunk_hi = (lane >> 3) & 1;

        // Fused cache write ("append, then attend"): the warp that owns the tile
        // holding position L-1 fetches the new token's K row (lanes 0..15) and
        // V row (lanes 16..31) up front, stores them to the pool, and patches
        // them into its staged tile before computing.  The block receiving the
        // token is owned by this sequence alone (copy-on-write), so no other
        // CTA reads that row.
        int i_new = -1;
        if (APPEND && !pre && L == L_raw && L > 0 && L - 1 >= tok_begin && L - 1 < tok_end) {
            const int it = (L - 1 - tok_begin) / kTileTokens;
            if (it % kConsumerWarps == warp) {
                i_new = it;
                const int c = lane & 15;
                if (c < HEAD_DIM / 8 && (!C::kTc || lane >= 16)) {  // tcgen05: the MMA warp writes K
                    const uint16_t *src = (lane < 16 ? p.k_new : p.v_new) +
                                          ((int64_t)b * p.num_kv_heads + h) * HEAD_DIM + c * 8;
                    cp_async16(smem_addr(append_row + lane), src);
                }
                if (lane == (C::kTc ? 16 : 0))
                    cp_async4(smem_addr(append_phys + (C::kTc ? 1 : 0)),
                              p.block_tables + (int64_t)b * p.max_blocks + (L - 1) / p.block_size);
                cp_async_commit();
            }
        }
        // This lane's share of the fused write at the tile that holds L-1: returns the
        // bf16 row chunk and the pool index of its 8 values (-1 if the block id is bad).
        auto append_fetch = [&](uint4 &row) -> int64_t {
            cp_async_wait_all();
            __syncwarp();
            const int64_t phys = *reinterpret_cast<volatile int *>(append_phys + (C::kTc ? 1 : 0));
            row = !C::kTc || lane >= 16 ? append_row[lane] : make_uint4(0u, 0u, 0u, 0u);
            if (phys < 0 || phys >= p.num_blocks) return -1;
            return ((phys * p.num_kv_heads + h) * p.block_size + (L - 1) % p.block_size) * (HEAD_DIM / 8) +
                   (lane & 15);
        };

        for (int i = warp; i < n_tiles; i += kConsumerWarps) {
            const int s = i % C::kStages;
            const int chunk = i / kConsumerWarps;  // tcgen05 scores: the chunk of four tiles
            const int sb = chunk % C::kScoreBufs;
            bool got = mbar_wait_bounded(&full[s], (i / C::kStages) & 1, p.err_flag);
            if constexpr (C::kTc)
                got = got && mbar_wait_bounded(&score_full[sb], (chunk / C::kScoreBufs) & 1, p.err_flag);
            if (!__all_sync(0xffffffffu, got)) break;
            float tc_s[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (C::kTc) {
                // The tile's 16 rows are in TMEM lanes 32 warp .. +15, this warp's quarter.
                tc_fence_after();
                tmem_ld_16x256b(tmem + ((uint32_t)(32 * warp) << 16) + 8 * sb, tc_s);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&score_free[sb]);
            }
            const int valid = min(kTileTokens, tok_end - (tok_begin + i * kTileTokens));
            if (tile_ok[s]) {
                uint32_t kbase = smem_addr(smem + C::k_off(s));
                uint32_t vbase = smem_addr(smem + C::v_off(s));
                uint32_t ring_k = kbase;  // fp8 direct-K: K stays in the ring until QK is done
                if constexpr (C::kDirect) {
                    // The fused cache write lands in the (swizzled) fp8 tile first, and in the pool.
                    if (APPEND && i == i_new) {
                        const int r = (L - 1 - tok_begin) - i_new * kTileTokens;
                        const int c = lane & 15;  // 8-byte piece of the 128-byte row
                        uint4 row;
                        const int64_t dst = append_fetch(row);
                        if (!C::kTc || lane >= 16) {  // tcgen05: the K half is the MMA warp's
                            const uint2 q8 = bf16x8_to_e4m3x8(row, lane < 16 ? p.k_inv_scale : p.v_inv_scale);
                            const uint32_t a = (lane < 16 ? kbase : vbase) + fp8_tile_offset(r, c * 8);
                            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(q8.x), "r"(q8.y) : "memory");
                            if (dst >= 0) reinterpret_cast<uint2 *>(lane < 16 ? p.k_pool : p.v_pool)[dst] = q8;
                        }
                        __syncwarp();
                    }
                } else if constexpr (FP8) {
                    // head_dim 64: the fused write lands in the unswizzled fp8 tile first.
                    if (APPEND && i == i_new) {
                        const int r = (L - 1 - tok_begin) - i_new * kTileTokens;
                        const int c = lane & 15;
                        uint4 row;
                        const int64_t dst = append_fetch(row);
                        if (c < HEAD_DIM / 8) {
                            const uint2 q8 = bf16x8_to_e4m3x8(row, lane < 16 ? p.k_inv_scale : p.v_inv_scale);
                            const uint32_t a = (lane < 16 ? kbase : vbase) + r * HEAD_DIM + c * 8;
                            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(q8.x), "r"(q8.y)
                                         : "memory");
                            if (dst >= 0) reinterpret_cast<uint2 *>(lane < 16 ? p.k_pool : p.v_pool)[dst] = q8;
                        }
                        __syncwarp();
                    }
                    // Expand K and V into this warp's 16-bit tiles (E4M3 -> f16 is exact),
                    // laid out like a TMA-swizzled bf16 tile so the code below is shared.
                    const uint32_t stg_k = smem_addr(smem + C::kRingBytes + warp * 2 * C::kTile16Bytes);
                    const uint32_t stg_v = stg_k + C::kTile16Bytes;
                    constexpr int kChunksPerRow = HEAD_DIM / 16;  // 16 fp8 values per 16-byte chunk
#pragma unroll
                    for (int x = lane; x < kTileTokens * kChunksPerRow; x += 32) {
                        const int r = x / kChunksPerRow;
                        const int c16 = x - r * kChunksPerRow;
#pragma unroll
                        for (int kv = 0; kv < 2; ++kv) {
                            const uint4 w = lds128((kv ? vbase : kbase) + x * 16);
                            const uint32_t dst = kv ? stg_v : stg_k;
                            const uint4 lo = e4m3x8_to_f16x8(w.x, w.y);
                            const uint4 hi = e4m3x8_to_f16x8(w.z, w.w);
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + tile_offset(r, 2 * c16)),
                                         "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w)
                                         : "memory");
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + tile_offset(r, 2 * c16 + 1)),
                                         "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
                                         : "memory");
                        }
                    }
                    if (APPEND && i == i_new) fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);  // the ring slot is free again
                    kbase = stg_k;
                    vbase = stg_v;
                }
                if (!C::kDirect && valid < kTileTokens) {
                    // Rows past the sequence end hold stale data: zero them so
                    // that P = 0 times V cannot produce NaN.  (fp8, head_dim 128
                    // masks them in registers instead, below.)
                    constexpr int kBoxes16 = HEAD_DIM / 64;  // boxes of the 16-bit tile
                    const int lines = (kTileTokens - valid) * kBoxes16;
                    for (int x = lane; x < lines * 8; x += 32) {
                        const int line = x >> 3;
                        const int r = valid + line / kBoxes16;
                        const int bx = line % kBoxes16;
                        const uint32_t a = vbase + bx * kBox16Bytes + r * 128 + ((x & 7) << 4);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u)
                                     : "memory");
                    }
                    __syncwarp();
                }
                if (APPEND && !FP8 && i == i_new) {
                    const int r = (L - 1 - tok_begin) - i_new * kTileTokens;  // row of L-1 in this tile
                    const int c = lane & 15;
                    uint4 row;
                    const int64_t dst = append_fetch(row);
                    if (c < HEAD_DIM / 8) {
                        const uint32_t a = (lane < 16 ? kbase : vbase) + tile_offset(r, c);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(row.x), "r"(row.y),
                                     "r"(row.z), "r"(row.w)
                                     : "memory");
                        if (dst >= 0) reinterpret_cast<uint4 *>(lane < 16 ? p.k_pool : p.v_pool)[dst] = row;
                    }
                    __syncwarp();
                }
#if PA_DECODE_SIMT_G1
                if (simt) {
                    // scores: lanes 2t and 2t+1 each dot half of token t's row with q
                    const int t = lane >> 1;
                    float acc = 0.f;
#pragma unroll
                    for (int c = 0; c < HEAD_DIM / 16; ++c) {
                        const uint4 kv = lds128(kbase + tile_offset(t, (lane & 1) * (HEAD_DIM / 16) + c));
                        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            acc = fmaf(bf16_lo_to_float(kw[e]), bf16_lo_to_float(sq[4 * c + e]), acc);
                            acc = fmaf(bf16_hi_to_float(kw[e]), bf16_hi_to_float(sq[4 * c + e]), acc);
                        }
                    }
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    const float sc = t < valid ? acc * s_scale : -INFINITY;
                    float mx = sc;
#pragma unroll
                    for (int off = 2; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    const float mn = fmaxf(sm, mx);
                    const float alpha = fast_exp2(sm - mn);
                    const float pt = fast_exp2(sc - mn);
                    float ps = pt;
#pragma unroll
                    for (int off = 2; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
                    sl = sl * alpha + ps;
                    sm = mn;
#pragma unroll
                    for (int k = 0; k < HEAD_DIM / 32; ++k) so[k] *= alpha;
                    // PV: this lane's HEAD_DIM/32 dims of every token row
#pragma unroll
                    for (int u = 0; u < kTileTokens; ++u) {
                        const float pu = __shfl_sync(0xffffffffu, pt, 2 * u);
                        if constexpr (HEAD_DIM == 128) {
                            uint32_t v0, v1;
                            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                         : "=r"(v0), "=r"(v1)
                                         : "r"(vbase + tile_offset(u, lane >> 1) + (lane & 1) * 8));
                            so[0] = fmaf(pu, bf16_lo_to_float(v0), so[0]);
                            so[1] = fmaf(pu, bf16_hi_to_float(v0), so[1]);
                            so[2] = fmaf(pu, bf16_lo_to_float(v1), so[2]);
                            so[3] = fmaf(pu, bf16_hi_to_float(v1), so[3]);
                        } else {
                            uint32_t v0;
                            asm volatile("ld.shared.u32 %0, [%1];"
                                         : "=r"(v0)
                                         : "r"(vbase + tile_offset(u, lane >> 2) + (lane & 3) * 4));
                            so[0] = fmaf(pu, bf16_lo_to_float(v0), so[0]);
                            so[1] = fmaf(pu, bf16_hi_to_float(v0), so[1]);
                        }
                    }
                } else
#endif
                {
                // ---- S^T = K Q^T ----
                float sacc[4] = {tc_s[0], tc_s[1], tc_s[2], tc_s[3]};  // tcgen05: already computed
#pragma unroll
                for (int j = 0; j < (C::kTc ? 0 : HEAD_DIM / 32); ++j) {
                    uint4 ka, kb;
                    if constexpr (C::kDirect) {
                        // 8 fp8 codes (dims 32j+8t .. +7) of rows tau and tau+8, expanded in registers
                        uint32_t a0, a1, b0, b1;
                        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                     : "=r"(a0), "=r"(a1)
                                     : "r"(ring_k + fp8_tile_offset(tau, 32 * j + 8 * tig)));
                        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                     : "=r"(b0), "=r"(b1)
                                     : "r"(ring_k + fp8_tile_offset(tau + 8, 32 * j + 8 * tig)));
                        ka = e4m3x8_to_f16x8(a0, a1);
                        kb = e4m3x8_to_f16x8(b0, b1);
                    } else {
                        const int c = 4 * j + tig;
                        ka = lds128(kbase + tile_offset(tau, c));
                        kb = lds128(kbase + tile_offset(tau + 8, c));
                    }
                    mma_16816<FP8>(sacc, ka.x, kb.x, ka.y, kb.y, qf[2 * j][0], qf[2 * j][1]);
                    mma_16816<FP8>(sacc, ka.z, kb.z, ka.w, kb.w, qf[2 * j + 1][0], qf[2 * j + 1][1]);
                }
                // sacc: (token tau, col 2t), (tau, 2t+1), (tau+8, 2t), (tau+8, 2t+1)
                const float s0 = tau < valid ? sacc[0] * s_scale : -INFINITY;
                const float s1 = tau < valid ? sacc[1] * s_scale : -INFINITY;
                const float s2 = tau + 8 < valid ? sacc[2] * s_scale : -INFINITY;
                const float s3 = tau + 8 < valid ? sacc[3] * s_scale : -INFINITY;
                float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
                const float a0 = fast_exp2(m_run[0] - mn0), a1 = fast_exp2(m_run[1] - mn1);
                m_run[0] = mn0;
                m_run[1] = mn1;
                const float p0 = fast_exp2(s0 - mn0), p1 = fast_exp2(s1 - mn1);
                const float p2 = fast_exp2(s2 - mn0), p3 = fast_exp2(s3 - mn1);
                l_run[0] = l_run[0] * a0 + (p0 + p2);
                l_run[1] = l_run[1] * a1 + (p1 + p3);
                if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
                    for (int mt = 0; mt < HEAD_DIM / 16; ++mt) {
                        o[mt][0] *= a0;
                        o[mt][1] *= a1;
                        o[mt][2] *= a0;
                        o[mt][3] *= a1;
                    }
                }
                // ---- P^T as B fragments: hi + lo bf16 parts (fp8 pools: one f16 part) ----
                constexpr bool kPLo = !FP8 || PA_DECODE_FP8_P_LO;
                uint32_t h01, h23, l01 = 0u, l23 = 0u;
                if constexpr (FP8) {
                    h01 = pack_f16x2(p0, p1);
                    h23 = pack_f16x2(p2, p3);
                    if (kPLo) {
                        l01 = pack_f16x2(p0 - f16_lo_to_float(h01), p1 - f16_hi_to_float(h01));
                        l23 = pack_f16x2(p2 - f16_lo_to_float(h23), p3 - f16_hi_to_float(h23));
                    }
                } else {
                    h01 = pack_bf16x2(p0, p1);
                    h23 = pack_bf16x2(p2, p3);
                    l01 = pack_bf16x2(p0 - bf16_lo_to_float(h01), p1 - bf16_hi_to_float(h01));
                    l23 = pack_bf16x2(p2 - bf16_lo_to_float(h23), p3 - bf16_hi_to_float(h23));
                }
                const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
                const uint32_t bl0 = kPLo ? movmatrix_trans(l01) : 0u, bl1 = kPLo ? movmatrix_trans(l23) : 0u;
                // ---- O^T += V^T P^T ----
                if constexpr (C::kDirect) {
                    // V^T fragments straight from the swizzled fp8 tile.  ldmatrix.trans on
                    // 16-bit pairs hands each lane, per register, the codes of tokens
                    // (k, k+1) for two neighbouring dims; split into an even-dim and an
                    // odd-dim m-tile and widened to f16 they are the A fragments.  M-tile
                    // 2c+e holds dims 32c + 2r + e (row r < 8) and 32c + 16 + 2(r-8) + e.
                    // Matrices: rows tau (+8 for 1, 3) of byte columns 32c (+16 for 2, 3).
                    const int mtx = lane >> 3;
                    const uint32_t v_addr = vbase + fp8_tile_offset(token_of(lane & 7) + ((mtx & 1) << 3), (mtx >> 1) << 4);
                    const bool partial = valid < kTileTokens;
                    uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;  // tokens past the end read as 0
                    if (partial) {
                        const int k0 = token_of(2 * tig), k1 = token_of(2 * tig + 1);
                        keep_lo = (k0 < valid ? 0x0000ffffu : 0u) | (k1 < valid ? 0xffff0000u : 0u);
                        keep_hi = (k0 + 8 < valid ? 0x0000ffffu : 0u) | (k1 + 8 < valid ? 0xffff0000u : 0u);
                    }
#pragma unroll
                    for (int c = 0; c < HEAD_DIM / 32; ++c) {
                        uint32_t r0, r1, r2, r3;
                        // + 32c bytes: the swizzle only permutes 16-byte chunks within 128, so
                        // chunk (2c + hi) ^ (row & 7) is reached by xor-ing 2c into the chunk bits
                        ldmatrix_x4_trans(v_addr ^ ((uint32_t)(2 * c) << 4), r0, r1, r2, r3);
                        const uint32_t m[4] = {r0, r2, r1, r3};  // a0: tokens k, rows < 8; a1: rows >= 8; a2, a3: +8 tokens
                        uint32_t ev[4], od[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            e4m3x4_to_f16x4(__byte_perm(m[q], 0u, 0x3120), ev[q], od[q]);
                            if (partial) {
                                ev[q] &= q < 2 ? keep_lo : keep_hi;
                                od[q] &= q < 2 ? keep_lo : keep_hi;
                            }
                        }
                        mma_16816<FP8>(o[2 * c], ev[0], ev[1], ev[2], ev[3], bh0, bh1);
                        if (kPLo) mma_16816<FP8>(o[2 * c], ev[0], ev[1], ev[2], ev[3], bl0, bl1);
                        mma_16816<FP8>(o[2 * c + 1], od[0], od[1], od[2], od[3], bh0, bh1);
                        if (kPLo) mma_16816<FP8>(o[2 * c + 1], od[0], od[1], od[2], od[3], bl0, bl1);
                    }
                    // K and V have left the ring: hand the slot back to the producer.
                    if (APPEND && i == i_new) fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);
                } else {
#pragma unroll
                    for (int mt = 0; mt < HEAD_DIM / 16; ++mt) {
                        uint32_t a0r, a1r, a2r, a3r;
                        ldmatrix_x4_trans(vbase + tile_offset(v_row, 2 * mt + v_chunk_hi), a0r, a1r, a2r, a3r);
                        mma_16816<FP8>(o[mt], a0r, a1r, a2r, a3r, bh0, bh1);
                        if (kPLo) mma_16816<FP8>(o[mt], a0r, a1r, a2r, a3r, bl0, bl1);
                    }
                }
                }
                if (!FP8 && (valid < kTileTokens || (APPEND && i == i_new))) fence_proxy_async_smem();
            } else if (FP8) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);  // skipped tile: release it here
            }
            if constexpr (!FP8) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
        }
        if (APPEND && i_new >= 0) cp_async_wait_all();  // never leave copies in flight
        // Row sums over this warp's tokens (lanes with the same tig share a column).
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
            l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
        }
    }

    // ---------------- merge the warps' states (ring memory is free now) ----------------
    __syncthreads();
    if constexpr (C::kTc) {
        if (warp == kConsumerWarps + 1) {  // every MMA and TMEM read is complete
            tc_fence_after();
            tmem_dealloc(tmem, C::kTmemCols);
        }
    }
    float *mo = reinterpret_cast<float *>(smem);                      // [W][8][kMergeStride]
    float *mm = mo + kConsumerWarps * 8 * C::kMergeStride;            // [W][8]
    float *ml = mm + kConsumerWarps * 8;                              // [W][8]
    if (warp < kConsumerWarps) {
        const int gid = lane >> 2, tig = lane & 3;
        float *w0 = mo + (warp * 8 + 2 * tig) * C::kMergeStride;
        float *w1 = w0 + C::kMergeStride;
#pragma unroll
        for (int mt = 0; mt < HEAD_DIM / 16; ++mt) {
            // dims of rows gid and gid + 8 of m-tile mt (fp8 head_dim 128: even/odd-dim m-tiles)
            const int d0 = C::kDirect ? 32 * (mt >> 1) + 2 * gid + (mt & 1) : 16 * mt + gid;
            const int d1 = C::kDirect ? d0 + 16 : d0 + 8;
            w0[d0] = o[mt][0];
            w1[d0] = o[mt][1];
            w0[d1] = o[mt][2];
            w1[d1] = o[mt][3];
        }
        if (gid == 0) {
            mm[warp * 8 + 2 * tig] = m_run[0];
            mm[warp * 8 + 2 * tig + 1] = m_run[1];
            ml[warp * 8 + 2 * tig] = l_run[0];
            ml[warp * 8 + 2 * tig + 1] = l_run[1];
        }
#if PA_DECODE_SIMT_G1
        if (simt) {  // column 0 holds the CUDA-core state
            __syncwarp();
#pragma unroll
            for (int k = 0; k < HEAD_DIM / 32; ++k) mo[(warp * 8) * C::kMergeStride + lane * (HEAD_DIM / 32) + k] = so[k];
            if (lane == 0) {
                mm[warp * 8] = sm;
                ml[warp * 8] = sl;
            }
        }
#endif
    }
    __syncthreads();
    const int G = p.group;
    // Column n is query head n % G of member b + n / G; in the split variant
    // its partial state goes to slot `slot` of that row.
    const int slot = PREFIX && !pre ? p.num_parts + part : part;
    for (int x = threadIdx.x; x < (PREFIX ? nmem : 1) * G * HEAD_DIM; x += C::kThreads) {
        const int n = x / HEAD_DIM;
        const int d = x - n * HEAD_DIM;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mm[w * 8 + n]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float f = fast_exp2(mm[w * 8 + n] - M);
                num += f * mo[(w * 8 + n) * C::kMergeStride + d];
                den += f * ml[w * 8 + n];
            }
        }
        const int64_t row = PREFIX ? (int64_t)(b + n / G) * p.num_q_heads + (int64_t)h * G + n % G
                                   : (int64_t)b * p.num_q_heads + (int64_t)h * G + n;
        if (FP8) num *= p.v_scale;
        if (SPLIT && !direct) {
            p.part_o[(row * p.num_slots + slot) * HEAD_DIM + d] = den == 0.f ? 0.f : num / den;
            if (d == 0) {
                p.part_ml[(row * p.num_slots + slot) * 2] = M;
                p.part_ml[(row * p.num_slots + slot) * 2 + 1] = den;
            }
        } else {
            // No tokens: a zero row.  A NaN read from an attended row stays NaN.
            p.out[row * HEAD_DIM + d] = den == 0.f ? 0.f : num / den;
        }
    }
}

// Log-sum-exp merge of the partial states of one (sequence, query head):
//   out = sum_p 2^(m_p - M) l_p o_p / sum_p 2^(m_p - M) l_p,  M = max_p m_p,
// over the shared-prefix slots [0, n_pre) and the sequence's own slots
// [s0, s0 + n_own).  Rows with a single partial state were written by the
// decode itself and are skipped.  Four warps split the slots; each lane owns
// HEAD_DIM/32 output dims.
constexpr int kReduceThreads = 128;

template <int HEAD_DIM, bool PREFIX>
__global__ void __launch_bounds__(kReduceThreads) lse_reduce_kernel(const DecodeParams p) {
    constexpr int kWarps = kReduceThreads / 32;
    constexpr int V = HEAD_DIM / 32;  // dims per lane: 4 or 2
    __shared__ float s_max[kWarps];
    __shared__ float s_den[kWarps];
    __shared__ float s_acc[kWarps][HEAD_DIM];
    const int hq = blockIdx.x;
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int shared = PREFIX ? group_shared_tokens(p, b / p.group_size) : 0;
    const int L = clamp_len(__ldg(p.seq_lens + b), p);
    const int n_pre = parts_of(shared, p.part_tokens);
    const int n_own = parts_of(L - shared, p.part_tokens);
    const int n = n_pre + n_own;
    // Launched as a programmatic dependent of the decode grid, so it may start
    // before the decode has finished.  Which rows need a merge follows from the
    // lengths alone (the decode does not write them): rows written by the
    // decode itself leave at once, without holding a slot through the decode's
    // last wave (0.5 % less time per call on the Llama-3-8B-shaped workload);
    // the others wait for the decode's results.
    if (n_pre == 0 && n_own <= 1) return;  // written by the decode
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int s0 = PREFIX ? p.num_parts : 0;
    auto slot_of = [&](int k) { return k < n_pre ? k : s0 + k - n_pre; };
    const int64_t row = (int64_t)b * p.num_q_heads + hq;
    const float2 *ml = reinterpret_cast<const float2 *>(p.part_ml) + row * p.num_slots;
    const float *po = p.part_o + row * p.num_slots * HEAD_DIM + lane * V;

    float M = -INFINITY;
    for (int i = threadIdx.x; i < n; i += kReduceThreads) M = fmaxf(M, __ldg(&ml[slot_of(i)].x));
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) s_max[warp] = M;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_max[w]);

    float acc[V];
#pragma unroll
    for (int k = 0; k < V; ++k) acc[k] = 0.f;
    float den = 0.f;
    if (M != -INFINITY) {
#pragma unroll 4
        for (int i = warp; i < n; i += kWarps) {
            const int64_t s = slot_of(i);
            const float2 mlv = __ldg(&ml[s]);
            const float w = fast_exp2(mlv.x - M) * mlv.y;
            if constexpr (V == 4) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(po + s * HEAD_DIM));
                acc[0] += w * v.x;
                acc[1] += w * v.y;
                acc[2] += w * v.z;
                acc[3] += w * v.w;
            } else {
                const float2 v = __ldg(reinterpret_cast<const float2 *>(po + s * HEAD_DIM));
                acc[0] += w * v.x;
                acc[1] += w * v.y;
            }
            den += w;
        }
    }
#pragma unroll
    for (int k = 0; k < V; ++k) s_acc[warp][lane * V + k] = acc[k];
    if (lane == 0) s_den[warp] = den;
    __syncthreads();
    for (int x = threadIdx.x; x < HEAD_DIM; x += kReduceThreads) {
        float num = 0.f, dd = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            num += s_acc[w][x];
            dd += s_den[w];
        }
        p.out[row * HEAD_DIM + x] = dd == 0.f ? 0.f : num / dd;  // no tokens: zeros; a NaN stays NaN
    }
}

}  // namespace
}  // namespace pa

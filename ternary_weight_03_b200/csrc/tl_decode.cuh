// tl_decode.cuh -- a batch of decode-shaped ternary layers (M = 1..8 tokens
// each; 2-bit or 1.6-bit packing) in ONE persistent launch:
//   for every layer l:  Y_l[m][n] = fp16_rn(alpha_l * sum_k T_l[n][k] X_l[m][k]).
//
// Decoding streams every packed weight once and is bound by memory bandwidth
// ("Pith review of Spectra 1.1", "What carries the argument"), so the kernel
// is built around keeping HBM busy: one CTA per SM walks a queue of work
// items (layer, 256-row tile, K-part) across all layers of the batch, and the
// instructions spent per packed byte must stay far below what the SM can
// issue.  Two tensor-core engines, chosen per item by its token count:
//
//  * M <= 2, exact integer engine (mma.sync m16n8k32, u8 x u8 -> s32).  A
//    holds the 2-bit digits d = t + 1 of one digit position j of every byte
//    of a packed word, left in place (one AND: values d * 4^j), with one
//    accumulator per position.  B holds the activations as exact integers:
//    every binary16 x has x * 2^24 integral and |x * 2^24| < 2^40, so
//    z = x * 2^24 + 2^40 is a 41-bit natural number, stored as six u8 planes
//    (B columns), next to one column of ones.  Then
//      sum_k t_k x_k * 2^24 = sum_p 256^p S_p - 2^40 S_1 - Q,
//    with S_p = sum_k d_k u_p(k) (MMA columns, exact in s32 per item),
//    S_1 = sum_k d_k (the ones column) and Q = sum_k x_k 2^24 (exact).  The
//    sum is exact in int64, so a layer's result is the single rounding
//    fp16_rn(alpha * V * 2^-24) whatever the split of K.
//  * M >= 3, fp16 engine (mma.sync m16n8k16, fp16 -> fp32): masking digit
//    position j of every byte of a packed word leaves the digits as subnormal
//    halves d * 2^(2j-24) (one AND per register); one accumulator per digit
//    position, combined with exact power-of-two scales; sum_k x_k is
//    subtracted at the end (d = t + 1).
//  * Base 3 (1.6-bit, decode2_kernel<16>): the same roles and engines, with
//    the digits' quotients floor(v / 3^p) taken two bytes per IMAD in 16-bit
//    lanes (see "base 3" below): the integer engine multiplies the quotients
//    themselves against telescoped activations, the fp16 engine the digits.
//
// Weights arrive by TMA in boxes of 256 rows x 128 bytes (512 trits per row
// at 2 bits, 640 at 1.6 bits) with the 128-byte swizzle, one box per stage.
// A consumer lane (g, c) reads 16-byte chunk 4v + c of rows g and g + 8 of a
// 16-row tile; MMA row g is physical row pi(g) = ((g & 1) << 2) | (g >> 1),
// so the two rows of every quarter-warp differ in bit 2 and each LDS.128
// touches every bank once.
//
// Activations go into the B layout of their engine once per (layer, stage),
// not once per item: every warp except the producer first converts such
// units (unit u by converting warp u mod their number) into the workspace
// and counts them per layer; a stage's converted operands then arrive by one
// bulk copy next to its weights.  The first item of every CTA (so no CTA
// starts by waiting for others) and items of layers flagged as reading an
// earlier layer's output (their X is written during this launch) for the
// integer engine are converted per item instead, from X in global memory, by
// stager warps; such layers for the fp16 engine convert their X once, after
// the layers they read are complete, by the stagers of their items.  A
// dependent layer waits only for the earlier layers whose Y overlaps its X.
//
// Warp roles of a CTA (768 threads):
//  * warp 0, producer: issues each stage's copies into a ring and queues items
//    (items come from a workspace counter, fetched one item ahead);
//  * warps 1..3, stagers (warp 1 + i owns the ring slots s with s mod 3 = i);
//  * warps 4..7, epilogues (item i goes to warp 4 + i mod 4, or mod 2 when
//    only two partial buffers fit): sum the consumer
//    partials of an item in a fixed order, then write Y, or a partial of a
//    split tile to the workspace where the last part to arrive adds the parts
//    in part order;
//  * warps 8..23, consumers: warp w takes row tiles 2 (w & 7) and 2 (w & 7) + 1
//    and the half w >> 3 of every stage (chunks 4 (w >> 3) .. +3).
// The cross-warp and cross-CTA sums follow the pages' shared-memory tree
// reduction of per-warp partials (Figure 11 caption text on appendix G.4 of the
// same page), in a fixed order.  All waits are bounded; a timeout sets the
// device error word.  The last CTA to finish resets the workspace counters, so
// they stay zero between launches.
#pragma once
#include <cuda.h>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>
#include "tl_common.cuh"
#include "tl_sm100.cuh"

namespace tlk {

constexpr int kDkTiles = 16;                             // 16-row MMA tiles per item
constexpr int kDkRows = 16 * kDkTiles;                   // 256 weight rows per item
constexpr int kDkStageW = 128;                           // packed bytes per row per stage (one box)
constexpr int kDkWords = kDkStageW / 4;                  // 32 packed words per row per stage
constexpr int kDkWBytes = kDkRows * kDkStageW;           // 32 KB of weights per stage
constexpr int kDkConsumers = 16;
constexpr int kDkStagers = 3;
constexpr int kDkEpilogues = 4;
constexpr int kDkFirstEpi = 1 + kDkStagers;
constexpr int kDkFirstCons = kDkFirstEpi + kDkEpilogues;
constexpr int kDkWarps = kDkFirstCons + kDkConsumers;  // 24
constexpr int kDkThreads = 32 * kDkWarps;              // 768
constexpr int kDkMaxStages = 6;
constexpr int kDkQueue = 16;
constexpr int kDkMaxPartBufs = 4;  // consumer -> epilogue buffers (2 when large, in long launches)
constexpr int kDkImmaMaxM = 2;                          // exact integer engine up to 2 tokens
constexpr int kDkRefSms = 148;                          // scheduling reference: SMs of a B200
constexpr int kDkMaxItemStages = 64;                    // s32 sums of an item stay exact
constexpr uint32_t kDkSmemBudget = 232448u;             // 227 KB
constexpr int kDkMetaBytes = 64;                        // per stage: per-token offsets, first

// Workspace counters (u32 words of the 256-byte header).
constexpr int kDkCtrDone = 2;       // CTAs that have finished
constexpr int kDkCtrItems = 3;      // items handed out beyond the first 2 gridDim.x
constexpr int kDkCtrUnitsDone = 5;  // CTAs whose conversion units are all written

// Activations per stage: 128 packed bytes of 4 (2-bit) or 5 (1.6-bit) trits.
__host__ __device__ constexpr int dk_trits(int fmt) { return fmt == 2 ? 4 * kDkStageW : 5 * kDkStageW; }
// Bytes of converted B operands of one stage of a layer with M tokens: the
// integer engine needs one byte per activation and column of a group of 8
// (2 groups at M = 2), the fp16 engine 2 bytes per activation and token
// (tokens rounded up to even).
__host__ __device__ constexpr uint32_t dk_stage_b(int fmt, int M) {
    return M <= 2 ? 8u * (uint32_t)dk_trits(fmt) * (uint32_t)M
                  : 2u * (uint32_t)dk_trits(fmt) * (uint32_t)(M + (M & 1));
}
// The largest stage of a batch whose layers have at most maxM tokens.
__host__ __device__ constexpr uint32_t dk_slot_b(int fmt, int maxM) {
    return dk_stage_b(fmt, maxM < 2 ? maxM : 2) > dk_stage_b(fmt, maxM) ? dk_stage_b(fmt, maxM < 2 ? maxM : 2)
                                                                      : dk_stage_b(fmt, maxM);
}
// Consumer -> epilogue buffer: [token][warp][tile][row] of int64 (M <= 2) or fp32.
__host__ __device__ constexpr uint32_t dk_part_bytes(int maxM) {
    return (maxM <= 1 ? 4096u : 8192u) > 2048u * (uint32_t)maxM ? (maxM <= 1 ? 4096u : 8192u)
                                                                 : 2048u * (uint32_t)maxM;
}

// One work item as the producer reads it (96 bytes): everything the CTA's
// roles need, so no lookup chain stands between items.
struct DkItemRec {
    const uint16_t *X;
    uint16_t *Y;
    const uint8_t *B;  // converted operands of the layer ([meta][B] per stage), or null
    int64_t part_off;  // first 8-byte partial slot of the item's layer
    float alpha;
    int layer;         // low 16 bits: the layer (its tensor map); high 16 bits: the
                       // layer whose conversion of X it uses (its ready counter)
    int tile, part, s0, s1;
    int M, K, N, ldx, ldy;
    int parts;         // K-parts per tile of the layer
    int tile_begin;    // global index of the layer's first tile
    int deps;          // 0: X is final at the start; else (lo << 16) | (hi + 1): X is
                       // read once layers lo .. hi (the earlier layers whose Y overlaps
                       // it) have stored all their outputs
    int need;          // conversion units of X (stages x M) when B is given, else 0
    int bstride;       // bytes per stage of B (64 + dk_stage_b(M))
    int flags;         // kDkItemSwiglu, kDkItemCoop
    int pad_[3];
};
static_assert(sizeof(DkItemRec) == 112, "item record is seven 16-byte loads");
// DkItemRec.flags: X rows hold [gate | up] halves (SwiGLU input); X is written
// by earlier layers and converted into B once, after they complete, by the
// stagers of whichever CTAs hold the layer's items (units claimed from a
// per-layer counter), instead of on chip by every item.
constexpr int kDkItemSwiglu = 1;
constexpr int kDkItemCoop = 2;

// One conversion unit: one stage of one token of one layer.
struct DkUnitRec {
    const uint16_t *X;  // the layer's activations
    uint8_t *dst;       // [meta][B] of (layer, stage)
    int layer, stage, m, M, K, ldx;
    int pad_[2];
};
static_assert(sizeof(DkUnitRec) == 48, "unit record is three 16-byte loads");

// Workspace layout (every region 256-byte aligned):
//   header  : 64 u32 counters (kDkCtr*)
//   maps    : count x CUtensorMap
//   items   : total_items x DkItemRec
//   units   : total_units x DkUnitRec
//   ready   : count x u32, conversion units written per layer; then count x u32,
//             final tiles per layer; count x u32, tiles per layer; count x u32,
//             conversion units claimed per layer (kDkItemCoop)
//   tiles   : total_tiles x u32, parts of each tile that have arrived
//   partials: 8-byte partial sums of split tiles (int64 for M <= 2, double above)
//   staged  : converted operands, per layer stages x (64 + dk_stage_b(M)) bytes
struct DkWsLayout {
    size_t maps, items, units, ready, tiles, partials, staged, total;
    DkWsLayout(int count, int total_items, int total_units, int total_tiles, int64_t slots,
               int64_t staged_bytes) {
        auto up = [](size_t v) { return (v + 255u) & ~(size_t)255u; };
        maps = 256;
        items = up(maps + (size_t)count * sizeof(CUtensorMap));
        units = up(items + (size_t)total_items * sizeof(DkItemRec));
        ready = up(units + (size_t)total_units * sizeof(DkUnitRec));
        tiles = up(ready + (size_t)count * 16u);
        partials = up(tiles + (size_t)total_tiles * 4u);
        staged = up(partials + (size_t)slots * 8u);
        total = up(staged + (size_t)staged_bytes);
    }
};

struct DkArgs {
    uint32_t *ctr;
    const CUtensorMap *maps;
    const DkItemRec *items;
    const DkUnitRec *units;
    uint32_t *ready;
    uint32_t *lfinal;        // final tiles per layer (batches with dependencies)
    const uint32_t *ltiles;  // tiles per layer
    uint32_t *claim;         // conversion units claimed per layer (kDkItemCoop)
    uint32_t *tile_ctr;
    int64_t *partials;
    int count;
    int total_items;
    int total_units;
    int maxM;
    int chained;  // 1: some layer reads an earlier layer's output; 2: and one has a SwiGLU input
    int drop_arrive;  // failure-detection hook (debug library only), else 0
    int wide;         // four consumer -> epilogue buffers even for large partials
};

struct DkQEntry {
    uint16_t *Y;
    const uint16_t *X;
    int64_t part_off;
    float alpha;
    int item;  // -1: no more items
    int tile, part, s0, s1, M, K, N, ldx, ldy, parts, tile_begin;
    int pre;      // 1: converted operands arrive with the weights; 0: a stager converts X
    int chained;  // X is written by earlier layers of this launch
    int swiglu;   // X rows hold [gate | up]; the input is silu(gate) * up
    int layer;    // the item's layer
    int coop;     // the stagers first help convert the layer's X into B (kDkItemCoop)
};

struct DkLayout {
    uint32_t ns, nbufs, slot_b, parts, w_off, st_off, part_off, q_off, bar_off, total;
    __host__ __device__ DkLayout(int fmt, int maxM, bool wide) {
        slot_b = dk_slot_b(fmt, maxM) + kDkMetaBytes;  // [meta][B]
        parts = dk_part_bytes(maxM);
        nbufs = parts <= 8192u || wide ? (uint32_t)kDkMaxPartBufs : 2u;
        const uint32_t per_stage = (uint32_t)kDkWBytes + slot_b;
        const uint32_t fixed = nbufs * parts + kDkQueue * (uint32_t)sizeof(DkQEntry) +
                               8u * (3u * kDkMaxStages + 2u * kDkQueue + 2u * kDkMaxPartBufs) +
                               16u + 4u * kDkQueue + 1024u;  // counter, ready words, base slack
        const uint32_t n = (kDkSmemBudget - fixed) / per_stage;
        ns = n > (uint32_t)kDkMaxStages ? (uint32_t)kDkMaxStages : n;  // >= 3 for maxM <= 8
        w_off = 0;
        st_off = ns * (uint32_t)kDkWBytes;
        part_off = st_off + ns * slot_b;
        q_off = part_off + nbufs * parts;
        bar_off = (q_off + kDkQueue * (uint32_t)sizeof(DkQEntry) + 7u) & ~7u;
        total = bar_off + 8u * (3u * ns + 2u * kDkQueue + 2u * nbufs) + 16u + 4u * kDkQueue + 1024u;
    }
};

template <typename R, int N16>
__device__ __forceinline__ R dk_load_rec(const R *base, int idx) {
    const uint4 *p = reinterpret_cast<const uint4 *>(base + idx);
    uint4 v[N16];
#pragma unroll
    for (int i = 0; i < N16; ++i) v[i] = __ldg(p + i);
    R r;
    memcpy(&r, v, sizeof(r));
    return r;
}

__device__ __forceinline__ void dk_bulk_load(void *smem_dst, const void *src, uint32_t bytes,
                                             uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void dk_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ uint32_t dk_ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Orders this thread's generic-proxy accesses to global memory with its
// async-proxy (bulk copy) accesses.
__device__ __forceinline__ void dk_fence_proxy_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ bool dk_warp_wait(uint64_t *bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ bool dk_next_item(const DkQEntry *queue, uint64_t *qfull,
                                             uint64_t *qempty, int &qi, DkQEntry &e) {
    const int q = qi % kDkQueue;
    if (!dk_warp_wait(&qfull[q], (uint32_t)(qi / kDkQueue) & 1u)) return false;
    e = queue[q];
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&qempty[q]);
    ++qi;
    return e.item >= 0;
}
// Lane 0 spins (bounded) until *p >= target, or until *all_p >= all_target
// when all_p is given (then *all_seen is set); false on a timeout.  The
// result is the same in every lane.
__device__ __forceinline__ bool dk_wait_count(const uint32_t *p, uint32_t target,
                                              const uint32_t *all_p, uint32_t all_target,
                                              bool *all_seen) {
    bool good = true, all = false;
    if ((threadIdx.x & 31) == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (true) {
            // both counters are read before either is tested (one round trip per poll)
            const uint32_t va = all_p ? dk_ld_acquire(all_p) : 0u;
            const uint32_t vp = dk_ld_acquire(p);
            if (all_p && va >= all_target) {
                all = true;
                break;
            }
            if (vp >= target) break;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicOr(&g_error_word, kErrTimeout);
                good = false;
                break;
            }
            __nanosleep(32);
        }
    }
    all = __shfl_sync(0xffffffffu, all ? 1 : 0, 0) != 0;
    if (all_seen && all) *all_seen = true;
    return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
}

// Lane 0 spins (bounded) until the shared word holds `item`; the result is the
// same in every lane, and the producer's view of global memory (it saw the
// earlier layers complete) is ordered before this warp's reads that follow.
__device__ __forceinline__ bool dk_wait_ready(volatile int *word, int item) {
    bool good = true;
    if ((threadIdx.x & 31) == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (*word != item) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicOr(&g_error_word, kErrTimeout);
                good = false;
                break;
            }
            __nanosleep(32);
        }
        __threadfence_block();
    }
    return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ uint4 dk_lds128(const uint8_t *p) {
    return *reinterpret_cast<const uint4 *>(p);
}
__device__ __forceinline__ uint32_t dk_word(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// D (16x8 s32) += A (16x32 u8, row) * B (32x8 u8, col)
__device__ __forceinline__ void mma_u8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Integer engine: B column of token m's plane p, and of the ones column.
__host__ __device__ constexpr int dk_col(int m, int p) { return 6 * m + p; }
__host__ __device__ constexpr int dk_ones_col(int M) { return 6 * M; }

// Offset of the 16-byte B block of (16-trit word w of the stage, column col)
// in the integer engine's layout: [cg][v][i][col & 7][c], where
// w = (4 v + c) * 4 + i.  A consumer quarter-warp reads two columns x four c:
// 128 contiguous bytes.
__device__ __forceinline__ uint32_t dk_iblock(int w, int col) {
    const int ch = w >> 2, i = w & 3, v = ch >> 2, c = ch & 3;
    return (uint32_t)((col >> 3) * 4096 + (((v * 4 + i) * 8 + (col & 7)) * 4 + c) * 16);
}
// fp16 engine: offset of the 16-byte half `hf` (digit positions 2hf, 2hf+1)
// of the B operands of (word w, token m): [v][i][hf][m][c], Mp = tokens rounded
// up to even (a quarter-warp reads tokens 2p, 2p+1 x four c).
__device__ __forceinline__ uint32_t dk_hblock(int w, int m, int hf, int Mp) {
    const int ch = w >> 2, i = w & 3, v = ch >> 2, c = ch & 3;
    return (uint32_t)(((((v * 4 + i) * 2 + hf) * Mp + m) * 4 + c) * 16);
}

// MMA row g of a 16-row tile reads physical row pi(g) (and pi(g) + 8).
__host__ __device__ constexpr int dk_pi(int g) { return ((g & 1) << 2) | (g >> 1); }
__host__ __device__ constexpr int dk_pi_inv(int p) { return ((p & 3) << 1) | (p >> 2); }

// The 16 activations of word w (elements 16w .. 16w + 15 of a stage that
// starts at src), zero at elements >= valid.  Only whole 8-element halves that
// start below `valid` are read, so reads of global activations stay inside
// the row (ldx is a multiple of 8 and >= K).
__device__ __forceinline__ void dk_read_word(const uint16_t *src, int w, int valid,
                                             uint32_t (&r)[8]) {
    const int e0 = 16 * w;
    uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
    if (e0 < valid) lo = *reinterpret_cast<const uint4 *>(src + e0);
    if (e0 + 8 < valid) hi = *reinterpret_cast<const uint4 *>(src + e0 + 8);
    r[0] = lo.x; r[1] = lo.y; r[2] = lo.z; r[3] = lo.w;
    r[4] = hi.x; r[5] = hi.y; r[6] = hi.z; r[7] = hi.w;
    const int keep = valid - e0;
    if (keep < 16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t l = 2 * i < keep ? 0x0000FFFFu : 0u;
            const uint32_t h = 2 * i + 1 < keep ? 0xFFFF0000u : 0u;
            r[i] &= l | h;
        }
    }
}

// The same for a SwiGLU input: element e of the word is
// fp16_rn(silu(g_e) * u_e) in fp32, g from src and u from up = src + K (the
// row's second half); zero at e >= valid.
__device__ __forceinline__ uint32_t dk_glu2(uint32_t g, uint32_t u) {
    const float2 gf = __half22float2(*reinterpret_cast<const __half2 *>(&g));
    const float2 uf = __half22float2(*reinterpret_cast<const __half2 *>(&u));
    const float a = __fdividef(gf.x, 1.0f + __expf(-gf.x)) * uf.x;
    const float b = __fdividef(gf.y, 1.0f + __expf(-gf.y)) * uf.y;
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ void dk_read_word_glu(const uint16_t *src, const uint16_t *up, int w,
                                                 int valid, uint32_t (&r)[8]) {
    uint32_t g[8], u[8];
    dk_read_word(src, w, valid, g);
    dk_read_word(up, w, valid, u);
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = dk_glu2(g[i], u[i]);
}
// One word of a stage's activations: plain, or the SwiGLU product (up != null).
__device__ __forceinline__ void dk_load_word(const uint16_t *src, const uint16_t *up, int w,
                                             int valid, uint32_t (&r)[8]) {
    if (up)
        dk_read_word_glu(src, up, w, valid, r);
    else
        dk_read_word(src, w, valid, r);
}

// One warp converts one stage of token m for the integer engine: z = x 2^24 +
// 2^40 as six u8 planes, each 16-byte block the 4x4 transpose of a word's
// elements (byte 4j + b = element 4b + j), the ones column (m == 0), and
// Q = sum x 2^24 into meta[m] (exact: the partial sums of binary16 values are
// multiples of 2^-24 below 2^26, within a double's 53 bits).
__device__ __forceinline__ void dk_conv_imma(const uint16_t *src, const uint16_t *up, int valid,
                                             int m, int M, uint8_t *dstB, uint8_t *meta, int lane) {
    const int ones = dk_ones_col(M);
    double qd = 0.0;
    for (int w = lane; w < kDkWords; w += 32) {
        uint32_t r[8];
        dk_load_word(src, up, w, valid, r);
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; e2 += 2) {
            const float2 xf2 = __half22float2(*reinterpret_cast<const __half2 *>(&r[e2 >> 1]));
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float xf = u ? xf2.y : xf2.x;
                const float fl = floorf(xf);
                lo[e2 + u] = (uint32_t)((xf - fl) * 16777216.0f);
                hi[e2 + u] = (uint32_t)(fl + 65536.0f);
                qd += (double)xf;
            }
        }
        // bytes 0..2 of lo[] are planes 0..2, bytes 0..2 of hi[] planes 3..5
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t *s = half ? hi : lo;
            uint32_t pl[3][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t A0 = prmt(s[j], s[4 + j], 0x5140u);
                const uint32_t B0 = prmt(s[8 + j], s[12 + j], 0x5140u);
                const uint32_t C0 = prmt(s[j], s[4 + j], 0x7362u);
                const uint32_t D0 = prmt(s[8 + j], s[12 + j], 0x7362u);
                pl[0][j] = prmt(A0, B0, 0x5410u);
                pl[1][j] = prmt(A0, B0, 0x7632u);
                pl[2][j] = prmt(C0, D0, 0x5410u);
            }
#pragma unroll
            for (int p = 0; p < 3; ++p)
                *reinterpret_cast<uint4 *>(dstB + dk_iblock(w, dk_col(m, 3 * half + p))) =
                    make_uint4(pl[p][0], pl[p][1], pl[p][2], pl[p][3]);
        }
        if (m == 0)
            *reinterpret_cast<uint4 *>(dstB + dk_iblock(w, ones)) =
                make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) qd += __shfl_xor_sync(0xffffffffu, qd, o);
    if (lane == 0) reinterpret_cast<int64_t *>(meta)[m] = (int64_t)(qd * 16777216.0);
}

// One warp converts one stage of token m for the fp16 engine: per word and
// digit position j the pairs (x_j, x_{8+j}) and (x_{4+j}, x_{12+j}), and
// sum_k x into meta[m] (fp32).
__device__ __forceinline__ void dk_conv_hmma(const uint16_t *src, const uint16_t *up, int valid,
                                             int m, int Mp, uint8_t *dstB, uint8_t *meta, int lane) {
    float sx = 0.f;
    for (int w = lane; w < kDkWords; w += 32) {
        uint32_t r[8];
        dk_load_word(src, up, w, valid, r);
        uint32_t b[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
            b[2 * j] = prmt(r[j >> 1], r[4 + (j >> 1)], sel);
            b[2 * j + 1] = prmt(r[2 + (j >> 1)], r[6 + (j >> 1)], sel);
        }
        *reinterpret_cast<uint4 *>(dstB + dk_hblock(w, m, 0, Mp)) = make_uint4(b[0], b[1], b[2], b[3]);
        *reinterpret_cast<uint4 *>(dstB + dk_hblock(w, m, 1, Mp)) = make_uint4(b[4], b[5], b[6], b[7]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 fv = __half22float2(*reinterpret_cast<const __half2 *>(&r[i]));
            sx += fv.x + fv.y;
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
    if (lane == 0) reinterpret_cast<float *>(meta)[m] = sx;
}

// ---- base 3 (1.6-bit) ----
// A packed byte v = sum_i d_i 3^i (d = t + 1) holds five trits; with
// q_i = floor(v / 3^i) (q_0 = v), d_i = q_i - 3 q_{i+1} and d_4 = q_4, so for
// the activations xi_{5b+i} of byte b
//   sum_i d_i xi_{5b+i} = q_0 xi_{5b} + sum_{p=1..4} q_p (xi_{5b+p} - 3 xi_{5b+p-1}).
// The quotients of the four bytes of a word come out of 16-bit lanes: for
// v < 256, floor(85 (v + 1) / 256) = floor(v / 3) (exact for v < 243, the
// valid codes), and 85 (v + 1) < 2^16, so one IMAD serves two bytes and the
// quotient is the product's high byte.

// The 20 activations of packed word w of a base-3 stage (elements 20w ..
// 20w + 19 of a stage that starts at src), zero at elements >= valid.  Only
// whole 4-element groups that start below `valid` are read (ldx is a multiple
// of 8 and >= K, so they stay inside the row).
__device__ __forceinline__ void dk_read20(const uint16_t *src, int w, int valid, uint32_t (&r)[10]) {
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        const int e = 20 * w + 4 * i;
        uint2 v = make_uint2(0u, 0u);
        if (e < valid) v = *reinterpret_cast<const uint2 *>(src + e);
        const int keep = valid - e;
        if (keep < 4) {
            v.x &= (keep > 0 ? 0x0000FFFFu : 0u) | (keep > 1 ? 0xFFFF0000u : 0u);
            v.y &= (keep > 2 ? 0x0000FFFFu : 0u);
        }
        r[2 * i] = v.x;
        r[2 * i + 1] = v.y;
    }
}
// The same, plain or as the SwiGLU product (up != null).
__device__ __forceinline__ void dk_load20(const uint16_t *src, const uint16_t *up, int w, int valid,
                                          uint32_t (&r)[10]) {
    dk_read20(src, w, valid, r);
    if (up) {
        uint32_t u[10];
        dk_read20(up, w, valid, u);
#pragma unroll
        for (int i = 0; i < 10; ++i) r[i] = dk_glu2(r[i], u[i]);
    }
}
// Element e (0..19) of a word read by dk_read20 as the halves of r.
template <int E0, int E1>
__device__ __forceinline__ uint32_t dk_pair20(const uint32_t (&r)[10]) {
    return prmt(r[E0 >> 1], r[E1 >> 1], ((E0 & 1) ? 0x32u : 0x10u) | ((E1 & 1) ? 0x7600u : 0x5400u));
}

// Integer engine, base 3: offset of the 8-byte B entry of (half v, word pair
// pr, position p, column col, lane column c): words 2pr and 2pr + 1 of chunk
// 4v + c, four bytes each.  A quarter-warp reads 64 contiguous bytes.
__host__ __device__ constexpr uint32_t dk_i3off(int v, int pr, int p, int col, int c) {
    return (uint32_t)((col >> 3) * 5 * 1024 + ((((v * 2 + pr) * 5 + p) * 8 + (col & 7)) * 4 + c) * 8);
}
// fp16 engine, base 3: offset of the 8-byte B entry of (half v, word i of the
// chunk, digit p, token m, lane column c), Mp tokens rounded up to even.
__host__ __device__ constexpr uint32_t dk_h3off(int v, int i, int p, int m, int c, int Mp) {
    return (uint32_t)(((((v * 4 + i) * 5 + p) * Mp + m) * 4 + c) * 8);
}

// One warp converts one base-3 stage of token m for the integer engine.  Lane
// w takes packed word w (bytes 4w .. 4w + 3).  With xi = x 2^24 (an integer,
// |xi| < 2^40), position p of byte b has the B operand
//   p = 0: xi_{5b} + 2^42,   p >= 1: xi_{5b+p} - 3 xi_{5b+p-1} + 2^42,
// a natural number below 2^43 stored as six u8 planes; the 2^42 offsets come
// back out as 2^42 times the ones column's sum of A.  Q = sum xi into meta[m]
// (exact in a double: below 2^50).
__device__ __forceinline__ void dk_conv_imma3(const uint16_t *src, const uint16_t *up, int valid,
                                              int m, int M, uint8_t *dstB, uint8_t *meta, int lane) {
    const int w = lane, ch = w >> 2, i = w & 3, v = ch >> 2, c = ch & 3, pr = i >> 1, hf = i & 1;
    uint32_t r[10];
    dk_load20(src, up, w, valid, r);
    int64_t xi[20];
    double qd = 0.0;
#pragma unroll
    for (int k = 0; k < 10; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r[k]));
        xi[2 * k] = (int64_t)(f.x * 16777216.0f);  // exact: a binary16 times 2^24
        xi[2 * k + 1] = (int64_t)(f.y * 16777216.0f);
        qd += (double)xi[2 * k] + (double)xi[2 * k + 1];
    }
    const int ones = dk_ones_col(M);
#pragma unroll
    for (int p = 0; p < 5; ++p) {
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t b = (p == 0 ? xi[5 * e] : xi[5 * e + p] - 3 * xi[5 * e + p - 1]) + (1ll << 42);
            lo[e] = (uint32_t)b;
            hi[e] = (uint32_t)(b >> 32);
        }
        // plane j's word holds byte j of the four bytes' operands
        const uint32_t a01 = prmt(lo[0], lo[1], 0x5140u), a23 = prmt(lo[2], lo[3], 0x5140u);
        const uint32_t c01 = prmt(lo[0], lo[1], 0x7362u), c23 = prmt(lo[2], lo[3], 0x7362u);
        const uint32_t h01 = prmt(hi[0], hi[1], 0x5140u), h23 = prmt(hi[2], hi[3], 0x5140u);
        const uint32_t pl[6] = {prmt(a01, a23, 0x5410u), prmt(a01, a23, 0x7632u),
                                prmt(c01, c23, 0x5410u), prmt(c01, c23, 0x7632u),
                                prmt(h01, h23, 0x5410u), prmt(h01, h23, 0x7632u)};
#pragma unroll
        for (int j = 0; j < 6; ++j)
            *reinterpret_cast<uint32_t *>(dstB + dk_i3off(v, pr, p, dk_col(m, j), c) + 4 * hf) = pl[j];
        if (m == 0)
            *reinterpret_cast<uint32_t *>(dstB + dk_i3off(v, pr, p, ones, c) + 4 * hf) = 0x01010101u;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) qd += __shfl_xor_sync(0xffffffffu, qd, o);
    if (lane == 0) reinterpret_cast<int64_t *>(meta)[m] = (int64_t)qd;
}

// One warp converts one base-3 stage of token m for the fp16 engine: per word
// and digit p the pairs (x_p, x_{10+p}) and (x_{5+p}, x_{15+p}) of the word's
// elements (bytes 0 and 2, bytes 1 and 3), and sum x into meta[m] (fp32).
__device__ __forceinline__ void dk_conv_hmma3(const uint16_t *src, const uint16_t *up, int valid,
                                              int m, int Mp, uint8_t *dstB, uint8_t *meta, int lane) {
    const int w = lane, ch = w >> 2, i = w & 3, v = ch >> 2, c = ch & 3;
    uint32_t r[10];
    dk_load20(src, up, w, valid, r);
    float sx = 0.f;
#pragma unroll
    for (int k = 0; k < 10; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r[k]));
        sx += f.x + f.y;
    }
    uint2 *d = reinterpret_cast<uint2 *>(dstB);
    d[dk_h3off(v, i, 0, m, c, Mp) / 8] = make_uint2(dk_pair20<0, 10>(r), dk_pair20<5, 15>(r));
    d[dk_h3off(v, i, 1, m, c, Mp) / 8] = make_uint2(dk_pair20<1, 11>(r), dk_pair20<6, 16>(r));
    d[dk_h3off(v, i, 2, m, c, Mp) / 8] = make_uint2(dk_pair20<2, 12>(r), dk_pair20<7, 17>(r));
    d[dk_h3off(v, i, 3, m, c, Mp) / 8] = make_uint2(dk_pair20<3, 13>(r), dk_pair20<8, 18>(r));
    d[dk_h3off(v, i, 4, m, c, Mp) / 8] = make_uint2(dk_pair20<4, 14>(r), dk_pair20<9, 19>(r));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, o);
    if (lane == 0) reinterpret_cast<float *>(meta)[m] = sx;
}

// One stage of token m in the B layout of the item's engine.
template <int FMT>
__device__ __forceinline__ void dk_convert(const uint16_t *src, const uint16_t *up, int valid, int m,
                                           int M, uint8_t *slot, int lane) {
    if constexpr (FMT == 2) {
        if (M <= kDkImmaMaxM)
            dk_conv_imma(src, up, valid, m, M, slot + kDkMetaBytes, slot, lane);
        else
            dk_conv_hmma(src, up, valid, m, M + (M & 1), slot + kDkMetaBytes, slot, lane);
    } else {
        if (M <= kDkImmaMaxM)
            dk_conv_imma3(src, up, valid, m, M, slot + kDkMetaBytes, slot, lane);
        else
            dk_conv_hmma3(src, up, valid, m, M + (M & 1), slot + kDkMetaBytes, slot, lane);
    }
}

// The last part of a split tile adds the tile's parts in part order and stores
// fp16_rn(alpha * sum): int64 partials (integer engine, exact, V * 2^-24) or
// fp32 partials summed in double.  A lane takes 8 consecutive rows of one
// token at a time and keeps the loads of several parts in flight.  Not
// inlined, so its registers do not weigh on the consumer loops.
__device__ __noinline__ void dk_finalize(const int64_t *base, int cnt, int parts, bool exact,
                                         float alpha, uint16_t *Y, int64_t ldy, int n0, int N,
                                         int lane) {
    for (int gi = lane; gi < cnt / 8; gi += 32) {
        const int idx0 = gi * 8;  // token idx0 / 256, rows idx0 % 256 ..
        const int m = idx0 / kDkRows, r0 = idx0 % kDkRows;
        uint32_t h[4];
        if (exact) {
            int64_t acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            int q = 0;
            for (; q + 2 <= parts; q += 2) {
                const longlong2 *p0 =
                    reinterpret_cast<const longlong2 *>(base + (int64_t)q * cnt + idx0);
                const longlong2 *p1 = reinterpret_cast<const longlong2 *>(
                    base + (int64_t)(q + 1) * cnt + idx0);
                longlong2 u[4], w[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    u[j] = __ldcg(p0 + j);
                    w[j] = __ldcg(p1 + j);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[2 * j] += u[j].x + w[j].x;
                    acc[2 * j + 1] += u[j].y + w[j].y;
                }
            }
            if (q < parts) {
                const longlong2 *p0 =
                    reinterpret_cast<const longlong2 *>(base + (int64_t)q * cnt + idx0);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const longlong2 u = __ldcg(p0 + j);
                    acc[2 * j] += u.x;
                    acc[2 * j + 1] += u.y;
                }
            }
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const uint16_t lo = __half_as_ushort(__double2half(
                    (double)alpha * ((double)acc[j] * 5.9604644775390625e-8)));
                const uint16_t hi = __half_as_ushort(__double2half(
                    (double)alpha * ((double)acc[j + 1] * 5.9604644775390625e-8)));
                h[j / 2] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
        } else {
            // fp32 partials, summed in double in part order
            double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int q0 = 0; q0 < parts; q0 += 4) {
                const int nq = parts - q0 < 4 ? parts - q0 : 4;
                float4 u[4][2];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < nq) {
                        const float4 *f = reinterpret_cast<const float4 *>(
                            reinterpret_cast<const float *>(base + (int64_t)(q0 + q) * cnt) +
                            idx0);
                        u[q][0] = __ldcg(f);
                        u[q][1] = __ldcg(f + 1);
                    }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < nq) {
                        acc[0] += u[q][0].x;
                        acc[1] += u[q][0].y;
                        acc[2] += u[q][0].z;
                        acc[3] += u[q][0].w;
                        acc[4] += u[q][1].x;
                        acc[5] += u[q][1].y;
                        acc[6] += u[q][1].z;
                        acc[7] += u[q][1].w;
                    }
            }
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const uint16_t lo = f32_to_f16_bits(alpha * (float)acc[j]);
                const uint16_t hi = f32_to_f16_bits(alpha * (float)acc[j + 1]);
                h[j / 2] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
        }
        uint16_t *yr = Y + (int64_t)m * ldy + n0 + r0;
        if (n0 + r0 + 8 <= N) {
            *reinterpret_cast<uint4 *>(yr) = make_uint4(h[0], h[1], h[2], h[3]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (n0 + r0 + j < N) yr[j] = (uint16_t)(h[j / 2] >> (16 * (j & 1)));
        }
    }
}

// kGlu: the batch has SwiGLU-input layers (a separate instantiation, so that
// the conversion's fp32 silu code is not part of every other batch's kernel).
// A dependent layer's X converted once (kDkItemCoop): a warp claims the
// layer's units (stage, token) one at a time until none is left, converts each
// into the layer's B in the workspace and counts it in `ready`.  Not inlined,
// so its registers do not weigh on the kernel's other roles.
template <int FMT>
__device__ __noinline__ void dk_coop_convert(const DkItemRec *ir, const uint16_t *X, int ldx, int M,
                                             int K, bool swiglu, uint32_t *claim, uint32_t *ready,
                                             int lane) {
    constexpr int TS = dk_trits(FMT);
    uint8_t *B = const_cast<uint8_t *>(ir->B);
    const int need = ir->need, bstride = ir->bstride;
    while (true) {
        uint32_t u = 0;
        if (lane == 0) u = atomicAdd(claim, 1u);
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= (uint32_t)need) break;
        const int us = (int)u / M, um = (int)u % M;
        const int valid = min(K - us * TS, TS);
        const uint16_t *src = X + (int64_t)um * ldx + (int64_t)us * TS;
        dk_convert<FMT>(src, swiglu ? src + K : nullptr, valid, um, M, B + (int64_t)us * bstride, lane);
        // read by bulk copies of other CTAs
        dk_fence_proxy_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(ready, 1u);
    }
}

template <int FMT, bool kGlu>
__global__ void __launch_bounds__(kDkThreads, 1) decode2_kernel(const __grid_constant__ DkArgs a) {
    constexpr int TS = dk_trits(FMT);  // activations per stage
    extern __shared__ __align__(1024) uint8_t dk_smem_raw[];
    const DkLayout lay(FMT, a.maxM, a.wide != 0);
    const int NS = (int)lay.ns;
    // 1024-byte alignment for the 128-byte swizzle of the weight boxes
    uint8_t *smem = dk_smem_raw + ((1024u - (smem_u32(dk_smem_raw) & 1023u)) & 1023u);
    uint8_t *wring = smem + lay.w_off;
    uint8_t *sslot = smem + lay.st_off;  // per slot: [meta 64 B][B operands]
    uint8_t *parts = smem + lay.part_off;
    DkQEntry *queue = reinterpret_cast<DkQEntry *>(smem + lay.q_off);
    uint64_t *wfull = reinterpret_cast<uint64_t *>(smem + lay.bar_off);  // copies landed
    uint64_t *xfull = wfull + NS;  // stager -> consumers (stages converted on chip only)
    uint64_t *empty = xfull + NS;                                         // consumers -> producer
    uint64_t *qfull = empty + NS;
    uint64_t *qempty = qfull + kDkQueue;
    const int NB = (int)lay.nbufs;
    uint64_t *pfull = qempty + kDkQueue;  // consumers -> epilogue
    uint64_t *pempty = pfull + NB;
    uint32_t *conv_done = reinterpret_cast<uint32_t *>(pempty + NB);  // warps done converting
    // per queue slot: the index of the dependent item whose inputs are final
    volatile int *iready = reinterpret_cast<volatile int *>(conv_done + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&wfull[i], 1);
            mbar_init(&xfull[i], 32);  // every stager lane arrives
            mbar_init(&empty[i], kDkConsumers);
        }
        for (int i = 0; i < kDkQueue; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], kDkConsumers + kDkStagers + kDkEpilogues);
        }
        for (int i = 0; i < NB; ++i) {
            mbar_init(&pfull[i], kDkConsumers);
            mbar_init(&pempty[i], 1);
        }
        *conv_done = 0u;
        for (int i = 0; i < kDkQueue; ++i) iready[i] = -1;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp != 0) {
        // ---- every warp but the producer: convert activations, one unit at a time ----
        pdl_wait();  // X may be written by the preceding grid; Y may still be in use
        // unit u goes to CTA u mod gridDim.x, so that every CTA converts a few
        // units at once (one per warp) rather than a few CTAs many; within a
        // CTA the stagers come last, as they convert the CTA's first item next
        constexpr int kConv = kDkWarps - 1;
        const int crank = warp > kDkStagers ? warp - 1 - kDkStagers : kConv - kDkStagers + warp - 1;
        for (int u = crank * (int)gridDim.x + (int)blockIdx.x; u < a.total_units;
             u += (int)gridDim.x * kConv) {
            const DkUnitRec U = dk_load_rec<DkUnitRec, 3>(a.units, u);
            const int valid = min(U.K - U.stage * TS, TS);
            const uint16_t *src = U.X + (int64_t)U.m * U.ldx + (int64_t)U.stage * TS;
            dk_convert<FMT>(src, nullptr, valid, U.m, U.M, U.dst, lane);
            // the converted unit is read by bulk copies of other CTAs
            dk_fence_proxy_global();
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(&a.ready[U.layer], 1u);
        }
        // the last converting warp of the CTA counts the CTA as done
        if (lane == 0 && atomicAdd(conv_done, 1u) == (uint32_t)kConv - 1) {
            __threadfence();
            atomicAdd(&a.ctr[kDkCtrUnitsDone], 1u);
        }
    }

    if (warp == 0) {
        // ---------------- producer ----------------
        // Items are handed out dynamically: the first one is blockIdx.x, each
        // later one comes from the workspace counter (plus gridDim.x).  The
        // index of the item after next and the record of the next item are
        // fetched while the current item streams.
        uint32_t stage = 0;
        int ps = 0;
        uint32_t pph = 0;
        bool wrapped = false;
        int qi = 0;
        bool waited = false, ok = true, all_ready = a.total_units == 0, fenced = true;
        const int G = (int)gridDim.x;
        int item = (int)blockIdx.x;
        DkItemRec R{};
        if (item < a.total_items) R = dk_load_rec<DkItemRec, 7>(a.items, item);
        int next = a.total_items;
        while (ok) {
            const int q = qi % kDkQueue;
            if (qi >= kDkQueue && !dk_warp_wait(&qempty[q], (uint32_t)((qi / kDkQueue) - 1) & 1u)) {
                ok = false;
                break;
            }
            const bool valid = item < a.total_items;
            // the CTA's first item is converted on chip by the stagers (integer
            // engine: one or two tokens per stage), so the CTA starts without
            // waiting for other CTAs' conversions
            const bool pre = valid && R.B != nullptr && (waited || R.M > kDkImmaMaxM);
            if (lane == 0) {
                DkQEntry e{};
                e.item = valid ? item : -1;
                if (valid) {
                    e.Y = R.Y;
                    e.X = R.X;
                    e.ldx = R.ldx;
                    e.part_off = R.part_off;
                    e.alpha = R.alpha;
                    e.tile = R.tile;
                    e.part = R.part;
                    e.s0 = R.s0;
                    e.s1 = R.s1;
                    e.M = R.M;
                    e.K = R.K;
                    e.N = R.N;
                    e.ldy = R.ldy;
                    e.parts = R.parts;
                    e.tile_begin = R.tile_begin;
                    e.pre = pre ? 1 : 0;
                    e.chained = R.deps != 0 ? 1 : 0;
                    e.swiglu = (R.flags & kDkItemSwiglu) ? 1 : 0;
                    e.layer = R.layer & 0xFFFF;
                    e.coop = (R.flags & kDkItemCoop) ? 1 : 0;
                }
                queue[q] = e;
                mbar_arrive(&qfull[q]);
            }
            ++qi;
            if (!valid) break;
            const CUtensorMap *tmap = a.maps + (R.layer & 0xFFFF);
            const int n0 = R.tile * kDkRows;
            // bytes of a stage besides the weights: the converted operands
            auto extra = [&](int) -> uint32_t { return pre ? (uint32_t)R.bstride : 0u; };
            auto issue_w = [&](int slot, int s) {
                tma_load_2d(wring + slot * kDkWBytes, tmap, &wfull[slot], s * kDkStageW, n0);
            };
            auto issue_x = [&](int slot, int s) {
                if (pre)
                    dk_bulk_load(sslot + slot * lay.slot_b, R.B + (int64_t)s * R.bstride,
                                 (uint32_t)R.bstride, &wfull[slot]);
            };
            const bool coop = (R.flags & kDkItemCoop) != 0;
            // the item's activations may be read: the earlier layers that write
            // X are complete (dependent layers), and the layer's units are
            // converted (operands that arrive with the weights)
            auto wait_inputs = [&]() -> bool {
                bool good = true;
                if (R.deps != 0) {
                    // every layer that writes this layer's X has stored all its tiles
                    const int hi = (R.deps & 0xFFFF) - 1;
                    for (int j = R.deps >> 16; j <= hi && good; ++j)
                        good = dk_wait_count(&a.lfinal[j], a.ltiles[j], nullptr, 0u, nullptr);
                    fenced = false;
                }
                if (good && R.deps != 0) {
                    // the stagers may read X: to convert the item's stages, or
                    // (coop) to help convert the layer's units
                    if (lane == 0) {
                        __threadfence_block();
                        iready[q] = item;
                    }
                    __syncwarp();
                }
                if (good && pre) {
                    if (coop) {
                        // units of a dependent layer: converted during this launch
                        good = dk_wait_count(&a.ready[R.layer & 0xFFFF], (uint32_t)R.need, nullptr, 0u,
                                             nullptr);
                        fenced = false;
                    } else if (!all_ready) {
                        good = dk_wait_count(&a.ready[R.layer >> 16], (uint32_t)R.need,
                                             &a.ctr[kDkCtrUnitsDone], gridDim.x, &all_ready);
                        fenced = false;
                    }
                }
                // what was observed above is read next by bulk copies (async proxy)
                if (!fenced) {
                    dk_fence_proxy_global();
                    fenced = true;
                }
                return good;
            };
            int s = R.s0;
            if (!waited) {
                // first item: weights of up to a ring's worth of stages before the
                // previous grid ends (expected bytes raised now, the arrival later)
                const int pre_n = min(R.s1 - R.s0, NS);
                if (lane == 0) {
                    tma_prefetch_desc(tmap);
                    for (int i = 0; i < pre_n; ++i) {
                        const int slot = (int)((stage + i) % NS);
                        dk_expect_tx(&wfull[slot], kDkWBytes);
                        issue_w(slot, R.s0 + i);
                    }
                }
                pdl_wait();
                waited = true;
                // the second item is static too (blockIdx.x + G): no counter round
                // trip before the CTA's first stages; later ones come from the
                // counter, which the previous grid's last CTA reset
                next = item + G;
                const bool in_ok = wait_inputs();
                if (lane == 0) {
                    for (int i = 0; i < pre_n; ++i) {
                        const int slot = (int)((stage + i) % NS);
                        const int si = R.s0 + i;
                        mbar_arrive_expect_tx(&wfull[slot], in_ok ? extra(si) : 0u);
                        if (in_ok) issue_x(slot, si);
                    }
                }
                __syncwarp();
                stage += pre_n;
                s += pre_n;
                ps = pre_n;
                if (ps == NS) {
                    ps = 0;
                    pph = 1;
                    wrapped = true;
                }
                if (!in_ok) {
                    ok = false;
                    break;
                }
            } else {
                int pre_n = 0;
                const int s_pre = s, ps_pre = ps;
                if (R.deps != 0 || coop) {
                    // a dependent item: its weights do not depend on the earlier
                    // layers, so up to a ring's worth streams while it waits (the
                    // slots are freed by earlier items, never by this one); with
                    // converted operands the stage completes only once they follow
                    pre_n = min(R.s1 - s, NS);
                    for (int i = 0; i < pre_n; ++i, ++s, ++stage) {
                        const int slot = ps;
                        if (wrapped && !dk_warp_wait(&empty[slot], pph ^ 1u)) {
                            ok = false;
                            break;
                        }
                        if (++ps == NS) {
                            ps = 0;
                            pph ^= 1u;
                            wrapped = true;
                        }
                        if (lane == 0) {
                            if (pre)
                                dk_expect_tx(&wfull[slot], kDkWBytes);
                            else
                                mbar_arrive_expect_tx(&wfull[slot], kDkWBytes);
                            issue_w(slot, s);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                }
                const bool in_ok = wait_inputs();
                if (pre && lane == 0) {
                    for (int i = 0; i < pre_n; ++i) {
                        const int slot = (ps_pre + i) % NS;
                        mbar_arrive_expect_tx(&wfull[slot], in_ok ? extra(s_pre + i) : 0u);
                        if (in_ok) issue_x(slot, s_pre + i);
                    }
                }
                __syncwarp();
                if (!in_ok) {
                    ok = false;
                    break;
                }
            }
            // fetched now, used after this item's stages are issued
            DkItemRec NR{};
            if (next < a.total_items) NR = dk_load_rec<DkItemRec, 7>(a.items, next);
            int nx2 = 0;
            if (lane == 0 && next < a.total_items)
                nx2 = 2 * G + (int)atomicAdd(&a.ctr[kDkCtrItems], 1u);
            for (; s < R.s1; ++s, ++stage) {
                const int slot = ps;
                if (wrapped && !dk_warp_wait(&empty[slot], pph ^ 1u)) {
                    ok = false;
                    break;
                }
                if (++ps == NS) {
                    ps = 0;
                    pph ^= 1u;
                    wrapped = true;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&wfull[slot], kDkWBytes + extra(s));
                    issue_w(slot, s);
                    issue_x(slot, s);
                }
                __syncwarp();
            }
            if (!ok) break;
            item = next;
            R = NR;
            next = next < a.total_items ? __shfl_sync(0xffffffffu, nx2, 0) : a.total_items;
            if (item < a.total_items && lane == 0) tma_prefetch_desc(a.maps + (R.layer & 0xFFFF));
        }
        if (!waited) pdl_wait();
        // the CTA may not exit with copies still landing in its shared memory
        for (uint32_t t = stage > (uint32_t)NS ? stage - NS : 0; t < stage; ++t)
            mbar_wait(&wfull[t % NS], (t / NS) & 1u);
    } else if (warp < kDkFirstEpi) {
        // ---------------- stagers ----------------
        // Stages whose operands were converted beforehand pass them by; the
        // others (a CTA's first item, chained layers) are converted here from X
        // in global memory.  xfull is never arrived on a round ahead: a slot's
        // round r >= 1 starts only once the consumers released round r - 1.
        const int sw = warp - 1;
        int ss = 0;
        uint32_t sph = 0;
        bool first_round = true;  // no earlier use of any slot to wait out
        int qi = 0;
        bool ok = true;
        DkQEntry e;
        while (ok && dk_next_item(queue, qfull, qempty, qi, e)) {
            const int M = e.M, K = e.K;
            const int eq = (qi - 1) % kDkQueue;  // the entry's queue slot
            bool inputs = !e.chained;            // X of a dependent item: after iready
            if (e.coop) {
                // the layer's X is converted once: claim its units (stage, token)
                // one at a time until none is left; the producer waits for all of
                // them before it copies the item's operands in
                if (e.chained && !dk_wait_ready(&iready[eq], e.item)) {
                    ok = false;
                    break;
                }
                dk_coop_convert<FMT>(a.items + e.item, e.X, e.ldx, M, K, kGlu && e.swiglu,
                                     &a.claim[e.layer], &a.ready[e.layer], lane);
            }
            for (int s = e.s0; s < e.s1; ++s) {
                const int slot = ss;
                const uint32_t ph = sph;
                const bool fresh = first_round;
                if (++ss == NS) {
                    ss = 0;
                    sph ^= 1u;
                    first_round = false;
                }
                if (e.pre || slot % kDkStagers != sw) continue;  // converted, or another stager's
                // A slot's first use needs no wait (X of a layer without
                // dependencies is final since pdl_wait).  A later use waits for the
                // consumers to release the slot's previous round: on `empty`, not on
                // the weights of this round -- a stager that skipped its first-round
                // wait may reach round 1 while the slot is still in phase 0, and a
                // parity wait on wfull would then pass a phase early.  A
                // dependent item's X is read once the producer has seen every
                // earlier layer complete and published the item in iready.
                if (!fresh && !dk_warp_wait(&empty[slot], ph ^ 1u)) {
                    ok = false;
                    break;
                }
                if (!inputs) {
                    if (!dk_wait_ready(&iready[eq], e.item)) {
                        ok = false;
                        break;
                    }
                    inputs = true;
                }
                const int valid = min(K - s * TS, TS);
                uint8_t *dst = sslot + slot * lay.slot_b;
                for (int m = 0; m < M; ++m) {
                    const uint16_t *src = e.X + (int64_t)m * e.ldx + (int64_t)s * TS;
                    const uint16_t *up = kGlu && e.swiglu ? src + K : nullptr;  // [gate | up] rows
                    dk_convert<FMT>(src, up, valid, m, M, dst, lane);
                }
#ifdef TL_DEBUG_HOOKS
                // the hook: CTA 0's first stage converted here is never published
                if (a.drop_arrive && blockIdx.x == 0 && s == e.s0 && e.item == (int)blockIdx.x)
                    continue;
#endif
                mbar_arrive(&xfull[slot]);
            }
        }
    } else if (warp < kDkFirstCons) {
        // ---------------- epilogues ----------------
        // Item i uses buffer i mod NB and goes to epilogue warp i mod EA, with
        // EA = min(warps, NB) dividing NB: each warp owns its buffers and waits
        // on their phases in order (a parity wait must never be a phase ahead).
        const int ew = warp - kDkFirstEpi;
        const int EA = NB < kDkEpilogues ? NB : kDkEpilogues;
        int qi = 0, pi = -1;
        DkQEntry e;
        while (dk_next_item(queue, qfull, qempty, qi, e)) {
            if (++pi % EA != ew) continue;
            const int b = pi % NB;
            if (!dk_warp_wait(&pfull[b], (uint32_t)(pi / NB) & 1u)) break;
            const uint8_t *pb = parts + b * lay.parts;
            const int M = e.M, n0 = e.tile * kDkRows, cnt = kDkRows * M;
            const bool exact = M <= kDkImmaMaxM;
            int64_t *slot = e.parts > 1 ? a.partials + e.part_off +
                                              (int64_t)(e.tile * e.parts + e.part) * cnt
                                        : nullptr;
            // partial of (token m, warp cw, tile t of the warp, MMA row rho) at
            // ((m*16 + cw)*2 + t)*16 + rho; the two warps of a row tile (cw, cw + 8)
            // are 256 entries apart.  A lane takes 8 consecutive rows r0 .. r0 + 7
            // of one token: MMA rows (r0 & 8) + pi^-1(0..7), 8 consecutive entries.
            for (int gi = lane; gi < cnt / 8; gi += 32) {
                const int m = gi / (kDkRows / 8), r0 = (gi % (kDkRows / 8)) * 8;
                const int t = r0 >> 4, tp = t >> 1, tl = t & 1;
                const int base = ((m * 16 + tp) * 2 + tl) * 16 + (r0 & 8);
                float y[8];
                int64_t iv[8];
                if (exact) {
                    const int64_t *p = reinterpret_cast<const int64_t *>(pb) + base;
#pragma unroll
                    for (int q = 0; q < 8; q += 2) {
                        const longlong2 u = *reinterpret_cast<const longlong2 *>(p + q);
                        const longlong2 w = *reinterpret_cast<const longlong2 *>(p + 256 + q);
                        iv[dk_pi(q)] = u.x + w.x;  // MMA row q holds physical row pi(q)
                        iv[dk_pi(q + 1)] = u.y + w.y;
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        y[j] = (float)((double)e.alpha * ((double)iv[j] * 5.9604644775390625e-8));
                } else {
                    const float *p = reinterpret_cast<const float *>(pb) + base;
                    const float4 u0 = *reinterpret_cast<const float4 *>(p);
                    const float4 u1 = *reinterpret_cast<const float4 *>(p + 4);
                    const float4 w0 = *reinterpret_cast<const float4 *>(p + 256);
                    const float4 w1 = *reinterpret_cast<const float4 *>(p + 260);
                    const float v[8] = {u0.x + w0.x, u0.y + w0.y, u0.z + w0.z, u0.w + w0.w,
                                        u1.x + w1.x, u1.y + w1.y, u1.z + w1.z, u1.w + w1.w};
#pragma unroll
                    for (int q = 0; q < 8; ++q) y[dk_pi(q)] = v[q];
                }
                const int idx0 = m * kDkRows + r0;
                if (slot) {
                    // this part's partial of a split tile: int64 entries, or fp32
                    // entries packed into the first half of the part's region
                    if (exact) {
#pragma unroll
                        for (int j = 0; j < 8; j += 2)
                            *reinterpret_cast<longlong2 *>(slot + idx0 + j) =
                                make_longlong2(iv[j], iv[j + 1]);
                    } else {
                        float4 *f = reinterpret_cast<float4 *>(reinterpret_cast<float *>(slot) + idx0);
                        f[0] = make_float4(y[0], y[1], y[2], y[3]);
                        f[1] = make_float4(y[4], y[5], y[6], y[7]);
                    }
                } else {
                    // fp16_rn(alpha * v): exact items round once from double
                    uint32_t h[4];
#pragma unroll
                    for (int j = 0; j < 8; j += 2) {
                        uint16_t lo, hi;
                        if (exact) {
                            lo = __half_as_ushort(__double2half(
                                (double)e.alpha * ((double)iv[j] * 5.9604644775390625e-8)));
                            hi = __half_as_ushort(__double2half(
                                (double)e.alpha * ((double)iv[j + 1] * 5.9604644775390625e-8)));
                        } else {
                            lo = f32_to_f16_bits(e.alpha * y[j]);
                            hi = f32_to_f16_bits(e.alpha * y[j + 1]);
                        }
                        h[j / 2] = (uint32_t)lo | ((uint32_t)hi << 16);
                    }
                    uint16_t *yr = e.Y + (int64_t)m * e.ldy + n0 + r0;
                    if (n0 + r0 + 8 <= e.N) {
                        *reinterpret_cast<uint4 *>(yr) = make_uint4(h[0], h[1], h[2], h[3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (n0 + r0 + j < e.N) yr[j] = (uint16_t)(h[j / 2] >> (16 * (j & 1)));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[b]);
            bool final_tile = true;
            if (slot) {
                __threadfence();
                __syncwarp();
                uint32_t prev = 0;
                if (lane == 0) prev = atomicAdd(&a.tile_ctr[e.tile_begin + e.tile], 1u);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                final_tile = prev == (uint32_t)(e.parts - 1);
                if (final_tile) {
                    // last part of the tile: add the parts in part order.  A lane
                    // takes 8 consecutive rows of one token at a time and keeps
                    // the loads of several parts in flight (16-byte loads).
                    __threadfence();
                    dk_finalize(a.partials + e.part_off + (int64_t)e.tile * e.parts * cnt, cnt,
                                e.parts, exact, e.alpha, e.Y, e.ldy, n0, e.N, lane);
                    if (lane == 0) a.tile_ctr[e.tile_begin + e.tile] = 0u;
                }
            }
            if (final_tile && a.chained) {
                // the tile's outputs are stored: count it for its layer (a layer
                // whose count reaches its tiles is complete for its readers)
                dk_fence_proxy_global();
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(&a.lfinal[e.layer], 1u);
            }
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - kDkFirstCons;
        const int tp = cw & 7, v = cw >> 3;  // tile pair, half of the stage's 128 bytes
        const int qv = v;                     // the warp that subtracts the offsets: v == 0
        const int g = lane >> 2, c = lane & 3;
        const int pg = dk_pi(g);
        // tile 2tp, MMA row g: physical row 32 tp + pg; the 4 rows of this lane
        // (tiles 2tp / 2tp+1, rows g / g+8) are 8 rows apart
        const uint32_t aoff = (uint32_t)((32 * tp + pg) * kDkStageW + (((4 * v + c) ^ pg) << 4));
        int cs = 0;
        uint32_t cph = 0;
        uint32_t xph = 0;  // bit s: parity of slot s's next xfull phase
        int qi = 0, pi = 0;
        bool ok = true;
        DkQEntry e{};
        // waits for the stage's copies (and its conversion on chip); false on a timeout
        auto wait_stage = [&](int slot) -> bool {
            if (!dk_warp_wait(&wfull[slot], cph)) return false;
            if (e.pre) return true;
            const bool good = dk_warp_wait(&xfull[slot], (xph >> slot) & 1u);
            xph ^= 1u << slot;
            return good;
        };
        auto release = [&](int slot) {
            // the shared-memory values are consumed (in registers) before the release
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            if (++cs == NS) {
                cs = 0;
                cph ^= 1u;
            }
        };
        while (ok && dk_next_item(queue, qfull, qempty, qi, e)) {
            const int M = e.M;
            const int b = pi % NB;
            uint8_t *pb = parts + b * lay.parts;
            if constexpr (FMT == 2) {
                if (M == 1) {
                    // ---- integer engine, one token: one accumulator per digit
                    // position j (A = digits * 4^j, one AND per register) ----
                    int acc[2][4][4];  // [tile][digit position][D]
    #pragma unroll
                    for (int t = 0; t < 2; ++t)
    #pragma unroll
                        for (int j = 0; j < 4; ++j) acc[t][j][0] = acc[t][j][1] = acc[t][j][2] = acc[t][j][3] = 0;
                    int64_t qsum = 0;
                    for (int s = e.s0; s < e.s1; ++s) {
                        const int slot = cs;
                        if (!wait_stage(slot)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *wb = wring + slot * kDkWBytes + aoff;
                        const uint4 A00 = dk_lds128(wb);                     // tile 2tp, row g
                        const uint4 A01 = dk_lds128(wb + 8 * kDkStageW);   // tile 2tp, row g + 8
                        const uint4 A10 = dk_lds128(wb + 16 * kDkStageW);  // tile 2tp + 1, row g
                        const uint4 A11 = dk_lds128(wb + 24 * kDkStageW);  // tile 2tp + 1, row g + 8
                        const uint8_t *sb = sslot + slot * lay.slot_b;
                        qsum += reinterpret_cast<const int64_t *>(sb)[0];
                        const uint8_t *xg = sb + kDkMetaBytes + ((v * 32 + g) * 4 + c) * 16;
    #pragma unroll
                        for (int pr = 0; pr < 2; ++pr) {
                            const int i0 = 2 * pr, i1 = i0 + 1;
                            const uint4 B0 = dk_lds128(xg + i0 * 512), B1 = dk_lds128(xg + i1 * 512);
    #pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint32_t m = 0x03030303u << (2 * j);
                                const uint32_t b0 = dk_word(B0, j), b1 = dk_word(B1, j);
                                mma_u8_16832(acc[0][j], dk_word(A00, i0) & m, dk_word(A01, i0) & m,
                                             dk_word(A00, i1) & m, dk_word(A01, i1) & m, b0, b1);
                                mma_u8_16832(acc[1][j], dk_word(A10, i0) & m, dk_word(A11, i0) & m,
                                             dk_word(A10, i1) & m, dk_word(A11, i1) & m, b0, b1);
                            }
                        }
                        release(slot);
                    }
                    if (!ok) break;
                    if (pi >= NB && !dk_warp_wait(&pempty[b], (uint32_t)((pi / NB) - 1) & 1u))
                        break;
                    // V = sum_p 256^p S_p - 2^40 S_ones - Q; this lane holds columns
                    // 2c, 2c + 1 (planes 2c, 2c + 1, or the ones column at c = 3)
                    // D = 64 S exactly: position j carries 4^j, so acc0*64 + acc1*16 +
                    // acc2*4 + acc3 = 64 sum_j acc_j 4^-j (below 2^31 for items of at most
                    // kDkMaxItemStages stages); lane c's columns give t_c = D_2c + 256 D_2c+1
                    // (lane 3: the ones column), and lane 0 forms
                    // 64 V = t_0 + 2^16 t_1 + 2^32 t_2 - 2^40 t_3 - 64 Q (modulo 2^64).
    #pragma unroll
                    for (int t = 0; t < 2; ++t) {
    #pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            uint32_t d[2];
    #pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int q = 2 * rr + u;
                                d[u] = (uint32_t)(acc[t][0][q] * 64 + acc[t][1][q] * 16 + acc[t][2][q] * 4 +
                                                  acc[t][3][q]);
                            }
                            const uint64_t tc = c < 3 ? (uint64_t)d[0] + ((uint64_t)d[1] << 8) : (uint64_t)d[0];
                            const uint64_t t1 = __shfl_sync(0xffffffffu, tc, (lane & ~3) | 1);
                            const uint64_t t2 = __shfl_sync(0xffffffffu, tc, (lane & ~3) | 2);
                            const uint64_t t3 = __shfl_sync(0xffffffffu, tc, (lane & ~3) | 3);
                            if (c == 0) {
                                uint64_t v64 = tc + (t1 << 16) + (t2 << 32) - (t3 << 40);
                                if (qv == 0) v64 -= (uint64_t)qsum << 6;
                                reinterpret_cast<int64_t *>(pb)[(cw * 2 + t) * 16 + g + 8 * rr] =
                                    (int64_t)v64 >> 6;
                            }
                        }
                    }
                } else if (M == 2) {
                    // ---- integer engine, two tokens: two column groups share the
                    // decoded digits (shifted to the low bits, one accumulator) ----
                    int iacc[2][2][4];  // [tile][column group][D]
    #pragma unroll
                    for (int t = 0; t < 2; ++t)
    #pragma unroll
                        for (int q = 0; q < 8; ++q) iacc[t][q >> 2][q & 3] = 0;
                    int64_t qsum0 = 0, qsum1 = 0;
                    for (int s = e.s0; s < e.s1; ++s) {
                        const int slot = cs;
                        if (!wait_stage(slot)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *wb = wring + slot * kDkWBytes + aoff;
                        const uint4 A00 = dk_lds128(wb);
                        const uint4 A01 = dk_lds128(wb + 8 * kDkStageW);
                        const uint4 A10 = dk_lds128(wb + 16 * kDkStageW);
                        const uint4 A11 = dk_lds128(wb + 24 * kDkStageW);
                        const uint8_t *sb = sslot + slot * lay.slot_b;
                        qsum0 += reinterpret_cast<const int64_t *>(sb)[0];
                        qsum1 += reinterpret_cast<const int64_t *>(sb)[1];
                        const uint8_t *xg = sb + kDkMetaBytes + ((v * 32 + g) * 4 + c) * 16;
    #pragma unroll
                        for (int pr = 0; pr < 2; ++pr) {
                            const int i0 = 2 * pr, i1 = i0 + 1;
                            const uint4 B00 = dk_lds128(xg + i0 * 512), B01 = dk_lds128(xg + i1 * 512);
                            const uint4 B10 = dk_lds128(xg + 4096 + i0 * 512);
                            const uint4 B11 = dk_lds128(xg + 4096 + i1 * 512);
    #pragma unroll 2
                            for (int j = 0; j < 4; ++j) {
                                constexpr uint32_t m = 0x03030303u;
                                const uint32_t a00 = (dk_word(A00, i0) >> (2 * j)) & m;
                                const uint32_t a01 = (dk_word(A01, i0) >> (2 * j)) & m;
                                const uint32_t a02 = (dk_word(A00, i1) >> (2 * j)) & m;
                                const uint32_t a03 = (dk_word(A01, i1) >> (2 * j)) & m;
                                const uint32_t a10 = (dk_word(A10, i0) >> (2 * j)) & m;
                                const uint32_t a11 = (dk_word(A11, i0) >> (2 * j)) & m;
                                const uint32_t a12 = (dk_word(A10, i1) >> (2 * j)) & m;
                                const uint32_t a13 = (dk_word(A11, i1) >> (2 * j)) & m;
                                const uint32_t b00 = dk_word(B00, j), b01 = dk_word(B01, j);
                                const uint32_t b10 = dk_word(B10, j), b11 = dk_word(B11, j);
                                mma_u8_16832(iacc[0][0], a00, a01, a02, a03, b00, b01);
                                mma_u8_16832(iacc[1][0], a10, a11, a12, a13, b00, b01);
                                mma_u8_16832(iacc[0][1], a00, a01, a02, a03, b10, b11);
                                mma_u8_16832(iacc[1][1], a10, a11, a12, a13, b10, b11);
                            }
                        }
                        release(slot);
                    }
                    if (!ok) break;
                    if (pi >= NB && !dk_warp_wait(&pempty[b], (uint32_t)((pi / NB) - 1) & 1u))
                        break;
                    // columns: token 0 planes 0..5 (group 0, c 0..2), token 1 planes
                    // 0..1 (group 0, c 3) and 2..5 (group 1, c 0..1), ones (group 1, c 2)
    #pragma unroll
                    for (int t = 0; t < 2; ++t) {
    #pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            const int64_t d0 = iacc[t][0][2 * rr], d1 = iacc[t][0][2 * rr + 1];
                            const int64_t e0 = iacc[t][1][2 * rr], e1 = iacc[t][1][2 * rr + 1];
                            int64_t v0 = 0, v1 = 0;
                            if (c < 3) v0 = (d0 << (16 * c)) + (d1 << (16 * c + 8));
                            else v1 = d0 + (d1 << 8);
                            if (c < 2) {
                                v1 += (e0 << (16 * c + 16)) + (e1 << (16 * c + 24));
                            } else if (c == 2) {
                                v0 -= e0 << 40;
                                v1 -= e0 << 40;
                            }
                            v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
                            v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
                            v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
                            v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
                            if (qv == 0) {
                                v0 -= qsum0;
                                v1 -= qsum1;
                            }
                            if (c == 0) {
                                int64_t *p = reinterpret_cast<int64_t *>(pb);
                                p[(cw * 2 + t) * 16 + g + 8 * rr] = v0;
                                p[((16 + cw) * 2 + t) * 16 + g + 8 * rr] = v1;
                            }
                        }
                    }
                } else {
                    // ---- fp16 engine ----
                    const int Mp = M + (M & 1);
                    float facc[2][4][4];  // [tile][digit position][D]
    #pragma unroll
                    for (int t = 0; t < 2; ++t)
    #pragma unroll
                        for (int q = 0; q < 4; ++q)
                            facc[t][q][0] = facc[t][q][1] = facc[t][q][2] = facc[t][q][3] = 0.f;
                    float sx0 = 0.f, sx1 = 0.f;  // sum x of this lane's tokens 2c, 2c + 1
                    for (int s = e.s0; s < e.s1; ++s) {
                        const int slot = cs;
                        if (!wait_stage(slot)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *wb = wring + slot * kDkWBytes + aoff;
                        const uint4 A00 = dk_lds128(wb);
                        const uint4 A01 = dk_lds128(wb + 8 * kDkStageW);
                        const uint4 A10 = dk_lds128(wb + 16 * kDkStageW);
                        const uint4 A11 = dk_lds128(wb + 24 * kDkStageW);
                        const uint8_t *sb = sslot + slot * lay.slot_b;
                        const float *mt = reinterpret_cast<const float *>(sb);
                        if (2 * c < M) sx0 += mt[2 * c];
                        if (2 * c + 1 < M) sx1 += mt[2 * c + 1];
                        const uint8_t *xb = sb + kDkMetaBytes;
    #pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint4 B0 = make_uint4(0u, 0u, 0u, 0u), B1 = B0;
                            if (g < M) {
                                const int w = (4 * v + c) * 4 + i;
                                B0 = dk_lds128(xb + dk_hblock(w, g, 0, Mp));
                                B1 = dk_lds128(xb + dk_hblock(w, g, 1, Mp));
                            }
                            const uint32_t bb[8] = {B0.x, B0.y, B0.z, B0.w, B1.x, B1.y, B1.z, B1.w};
                            const uint32_t W0 = dk_word(A00, i), V0 = dk_word(A01, i);
                            const uint32_t W1 = dk_word(A10, i), V1 = dk_word(A11, i);
                            const uint32_t hW0 = W0 >> 8, hV0 = V0 >> 8, hW1 = W1 >> 8, hV1 = V1 >> 8;
    #pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint32_t m = 0x00030003u << (2 * j);
                                mma_16816(facc[0][j], W0 & m, V0 & m, hW0 & m, hV0 & m, bb[2 * j],
                                          bb[2 * j + 1]);
                                mma_16816(facc[1][j], W1 & m, V1 & m, hW1 & m, hV1 & m, bb[2 * j],
                                          bb[2 * j + 1]);
                            }
                        }
                        release(slot);
                    }
                    if (!ok) break;
                    if (pi >= NB && !dk_warp_wait(&pempty[b], (uint32_t)((pi / NB) - 1) & 1u))
                        break;
                    float *p = reinterpret_cast<float *>(pb);
    #pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        float sv[4];
    #pragma unroll
                        for (int q = 0; q < 4; ++q)
                            sv[q] = facc[t][0][q] * 16777216.0f + facc[t][1][q] * 4194304.0f +
                                    facc[t][2][q] * 1048576.0f + facc[t][3][q] * 262144.0f;
                        if (qv == 0) {
                            sv[0] -= sx0;
                            sv[1] -= sx1;
                            sv[2] -= sx0;
                            sv[3] -= sx1;
                        }
                        const int m0 = 2 * c, m1 = 2 * c + 1;
                        if (m0 < M) {
                            p[((m0 * 16 + cw) * 2 + t) * 16 + g] = sv[0];
                            p[((m0 * 16 + cw) * 2 + t) * 16 + g + 8] = sv[2];
                        }
                        if (m1 < M) {
                            p[((m1 * 16 + cw) * 2 + t) * 16 + g] = sv[1];
                            p[((m1 * 16 + cw) * 2 + t) * 16 + g + 8] = sv[3];
                        }
                    }
                }
            } else {
                if (M == 1) {
                    // ---- base-3 integer engine, one token: positions p = 0..4 (the
                    // bytes, then their quotients by 3, 9, 27, 81) share one
                    // accumulator; B carries each position's activations ----
                    int acc[2][4];  // [tile][D]
    #pragma unroll
                    for (int t = 0; t < 2; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0;
                    int64_t qsum = 0;
                    for (int s = e.s0; s < e.s1; ++s) {
                        const int slot = cs;
                        if (!wait_stage(slot)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *wb = wring + slot * kDkWBytes + aoff;
                        const uint4 A[2][2] = {{dk_lds128(wb), dk_lds128(wb + 8 * kDkStageW)},
                                               {dk_lds128(wb + 16 * kDkStageW), dk_lds128(wb + 24 * kDkStageW)}};
                        const uint8_t *sb = sslot + slot * lay.slot_b;
                        qsum += reinterpret_cast<const int64_t *>(sb)[0];
                        const uint8_t *xg = sb + kDkMetaBytes + dk_i3off(v, 0, 0, g, c);
    #pragma unroll
                        for (int pr = 0; pr < 2; ++pr) {
                            // [tile][row g / g + 8][word 2pr / 2pr + 1]: A words, and their
                            // even / odd bytes in 16-bit lanes
                            uint32_t P[2][2][2], E[2][2][2], O[2][2][2];
    #pragma unroll
                            for (int t = 0; t < 2; ++t)
    #pragma unroll
                                for (int r = 0; r < 2; ++r)
    #pragma unroll
                                    for (int h = 0; h < 2; ++h) {
                                        P[t][r][h] = dk_word(A[t][r], 2 * pr + h);
                                        E[t][r][h] = prmt(P[t][r][h], 0u, 0x4240u);
                                        O[t][r][h] = prmt(P[t][r][h], 0u, 0x4341u);
                                    }
    #pragma unroll
                            for (int p = 0; p < 5; ++p) {
                                if (p > 0) {
    #pragma unroll
                                    for (int t = 0; t < 2; ++t)
    #pragma unroll
                                        for (int r = 0; r < 2; ++r)
    #pragma unroll
                                            for (int h = 0; h < 2; ++h) {
                                                const uint32_t tE = E[t][r][h] * 85u + 0x00550055u;
                                                const uint32_t tO = O[t][r][h] * 85u + 0x00550055u;
                                                P[t][r][h] = prmt(tE, tO, 0x7351u);
                                                E[t][r][h] = prmt(tE, 0u, 0x4341u);
                                                O[t][r][h] = prmt(tO, 0u, 0x4341u);
                                            }
                                }
                                const uint2 bq = *reinterpret_cast<const uint2 *>(xg + dk_i3off(0, pr, p, 0, 0));
    #pragma unroll
                                for (int t = 0; t < 2; ++t)
                                    mma_u8_16832(acc[t], P[t][0][0], P[t][1][0], P[t][0][1], P[t][1][1], bq.x,
                                                 bq.y);
                            }
                        }
                        release(slot);
                    }
                    if (!ok) break;
                    if (pi >= NB && !dk_warp_wait(&pempty[b], (uint32_t)((pi / NB) - 1) & 1u))
                        break;
                    // V = sum_p 256^p S_p - 2^42 S_ones - Q; lane c holds columns 2c,
                    // 2c + 1 (planes, or the ones column at c = 3), and lane 0 of the
                    // quad forms V (modulo 2^64)
    #pragma unroll
                    for (int t = 0; t < 2; ++t) {
    #pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            const uint64_t d0 = (uint32_t)acc[t][2 * rr], d1 = (uint32_t)acc[t][2 * rr + 1];
                            const uint64_t tc = c < 3 ? d0 + (d1 << 8) : d0;
                            const uint64_t t1 = __shfl_sync(0xffffffffu, tc, (lane & ~3) | 1);
                            const uint64_t t2 = __shfl_sync(0xffffffffu, tc, (lane & ~3) | 2);
                            const uint64_t t3 = __shfl_sync(0xffffffffu, tc, (lane & ~3) | 3);
                            if (c == 0) {
                                uint64_t v64 = tc + (t1 << 16) + (t2 << 32) - (t3 << 42);
                                if (qv == 0) v64 -= (uint64_t)qsum;
                                reinterpret_cast<int64_t *>(pb)[(cw * 2 + t) * 16 + g + 8 * rr] = (int64_t)v64;
                            }
                        }
                    }
                } else if (M == 2) {
                    // ---- base-3 integer engine, two tokens: two column groups ----
                    int iacc[2][2][4];  // [tile][column group][D]
    #pragma unroll
                    for (int t = 0; t < 2; ++t)
    #pragma unroll
                        for (int q = 0; q < 8; ++q) iacc[t][q >> 2][q & 3] = 0;
                    int64_t qsum0 = 0, qsum1 = 0;
                    for (int s = e.s0; s < e.s1; ++s) {
                        const int slot = cs;
                        if (!wait_stage(slot)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *wb = wring + slot * kDkWBytes + aoff;
                        const uint4 A[2][2] = {{dk_lds128(wb), dk_lds128(wb + 8 * kDkStageW)},
                                               {dk_lds128(wb + 16 * kDkStageW), dk_lds128(wb + 24 * kDkStageW)}};
                        const uint8_t *sb = sslot + slot * lay.slot_b;
                        qsum0 += reinterpret_cast<const int64_t *>(sb)[0];
                        qsum1 += reinterpret_cast<const int64_t *>(sb)[1];
                        const uint8_t *xg = sb + kDkMetaBytes + dk_i3off(v, 0, 0, g, c);
    #pragma unroll
                        for (int pr = 0; pr < 2; ++pr) {
                            uint32_t P[2][2][2], E[2][2][2], O[2][2][2];
    #pragma unroll
                            for (int t = 0; t < 2; ++t)
    #pragma unroll
                                for (int r = 0; r < 2; ++r)
    #pragma unroll
                                    for (int h = 0; h < 2; ++h) {
                                        P[t][r][h] = dk_word(A[t][r], 2 * pr + h);
                                        E[t][r][h] = prmt(P[t][r][h], 0u, 0x4240u);
                                        O[t][r][h] = prmt(P[t][r][h], 0u, 0x4341u);
                                    }
    #pragma unroll
                            for (int p = 0; p < 5; ++p) {
                                if (p > 0) {
    #pragma unroll
                                    for (int t = 0; t < 2; ++t)
    #pragma unroll
                                        for (int r = 0; r < 2; ++r)
    #pragma unroll
                                            for (int h = 0; h < 2; ++h) {
                                                const uint32_t tE = E[t][r][h] * 85u + 0x00550055u;
                                                const uint32_t tO = O[t][r][h] * 85u + 0x00550055u;
                                                P[t][r][h] = prmt(tE, tO, 0x7351u);
                                                E[t][r][h] = prmt(tE, 0u, 0x4341u);
                                                O[t][r][h] = prmt(tO, 0u, 0x4341u);
                                            }
                                }
                                const uint32_t off = dk_i3off(0, pr, p, 0, 0);
                                const uint2 bq0 = *reinterpret_cast<const uint2 *>(xg + off);
                                const uint2 bq1 = *reinterpret_cast<const uint2 *>(xg + 5 * 1024 + off);
    #pragma unroll
                                for (int t = 0; t < 2; ++t) {
                                    mma_u8_16832(iacc[t][0], P[t][0][0], P[t][1][0], P[t][0][1], P[t][1][1],
                                                 bq0.x, bq0.y);
                                    mma_u8_16832(iacc[t][1], P[t][0][0], P[t][1][0], P[t][0][1], P[t][1][1],
                                                 bq1.x, bq1.y);
                                }
                            }
                        }
                        release(slot);
                    }
                    if (!ok) break;
                    if (pi >= NB && !dk_warp_wait(&pempty[b], (uint32_t)((pi / NB) - 1) & 1u))
                        break;
                    // columns: token 0 planes 0..5 (group 0, c 0..2), token 1 planes
                    // 0..1 (group 0, c 3) and 2..5 (group 1, c 0..1), ones (group 1, c 2)
    #pragma unroll
                    for (int t = 0; t < 2; ++t) {
    #pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            const int64_t d0 = (uint32_t)iacc[t][0][2 * rr], d1 = (uint32_t)iacc[t][0][2 * rr + 1];
                            const int64_t e0 = (uint32_t)iacc[t][1][2 * rr], e1 = (uint32_t)iacc[t][1][2 * rr + 1];
                            int64_t v0 = 0, v1 = 0;
                            if (c < 3) v0 = (d0 << (16 * c)) + (d1 << (16 * c + 8));
                            else v1 = d0 + (d1 << 8);
                            if (c < 2) {
                                v1 += (e0 << (16 * c + 16)) + (e1 << (16 * c + 24));
                            } else if (c == 2) {
                                v0 -= e0 << 42;
                                v1 -= e0 << 42;
                            }
                            v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
                            v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
                            v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
                            v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
                            if (qv == 0) {
                                v0 -= qsum0;
                                v1 -= qsum1;
                            }
                            if (c == 0) {
                                int64_t *p = reinterpret_cast<int64_t *>(pb);
                                p[(cw * 2 + t) * 16 + g + 8 * rr] = v0;
                                p[((16 + cw) * 2 + t) * 16 + g + 8 * rr] = v1;
                            }
                        }
                    }
                } else {
                    // ---- base-3 fp16 engine: digits as subnormal halves d 2^-24 in
                    // 16-bit lanes (even bytes, odd bytes), one accumulator ----
                    const int Mp = M + (M & 1);
                    float facc[2][4];  // [tile][D]
    #pragma unroll
                    for (int t = 0; t < 2; ++t) facc[t][0] = facc[t][1] = facc[t][2] = facc[t][3] = 0.f;
                    float sx0 = 0.f, sx1 = 0.f;  // sum x of this lane's tokens 2c, 2c + 1
                    for (int s = e.s0; s < e.s1; ++s) {
                        const int slot = cs;
                        if (!wait_stage(slot)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *wb = wring + slot * kDkWBytes + aoff;
                        const uint4 A[2][2] = {{dk_lds128(wb), dk_lds128(wb + 8 * kDkStageW)},
                                               {dk_lds128(wb + 16 * kDkStageW), dk_lds128(wb + 24 * kDkStageW)}};
                        const uint8_t *sb = sslot + slot * lay.slot_b;
                        const float *mt = reinterpret_cast<const float *>(sb);
                        if (2 * c < M) sx0 += mt[2 * c];
                        if (2 * c + 1 < M) sx1 += mt[2 * c + 1];
                        const uint8_t *xb = sb + kDkMetaBytes;
    #pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint32_t E[2][2], O[2][2];  // [tile][row g / g + 8]
    #pragma unroll
                            for (int t = 0; t < 2; ++t)
    #pragma unroll
                                for (int r = 0; r < 2; ++r) {
                                    const uint32_t W = dk_word(A[t][r], i);
                                    E[t][r] = prmt(W, 0u, 0x4240u);
                                    O[t][r] = prmt(W, 0u, 0x4341u);
                                }
    #pragma unroll
                            for (int p = 0; p < 5; ++p) {
                                uint2 bq = make_uint2(0u, 0u);
                                if (g < M) bq = *reinterpret_cast<const uint2 *>(xb + dk_h3off(v, i, p, g, c, Mp));
                                uint32_t dE[2][2], dO[2][2];
    #pragma unroll
                                for (int t = 0; t < 2; ++t)
    #pragma unroll
                                    for (int r = 0; r < 2; ++r) {
                                        if (p < 4) {
                                            // d_p = q_p - 3 q_{p+1} per lane (never negative)
                                            const uint32_t e1 = prmt(E[t][r] * 85u + 0x00550055u, 0u, 0x4341u);
                                            const uint32_t o1 = prmt(O[t][r] * 85u + 0x00550055u, 0u, 0x4341u);
                                            dE[t][r] = E[t][r] - 3u * e1;
                                            dO[t][r] = O[t][r] - 3u * o1;
                                            E[t][r] = e1;
                                            O[t][r] = o1;
                                        } else {
                                            dE[t][r] = E[t][r];
                                            dO[t][r] = O[t][r];
                                        }
                                    }
    #pragma unroll
                                for (int t = 0; t < 2; ++t)
                                    mma_16816(facc[t], dE[t][0], dE[t][1], dO[t][0], dO[t][1], bq.x, bq.y);
                            }
                        }
                        release(slot);
                    }
                    if (!ok) break;
                    if (pi >= NB && !dk_warp_wait(&pempty[b], (uint32_t)((pi / NB) - 1) & 1u))
                        break;
                    float *p = reinterpret_cast<float *>(pb);
    #pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        float sv[4];
    #pragma unroll
                        for (int q = 0; q < 4; ++q) sv[q] = facc[t][q] * 16777216.0f;
                        if (qv == 0) {
                            sv[0] -= sx0;
                            sv[1] -= sx1;
                            sv[2] -= sx0;
                            sv[3] -= sx1;
                        }
                        const int m0 = 2 * c, m1 = 2 * c + 1;
                        if (m0 < M) {
                            p[((m0 * 16 + cw) * 2 + t) * 16 + g] = sv[0];
                            p[((m0 * 16 + cw) * 2 + t) * 16 + g + 8] = sv[2];
                        }
                        if (m1 < M) {
                            p[((m1 * 16 + cw) * 2 + t) * 16 + g] = sv[1];
                            p[((m1 * 16 + cw) * 2 + t) * 16 + g + 8] = sv[3];
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[b]);
            ++pi;
        }
    }

    __syncthreads();
    if (threadIdx.x == 0) {
        // the last CTA out leaves the workspace counters at zero for the next launch
        __threadfence();
        const uint32_t done = atomicAdd(&a.ctr[kDkCtrDone], 1u);
        if (done == gridDim.x - 1) {
            __threadfence();
            a.ctr[kDkCtrItems] = 0u;
            a.ctr[kDkCtrUnitsDone] = 0u;
            for (int l = 0; l < a.count; ++l) a.ready[l] = a.lfinal[l] = a.claim[l] = 0u;
            a.ctr[kDkCtrDone] = 0u;
        }
    }
}

}  // namespace tlk

// ---- host side ---------------------------------------------------------------
namespace tlk {

// Relative cost of a stage: the fp16 engine (M >= 3) takes about twice (2-bit)
// or three times (base 3, whose digits take a division each) as long per
// stage as the integer engine.
inline int dk_stage_cost(int fmt, int M) { return M <= kDkImmaMaxM ? 1 : (fmt == 2 ? 2 : 3); }
// Cost per item for a batch of total cost `total` (in integer-engine stages):
// a few items per SM of a B200, so that the longest-first order leaves a
// short tail, but 4..16 integer-engine stages of cost, so item boundaries
// (and the epilogue work per item) stay rare.  Three items per SM for 2-bit
// and four for base 3, whose ALU-bound stages gain nothing from the extra
// bandwidth the last CTAs of a launch find (measured on batches of the six
// decode shapes at M = 1, 8 and both: 2-bit both 45.4 -> 43.0 us with three
// instead of four, the rest unchanged; base 3 slower with fewer items).
inline int dk_item_cost(int fmt, int64_t total) {
    const int64_t t = total / ((fmt == 2 ? 3 : 4) * kDkRefSms);
    return t < 4 ? 4 : (t > 16 ? 16 : (int)t);
}
// K-parts of a layer: items of about `target` stages, cut at stage
// boundaries, never more than kDkMaxItemStages stages per item.
inline int dk_parts(int stages, int target) {
    if (target < 1) target = 1;
    int parts = (stages + target / 2) / target;
    if (parts < 1) parts = 1;
    while ((stages + parts - 1) / parts > kDkMaxItemStages) ++parts;
    if (parts > stages) parts = stages;
    return parts;
}

struct DkHostLayer {
    const uint8_t *T;
    const uint16_t *X;
    uint16_t *Y;
    int64_t ldp, ldx, ldy;
    float alpha;
    int M, N, K;
    bool reads_earlier;
    bool swiglu;  // X rows hold [gate | up] (only with reads_earlier)
};

struct DkSchedule {
    int count = 0, total_items = 0, total_units = 0, total_tiles = 0, maxM = 1, chained = 0;
    int64_t slots = 0, staged = 0;
    size_t bytes = 0;
};

// Packed bytes of a row of K trits: 4 (2-bit) or 5 (1.6-bit) trits per byte.
inline int64_t dk_row_bytes(int fmt, int64_t K) { return fmt == 2 ? (K + 3) / 4 : (K + 4) / 5; }

// Sizes of a batch; with `items` and `units` given, also their tables, holding
// pointers into the workspace at `ws`.  Items are in layer order, then tile,
// then part (longest first when no layer reads an earlier one); units in
// layer order, then stage, then token.
inline DkSchedule dk_schedule(int fmt, int count, const DkHostLayer *in, uint8_t *ws,
                              std::vector<DkItemRec> *items, std::vector<DkUnitRec> *units) {
    DkSchedule sc;
    sc.count = count;
    auto stages_of = [fmt](const DkHostLayer &h) {
        return (int)((dk_row_bytes(fmt, h.K) + kDkStageW - 1) / kDkStageW);
    };
    auto stage_cost = [fmt](int M) { return dk_stage_cost(fmt, M); };
    int64_t total = 0;
    for (int l = 0; l < count; ++l)
        total += (int64_t)stages_of(in[l]) * ((in[l].N + kDkRows - 1) / kDkRows) *
                 stage_cost(in[l].M);
    const int cost = dk_item_cost(fmt, total);
    // fp16-engine items stay at 8 stages or more: their epilogue (M outputs
    // per row) must keep up with the consumers.  A layer that waits for the
    // earlier layers starts alone, so its items are sized to spread it over
    // about one CTA per SM instead (at most 8 parts per tile for the integer
    // engine, 2 for the fp16 engine, whose final sums of split tiles cost more).
    auto target_of = [&](const DkHostLayer &h) {
        if (h.reads_earlier) {
            const int64_t units = (int64_t)stages_of(h) * ((h.N + kDkRows - 1) / kDkRows);
            const int t = (int)((units + kDkRefSms - 1) / kDkRefSms);
            const int min_t = (stages_of(h) + (h.M > kDkImmaMaxM ? 1 : 7)) / (h.M > kDkImmaMaxM ? 2 : 8);
            return t > min_t ? t : (min_t > 0 ? min_t : 1);
        }
        const int t = cost / stage_cost(h.M);
        return h.M > kDkImmaMaxM && t < 8 ? 8 : t;
    };
    // An independent layer whose X (pointer, stride, K, M) is an earlier
    // independent layer's uses that layer's conversion (Q, K and V of one
    // token batch convert X once); src[l] is the layer that converts.
    std::vector<int> src(count);
    for (int l = 0; l < count; ++l) {
        src[l] = l;
        if (in[l].reads_earlier) continue;
        for (int j = 0; j < l; ++j)
            if (src[j] == j && !in[j].reads_earlier && in[j].X == in[l].X &&
                in[j].ldx == in[l].ldx && in[j].K == in[l].K && in[j].M == in[l].M) {
                src[l] = j;
                break;
            }
    }
    // The earlier layers whose Y overlaps a dependent layer's X (its rows of K,
    // or 2K with the SwiGLU input, elements): deps[l] = (lo << 16) | (hi + 1)
    // for the first and last of them, 0 if none (X is then final at the start).
    std::vector<int> deps(count, 0);
    for (int l = 0; l < count; ++l) {
        if (!in[l].reads_earlier) continue;
        const DkHostLayer &h = in[l];
        const uint8_t *x0 = reinterpret_cast<const uint8_t *>(h.X);
        const uint8_t *x1 = x0 + 2 * ((int64_t)(h.M - 1) * h.ldx + (h.swiglu ? 2 * (int64_t)h.K : h.K));
        int lo = -1, hi = -1;
        for (int j = 0; j < l; ++j) {
            const uint8_t *y0 = reinterpret_cast<const uint8_t *>(in[j].Y);
            const uint8_t *y1 = y0 + 2 * ((int64_t)(in[j].M - 1) * in[j].ldy + in[j].N);
            if (y0 < x1 && x0 < y1) {
                if (lo < 0) lo = j;
                hi = j;
            }
        }
        if (lo >= 0) deps[l] = (lo << 16) | (hi + 1);
    }
    for (int l = 0; l < count; ++l) {
        const DkHostLayer &h = in[l];
        const int stages = stages_of(h);
        const int parts = dk_parts(stages, target_of(h));
        const int tiles = (h.N + kDkRows - 1) / kDkRows;
        sc.total_items += tiles * parts;
        sc.total_tiles += tiles;
        if (h.reads_earlier) {
            if (sc.chained == 0) sc.chained = 1;
            if (h.swiglu) sc.chained = 2;
            if (h.M > kDkImmaMaxM)  // kDkItemCoop: converted once, during the launch
                sc.staged += (int64_t)stages * (kDkMetaBytes + dk_stage_b(fmt, h.M));
        } else if (src[l] == l) {
            sc.total_units += stages * h.M;
            sc.staged += (int64_t)stages * (kDkMetaBytes + dk_stage_b(fmt, h.M));
        }
        if (parts > 1) sc.slots += (int64_t)tiles * parts * kDkRows * h.M;
        if (h.M > sc.maxM) sc.maxM = h.M;
    }
    const DkWsLayout wl(count, sc.total_items, sc.total_units, sc.total_tiles, sc.slots, sc.staged);
    sc.bytes = wl.total;
    if (!items || !units) return sc;
    int64_t slots = 0, staged = 0;
    int tile_begin = 0;
    std::vector<uint8_t *> Bs(count, nullptr);  // each layer's converted X
    for (int l = 0; l < count; ++l) {
        const DkHostLayer &h = in[l];
        const int stages = stages_of(h);
        const int parts = dk_parts(stages, target_of(h));
        const int tiles = (h.N + kDkRows - 1) / kDkRows;
        const int bstride = kDkMetaBytes + (int)dk_stage_b(fmt, h.M);
        // A dependent layer for the fp16 engine converts its X once, during the
        // launch (kDkItemCoop); one for the integer engine converts per item on
        // chip (one or two tokens per stage: cheaper than a round trip)
        const bool coop = h.reads_earlier && h.M > kDkImmaMaxM;
        const bool converts = (!h.reads_earlier && src[l] == l) || coop;
        uint8_t *B = h.reads_earlier && !coop ? nullptr : (converts ? ws + wl.staged + staged : Bs[src[l]]);
        Bs[l] = B;
        for (int t = 0; t < tiles; ++t)
            for (int q = 0; q < parts; ++q) {
                DkItemRec r{};
                r.X = h.X;
                r.Y = h.Y;
                r.B = B;
                r.part_off = slots;
                r.alpha = h.alpha;
                r.layer = l | (src[l] << 16);
                r.tile = t;
                r.part = q;
                r.s0 = (int)((int64_t)stages * q / parts);
                r.s1 = (int)((int64_t)stages * (q + 1) / parts);
                r.M = h.M;
                r.K = h.K;
                r.N = h.N;
                r.ldx = (int)h.ldx;
                r.ldy = (int)h.ldy;
                r.parts = parts;
                r.tile_begin = tile_begin;
                r.deps = deps[l];
                r.need = B ? stages * h.M : 0;
                r.bstride = bstride;
                r.flags = (h.swiglu ? kDkItemSwiglu : 0) | (coop ? kDkItemCoop : 0);
                items->push_back(r);
            }
        if (converts && !coop)
            for (int s = 0; s < stages; ++s)
                for (int m = 0; m < h.M; ++m) {
                    DkUnitRec u{};
                    u.X = h.X;
                    u.dst = B + (int64_t)s * bstride;
                    u.layer = l;
                    u.stage = s;
                    u.m = m;
                    u.M = h.M;
                    u.K = h.K;
                    u.ldx = (int)h.ldx;
                    units->push_back(u);
                }
        if (parts > 1) slots += (int64_t)tiles * parts * kDkRows * h.M;
        if (converts) staged += (int64_t)stages * bstride;
        tile_begin += tiles;
    }
    // Items are handed out in table order.  Without dependencies between
    // layers, the costliest items go first, so the last ones handed out (the
    // launch's tail) are the cheapest.  A part of a split tile also counts
    // the finish its tile may need (one round of loads per token and per
    // four parts, about a stage each), so split tiles finish early.
    if (!sc.chained) {
        std::stable_sort(items->begin(), items->end(), [&](const DkItemRec &x, const DkItemRec &y) {
            auto cost = [&](const DkItemRec &r) {
                return (r.s1 - r.s0) * stage_cost(r.M) + (r.parts > 1 ? r.M * ((r.parts + 3) / 4) : 0);
            };
            return cost(x) > cost(y);
        });
        return sc;
    }
    // With dependencies, a dependent layer's items must follow every item of
    // the layers it reads (then everything it waits for was handed out before
    // it); they follow every earlier layer's.  Within that rule, each dependent layer's items are handed out
    // after the independent layers that follow it, just before the next
    // dependent layer's: a CTA that takes a dependent item then mostly finds
    // its inputs complete instead of waiting while independent work remains.
    // A chain of dependent layers keeps its order.
    std::vector<DkItemRec> ordered;
    ordered.reserve(items->size());
    size_t i = 0, pending_begin = 0, pending_end = 0;  // the held-back dependent layer
    while (i < items->size()) {
        const int layer = (*items)[i].layer & 0xFFFF;
        size_t j = i;
        while (j < items->size() && ((*items)[j].layer & 0xFFFF) == layer) ++j;
        if ((*items)[i].deps != 0) {
            ordered.insert(ordered.end(), items->begin() + pending_begin,
                           items->begin() + pending_end);
            pending_begin = i;
            pending_end = j;
        } else {
            ordered.insert(ordered.end(), items->begin() + i, items->begin() + j);
        }
        i = j;
    }
    ordered.insert(ordered.end(), items->begin() + pending_begin, items->begin() + pending_end);
    items->swap(ordered);
    return sc;
}

// Tensor map of a layer's packed weights: bytes x rows, boxes of 128 bytes x
// 256 rows with the 128-byte swizzle, zero fill outside [0, row bytes) x [0, N).
inline bool dk_encode_map(int fmt, const DkHostLayer &h, CUtensorMap *map) {
    auto encode = tensor_map_encoder();
    if (!encode) return false;
    const int64_t rowbytes = dk_row_bytes(fmt, h.K);
    cuuint64_t dims[2] = {(cuuint64_t)rowbytes, (cuuint64_t)h.N};
    cuuint64_t strides[1] = {(cuuint64_t)h.ldp};
    cuuint32_t box[2] = {(cuuint32_t)kDkStageW, (cuuint32_t)kDkRows};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(h.T), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline DkArgs dk_args(void *ws, int count, int total_items, int total_units, int total_tiles,
                      int maxM, int chained) {
    const DkWsLayout wl(count, total_items, total_units, total_tiles, 0, 0);
    uint8_t *b = reinterpret_cast<uint8_t *>(ws);
    DkArgs a;
    a.ctr = reinterpret_cast<uint32_t *>(b);
    a.maps = reinterpret_cast<const CUtensorMap *>(b + wl.maps);
    a.items = reinterpret_cast<const DkItemRec *>(b + wl.items);
    a.units = reinterpret_cast<const DkUnitRec *>(b + wl.units);
    a.ready = reinterpret_cast<uint32_t *>(b + wl.ready);
    a.lfinal = a.ready + count;
    a.ltiles = a.ready + 2 * count;
    a.claim = a.ready + 3 * count;
    a.tile_ctr = reinterpret_cast<uint32_t *>(b + wl.tiles);
    a.partials = reinterpret_cast<int64_t *>(b + wl.partials);
    a.count = count;
    a.total_items = total_items;
    a.total_units = total_units;
    a.maxM = maxM;
    a.chained = chained;
    a.drop_arrive = 0;
    // short launches with large partials (M > 4, under 8 items per SM):
    // their epilogues and tail, not the stream, set the pace, so four
    // epilogue buffers pay for one stage less of ring
    a.wide = maxM > 4 && total_items < 8 * kDkRefSms ? 1 : 0;
    return a;
}

template <int FMT>
inline int launch_decode2(const DkArgs &a, int num_sms, bool pdl, cudaStream_t stream,
                          int *last_cuda_error) {
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static cudaError_t attr_err[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        *last_cuda_error = (int)e;
        return 5;
    }
    std::call_once(once[dev], [dev] {
        uint32_t most = 0;
        for (int m = 1; m <= 8; ++m) {
            for (int w = 0; w < 2; ++w) {
                const uint32_t t = DkLayout(FMT, m, w != 0).total;
                most = t > most ? t : most;
            }
        }
        attr_err[dev] = cudaFuncSetAttribute(decode2_kernel<FMT, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
        if (attr_err[dev] == cudaSuccess)
            attr_err[dev] = cudaFuncSetAttribute(
                decode2_kernel<FMT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
    });
    if (attr_err[dev] != cudaSuccess) {
        *last_cuda_error = (int)attr_err[dev];
        return 5;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.total_items < num_sms ? a.total_items : num_sms));
    cfg.blockDim = dim3(kDkThreads);
    cfg.dynamicSmemBytes = DkLayout(FMT, a.maxM, a.wide != 0).total;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 1 : 0;
    e = a.chained == 2 ? cudaLaunchKernelEx(&cfg, decode2_kernel<FMT, true>, a)
                       : cudaLaunchKernelEx(&cfg, decode2_kernel<FMT, false>, a);
    if (e != cudaSuccess) (void)cudaGetLastError();  // the error is returned here, once
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

}  // namespace tlk

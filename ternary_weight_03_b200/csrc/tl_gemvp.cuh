// tl_gemvp.cuh -- a batch of decode-shaped ternary layers (M = 1..8 tokens
// each) in ONE persistent launch:
//   for every layer l:  Y_l[m][n] = fp16_rn(alpha_l * sum_k T_l[n][k] X_l[m][k]).
//
// Why: the pages' decode phase is bound by streaming the packed weights once
// ("Pith review of Spectra 1.1", "What carries the argument": memory bandwidth,
// not compute, is the bottleneck of decoding).  A 2-15 MB layer read by its own
// launch spends as long starting, staging and draining as streaming; one
// launch per layer cannot approach HBM speed.  Here one CTA per SM streams a
// queue of work items across all the layers of the batch without pausing at
// layer boundaries.
//
// Work item = (layer, tile of 120 weight rows, K-part).  A layer's K-groups
// (64 packed bytes per row each) are cut into `parts` contiguous ranges so
// that items are all about the same size; CTA b of G takes the items b,
// b + G, b + 2G, ... (its first item's weights are fetched before the
// previous grid finishes, and the next item's record is loaded while the
// current one streams).
//
// Every copy is a TMA copy: per stage (gp_sg K-groups) one 2D tensor-map box
// of the tile's 120 rows (zero-filled past N and past the row), and one 1D
// bulk copy per token of the activations at those K positions.  (Per-thread
// cp.async through L1 was measured at ~8-10 GB/s per SM here, far below the
// ~40 GB/s per SM that HBM speed needs.)  The per-layer tensor maps and the
// layer table live in the workspace, written once by tl_gemv_batch_plan.
//
// Warp roles of a CTA (704 threads):
//  * warp 0, producer: one elected lane issues each stage's copies into a ring
//    of stages (completion counted in bytes on the stage's mbarrier) and
//    queues the items for the other roles;
//  * warps 1..3, stagers (warp 1 + i owns the ring slots s with s mod 3 = i):
//    rewrite each stage's activations from natural order into the consumers'
//    layout (2-bit: the
//    pair order of the class-masked decode, see g3_word2; 1.6-bit: the
//    interleaved units of gemv16_word), with zeros at k >= K;
//  * warps 6..21, consumers: the decode + mma.sync of tl_gemv3.cuh (15 weight
//    rows and the all-ones row per warp; the two warps of a row tile take
//    alternate K-groups of each stage), accumulating over the item's stages,
//    then handing the item's 2 x 120 x M sums to
//  * warps 4 and 5, epilogues (alternate items): y = alpha * (sum - ones-row
//    sum) to Y when the layer has one part; otherwise the part's fp32
//    partial goes to the workspace and the
//    last of the tile's parts to arrive (per-tile counter) adds the parts in
//    part order (deterministic) and stores Y.  The tree reduction of per-warp
//    partials through shared memory follows the Figure 11 caption text on
//    appendix G.4 of the same page; the cross-CTA step is this file's own.
// Layers flagged as reading an earlier layer's output wait (bounded) until
// every tile of the earlier layers is final.  All waits are bounded; a
// timeout sets the device error word.  The last CTA to finish resets the
// workspace counters, so they stay zero between launches.
#pragma once
#include <cuda.h>
#include <mutex>
#include "tl_common.cuh"
#include "tl_sm100.cuh"
#include "tl_gemv.cuh"
#include "tl_gemv3.cuh"

namespace tlk {

constexpr int kGpRowTiles = 8;                               // 15-row tiles per item
constexpr int kGpConsumers = 2 * kGpRowTiles;                 // two warps per row tile
constexpr int kGpStagers = 3;                                 // stager warps (each owns ring slots)
constexpr int kGpEpilogues = 2;                               // epilogue warps (alternate items)
constexpr int kGpFirstEpi = 1 + kGpStagers;                   // warp index of the first epilogue
constexpr int kGpFirstCons = kGpFirstEpi + kGpEpilogues;      // warp index of the first consumer
constexpr int kGpWarps = kGpFirstCons + kGpConsumers;
constexpr int kGpThreads = 32 * kGpWarps;                    // 704
constexpr int kGpRows = kGpRowTiles * kG3TileRows;            // 120 weight rows per item
// K-groups per stage: 4 for 2-bit (256 B per row, 30 KB of weights per stage),
// 2 for 1.6-bit, whose larger activation slots would otherwise leave too few
// stages in shared memory at M = 8.
__host__ __device__ constexpr int gp_sg(int fmt) { return fmt == 2 ? 4 : 2; }
__host__ __device__ constexpr int gp_stage_w(int fmt) { return gp_sg(fmt) * kGemvGroupBytes; }
__host__ __device__ constexpr int gp_wbytes(int fmt) { return kGpRows * gp_stage_w(fmt); }
constexpr int kGpMaxStages = 8;
constexpr int kGpQueue = 32;                                  // items in flight per CTA
constexpr int kGpPartBufs = 2;                                // consumer -> epilogue buffers
constexpr int kGpPartFloats = kGpConsumers * 16 * 8;          // 2048 floats per buffer
constexpr uint32_t kGpSmemBudget = 220u * 1024u;
constexpr int kGpHeaderWords = 64;                            // workspace counters (256 B)

// One layer of a batch as the kernel reads it from the workspace.
struct GpLayer {
    const uint8_t *T;
    const uint16_t *X;
    uint16_t *Y;
    int64_t ldp;       // bytes
    int64_t part_off;  // first float of this layer's partial slots
    int ldx, ldy;      // elements
    float alpha;
    int M, N, K;
    int groups;        // 64-byte K-groups per packed row
    int parts;         // K-parts per tile
    int tiles;         // 120-row tiles
    int item_begin;    // global index of the layer's first item
    int tile_begin;    // global index of the layer's first tile
    int wait_tiles;    // tiles that must be final before X is read (0: none)
    int pad_;
};

// Workspace layout of a planned batch (every region 256-byte aligned):
//   header  : kGpHeaderWords u32 counters: [1] final tiles, [2] CTAs done ([0] unused)
//   layers  : count x GpLayer
//   maps    : count x CUtensorMap (the packed weights of each layer)
//   tiles   : total_tiles x u32, parts of each tile that have arrived
//   partials: fp32 partial sums of split tiles
struct GpWsLayout {
    size_t layers, maps, tiles, partials, total;
    GpWsLayout(int count, int total_tiles, int64_t floats) {
        auto up = [](size_t v) { return (v + 255u) & ~(size_t)255u; };
        layers = 256;
        maps = up(layers + (size_t)count * sizeof(GpLayer));
        tiles = up(maps + (size_t)count * sizeof(CUtensorMap));
        partials = up(tiles + (size_t)total_tiles * 4u);
        total = up(partials + (size_t)floats * 4u);
    }
};

// Kernel parameters: pointers into the workspace and the batch's sizes.
struct GpArgs {
    uint32_t *ctr;
    const GpLayer *L;
    const CUtensorMap *maps;
    uint32_t *tile_ctr;
    float *partials;
    int count;
    int total_items;
    int maxM;
};

// What the producer tells the other roles about an item (shared memory).
struct GpQEntry {
    uint16_t *Y;
    int64_t part_off;
    float alpha;
    int item;  // -1: no more items
    int tile, part, g0, g1, M, K, N, ldy, parts, tile_begin;
};

// Shared-memory layout of one launch; maxM = the most tokens of any layer.
struct GpLayout {
    uint32_t ns, xtok, raw_tok, raw_stage, x_stage, raw_off, x_off, part_off, q_off, bar_off,
        total;
    __host__ __device__ GpLayout(int fmt, int maxM) {
        const uint32_t group_bytes = fmt == 2 ? 512u : 640u;  // activations per token per group
        raw_tok = gp_sg(fmt) * group_bytes;                 // natural order, as copied
        xtok = gp_sg(fmt) * group_bytes + 64u;              // staged token stride (bank offset)
        raw_stage = (raw_tok * (uint32_t)maxM + 127u) & ~127u;
        x_stage = (xtok * (uint32_t)maxM + 127u) & ~127u;
        const uint32_t per_stage = (uint32_t)gp_wbytes(fmt) + raw_stage + x_stage;
        const uint32_t fixed = (uint32_t)kGpPartBufs * kGpPartFloats * 4u +
                               kGpQueue * (uint32_t)sizeof(GpQEntry) +
                               8u * (3u * kGpMaxStages + 2u * kGpQueue + 2u * kGpPartBufs) + 256u;
        const uint32_t n = (kGpSmemBudget - fixed) / per_stage;
        ns = n > (uint32_t)kGpMaxStages ? (uint32_t)kGpMaxStages : n;  // >= 3 for M <= 8
        raw_off = ns * (uint32_t)gp_wbytes(fmt);
        x_off = raw_off + ns * raw_stage;
        part_off = x_off + ns * x_stage;
        q_off = part_off + (uint32_t)kGpPartBufs * kGpPartFloats * 4u;
        bar_off = (q_off + kGpQueue * (uint32_t)sizeof(GpQEntry) + 7u) & ~7u;
        total = bar_off + 8u * (3u * ns + 2u * kGpQueue + 2u * kGpPartBufs) + 128u;
    }
};

struct GpItem {
    int l, tile, part, g0, g1;
};

template <int SG>
__device__ __forceinline__ GpItem gp_decode(const GpArgs &a, int item) {
    int lo = 0, hi = a.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(&a.L[mid].item_begin) <= item) lo = mid;
        else hi = mid - 1;
    }
    const GpLayer *L = a.L + lo;
    const int parts = __ldg(&L->parts), groups = __ldg(&L->groups);
    const int local = item - __ldg(&L->item_begin);
    GpItem it;
    it.l = lo;
    it.tile = local / parts;
    it.part = local % parts;
    // parts cut at stage (SG-group) boundaries
    const int stages = (groups + SG - 1) / SG;
    it.g0 = SG * (int)((int64_t)stages * it.part / parts);
    it.g1 = min(groups, SG * (int)((int64_t)stages * (it.part + 1) / parts));
    return it;
}

// 1D bulk copy global -> shared (TMA, no tensor map), completing `bytes` on `bar`.
// Addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Raise the bytes a phase expects without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Every lane waits; the warp proceeds only if all lanes saw the phase.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// Read the next queued item and release its queue slot; false at the end
// of the queue (or on a timeout).
__device__ __forceinline__ bool gp_next_item(const GpQEntry *queue, uint64_t *qfull,
                                             uint64_t *qempty, int &qi, GpQEntry &e) {
    const int q = qi % kGpQueue;
    if (!warp_wait(&qfull[q], (uint32_t)(qi / kGpQueue) & 1u)) return false;
    e = queue[q];
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&qempty[q]);
    ++qi;
    return e.item >= 0;
}

template <int FMT>
__global__ void __launch_bounds__(kGpThreads, 1) gemvp_kernel(const __grid_constant__ GpArgs a) {
    constexpr int TPB = FMT == 2 ? 4 : 5;
    constexpr int TRITS_GROUP = kGemvGroupBytes * TPB;  // 256 / 320 activations per group
    constexpr int SG = gp_sg(FMT);                       // K-groups per stage
    constexpr int STAGE_W = gp_stage_w(FMT);             // weight bytes per row per stage
    constexpr int WBYTES = gp_wbytes(FMT);               // weight bytes per stage
    constexpr int TRITS_STAGE = SG * TRITS_GROUP;        // activations per token per stage
    constexpr int XUNITS = TRITS_STAGE / 8;              // 16-byte units per token per stage
    constexpr int GBYTES = G3X<FMT>::group_bytes;        // staged bytes per token per group
    constexpr uint32_t ONES = FMT == 2 ? 0x55555555u : 0x79797979u;  // every digit 1
    extern __shared__ __align__(128) uint8_t gp_smem_raw[];
    __shared__ uint32_t lut_even[FMT == 2 ? 1 : 256];
    __shared__ uint32_t lut_odd[FMT == 2 ? 1 : 256];

    const GpLayout lay(FMT, a.maxM);
    const int NS = (int)lay.ns;
    uint8_t *smem = gp_smem_raw + ((128u - (smem_u32(gp_smem_raw) & 127u)) & 127u);
    uint8_t *wring = smem;
    uint8_t *rawx = smem + lay.raw_off;
    uint8_t *xs = smem + lay.x_off;
    float *parts = reinterpret_cast<float *>(smem + lay.part_off);
    GpQEntry *queue = reinterpret_cast<GpQEntry *>(smem + lay.q_off);
    uint64_t *wfull = reinterpret_cast<uint64_t *>(smem + lay.bar_off);  // copies landed
    uint64_t *xfull = wfull + NS;                                         // stager -> consumers
    uint64_t *empty = xfull + NS;                                         // consumers -> producer
    uint64_t *qfull = empty + NS;
    uint64_t *qempty = qfull + kGpQueue;
    uint64_t *pfull = qempty + kGpQueue;  // consumers -> epilogue
    uint64_t *pempty = pfull + kGpPartBufs;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&wfull[i], 1);
            mbar_init(&xfull[i], 32);
            mbar_init(&empty[i], kGpConsumers);
        }
        for (int i = 0; i < kGpQueue; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], kGpConsumers + kGpStagers + kGpEpilogues);
        }
        for (int i = 0; i < kGpPartBufs; ++i) {
            mbar_init(&pfull[i], kGpConsumers);
            mbar_init(&pempty[i], 1);
        }
        fence_mbar_init();
    }
    if constexpr (FMT != 2) build_lut16(lut_even, lut_odd);
    __syncthreads();
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- producer ----------------
        // Items b, b + G, b + 2G, ... (G CTAs): the next item is known at once, so
        // its layer record is loaded while the current item streams.
        uint32_t stage = 0;
        int ps = 0;               // ring slot of the next stage
        uint32_t pph = 0;         // its round's parity
        bool wrapped = false;     // the ring has been filled once
        int qi = 0;
        bool waited = false, ok = true;
        uint32_t final_seen = 0;  // lower bound of the final-tile counter
        int item = (int)blockIdx.x;
        GpItem it{};
        GpLayer L{};
        if (item < a.total_items) {
            it = gp_decode<SG>(a, item);
            L = a.L[it.l];
        }
        while (ok) {
            const int q = qi % kGpQueue;
            if (qi >= kGpQueue && !warp_wait(&qempty[q], (uint32_t)((qi / kGpQueue) - 1) & 1u)) {
                ok = false;
                break;
            }
            const bool valid = item < a.total_items;
            if (lane == 0) {
                GpQEntry e{};
                e.item = valid ? item : -1;
                if (valid) {
                    e.Y = L.Y;
                    e.part_off = L.part_off;
                    e.alpha = L.alpha;
                    e.tile = it.tile;
                    e.part = it.part;
                    e.g0 = it.g0;
                    e.g1 = it.g1;
                    e.M = L.M;
                    e.K = L.K;
                    e.N = L.N;
                    e.ldy = L.ldy;
                    e.parts = L.parts;
                    e.tile_begin = L.tile_begin;
                }
                queue[q] = e;
                mbar_arrive(&qfull[q]);
            }
            ++qi;
            if (!valid) break;
            // the item after this one: decode it and start loading its record now
            const int next = item + (int)gridDim.x;
            GpItem nit{};
            GpLayer NL{};
            if (next < a.total_items) {
                nit = gp_decode<SG>(a, next);
                NL = a.L[nit.l];
            }
            const CUtensorMap *tmap = a.maps + it.l;
            const int n0 = it.tile * kGpRows;
            // activation bytes of the stage at group g for one token (whole 16-byte units)
            auto xbytes = [&](int g) -> uint32_t {
                const int rem = L.K - g * TRITS_GROUP;
                const int n = rem < TRITS_STAGE ? ((rem + 7) & ~7) : TRITS_STAGE;
                return 2u * (uint32_t)n;
            };
            auto issue_x = [&](int s, int g) {
                const uint32_t b = xbytes(g);
                for (int m = 0; m < L.M; ++m)
                    bulk_load(rawx + s * lay.raw_stage + m * lay.raw_tok,
                              L.X + (int64_t)m * L.ldx + g * TRITS_GROUP, b, &wfull[s]);
            };
            auto wait_deps = [&]() -> bool {
                if (L.wait_tiles <= 0 || final_seen >= (uint32_t)L.wait_tiles) return true;
                bool good = true;
                if (lane == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    uint32_t v = ld_acquire_gpu(&a.ctr[1]);
                    while (v < (uint32_t)L.wait_tiles) {
                        if (globaltimer_ns() - t0 > kWaitLimitNs) {
                            atomicOr(&g_error_word, kErrTimeout);
                            good = false;
                            break;
                        }
                        __nanosleep(64);
                        v = ld_acquire_gpu(&a.ctr[1]);
                    }
                    final_seen = v;
                }
                final_seen = __shfl_sync(0xffffffffu, final_seen, 0);
                return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
            };
            int g = it.g0;
            if (!waited) {
                // first item: weights of up to a ring's worth of stages before the
                // previous grid ends (expected bytes raised now, the arrival later)
                const int nst = (it.g1 - it.g0 + SG - 1) / SG;
                const int pre = min(nst, NS);
                if (lane == 0) {
                    tma_prefetch_desc(tmap);
                    for (int i = 0; i < pre; ++i) {
                        const int s = (int)((stage + i) % NS);
                        mbar_expect_tx(&wfull[s], WBYTES);
                        tma_load_2d(wring + s * WBYTES, tmap, &wfull[s],
                                    (it.g0 + SG * i) * kGemvGroupBytes, n0);
                    }
                }
                pdl_wait();
                waited = true;
                const bool deps = wait_deps();
                // the stages already counted on their barriers still get their arrival
                if (lane == 0) {
                    for (int i = 0; i < pre; ++i) {
                        const int s = (int)((stage + i) % NS);
                        const int gi = it.g0 + SG * i;
                        mbar_arrive_expect_tx(&wfull[s], deps ? (uint32_t)L.M * xbytes(gi) : 0u);
                        if (deps) issue_x(s, gi);
                    }
                }
                __syncwarp();
                stage += pre;
                g += SG * pre;
                ps = pre;
                if (ps == NS) { ps = 0; pph = 1; wrapped = true; }
                if (!deps) { ok = false; break; }
            } else if (!wait_deps()) {
                ok = false;
                break;
            }
            for (; g < it.g1; g += SG, ++stage) {
                const int s = ps;
                if (wrapped && !warp_wait(&empty[s], pph ^ 1u)) {
                    ok = false;
                    break;
                }
                if (++ps == NS) {
                    ps = 0;
                    pph ^= 1u;
                    wrapped = true;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&wfull[s], WBYTES + (uint32_t)L.M * xbytes(g));
                    tma_load_2d(wring + s * WBYTES, tmap, &wfull[s], g * kGemvGroupBytes, n0);
                    issue_x(s, g);
                }
                __syncwarp();
            }
            if (!ok) break;
            item = next;
            it = nit;
            L = NL;
        }
        if (!waited) pdl_wait();
        // the CTA may not exit with copies still landing in its shared memory
        for (uint32_t t = stage > (uint32_t)NS ? stage - NS : 0; t < stage; ++t)
            mbar_wait(&wfull[t % NS], (t / NS) & 1u);
    } else if (warp < kGpFirstEpi) {
        // ---------------- stagers: warp 1 + i takes the ring slots s with s % kGpStagers == i ----
        // (owning slots, not every k-th stage: a stager then waits every round of
        // its slots in order, so a parity wait never sees a phase two rounds back)
        const int sw = warp - 1;
        int ss = 0;
        uint32_t sph = 0;
        int qi = 0;
        bool ok = true;
        GpQEntry e;
        while (ok && gp_next_item(queue, qfull, qempty, qi, e)) {
            const int M = e.M, K = e.K;
            for (int g = e.g0; g < e.g1; g += SG) {
                const int s = ss;
                const uint32_t ph = sph;
                if (++ss == NS) {
                    ss = 0;
                    sph ^= 1u;
                }
                if (s % kGpStagers != sw) continue;  // another stager's slot
                if (!warp_wait(&wfull[s], ph)) {
                    ok = false;
                    break;
                }
                // activations of this stage below K (and below the item's last group)
                const int valid = min(K - g * TRITS_GROUP, (e.g1 - g) * TRITS_GROUP);
                const uint8_t *raw = rawx + s * lay.raw_stage;
                uint8_t *dst = xs + s * lay.x_stage;
                // unit v of a token keeps its first clamp(valid - 8 v, 0, 8) activations
                auto load_unit = [&](int m, int v) -> uint4 {
                    const int keep = valid - 8 * v;
                    if (keep <= 0) return make_uint4(0u, 0u, 0u, 0u);
                    uint4 u = *reinterpret_cast<const uint4 *>(raw + m * lay.raw_tok + 16 * v);
                    if (keep < 8) {
                        uint32_t *w = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint32_t lo = 2 * i < keep ? 0x0000FFFFu : 0u;
                            const uint32_t hi = 2 * i + 1 < keep ? 0xFFFF0000u : 0u;
                            w[i] &= lo | hi;
                        }
                    }
                    return u;
                };
                if constexpr (FMT == 2) {
                    // natural order -> (x_i, x_{8+i}) pairs of each 16-activation word;
                    // item (token m, group h, lane chunk c, word j)
                    for (int w = lane; w < M * 16 * SG; w += 32) {
                        const int m = w / (16 * SG), r = w % (16 * SG);
                        const int h = r >> 4, c = (r >> 2) & 3, j = r & 3;
                        const int v0 = 32 * h + 8 * c + 2 * j;
                        const uint4 lo4 = load_unit(m, v0), hi4 = load_unit(m, v0 + 1);
                        const uint32_t *lo = reinterpret_cast<const uint32_t *>(&lo4);
                        const uint32_t *hi = reinterpret_cast<const uint32_t *>(&hi4);
                        uint32_t pr[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pr[i] = prmt(lo[i >> 1], hi[i >> 1], (i & 1) ? 0x7632u : 0x5410u);
                        uint8_t *d = dst + m * lay.xtok + h * GBYTES;
                        *reinterpret_cast<uint4 *>(d + ((2 * j) * 4 + c) * 16) =
                            make_uint4(pr[0], pr[1], pr[2], pr[3]);
                        *reinterpret_cast<uint4 *>(d + ((2 * j + 1) * 4 + c) * 16) =
                            make_uint4(pr[4], pr[5], pr[6], pr[7]);
                    }
                } else {
                    // natural order -> unit v of group h at (v % 10) * 4 + v / 10
                    for (int w = lane; w < M * XUNITS; w += 32) {
                        const int m = w / XUNITS, vv = w % XUNITS;
                        const int h = vv / 40, v = vv % 40;
                        *reinterpret_cast<uint4 *>(dst + m * lay.xtok + h * GBYTES +
                                                   ((v % 10) * 4 + v / 10) * 16) =
                            load_unit(m, vv);
                    }
                }
                mbar_arrive(&xfull[s]);
            }
        }
    } else if (warp < kGpFirstCons) {
        // ---------------- epilogues: warp 4 + i takes the items i, i + 2, ... ----------------
        const int ew = warp - kGpFirstEpi;
        pdl_wait();  // Y and the workspace may still be in use by the previous grid
        int qi = 0, pi = -1;
        GpQEntry e;
        while (gp_next_item(queue, qfull, qempty, qi, e)) {
            if (++pi % kGpEpilogues != ew) continue;  // another epilogue warp's item
            const int b = pi % kGpPartBufs;
            if (!warp_wait(&pfull[b], (uint32_t)(pi / kGpPartBufs) & 1u)) break;
            const float *pb = parts + b * kGpPartFloats;
            const int M = e.M, n0 = e.tile * kGpRows, cnt = kGpRows * M;
            float *slot = e.parts > 1 ? a.partials + e.part_off +
                                            (int64_t)(e.tile * e.parts + e.part) * cnt
                                      : nullptr;
            for (int idx = lane; idx < cnt; idx += 32) {
                const int r = idx % kGpRows, m = idx / kGpRows;  // consecutive lanes: consecutive n
                const int w = r / kG3TileRows, rr = r % kG3TileRows;
                const float *p0 = pb + w * 128, *p1 = pb + (w + kGpRowTiles) * 128;
                const float v = (p0[rr * 8 + m] - p0[15 * 8 + m]) + (p1[rr * 8 + m] - p1[15 * 8 + m]);
                if (slot) {
                    slot[idx] = v;
                } else if (n0 + r < e.N) {
                    e.Y[(int64_t)m * e.ldy + n0 + r] = f32_to_f16_bits(e.alpha * v);
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
                    // last part of the tile: add the parts in part order
                    __threadfence();
                    const float *base = a.partials + e.part_off + (int64_t)e.tile * e.parts * cnt;
                    for (int i0 = 0; i0 < cnt; i0 += 32 * 8) {
                        float acc[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) acc[t] = 0.f;
                        for (int q = 0; q < e.parts; ++q) {
#pragma unroll
                            for (int t = 0; t < 8; ++t) {
                                const int idx = i0 + lane + 32 * t;
                                if (idx < cnt) acc[t] += __ldcg(base + (int64_t)q * cnt + idx);
                            }
                        }
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int idx = i0 + lane + 32 * t;
                            const int r = idx % kGpRows, m = idx / kGpRows;
                            if (idx < cnt && n0 + r < e.N)
                                e.Y[(int64_t)m * e.ldy + n0 + r] = f32_to_f16_bits(e.alpha * acc[t]);
                        }
                    }
                    if (lane == 0) a.tile_ctr[e.tile_begin + e.tile] = 0u;
                }
            }
            if (final_tile) {
                // the tile's outputs are stored: count it for layers that read them
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(&a.ctr[1], 1u);
            }
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - kGpFirstCons;
        const int rt = cw % kGpRowTiles, hw = cw / kGpRowTiles;  // row tile, first group
        constexpr int kHStep = kGpConsumers / kGpRowTiles;        // warps per row tile
        const int g = lane >> 2, c = lane & 3;
        const bool onesB = (g == 7);
        const int rowA = rt * kG3TileRows + g, rowB = rowA + 8;
        int cs = 0;
        uint32_t cph = 0;
        int qi = 0, pi = 0;
        bool ok = true;
        GpQEntry e;
        while (ok && gp_next_item(queue, qfull, qempty, qi, e)) {
            const int tok = g < e.M ? g : 0;
            float acc[4][4], acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
            for (int gg = e.g0; gg < e.g1; gg += SG) {
                const int s = cs;
                if (!warp_wait(&wfull[s], cph) || !warp_wait(&xfull[s], cph)) {
                    ok = false;
                    break;
                }
                if (++cs == NS) {
                    cs = 0;
                    cph ^= 1u;
                }
                for (int h = hw; h < SG && gg + h < e.g1; h += kHStep) {  // groups of this warp
                    const uint8_t *box = wring + s * WBYTES + h * kGemvGroupBytes + 16 * c;
                    const uint4 wa = *reinterpret_cast<const uint4 *>(box + rowA * STAGE_W);
                    uint4 wb = make_uint4(ONES, ONES, ONES, ONES);
                    if (!onesB) wb = *reinterpret_cast<const uint4 *>(box + rowB * STAGE_W);
                    g3_group<FMT>(wa, wb, xs + s * lay.x_stage + tok * lay.xtok + h * GBYTES, c,
                                  lut_even, lut_odd, acc, acc4);
                }
                // the values read above are consumed (in registers) before the
                // release, after which TMA may refill the stage
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;
            float sv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if constexpr (FMT == 2)
                    sv[q] = acc[0][q] * 16777216.0f + acc[1][q] * 4194304.0f +
                            acc[2][q] * 1048576.0f + acc[3][q] * 262144.0f;
                else
                    sv[q] = (acc[0][q] + acc[1][q]) * 16777216.0f +
                            (acc[2][q] + acc[3][q]) * 1048576.0f + acc4[q] * 65536.0f;
            }
            const int b = pi % kGpPartBufs;
            if (pi >= kGpPartBufs &&
                !warp_wait(&pempty[b], (uint32_t)((pi / kGpPartBufs) - 1) & 1u))
                break;
            float *pw = parts + b * kGpPartFloats + cw * 128;
            pw[g * 8 + 2 * c] = sv[0];
            pw[g * 8 + 2 * c + 1] = sv[1];
            pw[(g + 8) * 8 + 2 * c] = sv[2];
            pw[(g + 8) * 8 + 2 * c + 1] = sv[3];
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[b]);
            ++pi;
        }
    }

    __syncthreads();
    if (threadIdx.x == 0) {
        // the last CTA out leaves the workspace counters at zero for the next launch
        __threadfence();
        const uint32_t done = atomicAdd(&a.ctr[2], 1u);
        if (done == gridDim.x - 1) {
            __threadfence();
            a.ctr[1] = 0u;
            a.ctr[2] = 0u;
        }
    }
}

}  // namespace tlk

// ---- host side ---------------------------------------------------------------
namespace tlk {

// K-parts of a layer: items of about eight stages (32 K-groups for 2-bit, 16
// for 1.6-bit), so the per-item hand-offs stay small against the streaming;
// parts are cut at stage boundaries, so there are at most as many parts as
// stages.
inline int gp_parts(int fmt, int groups, int M) {
    const int target = 8 * gp_sg(fmt);
    const int stages = (groups + gp_sg(fmt) - 1) / gp_sg(fmt);
    int parts = (groups + target / 2) / target;
    if (parts < 1) parts = 1;
    if (parts > stages) parts = stages;
    return parts;
}

// One validated layer as the planner takes it.
struct GpHostLayer {
    const uint8_t *T;
    const uint16_t *X;
    uint16_t *Y;
    int64_t ldp, ldx, ldy;
    float alpha;
    int M, N, K;
    bool reads_earlier;
    bool swiglu = false;  // X holds gate and up halves (2-bit batch only)
};

struct GpSchedule {
    int count = 0, total_items = 0, total_tiles = 0, maxM = 1;
    int64_t floats = 0;
    size_t bytes = 0;
};

// Fills the kernel's layer table (host copy) and returns the batch's sizes.
inline GpSchedule gp_schedule(int fmt, int count, const GpHostLayer *in, GpLayer *out) {
    GpSchedule sc;
    sc.count = count;
    bool after_dependent = false;
    for (int l = 0; l < count; ++l) {
        const GpHostLayer &h = in[l];
        GpLayer &L = out[l];
        const int64_t rowbytes = fmt == 2 ? ((int64_t)h.K + 3) / 4 : ((int64_t)h.K + 4) / 5;
        L = GpLayer{};
        L.T = h.T;
        L.X = h.X;
        L.Y = h.Y;
        L.ldp = h.ldp;
        L.ldx = (int)h.ldx;
        L.ldy = (int)h.ldy;
        L.alpha = h.alpha;
        L.M = h.M;
        L.N = h.N;
        L.K = h.K;
        L.groups = (int)((rowbytes + kGemvGroupBytes - 1) / kGemvGroupBytes);
        L.parts = gp_parts(fmt, L.groups, h.M);
        L.tiles = (h.N + kGpRows - 1) / kGpRows;
        L.item_begin = sc.total_items;
        L.tile_begin = sc.total_tiles;
        // A layer after a dependent one waits too: the final-tile counter only
        // says how many tiles are final, so a later independent layer's tiles
        // must not be able to stand in for an earlier layer's missing ones.
        after_dependent = after_dependent || h.reads_earlier;
        L.wait_tiles = after_dependent ? sc.total_tiles : 0;
        L.part_off = sc.floats;
        if (L.parts > 1) sc.floats += (int64_t)L.tiles * L.parts * kGpRows * h.M;
        sc.total_items += L.tiles * L.parts;
        sc.total_tiles += L.tiles;
        if (h.M > sc.maxM) sc.maxM = h.M;
    }
    sc.bytes = GpWsLayout(count, sc.total_tiles, sc.floats).total;
    return sc;
}

// Tensor map of a layer's packed weights: bytes x rows, boxes of one stage
// (gp_stage_w bytes x 120 rows), zero fill outside [0, row bytes) x [0, N).
inline bool gp_encode_map(int fmt, const GpHostLayer &h, CUtensorMap *map) {
    auto encode = tensor_map_encoder();
    if (!encode) return false;
    const int64_t rowbytes = fmt == 2 ? ((int64_t)h.K + 3) / 4 : ((int64_t)h.K + 4) / 5;
    cuuint64_t dims[2] = {(cuuint64_t)rowbytes, (cuuint64_t)h.N};
    cuuint64_t strides[1] = {(cuuint64_t)h.ldp};
    cuuint32_t box[2] = {(cuuint32_t)gp_stage_w(fmt), (cuuint32_t)kGpRows};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(h.T), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline GpArgs gp_args(void *ws, int count, int total_items, int total_tiles, int maxM) {
    const GpWsLayout wl(count, total_tiles, 0);
    uint8_t *b = reinterpret_cast<uint8_t *>(ws);
    GpArgs a;
    a.ctr = reinterpret_cast<uint32_t *>(b);
    a.L = reinterpret_cast<const GpLayer *>(b + wl.layers);
    a.maps = reinterpret_cast<const CUtensorMap *>(b + wl.maps);
    a.tile_ctr = reinterpret_cast<uint32_t *>(b + wl.tiles);
    a.partials = reinterpret_cast<float *>(b + wl.partials);
    a.count = count;
    a.total_items = total_items;
    a.maxM = maxM;
    return a;
}

template <int FMT>
inline int launch_gemvp(const GpArgs &a, int num_sms, bool pdl, cudaStream_t stream,
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
            const uint32_t t = GpLayout(FMT, m).total;
            most = t > most ? t : most;
        }
        attr_err[dev] = cudaFuncSetAttribute(gemvp_kernel<FMT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
    });
    if (attr_err[dev] != cudaSuccess) {
        *last_cuda_error = (int)attr_err[dev];
        return 5;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.total_items < num_sms ? a.total_items : num_sms));
    cfg.blockDim = dim3(kGpThreads);
    cfg.dynamicSmemBytes = GpLayout(FMT, a.maxM).total;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, gemvp_kernel<FMT>, a);
    if (e != cudaSuccess) (void)cudaGetLastError();  // the error is returned here, once
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

}  // namespace tlk

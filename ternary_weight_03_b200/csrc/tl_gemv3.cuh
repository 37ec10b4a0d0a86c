// tl_gemv3.cuh -- decode-shaped ternary layer (M = 1..8 tokens), TMA-fed:
//   Y[m][n] = fp16_rn(alpha * sum_k T[n][k] * X[m][k]),  2-bit or 1.6-bit T.
//
// Why mma.sync here and not tcgen05: a tcgen05.mma with A in tensor memory
// (M = 128, K = 16) costs ~176 SM cycles whatever N is, so with N = 16 tokens
// it covers only ~12 trits per cycle per SM -- far below what streaming the
// packed weights at HBM speed needs (~70).  The legacy m16n8k16 MMA, measured
// at 0.9 instructions per ns per SM on B200, covers ten times more.
//
// Per CTA (one producer warp + W consumer warps, W = kG3Warps):
//  * the CTA owns W row tiles of 15 weight rows; a thread-block cluster of S
//    CTAs splits K, and the S partial sums are reduced through distributed
//    shared memory in a fixed order (the pages' shared-memory tree reduction of
//    per-warp partials, Figure 11 caption text on appendix G.4 of "Pith review
//    of Spectra 1.1", lifted to the CTAs of a cluster);
//  * the producer streams, per 64-byte-per-row K-group, one TMA box of the
//    CTA's 120 rows x 64 bytes into a ring deep enough for every K-group the
//    CTA owns, so all weight loads are in flight from the start;
//  * the consumer warps meanwhile stage the CTA's activation slice in shared
//    memory (zero past K), in an interleaved layout that makes every consumer
//    load bank-conflict free; consumers then never wait on global memory;
//  * a consumer warp decodes its 15 rows plus a sixteenth row of all-1 digits
//    (the "ones row" that accumulates sum_k x) into subnormal fp16 lanes and
//    multiplies them on mma.sync with fp32 accumulation: 2-bit words by digit
//    class (one LOP3 per register, see g3_word2, with activations staged in
//    the matching pair order), 1.6-bit bytes through the shared-memory tables
//    of tl_gemv.cuh (gemv16_word);
//  * each warp pushes its partial sums into the shared memory of the CTA that
//    owns its tile (warp tile w belongs to rank w mod S); after one cluster
//    barrier every CTA sums what it received, in rank order, and stores Y.
// Bounded mbarrier waits set the device error word on timeout.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include "tl_common.cuh"
#include "tl_sm100.cuh"
#include "tl_gemv.cuh"

namespace tlk {

constexpr int kG3Warps = 8;                      // consumer warps per CTA
constexpr int kG3Threads = 32 * (kG3Warps + 1);  // + one producer warp
constexpr int kG3TileRows = 15;                  // weight rows per consumer warp
constexpr int kG3CtaRows = kG3Warps * kG3TileRows;  // 120
constexpr int kG3Groups = 8;                     // most K-groups per CTA (= ring depth)
constexpr int kG3StageBytes = kG3CtaRows * kGemvGroupBytes;  // one TMA box: 120 rows x 64 B
constexpr int kG3MaxCluster = 8;

// Activation staging: per token row, per K-group, the lane chunks' 16-byte
// units interleaved so that unit u of lane chunk c sits at (u * 4 + c) * 16.
// The row stride is a multiple of 128 plus 64 bytes, so tokens g and g + 1
// of one load phase fall in different halves of the banks.
template <int FMT>
struct G3X {
    static constexpr int units = FMT == 2 ? 8 : 10;        // 16-byte units per lane chunk
    static constexpr int group_bytes = 4 * units * 16;     // 512 / 640
};

constexpr int kG3PartBytes = kG3Warps * 16 * 8 * 4;  // 4 KB of pushed partial sums

// Shared-memory layout of one launch, sized for its K-groups per CTA (ngmax)
// and tokens (M), so that small calls leave room for the next call's CTAs.
struct G3Layout {
    uint32_t x_off, xrow_bytes, part_off, bar_off, total;
    __host__ __device__ G3Layout(int group_bytes, int ngmax, int M) {
        const uint32_t ring = (uint32_t)ngmax * kG3StageBytes;  // ring at offset 0
        xrow_bytes = (uint32_t)ngmax * group_bytes + 64;
        x_off = ring;
        part_off = x_off + (((uint32_t)M * xrow_bytes + 127u) & ~127u);
        bar_off = part_off + kG3PartBytes;
        total = bar_off + 8u * (uint32_t)(ngmax + 1) + 128u;  // + slack for 128-byte alignment
    }
};

// Load activations x[m][k .. k + 8) (zero at positions >= K) as a uint4.
__device__ __forceinline__ uint4 g3_load8(const uint16_t *xr, int k, int K) {
    if (k + 8 <= K) return ld_shared_ro(xr + k);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (k < K) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t lo = k + 2 * q < K ? xr[k + 2 * q] : 0u;
            const uint32_t hi = k + 2 * q + 1 < K ? xr[k + 2 * q + 1] : 0u;
            w[q] = lo | (hi << 16);
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Stage the activations x[m][k_base + i] (i < groups * trits per group) of
// tokens m < M into shared memory, zero at k >= K.  2-bit: every 16-element
// word is stored as its 8 pairs (x_i, x_{8+i}), i = 0..7 (the B operand of
// the class-masked decode, see g3_group); 1.6-bit: natural order.
template <int FMT>
__device__ __forceinline__ void g3_stage_x(uint8_t *xs, const uint16_t *__restrict__ X,
                                           int64_t ldx, int M, int K, int k_base, int groups,
                                           uint32_t xrow_bytes, int tid, int nthreads) {
    constexpr int U = G3X<FMT>::units;
    constexpr int TRITS_LANE = 8 * U;  // 64 / 80 activations per lane chunk
    constexpr int UI = FMT == 2 ? 2 : 1;  // 16-byte units per staging item
    const int per_row = groups * 4 * U / UI;  // items per token row
    const int total = M * per_row;
    constexpr int B = FMT == 2 ? 4 : 8;  // items loaded together per thread
    for (int base = tid; base < total; base += B * nthreads) {
        uint4 v[B][UI];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int it = base + b * nthreads;
            if (it < total) {
                const int m = it / per_row, r = (it % per_row) * UI;
                const int grp = r / (4 * U), rr = r % (4 * U);
                const int c = rr / U, u = rr % U;
                const int k = k_base + grp * 4 * TRITS_LANE + c * TRITS_LANE + u * 8;
                const uint16_t *xr = X + (int64_t)m * ldx;
#pragma unroll
                for (int h = 0; h < UI; ++h) v[b][h] = g3_load8(xr, k + 8 * h, K);
            }
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int it = base + b * nthreads;
            if (it < total) {
                const int m = it / per_row, r = (it % per_row) * UI;
                const int grp = r / (4 * U), rr = r % (4 * U);
                const int c = rr / U, u = rr % U;
                uint8_t *dst = xs + m * xrow_bytes + grp * G3X<FMT>::group_bytes;
                if constexpr (FMT == 2) {
                    const uint32_t *lo = reinterpret_cast<const uint32_t *>(&v[b][0]);
                    const uint32_t *hi = reinterpret_cast<const uint32_t *>(&v[b][1]);
                    uint32_t p[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)  // (x_i, x_{8+i})
                        p[i] = prmt(lo[i >> 1], hi[i >> 1], (i & 1) ? 0x7632u : 0x5410u);
                    *reinterpret_cast<uint4 *>(dst + (u * 4 + c) * 16) =
                        make_uint4(p[0], p[1], p[2], p[3]);
                    *reinterpret_cast<uint4 *>(dst + ((u + 1) * 4 + c) * 16) =
                        make_uint4(p[4], p[5], p[6], p[7]);
                } else {
                    *reinterpret_cast<uint4 *>(dst + (u * 4 + c) * 16) = v[b][0];
                }
            }
        }
    }
}

// One K-group of one consumer lane: words wa (row g) and wb (row g + 8 or the
// ones row) against the lane's activations, read from the staged layout.
// One 2-bit word pair (rows g and g+8) by digit class: digit i of a word sits
// at bits 2i; masking bit pair c of each byte of W (and of W >> 8) leaves
// digits (c, 8+c) and (c+4, 12+c) as subnormal fp16 halves d * 2^(2c-24).
// One MMA per class, with the staged activation pairs p_c and p_{c+4}
// (p_i = (x_i, x_{8+i})) as B; acc[c] collects class c.
__device__ __forceinline__ void g3_word2(uint32_t W, uint32_t V, const uint32_t *p,
                                         float (&acc)[4][4]) {
    const uint32_t hW = W >> 8, hV = V >> 8;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t m = 0x00030003u << (2 * c);
        mma_16816(acc[c], W & m, V & m, hW & m, hV & m, p[c], p[4 + c]);
    }
}

// One K-group of one consumer lane: words wa (row g) and wb (row g + 8 or the
// ones row) against the lane's activations, read from the staged layout.
template <int FMT>
__device__ __forceinline__ void g3_group(const uint4 &wa, const uint4 &wb, const uint8_t *xg,
                                         int c, const uint32_t *lut_even,
                                         const uint32_t *lut_odd, float (&acc)[4][4],
                                         float (&acc4)[4]) {
    if constexpr (FMT == 2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 xv[2];
            xv[0] = *reinterpret_cast<const uint4 *>(xg + ((2 * j) * 4 + c) * 16);
            xv[1] = *reinterpret_cast<const uint4 *>(xg + ((2 * j + 1) * 4 + c) * 16);
            g3_word2(u4get(wa, j), u4get(wb, j), reinterpret_cast<const uint32_t *>(xv), acc);
        }
    } else {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            uint4 xv[5];
#pragma unroll
            for (int i = 0; i < 5; ++i)
                xv[i] = *reinterpret_cast<const uint4 *>(xg + ((5 * jj + i) * 4 + c) * 16);
            const uint32_t *xp = reinterpret_cast<const uint32_t *>(xv);
            // 1.6-bit classes: acc[0] / acc[1] digit class 0, acc[2] / acc[3] class 2
            gemv16_word(u4get(wa, 2 * jj), u4get(wb, 2 * jj), xp, lut_even, lut_odd, acc[0],
                        acc[2], acc4);
            gemv16_word(u4get(wa, 2 * jj + 1), u4get(wb, 2 * jj + 1), xp + 10, lut_even,
                        lut_odd, acc[1], acc[3], acc4);
        }
    }
}

template <int FMT>
__global__ void __launch_bounds__(kG3Threads, 2)
gemv3_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t *__restrict__ X,
             int64_t ldx, float alpha, uint16_t *__restrict__ Y, int64_t ldy, int M, int N, int K,
             int groups_total) {
    constexpr int TPB = FMT == 2 ? 4 : 5;
    constexpr int TRITS_GROUP = kGemvGroupBytes * TPB;  // 256 / 320
    constexpr uint32_t ONES = FMT == 2 ? 0x55555555u : 0x79797979u;  // every digit 1
    extern __shared__ __align__(1024) uint8_t g3_smem_raw[];
    __shared__ uint32_t lut_even[FMT == 2 ? 1 : 256];
    __shared__ uint32_t lut_odd[FMT == 2 ? 1 : 256];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t S = cluster_nctarank();
    const uint32_t rank = cluster_ctarank();
    const int tile = blockIdx.x / (int)S;
    const int n0 = tile * kG3CtaRows;
    const int g_b = (int)((int64_t)groups_total * rank / S);
    const int g_e = (int)((int64_t)groups_total * (rank + 1) / S);
    const int ng = g_e - g_b;  // K-groups of this CTA
    const int ngmax = (groups_total + (int)S - 1) / (int)S;
    const G3Layout lay(G3X<FMT>::group_bytes, ngmax, M);
    // TMA destinations need 128-byte alignment
    uint8_t *smem = g3_smem_raw + ((128u - (smem_u32(g3_smem_raw) & 127u)) & 127u);
    uint8_t *ring = smem;
    uint8_t *xs = smem + lay.x_off;
    float *part = reinterpret_cast<float *>(smem + lay.part_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.bar_off);  // [ngmax]
    uint64_t *redbar = full + ngmax;  // pushed partial sums have landed (S > 1)

    if (threadIdx.x == 0) {
        for (int i = 0; i < ngmax; ++i) mbar_init(&full[i], 1);
        mbar_init(redbar, 1);
        if (S > 1) mbar_arrive_expect_tx(redbar, kG3PartBytes);
        fence_mbar_init();
        tma_prefetch_desc(&tmap_w);
    }
    if constexpr (FMT != 2) build_lut16(lut_even, lut_odd);
    __syncthreads();

    // every weight load of this CTA is issued now (the ring holds all groups)
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < ng; ++i) {
            mbar_arrive_expect_tx(&full[i], kG3StageBytes);
            tma_load_2d(ring + i * kG3StageBytes, &tmap_w, &full[i], (g_b + i) * kGemvGroupBytes,
                        n0);
        }
    }
    // peers may push partial sums to this CTA only after its barrier exists
    if (S > 1) cluster_sync();
    // activations may be produced by the preceding kernel on the stream
    pdl_launch_dependents();
    pdl_wait();
    if (warp > 0)
        g3_stage_x<FMT>(xs, X, ldx, M, K, g_b * TRITS_GROUP, ng, lay.xrow_bytes, threadIdx.x - 32,
                        32 * kG3Warps);
    __syncthreads();

    if (warp > 0) {
        const int cw = warp - 1;
        const int g = lane >> 2, c = lane & 3;
        const bool onesB = (g == 7);
        const int rowA = cw * kG3TileRows + g, rowB = rowA + 8;  // rows within the box
        const uint8_t *xrow = xs + (g < M ? g : 0) * lay.xrow_bytes;
        float acc[4][4], acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
        for (int i = 0; i < ng; ++i) {
            if (!mbar_wait(&full[i], 0)) break;
            const uint8_t *box = ring + i * kG3StageBytes;
            const uint4 wa = *reinterpret_cast<const uint4 *>(box + rowA * kGemvGroupBytes + 16 * c);
            uint4 wb = make_uint4(ONES, ONES, ONES, ONES);
            if (!onesB) wb = *reinterpret_cast<const uint4 *>(box + rowB * kGemvGroupBytes + 16 * c);
            g3_group<FMT>(wa, wb, xrow + i * G3X<FMT>::group_bytes, c, lut_even, lut_odd, acc,
                          acc4);
        }
        // combine classes with exact power-of-two scales: sum_k d * x
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
        // the owner of warp tile cw is rank cw mod S; it keeps the S partials
        // of each tile it owns at part[(source rank * tiles per rank + cw / S)]
        const uint32_t owner = (uint32_t)cw % S;
        const uint32_t slot = rank * (kG3Warps / S) + (uint32_t)cw / S;
        const uint32_t o0 = (uint32_t)(g * 8 + 2 * c), o1 = (uint32_t)((g + 8) * 8 + 2 * c);
        if (S > 1) {
            const uint32_t base = smem_u32(part) + slot * 512u;
            st_async_v2_f32(base + o0 * 4u, owner, smem_u32(redbar), sv[0], sv[1]);
            st_async_v2_f32(base + o1 * 4u, owner, smem_u32(redbar), sv[2], sv[3]);
        } else {
            float *pw = part + slot * 128u;
            pw[o0] = sv[0];
            pw[o0 + 1] = sv[1];
            pw[o1] = sv[2];
            pw[o1 + 1] = sv[3];
        }
    }
    if (S > 1)
        mbar_wait_cluster(redbar, 0);  // all S x (tiles owned) partials have arrived
    else
        __syncthreads();
    {
        // this CTA owns warp tiles w = lt * S + rank; sum the S partials in rank order
        const int per_rank = kG3Warps / (int)S;
        const int items = per_rank * kG3TileRows * M;
        for (int it = threadIdx.x; it < items; it += blockDim.x) {
            const int lt = it / (kG3TileRows * M), rem = it % (kG3TileRows * M);
            const int r = rem / M, m = rem % M;
            const int cw = lt * (int)S + (int)rank;
            const int n = n0 + cw * kG3TileRows + r;
            float acc = 0.f, sx = 0.f;
            for (int q = 0; q < (int)S; ++q) {
                const float *pq = part + (q * per_rank + lt) * 128;
                acc += pq[r * 8 + m];
                sx += pq[15 * 8 + m];
            }
            if (n < N) Y[(int64_t)m * ldy + n] = f32_to_f16_bits(alpha * (acc - sx));
        }
    }
    // no CTA leaves while a peer may still push into its shared memory (a peer
    // whose own wait timed out above still gets here: every wait is bounded)
    if (S > 1) cluster_sync();
}

// ---- host side ---------------------------------------------------------------
template <int FMT>
inline int g3_groups(int K) {
    const int64_t rowbytes = FMT == 2 ? ((int64_t)K + 3) / 4 : ((int64_t)K + 4) / 5;
    return (int)((rowbytes + kGemvGroupBytes - 1) / kGemvGroupBytes);
}

// K fits when a cluster of at most kG3MaxCluster CTAs holds every K-group.
template <int FMT>
inline bool gemv3_supported(int K) {
    return (g3_groups<FMT>(K) + kG3MaxCluster - 1) / kG3MaxCluster <= kG3Groups;
}

// Co-resident CTAs of gemv3_kernel<FMT> for a cluster size and a dynamic
// shared-memory size (cudaOccupancyMaxActiveClusters x cluster size), cached
// per device.  Returns -1 on a CUDA error.
template <int FMT>
inline int g3_resident(int dev, int S, uint32_t smem) {
    struct Entry { int dev, S; uint32_t smem; int ctas; };
    static std::mutex mu;
    static Entry cache[256];
    static int used = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i)
            if (cache[i].dev == dev && cache[i].S == S && cache[i].smem == smem) return cache[i].ctas;
    }
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(1024);
    q.blockDim = dim3(kG3Threads);
    q.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)S;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    q.attrs = at;
    q.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemv3_kernel<FMT>, &q) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (used < 256) cache[used++] = Entry{dev, S, smem, clusters * S};
    return clusters * S;
}

// Smallest power-of-two cluster that fits K, then doubled while each CTA
// keeps >= 1 K-group and the grid stays within both one wave of co-resident
// CTAs and two CTAs per SM -- the rest of each SM is left to the next call on
// the stream, which (under programmatic dependent launch) streams its weights
// while this one drains.
template <int FMT>
inline int gemv3_pick_cluster(int dev, int N, int K, int M, int num_sms, int *resident_out) {
    const int groups = g3_groups<FMT>(K);
    const int tiles = (N + kG3CtaRows - 1) / kG3CtaRows;
    int S = 1;
    while (S < kG3MaxCluster && (groups + S - 1) / S > kG3Groups) S *= 2;
    auto fits = [&](int s) {
        const int ngmax = (groups + s - 1) / s;
        const int r = g3_resident<FMT>(dev, s, G3Layout(G3X<FMT>::group_bytes, ngmax, M).total);
        if (r < 0) return -1;
        return (int64_t)tiles * s <= r && (int64_t)tiles * s <= 2 * num_sms ? 1 : 0;
    };
    while (S < kG3MaxCluster && 2 * S <= groups) {
        const int f = fits(2 * S);
        if (f < 0) return -1;
        if (!f) break;
        S *= 2;
    }
    if (resident_out)
        *resident_out =
            g3_resident<FMT>(dev, S, G3Layout(G3X<FMT>::group_bytes, (groups + S - 1) / S, M).total);
    return S;
}

template <int FMT>
inline int launch_gemv3(const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                        int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K, int num_sms,
                        bool pdl, cudaStream_t stream, int *last_cuda_error) {
    auto encode = tensor_map_encoder();
    if (!encode) return 5;
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static cudaError_t err[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        *last_cuda_error = (int)e;
        return 5;
    }
    std::call_once(once[dev], [dev] {
        const uint32_t most = G3Layout(G3X<FMT>::group_bytes, kG3Groups, 8).total;
        err[dev] = cudaFuncSetAttribute(gemv3_kernel<FMT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
    });
    if (err[dev] != cudaSuccess) {
        *last_cuda_error = (int)err[dev];
        return 5;
    }
    int resident = 0;
    const int S = gemv3_pick_cluster<FMT>(dev, N, K, M, num_sms, &resident);
    if (S < 0 || resident < 1) {
        *last_cuda_error = (int)cudaGetLastError();
        return 5;
    }
    const int groups = g3_groups<FMT>(K);
    const int tiles = (N + kG3CtaRows - 1) / kG3CtaRows;
    const G3Layout lay(G3X<FMT>::group_bytes, (groups + S - 1) / S, M);
    CUtensorMap tw;
    const int64_t rowbytes = FMT == 2 ? ((int64_t)K + 3) / 4 : ((int64_t)K + 4) / 5;
    cuuint64_t dims[2] = {(cuuint64_t)rowbytes, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)ldp};
    cuuint32_t box[2] = {kGemvGroupBytes, kG3CtaRows};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(dT), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return 5;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * S), 1, 1);
    cfg.blockDim = dim3(kG3Threads, 1, 1);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, gemv3_kernel<FMT>, tw, dX, ldx, alpha, dY, ldy, M, N, K, groups);
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

}  // namespace tlk

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
//    multiplies them on mma.sync with fp32 accumulation, exactly as in
//    tl_gemv.cuh (gemv2_word / gemv16_word);
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
// Row stride = groups * group bytes + 64, i.e. 64 mod 128, so tokens g and
// g + 1 of one load phase fall in different halves of the banks.
template <int FMT>
struct G3X {
    static constexpr int units = FMT == 2 ? 8 : 10;        // 16-byte units per lane chunk
    static constexpr int group_bytes = 4 * units * 16;     // 512 / 640
    static constexpr int row_bytes = kG3Groups * group_bytes + 64;
    static constexpr int bytes = 8 * row_bytes;            // M <= 8 tokens
};

template <int FMT>
struct G3Smem {
    static constexpr uint32_t ring_off = 0;
    static constexpr uint32_t ring_bytes = kG3Groups * kG3StageBytes;        // 64 KB
    static constexpr uint32_t x_off = ring_off + ring_bytes;
    static constexpr uint32_t x_bytes = G3X<FMT>::bytes;                     // 32.5 / 40.5 KB
    static constexpr uint32_t part_off = x_off + x_bytes;
    // partial sums pushed by the cluster: [source rank][owned warp tile][16][8]
    static constexpr uint32_t part_bytes = kG3Warps * 16 * 8 * 4;           // 4 KB
    static constexpr uint32_t bar_off = part_off + part_bytes;
    static constexpr uint32_t total = bar_off + kG3Groups * 8 + 128;        // + alignment slack
};

// Stage the activations x[m][k_base + i] (i < groups * trits per group) of
// tokens m < M into shared memory, zero at k >= K.
template <int FMT>
__device__ __forceinline__ void g3_stage_x(uint8_t *xs, const uint16_t *__restrict__ X,
                                           int64_t ldx, int M, int K, int k_base, int groups,
                                           int tid, int nthreads) {
    constexpr int U = G3X<FMT>::units;
    constexpr int TRITS_LANE = 8 * U;  // 64 / 80 activations per lane chunk
    const int per_row = groups * 4 * U;  // 16-byte units per token row
    const int total = M * per_row;
    constexpr int B = 8;  // units loaded together per thread
    for (int base = tid; base < total; base += B * nthreads) {
        uint4 v[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int it = base + b * nthreads;
            v[b] = make_uint4(0, 0, 0, 0);
            if (it < total) {
                const int m = it / per_row, r = it % per_row;
                const int grp = r / (4 * U), rr = r % (4 * U);
                const int c = rr / U, u = rr % U;
                const int k = k_base + grp * 4 * TRITS_LANE + c * TRITS_LANE + u * 8;
                const uint16_t *xr = X + (int64_t)m * ldx;
                if (k + 8 <= K) {
                    v[b] = ld_shared_ro(xr + k);
                } else if (k < K) {
                    uint32_t w[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t lo = k + 2 * q < K ? xr[k + 2 * q] : 0u;
                        const uint32_t hi = k + 2 * q + 1 < K ? xr[k + 2 * q + 1] : 0u;
                        w[q] = lo | (hi << 16);
                    }
                    v[b] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int it = base + b * nthreads;
            if (it < total) {
                const int m = it / per_row, r = it % per_row;
                const int grp = r / (4 * U), rr = r % (4 * U);
                const int c = rr / U, u = rr % U;
                *reinterpret_cast<uint4 *>(xs + m * G3X<FMT>::row_bytes +
                                           grp * G3X<FMT>::group_bytes + (u * 4 + c) * 16) = v[b];
            }
        }
    }
}


// One K-group of one consumer lane: words wa (row g) and wb (row g + 8 or the
// ones row) against the lane's activations, read from the staged layout.
template <int FMT>
__device__ __forceinline__ void g3_group(const uint4 &wa, const uint4 &wb, const uint8_t *xg,
                                         int c, const uint32_t *lut_even,
                                         const uint32_t *lut_odd, float (&acc0a)[4],
                                         float (&acc0b)[4], float (&acc2a)[4],
                                         float (&acc2b)[4], float (&acc4)[4]) {
    if constexpr (FMT == 2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 xv[2];
            xv[0] = *reinterpret_cast<const uint4 *>(xg + ((2 * j) * 4 + c) * 16);
            xv[1] = *reinterpret_cast<const uint4 *>(xg + ((2 * j + 1) * 4 + c) * 16);
            gemv2_word(u4get(wa, j), u4get(wb, j), reinterpret_cast<const uint32_t *>(xv), acc0a,
                       acc0b, acc2a, acc2b);
        }
    } else {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            uint4 xv[5];
#pragma unroll
            for (int i = 0; i < 5; ++i)
                xv[i] = *reinterpret_cast<const uint4 *>(xg + ((5 * jj + i) * 4 + c) * 16);
            const uint32_t *xp = reinterpret_cast<const uint32_t *>(xv);
            gemv16_word(u4get(wa, 2 * jj), u4get(wb, 2 * jj), xp, lut_even, lut_odd, acc0a,
                        acc2a, acc4);
            gemv16_word(u4get(wa, 2 * jj + 1), u4get(wb, 2 * jj + 1), xp + 10, lut_even,
                        lut_odd, acc0b, acc2b, acc4);
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
    // TMA destinations need 128-byte alignment
    uint8_t *smem = g3_smem_raw + ((128u - (smem_u32(g3_smem_raw) & 127u)) & 127u);
    uint8_t *ring = smem + G3Smem<FMT>::ring_off;
    uint8_t *xs = smem + G3Smem<FMT>::x_off;
    float *part = reinterpret_cast<float *>(smem + G3Smem<FMT>::part_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + G3Smem<FMT>::bar_off);
    __shared__ uint32_t lut_even[FMT == 2 ? 1 : 256];
    __shared__ uint32_t lut_odd[FMT == 2 ? 1 : 256];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t S = cluster_nctarank();
    const uint32_t rank = cluster_ctarank();
    const int tile = blockIdx.x / (int)S;
    const int n0 = tile * kG3CtaRows;
    const int g_b = (int)((int64_t)groups_total * rank / S);
    const int g_e = (int)((int64_t)groups_total * (rank + 1) / S);
    const int ng = g_e - g_b;  // K-groups of this CTA (<= kG3Groups)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kG3Groups; ++s) mbar_init(&full[s], 1);
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
    // activations may be produced by the preceding kernel on the stream
    pdl_launch_dependents();
    pdl_wait();
    if (warp > 0) g3_stage_x<FMT>(xs, X, ldx, M, K, g_b * TRITS_GROUP, ng, threadIdx.x - 32,
                                  32 * kG3Warps);
    __syncthreads();

    if (warp > 0) {
        const int cw = warp - 1;
        const int g = lane >> 2, c = lane & 3;
        const bool onesB = (g == 7);
        const int rowA = cw * kG3TileRows + g, rowB = rowA + 8;  // rows within the box
        const uint8_t *xrow = xs + (g < M ? g : 0) * G3X<FMT>::row_bytes;
        float acc0a[4] = {0.f, 0.f, 0.f, 0.f}, acc0b[4] = {0.f, 0.f, 0.f, 0.f};
        float acc2a[4] = {0.f, 0.f, 0.f, 0.f}, acc2b[4] = {0.f, 0.f, 0.f, 0.f};
        float acc4[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i = 0; i < ng; ++i) {
            if (!mbar_wait(&full[i], 0)) break;
            const uint8_t *box = ring + i * kG3StageBytes;
            const uint4 wa = *reinterpret_cast<const uint4 *>(box + rowA * kGemvGroupBytes + 16 * c);
            uint4 wb = make_uint4(ONES, ONES, ONES, ONES);
            if (!onesB) wb = *reinterpret_cast<const uint4 *>(box + rowB * kGemvGroupBytes + 16 * c);
            g3_group<FMT>(wa, wb, xrow + i * G3X<FMT>::group_bytes, c, lut_even, lut_odd, acc0a,
                          acc0b, acc2a, acc2b, acc4);
        }
        float sv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            sv[q] = (acc0a[q] + acc0b[q]) * 16777216.0f + (acc2a[q] + acc2b[q]) * 1048576.0f;
            if constexpr (FMT != 2) sv[q] += acc4[q] * 65536.0f;
        }
        // push to the owner of this warp tile: part[rank][cw / S][16][8] there
        const uint32_t owner = (uint32_t)cw % S;
        const uint32_t per_rank = kG3Warps / S;
        const uint32_t base = smem_u32(part) +
            ((rank * per_rank + (uint32_t)cw / S) * 128u) * 4u;
        st_dsmem_f32(base + (uint32_t)(g * 8 + 2 * c) * 4u, owner, sv[0]);
        st_dsmem_f32(base + (uint32_t)(g * 8 + 2 * c + 1) * 4u, owner, sv[1]);
        st_dsmem_f32(base + (uint32_t)((g + 8) * 8 + 2 * c) * 4u, owner, sv[2]);
        st_dsmem_f32(base + (uint32_t)((g + 8) * 8 + 2 * c + 1) * 4u, owner, sv[3]);
    }
    cluster_sync();  // every pushed partial sum has landed
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
}

// ---- host side ---------------------------------------------------------------
struct G3Shape {
    int cluster;  // CTAs splitting K
    int tiles;    // row tiles of 120 rows
    int groups;   // 64-byte K-groups per packed row
};

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

// Smallest power-of-two cluster that fits K, then doubled while the grid
// stays within one wave of co-resident clusters and every CTA keeps >= 1
// group.  resident[i] = CTAs that can be resident with clusters of 2^i.
template <int FMT>
inline G3Shape gemv3_shape(int N, int K, const int *resident) {
    const int groups = g3_groups<FMT>(K);
    const int tiles = (N + kG3CtaRows - 1) / kG3CtaRows;
    int S = 1, log2s = 0;
    while (S < kG3MaxCluster && (groups + S - 1) / S > kG3Groups) S *= 2, ++log2s;
    while (S < kG3MaxCluster && 2 * S <= groups &&
           (int64_t)tiles * S * 2 <= resident[log2s + 1])
        S *= 2, ++log2s;
    return G3Shape{S, tiles, groups};
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
    static int resident[kMaxDev][4];  // co-resident CTAs for clusters of 1, 2, 4, 8
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        *last_cuda_error = (int)e;
        return 5;
    }
    std::call_once(once[dev], [dev] {
        err[dev] = cudaFuncSetAttribute(gemv3_kernel<FMT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)G3Smem<FMT>::total);
        for (int i = 0; i < 4 && err[dev] == cudaSuccess; ++i) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(1024);
            q.blockDim = dim3(kG3Threads);
            q.dynamicSmemBytes = G3Smem<FMT>::total;
            cudaLaunchAttribute a[1];
            a[0].id = cudaLaunchAttributeClusterDimension;
            a[0].val.clusterDim.x = 1u << i;
            a[0].val.clusterDim.y = 1;
            a[0].val.clusterDim.z = 1;
            q.attrs = a;
            q.numAttrs = 1;
            int clusters = 0;
            err[dev] = cudaOccupancyMaxActiveClusters(&clusters, gemv3_kernel<FMT>, &q);
            resident[dev][i] = clusters << i;
        }
    });
    (void)num_sms;
    if (err[dev] != cudaSuccess || resident[dev][0] < 1) {
        *last_cuda_error = (int)err[dev];
        return 5;
    }
    const G3Shape sh = gemv3_shape<FMT>(N, K, resident[dev]);
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
    cfg.gridDim = dim3((unsigned)(sh.tiles * sh.cluster), 1, 1);
    cfg.blockDim = dim3(kG3Threads, 1, 1);
    cfg.dynamicSmemBytes = G3Smem<FMT>::total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)sh.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, gemv3_kernel<FMT>, tw, dX, ldx, alpha, dY, ldy, M, N, K,
                           sh.groups);
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

}  // namespace tlk

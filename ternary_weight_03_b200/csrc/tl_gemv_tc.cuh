// tl_gemv_tc.cuh -- decode-shaped ternary layer (M = 1..8) on the tcgen05
// tensor cores, 2-bit packing:  Y[m][n] = fp16_rn(alpha * sum_k T[n][k] X[m][k]).
//
// Work decomposition: a row tile is 127 weight rows (TMEM lanes 0..126) plus
// one "ones" lane (127) whose digits are all 1; a thread-block cluster of S
// CTAs splits the tile's K range, and the S partial results are summed through
// distributed shared memory in a fixed order (the pages' shared-memory tree
// reduction of per-warp partials -- Figure 11 caption text on appendix G.4 of
// "Pith review of Spectra 1.1" -- lifted to the CTAs of a cluster).
//
// Per CTA:
//  * warp 0 streams packed stages (127+1 rows x 64 bytes = 256 trits per row)
//    with TMA (64-byte swizzle, no multicast) into a 4-deep ring;
//  * all warps first copy the CTA's slice of the activations into shared
//    memory, permuted so that it is the MMA B operand for the digit classes
//    below (tokens m >= M are left undefined: their outputs are never stored);
//  * eight decode warps (thread = weight row = TMEM lane) turn each 32-bit word
//    of 16 digits into 8 fp16x2 registers with one LOP3 each (plus one shift
//    per word): digit d = t + 1 masked in place reads as the subnormal
//    d * 2^(2c-24), c = 0..3 the digit's bit pair within its byte ("class");
//    the registers go to a 3-slot ring in tensor memory with tcgen05.st as the
//    MMA A operand;
//  * one thread issues tcgen05.mma.kind::f16 (M = 128 rows, N = 16 tokens,
//    K = 16), one fp32 accumulator per class, and recycles the A slots with
//    tcgen05.commit;
//  * epilogue: classes combined with exact power-of-two scales, partial sums
//    to shared memory, cluster barrier, each CTA reduces a slice of rows over
//    the cluster, subtracts the ones lane (sum_k x, the t = d - 1 offset),
//    scales by alpha and stores fp16.
// Bounded mbarrier waits set the device error word on timeout.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include "tl_common.cuh"
#include "tl_sm100.cuh"

namespace tlk {

constexpr int kTcWRows = 127;          // weight rows per tile (lane 127 = ones row)
constexpr int kTcStageRowBytes = 64;   // bytes per row per stage (256 trits)
constexpr int kTcStages = 4;           // TMA ring depth
constexpr int kTcThreads = 320;        // warp 0 TMA, warp 1 MMA, warps 2..9 decode
constexpr int kTcMaxStagesPerCta = 8;  // K range per CTA <= 2048 trits
constexpr int kTcTmemCols = 256;       // 4 class accumulators x 16 + 3 A slots x 64
constexpr int kTcAccCol = 0;           // class c accumulator at columns [16c, 16c + 16)
constexpr int kTcSlotCol = 64;         // A slot i at [64 + 64i, 64 + 64i + 64)
constexpr int kTcSlots = 3;
constexpr int kTcBlockBytes = 4096;    // permuted activations per 128-trit block (8 x 512)
constexpr int kTcMaxCluster = 8;

// class-part ci (0..7) holds digits (ci, 8 + ci) of a word; its bit pair
// within the byte, and so its accumulator class, is ci & 3.
__host__ __device__ constexpr int tc_shift(int ci) { return ci; }
__host__ __device__ constexpr int tc_class(int ci) { return ci & 3; }

struct TcSmem {
    static constexpr uint32_t wstage_bytes = 128u * kTcStageRowBytes;  // 8 KB
    static constexpr uint32_t xperm_bytes = 2u * kTcMaxStagesPerCta * kTcBlockBytes;  // 64 KB
    static constexpr uint32_t partial_bytes = 128u * 16u * 4u;  // 8 KB
    static constexpr uint32_t wstage_off = 0;
    static constexpr uint32_t xperm_off = wstage_off + kTcStages * wstage_bytes;
    static constexpr uint32_t partial_off = xperm_off + xperm_bytes;
    static constexpr uint32_t bar_off = partial_off + partial_bytes;
    static constexpr uint32_t total = bar_off + 64 * 8 + 1024;  // + barriers + alignment slack
};

// Shared-memory descriptor, K-major, no swizzle: 8-row x 16-byte core
// matrices; LBO = byte distance between the two core matrices along K,
// SBO = byte distance between 8-row groups.
__device__ __forceinline__ uint64_t sdesc_kinter(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;  // sm_100 descriptor version
    return d;                // layout type 0: no swizzle
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}
__device__ __forceinline__ void tmem_st_32x32b_x64(uint32_t taddr, const uint32_t (&v)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, "
        "%45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, "
        "%62, %63, %64};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31]), "r"(v[32]), "r"(v[33]), "r"(v[34]), "r"(v[35]),
        "r"(v[36]), "r"(v[37]), "r"(v[38]), "r"(v[39]), "r"(v[40]), "r"(v[41]), "r"(v[42]),
        "r"(v[43]), "r"(v[44]), "r"(v[45]), "r"(v[46]), "r"(v[47]), "r"(v[48]), "r"(v[49]),
        "r"(v[50]), "r"(v[51]), "r"(v[52]), "r"(v[53]), "r"(v[54]), "r"(v[55]), "r"(v[56]),
        "r"(v[57]), "r"(v[58]), "r"(v[59]), "r"(v[60]), "r"(v[61]), "r"(v[62]), "r"(v[63])
        : "memory");
}

// Class-masked registers of one 32-bit word (16 digits, digit i at bits 2i):
// register ci holds digits (ci, 8 + ci) of the word in its low / high half,
// at bit pair ci & 3 of the half's low byte (digits 4..7 and 12..15 come from
// the word shifted right by 8).
__device__ __forceinline__ void tc_decode_word(uint32_t w, uint32_t *r8 /* stride 8 */) {
    const uint32_t h = w >> 8;
    r8[0 * 8] = w & 0x00030003u;  // digits 0, 8   class 0
    r8[1 * 8] = w & 0x000C000Cu;  // digits 1, 9   class 1
    r8[2 * 8] = w & 0x00300030u;  // digits 2, 10  class 2
    r8[3 * 8] = w & 0x00C000C0u;  // digits 3, 11  class 3
    r8[4 * 8] = h & 0x00030003u;  // digits 4, 12  class 0
    r8[5 * 8] = h & 0x000C000Cu;  // digits 5, 13  class 1
    r8[6 * 8] = h & 0x00300030u;  // digits 6, 14  class 2
    r8[7 * 8] = h & 0x00C000C0u;  // digits 7, 15  class 3
}

__global__ void __launch_bounds__(kTcThreads, 2)
gemv2_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t *__restrict__ X,
                int64_t ldx, float alpha, uint16_t *__restrict__ Y, int64_t ldy, int M, int N,
                int K, int stages_total) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *wst = smem + TcSmem::wstage_off;
    uint8_t *xperm = smem + TcSmem::xperm_off;
    float *partial = reinterpret_cast<float *>(smem + TcSmem::partial_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TcSmem::bar_off);
    uint64_t *wfull = bars;                   // [kTcStages] TMA -> decoders
    uint64_t *wempty = wfull + kTcStages;     // [kTcStages] decoders -> TMA
    uint64_t *afull = wempty + kTcStages;     // [kTcSlots] decoders -> MMA
    uint64_t *aempty = afull + kTcSlots;      // [kTcSlots] MMA commit -> decoders
    uint64_t *done = aempty + kTcSlots;       // last MMA committed -> epilogue
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t S = cluster_nctarank();
    const uint32_t rank = cluster_ctarank();
    const int tile = blockIdx.x / (int)S;
    const int n0 = tile * kTcWRows;
    // this CTA's stages of the row: [st_b, st_e)
    const int st_b = (int)((int64_t)stages_total * rank / S);
    const int st_e = (int)((int64_t)stages_total * (rank + 1) / S);
    const int nst = st_e - st_b;
    const int nblk = 2 * nst;
    const int k_base = st_b * 4 * kTcStageRowBytes;  // first trit of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], 256);
        }
        for (int i = 0; i < kTcSlots; ++i) {
            mbar_init(&afull[i], 128);
            mbar_init(&aempty[i], 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmap_w);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // the producer starts streaming weights before the activation permute
    if (warp == 0 && lane == 0) {
        for (int st = 0; st < nst && st < kTcStages; ++st) {
            mbar_arrive_expect_tx(&wfull[st], TcSmem::wstage_bytes);
            tma_load_2d(wst + st * TcSmem::wstage_bytes, &tmap_w, &wfull[st],
                        (st_b + st) * kTcStageRowBytes, n0);
        }
    }

    // ---- permuted activations: B operand of every (block, class-part) MMA ----
    // item = (token m < M, local block lb, word j): 16 activations
    // x[m][k_base + 128 lb + 16 j + 0..15]; class-part ci takes the pair
    // (s', 8 + s') into logical k (2j, 2j+1) of its 16 x 16 B tile.
    {
        const int items = M * nblk * 8;
        for (int it = threadIdx.x; it < items; it += blockDim.x) {
            const int j = it & 7;
            const int lb = (it >> 3) % nblk;
            const int m = (it >> 3) / nblk;
            const int k0 = k_base + 128 * lb + 16 * j;
            const uint16_t *xr = X + (int64_t)m * ldx;
            uint32_t v[8];
            if (k0 + 16 <= K) {
                const uint4 a = ld_shared_ro(xr + k0), b = ld_shared_ro(xr + k0 + 8);
                v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
                v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int k = k0 + 2 * q;
                    const uint32_t lo = k < K ? xr[k] : 0u;
                    const uint32_t hi = k + 1 < K ? xr[k + 1] : 0u;
                    v[q] = lo | (hi << 16);
                }
            }
            // logical k = 2j -> core matrix kc = j / 4, element e = 2j % 8
            const uint32_t sub = (uint32_t)((m >> 3) * 256 + (j >> 2) * 128 + (m & 7) * 16 +
                                            ((2 * j) & 7) * 2);
#pragma unroll
            for (int ci = 0; ci < 8; ++ci) {
                const int s = tc_shift(ci);
                // pair (x[s], x[8 + s]): halves s & 1 of words s >> 1 and 4 + (s >> 1)
                const uint32_t pair =
                    prmt(v[s >> 1], v[4 + (s >> 1)], (s & 1) ? 0x7632u : 0x5410u);
                *reinterpret_cast<uint32_t *>(xperm + (lb * 8 + ci) * 512 + sub) = pair;
            }
        }
    }
    // generic-proxy writes of the B operand must be visible to the tensor core
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    if (warp == 0) {
        // ---- TMA producer (continues the ring) ----
        if (lane == 0) {
            for (int st = kTcStages; st < nst; ++st) {
                const int s = st % kTcStages;
                if (!mbar_wait(&wempty[s], ((st / kTcStages) - 1) & 1)) break;
                mbar_arrive_expect_tx(&wfull[s], TcSmem::wstage_bytes);
                tma_load_2d(wst + s * TcSmem::wstage_bytes, &tmap_w, &wfull[s],
                            (st_b + st) * kTcStageRowBytes, n0);
            }
            for (int st = nst - kTcStages > 0 ? nst - kTcStages : 0; st < nst; ++st)
                mbar_wait(&wfull[st % kTcStages], (st / kTcStages) & 1);
        }
    } else if (warp == 1) {
        // ---- MMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(128, 16);
            const uint32_t xbase = smem_u32(xperm);
            for (int lb = 0; lb < nblk; ++lb) {
                const int slot = lb % kTcSlots;
                if (!mbar_wait(&afull[slot], (lb / kTcSlots) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int ci = 0; ci < 8; ++ci) {
                    const uint64_t bdesc =
                        sdesc_kinter(xbase + (uint32_t)(lb * 8 + ci) * 512u, 128u, 256u);
                    const uint32_t acc = tmem + kTcAccCol + 16 * tc_class(ci);
                    const uint32_t a = tmem + kTcSlotCol + 64 * slot + 8 * ci;
                    const bool first = lb == 0 && ci < 4;
                    tc_mma_ts(acc, a, bdesc, idesc, first ? 0u : 1u);
                }
                tc_commit(&aempty[slot]);
            }
            tc_commit(done);
        }
    } else {
        // ---- decode warps 2..9: set h = (warp - 2) / 4 takes blocks lb = 2 st + h ----
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        const uint32_t swz = (uint32_t)((row >> 1) & 3);
        bool ok = true;
        for (int st = 0; st < nst && ok; ++st) {
            const int s = st % kTcStages;
            ok = mbar_wait(&wfull[s], (st / kTcStages) & 1);
            if (!ok) break;
            const uint8_t *rowp = wst + s * TcSmem::wstage_bytes + row * kTcStageRowBytes;
            uint4 c0 = *reinterpret_cast<const uint4 *>(rowp + (((2 * h) ^ swz) << 4));
            uint4 c1 = *reinterpret_cast<const uint4 *>(rowp + (((2 * h + 1) ^ swz) << 4));
            if (row == 127) {  // the ones row: every digit 1
                c0 = make_uint4(0x55555555u, 0x55555555u, 0x55555555u, 0x55555555u);
                c1 = c0;
            }
            const int lb = 2 * st + h;
            const int slot = lb % kTcSlots;
            if (lb >= kTcSlots && !(ok = mbar_wait(&aempty[slot], ((lb / kTcSlots) - 1) & 1)))
                break;
            tc_fence_after();
            uint32_t a[64];
            tc_decode_word(c0.x, a + 0);
            tc_decode_word(c0.y, a + 1);
            tc_decode_word(c0.z, a + 2);
            tc_decode_word(c0.w, a + 3);
            tc_decode_word(c1.x, a + 4);
            tc_decode_word(c1.y, a + 5);
            tc_decode_word(c1.z, a + 6);
            tc_decode_word(c1.w, a + 7);
            // release the weight stage only once its bytes have been consumed; the
            // proxy fence orders these generic reads before the next TMA write
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&wempty[s]);
            tmem_st_32x32b_x64(tmem + lane_addr + kTcSlotCol + 64 * slot, a);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&afull[slot]);
        }
        // ---- epilogue part 1: combine classes, partial sums to shared memory ----
        if (h == 0) {
            if (ok) ok = mbar_wait(done, 0);
            float s16[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) s16[m] = 0.f;
            if (ok && nblk > 0) {
                tc_fence_after();
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + lane_addr + kTcAccCol + 32 * part, v);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int cls = 2 * part + (i >> 4);  // columns 16 c + m
                        const float scale = cls == 0 ? 16777216.f : cls == 1 ? 4194304.f
                                          : cls == 2 ? 1048576.f : 262144.f;
                        s16[i & 15] += __uint_as_float(v[i]) * scale;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) partial[row * 16 + m] = s16[m];
        }
    }

    // ---- teardown of TMEM, then the cluster-wide reduction ----
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        if (lane == 0) mbar_wait(done, 0);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
    cluster_sync();  // every CTA's partial sums are written
    {
        const int rows_per = (128 + (int)S - 1) / (int)S;
        const int r0 = (int)rank * rows_per;
        const int r1 = min(r0 + rows_per, kTcWRows);
        const uint32_t pbase = smem_u32(partial);
        for (int it = threadIdx.x; it < (r1 > r0 ? (r1 - r0) * M : 0); it += blockDim.x) {
            const int row = r0 + it / M, m = it % M;
            const int n = n0 + row;
            float acc = 0.f, sx = 0.f;
            for (uint32_t qr = 0; qr < S; ++qr) {
                acc += ld_dsmem_f32(pbase + (uint32_t)(row * 16 + m) * 4u, qr);
                sx += ld_dsmem_f32(pbase + (uint32_t)(127 * 16 + m) * 4u, qr);
            }
            if (n < N) Y[(int64_t)m * ldy + n] = f32_to_f16_bits(alpha * (acc - sx));
        }
    }
    cluster_sync();  // no CTA leaves while others may still read its partial sums
}

// ---- host side ---------------------------------------------------------------
struct GemvTcShape {
    int cluster;
    int tiles;
    int stages_total;
};

inline GemvTcShape gemv_tc_shape(int N, int K, int num_sms) {
    const int64_t rowbytes = ((int64_t)K + 3) / 4;
    const int ns = (int)((rowbytes + kTcStageRowBytes - 1) / kTcStageRowBytes);
    const int tiles = (N + kTcWRows - 1) / kTcWRows;
    int S = 1;
    while (S < kTcMaxCluster && (ns + S - 1) / S > kTcMaxStagesPerCta) S *= 2;
    // more CTAs while they still fit two per SM and each keeps at least one stage
    while (S < kTcMaxCluster && 2 * S <= ns && (int64_t)tiles * S * 2 <= 2 * num_sms) S *= 2;
    return GemvTcShape{S, tiles, ns};
}

inline bool gemv_tc_supported(int N, int K) {
    const int64_t rowbytes = ((int64_t)K + 3) / 4;
    const int ns = (int)((rowbytes + kTcStageRowBytes - 1) / kTcStageRowBytes);
    (void)N;
    return (ns + kTcMaxCluster - 1) / kTcMaxCluster <= kTcMaxStagesPerCta;
}

inline int launch_gemv_tc(const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                          int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K,
                          int num_sms, cudaStream_t stream, int *last_cuda_error) {
    auto encode = tensor_map_encoder();
    if (!encode) return 5;
    const GemvTcShape sh = gemv_tc_shape(N, K, num_sms);
    CUtensorMap tw;
    const int64_t rowbytes = ((int64_t)K + 3) / 4;
    cuuint64_t dims[2] = {(cuuint64_t)rowbytes, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)ldp};
    cuuint32_t box[2] = {kTcStageRowBytes, 128};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(dT), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return 5;
    constexpr int kMaxDev = 64;
    static std::once_flag attr_once[kMaxDev];
    static cudaError_t attr_err[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        *last_cuda_error = (int)e;
        return 5;
    }
    std::call_once(attr_once[dev], [dev] {
        attr_err[dev] = cudaFuncSetAttribute(gemv2_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)TcSmem::total);
    });
    if (attr_err[dev] != cudaSuccess) {
        *last_cuda_error = (int)attr_err[dev];
        return 5;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sh.tiles * sh.cluster), 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = TcSmem::total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)sh.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gemv2_tc_kernel, tw, dX, ldx, alpha, dY, ldy, M, N, K,
                           sh.stages_total);
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

}  // namespace tlk

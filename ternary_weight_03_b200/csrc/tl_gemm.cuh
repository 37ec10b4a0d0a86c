// tl_gemm.cuh -- batched / prefill ternary linear layer, M >= 16:
//   Y[m][n] = fp16_rn(alpha * sum_k T[n][k] * X[m][k])
// on the sm_100a tensor cores (tcgen05, fp32 accumulators in tensor memory).
//
// The pages' GPU kernel is an FP16 x INT2 tensor-core kernel with
// asynchronous copies and fused dequantisation ("Pith review of Spectra
// 1.1", "What carries the argument").  Here, per CTA and output tile of
// 128 weight rows x BN tokens:
//  * a TMA warp streams, per K-step of 64, the packed tile (128 rows x 16 B)
//    and the activation tile (BN tokens x 64 fp16, 128-byte swizzle) into a
//    shared-memory ring (no multicast);
//  * four decode warps (thread = weight row = TMEM lane) expand the row's 64
//    trits to exact fp16 -1 / 0 / +1 and write them with tcgen05.st straight
//    into tensor memory, where they are the MMA's A operand -- the expanded
//    weights never touch shared memory;
//  * one thread issues tcgen05.mma.kind::f16 (A from TMEM, B = activations
//    from shared memory) into an fp32 accumulator in TMEM and commits to
//    mbarriers that recycle the ring stages;
//  * the decode warps then read the accumulator with tcgen05.ld, scale by
//    alpha and store fp16.
// Every mbarrier wait is bounded; a timeout sets the device error word.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include "tl_common.cuh"
#include "tl_sm100.cuh"

namespace tlk {

constexpr int kGemmRows = 128;        // weight rows per tile (TMEM lanes)
constexpr int kGemmKStep = 64;        // trits per K-step (4 MMAs of K = 16)
constexpr int kGemmStages = 4;        // ring depth (the A stages in TMEM follow it)
constexpr int kGemmThreads = 192;     // warp 0 TMA, warp 1 MMA, warps 2..5 decode/epilogue
// TMEM columns: the accumulator takes BN (at least 32) columns, then the four
// A stages take 32 columns each; the allocation is a power of two.
__host__ __device__ constexpr int gemm_acol_base(int bn) { return bn < 32 ? 32 : bn; }
__host__ __device__ constexpr int gemm_tmem_cols(int bn) {
    return gemm_acol_base(bn) + 32 * 4 <= 256 ? 256 : 512;
}

struct GemmSmem {
    // per-stage byte offsets inside the dynamic shared memory block
    __host__ __device__ static constexpr uint32_t x_stage_bytes(int bn) { return (uint32_t)bn * 128u; }
    static constexpr uint32_t w_stage_bytes = kGemmRows * 16u;
};

// Exact decode of one 32-bit word of 2-bit digits (16 trits, natural order)
// into 8 fp16x2 registers (t_2i, t_2i+1), values -1, 0, +1.
__device__ __forceinline__ void decode2_exact(uint32_t w, uint32_t *out) {
    const uint32_t m = 0x03030303u;
    const uint32_t e0 = w & m, e1 = (w >> 2) & m, e2 = (w >> 4) & m, e3 = (w >> 6) & m;
    // bytes of e0..e3 hold one digit each (MSB 0), so selector nibble 8 gives 0x00
    const __half2 off = __halves2half2(__ushort_as_half(0x6401), __ushort_as_half(0x6401));
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t sel = 0x8080u | (uint32_t)b | ((uint32_t)(4 + b) << 8);
        uint32_t lo = prmt(e0, e1, sel) | 0x64006400u;  // 1024 + d
        uint32_t hi = prmt(e2, e3, sel) | 0x64006400u;
        __half2 hlo = __hsub2(*reinterpret_cast<__half2 *>(&lo), off);  // d - 1 = t
        __half2 hhi = __hsub2(*reinterpret_cast<__half2 *>(&hi), off);
        out[2 * b] = *reinterpret_cast<uint32_t *>(&hlo);
        out[2 * b + 1] = *reinterpret_cast<uint32_t *>(&hhi);
    }
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm2_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
             float alpha, uint16_t *__restrict__ Y, int64_t ldy, int M, int N, int K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled activation stages
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *xs = smem;                                            // kGemmStages x BN x 128 B
    uint8_t *ws = xs + kGemmStages * GemmSmem::x_stage_bytes(BN);  // kGemmStages x 128 x 16 B
    uint64_t *full = reinterpret_cast<uint64_t *>(ws + kGemmStages * GemmSmem::w_stage_bytes);
    uint64_t *afull = full + kGemmStages;   // decoders -> MMA (A stage written)
    uint64_t *empty = afull + kGemmStages;  // MMA commit -> producer / decoders
    uint64_t *done = empty + kGemmStages;   // last MMA committed -> epilogue
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kGemmRows;
    const int m0 = blockIdx.y * BN;
    const int nk = (K + kGemmKStep - 1) / kGemmKStep;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&afull[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmap_w);
        tma_prefetch_desc(&tmap_x);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_slot, gemm_tmem_cols(BN));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    if (warp == 0) {
        // ---- TMA producer ----
        if (lane == 0) {
            const uint32_t bytes = GemmSmem::x_stage_bytes(BN) + GemmSmem::w_stage_bytes;
            for (int k = 0; k < nk; ++k) {
                const int s = k % kGemmStages;
                if (k >= kGemmStages && !mbar_wait(&empty[s], ((k / kGemmStages) - 1) & 1))
                    break;
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(xs + s * GemmSmem::x_stage_bytes(BN), &tmap_x, &full[s],
                            k * kGemmKStep, m0);
                tma_load_2d(ws + s * GemmSmem::w_stage_bytes, &tmap_w, &full[s], k * 16, n0);
            }
            // drain: make sure every issued copy has landed before the CTA may exit
            for (int k = nk - kGemmStages > 0 ? nk - kGemmStages : 0; k < nk; ++k) {
                const int s = k % kGemmStages;
                mbar_wait(&full[s], (k / kGemmStages) & 1);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(kGemmRows, BN);
            for (int k = 0; k < nk; ++k) {
                const int s = k % kGemmStages;
                // the decoders saw this stage's TMA complete before arriving; wait on
                // it here too so the tensor core's reads are ordered after the copy
                if (!mbar_wait(&full[s], (k / kGemmStages) & 1) ||
                    !mbar_wait(&afull[s], (k / kGemmStages) & 1))
                    break;
                tc_fence_after();
                const uint32_t xaddr = smem_u32(xs + s * GemmSmem::x_stage_bytes(BN));
#pragma unroll
                for (int j = 0; j < kGemmKStep / 16; ++j) {
                    const uint64_t bdesc = sdesc_k128(xaddr + 32 * j);
                    const uint32_t a_tmem = tmem + gemm_acol_base(BN) + 32 * s + 8 * j;
                    tc_mma_ts(tmem, a_tmem, bdesc, idesc, (k > 0 || j > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            tc_commit(done);  // also on abort, so teardown can wait for issued MMAs
        }
    } else {
        // ---- decode warps (2..5): thread = weight row = TMEM lane ----
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;      // row within the tile
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        for (int k = 0; k < nk && ok; ++k) {
            const int s = k % kGemmStages;
            ok = mbar_wait(&full[s], (k / kGemmStages) & 1);
            if (ok && k >= kGemmStages) ok = mbar_wait(&empty[s], ((k / kGemmStages) - 1) & 1);
            if (!ok) break;
            const uint4 pw = *reinterpret_cast<const uint4 *>(ws + s * GemmSmem::w_stage_bytes +
                                                               row * 16);
            uint32_t a[32];
            decode2_exact(pw.x, a);
            decode2_exact(pw.y, a + 8);
            decode2_exact(pw.z, a + 16);
            decode2_exact(pw.w, a + 24);
            // the packed bytes are consumed; order these generic reads before the
            // TMA write that will refill this stage once the MMA releases it
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_after();
            tmem_st_32x32b_x32(tmem + lane_addr + gemm_acol_base(BN) + 32 * s, a);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&afull[s]);
        }
        // ---- epilogue: accumulator -> alpha -> fp16 -> Y ----
        if (ok) ok = mbar_wait(done, 0);
        if (ok) {
            tc_fence_after();
            const int n = n0 + row;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + lane_addr + c, v);
                tc_wait_ld();
                if (n < N) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + c + j;
                        if (c + j < BN && m < M)  // BN = 16 reads 16 columns past the tile
                            Y[(int64_t)m * ldy + n] = f32_to_f16_bits(alpha * __uint_as_float(v[j]));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        if (lane == 0) mbar_wait(done, 0);  // no MMA may still write TMEM
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, gemm_tmem_cols(BN));
    }
}

// ---- host side ---------------------------------------------------------------
inline size_t gemm_smem_bytes(int bn) {
    return 1024 + kGemmStages * ((size_t)bn * 128 + kGemmRows * 16) + (3 * kGemmStages + 1) * 8 +
           16;
}

template <int BN>
inline int launch_gemm_bn(const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                          int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K,
                          cudaStream_t stream, int *last_cuda_error) {
    auto encode = tensor_map_encoder();
    if (!encode) return 5;  // TL_ERR_CUDA
    CUtensorMap tw, tx;
    const int64_t rowbytes = ((int64_t)K + 3) / 4;
    {
        cuuint64_t dims[2] = {(cuuint64_t)rowbytes, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)ldp};
        cuuint32_t box[2] = {16, kGemmRows};
        cuuint32_t estr[2] = {1, 1};
        if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(dT), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return 5;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
        cuuint32_t box[2] = {kGemmKStep, BN};
        cuuint32_t estr[2] = {1, 1};
        if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(dX), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return 5;
    }
    const size_t smem = gemm_smem_bytes(BN);
    // the dynamic shared memory limit is a per-device function attribute
    constexpr int kMaxDev = 64;
    static std::once_flag attr_once[kMaxDev];
    static cudaError_t attr_err[kMaxDev];
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        *last_cuda_error = (int)e0;
        return 5;
    }
    std::call_once(attr_once[dev], [smem, dev] {
        attr_err[dev] = cudaFuncSetAttribute(gemm2_kernel<BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (attr_err[dev] != cudaSuccess) {
        *last_cuda_error = (int)attr_err[dev];
        return 5;
    }
    dim3 grid((unsigned)((N + kGemmRows - 1) / kGemmRows), (unsigned)((M + BN - 1) / BN));
    gemm2_kernel<BN><<<grid, kGemmThreads, smem, stream>>>(tw, tx, alpha, dY, ldy, M, N, K);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

inline int launch_gemm(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                       int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K,
                       cudaStream_t stream, int *last_cuda_error) {
    if (fmt != 2) return 7;  // TL_ERR_UNSUPPORTED: the 1.6-bit tensor-core kernel is not built yet
    if (M >= 256) return launch_gemm_bn<256>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, last_cuda_error);
    if (M >= 128) return launch_gemm_bn<128>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, last_cuda_error);
    if (M >= 64) return launch_gemm_bn<64>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, last_cuda_error);
    if (M >= 32) return launch_gemm_bn<32>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, last_cuda_error);
    return launch_gemm_bn<16>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, last_cuda_error);
}

}  // namespace tlk

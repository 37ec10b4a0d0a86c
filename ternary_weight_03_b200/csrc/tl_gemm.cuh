// tl_gemm.cuh -- batched / prefill ternary linear layer, M >= 16:
//   Y[m][n] = fp16_rn(alpha * sum_k T[n][k] * X[m][k])
// on the sm_100a tensor cores (tcgen05, fp32 accumulators in tensor memory),
// for both storage formats (2-bit base 4 and 1.6-bit base 3).
//
// The pages' GPU kernel is an FP16 x INT2 tensor-core kernel with
// asynchronous copies and fused dequantisation ("Pith review of Spectra
// 1.1", "What carries the argument").  Here, per CTA and output tile of
// 128 weight rows x BN tokens:
//  * a TMA warp streams, per K-step of 64, the activation tile (BN tokens x
//    64 fp16, 128-byte swizzle) and, for the 2-bit format, the packed tile
//    (128 rows x 16 B) into a shared-memory ring (no multicast).  A 1.6-bit
//    row holds 64 trits in 12.8 bytes, so its packed tiles come in blocks of
//    320 trits (128 rows x 64 B, five K-steps) through a separate 2-deep ring;
//  * sets of four decode warps (four sets for 2-bit, two for 1.6-bit), the
//    sets taking the K-steps in turn (thread = weight row = TMEM lane),
//    expand the row's 64
//    trits to exact fp16 -1 / 0 / +1 and write them with tcgen05.st straight
//    into tensor memory, where they are the MMA's A operand -- the expanded
//    weights never touch shared memory;
//  * one thread issues tcgen05.mma.kind::f16 (A from TMEM, B = activations
//    from shared memory) into an fp32 accumulator in TMEM and commits to
//    mbarriers that recycle the ring stages;
//  * the decode warps then read the accumulator with tcgen05.ld (the sets
//    taking its 32-column chunks in turn), scale by
//    alpha and store fp16.
// Split-K, for shapes with fewer output tiles than SMs: a cluster of S CTAs
// shares one output tile, rank r taking K-steps [r nk / S, (r + 1) nk / S)
// (1.6-bit: whole 320-trit blocks, so every rank starts on a block).
// After one cluster barrier (every ring is then idle), the accumulator is
// cut into units of 32 rows (a TMEM lane quarter) x 16 columns; unit u is
// owned by rank u mod S, and a quarter's owned units go to its warps in turn.  Each CTA pushes the units it does not own from
// TMEM into the owner's activation ring with st.async, and the owner sums
// the S partials of its units in rank order -- deterministic, no global
// workspace.
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
// warp 0 TMA, warp 1 MMA, then gemm_dec_sets<FMT> sets of four decode warps
// (one per TMEM lane quarter); set d takes the K-steps k with k mod sets = d
// (and the 32-column chunks c of the accumulator with c / 32 mod sets = d in
// the epilogue).  2-bit: four sets; 1.6-bit: two, since every set reads
// each packed block whole.
template <int FMT>
__host__ __device__ constexpr int gemm_dec_sets() { return FMT == 2 ? 4 : 2; }
template <int FMT>
__host__ __device__ constexpr int gemm_threads() { return 64 + 128 * gemm_dec_sets<FMT>(); }
static_assert(kGemmStages % gemm_dec_sets<2>() == 0 && kGemmStages % gemm_dec_sets<16>() == 0,
              "each ring stage belongs to one decoder set");
// TMEM columns: the accumulator takes BN (at least 32) columns, then the four
// A stages take 32 columns each; the allocation is a power of two.
__host__ __device__ constexpr int gemm_acol_base(int bn) { return bn < 32 ? 32 : bn; }
__host__ __device__ constexpr int gemm_tmem_cols(int bn) {
    return gemm_acol_base(bn) + 32 * 4 <= 256 ? 256 : 512;
}

template <int FMT>
struct GemmSmem {
    // per-stage byte sizes inside the dynamic shared memory block
    __host__ __device__ static constexpr uint32_t x_stage_bytes(int bn) { return (uint32_t)bn * 128u; }
    // 2-bit: one packed tile (128 rows x 16 B = 64 trits) per K-step, filled
    // with the activation stage of the same K-step.  1.6-bit: 64 trits are
    // 12.8 bytes, so packed tiles come in blocks of 320 trits (128 rows x 64 B,
    // five K-steps) through a 2-deep ring of their own.
    static constexpr uint32_t w_row_bytes = FMT == 2 ? 16u : 64u;
    static constexpr uint32_t w_stage_bytes = kGemmRows * w_row_bytes;
    static constexpr int w_stages = FMT == 2 ? kGemmStages : 2;
    static constexpr int ksteps_per_w = FMT == 2 ? 1 : 5;
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

// Base-3 digits of the four bytes of w (byte = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4):
// E[i] holds digit i of byte b in its byte lane b.  The bytes are spread over
// two registers of 16-bit lanes, so one IMAD divides two bytes at once.
__device__ __forceinline__ void digits3_word(uint32_t w, uint32_t (&E)[5]) {
    uint32_t lo = prmt(w, 0u, 0x4240u);  // bytes 0 and 2 in 16-bit lanes
    uint32_t hi = prmt(w, 0u, 0x4341u);  // bytes 1 and 3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // floor(v / 3) = floor(85 (v + 1) / 256) for the valid codes v < 243
        // (85 (v + 1) < 2^16): the product's high byte, moved back into the
        // lane's low byte by the PRMT
        const uint32_t qlo = prmt(lo * 85u + 0x00550055u, 0u, 0x4341u);
        const uint32_t qhi = prmt(hi * 85u + 0x00550055u, 0u, 0x4341u);
        E[i] = prmt(lo - 3u * qlo, hi - 3u * qhi, 0x6240u);  // v mod 3, byte by byte
        lo = qlo;
        hi = qhi;
    }
    E[4] = prmt(lo, hi, 0x6240u);
}

// Exact decode of K-step J (trits 64 J .. 64 J + 63) of a 320-trit block of
// 1.6-bit codes (64 bytes in w[0..15]; trit 5 b + i is digit i of byte b) into
// 32 fp16x2 registers (t_2c, t_2c+1), values -1, 0, +1.  Once the loops
// unroll, every word, digit and byte index below is a compile-time constant.
template <int J>
__device__ __forceinline__ void decode16_kstep(const uint32_t (&w)[16], uint32_t (&out)[32]) {
    constexpr int kW0 = (64 * J / 5) / 4, kW1 = ((64 * J + 63) / 5) / 4;
    uint32_t E[kW1 - kW0 + 1][5];
#pragma unroll
    for (int q = 0; q <= kW1 - kW0; ++q) digits3_word(w[kW0 + q], E[q]);
    const __half2 off = __halves2half2(__ushort_as_half(0x6401), __ushort_as_half(0x6401));
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const int t0 = 64 * J + 2 * c, t1 = t0 + 1;
        const int b0 = t0 / 5, b1 = t1 / 5;
        // result bytes: digit of t0, 0x00 (sign of a digit byte), digit of t1, 0x00
        const uint32_t sel =
            (uint32_t)(b0 & 3) | 0x80u | ((uint32_t)(4 + (b1 & 3)) << 8) | 0x8000u;
        uint32_t p = prmt(E[b0 / 4 - kW0][t0 % 5], E[b1 / 4 - kW0][t1 % 5], sel) | 0x64006400u;
        __half2 h = __hsub2(*reinterpret_cast<__half2 *>(&p), off);  // 1024 + d - 1025 = t
        out[c] = *reinterpret_cast<uint32_t *>(&h);
    }
}

__device__ __forceinline__ void decode16_kstep(int j, const uint32_t (&w)[16], uint32_t (&out)[32]) {
    switch (j) {
        case 0: decode16_kstep<0>(w, out); break;
        case 1: decode16_kstep<1>(w, out); break;
        case 2: decode16_kstep<2>(w, out); break;
        case 3: decode16_kstep<3>(w, out); break;
        default: decode16_kstep<4>(w, out); break;
    }
}

template <int FMT, int BN>
__global__ void __launch_bounds__(gemm_threads<FMT>(), 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
            float alpha, uint16_t *__restrict__ Y, int64_t ldy, int M, int N, int K) {
    using L = GemmSmem<FMT>;
    constexpr int kGemmDecSets = gemm_dec_sets<FMT>();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled activation stages
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *xs = smem;                                         // kGemmStages x BN x 128 B
    uint8_t *ws = xs + kGemmStages * L::x_stage_bytes(BN);      // w_stages x 128 x w_row_bytes
    uint64_t *full = reinterpret_cast<uint64_t *>(ws + L::w_stages * L::w_stage_bytes);
    uint64_t *afull = full + kGemmStages;   // decoders -> MMA (A stage written)
    uint64_t *empty = afull + kGemmStages;  // MMA commit -> producer / decoders
    uint64_t *done = empty + kGemmStages;   // last MMA committed -> epilogue
    uint64_t *redbar = done + 1;            // split-K: the partials pushed to this CTA landed
    uint64_t *wfull = redbar + 1;           // 1.6-bit: packed block landed
    uint64_t *wempty = wfull + 2;           // 1.6-bit: packed block read by all 128 decoders
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(wempty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kGemmRows;
    const int m0 = blockIdx.y * BN;
    const int nk_all = (K + kGemmKStep - 1) / kGemmKStep;
    // split-K rank and K-step range, cut in units of KU K-steps (one packed
    // block) so that every rank starts on a block; the host keeps S <= the
    // number of units, so no range is empty
    constexpr int KU = L::ksteps_per_w;
    const uint32_t S = cluster_nctarank(), rank = cluster_ctarank();
    const int nu = (nk_all + KU - 1) / KU;
    const int kb = KU * (int)(((int64_t)nu * rank) / S);
    const int ke = min(nk_all, KU * (int)(((int64_t)nu * (rank + 1)) / S));
    const int nk = ke - kb;
    // split-K accumulator units: 4 lane quarters x kChunks column chunks of kChunkW
    constexpr int kChunkW = 16;
    constexpr int kChunks = BN / kChunkW;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&afull[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(redbar, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], 128 * kGemmDecSets);  // every set reads every full block
        }
        // bytes pushed here: (S - 1) sources x the tile's 128 x BN floats / S
        if (S > 1) mbar_arrive_expect_tx(redbar, (S - 1) * (uint32_t)(kGemmRows * BN * 4) / S);
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
            const uint32_t bytes = L::x_stage_bytes(BN) + (FMT == 2 ? L::w_stage_bytes : 0u);
            int issued = 0, wissued = 0;
            for (int k = 0; k < nk; ++k) {
                const int s = k % kGemmStages;
                if (k >= kGemmStages && !mbar_wait(&empty[s], ((k / kGemmStages) - 1) & 1))
                    break;
                if (FMT != 2 && k % KU == 0) {
                    // next packed block, once all decoders have read the one two back
                    const int b = k / KU, wsl = b & 1;
                    if (b >= 2 && !mbar_wait(&wempty[wsl], ((b >> 1) - 1) & 1)) break;
                    mbar_arrive_expect_tx(&wfull[wsl], L::w_stage_bytes);
                    tma_load_2d(ws + wsl * L::w_stage_bytes, &tmap_w, &wfull[wsl],
                                (kb / KU + b) * (int)L::w_row_bytes, n0);
                    wissued = b + 1;
                }
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(xs + s * L::x_stage_bytes(BN), &tmap_x, &full[s],
                            (kb + k) * kGemmKStep, m0);
                if (FMT == 2)
                    tma_load_2d(ws + s * L::w_stage_bytes, &tmap_w, &full[s], (kb + k) * 16, n0);
                issued = k + 1;
            }
            // drain: make sure every issued copy has landed before the CTA may exit
            for (int k = issued > kGemmStages ? issued - kGemmStages : 0; k < issued; ++k)
                mbar_wait(&full[k % kGemmStages], (k / kGemmStages) & 1);
            for (int b = wissued > 2 ? wissued - 2 : 0; b < wissued; ++b)
                mbar_wait(&wfull[b & 1], (b >> 1) & 1);
        }
    } else if (warp == 1) {
        // ---- MMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(kGemmRows, BN);
            for (int k = 0; k < nk; ++k) {
                const int s = k % kGemmStages;
                // the activation stage has landed and the decoders wrote A stage s
                // (2-bit: after seeing the same copy complete)
                if (!mbar_wait(&full[s], (k / kGemmStages) & 1) ||
                    !mbar_wait(&afull[s], (k / kGemmStages) & 1))
                    break;
                tc_fence_after();
                const uint32_t xaddr = smem_u32(xs + s * L::x_stage_bytes(BN));
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
        // ---- decode warps: thread = weight row = TMEM lane; set `half` takes
        // the K-steps k = half mod kGemmDecSets ----
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;      // row within the tile
        const int half = (warp - 2) >> 2;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        uint32_t blk[16];  // 1.6-bit: this row's current 320-trit block
        int have_blk = -1;  // 1.6-bit: index of the block in blk
        for (int k = half; k < nk && ok; k += kGemmDecSets) {
            const int s = k % kGemmStages;
            uint32_t a[32];
            if constexpr (FMT == 2) {
                ok = mbar_wait(&full[s], (k / kGemmStages) & 1);
                if (ok && k >= kGemmStages) ok = mbar_wait(&empty[s], ((k / kGemmStages) - 1) & 1);
                if (!ok) break;
                const uint4 pw = *reinterpret_cast<const uint4 *>(ws + s * L::w_stage_bytes +
                                                                   row * 16);
                decode2_exact(pw.x, a);
                decode2_exact(pw.y, a + 8);
                decode2_exact(pw.z, a + 16);
                decode2_exact(pw.w, a + 24);
                // the packed bytes are consumed; order these generic reads before the
                // TMA write that will refill this stage once the MMA releases it
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            } else {
                const int j = k % KU;
                if (k / KU != have_blk) {
                    // this set's first K-step of the block
                    const int b = k / KU, wsl = b & 1;
                    have_blk = b;
                    ok = mbar_wait(&wfull[wsl], (b >> 1) & 1);
                    if (!ok) break;
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        ws + wsl * L::w_stage_bytes + row * L::w_row_bytes);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 v = src[q];
                        blk[4 * q] = v.x;
                        blk[4 * q + 1] = v.y;
                        blk[4 * q + 2] = v.z;
                        blk[4 * q + 3] = v.w;
                    }
                    // order the generic reads before the TMA write that refills the slot
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive(&wempty[wsl]);
                }
                if (k >= kGemmStages && !mbar_wait(&empty[s], ((k / kGemmStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                decode16_kstep(j, blk, a);
            }
            tc_fence_after();
            tmem_st_32x32b_x32(tmem + lane_addr + gemm_acol_base(BN) + 32 * s, a);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&afull[s]);
        }
        // ---- epilogue: accumulator -> alpha -> fp16 -> Y ----
        // (split-K waits for the MMAs as well: TMEM and the ring are reused below)
        const bool fin = mbar_wait(done, 0);
        if (S == 1 && ok && fin) {
            tc_fence_after();
            const int n = n0 + row;
#pragma unroll 1
            for (int c = 32 * half; c < BN; c += 32 * kGemmDecSets) {
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
    if (S > 1) {
        // every CTA of the cluster has finished its MMAs, so its activation ring
        // is idle and can take the partials; the proxy fence orders the tensor
        // core's reads of the ring before the stores that will overwrite it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        cluster_sync();
        if (warp >= 2) {
            tc_fence_after();
            const int quarter = warp & 3;
            const int half = (warp - 2) >> 2;  // the warps of a quarter take chunks in turn
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            const int per = 4 * kChunks / (int)S;  // units owned per rank
            const uint32_t xs_addr = smem_u32(xs);
            // push: unit u = quarter * kChunks + c goes to rank u % S, slot
            // [source rank][u / S][kChunkW / 4 groups of 4 floats][32 lanes]
#pragma unroll 1
            for (int c = half; c < kChunks; c += kGemmDecSets) {
                const int u = quarter * kChunks + c;
                const uint32_t owner = (uint32_t)u % S;
                if (owner == rank) continue;
                uint32_t v[kChunkW];
                tmem_ld_32x32b_x16(tmem + lane_addr + c * kChunkW, v);
                tc_wait_ld();
                const uint32_t slot = rank * per + (uint32_t)u / S;
                const uint32_t dst = mapa_shared(
                    xs_addr + (slot * (kChunkW / 4) * 32 + lane) * 16u, owner);
                const uint32_t rbar = mapa_shared(smem_u32(redbar), owner);
#pragma unroll
                for (int c4 = 0; c4 < kChunkW / 4; ++c4)
                    st_async_v4_f32_mapped(dst + c4 * 32 * 16, rbar, __uint_as_float(v[4 * c4]),
                                           __uint_as_float(v[4 * c4 + 1]),
                                           __uint_as_float(v[4 * c4 + 2]),
                                           __uint_as_float(v[4 * c4 + 3]));
            }
            // reduce the units this CTA owns, in rank order; the owned units of
            // a quarter (c = first, first + S, ...) go to its warps in turn
            if (mbar_wait_cluster(redbar, 0)) {
                const int n = n0 + quarter * 32 + lane;
                const int first = (int)((rank + S - (uint32_t)(quarter * kChunks) % S) % S);
                int turn = 0;
#pragma unroll 1
                for (int c = first; c < kChunks; c += (int)S, ++turn) {
                    if (turn % kGemmDecSets != half) continue;
                    const int u = quarter * kChunks + c;  // u mod S == rank
                    uint32_t v[kChunkW];
                    tmem_ld_32x32b_x16(tmem + lane_addr + c * kChunkW, v);
                    tc_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < kChunkW / 4; ++c4) {
                        float a[4] = {0.f, 0.f, 0.f, 0.f};
                        for (uint32_t r = 0; r < S; ++r) {
                            float4 p;
                            if (r == rank) {
                                p = make_float4(__uint_as_float(v[4 * c4]),
                                                __uint_as_float(v[4 * c4 + 1]),
                                                __uint_as_float(v[4 * c4 + 2]),
                                                __uint_as_float(v[4 * c4 + 3]));
                            } else {
                                const uint32_t slot = r * per + (uint32_t)u / S;
                                p = *reinterpret_cast<const float4 *>(
                                    xs + (slot * (kChunkW / 4) * 32 + c4 * 32 + lane) * 16u);
                            }
                            a[0] += p.x;
                            a[1] += p.y;
                            a[2] += p.z;
                            a[3] += p.w;
                        }
                        if (n < N) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int m = m0 + c * kChunkW + 4 * c4 + j;
                                if (m < M)
                                    Y[(int64_t)m * ldy + n] = f32_to_f16_bits(alpha * a[j]);
                            }
                        }
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
// Every CTA asks for more than half of an SM's 228 KB of shared memory, so at
// most one CTA of this kernel (of any format or BN, from any number of
// concurrent launches) is resident per SM and its TMEM allocation (<= 512
// columns) never waits.  tcgen05.alloc blocks while columns are taken; with
// split-K clusters such a wait could close a cycle (a CTA holding TMEM at the
// cluster barrier for a peer that waits for TMEM behind it).
constexpr size_t kGemmMinSmem = 116 * 1024 + 1;
template <int FMT>
inline size_t gemm_smem_bytes(int bn) {
    using L = GemmSmem<FMT>;
    const size_t need = 1024 + kGemmStages * (size_t)L::x_stage_bytes(bn) +
                        (size_t)L::w_stages * L::w_stage_bytes + (3 * kGemmStages + 6) * 8 + 16;
    return need > kGemmMinSmem ? need : kGemmMinSmem;
}

// CTAs of gemm_kernel<FMT, BN> that can be resident at once in clusters of S
// (cached per device and S; -1 if the occupancy query fails).
template <int FMT, int BN>
inline int gemm_resident(int dev, int S, size_t smem) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static int cache[kMaxDev][4] = {};  // S = 1, 2, 4, 8; 0 = not queried yet
    const int si = S == 1 ? 0 : S == 2 ? 1 : S == 4 ? 2 : 3;
    if (dev < 0 || dev >= kMaxDev) return -1;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (cache[dev][si] != 0) return cache[dev][si];
    }
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(1, 1, 1024);
    q.blockDim = dim3(gemm_threads<FMT>());
    q.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = (unsigned)S;
    q.attrs = at;
    q.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemm_kernel<FMT, BN>, &q) != cudaSuccess)
        return -1;
    std::lock_guard<std::mutex> lock(mu);
    cache[dev][si] = clusters * S > 0 ? clusters * S : -1;
    return cache[dev][si];
}

// Split-K factor: the largest S in {1, 2, 4, 8} such that the S-CTA clusters
// of all output tiles are resident at once, S divides the accumulator's
// 4 x BN / 16 units and every rank keeps at least one K-range unit
// (a K-step of 64 trits; 1.6-bit: a packed block of 320 trits).
template <int FMT, int BN>
inline int gemm_split(int dev, int M, int N, int K, size_t smem) {
    const int64_t tiles = (int64_t)((N + kGemmRows - 1) / kGemmRows) * ((M + BN - 1) / BN);
    const int units = 4 * (BN / 16);
    const int ku = GemmSmem<FMT>::ksteps_per_w * kGemmKStep;
    const int nk = (K + ku - 1) / ku;
    int S = 1;
    while (2 * S <= 8 && units % (2 * S) == 0 && 2 * S <= nk) {
        const int r = gemm_resident<FMT, BN>(dev, 2 * S, smem);
        if (r <= 0 || tiles * 2 * S > r) break;
        S *= 2;
    }
    return S;
}

template <int FMT, int BN>
inline int launch_gemm_bn(const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                          int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K,
                          cudaStream_t stream, int *last_cuda_error) {
    using L = GemmSmem<FMT>;
    auto encode = tensor_map_encoder();
    if (!encode) return 5;  // TL_ERR_CUDA
    CUtensorMap tw, tx;
    // packed row bytes: ceil(K / 4) (2-bit) or ceil(K / 5) (1.6-bit); boxes
    // past the row's end read zeros, whose trits meet zero-filled activations
    const int64_t rowbytes = FMT == 2 ? ((int64_t)K + 3) / 4 : ((int64_t)K + 4) / 5;
    {
        cuuint64_t dims[2] = {(cuuint64_t)rowbytes, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)ldp};
        cuuint32_t box[2] = {L::w_row_bytes, kGemmRows};
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
    const size_t smem = gemm_smem_bytes<FMT>(BN);
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
        attr_err[dev] = cudaFuncSetAttribute(gemm_kernel<FMT, BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (attr_err[dev] != cudaSuccess) {
        *last_cuda_error = (int)attr_err[dev];
        return 5;
    }
    const int S = gemm_split<FMT, BN>(dev, M, N, K, smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + kGemmRows - 1) / kGemmRows), (unsigned)((M + BN - 1) / BN),
                       (unsigned)S);
    cfg.blockDim = dim3(gemm_threads<FMT>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = (unsigned)S;
    cfg.attrs = at;
    cfg.numAttrs = S > 1 ? 1 : 0;  // S = 1: a plain launch
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_kernel<FMT, BN>, tw, tx, alpha, dY, ldy, M, N, K);
    if (e != cudaSuccess) (void)cudaGetLastError();  // the error is returned here, once
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

template <int FMT>
inline int launch_gemm_fmt(const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                           int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K,
                           cudaStream_t stream, int *err) {
    if (M >= 256) return launch_gemm_bn<FMT, 256>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, err);
    if (M >= 128) return launch_gemm_bn<FMT, 128>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, err);
    if (M >= 64) return launch_gemm_bn<FMT, 64>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, err);
    if (M >= 32) return launch_gemm_bn<FMT, 32>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, err);
    return launch_gemm_bn<FMT, 16>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, err);
}

inline int launch_gemm(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
                       int64_t ldx, uint16_t *dY, int64_t ldy, int M, int N, int K,
                       cudaStream_t stream, int *last_cuda_error) {
    if (fmt == 2)
        return launch_gemm_fmt<2>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, last_cuda_error);
    return launch_gemm_fmt<16>(dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, stream, last_cuda_error);
}

}  // namespace tlk

// tl_gemv.cuh -- decode-shaped ternary linear layer, M = 1..8 tokens:
//   Y[m][n] = fp16_rn(alpha * sum_k T[n][k] * X[m][k])
// with T streamed from its 2-bit (base-4) or 1.6-bit (base-3) packing
// ("Pith review of Spectra 1.1", "Core claim" / "What carries the argument").
//
// Design (sm_100a):
//  * Work unit: a CTA owns tiles of 15 output rows; its W warps split the
//    reduction dimension K into contiguous ranges of 64-byte-per-row groups,
//    each warp keeping 4 groups in flight.  Every packed byte is read once
//    with a 128-bit streaming load.  W and the tiles per CTA are chosen at
//    launch from the shape and the kernel's occupancy so that all CTAs are
//    resident at once and carry equal work.
//  * Trits never become +-1 values.  A 2-bit digit d = t + 1 is moved with
//    one PRMT + one LOP3 into the low bits of an fp16 lane, where it reads as
//    the subnormal d * 2^-24 (or d * 2^-20, d * 2^-16 for digits that sit two
//    or four bits higher).  Tensor cores (mma.sync m16n8k16, fp32
//    accumulation) multiply these exactly by the activations; each digit
//    position ("class") has its own accumulator and the classes are combined
//    with exact power-of-two scales at the end.
//  * The offset of d = t + 1 is removed with a sixteenth tile row whose
//    digits are all 1: it accumulates sum_k x[m][k] alongside the 15 weight
//    rows, and y = alpha * (sum_k d x - sum_k x).
//  * 1.6-bit bytes are turned into the same lane layout by two 256-entry
//    tables in shared memory (one lookup per byte).
//  * Warp partials are merged through shared memory by a fixed tree
//    (Pith review, Figure 11 caption text on the paper's appendix G.4:
//    partial sums of a thread block are combined across warps in shared
//    memory by a tree summation), so results are run-to-run deterministic.
#pragma once
#include "tl_common.cuh"

namespace tlk {

constexpr int kGemvMaxWarps = 16;  // warps per CTA (split of K), 2..16
constexpr int kGemvDepth = 4;      // K-groups in flight per warp
constexpr int kGemvRows = 15;  // weight rows per CTA; tile row 15 is the ones row
constexpr int kGemvGroupBytes = 64;  // bytes per row per K-group (4 lanes x 16 B)

// PRMT selectors: output bytes [w.b_q, 0, y.b_q, 0] with y = w >> 2, where the
// zero comes from replicating the sign of y's top byte (always 0).
__device__ __forceinline__ uint32_t sel_q(int q) {
    return 0xF0F0u | (uint32_t)q | ((uint32_t)(4 + q) << 8);
}

// Load the 8 (or 10) uint4 of activations x[g][k0 .. k0 + 8*NV) with lanes
// beyond K zeroed.  `ok` false -> all zero (token g >= M).
template <int NV>
__device__ __forceinline__ void load_x(uint4 (&xv)[NV], const uint16_t *xrow, int k0, int K,
                                       bool ok) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = k0 + 8 * i;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (ok && e < K) {
            v = ld_shared_ro(xrow + e);
            if (e + 8 > K) {
                // zero the halves at positions >= K (K - e in 1..7 valid halves)
                const int valid = K - e;
                uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int lo = 2 * h, hi = 2 * h + 1;
                    uint32_t m = (lo < valid ? 0x0000FFFFu : 0u) | (hi < valid ? 0xFFFF0000u : 0u);
                    w[h] &= m;
                }
            }
        }
        xv[i] = v;
    }
}

__device__ __forceinline__ uint32_t u4get(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// One 2-bit word pair (rows g and g+8, 16 trits each at the same k) against
// the 8 activation pairs xp[0..7] of those 16 trits.  Two accumulators per
// digit class (a / b) keep the dependent MMA chains short.
__device__ __forceinline__ void gemv2_word(uint32_t W, uint32_t V, const uint32_t *xp,
                                           float (&acc0a)[4], float (&acc0b)[4],
                                           float (&acc2a)[4], float (&acc2b)[4]) {
    const uint32_t yW = W >> 2, yV = V >> 2;
    uint32_t PW[4], PV[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        PW[q] = prmt(W, yW, sel_q(q));
        PV[q] = prmt(V, yV, sel_q(q));
    }
    constexpr uint32_t M0 = 0x00030003u, M2 = 0x00300030u;
    // class 0: trits (4q, 4q+1) -> activation pair 2q; class 2: (4q+2, 4q+3) -> 2q+1
    mma_16816(acc0a, PW[0] & M0, PV[0] & M0, PW[1] & M0, PV[1] & M0, xp[0], xp[2]);
    mma_16816(acc2a, PW[0] & M2, PV[0] & M2, PW[1] & M2, PV[1] & M2, xp[1], xp[3]);
    mma_16816(acc0b, PW[2] & M0, PV[2] & M0, PW[3] & M0, PV[3] & M0, xp[4], xp[6]);
    mma_16816(acc2b, PW[2] & M2, PV[2] & M2, PW[3] & M2, PV[3] & M2, xp[5], xp[7]);
}

// Shared-memory tables for 1.6-bit bytes.  For b = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4:
//  even[b]: d0 @0, d2 @4, d4 @8 (low half); d1 @16, d3 @20 (high half)
//  odd[b] : d1 @0, d3 @4, d0 @8 (low half); d2 @16, d4 @20 (high half)
// Bytes >= 243 map to 0.
__device__ __forceinline__ void build_lut16(uint32_t *even, uint32_t *odd) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
        uint32_t e = 0, o = 0;
        if (b < 243) {
            int r = b, d[5];
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                d[i] = r % 3;
                r /= 3;
            }
            e = (uint32_t)d[0] | ((uint32_t)d[2] << 4) | ((uint32_t)d[4] << 8) |
                ((uint32_t)d[1] << 16) | ((uint32_t)d[3] << 20);
            o = (uint32_t)d[1] | ((uint32_t)d[3] << 4) | ((uint32_t)d[0] << 8) |
                ((uint32_t)d[2] << 16) | ((uint32_t)d[4] << 20);
        }
        even[b] = e;
        odd[b] = o;
    }
}

// One 1.6-bit 32-bit word pair (4 bytes = 20 trits per row) against the 10
// activation pairs xp[0..9] of those trits.
__device__ __forceinline__ void gemv16_word(uint32_t W, uint32_t V, const uint32_t *xp,
                                            const uint32_t *even, const uint32_t *odd,
                                            float (&acc0)[4], float (&acc2)[4],
                                            float (&acc4)[4]) {
    constexpr uint32_t M0 = 0x00030003u, M2 = 0x00300030u, M4 = 0x03000300u;
    uint32_t R2W[2], R2V[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {  // byte pairs (0,1) and (2,3) of the word
        const uint32_t leW = even[(W >> (16 * p)) & 0xFF], loW = odd[(W >> (16 * p + 8)) & 0xFF];
        const uint32_t leV = even[(V >> (16 * p)) & 0xFF], loV = odd[(V >> (16 * p + 8)) & 0xFF];
        // trits (0,1) and (6,7) of this pair: class 0, activation pairs 5p+0 and 5p+3
        mma_16816(acc0, leW & M0, leV & M0, loW & M0, loV & M0, xp[5 * p + 0], xp[5 * p + 3]);
        // trits (2,3) and (8,9): class 2, pairs 5p+1 and 5p+4
        mma_16816(acc2, leW & M2, leV & M2, loW & M2, loV & M2, xp[5 * p + 1], xp[5 * p + 4]);
        // trits (4,5) straddle the two bytes: class 4
        R2W[p] = (leW | (loW << 16)) & M4;
        R2V[p] = (leV | (loV << 16)) & M4;
    }
    mma_16816(acc4, R2W[0], R2V[0], R2W[1], R2V[1], xp[2], xp[7]);
}

// A 64-byte row whose digits are all 1 (2-bit: 0x55, 1.6-bit: 121 = 11111 in
// base 3): the source of the ones row (tile row 15).
__device__ __align__(16) const uint8_t g_ones_row2[kGemvGroupBytes] = {
    0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55,
    0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55,
    0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55,
    0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55};
__device__ __align__(16) const uint8_t g_ones_row16[kGemvGroupBytes] = {
    121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121,
    121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121,
    121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121,
    121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121, 121};

// All MMAs of one K-group for one lane: 4 words of rows g and g+8 (wa, wb)
// against the activations of the lane's chunk starting at element k0.
// MASK: zero activations at k >= K (only for the last, partial group).
template <int FMT, bool MASK>
__device__ __forceinline__ void gemv_group(const uint4 &wa, const uint4 &wb, const uint16_t *xrow,
                                           int k0, int K, const uint32_t *lut_even,
                                           const uint32_t *lut_odd, float (&acc0a)[4],
                                           float (&acc0b)[4], float (&acc2a)[4],
                                           float (&acc2b)[4], float (&acc4)[4]) {
    if constexpr (FMT == 2) {
        // one 32-bit word = 16 trits = 2 uint4 of activations (32 B aligned)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 xv[2];
            if constexpr (MASK) {
                load_x<2>(xv, xrow, k0 + 16 * j, K, true);
            } else {
                xv[0] = ld_shared_ro(xrow + k0 + 16 * j);
                xv[1] = ld_shared_ro(xrow + k0 + 16 * j + 8);
            }
            const uint32_t *xp = reinterpret_cast<const uint32_t *>(xv);
            gemv2_word(u4get(wa, j), u4get(wb, j), xp, acc0a, acc0b, acc2a, acc2b);
        }
    } else {
        // two 32-bit words = 40 trits = 5 uint4 of activations (80 B, aligned
        // because the lane chunk k0 starts at a multiple of 80 trits)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            uint4 xv[5];
            if constexpr (MASK) {
                load_x<5>(xv, xrow, k0 + 40 * jj, K, true);
            } else {
#pragma unroll
                for (int i = 0; i < 5; ++i) xv[i] = ld_shared_ro(xrow + k0 + 40 * jj + 8 * i);
            }
            const uint32_t *xp = reinterpret_cast<const uint32_t *>(xv);
            gemv16_word(u4get(wa, 2 * jj), u4get(wb, 2 * jj), xp, lut_even, lut_odd, acc0a,
                        acc2a, acc4);
            gemv16_word(u4get(wa, 2 * jj + 1), u4get(wb, 2 * jj + 1), xp + 10, lut_even,
                        lut_odd, acc0b, acc2b, acc4);
        }
    }
}

// Launch shape: blockDim.x = 32 * W (W warps split K), each CTA handles
// `tiles_per_cta` row tiles of 15 rows, strided by gridDim.x.
//
// Lanes never branch on their own row or token: lanes of tokens m >= M read
// token 0's activations and lanes of rows n >= N read row 0's bytes; those
// outputs are computed but never stored.  Lanes of the ones row read a
// constant 64-byte row with a zero stride.
template <int FMT>
__global__ void __launch_bounds__(32 * kGemvMaxWarps)
gemv_kernel(const uint8_t *__restrict__ P, int64_t ldp, float alpha, const uint16_t *__restrict__ X,
            int64_t ldx, uint16_t *__restrict__ Y, int64_t ldy, int M, int N, int K,
            int tiles_per_cta) {
    constexpr int TPB = FMT == 2 ? 4 : 5;              // trits per byte
    constexpr int TRITS_LANE = 16 * TPB;               // trits per lane per group (64 / 80)
    constexpr int TRITS_GROUP = kGemvGroupBytes * TPB; // trits per row per group (256 / 320)

    __shared__ float red[kGemvMaxWarps][16][8];
    __shared__ uint32_t lut_even[FMT == 2 ? 1 : 256];
    __shared__ uint32_t lut_odd[FMT == 2 ? 1 : 256];
    if constexpr (FMT != 2) {
        build_lut16(lut_even, lut_odd);
        __syncthreads();
    }

    const int nwarps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const bool onesB = (g == 7);
    const uint16_t *xrow = X + (int64_t)(g < M ? g : 0) * ldx;
    const int64_t rowbytes = FMT == 2 ? ((int64_t)K + 3) / 4 : ((int64_t)K + 4) / 5;
    const int KG = (int)((rowbytes + kGemvGroupBytes - 1) / kGemvGroupBytes);
    const int KG_full = K / TRITS_GROUP;  // groups with every activation index < K
    // this warp's contiguous range of K-groups; [kg_begin, kmain) needs no masking
    const int kg_begin = (int)((int64_t)KG * warp / nwarps);
    const int kg_end = (int)((int64_t)KG * (warp + 1) / nwarps);
    const int kmain = kg_end < KG_full ? kg_end : KG_full;
    const int ntiles = (N + kGemvRows - 1) / kGemvRows;
    const uint8_t *ones = FMT == 2 ? g_ones_row2 : g_ones_row16;

    for (int it = 0; it < tiles_per_cta; ++it) {
        const int tile = blockIdx.x + it * gridDim.x;
        if (tile >= ntiles) break;  // uniform across the CTA
        const int n0 = tile * kGemvRows;
        const int rA = n0 + g, rB = n0 + g + 8;
        const uint8_t *pA = P + (int64_t)(rA < N ? rA : 0) * ldp + 16 * c;
        const uint8_t *pB = onesB ? ones + 16 * c : P + (int64_t)(rB < N ? rB : 0) * ldp + 16 * c;
        const int64_t strideB = onesB ? 0 : kGemvGroupBytes;

        float acc0a[4] = {0.f, 0.f, 0.f, 0.f}, acc0b[4] = {0.f, 0.f, 0.f, 0.f};
        float acc2a[4] = {0.f, 0.f, 0.f, 0.f}, acc2b[4] = {0.f, 0.f, 0.f, 0.f};
        float acc4[4] = {0.f, 0.f, 0.f, 0.f};

        // main part: ring of kGemvDepth K-groups in flight per warp, no masking
        uint4 ra[kGemvDepth], rb[kGemvDepth];
#pragma unroll
        for (int i = 0; i < kGemvDepth; ++i) {
            if (kg_begin + i < kmain) {
                ra[i] = ld_stream(pA + (int64_t)(kg_begin + i) * kGemvGroupBytes);
                rb[i] = ld_stream(pB + (int64_t)(kg_begin + i) * strideB);
            }
        }
        if (it == 0) {
            // weights requested; activations and outputs may belong to preceding work
            pdl_launch_dependents();
            pdl_wait();
        }
        for (int base = kg_begin; base < kmain; base += kGemvDepth) {
#pragma unroll
            for (int i = 0; i < kGemvDepth; ++i) {
                const int kg = base + i;
                if (kg < kmain) {
                    const uint4 wa = ra[i], wb = rb[i];
                    if (kg + kGemvDepth < kmain) {
                        ra[i] = ld_stream(pA + (int64_t)(kg + kGemvDepth) * kGemvGroupBytes);
                        rb[i] = ld_stream(pB + (int64_t)(kg + kGemvDepth) * strideB);
                    }
                    gemv_group<FMT, false>(wa, wb, xrow, kg * TRITS_GROUP + c * TRITS_LANE, K,
                                           lut_even, lut_odd, acc0a, acc0b, acc2a, acc2b, acc4);
                }
            }
        }
        // tail: the last, partial K-group (at most one per row), masked
        for (int kg = kmain > kg_begin ? kmain : kg_begin; kg < kg_end; ++kg) {
            const int64_t boff = (int64_t)kg * kGemvGroupBytes + 16 * c;
            uint4 wa = make_uint4(0, 0, 0, 0), wb = make_uint4(0, 0, 0, 0);
            if (boff < rowbytes) {
                wa = ld_stream(pA + (int64_t)kg * kGemvGroupBytes);
                wb = ld_stream(pB + (int64_t)kg * strideB);
            }
            gemv_group<FMT, true>(wa, wb, xrow, kg * TRITS_GROUP + c * TRITS_LANE, K, lut_even,
                                  lut_odd, acc0a, acc0b, acc2a, acc2b, acc4);
        }

        // combine digit classes with exact power-of-two scales: sum_k d * x
        float s[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s[i] = (acc0a[i] + acc0b[i]) * 16777216.0f + (acc2a[i] + acc2b[i]) * 1048576.0f;
            if constexpr (FMT != 2) s[i] += acc4[i] * 65536.0f;
        }
        red[warp][g][2 * c] = s[0];
        red[warp][g][2 * c + 1] = s[1];
        red[warp][g + 8][2 * c] = s[2];
        red[warp][g + 8][2 * c + 1] = s[3];
        __syncthreads();
        for (int t = threadIdx.x; t < kGemvRows * 8; t += blockDim.x) {
            const int row = t >> 3, m = t & 7;
            if (m < M && n0 + row < N) {
                // pairwise tree over the warps' partials (fixed order)
                float tot[kGemvMaxWarps], sx[kGemvMaxWarps];
#pragma unroll
                for (int w = 0; w < kGemvMaxWarps; ++w) {
                    tot[w] = w < nwarps ? red[w][row][m] : 0.f;
                    sx[w] = w < nwarps ? red[w][15][m] : 0.f;
                }
#pragma unroll
                for (int span = 1; span < kGemvMaxWarps; span *= 2)
#pragma unroll
                    for (int w = 0; w + span < kGemvMaxWarps; w += 2 * span) {
                        tot[w] += tot[w + span];
                        sx[w] += sx[w + span];
                    }
                Y[(int64_t)m * ldy + n0 + row] = f32_to_f16_bits(alpha * (tot[0] - sx[0]));
            }
        }
        __syncthreads();
    }
}

// Host-side launch shape for a GEMV: warps per CTA (split of K) and tiles
// per CTA, chosen so that every CTA is resident in one wave and all CTAs
// carry the same number of row tiles.
struct GemvShape {
    int warps;
    int tiles_per_cta;
    int grid;
};

template <int FMT>
inline GemvShape gemv_shape(int N, int K, int num_sms, int (*occupancy)(int fmt, int warps)) {
    const int64_t rowbytes = FMT == 2 ? ((int64_t)K + 3) / 4 : ((int64_t)K + 4) / 5;
    const int KG = (int)((rowbytes + kGemvGroupBytes - 1) / kGemvGroupBytes);
    const int ntiles = (N + kGemvRows - 1) / kGemvRows;
    GemvShape best{4, 1, ntiles};
    double best_cost = 1e30;
    for (int w = 2; w <= kGemvMaxWarps; w += 2) {
        if (w > 4 && w > KG) break;
        const int occ = occupancy(FMT, w);
        if (occ < 1) continue;
        const int slots = num_sms * occ;
        const int t = (ntiles + slots - 1) / slots;
        const int grid = (ntiles + t - 1) / t;
        const int groups_per_warp = (KG + w - 1) / w;
        // critical path in K-groups, plus a penalty when fewer than one CTA per SM
        // or few warps in flight per SM
        const double warps_per_sm = (double)grid * w / num_sms;
        double cost = (double)t * groups_per_warp + 0.5 * t;
        if (warps_per_sm < 8) cost *= 8.0 / warps_per_sm;
        if (grid < num_sms) cost *= (double)num_sms / grid;
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = GemvShape{w, t, grid};
        }
    }
    return best;
}

}  // namespace tlk

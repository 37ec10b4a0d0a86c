// tl_ternarise.cuh -- device ternariser + packer: fp16 weights W [N][K] ->
// shared scale alpha and packed trits (2-bit or 1.6-bit rows).
//
// The pages ("Pith review of Spectra 1.1", "What carries the argument") give
// the layer's weights as {-1, 0, 1} times one shared floating-point scale,
// obtained by rounding to the nearest ternary value; they give no formula
// for the scale.  Reading taken here: alpha = mean |W| over the matrix, and
// t = the nearest of {-1, 0, 1} to w / alpha with ties to 0.
//
// Three launches, stream-ordered, no allocation:
//  1. absum_kernel: every |w| is an integer number of 2^-24 units (binary16
//     subnormals are multiples of 2^-24), so the sum S is taken exactly in
//     128-bit integers; each block writes its partial to the workspace.
//     Integer addition is associative, so alpha does not depend on the grid.
//  2. scale_kernel (one block): S = sum of the partials, then
//     alpha = fp32_rn(fp64_rn(fp64_rn(S) / (N K)) * 2^-24), stored to *alpha.
//  3. ternarise_pack_kernel<FMT>: per packed 32-bit word (16 or 20 trits),
//     t = sign(w) if 2 |w| > alpha else 0, digits d = t + 1, bytes
//     sum d_i b^i (b = 4 or 3, least significant first), pad digit 1 for
//     trits past K, bytes past the row's end written as 0.
//     2 |w| > alpha is exactly the fp32 rule fp32_rn(w / alpha) > 0.5: 0.5
//     is an fp32 value, and an fp32 alpha within rounding distance of 2 |w|
//     (relative 2^-24) other than 2 |w| itself does not exist, so the
//     rounded quotient lies above 0.5 exactly when the true one does.
#pragma once
#include <cstdint>
#include "tl_common.cuh"

namespace tlk {

constexpr int kTzThreads = 256;
constexpr int kTzMaxPartials = 1024;  // 16 B each: the workspace holds 16 KiB

struct U128 {
    uint64_t lo, hi;
};

__device__ __forceinline__ void add128(U128 &a, uint64_t lo, uint64_t hi) {
    a.lo += lo;
    a.hi += hi + (a.lo < lo ? 1u : 0u);
}

// |w| of a binary16 bit pattern in 2^-24 units (exact; < 2^41).
__device__ __forceinline__ uint64_t half_abs_units(uint32_t h) {
    const uint32_t e = (h >> 10) & 31u, m = h & 1023u;
    return e == 0 ? (uint64_t)m : (uint64_t)(1024u + m) << (e - 1);
}

// Sum of v over the block (kTzThreads threads); the result is valid in thread 0.
__device__ __forceinline__ U128 block_sum128(U128 v) {
    __shared__ uint64_t s_lo[kTzThreads / 32], s_hi[kTzThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t lo = __shfl_xor_sync(0xffffffffu, v.lo, off);
        const uint64_t hi = __shfl_xor_sync(0xffffffffu, v.hi, off);
        add128(v, lo, hi);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_lo[warp] = v.lo;
        s_hi[warp] = v.hi;
    }
    __syncthreads();
    U128 r{0, 0};
    if (warp == 0) {
        if (lane < kTzThreads / 32) r = U128{s_lo[lane], s_hi[lane]};
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint64_t lo = __shfl_xor_sync(0xffffffffu, r.lo, off);
            const uint64_t hi = __shfl_xor_sync(0xffffffffu, r.hi, off);
            add128(r, lo, hi);
        }
    }
    return r;
}

// Pass 1.  Work unit: 16 consecutive entries of one row (32 bytes, two
// 16-byte loads when the unit lies inside the row).  Blocks walk (row, group
// of 256 units) pairs, so one 64-bit division per block step is all the index
// arithmetic.
__global__ void __launch_bounds__(kTzThreads)
absum_kernel(const uint16_t *__restrict__ W, int64_t ldw, int N, int K, U128 *partials) {
    const int units = (K + 15) / 16;
    const int groups = (units + kTzThreads - 1) / kTzThreads;
    U128 acc{0, 0};
    for (int64_t r = blockIdx.x; r < (int64_t)N * groups; r += gridDim.x) {
        const int64_t n = r / groups;
        const int u = (int)(r - n * groups) * kTzThreads + (int)threadIdx.x;
        if (u >= units) continue;
        const uint16_t *row = W + n * ldw;
        const int k0 = 16 * u;
        uint64_t s = 0;  // 16 x < 2^41
        if (k0 + 16 <= K) {
            // cached loads: pass 3 reads W again, and a matrix below the L2's
            // size can partly stay there; pass 3 streams it out (last use)
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(row + k0));
            const uint4 b = __ldg(reinterpret_cast<const uint4 *>(row + k0) + 1);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
                s += half_abs_units(w[i] & 0xFFFFu) + half_abs_units(w[i] >> 16);
        } else {
            for (int k = k0; k < K; ++k) s += half_abs_units(row[k]);
        }
        add128(acc, s, 0);
    }
    const U128 tot = block_sum128(acc);
    if (threadIdx.x == 0) partials[blockIdx.x] = tot;
}

// 128-bit unsigned integer to double, rounded to nearest even.
__device__ __forceinline__ double u128_to_double_rn(U128 v) {
    if (v.hi == 0) return __ull2double_rn(v.lo);
    const int lz = __clzll((long long)v.hi);
    // the 64 leading bits, with every bit below them folded into bit 0 (far
    // below double's rounding position, so it only decides exact halves)
    uint64_t top = lz ? (v.hi << lz) | (v.lo >> (64 - lz)) : v.hi;
    const uint64_t rest = lz ? v.lo << lz : v.lo;
    top |= rest != 0 ? 1u : 0u;
    return ldexp(__ull2double_rn(top), 64 - lz);
}

// Pass 2 (one block).
__global__ void __launch_bounds__(kTzThreads)
scale_kernel(const U128 *__restrict__ partials, int count, int64_t NK, float *alpha) {
    U128 acc{0, 0};
    for (int i = threadIdx.x; i < count; i += kTzThreads) add128(acc, partials[i].lo, partials[i].hi);
    const U128 S = block_sum128(acc);
    if (threadIdx.x == 0) {
        const double mean_units = __ddiv_rn(u128_to_double_rn(S), (double)NK);
        *alpha = __double2float_rn(mean_units * 0x1p-24);
    }
}

// Digit d = t + 1 of one binary16 weight: 2 if w > alpha / 2, 0 if
// w < -alpha / 2, else 1 (2 |w| is exact in fp32).
__device__ __forceinline__ uint32_t trit_digit(uint32_t h, float alpha) {
    const float a2 = 2.0f * fabsf(__half2float(__ushort_as_half((unsigned short)h)));
    return a2 > alpha ? ((h & 0x8000u) ? 0u : 2u) : 1u;
}

// Pass 3.  Work unit: one packed 32-bit word = 4 bytes = 16 (2-bit) or 20
// (1.6-bit) trits = 32 or 40 bytes of W at an 8-byte-aligned offset.
template <int FMT>
__global__ void __launch_bounds__(kTzThreads)
ternarise_pack_kernel(const uint16_t *__restrict__ W, int64_t ldw, int N, int K,
                      uint8_t *__restrict__ P, int64_t ldp, const float *__restrict__ alpha_p) {
    constexpr int D = FMT == 2 ? 4 : 5;  // trits per byte
    constexpr int TW = 4 * D;            // trits per word
    constexpr uint32_t B = FMT == 2 ? 4u : 3u;
    const float alpha = *alpha_p;
    const int64_t rb = FMT == 2 ? ((int64_t)K + 3) / 4 : ((int64_t)K + 4) / 5;
    const int words = (int)(ldp / 4);
    const int groups = (words + kTzThreads - 1) / kTzThreads;
    for (int64_t r = blockIdx.x; r < (int64_t)N * groups; r += gridDim.x) {
        const int64_t n = r / groups;
        const int g = (int)(r - n * groups) * kTzThreads + (int)threadIdx.x;
        if (g >= words) continue;
        const uint16_t *row = W + n * ldw;
        const int64_t k0 = (int64_t)g * TW;
        uint32_t h[TW];
        if (k0 + TW <= K) {
            if constexpr (FMT == 2) {
                const uint4 a = __ldcs(reinterpret_cast<const uint4 *>(row + k0));
                const uint4 b = __ldcs(reinterpret_cast<const uint4 *>(row + k0) + 1);
                const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    h[2 * i] = w[i] & 0xFFFFu;
                    h[2 * i + 1] = w[i] >> 16;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 5; ++i) {
                    const uint2 v = __ldcs(reinterpret_cast<const uint2 *>(row + k0) + i);
                    h[4 * i] = v.x & 0xFFFFu;
                    h[4 * i + 1] = v.x >> 16;
                    h[4 * i + 2] = v.y & 0xFFFFu;
                    h[4 * i + 3] = v.y >> 16;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < TW; ++i) h[i] = k0 + i < K ? row[k0 + i] : 0u;
        }
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if ((int64_t)4 * g + b >= rb) continue;  // past the row's end: 0
            uint32_t byte = 0, place = 1;
#pragma unroll
            for (int i = 0; i < D; ++i) {
                const int idx = b * D + i;
                const uint32_t d = k0 + idx < K ? trit_digit(h[idx], alpha) : 1u;  // pad: 0-trit
                byte += d * place;
                place *= B;
            }
            word |= byte << (8 * b);
        }
        *reinterpret_cast<uint32_t *>(P + n * ldp + 4 * (int64_t)g) = word;
    }
}

// Host: the three launches on `stream`.  Returns 0 or 5 (TL_ERR_CUDA, with
// the CUDA error in *last_cuda_error).
inline int launch_ternarise(int fmt, const uint16_t *dW, int64_t ldw, int N, int K, uint8_t *dP,
                            int64_t ldp, float *dAlpha, void *workspace, int num_sms,
                            cudaStream_t stream, int *last_cuda_error) {
    U128 *partials = reinterpret_cast<U128 *>(workspace);
    const int units = (K + 15) / 16;
    const int64_t steps1 = (int64_t)N * ((units + kTzThreads - 1) / kTzThreads);
    int g1 = 4 * num_sms;
    if (g1 > kTzMaxPartials) g1 = kTzMaxPartials;
    if (steps1 < g1) g1 = (int)steps1;
    (void)cudaGetLastError();  // an error of an earlier call was returned by that call
    absum_kernel<<<g1, kTzThreads, 0, stream>>>(dW, ldw, N, K, partials);
    scale_kernel<<<1, kTzThreads, 0, stream>>>(partials, g1, (int64_t)N * K, dAlpha);
    const int words = (int)(ldp / 4);
    const int64_t steps3 = (int64_t)N * ((words + kTzThreads - 1) / kTzThreads);
    int64_t g3 = (int64_t)8 * num_sms;
    if (steps3 < g3) g3 = steps3;
    if (fmt == 2)
        ternarise_pack_kernel<2><<<(unsigned)g3, kTzThreads, 0, stream>>>(dW, ldw, N, K, dP, ldp, dAlpha);
    else
        ternarise_pack_kernel<16><<<(unsigned)g3, kTzThreads, 0, stream>>>(dW, ldw, N, K, dP, ldp, dAlpha);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *last_cuda_error = (int)e;
        return 5;
    }
    return 0;
}

}  // namespace tlk

// tl_host.cpp -- host-side codec of libternary: tl_pack2, tl_pack16,
// tl_unpack, tl_packed_row_bytes, tl_status_str.
//
// Formats ("Pith review of Spectra 1.1", "Core claim" and "What carries the
// argument"): 2-bit = four trits per byte as base-4 digits, 1.6-bit = five
// trits per byte as base-3 digits (3^5 = 243 <= 2^8).  The digit of a trit t
// is t + 1; trit k of a row is digit k % g of byte k / g; digit i weighs b^i.
//
// The packers are table driven: every byte is assembled from per-position
// digit contributions, and the unpacker decodes a byte with one table row.
// Large matrices are split across host threads by rows.
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

#include "tl.h"

namespace {

// Contribution of trit value t (index t + 1) at digit position i:
// 2-bit: (t + 1) << 2i;  1.6-bit: (t + 1) * 3^i.
struct PackTables {
    uint8_t two[4][3];
    uint8_t three[5][3];
    PackTables() {
        for (int i = 0; i < 4; ++i)
            for (int d = 0; d < 3; ++d) two[i][d] = (uint8_t)(d << (2 * i));
        int w = 1;
        for (int i = 0; i < 5; ++i, w *= 3)
            for (int d = 0; d < 3; ++d) three[i][d] = (uint8_t)(d * w);
    }
};

// Decode tables: valid flag and the g trits of every byte value.
struct UnpackTables {
    int8_t two[256][4];
    bool two_ok[256];
    int8_t three[256][5];
    bool three_ok[256];
    UnpackTables() {
        for (int v = 0; v < 256; ++v) {
            bool ok = true;
            for (int i = 0; i < 4; ++i) {
                int d = (v >> (2 * i)) & 3;
                ok = ok && d != 3;
                two[v][i] = (int8_t)(d - 1);
            }
            two_ok[v] = ok;
            int r = v;
            for (int i = 0; i < 5; ++i) {
                three[v][i] = (int8_t)(r % 3 - 1);
                r /= 3;
            }
            three_ok[v] = v < 243;
        }
    }
};

const PackTables &pack_tables() {
    static const PackTables t;
    return t;
}
const UnpackTables &unpack_tables() {
    static const UnpackTables t;
    return t;
}

inline bool trit_ok(int8_t t) { return t >= -1 && t <= 1; }

template <int G>
void pack_rows(const int8_t *T, int64_t n0, int64_t n1, int64_t K, int64_t ldt, uint8_t *P,
               int64_t ldp, const uint8_t (*tab)[3]) {
    const int64_t full = K / G, rem = K % G;
    const int64_t rb = full + (rem ? 1 : 0);
    for (int64_t n = n0; n < n1; ++n) {
        const int8_t *t = T + n * ldt;
        uint8_t *p = P + n * ldp;
        for (int64_t j = 0; j < full; ++j, t += G) {
            unsigned v = 0;
            for (int i = 0; i < G; ++i) v += tab[i][t[i] + 1];
            p[j] = (uint8_t)v;
        }
        if (rem) {
            unsigned v = 0;
            for (int i = 0; i < G; ++i) v += tab[i][(i < rem ? t[i] : 0) + 1];
            p[full] = (uint8_t)v;
        }
        if (ldp > rb) std::memset(p + rb, 0, (size_t)(ldp - rb));
    }
}

int threads_for(int64_t work) {
    if (work < (int64_t)1 << 22) return 1;
    unsigned hc = std::thread::hardware_concurrency();
    int n = (int)std::min<unsigned>(hc ? hc : 1, 64);
    return std::max(1, n);
}

template <class F>
void parallel_rows(int64_t N, int nthreads, F &&f) {
    if (nthreads <= 1 || N < 2 * nthreads) {
        f(0, N);
        return;
    }
    std::vector<std::thread> pool;
    pool.reserve(nthreads - 1);
    for (int i = 1; i < nthreads; ++i)
        pool.emplace_back([&, i] { f(N * i / nthreads, N * (i + 1) / nthreads); });
    f(0, N / nthreads);
    for (auto &th : pool) th.join();
}

int pack_impl(int fmt, const int8_t *T, int64_t N, int64_t K, int64_t ldt, uint8_t *P,
              int64_t ldp) {
    const int64_t rb = tl_packed_row_bytes(fmt, K);
    if (rb < 0 || N < 0 || ldt < K || ldp < rb || ldp < 0) return TL_ERR_INVALID_ARG;
    if (N > 0 && ldp > 0 && P == nullptr) return TL_ERR_INVALID_ARG;
    if (N > 0 && K > 0 && T == nullptr) return TL_ERR_INVALID_ARG;
    if (N == 0) return TL_OK;
    const int nt = threads_for(N * K);
    // validate first so that a bad trit leaves no partial guarantee to reason about
    std::vector<char> bad(std::max(nt, 1), 0);
    {
        std::vector<std::thread> pool;
        auto check = [&](int slot, int64_t a, int64_t b) {
            for (int64_t n = a; n < b && !bad[slot]; ++n) {
                const int8_t *t = T + n * ldt;
                for (int64_t k = 0; k < K; ++k)
                    if (!trit_ok(t[k])) {
                        bad[slot] = 1;
                        break;
                    }
            }
        };
        if (nt <= 1 || N < 2 * nt) {
            check(0, 0, N);
        } else {
            for (int i = 1; i < nt; ++i)
                pool.emplace_back(check, i, N * i / nt, N * (i + 1) / nt);
            check(0, 0, N / nt);
            for (auto &th : pool) th.join();
        }
    }
    for (char b : bad)
        if (b) return TL_ERR_BAD_TRIT;
    const PackTables &pt = pack_tables();
    parallel_rows(N, nt, [&](int64_t a, int64_t b) {
        if (fmt == TL_FMT_2BIT)
            pack_rows<4>(T, a, b, K, ldt, P, ldp, pt.two);
        else
            pack_rows<5>(T, a, b, K, ldt, P, ldp, pt.three);
    });
    return TL_OK;
}

}  // namespace

extern "C" {

const char *tl_status_str(int status) {
    switch (status) {
        case TL_OK: return "TL_OK";
        case TL_ERR_INVALID_ARG: return "TL_ERR_INVALID_ARG: invalid argument";
        case TL_ERR_BAD_TRIT: return "TL_ERR_BAD_TRIT: trit outside {-1, 0, 1}";
        case TL_ERR_BAD_CODE: return "TL_ERR_BAD_CODE: byte is not a valid packed code";
        case TL_ERR_ALIGN: return "TL_ERR_ALIGN: pointer or stride misaligned";
        case TL_ERR_CUDA: return "TL_ERR_CUDA: CUDA runtime error";
        case TL_ERR_TIMEOUT: return "TL_ERR_TIMEOUT: a device wait ran out";
        case TL_ERR_UNSUPPORTED: return "TL_ERR_UNSUPPORTED: no kernel for this case";
        default: return "unknown tl status";
    }
}

int64_t tl_packed_row_bytes(int fmt, int64_t K) {
    if (K < 0) return -1;
    if (fmt == TL_FMT_2BIT) return (K + 3) / 4;
    if (fmt == TL_FMT_1P6BIT) return (K + 4) / 5;
    return -1;
}

int tl_pack2(const int8_t *T, int64_t N, int64_t K, int64_t ldt, uint8_t *P, int64_t ldp) {
    return pack_impl(TL_FMT_2BIT, T, N, K, ldt, P, ldp);
}

int tl_pack16(const int8_t *T, int64_t N, int64_t K, int64_t ldt, uint8_t *P, int64_t ldp) {
    return pack_impl(TL_FMT_1P6BIT, T, N, K, ldt, P, ldp);
}

int tl_unpack(int fmt, const uint8_t *P, int64_t N, int64_t K, int64_t ldp, int8_t *T,
              int64_t ldt, int64_t *bad_index) {
    const int64_t rb = tl_packed_row_bytes(fmt, K);
    if (rb < 0 || N < 0 || ldt < K || ldp < rb) return TL_ERR_INVALID_ARG;
    if (N > 0 && rb > 0 && P == nullptr) return TL_ERR_INVALID_ARG;
    if (N > 0 && K > 0 && T == nullptr) return TL_ERR_INVALID_ARG;
    const UnpackTables &ut = unpack_tables();
    const int g = fmt == TL_FMT_2BIT ? 4 : 5;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *p = P + n * ldp;
        int8_t *t = T + n * ldt;
        for (int64_t j = 0; j < rb; ++j) {
            const unsigned v = p[j];
            const bool ok = fmt == TL_FMT_2BIT ? ut.two_ok[v] : ut.three_ok[v];
            if (!ok) {
                if (bad_index) *bad_index = n * ldp + j;
                return TL_ERR_BAD_CODE;
            }
            const int8_t *digits = fmt == TL_FMT_2BIT ? ut.two[v] : ut.three[v];
            const int64_t k0 = j * g;
            const int cnt = (int)std::min<int64_t>(g, K - k0);
            std::memcpy(t + k0, digits, (size_t)cnt);
        }
    }
    return TL_OK;
}

}  // extern "C"

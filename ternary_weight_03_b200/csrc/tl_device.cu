// tl_device.cu -- device entry points of libternary: argument validation,
// kernel selection and launch for tl_gemv / tl_gemm, and the device error
// word behind tl_device_status.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "tl.h"
#include "tl_common.cuh"
#include "tl_gemv.cuh"
#include "tl_gemm.cuh"
#include "tl_gemv3.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return TL_ERR_CUDA;
}

// Per-device facts queried once: SM count and the GEMV kernels' occupancy
// (resident CTAs per SM) for every warps-per-CTA choice.
struct DeviceInfo {
    int num_sms = 0;
    int occ[2][tlk::kGemvMaxWarps + 1] = {};
};

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::once_flag g_device_once[kMaxDevices];
bool g_device_ok[kMaxDevices];

const DeviceInfo *device_info() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cuda_fail(e);
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_device_once[dev], [dev] {
        DeviceInfo &d = g_devices[dev];
        bool ok = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) ==
                  cudaSuccess;
        for (int w = 1; w <= tlk::kGemvMaxWarps && ok; ++w) {
            ok = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ[0][w], tlk::gemv_kernel<2>,
                                                               32 * w, 0) == cudaSuccess &&
                 cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ[1][w], tlk::gemv_kernel<16>,
                                                               32 * w, 0) == cudaSuccess;
        }
        g_device_ok[dev] = ok;
    });
    if (!g_device_ok[dev]) {
        cuda_fail(cudaGetLastError());
        return nullptr;
    }
    return &g_devices[dev];
}

int gemv_occupancy(int fmt, int warps) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    return g_devices[dev].occ[fmt == TL_FMT_2BIT ? 0 : 1][warps];
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Shared argument rules of tl_gemv / tl_gemm.
int check_layer_args(int fmt, const uint8_t *dT, int64_t ldp, const uint16_t *dX, int64_t ldx,
                     uint16_t *dY, int64_t ldy, int64_t N, int64_t K) {
    if (fmt != TL_FMT_2BIT && fmt != TL_FMT_1P6BIT) return TL_ERR_INVALID_ARG;
    if (!dT || !dX || !dY) return TL_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || N > INT32_MAX - 64 || K > INT32_MAX - 512) return TL_ERR_INVALID_ARG;
    const int64_t rb = tl_packed_row_bytes(fmt, K);
    if (ldp < rb || ldx < K || ldy < N) return TL_ERR_INVALID_ARG;
    if (!aligned16(dT) || !aligned16(dX) || !aligned16(dY)) return TL_ERR_ALIGN;
    if (ldp % 16 != 0 || ldx % 8 != 0 || ldy % 8 != 0) return TL_ERR_ALIGN;
    return TL_OK;
}

}  // namespace

extern "C" {

int tl_last_cuda_error(void) { return t_last_cuda_error; }

int tl_gemv_ex(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
               int64_t ldx, uint16_t *dY, int64_t ldy, int M, int64_t N, int64_t K,
               unsigned int flags, void *stream) {
    if (M < 1 || M > TL_GEMV_MAX_M) return TL_ERR_INVALID_ARG;
    if (flags & ~(unsigned int)TL_FLAG_PDL) return TL_ERR_INVALID_ARG;
    int rc = check_layer_args(fmt, dT, ldp, dX, ldx, dY, ldy, N, K);
    if (rc != TL_OK) return rc;
    const DeviceInfo *dev = device_info();
    if (!dev) return TL_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const bool pdl = (flags & TL_FLAG_PDL) != 0;
    if (fmt == TL_FMT_2BIT && tlk::gemv3_supported<2>((int)K))
        return tlk::launch_gemv3<2>(dT, ldp, alpha, dX, ldx, dY, ldy, M, (int)N, (int)K,
                                    dev->num_sms, pdl, s, &t_last_cuda_error);
    if (fmt == TL_FMT_1P6BIT && tlk::gemv3_supported<16>((int)K))
        return tlk::launch_gemv3<16>(dT, ldp, alpha, dX, ldx, dY, ldy, M, (int)N, (int)K,
                                     dev->num_sms, pdl, s, &t_last_cuda_error);
    // K beyond what one cluster can stage: the register-streaming kernel
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cfg.stream = s;
    cudaError_t e;
    if (fmt == TL_FMT_2BIT) {
        const tlk::GemvShape sh = tlk::gemv_shape<2>((int)N, (int)K, dev->num_sms, gemv_occupancy);
        cfg.gridDim = dim3((unsigned)sh.grid);
        cfg.blockDim = dim3((unsigned)(32 * sh.warps));
        e = cudaLaunchKernelEx(&cfg, tlk::gemv_kernel<2>, dT, ldp, alpha, dX, ldx, dY, ldy, M,
                               (int)N, (int)K, sh.tiles_per_cta);
    } else {
        const tlk::GemvShape sh = tlk::gemv_shape<16>((int)N, (int)K, dev->num_sms, gemv_occupancy);
        cfg.gridDim = dim3((unsigned)sh.grid);
        cfg.blockDim = dim3((unsigned)(32 * sh.warps));
        e = cudaLaunchKernelEx(&cfg, tlk::gemv_kernel<16>, dT, ldp, alpha, dX, ldx, dY, ldy, M,
                               (int)N, (int)K, sh.tiles_per_cta);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return TL_OK;
}

int tl_gemv(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
            int64_t ldx, uint16_t *dY, int64_t ldy, int M, int64_t N, int64_t K, void *stream) {
    return tl_gemv_ex(fmt, dT, ldp, alpha, dX, ldx, dY, ldy, M, N, K, 0u, stream);
}

int tl_gemm(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
            int64_t ldx, uint16_t *dY, int64_t ldy, int M, int64_t N, int64_t K, void *stream) {
    if (M < TL_GEMM_MIN_M) return TL_ERR_INVALID_ARG;
    int rc = check_layer_args(fmt, dT, ldp, dX, ldx, dY, ldy, N, K);
    if (rc != TL_OK) return rc;
    return tlk::launch_gemm(fmt, dT, ldp, alpha, dX, ldx, dY, ldy, M, (int)N, (int)K,
                            (cudaStream_t)stream, &t_last_cuda_error);
}

int tl_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int word = 0;
    e = cudaMemcpyFromSymbol(&word, tlk::g_error_word, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(tlk::g_error_word, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e);
        return TL_ERR_TIMEOUT;
    }
    return TL_OK;
}

}  // extern "C"

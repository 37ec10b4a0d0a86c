// tl_device.cu -- device entry points of libternary: argument validation,
// kernel selection and launch for tl_gemv / tl_gemm / tl_gemv_batch /
// tl_ternarise, and the device error word behind tl_device_status.
#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>
#include <cuda_runtime.h>

#include "tl.h"
#ifdef TL_DEBUG_HOOKS
#include "tl_debug.h"
#endif
#include "tl_common.cuh"
#include "tl_gemv.cuh"
#include "tl_gemm.cuh"
#include "tl_gemv3.cuh"
#include "tl_decode.cuh"
#include "tl_ternarise.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

// Workspace of tl_gemv_batch_plan_static: one fixed array per device, part of
// the library's device image (no allocation call ever creates it).
__device__ __align__(256) uint8_t g_static_workspace[TL_STATIC_WORKSPACE_BYTES];

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

// Per device: the number of the latest static plan (0: none yet).  A static
// plan whose number is older describes a table that has been overwritten.
std::atomic<uint64_t> g_static_generation[kMaxDevices];

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

// Validates a batch and converts it into the persistent kernel's host layers.
int batch_layers(int fmt, int count, const tl_gemv_layer *layers, tlk::DkHostLayer *out) {
    if (fmt != TL_FMT_2BIT && fmt != TL_FMT_1P6BIT) return TL_ERR_INVALID_ARG;
    if (count < 1 || count > TL_GEMV_BATCH_MAX || !layers) return TL_ERR_INVALID_ARG;
    int64_t items = 0;
    for (int l = 0; l < count; ++l) {
        const tl_gemv_layer &a = layers[l];
        if (a.M < 1 || a.M > TL_GEMV_MAX_M) return TL_ERR_INVALID_ARG;
        constexpr unsigned int kFlags = TL_LAYER_READS_EARLIER | TL_LAYER_SWIGLU_INPUT;
        if (a.flags & ~kFlags) return TL_ERR_INVALID_ARG;
        if (l == 0 && (a.flags & TL_LAYER_READS_EARLIER)) return TL_ERR_INVALID_ARG;
        const bool swiglu = (a.flags & TL_LAYER_SWIGLU_INPUT) != 0;
        if (swiglu && !(a.flags & TL_LAYER_READS_EARLIER)) return TL_ERR_INVALID_ARG;
        int rc = check_layer_args(fmt, a.dT, a.ldp, a.dX, a.ldx, a.dY, a.ldy, a.N, a.K);
        if (rc != TL_OK) return rc;
        if (swiglu) {
            // X rows hold [gate | up]: 2K elements, the up half 16-byte aligned
            if (a.ldx < 2 * a.K) return TL_ERR_INVALID_ARG;
            if (a.K % 8 != 0) return TL_ERR_ALIGN;
        }
        if (a.ldx > INT32_MAX || a.ldy > INT32_MAX) return TL_ERR_INVALID_ARG;
        const int64_t stages = (tl_packed_row_bytes(fmt, a.K) + tlk::kDkStageW - 1) / tlk::kDkStageW;
        items += ((a.N + tlk::kDkRows - 1) / tlk::kDkRows) * stages;  // upper bound
        if (items > INT32_MAX / 2) return TL_ERR_INVALID_ARG;
        out[l] = tlk::DkHostLayer{a.dT, a.dX, a.dY, a.ldp, a.ldx, a.ldy, a.alpha, a.M, (int)a.N,
                                  (int)a.K, (a.flags & TL_LAYER_READS_EARLIER) != 0, swiglu};
    }
    return TL_OK;
}

// tl_gemv_batch_plan (tl_decode.cuh): layer table, tensor maps and zeroed
// counters written into the workspace.
int plan_decode2(int fmt, int count, const std::vector<tlk::DkHostLayer> &dh, void *dWorkspace,
                 size_t workspace_bytes, tl_gemv_plan *plan) {
    uint8_t *ws = reinterpret_cast<uint8_t *>(dWorkspace);
    std::vector<tlk::DkItemRec> items;
    std::vector<tlk::DkUnitRec> units;
    const tlk::DkSchedule sc = tlk::dk_schedule(fmt, count, dh.data(), ws, &items, &units);
    if (sc.bytes > workspace_bytes) return TL_ERR_INVALID_ARG;
    std::vector<CUtensorMap> maps(count);
    for (int l = 0; l < count; ++l)
        if (!tlk::dk_encode_map(fmt, dh[l], &maps[l])) return TL_ERR_CUDA;
    if (!device_info()) return TL_ERR_CUDA;
    const tlk::DkWsLayout wl(count, sc.total_items, sc.total_units, sc.total_tiles, sc.slots,
                             sc.staged);
    cudaError_t e = cudaMemset(ws, 0, wl.maps);  // counters
    if (e == cudaSuccess)
        e = cudaMemcpy(ws + wl.maps, maps.data(), sizeof(CUtensorMap) * count,
                       cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(ws + wl.items, items.data(), sizeof(tlk::DkItemRec) * items.size(),
                       cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !units.empty())
        e = cudaMemcpy(ws + wl.units, units.data(), sizeof(tlk::DkUnitRec) * units.size(),
                       cudaMemcpyHostToDevice);
    // ready, per-layer final tiles, per-layer tile counts, tile counters
    if (e == cudaSuccess) e = cudaMemset(ws + wl.ready, 0, wl.partials - wl.ready);
    std::vector<uint32_t> ltiles(count);
    for (int l = 0; l < count; ++l) ltiles[l] = (uint32_t)((dh[l].N + tlk::kDkRows - 1) / tlk::kDkRows);
    if (e == cudaSuccess)
        e = cudaMemcpy(ws + wl.ready + 8 * (size_t)count, ltiles.data(), 4 * (size_t)count,
                       cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
    plan->fmt = fmt;
    plan->count = count;
    plan->max_m = sc.maxM;
    plan->total_items = sc.total_items;
    plan->total_tiles = sc.total_tiles;
    plan->total_units = sc.total_units;
    plan->chained = sc.chained;
    plan->dWorkspace = dWorkspace;
    plan->workspace_bytes = workspace_bytes;
    plan->generation = 0;
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
    if (e != cudaSuccess) (void)cudaGetLastError();  // the error is returned here, once
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

int tl_ternarise(int fmt, const uint16_t *dW, int64_t ldw, int64_t N, int64_t K, uint8_t *dP,
                 int64_t ldp, float *dAlpha, void *dWorkspace, void *stream) {
    if (fmt != TL_FMT_2BIT && fmt != TL_FMT_1P6BIT) return TL_ERR_INVALID_ARG;
    if (!dW || !dP || !dAlpha || !dWorkspace) return TL_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || N > INT32_MAX || K > INT32_MAX - 512) return TL_ERR_INVALID_ARG;
    if (ldw < K || ldp < tl_packed_row_bytes(fmt, K) || ldp > INT32_MAX) return TL_ERR_INVALID_ARG;
    if (!aligned16(dW) || !aligned16(dP) || !aligned16(dWorkspace) || ((uintptr_t)dAlpha & 3u))
        return TL_ERR_ALIGN;
    if (ldw % 8 != 0 || ldp % 16 != 0) return TL_ERR_ALIGN;
    const DeviceInfo *dev = device_info();
    if (!dev) return TL_ERR_CUDA;
    return tlk::launch_ternarise(fmt, dW, ldw, (int)N, (int)K, dP, ldp, dAlpha, dWorkspace,
                                 dev->num_sms, (cudaStream_t)stream, &t_last_cuda_error);
}

int tl_gemv_batch_bytes(int fmt, int count, const tl_gemv_layer *layers, size_t *bytes) {
    if (!bytes) return TL_ERR_INVALID_ARG;
    std::vector<tlk::DkHostLayer> h(count > 0 && count <= TL_GEMV_BATCH_MAX ? count : 0);
    int rc = batch_layers(fmt, count, layers, h.data());
    if (rc != TL_OK) return rc;
    *bytes = tlk::dk_schedule(fmt, count, h.data(), nullptr, nullptr, nullptr).bytes;
    return TL_OK;
}

int tl_gemv_batch_plan(int fmt, int count, const tl_gemv_layer *layers, void *dWorkspace,
                       size_t workspace_bytes, tl_gemv_plan *plan) {
    if (!plan || !dWorkspace) return TL_ERR_INVALID_ARG;
    if (((uintptr_t)dWorkspace & 255u) != 0) return TL_ERR_ALIGN;
    std::vector<tlk::DkHostLayer> h(count > 0 && count <= TL_GEMV_BATCH_MAX ? count : 0);
    int rc = batch_layers(fmt, count, layers, h.data());
    if (rc != TL_OK) return rc;
    return plan_decode2(fmt, count, h, dWorkspace, workspace_bytes, plan);
}

int tl_gemv_batch_plan_static(int fmt, int count, const tl_gemv_layer *layers,
                              tl_gemv_plan *plan) {
    if (!plan) return TL_ERR_INVALID_ARG;
    size_t need = 0;
    int rc = tl_gemv_batch_bytes(fmt, count, layers, &need);
    if (rc != TL_OK) return rc;
    if (need > (size_t)TL_STATIC_WORKSPACE_BYTES) return TL_ERR_INVALID_ARG;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return TL_ERR_INVALID_ARG;
    void *addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_static_workspace);  // this device's copy
    if (e != cudaSuccess) return cuda_fail(e);
    // no run of an earlier static plan may still be reading the array
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
    // every earlier static plan of this device is stale from here on, even if
    // the rewrite below fails half way
    const uint64_t gen = g_static_generation[dev].fetch_add(1) + 1;
    rc = tl_gemv_batch_plan(fmt, count, layers, addr, (size_t)TL_STATIC_WORKSPACE_BYTES, plan);
    if (rc != TL_OK) return rc;
    plan->generation = gen;
    return TL_OK;
}

int tl_gemv_batch_run(const tl_gemv_plan *plan, unsigned int flags, void *stream) {
    if (!plan || !plan->dWorkspace) return TL_ERR_INVALID_ARG;
#ifdef TL_DEBUG_HOOKS
    constexpr unsigned int kRunFlags = TL_FLAG_PDL | TL_FLAG_DEBUG_DROP_ARRIVE;
#else
    constexpr unsigned int kRunFlags = TL_FLAG_PDL;
#endif
    if (flags & ~kRunFlags) return TL_ERR_INVALID_ARG;
    if (plan->fmt != TL_FMT_2BIT && plan->fmt != TL_FMT_1P6BIT) return TL_ERR_INVALID_ARG;
    if (plan->count < 1 || plan->count > TL_GEMV_BATCH_MAX || plan->max_m < 1 ||
        plan->max_m > TL_GEMV_MAX_M || plan->total_items < 1 || plan->total_tiles < 1 ||
        plan->total_units < 0 || plan->chained < 0 || plan->chained > 2)
        return TL_ERR_INVALID_ARG;
    const DeviceInfo *dev = device_info();
    if (!dev) return TL_ERR_CUDA;
    if (plan->generation != 0) {
        // a static plan: only the device's latest, on the device that planned it
        int d = 0;
        cudaError_t e = cudaGetDevice(&d);
        if (e != cudaSuccess) return cuda_fail(e);
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_static_workspace);
        if (e != cudaSuccess) return cuda_fail(e);
        if (plan->dWorkspace != addr || plan->generation != g_static_generation[d].load())
            return TL_ERR_INVALID_ARG;
    }
    const bool pdl = (flags & TL_FLAG_PDL) != 0;
    tlk::DkArgs da = tlk::dk_args(plan->dWorkspace, plan->count, plan->total_items,
                                  plan->total_units, plan->total_tiles, plan->max_m, plan->chained);
    da.drop_arrive = (flags & TL_FLAG_DEBUG_DROP_ARRIVE) ? 1 : 0;
    return plan->fmt == TL_FMT_2BIT
               ? tlk::launch_decode2<2>(da, dev->num_sms, pdl, (cudaStream_t)stream,
                                        &t_last_cuda_error)
               : tlk::launch_decode2<16>(da, dev->num_sms, pdl, (cudaStream_t)stream,
                                         &t_last_cuda_error);
}

#ifdef TL_DEBUG_HOOKS
int tl_debug_batch_items(int fmt, int count, const tl_gemv_layer *layers, void *items,
                         size_t items_bytes, int *n_items) {
    static_assert(sizeof(tlk::DkItemRec) == TL_DEBUG_ITEM_BYTES, "record size");
    if (!n_items || (!items && items_bytes > 0)) return TL_ERR_INVALID_ARG;
    std::vector<tlk::DkHostLayer> h(count > 0 && count <= TL_GEMV_BATCH_MAX ? count : 0);
    int rc = batch_layers(fmt, count, layers, h.data());
    if (rc != TL_OK) return rc;
    // a workspace base that is never dereferenced: the table only holds addresses
    uint8_t *ws = reinterpret_cast<uint8_t *>((uintptr_t)1 << 40);
    std::vector<tlk::DkItemRec> recs;
    std::vector<tlk::DkUnitRec> units;
    tlk::dk_schedule(fmt, count, h.data(), ws, &recs, &units);
    const size_t n = std::min(recs.size(), items_bytes / sizeof(tlk::DkItemRec));
    if (n) std::memcpy(items, recs.data(), n * sizeof(tlk::DkItemRec));
    *n_items = (int)recs.size();
    return TL_OK;
}
#endif

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

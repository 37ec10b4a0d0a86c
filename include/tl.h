/*
 * tl.h -- C ABI of libternary: the ternary linear layer y = alpha * (T x) on
 * one NVIDIA B200 (sm_100a), with T in {-1, 0, 1} packed losslessly at
 * 2 bits (4 trits per byte) or 1.6 bits (5 trits per byte).
 *
 * Defining passages ("Pith review of Spectra 1.1: Scaling Laws and
 * Efficient Inference for Ternary Language Models", pith.science):
 *   - "What carries the argument": a ternary linear layer is a linear layer
 *     whose weight matrix is restricted to {-1,0,1} times one shared
 *     floating-point scale; k trits fit p bits when 2^p > 3^k, so 5 trits
 *     fit one byte (1.6 bits per weight).
 *   - "Core claim": lossless packing at 2 bits by a base-4 encoding and at
 *     1.6 bits by a base-3 encoding.
 *   - Referee report, minor comment 5 (paper section 3.2): decoding by
 *     running quotients; the partial final block is left open.
 *
 * Conventions fixed by this library where the pages are silent:
 *   - Trit t is stored as digit d = t + 1 (so -1 -> 0, 0 -> 1, +1 -> 2).
 *   - T is N x K (output rows x reduction).  Row n of T is packed into row n
 *     of P, row stride ldp bytes.  Trit k of a row is digit (k mod g) of byte
 *     floor(k / g), g = 4 (2-bit) or 5 (1.6-bit); digit i has weight b^i,
 *     b = 4 or 3 (least-significant digit first).
 *     2-bit:   byte = d0 + 4 d1 + 16 d2 + 64 d3  (a field value 3 is invalid)
 *     1.6-bit: byte = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4  (bytes >= 243 invalid)
 *   - A partial last byte is completed with 0-trits (digit 1).  Bytes in
 *     [row_bytes, ldp) are written as 0 by the packers and never interpreted.
 *   - X is M x K, Y is M x N, both IEEE binary16 (passed as uint16_t bit
 *     patterns), row-major with row strides ldx / ldy elements:
 *     Y[m][n] = fp16_rn(alpha * sum_k T[n][k] * X[m][k]), the sum taken in
 *     fp32 (products are exact; the order of the additions is unspecified).
 *
 * All functions return a status code (TL_OK = 0) and never throw.  They
 * keep no state between calls except a per-device error word set by the
 * kernels' bounded waits (see tl_device_status) and lazily created
 * per-device launch parameters; they are safe to call concurrently from
 * several host threads on different streams.
 */
#ifndef TERNARY_TL_H
#define TERNARY_TL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TL_FMT_2BIT 2    /* 4 trits per byte, base 4 */
#define TL_FMT_1P6BIT 16 /* 5 trits per byte, base 3 */

#define TL_GEMV_MAX_M 8   /* tl_gemv: 1 <= M <= 8 */
#define TL_GEMM_MIN_M 16  /* tl_gemm: M >= 16 */

enum tl_status {
    TL_OK = 0,
    TL_ERR_INVALID_ARG = 1, /* null pointer, size out of range, bad format, bad stride */
    TL_ERR_BAD_TRIT = 2,    /* a trit outside {-1, 0, 1} given to a packer */
    TL_ERR_BAD_CODE = 3,    /* a byte that is not a valid code given to tl_unpack */
    TL_ERR_ALIGN = 4,       /* a device pointer or stride breaks the alignment rules */
    TL_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
    TL_ERR_TIMEOUT = 6,     /* a kernel's bounded wait ran out (see tl_device_status) */
    TL_ERR_UNSUPPORTED = 7  /* reserved: no kernel for a (format, shape); no call returns it now */
};

/* Static, human-readable name of a status code (never NULL). */
const char *tl_status_str(int status);

/* The CUDA error code (cudaError_t value) behind the last TL_ERR_CUDA
 * returned on the calling host thread, or 0. */
int tl_last_cuda_error(void);

/* Bytes per packed row: ceil(K / 4) for TL_FMT_2BIT, ceil(K / 5) for
 * TL_FMT_1P6BIT.  Returns -1 for an unknown format or K < 0.  Pure. */
int64_t tl_packed_row_bytes(int fmt, int64_t K);

/* Pack int8 trits T[N][ldt] (host memory) into P[N][ldp] (host memory) at
 * 2 bits per trit ("Core claim": base-4 encoding).  Requires ldt >= K and
 * ldp >= tl_packed_row_bytes(TL_FMT_2BIT, K); P must hold N * ldp bytes and
 * may not overlap T.  Every trit must be -1, 0 or 1, else TL_ERR_BAD_TRIT
 * and P is left unspecified.  The caller owns both buffers; nothing is
 * allocated.  N == 0 or K == 0 is valid (pads only). */
int tl_pack2(const int8_t *T, int64_t N, int64_t K, int64_t ldt, uint8_t *P, int64_t ldp);

/* The same at 1.6 bits per trit ("What carries the argument": 5 trits in
 * one byte, base 3, valid since 3^5 = 243 <= 2^8).  ldp >=
 * tl_packed_row_bytes(TL_FMT_1P6BIT, K). */
int tl_pack16(const int8_t *T, int64_t N, int64_t K, int64_t ldt, uint8_t *P, int64_t ldp);

/* Unpack P[N][ldp] (host) into int8 trits T[N][ldt] (host), the map U of
 * the packing theorem (U(P(t)) = t, "Circularity Check").  Every byte in
 * [0, row_bytes) of every row is validated: a 2-bit byte with a field equal
 * to 3, or a 1.6-bit byte >= 243, returns TL_ERR_BAD_CODE and, when
 * bad_index is not NULL, stores the offset n * ldp + j of the first such
 * byte in row-major order (T is then partly written).  Digits of the last
 * byte beyond K and bytes past row_bytes are not returned. */
int tl_unpack(int fmt, const uint8_t *P, int64_t N, int64_t K, int64_t ldp, int8_t *T,
              int64_t ldt, int64_t *bad_index);

/* Decode-shaped layer, 1 <= M <= TL_GEMV_MAX_M:
 *   Y[m][n] = fp16_rn(alpha * sum_k T[n][k] X[m][k]),  m < M, n < N.
 * dT: packed T on the device, N rows of ldp bytes, format fmt.
 * dX: binary16 activations on the device, M rows of ldx elements.
 * dY: binary16 outputs on the device, M rows of ldy elements; every
 *     element m < M, n < N is overwritten (no accumulation into Y).
 * alpha: the layer's shared scale ("What carries the argument").
 * stream: a cudaStream_t (NULL = the legacy default stream).
 * Rules: dT, dX, dY 16-byte aligned; ldp % 16 == 0 and ldp >= row bytes;
 * ldx % 8 == 0, ldx >= K; ldy % 8 == 0, ldy >= N; N >= 1, K >= 1 (else
 * TL_ERR_INVALID_ARG / TL_ERR_ALIGN before anything is enqueued).  The
 * kernels read only [0, ldp) of each packed row, X[m][0..ldx) and write
 * only Y[m][0..N).  The call is asynchronous and stream-ordered: it returns
 * once the work is enqueued, allocates nothing and does not synchronize.
 * Codes are not validated on the device: an invalid byte yields an
 * unspecified (but finite-time, in-bounds) result.  The buffers are the
 * caller's and must stay valid until the stream reaches this work. */
int tl_gemv(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
            int64_t ldx, uint16_t *dY, int64_t ldy, int M, int64_t N, int64_t K, void *stream);

/* Flags of tl_gemv_ex. */
#define TL_FLAG_PDL 1u /* programmatic dependent launch, see tl_gemv_ex */

/* tl_gemv with launch flags (tl_gemv is tl_gemv_ex with flags = 0).
 * TL_FLAG_PDL: the kernel is launched with programmatic stream
 * serialization, so it may begin while the preceding kernel on `stream` is
 * still running.  Before it waits for that kernel it only streams the packed
 * weights dT; it reads X and writes Y after the preceding work has completed
 * and its memory is visible.  The caller therefore promises that dT is not
 * written by any work still in flight on the stream (true of static layer
 * weights).  Works inside CUDA-graph capture.  Other flag bits:
 * TL_ERR_INVALID_ARG. */
int tl_gemv_ex(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
               int64_t ldx, uint16_t *dY, int64_t ldy, int M, int64_t N, int64_t K,
               unsigned int flags, void *stream);

/* ---- a batch of decode-shaped layers in one launch ---------------------- */

#define TL_GEMV_BATCH_MAX 4096    /* layers per batch */
#define TL_LAYER_READS_EARLIER 1u /* tl_gemv_layer.flags, see tl_gemv_batch_plan */
#define TL_LAYER_SWIGLU_INPUT 2u  /* tl_gemv_layer.flags, see tl_gemv_batch_plan */

/* One layer of a batch: the arguments of tl_gemv for that layer. */
typedef struct tl_gemv_layer {
    const uint8_t *dT;   /* packed T, N rows of ldp bytes (device) */
    int64_t ldp;
    float alpha;
    const uint16_t *dX;  /* M x K binary16 activations, row stride ldx (device) */
    int64_t ldx;
    uint16_t *dY;        /* M x N binary16 outputs, row stride ldy (device) */
    int64_t ldy;
    int M;               /* 1 .. TL_GEMV_MAX_M */
    int64_t N, K;
    unsigned int flags;  /* 0, TL_LAYER_READS_EARLIER, or that | TL_LAYER_SWIGLU_INPUT */
} tl_gemv_layer;

/* A planned batch: filled by tl_gemv_batch_plan, read by tl_gemv_batch_run.
 * Plain data owned by the caller; treat the fields as read-only. */
typedef struct tl_gemv_plan {
    int fmt, count, max_m, total_items, total_tiles;
    int total_units;  /* activation conversion units of the launch */
    int chained;      /* 1 if some layer has TL_LAYER_READS_EARLIER, 2 if one
                         also has TL_LAYER_SWIGLU_INPUT, else 0 */
    void *dWorkspace;
    size_t workspace_bytes;
    uint64_t generation; /* 0, or the static plan's number (tl_gemv_batch_plan_static) */
} tl_gemv_plan;

/* Workspace bytes a batch needs: counters (16 bytes per layer), one TMA
 * descriptor per layer, a 112-byte record per work item (256 output rows x a K-part of whole stages;
 * a stage is 128 packed bytes per row, 512 trits at 2 bits or 640 at 1.6
 * bits), the layers' activations converted once into the tensor-core
 * operand layout (per stage 64 B plus 8 B per trit x M at M <= 2, 2 B per
 * trit x M rounded up to even at M >= 3; none for TL_LAYER_READS_EARLIER
 * layers with M <= 2, which convert on chip) with a 48-byte record per stage
 * and token (none for TL_LAYER_READS_EARLIER layers),
 * and 8-byte partial sums of rows split into K-parts (N * M * 8 bytes per
 * part).  Validates the batch like tl_gemv_batch_plan.  Pure host
 * function. */
int tl_gemv_batch_bytes(int fmt, int count, const tl_gemv_layer *layers, size_t *bytes);

/* Plans count (1 .. TL_GEMV_BATCH_MAX) decode-shaped layers of one format (2-
 * or 1.6-bit, both run by the same persistent kernel)
 * for single-launch execution by tl_gemv_batch_run.  Every layer follows the
 * argument rules of tl_gemv; layers[] is host memory, read before the call
 * returns.  Writes the layer table and the layers' TMA descriptors into
 * dWorkspace (device memory of at least tl_gemv_batch_bytes() bytes,
 * 256-byte aligned, owned by the caller) and zeroes its counters, with
 * blocking copies: the call synchronizes the device and may not be captured
 * into a CUDA graph.  Plan once, run many times; the plan holds the
 * pointers of T, X and Y, so a batch on other buffers needs a new plan.
 * Dependencies: a layer with TL_LAYER_READS_EARLIER (not allowed on layer
 * 0) may consume the outputs of earlier layers of the batch: it reads its X
 * only after every earlier layer whose Y overlaps that X (rows m < M of K
 * elements at stride ldx, 2K with the SwiGLU input; compared by address) has
 * stored all of its Y.  Layers it does not read from run concurrently with
 * it, so independent chains (one per decoder block, say) overlap.  Without
 * the flag, X must not be written by any layer of the batch.  No Y may
 * overlap another layer's Y or T, nor the X of an earlier layer.
 * SwiGLU input (TL_LAYER_SWIGLU_INPUT together with
 * TL_LAYER_READS_EARLIER): row m of dX holds a gated unit's two inputs, the
 * gate values g in elements [0, K) and the up values u in [K, 2K) (typically
 * the outputs of two earlier layers writing the halves of one buffer), and
 * the layer's input is x_k = fp16_rn(silu(g_k) * u_k), silu(g) = g / (1 +
 * exp(-g)), evaluated in fp32 -- the gated feed-forward unit of a LLaMA-style
 * decoder fused into its down projection, so the product never goes to
 * memory.  Needs ldx >= 2 K and K % 8 == 0 (else TL_ERR_INVALID_ARG /
 * TL_ERR_ALIGN).
 * Independent layers with the same X (pointer, ldx, K and M; no
 * TL_LAYER_READS_EARLIER), such as the Q, K and V projections of one token
 * batch, share one conversion of X: it is staged once per launch, and each
 * layer keeps its own alpha.
 * Errors: TL_ERR_INVALID_ARG (bad layer, count or workspace too small),
 * TL_ERR_ALIGN, TL_ERR_CUDA. */
int tl_gemv_batch_plan(int fmt, int count, const tl_gemv_layer *layers, void *dWorkspace,
                       size_t workspace_bytes, tl_gemv_plan *plan);

/* Bytes of the library's own per-device workspace (see
 * tl_gemv_batch_plan_static). */
#define TL_STATIC_WORKSPACE_BYTES (16u << 20)

/* tl_gemv_batch_plan without caller memory: the workspace is a fixed array of
 * TL_STATIC_WORKSPACE_BYTES bytes inside the library's device code, one per
 * device, located with cudaGetSymbolAddress on the current device.  Nothing
 * is allocated.  A batch whose tl_gemv_batch_bytes exceeds
 * TL_STATIC_WORKSPACE_BYTES is rejected with TL_ERR_INVALID_ARG before
 * anything is written.  Races: the array is shared by every caller in the
 * process on that device, so planning again replaces the previous static
 * plan.  Each static plan carries a per-device number (plan->generation);
 * the call takes a new number before it writes the array, and
 * tl_gemv_batch_run returns TL_ERR_INVALID_ARG, without launching, for a
 * static plan whose number is no longer the device's latest (or that was
 * planned on another device): plan again instead.  Do not plan from several
 * host threads at once.  The call synchronizes the device first, so no run
 * of an earlier static plan is still reading the array when it is rewritten.
 * Clearing: the call zeroes the array's counters; every completed
 * tl_gemv_batch_run leaves them zero; after a run that ends in
 * TL_ERR_TIMEOUT, plan again before the next run.  Otherwise as
 * tl_gemv_batch_plan (blocking, not capturable). */
int tl_gemv_batch_plan_static(int fmt, int count, const tl_gemv_layer *layers,
                              tl_gemv_plan *plan);

/* Runs a planned batch in ONE persistent launch: every layer computes
 * exactly what tl_gemv computes.  The launch streams the packed weights of
 * all layers back to back ("What carries the argument": decoding is bound by
 * memory bandwidth), splitting long rows across CTAs; split rows are summed
 * in a fixed order, so results are deterministic.  Each launch that
 * completes leaves the workspace counters at zero, so the plan can be run
 * again without clearing; after a launch that ends in TL_ERR_TIMEOUT
 * (tl_device_status) plan again.  Launches of one plan (one workspace) must
 * be ordered on one stream.  flags: 0 or TL_FLAG_PDL (as for tl_gemv_ex:
 * the first weights are fetched while the preceding kernel finishes; X, Y
 * and the workspace counters are touched only after it completed).
 * Asynchronous, allocates nothing, may be captured into a CUDA graph.
 * Errors: TL_ERR_INVALID_ARG (plan not filled by tl_gemv_batch_plan, a
 * static plan replaced by a later tl_gemv_batch_plan_static, bad flags),
 * TL_ERR_CUDA. */
int tl_gemv_batch_run(const tl_gemv_plan *plan, unsigned int flags, void *stream);

/* Failure-detection hook of tl_gemv_batch_run, honoured only by the debug
 * library (libternary_debug.so, the same sources compiled with
 * TL_DEBUG_HOOKS); the product library rejects the bit with
 * TL_ERR_INVALID_ARG.  With it, the 2-bit batch kernel's CTA 0 leaves out
 * the shared-memory barrier arrival that publishes its first operand stage
 * converted on chip (a batch whose first item has M <= 2).  Its consumers'
 * bounded wait then runs out: every warp of the launch gives up its work
 * within the wait limit (1 s), the CTA waits for its own copies in flight
 * and exits, and tl_device_status returns TL_ERR_TIMEOUT.  No hardware
 * completion is ever skipped. */
#define TL_FLAG_DEBUG_DROP_ARRIVE 0x80000000u

/* Batched / prefill-shaped layer, M >= TL_GEMM_MIN_M, same arguments and
 * rules as tl_gemv, both formats ("Pith review of Spectra 1.1", "What carries
 * the argument": an FP16 x INT2 tensor-core kernel with fused dequantisation;
 * the 1.6-bit packing of "Core claim" goes through the same kernel).  Packed
 * tiles are expanded on chip to exact fp16 -1 / 0 / +1 and multiplied with
 * tcgen05 MMAs accumulating in fp32.  For a given format and shape the
 * summation order is fixed, so repeated calls agree bit for bit. */
int tl_gemm(int fmt, const uint8_t *dT, int64_t ldp, float alpha, const uint16_t *dX,
            int64_t ldx, uint16_t *dY, int64_t ldy, int M, int64_t N, int64_t K, void *stream);

/* Device ternariser + packer: fp16 weights W [N][ldw] -> the shared scale
 * *dAlpha and the packed trits P [N][ldp] (format fmt), the step before the
 * layer: its weights are {-1, 0, 1} times one shared floating-point scale,
 * obtained by rounding to the nearest ternary value ("Pith review of
 * Spectra 1.1", "What carries the argument", and the round-to-nearest
 * quantisation named among its domain assumptions).  The pages give no
 * scale formula; this library takes
 *   alpha = mean |W| over all N K entries: the sum of |w| is exact (integer
 *           multiples of 2^-24), then alpha = fp32_rn(fp64_rn(fp64_rn(S) /
 *           (N K)) * 2^-24), independent of the summation order;
 *   t     = +1 if w > alpha / 2, -1 if w < -alpha / 2, else 0 (the nearest
 *           ternary value to w / alpha in fp32, ties to 0; all-zero W gives
 *           alpha = 0 and T = 0);
 * and packs T exactly as tl_pack2 / tl_pack16 do (pad trits 0, bytes from
 * the row's end to ldp written as 0).  W must be finite (NaN / Inf give
 * unspecified T and alpha, never a fault).
 * Device pointers, caller-owned: dW (16-byte aligned, ldw >= K, ldw % 8 ==
 * 0), dP (16-byte aligned, tl_packed_row_bytes <= ldp <= INT32_MAX,
 * ldp % 16 == 0; must not overlap dW), dAlpha (one float, 4-byte aligned),
 * dWorkspace
 * (TL_TERNARISE_WORKSPACE_BYTES, 16-byte aligned, contents need no
 * clearing; calls sharing it must be ordered on one stream).  Three
 * stream-ordered launches, asynchronous, no allocation, may be captured
 * into a CUDA graph.  Errors: TL_ERR_INVALID_ARG (format, null pointer,
 * sizes), TL_ERR_ALIGN, TL_ERR_CUDA. */
#define TL_TERNARISE_WORKSPACE_BYTES 16384u
int tl_ternarise(int fmt, const uint16_t *dW, int64_t ldw, int64_t N, int64_t K, uint8_t *dP,
                 int64_t ldp, float *dAlpha, void *dWorkspace, void *stream);

/* Synchronizes `stream`, then reads and clears the current device's error
 * word, which kernels set when one of their bounded waits gives up instead
 * of spinning forever.  Returns TL_OK, TL_ERR_TIMEOUT, or TL_ERR_CUDA if
 * the synchronization itself failed. */
int tl_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TERNARY_TL_H */

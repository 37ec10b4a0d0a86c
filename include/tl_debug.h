/* tl_debug.h -- test hooks of libternary_debug.so (the same sources as
 * libternary.so, compiled with TL_DEBUG_HOOKS).  The product library does not
 * export these functions.  They expose internal tables for tests and may
 * change with the kernels. */
#ifndef TL_DEBUG_H
#define TL_DEBUG_H

#include <stddef.h>
#include <stdint.h>
#include "tl.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of one record written by tl_debug_batch_items. */
#define TL_DEBUG_ITEM_BYTES 112

/* The work items tl_gemv_batch_plan would write for this batch, in the order
 * the persistent kernel hands them out, without touching any device: pure host
 * function.  The layers are validated like tl_gemv_batch_plan (same errors);
 * their pointers are only compared, never dereferenced.  Writes
 * min(count of items, items_bytes / TL_DEBUG_ITEM_BYTES) records to items
 * (host memory, caller-owned) and the count of items to *n_items.  Record
 * layout (little-endian, byte offsets): 0 X, 8 Y, 16 converted-operand
 * region (u64 addresses into a workspace based at 2^40), 24 int64 first
 * partial slot, 32 float alpha, then int32 at 36 layer | (converting layer
 * << 16), 40 tile, 44 part, 48 first stage, 52 end stage, 56 M, 60 K, 64 N,
 * 68 ldx, 72 ldy, 76 parts per tile, 80 first tile of the layer, 84
 * dependency range ((lo << 16) | (hi + 1), 0 for none), 88 conversion units,
 * 92 bytes per stage of converted operands, 96 flags (1: SwiGLU input,
 * 2: input converted once per launch by the layer's items), 100..111 unused.
 * A stage is 128 packed bytes of a row (512 trits at 2 bits, 640 at 1.6). */
int tl_debug_batch_items(int fmt, int count, const tl_gemv_layer *layers, void *items,
                         size_t items_bytes, int *n_items);

#ifdef __cplusplus
}
#endif

#endif /* TL_DEBUG_H */

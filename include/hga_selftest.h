/*
 * hga_selftest.h -- hardware self test of libhga.so.
 *
 * The article has no counterpart to this call.  It checks, on the device at
 * hand, the tensor-core operand arrangements that the attention kernels rely
 * on (shared-memory descriptors with 128-byte swizzle in K-major and MN-major
 * form, and the packed-bf16 tensor-memory A operand), by computing one
 * 128 x 128 x 128 bf16 product with fp32 accumulation.
 */
#ifndef HGA_SELFTEST_H
#define HGA_SELFTEST_H

#include "hga.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * form 0: d = a . b^T  (a [M=128][K=128], b [N=128][K=128], both from shared memory)
 * form 1: d = a . b    (a [M][K] from shared memory, b [K][N] MN-major)
 * form 2: d = a . b    (a from tensor memory, b [K][N] MN-major)
 * form 3: d = a . b^T  (a from tensor memory, b [N][K] K-major)
 * a, b: device bf16, row-major, 16-byte aligned; d: device fp32 [128][128]
 * row-major.  Enqueued on `stream`.  Errors: HGA_ERR_INVALID_ARG (null pointer,
 * bad form), HGA_ERR_CUDA.
 */
HGA_API hga_status hga_selftest_umma(int form, const void* a, const void* b, float* d, hga_stream_t stream);

/*
 * Self test of the device-side timeout path (the article has no counterpart).
 * Runs the tensor-core forward of hga_attn_fwd (same arguments; bf16, d = 128,
 * block = 128, even group size, else HGA_ERR_UNSUPPORTED) with its K/V tile
 * loads withheld, so that a pipeline wait can never be satisfied.  Every
 * wait in the kernels is bounded (1 s): the CTA that gives up raises its
 * abort flag, every role leaves its loop, the CTA waits (bounded) for its own
 * copies and tensor-core work in flight, frees its tensor memory and returns.
 * The next hga_device_status() then reports HGA_ERR_TIMEOUT, and the CUDA
 * context stays usable.  o and lse are left unwritten.  Expect about one
 * second of device time per call.
 */
HGA_API hga_status hga_selftest_attn_fwd_stalled(const hga_dims* dims, const void* q, const void* k_seg,
                                                 const void* v_seg, const void* k_hist, const void* v_hist,
                                                 int n_kv_blocks, const int32_t* idx, void* o, float* lse,
                                                 hga_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif

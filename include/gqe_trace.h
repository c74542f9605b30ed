/* gqe_trace.h -- diagnostic entry point of the traced build of the library.
 *
 * `python moe_gqa_query_b200/build.py --trace` builds libgqe_trace.so: the
 * same library, with the d_head = 64 prefill attention kernel (gqe_attn_prefill)
 * recording a timeline of every CTA in a device array.  The normal build
 * (libgqe.so) has no trace and does not export this function.
 */
#ifndef GQE_TRACE_H_
#define GQE_TRACE_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Copies the first `bytes` of the trace array to `host` (synchronous; host
 * memory owned by the caller).  Layout: 12 unsigned 64-bit values per CTA of
 * the last gqe_attn_prefill launch with d_head = 64, indexed by blockIdx.x
 * (the first 16384 CTAs are recorded):
 *   [0]  SM id | key tiles << 16 | routed << 31
 *   [1]  CTA entry, [2] set-up done (barriers, tensor memory, dependent-launch
 *        wait), [3] Q tile arrived, [4] first S tile ready, [5] first P
 *        published, [6] softmax loop done, [7] last P V done, [8] output
 *        written, [9] CTA exit: globaltimer nanoseconds
 *   [10] time the softmax waited for S tiles after the first, [11] time it
 *        waited for P V before overwriting P (nanoseconds, summed).
 * Returns 0, 1 (null host or more bytes than the array), 4 (CUDA error). */
int gqe_debug_attn_trace(void* host, size_t bytes);

#ifdef __cplusplus
}
#endif

#endif  /* GQE_TRACE_H_ */

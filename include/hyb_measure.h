/*
 * hyb_measure.h -- measurement support of the B200 hybrid_v2 KV-cache decode
 * library: a plain streaming read of a device buffer, the reference against
 * which a decode launch's achieved HBM bandwidth is read at the same byte count.
 *
 * Why it exists: web page "DeepSeek V4混合式KV Cache推理优化实战解析", section
 * 2.1, judges a decode backend by the fraction of the memory bandwidth it
 * uses.  At small byte counts (a few tens of MB per decode step) no kernel
 * reaches the copy bandwidth: launch, ramp-up and drain cost a fixed few
 * microseconds.  hyb_stream_read reads the same number of bytes with nothing
 * else in the way -- no block-table lookup, no dependent load, no arithmetic
 * beyond an XOR -- so its time at a given byte count is the attainable floor
 * of any kernel that has to read those bytes once.
 *
 * Same library as hyb_kv.h (libhybkv.so); return codes are those of hyb_kv.h.
 */
#ifndef HYB_MEASURE_H
#define HYB_MEASURE_H

#include <stddef.h>
#include <stdint.h>

#include "hyb_kv.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * hyb_stream_read: read `bytes` bytes of device memory at `src` once, in
 * 16-byte coalesced loads spread over a grid of 8 CTAs of 256 threads per SM,
 * and XOR the XOR of all of its 32-bit words into *sink (device memory).
 *
 *   src     device pointer, 16-byte aligned; not modified; not retained.
 *   bytes   a multiple of 16; 0 launches nothing and checks no pointer.
 *   sink    device pointer to one uint32_t; the caller sets its start value
 *           (zero to get the buffer's XOR); updated with atomic XORs.
 *   stream  the CUDA stream of the launch (NULL: the legacy default stream).
 *
 * Asynchronous: returns after the launch; the result is in *sink once the
 * stream reaches it.  Returns HYB_OK, HYB_ERR_INVALID_VALUE (null pointer,
 * misaligned src or sink, bytes not a multiple of 16) or HYB_ERR_CUDA (the
 * launch failed; hyb_last_cuda_error gives the CUDA error).
 */
int hyb_stream_read(const void *src, size_t bytes, uint32_t *sink, hyb_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HYB_MEASURE_H */

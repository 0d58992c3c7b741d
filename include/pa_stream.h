/*
 * pa_stream.h — measurement helper of the paged-attention library (not part of
 * the decode path): a read-only streaming kernel that gives the HBM read
 * bandwidth this GPU sustains, the reference a read-dominated kernel is
 * compared with next to the copy (read + write) bandwidth.
 *
 * pa_stream_read — read every byte of `src` once and write one 32-bit checksum
 * per CTA to `partial` (device, num_ctas entries). Each of the `num_ctas` CTAs
 * (two fit on an SM) streams 16 KiB chunks c, c + num_ctas, ... through a
 * 6-stage shared-memory ring with bulk asynchronous copies (cp.async.bulk, no
 * multicast), the way the decode kernels read the cache. `bytes` must be a
 * multiple of 16 and `src` 16-byte aligned. Asynchronous on `stream` (a
 * cudaStream_t, NULL = the default stream). Returns 0, -1 on bad arguments,
 * -5 if the launch failed.
 */
#ifndef PA_STREAM_H
#define PA_STREAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int pa_stream_read(const void* src, size_t bytes, uint32_t* partial, int32_t num_ctas,
                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_STREAM_H */

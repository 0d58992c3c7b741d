/*
 * pa_test.h — test hook of the paged-attention library; not for production use.
 *
 * pa_test_skip_load — while `position` >= 0, every following pa_decode call
 * (from any thread) leaves ring position `position` of each CTA's K/V pipeline
 * unloaded. The consumer waiting for that position gives up after its bounded
 * wait (about one second), the producer and the other waiters then give up in
 * turn, the kernel still terminates, its outputs are invalid, and pa_sync_check
 * returns PA_ERR_TIMEOUT; the CUDA context stays usable. -1 restores normal
 * operation. It exists only so that the timeout path can be tested without a
 * fault or a hang.
 *
 * pa_test_last_decode_kernel — which decode kernel the calling thread's last
 * successful pa_decode / pa_decode_grouped / pa_decode_noalloc enqueued:
 * PA_KERNEL_SIMT (CUDA-core consumer), PA_KERNEL_MMA (tensor-core GQA
 * consumer), PA_KERNEL_GROUPED (grouped sequences / multi-token queries),
 * PA_KERNEL_GROUPED_TCGEN05 (the same on the tcgen05 consumer, see
 * pa_set_grouped_consumer), or -1 if none yet. Lets
 * tests confirm which path a shape takes.
 */
#define PA_KERNEL_SIMT 0
#define PA_KERNEL_MMA 1
#define PA_KERNEL_GROUPED 2
#define PA_KERNEL_GROUPED_TCGEN05 3
#ifndef PA_TEST_H
#define PA_TEST_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

void pa_test_skip_load(int32_t position);
int pa_test_last_decode_kernel(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_TEST_H */

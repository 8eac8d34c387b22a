/* Self-test entry point of libabattn_selftest.so, a test library beside
 * libabattn.so.  It checks the device-side failure detection that every
 * abattn kernel relies on: bounded mbarrier waits (about a second of SM
 * clock) that give up, set the device error word and return, so that a
 * stalled pipeline ends as a status code instead of a hung GPU.
 *
 * Status codes are those of abattn.h. */
#ifndef ABATTN_SELFTEST_H
#define ABATTN_SELFTEST_H

#ifdef __cplusplus
extern "C" {
#endif

/* Launches one warp that waits, with the kernels' own bounded wait, on an
 * mbarrier that nothing arrives on, then synchronizes `stream` (a
 * cudaStream_t, NULL for the default stream) and reads and clears this
 * library's device error word.
 *   waited  host int, out: 1 if the wait completed (it must not), 0 if it
 *           gave up, -1 if the kernel did not run.
 * Returns ABATTN_ERR_TIMEOUT when the wait ran out as designed, ABATTN_OK if
 * it did not, ABATTN_ERR_NULL for a NULL `waited`, ABATTN_ERR_CUDA when a
 * CUDA call failed.  Takes about a second; allocates and frees one int of
 * device memory. */
int abattn_selftest_stalled_wait(int *waited, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ABATTN_SELFTEST_H */

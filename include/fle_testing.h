/*
 * fle_testing.h -- test and diagnostic hooks of libfle.
 *
 * These entry points are not part of the fused Linear + epilogue call; they
 * exist so that tests can reach code paths that ordinary inputs leave to
 * timing (which CTA finishes a tile split over several CTAs), check the
 * device-side waits without making the real kernel stall, and bound the
 * epilogue's scalar math against CUDA's own functions.  They never change
 * what fle_forward computes, only which of its correct paths runs.  Same
 * conventions as fle.h: plain C, device pointers, stream-ordered.
 */
#ifndef FLE_TESTING_H
#define FLE_TESTING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Test hook for the bounded-wait machinery: launches one CTA whose thread
 * waits on a shared-memory barrier that nothing ever arrives on, with a wait
 * limit of timeout_us microseconds.  The wait gives up, records
 * FLE_ERR_TIMEOUT in the device status word and the kernel returns normally,
 * so the context stays usable.  Returns the launch status; read the recorded
 * status with fle_device_status().
 */
int fle_test_bounded_wait(uint32_t timeout_us, void* stream);

/*
 * Test hook for the epilogue's scalar math: out[i] = f(in[i]) for device
 * arrays of n floats, with f = erf (which = 0), exact-form GELU (1),
 * x * sigmoid(x) (2), tanh-form GELU (3) or exact-form GELU on |x| <= 2 by
 * the polynomial epilogue (a) uses there (4), evaluated either as the fused
 * epilogue evaluates it (reference = 0) or with CUDA's erff/expf/tanhf and
 * IEEE division (reference = 1), so tests can bound the difference.
 * Stream-ordered.
 */
int fle_test_epilogue_math(const float* in, float* out, int64_t n, int32_t which, int32_t reference,
                           void* stream);

/*
 * Who finishes a tile whose k-blocks the schedule split over several CTAs
 * (or CTA pairs).  Every contributor but one parks its fp32 partial tile in
 * the workspace and counts its arrival; the tile is then finished either
 *   FLE_FINISH_OWN:  by the CTA holding the tile's k-block 0, which adds the
 *                    parked partials to its own accumulator (when it finds
 *                    every other contributor already arrived), or
 *   FLE_FINISH_LAST: by whichever contributor arrives last, which sums all
 *                    parked partials starting from zero.
 * Both give the same result (partials are summed in contributor order).
 * With FLE_FINISH_AUTO (the default) the k-block-0 CTA waits up to 20 us for
 * the others to arrive, then decides; timing decides per tile.
 * FLE_FINISH_OWN makes that wait up to 50 ms, so that it finishes whenever
 * the others arrive (it parks if they have not by then); FLE_FINISH_LAST makes
 * it always park.
 * fle_test_set_finisher sets the mode for later fle_forward calls in this
 * process (all devices) and returns the previous one, or -1 for an unknown
 * mode (nothing changes).
 */
enum { FLE_FINISH_AUTO = 0, FLE_FINISH_OWN = 1, FLE_FINISH_LAST = 2 };
int fle_test_set_finisher(int32_t mode);

/*
 * Reads how many split tiles were finished each way on the current device
 * since the counts were last cleared: counts[0] by FLE_FINISH_OWN, counts[1]
 * by FLE_FINISH_LAST (a CTA of a pair counts its own 128 rows).  Synchronises
 * `stream` first; clears the counts when reset != 0.  Host array of two
 * uint32.  Returns FLE_OK or FLE_ERR_NULL / FLE_ERR_CUDA.
 */
int fle_test_finisher_counts(uint32_t* counts, int32_t reset, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLE_TESTING_H */

/*
 * hyena_conv_testing.h -- test-only entry point of libhyena_conv.so.  Not part of the
 * operation's interface (hyena_conv.h); the pages have no counterpart.  It exists so that a
 * test can make the tensor-core forward's failure detection fire without faulting the GPU.
 */
#ifndef HYENA_CONV_TESTING_H
#define HYENA_CONV_TESTING_H

#include <stdint.h>

#include "hyena_conv.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * The tensor-core forward (HYENA_ALGO_TENSOR of hyena_conv_fwd_ex, bf16) with two test
 * settings.  Every wait between the kernel's warp roles (TMA producers, MMA issuer, operand
 * build, epilogue) is bounded; `wait_ns` replaces its limit (2 s in the product path) and must
 * lie in [1 ms, 2 s].  fault == 1 makes the MMA issuer withhold its arrive for the first tile's
 * accumulator, so the epilogue's bounded wait runs out: the kernel sets HYENA_DEVICE_TIMEOUT in
 * the status word (hyena_device_status), every role leaves its loop, in-flight copies and
 * MMAs are drained (under the full 2 s limit), tensor memory is freed and the kernel returns;
 * y is then incomplete.  The CUDA context stays usable.  fault == 0 runs the kernel normally
 * under the given limit.  Arguments and errors as hyena_conv_fwd_ex, plus HYENA_ERR_INVALID_ARG
 * for fault not in {0, 1} or wait_ns outside [1 ms, 2 s] and HYENA_ERR_UNSUPPORTED for a
 * shape the tensor path does not take.
 */
int hyena_testing_fwd_fault(const void *q, const void *k, const void *v, const float *h, void *y,
                            int64_t B, int64_t L, int64_t D, int d_g, int l_h, int fault,
                            uint64_t wait_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_CONV_TESTING_H */

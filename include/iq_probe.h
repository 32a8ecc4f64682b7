/*
 * iq_probe.h -- probes of libiq_b200.so (measurement and device checks, not part of the
 * encoder path): the FP32 issue rate, and the bounded wait on bulk copies.
 *
 * The encoder searches are exhaustive argmins whose per-candidate work is a two-term fma and a
 * minimum: FP32 ALU work with no contraction in it, so their roofline is the rate at which the
 * GPU retires FP32 lane operations. These calls measure that rate on the device at hand, so the
 * roofline fraction divides by a measured number rather than a nominal lanes x clock product.
 *
 *   iq_probe_fp32(kind, blocks, iters, out, stream)
 *     launches `blocks` CTAs of 256 threads; each thread runs `iters` iterations of 8 independent
 *     chains of the given kind and stores one float in out[blocks * 256] (device memory owned by
 *     the caller; its values mean nothing). Asynchronous on `stream`; time it with events.
 *       kind 0  scalar fma.rn.f32
 *       kind 1  packed fma.rn.f32x2
 *       kind 2  per candidate pair two fma.rn.f32 and one three-input min.f32 (the encoders'
 *               candidate fold)
 *       kind 3  kind 2 with the two fmas packed into one fma.rn.f32x2
 *     Returns 0, 1 for a bad argument (nothing launched) or 3 if the launch failed.
 *   iq_probe_fp32_ops_per_iter(kind)
 *     FP32 lane ops per thread and iteration (an fma and a min each count one): 8 for kinds 0
 *     and 1, 16 for kinds 2 and 3; 0 for an unknown kind.
 * Lane ops per launch = blocks x 256 x iters x iq_probe_fp32_ops_per_iter(kind).
 *
 * A check of the bounded wait on bulk copies (the choice search's H panels). The pages have no
 * counterpart; it exists to test the copy protocol and its timeout path on the device:
 *   iq_probe_bulk_wait(src, bytes, arm, limit_cycles, out, stream)
 *     one CTA initialises an mbarrier; with arm != 0 it copies `bytes` (16..4096, a multiple of
 *     16) of device memory `src` (16-byte aligned) into shared memory with cp.async.bulk completing
 *     on that barrier; with arm == 0 it issues nothing. Every thread then waits for the barrier's
 *     first phase for at most `limit_cycles` SM cycles. out (device uint32[2]): out[0] = 1 if all
 *     threads saw the phase complete, 0 if the bound ran out; out[1] = sum over the copied words
 *     w_i of w_i (2 i + 1) mod 2^32 (0 when out[0] = 0). Asynchronous on `stream`. Returns 0, 1 for
 *     a bad argument (nothing launched) or 3 if the launch failed.
 */
#ifndef IQ_PROBE_H
#define IQ_PROBE_H

#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

int32_t iq_probe_fp32(int32_t kind, int64_t blocks, int64_t iters, float *out, cudaStream_t stream);
int64_t iq_probe_fp32_ops_per_iter(int32_t kind);
int32_t iq_probe_bulk_wait(const void *src, int64_t bytes, int32_t arm, int64_t limit_cycles, uint32_t *out,
                           cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* IQ_PROBE_H */

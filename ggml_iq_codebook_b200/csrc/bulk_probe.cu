// bulk_probe.cu -- a check of the bulk-copy wait that the choice search stages its H panels with:
// one CTA copies a caller's buffer into shared memory with the same helpers (cp.async.bulk
// completing on an mbarrier, waited on with a bounded try_wait), or arms nothing so that the
// bounded wait has to run out. It tests the protocol and its timeout path without a fault: the
// wait that runs out is on a barrier no copy was ever issued for.
#include <cuda_runtime.h>
#include <stdint.h>

#include "iq_device.cuh"
#include "iq_probe.h"

namespace {

constexpr int kProbeBytes = 4096;  // largest copy the probe stages

__global__ void bulk_probe_kernel(const uint32_t* src, int bytes, int arm, long long limit, uint32_t* out) {
    __shared__ __align__(16) uint32_t buf[kProbeBytes / 4];
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        iqk::mbar_init(&bar);
        if (arm) iqk::bulk_load(buf, src, static_cast<uint32_t>(bytes), &bar);
    }
    __syncthreads();
    const bool done = iqk::mbar_wait(&bar, 0u, limit);
    const uint32_t all = __syncthreads_and(done);
    if (threadIdx.x == 0) {
        uint32_t sum = 0u;
        if (all)
            for (int i = 0; i < bytes / 4; ++i) sum += buf[i] * static_cast<uint32_t>(2 * i + 1);
        out[0] = all;
        out[1] = sum;
    }
}

}  // namespace

extern "C" int32_t iq_probe_bulk_wait(const void* src, int64_t bytes, int32_t arm, int64_t limit_cycles,
                                      uint32_t* out, cudaStream_t stream) {
    if (out == nullptr || limit_cycles <= 0 || (arm && (src == nullptr || bytes <= 0 || bytes > kProbeBytes ||
                                                         (bytes & 15) != 0 || (reinterpret_cast<uintptr_t>(src) & 15) != 0)))
        return 1;
    bulk_probe_kernel<<<1, 128, 0, stream>>>(static_cast<const uint32_t*>(src), arm ? static_cast<int>(bytes) : 0, arm,
                                             static_cast<long long>(limit_cycles), out);
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

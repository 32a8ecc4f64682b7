// fp32_probe.cu -- issue-rate probes that give the FP32 roofline its measured denominator.
//
// The search kernels are bound by FP32 ALU work (exhaustive argmins with a two-term fma per
// candidate), not by a contraction, so their roofline is the rate at which one B200 retires
// FP32 lane operations. These kernels measure that rate: every thread runs 8 independent chains
// (enough independent work to hide the pipeline latency at 8 warps per scheduler) of
//   kind 0  scalar fma.rn.f32                     (1 FP32 op per instruction)
//   kind 1  packed fma.rn.f32x2                   (2 FP32 ops per instruction)
//   kind 2  the encoders' candidate mix: per pair of candidates two fma.rn.f32 and one
//           three-input min.f32 (the running-minimum fold), counted as 4 ops (fma + min each)
//   kind 3  kind 2 with the two fmas packed into one fma.rn.f32x2
// and the result is stored so that nothing is optimised away. Lane ops per launch =
// blocks x 256 threads x iters x ops per iteration (see iq_probe.h).
#include <cuda_runtime.h>
#include <stdint.h>

#include "iq_probe.h"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float min3(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int KIND>
__global__ void __launch_bounds__(kThreads) fp32_probe_kernel(float* out, int64_t iters, float a, float b) {
    const float t = static_cast<float>(threadIdx.x) * 1e-7f;
    float x[8], m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[i] = t + static_cast<float>(i) * 1e-3f;
        m[i] = 1e30f;
    }
    for (int64_t it = 0; it < iters; ++it) {
        if (KIND == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = __fmaf_rn(x[i], a, b);
        } else if (KIND == 1) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 r = __ffma2_rn(make_float2(x[i], x[i + 1]), make_float2(a, a), make_float2(b, b));
                x[i] = r.x;
                x[i + 1] = r.y;
            }
        } else if (KIND == 2) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                x[i] = __fmaf_rn(x[i], a, b);
                x[i + 1] = __fmaf_rn(x[i + 1], a, b);
                m[i] = min3(m[i], x[i], x[i + 1]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 r = __ffma2_rn(make_float2(x[i], x[i + 1]), make_float2(a, a), make_float2(b, b));
                x[i] = r.x;
                x[i + 1] = r.y;
                m[i] = min3(m[i], x[i], x[i + 1]);
            }
        }
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s += x[i] + (KIND >= 2 ? m[i] : 0.0f);
    out[static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x] = s;
}

}  // namespace

extern "C" {

int64_t iq_probe_fp32_ops_per_iter(int32_t kind) {
    // FP32 lane ops per thread and iteration: every kind advances the 8 chains once (8 fma);
    // kinds 2 and 3 also fold the 8 new values into running minima (8 min ops in 4 instructions)
    return kind == 0 || kind == 1 ? 8 : kind == 2 || kind == 3 ? 16 : 0;
}

int32_t iq_probe_fp32(int32_t kind, int64_t blocks, int64_t iters, float* out, cudaStream_t stream) {
    if (out == nullptr || blocks <= 0 || blocks > (1 << 20) || iters <= 0) return 1;
    const float a = 0.999999f, b = 1e-6f;
    switch (kind) {
        case 0: fp32_probe_kernel<0><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(out, iters, a, b); break;
        case 1: fp32_probe_kernel<1><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(out, iters, a, b); break;
        case 2: fp32_probe_kernel<2><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(out, iters, a, b); break;
        case 3: fp32_probe_kernel<3><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(out, iters, a, b); break;
        default: return 1;
    }
    return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

}  // extern "C"

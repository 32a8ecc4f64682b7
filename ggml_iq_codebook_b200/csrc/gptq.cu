// gptq.cu -- the per-block calibration loop's propagation kernels (sm_100a).
//
// PR #3218 ("[4/4] Run the local-Hessian choice search as one CUDA kernel") times the search
// inside GPTQ, which quantises a weight one block at a time. After block b has been quantised with
// error E = x_b - q_b (per row), GPTQ (Frantar et al. 2022, a whole 256-column block as one lazy
// batch) moves the later columns to the optimal compensation
//     W[:, rest] -= (E U_bb^-1) U_b,rest,      H^-1 = U^T U (U upper triangular).
// Arithmetic convention (identical to the CPU oracle), per row:
//   Y = E U_bb^-1 by forward substitution: column j starts from E_j, takes fma(-Y_k, U[k][j], .)
//       for k < j ascending, and Y_j = acc / U[j][j] (IEEE division);
//   every later column j' starts from w[j'] and takes fma(-Y_k, U[b 256 + k][j'], .) for
//       k = 0..255 ascending.
// Design (B200): the solve runs a warp per row, lane L owning columns 8L..8L+7 (a lane resolves
// its 8 columns, one shuffle round broadcasts them, all later columns advance their chains; the
// CTA's rows share U_bb's rows through shared memory); the update is an
// FP32 register-tiled GEMM (8 rows x 8 columns per thread, k staged through shared memory in
// ascending chunks) whose column pairs run as packed fma.rn.f32x2, so every output is still one
// sequential IEEE fma chain over k.
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

__global__ void bf16_to_f32_kernel(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw, float* out) {
    const int64_t n8 = rows * (cols / 8);
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n8;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = t / (cols / 8), c8 = t - r * (cols / 8);
        float x[8];
        unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(w + r * ldw) + c8), x);
        float4* dst = reinterpret_cast<float4*>(out + r * cols + 8 * c8);
        dst[0] = make_float4(x[0], x[1], x[2], x[3]);
        dst[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
}

constexpr int kSolveWarps = 8;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// e [rows][256] holds E on entry and Y = E U_bb^-1 on exit; ubb points at U[o][o], row stride ldu.
// A warp per row, lane L owning columns 8L..8L+7. Column group kb resolves in one lane: lane kb
// takes its 8 Y's in order (each division, then the fmas into its own later columns), broadcasts
// them, and every later lane applies the 8 to its columns, k ascending -- the forward
// substitution's chains in the oracle's order, with one cross-lane round trip per 8 columns.
// The CTA's warps share the rows 8 kb .. 8 kb + 7 of U_bb, staged in shared memory (double
// buffered with cp.async: the next group's 8 KiB stream in while this group resolves). A row's
// 16-byte slots are stored swizzled (slot q at q ^ (q >> 3 & 1)) so that a warp's reads of its
// lanes' 32-byte column chunks spread over every bank.
__global__ void __launch_bounds__(32 * kSolveWarps) gptq_solve_kernel(float* e, const float* ubb, int64_t ldu,
                                                                      int64_t rows) {
    __shared__ __align__(16) float us[2][8][kBlock];
    auto swz = [](int q) { return q ^ ((q >> 3) & 1); };  // 16-byte slot of logical slot q
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kSolveWarps + (threadIdx.x >> 5);
    const bool active = row < rows;
    auto stage = [&](int kb, int buf) {
        for (int i = threadIdx.x; i < 8 * kBlock / 4; i += 32 * kSolveWarps) {
            const int r = i / (kBlock / 4), c4 = i - r * (kBlock / 4);
            cp_async16(&us[buf][r][4 * swz(c4)], ubb + (8 * kb + r) * ldu + 4 * c4);
        }
        cp_async_commit();
    };
    float* er = e + (active ? row : 0) * kBlock + 8 * lane;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0}, y[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (active) {
        const float4 a = reinterpret_cast<const float4*>(er)[0], b = reinterpret_cast<const float4*>(er)[1];
        acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w; acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    }
    stage(0, 0);
#pragma unroll 1
    for (int kb = 0; kb < 32; ++kb) {
        cp_async_wait_all();
        __syncthreads();  // group kb's rows have landed; every warp is done with the other buffer
        if (kb + 1 < 32) stage(kb + 1, (kb + 1) & 1);
        const float(*u)[kBlock] = us[kb & 1];
        auto at = [&](int r, int c) { return u[r][4 * swz(c >> 2) + (c & 3)]; };  // U[8 kb + r][c]
        float ys[8];
        if (lane == kb) {
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                ys[s] = __fdiv_rn(acc[s], at(s, 8 * kb + s));  // U[k][k], k = 8 kb + s
                y[s] = ys[s];
#pragma unroll
                for (int t = s + 1; t < 8; ++t) acc[t] = __fmaf_rn(-ys[s], at(s, 8 * kb + t), acc[t]);
            }
        }
#pragma unroll
        for (int s = 0; s < 8; ++s) ys[s] = __shfl_sync(0xffffffffu, ys[s], kb);
        if (lane > kb) {
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const float4 ua = *reinterpret_cast<const float4*>(&u[s][4 * swz(2 * lane)]);
                const float4 ub = *reinterpret_cast<const float4*>(&u[s][4 * swz(2 * lane + 1)]);
                const float uv[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(-ys[s], uv[i], acc[i]);
            }
        }
    }
    cp_async_wait_all();
    if (active) {
        reinterpret_cast<float4*>(er)[0] = make_float4(y[0], y[1], y[2], y[3]);
        reinterpret_cast<float4*>(er)[1] = make_float4(y[4], y[5], y[6], y[7]);
    }
}

constexpr int kBM = 128, kBN = 128, kBK = 16, kUpdThreads = 256;

// W[r][col0 + n] -= sum_k Y[r][k] U[k][col0 + n]: CTA tile 128 rows x 128 columns, 16 x 16
// threads each owning 8 rows x 8 columns; k advances in chunks of 16 (ascending).
__global__ void __launch_bounds__(kUpdThreads, 2) gptq_update_kernel(const GptqUpdateParams p) {
    __shared__ __align__(16) float ys[kBK][kBM];  // -Y, k-major
    __shared__ __align__(16) float us[kBK][kBN];
    const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM, n0 = p.col0 + static_cast<int64_t>(blockIdx.x) * kBN;
    float2 acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = m0 + 8 * tm + i;
        if (r < p.rows) {
            const float4* src = reinterpret_cast<const float4*>(p.w + r * p.ldw + n0 + 8 * tn);
            const float4 a = src[0], b = src[1];
            acc[i][0] = make_float2(a.x, a.y); acc[i][1] = make_float2(a.z, a.w);
            acc[i][2] = make_float2(b.x, b.y); acc[i][3] = make_float2(b.z, b.w);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
        }
    }
#pragma unroll 1
    for (int k0 = 0; k0 < kBlock; k0 += kBK) {
        __syncthreads();  // the previous chunk is consumed
        // -Y[m0 .. m0 + 127][k0 .. k0 + 15] -> ys[k][m]: each thread one row's 8 k values
        {
            const int m = tid >> 1, kk = 8 * (tid & 1);
            const int64_t r = m0 + m;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (r < p.rows) {
                const float4* src = reinterpret_cast<const float4*>(p.y + r * kBlock + k0 + kk);
                const float4 a = __ldg(src), b = __ldg(src + 1);
                v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) ys[kk + j][m] = -v[j];
        }
        // U[k0 .. k0 + 15][n0 .. n0 + 127] -> us[k][n]: each thread 8 consecutive columns
        {
            const int k = tid >> 4, nn = 8 * (tid & 15);
            const float4* src = reinterpret_cast<const float4*>(p.u + (k0 + k) * p.ldu + n0 + nn);
            reinterpret_cast<float4*>(&us[k][nn])[0] = __ldg(src);
            reinterpret_cast<float4*>(&us[k][nn])[1] = __ldg(src + 1);
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kBK; ++k) {
            const float4 y0 = reinterpret_cast<const float4*>(&ys[k][8 * tm])[0];
            const float4 y1 = reinterpret_cast<const float4*>(&ys[k][8 * tm])[1];
            const float4 u0 = reinterpret_cast<const float4*>(&us[k][8 * tn])[0];
            const float4 u1 = reinterpret_cast<const float4*>(&us[k][8 * tn])[1];
            const float yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
            const float2 up[4] = {make_float2(u0.x, u0.y), make_float2(u0.z, u0.w), make_float2(u1.x, u1.y),
                                  make_float2(u1.z, u1.w)};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 y2 = make_float2(yv[i], yv[i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __ffma2_rn(up[j], y2, acc[i][j]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = m0 + 8 * tm + i;
        if (r < p.rows) {
            float4* dst = reinterpret_cast<float4*>(p.w + r * p.ldw + n0 + 8 * tn);
            dst[0] = make_float4(acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y);
            dst[1] = make_float4(acc[i][2].x, acc[i][2].y, acc[i][3].x, acc[i][3].y);
        }
    }
}

}  // namespace

cudaError_t launch_bf16_to_f32(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw, float* out, cudaStream_t s) {
    const int64_t n8 = rows * (cols / 8);
    if (n8 == 0) return cudaSuccess;
    const int64_t blocks = (n8 + 255) / 256;
    bf16_to_f32_kernel<<<static_cast<unsigned>(blocks < 65535 ? blocks : 65535), 256, 0, s>>>(w, rows, cols, ldw, out);
    return cudaGetLastError();
}

cudaError_t launch_gptq_solve(float* e, const float* ubb, int64_t ldu, int64_t rows, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int64_t blocks = (rows + kSolveWarps - 1) / kSolveWarps;
    gptq_solve_kernel<<<static_cast<unsigned>(blocks), 32 * kSolveWarps, 0, s>>>(e, ubb, ldu, rows);
    return cudaGetLastError();
}

cudaError_t launch_gptq_update(const GptqUpdateParams& p, int /*num_sms*/, cudaStream_t s) {
    if (p.rows == 0 || p.ncols == 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(p.ncols / kBN), static_cast<unsigned>((p.rows + kBM - 1) / kBM));
    gptq_update_kernel<<<grid, kUpdThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace iqk

// choice_search.cu -- local-Hessian choice search (sm_100a).
//
// Method (PR #3158, local_hessian for GGML IQ; fused into one launch in PR #3218): for one row of
// a 256-column block with block Hessian H and the every-choice candidates (PR #3159):
//   (1) Delta(c) = x - decode(candidate c)
//   (2) each choice group g takes argmin_c Delta_g(c)^T H_gg Delta_g(c)
//   (3) grad = H Delta, then two sweeps over the groups in order: for every c,
//       u = Delta_g(c) - Delta_g(cur), gain = 2 u^T grad_g + u^T H_gg u; the lowest c of least
//       gain is taken iff its gain < 0, then grad += H[:, g] u.
//   (4) picks, and the payload with each group's fields from its picked candidate.
// Arithmetic convention (identical to the CPU oracle): (H v)_i restricted to a group is the fma
// chain over k ascending of H[k][i] v_k starting from the product; grad_i is the same chain over
// all 256 k; sums over i inside a group are a pairwise tree; gain = fma(2, t1, t2); switching
// updates grad_i by an fma chain over the group's k. NaN and +inf scores never win.
//
// Design (B200): one CTA = 8 warps = 8 rows of one block. The rows run the group steps in
// lockstep, so each step stages one panel of H (the group's W rows, W x 256 fp32) in shared memory
// once for all 8 rows, double-buffered with cp.async so the next panel streams in while this one
// is used; H is read from L2 three times per CTA (step 2 + initial gradient fused in one pass,
// then one pass per sweep). Inside a warp the 16 choices x W columns of a group are spread as
// (choice pair, column quad) per lane: a lane keeps its two choices' W-vectors in registers and
// runs 2 x W/4 fma chains that share each 16-byte panel read. The gradient is accumulated
// column-per-thread for all 8 rows at once, and a switch updates grad with 16-byte panel reads,
// 8 columns per lane. The grid is staged in shared memory for the candidate decodes.
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

constexpr int kRows = 8;  // rows per CTA, one warp each

template <int FMT>
struct Cfg {
    static constexpr int G = FMT == IQ_FMT_IQ1_S ? 8 : 16;     // choice groups per block
    static constexpr int W = kBlock / G;                        // columns per choice group
    static constexpr int Q = W / 4;                             // columns per lane (quad split)
    static constexpr int B = FMT == IQ_FMT_IQ1_S ? kIq1sBytes : kIq2xsBytes;
    static constexpr int E = FMT == IQ_FMT_IQ1_S ? kIq1sEntries : kIq2xsEntries;
    static constexpr int BPAD = (kChoices * B + 15) / 16 * 16;  // candidate bytes per row
    static constexpr int DSTR = W + 4;                          // padded row of Dg (16-byte rows)
    // shared memory layout (bytes)
    static constexpr int oHp = 0;                               // float [2][W][256], double buffer
    static constexpr int oCurT = oHp + 2 * W * kBlock * 4;      // float [256][kRows]
    static constexpr int oGrid = oCurT + kBlock * kRows * 4;    // int2 [E]
    static constexpr int oRows = oGrid + E * 8;                 // per-row records
    static constexpr int rX = 0;                                // float [256]
    static constexpr int rCur = rX + kBlock * 4;                // float [256]
    static constexpr int rGrad = rCur + kBlock * 4;             // float [256]
    static constexpr int rDg = rGrad + kBlock * 4;              // float [16][DSTR]
    static constexpr int rU = rDg + kChoices * DSTR * 4;        // float [W]
    static constexpr int rPick = rU + W * 4;                    // int [G]
    static constexpr int rCand = rPick + G * 4;                 // uint8 [16][B]
    static constexpr int rBytes = (rCand + BPAD + 15) / 16 * 16;
    static constexpr int smem = oRows + kRows * rBytes;
};

__device__ __forceinline__ void grid_row(const int2* sgrid, int idx, float g[8]) {
    const int2 raw = sgrid[idx];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        g[j] = static_cast<float>(static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF));
}

// Dg[c][k] = x[gW + k] - decode(candidate c)[gW + k] for all 16 c, k < W. Lane: c = lane / 2,
// half = lane & 1 decodes W/2 columns.
template <int FMT>
__device__ __forceinline__ void decode_group(const uint8_t* cand, const float* x, float* Dg, const int2* grid,
                                             int g, int lane) {
    using C = Cfg<FMT>;
    const int c = lane >> 1, half = lane & 1;
    const uint8_t* pc = cand + c * C::B;
    const float d = half_bits_to_f32(static_cast<uint32_t>(pc[0]) | (static_cast<uint32_t>(pc[1]) << 8));
    float gv[8];
    if (FMT == IQ_FMT_IQ2_XS) {
        const int grp = 2 * g + half;  // 8-weight group inside the block
        const uint32_t code = static_cast<uint32_t>(pc[2 + 2 * grp]) | (static_cast<uint32_t>(pc[3 + 2 * grp]) << 8);
        const uint32_t sc = pc[66 + (g >> 1)];
        const int ls = static_cast<int>((g & 1) ? (sc >> 4) : (sc & 15u));
        const float s = __fmul_rn(d, static_cast<float>(2 * ls + 1));
        const uint32_t sign7 = code >> 9;
        const uint32_t neg = sign7 | (static_cast<uint32_t>(__popc(sign7) & 1) << 7);
        grid_row(grid, static_cast<int>(code & 511u), gv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float a = __fmul_rn(s, gv[j]);
            const float xh = ((neg >> j) & 1u) ? -a : a;
            Dg[c * C::DSTR + 8 * half + j] = __fsub_rn(x[g * C::W + 8 * half + j], xh);
        }
    } else {
        const uint32_t qh = static_cast<uint32_t>(pc[34 + 2 * g]) | (static_cast<uint32_t>(pc[35 + 2 * g]) << 8);
        const float s = __fmul_rn(d, static_cast<float>(2 * static_cast<int>((qh >> 12) & 7u) + 1));
        const float delta = (qh & 0x8000u) ? -0.125f : 0.125f;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int i4 = 2 * half + t;  // group within the sub-block
            const int idx = static_cast<int>(pc[2 + 4 * g + i4]) | static_cast<int>(((qh >> (3 * i4)) & 7u) << 8);
            grid_row(grid, idx, gv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float xh = __fmul_rn(s, __fadd_rn(gv[j], delta));
                Dg[c * C::DSTR + 8 * i4 + j] = __fsub_rn(x[g * C::W + 8 * i4 + j], xh);
            }
        }
    }
}

// Pairwise tree over this lane's Q leaves, then across the 4 column quads (lane bits 0..1).
template <int Q>
__device__ __forceinline__ float quad_tree(float p[Q]) {
#pragma unroll
    for (int width = 1; width < Q; width *= 2)
#pragma unroll
        for (int t = 0; t + width < Q; t += 2 * width) p[t] = __fadd_rn(p[t], p[t + width]);
    float v = p[0];
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 1));
    v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 2));
    return v;
}

// Warp argmin over (key(value), c) with the lowest c on ties; each lane offers two choices.
__device__ __forceinline__ void warp_argmin(float v0, int c0, float v1, int c1, float& best, int& cbest) {
    float k = argmin_key(v0);
    int c = c0;
    const float k1 = argmin_key(v1);
    if (k1 < k) { k = k1; c = c1; }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        const float ko = __shfl_xor_sync(0xffffffffu, k, o);
        const int co = __shfl_xor_sync(0xffffffffu, c, o);
        if (ko < k || (ko == k && co < c)) { k = ko; c = co; }
    }
    best = k;
    cbest = c;
}

template <int N>
__device__ __forceinline__ void load_vec(const float* src, float v[N]) {
#pragma unroll
    for (int t = 0; t < N / 4; ++t) {
        const float4 a = reinterpret_cast<const float4*>(src)[t];
        v[4 * t] = a.x; v[4 * t + 1] = a.y; v[4 * t + 2] = a.z; v[4 * t + 3] = a.w;
    }
}

// v_h[t] = sum over k < W (fma chain, k ascending) of Hp[k][col0 + t] * a_h[k], for two vectors.
template <int W, int Q>
__device__ __forceinline__ void group_matvec2(const float* Hp, int col0, const float a0[W], const float a1[W],
                                              float v0[Q], float v1[Q]) {
    float h[Q];
    load_vec<Q>(Hp + col0, h);
#pragma unroll
    for (int t = 0; t < Q; ++t) { v0[t] = __fmul_rn(h[t], a0[0]); v1[t] = __fmul_rn(h[t], a1[0]); }
#pragma unroll
    for (int k = 1; k < W; ++k) {
        load_vec<Q>(Hp + k * kBlock + col0, h);
#pragma unroll
        for (int t = 0; t < Q; ++t) {
            v0[t] = __fmaf_rn(h[t], a0[k], v0[t]);
            v1[t] = __fmaf_rn(h[t], a1[k], v1[t]);
        }
    }
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <int FMT>
__global__ void __launch_bounds__(kRows * 32) choice_search_kernel(const ChoiceParams p) {
    using C = Cfg<FMT>;
    constexpr int W = C::W, Q = C::Q, G = C::G;
    extern __shared__ __align__(16) char smem[];
    float* curT = reinterpret_cast<float*>(smem + C::oCurT);
    int2* sgrid = reinterpret_cast<int2*>(smem + C::oGrid);

    const int64_t row_tiles = (p.rows + kRows - 1) / kRows;
    const int64_t blk = blockIdx.x / row_tiles;
    const int64_t row0 = (blockIdx.x - blk * row_tiles) * kRows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = row0 + warp;
    const bool active = row < p.rows;
    char* rec = smem + C::oRows + warp * C::rBytes;
    float* x = reinterpret_cast<float*>(rec + C::rX);
    float* cur = reinterpret_cast<float*>(rec + C::rCur);
    float* grad = reinterpret_cast<float*>(rec + C::rGrad);
    float* Dg = reinterpret_cast<float*>(rec + C::rDg);
    float* ustar = reinterpret_cast<float*>(rec + C::rU);
    int* pick = reinterpret_cast<int*>(rec + C::rPick);
    uint8_t* cand = reinterpret_cast<uint8_t*>(rec + C::rCand);
    const float* H = p.hess + blk * kBlock * kBlock;

    // H panels (the W rows of one choice group) stream through a double buffer: step p of the
    // 3G group steps (step 2, then two sweeps) uses panel p % G from buffer p & 1.
    auto panel = [&](int step) { return reinterpret_cast<float*>(smem + C::oHp + (step & 1) * W * kBlock * 4); };
    auto prefetch = [&](int step) {
        const char* src = reinterpret_cast<const char*>(H + (step % G) * W * kBlock);
        char* dst = reinterpret_cast<char*>(panel(step));
        for (int i = threadIdx.x; i < W * kBlock / 4; i += blockDim.x) cp_async16(dst + 16 * i, src + 16 * i);
        cp_async_commit();
    };
    prefetch(0);

    // ---- stage the grid, the row's x (fp32) and its 16 candidate payloads
    for (int q = threadIdx.x; q < C::E; q += blockDim.x) sgrid[q] = __ldg(reinterpret_cast<const int2*>(p.grid) + q);
    if (active) {
        float xv[8];
        unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(p.w + row * p.ldw + blk * kBlock) + lane), xv);
        bool nonfinite = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            x[8 * lane + j] = xv[j];
            nonfinite |= !isfinite(xv[j]);
        }
        if (__any_sync(0xffffffffu, nonfinite) && lane == 0) raise_flags(p.flags, IQ_FLAG_NONFINITE);
        for (int c = 0; c < kChoices; ++c) {
            const uint8_t* src = p.cand + c * p.cand_cstride + (row * p.cand_ld + blk) * C::B;
            for (int i = lane; i < C::B; i += 32) cand[c * C::B + i] = src[i];
        }
    } else {
        for (int i = lane; i < kBlock; i += 32) curT[i * kRows + warp] = 0.0f;
    }

    const int cp = lane >> 2, iq = lane & 3;
    const int c0 = 2 * cp, c1 = 2 * cp + 1;
    const float* D0 = Dg + c0 * C::DSTR;
    const float* D1 = Dg + c1 * C::DSTR;

    // ---- step 2 (own diagonal block) fused with the initial gradient grad = H Delta
    float gacc[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) gacc[r] = 0.0f;
    for (int g = 0; g < G; ++g) {
        cp_async_wait_all();
        __syncthreads();  // panel g has landed; every thread is done with the other buffer
        prefetch(g + 1);
        const float* Hp = panel(g);
        if (active) {
            decode_group<FMT>(cand, x, Dg, sgrid, g, lane);
            __syncwarp();
            float a0[W], a1[W], v0[Q], v1[Q], e0[Q], e1[Q];
            load_vec<W>(D0, a0);
            load_vec<W>(D1, a1);
            group_matvec2<W, Q>(Hp, g * W + iq * Q, a0, a1, v0, v1);
            load_vec<Q>(D0 + iq * Q, e0);
            load_vec<Q>(D1 + iq * Q, e1);
#pragma unroll
            for (int t = 0; t < Q; ++t) { v0[t] = __fmul_rn(e0[t], v0[t]); v1[t] = __fmul_rn(e1[t], v1[t]); }
            const float s0 = quad_tree<Q>(v0), s1 = quad_tree<Q>(v1);
            float best;
            int cstar;
            warp_argmin(s0, c0, s1, c1, best, cstar);
            if (lane < W) {
                const float dv = Dg[cstar * C::DSTR + lane];
                cur[g * W + lane] = dv;
                curT[(g * W + lane) * kRows + warp] = dv;
            }
            if (lane == 0) pick[g] = cstar;
        }
        __syncthreads();
        // grad_i += H[k][i] cur_k over this group's k, for all rows (thread = column i)
        {
            const int i = threadIdx.x;
#pragma unroll 4
            for (int k = 0; k < W; ++k) {
                const float h = Hp[k * kBlock + i];
                const float4 ca = *reinterpret_cast<const float4*>(curT + (g * W + k) * kRows);
                const float4 cb = *reinterpret_cast<const float4*>(curT + (g * W + k) * kRows + 4);
                const float cv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
                if (g == 0 && k == 0) {
#pragma unroll
                    for (int r = 0; r < kRows; ++r) gacc[r] = __fmul_rn(h, cv[r]);
                } else {
#pragma unroll
                    for (int r = 0; r < kRows; ++r) gacc[r] = __fmaf_rn(h, cv[r], gacc[r]);
                }
            }
        }
    }
    {
        const int i = threadIdx.x;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float* gr = reinterpret_cast<float*>(smem + C::oRows + r * C::rBytes + C::rGrad);
            gr[i] = gacc[r];
        }
    }

    // ---- step 3: two sweeps over the groups
    for (int step = G; step < 3 * G; ++step) {
        const int g = step % G;
        cp_async_wait_all();
        __syncthreads();
        if (step + 1 < 3 * G) prefetch(step + 1);
        const float* Hp = panel(step);
        if (!active) continue;
        decode_group<FMT>(cand, x, Dg, sgrid, g, lane);
        __syncwarp();
        float u0[W], u1[W], v0[Q], v1[Q];
        {
            float cg[W];
            load_vec<W>(cur + g * W, cg);
            load_vec<W>(D0, u0);
            load_vec<W>(D1, u1);
#pragma unroll
            for (int k = 0; k < W; ++k) { u0[k] = __fsub_rn(u0[k], cg[k]); u1[k] = __fsub_rn(u1[k], cg[k]); }
        }
        group_matvec2<W, Q>(Hp, g * W + iq * Q, u0, u1, v0, v1);
        float gain0, gain1;
        {
            float cq[Q], e0[Q], e1[Q], gq[Q], p0[Q], p1[Q];
            load_vec<Q>(cur + g * W + iq * Q, cq);
            load_vec<Q>(D0 + iq * Q, e0);
            load_vec<Q>(D1 + iq * Q, e1);
            load_vec<Q>(grad + g * W + iq * Q, gq);
#pragma unroll
            for (int t = 0; t < Q; ++t) {
                e0[t] = __fsub_rn(e0[t], cq[t]);  // u_i of this lane's columns
                e1[t] = __fsub_rn(e1[t], cq[t]);
                p0[t] = __fmul_rn(e0[t], gq[t]);
                p1[t] = __fmul_rn(e1[t], gq[t]);
                v0[t] = __fmul_rn(e0[t], v0[t]);
                v1[t] = __fmul_rn(e1[t], v1[t]);
            }
            const float t10 = quad_tree<Q>(p0), t11 = quad_tree<Q>(p1);
            const float t20 = quad_tree<Q>(v0), t21 = quad_tree<Q>(v1);
            gain0 = __fmaf_rn(2.0f, t10, t20);
            gain1 = __fmaf_rn(2.0f, t11, t21);
        }
        float best;
        int cstar;
        warp_argmin(gain0, c0, gain1, c1, best, cstar);
        if (best < 0.0f) {
            if (lane < W) ustar[lane] = __fsub_rn(Dg[cstar * C::DSTR + lane], cur[g * W + lane]);
            __syncwarp();
            // grad[i] += sum_k H[k][i] u_k (fma chain over the group's k), 8 columns per lane
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int i0 = half * 128 + 4 * lane;
                float4 acc = *reinterpret_cast<const float4*>(grad + i0);
#pragma unroll 4
                for (int k = 0; k < W; ++k) {
                    const float uk = ustar[k];
                    const float4 hv = *reinterpret_cast<const float4*>(Hp + k * kBlock + i0);
                    acc.x = __fmaf_rn(hv.x, uk, acc.x);
                    acc.y = __fmaf_rn(hv.y, uk, acc.y);
                    acc.z = __fmaf_rn(hv.z, uk, acc.z);
                    acc.w = __fmaf_rn(hv.w, uk, acc.w);
                }
                *reinterpret_cast<float4*>(grad + i0) = acc;
            }
            __syncwarp();
            if (lane < W) cur[g * W + lane] = Dg[cstar * C::DSTR + lane];
            if (lane == 0) pick[g] = cstar;
        }
        __syncwarp();
    }

    // ---- step 4: picks and the payload assembled from the picked candidates
    if (active) {
        __syncwarp();
        for (int g = lane; g < G; g += 32) p.picks[(row * p.nblk + blk) * G + g] = static_cast<uint8_t>(pick[g]);
        uint8_t* out = p.payload + (row * p.payload_ld + blk) * C::B;
        for (int i = lane; i < C::B; i += 32) {
            uint8_t v;
            if (i < 2) {
                v = cand[i];
            } else if (FMT == IQ_FMT_IQ2_XS) {
                if (i < 66) {
                    v = cand[pick[(i - 2) >> 2] * C::B + i];
                } else {
                    const int k = 2 * (i - 66);
                    v = static_cast<uint8_t>((cand[pick[k] * C::B + i] & 0x0Fu) | (cand[pick[k + 1] * C::B + i] & 0xF0u));
                }
            } else {
                const int g = i < 34 ? (i - 2) >> 2 : (i - 34) >> 1;
                v = cand[pick[g] * C::B + i];
            }
            out[i] = v;
        }
    }
}

template <int FMT>
cudaError_t launch(const ChoiceParams& p, cudaStream_t s) {
    using C = Cfg<FMT>;
    auto kern = choice_search_kernel<FMT>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::smem);
    if (err != cudaSuccess) return err;
    const int64_t ctas = p.nblk * ((p.rows + kRows - 1) / kRows);
    kern<<<static_cast<unsigned>(ctas), kRows * 32, C::smem, s>>>(p);
    return cudaGetLastError();
}

__global__ void sqrt_diag_kernel(const float* hess, int64_t nblk, float* out) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= nblk * kBlock) return;
    const int64_t b = t / kBlock, i = t - b * kBlock;
    out[t] = __fsqrt_rn(hess[b * kBlock * kBlock + i * kBlock + i]);
}

}  // namespace

cudaError_t launch_choice_search(int fmt, const ChoiceParams& p, int /*num_sms*/, cudaStream_t s) {
    if (p.rows == 0 || p.nblk == 0) return cudaSuccess;
    return fmt == IQ_FMT_IQ1_S ? launch<IQ_FMT_IQ1_S>(p, s) : launch<IQ_FMT_IQ2_XS>(p, s);
}

cudaError_t launch_sqrt_diag(const float* hess, int64_t nblk, float* out, cudaStream_t s) {
    if (nblk == 0) return cudaSuccess;
    const int64_t n = nblk * kBlock;
    sqrt_diag_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(hess, nblk, out);
    return cudaGetLastError();
}

}  // namespace iqk

// iq_decode.cu -- IQ1_S / IQ2_XS decoders (sm_100a), HBM-bound.
//
// Values (PR #2450 review comments):
//   IQ1_S  x = d (2 ls + 1) (q_j + delta), index = low | ((qh >> 3i) & 7) << 8, ls = qh bits
//          12..14, delta = -1/8 if qh bit 15 else +1/8.
//   IQ2_XS x = d (2 ls + 1) g_j (-1)^sign_j, code = index | sign7 << 9, sign_7 = parity(sign7),
//          ls of sub-block k in nibble (k & 1) of byte 66 + k/2.
// Every value is a product of at most 20 significant bits, so the fp32 result is exact; the bf16
// output is its round-to-nearest-even. Each block decodes independently, so the output does not
// depend on how a caller chunks the blocks.
//
// Design: one warp per block, one lane per 8-weight group. The warp reads the block's payload as
// 16-bit words (one per lane, coalesced into one or two sectors) and hands each lane its fields
// with warp shuffles. Each warp works on 8 blocks at a time and issues the payload loads of its
// next 8 blocks before decoding the current ones, so HBM latency overlaps the work; the grid
// (16 KiB / 4 KiB) is staged once per CTA in shared memory, so no global load depends on another.
// Each lane writes its 8 outputs with one 16-byte (bf16) or two 16-byte (fp32) streaming stores:
// a warp writes 512 or 1024 contiguous bytes per block.
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;  // blocks per warp per iteration (and as many prefetched)

template <bool BF16>
__device__ __forceinline__ void store8(void* out, int64_t group, const float v[8]) {
    if (BF16) {
        uint4 o;
        o.x = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[0]))) |
              (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[1]))) << 16);
        o.y = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2]))) |
              (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[3]))) << 16);
        o.z = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[4]))) |
              (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[5]))) << 16);
        o.w = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[6]))) |
              (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[7]))) << 16);
        __stcs(reinterpret_cast<uint4*>(out) + group, o);
    } else {
        float4* o = reinterpret_cast<float4*>(out) + 2 * group;
        __stcs(o, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(o + 1, make_float4(v[4], v[5], v[6], v[7]));
    }
}

__device__ __forceinline__ void grid_row(const int2* grid, int idx, float g[8]) {
    const int2 raw = grid[idx];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        g[j] = static_cast<float>(static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF));
}

// Fields of this lane's group from the block's 16-bit words (v0: word `lane`, v1: word 32+lane).
template <int FMT>
__device__ __forceinline__ void group_fields(uint32_t v0, uint32_t v1, int lane, float& s, float& delta,
                                             int& idx, uint32_t& neg) {
    const float d = half_bits_to_f32(__shfl_sync(0xffffffffu, v0, 0));
    if (FMT == IQ_FMT_IQ1_S) {
        const uint32_t lw = __shfl_sync(0xffffffffu, v0, 1 + (lane >> 1));
        const uint32_t qh = __shfl_sync(0xffffffffu, v0, 17 + (lane >> 2));
        const uint32_t low = (lane & 1) ? (lw >> 8) : (lw & 0xFFu);
        idx = static_cast<int>(low | (((qh >> (3 * (lane & 3))) & 7u) << 8));
        s = __fmul_rn(d, static_cast<float>(2 * static_cast<int>((qh >> 12) & 7u) + 1));
        delta = (qh & 0x8000u) ? -0.125f : 0.125f;
        neg = 0;
    } else {
        const uint32_t ca = __shfl_sync(0xffffffffu, v0, lane < 31 ? lane + 1 : 31);
        const uint32_t cb = __shfl_sync(0xffffffffu, v1, 0);
        const uint32_t code = lane < 31 ? ca : cb;
        const uint32_t sw = __shfl_sync(0xffffffffu, v1, 1 + (lane >> 3));  // bytes 66 + 2m, 67 + 2m
        const uint32_t sc = ((lane >> 2) & 1) ? (sw >> 8) : (sw & 0xFFu);
        const int ls = static_cast<int>(((lane >> 1) & 1) ? (sc >> 4) : (sc & 15u));
        s = __fmul_rn(d, static_cast<float>(2 * ls + 1));
        delta = 0.0f;
        idx = static_cast<int>(code & 511u);
        const uint32_t sign7 = code >> 9;
        neg = sign7 | (static_cast<uint32_t>(__popc(sign7) & 1) << 7);
    }
}

template <int WORDS>
__device__ __forceinline__ void load_words(const uint16_t* words, int64_t b0, int64_t nblocks, int lane,
                                           uint32_t v0[kUnroll], uint32_t v1[kUnroll]) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t b = b0 + u;
        v0[u] = 0;
        v1[u] = 0;
        if (b < nblocks) {
            if (lane < WORDS) v0[u] = __ldcs(words + b * WORDS + lane);
            if (WORDS > 32 && lane < WORDS - 32) v1[u] = __ldcs(words + b * WORDS + 32 + lane);
        }
    }
}

template <int FMT, bool BF16>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
    constexpr int BYTES = FMT == IQ_FMT_IQ1_S ? kIq1sBytes : kIq2xsBytes;
    constexpr int WORDS = BYTES / 2;
    constexpr int E = FMT == IQ_FMT_IQ1_S ? kIq1sEntries : kIq2xsEntries;
    __shared__ int2 sgrid[E];
    for (int q = threadIdx.x; q < E; q += kThreads) sgrid[q] = __ldg(reinterpret_cast<const int2*>(p.grid) + q);
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
    const int64_t stride = nwarps * kUnroll;
    const uint16_t* words = reinterpret_cast<const uint16_t*>(p.payload);

    uint32_t v0[kUnroll], v1[kUnroll];
    int64_t b0 = warp * kUnroll;
    load_words<WORDS>(words, b0, p.nblocks, lane, v0, v1);
    for (; b0 < p.nblocks; b0 += stride) {
        uint32_t n0[kUnroll], n1[kUnroll];
        load_words<WORDS>(words, b0 + stride, p.nblocks, lane, n0, n1);  // next batch, in flight
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t b = b0 + u;
            if (b >= p.nblocks) break;  // warp-uniform
            float s, delta;
            int idx;
            uint32_t neg;
            group_fields<FMT>(v0[u], v1[u], lane, s, delta, idx, neg);
            float g[8], v[8];
            grid_row(sgrid, idx, g);
            if (FMT == IQ_FMT_IQ1_S) {
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(s, __fadd_rn(g[j], delta));
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float a = __fmul_rn(s, g[j]);
                    v[j] = ((neg >> j) & 1u) ? -a : a;
                }
            }
            store8<BF16>(p.out, b * 32 + lane, v);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) { v0[u] = n0[u]; v1[u] = n1[u]; }
    }
}

template <int FMT, bool BF16>
cudaError_t launch(const DecodeParams& p, int num_sms, cudaStream_t s) {
    const int64_t warps_needed = (p.nblocks + kUnroll - 1) / kUnroll;
    const int64_t ctas_needed = (warps_needed + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = 8LL * num_sms;  // 8 CTAs of 256 threads fill an SM
    const int64_t ctas = ctas_needed < cap ? ctas_needed : cap;
    decode_kernel<FMT, BF16><<<static_cast<unsigned>(ctas), kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int fmt, bool bf16, const DecodeParams& p, int num_sms, cudaStream_t s) {
    if (p.nblocks == 0) return cudaSuccess;
    if (fmt == IQ_FMT_IQ1_S) return bf16 ? launch<IQ_FMT_IQ1_S, true>(p, num_sms, s) : launch<IQ_FMT_IQ1_S, false>(p, num_sms, s);
    return bf16 ? launch<IQ_FMT_IQ2_XS, true>(p, num_sms, s) : launch<IQ_FMT_IQ2_XS, false>(p, num_sms, s);
}

}  // namespace iqk

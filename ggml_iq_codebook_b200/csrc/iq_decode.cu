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
// Design: one thread per 8-weight group (a warp per block), writing 16 B (bf16) or 32 B (fp32)
// per thread, coalesced; each CTA stages its tile of payload bytes in shared memory with 16-byte
// loads when the tile is 16-byte aligned. The grid (16 KiB / 4 KiB) is read through the L1 cache.
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

constexpr int kThreads = 256;
constexpr int kTileBlocks = 32;  // blocks per CTA iteration (4 groups per thread)

template <int BYTES>
__device__ __forceinline__ void stage_tile(uint8_t* sp, const uint8_t* src, int nbytes) {
    // BYTES * kTileBlocks is a multiple of 16; a full tile whose start is 16-aligned moves in
    // 16-byte vectors, anything else byte by byte.
    if (nbytes == BYTES * kTileBlocks && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        uint4* d4 = reinterpret_cast<uint4*>(sp);
        for (int i = threadIdx.x; i < nbytes / 16; i += kThreads) d4[i] = __ldg(s4 + i);
    } else {
        for (int i = threadIdx.x; i < nbytes; i += kThreads) sp[i] = src[i];
    }
}

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

__device__ __forceinline__ void grid_row(const int8_t* grid, int idx, float g[8]) {
    const int2 raw = __ldg(reinterpret_cast<const int2*>(grid) + idx);
#pragma unroll
    for (int j = 0; j < 8; ++j)
        g[j] = static_cast<float>(static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF));
}

template <int FMT, bool BF16>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
    constexpr int BYTES = FMT == IQ_FMT_IQ1_S ? kIq1sBytes : kIq2xsBytes;
    __shared__ __align__(16) uint8_t tile[BYTES * kTileBlocks];
    const int64_t ntiles = (p.nblocks + kTileBlocks - 1) / kTileBlocks;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int64_t b0 = t * kTileBlocks;
        const int nb = static_cast<int>(p.nblocks - b0 < kTileBlocks ? p.nblocks - b0 : kTileBlocks);
        __syncthreads();  // the previous tile is no longer read
        stage_tile<BYTES>(tile, p.payload + b0 * BYTES, nb * BYTES);
        __syncthreads();
#pragma unroll
        for (int rep = 0; rep < kTileBlocks * 32 / kThreads; ++rep) {
            const int gl = rep * kThreads + threadIdx.x;  // group within the tile
            const int bl = gl >> 5, grp = gl & 31;
            if (bl >= nb) break;
            const uint8_t* pb = tile + bl * BYTES;
            const float d = half_bits_to_f32(static_cast<uint32_t>(pb[0]) | (static_cast<uint32_t>(pb[1]) << 8));
            float g[8], v[8];
            if (FMT == IQ_FMT_IQ1_S) {
                const int k = grp >> 2;
                const uint32_t qh = static_cast<uint32_t>(pb[34 + 2 * k]) | (static_cast<uint32_t>(pb[35 + 2 * k]) << 8);
                const int idx = static_cast<int>(pb[2 + grp]) | static_cast<int>(((qh >> (3 * (grp & 3))) & 7u) << 8);
                const float s = __fmul_rn(d, static_cast<float>(2 * static_cast<int>((qh >> 12) & 7u) + 1));
                const float delta = (qh & 0x8000u) ? -0.125f : 0.125f;
                grid_row(p.grid, idx, g);
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(s, __fadd_rn(g[j], delta));
            } else {
                const uint32_t code = static_cast<uint32_t>(pb[2 + 2 * grp]) | (static_cast<uint32_t>(pb[3 + 2 * grp]) << 8);
                const int k = grp >> 1;
                const uint32_t sc = pb[66 + (k >> 1)];
                const int ls = static_cast<int>((k & 1) ? (sc >> 4) : (sc & 15u));
                const float s = __fmul_rn(d, static_cast<float>(2 * ls + 1));
                const uint32_t sign7 = code >> 9;
                const uint32_t neg = sign7 | (static_cast<uint32_t>(__popc(sign7) & 1) << 7);
                grid_row(p.grid, static_cast<int>(code & 511u), g);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float a = __fmul_rn(s, g[j]);
                    v[j] = ((neg >> j) & 1u) ? -a : a;
                }
            }
            store8<BF16>(p.out, (b0 + bl) * 32 + grp, v);
        }
    }
}

template <int FMT, bool BF16>
cudaError_t launch(const DecodeParams& p, int num_sms, cudaStream_t s) {
    const int64_t ntiles = (p.nblocks + kTileBlocks - 1) / kTileBlocks;
    const int64_t cap = 8LL * num_sms;  // 8 CTAs of 256 threads fill an SM
    const int64_t ctas = ntiles < cap ? ntiles : cap;
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

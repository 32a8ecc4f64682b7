// iq_decode.cu -- IQ1_S / IQ2_XS / IQ1_M / IQ2_S decoders (sm_100a), HBM-bound.
//
// Values (PR #2450 review comments):
//   IQ1_S  x = d (2 ls + 1) (q_j + delta), index = low | ((qh >> 3i) & 7) << 8, ls = qh bits
//          12..14, delta = -1/8 if qh bit 15 else +1/8.
//   IQ2_XS x = d (2 ls + 1) g_j (-1)^sign_j, code = index | sign7 << 9, sign_7 = parity(sign7),
//          ls of sub-block k in nibble (k & 1) of byte 66 + k/2.
//   IQ1_M  (PR #2513) x = d (2 ls + 1) (q_j + delta), d = the top nibbles of the four scale words
//          at bytes 48..55, ls of choice group k = bits 3(k%4).. of word k/4, group g's index
//          = byte g | (nibble g of bytes 32.. & 7) << 8, delta = -1/8 if that nibble's bit 3.
//   IQ2_S  (PR #2512) x = d (2 ls + 1) g_j (-1)^sign_j, index = byte 2 + g | 2 bits at shift
//          2 (g % 4) of byte 66 + g/4 << 8, sign mask = byte 34 + g, ls as IQ2_XS at bytes 74...
// Every value is a product of at most 20 significant bits, so the fp32 result is exact; the bf16
// output is its round-to-nearest-even. Each block decodes independently, so the output does not
// depend on how a caller chunks the blocks.
//
// Design: persistent CTAs walk tiles of 256 blocks. A tile's payload bytes (12.5, 14, 18.5 or
// 20.5 KiB for IQ1_S, IQ1_M, IQ2_XS, IQ2_S)
// stream into shared memory with 16-byte cp.async copies, double-buffered, so the next tile's
// reads are in flight while this one is decoded and no warp waits on its own small global loads.
// A half-warp decodes one block, two adjacent 8-weight groups per lane, reading its fields from
// the staged bytes; the grid is staged once per CTA as 16-bit element codes (4, 1 or 2 KiB), and
// outputs are picked from a lane's precomputed products (no int-to-float conversions, which
// throttle the MIO queue). Each lane writes its 16 outputs with 32-byte streaming stores
// (st.global.v8): one for bf16, two for fp32.
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

constexpr int kThreads = 256;
constexpr int kMinCtas = 1;      // launch-bounds occupancy hint (CTAs per SM)
constexpr int kTileBlocks = 256;  // blocks per staged payload tile
constexpr int kCtasPerSm = 5;     // persistent CTAs per SM

// Two fp32 values rounded to bf16 (nearest even) in one packed conversion: a in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void st_global_v8(void* ptr, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                             uint32_t f, uint32_t g, uint32_t h) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(a), "r"(b), "r"(c),
                 "r"(d), "r"(e), "r"(f), "r"(g), "r"(h)
                 : "memory");
}

// Store 16 consecutive outputs (two groups) starting at output element 8 * group.
template <bool BF16>
__device__ __forceinline__ void store16(void* out, int64_t group, const float v[16]) {
    if (BF16) {
        uint32_t w[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) w[t] = pack_bf16x2(v[2 * t], v[2 * t + 1]);
        st_global_v8(reinterpret_cast<uint4*>(out) + group, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    } else {
        float4* o = reinterpret_cast<float4*>(out) + 2 * group;
#pragma unroll
        for (int h = 0; h < 2; ++h)
            st_global_v8(o + 2 * h, __float_as_uint(v[8 * h]), __float_as_uint(v[8 * h + 1]),
                         __float_as_uint(v[8 * h + 2]), __float_as_uint(v[8 * h + 3]), __float_as_uint(v[8 * h + 4]),
                         __float_as_uint(v[8 * h + 5]), __float_as_uint(v[8 * h + 6]), __float_as_uint(v[8 * h + 7]));
    }
}


__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// A half-warp decodes one block from its staged payload bytes `pb` (2-byte aligned); lane
// h = lane & 15 decodes groups 2h and 2h + 1 (for IQ1_M: exactly choice group h). No int-to-float conversion on the way: a lane
// forms the few products a group can take (IQ1_S: s (q + delta) for q in {-1, 0, 1}; IQ2_XS:
// s g for g in {1, 3, 5, 7}), each rounded exactly as the direct formula rounds it, and picks
// per element from the staged grid codes.
template <int FMT, bool BF16>
__device__ __forceinline__ void decode_pair(const uint8_t* pb, int h, const uint16_t* sgrid, void* out, int64_t b) {
    const uint16_t* pw = reinterpret_cast<const uint16_t*>(pb);
    float v[16];
    if (FMT == IQ_FMT_IQ1_M) {
        const uint32_t w0 = pw[24], w1 = pw[25], w2 = pw[26], w3 = pw[27];
        const float d = half_bits_to_f32(iq1m_d_bits(w0, w1, w2, w3));
        const uint32_t wk = pw[24 + (h >> 2)];
        const float s = __fmul_rn(d, small_int_to_float(2u * ((wk >> (3 * (h & 3))) & 7u) + 1u));
        const uint32_t lw = pw[h];      // low index bytes of groups 2h, 2h + 1
        const uint32_t nb = pb[32 + h];  // their nibbles
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t nib = (nb >> (4 * t)) & 15u;
            const float delta = (nib & 8u) ? -0.125f : 0.125f;
            const float vp = __fmul_rn(s, __fadd_rn(1.0f, delta));
            const float v0 = __fmul_rn(s, __fadd_rn(0.0f, delta));
            const float vn = __fmul_rn(s, __fadd_rn(-1.0f, delta));
            const int idx = static_cast<int>(((lw >> (8 * t)) & 0xFFu) | ((nib & 7u) << 8));
            const uint32_t m = sgrid[idx];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[8 * t + j] = ((m >> j) & 1u) ? vp : (((m >> (8 + j)) & 1u) ? vn : v0);
        }
        store16<BF16>(out, b * 32 + 2 * h, v);
        return;
    }
    const float d = half_bits_to_f32(pw[0]);
    if (FMT == IQ_FMT_IQ2_S) {
        const uint32_t sc = pb[74 + (h >> 1)];
        const int ls = static_cast<int>((h & 1) ? (sc >> 4) : (sc & 15u));
        const float s = __fmul_rn(d, small_int_to_float(static_cast<uint32_t>(2 * ls + 1)));
        const float m1 = __fmul_rn(s, 1.0f), m3 = __fmul_rn(s, 3.0f), m5 = __fmul_rn(s, 5.0f), m7 = __fmul_rn(s, 7.0f);
        const uint32_t lw = pw[1 + h];                  // low index bytes of groups 2h, 2h + 1
        const uint32_t sg = pw[17 + h];                 // their sign bytes
        const uint32_t hb = pb[66 + (h >> 1)] >> (4 * (h & 1));
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t idx = ((lw >> (8 * t)) & 0xFFu) | (((hb >> (2 * t)) & 3u) << 8);
            const uint32_t neg = (sg >> (8 * t)) & 0xFFu;
            const uint32_t e = sgrid[idx];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t cj = (e >> (2 * j)) & 3u;
                const float a = (cj & 2u) ? ((cj & 1u) ? m7 : m5) : ((cj & 1u) ? m3 : m1);
                v[8 * t + j] = ((neg >> j) & 1u) ? -a : a;
            }
        }
        store16<BF16>(out, b * 32 + 2 * h, v);
        return;
    }
    if (FMT == IQ_FMT_IQ1_S) {
        const uint32_t lw = pw[1 + h];          // low index bytes of groups 2h, 2h + 1
        const uint32_t qh = pw[17 + (h >> 1)];  // the sub-block's qh
        const float s = __fmul_rn(d, small_int_to_float(2u * ((qh >> 12) & 7u) + 1u));
        const float delta = (qh & 0x8000u) ? -0.125f : 0.125f;
        const float vp = __fmul_rn(s, __fadd_rn(1.0f, delta));   // q = +1
        const float v0 = __fmul_rn(s, __fadd_rn(0.0f, delta));   // q = 0
        const float vn = __fmul_rn(s, __fadd_rn(-1.0f, delta));  // q = -1
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int grp = 2 * h + t;
            const int idx = static_cast<int>(((lw >> (8 * t)) & 0xFFu) | (((qh >> (3 * (grp & 3))) & 7u) << 8));
            const uint32_t m = sgrid[idx];  // bit j: q_j = +1; bit 8 + j: q_j = -1
#pragma unroll
            for (int j = 0; j < 8; ++j) v[8 * t + j] = ((m >> j) & 1u) ? vp : (((m >> (8 + j)) & 1u) ? vn : v0);
        }
    } else {
        const uint32_t ca = pw[1 + 2 * h], cb = pw[2 + 2 * h];  // codes of groups 2h, 2h + 1
        const uint32_t sc = pb[66 + (h >> 1)];                   // scales of sub-blocks 2(h/2), +1
        const int ls = static_cast<int>((h & 1) ? (sc >> 4) : (sc & 15u));
        const float s = __fmul_rn(d, small_int_to_float(static_cast<uint32_t>(2 * ls + 1)));
        const float m1 = __fmul_rn(s, 1.0f), m3 = __fmul_rn(s, 3.0f), m5 = __fmul_rn(s, 5.0f), m7 = __fmul_rn(s, 7.0f);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t code = t ? cb : ca;
            const uint32_t sign7 = code >> 9;
            const uint32_t neg = sign7 | (static_cast<uint32_t>(__popc(sign7) & 1) << 7);
            const uint32_t e = sgrid[code & 511u];  // 2 bits per element: g = 2 * bits + 1
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t cj = (e >> (2 * j)) & 3u;
                const float a = (cj & 2u) ? ((cj & 1u) ? m7 : m5) : ((cj & 1u) ? m3 : m1);
                v[8 * t + j] = ((neg >> j) & 1u) ? -a : a;
            }
        }
    }
    store16<BF16>(out, b * 32 + 2 * h, v);
}

template <int FMT>
struct DecodeCfg {
    static constexpr int BYTES = FMT == IQ_FMT_IQ1_S   ? kIq1sBytes
                                 : FMT == IQ_FMT_IQ1_M ? kIq1mBytes
                                 : FMT == IQ_FMT_IQ2_S ? kIq2sBytes
                                                       : kIq2xsBytes;
    static constexpr bool IQ2 = FMT == IQ_FMT_IQ2_XS || FMT == IQ_FMT_IQ2_S;
    static constexpr int E = FMT == IQ_FMT_IQ2_XS ? kIq2xsEntries : FMT == IQ_FMT_IQ2_S ? kIq2sEntries : kIq1sEntries;
    static constexpr int TILE_BYTES = kTileBlocks * BYTES;  // a multiple of 16
    static constexpr int GRID_BYTES = (E * 2 + 15) / 16 * 16;
    static constexpr int smem = GRID_BYTES + 2 * TILE_BYTES;
};

// The grid as 16-bit codes: IQ1_S, IQ1_M (+1 mask) | (-1 mask) << 8; IQ2_XS two bits (g - 1) / 2 per
// element. Values outside the format's alphabet are not representable here.
template <int FMT>
__device__ __forceinline__ uint16_t grid_code(int2 raw) {
    uint32_t c = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
        if (!DecodeCfg<FMT>::IQ2) c |= (static_cast<uint32_t>(v == 1) << j) | (static_cast<uint32_t>(v == -1) << (8 + j));
        else c |= (static_cast<uint32_t>((v - 1) >> 1) & 3u) << (2 * j);
    }
    return static_cast<uint16_t>(c);
}

template <int FMT, bool BF16>
__global__ void __launch_bounds__(kThreads, kMinCtas) decode_kernel(const DecodeParams p) {
    using C = DecodeCfg<FMT>;
    extern __shared__ __align__(16) char smem[];
    uint16_t* sgrid = reinterpret_cast<uint16_t*>(smem);
    uint8_t* tiles = reinterpret_cast<uint8_t*>(smem + C::GRID_BYTES);
    for (int q = threadIdx.x; q < C::E; q += kThreads)
        sgrid[q] = grid_code<FMT>(__ldg(reinterpret_cast<const int2*>(p.grid) + q));

    const int64_t ntiles = (p.nblocks + kTileBlocks - 1) / kTileBlocks;
    const bool aligned16 = (reinterpret_cast<uintptr_t>(p.payload) & 15u) == 0;
    // Stage tile t into buffer buf: 16-byte async copies when the tile is whole and aligned,
    // plain byte copies otherwise (made visible by the barrier before the tile is read).
    auto stage = [&](int64_t t, int buf) {
        if (t < ntiles) {
            const int64_t nb = p.nblocks - t * kTileBlocks < kTileBlocks ? p.nblocks - t * kTileBlocks : kTileBlocks;
            const int bytes = static_cast<int>(nb) * C::BYTES;
            const uint8_t* src = p.payload + t * C::TILE_BYTES;
            uint8_t* dst = tiles + buf * C::TILE_BYTES;
            if (aligned16 && (bytes & 15) == 0) {
                for (int i = threadIdx.x; i < bytes / 16; i += kThreads) cp_async16(dst + 16 * i, src + 16 * i);
            } else {
                for (int i = threadIdx.x; i < bytes; i += kThreads) dst[i] = src[i];
            }
        }
        cp_async_commit();
    };

    const int hw = threadIdx.x >> 4, h = threadIdx.x & 15;  // half-warp, lane within it
    int buf = 0;
    stage(blockIdx.x, 0);
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, buf ^= 1) {
        stage(t + gridDim.x, buf ^ 1);  // the next tile streams in while this one is decoded
        cp_async_wait<1>();
        __syncthreads();
        const int64_t nb = p.nblocks - t * kTileBlocks < kTileBlocks ? p.nblocks - t * kTileBlocks : kTileBlocks;
        const uint8_t* tile = tiles + buf * C::TILE_BYTES;
        for (int k = hw; k < nb; k += kThreads / 16)
            decode_pair<FMT, BF16>(tile + k * C::BYTES, h, sgrid, p.out, t * kTileBlocks + k);
        __syncthreads();  // the buffer is refilled next iteration
    }
    cp_async_wait<0>();
}

template <int FMT, bool BF16>
cudaError_t launch(const DecodeParams& p, int num_sms, cudaStream_t s) {
    using C = DecodeCfg<FMT>;
    auto kern = decode_kernel<FMT, BF16>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::smem);
    if (err != cudaSuccess) return err;
    const int64_t ntiles = (p.nblocks + kTileBlocks - 1) / kTileBlocks;
    const int64_t cap = static_cast<int64_t>(kCtasPerSm) * num_sms;
    const int64_t ctas = ntiles < cap ? ntiles : cap;
    kern<<<static_cast<unsigned>(ctas), kThreads, C::smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int fmt, bool bf16, const DecodeParams& p, int num_sms, cudaStream_t s) {
    if (p.nblocks == 0) return cudaSuccess;
    if (fmt == IQ_FMT_IQ1_S) return bf16 ? launch<IQ_FMT_IQ1_S, true>(p, num_sms, s) : launch<IQ_FMT_IQ1_S, false>(p, num_sms, s);
    if (fmt == IQ_FMT_IQ1_M) return bf16 ? launch<IQ_FMT_IQ1_M, true>(p, num_sms, s) : launch<IQ_FMT_IQ1_M, false>(p, num_sms, s);
    if (fmt == IQ_FMT_IQ2_S) return bf16 ? launch<IQ_FMT_IQ2_S, true>(p, num_sms, s) : launch<IQ_FMT_IQ2_S, false>(p, num_sms, s);
    return bf16 ? launch<IQ_FMT_IQ2_XS, true>(p, num_sms, s) : launch<IQ_FMT_IQ2_XS, false>(p, num_sms, s);
}

}  // namespace iqk

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
// 20.5 KiB for IQ1_S, IQ1_M, IQ2_XS, IQ2_S) stream into shared memory with 16-byte cp.async
// copies, double-buffered, so the next tile's reads are in flight while this one is decoded and
// no warp waits on its own small global loads. A half-warp decodes one block, two adjacent
// 8-weight groups per lane, reading its fields from the staged bytes.
//
// A group's 8 outputs take at most four distinct magnitudes (IQ1: s (q + delta) for q = 0, +1,
// -1; IQ2: s g for g = 1, 3, 5, 7), each formed once per lane and rounded exactly as the direct
// formula rounds it, so no int-to-float conversion runs per element. The grid is staged once per
// CTA in the form each family reads fastest (measured on B200, 6M-block launches):
//   IQ1: 16-bit masks (+1 mask | -1 mask << 8); each element selects among its group's three
//        values, and bf16 pairs are rounded in one packed conversion.
//   IQ2: byte-permute selectors, 8 bytes per entry (four 16-bit selectors, one per output pair).
//        For bf16 the four rounded values sit in two registers as a byte table, so an output
//        pair is one byte permute plus one XOR with the pair's sign word, read from a staged
//        table indexed by the group's sign byte (IQ2_XS: by its 7 stored signs, the parity bit
//        folded in). For fp32 each element picks by the 2-bit code inside its selector.
// The selector form is about 5% faster than per-element selects for IQ2 and about 8% slower for
// IQ1_S. Each lane writes its 16 outputs with 32-byte streaming stores (st.global.v8): one for
// bf16, two for fp32.
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

constexpr int kThreads = 256;
constexpr int kMinCtas = 1;      // launch-bounds occupancy hint (CTAs per SM)
constexpr int kTileBlocks = 256;  // blocks per staged payload tile
constexpr int kCtasPerSm = 5;     // persistent CTAs per SM, at most (fewer when shared memory runs out)

template <int FMT>
struct DecodeCfg {
    static constexpr int BYTES = FMT == IQ_FMT_IQ1_S   ? kIq1sBytes
                                 : FMT == IQ_FMT_IQ1_M ? kIq1mBytes
                                 : FMT == IQ_FMT_IQ2_S ? kIq2sBytes
                                                       : kIq2xsBytes;
    static constexpr bool IQ2 = FMT == IQ_FMT_IQ2_XS || FMT == IQ_FMT_IQ2_S;
    static constexpr int E = FMT == IQ_FMT_IQ2_XS ? kIq2xsEntries : FMT == IQ_FMT_IQ2_S ? kIq2sEntries : kIq1sEntries;
    // sign-word table entries: IQ2_XS by its 7 stored sign bits, IQ2_S by its sign byte
    static constexpr int SIGNS = FMT == IQ_FMT_IQ2_XS ? 128 : FMT == IQ_FMT_IQ2_S ? 256 : 0;
    static constexpr int TILE_BYTES = kTileBlocks * BYTES;  // a multiple of 16
    static constexpr int SEL_BYTES = IQ2 ? E * 8 : (E * 2 + 15) / 16 * 16;  // selectors or masks
    static constexpr int SIGN_BYTES = SIGNS * 16;
    static constexpr int smem = SEL_BYTES + SIGN_BYTES + 2 * TILE_BYTES;
};

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

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

// IQ1 grid entry as masks: bit j set when q_j = +1, bit 8 + j when q_j = -1.
__device__ __forceinline__ uint16_t grid_masks(int2 raw) {
    uint32_t m = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
        m |= (static_cast<uint32_t>(v == 1) << j) | (static_cast<uint32_t>(v == -1) << (8 + j));
    }
    return static_cast<uint16_t>(m);
}

// An IQ2 grid entry as four byte-permute selectors, one per output pair (elements 2p, 2p + 1) at
// bits 16p..16p+15 of the 64-bit entry: nibbles (2 c0, 2 c0 + 1, 2 c1, 2 c1 + 1) pick the two
// 16-bit table entries c0, c1, where c = (g - 1) / 2. Values outside {1, 3, 5, 7} are not
// representable here.
__device__ __forceinline__ uint2 grid_selectors(int2 raw) {
    uint32_t sel[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
        const uint32_t c = static_cast<uint32_t>((v - 1) >> 1) & 3u;
        sel[j >> 2] |= ((2u * c) | ((2u * c + 1u) << 4)) << (8 * (j & 3));  // the element's two byte selectors
    }
    return make_uint2(sel[0], sel[1]);
}

// The four sign words of a group whose sign bits are n: bit 2p lands on bit 15 of word p (the
// low output of pair p), bit 2p + 1 on bit 31.
__device__ __forceinline__ uint4 sign_words(uint32_t n) {
    uint32_t w[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) w[p] = (((n >> (2 * p)) & 1u) << 15) | (((n >> (2 * p + 1)) & 1u) << 31);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// A group's 8 bf16 outputs as four packed words from its byte table (lo, hi), its selectors and
// its sign words.
__device__ __forceinline__ void bf16_group(uint32_t lo, uint32_t hi, uint2 sel, uint4 sg, uint32_t* w) {
    w[0] = __byte_perm(lo, hi, sel.x) ^ sg.x;
    w[1] = __byte_perm(lo, hi, sel.x >> 16) ^ sg.y;
    w[2] = __byte_perm(lo, hi, sel.y) ^ sg.z;
    w[3] = __byte_perm(lo, hi, sel.y >> 16) ^ sg.w;
}

// A group's 8 fp32 outputs: element j takes entry c_j of (v0, v1, v2, v3), the code read back
// from its selector, negated when bit j of neg is set.
__device__ __forceinline__ void f32_group(float v0, float v1, float v2, float v3, uint2 sel, uint32_t neg, float* o) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t c = ((j < 4 ? sel.x : sel.y) >> (8 * (j & 3) + 1)) & 3u;
        const float a = (c & 2u) ? ((c & 1u) ? v3 : v2) : ((c & 1u) ? v1 : v0);
        o[j] = ((neg >> j) & 1u) ? -a : a;
    }
}

// A half-warp decodes one block from its staged payload bytes `pb` (2-byte aligned); lane
// h = lane & 15 decodes groups 2h and 2h + 1 (for IQ1_M: exactly choice group h).
template <int FMT, bool BF16>
__device__ __forceinline__ void decode_iq1(const uint8_t* pb, int h, const uint16_t* smask, void* out, int64_t b) {
    const uint16_t* pw = reinterpret_cast<const uint16_t*>(pb);
    float vp[2], v0[2], vn[2];  // per group t of the lane's two: its values for q = +1, 0, -1
    uint32_t m[2];              // its masks
    if (FMT == IQ_FMT_IQ1_M) {
        const uint32_t w0 = pw[24], w1 = pw[25], w2 = pw[26], w3 = pw[27];
        const float d = half_bits_to_f32(iq1m_d_bits(w0, w1, w2, w3));
        const uint32_t wk = pw[24 + (h >> 2)];
        const float s = __fmul_rn(d, small_int_to_float(2u * ((wk >> (3 * (h & 3))) & 7u) + 1u));
        const uint32_t lw = pw[h];       // low index bytes of groups 2h, 2h + 1
        const uint32_t nb = pb[32 + h];  // their nibbles
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t nib = (nb >> (4 * t)) & 15u;
            const float delta = (nib & 8u) ? -0.125f : 0.125f;
            vp[t] = __fmul_rn(s, __fadd_rn(1.0f, delta));
            v0[t] = __fmul_rn(s, __fadd_rn(0.0f, delta));
            vn[t] = __fmul_rn(s, __fadd_rn(-1.0f, delta));
            m[t] = smask[((lw >> (8 * t)) & 0xFFu) | ((nib & 7u) << 8)];
        }
    } else {
        const float d = half_bits_to_f32(pw[0]);
        const uint32_t lw = pw[1 + h];          // low index bytes of groups 2h, 2h + 1
        const uint32_t qh = pw[17 + (h >> 1)];  // the sub-block's qh
        const float s = __fmul_rn(d, small_int_to_float(2u * ((qh >> 12) & 7u) + 1u));
        const float delta = (qh & 0x8000u) ? -0.125f : 0.125f;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            vp[t] = __fmul_rn(s, __fadd_rn(1.0f, delta));
            v0[t] = __fmul_rn(s, __fadd_rn(0.0f, delta));
            vn[t] = __fmul_rn(s, __fadd_rn(-1.0f, delta));
            const int grp = 2 * h + t;
            m[t] = smask[((lw >> (8 * t)) & 0xFFu) | (((qh >> (3 * (grp & 3))) & 7u) << 8)];
        }
    }
    float o[16];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 8; ++j) o[8 * t + j] = ((m[t] >> j) & 1u) ? vp[t] : (((m[t] >> (8 + j)) & 1u) ? vn[t] : v0[t]);
    store16<BF16>(out, b * 32 + 2 * h, o);
}

// The same for IQ2_XS and IQ2_S, from the staged selectors and sign words.
template <int FMT, bool BF16>
__device__ __forceinline__ void decode_iq2(const uint8_t* pb, int h, const uint2* ssel, const uint4* ssgn, void* out,
                                           int64_t b) {
    const uint16_t* pw = reinterpret_cast<const uint16_t*>(pb);
    uint2 sel[2];    // per group t of the lane's two: its selectors
    uint32_t neg[2];  // its sign bits (IQ2_XS: the 7 stored ones)
    const float d = half_bits_to_f32(pw[0]);
    // IQ2_XS scales at byte 66 + h / 2, IQ2_S at 74 + h / 2 (the lane's sub-block h)
    const uint32_t sc = pb[(FMT == IQ_FMT_IQ2_S ? 74 : 66) + (h >> 1)];
    const int ls = static_cast<int>((h & 1) ? (sc >> 4) : (sc & 15u));
    const float s = __fmul_rn(d, small_int_to_float(static_cast<uint32_t>(2 * ls + 1)));
    const float v1 = __fmul_rn(s, 1.0f), v3 = __fmul_rn(s, 3.0f), v5 = __fmul_rn(s, 5.0f), v7 = __fmul_rn(s, 7.0f);
    if (FMT == IQ_FMT_IQ2_S) {
        const uint32_t lw = pw[1 + h];   // low index bytes of groups 2h, 2h + 1
        const uint32_t sg = pw[17 + h];  // their sign bytes
        const uint32_t hb = pb[66 + (h >> 1)] >> (4 * (h & 1));
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            sel[t] = ssel[((lw >> (8 * t)) & 0xFFu) | (((hb >> (2 * t)) & 3u) << 8)];
            neg[t] = (sg >> (8 * t)) & 0xFFu;
        }
    } else {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t cw = pw[1 + 2 * h + t];  // index | sign7 << 9
            sel[t] = ssel[cw & 511u];
            neg[t] = cw >> 9;
        }
    }
    if (BF16) {
        const uint32_t lo = pack_bf16x2(v1, v3), hi = pack_bf16x2(v5, v7);
        uint32_t w[8];
#pragma unroll
        for (int t = 0; t < 2; ++t) bf16_group(lo, hi, sel[t], ssgn[neg[t]], w + 4 * t);
        st_global_v8(reinterpret_cast<uint4*>(out) + b * 32 + 2 * h, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    } else {
        float o[16];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint32_t n = FMT == IQ_FMT_IQ2_XS ? neg[t] | (static_cast<uint32_t>(__popc(neg[t]) & 1) << 7) : neg[t];
            f32_group(v1, v3, v5, v7, sel[t], n, o + 8 * t);
        }
        store16<false>(out, b * 32 + 2 * h, o);
    }
}

template <int FMT, bool BF16>
__global__ void __launch_bounds__(kThreads, kMinCtas) decode_kernel(const DecodeParams p) {
    using C = DecodeCfg<FMT>;
    extern __shared__ __align__(16) char smem[];
    uint2* ssel = reinterpret_cast<uint2*>(smem);       // IQ2: selectors
    uint16_t* smask = reinterpret_cast<uint16_t*>(smem);  // IQ1: masks
    uint4* ssgn = reinterpret_cast<uint4*>(smem + C::SEL_BYTES);
    uint8_t* tiles = reinterpret_cast<uint8_t*>(smem + C::SEL_BYTES + C::SIGN_BYTES);
    for (int q = threadIdx.x; q < C::E; q += kThreads) {
        const int2 raw = __ldg(reinterpret_cast<const int2*>(p.grid) + q);
        if (C::IQ2) ssel[q] = grid_selectors(raw);
        else smask[q] = grid_masks(raw);
    }
    for (int q = threadIdx.x; q < C::SIGNS; q += kThreads) {
        const uint32_t n = FMT == IQ_FMT_IQ2_XS ? q | (static_cast<uint32_t>(__popc(q) & 1) << 7) : q;
        ssgn[q] = sign_words(n);
    }

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
        {
            if (C::IQ2) decode_iq2<FMT, BF16>(tile + k * C::BYTES, h, ssel, ssgn, p.out, t * kTileBlocks + k);
            else decode_iq1<FMT, BF16>(tile + k * C::BYTES, h, smask, p.out, t * kTileBlocks + k);
        }
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
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, C::smem);
    if (err != cudaSuccess) return err;
    if (per_sm > kCtasPerSm) per_sm = kCtasPerSm;
    if (per_sm < 1) per_sm = 1;
    const int64_t ntiles = (p.nblocks + kTileBlocks - 1) / kTileBlocks;
    const int64_t cap = static_cast<int64_t>(per_sm) * num_sms;
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

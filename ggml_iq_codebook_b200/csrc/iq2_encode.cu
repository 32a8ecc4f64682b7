// iq2_encode.cu -- IQ2_XS and IQ2_S encoders: weighted exhaustive magnitude search + pack.
//
// Method (PR #2450 review comments; IQ2_S codec commit text on the PR #2525 page): 32 groups of
// 8 weights per 256-weight block, each coded as a 9-bit index into a 512 x 8 magnitude grid plus
// a 7-bit sign mask whose 8th sign is implied by even parity; one 4-bit local scale ls per 16
// weights, s = d (2 ls + 1). Signs come from x; an odd count of negatives is fixed by flipping
// the weakest element, then the search runs on magnitudes.
//
// Score convention (identical, op for op, to the CPU oracle):
//   signs   neg_j = x_j < 0; if popcount(neg) is odd, flip k = argmin_j (x_j x_j) w_j (lowest j)
//   target  a_j = |x_j|, a_k = -|x_k| for the flipped k;  V_j = -2 (w_j a_j)
//   entry   A = w_0 g_0^2, then A = fma(w_j, g_j^2, A) for j = 1..7;
//           B = V_0 g_0,  then B = fma(V_j, g_j, B);   m = fma(s, A, B)
//   argmin_g m (lowest entry on ties); e = s m_min; sub-block E = e_even + e_odd; argmin_ls E.
//
// IQ2_S (PR #2512 codec, PR #2565 CUDA encoder commit texts): a 1024-entry grid and eight sign
// bits for each group, so the input's signs are kept (nothing is flipped) and a_j = |x_j|; the
// 82-byte block holds d, the low index bytes, the sign bytes, the 2-bit high index fields (group
// g at shift 2 (g % 4) of byte 66 + g/4) and the scale nibbles at bytes 74..81.
//
// Kernel design (B200): one warp per block, one lane per group; the entry loop (512 entries for
// IQ2_XS, 1024 for IQ2_S) is warp-uniform and reads each entry's 8 magnitudes and 8 squares
// (64 B) with broadcast 16-byte shared-memory loads. Argmin bookkeeping as in the IQ1_S kernel: running minima, chunk of first appearance,
// one-chunk rescan for the index; the rescans, whose entries differ from lane to lane, read a
// packed 8-byte copy of the grid instead of the 64-byte float rows.
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

constexpr int kWarps = 8;

template <int FMT>
struct Iq2Cfg {
    static constexpr bool S = FMT == IQ_FMT_IQ2_S;
    static constexpr int E = S ? kIq2sEntries : kIq2xsEntries;
    static constexpr int BYTES = S ? kIq2sBytes : kIq2xsBytes;
    static constexpr int FLOAT_GRID_BYTES = E * 16 * 4;           // per entry: g[8] then g^2[8] as fp32
    static constexpr int SMEM = FLOAT_GRID_BYTES + E * 8;         // + the packed int8 grid
};

struct Entry {
    float g[8], gg[8];
};

__device__ __forceinline__ void load_entry(const float4* sg, int q, Entry& en) {
    const float4 a = sg[4 * q], b = sg[4 * q + 1], c = sg[4 * q + 2], d = sg[4 * q + 3];
    en.g[0] = a.x; en.g[1] = a.y; en.g[2] = a.z; en.g[3] = a.w;
    en.g[4] = b.x; en.g[5] = b.y; en.g[6] = b.z; en.g[7] = b.w;
    en.gg[0] = c.x; en.gg[1] = c.y; en.gg[2] = c.z; en.gg[3] = c.w;
    en.gg[4] = d.x; en.gg[5] = d.y; en.gg[6] = d.z; en.gg[7] = d.w;
}

// The same entry rebuilt from the packed int8 grid (one 8-byte read): the rescans of single
// chunks read entries at lane-dependent addresses, where 8 bytes beat 64. (Converting with the
// exact bit trick instead of int-to-float conversions measured slower here.)
__device__ __forceinline__ void load_entry_packed(const int2* sp, int q, Entry& en) {
    const int2 raw = sp[q];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        en.g[j] = static_cast<float>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
        en.gg[j] = __fmul_rn(en.g[j], en.g[j]);
    }
}

__device__ __forceinline__ void entry_AB(const Entry& en, const float w[8], const float V[8], float& A,
                                         float& B) {
    A = __fmul_rn(w[0], en.gg[0]);
    B = __fmul_rn(V[0], en.g[0]);
#pragma unroll
    for (int j = 1; j < 8; ++j) {
        A = __fmaf_rn(w[j], en.gg[j], A);
        B = __fmaf_rn(V[j], en.g[j], B);
    }
}

template <int BYTES>
__device__ __forceinline__ void write_zero_block(uint8_t* out, int lane) {
    for (int i = lane; i < BYTES / 2; i += 32) reinterpret_cast<uint16_t*>(out)[i] = 0;
}

// lane = group: code = idx | sign7 << 9; ls = its sub-block's local scale.
__device__ __forceinline__ void pack_block(uint8_t* out, int lane, int idx, uint32_t neg, int ls,
                                           uint16_t d_half) {
    *reinterpret_cast<uint16_t*>(out + 2 + 2 * lane) =
        static_cast<uint16_t>(static_cast<uint32_t>(idx) | ((neg & 0x7Fu) << 9));
    const int hi = __shfl_down_sync(0xffffffffu, ls, 2);  // sub-block 2i+1 sits 2 lanes up
    if ((lane & 3) == 0) out[66 + (lane >> 2)] = static_cast<uint8_t>(ls | (hi << 4));
    if (lane == 0) *reinterpret_cast<uint16_t*>(out) = d_half;
}

// IQ2_S: lane = group: low index byte, sign byte, 2 high index bits (4 groups per byte), and the
// sub-block's scale nibble.
__device__ __forceinline__ void pack_block_s(uint8_t* out, int lane, int idx, uint32_t neg, int ls,
                                             uint16_t d_half) {
    out[2 + lane] = static_cast<uint8_t>(idx & 0xFF);
    out[34 + lane] = static_cast<uint8_t>(neg);
    uint32_t v = static_cast<uint32_t>((idx >> 8) & 3) << (2 * (lane & 3));
    v |= __shfl_xor_sync(0xffffffffu, v, 1);
    v |= __shfl_xor_sync(0xffffffffu, v, 2);
    const int hi = __shfl_down_sync(0xffffffffu, ls, 2);  // sub-block 2i+1 sits 2 lanes up
    if ((lane & 3) == 0) {
        out[66 + (lane >> 2)] = static_cast<uint8_t>(v);
        out[74 + (lane >> 2)] = static_cast<uint8_t>(ls | (hi << 4));
    }
    if (lane == 0) *reinterpret_cast<uint16_t*>(out) = d_half;
}

template <int FMT>
__device__ __forceinline__ void pack(uint8_t* out, int lane, int idx, uint32_t neg, int ls, uint16_t d_half) {
    if (Iq2Cfg<FMT>::S) pack_block_s(out, lane, idx, neg, ls, d_half);
    else pack_block(out, lane, idx, neg, ls, d_half);
}

template <int FMT, int MODE, int K, bool BF16IN>
__global__ void __launch_bounds__(kWarps * 32, 2) iq2_encode_kernel(const EncodeParams p) {
    using Cfg = Iq2Cfg<FMT>;
    extern __shared__ __align__(16) char smem[];
    float* sgf = reinterpret_cast<float*>(smem);
    const float4* sg = reinterpret_cast<const float4*>(smem);
    int2* sgp = reinterpret_cast<int2*>(smem + Cfg::FLOAT_GRID_BYTES);

    bool bad = false;
    for (int q = threadIdx.x; q < Cfg::E; q += blockDim.x) {
        const int2 raw = __ldg(reinterpret_cast<const int2*>(p.grid) + q);
        sgp[q] = raw;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
            bad |= !(v == 1 || v == 3 || v == 5 || v == 7);
            sgf[16 * q + j] = static_cast<float>(v);
            sgf[16 * q + 8 + j] = static_cast<float>(v * v);
        }
    }
    bad = __syncthreads_or(bad);
    if (bad && threadIdx.x == 0) raise_flags(p.flags, IQ_FLAG_GRID);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t per_batch = p.rows * p.nblk;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;

    for (int64_t b = static_cast<int64_t>(blockIdx.x) * kWarps + warp; b < p.nb; b += stride) {
        const int64_t e = b / per_batch, rem = b - e * per_batch;
        const int64_t r = rem / p.nblk, blk = rem - r * p.nblk;
        uint8_t* out = p.payload + b * Cfg::BYTES;
        const int64_t every_stride = p.nb * Cfg::BYTES;

        float x[8], w[8];
        load_weights8<BF16IN>(p.w, p.w_dtype, e * p.w_bstride + r * p.ldw + blk * kBlock + 8 * lane, x);
        if (p.imp != nullptr) {
            const float4* ip = reinterpret_cast<const float4*>(p.imp + e * p.imp_bstride + blk * kBlock) + 2 * lane;
            const float4 a = __ldg(ip), c = __ldg(ip + 1);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = c.x; w[5] = c.y; w[6] = c.z; w[7] = c.w;
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) w[j] = 1.0f;
        }
        uint32_t f = 0;
        float am = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (!isfinite(x[j])) f |= IQ_FLAG_NONFINITE;
            else am = fmaxf(am, fabsf(x[j]));
            if (!isfinite(w[j]) || w[j] < 0.0f) f |= IQ_FLAG_IMPORTANCE;
        }
        int fixed_c = 0;
        if (MODE == kFixed) {
            fixed_c = p.choices[b * 16 + (lane >> 1)];
            if (fixed_c >= kChoices) f |= IQ_FLAG_CHOICE;
        }
        f = __reduce_or_sync(0xffffffffu, f);
        const float amax = warp_max(am);
        uint16_t d_half = 0;
        if (p.scales != nullptr) {
            d_half = __ldg(p.scales + b * p.scales_stride);
            if (given_d_bad(d_half)) f |= IQ_FLAG_RANGE;
        } else if (f == 0 && !bad) {
            d_half = predict_d(amax, 217.0f, p.anchor);
            if ((d_half & 0x7FFFu) == 0x7C00u) f = IQ_FLAG_RANGE;
        }
        if (f != 0 || bad || (d_half & 0x7FFFu) == 0) {
            if (MODE == kEvery) {
                for (int c = 0; c < kChoices; ++c) write_zero_block<Cfg::BYTES>(out + c * every_stride, lane);
            } else {
                write_zero_block<Cfg::BYTES>(out, lane);
            }
            if (lane == 0) raise_flags(p.flags, f);
            continue;
        }
        const float d = half_bits_to_f32(d_half);

        // ---- signs with even parity, magnitudes as targets
        uint32_t neg = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) neg |= static_cast<uint32_t>(x[j] < 0.0f) << j;
        int flipped = -1;
        if (!Cfg::S && (__popc(neg) & 1)) {
            int k = 0;
            float tk = __fmul_rn(__fmul_rn(x[0], x[0]), w[0]);
#pragma unroll
            for (int j = 1; j < 8; ++j) {
                const float tj = __fmul_rn(__fmul_rn(x[j], x[j]), w[j]);
                if (tj < tk) { tk = tj; k = j; }
            }
            neg ^= 1u << k;
            flipped = k;
        }
        float V[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float a = (j == flipped) ? -fabsf(x[j]) : fabsf(x[j]);
            V[j] = __fmul_rn(-2.0f, __fmul_rn(w[j], a));
        }
        float s[16];
#pragma unroll
        for (int ls = 0; ls < 16; ++ls) s[ls] = __fmul_rn(d, static_cast<float>(2 * ls + 1));

        if constexpr (MODE == kFixed) {
            float sv = s[0];
#pragma unroll
            for (int ls = 1; ls < 16; ++ls) if (fixed_c == ls) sv = s[ls];
            float best = INFINITY;
            int bi = 0;
#pragma unroll 2
            for (int q = 0; q < Cfg::E; ++q) {
                Entry en;
                load_entry(sg, q, en);
                float A, B;
                entry_AB(en, w, V, A, B);
                const float m = __fmaf_rn(sv, A, B);
                if (m < best) { best = m; bi = q; }
            }
            pack<FMT>(out, lane, bi, neg, fixed_c, d_half);
        } else {
            float best[kChoices];
            int bch[kChoices];
#pragma unroll
            for (int c = 0; c < kChoices; ++c) { best[c] = INFINITY; bch[c] = 0; }
            for (int ch = 0; ch < Cfg::E / K; ++ch) {
                float cm[kChoices];
                {
                    Entry ea, eb;
                    load_entry(sg, ch * K, ea);
                    load_entry(sg, ch * K + 1, eb);
                    float Aa, Ba, Ab, Bb;
                    entry_AB(ea, w, V, Aa, Ba);
                    entry_AB(eb, w, V, Ab, Bb);
#pragma unroll
                    for (int c = 0; c < kChoices; ++c) cm[c] = fminf(__fmaf_rn(s[c], Aa, Ba), __fmaf_rn(s[c], Ab, Bb));
                }
#pragma unroll 1
                for (int q = ch * K + 2; q < ch * K + K; q += 2) {
                    Entry ea, eb;
                    load_entry(sg, q, ea);
                    load_entry(sg, q + 1, eb);
                    float Aa, Ba, Ab, Bb;
                    entry_AB(ea, w, V, Aa, Ba);
                    entry_AB(eb, w, V, Ab, Bb);
#pragma unroll
                    for (int c = 0; c < kChoices; ++c)
                        cm[c] = min3f(cm[c], __fmaf_rn(s[c], Aa, Ba), __fmaf_rn(s[c], Ab, Bb));
                }
#pragma unroll
                for (int c = 0; c < kChoices; ++c) {
                    if (cm[c] < best[c]) { best[c] = cm[c]; bch[c] = ch; }
                }
            }

            auto entry_of = [&](int c) -> int {
                float target = best[0], sv = s[0];
                int ch = bch[0];
#pragma unroll
                for (int k = 1; k < kChoices; ++k) if (k == c) { target = best[k]; ch = bch[k]; sv = s[k]; }
                if (!(target < INFINITY)) return 0;
                for (int q = ch * K; q < ch * K + K; ++q) {
                    Entry en;
                    load_entry_packed(sgp, q, en);
                    float A, B;
                    entry_AB(en, w, V, A, B);
                    if (__fmaf_rn(sv, A, B) == target) return q;
                }
                return ch * K;  // not reached: the same arithmetic reproduces target
            };

            if (MODE == kEvery) {
                for (int c = 0; c < kChoices; ++c) pack<FMT>(out + c * every_stride, lane, entry_of(c), neg, c, d_half);
                continue;
            }

            int cstar = 0;
            float bestE = INFINITY;
#pragma unroll
            for (int c = 0; c < kChoices; ++c) {
                const float e0 = __fmul_rn(s[c], best[c]);
                const float E = __fadd_rn(e0, __shfl_xor_sync(0xffffffffu, e0, 1));
                if (E < bestE) { bestE = E; cstar = c; }
            }
            pack<FMT>(out, lane, entry_of(cstar), neg, cstar, d_half);
        }
    }
}

template <int FMT, int MODE, int K>
cudaError_t launch_mode(const EncodeParams& p, int num_sms, cudaStream_t s) {
    constexpr int smem = Iq2Cfg<FMT>::SMEM;
    auto kern = p.w_dtype == IQ_IN_BF16 ? iq2_encode_kernel<FMT, MODE, K, true> : iq2_encode_kernel<FMT, MODE, K, false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    const int64_t ctas_needed = (p.nb + kWarps - 1) / kWarps;
    const int64_t ctas = ctas_needed < 2LL * num_sms ? ctas_needed : 2LL * num_sms;
    kern<<<static_cast<unsigned>(ctas), kWarps * 32, smem, s>>>(p);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(const EncodeParams& p, int mode, int num_sms, cudaStream_t s) {
    switch (mode) {
        case kSearch: return launch_mode<FMT, kSearch, 32>(p, num_sms, s);
        case kFixed: return launch_mode<FMT, kFixed, 32>(p, num_sms, s);
        default: return launch_mode<FMT, kEvery, 8>(p, num_sms, s);
    }
}

}  // namespace

cudaError_t launch_iq2_encode(int fmt, const EncodeParams& p, int mode, int num_sms, cudaStream_t s) {
    if (p.nb == 0) return cudaSuccess;
    return fmt == IQ_FMT_IQ2_S ? launch_fmt<IQ_FMT_IQ2_S>(p, mode, num_sms, s)
                               : launch_fmt<IQ_FMT_IQ2_XS>(p, mode, num_sms, s);
}

}  // namespace iqk

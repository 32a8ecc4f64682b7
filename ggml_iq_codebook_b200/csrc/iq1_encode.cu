// iq1_encode.cu -- IQ1_S and IQ1_M encoders: weighted exhaustive shifted-grid search + pack
// (sm_100a).
//
// Method (PR #2723 "Weight the IQ1 encoders by the square root of GPTQ's Hessian diagonal";
// PR #2450 review comments): each 8-weight group x is approximated by s (q + delta) with q one
// of 2048 ternary grid entries, delta = +-1/8 and s = d (2 ls + 1), ls in 0..7. The local scale
// and delta are shared by the 4 groups of a 32-weight sub-block (16 choices c = ls + 8 [delta<0]);
// each group picks its own entry. The objective is sum_j w_j (x_j - s (q_j + delta))^2.
//
// Score convention (identical, op for op, to the CPU oracle):
//   per group  T_j = -2 (w_j x_j);  S(v, M) = (sum over M's low-nibble bits, ascending from 0)
//              + (sum over its high-nibble bits, ascending from 0);  W = S(w, all), Tall = S(T, all)
//   per entry  P/N = positions of +1/-1;  A = S(w,P) + S(w,N);  R = S(w,P) - S(w,N);
//              C = S(T,P) - S(T,N)
//   per choice A_delta = fma(delta^2, W, fma(2 delta, R, A));  C_delta = fma(delta, Tall, C);
//              m = fma(s, A_delta, C_delta)
//   per (group, c)     argmin_q m (lowest q on ties), e = s * m_min
//   per (sub-block, c) E = (e0 + e1) + (e2 + e3);  choice = argmin_c E (lowest c on ties)
//
// IQ1_M (PR #2513 codec, PR #2595 CUDA encoder commit texts) runs the same search and selects
// differently: a choice group is two 8-weight groups sharing ls (8 choices); per group and ls the
// delta with the smaller m wins (+1/8 on equal m), e = s * m, E = e_even + e_odd, lowest ls on
// ties. Its d anchor is clamp(0.58 + 0.035 amax / rms, 0.65, 0.95), with rms = sqrt(ss / 256):
// each lane sums its 8 squares in order, the 32 lane sums meet in the xor-butterfly tree.
//
// Kernel design (B200): one warp per 256-weight block, one lane per group, so the 2048-entry
// loop is warp-uniform: the entry's four subset-sum row offsets come from one broadcast
// shared-memory read, and each lane then reads its own group's nibble tables (S(w), S(T) for the
// 16 low and 16 high nibble values, 8 KiB per warp, conflict-free rows). The argmin keeps only
// running minima (fminf) in registers plus the chunk of K entries where each choice's minimum
// first appeared (two candidates fold into one three-input min); the winning entry index is
// recovered afterwards by rescanning that one chunk with the identical arithmetic. Persistent
// CTAs walk the blocks with a static stride: every block costs the same, so no work queue (and
// no scratch memory) is needed. Weights arrive as bf16 (its own instantiation), f16 or fp32, all
// converted exactly; d is predicted from amax or given per block (static scales, PR #3197).
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

constexpr int kWarps = 8;                      // warps per CTA
constexpr int kGridBytes = kIq1sEntries * 16;  // uint4 of 4 table-row byte offsets per entry
constexpr int kTabBytes = 32 * 32 * 8;         // 32 rows x 32 lanes x float2, per warp
constexpr int kSmemBytes = kGridBytes + kWarps * kTabBytes;

template <int FMT>
struct Iq1Cfg {
    static constexpr bool M = FMT == IQ_FMT_IQ1_M;
    static constexpr int BYTES = M ? kIq1mBytes : kIq1sBytes;
    static constexpr int NCH = M ? kIq1mChoices : kChoices;  // choices per choice group
    static constexpr int G = M ? 16 : 8;                     // choice groups per block
    static constexpr int LANES_PER_CHOICE = 32 / G;          // groups (lanes) per choice group
};

struct Terms {
    float Ap, An, Cp, Cn;  // A_delta and C_delta for delta = +1/8 and -1/8
};

// Subset-sum terms of one grid entry for this lane's group.
__device__ __forceinline__ Terms entry_terms(const char* smem, uint32_t lane_base, uint4 o, float W,
                                             float Tall) {
    const float2 plo = *reinterpret_cast<const float2*>(smem + lane_base + o.x);
    const float2 phi = *reinterpret_cast<const float2*>(smem + lane_base + o.y);
    const float2 nlo = *reinterpret_cast<const float2*>(smem + lane_base + o.z);
    const float2 nhi = *reinterpret_cast<const float2*>(smem + lane_base + o.w);
    const float Wp = __fadd_rn(plo.x, phi.x), Tp = __fadd_rn(plo.y, phi.y);
    const float Wn = __fadd_rn(nlo.x, nhi.x), Tn = __fadd_rn(nlo.y, nhi.y);
    const float A = __fadd_rn(Wp, Wn), R = __fsub_rn(Wp, Wn), C = __fsub_rn(Tp, Tn);
    Terms t;
    t.Ap = __fmaf_rn(0.015625f, W, __fmaf_rn(0.25f, R, A));
    t.An = __fmaf_rn(0.015625f, W, __fmaf_rn(-0.25f, R, A));
    t.Cp = __fmaf_rn(0.125f, Tall, C);
    t.Cn = __fmaf_rn(-0.125f, Tall, C);
    return t;
}

// The same terms with both shifts side by side, A = (A_+, A_-) and C = (C_+, C_-), so that one
// packed fma.rn.f32x2 scores an entry under both shifts of a local scale. Every element is the
// scalar version's op sequence (the packed ops are independent IEEE operations per element).
struct Terms2 {
    float2 A, C;
};

__device__ __forceinline__ Terms2 entry_terms2(const char* smem, uint32_t lane_base, uint4 o, float2 W2,
                                               float Tall) {
    const float2 plo = *reinterpret_cast<const float2*>(smem + lane_base + o.x);
    const float2 phi = *reinterpret_cast<const float2*>(smem + lane_base + o.y);
    const float2 nlo = *reinterpret_cast<const float2*>(smem + lane_base + o.z);
    const float2 nhi = *reinterpret_cast<const float2*>(smem + lane_base + o.w);
    const float2 p = __fadd2_rn(plo, phi), n = __fadd2_rn(nlo, nhi);  // (Wp, Tp), (Wn, Tn)
    const float A = __fadd_rn(p.x, n.x), R = __fsub_rn(p.x, n.x), C = __fsub_rn(p.y, n.y);
    Terms2 t;
    t.A = __ffma2_rn(make_float2(0.015625f, 0.015625f), W2,
                     make_float2(__fmaf_rn(0.25f, R, A), __fmaf_rn(-0.25f, R, A)));
    t.C = make_float2(__fmaf_rn(0.125f, Tall, C), __fmaf_rn(-0.125f, Tall, C));
    return t;
}

template <int BYTES>
__device__ __forceinline__ void write_zero_block(uint8_t* out, int lane) {
    for (int i = lane; i < BYTES / 2; i += 32) reinterpret_cast<uint16_t*>(out)[i] = 0;
}

// Pack one block: lane = group, idx = its entry, c = its sub-block's choice.
__device__ __forceinline__ void pack_block(uint8_t* out, int lane, int idx, int c, uint16_t d_half) {
    uint32_t v = static_cast<uint32_t>((idx >> 8) & 7) << (3 * (lane & 3));
    v |= __shfl_xor_sync(0xffffffffu, v, 1);
    v |= __shfl_xor_sync(0xffffffffu, v, 2);
    const uint32_t qh = v | (static_cast<uint32_t>(c & 7) << 12) | (static_cast<uint32_t>(c >> 3) << 15);
    out[2 + lane] = static_cast<uint8_t>(idx & 0xFF);
    if ((lane & 3) == 0) *reinterpret_cast<uint16_t*>(out + 34 + 2 * (lane >> 2)) = static_cast<uint16_t>(qh);
    if (lane == 0) *reinterpret_cast<uint16_t*>(out) = d_half;
}

// Pack one IQ1_M block: lane = group, idx = its entry, neg = its delta bit, ls = its choice
// group's local scale. Bytes 0..31 low index bytes; 32..47 a nibble per group (even group low);
// 48..55 four scale words: ls of choice groups 4i..4i+3 at shifts 0,3,6,9, d's nibble i on top.
__device__ __forceinline__ void pack_block_m(uint8_t* out, int lane, int idx, int ls, int neg, uint16_t d_half) {
    out[lane] = static_cast<uint8_t>(idx & 0xFF);
    uint32_t v = (static_cast<uint32_t>((idx >> 8) & 7) | (static_cast<uint32_t>(neg) << 3)) << (4 * (lane & 1));
    v |= __shfl_xor_sync(0xffffffffu, v, 1);
    if ((lane & 1) == 0) out[32 + (lane >> 1)] = static_cast<uint8_t>(v);
    uint32_t wv = (lane & 1) ? 0u : static_cast<uint32_t>(ls) << (3 * ((lane >> 1) & 3));
    wv |= __shfl_xor_sync(0xffffffffu, wv, 1);
    wv |= __shfl_xor_sync(0xffffffffu, wv, 2);
    wv |= __shfl_xor_sync(0xffffffffu, wv, 4);
    if ((lane & 7) == 0) {
        const int i = lane >> 3;
        *reinterpret_cast<uint16_t*>(out + 48 + 2 * i) =
            static_cast<uint16_t>(wv | ((static_cast<uint32_t>(d_half >> (4 * i)) & 15u) << 12));
    }
}

template <int FMT, int MODE, int K, bool BF16IN>
__global__ void __launch_bounds__(kWarps * 32, 2) iq1_encode_kernel(const EncodeParams p) {
    using Cfg = Iq1Cfg<FMT>;
    extern __shared__ __align__(16) char smem[];
    uint4* sgrid = reinterpret_cast<uint4*>(smem);

    // Grid prologue: per entry, the byte offsets of its four table rows
    // (low nibble of P, high nibble of P, low nibble of N, high nibble of N).
    bool bad = false;
    for (int q = threadIdx.x; q < kIq1sEntries; q += blockDim.x) {
        const int2 raw = __ldg(reinterpret_cast<const int2*>(p.grid) + q);
        uint32_t pos = 0, neg = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
            pos |= static_cast<uint32_t>(v == 1) << j;
            neg |= static_cast<uint32_t>(v == -1) << j;
            bad |= (v < -1) || (v > 1);
        }
        sgrid[q] = make_uint4((pos & 15u) << 8, (16u + (pos >> 4)) << 8, (neg & 15u) << 8,
                              (16u + (neg >> 4)) << 8);
    }
    bad = __syncthreads_or(bad);
    if (bad && threadIdx.x == 0) raise_flags(p.flags, IQ_FLAG_GRID);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lane_base = kGridBytes + warp * kTabBytes + lane * 8;
    const int64_t per_batch = p.rows * p.nblk;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;

    for (int64_t b = static_cast<int64_t>(blockIdx.x) * kWarps + warp; b < p.nb; b += stride) {
        const int64_t e = b / per_batch, rem = b - e * per_batch;
        const int64_t r = rem / p.nblk, blk = rem - r * p.nblk;
        uint8_t* out = p.payload + b * Cfg::BYTES;
        const int64_t every_stride = p.nb * Cfg::BYTES;

        // ---- load + validate (8 weights and importances per lane, 16-byte vector loads)
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
            fixed_c = p.choices[b * Cfg::G + lane / Cfg::LANES_PER_CHOICE];
            if (fixed_c >= Cfg::NCH) f |= IQ_FLAG_CHOICE;
        }
        f = __reduce_or_sync(0xffffffffu, f);
        const float amax = warp_max(am);
        uint16_t d_half = 0;
        if (p.scales != nullptr) {
            d_half = __ldg(p.scales + b * p.scales_stride);
            if (given_d_bad(d_half)) f |= IQ_FLAG_RANGE;
        } else if (f == 0 && !bad) {
            float anchor = p.anchor;
            if (Cfg::M) {
                float ss = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) ss = __fadd_rn(ss, __fmul_rn(x[j], x[j]));
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
                const float rms = __fsqrt_rn(__fdiv_rn(ss, 256.0f));
                const float ratio = __fdiv_rn(amax, rms);
                anchor = fminf(fmaxf(__fadd_rn(0.58f, __fmul_rn(0.035f, ratio)), 0.65f), 0.95f);
            }
            d_half = predict_d(amax, 16.875f, anchor);
            if ((d_half & 0x7FFFu) == 0x7C00u) f = IQ_FLAG_RANGE;
        }
        if (f != 0 || bad || (d_half & 0x7FFFu) == 0) {
            if (MODE == kEvery) {
                for (int c = 0; c < Cfg::NCH; ++c) write_zero_block<Cfg::BYTES>(out + c * every_stride, lane);
            } else {
                write_zero_block<Cfg::BYTES>(out, lane);
            }
            if (lane == 0) raise_flags(p.flags, f);
            continue;
        }
        const float d = half_bits_to_f32(d_half);

        // ---- per-group nibble subset-sum tables: rows 0..15 low nibble, 16..31 high nibble
        float t[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = __fmul_rn(-2.0f, __fmul_rn(w[j], x[j]));
        float lw[16], lt[16], hw[16], ht[16];
        lw[0] = 0.0f; lt[0] = 0.0f; hw[0] = 0.0f; ht[0] = 0.0f;
#pragma unroll
        for (int bit = 0; bit < 4; ++bit) {
#pragma unroll
            for (int k = 1 << bit; k < (2 << bit); ++k) {
                lw[k] = __fadd_rn(lw[k - (1 << bit)], w[bit]);
                lt[k] = __fadd_rn(lt[k - (1 << bit)], t[bit]);
                hw[k] = __fadd_rn(hw[k - (1 << bit)], w[4 + bit]);
                ht[k] = __fadd_rn(ht[k - (1 << bit)], t[4 + bit]);
            }
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            *reinterpret_cast<float2*>(smem + lane_base + k * 256) = make_float2(lw[k], lt[k]);
            *reinterpret_cast<float2*>(smem + lane_base + (16 + k) * 256) = make_float2(hw[k], ht[k]);
        }
        const float W = __fadd_rn(lw[15], hw[15]);
        const float Tall = __fadd_rn(lt[15], ht[15]);
        float s[8];
#pragma unroll
        for (int ls = 0; ls < 8; ++ls) s[ls] = __fmul_rn(d, static_cast<float>(2 * ls + 1));

        if constexpr (MODE == kFixed) {
            if constexpr (Cfg::M) {
                // The lane's local scale is given; both deltas are searched, each keeping its lowest
                // entry, and the negative shift wins only with a strictly smaller m.
                float sv = s[0];
#pragma unroll
                for (int ls = 1; ls < 8; ++ls) if (fixed_c == ls) sv = s[ls];
                float bp = INFINITY, bn = INFINITY;
                int qp = 0, qn = 0;
#pragma unroll 4
                for (int q = 0; q < kIq1sEntries; ++q) {
                    const Terms tm = entry_terms(smem, lane_base, sgrid[q], W, Tall);
                    const float mp = __fmaf_rn(sv, tm.Ap, tm.Cp), mn = __fmaf_rn(sv, tm.An, tm.Cn);
                    if (mp < bp) { bp = mp; qp = q; }
                    if (mn < bn) { bn = mn; qn = q; }
                }
                const int neg = bn < bp;
                pack_block_m(out, lane, neg ? qn : qp, fixed_c, neg, d_half);
            } else {
                // One choice per lane: direct argmin with the index (lowest entry on ties).
                float sv = s[0];
#pragma unroll
                for (int ls = 1; ls < 8; ++ls) if ((fixed_c & 7) == ls) sv = s[ls];
                const bool negd = fixed_c >= 8;
                float best = INFINITY;
                int bi = 0;
#pragma unroll 4
                for (int q = 0; q < kIq1sEntries; ++q) {
                    const Terms tm = entry_terms(smem, lane_base, sgrid[q], W, Tall);
                    const float m = negd ? __fmaf_rn(sv, tm.An, tm.Cn) : __fmaf_rn(sv, tm.Ap, tm.Cp);
                    if (m < best) { best = m; bi = q; }
                }
                pack_block(out, lane, bi, fixed_c, d_half);
            }
        } else {
            // ---- search: running minima per choice, chunk of first appearance
            float best[kChoices];
            int bch[kChoices];
#pragma unroll
            for (int c = 0; c < kChoices; ++c) { best[c] = INFINITY; bch[c] = 0; }
            // m for both shifts of a local scale in one packed fma: (s, s) * (A_+, A_-) + (C_+, C_-)
            const float2 W2 = make_float2(W, W);
            float2 s2[8];
#pragma unroll
            for (int ls = 0; ls < 8; ++ls) s2[ls] = make_float2(s[ls], s[ls]);
            for (int ch = 0; ch < kIq1sEntries / K; ++ch) {
                float cm[kChoices];
                {
                    const Terms2 ta = entry_terms2(smem, lane_base, sgrid[ch * K], W2, Tall);
                    const Terms2 tb = entry_terms2(smem, lane_base, sgrid[ch * K + 1], W2, Tall);
#pragma unroll
                    for (int ls = 0; ls < 8; ++ls) {
                        const float2 ma = __ffma2_rn(s2[ls], ta.A, ta.C), mb = __ffma2_rn(s2[ls], tb.A, tb.C);
                        cm[ls] = fminf(ma.x, mb.x);
                        cm[8 + ls] = fminf(ma.y, mb.y);
                    }
                }
#pragma unroll 2
                for (int q = ch * K + 2; q < ch * K + K; q += 2) {
                    const Terms2 ta = entry_terms2(smem, lane_base, sgrid[q], W2, Tall);
                    const Terms2 tb = entry_terms2(smem, lane_base, sgrid[q + 1], W2, Tall);
#pragma unroll
                    for (int ls = 0; ls < 8; ++ls) {
                        const float2 ma = __ffma2_rn(s2[ls], ta.A, ta.C), mb = __ffma2_rn(s2[ls], tb.A, tb.C);
                        cm[ls] = min3f(cm[ls], ma.x, mb.x);
                        cm[8 + ls] = min3f(cm[8 + ls], ma.y, mb.y);
                    }
                }
#pragma unroll
                for (int c = 0; c < kChoices; ++c) {
                    if (cm[c] < best[c]) { best[c] = cm[c]; bch[c] = ch; }
                }
            }

            // Recover the first entry of choice c that reached best[c] (0 if nothing beat +inf).
            auto entry_of = [&](int c) -> int {
                float target = best[0];
                int ch = bch[0];
                float sv = s[0];
#pragma unroll
                for (int k = 1; k < kChoices; ++k) if (k == c) { target = best[k]; ch = bch[k]; }
#pragma unroll
                for (int ls = 1; ls < 8; ++ls) if ((c & 7) == ls) sv = s[ls];
                if (!(target < INFINITY)) return 0;
                const bool negd = c >= 8;
                for (int q = ch * K; q < ch * K + K; ++q) {
                    const Terms tm = entry_terms(smem, lane_base, sgrid[q], W, Tall);
                    const float m = negd ? __fmaf_rn(sv, tm.An, tm.Cn) : __fmaf_rn(sv, tm.Ap, tm.Cp);
                    if (m == target) return q;
                }
                return ch * K;  // not reached: the same arithmetic reproduces target
            };

            if (Cfg::M) {
                // per ls: the group's delta (bit ls of negmask: -1/8 only with a strictly smaller m)
                uint32_t negmask = 0;
#pragma unroll
                for (int ls = 0; ls < kIq1mChoices; ++ls) negmask |= static_cast<uint32_t>(best[8 + ls] < best[ls]) << ls;
                if (MODE == kEvery) {
                    for (int ls = 0; ls < kIq1mChoices; ++ls) {
                        const int neg = (negmask >> ls) & 1;
                        pack_block_m(out + ls * every_stride, lane, entry_of(ls + 8 * neg), ls, neg, d_half);
                    }
                    continue;
                }
                // e = s m under the group's delta, E = e_even + e_odd over the choice group
                int lstar = 0;
                float bestE = INFINITY;
#pragma unroll
                for (int ls = 0; ls < kIq1mChoices; ++ls) {
                    const float mm = ((negmask >> ls) & 1) ? best[8 + ls] : best[ls];
                    const float e = __fmul_rn(s[ls], mm);
                    const float E = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, 1));
                    if (E < bestE) { bestE = E; lstar = ls; }
                }
                const int neg = (negmask >> lstar) & 1;
                pack_block_m(out, lane, entry_of(lstar + 8 * neg), lstar, neg, d_half);
                continue;
            }
            if (MODE == kEvery) {
                for (int c = 0; c < kChoices; ++c) pack_block(out + c * every_stride, lane, entry_of(c), c, d_half);
                continue;
            }

            // group errors, sub-block sums over the 4 lanes of a sub-block, choice argmin
            int cstar = 0;
            float bestE = INFINITY;
#pragma unroll
            for (int c = 0; c < kChoices; ++c) {
                const float e0 = __fmul_rn(s[c & 7], best[c]);
                const float t2 = __fadd_rn(e0, __shfl_xor_sync(0xffffffffu, e0, 1));
                const float E = __fadd_rn(t2, __shfl_xor_sync(0xffffffffu, t2, 2));
                if (E < bestE) { bestE = E; cstar = c; }
            }
        pack_block(out, lane, entry_of(cstar), cstar, d_half);
        }
    }
}

template <int FMT, int MODE, int K>
cudaError_t launch_mode(const EncodeParams& p, int num_sms, cudaStream_t s) {
    auto kern = p.w_dtype == IQ_IN_BF16 ? iq1_encode_kernel<FMT, MODE, K, true> : iq1_encode_kernel<FMT, MODE, K, false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    const int64_t ctas_needed = (p.nb + kWarps - 1) / kWarps;
    const int64_t ctas = ctas_needed < 2LL * num_sms ? ctas_needed : 2LL * num_sms;
    kern<<<static_cast<unsigned>(ctas), kWarps * 32, kSmemBytes, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

template <int FMT>
cudaError_t launch_fmt(const EncodeParams& p, int mode, int num_sms, cudaStream_t s) {
    switch (mode) {
        case kSearch: return launch_mode<FMT, kSearch, 32>(p, num_sms, s);
        case kFixed: return launch_mode<FMT, kFixed, 32>(p, num_sms, s);
        default: return launch_mode<FMT, kEvery, 8>(p, num_sms, s);
    }
}

cudaError_t launch_iq1_encode(int fmt, const EncodeParams& p, int mode, int num_sms, cudaStream_t s) {
    if (p.nb == 0) return cudaSuccess;
    return fmt == IQ_FMT_IQ1_M ? launch_fmt<IQ_FMT_IQ1_M>(p, mode, num_sms, s)
                               : launch_fmt<IQ_FMT_IQ1_S>(p, mode, num_sms, s);
}

}  // namespace iqk

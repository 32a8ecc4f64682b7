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
// Formats: IQ1_S (8 groups of 32 columns), IQ2_XS and IQ2_S (16 groups of 16 columns), 16 choices;
// and a layout with eight candidates per 8-weight group (IQ2_XS candidates for ls = 8..15 over 32
// groups of 8 columns; picks only, since no payload stores a scale per 8 weights);
// IQ1_M (16 groups of 16 columns, 8 choices). With 8 choices two lanes share a candidate and each
// forms half of the group's H_gg u columns and half of each score's products; a 16-wide pairwise
// tree ends by adding its two 8-wide subtrees, so the halves join with one shuffle and one add.
//
// Experts: a stack of weights sharing a row layout runs in the same launch, row r taking Hessian
// set r / rows_per_hess (PR #3218's reason for one launch: thousands of small expert weights).
//
// Design (B200): one CTA = 16 rows (8 for IQ1_S) of one block, a half-warp per row and one lane per
// choice. Step 2 first stages all G diagonal blocks H_gg together (they fill one panel buffer), so
// each row scores its groups with no CTA barrier: a lane decodes its own candidate's group straight
// into registers and keeps all W accumulators of H_gg u, W independent fma chains fed by broadcast
// 16-byte reads; its two trees are local, and the only cross-lane step is the argmin over the
// half-warp. The initial gradient H Delta then streams H panel by panel (the group's W rows, W x 256
// contiguous fp32, double-buffered; one thread issues each panel as one bulk copy that completes
// on the buffer's mbarrier, every thread waits with a bound) as 4-row x 4-column register tiles
// (per k one 16-byte read of the rows' values and one of H, then 16 fmas). The sweeps run the rows in lockstep over the same
// panel stream, so each panel is staged once for all rows: each row decides from its stored
// curvature terms and its gradient, and the gradients of the rows that switched are updated by all
// threads, a column pair per thread in packed fmas. H is read from L2 three times per CTA, plus
// its diagonal blocks once. The grid is staged per format so that decoding needs no int-to-float
// conversion: IQ1 as 16-bit +1/-1 masks, each element selecting among its group's three values;
// IQ2 as byte-permute selectors over tables of the four magnitudes' 16-bit halves (two permutes
// per pair of halves, two to join them into floats, the signs by XOR). The block's H is checked for
// non-finite entries through the initial gradient: every entry enters a chain of every row, so
// the explicit scan runs only in a CTA whose gradient came out non-finite. On request each row's
// final Delta^T H Delta is reported as sum_i cur_i grad_i (a pairwise tree over the 256 columns).
#include "iq_device.cuh"
#include "iq_kernels.h"

namespace iqk {
namespace {

template <int N>
__device__ __forceinline__ void load_vec(const float* src, float v[N]) {
#pragma unroll
    for (int t = 0; t < N / 4; ++t) {
        const float4 a = reinterpret_cast<const float4*>(src)[t];
        v[4 * t] = a.x; v[4 * t + 1] = a.y; v[4 * t + 2] = a.z; v[4 * t + 3] = a.w;
    }
}

// An IQ1 grid entry as masks: bit j set when q_j = +1, bit 8 + j when q_j = -1.
__device__ __forceinline__ uint16_t grid_masks(int2 raw) {
    uint32_t c = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
        c |= (static_cast<uint32_t>(v == 1) << j) | (static_cast<uint32_t>(v == -1) << (8 + j));
    }
    return static_cast<uint16_t>(c);
}

// An IQ2 grid entry as four byte-permute selectors, one per element pair (2p, 2p + 1) at bits
// 16p..16p+15 of the 64-bit entry: nibbles (2 c0, 2 c0 + 1, 2 c1, 2 c1 + 1) pick the 16-bit
// entries c0 and c1 of a four-entry table, c = (g - 1) / 2.
__device__ __forceinline__ uint2 grid_selectors(int2 raw) {
    uint32_t sel[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
        const uint32_t c = static_cast<uint32_t>((v - 1) >> 1) & 3u;
        sel[j >> 2] |= ((2u * c) | ((2u * c + 1u) << 4)) << (8 * (j & 3));
    }
    return make_uint2(sel[0], sel[1]);
}

// The 8 values m(c_j), negated where bit j of neg is set, with the four magnitudes (m1, m3, m5,
// m7) split into a table of their low halves and one of their high halves: a pair's two low
// halves are one byte permute, its two high halves another, and two more join them into the
// pair's floats. The sign is the float's top bit, so negation is an XOR (also for zero).
__device__ __forceinline__ void pick8(uint2 sel, float m1, float m3, float m5, float m7, uint32_t neg, float xh[8]) {
    const uint32_t u1 = __float_as_uint(m1), u3 = __float_as_uint(m3), u5 = __float_as_uint(m5), u7 = __float_as_uint(m7);
    const uint32_t la = __byte_perm(u1, u3, 0x5410), lb = __byte_perm(u5, u7, 0x5410);
    const uint32_t ha = __byte_perm(u1, u3, 0x7632), hb = __byte_perm(u5, u7, 0x7632);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t w = p < 2 ? sel.x : sel.y;
        const uint32_t sp = (p & 1) ? (w >> 16) : w;
        const uint32_t lo = __byte_perm(la, lb, sp), hi = __byte_perm(ha, hb, sp);
        const uint32_t e0 = __byte_perm(lo, hi, 0x5410) ^ ((neg << (31 - 2 * p)) & 0x80000000u);
        const uint32_t e1 = __byte_perm(lo, hi, 0x7632) ^ ((neg << (30 - 2 * p)) & 0x80000000u);
        xh[2 * p] = __uint_as_float(e0);
        xh[2 * p + 1] = __uint_as_float(e1);
    }
}

// The decoded values of one 8-weight group of candidate `pc`: xh[j] = value of element j of
// 8-weight group `grp8` (inside the block) in choice group g. The products the group can take are
// formed once (IQ1_S: s (q + delta), q in {-1, 0, 1}; IQ2_XS: s g, g in {1, 3, 5, 7}), each
// rounded exactly as the direct formula rounds it, and picked per element (no int-to-float) from
// the staged grid: `sgrid_v` holds 16-bit masks for IQ1_S and IQ1_M, 64-bit selectors for IQ2.
template <int FMT>
__device__ __forceinline__ void decode8(const uint8_t* pc, const void* sgrid_v, int g, int grp8, float xh[8]) {
    const uint16_t* sgrid = static_cast<const uint16_t*>(sgrid_v);
    if (FMT == IQ_FMT_IQ1_M) {
        // 56-byte layout: low index byte grp8; its nibble in byte 32 + grp8 / 2 (3 high index
        // bits, bit 3 = delta -1/8); choice group g's 3-bit scale in word 48 + 2 (g / 4); d in
        // the words' top nibbles
        const uint16_t* pw = reinterpret_cast<const uint16_t*>(pc);
        const float dm = half_bits_to_f32(iq1m_d_bits(pw[24], pw[25], pw[26], pw[27]));
        const float s = __fmul_rn(dm, small_int_to_float(2u * ((static_cast<uint32_t>(pw[24 + (g >> 2)]) >> (3 * (g & 3))) & 7u) + 1u));
        const uint32_t nib = (static_cast<uint32_t>(pc[32 + (grp8 >> 1)]) >> (4 * (grp8 & 1))) & 15u;
        const float delta = (nib & 8u) ? -0.125f : 0.125f;
        const float vp = __fmul_rn(s, __fadd_rn(1.0f, delta));
        const float v0 = __fmul_rn(s, __fadd_rn(0.0f, delta));
        const float vn = __fmul_rn(s, __fadd_rn(-1.0f, delta));
        const uint32_t m = sgrid[static_cast<uint32_t>(pc[grp8]) | ((nib & 7u) << 8)];
#pragma unroll
        for (int j = 0; j < 8; ++j) xh[j] = ((m >> j) & 1u) ? vp : (((m >> (8 + j)) & 1u) ? vn : v0);
        return;
    }
    const float d = half_bits_to_f32(*reinterpret_cast<const uint16_t*>(pc));
    if (FMT == IQ_FMT_IQ2_S) {
        // 82-byte layout: low index byte 2 + grp8, sign byte 34 + grp8, 2 high index bits at
        // shift 2 (grp8 % 4) of byte 66 + grp8 / 4, choice group g's scale nibble at 74 + g / 2
        const uint32_t sc = pc[74 + (g >> 1)];
        const int ls = static_cast<int>((g & 1) ? (sc >> 4) : (sc & 15u));
        const float s = __fmul_rn(d, small_int_to_float(static_cast<uint32_t>(2 * ls + 1)));
        const float m1 = __fmul_rn(s, 1.0f), m3 = __fmul_rn(s, 3.0f), m5 = __fmul_rn(s, 5.0f), m7 = __fmul_rn(s, 7.0f);
        const uint32_t idx = static_cast<uint32_t>(pc[2 + grp8]) | (((static_cast<uint32_t>(pc[66 + (grp8 >> 2)]) >> (2 * (grp8 & 3))) & 3u) << 8);
        const uint32_t neg = pc[34 + grp8];
        pick8(static_cast<const uint2*>(sgrid_v)[idx], m1, m3, m5, m7, neg, xh);
    } else if (FMT == IQ_FMT_IQ2_XS) {
        const uint32_t code = *reinterpret_cast<const uint16_t*>(pc + 2 + 2 * grp8);
        const uint32_t sc = pc[66 + (g >> 1)];
        const int ls = static_cast<int>((g & 1) ? (sc >> 4) : (sc & 15u));
        const float s = __fmul_rn(d, small_int_to_float(static_cast<uint32_t>(2 * ls + 1)));
        const float m1 = __fmul_rn(s, 1.0f), m3 = __fmul_rn(s, 3.0f), m5 = __fmul_rn(s, 5.0f), m7 = __fmul_rn(s, 7.0f);
        const uint32_t sign7 = code >> 9;
        const uint32_t neg = sign7 | (static_cast<uint32_t>(__popc(sign7) & 1) << 7);
        pick8(static_cast<const uint2*>(sgrid_v)[code & 511u], m1, m3, m5, m7, neg, xh);
    } else {
        const uint32_t qh = *reinterpret_cast<const uint16_t*>(pc + 34 + 2 * g);
        const float s = __fmul_rn(d, small_int_to_float(2u * ((qh >> 12) & 7u) + 1u));
        const float delta = (qh & 0x8000u) ? -0.125f : 0.125f;
        const float vp = __fmul_rn(s, __fadd_rn(1.0f, delta));
        const float v0 = __fmul_rn(s, __fadd_rn(0.0f, delta));
        const float vn = __fmul_rn(s, __fadd_rn(-1.0f, delta));
        const int i4 = grp8 & 3;  // group within the sub-block
        const int idx = static_cast<int>(pc[2 + 4 * g + i4]) | static_cast<int>(((qh >> (3 * i4)) & 7u) << 8);
        const uint32_t m = sgrid[idx];
#pragma unroll
        for (int j = 0; j < 8; ++j) xh[j] = ((m >> j) & 1u) ? vp : (((m >> (8 + j)) & 1u) ? vn : v0);
    }
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }


template <int FMT>
struct Cfg {
    static constexpr bool G8 = FMT == kChoiceIq2xsG8;          // eight candidates per 8-weight group
    static constexpr int DF = G8 ? IQ_FMT_IQ2_XS : FMT;         // the candidates' payload format
    static constexpr int PICK0 = G8 ? kChoiceG8FirstLs : 0;     // reported pick of candidate 0
    static constexpr int R = FMT == IQ_FMT_IQ1_S ? 8 : 16;      // rows per CTA (shared-memory budget)
    static constexpr int T = R * 16;                            // threads: a half-warp per row
    static constexpr int RG = R / 4;                            // 4-row groups of the gradient tiles
    static constexpr int G = FMT == IQ_FMT_IQ1_S ? 8 : G8 ? 32 : 16;  // choice groups per block
    static constexpr int W = kBlock / G;                        // columns per choice group
    static constexpr int B = DF == IQ_FMT_IQ1_S   ? kIq1sBytes
                             : DF == IQ_FMT_IQ1_M ? kIq1mBytes
                             : DF == IQ_FMT_IQ2_S ? kIq2sBytes
                                                  : kIq2xsBytes;
    static constexpr int E = DF == IQ_FMT_IQ2_XS ? kIq2xsEntries : DF == IQ_FMT_IQ2_S ? kIq2sEntries : kIq1sEntries;
    static constexpr int NC = FMT == IQ_FMT_IQ1_M ? kIq1mChoices : G8 ? 8 : kChoices;  // candidates per row
    static constexpr int SPLIT = kChoices / NC;                 // lanes per candidate
    static constexpr int WO = W / SPLIT;                        // group columns per lane
    static constexpr int BPAD = (kChoices * B + 15) / 16 * 16;  // candidate bytes per row
    // shared memory layout (bytes)
    static constexpr int oHp = 0;                             // float [2][W][256], double buffer
    static constexpr int oCurT = oHp + 2 * W * kBlock * 4;    // float [256][R]: the rows' current Delta
    static constexpr int oUR = oCurT + kBlock * R * 4;        // float [R][W]: u of the rows that switched
    static constexpr int oT2 = oUR + R * W * 4;               // float [R][G][NC]: u^T H_gg u per candidate
    static constexpr int oSw = oT2 + R * G * NC * 4;          // uint32 [2]: rows that switched, by step parity
    static constexpr bool IQ2 = DF == IQ_FMT_IQ2_XS || DF == IQ_FMT_IQ2_S;
    static constexpr int oBar = oSw + R * 4;   // uint64 [2] panel barriers, uint32 abort word
    static constexpr int oGrid = oBar + 32;    // IQ2: uint2 [E] selectors; IQ1: uint16 [E] masks
    static constexpr int oRows = oGrid + (IQ2 ? E * 8 : (E * 2 + 15) / 16 * 16);  // per-row records
    static constexpr int rGrad = 0;                               // float [256]
    static constexpr int rPick = rGrad + kBlock * 4;              // int [G]
    static constexpr int rCand = (rPick + G * 4 + 15) / 16 * 16;  // uint8 [16][B]
    static constexpr int rBytes = (rCand + BPAD + 15) / 16 * 16;
    static constexpr int smem = oRows + R * rBytes;
    // two CTAs share an SM (228 KiB of shared memory, 1 KiB reserved per CTA)
    static_assert(2 * (smem + 1024) <= 228 * 1024, "two CTAs per SM");
};

// Pairwise tree over N values: (p0 + p1), (p2 + p3), ... then up, as the oracle sums.
template <int N>
__device__ __forceinline__ float tree_sum(float p[N]) {
#pragma unroll
    for (int width = 1; width < N; width *= 2)
#pragma unroll
        for (int t = 0; t + width < N; t += 2 * width) p[t] = __fadd_rn(p[t], p[t + width]);
    return p[0];
}

// Argmin over the 16 lanes of a half-warp of (key(value), choice), lowest choice on ties, where
// lane c of the half-warp holds choice c. The key (NaN and +inf as +inf, -0 as +0, so that equal
// floats are equal keys) is mapped to an order-preserving unsigned and reduced with one redux;
// the lowest lane holding the minimum is the choice.
__device__ __forceinline__ void half_argmin(float v, int /*c*/, unsigned mask, float& best, int& cbest) {
    const uint32_t u = __float_as_uint(__fadd_rn(argmin_key(v), 0.0f));
    const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    const uint32_t m = __reduce_min_sync(mask, o);
    cbest = (__ffs(__ballot_sync(mask, o == m) & mask) - 1) & 15;
    best = __uint_as_float((m & 0x80000000u) ? (m & 0x7FFFFFFFu) : ~m);
}

// v[i] = sum over k < W (fma chain, k ascending, starting from the product) of
// Hp[k][col0 + i] * a[k], for NO columns, Hp's rows LD floats apart. Adjacent columns run as one
// packed fma.rn.f32x2 (two independent IEEE fmas, so every chain rounds exactly as the scalar
// one); the next row is loaded while the current one is used.
template <int W, int NO, int LD>
__device__ __forceinline__ void group_matvec(const float* Hp, int col0, const float a[W], float v[NO]) {
    static_assert(NO % 4 == 0, "16-byte panel reads");
    float h[NO], hn[NO];
    float2 acc[NO / 2];
    load_vec<NO>(Hp + col0, h);
    load_vec<NO>(Hp + LD + col0, hn);
    {
        const float2 a0 = make_float2(a[0], a[0]);
#pragma unroll
        for (int t = 0; t < NO / 2; ++t) acc[t] = __fmul2_rn(make_float2(h[2 * t], h[2 * t + 1]), a0);
    }
#pragma unroll
    for (int k = 1; k < W; ++k) {
#pragma unroll
        for (int i = 0; i < NO; ++i) h[i] = hn[i];
        if (k + 1 < W) load_vec<NO>(Hp + (k + 1) * LD + col0, hn);
        const float2 ak = make_float2(a[k], a[k]);
#pragma unroll
        for (int t = 0; t < NO / 2; ++t) acc[t] = __ffma2_rn(make_float2(h[2 * t], h[2 * t + 1]), ak, acc[t]);
    }
#pragma unroll
    for (int t = 0; t < NO / 2; ++t) {
        v[2 * t] = acc[t].x;
        v[2 * t + 1] = acc[t].y;
    }
}

// A 4-row x 4-column register tile of gradient chains: acc[r][c] = fma(h[c], x[r], acc[r][c]) for
// one k, as two packed fmas per row (the pairs are two independent columns).
__device__ __forceinline__ void tile_fma(float2 acc[4][2], const float4 hv, const float4 xv, bool first) {
    const float2 h01 = make_float2(hv.x, hv.y), h23 = make_float2(hv.z, hv.w);
    const float xr[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const float2 x2 = make_float2(xr[rr], xr[rr]);
        if (first) {
            acc[rr][0] = __fmul2_rn(h01, x2);
            acc[rr][1] = __fmul2_rn(h23, x2);
        } else {
            acc[rr][0] = __ffma2_rn(h01, x2, acc[rr][0]);
            acc[rr][1] = __ffma2_rn(h23, x2, acc[rr][1]);
        }
    }
}

// This lane's half of a group vector (register indices stay static), or all of it.
template <int W, int WO>
__device__ __forceinline__ void lane_part(const float a[W], int part, float out[WO]) {
#pragma unroll
    for (int i = 0; i < WO; ++i) out[i] = (WO < W && part) ? a[WO + i] : a[i];
}

// Joins the two halves' tree sums (lanes c and c + NC) when a candidate spans two lanes.
template <int SPLIT, int NC>
__device__ __forceinline__ float join_parts(float t, unsigned mask) {
    return SPLIT == 1 ? t : __fadd_rn(t, __shfl_xor_sync(mask, t, NC));
}

// u^T H_gg u over this lane's candidate: (H_gg u) for this lane's columns, the products with u,
// and the pairwise tree over the group's W columns (joined across the lanes of a candidate).
// Hg is H_gg's first row, the group's first column at col0, rows LD floats apart: a panel
// (LD = 256, col0 = g W) or a staged diagonal block (LD = W, col0 = 0).
template <int W, int WO, int SPLIT, int NC, int LD>
__device__ __forceinline__ float quad_form(const float* Hg, int col0, int part, const float u[W], unsigned mask) {
    float v[WO], up[WO];
    group_matvec<W, WO, LD>(Hg, col0 + part * WO, u, v);
    lane_part<W, WO>(u, part, up);
#pragma unroll
    for (int i = 0; i < WO; ++i) v[i] = __fmul_rn(up[i], v[i]);
    return join_parts<SPLIT, NC>(tree_sum<WO>(v), mask);
}

// Whether a staged grid row lies in the candidates' alphabet ({-1, 0, 1} or {1, 3, 5, 7}).
template <int DF>
__device__ __forceinline__ bool grid_row_ok(int2 raw) {
    bool ok = true;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int v = static_cast<int8_t>(((j < 4 ? raw.x : raw.y) >> (8 * (j & 3))) & 0xFF);
        ok &= (DF == IQ_FMT_IQ1_S || DF == IQ_FMT_IQ1_M) ? (v >= -1 && v <= 1) : (v == 1 || v == 3 || v == 5 || v == 7);
    }
    return ok;
}

// Eight consecutive weights of a row as fp32 (exact): bf16 bits, or fp32 values.
template <bool F32>
__device__ __forceinline__ void load_x8(const void* xrow, int i8, float xv[8]) {
    if (F32) {
        const float4* q = reinterpret_cast<const float4*>(xrow) + 2 * i8;
        const float4 a = __ldg(q), b = __ldg(q + 1);
        xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w; xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
    } else {
        unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(xrow) + i8), xv);
    }
}

template <int FMT, bool F32>
__global__ void __launch_bounds__(Cfg<FMT>::T, 2) choice_search_kernel(const ChoiceParams p) {
    using C = Cfg<FMT>;
    constexpr int W = C::W, G = C::G, kRows = C::R, kThreads = C::T, WO = C::WO, NC = C::NC;
    static_assert(C::SPLIT * NC == kChoices && (W & (W - 1)) == 0, "halves join as the tree's last level");
    static_assert(kThreads == C::RG * 64, "gradient tiles: 4 rows x 4 columns per thread");
    extern __shared__ __align__(16) char smem[];
    float* curT = reinterpret_cast<float*>(smem + C::oCurT);
    float* uR = reinterpret_cast<float*>(smem + C::oUR);
    uint32_t* swbits = reinterpret_cast<uint32_t*>(smem + C::oSw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::oBar);
    volatile uint32_t* abort_word = reinterpret_cast<volatile uint32_t*>(smem + C::oBar + 16);
    uint16_t* sgrid = reinterpret_cast<uint16_t*>(smem + C::oGrid);

    // CTA -> (block, expert, row tile): a tile never straddles two experts, and the CTAs that
    // share one Hessian block are adjacent in launch order.
    const int64_t nexp = p.rows / p.rows_per_hess;
    const int64_t tiles_e = (p.rows_per_hess + kRows - 1) / kRows;
    const int64_t blk_rel = blockIdx.x / (nexp * tiles_e);
    const int64_t blk = p.blk0 + blk_rel;
    const int64_t rem = blockIdx.x - blk_rel * nexp * tiles_e;
    const int64_t expert = rem / tiles_e;
    const int64_t tile_row0 = (rem - expert * tiles_e) * kRows;
    const int tid = threadIdx.x, hr = tid >> 4, c = tid & 15;
    const int ch = c % NC, part = c / NC;  // this lane's candidate, and its half of the columns
    const unsigned hmask = 0xFFFFu << (16 * (hr & 1));  // this half-warp's lanes within the warp
    const int64_t row = expert * p.rows_per_hess + tile_row0 + hr;
    const bool active = tile_row0 + hr < p.rows_per_hess;
    char* rec = smem + C::oRows + hr * C::rBytes;
    float* grad = reinterpret_cast<float*>(rec + C::rGrad);
    int* pick = reinterpret_cast<int*>(rec + C::rPick);
    uint8_t* cand = reinterpret_cast<uint8_t*>(rec + C::rCand);
    float* t2row = reinterpret_cast<float*>(smem + C::oT2) + hr * G * NC;  // [G][NC]
    const float* H = p.hess + (expert * p.nblk + blk) * kBlock * kBlock;
    const void* xrow = F32 ? static_cast<const void*>(static_cast<const float*>(p.w) + row * p.ldw + blk * kBlock)
                           : static_cast<const void*>(static_cast<const uint16_t*>(p.w) + row * p.ldw + blk * kBlock);

    // H panels (the W rows of one choice group, W x 256 contiguous fp32) stream through a double
    // buffer: step s of the 3G panel steps (the initial gradient, then two sweeps) uses panel
    // s % G from buffer s & 1. One thread issues each panel as one bulk copy completing on the
    // buffer's barrier; every thread waits for that phase (parity (s >> 1) & 1, the buffer's
    // (s >> 1)-th use) with a bound. A wait that runs out marks the CTA aborted: its waits stop,
    // and its row-blocks are written as findings (IQ_FLAG_TIMEOUT).
    auto panel = [&](int step) { return reinterpret_cast<float*>(smem + C::oHp + (step & 1) * W * kBlock * 4); };
    auto prefetch = [&](int step) {  // thread 0, after a CTA barrier that freed the buffer
        bulk_load(panel(step), H + (step % G) * W * kBlock, W * kBlock * 4, bars + (step & 1));
    };
    bool timed_out = false;
    auto wait_panel = [&](int step) {
        if (*abort_word == 0u && !mbar_wait(bars + (step & 1), (step >> 1) & 1, kBulkWaitCycles)) {
            timed_out = true;
            *abort_word = 1u;
        }
    };
    if (tid == 0) {
        mbar_init(bars);
        mbar_init(bars + 1);
        *abort_word = 0u;
        prefetch(0);
    }

    // ---- stage the grid (checking the alphabet) and the row's candidate payloads (lanes
    // past the format's NC candidates stage zeros and never win); a non-finite weight taints the row
    bool grid_bad = false, h_bad = false, row_bad = false;
    for (int q = tid; q < C::E; q += kThreads) {
        const int2 raw = __ldg(reinterpret_cast<const int2*>(p.grid) + q);
        if (C::IQ2) reinterpret_cast<uint2*>(sgrid)[q] = grid_selectors(raw);
        else sgrid[q] = grid_masks(raw);
        grid_bad |= !grid_row_ok<C::DF>(raw);
    }
    if (active) {
        bool nonfinite = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            float xv[8];
            load_x8<F32>(xrow, 2 * c + t, xv);
#pragma unroll
            for (int j = 0; j < 8; ++j) nonfinite |= !isfinite(xv[j]);
        }
        row_bad = __any_sync(hmask, nonfinite);
        // 2-byte copies (B is even and the caller's candidates are 2-byte aligned), all loads
        // issued before the stores
        uint16_t* dst = reinterpret_cast<uint16_t*>(cand + c * C::B);
        if (c < C::NC) {
            const uint16_t* src = reinterpret_cast<const uint16_t*>(
                p.cand + c * p.cand_cstride + (row * p.cand_ld + (blk - p.cand_blk0)) * C::B);
            uint16_t stage[C::B / 2];
#pragma unroll
            for (int i = 0; i < C::B / 2; ++i) stage[i] = __ldg(src + i);
#pragma unroll
            for (int i = 0; i < C::B / 2; ++i) dst[i] = stage[i];
        } else {
#pragma unroll
            for (int i = 0; i < C::B / 2; ++i) dst[i] = 0;
        }
    } else {
        for (int i = c; i < kBlock; i += 16) curT[i * kRows + hr] = 0.0f;
    }

    // Delta(c) over choice group g, decoded from this lane's candidate into registers.
    auto delta_of = [&](int g, float dl[W]) {
#pragma unroll
        for (int t = 0; t < W / 8; ++t) {
            float xh[8], xv[8];
            // decode8 takes the format's own choice group: for 8-column groups, the 16-column
            // group that holds the scale nibble
            decode8<C::DF>(cand + ch * C::B, sgrid, C::G8 ? (g >> 1) : g, (g * W + 8 * t) >> 3, xh);
            load_x8<F32>(xrow, (g * W) / 8 + t, xv);
#pragma unroll
            for (int j = 0; j < 8; ++j) dl[8 * t + j] = __fsub_rn(xv[j], xh[j]);
        }
    };

    // Gradient tiles: this thread owns rows 4 rg .. 4 rg + 3 and columns 4 cg .. 4 cg + 3.
    const int rg = tid >> 6, cg = tid & 63;
    auto grad_row = [&](int r) {
        return reinterpret_cast<float*>(smem + C::oRows + r * C::rBytes + C::rGrad);
    };

    // ---- step 2: each group's pick from its own diagonal block, and the first sweep's curvature
    // terms (u = Delta(c) - Delta(pick) changes only when group g itself switches, so u^T H_gg u is
    // scored here, once). The G diagonal blocks H_gg (G W^2 floats, one panel buffer) are staged
    // together in buffer 1 while panel 0 streams into buffer 0, so each row runs its G groups
    // without waiting for the other rows.
    float* Hd = panel(1);
    for (int i = tid; i < G * W * W / 4; i += kThreads) {
        const int gk = i / (W / 4), c4 = i % (W / 4);  // H row gk = g W + k, its 16-byte chunk c4 of H_gg
        cp_async16(Hd + gk * W + 4 * c4, H + gk * kBlock + (gk / W) * W + 4 * c4);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    if (active) {
        for (int g = 0; g < G; ++g) {
            const float* Hg = Hd + g * W * W;
            float dl[W];
            delta_of(g, dl);
            const float sq = quad_form<W, WO, C::SPLIT, NC, W>(Hg, 0, part, dl, hmask);  // every lane joins
            const float score = c < NC ? sq : INFINITY;
            float best;
            int cstar;
            half_argmin(score, c, hmask, best, cstar);
            if (c == cstar) {
#pragma unroll
                for (int i = 0; i < W; ++i) curT[(g * W + i) * kRows + hr] = dl[i];
                pick[g] = c;
            }
            // the winner's Delta by shuffles, then u = Delta(c) - Delta(pick) in place
#pragma unroll
            for (int i = 0; i < W; ++i) dl[i] = __fsub_rn(dl[i], __shfl_sync(hmask, dl[i], cstar, 16));
            const float t2 = quad_form<W, WO, C::SPLIT, NC, W>(Hg, 0, part, dl, hmask);
            if (part == 0) t2row[g * NC + ch] = t2;
        }
    }

    // ---- the initial gradient grad = H Delta(picks), panel by panel: grad_i += H[k][i] cur_k over
    // group g's k, a 4-row x 4-column tile per thread, fed by one 16-byte read of the rows' cur_k
    // and one of H[k][4 columns] per k
    float2 gacc[4][2];
    for (int g = 0; g < G; ++g) {
        __syncthreads();  // every thread is done with the other buffer (panel g - 1, or Hd)
        if (tid == 0) prefetch(g + 1);
        wait_panel(g);
        const float* Hp = panel(g);
#pragma unroll 4
        for (int k = 0; k < W; ++k) {
            const float4 cv = *reinterpret_cast<const float4*>(curT + (g * W + k) * kRows + 4 * rg);
            const float4 hv = *reinterpret_cast<const float4*>(Hp + k * kBlock + 4 * cg);
            tile_fma(gacc, hv, cv, g == 0 && k == 0);
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
        *reinterpret_cast<float4*>(grad_row(4 * rg + rr) + 4 * cg) =
            make_float4(gacc[rr][0].x, gacc[rr][0].y, gacc[rr][1].x, gacc[rr][1].y);
    // Every entry H[k][i] of the block enters column i's gradient chain of every row (inactive
    // rows with Delta = 0), and a non-finite product (inf * 0 is NaN) keeps the chain non-finite,
    // so a finite gradient tile everywhere proves the block finite. A non-finite one (which a
    // non-finite Delta or an overflow can also cause) sends the CTA to the exact scan of H.
    {
        bool tile_bad = false;
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
            tile_bad |= !(isfinite(gacc[rr][0].x) && isfinite(gacc[rr][0].y) && isfinite(gacc[rr][1].x) &&
                          isfinite(gacc[rr][1].y));
        if (__syncthreads_or(tile_bad)) {
            const float4* H4 = reinterpret_cast<const float4*>(H);
            for (int i = tid; i < kBlock * kBlock / 4; i += kThreads) {
                const float4 v = __ldg(H4 + i);
                h_bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
            }
        }
    }
    grid_bad = __syncthreads_or(grid_bad);
    h_bad = __syncthreads_or(h_bad);
    if (tid == 0) raise_flags(p.flags, (grid_bad ? IQ_FLAG_GRID : 0u) | (h_bad ? IQ_FLAG_NONFINITE : 0u));
    if (active && c == 0 && row_bad) raise_flags(p.flags, IQ_FLAG_NONFINITE);
    // The gradient tiles wanted the rows' Delta by column; the sweeps read and write whole
    // groups of one row, so the same area is rewritten row-major: cur[r][i].
    float* cur = curT;
    {
        float v[kBlock * kRows / kThreads];
#pragma unroll
        for (int t = 0; t < kBlock * kRows / kThreads; ++t) v[t] = curT[tid + t * kThreads];
        __syncthreads();
#pragma unroll
        for (int t = 0; t < kBlock * kRows / kThreads; ++t) {
            const int idx = tid + t * kThreads;  // = i * kRows + r
            cur[(idx % kRows) * kBlock + idx / kRows] = v[t];
        }
        if (tid == 0) swbits[0] = swbits[1] = 0u;
    }
    float* cur_row = cur + hr * kBlock;

    // ---- step 3: two sweeps over the groups. Each row decides (lane per choice) from the stored
    // curvature term and the current gradient; a row that switches in the first sweep rescores
    // that group's curvature terms around its new pick for the second. Then all threads update
    // the switched rows' gradients, a column pair per thread.
    for (int step = G; step < 3 * G; ++step) {
        const int g = step % G;
        __syncthreads();
        if (tid == 0 && step + 1 < 3 * G) prefetch(step + 1);
        wait_panel(step);
        const float* Hp = panel(step);
        int switched = 0;
        if (active) {
            float dl[W], u[W];
            delta_of(g, dl);
            {
                float cg[W];
                load_vec<W>(cur_row + g * W, cg);
#pragma unroll
                for (int i = 0; i < W; ++i) u[i] = __fsub_rn(dl[i], cg[i]);
            }
            float gain;
            {
                float gq[WO], p1[WO], up[WO];
                load_vec<WO>(grad + g * W + part * WO, gq);
                lane_part<W, WO>(u, part, up);
#pragma unroll
                for (int i = 0; i < WO; ++i) p1[i] = __fmul_rn(up[i], gq[i]);
                const float t1 = join_parts<C::SPLIT, NC>(tree_sum<WO>(p1), hmask);
                gain = c < NC ? __fmaf_rn(2.0f, t1, t2row[g * NC + ch]) : INFINITY;
            }
            float best;
            int cstar;
            half_argmin(gain, c, hmask, best, cstar);
            switched = best < 0.0f;  // uniform over the half-warp
            if (switched) {
                if (c == cstar) {
#pragma unroll
                    for (int i = 0; i < W; i += 4)
                        *reinterpret_cast<float4*>(uR + hr * W + i) = make_float4(u[i], u[i + 1], u[i + 2], u[i + 3]);
#pragma unroll
                    for (int i = 0; i < W; i += 4)
                        *reinterpret_cast<float4*>(cur_row + g * W + i) = make_float4(dl[i], dl[i + 1], dl[i + 2], dl[i + 3]);
                    pick[g] = c;
                }
                if (step < 2 * G) {  // the second sweep's curvature terms around the new pick
#pragma unroll
                    for (int i = 0; i < W; ++i) dl[i] = __fsub_rn(dl[i], __shfl_sync(hmask, dl[i], cstar, 16));
                    const float t2 = quad_form<W, WO, C::SPLIT, NC, kBlock>(Hp, g * W, part, dl, hmask);
                    if (part == 0) t2row[g * NC + ch] = t2;
                }
            }
        }
        if (c == 0 && switched) atomicOr(&swbits[step & 1], 1u << hr);
        __syncthreads();
        // grad[r][i] += sum_k H[k][i] u_k (fma chain over the group's k) for the rows that
        // switched: a column pair per thread, its H[k][2 cp .. 2 cp + 1] in registers, as two
        // independent chains in packed fmas; the CTA's thread sets split the switched rows by
        // their rank among them. (Register tiles over 4-row groups measured no faster for IQ2 and
        // 5% slower for IQ1_S.)
        const uint32_t swmask = swbits[step & 1];
        if (tid == 0) swbits[(step + 1) & 1] = 0u;  // every thread read it last step, before this step's first barrier
        if (swmask != 0) {
            constexpr int kSets = kThreads / (kBlock / 2);
            const int cp = tid % (kBlock / 2), set = tid / (kBlock / 2);
            float2 hcol[W];
#pragma unroll
            for (int k = 0; k < W; ++k) hcol[k] = *reinterpret_cast<const float2*>(Hp + k * kBlock + 2 * cp);
            int rank = 0;
            for (uint32_t m = swmask; m != 0; m &= m - 1, ++rank) {
                if (rank % kSets != set) continue;
                const int r = __ffs(m) - 1;
                float uk[W];
                load_vec<W>(uR + r * W, uk);
                float2* gr = reinterpret_cast<float2*>(grad_row(r)) + cp;
                float2 acc = *gr;
#pragma unroll
                for (int k = 0; k < W; ++k) acc = __ffma2_rn(hcol[k], make_float2(uk[k], uk[k]), acc);
                *gr = acc;
            }
        }
    }

    // every gradient update has landed; an aborted CTA waits once more (bounded) for copies in flight
    const bool cta_timed_out = __syncthreads_or(timed_out);
    if (cta_timed_out && tid == 0) {
        const int last = 3 * G - 1;  // the last panel step; its barrier phase and the other buffer's
        mbar_wait(bars + (last & 1), (last >> 1) & 1, kBulkWaitCycles);
        mbar_wait(bars + ((last - 1) & 1), ((last - 1) >> 1) & 1, kBulkWaitCycles);
        raise_flags(p.flags, IQ_FLAG_TIMEOUT);
    }
    // A row-block with a finding (a non-finite weight in the row, a non-finite entry in its
    // Hessian block, a grid value outside the alphabet, a copy wait that ran out) reports picks 0,
    // the all-zero payload and a NaN objective.
    const bool tainted = grid_bad || h_bad || row_bad || cta_timed_out;

    // ---- the final objective Delta^T H Delta = sum_i cur_i grad_i: lane c sums columns
    // 16c .. 16c + 15 by a pairwise tree, then the butterfly joins the 16 lanes pairwise
    if (p.objective != nullptr && active) {
        float pr[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) pr[j] = __fmul_rn(cur_row[16 * c + j], grad[16 * c + j]);
        float t = tree_sum<16>(pr);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) t = __fadd_rn(t, __shfl_xor_sync(hmask, t, o));
        if (c == 0) p.objective[row * p.nblk + blk] = tainted ? __uint_as_float(0x7FC00000u) : t;
    }

    // ---- the final Delta (one block per launch): what the per-block calibration loop
    // propagates; a row-block with a finding has the all-zero payload, so its Delta is x
    if (p.delta_out != nullptr && active) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            float xv[8], dv[8];
            load_x8<F32>(xrow, 2 * c + t, xv);
#pragma unroll
            for (int j = 0; j < 8; ++j) dv[j] = tainted ? xv[j] : cur_row[16 * c + 8 * t + j];
            float4* dst = reinterpret_cast<float4*>(p.delta_out + row * kBlock + 16 * c + 8 * t);
            dst[0] = make_float4(dv[0], dv[1], dv[2], dv[3]);
            dst[1] = make_float4(dv[4], dv[5], dv[6], dv[7]);
        }
    }

    // ---- step 4: picks and the payload assembled from the picked candidates
    if (active) {
        __syncwarp(hmask);
        for (int q = c; q < G; q += 16)
            p.picks[(row * p.nblk + blk) * G + q] = static_cast<uint8_t>(C::PICK0 + (tainted ? 0 : pick[q]));
    }
    if (!C::G8 && active) {  // 8-column groups report picks only: no payload stores their scales
        uint8_t* out = p.payload + (row * p.payload_ld + blk) * C::B;
        for (int i = c; i < C::B; i += 16) {
            uint8_t v;
            if (FMT == IQ_FMT_IQ1_M) {
                if (i < 32) {  // low index byte of 8-weight group i: choice group i / 2
                    v = cand[pick[i >> 1] * C::B + i];
                } else if (i < 48) {  // the nibbles of choice group i - 32's two groups
                    v = cand[pick[i - 32] * C::B + i];
                } else {  // scale word q: choice groups 4q..4q+3 at shifts 0,3,6,9; d's nibble on top
                    const int q = (i - 48) >> 1;
                    uint32_t wv = (static_cast<uint32_t>(cand[49 + 2 * q]) << 8) & 0xF000u;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint8_t* pc = cand + pick[4 * q + j] * C::B;
                        const uint32_t wj = static_cast<uint32_t>(pc[48 + 2 * q]) | (static_cast<uint32_t>(pc[49 + 2 * q]) << 8);
                        wv |= wj & (7u << (3 * j));
                    }
                    v = static_cast<uint8_t>((i & 1) ? (wv >> 8) : wv);
                }
            } else if (i < 2) {
                v = cand[i];
            } else if (FMT == IQ_FMT_IQ2_S) {
                if (i < 66) {  // low index and sign bytes of 8-weight group q8: choice group q8 / 2
                    v = cand[pick[((i - 2) & 31) >> 1] * C::B + i];
                } else if (i < 74) {  // 2-bit high index fields: groups 4q, 4q+1 | 4q+2, 4q+3
                    const int k = 2 * (i - 66);
                    v = static_cast<uint8_t>((cand[pick[k] * C::B + i] & 0x0Fu) | (cand[pick[k + 1] * C::B + i] & 0xF0u));
                } else {  // scale nibbles of choice groups 2q, 2q + 1
                    const int k = 2 * (i - 74);
                    v = static_cast<uint8_t>((cand[pick[k] * C::B + i] & 0x0Fu) | (cand[pick[k + 1] * C::B + i] & 0xF0u));
                }
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
            out[i] = tainted ? static_cast<uint8_t>(0) : v;
        }
    }
}

template <int FMT, bool F32>
cudaError_t launch(const ChoiceParams& p, cudaStream_t s) {
    using C = Cfg<FMT>;
    auto kern = choice_search_kernel<FMT, F32>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::smem);
    if (err != cudaSuccess) return err;
    const int64_t ctas = p.nblk_run * (p.rows / p.rows_per_hess) * ((p.rows_per_hess + C::R - 1) / C::R);
    kern<<<static_cast<unsigned>(ctas), C::T, C::smem, s>>>(p);
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
    if (p.rows == 0 || p.nblk_run == 0) return cudaSuccess;
    if (p.w_f32) {  // the per-block calibration loop's compensated weights
        if (fmt == IQ_FMT_IQ1_S) return launch<IQ_FMT_IQ1_S, true>(p, s);
        if (fmt == IQ_FMT_IQ2_S) return launch<IQ_FMT_IQ2_S, true>(p, s);
        if (fmt == IQ_FMT_IQ1_M) return launch<IQ_FMT_IQ1_M, true>(p, s);
        if (fmt == IQ_FMT_IQ2_XS) return launch<IQ_FMT_IQ2_XS, true>(p, s);
        return cudaErrorInvalidValue;
    }
    if (fmt == IQ_FMT_IQ1_S) return launch<IQ_FMT_IQ1_S, false>(p, s);
    if (fmt == IQ_FMT_IQ2_S) return launch<IQ_FMT_IQ2_S, false>(p, s);
    if (fmt == IQ_FMT_IQ1_M) return launch<IQ_FMT_IQ1_M, false>(p, s);
    if (fmt == kChoiceIq2xsG8) return launch<kChoiceIq2xsG8, false>(p, s);
    return launch<IQ_FMT_IQ2_XS, false>(p, s);
}

cudaError_t launch_sqrt_diag(const float* hess, int64_t nblk, float* out, cudaStream_t s) {
    if (nblk == 0) return cudaSuccess;
    const int64_t n = nblk * kBlock;
    sqrt_diag_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(hess, nblk, out);
    return cudaGetLastError();
}

}  // namespace iqk

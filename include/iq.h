/*
 * iq.h -- C ABI of the B200 GGML IQ encoder library (libiq_b200.so).
 *
 * What the library computes (Model-Optimizer pull-request pages):
 *   - IQ1_S and IQ2_XS weight encoding: every 256-weight super-block of a row is split into
 *     8-weight groups; each group gets an exhaustive, importance-weighted codebook search that
 *     minimises sum_j w_j (x_j - xhat_j)^2 over grid entry, sign/shift and local scale, and the
 *     block is packed into its fixed byte layout. Sources: PR #2723 "Weight the IQ1 encoders by
 *     the square root of GPTQ's Hessian diagonal" (objective, delta = +-1/8, unweighted d);
 *     PR #2450 "[OMNIML-5899] Add IQ tests and release notes", review comments (IQ1_S 50-byte and
 *     IQ2_XS 74-byte layouts, d = fp16((amax / 16.875) * 0.61), a choice among 16 with ties going
 *     to the lower index, even sign parity); the IQ2_S codec commit text on the PR #2525 page
 *     (IQ2_XS repairs an odd sign count at its weakest element).
 *   - fixed per-group choices (PR #3157) and the one-pass every-choice encode (PR #3159);
 *   - IQ1_M (PR #2513 codec and PR #2595 encoder commit texts): the IQ1_S search with a local
 *     scale per 16 weights, a delta per 8-weight group and d kept in four scale words;
 *   - IQ2_S (PR #2512 codec and PR #2565 encoder commit texts): the IQ2_XS search over a
 *     1024-entry grid with eight sign bits for each group (the input's signs, no parity flip);
 *   - decoding of the four layouts;
 *   - the local-Hessian choice search (PR #3158, fused in PR #3218 "[4/4] Run the local-Hessian
 *     choice search as one CUDA kernel"), and the same search over eight candidates per 8-weight
 *     group;
 *   - encoding under given block scales (PR #3197, static scales).
 *
 * The exact floating-point op sequence of every score is a fixed convention (it is what makes
 * payloads and picks bit-reproducible); it is documented next to each kernel.
 *
 * Memory: every pointer argument is DEVICE memory owned by the caller, except `desc`, which is a
 * host struct. The library never allocates device memory. Calls are asynchronous on `stream`:
 * they validate their arguments on the host, enqueue kernels and return. A non-IQ_OK status
 * means nothing was enqueued (except IQ_ECUDA, reported after a failed launch).
 *
 * Device-side findings (non-finite weights or Hessian values, bad importance, out-of-range
 * choices, d overflowing fp16, a grid value outside the format's alphabet) cannot be known on the
 * host. Blocks with a finding are written as the all-zero payload. How a call reports them depends
 * on `flags`:
 *   - flags != NULL (a caller-owned device uint32): the call stays asynchronous. It clears the word
 *     on `stream` and the kernels OR IQ_FLAG_* bits into it, so once the stream has passed the call
 *     the word holds exactly this call's findings; the status only covers the host-side checks.
 *   - flags == NULL: the call is SYNCHRONOUS. The kernels report into a word the library keeps on
 *     each device; the call waits for `stream` to finish it and returns the first finding as a
 *     status (IQ_ETIMEOUT, IQ_EGRID, IQ_ENONFINITE, IQ_EIMPORTANCE, IQ_ERANGE, IQ_ECHOICE, in that
 *     order of precedence), so bad data never comes back as IQ_OK. Such calls on one device are serialised
 *     by a host mutex held from clearing that word to reading it back.
 *
 * Requires an sm_100 (B200-class) device; other devices get IQ_EUNSUPPORTED.
 */
#ifndef IQ_B200_H
#define IQ_B200_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    IQ_OK = 0,
    IQ_EINVAL = 1,        /* NULL pointer, unknown format, bad descriptor or stride          */
    IQ_ESHAPE = 2,        /* empty tensor, or cols not a multiple of 256 ([512, 384] case)     */
    IQ_ECUDA = 3,         /* a CUDA runtime call or kernel launch failed                       */
    IQ_EUNSUPPORTED = 4,  /* the current device is not sm_100, or the call does not take the format */
    /* device-side findings, returned only by calls made with flags == NULL (see above)          */
    IQ_ENONFINITE = 5,    /* a weight (or, for the choice search, a Hessian value) is NaN or inf  */
    IQ_EIMPORTANCE = 6,   /* an importance value is NaN, infinite or negative (PR #2723 review)  */
    IQ_ERANGE = 7,        /* d rounds to fp16 infinity, or a given d is negative, infinite or NaN */
    IQ_ECHOICE = 8,       /* a given choice is >= the format's number of choices              */
    IQ_EGRID = 9,         /* a grid value lies outside the format's alphabet                   */
    IQ_ESCRATCH = 10,     /* iq_gptq_blocks_static: the call needs more than the library's 10 MiB */
    IQ_ETIMEOUT = 11      /* a kernel's bounded wait for its own copy ran out (see IQ_FLAG_TIMEOUT) */
} iq_status;

typedef enum { IQ_FMT_IQ1_S = 1, IQ_FMT_IQ2_XS = 2, IQ_FMT_IQ1_M = 3, IQ_FMT_IQ2_S = 4 } iq_format;

typedef enum { IQ_OUT_F32 = 0, IQ_OUT_BF16 = 1 } iq_out_dtype;

/* weight element types iq_encode takes (PR #2450: the encoders take fp32, f16 and bf16); each
 * converts to fp32 exactly and the search runs on those values */
typedef enum { IQ_IN_BF16 = 0, IQ_IN_F16 = 1, IQ_IN_F32 = 2 } iq_in_dtype;

/* device-side findings, ORed into *flags */
#define IQ_FLAG_NONFINITE 1u  /* a weight (choice search: or a Hessian value) is NaN or +-inf */
#define IQ_FLAG_IMPORTANCE 2u /* an importance value is NaN, +-inf or negative            */
#define IQ_FLAG_RANGE 4u      /* d rounds to fp16 infinity, or a given d is < 0, inf or NaN */
#define IQ_FLAG_CHOICE 8u     /* a given choice is >= 16                                  */
#define IQ_FLAG_GRID 16u      /* a grid value lies outside the format's alphabet           */
/* a CTA's bounded wait for one of its own bulk copies into shared memory ran out (about 0.1 s;
 * not expected on a working device): its row-blocks are written as the all-zero payload with
 * picks 0 and a NaN objective, and the CTA stops waiting */
#define IQ_FLAG_TIMEOUT 32u

/*
 * Codebook/convention descriptor (host struct; the grid it points to lives on the device).
 *   fmt           IQ_FMT_IQ1_S, IQ_FMT_IQ2_XS, IQ_FMT_IQ1_M or IQ_FMT_IQ2_S
 *   grid_entries  2048 (IQ1_S, IQ1_M), 512 (IQ2_XS) or 1024 (IQ2_S)
 *   grid          device int8 [grid_entries][8]; IQ1_S and IQ1_M values in {-1,0,1} (a ternary
 *                 grid, PR #2723; IQ1_M shares IQ1_S's, PR #2513), IQ2_XS and IQ2_S magnitudes in {1,3,5,7}.
 *                 Row q, column j multiplies weight j of a group.
 *   anchor        the scale predictor's anchor: d = fp16(fp32(amax / qmax) * anchor), with
 *                 qmax = 16.875 (IQ1_S, = 15 * 1.125, the largest |s (q + delta)| in units of d)
 *                 and 217 (IQ2_XS and IQ2_S, = 31 * 7). IQ1_S uses 0.61 (PR #2450 review). The
 *                 pages give no IQ2_XS or IQ2_S constant; this library's default is 0.9. IQ1_M ignores it: its anchor
 *                 is clamp(0.58 + 0.035 * amax / rms, 0.65, 0.95) per block (PR #2513), rms over
 *                 the block's 256 weights (squares summed per 8-weight group in order, the 32
 *                 group sums by a pairwise tree), with qmax = 16.875.
 */
typedef struct {
    int32_t fmt;
    int32_t grid_entries;
    const int8_t *grid;
    float anchor;
} iq_desc;
/*
 * Two convention values are deliberately not descriptor fields:
 *   - delta = +-1/8 (IQ1_S, IQ1_M; PR #2723, the PR #2450 worked example) belongs to the layout,
 *     not to the encoder: a payload stores only its sign bit, and every decoder of the format
 *     reads the value back as +-1/8. An encoder searching under another delta would write
 *     payloads that decode to values it never scored.
 *   - IQ1_M's anchor clamp(0.58 + 0.035 * peak_to_rms, 0.65, 0.95) is the format's own scale
 *     predictor (PR #2513); IQ1_S's flat 0.61 is the `anchor` field's default.
 */

/* Bytes per 256-weight block: 50 (IQ1_S), 74 (IQ2_XS), 56 (IQ1_M), 82 (IQ2_S); 0 for an unknown
 * format. */
size_t iq_block_bytes(int32_t fmt);

/* Payload bytes of a [rows, cols] weight: rows * (cols / 256) * iq_block_bytes(fmt); 0 for an
 * unknown format, a negative size or cols not a multiple of 256. */
size_t iq_payload_bytes(int32_t fmt, int64_t rows, int64_t cols);

/* Choice groups per block: 8 (IQ1_S, one per 32 weights: local scale + delta sign),
 * 16 (IQ2_XS and IQ2_S, one 4-bit local scale per 16 weights; IQ1_M, one 3-bit local scale per
 * 16 weights, each 8-weight group taking its own delta); 0 for an unknown format. */
int32_t iq_choice_groups(int32_t fmt);

/* Choices per group: 16 for IQ1_S (c = ls + 8 * [delta < 0]), IQ2_XS and IQ2_S (c = ls); 8 for
 * IQ1_M (c = ls); 0 for an unknown format. */
int32_t iq_num_choices(int32_t fmt);

/*
 * Encode `batch` weights of [rows, cols], elements of type w_dtype (IQ_IN_BF16 / IQ_IN_F16 bit
 * patterns, or IQ_IN_F32 values).
 *   w[e * w_batch_stride + r * ldw + col]        (elements; ldw >= cols)
 *   importance: NULL (all ones) or fp32 per input column,
 *     importance[e * imp_batch_stride + col]     (imp_batch_stride 0 shares one vector)
 *     values must be finite and >= 0 (PR #2723 review), else IQ_FLAG_IMPORTANCE.
 *   choices: NULL, or uint8 [batch][rows][cols/256][G] forcing each choice group's choice
 *     (PR #3157); entries, signs and IQ1_M's per-group deltas are still searched under it.
 *   scales: NULL to predict each block's d from its amax, or fp16 bit patterns giving every
 *     block's d (static scales, PR #3197, its "Static scales" item): block n of the flattened
 *     [batch][rows][cols/256] order takes d = scales[n * scales_stride] and is searched and packed
 *     under it whatever its amax. scales_stride >= 1 (uint16 elements): 1 for a dense array, or
 *     B/2 to read the d of an existing IQ1_S, IQ2_XS or IQ2_S payload in place (its first two
 *     bytes).
 *     A negative, infinite or NaN d gives the all-zero payload and IQ_FLAG_RANGE; d = +-0 gives
 *     the all-zero payload. Works with every mode.
 *   every_choice: 0, or 1 to write all C choices' payloads in one sweep (PR #3159):
 *     payload c equals the encode with choices = full(c). Must be 0 when choices != NULL.
 *   payload: uint8 [batch][rows][cols/256][B], or [C][batch][rows][cols/256][B] with every_choice
 *     (C = iq_num_choices(fmt)).
 * Per block ([#2450] layouts):
 *   IQ1_S  bytes 0-1 fp16 d; 2..33 low 8 bits of the 32 group indices; 34..49 eight LE uint16 qh,
 *          one per 32-weight sub-block: bits 0..11 the high 3 index bits of its 4 groups (shifts
 *          0,3,6,9), bits 12..14 local scale ls, bit 15 set for delta = -1/8.
 *   IQ2_XS bytes 0-1 fp16 d; 2..65 32 LE uint16 codes (9-bit index | 7-bit sign mask << 9, the
 *          8th sign by even parity); 66..73 sixteen 4-bit local scales, sub-block 2i in the low
 *          nibble of byte 66+i.
 *   IQ1_M  bytes 0..31 low 8 bits of the 32 group indices; 32..47 a nibble per group (group 2i in
 *          the low nibble of byte 32+i): 3 high index bits, bit 3 set for delta = -1/8; 48..55
 *          four LE uint16 scale words: word i holds the 3-bit ls of choice groups 4i..4i+3 at
 *          shifts 0,3,6,9 and bits 12..15 of word i are bits 4i..4i+3 of fp16 d (PR #2513).
 *   IQ2_S  bytes 0-1 fp16 d; 2..33 low 8 bits of the 32 group indices; 34..65 the groups' 8-bit
 *          sign masks (bit j set: element j negative); 66..73 the 2 high index bits, group g at
 *          shift 2 (g % 4) of byte 66 + g/4; 74..81 sixteen 4-bit local scales as IQ2_XS's.
 * Value of a weight: IQ1_S, IQ1_M d (2 ls + 1)(q + delta); IQ2_XS, IQ2_S d (2 ls + 1) g sign.
 * IQ1_M picks, per group and ls, the (delta, entry) of least error, the lower shift (+1/8) and
 * then the lower entry on equal error (PR #2595); a choice group's error is the sum of its two
 * groups'.
 * Without scales, amax == 0 or d rounding to fp16 zero gives the all-zero payload ([#2450]).
 * Alignment: w and importance 16-byte aligned, ldw and w_batch_stride multiples of 16 bytes (8
 * elements of bf16/f16, 4 of fp32),
 * imp_batch_stride a multiple of 4, payload and scales 2-byte aligned, grid 16-byte aligned
 * (IQ_EINVAL).
 */
iq_status iq_encode(const iq_desc *desc, const void *w, int32_t w_dtype, int64_t batch, int64_t rows,
                    int64_t cols, int64_t ldw, int64_t w_batch_stride, const float *importance,
                    int64_t imp_batch_stride, const uint8_t *choices, const uint16_t *scales,
                    int64_t scales_stride, int32_t every_choice, uint8_t *payload, uint32_t *flags, cudaStream_t stream);

/*
 * Decode nblocks contiguous payload blocks into [nblocks][256] values, fp32 (exact) or bf16
 * (round to nearest even of the exact value). Output is independent of how blocks are chunked.
 * payload must be 2-byte aligned and out 32-byte aligned (IQ_EINVAL otherwise). The grid must
 * lie in the format's alphabet (what iq_encode checks); other grid values decode unspecified.
 */
iq_status iq_decode(const iq_desc *desc, const uint8_t *payload, int64_t nblocks, int32_t out_dtype,
                    void *out, cudaStream_t stream);

/*
 * Local-Hessian choice search (PR #3158 steps; one fused launch as in PR #3218) for the first
 * nblk 256-column blocks of a [rows, ldw] bf16 weight, for every format (IQ1_M: 8 choices).
 *   hess: fp32 [rows / rows_per_hess][nblk][256][256], the symmetric diagonal blocks of the input
 *     Hessian, read as H[k][i] (row k, column i) for (H v)_i. Row r uses set r / rows_per_hess:
 *     a stack of experts that share a row layout runs in one call, each with its own Hessian
 *     (PR #3218: launch overhead dominated on MoE models). rows_per_hess = 0 means rows (one set);
 *     otherwise it must divide rows (IQ_ESHAPE).
 *   cand: the every-choice payloads of those blocks; candidate c of (row r, block b) starts at
 *     cand + c * cand_choice_stride + (r * cand_ld + b) * B   (bytes; cand_ld in blocks). cand is
 *     2-byte aligned and cand_choice_stride even (IQ_EINVAL otherwise).
 *   picks: uint8 [rows][nblk][G], the chosen choice of every choice group.
 *   payload: the final payload, block (r, b) at payload + (r * payload_ld + b) * B: each choice
 *     group's fields copied from its picked candidate, d from candidate 0 (the encode under the
 *     picks, PR #3157).
 *   objective: NULL, or fp32 [rows][nblk]: the final Delta^T H Delta of each row and block, as
 *     sum_i Delta_i grad_i over the search's final gradient (a pairwise tree over the columns).
 * Steps per (row, block): Delta(c) = x - decode(cand c); each group takes its best choice under
 * its own H_gg; grad = H Delta; two sweeps over the groups in order, each taking the choice with
 * the least gain 2 u^T grad_g + u^T H_gg u (u = Delta_g(c) - Delta_g(cur)) iff that gain < 0,
 * then grad += H[:, g] u. Lowest choice on equal score or gain.
 * Findings (IQ_FLAG_NONFINITE: a non-finite weight in the row-block or a non-finite entry of its
 * Hessian block; IQ_FLAG_GRID: a grid value outside the candidates' alphabet) make that
 * row-block report picks 0 (the first candidate), the all-zero payload and a NaN objective
 * (bits 0x7FC00000); the other row-blocks are unaffected. The kernel streams H in bulk copies
 * and bounds every wait for them; a wait that runs out (IQ_FLAG_TIMEOUT, not expected on a
 * working device) reports the row-blocks of its CTA the same way.
 */
iq_status iq_choice_search(const iq_desc *desc, const uint16_t *w, int64_t rows, int64_t nblk,
                           int64_t ldw, const float *hess, int64_t rows_per_hess, const uint8_t *cand,
                           int64_t cand_ld, int64_t cand_choice_stride, uint8_t *picks, uint8_t *payload,
                           int64_t payload_ld, float *objective, uint32_t *flags, cudaStream_t stream);

/*
 * The same search with eight candidates per 8-weight group: 32 groups of 8 columns per block,
 * each choosing among the IQ2_XS every-choice decodes for ls = 8..15 (PR #3158's steps, only the
 * grouping differs; the 16-column search above is IQ2_XS's native one). desc must be IQ2_XS
 * (IQ_EUNSUPPORTED otherwise). w, hess, rows_per_hess, objective and flags as above.
 *   cand: the 16-choice IQ2_XS every-choice payloads, addressed as above; only choices 8..15 are
 *     read.
 *   picks: uint8 [rows][nblk][32], the chosen ls (8..15) of every 8-column group.
 * No payload is written: no IQ layout stores a scale per 8 weights.
 */
iq_status iq_choice_search_g8(const iq_desc *desc, const uint16_t *w, int64_t rows, int64_t nblk, int64_t ldw,
                              const float *hess, int64_t rows_per_hess, const uint8_t *cand, int64_t cand_ld,
                              int64_t cand_choice_stride, uint8_t *picks, float *objective, uint32_t *flags,
                              cudaStream_t stream);

/*
 * The per-block calibration loop over one weight in a single call (PR #3218: "GPTQ with
 * local_hessian_scales searches one block at a time"), with GPTQ's error propagation between the
 * blocks (Frantar et al. 2022, "GPTQ: Accurate Post-Training Quantization for Generative
 * Pre-trained Transformers", one 256-column block per lazy batch). Every row independently:
 *   w_work = fp32(w); for b = 0 .. cols/256 - 1, in order:
 *     x = w_work[:, block b]; the every-choice encode of x under importance sqrt(diag H_b);
 *     the local-Hessian choice search of x under H_b (iq_choice_search's steps and findings)
 *       -> picks[:, b], payload[:, b] and E = x - decode(payload[:, b]);
 *     Y = E U_bb^-1 (forward substitution: column j starts from E_j, takes fma(-Y_k, U[k][j], .)
 *       for k < j ascending, then Y_j = acc / U[j][j]); every later column j' of w_work takes
 *       fma(-Y_k, U[256 b + k][j'], .) for k = 0..255 ascending.
 *   U is the upper-triangular Cholesky factor of the weight's inverse Hessian (H^-1 = U^T U),
 *   fp32 [cols][ldu], read on and above the diagonal; block b's local Hessian is
 *   H_b = U_bb^-1 U_bb^-T, given in hess [cols/256][256][256] as iq_choice_search reads it.
 *   w: bf16 [rows][ldw]; payload [rows][cols/256][B]; picks [rows][cols/256][G];
 *   w_work: fp32 [rows][cols], caller-owned output: on return its block b holds the weights
 *     block b was quantised from.
 *   workspace: device scratch of at least iq_gptq_workspace_bytes(fmt, rows) bytes, 256-byte
 *     aligned, owned by the caller (the candidates of one block, its error and its importance);
 *     its contents on return mean nothing.
 * All blocks are enqueued on `stream` in order, with no host synchronisation between them (with a
 * flags word; without one the call waits at its end, as every call does). Alignment: w, hess, U
 * and w_work 16-byte aligned, ldw a multiple of 8, ldu of 4 (IQ_EINVAL otherwise).
 */
size_t iq_gptq_workspace_bytes(int32_t fmt, int64_t rows);
iq_status iq_gptq_blocks(const iq_desc *desc, const uint16_t *w, int64_t rows, int64_t cols, int64_t ldw,
                         const float *hess, const float *U, int64_t ldu, void *workspace, size_t workspace_bytes,
                         uint8_t *payload, uint8_t *picks, float *w_work, uint32_t *flags, cudaStream_t stream);

/*
 * iq_gptq_blocks without a workspace argument, for callers that cannot allocate device memory
 * where they call it: code inside another framework's memory pool, which owns the free HBM;
 * code held to a fixed device-memory budget from the moment it was loaded; code on a path where
 * cudaMalloc's implicit device synchronisation cannot be afforded. The pages have no counterpart:
 * this entry point exists for those callers only.
 *   Scratch: a 10 MiB device array inside the library (every GPU that loads the library holds one
 *   until the process exits). Calls whose iq_gptq_workspace_bytes(fmt, rows) exceeds 10 MiB get
 *   IQ_ESCRATCH and enqueue nothing; 10 MiB covers 4096 rows in every format.
 *   Set-up: the first call on a device looks up that device's address of the array (with the
 *   device current); make that first call before any stream capture.
 *   Sharing: every call uses the same array and leaves its contents behind. Nothing in it needs
 *   clearing (each call writes every scratch byte it reads), but calls that overlap on the GPU,
 *   from two streams or two host threads, race on it: order them.
 *   Everything else (arguments, outputs, findings, statuses) is exactly iq_gptq_blocks's, and
 *   the call allocates no device memory.
 */
iq_status iq_gptq_blocks_static(const iq_desc *desc, const uint16_t *w, int64_t rows, int64_t cols, int64_t ldw,
                                const float *hess, const float *U, int64_t ldu, uint8_t *payload, uint8_t *picks,
                                float *w_work, uint32_t *flags, cudaStream_t stream);

/*
 * out[b * 256 + i] = sqrtf(hess[b][i][i]) for b < nblk: the search importance the local-Hessian
 * calibration uses for the every-choice candidates (square root of the Hessian diagonal, PR #3158).
 */
iq_status iq_sqrt_diag(const float *hess, int64_t nblk, float *out, cudaStream_t stream);

/* A static, human-readable name for a status code. */
const char *iq_status_string(iq_status s);

/* Build information: compiler, target architecture, kernel configuration. */
const char *iq_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* IQ_B200_H */

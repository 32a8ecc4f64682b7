// iq_kernels.h -- internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime_api.h>
#include <stdint.h>

namespace iqk {

enum EncodeMode { kSearch = 0, kFixed = 1, kEvery = 2 };

struct EncodeParams {
    const void* w;
    int w_dtype;  // IQ_IN_BF16, IQ_IN_F16 or IQ_IN_F32
    int64_t rows, nblk, ldw, w_bstride;
    const float* imp;  // nullptr: all ones
    int64_t imp_bstride;
    const uint8_t* choices;  // kFixed only
    const uint16_t* scales;  // nullptr: predict d from amax; else fp16 bits of block b's d at
    int64_t scales_stride;   // scales[b * scales_stride]
    uint8_t* payload;
    uint32_t* flags;
    const int8_t* grid;
    float anchor;
    int64_t nb;  // batch * rows * nblk
};

struct DecodeParams {
    const uint8_t* payload;
    int64_t nblocks;
    const int8_t* grid;
    void* out;
};

struct ChoiceParams {
    const void* w;     // bf16 bits, or fp32 values when w_f32
    int w_f32;
    int64_t rows, nblk, ldw;
    // the launch covers blocks blk0 .. blk0 + nblk_run - 1 of the nblk; candidate block b sits at
    // block index b - cand_blk0 of cand
    int64_t blk0, nblk_run, cand_blk0;
    const float* hess;
    int64_t rows_per_hess;  // row r uses Hessian set r / rows_per_hess (divides rows)
    const uint8_t* cand;
    int64_t cand_ld, cand_cstride;
    uint8_t* picks;
    uint8_t* payload;
    int64_t payload_ld;
    float* objective;  // nullptr, or [rows][nblk]: the final Delta^T H Delta
    float* delta_out;  // nullptr, or [rows][256] (one block per launch): the final Delta
    uint32_t* flags;
    const int8_t* grid;
};

struct GptqUpdateParams {
    float* w;           // the working weight [rows][ldw] (fp32), updated in place
    const float* y;     // [rows][256]: E U_bb^-1 of the block just quantised
    const float* u;     // rows o .. o + 255 of the inverse-Hessian factor, [256][ldu]
    int64_t rows, ldw, ldu;
    int64_t col0, ncols;  // the columns to update: col0 .. col0 + ncols - 1
};

// Choice-search layout code beside the iq_format values (not a payload format): IQ2_XS
// candidates searched over 32 groups of 8 columns, eight candidates (ls = 8..15) per group,
// picks only. The caller points cand at the candidate for ls = 8.
constexpr int kChoiceIq2xsG8 = 5;
constexpr int kChoiceG8FirstLs = 8;

// Each returns the cudaError_t of its launch (cudaSuccess when nothing had to run).
cudaError_t launch_iq1_encode(int fmt, const EncodeParams& p, int mode, int num_sms, cudaStream_t s);
cudaError_t launch_iq2_encode(int fmt, const EncodeParams& p, int mode, int num_sms, cudaStream_t s);
cudaError_t launch_decode(int fmt, bool bf16, const DecodeParams& p, int num_sms, cudaStream_t s);
cudaError_t launch_choice_search(int fmt, const ChoiceParams& p, int num_sms, cudaStream_t s);
cudaError_t launch_sqrt_diag(const float* hess, int64_t nblk, float* out, cudaStream_t s);
// The per-block calibration loop's pieces: bf16 -> fp32 copy of the weight; Y = E U_bb^-1 in
// place per row; W[:, cols] -= Y U_b,cols.
cudaError_t launch_bf16_to_f32(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw, float* out, cudaStream_t s);
cudaError_t launch_gptq_solve(float* e, const float* ubb, int64_t ldu, int64_t rows, cudaStream_t s);
cudaError_t launch_gptq_update(const GptqUpdateParams& p, int num_sms, cudaStream_t s);

}  // namespace iqk

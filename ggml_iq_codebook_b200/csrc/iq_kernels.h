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
    const uint16_t* w;
    int64_t rows, nblk, ldw;
    const float* hess;
    int64_t rows_per_hess;  // row r uses Hessian set r / rows_per_hess (divides rows)
    const uint8_t* cand;
    int64_t cand_ld, cand_cstride;
    uint8_t* picks;
    uint8_t* payload;
    int64_t payload_ld;
    float* objective;  // nullptr, or [rows][nblk]: the final Delta^T H Delta
    uint32_t* flags;
    const int8_t* grid;
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

}  // namespace iqk

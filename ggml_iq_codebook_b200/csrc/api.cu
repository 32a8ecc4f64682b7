// api.cu -- the C ABI (include/iq.h): argument validation on the host, then kernel launches.
#include <atomic>
#include <cmath>
#include <mutex>

#include "iq.h"
#include "iq_kernels.h"

#define IQ_STR_(x) #x
#define IQ_STR(x) IQ_STR_(x)

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];  // 0 unknown, -1 unsupported, >0 SM count

// The current device must be an sm_100 part; returns its SM count (cached per device).
iq_status device_sms(int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return IQ_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return IQ_EUNSUPPORTED;
    int v = g_sms[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        int major = 0, minor = 0, count = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return IQ_ECUDA;
        v = (major == 10 && minor == 0) ? count : -1;
        g_sms[dev].store(v, std::memory_order_relaxed);
    }
    if (v < 0) return IQ_EUNSUPPORTED;
    *sms = v;
    return IQ_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

iq_status check_desc(const iq_desc* d) {
    if (d == nullptr || d->grid == nullptr) return IQ_EINVAL;
    if (d->fmt == IQ_FMT_IQ1_S || d->fmt == IQ_FMT_IQ1_M) {
        if (d->grid_entries != 2048) return IQ_EINVAL;
    } else if (d->fmt == IQ_FMT_IQ2_XS) {
        if (d->grid_entries != 512) return IQ_EINVAL;
    } else if (d->fmt == IQ_FMT_IQ2_S) {
        if (d->grid_entries != 1024) return IQ_EINVAL;
    } else {
        return IQ_EINVAL;
    }
    if (!aligned(d->grid, 16)) return IQ_EINVAL;
    // IQ1_M derives its anchor from each block; the others take it from the descriptor.
    if (d->fmt != IQ_FMT_IQ1_M && (!std::isfinite(d->anchor) || !(d->anchor > 0.0f))) return IQ_EINVAL;
    return IQ_OK;
}

iq_status launched(cudaError_t e) { return e == cudaSuccess ? IQ_OK : IQ_ECUDA; }

}  // namespace

// The findings word of calls made without one: one per device (a __device__ variable has an
// instance on every device that loads the library). Such calls hold the device's mutex from
// clearing the word to reading it back, so two of them never share it.
__device__ uint32_t g_own_flags;

namespace {

std::mutex g_own_flags_mutex[kMaxDevices];

// The flags word a call reports through: the caller's device word (cleared on the stream, read
// by the caller), or, when the caller passes none, the library's own word, read back after the
// stream has finished the call and turned into a status.
class FlagsWord {
  public:
    explicit FlagsWord(uint32_t* caller) : caller_(caller) {}
    ~FlagsWord() {
        if (locked_) g_own_flags_mutex[dev_].unlock();
    }
    iq_status begin(cudaStream_t s) {
        uint32_t* w = caller_;
        if (w == nullptr) {
            if (cudaGetDevice(&dev_) != cudaSuccess) return IQ_ECUDA;
            if (dev_ < 0 || dev_ >= kMaxDevices) return IQ_EUNSUPPORTED;
            g_own_flags_mutex[dev_].lock();
            locked_ = true;
            if (cudaGetSymbolAddress(reinterpret_cast<void**>(&own_), g_own_flags) != cudaSuccess) return IQ_ECUDA;
            w = own_;
        }
        return cudaMemsetAsync(w, 0, sizeof(uint32_t), s) == cudaSuccess ? IQ_OK : IQ_ECUDA;
    }
    uint32_t* ptr() const { return caller_ != nullptr ? caller_ : own_; }
    // The call's status: `st` itself when the launch failed or the caller keeps the word;
    // otherwise the library's word is read once the stream is done, and a finding becomes
    // IQ_ETIMEOUT, IQ_EGRID, IQ_ENONFINITE, IQ_EIMPORTANCE, IQ_ERANGE or IQ_ECHOICE (first match
    // wins).
    iq_status finish(iq_status st, cudaStream_t s) {
        if (st != IQ_OK || caller_ != nullptr) return st;
        uint32_t f = 0;
        if (cudaMemcpyAsync(&f, own_, sizeof(f), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return IQ_ECUDA;
        if (f & IQ_FLAG_TIMEOUT) return IQ_ETIMEOUT;
        if (f & IQ_FLAG_GRID) return IQ_EGRID;
        if (f & IQ_FLAG_NONFINITE) return IQ_ENONFINITE;
        if (f & IQ_FLAG_IMPORTANCE) return IQ_EIMPORTANCE;
        if (f & IQ_FLAG_RANGE) return IQ_ERANGE;
        if (f & IQ_FLAG_CHOICE) return IQ_ECHOICE;
        return IQ_OK;
    }

  private:
    uint32_t* caller_;
    uint32_t* own_ = nullptr;
    int dev_ = 0;
    bool locked_ = false;
};

}  // namespace

extern "C" {

size_t iq_block_bytes(int32_t fmt) {
    return fmt == IQ_FMT_IQ1_S ? 50 : fmt == IQ_FMT_IQ2_XS ? 74 : fmt == IQ_FMT_IQ1_M ? 56 : fmt == IQ_FMT_IQ2_S ? 82 : 0;
}

int32_t iq_choice_groups(int32_t fmt) {
    return fmt == IQ_FMT_IQ1_S ? 8 : (fmt == IQ_FMT_IQ2_XS || fmt == IQ_FMT_IQ1_M || fmt == IQ_FMT_IQ2_S) ? 16 : 0;
}

int32_t iq_num_choices(int32_t fmt) {
    return (fmt == IQ_FMT_IQ1_S || fmt == IQ_FMT_IQ2_XS || fmt == IQ_FMT_IQ2_S) ? 16 : fmt == IQ_FMT_IQ1_M ? 8 : 0;
}

size_t iq_payload_bytes(int32_t fmt, int64_t rows, int64_t cols) {
    const size_t b = iq_block_bytes(fmt);
    if (b == 0 || rows < 0 || cols < 0 || cols % 256 != 0) return 0;
    return static_cast<size_t>(rows) * static_cast<size_t>(cols / 256) * b;
}

iq_status iq_encode(const iq_desc* desc, const void* w, int32_t w_dtype, int64_t batch, int64_t rows, int64_t cols,
                    int64_t ldw, int64_t w_batch_stride, const float* importance,
                    int64_t imp_batch_stride, const uint8_t* choices, const uint16_t* scales,
                    int64_t scales_stride, int32_t every_choice, uint8_t* payload, uint32_t* flags, cudaStream_t stream) {
    iq_status st = check_desc(desc);
    if (st != IQ_OK) return st;
    if (w == nullptr || payload == nullptr) return IQ_EINVAL;
    if (batch <= 0 || rows <= 0 || cols <= 0 || cols % 256 != 0) return IQ_ESHAPE;
    if (w_dtype != IQ_IN_BF16 && w_dtype != IQ_IN_F16 && w_dtype != IQ_IN_F32) return IQ_EINVAL;
    const int64_t vec = w_dtype == IQ_IN_F32 ? 4 : 8;  // elements per 16 bytes
    if (ldw < cols || ldw % vec != 0 || !aligned(w, 16)) return IQ_EINVAL;
    if (batch > 1 && (w_batch_stride < (rows - 1) * ldw + cols || w_batch_stride % vec != 0)) return IQ_EINVAL;
    if (importance != nullptr) {
        if (!aligned(importance, 16) || imp_batch_stride < 0 || imp_batch_stride % 4 != 0) return IQ_EINVAL;
        if (batch > 1 && imp_batch_stride != 0 && imp_batch_stride < cols) return IQ_EINVAL;
    }
    if (every_choice != 0 && every_choice != 1) return IQ_EINVAL;
    if (every_choice && choices != nullptr) return IQ_EINVAL;
    if (!aligned(payload, 2) || (scales != nullptr && (!aligned(scales, 2) || scales_stride < 1)))
        return IQ_EINVAL;
    int sms = 0;
    if ((st = device_sms(&sms)) != IQ_OK) return st;
    FlagsWord fw(flags);
    if ((st = fw.begin(stream)) != IQ_OK) return st;

    iqk::EncodeParams p;
    p.w = w;
    p.w_dtype = w_dtype;
    p.rows = rows;
    p.nblk = cols / 256;
    p.ldw = ldw;
    p.w_bstride = batch > 1 ? w_batch_stride : 0;
    p.imp = importance;
    p.imp_bstride = importance != nullptr ? imp_batch_stride : 0;
    p.choices = choices;
    p.scales = scales;
    p.scales_stride = scales != nullptr ? scales_stride : 0;
    p.payload = payload;
    p.flags = fw.ptr();
    p.grid = desc->grid;
    p.anchor = desc->anchor;
    p.nb = batch * rows * (cols / 256);
    const int mode = every_choice ? iqk::kEvery : (choices != nullptr ? iqk::kFixed : iqk::kSearch);
    const bool iq2 = desc->fmt == IQ_FMT_IQ2_XS || desc->fmt == IQ_FMT_IQ2_S;
    return fw.finish(launched(iq2 ? iqk::launch_iq2_encode(desc->fmt, p, mode, sms, stream)
                                  : iqk::launch_iq1_encode(desc->fmt, p, mode, sms, stream)),
                     stream);
}

iq_status iq_decode(const iq_desc* desc, const uint8_t* payload, int64_t nblocks, int32_t out_dtype,
                    void* out, cudaStream_t stream) {
    iq_status st = check_desc(desc);
    if (st != IQ_OK) return st;
    if (payload == nullptr || out == nullptr) return IQ_EINVAL;
    if (nblocks <= 0) return IQ_ESHAPE;
    if (out_dtype != IQ_OUT_F32 && out_dtype != IQ_OUT_BF16) return IQ_EINVAL;
    if (!aligned(out, 32) || !aligned(payload, 2)) return IQ_EINVAL;
    int sms = 0;
    if ((st = device_sms(&sms)) != IQ_OK) return st;
    iqk::DecodeParams p;
    p.payload = payload;
    p.nblocks = nblocks;
    p.grid = desc->grid;
    p.out = out;
    return launched(iqk::launch_decode(desc->fmt, out_dtype == IQ_OUT_BF16, p, sms, stream));
}

iq_status iq_choice_search(const iq_desc* desc, const uint16_t* w, int64_t rows, int64_t nblk,
                           int64_t ldw, const float* hess, int64_t rows_per_hess, const uint8_t* cand, int64_t cand_ld,
                           int64_t cand_choice_stride, uint8_t* picks, uint8_t* payload,
                           int64_t payload_ld, float* objective, uint32_t* flags, cudaStream_t stream) {
    iq_status st = check_desc(desc);
    if (st != IQ_OK) return st;
    if (w == nullptr || hess == nullptr || cand == nullptr || picks == nullptr || payload == nullptr)
        return IQ_EINVAL;
    if (rows <= 0 || nblk <= 0) return IQ_ESHAPE;
    if (ldw < nblk * 256 || ldw % 8 != 0 || !aligned(w, 16) || !aligned(hess, 16)) return IQ_EINVAL;
    if (cand_ld < nblk || payload_ld < nblk || cand_choice_stride < 0) return IQ_EINVAL;
    if (!aligned(cand, 2) || (cand_choice_stride & 1) != 0) return IQ_EINVAL;  // 2-byte staging
    if (rows_per_hess == 0) rows_per_hess = rows;
    if (rows_per_hess < 0 || rows % rows_per_hess != 0) return IQ_ESHAPE;
    int sms = 0;
    if ((st = device_sms(&sms)) != IQ_OK) return st;
    FlagsWord fw(flags);
    if ((st = fw.begin(stream)) != IQ_OK) return st;
    iqk::ChoiceParams p;
    p.w = w;
    p.w_f32 = 0;
    p.rows = rows;
    p.nblk = nblk;
    p.ldw = ldw;
    p.blk0 = 0;
    p.nblk_run = nblk;
    p.cand_blk0 = 0;
    p.delta_out = nullptr;
    p.hess = hess;
    p.rows_per_hess = rows_per_hess;
    p.cand = cand;
    p.cand_ld = cand_ld;
    p.cand_cstride = cand_choice_stride;
    p.picks = picks;
    p.payload = payload;
    p.payload_ld = payload_ld;
    p.objective = objective;
    p.flags = fw.ptr();
    p.grid = desc->grid;
    return fw.finish(launched(iqk::launch_choice_search(desc->fmt, p, sms, stream)), stream);
}

iq_status iq_choice_search_g8(const iq_desc* desc, const uint16_t* w, int64_t rows, int64_t nblk, int64_t ldw,
                              const float* hess, int64_t rows_per_hess, const uint8_t* cand, int64_t cand_ld,
                              int64_t cand_choice_stride, uint8_t* picks, float* objective, uint32_t* flags,
                              cudaStream_t stream) {
    iq_status st = check_desc(desc);
    if (st != IQ_OK) return st;
    if (desc->fmt != IQ_FMT_IQ2_XS) return IQ_EUNSUPPORTED;
    if (w == nullptr || hess == nullptr || cand == nullptr || picks == nullptr) return IQ_EINVAL;
    if (rows <= 0 || nblk <= 0) return IQ_ESHAPE;
    if (ldw < nblk * 256 || ldw % 8 != 0 || !aligned(w, 16) || !aligned(hess, 16)) return IQ_EINVAL;
    if (cand_ld < nblk || cand_choice_stride < 0) return IQ_EINVAL;
    if (!aligned(cand, 2) || (cand_choice_stride & 1) != 0) return IQ_EINVAL;  // 2-byte staging
    if (rows_per_hess == 0) rows_per_hess = rows;
    if (rows_per_hess < 0 || rows % rows_per_hess != 0) return IQ_ESHAPE;
    int sms = 0;
    if ((st = device_sms(&sms)) != IQ_OK) return st;
    FlagsWord fw(flags);
    if ((st = fw.begin(stream)) != IQ_OK) return st;
    iqk::ChoiceParams p;
    p.w = w;
    p.w_f32 = 0;
    p.rows = rows;
    p.nblk = nblk;
    p.ldw = ldw;
    p.blk0 = 0;
    p.nblk_run = nblk;
    p.cand_blk0 = 0;
    p.delta_out = nullptr;
    p.hess = hess;
    p.rows_per_hess = rows_per_hess;
    p.cand = cand + iqk::kChoiceG8FirstLs * cand_choice_stride;  // the candidate for ls = 8
    p.cand_ld = cand_ld;
    p.cand_cstride = cand_choice_stride;
    p.picks = picks;
    p.payload = nullptr;
    p.payload_ld = 0;
    p.objective = objective;
    p.flags = fw.ptr();
    p.grid = desc->grid;
    return fw.finish(launched(iqk::launch_choice_search(iqk::kChoiceIq2xsG8, p, sms, stream)), stream);
}

namespace {
size_t round256(size_t n) { return (n + 255) / 256 * 256; }
}  // namespace

size_t iq_gptq_workspace_bytes(int32_t fmt, int64_t rows) {
    const size_t b = iq_block_bytes(fmt), c = static_cast<size_t>(iq_num_choices(fmt));
    if (b == 0 || rows <= 0) return 0;
    const size_t r = static_cast<size_t>(rows);
    return round256(256 * sizeof(float)) + round256(c * r * b) + round256(r * 256 * sizeof(float));
}

iq_status iq_gptq_blocks(const iq_desc* desc, const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw,
                         const float* hess, const float* U, int64_t ldu, void* workspace, size_t workspace_bytes,
                         uint8_t* payload, uint8_t* picks, float* w_work, uint32_t* flags, cudaStream_t stream) {
    iq_status st = check_desc(desc);
    if (st != IQ_OK) return st;
    if (w == nullptr || hess == nullptr || U == nullptr || workspace == nullptr || payload == nullptr ||
        picks == nullptr || w_work == nullptr)
        return IQ_EINVAL;
    if (rows <= 0 || cols <= 0 || cols % 256 != 0) return IQ_ESHAPE;
    if (ldw < cols || ldw % 8 != 0 || !aligned(w, 16) || !aligned(hess, 16)) return IQ_EINVAL;
    if (ldu < cols || ldu % 4 != 0 || !aligned(U, 16) || !aligned(w_work, 16) || !aligned(payload, 2)) return IQ_EINVAL;
    if (!aligned(workspace, 256) || workspace_bytes < iq_gptq_workspace_bytes(desc->fmt, rows)) return IQ_EINVAL;
    int sms = 0;
    if ((st = device_sms(&sms)) != IQ_OK) return st;
    FlagsWord fw(flags);
    if ((st = fw.begin(stream)) != IQ_OK) return st;

    const int64_t nblk = cols / 256, B = static_cast<int64_t>(iq_block_bytes(desc->fmt));
    char* ws = static_cast<char*>(workspace);
    float* imp = reinterpret_cast<float*>(ws);
    uint8_t* cand = reinterpret_cast<uint8_t*>(ws + round256(256 * sizeof(float)));
    float* e = reinterpret_cast<float*>(ws + round256(256 * sizeof(float)) +
                                        round256(static_cast<size_t>(iq_num_choices(desc->fmt)) * rows * B));
    const bool iq2 = desc->fmt == IQ_FMT_IQ2_XS || desc->fmt == IQ_FMT_IQ2_S;

    cudaError_t err = iqk::launch_bf16_to_f32(w, rows, cols, ldw, w_work, stream);
    for (int64_t b = 0; b < nblk && err == cudaSuccess; ++b) {
        const int64_t o = 256 * b;
        // the block's candidates: the every-choice encode of the compensated weights under
        // sqrt(diag H_b)
        err = iqk::launch_sqrt_diag(hess + o * 256, 1, imp, stream);
        if (err != cudaSuccess) break;
        iqk::EncodeParams ep;
        ep.w = w_work + o;
        ep.w_dtype = IQ_IN_F32;
        ep.rows = rows;
        ep.nblk = 1;
        ep.ldw = cols;
        ep.w_bstride = 0;
        ep.imp = imp;
        ep.imp_bstride = 0;
        ep.choices = nullptr;
        ep.scales = nullptr;
        ep.scales_stride = 0;
        ep.payload = cand;
        ep.flags = fw.ptr();
        ep.grid = desc->grid;
        ep.anchor = desc->anchor;
        ep.nb = rows;
        err = iq2 ? iqk::launch_iq2_encode(desc->fmt, ep, iqk::kEvery, sms, stream)
                  : iqk::launch_iq1_encode(desc->fmt, ep, iqk::kEvery, sms, stream);
        if (err != cudaSuccess) break;
        // the local-Hessian search of block b, which also leaves the block's final Delta in e
        iqk::ChoiceParams cp;
        cp.w = w_work;
        cp.w_f32 = 1;
        cp.rows = rows;
        cp.nblk = nblk;
        cp.ldw = cols;
        cp.blk0 = b;
        cp.nblk_run = 1;
        cp.cand_blk0 = b;
        cp.hess = hess;
        cp.rows_per_hess = rows;
        cp.cand = cand;
        cp.cand_ld = 1;
        cp.cand_cstride = rows * B;
        cp.picks = picks;
        cp.payload = payload;
        cp.payload_ld = nblk;
        cp.objective = nullptr;
        cp.delta_out = e;
        cp.flags = fw.ptr();
        cp.grid = desc->grid;
        err = iqk::launch_choice_search(desc->fmt, cp, sms, stream);
        if (err != cudaSuccess || b + 1 == nblk) break;
        // GPTQ's compensation of the later columns
        err = iqk::launch_gptq_solve(e, U + o * ldu + o, ldu, rows, stream);
        if (err != cudaSuccess) break;
        iqk::GptqUpdateParams up;
        up.w = w_work;
        up.y = e;
        up.u = U + o * ldu;
        up.rows = rows;
        up.ldw = cols;
        up.ldu = ldu;
        up.col0 = o + 256;
        up.ncols = cols - o - 256;
        err = iqk::launch_gptq_update(up, sms, stream);
    }
    return fw.finish(launched(err), stream);
}

iq_status iq_sqrt_diag(const float* hess, int64_t nblk, float* out, cudaStream_t stream) {
    if (hess == nullptr || out == nullptr) return IQ_EINVAL;
    if (nblk <= 0) return IQ_ESHAPE;
    int sms = 0;
    iq_status st = device_sms(&sms);
    if (st != IQ_OK) return st;
    return launched(iqk::launch_sqrt_diag(hess, nblk, out, stream));
}

const char* iq_status_string(iq_status s) {
    switch (s) {
        case IQ_OK: return "ok";
        case IQ_EINVAL: return "invalid argument";
        case IQ_ESHAPE: return "invalid shape (empty, or columns not a multiple of 256)";
        case IQ_ECUDA: return "CUDA error";
        case IQ_EUNSUPPORTED: return "device is not sm_100, or the call does not take this format";
        case IQ_ENONFINITE: return "a weight or Hessian value is NaN or infinite";
        case IQ_EIMPORTANCE: return "an importance value is NaN, infinite or negative";
        case IQ_ERANGE: return "a block scale overflows fp16, or a given scale is negative, infinite or NaN";
        case IQ_ECHOICE: return "a given choice is out of the format's range";
        case IQ_EGRID: return "a grid value lies outside the format's alphabet";
        case IQ_ESCRATCH: return "the call needs more scratch than the library's static 10 MiB array";
        case IQ_ETIMEOUT: return "a kernel's bounded wait for its own copy ran out";
        default: return "unknown status";
    }
}

const char* iq_build_info(void) {
    return "libiq_b200: nvcc " IQ_STR(__CUDACC_VER_MAJOR__) "." IQ_STR(__CUDACC_VER_MINOR__)
           ", sm_100a, -fmad=false; encode: warp per block, lane per group, persistent CTAs";
}

}  // extern "C"

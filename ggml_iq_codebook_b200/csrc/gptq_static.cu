// gptq_static.cu -- the per-block calibration loop for callers that cannot allocate device memory.
//
// iq_gptq_blocks needs a few MiB of scratch per call (one block's candidates, its error rows and
// its importance), which its caller allocates and passes in. Some callers cannot do that at the
// point of the call: code running inside another framework's memory pool (which owns the free
// HBM and must not be bypassed by a cudaMalloc), code under a fixed device-memory budget set when
// it was loaded, or code on a path where cudaMalloc's implicit device synchronisation is not
// acceptable. For them this file keeps the scratch in the library itself: one file-scope device
// array of a fixed size, which every GPU that loads the library holds until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it is only a stand-in
// symbol), so each device's address is looked up once, with that device current, through
// cudaGetSymbolAddress, and passed to the kernels like any caller-owned workspace.
#include <mutex>

#include "iq.h"

namespace {
constexpr size_t kStaticScratchBytes = size_t{10} << 20;  // 10 MiB
constexpr int kMaxDevices = 64;
}  // namespace

// The scratch of iq_gptq_blocks_static: one instance on every device that loads the library.
static __device__ __align__(256) unsigned char g_gptq_scratch[kStaticScratchBytes];

namespace {

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices];  // device address per device, filled on its first call

// The current device's address of g_gptq_scratch (set up once per device, then cached).
iq_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return IQ_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return IQ_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gptq_scratch) != cudaSuccess || p == nullptr) return IQ_ECUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return IQ_OK;
}

}  // namespace

extern "C" iq_status iq_gptq_blocks_static(const iq_desc* desc, const uint16_t* w, int64_t rows, int64_t cols,
                                           int64_t ldw, const float* hess, const float* U, int64_t ldu,
                                           uint8_t* payload, uint8_t* picks, float* w_work, uint32_t* flags,
                                           cudaStream_t stream) {
    if (desc == nullptr) return IQ_EINVAL;
    if (rows <= 0) return IQ_ESHAPE;
    const size_t need = iq_gptq_workspace_bytes(desc->fmt, rows);
    if (need == 0) return IQ_EINVAL;
    if (need > kStaticScratchBytes) return IQ_ESCRATCH;
    void* scratch = nullptr;
    const iq_status st = scratch_address(&scratch);
    if (st != IQ_OK) return st;
    // Every scratch byte the loop reads is written earlier in the same call, so the previous
    // call's contents need no clearing.
    return iq_gptq_blocks(desc, w, rows, cols, ldw, hess, U, ldu, scratch, kStaticScratchBytes, payload, picks,
                          w_work, flags, stream);
}

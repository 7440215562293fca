// Allocation-free variant of the stand-alone entropy selection.
//
// wedlm_entropy_select takes the per-row flags and per-chunk (max, sum,
// weighted sum, argmax) partials it needs from cudaMallocAsync.  Some callers
// cannot allow that: a runtime that has already reserved the whole device for
// its own pool (so any further cudaMalloc fails or fragments what it
// manages), or a host thread that must not take the allocator's locks or risk
// the device-wide synchronisation an allocation can cause (the call still waits
// for the one stream it is given, as wedlm_entropy_select does).  This file
// gives them the same computation with its scratch in a fixed device array
// owned by the library image instead.
//
// The array lives in every GPU that loads the library until the process
// exits.  In host code its name is only a host-side stand-in for the symbol,
// never a device address, so the device address is fetched with
// cudaGetSymbolAddress once per device (with that device current) and cached
// for the life of the process (a cudaDeviceReset would invalidate it; the
// header tells callers not to use this entry point after one).
#include <mutex>

#include "kernels.cuh"

using namespace wedlm;

namespace {

constexpr int kChunks = 16;
constexpr size_t kPartBytes = (size_t)WEDLM_NOALLOC_MAX_ROWS * kChunks * sizeof(float4);
constexpr size_t kMaskBytes = (size_t)WEDLM_NOALLOC_MAX_ROWS;
constexpr size_t kErrBytes = 256;

// Scratch shared by every call on a device: the partials, the row flags, then
// the call's error word.
static __device__ __align__(256) unsigned char g_select_scratch[kPartBytes + kMaskBytes + kErrBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_addr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device (set up on first use).
wedlm_status scratch_address(unsigned char** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return WEDLM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return WEDLM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) return WEDLM_ERR_CUDA;
        g_addr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_addr[dev];
    return WEDLM_OK;
}

}  // namespace

extern "C" wedlm_status wedlm_entropy_select_noalloc(const float* logits, int32_t vocab, int32_t mask_id,
                                                     const uint8_t* filled, const int32_t* n, int32_t n_seq,
                                                     int32_t stride, const wedlm_step_params* params, float* htilde,
                                                     int32_t* argmax, uint8_t* fill, void* stream) {
    if (n_seq < 0 || stride < 1 || stride > kMaxWindow || vocab < 2 || mask_id < -1 || mask_id >= vocab || !params)
        return WEDLM_ERR_INVALID_ARG;
    if ((int64_t)n_seq * stride > WEDLM_NOALLOC_MAX_ROWS) return WEDLM_ERR_INVALID_ARG;
    if (!(params->logit_scale > 0.f)) return WEDLM_ERR_INVALID_ARG;
    if (n_seq == 0) return WEDLM_OK;
    if (!logits || !filled || !n || !htilde || !argmax || !fill) return WEDLM_ERR_INVALID_ARG;
    unsigned char* base = nullptr;
    wedlm_status s = scratch_address(&base);
    if (s) return s;
    float4* part = reinterpret_cast<float4*>(base);
    uint8_t* rowmask = base + kPartBytes;
    int* errw = reinterpret_cast<int*>(base + kPartBytes + kMaskBytes);
    cudaStream_t st = (cudaStream_t)stream;
    const int rows = n_seq * stride;
    StepKnobs kn{params->lambda, params->tau, params->logit_scale, params->tau_none};
    // Every row flag is rewritten below, every partial of a flagged row is
    // written before it is read and the error word is cleared first, so
    // nothing left by an earlier call is used.
    cudaMemsetAsync(errw, 0, sizeof(int), st);
    launch_rowmask_from_filled(filled, n, n_seq, stride, rowmask, st);
    launch_entropy_partials(logits, 1, 0, vocab, vocab, mask_id, params->logit_scale, rowmask, rows, kChunks, part, st);
    launch_select_only(part, kChunks, filled, n, n_seq, stride, kn, htilde, argmax, fill, errw, st);
    int herr = 0;
    cudaMemcpyAsync(&herr, errw, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (cudaGetLastError() != cudaSuccess) return WEDLM_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return WEDLM_ERR_CUDA;
    return herr == kErrNonFinite ? WEDLM_ERR_NONFINITE : herr ? WEDLM_ERR_DEVICE_ASSERT : WEDLM_OK;
}

// Shared device helpers of libwedlm (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/wedlm.h"

namespace wedlm {

using bf16 = __nv_bfloat16;

constexpr int kPage = WEDLM_PAGE_TOKENS;
constexpr int kMaxWindow = 64;

// Programmatic dependent launch.  A kernel launched with launch_pdl may begin
// while the previous kernel of its stream is still running: it must call
// griddep_wait() (which returns once that kernel has completed and its writes
// are visible) before touching memory that kernel reads or writes, and calls
// griddep_launch() after that wait (and after any TMEM allocation) to let the
// next kernel start early in turn.  Under a plain launch both are no-ops.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Global memory is never read through the non-coherent read-only path (no
// __ldg, no const __restrict__ kernel parameters): kernels started early by
// programmatic dependent launch read data that the kernel just before them
// wrote, and the read-only path is only guaranteed coherent for data that no
// one writes while the kernel runs.  Plain loads are compiled to bypass L1
// (-dlcm=cg, see build.py) and are served from L2; bulk data moves by TMA,
// also through L2.

// Device error word codes (mirrors of the wedlm_status values they map to).
constexpr int kErrBounds = 1;     // a bounds check refused an access
constexpr int kErrTimeout = 2;    // a bounded wait gave up
constexpr int kErrNonFinite = 3;  // a masked slot's logits held a NaN or an infinity

__device__ __forceinline__ void set_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024).  `scratch` holds 32 floats.
__device__ __forceinline__ float block_sum(float v, float* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float t = (lane < nw) ? scratch[lane] : 0.f;
    t = warp_sum(t);
    return t;
}

// Location of cache position p of a sequence in the paged KV pool.
// Pool layout: [layer][page][kv: 0=K,1=V][kv_head][16 tokens][head_dim].
struct KVLayout {
    int64_t layer_stride;   // elements per layer = num_pages * 2 * hkv * 16 * hd
    int hkv, hd, num_pages;
    __device__ __forceinline__ int64_t page_base(int layer, int page, int kv, int h) const {
        return (int64_t)layer * layer_stride + (((int64_t)page * 2 + kv) * hkv + h) * (int64_t)(kPage * hd);
    }
};

// Per-slot decode state living in device memory (structure of arrays).
struct SlotState {
    int32_t* S;        // [B] committed length (prompt + committed tokens)
    int32_t* end;      // [B] prompt_len + max_new_tokens
    int32_t* P;        // [B] prompt length
    int32_t* W;        // [B] window size (0 = slot unused)
    int32_t* wlen;     // [B] slots currently in the window
    int32_t* n;        // [B] rows of the current forward
    int32_t* k;        // [B] commit run of the current step
    int32_t* nf;       // [B] filled slots of the current step
    uint8_t* filled;   // [B][maxW]
    int32_t* token;    // [B][maxW]
    int32_t* page_table;   // [B][pages_per_seq]
    int32_t pages_per_seq;
    int32_t maxW;
    int64_t* counters; // [B][4]: steps, rows, committed, fills
    int32_t* gen;      // [B][gen_cap]: generated tokens in position order
    int32_t gen_cap;
    int32_t* out_count;     // [B]
    int32_t* out_tokens;    // [B][maxW]
    float* htilde;          // [B][maxW]
    int32_t* amax;          // [B][maxW]
    uint8_t* fillflag;      // [B][maxW]
};

// Per-row data of the current forward (row = entry * stride + r).
struct RowState {
    int32_t* pos;      // [Mmax] logical position
    int32_t* tok;      // [Mmax] token fed
    int32_t* perm;     // [Mmax] slot offset (decode) / r (prefill)
};

// Which rows of a forward belong to which slot: row = entry * stride + r,
// slot = slot_base + entry, row is live iff r < n[slot].
struct RowMap {
    int slot_base;
    int stride;
    const int32_t* n;
    __device__ __forceinline__ bool live(int row, int& slot, int& r) const {
        const int e = row / stride;
        r = row - e * stride;
        slot = slot_base + e;
        return r < n[slot];
    }
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// One non-blocking probe of an mbarrier phase (parity `parity` completed?).
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Waits at most ~limit_cycles (about one second at B200 clocks); gives up early
// once any CTA has recorded a timeout (a stall somewhere), so a launch that
// cannot finish drains quickly.  Bounds and non-finite errors are only
// recorded: the work that follows them completes normally.
__device__ __forceinline__ bool stalled(int* err) {
    return err && *reinterpret_cast<volatile int*>(err) == kErrTimeout;
}

// The same probe, but a thread whose phase is not complete is suspended until
// it completes or about `ns` nanoseconds have passed, instead of returning at
// once: waiting warps then take no issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity), "r"(ns) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int* err,
                                                  long long limit_cycles = 2000000000LL) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if ((it & 15u) == 0) {
            if (stalled(err)) return false;
            if (clock64() - t0 > limit_cycles) {
                set_error(err, kErrTimeout);
                return false;
            }
        }
    }
}

}  // namespace wedlm

// Stand-alone launches of single stages on caller-provided device buffers.
// They run exactly the kernels the decode step runs, so the tests can check
// each stage against the CPU oracle in isolation.
#include <string>

#include "gemm_tc.cuh"
#include "kernels.cuh"

using namespace wedlm;

namespace {

constexpr int kChunks = 16;

wedlm_status sync_status(cudaStream_t st) {
    if (cudaGetLastError() != cudaSuccess) return WEDLM_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return WEDLM_ERR_CUDA;
    return WEDLM_OK;
}

}  // namespace

extern "C" {

wedlm_status wedlm_reorder_window(const uint8_t* filled, const int32_t* n, const int32_t* S, int32_t n_seq,
                                  int32_t stride, int32_t* perm, int32_t* pos, int32_t* k, int32_t* nf,
                                  void* stream) {
    if (n_seq < 0 || stride < 1 || stride > kMaxWindow) return WEDLM_ERR_INVALID_ARG;
    if (n_seq == 0) return WEDLM_OK;
    if (!filled || !n || !S || !perm || !pos || !k || !nf) return WEDLM_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    launch_reorder_only(filled, n, S, n_seq, stride, perm, pos, k, nf, st);
    return sync_status(st);
}

wedlm_status wedlm_entropy_select(const float* logits, int32_t vocab, int32_t mask_id, const uint8_t* filled,
                                  const int32_t* n, int32_t n_seq, int32_t stride, const wedlm_step_params* params,
                                  float* htilde, int32_t* argmax, uint8_t* fill, void* stream) {
    if (n_seq < 0 || stride < 1 || stride > kMaxWindow || vocab < 2 || mask_id < -1 || mask_id >= vocab || !params)
        return WEDLM_ERR_INVALID_ARG;
    if (!(params->logit_scale > 0.f)) return WEDLM_ERR_INVALID_ARG;
    if (n_seq == 0) return WEDLM_OK;
    if (!logits || !filled || !n || !htilde || !argmax || !fill) return WEDLM_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const int rows = n_seq * stride;
    uint8_t* rowmask = nullptr;
    float4* part = nullptr;
    if (cudaMallocAsync((void**)&rowmask, rows, st) != cudaSuccess) return WEDLM_ERR_OOM_DEVICE;
    if (cudaMallocAsync((void**)&part, (size_t)rows * kChunks * sizeof(float4), st) != cudaSuccess) {
        cudaFreeAsync(rowmask, st);
        return WEDLM_ERR_OOM_DEVICE;
    }
    StepKnobs kn{params->lambda, params->tau, params->logit_scale, params->tau_none};
    launch_rowmask_from_filled(filled, n, n_seq, stride, rowmask, st);
    launch_entropy_partials(logits, 1, 0, vocab, vocab, mask_id, params->logit_scale, rowmask, rows, kChunks, part, st);
    launch_select_only(part, kChunks, filled, n, n_seq, stride, kn, htilde, argmax, fill, st);
    cudaFreeAsync(part, st);
    cudaFreeAsync(rowmask, st);
    return sync_status(st);
}

wedlm_status wedlm_linear_bf16(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t K, void* stream) {
    return wedlm_linear_bf16_plan(X, W, Y, M, N, K, 0, 0, stream);
}

static wedlm_status linear_bf16(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t K,
                                int32_t tile_n, int32_t k_splits, int32_t cg, int32_t hybrid, int32_t cluster_k,
                                void* stream) {
    if (M < 1 || N < 1 || K < 8 || K % 8 || !X || !W || !Y) return WEDLM_ERR_INVALID_ARG;
    if (tile_n != 0 && tile_n != 16 && tile_n != 32 && tile_n != 64 && tile_n != 128 && tile_n != 256)
        return WEDLM_ERR_INVALID_ARG;
    if (cg == 2 && tile_n != 128 && tile_n != 256) return WEDLM_ERR_INVALID_ARG;
    if (k_splits < 0 || k_splits > 16) return WEDLM_ERR_INVALID_ARG;
    if (((uintptr_t)X | (uintptr_t)W) & 15) return WEDLM_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cluster_k && (cg == 2 || hybrid || (tile_n != 128 && tile_n != 256) || k_splits < 2 || k_splits > 4 || N % 4))
        return WEDLM_ERR_INVALID_ARG;
    GemmPlan p = plan_gemm_bf16(M, N, K, sms, 16, tile_n, k_splits, 0, 0, -1, cg, hybrid, cluster_k);
    if (p.cg != (cg == 2 ? 2 : 1)) return WEDLM_ERR_INVALID_ARG;
    CUtensorMap tw, tx;
    if (!make_tmap_bf16(&tw, W, (uint64_t)N, (uint64_t)K, 128)) return WEDLM_ERR_CUDA;
    if (!make_tmap_bf16(&tx, X, (uint64_t)M, (uint64_t)K, (uint32_t)(p.bn / p.cg))) return WEDLM_ERR_CUDA;
    const size_t tiles = (size_t)p.m_tiles * p.n_tiles * p.cg;
    int* scratch = nullptr;  // error word, then tile tickets
    float* planes = nullptr;
    if (cudaMallocAsync((void**)&scratch, (1 + tiles) * sizeof(int), st) != cudaSuccess) return WEDLM_ERR_OOM_DEVICE;
    cudaMemsetAsync(scratch, 0, (1 + tiles) * sizeof(int), st);
    if (p.splits > 1 && cudaMallocAsync((void**)&planes, (size_t)p.splits * M * N * 4, st) != cudaSuccess) {
        cudaFreeAsync(scratch, st);
        return WEDLM_ERR_OOM_DEVICE;
    }
    EpiParams ep;
    ep.kind = EPI_STORE;
    ep.out = Y;
    ep.ws = planes;
    ep.counters = scratch + 1;
    ep.err = scratch;
    wedlm_status s = WEDLM_OK;
    if (launch_gemm_bf16(tw, tx, M, N, K, p, ep, st) != cudaSuccess) s = WEDLM_ERR_CUDA;
    int herr = 0;
    cudaMemcpyAsync(&herr, scratch, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (planes) cudaFreeAsync(planes, st);
    cudaFreeAsync(scratch, st);
    wedlm_status s2 = sync_status(st);
    if (s) return s;
    if (s2) return s2;
    if (herr == kErrTimeout) return WEDLM_ERR_TIMEOUT;
    if (herr) return WEDLM_ERR_DEVICE_ASSERT;
    return WEDLM_OK;
}

wedlm_status wedlm_linear_bf16_plan(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t K,
                                    int32_t tile_n, int32_t k_splits, void* stream) {
    return linear_bf16(X, W, Y, M, N, K, tile_n, k_splits, 1, 0, 0, stream);
}

wedlm_status wedlm_linear_bf16_sched(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t K,
                                     int32_t tile_n, int32_t k_splits, int32_t schedule, void* stream) {
    if (schedule & ~7) return WEDLM_ERR_INVALID_ARG;
    return linear_bf16(X, W, Y, M, N, K, tile_n, k_splits, (schedule & 1) ? 2 : 1, (schedule & 2) ? 1 : 0,
                       (schedule & 4) ? 1 : 0, stream);
}

}  // extern "C"

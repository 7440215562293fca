// Stand-alone launches of single stages on caller-provided device buffers.
// They run exactly the kernels the decode step runs, so the tests can check
// each stage against the CPU oracle in isolation.
#include <algorithm>
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

// Entropy selection on caller-provided scratch: `part` [rows][kChunks]
// partials, `rowmask` [rows] flags, `err` one device int (zeroed here).
static void enqueue_entropy_select(const float* logits, int32_t vocab, int32_t mask_id, const uint8_t* filled,
                                   const int32_t* n, int32_t n_seq, int32_t stride, const wedlm_step_params* params,
                                   float* htilde, int32_t* argmax, uint8_t* fill, float4* part, uint8_t* rowmask,
                                   int* err, cudaStream_t st) {
    const int rows = n_seq * stride;
    StepKnobs kn{params->lambda, params->tau, params->logit_scale, params->tau_none};
    cudaMemsetAsync(err, 0, sizeof(int), st);
    launch_rowmask_from_filled(filled, n, n_seq, stride, rowmask, st);
    launch_entropy_partials(logits, 1, 0, vocab, vocab, mask_id, params->logit_scale, rowmask, rows, kChunks, part, st);
    launch_select_only(part, kChunks, filled, n, n_seq, stride, kn, htilde, argmax, fill, err, st);
}

static bool entropy_args_ok(int32_t vocab, int32_t mask_id, int32_t n_seq, int32_t stride,
                            const wedlm_step_params* params) {
    return n_seq >= 0 && stride >= 1 && stride <= kMaxWindow && vocab >= 2 && mask_id >= -1 && mask_id < vocab &&
           params && params->logit_scale > 0.f;
}

static size_t entropy_ws_bytes(int32_t n_seq, int32_t stride) {
    const size_t rows = (size_t)n_seq * stride;
    return 256 + (rows * kChunks * sizeof(float4) + 255) / 256 * 256 + (rows + 255) / 256 * 256;
}

wedlm_status wedlm_entropy_select(const float* logits, int32_t vocab, int32_t mask_id, const uint8_t* filled,
                                  const int32_t* n, int32_t n_seq, int32_t stride, const wedlm_step_params* params,
                                  float* htilde, int32_t* argmax, uint8_t* fill, void* stream) {
    if (!entropy_args_ok(vocab, mask_id, n_seq, stride, params)) return WEDLM_ERR_INVALID_ARG;
    if (n_seq == 0) return WEDLM_OK;
    if (!logits || !filled || !n || !htilde || !argmax || !fill) return WEDLM_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t bytes = entropy_ws_bytes(n_seq, stride);
    char* ws = nullptr;
    if (cudaMallocAsync((void**)&ws, bytes, st) != cudaSuccess) return WEDLM_ERR_OOM_DEVICE;
    const size_t rows = (size_t)n_seq * stride;
    float4* part = reinterpret_cast<float4*>(ws + 256);
    uint8_t* rowmask = reinterpret_cast<uint8_t*>(ws + 256 + (rows * kChunks * sizeof(float4) + 255) / 256 * 256);
    enqueue_entropy_select(logits, vocab, mask_id, filled, n, n_seq, stride, params, htilde, argmax, fill, part,
                           rowmask, reinterpret_cast<int*>(ws), st);
    int herr = 0;
    cudaMemcpyAsync(&herr, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
    cudaFreeAsync(ws, st);
    wedlm_status s = sync_status(st);
    if (s) return s;
    return herr == kErrNonFinite ? WEDLM_ERR_NONFINITE : herr ? WEDLM_ERR_DEVICE_ASSERT : WEDLM_OK;
}

wedlm_status wedlm_entropy_select_workspace_bytes(int32_t n_seq, int32_t stride, int64_t* bytes) {
    if (!bytes || n_seq < 0 || stride < 1 || stride > kMaxWindow) return WEDLM_ERR_INVALID_ARG;
    *bytes = (int64_t)entropy_ws_bytes(n_seq, stride);
    return WEDLM_OK;
}

wedlm_status wedlm_entropy_select_async(const float* logits, int32_t vocab, int32_t mask_id, const uint8_t* filled,
                                        const int32_t* n, int32_t n_seq, int32_t stride,
                                        const wedlm_step_params* params, float* htilde, int32_t* argmax,
                                        uint8_t* fill, void* workspace, int64_t workspace_bytes, void* stream) {
    if (!entropy_args_ok(vocab, mask_id, n_seq, stride, params)) return WEDLM_ERR_INVALID_ARG;
    if (n_seq == 0) return WEDLM_OK;
    if (!logits || !filled || !n || !htilde || !argmax || !fill || !workspace) return WEDLM_ERR_INVALID_ARG;
    if (workspace_bytes < (int64_t)entropy_ws_bytes(n_seq, stride) || ((uintptr_t)workspace & 255))
        return WEDLM_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(workspace);
    const size_t rows = (size_t)n_seq * stride;
    enqueue_entropy_select(logits, vocab, mask_id, filled, n, n_seq, stride, params, htilde, argmax, fill,
                           reinterpret_cast<float4*>(ws + 256),
                           reinterpret_cast<uint8_t*>(ws + 256 + (rows * kChunks * sizeof(float4) + 255) / 256 * 256),
                           reinterpret_cast<int*>(ws), (cudaStream_t)stream);
    return cudaGetLastError() == cudaSuccess ? WEDLM_OK : WEDLM_ERR_CUDA;
}

// Workspace of the stand-alone attention: [0, 256) the device error word;
// then the (m, l) partials and the O partials of the key chunks, each piece
// 256-byte aligned.
struct AttnWs {
    int kv_chunk = 0, max_splits = 0;
    size_t off_ml = 0, off_o = 0, bytes = 0;
};

static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

static bool attn_ws_layout(int n_seq, int stride, int hq, int hkv, int max_ctx, AttnWs* w) {
    if (n_seq < 1 || stride < 1 || stride > kMaxWindow * 16 || hq < 1 || hkv < 1 || hq % hkv || hq / hkv > 128 ||
        max_ctx < 1)
        return false;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    w->kv_chunk = attn_kv_chunk_for(n_seq, stride, hq, hkv, max_ctx, sms);
    w->max_splits = (max_ctx + w->kv_chunk - 1) / w->kv_chunk;
    if (w->max_splits > attn_max_splits()) return false;
    const size_t rows = (size_t)n_seq * stride;
    w->off_ml = 256;
    const size_t parts = w->max_splits > 1 ? rows * hq * w->max_splits : 0;
    w->off_o = w->off_ml + round256(parts * sizeof(float2));
    w->bytes = w->off_o + round256(parts * 128 * sizeof(float));
    return true;
}

wedlm_status wedlm_attention_workspace_bytes(int32_t n_seq, int32_t stride, int32_t n_heads, int32_t n_kv_heads,
                                             int32_t max_ctx, int64_t* bytes) {
    AttnWs w;
    if (!bytes || !attn_ws_layout(n_seq, stride, n_heads, n_kv_heads, max_ctx, &w)) return WEDLM_ERR_INVALID_ARG;
    *bytes = (int64_t)w.bytes;
    return WEDLM_OK;
}

wedlm_status wedlm_attention_bf16(const void* q, const void* kv_pool, int32_t num_pages, int32_t n_heads,
                                  int32_t n_kv_heads, const int32_t* page_table, int32_t pages_per_seq,
                                  const int32_t* S, const int32_t* n, int32_t n_seq, int32_t stride, int32_t max_ctx,
                                  void* out, void* workspace, int64_t workspace_bytes, void* stream) {
    AttnWs w;
    if (!attn_ws_layout(n_seq, stride, n_heads, n_kv_heads, max_ctx, &w)) return WEDLM_ERR_INVALID_ARG;
    if (!q || !kv_pool || !page_table || !S || !n || !out || !workspace || num_pages < 1 || pages_per_seq < 1)
        return WEDLM_ERR_INVALID_ARG;
    if (workspace_bytes < (int64_t)w.bytes) return WEDLM_ERR_INVALID_ARG;
    if (((uintptr_t)q | (uintptr_t)kv_pool | (uintptr_t)out | (uintptr_t)workspace) & 255) return WEDLM_ERR_INVALID_ARG;
    const int hq = n_heads, hkv = n_kv_heads;
    KVLayout kvl;
    kvl.layer_stride = (int64_t)num_pages * 2 * hkv * kPage * 128;
    kvl.hkv = hkv;
    kvl.hd = 128;
    kvl.num_pages = num_pages;
    CUtensorMap tm_kv, tm_q, tm_qd;
    const int rows = n_seq * stride;
    if (!make_kv_tmap(&tm_kv, (const bf16*)kv_pool, kvl, 1) ||
        !make_q_tmap(&tm_q, (const bf16*)q, rows, hq, hkv, false) ||
        !make_q_tmap(&tm_qd, (const bf16*)q, rows, hq, hkv, true))
        return WEDLM_ERR_CUDA;
    SlotState ss{};
    ss.S = const_cast<int32_t*>(S);
    ss.n = const_cast<int32_t*>(n);
    ss.page_table = const_cast<int32_t*>(page_table);
    ss.pages_per_seq = pages_per_seq;
    RowMap rm{0, stride, n};
    char* ws = static_cast<char*>(workspace);
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e =
        launch_attn_bf16(tm_kv, tm_q, tm_qd, kvl, 0, hq, hkv, (bf16*)out, (float*)(ws + w.off_o),
                         (float2*)(ws + w.off_ml), n_seq, stride, w.kv_chunk,
                         w.max_splits, ss, rm, (int*)ws, st);
    return e == cudaSuccess ? WEDLM_OK : WEDLM_ERR_CUDA;
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

// Kernel launch interface of libwedlm (host-callable wrappers).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace wedlm {

struct StepKnobs {
    float lambda, tau, logit_scale;
    int tau_none;
    int blockwise;           // commit only whole windows (block-wise baseline)
    float temperature;       // > 0: Gumbel-max sampling of fill tokens
    unsigned long long seed;
};

// Window prepare for a decode step: refill, reorder, embed, first RMSNorm.
template <typename T>
void launch_decode_prepare(const T* embed, const float* norm_g, float eps, int d, int mask_id,
                           SlotState ss, RowState rs, uint8_t* rowmask, int n_entries, int stride,
                           float* x, T* h, int blockwise, cudaStream_t st);
// Prefill rows: tokens from `ids` (device), logical positions S0 + r.
template <typename T>
void launch_prefill_prepare(const T* embed, const float* norm_g, float eps, int d, const int32_t* ids,
                            int slot, int S0, int n, SlotState ss, RowState rs, float* x, T* h,
                            cudaStream_t st);
void launch_slot_admit(SlotState ss, int slot, int P, int end, int W, cudaStream_t st);
// Evict L2 before a timing run: a read-only sweep over `bytes` (> L2) of `buf`.
void launch_l2_evict(const void* buf, size_t bytes, float* sink, int num_sms, cudaStream_t st);
void launch_prefill_finish(SlotState ss, int slot, int P, cudaStream_t st);

// fp32 SIMT GEMM: C[M][N] = X[M][K] * W[N][K]^T.
void launch_gemm_f32(const float* X, const float* W, float* C, int M, int N, int K, cudaStream_t st);

template <typename T>
void launch_qkv_rope(const float* ws, int splits, int64_t split_stride, int M, int hq, int hkv, int hd,
                     T* q_out, T* kv_pool, KVLayout kvl, int layer, const float2* rope_cs, int rope_max_pos,
                     RowState rs, SlotState ss, RowMap rm, int* err, cudaStream_t st);

void launch_attn_f32(const float* q, const float* kv_pool, KVLayout kvl, int layer, int hq, int hkv, int hd,
                     float* out, int M, SlotState ss, RowMap rm, int* err, cudaStream_t st);

template <typename T>
void launch_residual_norm(const float* ws, int splits, int64_t split_stride, int M, int d, float* x, T* h,
                          const float* g, float eps, RowMap rm, cudaStream_t st);

// Packing of a decode step's masked rows for the LM head (row_map == nullptr:
// no packing).  Window e's masked rows are its physical rows nf..n-1; packed
// row i holds them in order over the windows, row_map[i] = the physical row,
// *count = the number of masked rows.
struct MaskedRows {
    const int32_t* nf = nullptr;  // [slots] filled rows of each window (ss.nf)
    int32_t* row_map = nullptr;   // [rows]
    int32_t* count = nullptr;     // [1]
    int n_entries = 0;
};

// bf16 mode: h = rmsnorm(x) * g (d % 4 == 0, d <= 8192); with mr.row_map the
// masked rows only, packed (see MaskedRows).
void launch_rmsnorm_bf16(const float* x, bf16* h, const float* g, float eps, int M, int d, RowMap rm,
                         cudaStream_t st, MaskedRows mr = MaskedRows());

template <typename T>
void launch_swiglu(const float* ws, int splits, int64_t split_stride, int M, int F, T* act, RowMap rm,
                   cudaStream_t st);

void launch_rope_table(float2* cs, int max_pos, int half, int hd, double theta, cudaStream_t st);

// Entropy / argmax partials over vocabulary chunks for rows with rowmask[row] != 0.
// Sampled fills: inv_t = 1 / temperature (0 = greedy, nothing sampled); row r
// belongs to slot r / stride, at logical position pos[r]; steps = the per-slot
// counters block (its first field counts the slot's decode steps); part gets
// one (best key, token) pair per (row, chunk).
struct SampleArgs {
    float inv_t = 0.f;
    unsigned long long seed = 0;
    int stride = 1;
    const int32_t* pos = nullptr;
    const int64_t* steps = nullptr;
    float2* part = nullptr;
};

void launch_entropy_partials(const float* logits, int splits, int64_t split_stride, int64_t ld, int V,
                             int mask_id, float scale, const uint8_t* rowmask, int rows, int chunks,
                             float4* part, cudaStream_t st, SampleArgs sa = SampleArgs());

// Fused LM-head entropy, second level: per-32-id partials [rows][npart] of the
// GEMM epilogue -> [rows][chunks] partials for the selection kernel.
void launch_entropy_merge(const float4* part, int npart, const uint8_t* rowmask, int rows, int chunks, float4* out,
                          cudaStream_t st);

// spart: the sampling partials (read only when knobs.temperature > 0).
void launch_select_commit(const float4* part, const float2* spart, int chunks, SlotState ss, RowState rs,
                          int n_entries, int stride, StepKnobs knobs, int* err, cudaStream_t st);

void launch_reorder_only(const uint8_t* filled, const int32_t* n, const int32_t* S, int n_seq, int stride,
                         int32_t* perm, int32_t* pos, int32_t* k, int32_t* nf, cudaStream_t st);

// Stand-alone selection; err (may be NULL) records kErrNonFinite when a masked
// row's logits held a NaN or an infinity (that slot: H~ NaN, argmax -1, no fill).
void launch_select_only(const float4* part, int chunks, const uint8_t* filled, const int32_t* n, int n_seq,
                        int stride, StepKnobs knobs, float* htilde, int32_t* argmax, uint8_t* fill, int* err,
                        cudaStream_t st);

void launch_rowmask_from_filled(const uint8_t* filled, const int32_t* n, int n_seq, int stride,
                                uint8_t* rowmask, cudaStream_t st);

// bf16 tensor-core paths (gemm_tc.cu, attn_tc.cu).
// Tensor map over the whole KV pool viewed as [rows][128] bf16, 16-row boxes
// of 64 dims with the 128-byte swizzle (one box = one page, one half).
bool make_kv_tmap(CUtensorMap* tm, const bf16* kv_pool, const KVLayout& kvl, int n_layers);
// Tensor map over q [rows][hq][128] with boxes of 64 dims x g heads x the
// attention's rows per tile (dual: the tile of windows with <= 64 query rows).
bool make_q_tmap(CUtensorMap* tm, const bf16* q, int rows, int hq, int hkv, bool dual);
// Decode/prefill attention (persistent: two CTAs per SM).  With more than one
// key chunk per row tile (kv_chunk < keys), chunk partials go to part_o
// [rows][hq][max_splits][128] / part_ml [rows][hq][max_splits] and a second
// kernel, launched behind the attention on the same stream, combines them
// into `out`; max_splits <= attn_max_splits(), and every sequence's S + n must
// fit in max_splits chunks (otherwise the bounds check fires).  kv_chunk is a
// multiple of 64.
cudaError_t launch_attn_bf16(const CUtensorMap& tm_kv, const CUtensorMap& tm_q, const CUtensorMap& tm_q_dual,
                             KVLayout kvl, int layer, int hq, int hkv, bf16* out, float* part_o, float2* part_ml,
                             int n_entries, int stride, int kv_chunk, int max_splits, SlotState ss, RowMap rm,
                             int* err, cudaStream_t st);
// Keys per chunk of the decode attention for a context's capacity (fixed per
// context, so a sequence's result does not depend on its batch neighbours).
int attn_kv_chunk_for(int max_batch, int max_window, int hq, int hkv, int max_ctx, int num_sms);
int attn_max_splits();
int attn_dual_rows_per_tile(int group);
int attn_rows_per_tile(int group);

}  // namespace wedlm

// bf16 dense projections on the 5th-generation tensor cores (tcgen05 + TMA),
// persistent, with the projection's epilogue fused in.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace wedlm {

// What the epilogue does with the fp32 accumulator Y[m][n]:
//   EPI_STORE     out[m][n] = Y                                  (LM head, test hook)
//   EPI_RESIDUAL  out[m][n] += Y, rows marked live only          (O and down projections)
//   EPI_SWIGLU    act[m][n/2] = silu(Y[m][n]) * Y[m][n+1], n even (gate/up rows interleaved)
//   EPI_QKV_ROPE  rotate q and k head dims (pairs interleaved in adjacent rows) at the
//                 row's logical position; q -> act[m][hq][128], k and v -> KV pages at
//                 cache index S + r of the row's sequence
//   EPI_ENTROPY   (LM head) logits are never stored: for every 32 vocab ids (one
//                 warp's TMEM lanes) and activation row m, the partial
//                 (max z, sum e^(z-max), sum e^(z-max)(z-max), lowest argmax) of
//                 z = scale * Y over ids != mask_id -> epart[m][npart]
enum EpiKind : int { EPI_STORE = 0, EPI_QKV_ROPE = 1, EPI_SWIGLU = 2, EPI_RESIDUAL = 3, EPI_ENTROPY = 4 };

struct EpiParams {
    int kind = EPI_STORE;
    float* out = nullptr;
    bf16* act = nullptr;
    bf16* kv_pool = nullptr;
    KVLayout kvl{};
    int layer = 0, hq = 0, hkv = 0;
    const float2* rope_cs = nullptr;
    int rope_max_pos = 0;
    RowState rs{};
    SlotState ss{};
    RowMap rm{};
    int check_rows = 0;        // 1: skip rows RowMap marks as padding
    float4* epart = nullptr;   // EPI_ENTROPY: partials [M][npart], npart = 4 per 128 weight rows
    int npart = 0;
    int mask_id = -1;
    float scale = 1.f;
    // Activation rows counted on the device (LM head over the packed masked
    // rows): rows >= *m_count are neither computed nor stored (the MMA width of
    // a tile shrinks to cover the live rows when the plan has no CTA pairs),
    // and an EPI_STORE / EPI_ENTROPY result of row m goes to row row_map[m].
    const int* m_count = nullptr;
    const int32_t* row_map = nullptr;
    float* ws = nullptr;       // split-K partial planes [splits][M][N]
    int* counters = nullptr;   // per-tile tickets; zero before and after every launch
    int* err = nullptr;
};

// How Y[M][N] = X[M][K] * W[N][K]^T is cut: tiles of 128 * wt weight rows
// (wt MMAs of M = 128 sharing the activation operand) by bn activation rows
// (MMA N), K in `splits` slices; units = tiles * splits are dealt round-robin
// to `grid` persistent CTAs (one per SM).  wt = 2 needs bn >= 128.  With
// cg = 2 a tile is 256 weight rows computed by a CTA pair (cta_group::2 MMAs,
// bn = 128 or 256 split between the two CTAs' shared memory), units are dealt
// to pairs, and `grid` counts CTAs (two per pair).
struct GemmPlan {
    int bn = 16;
    int wt = 1;
    int bk = 64;       // k-block depth: 64 (128-byte swizzle) or 32 (64-byte swizzle, bn >= 128)
    int coop = 1;      // K-split fixup: 1 the slices wait and share the reduction, 0 the last one reduces
    int cg = 1;        // 2: CTA pairs (clusters of two) share 256-row weight tiles; coop is then 0
    int hybrid = 0;    // 1: only the tiles of the last partial round are split (splits slices); coop is then 0
    int ks = 1;        // > 1: a tile's `splits` slices are the CTAs of one cluster, one unit per CTA, reduced
                       // through distributed shared memory (bn 128 or 256, wt 1, cg 1)
    int splits = 1;
    int kb_per_split = 1;
    int m_tiles = 1;
    int n_tiles = 1;
    int grid = 1;
};

// max_splits: the most K slices the caller's partial workspace holds (>= 1).
// force_bn / force_splits > 0 pin the tile width / split count, force_wt = 2
// selects 256-row weight tiles (tuning hooks).
// force_coop: 1 / 0 pick the K-split fixup, -1 the default (distributed for
// M > 128 rows, last arriver otherwise).  force_cg = 2 (with force_bn 128 or
// 256) selects CTA-pair tiles.
// force_hybrid = 1 (with force_splits > 1): the whole rounds of tiles run whole-K
// and only the last partial round is split.  force_cluster_k = 1 (with
// force_splits 2..4, force_bn 128 or 256): cluster K split.
GemmPlan plan_gemm_bf16(int M, int N, int K, int num_sms, int max_splits, int force_bn = 0, int force_splits = 0,
                        int force_wt = 0, int force_bk = 0, int force_coop = -1, int force_cg = 1,
                        int force_hybrid = 0, int force_cluster_k = 0);
GemmPlan plan_gemm_bf16_shape(int M, int N, int K, int num_sms, int max_splits, int force_bn, int force_splits,
                              int force_wt, int force_bk, int force_cg = 1, int force_hybrid = 0,
                              int force_cluster_k = 0);

// 2-D bf16 tensor map [rows][cols], boxes of bk columns (64: 128-byte swizzle,
// 32: 64-byte swizzle) by box_rows rows.
bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, int bk = 64);
// Any-rank bf16 tensor map with the 128-byte swizzle (box[0] * 2 bytes must be
// 128); gstride[i] is the byte stride of dimension i + 1.
bool encode_tmap_bf16(CUtensorMap* tm, const void* base, int rank, const cuuint64_t* gdim, const cuuint64_t* gstride,
                      const cuuint32_t* box);

// tmW: weights [N][K], box rows 128; tmX: activations [>=M][K], box rows
// plan.bn / plan.cg; both with boxes of plan.bk columns.
cudaError_t launch_gemm_bf16(const CUtensorMap& tmW, const CUtensorMap& tmX, int M, int N, int K,
                             const GemmPlan& plan, const EpiParams& ep, cudaStream_t st);

}  // namespace wedlm

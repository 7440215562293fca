// bf16 dense projections on the 5th-generation tensor cores (tcgen05 + TMA).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace wedlm {

// How one Y[M][N] = X[M][K] * W[N][K]^T is cut into CTAs: 128 weight rows per
// tile (the MMA's M), bn activation rows per tile (the MMA's N), and `splits`
// slices of K, each writing its own fp32 partial plane out[split][M][N].
struct GemmPlan {
    int bn = 16;
    int splits = 1;
    int kb_per_split = 1;
    int m_tiles = 1;
    int n_tiles = 1;
};

GemmPlan plan_gemm_bf16(int M, int N, int K, int num_sms);

// 2-D bf16 tensor map over a row-major [rows][cols] matrix with a 64-column,
// box_rows-row box and 128-byte swizzle.  Returns false if the driver refuses.
bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// tmW: weights [N][K] with box_rows 128; tmX: activations [>=M][K] with
// box_rows = plan.bn.  out: fp32 [plan.splits][M][N].
cudaError_t launch_gemm_bf16(const CUtensorMap& tmW, const CUtensorMap& tmX, float* out, int M, int N, int K,
                             const GemmPlan& plan, int* err, cudaStream_t st);

}  // namespace wedlm

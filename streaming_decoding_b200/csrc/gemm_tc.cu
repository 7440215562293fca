// bf16 GEMM on tcgen05 tensor cores with TMA-fed shared-memory stages.
//
// Y[M][N] = X[M][K] * W[N][K]^T for the dense projections (QKV, O, gate/up,
// down) and the LM head.  In decoding, M (window rows of the batch) is small
// (16..256) and N, K are the model's widths, so the kernel is laid out
// "swap-AB": the 128-row MMA M side is taken by the weights and the MMA N
// side by the activation rows.  Each CTA streams its weight tiles exactly once
// from HBM; the step is bound by weight bytes until M approaches the
// machine-balance point (about 250 rows), where it becomes tensor bound.
//
// Warp roles (192 threads):
//   warp 0      one elected thread issues TMA loads of A (weights, 128 x 64)
//               and B (activations, bn x 64) into a STAGES-deep ring,
//   warp 1      allocates TMEM and one elected thread issues tcgen05.mma
//               (kind::f16, bf16 inputs, fp32 accumulate in TMEM), releasing
//               each stage back to the producer with tcgen05.commit,
//   warps 2..5  epilogue: tcgen05.ld the 128 x bn fp32 accumulator (warp w
//               owns TMEM lanes 32*(w%4) .. +31) and store it row-major.
// Every mbarrier wait is bounded; on timeout the kernel records an error and
// unwinds (frees TMEM) instead of hanging.
#include <cmath>

#include <cudaTypedefs.h>

#include "gemm_tc.cuh"

namespace wedlm {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_STAGE_BYTES = BM * BK * 2;

template <int BN> struct TileCfg {
    static constexpr int B_STAGE_BYTES = BN * BK * 2;
    static constexpr int STAGES = BN <= 32 ? 5 : (BN <= 64 ? 4 : (BN <= 128 ? 6 : 4));
    static constexpr int TMEM_COLS = BN <= 32 ? 32 : BN;
    static constexpr int SMEM_BYTES = STAGES * (A_STAGE_BYTES + B_STAGE_BYTES) + 1024 /*align*/ + 256 /*barriers*/;
};

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major tile stored with the 128-byte
// swizzle (rows of 64 bf16 = 128 B; 8-row swizzle atoms 1024 B apart).
__device__ __forceinline__ uint64_t sdesc_k_sw128(const void* p) {
    const uint32_t a = smem_u32(p);
    uint64_t d = (uint64_t)((a >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;               // leading-dimension byte offset (unused with swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;     // stride byte offset between 8-row atoms
    d |= (uint64_t)1 << 46;               // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;               // 128-byte swizzle
    return d;
}

// Instruction descriptor: dense kind::f16, D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int BN>
__global__ void __launch_bounds__(192, 1) gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmW,
                                                              const __grid_constant__ CUtensorMap tmX,
                                                              float* __restrict__ out, int M, int N, int K,
                                                              int kb_per_split, int* err) {
    using C = TileCfg<BN>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::B_STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* accum = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BM, m0 = blockIdx.y * BN, split = blockIdx.z;
    const int KB = (K + BK - 1) / BK;
    const int kb0 = split * kb_per_split;
    const int nkb = min(KB, kb0 + kb_per_split) - kb0;

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (nkb > 0) {
        if (warp == 0) {
            if (lane == 0) {
                for (int i = 0; i < nkb; ++i) {
                    const int s = i % STAGES;
                    const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&empty[s]), ph ^ 1u, err)) break;
                    mbar_expect_tx(&full[s], A_STAGE_BYTES + C::B_STAGE_BYTES);
                    const int kx = (kb0 + i) * BK;
                    tma_load_2d(sA + s * A_STAGE_BYTES, &tmW, kx, n0, &full[s]);
                    tma_load_2d(sB + s * C::B_STAGE_BYTES, &tmX, kx, m0, &full[s]);
                }
            }
        } else if (warp == 1) {
            if (lane == 0) {
                constexpr uint32_t idesc = idesc_bf16(BM, BN);
                for (int i = 0; i < nkb; ++i) {
                    const int s = i % STAGES;
                    const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&full[s]), ph, err)) break;
                    tc_fence_after();
                    const uint8_t* a = sA + s * A_STAGE_BYTES;
                    const uint8_t* b = sB + s * C::B_STAGE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_bf16(tmem, sdesc_k_sw128(a + kk * 32), sdesc_k_sw128(b + kk * 32), idesc,
                                  (i > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                umma_commit(accum);
            }
        } else {
            const int q = warp & 3;
            const int n = n0 + q * 32 + lane;
            float* o = out + (int64_t)split * M * N;
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(accum), 0u, err));
            if (ok) {
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, v);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + c + j;
                        if (m < M && n < N) o[(int64_t)m * N + n] = __uint_as_float(v[j]);
                    }
                }
            }
        }
    } else if (warp >= 2) {
        const int n = n0 + (warp & 3) * 32 + lane;
        float* o = out + (int64_t)split * M * N;
        for (int j = 0; j < BN; ++j) {
            const int m = m0 + j;
            if (m < M && n < N) o[(int64_t)m * N + n] = 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& tmW, const CUtensorMap& tmX, float* out, int M, int N, int K,
                      const GemmPlan& p, int* err, cudaStream_t st) {
    using C = TileCfg<BN>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(p.n_tiles, p.m_tiles, p.splits);
    gemm_bf16_tc_kernel<BN><<<grid, 192, C::SMEM_BYTES, st>>>(tmW, tmX, out, M, N, K, p.kb_per_split, err);
    return cudaGetLastError();
}

}  // namespace

GemmPlan plan_gemm_bf16(int M, int N, int K, int num_sms) {
    GemmPlan p;
    p.bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    p.m_tiles = (M + p.bn - 1) / p.bn;
    p.n_tiles = (N + BM - 1) / BM;
    const int KB = (K + BK - 1) / BK;
    const int occ = p.bn <= 64 ? 2 : 1;
    const double slots = (double)num_sms * occ;
    const double tiles = (double)p.m_tiles * p.n_tiles;
    const double wbytes = 2.0 * N * K;
    double best = -1.0;
    for (int s = 1; s <= KB && s <= 32; ++s) {
        const int kbps = (KB + s - 1) / s;
        const int sp = (KB + kbps - 1) / kbps;
        if (sp != s) continue;
        const double ctas = tiles * sp;
        const double waves = std::ceil(ctas / slots);
        const double eff = ctas / (waves * slots);
        const double partial = sp > 1 ? (2.0 * sp * 4.0 * M * N) / wbytes : 0.0;
        const double score = eff / (1.0 + 0.5 * partial);
        if (score > best + 0.02) {
            best = score;
            p.splits = sp;
            p.kb_per_split = kbps;
        }
    }
    return p;
}

bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm_bf16(const CUtensorMap& tmW, const CUtensorMap& tmX, float* out, int M, int N, int K,
                             const GemmPlan& p, int* err, cudaStream_t st) {
    switch (p.bn) {
        case 16: return launch_bn<16>(tmW, tmX, out, M, N, K, p, err, st);
        case 32: return launch_bn<32>(tmW, tmX, out, M, N, K, p, err, st);
        case 64: return launch_bn<64>(tmW, tmX, out, M, N, K, p, err, st);
        case 128: return launch_bn<128>(tmW, tmX, out, M, N, K, p, err, st);
        case 256: return launch_bn<256>(tmW, tmX, out, M, N, K, p, err, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace wedlm

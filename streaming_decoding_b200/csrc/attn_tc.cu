// Reordered-causal GQA attention of window rows against the paged KV cache on
// the 5th-generation tensor cores (tcgen05, accumulators in TMEM, K/V pages
// brought in by TMA).
//
// [Method] (hyper.ai summary of arXiv 2512.22737, section "Method"): after
// Topological Reordering the window goes through a plain causal forward
// conditioned on the persistent KV cache; physical row r of a sequence with
// committed length S attends to cache positions 0..S-1 and to window rows
// 0..r, whose K/V the QKV epilogue of this same forward wrote at S..S+r.
//
// One CTA owns (batch entry, KV head, tile of RT window rows, key chunk).  Its
// 128 query rows (RT rows x g query heads sharing the KV head; unused rows are
// zero) are the M side of every MMA, so each K/V byte loaded serves all g heads:
//   S  = Q K^T   M=128, N=64 keys, K=128 dims  (A = Q, B = K: shared memory)
//   O += P V     M=128, N=128 dims, K=64 keys  (A = P in TMEM, B = V)
// A 16-token page is one TMA box per 64-dim half, so K and V blocks land as
// key rows of 128 bytes with the 128-byte swizzle: the K-major operand form
// for K and the MN-major (dims contiguous) form for V.
//
// TMEM: two S buffers of 64 columns (P overwrites the first 32 columns of its
// own S buffer as packed bf16) and O in 128 columns.  With two S buffers the
// MMA of S for block j+1 runs while the softmax works on block j.
// Warp roles (192 threads):
//   warps 0-3  softmax: thread i owns query row i (TMEM lane i); applies the
//              causal and chunk masks, keeps a running max m and sum l (exp2
//              domain); O is rescaled in TMEM only when a row's max grows by
//              more than 2^8 (otherwise P stays relative to the older max,
//              exactly); at the end normalises O and stores the row, or (when
//              the keys were split) stores the unnormalised partial, and the
//              last CTA of the tile merges the partials of all chunks,
//   warp 4     allocates 256 TMEM columns; one thread issues the MMAs,
//   warp 5     TMA loads: Q (two 3-D boxes of 64 dims x g heads x rows), then
//              K and V into two 2-stage rings (K released once S has been
//              computed, V once P V has); the chunk's page ids are read 128 at
//              a time into the warp's registers.
// All waits are bounded; a timeout sets the device error word.
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace wedlm {
namespace {

constexpr int HD = 128;
constexpr int KBLK = 64;
constexpr int QROWS = 128;
constexpr int NST = 2;                              // stages per ring (K and V)
constexpr int Q_BYTES = QROWS * HD * 2;             // two 64-dim halves of 16 KB
constexpr int HALF_BYTES = KBLK * 128;              // 64 keys x 64 dims
constexpr int BLK_BYTES = 2 * HALF_BYTES;           // one K or V block: 16 KB
constexpr int BOX_BYTES = kPage * 128;              // one page, one half: 2 KB
constexpr int NTHREADS = 192;
constexpr uint32_t TM_S = 0, TM_O = 128, TM_COLS = 256;  // S buffer b at TM_S + 64 b
constexpr int MAX_SPLITS = 32;  // key chunks per row tile (merge weights in smem)
constexpr int kMR = 8, kMS = 2;  // merge: rows x chunk partials in flight per lane
constexpr int SMEM_BYTES = Q_BYTES + 2 * NST * BLK_BYTES + 256 + 1024 /*block maxima*/ + 1024 /*align*/;

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// One box of the pool's tensor map (x = dim offset, y = pool row) into shared memory.
__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major tile with the 128-byte swizzle (128-byte rows, 8-row atoms 1024 B apart).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr) {
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// MN-major tile with the 128-byte swizzle: 128-byte rows along K (one key
// each, 64 dims), 8-row atoms 1024 B apart (SBO), the next 64 dims 8 KB on (LBO).
__device__ __forceinline__ uint64_t sdesc_mn(uint32_t addr) {
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)(HALF_BYTES >> 4) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Barrier among the 128 softmax threads only (named barrier 1).
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// A 3-D box of q: 64 dims x g heads x rt rows (one 64-dim half of a tile).
__device__ __forceinline__ void tma_box3(uint32_t dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

struct AttnParams {
    KVLayout kvl;
    int layer, hq, hkv;
    bf16* out;
    float* part_o;
    float2* part_ml;
    int* tickets;  // [entries][hkv][tiles], zero between launches
    int stride, kv_chunk, max_splits, rt, tiles;
    SlotState ss;
    RowMap rm;
    int* err;
};

// DUAL (valid query rows <= 64): rows 64..127 repeat rows 0..63, and the
// thread of row i + 64 takes keys 32..63 of every block while the thread of
// row i takes keys 0..31, each writing zeros into the other half of its P
// row; the two share the running max through shared memory, so O rows i and
// i + 64 hold the two halves of one result (summed at the end).  This halves
// the per-thread softmax work when a tile has 64 or fewer query rows.
template <bool DUAL>
__global__ void __launch_bounds__(NTHREADS, 2) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                                                              const __grid_constant__ CUtensorMap tm_q,
                                                              const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = smem + Q_BYTES;             // [NST] K blocks
    uint8_t* sV = sK + NST * BLK_BYTES;       // [NST] V blocks
    float* sX = reinterpret_cast<float*>(sK); // after the last block: exchange / merge scratch (64 KB)
    uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NST * BLK_BYTES);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;    // [NST]
    uint64_t* k_empty = bars + 3;   // [NST]
    uint64_t* v_full = bars + 5;    // [NST]
    uint64_t* v_empty = bars + 7;   // [NST]
    uint64_t* s_full = bars + 9;    // [2] per S buffer
    uint64_t* p_full = bars + 11;   // [2] per S buffer
    uint64_t* o_done = bars + 13;   // one completion per P V
    uint64_t* o_final = bars + 14;  // the last P V
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
    int* last_flag = reinterpret_cast<int*>(bars + 16);
    float* xmax = reinterpret_cast<float*>(bars + 32);  // [2][128] block maxima (DUAL)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int entry = blockIdx.z / p.max_splits, sp = blockIdx.z % p.max_splits;
    const int kvh = blockIdx.y;
    const int slot = p.rm.slot_base + entry;
    const int n = p.rm.n[slot];
    const int r0 = blockIdx.x * p.rt;
    if (r0 >= n) return;
    const int S = p.ss.S[slot];
    const int r_last = min(r0 + p.rt, n) - 1;
    const int kend = S + r_last + 1;
    const int nsplit = (kend + p.kv_chunk - 1) / p.kv_chunk;
    if (sp >= nsplit) return;
    const int ks = sp * p.kv_chunk;
    const int ke = min(kend, ks + p.kv_chunk);
    const int nblk = (ke - ks + KBLK - 1) / KBLK;
    const int g = p.hq / p.hkv;
    const int qrows = p.rt * g;  // query rows of the tile (<= 64 when DUAL)

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_kv)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
        mbar_init(q_full, 1);
        for (int s = 0; s < NST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 4);
        }
        mbar_init(o_done, 1);
        mbar_init(o_final, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 4) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int* err = p.err;
    // q and this layer's window K/V come from the QKV projection just before
    if (warp != 5) {
        griddep_wait();
        griddep_launch();
    }

    if (warp == 5) {
        // ---------------------------------------------------------- loader
        // Page ids of the chunk, 128 at a time, four per lane.  Keys past the
        // chunk end (and, after an error, unmapped pages) read a mapped page
        // instead: their scores are masked, and pool memory is zeroed at
        // creation and only ever holds finite K/V, so P = 0 times V stays 0.
        const int32_t* pt = p.ss.page_table + (int64_t)slot * p.ss.pages_per_seq;
        const int64_t row_k = p.kvl.page_base(p.layer, 0, 0, kvh) / HD;   // pool row of (page 0, K, kvh, token 0)
        const int64_t row_v = p.kvl.page_base(p.layer, 0, 1, kvh) / HD;
        const int64_t page_rows = (int64_t)2 * p.kvl.hkv * kPage;         // pool rows per page step
        const int page_first = ks / kPage, page_end = (ke + kPage - 1) / kPage;
        int batch = -1;
        int preg[4];
        auto load_batch = [&](int b) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pi = page_first + b * 128 + i * 32 + lane;
                int pg = -1;
                if (pi < page_end) {
                    pg = pi < p.ss.pages_per_seq ? __ldg(pt + pi) : -1;
                    if (pg < 0 || pg >= p.kvl.num_pages) {
                        set_error(err, kErrBounds);
                        pg = -1;
                    }
                }
                preg[i] = pg;
            }
            batch = b;
        };
        load_batch(0);
        griddep_wait();
        griddep_launch();
        if (lane == 0) {
            mbar_expect_tx(q_full, (DUAL ? 4 : 2) * 128 * qrows);
            const int z = entry * p.stride + r0, y = kvh * g;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tma_box3(smem_u32(sQ) + h * (QROWS * 128), &tm_q, h * 64, y, z, q_full);
                if (DUAL) tma_box3(smem_u32(sQ) + h * (QROWS * 128) + 64 * 128, &tm_q, h * 64, y, z, q_full);
            }
        }
        int fallback = __shfl_sync(0xffffffffu, preg[0], 0);
        if (fallback < 0) fallback = 0;
        bool ok = true;
        int k_issued = 0, v_issued = 0;
        for (int j = 0; j < nblk && ok; ++j) {
            const int st = j % NST;
            // this block's four pages: local index li = 4j + lane (lanes 0..3)
            const int li = j * 4 + (lane & 3);
            if ((li >> 7) != batch) load_batch(li >> 7);
            const int w = li & 127;
            const int c0 = __shfl_sync(0xffffffffu, preg[0], w & 31), c1 = __shfl_sync(0xffffffffu, preg[1], w & 31);
            const int c2 = __shfl_sync(0xffffffffu, preg[2], w & 31), c3 = __shfl_sync(0xffffffffu, preg[3], w & 31);
            int pg = (w >> 5) == 0 ? c0 : (w >> 5) == 1 ? c1 : (w >> 5) == 2 ? c2 : c3;
            if (pg < 0) pg = fallback;
            // K ring
            if (lane == 0) ok = mbar_wait_bounded(smem_u32(&k_empty[st]), ((j / NST) & 1) ^ 1, err);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) mbar_expect_tx(&k_full[st], BLK_BYTES);
            __syncwarp();
            if (lane < 4) {
                const int y = (int)(row_k + (int64_t)pg * page_rows);
                const uint32_t dst = smem_u32(sK + st * BLK_BYTES) + lane * BOX_BYTES;
                tma_box(dst, &tm_kv, 0, y, &k_full[st]);
                tma_box(dst + HALF_BYTES, &tm_kv, 64, y, &k_full[st]);
            }
            k_issued = j + 1;
            // V ring
            if (lane == 0) ok = mbar_wait_bounded(smem_u32(&v_empty[st]), ((j / NST) & 1) ^ 1, err);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) mbar_expect_tx(&v_full[st], BLK_BYTES);
            __syncwarp();
            if (lane < 4) {
                const int y = (int)(row_v + (int64_t)pg * page_rows);
                const uint32_t dst = smem_u32(sV + st * BLK_BYTES) + lane * BOX_BYTES;
                tma_box(dst, &tm_kv, 0, y, &v_full[st]);
                tma_box(dst + HALF_BYTES, &tm_kv, 64, y, &v_full[st]);
            }
            v_issued = j + 1;
        }
        // Copies still in flight (only after an error) must land before the CTA
        // exits: wait, bounded, for Q and the last blocks issued to each stage.
        if (lane == 0) {
            mbar_wait_bounded(smem_u32(q_full), 0, nullptr, 200000000LL);
            for (int j = max(0, k_issued - NST); j < k_issued; ++j)
                mbar_wait_bounded(smem_u32(&k_full[j % NST]), (j / NST) & 1, nullptr, 200000000LL);
            for (int j = max(0, v_issued - NST); j < v_issued; ++j)
                mbar_wait_bounded(smem_u32(&v_full[j % NST]), (j / NST) & 1, nullptr, 200000000LL);
        }
    } else if (warp == 4) {
        // -------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, KBLK);
            constexpr uint32_t idO = idesc_bf16(128, HD) | (1u << 16);  // B (V) MN-major
            const uint32_t qa = smem_u32(sQ);
            auto issue_s = [&](int j) -> bool {
                const int st = j % NST, b = j & 1;
                if (!mbar_wait_bounded(smem_u32(&k_full[st]), (j / NST) & 1, err)) return false;
                tc_fence_after();
                const uint32_t kb = smem_u32(sK + st * BLK_BYTES);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    mma_ss(tmem + TM_S + b * 64, sdesc(qa + (kk >> 2) * (QROWS * 128) + (kk & 3) * 32),
                           sdesc(kb + (kk >> 2) * HALF_BYTES + (kk & 3) * 32), idS, kk > 0 ? 1u : 0u);
                umma_commit(&k_empty[st]);
                umma_commit(&s_full[b]);
                return true;
            };
            bool ok = mbar_wait_bounded(smem_u32(q_full), 0, err);
            for (int j = 0; j < nblk && j < 2 && ok; ++j) ok = issue_s(j);
            for (int j = 0; j < nblk && ok; ++j) {
                const int st = j % NST, b = j & 1;
                if (!(ok = mbar_wait_bounded(smem_u32(&p_full[b]), (j >> 1) & 1, err))) break;
                if (!(ok = mbar_wait_bounded(smem_u32(&v_full[st]), (j / NST) & 1, err))) break;
                tc_fence_after();
                const uint32_t vb = smem_u32(sV + st * BLK_BYTES);
#pragma unroll
                for (int kk = 0; kk < KBLK / 16; ++kk)
                    mma_ts(tmem + TM_O, tmem + TM_S + b * 64 + kk * 8, sdesc_mn(vb + kk * 2048), idO,
                           (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&v_empty[st]);
                umma_commit(o_done);
                if (j + 2 < nblk) {
                    // S buffer b is read by this P V: wait for it before S(j+2) overwrites it
                    if (!(ok = mbar_wait_bounded(smem_u32(o_done), j & 1, err))) break;
                    ok = issue_s(j + 2);
                }
            }
            if (ok) umma_commit(o_final);
        }
    } else {
        // ---------------------------------------------------------- softmax
        const int tid = threadIdx.x;                // TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int qi = DUAL ? (tid & 63) : tid;     // query row this thread works for
        const int half = DUAL ? (tid >> 6) : 0;     // DUAL: key half of every block
        const int rr = r0 + qi / g;
        const bool qok = qi < qrows && rr < n;
        const int lim = S + (qok ? rr : r_last);    // last visible key
        const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
        constexpr int NC = DUAL ? 32 : 64;          // score columns per thread and block
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nblk && ok; ++j) {
            const int b = j & 1;
            const int kb0 = ks + j * KBLK + half * 32;
            const uint32_t tS = tmem + lane_base + TM_S + b * 64;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&s_full[b]), (j >> 1) & 1, err));
            if (!ok) break;
            tc_fence_after();
            uint32_t r[32];
            float s[NC];
            if constexpr (DUAL) {
                tmem_ld32(tS + half * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(r[c]);
            } else {
                uint32_t r2[32];
                tmem_ld32(tS, r);
                tmem_ld32(tS + 32, r2);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    s[c] = __uint_as_float(r[c]);
                    s[(32 + c) % NC] = __uint_as_float(r2[c]);
                }
            }
            float bmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int t = kb0 + c;
                s[c] = (t < ke && t <= lim) ? s[c] * sl2 : -INFINITY;
                bmax = fmaxf(bmax, s[c]);
            }
            if (DUAL) {
                float* xb = xmax + b * 128;
                xb[tid] = bmax;
                softmax_sync();
                bmax = fmaxf(bmax, xb[tid ^ 64]);
            }
            const bool need = bmax > m_ref + 8.0f;
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                // P V of the previous block must be done before O is rescaled
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(o_done), (j - 1) & 1, err));
                if (!ok) break;
                tc_fence_after();
                const float f = need ? exp2f(m_ref - bmax) : 1.0f;
#pragma unroll 1
                for (int c = 0; c < HD; c += 32) {
                    tmem_ld32(tmem + lane_base + TM_O + c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * f);
                    tmem_st32(tmem + lane_base + TM_O + c, r);
                }
                l *= f;
            }
            if (need) m_ref = bmax;
            const float ref = (m_ref == -INFINITY) ? 0.f : m_ref;
            float psum = 0.f;
            if constexpr (DUAL) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float a = exp2f(s[2 * c] - ref), bb = exp2f(s[2 * c + 1] - ref);
                    psum += a + bb;
                    pk[c] = pack_bf16(a, bb);
                }
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    r[c] = half ? 0u : pk[c];
                    r[16 + c] = half ? pk[c] : 0u;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float a = exp2f(s[(2 * c) % NC] - ref), bb = exp2f(s[(2 * c + 1) % NC] - ref);
                    psum += a + bb;
                    r[c] = pack_bf16(a, bb);
                }
            }
            l += psum;
            tmem_st32(tS, r);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[b]);
        }
        // (o_done may be one or two completions behind here, so the last P V
        // signals a barrier of its own)
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(o_final), 0, err));
        const int qrow = entry * p.stride + (qok ? rr : r_last);
        const int qhead = kvh * g + qi % g;
        const int64_t pbase = ((int64_t)qrow * p.hq + qhead) * p.max_splits;
        // The ring buffers are idle now (every block was consumed): reuse them.
        softmax_sync();
        if (ok) {
            tc_fence_after();
            if (DUAL && half) {
                // hand this half's O row and sum to the row's owner (thread qi)
#pragma unroll 1
                for (int c = 0; c < HD; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + TM_O + c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) sX[(c + x) * 64 + qi] = __uint_as_float(r[x]);
                }
                sX[HD * 64 + qi] = l;
            }
        }
        if (DUAL) softmax_sync();
        if (ok && !(DUAL && half)) {
            if (DUAL) l += sX[HD * 64 + qi];
            const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll 1
            for (int c = 0; c < HD; c += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_base + TM_O + c, r);
                tmem_wait_ld();
                if (DUAL) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) + sX[(c + x) * 64 + qi]);
                }
                if (!qok) continue;
                if (nsplit == 1) {
                    __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(p.out + ((int64_t)qrow * p.hq + qhead) * HD + c);
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        op[x] = __floats2bfloat162_rn(__uint_as_float(r[2 * x]) * inv, __uint_as_float(r[2 * x + 1]) * inv);
                } else {
                    float4* po = reinterpret_cast<float4*>(p.part_o + (pbase + sp) * HD + c);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        po[x] = make_float4(__uint_as_float(r[4 * x]), __uint_as_float(r[4 * x + 1]),
                                            __uint_as_float(r[4 * x + 2]), __uint_as_float(r[4 * x + 3]));
                }
            }
            if (qok && nsplit > 1) p.part_ml[pbase + sp] = make_float2(m_ref, l);
        }
        if (nsplit > 1) {
            // The last chunk of this (entry, KV head, tile) to finish merges all
            // chunks' partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
            __threadfence();
            softmax_sync();
            if (tid == 0) {
                int* ticket = p.tickets + ((int64_t)entry * p.hkv + kvh) * p.tiles + blockIdx.x;
                const int prev = atomicAdd(ticket, 1);
                const int last = prev == nsplit - 1;
                if (last) *ticket = 0;
                *last_flag = last;
            }
            softmax_sync();
            if (*last_flag) {
                __threadfence();
                // weights w_s / L per (row, chunk) into shared memory (all of a
                // row's (m, l) loads in flight at once)
                float* wsm = sX;  // [128 rows][MAX_SPLITS]
                if (tid < qrows && r0 + tid / g < n) {
                    const int64_t pb = ((int64_t)(entry * p.stride + r0 + tid / g) * p.hq + kvh * g + tid % g) *
                                       p.max_splits;
                    float2 ml[MAX_SPLITS];
#pragma unroll
                    for (int s2 = 0; s2 < MAX_SPLITS; ++s2)
                        ml[s2] = s2 < nsplit ? __ldcg(&p.part_ml[pb + s2]) : make_float2(-INFINITY, 0.f);
                    float M = -INFINITY;
#pragma unroll
                    for (int s2 = 0; s2 < MAX_SPLITS; ++s2) M = fmaxf(M, ml[s2].x);
                    float L = 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < MAX_SPLITS; ++s2) {
                        ml[s2].x = (ml[s2].x == -INFINITY) ? 0.f : exp2f(ml[s2].x - M);
                        L += ml[s2].x * ml[s2].y;
                    }
                    const float inv = L > 0.f ? 1.0f / L : 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < MAX_SPLITS; ++s2) wsm[tid * MAX_SPLITS + s2] = ml[s2].x * inv;
                }
                softmax_sync();
                // then the rows: a warp takes one row at a time, a lane 4 dims
                // (coalesced 512-byte reads per chunk partial)
#pragma unroll 1
                for (int row0 = warp; row0 < qrows; row0 += 4 * kMR) {
                    float4 acc[kMR];
                    int64_t pbr[kMR];
                    bool okr[kMR];
#pragma unroll
                    for (int u = 0; u < kMR; ++u) {
                        const int row = row0 + 4 * u;
                        okr[u] = row < qrows && r0 + row / g < n;
                        pbr[u] = ((int64_t)(entry * p.stride + r0 + row / g) * p.hq + kvh * g + row % g) *
                                 p.max_splits;
                        acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll 1
                    for (int s0 = 0; s0 < nsplit; s0 += kMS) {
                        float4 v[kMR][kMS];
#pragma unroll
                        for (int u = 0; u < kMR; ++u)
#pragma unroll
                            for (int q = 0; q < kMS; ++q)
                                v[u][q] = (okr[u] && s0 + q < nsplit)
                                              ? __ldcg(reinterpret_cast<const float4*>(p.part_o + (pbr[u] + s0 + q) * HD) + lane)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (int u = 0; u < kMR; ++u)
#pragma unroll
                            for (int q = 0; q < kMS; ++q) {
                                const float w = (okr[u] && s0 + q < nsplit) ? wsm[(row0 + 4 * u) * MAX_SPLITS + s0 + q] : 0.f;
                                acc[u].x += w * v[u][q].x;
                                acc[u].y += w * v[u][q].y;
                                acc[u].z += w * v[u][q].z;
                                acc[u].w += w * v[u][q].w;
                            }
                    }
#pragma unroll
                    for (int u = 0; u < kMR; ++u) {
                        if (!okr[u]) continue;
                        const int row = row0 + 4 * u;
                        uint2 o;
                        o.x = pack_bf16(acc[u].x, acc[u].y);
                        o.y = pack_bf16(acc[u].z, acc[u].w);
                        *reinterpret_cast<uint2*>(p.out + ((int64_t)(entry * p.stride + r0 + row / g) * p.hq + kvh * g +
                                                           row % g) * HD + lane * 4) = o;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TM_COLS) : "memory");
    }
}

}  // namespace

int attn_rows_per_tile(int group) { return QROWS / group; }
int attn_dual_rows_per_tile(int group) { return 64 / group; }
int attn_max_splits() { return MAX_SPLITS; }

bool make_kv_tmap(CUtensorMap* tm, const bf16* kv_pool, const KVLayout& kvl, int n_layers) {
    const uint64_t rows = (uint64_t)n_layers * (uint64_t)kvl.layer_stride / HD;
    return make_tmap_bf16(tm, kv_pool, rows, HD, kPage);
}

bool make_q_tmap(CUtensorMap* tm, const bf16* q, int rows, int hq, int hkv, bool dual) {
    const int g = hq / hkv;
    const cuuint64_t gdim[3] = {(cuuint64_t)HD, (cuuint64_t)hq, (cuuint64_t)rows};
    const cuuint64_t gstride[2] = {(cuuint64_t)HD * 2, (cuuint64_t)hq * HD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)g,
                               (cuuint32_t)(dual ? attn_dual_rows_per_tile(g) : attn_rows_per_tile(g))};
    return encode_tmap_bf16(tm, q, 3, gdim, gstride, box);
}

void launch_attn_bf16(const CUtensorMap& tm_kv, const CUtensorMap& tm_q, const CUtensorMap& tm_q_dual, KVLayout kvl,
                      int layer, int hq, int hkv, bf16* out, float* part_o, float2* part_ml, int* tickets,
                      int n_entries, int stride, int kv_chunk, int max_splits, SlotState ss, RowMap rm, int* err,
                      cudaStream_t st) {
    const int g = hq / hkv;
    // DUAL when every query row of a window fits in 64 (one tile of 64 / g rows)
    const bool dual = stride * g <= 64;
    const int rt = dual ? attn_dual_rows_per_tile(g) : attn_rows_per_tile(g);
    const int tiles = (stride + rt - 1) / rt;
    AttnParams p{kvl, layer, hq, hkv, out, part_o, part_ml, tickets, stride, kv_chunk, max_splits, rt, tiles,
                 ss, rm, err};
    dim3 grid(tiles, hkv, n_entries * max_splits);
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        attr_dev = dev;
    }
    if (dual)
        launch_pdl(attn_tc_kernel<true>, grid, dim3(NTHREADS), SMEM_BYTES, st, tm_kv, tm_q_dual, p);
    else
        launch_pdl(attn_tc_kernel<false>, grid, dim3(NTHREADS), SMEM_BYTES, st, tm_kv, tm_q, p);
}

}  // namespace wedlm

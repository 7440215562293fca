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
// Work item = (batch entry, row tile, KV head, key chunk).  A tile's 128
// query rows (RT window rows x g query heads sharing the KV head; unused rows
// are zero) are the M side of every MMA, so each K/V byte loaded serves all g
// heads:
//   S  = Q K^T   M=128, N=64 keys, K=128 dims  (A = Q, B = K: shared memory)
//   O += P V     M=128, N=128 dims, K=64 keys  (A = P in TMEM, B = V)
// A 16-token page is one TMA box per 64-dim half, so K and V blocks land as
// key rows of 128 bytes with the 128-byte swizzle: the K-major operand form
// for K and the MN-major (dims contiguous) form for V.
//
// The kernel is persistent: one CTA per SM walks its share of the items (the
// non-empty items of the launch, numbered in (entry, tile, KV head, chunk)
// order, dealt round-robin), and its K and V rings, Q buffers, S buffers and O
// accumulators run continuously across items, so the loads of the next item
// stream in while the current one finishes.  Keys below a sequence's committed
// length were written by earlier kernels, so the loaders start on them before
// waiting for the previous kernel (the QKV projection that writes q and the
// window's K/V).
//
// TMEM (512 columns): two S buffers of 64 columns (P overwrites the first 32
// columns of its own S buffer as packed bf16) and two O accumulators of 128.
// Warp roles (224 threads):
//   warps 0-3  softmax: thread i owns query row i (TMEM lane i); causal and
//              chunk masks, running max m and sum l (exp2 domain); O is
//              rescaled in TMEM only when a row's max grows by more than 2^8
//              (otherwise P stays relative to the older max, exactly); at the
//              end of an item O is normalised and stored, or (keys split over
//              chunks) stored unnormalised with (m, l), and the last chunk of
//              the (entry, tile, KV head) to finish merges the partials,
//   warp 4     allocates TMEM; one thread issues the MMAs,
//   warp 5     TMA loads of Q (two 3-D boxes of 64 dims x g heads x rows, into
//              one of two Q buffers) and of K blocks into a 4-stage ring,
//   warp 6     TMA loads of V blocks into a 4-stage ring.
// All waits are bounded; a timeout sets the device error word.
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace wedlm {
namespace {

constexpr int HD = 128;
constexpr int KBLK = 64;
constexpr int QROWS = 128;
constexpr int NK = 2;                               // K ring stages
constexpr int NV = 2;                               // V ring stages
constexpr int Q_BYTES = QROWS * HD * 2;             // two 64-dim halves of 16 KB
constexpr int HALF_BYTES = KBLK * 128;              // 64 keys x 64 dims
constexpr int BLK_BYTES = 2 * HALF_BYTES;           // one K or V block: 16 KB
constexpr int BOX_BYTES = kPage * 128;              // one page, one half: 2 KB
constexpr int NTHREADS = 224;
constexpr int CTAS_PER_SM = 2;                      // two independent item streams per SM
constexpr uint32_t TM_S = 0, TM_O = 128, TM_COLS = 256;  // S buffer b at 64 b, O at 128
constexpr int MAX_SPLITS = 32;  // key chunks per row tile
constexpr int kMR = 4, kMS = 2;  // merge: rows x chunk partials in flight per lane
constexpr int XCH_FLOATS = 32 * 64 + 2 * 64;        // DUAL exchange: 32 dims x 64 rows, then (m, l)
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;
constexpr int OFF_V = OFF_K + NK * BLK_BYTES;
constexpr int OFF_X = OFF_V + NV * BLK_BYTES;                    // DUAL exchange
constexpr int OFF_BAR = OFF_X + XCH_FLOATS * 4;
constexpr int BAR_BYTES = 512;                                    // barriers and flags
constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024 /*align*/;

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
    int n_entries, stride, kv_chunk, max_splits, rt, tiles;
    SlotState ss;
    RowMap rm;
    int* err;
};

// One work item and the sizes every role derives from it.
struct Item {
    int entry, tile, kvh, sp;
    int slot, S, n, r0, r_last, ks, ke, nblk, nsplit;
};

// The items of this CTA, in order: the launch's non-empty items are numbered
// over (entry, tile) groups -- group size hkv * nsplit, KV head then chunk
// within a group -- and CTA c takes numbers c, c + G, c + 2G, ...  Every role
// of the CTA runs its own copy and sees the same sequence (the sizes it reads
// do not change during the launch).  S and n are read through L2: the kernel
// may start before the previous kernel of the stream has finished.
struct ItemIter {
    int e = 0, t = 0;          // current group
    int base = 0;              // number of the group's first item
    int next = 0;              // next number this CTA takes
    int cnt = -1;              // items in the current group (-1: not computed)
    int S = 0, n = 0, nsplit = 0;
};

__device__ __forceinline__ bool next_item(ItemIter& it, const AttnParams& p, Item& o) {
    while (it.e < p.n_entries) {
        if (it.cnt < 0) {
            const int slot = p.rm.slot_base + it.e;
            it.n = __ldcg(p.rm.n + slot);
            it.S = __ldcg(p.ss.S + slot);
            const int r0 = it.t * p.rt;
            if (r0 >= it.n) {
                it.cnt = 0;
            } else {
                const int kend = it.S + min(r0 + p.rt, it.n);
                it.nsplit = (kend + p.kv_chunk - 1) / p.kv_chunk;
                it.cnt = p.hkv * it.nsplit;
                if (it.nsplit > p.max_splits || it.S < 0) {  // more keys than the launch has room for
                    set_error(p.err, kErrBounds);
                    it.cnt = 0;
                }
            }
        }
        if (it.next < it.base + it.cnt) {
            const int local = it.next - it.base;
            it.next += gridDim.x;
            o.entry = it.e;
            o.tile = it.t;
            o.kvh = local / it.nsplit;
            o.sp = local % it.nsplit;
            o.slot = p.rm.slot_base + it.e;
            o.S = it.S;
            o.n = it.n;
            o.nsplit = it.nsplit;
            o.r0 = it.t * p.rt;
            o.r_last = min(o.r0 + p.rt, it.n) - 1;
            const int kend = it.S + o.r_last + 1;
            o.ks = o.sp * p.kv_chunk;
            o.ke = min(kend, o.ks + p.kv_chunk);
            o.nblk = (o.ke - o.ks + KBLK - 1) / KBLK;
            return true;
        }
        it.base += it.cnt;
        it.cnt = -1;
        if (++it.t == p.tiles) {
            it.t = 0;
            ++it.e;
        }
    }
    return false;
}

// TMA loads of one KV ring (K or V, kv = 0 / 1) for every item of this CTA,
// issued by lane 0 of the calling warp; the warp's lanes hold the chunk's page
// ids, 128 at a time.  Keys past the chunk end (and, after an error, unmapped
// pages) read a mapped page instead: their scores are masked, and pool memory
// is zeroed at creation and only ever holds finite K/V, so P = 0 times V stays
// 0.  Blocks that reach the window rows (keys >= S) wait for the previous
// kernel first; with `with_q` the warp also loads each item's Q (after that
// wait) into its Q buffer.  Returns false after a failed wait.
template <bool DUAL, int NST>
__device__ __forceinline__ bool kv_loader(const AttnParams& p, const CUtensorMap* tm_kv, const CUtensorMap* tm_q,
                                          int kv, uint8_t* ring, uint64_t* full, uint64_t* empty, bool with_q,
                                          uint8_t* sQ, uint64_t* q_full, uint64_t* q_empty, int lane, bool& waited,
                                          uint32_t& issued, uint32_t& q_issued) {
    int* err = p.err;
    const int g = p.hq / p.hkv;
    ItemIter it;
    it.next = blockIdx.x;
    Item item;
    uint32_t gb = 0;
    int li = 0;
    bool ok = true;
    while (ok && next_item(it, p, item)) {
        const int32_t* pt = p.ss.page_table + (int64_t)item.slot * p.ss.pages_per_seq;
        const int64_t row0 = p.kvl.page_base(p.layer, 0, kv, item.kvh) / HD;  // pool row of (page 0, kv, head, 0)
        const int64_t page_rows = (int64_t)2 * p.kvl.hkv * kPage;            // pool rows per page step
        const int page_first = item.ks / kPage, page_end = (item.ke + kPage - 1) / kPage;
        int batch = -1;
        int preg[4];
        auto load_batch = [&](int b) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pi = page_first + b * 128 + i * 32 + lane;
                int pg = -1;
                if (pi < page_end) {
                    pg = pi < p.ss.pages_per_seq ? __ldcg(pt + pi) : -1;
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
        int fallback = __shfl_sync(0xffffffffu, preg[0], 0);
        if (fallback < 0) fallback = 0;
        // Q of this item (q comes from the previous kernel).  The first item's Q
        // is deferred until a block needs that kernel anyway, or the ring is
        // full (the MMAs that free it need Q): cache blocks go out first.
        const int qb = 0;  // one Q buffer: item li's load waits for item li-1's last S
        bool q_pending = with_q;
        auto issue_q = [&]() -> bool {
            if (!waited) {
                griddep_wait();
                waited = true;
            }
            bool qok = true;
            if (lane == 0) qok = mbar_wait_bounded(smem_u32(&q_empty[qb]), (li & 1) ^ 1, err);
            qok = __shfl_sync(0xffffffffu, qok, 0);
            if (qok) q_issued = (uint32_t)li + 1;
            if (qok && lane == 0) {
                const int qrows = p.rt * g;
                mbar_expect_tx(&q_full[qb], (DUAL ? 4 : 2) * 128 * qrows);
                const int z = item.entry * p.stride + item.r0, y = item.kvh * g;
                const uint32_t qa = smem_u32(sQ + qb * Q_BYTES);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tma_box3(qa + h * (QROWS * 128), tm_q, h * 64, y, z, &q_full[qb]);
                    if (DUAL) tma_box3(qa + h * (QROWS * 128) + 64 * 128, tm_q, h * 64, y, z, &q_full[qb]);
                }
            }
            q_pending = false;
            return qok;
        };
        if (q_pending && li > 0 && !(ok = issue_q())) break;
        for (int j = 0; j < item.nblk; ++j, ++gb) {
            const int st = gb % NST;
            // this block's four pages: local index li4 = 4j + lane (lanes 0..3)
            const int li4 = j * 4 + (lane & 3);
            if ((li4 >> 7) != batch) load_batch(li4 >> 7);
            const int w = li4 & 127;
            const int c0 = __shfl_sync(0xffffffffu, preg[0], w & 31), c1 = __shfl_sync(0xffffffffu, preg[1], w & 31);
            const int c2 = __shfl_sync(0xffffffffu, preg[2], w & 31), c3 = __shfl_sync(0xffffffffu, preg[3], w & 31);
            int pg = (w >> 5) == 0 ? c0 : (w >> 5) == 1 ? c1 : (w >> 5) == 2 ? c2 : c3;
            if (pg < 0) pg = fallback;
            // keys at or past S are the window's rows, written by the previous kernel
            const bool window = item.ks + (j + 1) * KBLK > item.S;
            if (q_pending && (window || gb >= (uint32_t)NST) && !(ok = issue_q())) break;
            if (!waited && window) {
                griddep_wait();
                waited = true;
            }
            if (lane == 0) ok = mbar_wait_bounded(smem_u32(&empty[st]), ((gb / NST) & 1) ^ 1, err);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) mbar_expect_tx(&full[st], BLK_BYTES);
            __syncwarp();
            if (lane < 4) {
                const int y = (int)(row0 + (int64_t)pg * page_rows);
                const uint32_t dst = smem_u32(ring + st * BLK_BYTES) + lane * BOX_BYTES;
                tma_box(dst, tm_kv, 0, y, &full[st]);
                tma_box(dst + HALF_BYTES, tm_kv, 64, y, &full[st]);
            }
            issued = gb + 1;
        }
        if (ok && q_pending) ok = issue_q();
        ++li;
    }
    return ok;
}

// DUAL (valid query rows <= 64): rows 64..127 repeat rows 0..63, and the
// thread of row i + 64 takes keys 32..63 of every block while the thread of
// row i takes keys 0..31, each writing zeros into the other half of its P
// row; the two share the running max through shared memory, so O rows i and
// i + 64 hold the two halves of one result (summed at the end).  This halves
// the per-thread softmax work when a tile has 64 or fewer query rows.
template <bool DUAL>
__global__ void __launch_bounds__(NTHREADS, CTAS_PER_SM) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                                                              const __grid_constant__ CUtensorMap tm_q,
                                                              const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + OFF_Q;  // Q buffer
    uint8_t* sK = smem + OFF_K;  // [NK] K blocks
    uint8_t* sV = smem + OFF_V;  // [NV] V blocks
    float* xch = reinterpret_cast<float*>(smem + OFF_X);  // DUAL exchange
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* q_full = bars + 0;    // [1]
    uint64_t* q_empty = bars + 1;   // [1]
    uint64_t* k_full = bars + 2;    // [NK]
    uint64_t* k_empty = bars + 4;   // [NK]
    uint64_t* v_full = bars + 6;    // [NV]
    uint64_t* v_empty = bars + 8;   // [NV]
    uint64_t* s_full = bars + 10;   // [2] per S buffer
    uint64_t* p_full = bars + 12;   // [2] per S buffer
    uint64_t* o_done = bars + 14;   // one completion per P V
    uint64_t* o_full = bars + 15;   // the item's last P V done
    uint64_t* o_free = bars + 16;   // O read out by the softmax warps
    uint64_t* drain = bars + 17;    // the MMA thread's last MMAs (error exit)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
    int* last_flag = reinterpret_cast<int*>(bars + 19);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.hq / p.hkv;
    const int qrows = p.rt * g;  // query rows of a tile (<= 64 when DUAL)

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_kv)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(o_full, 1);
        mbar_init(o_free, 4);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
        }
        for (int s = 0; s < NK; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
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

    if (warp == 5 || warp == 6) {
        // ---------------------------------------------------------- loaders
        bool waited = false;
        uint32_t issued = 0, q_issued = 0;
        if (warp == 5)
            kv_loader<DUAL, NK>(p, &tm_kv, &tm_q, 0, sK, k_full, k_empty, true, sQ, q_full, q_empty, lane, waited,
                                issued, q_issued);
        else
            kv_loader<DUAL, NV>(p, &tm_kv, &tm_q, 1, sV, v_full, v_empty, false, sQ, q_full, q_empty, lane, waited,
                                issued, q_issued);
        if (!waited) griddep_wait();
        griddep_launch();
        // Copies still in flight (only after an error) must land before the CTA
        // exits: wait, bounded, for the last blocks issued to each stage.
        if (lane == 0) {
            uint64_t* full = warp == 5 ? k_full : v_full;
            const uint32_t nst = warp == 5 ? NK : NV;
            for (uint32_t j = issued > nst ? issued - nst : 0u; j < issued; ++j)
                mbar_wait_bounded(smem_u32(&full[j % nst]), (j / nst) & 1, nullptr, 200000000LL);
            if (q_issued > 0) mbar_wait_bounded(smem_u32(q_full), (q_issued - 1) & 1, nullptr, 200000000LL);
        }
    } else if (warp == 4) {
        // -------------------------------------------------------------- MMA
        griddep_wait();
        griddep_launch();
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, KBLK);
            constexpr uint32_t idO = idesc_bf16(128, HD) | (1u << 16);  // B (V) MN-major
            // Two cursors over this CTA's blocks (in item order): `sc` issues
            // S = Q K^T two blocks ahead of `pv`, which issues O += P V.
            struct Cursor {
                ItemIter it;
                Item item;
                int li = -1, j = 0;
                uint32_t gb = 0;
                bool valid = false;
            };
            auto start = [&](Cursor& c) {
                c.it.next = blockIdx.x;
                c.valid = next_item(c.it, p, c.item);
                c.li = 0;
                c.j = 0;
                c.gb = 0;
            };
            auto advance = [&](Cursor& c) {
                ++c.gb;
                if (++c.j == c.item.nblk) {
                    c.j = 0;
                    ++c.li;
                    c.valid = next_item(c.it, p, c.item);
                }
            };
            auto issue_s = [&](const Cursor& c) -> bool {
                const uint32_t b = c.gb;
                const int qb = 0;
                if (c.j == 0 && !mbar_wait_bounded(smem_u32(q_full), c.li & 1, err)) return false;
                if (!mbar_wait_bounded(smem_u32(&k_full[b % NK]), (b / NK) & 1, err)) return false;
                tc_fence_after();
                const uint32_t qa = smem_u32(sQ + qb * Q_BYTES);
                const uint32_t kb = smem_u32(sK + (b % NK) * BLK_BYTES);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    mma_ss(tmem + TM_S + (b & 1) * 64, sdesc(qa + (kk >> 2) * (QROWS * 128) + (kk & 3) * 32),
                           sdesc(kb + (kk >> 2) * HALF_BYTES + (kk & 3) * 32), idS, kk > 0 ? 1u : 0u);
                umma_commit(&k_empty[b % NK]);
                umma_commit(&s_full[b & 1]);
                if (c.j == c.item.nblk - 1) umma_commit(&q_empty[qb]);
                return true;
            };
            Cursor sc, pv;
            start(sc);
            start(pv);
            bool ok = true;
            for (int a = 0; a < 2 && sc.valid && ok; ++a) {
                ok = issue_s(sc);
                advance(sc);
            }
            while (pv.valid && ok) {
                const uint32_t b = pv.gb;
                const int ob = 0;
                if (!(ok = mbar_wait_bounded(smem_u32(&p_full[b & 1]), (b >> 1) & 1, err))) break;
                if (pv.j == 0 && !(ok = mbar_wait_bounded(smem_u32(o_free), (pv.li & 1) ^ 1, err))) break;
                if (!(ok = mbar_wait_bounded(smem_u32(&v_full[b % NV]), (b / NV) & 1, err))) break;
                tc_fence_after();
                const uint32_t vb = smem_u32(sV + (b % NV) * BLK_BYTES);
#pragma unroll
                for (int kk = 0; kk < KBLK / 16; ++kk)
                    mma_ts(tmem + TM_O + ob * 128, tmem + TM_S + (b & 1) * 64 + kk * 8, sdesc_mn(vb + kk * 2048), idO,
                           (pv.j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&v_empty[b % NV]);
                umma_commit(o_done);
                if (pv.j == pv.item.nblk - 1) umma_commit(o_full);
                advance(pv);
                if (sc.valid) {
                    // S buffer b & 1 is read by this P V: wait for it before S(b + 2) overwrites it
                    if (!(ok = mbar_wait_bounded(smem_u32(o_done), b & 1, err))) break;
                    ok = issue_s(sc);
                    advance(sc);
                }
            }
            // every MMA issued has completed before TMEM may be released
            umma_commit(drain);
            mbar_wait_bounded(smem_u32(drain), 0, nullptr, 200000000LL);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------- softmax
        griddep_wait();
        griddep_launch();
        const int tid = threadIdx.x;                // TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int qi = DUAL ? (tid & 63) : tid;     // query row this thread works for
        const int half = DUAL ? (tid >> 6) : 0;     // DUAL: key half of every block
        const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
        constexpr int NC = DUAL ? 32 : 64;          // score columns per thread and block
        ItemIter it;
        it.next = blockIdx.x;
        Item item;
        uint32_t gb = 0;
        int li = 0;
        bool ok = true;
        while (ok && next_item(it, p, item)) {
            const int rr = item.r0 + qi / g;
            const bool qok = qi < qrows && rr < item.n;
            const int lim = item.S + (qok ? rr : item.r_last);  // last visible key
            // running max (exp2 domain) and sum of this thread's keys; in DUAL
            // mode each key half keeps its own and the two merge at the end
            float m_ref = -INFINITY, l = 0.f;
            for (int j = 0; j < item.nblk && ok; ++j, ++gb) {
                const int b = gb & 1;
                const int kb0 = item.ks + j * KBLK + half * 32;
                const uint32_t tS = tmem + lane_base + TM_S + b * 64;
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&s_full[b]), (gb >> 1) & 1, err));
                if (!ok) break;
                tc_fence_after();
                uint32_t r[32];
                float s[NC];
#pragma unroll
                for (int h = 0; h < NC / 32; ++h) {
                    tmem_ld32(tS + (DUAL ? half * 32 : h * 32), r);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int t = kb0 + h * 32 + c;
                        s[h * 32 + c] = (t < item.ke && t <= lim) ? __uint_as_float(r[c]) * sl2 : -INFINITY;
                    }
                }
                float bmax = -INFINITY;
#pragma unroll
                for (int c = 0; c < NC; ++c) bmax = fmaxf(bmax, s[c]);
                const bool need = bmax > m_ref + 8.0f;
                if (j > 0 && __any_sync(0xffffffffu, need)) {
                    // P V of the previous block must be done before O is rescaled
                    ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(o_done), (gb - 1) & 1, err));
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
                        const float a = exp2f(s[2 * c] - ref), bb = exp2f(s[2 * c + 1] - ref);
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
            if (!ok) break;
            // ---- item epilogue: O of this item is complete once its last P V is
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(o_full), li & 1, err));
            if (!ok) break;
            tc_fence_after();
            const int qrow = item.entry * p.stride + (qok ? rr : item.r_last);
            const int qhead = item.kvh * g + qi % g;
            const int64_t pbase = ((int64_t)qrow * p.hq + qhead) * p.max_splits;
            const uint32_t tO = tmem + lane_base + TM_O;
            // DUAL: the two key halves of row qi (rows qi and qi + 64 of O) merge:
            // O = 2^(m0 - M) O0 + 2^(m1 - M) O1, l likewise, M = max(m0, m1)
            float a_own = 1.f, a_other = 0.f;
            if (DUAL) {
                softmax_sync();  // the exchange buffer is free (previous item)
                if (half) {
                    xch[32 * 64 + qi] = m_ref;
                    xch[32 * 64 + 64 + qi] = l;
                }
                softmax_sync();
                if (!half) {
                    const float m1 = xch[32 * 64 + qi], l1 = xch[32 * 64 + 64 + qi];
                    const float M = fmaxf(m_ref, m1);
                    a_own = (M == -INFINITY) ? 0.f : exp2f(m_ref - M);
                    a_other = (M == -INFINITY) ? 0.f : exp2f(m1 - M);
                    l = a_own * l + a_other * l1;
                    m_ref = M;
                }
            }
            const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll 1
            for (int c = 0; c < HD; c += 32) {
                uint32_t r[32];
                tmem_ld32(tO + c, r);
                tmem_wait_ld();
                if (DUAL) {
                    // the other key half of row qi, through shared memory
                    softmax_sync();
                    if (half) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) xch[x * 64 + qi] = __uint_as_float(r[x]);
                    }
                    softmax_sync();
                    if (half) continue;
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        r[x] = __float_as_uint(a_own * __uint_as_float(r[x]) + a_other * xch[x * 64 + qi]);
                }
                if (!qok) continue;
                if (item.nsplit == 1) {
                    __nv_bfloat162* op =
                        reinterpret_cast<__nv_bfloat162*>(p.out + ((int64_t)qrow * p.hq + qhead) * HD + c);
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        op[x] = __floats2bfloat162_rn(__uint_as_float(r[2 * x]) * inv, __uint_as_float(r[2 * x + 1]) * inv);
                } else {
                    float4* po = reinterpret_cast<float4*>(p.part_o + (pbase + item.sp) * HD + c);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        po[x] = make_float4(__uint_as_float(r[4 * x]), __uint_as_float(r[4 * x + 1]),
                                            __uint_as_float(r[4 * x + 2]), __uint_as_float(r[4 * x + 3]));
                }
            }
            // O is read out: the MMA may accumulate the next item into it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
            if (qok && item.nsplit > 1 && !(DUAL && half)) p.part_ml[pbase + item.sp] = make_float2(m_ref, l);
            if (item.nsplit > 1) {
                // The last chunk of this (entry, tile, KV head) to finish merges all
                // chunks' partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
                __threadfence();
                softmax_sync();
                if (tid == 0) {
                    int* ticket = p.tickets + ((int64_t)item.entry * p.hkv + item.kvh) * p.tiles + item.tile;
                    const int prev = atomicAdd(ticket, 1);
                    const int last = prev == item.nsplit - 1;
                    if (last) *ticket = 0;
                    *last_flag = last;
                }
                softmax_sync();
                const int is_last = *last_flag;
                softmax_sync();  // every thread has read the flag before the next item may rewrite it
                if (is_last) {
                    __threadfence();
                    const int nsplit = item.nsplit;
                    // a warp takes kMR rows at a time (rows warp, warp + 4, ...), a lane
                    // 4 dims; lane s holds chunk s's weight 2^(m_s - M) / L of each of
                    // those rows (shuffles), and kMR rows x kMS chunk partials are in
                    // flight together
#pragma unroll 1
                    for (int row0 = warp; row0 < qrows; row0 += 4 * kMR) {
                        int64_t pbr[kMR];
                        bool okr[kMR];
                        float wl[kMR];
#pragma unroll
                        for (int u = 0; u < kMR; ++u) {
                            const int row = row0 + 4 * u;
                            okr[u] = row < qrows && item.r0 + row / g < item.n;
                            pbr[u] = ((int64_t)(item.entry * p.stride + item.r0 + row / g) * p.hq + item.kvh * g +
                                      row % g) * p.max_splits;
                        }
                        float2 ml[kMR];
#pragma unroll
                        for (int u = 0; u < kMR; ++u)
                            ml[u] = (okr[u] && lane < nsplit) ? __ldcg(&p.part_ml[pbr[u] + lane])
                                                              : make_float2(-INFINITY, 0.f);
#pragma unroll
                        for (int u = 0; u < kMR; ++u) {
                            float M = ml[u].x;
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
                            const float w = (ml[u].x == -INFINITY || M == -INFINITY) ? 0.f : exp2f(ml[u].x - M);
                            float L = w * ml[u].y;
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
                            wl[u] = L > 0.f ? w / L : 0.f;
                        }
                        float4 acc[kMR];
#pragma unroll
                        for (int u = 0; u < kMR; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
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
                                    const float w = __shfl_sync(0xffffffffu, wl[u], (s0 + q) & 31);
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
                            uint2 o2;
                            o2.x = pack_bf16(acc[u].x, acc[u].y);
                            o2.y = pack_bf16(acc[u].z, acc[u].w);
                            *reinterpret_cast<uint2*>(p.out + ((int64_t)(item.entry * p.stride + item.r0 + row / g) * p.hq +
                                                               item.kvh * g + row % g) * HD + lane * 4) = o2;
                        }
                    }
                }
            }
            ++li;
        }
    } else {
        griddep_wait();
        griddep_launch();
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

int attn_kv_chunk_for(int max_batch, int max_window, int hq, int hkv, int max_ctx, int num_sms) {
    // Fixed per context (a sequence's result does not depend on its batch
    // neighbours): a full batch at half the context length makes about two
    // items per SM; at least four 64-key blocks per chunk (below that the item
    // setup and the merge of many partials outweigh the extra parallelism), at
    // most 32 blocks, and at most attn_max_splits() chunks per row tile.
    const int g = hq / hkv;
    const int rt = attn_rows_per_tile(g);
    const long long tiles = (max_window + rt - 1) / rt;
    const long long pairs = (long long)max_batch * tiles * hkv;
    const long long blocks = pairs * std::max(1, (max_ctx / 2 + 63) / 64);
    long long cb = (blocks + 2LL * num_sms - 1) / (2LL * num_sms);
    cb = std::max(4LL, std::min(cb, 32LL));
    cb = std::max(cb, ((long long)max_ctx + 64LL * MAX_SPLITS - 1) / (64LL * MAX_SPLITS));
    return (int)(cb * 64);
}

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

cudaError_t launch_attn_bf16(const CUtensorMap& tm_kv, const CUtensorMap& tm_q, const CUtensorMap& tm_q_dual,
                             KVLayout kvl, int layer, int hq, int hkv, bf16* out, float* part_o, float2* part_ml,
                             int* tickets, int n_entries, int stride, int kv_chunk, int max_splits, SlotState ss,
                             RowMap rm, int* err, cudaStream_t st) {
    if (hq % hkv || hq / hkv > QROWS || max_splits < 1 || max_splits > MAX_SPLITS || kv_chunk < KBLK ||
        kv_chunk % KBLK || n_entries < 1 || stride < 1)
        return cudaErrorInvalidValue;
    const int g = hq / hkv;
    // DUAL when every query row of a window fits in 64 (one tile of 64 / g rows)
    const bool dual = stride * g <= 64;
    const int rt = dual ? attn_dual_rows_per_tile(g) : attn_rows_per_tile(g);
    const int tiles = (stride + rt - 1) / rt;
    AttnParams p{kvl, layer, hq, hkv, out, part_o, part_ml, tickets, n_entries, stride, kv_chunk, max_splits, rt, tiles,
                 ss, rm, err};
    static int attr_dev = -1;
    static int num_sms = 148;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
        attr_dev = dev;
    }
    // two persistent CTAs per SM, fewer when the launch has fewer items
    const long long items_max = (long long)n_entries * tiles * hkv * max_splits;
    const int grid = (int)std::max(1LL, std::min<long long>(items_max, (long long)CTAS_PER_SM * num_sms));
    if (dual) return launch_pdl(attn_tc_kernel<true>, dim3(grid), dim3(NTHREADS), SMEM_BYTES, st, tm_kv, tm_q_dual, p);
    return launch_pdl(attn_tc_kernel<false>, dim3(grid), dim3(NTHREADS), SMEM_BYTES, st, tm_kv, tm_q, p);
}

}  // namespace wedlm

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
// Persistent, two CTAs per SM: each CTA walks its share of the launch's
// non-empty items (numbered in (entry, tile, KV head, chunk) order, dealt
// round-robin) with every stage of its pipeline running ahead of the next:
// K and V rings of two 64-key blocks each (16 KB per block), a Q buffer, two S
// buffers and an O accumulator in TMEM (256 columns: S buffer s at 64 s, O at
// 128; P overwrites the first 32 columns of its S buffer as packed bf16).  The
// MMA thread issues S = Q K^T a block ahead of the softmax and O += P V as
// soon as a block's P is written; an item's output is read out by separate
// epilogue warps while the softmax moves on to the next item.  Two CTAs per SM
// because TMA loads of 2 KB page boxes are limited per CTA: one CTA per SM
// streamed random pages at about 3.8 TB/s whatever its ring depth, two CTAs
// at the HBM peak (measured on this hardware).  Keys below a sequence's
// committed length were written by earlier kernels, so the loaders start on
// them before waiting for the previous kernel (the QKV projection that writes
// q and the window's K/V).
//
// Warp roles (352 threads):
//   warps 0-3  softmax: thread i owns query row i (TMEM lane i), reading its
//              scores 32 columns at a time; causal and chunk masks on the
//              blocks that reach the window or the chunk end, running max m
//              and sum l; O is rescaled in TMEM only when a
//              row's max grows by more than 2^8 in the exp2 domain (otherwise
//              P stays relative to the older max, exactly); at the end of an
//              item (m, l) go to the epilogue warps through shared memory,
//   warps 4-7  epilogue: O of a finished item out of TMEM, normalised to bf16
//              (a single key chunk) or stored unnormalised with (m, l) as the
//              chunk's partial, which attn_merge_kernel combines,
//   warp 8     allocates TMEM; one thread issues the MMAs,
//   warp 9     TMA loads of Q (two 3-D boxes of 64 dims x g heads x rows) and
//              of the K blocks,
//   warp 10    TMA loads of the V blocks.
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
constexpr int NQ = 1;                               // Q buffers
constexpr int NSB = 2;                              // S buffers in TMEM
constexpr int NO = 1;                               // O accumulators in TMEM
constexpr int CTAS_PER_SM = 2;
constexpr int Q_BYTES = QROWS * HD * 2;             // two 64-dim halves of 16 KB
constexpr int HALF_BYTES = KBLK * 128;              // 64 keys x 64 dims
constexpr int BLK_BYTES = 2 * HALF_BYTES;           // one K or V block: 16 KB
constexpr int BOX_BYTES = kPage * 128;              // one page, one half: 2 KB
constexpr int NTHREADS = 352;
constexpr int WARP_EPI = 4, WARP_MMA = 8, WARP_KLOAD = 9, WARP_VLOAD = 10;
constexpr uint32_t TM_S = 0, TM_O = NSB * 64, TM_COLS = 256;
constexpr int MAX_SPLITS = 32;  // key chunks per row tile
constexpr int XCH_FLOATS = 32 * 64;                 // DUAL exchange: 32 dims x 64 rows
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
constexpr int OFF_V = OFF_K + NK * BLK_BYTES;
constexpr int OFF_X = OFF_V + NV * BLK_BYTES;                    // DUAL exchange
constexpr int OFF_ML = OFF_X + XCH_FLOATS * 4;                   // (m, l) per O buffer and row
constexpr int ENT_CAP = 256;                                     // entries whose (n, S) are cached
constexpr int GRP_CAP = 512;                                     // (entry, tile) groups with item prefix sums
constexpr int OFF_ENT = OFF_ML + NO * QROWS * 8;                  // (n, S) of the launch's entries
constexpr int OFF_GRP = OFF_ENT + ENT_CAP * 8;                    // item prefix sums per group (two)
constexpr int OFF_BAR = OFF_GRP + 2 * GRP_CAP * 4;
constexpr int BAR_BYTES = 512;                                    // barriers
constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024 /*align*/;
static_assert(CTAS_PER_SM * (SMEM_BYTES + 1024) <= 228 * 1024, "attention shared memory: two CTAs per SM");
// Row max growth (exp2 domain) tolerated before O is rescaled.
constexpr float kRescaleLog2 = 8.0f;

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
// Non-blocking probe: has the phase of parity `parity` completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// One box of the pool's tensor map (x = dim offset, y = pool row) into shared memory.
__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// A 3-D box of q: 64 dims x g heads x rt rows (one 64-dim half of a tile).
__device__ __forceinline__ void tma_box3(uint32_t dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
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
// Barrier among the 128 epilogue threads only (named barrier 1).
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// The same barrier, returning whether `v` holds in every epilogue thread: the
// DUAL exchange (which synchronises the four warps) is entered by all of them
// or by none, also when a bounded wait gave up in one warp only.
__device__ __forceinline__ bool epi_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}

// 2^x on the special-function unit (PTX ex2.approx, flush-to-zero): about 2
// ulp, ex2(-inf) = +0.  The softmax weights are rounded to bf16 right after.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

struct AttnParams {
    KVLayout kvl;
    int layer, hq, hkv;
    bf16* out;
    float* part_o;    // [rows][hq][max_splits][128] unnormalised chunk outputs
    float2* part_ml;  // [rows][hq][max_splits] (max in the exp2 domain, sum)
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
// do not change during the launch).  Each entry's (n, S) is read from global
// memory once per CTA, at kernel start, into shared memory (the first
// ENT_CAP entries; any beyond are read through L2 as they come): walking
// from one of the CTA's items to the next passes several groups, and a
// dependent L2 round trip per group would dominate short items.  The kernel
// may start before the previous kernel of the stream has finished; n and S
// are not written by it.
struct ItemIter {
    int g = 0, g2 = 0;         // current group of the full-chunk / last-chunk items (bisection)
    int e = 0, t = 0;          // current group
    int base = 0;              // number of the group's first item
    int next = 0;              // next number this CTA takes
    int cnt = -1;              // items in the current group (-1: not computed)
    int S = 0, n = 0, nsplit = 0;
};

// Key chunks of row tile t of a window with n rows over committed length S.
__device__ __forceinline__ int tile_splits(int S, int n, int t, int rt, int kv_chunk) {
    const int kend = S + min((t + 1) * rt, n);
    return (kend + kv_chunk - 1) / kv_chunk;
}

// (n, S) of entry e: shared memory for the first ENT_CAP entries, else L2.
__device__ __forceinline__ int2 entry_ns(const AttnParams& p, const int2* ent, int e) {
    if (e < ENT_CAP) return ent[e];
    const int slot = p.rm.slot_base + e;
    return make_int2(__ldcg(p.rm.n + slot), __ldcg(p.ss.S + slot));
}

// Items of group g = (entry g / tiles, tile g % tiles): hkv * nsplit, 0 for an
// empty tile or (bounds error) a tile with more chunks than the launch allows.
__device__ __forceinline__ int group_items(const AttnParams& p, const int2* ent, int g, int& S, int& n, int& nsplit) {
    const int e = g / p.tiles, t = g - e * p.tiles;
    const int2 v = entry_ns(p, ent, e);
    n = v.x;
    S = v.y;
    if (t * p.rt >= n) return 0;
    nsplit = tile_splits(S, n, t, p.rt, p.kv_chunk);
    if (nsplit > p.max_splits || S < 0) {  // more keys than the launch has room for
        set_error(p.err, kErrBounds);
        return 0;
    }
    return p.hkv * nsplit;
}

__device__ __forceinline__ void fill_item(const AttnParams& p, int g, int kvh, int sp, int S, int n, int nsplit,
                                          Item& o) {
    o.entry = g / p.tiles;
    o.tile = g - o.entry * p.tiles;
    o.kvh = kvh;
    o.sp = sp;
    o.slot = p.rm.slot_base + o.entry;
    o.S = S;
    o.n = n;
    o.nsplit = nsplit;
    o.r0 = o.tile * p.rt;
    o.r_last = min(o.r0 + p.rt, n) - 1;
    const int kend = S + o.r_last + 1;
    o.ks = o.sp * p.kv_chunk;
    o.ke = min(kend, o.ks + p.kv_chunk);
    o.nblk = (o.ke - o.ks + KBLK - 1) / KBLK;
}

// First g in [lo, G) with a[g] > x (a non-decreasing, a[G - 1] > x).
__device__ __forceinline__ int bisect(const int* a, int lo, int G, int x) {
    int hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] > x) hi = mid;
        else lo = mid + 1;
    }
    return lo;
}

// The CTA's next item.  With at most GRP_CAP groups the items are numbered
// full chunks first -- (group, KV head, chunk) for every chunk but a group's
// last -- then every group's last chunk (KV head order), and the number is
// looked up by bisection in per-group prefix sums built once per CTA (gend:
// full-chunk items, gend + GRP_CAP: last-chunk items).  Dealt round-robin,
// this puts a short tail chunk beside a full chunk on an SM's two CTAs, where
// the plain (group, head, chunk) order alternated them so that the two CTAs of
// an SM often both drew full chunks.  Otherwise the groups are walked one by
// one in (group, head, chunk) order.
__device__ __forceinline__ bool next_item(ItemIter& it, const AttnParams& p, const int2* ent, const int* gend,
                                          Item& o) {
    const int G = p.n_entries * p.tiles;
    if (G <= GRP_CAP) {
        if (G == 0) return false;
        const int* glast = gend + GRP_CAP;
        const int nfull = gend[G - 1];
        if (it.next >= nfull + glast[G - 1]) return false;
        int S, n, nsplit;
        if (it.next < nfull) {
            const int g = bisect(gend, it.g, G, it.next);
            it.g = g;
            group_items(p, ent, g, S, n, nsplit);
            const int local = it.next - (g ? gend[g - 1] : 0);
            fill_item(p, g, local / (nsplit - 1), local % (nsplit - 1), S, n, nsplit, o);
        } else {
            const int x = it.next - nfull;
            const int g = bisect(glast, it.g2, G, x);
            it.g2 = g;
            group_items(p, ent, g, S, n, nsplit);
            fill_item(p, g, x - (g ? glast[g - 1] : 0), nsplit - 1, S, n, nsplit, o);
        }
        it.next += gridDim.x;
        return true;
    }
    while (it.e < p.n_entries) {
        const int g = it.e * p.tiles + it.t;
        if (it.cnt < 0) it.cnt = group_items(p, ent, g, it.S, it.n, it.nsplit);
        if (it.next < it.base + it.cnt) {
            const int local = it.next - it.base;
            fill_item(p, g, local / it.nsplit, local % it.nsplit, it.S, it.n, it.nsplit, o);
            it.next += gridDim.x;
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
// wait) into Q buffer (item index mod NQ).  Returns false after a failed wait.
template <bool DUAL>
__device__ __forceinline__ bool kv_loader(const AttnParams& p, const int2* ent, const int* gend,
                                          const CUtensorMap* tm_kv,
                                          const CUtensorMap* tm_q, int kv, uint8_t* ring, uint64_t* full, uint64_t* empty, bool with_q,
                                          uint8_t* sQ, uint64_t* q_full, uint64_t* q_empty, int lane, bool& waited,
                                          uint32_t& issued, uint32_t& q_issued) {
    constexpr int NST = NK;
    static_assert(NK == NV, "one loader body serves both rings");
    int* err = p.err;
    const int g = p.hq / p.hkv;
    const int64_t page_rows = (int64_t)2 * p.kvl.hkv * kPage;  // pool rows per page step
    // Page ids of one item's pages [page_first + 128 b, +128): lane l holds
    // pages +l, +32+l, +64+l, +96+l (-1 past the chunk end or out of range).
    auto page_batch = [&](const Item& itm, int b, int (&out)[4]) {
        const int32_t* pt = p.ss.page_table + (int64_t)itm.slot * p.ss.pages_per_seq;
        const int page_first = itm.ks / kPage, page_end = (itm.ke + kPage - 1) / kPage;
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
            out[i] = pg;
        }
    };
    ItemIter it;
    it.next = blockIdx.x;
    Item item, nitem;
    bool has = next_item(it, p, ent, gend, item);
    int preg[4] = {-1, -1, -1, -1}, pnext[4] = {-1, -1, -1, -1};
    if (has) page_batch(item, 0, preg);
    uint32_t gb = 0;
    int li = 0;
    bool ok = true;
    while (ok && has) {
        // the next item's first page ids are fetched now, while this one streams
        const bool nhas = next_item(it, p, ent, gend, nitem);
        if (nhas) page_batch(nitem, 0, pnext);
        const int64_t row0 = p.kvl.page_base(p.layer, 0, kv, item.kvh) / HD;  // pool row of (page 0, kv, head, 0)
        int batch = 0;
        auto load_batch = [&](int b) {
            page_batch(item, b, preg);
            batch = b;
        };
        int fallback = __shfl_sync(0xffffffffu, preg[0], 0);
        if (fallback < 0) fallback = 0;
        // Q of this item (q comes from the previous kernel).  The first item's Q
        // is deferred until a block needs that kernel anyway, or the ring is
        // full (the MMAs that free it need Q): cache blocks go out first.
        const int qb = li % NQ;
        bool q_pending = with_q;
        auto issue_q = [&]() -> bool {
            if (!waited) {
                griddep_wait();
                waited = true;
            }
            bool qok = true;
            if (lane == 0) qok = mbar_wait_bounded(smem_u32(&q_empty[qb]), ((li / NQ) & 1) ^ 1, err);
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
        item = nitem;
        has = nhas;
#pragma unroll
        for (int i = 0; i < 4; ++i) preg[i] = pnext[i];
    }
    return ok;
}

// DUAL (valid query rows <= 64): rows 64..127 repeat rows 0..63, and the
// thread of row i + 64 takes keys 32..63 of every block while the thread of
// row i takes keys 0..31, each writing zeros into the other half of its P
// row; each half keeps its own running max and sum, so O rows i and i + 64
// hold the two halves of one result, which the epilogue combines.  This
// halves the per-thread softmax work when a tile has 64 or fewer query rows.
template <bool DUAL>
__global__ void __launch_bounds__(NTHREADS, CTAS_PER_SM) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                                                              const __grid_constant__ CUtensorMap tm_q,
                                                              const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + OFF_Q;  // [NQ] Q buffers
    uint8_t* sK = smem + OFF_K;  // [NK] K blocks
    uint8_t* sV = smem + OFF_V;  // [NV] V blocks
    float* xch = reinterpret_cast<float*>(smem + OFF_X);     // DUAL exchange
    float2* sml = reinterpret_cast<float2*>(smem + OFF_ML);  // [NO][128] (m, l) per row
    int2* ent = reinterpret_cast<int2*>(smem + OFF_ENT);      // [ENT_CAP] (n, S) per entry
    int* gend = reinterpret_cast<int*>(smem + OFF_GRP);       // [2][GRP_CAP] item prefix sums per group
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* q_full = bars;              // [NQ]
    uint64_t* q_empty = q_full + NQ;      // [NQ]
    uint64_t* k_full = q_empty + NQ;      // [NK]
    uint64_t* k_empty = k_full + NK;      // [NK]
    uint64_t* v_full = k_empty + NK;      // [NV]
    uint64_t* v_empty = v_full + NV;      // [NV]
    uint64_t* s_full = v_empty + NV;      // [NSB] S = Q K^T of the buffer's block done
    uint64_t* p_full = s_full + NSB;      // [NSB] its P written (the 4 softmax warps)
    uint64_t* s_free = p_full + NSB;      // [NSB] its P V done: the buffer may take the next S
    uint64_t* o_full = s_free + NSB;      // [NO] an item's last P V into the accumulator done
    uint64_t* o_free = o_full + NO;       // [NO] accumulator read out (the 4 epilogue warps)
    uint64_t* ml_full = o_free + NO;      // [NO] the item's (m, l) written (softmax warps)
    uint64_t* ml_free = ml_full + NO;     // [NO] (m, l) read (epilogue warps)
    uint64_t* drain = ml_free + NO;       // the MMA thread's last MMAs (error exit)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.hq / p.hkv;
    const int qrows = p.rt * g;  // query rows of a tile (<= 64 when DUAL)

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_kv)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
        for (int s = 0; s < NQ; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        for (int s = 0; s < NK; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < NSB; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
            mbar_init(&s_free[s], 1);
        }
        for (int s = 0; s < NO; ++s) {
            mbar_init(&o_full[s], 1);
            mbar_init(&o_free[s], 4);
            mbar_init(&ml_full[s], 4);
            mbar_init(&ml_free[s], 4);
        }
        mbar_init(drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    for (int e = threadIdx.x; e < min(p.n_entries, ENT_CAP); e += NTHREADS) {
        const int slot = p.rm.slot_base + e;
        ent[e] = make_int2(__ldcg(p.rm.n + slot), __ldcg(p.ss.S + slot));
    }
    __syncthreads();
    if (warp == 0 && p.n_entries * p.tiles <= GRP_CAP) {
        // full-chunk and last-chunk items per group, then inclusive prefix sums
        const int G = p.n_entries * p.tiles;
        int carry = 0, carry2 = 0;
        for (int g0 = 0; g0 < G; g0 += 32) {
            int S, n, nsplit, v = 0, v2 = 0;
            if (g0 + lane < G && group_items(p, ent, g0 + lane, S, n, nsplit) > 0) {
                v = p.hkv * (nsplit - 1);
                v2 = p.hkv;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                const int u2 = __shfl_up_sync(0xffffffffu, v2, o);
                if (lane >= o) {
                    v += u;
                    v2 += u2;
                }
            }
            if (g0 + lane < G) {
                gend[g0 + lane] = carry + v;
                gend[GRP_CAP + g0 + lane] = carry2 + v2;
            }
            carry += __shfl_sync(0xffffffffu, v, 31);
            carry2 += __shfl_sync(0xffffffffu, v2, 31);
        }
    }
    if (warp == WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int* err = p.err;
    const float sl2 = 1.4426950408889634f / sqrtf((float)HD);  // log2(e) / sqrt(head_dim)

    if (warp == WARP_KLOAD || warp == WARP_VLOAD) {
        // ---------------------------------------------------------- loaders
        bool waited = false;
        uint32_t issued = 0, q_issued = 0;
        const bool kw = warp == WARP_KLOAD;
        if (kw)
            kv_loader<DUAL>(p, ent, gend, &tm_kv, &tm_q, 0, sK, k_full, k_empty, true, sQ, q_full, q_empty, lane, waited, issued,
                            q_issued);
        else
            kv_loader<DUAL>(p, ent, gend, &tm_kv, &tm_q, 1, sV, v_full, v_empty, false, sQ, q_full, q_empty, lane, waited,
                            issued, q_issued);
        if (!waited) griddep_wait();
        griddep_launch();
        // Copies still in flight (only after an error) must land before the CTA
        // exits: wait, bounded, for the last blocks issued to each stage.
        if (lane == 0) {
            uint64_t* full = kw ? k_full : v_full;
            for (uint32_t j = issued > (uint32_t)NK ? issued - NK : 0u; j < issued; ++j)
                mbar_wait_bounded(smem_u32(&full[j % NK]), (j / NK) & 1, nullptr, 200000000LL);
            for (uint32_t j = q_issued > (uint32_t)NQ ? q_issued - NQ : 0u; j < q_issued; ++j)
                mbar_wait_bounded(smem_u32(&q_full[j % NQ]), (j / NQ) & 1, nullptr, 200000000LL);
        }
    } else if (warp == WARP_MMA) {
        // -------------------------------------------------------------- MMA
        griddep_wait();
        griddep_launch();
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, KBLK);
            constexpr uint32_t idO = idesc_bf16(128, HD) | (1u << 16);  // B (V) MN-major
            // Two cursors over this CTA's blocks (in item order): `sc` issues
            // S = Q K^T into S buffer (block mod NSB) as soon as the block's K,
            // the item's Q and the buffer are there (up to NSB blocks ahead);
            // `pv` issues O += P V once the softmax has written the block's P.
            struct Cursor {
                ItemIter it;
                Item item;
                int li = 0, j = 0;
                uint32_t gb = 0;
                bool valid = false;
            };
            auto start = [&](Cursor& c) {
                c.it.next = blockIdx.x;
                c.valid = next_item(c.it, p, ent, gend, c.item);
            };
            auto advance = [&](Cursor& c) {
                ++c.gb;
                if (++c.j == c.item.nblk) {
                    c.j = 0;
                    ++c.li;
                    c.valid = next_item(c.it, p, ent, gend, c.item);
                }
            };
            // 1: S of c's block may be issued; 0: not yet (probe only); -1: a wait failed.
            auto s_ready = [&](const Cursor& c, bool block) -> int {
                const uint32_t b = c.gb;
                const int qb = c.li % NQ;
                const uint32_t qpar = (c.li / NQ) & 1, fpar = ((b / NSB) & 1) ^ 1, kpar = (b / NK) & 1;
                if (block) {
                    if (c.j == 0 && !mbar_wait_bounded(smem_u32(&q_full[qb]), qpar, err)) return -1;
                    if (b >= (uint32_t)NSB && !mbar_wait_bounded(smem_u32(&s_free[b % NSB]), fpar, err)) return -1;
                    if (!mbar_wait_bounded(smem_u32(&k_full[b % NK]), kpar, err)) return -1;
                    return 1;
                }
                if (c.j == 0 && !mbar_test(&q_full[qb], qpar)) return 0;
                if (b >= (uint32_t)NSB && !mbar_test(&s_free[b % NSB], fpar)) return 0;
                return mbar_test(&k_full[b % NK], kpar) ? 1 : 0;
            };
            auto issue_s = [&](const Cursor& c) {
                const uint32_t b = c.gb;
                const int qb = c.li % NQ;
                tc_fence_after();
                const uint32_t qa = smem_u32(sQ + qb * Q_BYTES);
                const uint32_t kb = smem_u32(sK + (b % NK) * BLK_BYTES);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    mma_ss(tmem + TM_S + (b % NSB) * 64, sdesc(qa + (kk >> 2) * (QROWS * 128) + (kk & 3) * 32),
                           sdesc(kb + (kk >> 2) * HALF_BYTES + (kk & 3) * 32), idS, kk > 0 ? 1u : 0u);
                umma_commit(&k_empty[b % NK]);
                umma_commit(&s_full[b % NSB]);
                if (c.j == c.item.nblk - 1) umma_commit(&q_empty[qb]);
            };
            auto issue_pv = [&](const Cursor& c) -> bool {
                const uint32_t b = c.gb;
                const int sb = b % NSB, ob = c.li % NO;
                if (!mbar_wait_bounded(smem_u32(&p_full[sb]), (b / NSB) & 1, err)) return false;
                if (c.j == 0 && !mbar_wait_bounded(smem_u32(&o_free[ob]), ((c.li / NO) & 1) ^ 1, err)) return false;
                if (!mbar_wait_bounded(smem_u32(&v_full[b % NV]), (b / NV) & 1, err)) return false;
                tc_fence_after();
                const uint32_t vb = smem_u32(sV + (b % NV) * BLK_BYTES);
#pragma unroll
                for (int kk = 0; kk < KBLK / 16; ++kk)
                    mma_ts(tmem + TM_O + ob * 128, tmem + TM_S + sb * 64 + kk * 8, sdesc_mn(vb + kk * 2048), idO,
                           (c.j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&v_empty[b % NV]);
                umma_commit(&s_free[sb]);
                if (c.j == c.item.nblk - 1) umma_commit(&o_full[ob]);
                return true;
            };
            Cursor sc, pv;
            start(sc);
            start(pv);
            bool ok = true;
            while (pv.valid && ok) {
                // the softmax needs S of pv's block: issue up to it, waiting if need be
                while (sc.valid && sc.gb <= pv.gb) {
                    const int r = s_ready(sc, true);
                    if (r < 0) {
                        ok = false;
                        break;
                    }
                    issue_s(sc);
                    advance(sc);
                }
                if (!ok) break;
                // further S blocks whose inputs are already there
                while (sc.valid && sc.gb < pv.gb + NSB && s_ready(sc, false) > 0) {
                    issue_s(sc);
                    advance(sc);
                }
                if (!(ok = issue_pv(pv))) break;
                advance(pv);
            }
            // every MMA issued has completed before TMEM may be released
            umma_commit(drain);
            mbar_wait_bounded(smem_u32(drain), 0, nullptr, 200000000LL);
        }
    } else if (warp < WARP_EPI) {
        // ---------------------------------------------------------- softmax
        griddep_wait();
        griddep_launch();
        const int tid = threadIdx.x;                // TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int qi = DUAL ? (tid & 63) : tid;     // query row this thread works for
        const int half = DUAL ? (tid >> 6) : 0;     // DUAL: key half of every block
        const float thr = kRescaleLog2 / sl2;       // rescale threshold in raw score units
        ItemIter it;
        it.next = blockIdx.x;
        Item item;
        uint32_t gb = 0;
        int li = 0;
        bool ok = true;
        while (ok && next_item(it, p, ent, gend, item)) {
            const int ob = li % NO;
            const int rr = item.r0 + qi / g;
            const bool qok = qi < qrows && rr < item.n;
            const int lim = item.S + (qok ? rr : item.r_last);  // last visible key
            const int kfree = min(item.ke, item.S);             // keys below: visible to every row
            // running max (raw scores) and sum of this thread's keys; in DUAL
            // mode each key half keeps its own and the epilogue merges them
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < item.nblk && ok; ++j, ++gb) {
                const int sb = gb % NSB;
                const uint32_t tS = tmem + lane_base + TM_S + sb * 64;
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&s_full[sb]), (gb / NSB) & 1, err));
                if (!ok) break;
                tc_fence_after();
                uint32_t r[32];
                const int kb0 = item.ks + j * KBLK + half * 32;
                // the block reaches the window or the chunk end: mask by key position
                const bool edge = item.ks + (j + 1) * KBLK > kfree;
                // scores of columns [c0, c0 + 32) of this thread's block, masked
                auto load_scores = [&](int c0, float (&sv)[32]) {
                    tmem_ld32(tS + c0, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) sv[c] = __uint_as_float(r[c]);
                    if (edge) {
                        const int t0 = kb0 + (DUAL ? 0 : c0);
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (!(t0 + c < item.ke && t0 + c <= lim)) sv[c] = -INFINITY;
                    }
                };
                float sv[32];
                float bmax = -INFINITY;
                load_scores(DUAL ? half * 32 : 0, sv);
#pragma unroll
                for (int c = 0; c < 32; ++c) bmax = fmaxf(bmax, sv[c]);
                if (!DUAL) {
                    // the second half's max first; its scores are loaded again below
                    float sv2[32];
                    load_scores(32, sv2);
#pragma unroll
                    for (int c = 0; c < 32; ++c) bmax = fmaxf(bmax, sv2[c]);
                }
                const bool need = bmax > m + thr;
                if (j > 0 && __any_sync(0xffffffffu, need)) {
                    // P V of the previous block must be done before O is rescaled
                    const uint32_t pb = gb - 1;
                    ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&s_free[pb % NSB]), (pb / NSB) & 1, err));
                    if (!ok) break;
                    tc_fence_after();
                    const float f = need ? fast_exp2((m - bmax) * sl2) : 1.0f;
                    const uint32_t tO = tmem + lane_base + TM_O + ob * 128;
#pragma unroll 1
                    for (int c = 0; c < HD; c += 32) {
                        tmem_ld32(tO + c, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * f);
                        tmem_st32(tO + c, r);
                    }
                    l *= f;
                }
                if (need) m = bmax;
                const float neg = (m == -INFINITY) ? 0.f : -m * sl2;
                float psum = 0.f;
                uint32_t pk[32];
                if constexpr (DUAL) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float a = fast_exp2(fmaf(sv[2 * c], sl2, neg));
                        const float bb = fast_exp2(fmaf(sv[2 * c + 1], sl2, neg));
                        psum += a + bb;
                        const uint32_t v = pack_bf16(a, bb);
                        pk[c] = half ? 0u : v;
                        pk[16 + c] = half ? v : 0u;
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float a = fast_exp2(fmaf(sv[2 * c], sl2, neg));
                        const float bb = fast_exp2(fmaf(sv[2 * c + 1], sl2, neg));
                        psum += a + bb;
                        pk[c] = pack_bf16(a, bb);
                    }
                    load_scores(32, sv);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float a = fast_exp2(fmaf(sv[2 * c], sl2, neg));
                        const float bb = fast_exp2(fmaf(sv[2 * c + 1], sl2, neg));
                        psum += a + bb;
                        pk[16 + c] = pack_bf16(a, bb);
                    }
                }
                l += psum;
                tmem_st32(tS, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sb]);
            }
            if (!ok) break;
            // (m, l) of this item to the epilogue warps, m in the exp2 domain
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&ml_free[ob]), ((li / NO) & 1) ^ 1, err));
            if (!ok) break;
            sml[ob * QROWS + tid] = make_float2(m == -INFINITY ? -INFINITY : m * sl2, l);
            __syncwarp();
            if (lane == 0) mbar_arrive(&ml_full[ob]);
            ++li;
        }
    } else if (warp < WARP_MMA) {
        // --------------------------------------------------------- epilogue
        griddep_wait();
        griddep_launch();
        const int e = threadIdx.x - WARP_EPI * 32;  // TMEM lane
        const uint32_t lane_base = (uint32_t)((warp - WARP_EPI) * 32) << 16;
        const int qi = DUAL ? (e & 63) : e;
        const int half = DUAL ? (e >> 6) : 0;
        ItemIter it;
        it.next = blockIdx.x;
        Item item;
        int li = 0;
        bool ok = true;
        while (ok && next_item(it, p, ent, gend, item)) {
            const int ob = li % NO;
            const int rr = item.r0 + qi / g;
            const bool qok = qi < qrows && rr < item.n;
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&ml_full[ob]), (li / NO) & 1, err));
            float2 own = make_float2(-INFINITY, 0.f), oth = own;
            if (ok) {
                own = sml[ob * QROWS + e];
                if (DUAL) oth = sml[ob * QROWS + (e ^ 64)];
                __syncwarp();
                if (lane == 0) mbar_arrive(&ml_free[ob]);
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&o_full[ob]), (li / NO) & 1, err));
            }
            if (DUAL) ok = epi_all(ok);
            if (!ok) break;
            tc_fence_after();
            // DUAL: the two key halves of row qi (rows qi and qi + 64 of O) merge:
            // O = 2^(m0 - M) O0 + 2^(m1 - M) O1, l likewise, M = max(m0, m1)
            float m = own.x, l = own.y, a_own = 1.f, a_other = 0.f;
            if (DUAL) {
                const float M = fmaxf(own.x, oth.x);
                a_own = M == -INFINITY ? 0.f : fast_exp2(own.x - M);
                a_other = M == -INFINITY ? 0.f : fast_exp2(oth.x - M);
                l = a_own * own.y + a_other * oth.y;
                m = M;
            }
            const int qrow = item.entry * p.stride + (qok ? rr : item.r_last);
            const int qhead = item.kvh * g + qi % g;
            const int64_t pbase = ((int64_t)qrow * p.hq + qhead) * p.max_splits;
            const uint32_t tO = tmem + lane_base + TM_O + ob * 128;
            const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll 1
            for (int c = 0; c < HD; c += 32) {
                uint32_t r[32];
                tmem_ld32(tO + c, r);
                tmem_wait_ld();
                if (DUAL) {
                    // the other key half of row qi, through shared memory
                    epi_sync();
                    if (half) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) xch[x * 64 + qi] = __uint_as_float(r[x]);
                    }
                    epi_sync();
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
            // O is read out: the MMA may accumulate a later item into it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[ob]);
            if (qok && item.nsplit > 1 && !(DUAL && half)) p.part_ml[pbase + item.sp] = make_float2(m, l);
            ++li;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TM_COLS) : "memory");
    }
}

// Combine the key chunks of every (row, query head) whose row tile was split:
// O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s.  One warp
// per (row, head), a lane per 4 dims; lane s holds chunk s's (m, l), and all
// of a pair's chunk partials are in flight together.  Rows whose tile had one
// chunk were written by the attention kernel itself and are left alone.
struct MergeParams {
    const float* part_o;
    const float2* part_ml;
    bf16* out;
    int n_entries, stride, hq, rt, kv_chunk, max_splits;
    SlotState ss;
    RowMap rm;
};

__global__ void __launch_bounds__(256) attn_merge_kernel(const MergeParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t pair = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const bool have = pair < (int64_t)p.n_entries * p.stride * p.hq;
    const int row = have ? (int)(pair / p.hq) : 0, h = have ? (int)(pair % p.hq) : 0;
    const int e = row / p.stride, r = row - e * p.stride;
    const int slot = p.rm.slot_base + e;
    // n and S are not written by the attention kernel: read before the wait
    const int n = have ? __ldcg(p.rm.n + slot) : 0;
    const int S = have ? __ldcg(p.ss.S + slot) : 0;
    griddep_wait();
    griddep_launch();
    if (!have || r >= n) return;
    const int nsplit = tile_splits(S, n, r / p.rt, p.rt, p.kv_chunk);
    if (nsplit <= 1 || nsplit > p.max_splits) return;
    const int64_t pb = ((int64_t)row * p.hq + h) * p.max_splits;
    // the (m, l) of every chunk and the first 8 chunk outputs, all in flight
    const float2 ml = lane < nsplit ? __ldcg(p.part_ml + pb + lane) : make_float2(-INFINITY, 0.f);
    const float4* po = reinterpret_cast<const float4*>(p.part_o + pb * HD) + lane;
    float4 v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = q < nsplit ? __ldcg(po + (int64_t)q * (HD / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float M = warp_max(ml.x);
    const float w = (ml.x == -INFINITY || M == -INFINITY) ? 0.f : fast_exp2(ml.x - M);
    const float L = warp_sum(w * ml.y);
    const float wl = L > 0.f ? w / L : 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int s0 = 0; s0 < nsplit; s0 += 8) {
        if (s0 > 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                v[q] = s0 + q < nsplit ? __ldcg(po + (int64_t)(s0 + q) * (HD / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float wq = __shfl_sync(0xffffffffu, wl, (s0 + q) & 31);
            acc.x += wq * v[q].x;
            acc.y += wq * v[q].y;
            acc.z += wq * v[q].z;
            acc.w += wq * v[q].w;
        }
    }
    uint2 o2;
    o2.x = pack_bf16(acc.x, acc.y);
    o2.y = pack_bf16(acc.z, acc.w);
    *reinterpret_cast<uint2*>(p.out + ((int64_t)row * p.hq + h) * HD + lane * 4) = o2;
}

}  // namespace

int attn_rows_per_tile(int group) { return QROWS / group; }
int attn_dual_rows_per_tile(int group) { return 64 / group; }
int attn_max_splits() { return MAX_SPLITS; }

int attn_kv_chunk_for(int max_batch, int max_window, int hq, int hkv, int max_ctx, int num_sms) {
    // Fixed per context (a sequence's result does not depend on its batch
    // neighbours): a full batch at half the context length makes about one
    // item per CTA (two CTAs per SM; every further item of a CTA waits for its
    // Q to load, the CTA's one Q buffer being busy until the item before has
    // issued its last S); at least four 64-key blocks per chunk, at most 32
    // blocks, and at most attn_max_splits() chunks per row tile.
    const int g = hq / hkv;
    const int rt = attn_rows_per_tile(g);
    const long long tiles = (max_window + rt - 1) / rt;
    const long long pairs = (long long)max_batch * tiles * hkv;
    const long long blocks = pairs * std::max(1, (max_ctx / 2 + 63) / 64);
    const long long ctas = (long long)CTAS_PER_SM * num_sms;
    long long cb = (blocks + ctas - 1) / ctas;
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
                             int n_entries, int stride, int kv_chunk, int max_splits, SlotState ss, RowMap rm,
                             int* err, cudaStream_t st) {
    if (hq % hkv || hq / hkv > QROWS || max_splits < 1 || max_splits > MAX_SPLITS || kv_chunk < KBLK ||
        kv_chunk % KBLK || n_entries < 1 || stride < 1 || (max_splits > 1 && (!part_o || !part_ml)))
        return cudaErrorInvalidValue;
    const int g = hq / hkv;
    // DUAL when every query row of a window fits in 64 (one tile of 64 / g rows)
    const bool dual = stride * g <= 64;
    const int rt = dual ? attn_dual_rows_per_tile(g) : attn_rows_per_tile(g);
    const int tiles = (stride + rt - 1) / rt;
    AttnParams p{kvl, layer, hq, hkv, out, part_o, part_ml, n_entries, stride, kv_chunk, max_splits, rt, tiles,
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
    cudaError_t e = dual ? launch_pdl(attn_tc_kernel<true>, dim3(grid), dim3(NTHREADS), SMEM_BYTES, st, tm_kv,
                                      tm_q_dual, p)
                         : launch_pdl(attn_tc_kernel<false>, dim3(grid), dim3(NTHREADS), SMEM_BYTES, st, tm_kv, tm_q, p);
    if (e != cudaSuccess || max_splits == 1) return e;
    MergeParams mp{part_o, part_ml, out, n_entries, stride, hq, rt, kv_chunk, max_splits, ss, rm};
    const long long pairs = (long long)n_entries * stride * hq;
    return launch_pdl(attn_merge_kernel, dim3((unsigned)((pairs + 7) / 8)), dim3(256), 0, st, mp);
}

}  // namespace wedlm

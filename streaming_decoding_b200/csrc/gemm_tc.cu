// Persistent bf16 GEMM on tcgen05 tensor cores, TMA-fed, with fused epilogues.
//
// Y[M][N] = X[M][K] * W[N][K]^T for every dense projection of the step (QKV,
// O, gate/up, down) and the LM head.  In decoding M (window rows of the
// batch) is small, so the layout is "swap-AB": the 128-row MMA M side holds
// weight rows, the MMA N side (bn = 16..256) holds activation rows.  Every
// weight byte is read from HBM exactly once per launch; the kernel is bound by
// weight bytes until M nears the machine-balance point (~250 rows).
//
// One CTA per SM loops over work units (tile, K slice).  Warp roles (192
// threads):
//   warp 0      one thread issues TMA loads of A (weights, 128*wt x bk) and B
//               (activations, bn x bk) into a STAGES-deep shared-memory ring
//               that runs continuously across units,
//   warp 1      allocates TMEM (accumulators of wt*bn columns, two when they
//               fit) and one thread issues tcgen05.mma (kind::f16, fp32
//               accumulation), releasing ring stages with tcgen05.commit; with
//               two accumulators the next unit's MMAs overlap the previous
//               unit's epilogue,
//   warps 2..5  epilogue (warp w owns TMEM lanes 32*(w%4)..+31): 32 accumulator
//               columns at a time are loaded (tcgen05.ld), stored transposed to
//               shared memory and finished as float4 runs of weight rows for 8
//               activation rows each (coalesced rows, vector stores; the loads
//               the fused epilogue needs besides the accumulator are issued
//               first); the accumulator is released to the MMA thread right
//               after its last load.  With K split over several units each
//               slice writes its fp32 partial plane the same way and takes a
//               ticket; either the slices of a tile (co-resident by cooperative
//               launch) wait for each other and each reduces a share of the
//               rows, or the slice that finishes last reduces the tile alone
//               and nobody waits; both sum in fixed split order.  A hybrid
//               schedule splits only the tiles of the last partial round.
// CTA pairs (CG = 2, clusters of two): the pair computes a 256-row weight tile
// with tcgen05.mma.cta_group::2 issued by the even CTA.  Each CTA stages its own
// 128 weight rows and half of the activation rows; the MMA reads the operands
// from both CTAs' shared memory and writes each CTA's 128 accumulator lanes in
// its own TMEM.  A CTA stages 32 KB per 64-deep k-block for 128 x 256 outputs
// (a single-CTA 128 x 256 tile stages 48 KB): two thirds of the operand bytes
// streamed from L2 into the SMs per output (half those of 128 x 128 tiles), and
// room for a 6-stage ring.
// Loads of both CTAs complete on the even CTA's ring barrier; its commits
// release the ring stage and hand over the accumulator in both CTAs; both CTAs'
// epilogues release the accumulator on the even CTA's barrier.
// Every mbarrier wait is bounded; on timeout the kernel records an error in
// the device error word and unwinds (freeing TMEM) instead of hanging.
#include <algorithm>
#include <cmath>

#include <cudaTypedefs.h>

#include "gemm_tc.cuh"

namespace wedlm {
namespace {

constexpr int BM = 128;
constexpr int BK_DEFAULT = 64;  // k-block depth of the 128-byte-swizzle tiles

// BN activation rows (MMA N) by WT weight sub-tiles of 128 rows (one MMA each
// per k-step, sharing the activation operand: WT = 2 halves the activation
// bytes a CTA moves per output).  NACC accumulators of WT*BN TMEM columns
// (two when they fit, so a unit's MMAs overlap the previous unit's epilogue).
// BK = 64 (128-byte rows, 128-byte swizzle) or 32 (64-byte rows, 64-byte
// swizzle: half the bytes per stage, so twice the stages in flight).
// CG = 2: CTA pair, BN activation rows per pair (BN / 2 staged by each CTA).
template <int BN, int WT, int BK, int CG> struct PCfg {
    static_assert(CG == 1 || (CG == 2 && WT == 1 && BK == 64 && BN >= 64), "pair tiles: one weight sub-tile per CTA");
    static constexpr int SUB_A_BYTES = BM * BK * 2;  // one 128-row weight sub-tile of a stage
    static constexpr int A_STAGE_BYTES = WT * SUB_A_BYTES;
    static constexpr int B_ROWS = BN / CG;  // activation rows this CTA stages
    static constexpr int B_STAGE_BYTES = B_ROWS * BK * 2;
    static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
    static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 12 ? 12 : (200 * 1024) / STAGE_BYTES;
    static constexpr int ACC_COLS = WT * BN;
    static constexpr int NACC = 2 * ACC_COLS <= 512 ? 2 : 1;
    static constexpr int TMEM_COLS = NACC * ACC_COLS < 32 ? 32 : NACC * ACC_COLS;
    static constexpr int META_BYTES = BN * 16;  // per activation row: live, pos, cache-row offset
    // epilogue staging: 32 accumulator columns (activation rows) x 128 weight rows, fp32
    static constexpr int EPI_COLS = 32;
    static constexpr int EPI_BYTES = BN >= EPI_COLS ? EPI_COLS * BM * 4 : 0;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ + META_BYTES + EPI_BYTES;
};

// What the epilogue needs per activation row of the current unit, computed
// once per unit into shared memory so the element loops issue their global
// loads in batches (no load waits behind a store of the previous element).
struct RowMeta {
    int live;      // row < M (and < the device row count) and not padding
    int pos;       // logical position (RoPE); with a row map, the row the result goes to
    long long kv;  // element offset of (layer, page, K, head 0, token) in the pool; -1 if out of range
};

struct GemmArgs {
    int M, N, K, kb_per_split, splits, n_tiles, m_tiles;
    int coop;        // split fixup: 1 distributed (cooperative launch), 0 last arriver
    int full_tiles;  // tiles [0, full_tiles) run whole-K as one unit each; the rest in `splits` K slices
    int ks;          // > 1: the `splits` slices of a tile are the CTAs of one cluster (one unit per CTA),
                     // reduced through distributed shared memory
    EpiParams ep;
};

// One work unit: a tile (n-major over m tiles) and a K slice of it.
struct Unit {
    int tile, split, nsplit, kb0, nkb;
};
__device__ __forceinline__ Unit unit_of(const GemmArgs& g, int u, int KB) {
    Unit r;
    if (u < g.full_tiles) {
        r.tile = u;
        r.split = 0;
        r.nsplit = 1;
        r.kb0 = 0;
        r.nkb = KB;
    } else {
        const int v = u - g.full_tiles;
        r.tile = g.full_tiles + v / g.splits;
        r.split = v % g.splits;
        r.nsplit = g.splits;
        r.kb0 = r.split * g.kb_per_split;
        r.nkb = min(KB, r.kb0 + g.kb_per_split) - r.kb0;
    }
    return r;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- CTA-pair (cluster of two) primitives
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Address of the same shared-memory object in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t mapa_rank(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
// Barrier over every thread of both CTAs (each CTA's threads all reach it).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// TMA load into this CTA's shared memory that completes on an mbarrier of
// either CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait with cluster-scope acquire (arrivals from the peer CTA).
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity, int* err) {
    const long long t0 = clock64();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((it & 1023u) == 1023u) {
            if (stalled(err)) return false;
            if (clock64() - t0 > 2000000000LL) {
                set_error(err, kErrTimeout);
                return false;
            }
        }
    }
}

// Shared-memory matrix descriptor of a K-major tile of BK-element rows stored
// with the matching swizzle: BK = 64 -> 128-byte rows, 128-byte swizzle, 8-row
// atoms 1024 B apart; BK = 32 -> 64-byte rows, 64-byte swizzle, atoms 512 B apart.
template <int BK>
__device__ __forceinline__ uint64_t sdesc_k(const void* p) {
    static_assert(BK == 64 || BK == 32, "k-block depth");
    const uint32_t a = smem_u32(p);
    uint64_t d = (uint64_t)((a >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                      // leading-dimension byte offset (unused with swizzle)
    d |= (uint64_t)((8 * BK * 2) >> 4) << 32;    // stride byte offset between 8-row atoms
    d |= (uint64_t)1 << 46;                      // descriptor version for tcgen05
    d |= (uint64_t)(BK == 64 ? 2 : 4) << 61;     // 128-byte or 64-byte swizzle
    return d;
}

// Instruction descriptor: dense kind::f16, D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

template <int CG>
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (CG == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
            ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
            : "memory");
}

// Arrive on `bar` once the MMAs issued so far complete; a pair arrives on the
// barrier at the same offset in both CTAs (one commit per CTA, by cluster address).
template <int CG>
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    if constexpr (CG == 2) {
#pragma unroll
        for (uint32_t r = 0; r < 2; ++r)
            asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         ::"r"(mapa_rank(smem_u32(bar), r))
                         : "memory");
    } else
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                     : "memory");
}

// 32 consecutive fp32 accumulator columns of this warp's 32 TMEM lanes (one
// load and its wait in one statement, so no use is scheduled before the wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive fp32 accumulator columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier over the four epilogue warps that also ANDs a predicate across them,
// so they leave the unit loop together (every wait before it is bounded).
__device__ __forceinline__ bool epi_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}

// Fill meta[0..BN) for activation rows m0..m0+BN-1 (the 128 epilogue threads).
// Live activation rows of a launch: M, or fewer when the rows are counted on
// the device (read after the dependency wait: the previous kernel writes it).
__device__ __forceinline__ int live_rows(const EpiParams& ep, int M) {
    return ep.m_count ? min(M, __ldcg(ep.m_count)) : M;
}

template <int BN>
__device__ __forceinline__ void fill_row_meta(const EpiParams& ep, int m0, int M, RowMeta* meta, int et) {
    const int Ml = live_rows(ep, M);
    for (int k = et; k < BN; k += 128) {
        const int m = m0 + k;
        RowMeta rmeta{0, 0, -1};
        int slot = 0, r = m;
        if (m < Ml && (!ep.check_rows || ep.rm.live(m, slot, r))) {
            rmeta.live = 1;
            if (ep.row_map) rmeta.pos = __ldcg(ep.row_map + m);
            if (ep.kind == EPI_QKV_ROPE) {
                const int pos = __ldcg(ep.rs.pos + m);
                if (pos < 0 || pos >= ep.rope_max_pos) {
                    set_error(ep.err, kErrBounds);
                    rmeta.live = 0;
                } else {
                    rmeta.pos = pos;
                    const int p = __ldcg(ep.ss.S + slot) + r;
                    const int pidx = p / kPage;
                    const int page = pidx < ep.ss.pages_per_seq
                                         ? __ldcg(ep.ss.page_table + (int64_t)slot * ep.ss.pages_per_seq + pidx)
                                         : -1;
                    if (page < 0 || page >= ep.kvl.num_pages) {
                        set_error(ep.err, kErrBounds);
                    } else {
                        rmeta.kv = ep.kvl.page_base(ep.layer, page, 0, 0) + (int64_t)(p % kPage) * 128;
                    }
                }
            }
        }
        meta[k] = rmeta;
    }
}

// silu(x) * y for the gate/up pair, with the exponential and the division on
// the special-function unit (no branch: independent elements interleave); its
// error, about 1e-6 relative, is far below the bf16 rounding of the result.
__device__ __forceinline__ float silu_mul(float x, float y) { return __fdividef(x, 1.0f + __expf(-x)) * y; }

// Destination row of QKV head `head` for activation row m: the q buffer, or the
// row's K or V page entry (kv: the row's cache offset, -1 if it has none).
// Every argument is a register value: the epilogues read all parameters and row
// metadata before their first global store, since after a store through a
// generic pointer the compiler would have to reload anything it cannot prove
// unaliased, which serialises the element loop on load latency.
__device__ __forceinline__ bf16* qkv_dst(bf16* act, bf16* pool, int hq, int hkv, int head, int m, long long kv) {
    if (head < hq) return act + ((int64_t)m * hq + head) * 128;
    if (kv < 0) return nullptr;
    const int sel = head < hq + hkv ? 0 : 1;
    const int h = head - hq - sel * hkv;
    return pool + kv + (int64_t)(sel * hkv + h) * (kPage * 128);
}

// Fused epilogue on 16 accumulator columns (activation rows mbase..mbase+15,
// meta rows kbase..kbase+15) of weight row n held by this thread; row pairs
// (n even, n odd) sit in adjacent lanes.
__device__ __forceinline__ void epilogue16(const EpiParams& ep, int n0, int n, int mbase, int kbase,
                                           const RowMeta* meta, const float (&v)[16], int N, int lane) {
    const int kind = ep.kind;
    float* const out = ep.out;
    bf16* const act = ep.act;
    bool live[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) live[k] = meta[kbase + k].live && n < N;
    switch (kind) {
        case EPI_STORE:
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (live[k]) out[(int64_t)(ep.row_map ? meta[kbase + k].pos : mbase + k) * N + n] = v[k];
            break;
        case EPI_RESIDUAL: {
            float x[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) x[k] = live[k] ? out[(int64_t)(mbase + k) * N + n] : 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (live[k]) out[(int64_t)(mbase + k) * N + n] = x[k] + v[k];
            break;
        }
        case EPI_SWIGLU: {
            const int F = N >> 1;
            bf16 r[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float partner = __shfl_xor_sync(0xffffffffu, v[k], 1);
                r[k] = __float2bfloat16_rn(silu_mul(v[k], partner));
            }
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (!(lane & 1) && live[k]) act[(int64_t)(mbase + k) * F + (n >> 1)] = r[k];
            break;
        }
        case EPI_QKV_ROPE: {
            bf16* const pool = ep.kv_pool;
            const float2* const rope = ep.rope_cs;
            const int hq = ep.hq, hkv = ep.hkv;
            const int head = n0 >> 7;
            const int t = n - n0;
            const bool rot = head < hq + hkv;
            const int i = t >> 1, odd = t & 1;
            const int dim = rot ? (odd ? i + 64 : i) : t;
            float2 cs[16];
            bf16* dst[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const RowMeta rmk = meta[kbase + k];
                cs[k] = (rot && live[k]) ? __ldcg(rope + (int64_t)rmk.pos * 64 + i) : make_float2(1.f, 0.f);
                dst[k] = live[k] ? qkv_dst(act, pool, hq, hkv, head, mbase + k, rmk.kv) : nullptr;
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float partner = rot ? __shfl_xor_sync(0xffffffffu, v[k], 1) : 0.f;
                float val = v[k];
                if (rot) {
                    const float a = odd ? partner : val, b = odd ? val : partner;
                    val = odd ? (b * cs[k].x + a * cs[k].y) : (a * cs[k].x - b * cs[k].y);
                }
                if (dst[k]) dst[k][dim] = __float2bfloat16_rn(val);
            }
            break;
        }
        default: break;
    }
}

// LM-head epilogue without logits (EPI_ENTROPY): for each of 16 activation
// rows, this warp's 32 vocab ids (one per lane, id n) reduce to the partial
// (max, sum e^(z-max), sum e^(z-max)(z-max), lowest argmax) of z = scale * v
// over valid ids (n < N, n != mask id); lane k stores row k's partial.
__device__ __forceinline__ void entropy16(const EpiParams& ep, const float (&v)[16], bool valid, int n, int kbase,
                                          const RowMeta* meta, int m0, int pidx, int lane) {
    const float scale = ep.scale;
    float4* const epart = ep.epart;
    const int npart = ep.npart;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float z = valid ? v[k] * scale : -INFINITY;
        float m = z;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float e = 0.f, t = 0.f;
        if (valid && m != -INFINITY) {
            e = expf(z - m);
            t = e * (z - m);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            e += __shfl_xor_sync(0xffffffffu, e, o);
            t += __shfl_xor_sync(0xffffffffu, t, o);
        }
        int a = (valid && z == m) ? n : INT_MAX;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
        const RowMeta rk = meta[kbase + k];
        const int row = ep.row_map ? rk.pos : m0 + kbase + k;
        if (lane == k && rk.live) epart[(int64_t)row * npart + pidx] = make_float4(m, e, t, __int_as_float(a));
    }
}

// Fused epilogue on weight rows n..n+3 (both row pairs inside this thread) of
// eight activation rows m = mrow[u] (meta rows krow[u]), in two phases: epi_pre
// issues every load that does not depend on the accumulator (row metadata, the
// residual stream, RoPE cos/sin, destination rows) so its latency overlaps the
// staging of the accumulator; epi_fin does the arithmetic and the vector stores.
// All parameter reads precede the first store (see qkv_dst).
struct EpiPre {
    bool live[8];
    float4 x[8];          // EPI_RESIDUAL: residual stream values
    float2 c0[8], c1[8];  // EPI_QKV_ROPE: (cos, sin) of dims (i, i + 64) and (i + 1, i + 65)
    bf16* dst[8];         // EPI_QKV_ROPE: destination rows
};

template <int KIND>
__device__ __forceinline__ void epi_pre(const EpiParams& ep, int n0, int n, const int (&mrow)[8], const int (&krow)[8],
                                        const bool (&ok)[8], const RowMeta* meta, int N, EpiPre& p) {
#pragma unroll
    for (int u = 0; u < 8; ++u) p.live[u] = ok[u] && meta[krow[u]].live;
    if constexpr (KIND == EPI_RESIDUAL) {
        const float* out = ep.out;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            p.x[u] = p.live[u] ? *reinterpret_cast<const float4*>(out + (int64_t)mrow[u] * N + n)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if constexpr (KIND == EPI_QKV_ROPE) {
        bf16* const act = ep.act;
        bf16* const pool = ep.kv_pool;
        const float2* const rope = ep.rope_cs;
        const int hq = ep.hq, hkv = ep.hkv;
        const int head = n0 >> 7;
        const bool rot = head < hq + hkv;
        const int i = (n - n0) >> 1;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const RowMeta rmu = meta[krow[u]];
            const int64_t base = (int64_t)rmu.pos * 64 + i;
            p.c0[u] = (rot && p.live[u]) ? __ldcg(rope + base) : make_float2(1.f, 0.f);
            p.c1[u] = (rot && p.live[u]) ? __ldcg(rope + base + 1) : make_float2(1.f, 0.f);
            p.dst[u] = p.live[u] ? qkv_dst(act, pool, hq, hkv, head, mrow[u], rmu.kv) : nullptr;
        }
    }
}

template <int KIND>
__device__ __forceinline__ void epi_fin(const EpiParams& ep, int n0, int n, const int (&mrow)[8], const float4 (&v)[8],
                                        const EpiPre& p, int N) {
    if constexpr (KIND == EPI_STORE) {
        float* const out = ep.out;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (p.live[u]) *reinterpret_cast<float4*>(out + (int64_t)mrow[u] * N + n) = v[u];
    } else if constexpr (KIND == EPI_RESIDUAL) {
        float* const out = ep.out;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (p.live[u])
                *reinterpret_cast<float4*>(out + (int64_t)mrow[u] * N + n) =
                    make_float4(p.x[u].x + v[u].x, p.x[u].y + v[u].y, p.x[u].z + v[u].z, p.x[u].w + v[u].w);
    } else if constexpr (KIND == EPI_SWIGLU) {
        bf16* const act = ep.act;
        const int F = N >> 1;
        __nv_bfloat162 r[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = __floats2bfloat162_rn(silu_mul(v[u].x, v[u].y), silu_mul(v[u].z, v[u].w));
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (p.live[u]) *reinterpret_cast<__nv_bfloat162*>(act + (int64_t)mrow[u] * F + (n >> 1)) = r[u];
    } else if constexpr (KIND == EPI_QKV_ROPE) {
        const int head = n0 >> 7;
        const int t = n - n0;
        const bool rot = head < ep.hq + ep.hkv;
        const int i = t >> 1;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            bf16* const d = p.dst[u];
            if (!d) continue;
            if (rot) {
                // rows (t, t+1) = dims (i, i+64); rows (t+2, t+3) = dims (i+1, i+65)
                const float d0 = v[u].x * p.c0[u].x - v[u].y * p.c0[u].y;
                const float d2 = v[u].y * p.c0[u].x + v[u].x * p.c0[u].y;
                const float d1 = v[u].z * p.c1[u].x - v[u].w * p.c1[u].y;
                const float d3 = v[u].w * p.c1[u].x + v[u].z * p.c1[u].y;
                *reinterpret_cast<__nv_bfloat162*>(d + i) = __floats2bfloat162_rn(d0, d1);
                *reinterpret_cast<__nv_bfloat162*>(d + i + 64) = __floats2bfloat162_rn(d2, d3);
            } else {
                *reinterpret_cast<__nv_bfloat162*>(d + t) = __floats2bfloat162_rn(v[u].x, v[u].y);
                *reinterpret_cast<__nv_bfloat162*>(d + t + 2) = __floats2bfloat162_rn(v[u].z, v[u].w);
            }
        }
    }
}

// Both phases back to back, dispatched on the epilogue kind at run time.
__device__ __forceinline__ void epilogue_vec4x8(const EpiParams& ep, int n0, int n, const int (&mrow)[8],
                                                const int (&krow)[8], const bool (&ok)[8], const RowMeta* meta,
                                                const float4 (&v)[8], int N) {
    EpiPre p;
    switch (ep.kind) {
        case EPI_STORE:
            epi_pre<EPI_STORE>(ep, n0, n, mrow, krow, ok, meta, N, p);
            epi_fin<EPI_STORE>(ep, n0, n, mrow, v, p, N);
            break;
        case EPI_RESIDUAL:
            epi_pre<EPI_RESIDUAL>(ep, n0, n, mrow, krow, ok, meta, N, p);
            epi_fin<EPI_RESIDUAL>(ep, n0, n, mrow, v, p, N);
            break;
        case EPI_SWIGLU:
            epi_pre<EPI_SWIGLU>(ep, n0, n, mrow, krow, ok, meta, N, p);
            epi_fin<EPI_SWIGLU>(ep, n0, n, mrow, v, p, N);
            break;
        case EPI_QKV_ROPE:
            epi_pre<EPI_QKV_ROPE>(ep, n0, n, mrow, krow, ok, meta, N, p);
            epi_fin<EPI_QKV_ROPE>(ep, n0, n, mrow, v, p, N);
            break;
        default: break;
    }
}

// Single-slice epilogue through shared memory, for one epilogue kind: 32
// accumulator columns (activation rows) at a time are stored transposed to
// `stage` (row = activation row, 128 weight rows; each store instruction writes
// 32 consecutive words), then each thread finishes float4 runs of weight rows
// for 8 activation rows: coalesced rows and vector stores.  `release` is called
// once, right after the last accumulator load.
template <int KIND, int BN, int WT, typename Release>
__device__ __forceinline__ void staged_epilogue(const EpiParams& ep, int M, int N, int n0, int m0, uint32_t tacc,
                                                float* stage, const RowMeta* meta, int q, int lane,
                                                Release release) {
    constexpr int COLS = 32;
    const int c4 = 4 * lane;
#pragma unroll 1
    for (int w = 0; w < WT; ++w) {
        const int nw = n0 + w * BM, nn = nw + c4;
        const bool nok = nn < N;
#pragma unroll 1
        for (int c = 0; c < BN; c += COLS) {
            int mrow[8], krow[8];
            bool okr[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int rl = q + 4 * u;  // row within the staged columns
                krow[u] = c + rl;
                mrow[u] = m0 + c + rl;
                okr[u] = nok && mrow[u] < M;
                if (KIND == EPI_STORE && ep.row_map && okr[u] && meta[krow[u]].live) mrow[u] = meta[krow[u]].pos;
            }
            EpiPre p;
            epi_pre<KIND>(ep, nw, nn, mrow, krow, okr, meta, N, p);
            {
                float v[COLS];
                tmem_ld32(tacc + (uint32_t)(w * BN + c), v);
                if (w == WT - 1 && c + COLS >= BN) release();
                float* srow = stage + q * 32 + lane;
#pragma unroll
                for (int k = 0; k < COLS; ++k) srow[k * BM] = v[k];
            }
            epi_bar();
            float4 acc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] = *reinterpret_cast<const float4*>(stage + (q + 4 * u) * BM + c4);
            epi_fin<KIND>(ep, nw, nn, mrow, acc, p, N);
            epi_bar();
        }
    }
}

// K slices of one tile computed by the ks CTAs of a cluster (cluster rank =
// slice), reduced through distributed shared memory instead of partial planes
// in global memory.  Chunk c (32 accumulator columns) belongs to CTA c % ks;
// once every CTA's own MMAs are done its operand ring is idle and becomes the
// receive buffer: each CTA pushes its partial of every chunk it does not own
// into the owner's ring, then sums the slices of its own chunks in rank order
// (deterministic) and finishes them like staged_epilogue.  Waits are bounded;
// false when one gave up (the error word is set).
template <int KIND, int BN>
__device__ __forceinline__ bool cluster_epilogue(const EpiParams& ep, int M, int N, int n0, int m0, uint32_t tacc,
                                                 float* stage, float* recv, uint64_t* rfree, uint64_t* rfull,
                                                 const RowMeta* meta, int q, int lane, int ks, int rank, int* err) {
    constexpr int COLS = 32, NCH = BN / COLS, CH_FLOATS = COLS * BM;
    const int per_owner = (NCH + ks - 1) / ks;
    // this CTA's ring is idle: every other CTA may write into it
    if (threadIdx.x == 64)
        for (int r = 0; r < ks; ++r)
            if (r != rank) mbar_arrive_cluster(mapa_rank(smem_u32(rfree), (uint32_t)r));
    if (!epi_all(mbar_wait_cluster_bounded(smem_u32(rfree), 0, err))) return false;
    // push this slice's partial of every chunk another CTA owns
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
        const int o = c % ks;
        if (o == rank) continue;
        float v[COLS];
        tmem_ld32(tacc + (uint32_t)(c * COLS), v);
        const int slot = rank < o ? rank : rank - 1;  // this CTA's index among o's senders
        const uint32_t dst =
            mapa_rank(smem_u32(recv + (size_t)(slot * per_owner + c / ks) * CH_FLOATS + q * 32 + lane), (uint32_t)o);
#pragma unroll
        for (int k = 0; k < COLS; ++k) st_cluster_f32(dst + (uint32_t)(k * BM * 4), v[k]);
    }
    fence_acq_rel_cluster();
    __syncwarp();
    if (lane == 0)
        for (int o = 0; o < ks; ++o)
            if (o != rank) mbar_arrive_cluster(mapa_rank(smem_u32(rfull), (uint32_t)o));
    if (!epi_all(mbar_wait_cluster_bounded(smem_u32(rfull), 0, err))) return false;
    // this CTA's chunks: all slices summed in rank order, then the fused epilogue
    const int c4 = 4 * lane, nn = n0 + c4;
    const bool nok = nn < N;
#pragma unroll 1
    for (int c = rank; c < NCH; c += ks) {
        int mrow[8], krow[8];
        bool okr[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int rl = q + 4 * u;
            krow[u] = c * COLS + rl;
            mrow[u] = m0 + c * COLS + rl;
            okr[u] = nok && mrow[u] < M;
            if (KIND == EPI_STORE && ep.row_map && okr[u] && meta[krow[u]].live) mrow[u] = meta[krow[u]].pos;
        }
        EpiPre p;
        epi_pre<KIND>(ep, n0, nn, mrow, krow, okr, meta, N, p);
        {
            float v[COLS], a[COLS];
            tmem_ld32(tacc + (uint32_t)(c * COLS), v);
#pragma unroll
            for (int k = 0; k < COLS; ++k) a[k] = 0.f;
#pragma unroll 1
            for (int r = 0; r < ks; ++r) {
                if (r == rank) {
#pragma unroll
                    for (int k = 0; k < COLS; ++k) a[k] += v[k];
                } else {
                    const int slot = r < rank ? r : r - 1;
                    const float* src = recv + (size_t)(slot * per_owner + c / ks) * CH_FLOATS + q * 32 + lane;
#pragma unroll
                    for (int k = 0; k < COLS; ++k) a[k] += src[k * BM];
                }
            }
            float* srow = stage + q * 32 + lane;
#pragma unroll
            for (int k = 0; k < COLS; ++k) srow[k * BM] = a[k];
        }
        epi_bar();
        float4 acc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = *reinterpret_cast<const float4*>(stage + (q + 4 * u) * BM + c4);
        epi_fin<KIND>(ep, n0, nn, mrow, acc, p, N);
        epi_bar();
    }
    return true;
}

template <int BN, int WT, int BK, int CG>
__global__ void __launch_bounds__(192, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW,
                                                         const __grid_constant__ CUtensorMap tmX, const GemmArgs g) {
    using C = PCfg<BN, WT, BK, CG>;
    constexpr int SUB_A_BYTES = C::SUB_A_BYTES;
    constexpr int NACC = C::NACC;
    constexpr int TW = BM * WT * CG;  // weight rows per tile (of the pair when CG = 2)
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * C::A_STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::B_STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* acce = accf + 2;
    uint64_t* rfree = acce + 2;  // cluster K split: the other CTAs' rings are idle
    uint64_t* rfull = rfree + 1; // cluster K split: the other slices of this CTA's chunks have arrived
    uint64_t* mma_drain = rfull + 1;  // every MMA issued has completed (before TMEM is released)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
    int* last_flag = reinterpret_cast<int*>(tmem_slot + 1);  // epilogue warps: this CTA reduces the tile
    RowMeta* meta = reinterpret_cast<RowMeta*>(smem + STAGES * C::STAGE_BYTES + 256);
    float* epi_stage = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES + 256 + C::META_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = (g.K + BK - 1) / BK;
    const int units = g.full_tiles + (g.n_tiles * g.m_tiles - g.full_tiles) * g.splits;
    int* err = g.ep.err;
    // Unit schedule: units u0, u0 + ustep, ... (per CTA, or per pair).
    const uint32_t rank = CG == 2 ? cluster_rank() : 0u;
    const int u0 = CG == 2 ? (int)cluster_id() : (int)blockIdx.x;
    const int ustep = CG == 2 ? (int)cluster_count() : (int)gridDim.x;

    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 4 * CG);  // the epilogue warps of every CTA of the pair
        }
        mbar_init(rfree, g.ks > 1 ? g.ks - 1 : 1);
        mbar_init(rfull, g.ks > 1 ? 4 * (g.ks - 1) : 1);
        mbar_init(mma_drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        if constexpr (CG == 2) {  // one warp of each CTA of the pair, collectively
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(C::TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(C::TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    if (CG == 2 || g.ks > 1)
        cluster_sync();  // every CTA's barriers are initialised before another signals them
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // Weights never depend on the previous kernel: the first ring slots
            // of the first unit get their weight tiles before the dependency
            // wait (overlapping that kernel's tail), the activations after it.
            // A pair's loads all complete on the even CTA's ring barrier, which
            // expects the bytes of both CTAs.
            auto load = [&](void* dst, const CUtensorMap* tm, int x, int y, int s) {
                if constexpr (CG == 2)
                    tma_load_2d_pair(dst, tm, x, y, mapa_rank(smem_u32(&full[s]), 0));
                else
                    tma_load_2d(dst, tm, x, y, &full[s]);
            };
            auto expect = [&](int s) {
                if (rank == 0) mbar_expect_tx(&full[s], CG * C::STAGE_BYTES);
            };
            uint32_t it = 0;
            int pre = 0;
            if (u0 < units) {
                const Unit un = unit_of(g, u0, KB);
                const int na = (un.tile / g.m_tiles) * TW + (int)rank * BM;
                const int kb0 = un.kb0, nkb = un.nkb;
                pre = min(nkb, STAGES);
                for (int i = 0; i < pre; ++i) {
                    expect(i);
#pragma unroll
                    for (int w = 0; w < WT; ++w)
                        load(sA + i * C::A_STAGE_BYTES + w * SUB_A_BYTES, &tmW, (kb0 + i) * BK, na + w * BM, i);
                }
            }
            griddep_wait();
            griddep_launch();
            bool ok = true;
            for (int u = u0; u < units && ok; u += ustep) {
                const Unit un = unit_of(g, u, KB);
                const int na = (un.tile / g.m_tiles) * TW + (int)rank * BM;
                const int mb = (un.tile % g.m_tiles) * BN + (int)rank * C::B_ROWS;
                const int kb0 = un.kb0, nkb = un.nkb;
                for (int i = 0; i < nkb; ++i, ++it) {
                    const int s = it % STAGES;
                    const int kx = (kb0 + i) * BK;
                    if ((int)it >= pre) {
                        const uint32_t ph = (it / STAGES) & 1u;
                        if (!mbar_wait_bounded(smem_u32(&empty[s]), ph ^ 1u, err)) {
                            ok = false;
                            break;
                        }
                        expect(s);
#pragma unroll
                        for (int w = 0; w < WT; ++w)
                            load(sA + s * C::A_STAGE_BYTES + w * SUB_A_BYTES, &tmW, kx, na + w * BM, s);
                    }
                    load(sB + s * C::B_STAGE_BYTES, &tmX, kx, mb, s);
                }
            }
            if constexpr (CG == 2) {
                // Drain: every stage's last release (a commit from the even CTA)
                // lands before this CTA may exit.
                for (uint32_t f = it > (uint32_t)STAGES ? it - STAGES : 0u; f < it && ok; ++f)
                    ok = mbar_wait_bounded(smem_u32(&empty[f % STAGES]), (f / STAGES) & 1u, err);
            } else {
                // Drain: the loads of the last stages issued land before this CTA
                // may exit (they complete whether or not anything consumed them).
                for (uint32_t f = it > (uint32_t)STAGES ? it - STAGES : 0u; f < it; ++f)
                    mbar_wait_bounded(smem_u32(&full[f % STAGES]), (f / STAGES) & 1u, nullptr, 200000000LL);
            }
        } else {
            griddep_wait();
            griddep_launch();
        }
    } else if (warp == 1) {
        griddep_wait();
        griddep_launch();
        if (lane == 0 && rank == 0) {  // a pair's MMAs are issued by its even CTA
            constexpr uint32_t idesc_full = idesc_bf16(BM * CG, BN);
            const int Ml = live_rows(g.ep, g.M);
            uint32_t it = 0, j = 0;
            bool ok = true;
            for (int u = u0; u < units && ok; u += ustep, ++j) {
                const Unit un = unit_of(g, u, KB);
                const int nkb = un.nkb;
                // rows counted on the device: a tile past them issues no MMA, a
                // single-CTA tile narrows its MMA to the live rows (multiple of 16)
                const int live = Ml - (un.tile % g.m_tiles) * BN;
                const bool skip = live <= 0;
                const uint32_t idesc = (CG == 1 && live > 0 && live < BN)
                                           ? idesc_bf16(BM, (live + 15) & ~15) : idesc_full;
                const uint32_t b = j % NACC, use = j / NACC;
                const bool free_acc = CG == 2 ? mbar_wait_cluster_bounded(smem_u32(&acce[b]), (use & 1u) ^ 1u, err)
                                              : mbar_wait_bounded(smem_u32(&acce[b]), (use & 1u) ^ 1u, err);
                if (!free_acc) break;
                tc_fence_after();
                const uint32_t d = tmem + b * C::ACC_COLS;
                for (int i = 0; i < nkb; ++i, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&full[s]), ph, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t* a = sA + s * C::A_STAGE_BYTES;
                    const uint8_t* bb = sB + s * C::B_STAGE_BYTES;
                    if (!skip) {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
                            for (int w = 0; w < WT; ++w)
                                umma_bf16<CG>(d + w * BN, sdesc_k<BK>(a + w * SUB_A_BYTES + kk * 32),
                                              sdesc_k<BK>(bb + kk * 32), idesc, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit<CG>(&empty[s]);
                }
                umma_commit<CG>(&accf[b]);
            }
            // TMEM is released after the final barrier: every MMA issued (also
            // after a failed wait) must have completed by then
            umma_commit<CG>(mma_drain);
            mbar_wait_bounded(smem_u32(mma_drain), 0, nullptr, 200000000LL);
        }
        if (CG == 2 && lane == 0 && rank == 1)  // the pair's commit reaches this CTA's barrier too
            mbar_wait_bounded(smem_u32(mma_drain), 0, nullptr, 200000000LL);
    } else {
        griddep_wait();
        griddep_launch();
        const int q = warp & 3;
        // the accumulator is released on the even CTA's barrier
        auto release = [&](uint32_t b) {
            if constexpr (CG == 2)
                mbar_arrive_cluster(mapa_rank(smem_u32(&acce[b]), 0));
            else
                mbar_arrive(&acce[b]);
        };
        uint32_t j = 0;
        for (int u = u0; u < units; u += ustep, ++j) {
            const Unit un = unit_of(g, u, KB);
            const int split = un.split, tile = un.tile, nsplit = un.nsplit;
            // n0: this CTA's first weight row (its TMEM lanes); m0: the tile's first activation row
            const int n0 = (tile / g.m_tiles) * TW + (int)rank * BM, m0 = (tile % g.m_tiles) * BN;
            const uint32_t b = j % NACC, use = j / NACC;
            const bool ok = epi_all(mbar_wait_bounded(smem_u32(&accf[b]), use & 1u, err));
            if (!ok) break;
            tc_fence_after();
            fill_row_meta<BN>(g.ep, m0, g.M, meta, threadIdx.x - 64);
            epi_bar();
            const uint32_t tacc = tmem + b * C::ACC_COLS + ((uint32_t)(q * 32) << 16);
            if (nsplit == 1 && g.ep.kind == EPI_ENTROPY) {
#pragma unroll 1
                for (int w = 0; w < WT; ++w) {
                    const int n = n0 + w * BM + q * 32 + lane;
                    const bool valid = n < g.N && n != g.ep.mask_id;
                    const int pidx = (n0 / BM + w) * 4 + q;
#pragma unroll 1
                    for (int c = 0; c < BN; c += 16) {
                        float v[16];
                        tmem_ld16(tacc + (uint32_t)(w * BN + c), v);
                        entropy16(g.ep, v, valid, n, c, meta, m0, pidx, lane);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release(b);
            } else if (nsplit == 1 && BN >= C::EPI_COLS && (g.N & 3) == 0) {
                // the accumulator is fully read once the last chunk is loaded: the
                // next unit's MMAs may start while the stores finish
                auto rel = [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) release(b);
                };
                switch (g.ep.kind) {
                    case EPI_STORE:
                        staged_epilogue<EPI_STORE, BN, WT>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, meta, q, lane, rel);
                        break;
                    case EPI_RESIDUAL:
                        staged_epilogue<EPI_RESIDUAL, BN, WT>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, meta, q, lane,
                                                              rel);
                        break;
                    case EPI_SWIGLU:
                        staged_epilogue<EPI_SWIGLU, BN, WT>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, meta, q, lane, rel);
                        break;
                    case EPI_QKV_ROPE:
                        staged_epilogue<EPI_QKV_ROPE, BN, WT>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, meta, q, lane,
                                                              rel);
                        break;
                    default: rel(); break;
                }
            } else if (nsplit == 1) {
#pragma unroll 1
                for (int w = 0; w < WT; ++w) {
                    const int nw = n0 + w * BM, n = nw + q * 32 + lane;
#pragma unroll 1
                    for (int c = 0; c < BN; c += 16) {
                        float v[16];
                        tmem_ld16(tacc + (uint32_t)(w * BN + c), v);
                        epilogue16(g.ep, nw, n, m0 + c, c, meta, v, g.N, lane);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release(b);
            } else if (g.ks > 1) {
                bool ok2 = true;
                if constexpr (WT == 1 && CG == 1 && BN >= 128) {
                    const int rank = (int)cluster_rank();
                    float* recv = reinterpret_cast<float*>(sA);
                    switch (g.ep.kind) {
                        case EPI_STORE:
                            ok2 = cluster_epilogue<EPI_STORE, BN>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, recv, rfree,
                                                                  rfull, meta, q, lane, g.ks, rank, err);
                            break;
                        case EPI_RESIDUAL:
                            ok2 = cluster_epilogue<EPI_RESIDUAL, BN>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, recv,
                                                                     rfree, rfull, meta, q, lane, g.ks, rank, err);
                            break;
                        case EPI_SWIGLU:
                            ok2 = cluster_epilogue<EPI_SWIGLU, BN>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, recv, rfree,
                                                                   rfull, meta, q, lane, g.ks, rank, err);
                            break;
                        case EPI_QKV_ROPE:
                            ok2 = cluster_epilogue<EPI_QKV_ROPE, BN>(g.ep, g.M, g.N, n0, m0, tacc, epi_stage, recv,
                                                                     rfree, rfull, meta, q, lane, g.ks, rank, err);
                            break;
                        default: break;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) release(b);
                if (!ok2) break;
            } else {
                float* plane = g.ep.ws + (int64_t)split * g.M * g.N;
                if constexpr (BN >= C::EPI_COLS) {
                    // the slice's fp32 partial through the staged path (float4 rows);
                    // rows the epilogue skips are not written and never read back
                    EpiParams pe = g.ep;
                    pe.kind = EPI_STORE;
                    pe.out = plane;
                    pe.row_map = nullptr;  // planes are indexed by the tile's own rows
                    auto rel = [&]() {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) release(b);
                    };
                    staged_epilogue<EPI_STORE, BN, WT>(pe, g.M, g.N, n0, m0, tacc, epi_stage, meta, q, lane, rel);
                } else {
#pragma unroll 1
                    for (int w = 0; w < WT; ++w) {
                        const int n = n0 + w * BM + q * 32 + lane;
#pragma unroll 1
                        for (int c = 0; c < BN; c += 16) {
                            float v[16];
                            tmem_ld16(tacc + (uint32_t)(w * BN + c), v);
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                const int m = m0 + c + k;
                                if (meta[c + k].live && n < g.N) plane[(int64_t)m * g.N + n] = v[k];
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) release(b);
                }
                // Two fixups of the K slices (both sum in fixed split order, so
                // results are deterministic):
                //  - distributed (g.coop, cooperative launch: the slices of a tile
                //    run co-resident in the same round): every slice waits for all
                //    planes, then reduces its own share of the tile's rows; the
                //    ticket counts 2*splits arrivals (written, then done reading);
                //  - last arriver: every slice leaves its plane and takes a ticket;
                //    the one that arrives last reduces the whole tile and resets
                //    the ticket; nobody waits.
                __threadfence();
                epi_bar();
                int* ctr = g.ep.counters + tile * CG + rank;
                int r0 = 0, r1 = BN;
                if (g.coop) {
                    if (threadIdx.x == 64) {
                        atomicAdd(ctr, 1);
                        const long long t0 = clock64();
                        while (*reinterpret_cast<volatile int*>(ctr) < nsplit) {
                            if (clock64() - t0 > 2000000000LL) {
                                set_error(err, kErrTimeout);
                                break;
                            }
                            __nanosleep(64);
                        }
                        __threadfence();
                    }
                    epi_bar();
                    const int rows = (BN + nsplit - 1) / nsplit;
                    r0 = split * rows;
                    r1 = min(BN, r0 + rows);
                } else {
                    if (threadIdx.x == 64) *last_flag = (atomicAdd(ctr, 1) == nsplit - 1) ? 1 : 0;
                    epi_bar();
                    if (!*last_flag) continue;
                    __threadfence();
                }
                const int et = threadIdx.x - 64;
                const int mr = et >> 5;
#pragma unroll 1
                for (int w = 0; w < WT; ++w) {
                    const int nw = n0 + w * BM;
                    const int nn = nw + 4 * (et & 31);
                    const bool nok = nn < g.N;  // N % 4 == 0 whenever K is split
#pragma unroll 1
                    for (int rb = r0 + mr; rb < r1; rb += 4 * 8) {
                        float4 acc[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
                        for (int sp0 = 0; sp0 < nsplit; sp0 += 4) {
                            // up to 4 planes x 8 rows of independent loads in flight
                            float4 t4[4][8];
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const float* pl = g.ep.ws + (int64_t)(sp0 + jj) * g.M * g.N;
#pragma unroll
                                for (int u = 0; u < 8; ++u) {
                                    const int rr = rb + 4 * u, m = m0 + rr;
                                    t4[jj][u] = (sp0 + jj < nsplit && nok && rr < r1 && m < g.M)
                                                    ? __ldcg(reinterpret_cast<const float4*>(pl + (int64_t)m * g.N + nn))
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                                }
                            }
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                                for (int u = 0; u < 8; ++u) {
                                    acc[u].x += t4[jj][u].x;
                                    acc[u].y += t4[jj][u].y;
                                    acc[u].z += t4[jj][u].z;
                                    acc[u].w += t4[jj][u].w;
                                }
                        }
                        int mrow[8], krow[8];
                        bool okr[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int rr = rb + 4 * u;
                            krow[u] = rr < BN ? rr : 0;
                            mrow[u] = m0 + rr;
                            okr[u] = nok && rr < r1 && mrow[u] < g.M;
                            if (g.ep.kind == EPI_STORE && g.ep.row_map && okr[u] && meta[krow[u]].live)
                                mrow[u] = meta[krow[u]].pos;
                        }
                        epilogue_vec4x8(g.ep, nw, nn, mrow, krow, okr, meta, acc, g.N);
                    }
                }
                epi_bar();
                if (threadIdx.x == 64) {
                    if (!g.coop) *ctr = 0;
                    else if (atomicAdd(ctr, 1) == 2 * nsplit - 1) atomicExch(ctr, 0);
                }
            }
        }
    }
    tc_fence_before();
    if (CG == 2 || g.ks > 1)
        cluster_sync();  // no CTA leaves while another may still signal or read it
    else
        __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if constexpr (CG == 2)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                         : "memory");
        else
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

// Hybrid schedule (hybrid = true): the tiles that fill whole rounds of the
// launch run whole-K; only the tiles of the last, partial round are cut into
// a.splits K slices (reduced by the last slice to finish), so that round keeps
// every CTA busy.
inline void set_full_tiles(GemmArgs& a, bool hybrid, int per_round) {
    const int tiles = a.n_tiles * a.m_tiles;
    a.full_tiles = 0;
    if (!hybrid || a.splits == 1) return;
    a.full_tiles = (tiles / per_round) * per_round;
    if (a.full_tiles == tiles) a.splits = 1;  // no partial round
}

template <int BN, int WT, int BK, int CG = 1>
cudaError_t launch_bn(const CUtensorMap& tmW, const CUtensorMap& tmX, GemmArgs a, int grid, bool hybrid,
                      cudaStream_t st) {
    using C = PCfg<BN, WT, BK, CG>;
    auto kern = gemm_tc_kernel<BN, WT, BK, CG>;
    static int attr_dev = -1;
    static int max_pairs = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (CG == 2) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(2);
            q.blockDim = dim3(192);
            q.dynamicSmemBytes = C::SMEM_BYTES;
            cudaLaunchAttribute ca[1];
            ca[0].id = cudaLaunchAttributeClusterDimension;
            ca[0].val.clusterDim.x = 2;
            ca[0].val.clusterDim.y = 1;
            ca[0].val.clusterDim.z = 1;
            q.attrs = ca;
            q.numAttrs = 1;
            e = cudaOccupancyMaxActiveClusters(&max_pairs, kern, &q);
            if (e != cudaSuccess) return e;
            if (max_pairs < 1) return cudaErrorInvalidConfiguration;
        }
        attr_dev = dev;
    }
    if (CG == 2) {
        // Pairs run as clusters of two; the schedule strides over clusters, so
        // any even grid is correct and no more pairs than fit at once are launched.
        if (a.splits > 1 && a.coop) return cudaErrorInvalidValue;
        const int pairs = std::max(1, std::min(grid / 2, max_pairs));
        set_full_tiles(a, hybrid, pairs);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * pairs);
        cfg.blockDim = dim3(192);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, a);
    }
    if (a.ks > 1) {
        if (grid % a.ks) return cudaErrorInvalidValue;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(192);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = a.ks;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, a);
    }
    if (hybrid && a.coop) return cudaErrorInvalidValue;
    set_full_tiles(a, hybrid, grid);
    if (!(a.splits > 1 && a.coop))
        return launch_pdl(kern, dim3(grid), dim3(192), C::SMEM_BYTES, st, tmW, tmX, a);
    // The slices of a tile wait for one another: launch cooperatively so all CTAs
    // are resident at once (the launch fails instead of deadlocking).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, a);
}

}  // namespace

namespace {
int bn_for(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

GemmPlan make_plan(int M, int N, int K, int num_sms, int bn, int splits, int wt = 1, int bk = BK_DEFAULT,
                   int cg = 1, bool hybrid = false, bool cluster_k = false) {
    GemmPlan p;
    p.bn = bn;
    p.wt = wt;
    p.bk = bk;
    p.cg = cg;
    p.hybrid = hybrid && splits > 1;
    p.m_tiles = (M + bn - 1) / bn;
    p.n_tiles = (N + BM * wt * cg - 1) / (BM * wt * cg);
    const int KB = (K + bk - 1) / bk;
    p.kb_per_split = (KB + splits - 1) / splits;
    p.splits = (KB + p.kb_per_split - 1) / p.kb_per_split;
    // Units are dealt in rounds of `grid`; a multiple of the split count keeps
    // the splits of every tile in one round (they wait for each other).
    const long units = (long)p.m_tiles * p.n_tiles * p.splits;
    if (cluster_k && p.splits > 1 && cg == 1 && wt == 1) {  // one unit per CTA, a tile's slices one cluster
        p.ks = p.splits;
        p.coop = 0;
        p.hybrid = 0;
        p.grid = (int)units;
        return p;
    }
    if (cg == 2) {  // CTA pairs; the K-split fixup of pairs is the last-arriver one
        p.coop = 0;
        p.grid = 2 * (int)std::min<long>(units, std::max(1, num_sms / 2));
        return p;
    }
    if (p.hybrid) {  // whole rounds of full tiles: every SM
        p.coop = 0;
        p.grid = (int)std::min<long>(units, num_sms);
        return p;
    }
    const int per_round = std::max(p.splits, (num_sms / p.splits) * p.splits);
    p.grid = (int)std::min<long>(units, per_round);
    return p;
}
}  // namespace

GemmPlan plan_gemm_bf16(int M, int N, int K, int num_sms, int max_splits, int force_bn, int force_splits,
                        int force_wt, int force_bk, int force_coop, int force_cg, int force_hybrid, int force_cluster_k) {
    GemmPlan p = plan_gemm_bf16_shape(M, N, K, num_sms, max_splits, force_bn, force_splits, force_wt, force_bk,
                                      force_cg, force_hybrid, force_cluster_k);
    p.coop = (p.cg == 2 || p.hybrid || p.ks > 1) ? 0 : force_coop >= 0 ? (force_coop ? 1 : 0) : (M > 128 ? 1 : 0);
    return p;
}

GemmPlan plan_gemm_bf16_shape(int M, int N, int K, int num_sms, int max_splits, int force_bn, int force_splits,
                              int force_wt, int force_bk, int force_cg, int force_hybrid, int force_cluster_k) {
    const int KB = (K + BK_DEFAULT - 1) / BK_DEFAULT;
    // the split-K reduction reads float4 runs of a row, so N must be a multiple of 4
    const int smax = (N % 4) ? 1 : std::max(1, std::min({max_splits, KB, 16}));
    if (force_bn > 0 || force_splits > 0) {
        const int bn = force_bn > 0 ? force_bn : bn_for(M);
        const int cg = (force_cg == 2 && (bn == 128 || bn == 256)) ? 2 : 1;
        const int wt = (cg == 1 && force_wt == 2 && bn >= 128) ? 2 : 1;
        const int bk = (cg == 1 && force_bk == 32 && bn >= 128) ? 32 : BK_DEFAULT;
        const bool ck = force_cluster_k != 0 && cg == 1 && wt == 1 && bk == BK_DEFAULT && bn >= 128;
        return make_plan(M, N, K, num_sms, bn, std::max(1, std::min(force_splits > 0 ? force_splits : 1, ck ? 4 : smax)),
                         ck ? 1 : wt, bk, cg, force_hybrid != 0 && !ck, ck);
    }
    // Cost in units of one 256-column k-block per CTA: rounds x k-block time x
    // (k-blocks per unit + per-unit overhead + the partial plane's round trip
    // when K is split).  Narrow tiles are bound by their weight stream, so a
    // k-block costs at least a quarter of a full-width one.
    GemmPlan best_p = make_plan(M, N, K, num_sms, bn_for(M), 1);
    double best = 1e30;
    int cands[2] = {bn_for(M), M > 128 ? 128 : 0};
    for (int bn : cands) {
        if (!bn) continue;
        const long tiles = (long)((M + bn - 1) / bn) * ((N + BM - 1) / BM);
        const double tkb = std::max(bn, 64) / 256.0;
        for (int sp = 1; sp <= smax; ++sp) {
            const int kbps = (KB + sp - 1) / sp;
            if ((KB + kbps - 1) / kbps != sp) continue;
            const int per_round = std::max(sp, (num_sms / sp) * sp);
            const double rounds = std::ceil((double)(tiles * sp) / per_round);
            const double cost = rounds * tkb * (kbps + 1.0 + (sp > 1 ? bn / 32.0 : 0.0));
            if (cost < best * 0.98) {
                best = cost;
                best_p = make_plan(M, N, K, num_sms, bn, sp);
            }
        }
    }
    return best_p;
}

bool encode_tmap_bf16(CUtensorMap* tm, const void* base, int rank, const cuuint64_t* gdim, const cuuint64_t* gstride,
                      const cuuint32_t* box) {
    auto fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return false;
    cuuint32_t estride[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                    const_cast<cuuint64_t*>(gdim), const_cast<cuuint64_t*>(gstride), const_cast<cuuint32_t*>(box),
                    estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, int bk) {
    auto fn = encode_fn();
    if (!fn || (bk != 64 && bk != 32)) return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)bk, box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, bk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm_bf16(const CUtensorMap& tmW, const CUtensorMap& tmX, int M, int N, int K, const GemmPlan& p,
                             const EpiParams& ep, cudaStream_t st) {
    if (p.splits > 1 && (!ep.ws || !ep.counters)) return cudaErrorInvalidValue;
    const int tw = 128 * p.wt * p.cg;
    if (ep.kind == EPI_ENTROPY && (p.splits != 1 || !ep.epart || ep.npart < ((N + tw - 1) / tw) * p.wt * p.cg * 4))
        return cudaErrorInvalidValue;
    GemmArgs a{M, N, K, p.kb_per_split, p.splits, p.n_tiles, p.m_tiles, p.coop, 0, p.ks, ep};
    const bool hy = p.hybrid != 0;
    if (p.ks > 1) {
        // cluster K split: one unit per CTA, a tile's slices are one cluster
        if (p.splits != p.ks || p.wt != 1 || p.cg != 1 || p.bk != 64 || (N & 3) || ep.kind == EPI_ENTROPY ||
            p.grid != p.n_tiles * p.m_tiles * p.ks)
            return cudaErrorInvalidValue;
        if (p.bn == 256) return launch_bn<256, 1, 64>(tmW, tmX, a, p.grid, false, st);
        if (p.bn == 128) return launch_bn<128, 1, 64>(tmW, tmX, a, p.grid, false, st);
        return cudaErrorInvalidValue;
    }
    if (p.cg == 2) {
        if (p.wt != 1 || p.bk != 64) return cudaErrorInvalidValue;
        if (p.bn == 256) return launch_bn<256, 1, 64, 2>(tmW, tmX, a, p.grid, hy, st);
        if (p.bn == 128) return launch_bn<128, 1, 64, 2>(tmW, tmX, a, p.grid, hy, st);
        return cudaErrorInvalidValue;
    }
    if (p.bk == 32) {
        if (p.wt == 2 && p.bn == 256) return launch_bn<256, 2, 32>(tmW, tmX, a, p.grid, hy, st);
        if (p.wt == 2 && p.bn == 128) return launch_bn<128, 2, 32>(tmW, tmX, a, p.grid, hy, st);
        if (p.wt == 1 && p.bn == 256) return launch_bn<256, 1, 32>(tmW, tmX, a, p.grid, hy, st);
        return cudaErrorInvalidValue;
    }
    if (p.wt == 2) {
        switch (p.bn) {
            case 128: return launch_bn<128, 2, 64>(tmW, tmX, a, p.grid, hy, st);
            case 256: return launch_bn<256, 2, 64>(tmW, tmX, a, p.grid, hy, st);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (p.bn) {
        case 16: return launch_bn<16, 1, 64>(tmW, tmX, a, p.grid, hy, st);
        case 32: return launch_bn<32, 1, 64>(tmW, tmX, a, p.grid, hy, st);
        case 64: return launch_bn<64, 1, 64>(tmW, tmX, a, p.grid, hy, st);
        case 128: return launch_bn<128, 1, 64>(tmW, tmX, a, p.grid, hy, st);
        case 256: return launch_bn<256, 1, 64>(tmW, tmX, a, p.grid, hy, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace wedlm

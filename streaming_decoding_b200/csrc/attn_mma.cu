// Reordered-causal GQA attention of window rows against the paged KV cache
// (bf16 storage, fp32 softmax), tensor cores via mma.sync m16n8k16.
//
// [Method] (hyper.ai summary of arXiv 2512.22737, section "Method"): after
// Topological Reordering the window is processed by a plain causal forward
// conditioned on the persistent KV cache; physical row r of a sequence with
// committed length S attends to cache positions 0..S-1 and window rows 0..r,
// whose K/V the QKV epilogue of this same forward wrote at positions S..S+r.
//
// One CTA owns (batch entry, KV head, tile of RT window rows, key split).  Its
// query rows are the RT rows times the g = hq/hkv query heads sharing the KV
// head (g*RT <= 16*NW; one warp per 16 query rows), so every K/V byte loaded
// serves all g heads.  The CTA's slice of the page table is staged in shared
// memory; keys stream through a 3-stage cp.async ring of 64-key blocks (4
// pages) with an XOR swizzle of 16-byte chunks that keeps ldmatrix
// conflict-free.  Online softmax in the exp2 domain.
// With more than one key split, unnormalised partial outputs plus (max, sum)
// go to a workspace and attn_combine_kernel merges them.
#include "kernels.cuh"

namespace wedlm {
namespace {

constexpr int HD = 128;
constexpr int KBLK = 64;
constexpr int CHUNKS = HD / 8;              // 16-byte chunks per key row
constexpr int TILE_BYTES = KBLK * HD * 2;   // one K or V block in shared memory
constexpr int ASTAGES = 3;                  // K/V blocks in flight per CTA
constexpr int MAX_PAGES_SMEM = 2048;        // page-table entries staged per CTA (32k keys)

__device__ __forceinline__ uint32_t swz(int key, int chunk) {
    return (uint32_t)(key * (HD * 2) + (((chunk ^ (key & 7))) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

struct AttnParams {
    const bf16* q;
    const bf16* kv_pool;
    KVLayout kvl;
    int layer, hq, hkv;
    bf16* out;
    float* part_o;
    float2* part_ml;
    int stride, kv_chunk, max_splits, rt;
    SlotState ss;
    RowMap rm;
    int* err;
};

// Issue cp.async copies of keys [kb0, kb0 + 64) (rows past ke zero-filled)
// into one K and one V stage; pages come from the CTA's staged page list.
__device__ __forceinline__ void load_kv_block(uint32_t sK, uint32_t sV, const AttnParams& p, int kvh,
                                              const int32_t* spages, int page0, int npages, int kb0, int ke,
                                              int nthreads) {
    for (int i = threadIdx.x; i < KBLK * CHUNKS; i += nthreads) {
        const int key = i / CHUNKS, ch = i - key * CHUNKS;
        const int t = kb0 + key;
        const bf16* srcK = p.kv_pool;
        const bf16* srcV = p.kv_pool;
        int bytes = 0;
        if (t < ke) {
            const int pi = t / kPage - page0;
            const int page = (pi >= 0 && pi < npages) ? spages[pi] : -1;
            if (page >= 0 && page < p.kvl.num_pages) {
                const int64_t o = (int64_t)(t % kPage) * HD + ch * 8;
                srcK = p.kv_pool + p.kvl.page_base(p.layer, page, 0, kvh) + o;
                srcV = p.kv_pool + p.kvl.page_base(p.layer, page, 1, kvh) + o;
                bytes = 16;
            } else {
                set_error(p.err, kErrBounds);
            }
        }
        cp_async16(sK + swz(key, ch), srcK, bytes);
        cp_async16(sV + swz(key, ch), srcV, bytes);
    }
}

template <int NW>
__global__ void __launch_bounds__(NW * 32) attn_bf16_kernel(const AttnParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
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
    const int g = p.hq / p.hkv;
    const int32_t* pt = p.ss.page_table + (int64_t)slot * p.ss.pages_per_seq;

    // This thread's two query rows (qa, qb = qa + 8) within the CTA tile.
    const int t4 = lane & 3, g8 = lane >> 2;
    int qrow[2], qhead[2], qlim[2];
    bool qok[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int qi = warp * 16 + g8 + 8 * u;
        const int rr = r0 + qi / g;
        qok[u] = (qi < p.rt * g) && (rr < n);
        const int rc = qok[u] ? rr : r_last;
        qrow[u] = entry * p.stride + rc;
        qhead[u] = kvh * g + (qi % g);
        qlim[u] = S + rc;  // last visible key (inclusive)
    }
    // Q fragments for the 8 k-steps of head_dim 128.
    uint32_t qf[8][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const uint32_t* qp = reinterpret_cast<const uint32_t*>(p.q + ((int64_t)qrow[u] * p.hq + qhead[u]) * HD);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qf[kk][u] = qok[u] ? qp[(16 * kk + 2 * t4) >> 1] : 0u;
            qf[kk][2 + u] = qok[u] ? qp[(16 * kk + 8 + 2 * t4) >> 1] : 0u;
        }
    }

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    const float sl2 = 1.4426950408889634f / sqrtf((float)HD);

    // stage this CTA's slice of the page table in shared memory
    int32_t* spages = reinterpret_cast<int32_t*>(smem + ASTAGES * 2 * TILE_BYTES);
    const int page0 = ks / kPage;
    const int npages = min((ke + kPage - 1) / kPage - page0, MAX_PAGES_SMEM);
    for (int i = threadIdx.x; i < npages; i += NW * 32)
        spages[i] = (page0 + i < p.ss.pages_per_seq) ? pt[page0 + i] : -1;
    __syncthreads();

    const uint32_t sbase = smem_u32(smem);
    const int nblk = (ke - ks + KBLK - 1) / KBLK;
#pragma unroll
    for (int st = 0; st < ASTAGES - 1; ++st) {
        if (st < nblk) {
            const uint32_t sK = sbase + st * 2 * TILE_BYTES;
            load_kv_block(sK, sK + TILE_BYTES, p, kvh, spages, page0, npages, ks + st * KBLK, ke, NW * 32);
        }
        cp_async_commit();
    }
    for (int b = 0; b < nblk; ++b) {
        const int kb0 = ks + b * KBLK;
        {
            const int nb = b + ASTAGES - 1;
            if (nb < nblk) {
                const uint32_t nK = sbase + (nb % ASTAGES) * 2 * TILE_BYTES;
                load_kv_block(nK, nK + TILE_BYTES, p, kvh, spages, page0, npages, ks + nb * KBLK, ke, NW * 32);
            }
            cp_async_commit();
        }
        cp_async_wait<ASTAGES - 1>();
        __syncthreads();
        const uint32_t sK = sbase + (b % ASTAGES) * 2 * TILE_BYTES;
        const uint32_t sV = sK + TILE_BYTES;

        // S = Q K^T for 64 keys: 8 key tiles of 8.
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sK + swz(8 * nt + (lane & 7), 2 * kk + (lane >> 3)), b0, b1, b2, b3);
                mma_bf16(s[nt], qf[kk], b0, b1);
                mma_bf16(s[nt], qf[kk + 1], b2, b3);
            }
        }
        // Mask (split range and causal limit) and online softmax.
        float bmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int u = e >> 1;
                const int key = kb0 + 8 * nt + 2 * t4 + (e & 1);
                const bool ok = key < ke && key <= qlim[u];
                s[nt][e] = ok ? s[nt][e] * sl2 : -INFINITY;
                bmax[u] = fmaxf(bmax[u], s[nt][e]);
            }
        }
        float corr[2], ref[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            bmax[u] = fmaxf(bmax[u], __shfl_xor_sync(0xffffffffu, bmax[u], 1));
            bmax[u] = fmaxf(bmax[u], __shfl_xor_sync(0xffffffffu, bmax[u], 2));
            const float mn = fmaxf(mrow[u], bmax[u]);
            ref[u] = (mn == -INFINITY) ? 0.f : mn;
            corr[u] = exp2f(mrow[u] - ref[u]);
            mrow[u] = mn;
        }
        float psum[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int u = e >> 1;
                const float pe = exp2f(s[nt][e] - ref[u]);
                s[nt][e] = pe;
                psum[u] += pe;
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) lrow[u] = lrow[u] * corr[u] + psum[u];
#pragma unroll
        for (int dn = 0; dn < 16; ++dn) {
            o[dn][0] *= corr[0];
            o[dn][1] *= corr[0];
            o[dn][2] *= corr[1];
            o[dn][3] *= corr[1];
        }
        // O += P V (P from the S accumulators, V via transposed ldmatrix).
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t pa[4];
            pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
            pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
            pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
            const int vkey = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int dn = 0; dn < 16; dn += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sV + swz(vkey, dn + (lane >> 4)), b0, b1, b2, b3);
                mma_bf16(o[dn], pa, b0, b1);
                mma_bf16(o[dn + 1], pa, b2, b3);
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int u = 0; u < 2; ++u) {
        lrow[u] += __shfl_xor_sync(0xffffffffu, lrow[u], 1);
        lrow[u] += __shfl_xor_sync(0xffffffffu, lrow[u], 2);
    }
    if (nsplit == 1) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!qok[u]) continue;
            const float inv = lrow[u] > 0.f ? 1.0f / lrow[u] : 0.f;
            bf16* op = p.out + ((int64_t)qrow[u] * p.hq + qhead[u]) * HD;
#pragma unroll
            for (int dn = 0; dn < 16; ++dn) {
                const int c = 8 * dn + 2 * t4;
                *reinterpret_cast<__nv_bfloat162*>(op + c) =
                    __floats2bfloat162_rn(o[dn][2 * u] * inv, o[dn][2 * u + 1] * inv);
            }
        }
    } else {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!qok[u]) continue;
            const int64_t pi = ((int64_t)qrow[u] * p.hq + qhead[u]) * p.max_splits + sp;
            float* po = p.part_o + pi * HD;
#pragma unroll
            for (int dn = 0; dn < 16; ++dn) {
                const int c = 8 * dn + 2 * t4;
                *reinterpret_cast<float2*>(po + c) = make_float2(o[dn][2 * u], o[dn][2 * u + 1]);
            }
            if (t4 == 0) p.part_ml[pi] = make_float2(mrow[u], lrow[u]);
        }
    }
}

__global__ void __launch_bounds__(128) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float2* __restrict__ part_ml, bf16* __restrict__ out,
                                                           int hq, int kv_chunk, int max_splits, int rt, SlotState ss,
                                                           RowMap rm) {
    const int row = blockIdx.x, head = blockIdx.y;
    int slot, r;
    if (!rm.live(row, slot, r)) return;
    const int n = rm.n[slot];
    const int r0 = (r / rt) * rt;
    const int r_last = min(r0 + rt, n) - 1;
    const int kend = ss.S[slot] + r_last + 1;
    const int ns = (kend + kv_chunk - 1) / kv_chunk;
    if (ns <= 1) return;
    const int64_t pi = ((int64_t)row * hq + head) * max_splits;
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, part_ml[pi + s].x);
    float L = 0.f, acc = 0.f;
    const int c = threadIdx.x;
    for (int s = 0; s < ns; ++s) {
        const float2 ml = part_ml[pi + s];
        const float w = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
        L += w * ml.y;
        acc += w * part_o[(pi + s) * HD + c];
    }
    out[((int64_t)row * hq + head) * HD + c] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
}

}  // namespace

int attn_rows_per_tile(int group) {
    // 4 warps (64 query rows) when they hold 16 window rows, else 8 warps.
    return (64 / group >= 16) ? 64 / group : 128 / group;
}

static int attn_warps(int group) { return (64 / group >= 16) ? 4 : 8; }

void launch_attn_bf16(const bf16* q, const bf16* kv_pool, KVLayout kvl, int layer, int hq, int hkv, int hd, bf16* out,
                      float* part_o, float2* part_ml, int n_entries, int stride, int kv_chunk, int max_splits,
                      SlotState ss, RowMap rm, int* err, cudaStream_t st) {
    (void)hd;
    const int g = hq / hkv;
    AttnParams p{q, kv_pool, kvl, layer, hq, hkv, out, part_o, part_ml, stride, kv_chunk, max_splits,
                 attn_rows_per_tile(g), ss, rm, err};
    const int tiles = (stride + p.rt - 1) / p.rt;
    dim3 grid(tiles, hkv, n_entries * max_splits);
    const int smem = ASTAGES * 2 * TILE_BYTES + MAX_PAGES_SMEM * 4;
    if (attn_warps(g) == 4) {
        static bool set4 = false;
        if (!set4) {
            cudaFuncSetAttribute(attn_bf16_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            set4 = true;
        }
        attn_bf16_kernel<4><<<grid, 128, smem, st>>>(p);
    } else {
        static bool set8 = false;
        if (!set8) {
            cudaFuncSetAttribute(attn_bf16_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            set8 = true;
        }
        attn_bf16_kernel<8><<<grid, 256, smem, st>>>(p);
    }
}

void launch_attn_combine(const float* part_o, const float2* part_ml, bf16* out, int M, int hq, int hd, int kv_chunk,
                         int max_splits, int rows_per_tile, SlotState ss, RowMap rm, cudaStream_t st) {
    (void)hd;
    dim3 grid(M, hq);
    attn_combine_kernel<<<grid, 128, 0, st>>>(part_o, part_ml, out, hq, kv_chunk, max_splits, rows_per_tile, ss, rm);
}

}  // namespace wedlm

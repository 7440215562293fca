// Window, epilogue, fp32 and selection kernels of libwedlm.
//
// Method references (by page and section):
//   [Method]  hyper.ai summary of arXiv 2512.22737, section "Method":
//             Topological Reordering, Streaming Parallel Decoding,
//             distance-penalised entropy selection.
//   [Review]  sai.science review "WeDLM: Reconciling Diffusion Language Models
//             with Standard Causal Attention for Fast Inference".
#include <cfloat>
#include <cmath>

#include "kernels.cuh"

namespace wedlm {

// ---------------------------------------------------------------------------
// Embedding gather + RMSNorm of one row: x = E[tok] (fp32), h = x / rms * g.
template <typename T>
__device__ void embed_norm_row(const T* E, int d, int tok, const float* g,
                               float eps, float* x, T* h, float* red) {
    float ss = 0.f;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        const float v = to_f32<T>(E[(int64_t)tok * d + c]);
        x[c] = v;
        ss += v * v;
    }
    ss = block_sum(ss, red);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    for (int c = threadIdx.x; c < d; c += blockDim.x) h[c] = from_f32<T>(x[c] * inv * g[c]);
}

// Decode step window preparation [Method]: refill with masks to
// min(W, end - S) slots; k = leftmost filled run; stable partition (filled
// ascending, then masks ascending); logical position S + offset per physical
// row; embed + first RMSNorm.  One CTA per (batch entry, physical row): each
// derives its entry's partition in shared memory from the window as it was
// before this step's refill (slots past the old window length count as
// masks), and CTA (entry, 0) writes the entry's updated window state.
template <typename T>
__global__ void __launch_bounds__(256) decode_prepare_kernel(const T* embed, const float* g,
                                                             float eps, int d, int mask_id, SlotState ss, RowState rs,
                                                             uint8_t* rowmask, int stride,
                                                             float* x, T* h, int blockwise) {
    griddep_wait();
    griddep_launch();
    __shared__ float red[32];
    __shared__ uint8_t s_f[kMaxWindow];
    __shared__ int32_t s_t[kMaxWindow];
    __shared__ int32_t s_perm[kMaxWindow];
    __shared__ int s_k, s_nf;
    const int slot = blockIdx.x, r = blockIdx.y;
    const int base = slot * stride;
    const int W = ss.W[slot], S = ss.S[slot], end = ss.end[slot], wlen = ss.wlen[slot];
    const bool active = W > 0 && S < end;
    const int n = active ? min(min(W, end - S), stride) : 0;
    uint8_t* f = ss.filled + (int64_t)slot * ss.maxW;
    int32_t* t = ss.token + (int64_t)slot * ss.maxW;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const bool fj = j < wlen && f[j];
        s_f[j] = fj ? 1 : 0;
        s_t[j] = fj ? t[j] : mask_id;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int nf = 0;
        for (int j = 0; j < n; ++j)
            if (s_f[j]) s_perm[nf++] = j;
        int m = nf;
        for (int j = 0; j < n; ++j)
            if (!s_f[j]) s_perm[m++] = j;
        int k = 0;
        while (k < n && s_f[k]) ++k;
        if (blockwise && k < n) k = 0;  // block-wise baseline: the whole window or nothing
        s_k = k;
        s_nf = nf;
    }
    __syncthreads();
    if (r == 0) {
        for (int j = wlen + threadIdx.x; j < n; j += blockDim.x) {  // refill
            f[j] = 0;
            t[j] = mask_id;
        }
        // (the window length itself is rewritten by the step's commit: every
        // CTA of this launch reads the old value)
        if (threadIdx.x == 0) {
            ss.n[slot] = n;
            ss.k[slot] = s_k;
            ss.nf[slot] = s_nf;
        }
    }
    float* xr = x + (int64_t)(base + r) * d;
    T* hr = h + (int64_t)(base + r) * d;
    if (r < n) {
        const int j = s_perm[r];
        const int tok = s_f[j] ? s_t[j] : mask_id;
        if (threadIdx.x == 0) {
            rs.perm[base + r] = j;
            rs.pos[base + r] = S + j;
            rs.tok[base + r] = tok;
            rowmask[base + r] = s_f[j] ? 0 : 1;
        }
        embed_norm_row<T>(embed, d, tok, g, eps, xr, hr, red);
    } else {
        if (threadIdx.x == 0) {
            rs.perm[base + r] = -1;
            rs.pos[base + r] = -1;
            rs.tok[base + r] = -1;
            rowmask[base + r] = 0;
        }
        for (int c = threadIdx.x; c < d; c += blockDim.x) {
            xr[c] = 0.f;
            hr[c] = from_f32<T>(0.f);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(256) prefill_prepare_kernel(const T* embed, const float* g,
                                                              float eps, int d, const int32_t* ids,
                                                              int slot, int S0, int n, SlotState ss, RowState rs,
                                                              float* x, T* h) {
    __shared__ float red[32];
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        ss.S[slot] = S0;
        ss.n[slot] = n;
    }
    for (int r = blockIdx.x; r < n; r += gridDim.x) {
        if (threadIdx.x == 0) {
            rs.pos[r] = S0 + r;
            rs.tok[r] = ids[r];
            rs.perm[r] = r;
        }
        embed_norm_row<T>(embed, d, ids[r], g, eps, x + (int64_t)r * d, h + (int64_t)r * d, red);
    }
}

__global__ void slot_admit_kernel(SlotState ss, int slot, int P, int end, int W) {
    ss.S[slot] = P;
    ss.P[slot] = P;
    ss.end[slot] = end;
    ss.W[slot] = W;
    ss.wlen[slot] = 0;
    ss.n[slot] = 0;
    ss.k[slot] = 0;
    ss.nf[slot] = 0;
    for (int j = 0; j < ss.maxW; ++j) {
        ss.filled[(int64_t)slot * ss.maxW + j] = 0;
        ss.token[(int64_t)slot * ss.maxW + j] = 0;
    }
    for (int c = 0; c < 4; ++c) ss.counters[slot * 4 + c] = 0;
    ss.out_count[slot] = 0;
}

__global__ void prefill_finish_kernel(SlotState ss, int slot, int P) {
    ss.S[slot] = P;
    ss.n[slot] = 0;
}

// ---------------------------------------------------------------------------
// fp32 SIMT GEMM (exact-parity mode): C[M][N] = X[M][K] * W[N][K]^T, fp32 FMA
// accumulation in ascending k.  64x64 tiles, 16-deep k slabs, 4x4 per thread.
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* X, const float* Wt,
                                                       float* C, int M, int N, int K) {
    __shared__ float Xs[16][64 + 1];
    __shared__ float Ws[16][64 + 1];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int i = tid; i < 64 * 16; i += 256) {
            const int rr = i / 16, kk = i % 16;
            const int m = m0 + rr, n = n0 + rr, k = k0 + kk;
            Xs[kk][rr] = (m < M && k < K) ? X[(int64_t)m * K + k] : 0.f;
            Ws[kk][rr] = (n < N && k < K) ? Wt[(int64_t)n * K + k] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = Xs[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
            if (m < M && n < N) C[(int64_t)m * N + n] = acc[i][j];
        }
}

// ---------------------------------------------------------------------------
// QKV epilogue: sum split-K partials, rotate q and k at the row's logical
// position (rotate-half pairs (i, i + hd/2); [Method]: RoPE keeps logical
// positions through the reordering), write q to q_out[row][hq][hd] and k, v to
// the paged cache at physical index S + r of the row's sequence (rows 0..k-1
// of the window are the committed run, so their K/V land at their final
// cache positions without a copy).
template <typename T>
__global__ void __launch_bounds__(256) qkv_rope_kernel(const float* ws, int splits, int64_t sstride,
                                                       int hq, int hkv, int hd, T* q_out,
                                                       T* kv_pool, KVLayout kvl, int layer,
                                                       const float2* rope_cs, int rope_max_pos,
                                                       RowState rs, SlotState ss, RowMap rm, int* err) {
    const int row = blockIdx.x;
    int slot, r;
    if (!rm.live(row, slot, r)) return;
    const int pos = rs.pos[row];
    const int p = ss.S[slot] + r;
    const int pidx = p / kPage, off = p % kPage;
    if (pidx >= ss.pages_per_seq || pos < 0 || pos >= rope_max_pos) {
        if (threadIdx.x == 0) set_error(err, kErrBounds);
        return;
    }
    const int page = ss.page_table[(int64_t)slot * ss.pages_per_seq + pidx];
    if (page < 0 || page >= kvl.num_pages) {
        if (threadIdx.x == 0) set_error(err, kErrBounds);
        return;
    }
    const int half = hd / 2;
    const int ncols = (hq + 2 * hkv) * hd;
    const int npairs = (hq + 2 * hkv) * half;
    for (int pr = threadIdx.x; pr < npairs; pr += blockDim.x) {
        const int head = pr / half, i = pr - head * half;
        const int col = head * hd + i;
        float a = 0.f, b = 0.f;
        for (int s = 0; s < splits; ++s) {
            const float* w = ws + s * sstride + (int64_t)row * ncols;
            a += w[col];
            b += w[col + half];
        }
        if (head < hq + hkv) {
            const float2 cs = rope_cs[(int64_t)pos * half + i];
            const float a2 = a * cs.x - b * cs.y;
            const float b2 = b * cs.x + a * cs.y;
            a = a2;
            b = b2;
        }
        if (head < hq) {
            T* qo = q_out + (int64_t)row * hq * hd + head * hd;
            qo[i] = from_f32<T>(a);
            qo[i + half] = from_f32<T>(b);
        } else {
            const int kv = head < hq + hkv ? 0 : 1;
            const int h = head - hq - kv * hkv;
            T* dst = kv_pool + kvl.page_base(layer, page, kv, h) + (int64_t)off * hd;
            dst[i] = from_f32<T>(a);
            dst[i + half] = from_f32<T>(b);
        }
    }
}

// fp32 attention (exact-parity mode): one warp per (row, query head).  Row r
// of a sequence with committed length S attends to cache positions 0..S+r
// (the window rows before it in physical order, then itself) [Method].
__global__ void __launch_bounds__(128) attn_f32_kernel(const float* q, const float* kv_pool,
                                                       KVLayout kvl, int layer, int hq, int hkv, int hd,
                                                       float* out, SlotState ss, RowMap rm, int* err) {
    const int row = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.y * 4 + warp;
    if (head >= hq) return;
    int slot, r;
    float* o = out + (int64_t)row * hq * hd + head * hd;
    if (!rm.live(row, slot, r)) {
        for (int c = lane; c < hd; c += 32) o[c] = 0.f;
        return;
    }
    const int kvh = head / (hq / hkv);
    const int T = ss.S[slot] + r + 1;
    const float* qr = q + (int64_t)row * hq * hd + head * hd;
    constexpr int MAXD = 4;  // head_dim <= 128
    float qv[MAXD], acc[MAXD];
    const int nd = hd / 32;
#pragma unroll
    for (int j = 0; j < MAXD; ++j) {
        qv[j] = (j < nd) ? qr[lane + 32 * j] : 0.f;
        acc[j] = 0.f;
    }
    const float scale = 1.0f / sqrtf((float)hd);
    float m = -INFINITY, l = 0.f;
    const int32_t* pt = ss.page_table + (int64_t)slot * ss.pages_per_seq;
    for (int t = 0; t < T; ++t) {
        const int pidx = t / kPage;
        const int page = (pidx < ss.pages_per_seq) ? pt[pidx] : -1;
        if (page < 0 || page >= kvl.num_pages) {
            if (lane == 0) set_error(err, kErrBounds);
            break;
        }
        const float* kp = kv_pool + kvl.page_base(layer, page, 0, kvh) + (int64_t)(t % kPage) * hd;
        const float* vp = kv_pool + kvl.page_base(layer, page, 1, kvh) + (int64_t)(t % kPage) * hd;
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < MAXD; ++j)
            if (j < nd) s = fmaf(qv[j], kp[lane + 32 * j], s);
        s = warp_sum(s) * scale;
        const float mn = fmaxf(m, s);
        const float c = expf(m - mn);
        const float pe = expf(s - mn);
        l = l * c + pe;
#pragma unroll
        for (int j = 0; j < MAXD; ++j)
            if (j < nd) acc[j] = acc[j] * c + pe * vp[lane + 32 * j];
        m = mn;
    }
    const float inv = (l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
    for (int j = 0; j < MAXD; ++j)
        if (j < nd) o[lane + 32 * j] = acc[j] * inv;
}

// Residual add of the summed split-K partials, then RMSNorm with gain g:
// x += sum_s ws[s]; h = x / rms(x) * g.
template <typename T>
__global__ void __launch_bounds__(256) residual_norm_kernel(const float* ws, int splits, int64_t sstride,
                                                            int d, float* x, T* h,
                                                            const float* g, float eps, RowMap rm) {
    __shared__ float red[32];
    const int row = blockIdx.x;
    int slot, r;
    if (!rm.live(row, slot, r)) return;
    float* xr = x + (int64_t)row * d;
    float ss = 0.f;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float v = xr[c];
        for (int s = 0; s < splits; ++s) v += ws[s * sstride + (int64_t)row * d + c];
        xr[c] = v;
        ss += v * v;
    }
    ss = block_sum(ss, red);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    T* hr = h + (int64_t)row * d;
    for (int c = threadIdx.x; c < d; c += blockDim.x) hr[c] = from_f32<T>(xr[c] * inv * g[c]);
}

// RMSNorm of the residual stream into the next GEMM's bf16 input:
// h = x / rms(x) * g, one CTA per row, the row held in registers (float4
// loads; d % 4 == 0 and d <= 4 * 256 * kNormVec).
constexpr int kNormVec = 8;
__global__ void __launch_bounds__(256) rmsnorm_bf16_kernel(const float* x, bf16* h,
                                                           const float* g, float eps, int d, RowMap rm,
                                                           MaskedRows mr) {
    __shared__ float red[32];
    const int row = blockIdx.x;
    const float4* gr = reinterpret_cast<const float4*>(g);
    const int nv = d >> 2;
    float4 v[kNormVec], gv[kNormVec];
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {  // the gains are weights: read before the dependency wait
        const int c = threadIdx.x + i * blockDim.x;
        gv[i] = c < nv ? __ldcg(gr + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    griddep_wait();
    griddep_launch();
    int slot, r;
    int dst = row;
    if (mr.row_map) {
        // Only the masked rows (physical rows nf..n-1 of each window) feed the LM
        // head: they are packed in order, row i of the packed block being
        // sum over earlier windows of (n - nf) + (r - nf).
        const int e = row / rm.stride;
        if (row == 0 && threadIdx.x == 0) {
            int total = 0;
            for (int e2 = 0; e2 < mr.n_entries; ++e2)
                total += max(0, rm.n[rm.slot_base + e2] - mr.nf[rm.slot_base + e2]);
            *mr.count = total;
        }
        if (!rm.live(row, slot, r) || r < mr.nf[slot]) return;
        int before = 0;
        for (int e2 = 0; e2 < e; ++e2) before += max(0, rm.n[rm.slot_base + e2] - mr.nf[rm.slot_base + e2]);
        dst = before + r - mr.nf[slot];
        if (threadIdx.x == 0) mr.row_map[dst] = row;
    } else if (!rm.live(row, slot, r)) {
        return;
    }
    const float4* xr = reinterpret_cast<const float4*>(x + (int64_t)row * d);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = threadIdx.x + i * blockDim.x;
        v[i] = c < nv ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    }
    ss = block_sum(ss, red);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    __nv_bfloat162* hr = reinterpret_cast<__nv_bfloat162*>(h + (int64_t)dst * d);
#pragma unroll
    for (int i = 0; i < kNormVec; ++i) {
        const int c = threadIdx.x + i * blockDim.x;
        if (c < nv) {
            hr[2 * c] = __floats2bfloat162_rn(v[i].x * inv * gv[i].x, v[i].y * inv * gv[i].y);
            hr[2 * c + 1] = __floats2bfloat162_rn(v[i].z * inv * gv[i].z, v[i].w * inv * gv[i].w);
        }
    }
}

void launch_rmsnorm_bf16(const float* x, bf16* h, const float* g, float eps, int M, int d, RowMap rm,
                         cudaStream_t st, MaskedRows mr) {
    launch_pdl(rmsnorm_bf16_kernel, dim3(M), dim3(256), 0, st, x, h, g, eps, d, rm, mr);
}

// SwiGLU: act = silu(gate) * up, gate = columns [0, F), up = [F, 2F).
template <typename T>
__global__ void __launch_bounds__(256) swiglu_kernel(const float* ws, int splits, int64_t sstride, int F,
                                                     T* act, RowMap rm) {
    const int row = blockIdx.x;
    int slot, r;
    if (!rm.live(row, slot, r)) return;
    for (int c = threadIdx.x; c < F; c += blockDim.x) {
        float gv = 0.f, uv = 0.f;
        for (int s = 0; s < splits; ++s) {
            const float* w = ws + s * sstride + (int64_t)row * 2 * F;
            gv += w[c];
            uv += w[F + c];
        }
        act[(int64_t)row * F + c] = from_f32<T>(gv / (1.0f + expf(-gv)) * uv);
    }
}

__global__ void rope_table_kernel(float2* cs, int max_pos, int half, int hd, double theta) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)max_pos * half) return;
    const int pos = (int)(idx / half), i = (int)(idx % half);
    const double inv = pow(theta, -2.0 * (double)i / (double)hd);
    const double ang = (double)pos * inv;
    cs[idx] = make_float2((float)cos(ang), (float)sin(ang));
}

// ---------------------------------------------------------------------------
// Entropy and argmax of softmax(scale * z) over ids != mask_id, as one
// streaming pass [Method; Review, Weaknesses]: per chunk of the vocabulary a
// running (M, s, t, amax) with M = max, s = sum e^(z-M), t = sum e^(z-M)(z-M);
// then H = log s - t/s.  Probabilities are never stored.
struct EntAcc {
    float m, s, t;
    int a;
};

__device__ __forceinline__ void ent_push(EntAcc& e, float z, int idx) {
    if (z > e.m) {
        if (e.s > 0.f) {
            const float al = expf(e.m - z);
            e.t = al * (e.t + (e.m - z) * e.s);
            e.s = al * e.s;
        }
        e.s += 1.f;
        e.m = z;
        e.a = idx;
    } else {
        const float ex = expf(z - e.m);
        e.s += ex;
        e.t += ex * (z - e.m);
    }
}

__device__ __forceinline__ EntAcc ent_merge(const EntAcc& x, const EntAcc& y) {
    if (y.s == 0.f) return x;
    if (x.s == 0.f) return y;
    EntAcc o;
    o.m = fmaxf(x.m, y.m);
    const float ax = expf(x.m - o.m), ay = expf(y.m - o.m);
    o.s = ax * x.s + ay * y.s;
    o.t = ax * (x.t + (x.m - o.m) * x.s) + ay * (y.t + (y.m - o.m) * y.s);
    o.a = (x.m > y.m) ? x.a : (y.m > x.m) ? y.a : min(x.a, y.a);
    return o;
}

__device__ __forceinline__ EntAcc ent_shfl_merge(EntAcc e, int o) {
    EntAcc y;
    y.m = __shfl_xor_sync(0xffffffffu, e.m, o);
    y.s = __shfl_xor_sync(0xffffffffu, e.s, o);
    y.t = __shfl_xor_sync(0xffffffffu, e.t, o);
    y.a = __shfl_xor_sync(0xffffffffu, e.a, o);
    return ent_merge(e, y);
}

// Sampled fills (temperature T > 0): Gumbel-max, token = argmax_v
// (scale z_v / T + G_v), G_v = -log(-log u_v), with u_v from a counter-based
// generator on the SplitMix64 output function (Steele, Lea and Flood, OOPSLA
// 2014) keyed by (seed, slot, the slot's decode step, position, v).
__device__ __forceinline__ unsigned long long splitmix_out(unsigned long long z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

struct SampAcc {
    float k;
    int a;
};

__device__ __forceinline__ void samp_push(SampAcc& q, float key, int idx) {
    if (key > q.k || (key == q.k && idx < q.a)) {
        q.k = key;
        q.a = idx;
    }
}

__device__ __forceinline__ SampAcc samp_merge(SampAcc x, SampAcc y) {
    return (y.k > x.k || (y.k == x.k && y.a < x.a)) ? y : x;
}

// Greedy steps (no sampling, one plane of logits, rows a multiple of 4 floats
// apart): each thread issues its share of a chunk -- up to kScanVec float4 --
// as independent loads, then reduces them with one reference maximum: m = max
// z, s = sum e^(z-m), t = sum e^(z-m)(z-m), the first index of the maximum.
// A NaN or an infinity among z leaves a NaN in s or t (R22: the row is then
// reported invalid by the selection).
constexpr int kScanVec = 10;
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__global__ void __launch_bounds__(256) entropy_scan_kernel(const float* logits, int64_t ld, int V,
                                                           int mask_id, float scale,
                                                           const uint8_t* rowmask, int chunks,
                                                           float4* part) {
    griddep_wait();
    griddep_launch();
    const int row = blockIdx.y, c = blockIdx.x;
    if (!rowmask[row]) return;
    const int csz = ((V + chunks - 1) / chunks + 3) & ~3;
    const int v0 = c * csz, v1 = min(V, v0 + csz);
    const int nvec = max(0, v1 - v0) >> 2;
    const float4* z4 = reinterpret_cast<const float4*>(logits + (int64_t)row * ld + v0);
    constexpr float kLog2e = 1.4426950408889634f;
    EntAcc acc{-INFINITY, 0.f, 0.f, INT_MAX};
    // The mask id and ids past the chunk end read -FLT_MAX: never a maximum
    // (ties do not replace), weight 2^(-288) = 0 below.  Non-finite logits are
    // caught by chk = sum z * 0 (NaN as soon as one z is a NaN or an
    // infinity), which makes the partial's sums NaN (the row is then invalid).
    float chk = 0.f;
    for (int b = 0; b < nvec; b += 256 * kScanVec) {
        float4 v[kScanVec];
        // all loads of the block first, in flight together
#pragma unroll
        for (int k = 0; k < kScanVec; ++k) {
            const int i = b + threadIdx.x + k * 256;
            v[k] = i < nvec ? __ldcg(z4 + i) : make_float4(-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX);
        }
#pragma unroll
        for (int k = 0; k < kScanVec; ++k) {
            const unsigned off = (unsigned)(mask_id - (v0 + 4 * (b + threadIdx.x + k * 256)));
            if (off < 4u) {
                if (off == 0) v[k].x = -FLT_MAX;
                else if (off == 1) v[k].y = -FLT_MAX;
                else if (off == 2) v[k].z = -FLT_MAX;
                else v[k].w = -FLT_MAX;
            }
        }
        // maximum and its first index, compared on the raw logits (scale > 0
        // keeps their order)
        float zm = -FLT_MAX;
        int a = INT_MAX;
        float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < kScanVec; ++k) {
            const int id = v0 + 4 * (b + threadIdx.x + k * 256);
            if (v[k].x > zm) { zm = v[k].x; a = id; }
            if (v[k].y > zm) { zm = v[k].y; a = id + 1; }
            if (v[k].z > zm) { zm = v[k].z; a = id + 2; }
            if (v[k].w > zm) { zm = v[k].w; a = id + 3; }
            c4[0] = fmaf(v[k].x, 0.f, c4[0]);
            c4[1] = fmaf(v[k].y, 0.f, c4[1]);
            c4[2] = fmaf(v[k].z, 0.f, c4[2]);
            c4[3] = fmaf(v[k].w, 0.f, c4[3]);
        }
        chk += (c4[0] + c4[1]) + (c4[2] + c4[3]);
        if (a == INT_MAX) continue;  // nothing but the mask id and padding
        // e = 2^(d log2 e), d = scale z - m (clamped at -200: e is 0 there);
        // four independent partial sums per thread
        const float m = scale * zm;
        float sum[4] = {0.f, 0.f, 0.f, 0.f}, tw[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < kScanVec; ++k) {
            const float zz[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float d = fmaxf(fmaf(scale, zz[q], -m), -200.f);
                const float e = ex2_ftz(d * kLog2e);
                sum[q] += e;
                tw[q] = fmaf(e, d, tw[q]);
            }
        }
        acc = ent_merge(acc, EntAcc{m, (sum[0] + sum[1]) + (sum[2] + sum[3]), (tw[0] + tw[1]) + (tw[2] + tw[3]), a});
    }
    if (chk != 0.f) {  // a NaN or an infinity among this thread's logits
        acc.s = __int_as_float(0x7fc00000);
        acc.t = acc.s;
    }
    // the chunk's last (v1 - v0) % 4 ids
    for (int id = v0 + 4 * nvec + threadIdx.x; id < v1; id += blockDim.x)
        if (id != mask_id) ent_push(acc, scale * logits[(int64_t)row * ld + id], id);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc = ent_shfl_merge(acc, o);
    __shared__ EntAcc sh[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        EntAcc t = sh[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) t = ent_merge(t, sh[w]);
        part[(int64_t)row * chunks + c] = make_float4(t.m, t.s, t.t, __int_as_float(t.a));
    }
}

__global__ void __launch_bounds__(256) entropy_partial_kernel(const float* logits, int splits,
                                                              int64_t sstride, int64_t ld, int V, int mask_id,
                                                              float scale, const uint8_t* rowmask,
                                                              int chunks, float4* part, SampleArgs sa) {
    griddep_wait();
    griddep_launch();
    const int row = blockIdx.y, c = blockIdx.x;
    if (!rowmask[row]) return;
    const int csz = ((V + chunks - 1) / chunks + 3) & ~3;
    const int v0 = c * csz, v1 = min(V, v0 + csz);
    EntAcc e{-INFINITY, 0.f, 0.f, INT_MAX};
    SampAcc q{-INFINITY, INT_MAX};
    const bool sampling = sa.inv_t > 0.f;
    unsigned long long hrow = 0;
    if (sampling) {
        const int slot = row / sa.stride;
        hrow = splitmix_out(sa.seed ^ (unsigned long long)slot);
        hrow = splitmix_out(hrow ^ (unsigned long long)sa.steps[(int64_t)slot * 4]);
        hrow = splitmix_out(hrow ^ (unsigned long long)(long long)sa.pos[row]);
    }
    const float kz = scale * sa.inv_t;
    auto push = [&](float z, int id) {
        ent_push(e, scale * z, id);
        if (sampling) {
            const unsigned long long h = splitmix_out(hrow ^ (unsigned long long)id);
            const float u = ((float)(h >> 40) + 0.5f) * 5.9604644775390625e-8f;  // 2^-24
            samp_push(q, kz * z - logf(-logf(u)), id);
        }
    };
    const float* zr = logits + (int64_t)row * ld;
    if (splits == 1 && (ld & 3) == 0) {
        const int nvec = (v1 - v0) >> 2;
        const float4* z4 = reinterpret_cast<const float4*>(zr + v0);
        for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
            const float4 z = __ldcg(z4 + i);
            const int id = v0 + 4 * i;
            if (id != mask_id) push(z.x, id);
            if (id + 1 != mask_id) push(z.y, id + 1);
            if (id + 2 != mask_id) push(z.z, id + 2);
            if (id + 3 != mask_id) push(z.w, id + 3);
        }
        for (int id = v0 + 4 * nvec + threadIdx.x; id < v1; id += blockDim.x)
            if (id != mask_id) push(zr[id], id);
    } else {
        for (int id = v0 + threadIdx.x; id < v1; id += blockDim.x) {
            if (id == mask_id) continue;
            float z = 0.f;
            for (int s = 0; s < splits; ++s) z += logits[s * sstride + (int64_t)row * ld + id];
            push(z, id);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        e = ent_shfl_merge(e, o);
        SampAcc y{__shfl_xor_sync(0xffffffffu, q.k, o), __shfl_xor_sync(0xffffffffu, q.a, o)};
        q = samp_merge(q, y);
    }
    __shared__ EntAcc sh[8];
    __shared__ SampAcc shq[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        sh[warp] = e;
        shq[warp] = q;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        EntAcc t = sh[0];
        SampAcc tq = shq[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
            t = ent_merge(t, sh[w]);
            tq = samp_merge(tq, shq[w]);
        }
        part[(int64_t)row * chunks + c] = make_float4(t.m, t.s, t.t, __int_as_float(t.a));
        if (sampling) sa.part[(int64_t)row * chunks + c] = make_float2(tq.k, __int_as_float(tq.a));
    }
}

// Second level of the fused LM-head entropy: merge the GEMM epilogue's
// per-32-id partials of a masked row into `chunks` partials (the layout the
// selection kernel reads).
__global__ void __launch_bounds__(256) entropy_merge_kernel(const float4* part, int npart,
                                                            const uint8_t* rowmask, int chunks,
                                                            float4* out) {
    griddep_wait();
    griddep_launch();
    const int row = blockIdx.y, c = blockIdx.x;
    if (!rowmask[row]) return;
    const int seg = (npart + chunks - 1) / chunks;
    const int p0 = c * seg, p1 = min(npart, p0 + seg);
    EntAcc e{-INFINITY, 0.f, 0.f, INT_MAX};
    for (int i = p0 + threadIdx.x; i < p1; i += blockDim.x) {
        const float4 q = __ldcg(part + (int64_t)row * npart + i);
        e = ent_merge(e, EntAcc{q.x, q.y, q.z, __float_as_int(q.w)});
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e = ent_shfl_merge(e, o);
    __shared__ EntAcc sh[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[warp] = e;
    __syncthreads();
    if (threadIdx.x == 0) {
        EntAcc t = sh[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) t = ent_merge(t, sh[w]);
        out[(int64_t)row * chunks + c] = make_float4(t.m, t.s, t.t, __int_as_float(t.a));
    }
}

__device__ __forceinline__ int combine_sample(const float2* part, int chunks, int row) {
    SampAcc q{-INFINITY, INT_MAX};
    for (int c = 0; c < chunks; ++c) {
        const float2 v = part[(int64_t)row * chunks + c];
        q = samp_merge(q, SampAcc{v.x, __float_as_int(v.y)});
    }
    return q.a;
}

// H and the argmax of a masked row from its chunk partials.  A NaN or an
// infinity among the row's logits leaves a NaN in the running sums (the
// exponential of a NaN, or 0 times an infinite offset), so such a row comes
// out with H = NaN: the caller treats it as invalid (never filled, argmax -1).
__device__ __forceinline__ void combine_entropy(const float4* part, int chunks, int row, float& H, int& a) {
    EntAcc e{-INFINITY, 0.f, 0.f, INT_MAX};
    for (int c = 0; c < chunks; ++c) {
        const float4 q = part[(int64_t)row * chunks + c];
        EntAcc y{q.x, q.y, q.z, __float_as_int(q.w)};
        e = ent_merge(e, y);
    }
    H = (e.s > 0.f) ? logf(e.s) - e.t / e.s : (e.s == 0.f ? 0.f : NAN);
    if (!isfinite(H) || !isfinite(e.m)) {
        H = NAN;
        a = -1;
        return;
    }
    a = e.a;
}

// Fill decisions for one window from H~ of its masked slots (R5): every
// masked slot with H~ < tau; if none (or tau_none) the argmin, lowest offset
// on ties.  ht[j] is NaN for non-masked slots.
__device__ __forceinline__ int choose_fills(const float* ht, const uint8_t* masked, int n, StepKnobs kn,
                                            uint8_t* fill) {
    int count = 0;
    for (int j = 0; j < n; ++j) {
        fill[j] = 0;
        if (!kn.tau_none && masked[j] && ht[j] < kn.tau) {
            fill[j] = 1;
            ++count;
        }
    }
    if (count == 0) {
        int best = -1;
        for (int j = 0; j < n; ++j)
            if (masked[j] && (best < 0 || ht[j] < ht[best])) best = j;
        if (best >= 0) {
            fill[best] = 1;
            count = 1;
        }
    }
    return count;
}

// Selection, commit and slide for one decode step, one CTA per batch entry
// [Method]: H~_j = H_j + lambda * j over masked slots; commit the k slots of
// the leftmost filled run (their K/V already sit at cache positions S..S+k-1);
// fill the chosen masks with their argmax tokens; slide the window by k.
__global__ void __launch_bounds__(64) select_commit_kernel(const float4* part,
                                                           const float2* spart, int chunks, SlotState ss,
                                                           RowState rs, int stride, StepKnobs kn, int* err) {
    griddep_wait();
    griddep_launch();
    const int slot = blockIdx.x;
    const int n = ss.n[slot];
    __shared__ float sh[kMaxWindow];
    __shared__ int sa[kMaxWindow];
    __shared__ uint8_t smask[kMaxWindow];
    __shared__ uint8_t sfill[kMaxWindow];
    const int maxW = ss.maxW;
    if (n == 0) {
        if (threadIdx.x == 0) ss.out_count[slot] = 0;
        for (int j = threadIdx.x; j < maxW; j += blockDim.x) {
            ss.htilde[(int64_t)slot * maxW + j] = NAN;
            ss.amax[(int64_t)slot * maxW + j] = -1;
            ss.fillflag[(int64_t)slot * maxW + j] = 0;
        }
        return;
    }
    const int k = ss.k[slot], nf = ss.nf[slot];
    const uint8_t* f = ss.filled + (int64_t)slot * maxW;
    for (int j = threadIdx.x; j < kMaxWindow; j += blockDim.x) {
        sh[j] = NAN;
        sa[j] = -1;
        smask[j] = (j < n && !f[j]) ? 1 : 0;
    }
    __syncthreads();
    for (int r = nf + threadIdx.x; r < n; r += blockDim.x) {
        const int row = slot * stride + r;
        const int j = rs.perm[row];
        float H;
        int a;
        combine_entropy(part, chunks, row, H, a);
        if (kn.temperature > 0.f && a >= 0) a = combine_sample(spart, chunks, row);  // the fill's sampled token
        if (j >= 0 && j < n) {
            sh[j] = H + kn.lambda * (float)j;
            sa[j] = a;
            if (a < 0) {  // non-finite logits: reported, never filled
                smask[j] = 0;
                set_error(err, kErrNonFinite);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int nfill = choose_fills(sh, smask, n, kn, sfill);
        int32_t* tok = ss.token + (int64_t)slot * maxW;
        uint8_t* fl = ss.filled + (int64_t)slot * maxW;
        const int S = ss.S[slot], P = ss.P[slot];
        for (int j = 0; j < k; ++j) {
            ss.out_tokens[(int64_t)slot * maxW + j] = tok[j];
            const int gi = S - P + j;
            if (gi >= 0 && gi < ss.gen_cap) ss.gen[(int64_t)slot * ss.gen_cap + gi] = tok[j];
            else set_error(err, kErrBounds);
        }
        for (int j = 0; j < n; ++j) {
            ss.htilde[(int64_t)slot * maxW + j] = sh[j];
            ss.amax[(int64_t)slot * maxW + j] = sa[j];
            ss.fillflag[(int64_t)slot * maxW + j] = sfill[j];
            if (sfill[j]) {
                fl[j] = 1;
                tok[j] = sa[j];
            }
        }
        for (int j = n; j < maxW; ++j) {
            ss.htilde[(int64_t)slot * maxW + j] = NAN;
            ss.amax[(int64_t)slot * maxW + j] = -1;
            ss.fillflag[(int64_t)slot * maxW + j] = 0;
        }
        for (int j = k; j < n; ++j) {  // slide
            fl[j - k] = fl[j];
            tok[j - k] = tok[j];
        }
        ss.wlen[slot] = n - k;
        ss.S[slot] = S + k;
        int64_t* cnt = ss.counters + (int64_t)slot * 4;
        cnt[0] += 1;
        cnt[1] += n;
        cnt[2] += k;
        cnt[3] += nfill;
        ss.out_count[slot] = k;
    }
}

// Stand-alone stages (test hooks) ------------------------------------------
__global__ void reorder_only_kernel(const uint8_t* filled, const int32_t* n,
                                    const int32_t* S, int n_seq, int stride, int32_t* perm,
                                    int32_t* pos, int32_t* kout, int32_t* nfout) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= n_seq) return;
    const uint8_t* f = filled + (int64_t)b * stride;
    const int nb = min(n[b], stride);
    int k = 0;
    while (k < nb && f[k]) ++k;
    int nf = 0;
    for (int j = 0; j < nb; ++j)
        if (f[j]) perm[(int64_t)b * stride + nf++] = j;
    int m = nf;
    for (int j = 0; j < nb; ++j)
        if (!f[j]) perm[(int64_t)b * stride + m++] = j;
    for (int r = 0; r < stride; ++r) {
        if (r < nb) pos[(int64_t)b * stride + r] = S[b] + perm[(int64_t)b * stride + r];
        else {
            perm[(int64_t)b * stride + r] = -1;
            pos[(int64_t)b * stride + r] = -1;
        }
    }
    kout[b] = k;
    nfout[b] = nf;
}

__global__ void rowmask_kernel(const uint8_t* filled, const int32_t* n, int n_seq, int stride, uint8_t* rowmask) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_seq * stride) return;
    const int b = i / stride, j = i % stride;
    rowmask[i] = (j < n[b] && !filled[i]) ? 1 : 0;
}

__global__ void __launch_bounds__(64) select_only_kernel(const float4* part, int chunks,
                                                         const uint8_t* filled, const int32_t* n,
                                                         int stride, StepKnobs kn, float* htilde, int32_t* amax,
                                                         uint8_t* fill, int* err) {
    const int b = blockIdx.x;
    const int nb = min(n[b], min(stride, kMaxWindow));
    __shared__ float sh[kMaxWindow];
    __shared__ uint8_t smask[kMaxWindow];
    __shared__ uint8_t sfill[kMaxWindow];
    __shared__ int sa[kMaxWindow];
    for (int j = threadIdx.x; j < kMaxWindow; j += blockDim.x) {
        const bool m = j < nb && !filled[(int64_t)b * stride + j];
        smask[j] = m ? 1 : 0;
        sfill[j] = 0;
        sh[j] = NAN;
        sa[j] = -1;
        if (m) {
            float H;
            int a;
            combine_entropy(part, chunks, b * stride + j, H, a);
            sh[j] = H + kn.lambda * (float)j;
            sa[j] = a;
            if (a < 0) {  // non-finite logits: reported, never filled
                smask[j] = 0;
                set_error(err, kErrNonFinite);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) choose_fills(sh, smask, nb, kn, sfill);
    __syncthreads();
    for (int j = threadIdx.x; j < stride; j += blockDim.x) {
        const bool in = j < kMaxWindow;
        htilde[(int64_t)b * stride + j] = in ? sh[j] : NAN;
        amax[(int64_t)b * stride + j] = in ? sa[j] : -1;
        fill[(int64_t)b * stride + j] = in ? sfill[j] : 0;
    }
}

// L2 eviction for timing runs: a read-only sweep over a buffer larger than L2
// leaves it full of clean lines (a memset would leave dirty lines that the
// timed kernel then pays to write back).
__global__ void __launch_bounds__(256) l2_evict_kernel(const float4* p, size_t n, float* sink) {
    float acc = 0.f;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = p[i];
        acc += v.x + v.y + v.z + v.w;
    }
    if (acc == 1234.5678f) *sink = acc;  // keeps the loads; the buffer is zero
}

// ---------------------------------------------------------------------------
// Host launch wrappers.
template <typename T>
void launch_decode_prepare(const T* embed, const float* g, float eps, int d, int mask_id, SlotState ss, RowState rs,
                           uint8_t* rowmask, int n_entries, int stride, float* x, T* h, int blockwise,
                           cudaStream_t st) {
    launch_pdl(decode_prepare_kernel<T>, dim3(n_entries, stride), dim3(256), 0, st, embed, g, eps, d, mask_id, ss, rs,
               rowmask, stride, x, h, blockwise);
}

template <typename T>
void launch_prefill_prepare(const T* embed, const float* g, float eps, int d, const int32_t* ids, int slot, int S0,
                            int n, SlotState ss, RowState rs, float* x, T* h, cudaStream_t st) {
    const int grid = n < 592 ? n : 592;
    prefill_prepare_kernel<T><<<grid > 0 ? grid : 1, 256, 0, st>>>(embed, g, eps, d, ids, slot, S0, n, ss, rs, x, h);
}

void launch_l2_evict(const void* buf, size_t bytes, float* sink, int num_sms, cudaStream_t st) {
    l2_evict_kernel<<<4 * num_sms, 256, 0, st>>>(reinterpret_cast<const float4*>(buf), bytes / 16, sink);
}

void launch_slot_admit(SlotState ss, int slot, int P, int end, int W, cudaStream_t st) {
    slot_admit_kernel<<<1, 1, 0, st>>>(ss, slot, P, end, W);
}

void launch_prefill_finish(SlotState ss, int slot, int P, cudaStream_t st) {
    prefill_finish_kernel<<<1, 1, 0, st>>>(ss, slot, P);
}

void launch_gemm_f32(const float* X, const float* W, float* C, int M, int N, int K, cudaStream_t st) {
    dim3 grid((N + 63) / 64, (M + 63) / 64);
    gemm_f32_kernel<<<grid, 256, 0, st>>>(X, W, C, M, N, K);
}

template <typename T>
void launch_qkv_rope(const float* ws, int splits, int64_t sstride, int M, int hq, int hkv, int hd, T* q_out,
                     T* kv_pool, KVLayout kvl, int layer, const float2* rope_cs, int rope_max_pos, RowState rs,
                     SlotState ss, RowMap rm, int* err, cudaStream_t st) {
    qkv_rope_kernel<T><<<M, 256, 0, st>>>(ws, splits, sstride, hq, hkv, hd, q_out, kv_pool, kvl, layer, rope_cs,
                                          rope_max_pos, rs, ss, rm, err);
}

void launch_attn_f32(const float* q, const float* kv_pool, KVLayout kvl, int layer, int hq, int hkv, int hd,
                     float* out, int M, SlotState ss, RowMap rm, int* err, cudaStream_t st) {
    dim3 grid(M, (hq + 3) / 4);
    attn_f32_kernel<<<grid, 128, 0, st>>>(q, kv_pool, kvl, layer, hq, hkv, hd, out, ss, rm, err);
}

template <typename T>
void launch_residual_norm(const float* ws, int splits, int64_t sstride, int M, int d, float* x, T* h, const float* g,
                          float eps, RowMap rm, cudaStream_t st) {
    residual_norm_kernel<T><<<M, 256, 0, st>>>(ws, splits, sstride, d, x, h, g, eps, rm);
}

template <typename T>
void launch_swiglu(const float* ws, int splits, int64_t sstride, int M, int F, T* act, RowMap rm, cudaStream_t st) {
    swiglu_kernel<T><<<M, 256, 0, st>>>(ws, splits, sstride, F, act, rm);
}

void launch_rope_table(float2* cs, int max_pos, int half, int hd, double theta, cudaStream_t st) {
    const int64_t n = (int64_t)max_pos * half;
    rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(cs, max_pos, half, hd, theta);
}

void launch_entropy_partials(const float* logits, int splits, int64_t sstride, int64_t ld, int V, int mask_id,
                             float scale, const uint8_t* rowmask, int rows, int chunks, float4* part, cudaStream_t st,
                             SampleArgs sa) {
    dim3 grid(chunks, rows);
    if (sa.inv_t <= 0.f && splits == 1 && (ld & 3) == 0 && ((uintptr_t)logits & 15) == 0) {
        launch_pdl(entropy_scan_kernel, grid, dim3(256), 0, st, logits, ld, V, mask_id, scale, rowmask, chunks, part);
        return;
    }
    launch_pdl(entropy_partial_kernel, grid, dim3(256), 0, st, logits, splits, sstride, ld, V, mask_id, scale, rowmask,
               chunks, part, sa);
}

void launch_entropy_merge(const float4* part, int npart, const uint8_t* rowmask, int rows, int chunks, float4* out,
                          cudaStream_t st) {
    launch_pdl(entropy_merge_kernel, dim3(chunks, rows), dim3(256), 0, st, part, npart, rowmask, chunks, out);
}

void launch_select_commit(const float4* part, const float2* spart, int chunks, SlotState ss, RowState rs,
                          int n_entries, int stride, StepKnobs kn, int* err, cudaStream_t st) {
    launch_pdl(select_commit_kernel, dim3(n_entries), dim3(64), 0, st, part, spart, chunks, ss, rs, stride, kn, err);
}

void launch_reorder_only(const uint8_t* filled, const int32_t* n, const int32_t* S, int n_seq, int stride,
                         int32_t* perm, int32_t* pos, int32_t* k, int32_t* nf, cudaStream_t st) {
    reorder_only_kernel<<<(n_seq + 63) / 64, 64, 0, st>>>(filled, n, S, n_seq, stride, perm, pos, k, nf);
}

void launch_select_only(const float4* part, int chunks, const uint8_t* filled, const int32_t* n, int n_seq,
                        int stride, StepKnobs kn, float* htilde, int32_t* argmax, uint8_t* fill, int* err,
                        cudaStream_t st) {
    select_only_kernel<<<n_seq, 64, 0, st>>>(part, chunks, filled, n, stride, kn, htilde, argmax, fill, err);
}

void launch_rowmask_from_filled(const uint8_t* filled, const int32_t* n, int n_seq, int stride, uint8_t* rowmask,
                                cudaStream_t st) {
    const int tot = n_seq * stride;
    rowmask_kernel<<<(tot + 255) / 256, 256, 0, st>>>(filled, n, n_seq, stride, rowmask);
}

// Explicit instantiations.
#define WEDLM_INST(T)                                                                                             \
    template void launch_decode_prepare<T>(const T*, const float*, float, int, int, SlotState, RowState, uint8_t*, \
                                           int, int, float*, T*, int, cudaStream_t);                              \
    template void launch_prefill_prepare<T>(const T*, const float*, float, int, const int32_t*, int, int, int,     \
                                            SlotState, RowState, float*, T*, cudaStream_t);                       \
    template void launch_qkv_rope<T>(const float*, int, int64_t, int, int, int, int, T*, T*, KVLayout, int,        \
                                     const float2*, int, RowState, SlotState, RowMap, int*, cudaStream_t);        \
    template void launch_residual_norm<T>(const float*, int, int64_t, int, int, float*, T*, const float*, float,  \
                                          RowMap, cudaStream_t);                                                  \
    template void launch_swiglu<T>(const float*, int, int64_t, int, int, T*, RowMap, cudaStream_t);
WEDLM_INST(float)
WEDLM_INST(bf16)
#undef WEDLM_INST

}  // namespace wedlm

// libwedlm: context, weights, prefill and the Streaming Parallel Decoding step
// behind the C ABI declared in include/wedlm.h.
//
// One decode step (hyper.ai summary of arXiv 2512.22737, section "Method") is
// a fixed sequence of kernel launches on the context's stream:
//   decode_prepare      refill + topological reorder + embed + RMSNorm
//   per layer (x L):    QKV GEMM -> qkv_rope (RoPE at logical positions,
//                       K/V into the paged cache) -> attention (+ combine)
//                       -> O GEMM -> residual+RMSNorm -> gate/up GEMM
//                       -> SwiGLU -> down GEMM -> residual+RMSNorm
//   LM-head GEMM        (all window rows; only masked rows are read)
//   entropy_partials    online (max, sum e, sum e*z, argmax) per vocab chunk
//   select_commit       H~ = H + lambda*j, threshold/argmin fills, commit run,
//                       slide
// followed by one device->host copy of the per-slot results.  Every size a
// kernel needs per step lives in device memory, so a step is replayable
// without host involvement.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <deque>
#include <map>
#include <string>
#include <vector>

#include "gemm_tc.cuh"
#include "kernels.cuh"

using namespace wedlm;

namespace {

constexpr int kEntropyChunks = 16;
constexpr size_t kEvictBytes = (size_t)256 << 20;  // > 2x the 126 MB L2

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Arena {
    // One cudaMalloc carved into 256-byte aligned pieces.
    char* base = nullptr;
    size_t size = 0, used = 0;
    std::vector<std::pair<void**, size_t>> plan;
    void add(void** p, size_t bytes) { plan.emplace_back(p, align_up(bytes ? bytes : 1, 256)); }
    // Zeroed on the context's stream: work the context enqueues later on that
    // stream (the RoPE table, the first prefill) is ordered after the zeroing,
    // which it would not be on the legacy default stream when the context's
    // stream is a non-blocking one.
    cudaError_t commit(cudaStream_t st) {
        size = 0;
        for (auto& e : plan) size += e.second;
        cudaError_t err = cudaMalloc(&base, size);
        if (err != cudaSuccess) return err;
        size_t off = 0;
        for (auto& e : plan) {
            *e.first = base + off;
            off += e.second;
        }
        return cudaMemsetAsync(base, 0, size, st);
    }
    void release() {
        if (base) cudaFree(base);
        base = nullptr;
    }
};

}  // namespace

struct wedlm_ctx {
    wedlm_model_cfg cfg{};
    int device = 0;
    int num_sms = 148;
    cudaStream_t stream = nullptr;
    bool bf16 = false;
    size_t elt = 4;
    std::string last_error;
    int64_t launches = 0;

    int L, d, hq, hkv, hd, F, V, Nqkv;
    int maxB, maxW, max_ctx, num_pages, pages_per_seq, chunk;
    int Mdec, Mmax;

    Arena weights_arena, state_arena, scratch_arena;
    // weights
    void* embed = nullptr;
    void* lm_head = nullptr;
    float* final_norm = nullptr;
    std::vector<float*> attn_norm, ffn_norm;
    std::vector<void*> wqkv, wo, wgu, wd;
    std::vector<uint8_t> loaded;  // per tensor slot
    bool weights_ready = false;
    // bf16 tensor maps of the weights (box 128 rows)
    // Weight tensor maps for both k-block depths (64: 128-byte swizzle, 32: 64-byte).
    struct WMap {
        CUtensorMap k64{}, k32{};
        const CUtensorMap& of(int bk) const { return bk == 32 ? k32 : k64; }
    };
    std::vector<WMap> tm_qkv, tm_o, tm_gu, tm_d;
    WMap tm_lm{};
    bool maps_ready = false;
    // KV pool
    void* kv_pool = nullptr;
    KVLayout kvl{};
    float2* rope_cs = nullptr;
    // slot state (device)
    SlotState ss{};
    RowState rs{};
    uint8_t* rowmask = nullptr;
    int* err = nullptr;
    // scratch
    float* x = nullptr;
    void* h = nullptr;
    void* q = nullptr;
    void* attn_out = nullptr;
    void* act = nullptr;
    float* ws = nullptr;           // split-K partial planes
    size_t ws_floats = 0;
    int* tile_counters = nullptr;  // per-tile tickets of the split-K reduction
    size_t n_tile_counters = 0;
    // GEMM launch shapes chosen by timing candidates, per (projection kind, rows)
    bool autotune = true;
    struct Tuned {
        GemmPlan plan;
        float us;
    };
    std::map<std::pair<int, int>, Tuned> tuned;
    // CUDA graph of one decode step, replayed while its shape and knobs match
    bool use_graphs = true;
    cudaGraphExec_t graph_exec = nullptr;
    int64_t graph_launches = 0;
    struct StepKey {
        int n_entries = -1, stride = -1, tau_none = 0, blockwise = 0;
        float lambda = 0.f, tau = 0.f, scale = 0.f, temperature = 0.f;
        uint64_t seed = 0;
        bool operator==(const StepKey& o) const {
            return n_entries == o.n_entries && stride == o.stride && tau_none == o.tau_none &&
                   blockwise == o.blockwise && lambda == o.lambda && tau == o.tau && scale == o.scale &&
                   temperature == o.temperature && seed == o.seed;
        }
    };
    StepKey graph_key, eager_key;
    float* logits = nullptr;
    size_t logits_floats = 0;
    void* evict = nullptr;        // zeroed buffer larger than L2, swept before every tuning launch
    float* evict_sink = nullptr;
    float4* ent_part = nullptr;
    float2* samp_part = nullptr;  // Gumbel-max partials of sampled fills
    float* dbg_resid = nullptr;   // test hook: residual stream before each layer and after the last [L+1][Mdec][d]
    float4* lm_part = nullptr;    // fused LM-head entropy partials [Mdec][lm_npart]
    int32_t* lm_rows = nullptr;   // [Mdec] physical row of each packed masked row (LM-head input)
    int32_t* lm_count = nullptr;  // [1] masked rows of the current step
    int lm_npart = 0;
    bool keep_logits = false;     // test hook: write logits (unfused LM head + entropy pass)
    bool force_fused = false;     // test hook: greedy bf16 steps always take the fused LM-head entropy
    std::map<int, bool> fuse_choice;  // rows -> fused LM-head entropy is the faster path
    bool capturing = false;           // a step is being captured into a CUDA graph: no timing runs
    float* attn_po = nullptr;
    float2* attn_pml = nullptr;
    CUtensorMap tm_kv{};
    CUtensorMap tm_q{}, tm_q_dual{};
    int attn_kv_chunk = 1 << 30, attn_max_splits = 1;
    int32_t* ids_dev = nullptr;
    // step results block for one device->host copy: counts[B], S[B], tokens[B][maxW], err
    int32_t* res_dev = nullptr;
    int32_t* res_host = nullptr;  // pinned
    // activation tensor maps keyed by (buffer, rows, cols, box)
    struct XMap {
        const void* p;
        uint64_t rows, cols;
        uint32_t box;
        int bk;
        CUtensorMap tm;
    };
    std::deque<XMap> xmaps;
    // host mirrors
    std::vector<int> h_W, h_S, h_end, h_P;
    std::vector<std::vector<int>> h_pages;
    std::vector<int> free_pages;
    int last_stride = 0;
    int logits_splits_last = 1;
    int last_M = 0;
    // per-kernel timing (wedlm_profile_enable)
    bool prof = false;
    std::vector<cudaEvent_t> ev_pool;
    size_t ev_used = 0;
    std::vector<std::pair<int, size_t>> ev_marks;  // (kind, index of the start event)
    double prof_ms[WEDLM_PROF_KINDS] = {};
    int64_t prof_n[WEDLM_PROF_KINDS] = {};
};

namespace {

wedlm_status fail(wedlm_ctx* c, wedlm_status s, const std::string& msg) {
    if (c) c->last_error = msg;
    return s;
}

// Profiling: bracket a launch with events when enabled.
cudaEvent_t prof_event(wedlm_ctx* c) {
    if (c->ev_used == c->ev_pool.size()) {
        cudaEvent_t e;
        cudaEventCreate(&e);
        c->ev_pool.push_back(e);
    }
    return c->ev_pool[c->ev_used++];
}

struct ProfScope {
    wedlm_ctx* c;
    int kind;
    ProfScope(wedlm_ctx* c_, int kind_) : c(c_), kind(kind_) {
        if (c->prof) {
            c->ev_marks.emplace_back(kind, c->ev_used);
            cudaEventRecord(prof_event(c), c->stream);
        }
        c->launches++;
    }
    ~ProfScope() {
        if (c->prof) cudaEventRecord(prof_event(c), c->stream);
    }
};

void prof_collect(wedlm_ctx* c) {
    if (c->ev_marks.empty()) return;
    cudaStreamSynchronize(c->stream);
    for (auto& m : c->ev_marks) {
        float ms = 0.f;
        cudaEventElapsedTime(&ms, c->ev_pool[m.second], c->ev_pool[m.second + 1]);
        c->prof_ms[m.first] += ms;
        c->prof_n[m.first] += 1;
    }
    c->ev_marks.clear();
    c->ev_used = 0;
}

#define CK(call)                                                                                  \
    do {                                                                                          \
        cudaError_t e_ = (call);                                                                  \
        if (e_ != cudaSuccess)                                                                    \
            return fail(ctx, WEDLM_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
    } while (0)

int tensor_slot(const wedlm_ctx* c, int tensor, int layer) {
    switch (tensor) {
        case WEDLM_T_EMBED: return 0;
        case WEDLM_T_LM_HEAD: return 1;
        case WEDLM_T_FINAL_NORM: return 2;
        default: break;
    }
    if (tensor < WEDLM_T_ATTN_NORM || tensor > WEDLM_T_WD || layer < 0 || layer >= c->L) return -1;
    return 3 + layer * 9 + (tensor - WEDLM_T_ATTN_NORM);
}

const CUtensorMap* xmap(wedlm_ctx* c, const void* p, uint64_t rows, uint64_t cols, uint32_t box, int bk) {
    for (auto& m : c->xmaps)
        if (m.p == p && m.rows == rows && m.cols == cols && m.box == box && m.bk == bk) return &m.tm;
    wedlm_ctx::XMap m{p, rows, cols, box, bk, {}};
    if (!make_tmap_bf16(&m.tm, p, rows, cols, box, bk)) return nullptr;
    c->xmaps.push_back(m);
    return &c->xmaps.back().tm;
}

// fp32 mode: C[M][N] = X[M][K] * W[N][K]^T into `out` (the epilogue kernels follow).
wedlm_status gemm_f32(wedlm_ctx* ctx, int kind, const float* X, const float* W, int M, int N, int K) {
    if ((size_t)M * N > ctx->ws_floats) return fail(ctx, WEDLM_ERR_STATE, "gemm workspace too small");
    ProfScope ps(ctx, kind);
    launch_gemm_f32(X, W, ctx->ws, M, N, K, ctx->stream);
    return WEDLM_OK;
}

// Time the candidate launch shapes of one projection (kind, M) on its real
// weights with its real epilogue, and keep the fastest.  The residual add is
// redirected into the logits scratch; the other epilogues write buffers the
// launch that follows rewrites anyway (the q / activation scratch, and K/V
// at the window's own cache positions).  Runs once per (kind, M) on the
// context's stream; candidates that do not fit the scratch buffers are skipped.
// Tuning key of a projection: the LM head with the entropy epilogue is tuned
// apart from the plain LM head (its epilogue costs differ).
int tune_kind(int kind, const EpiParams& ep) { return ep.kind == EPI_ENTROPY ? kind + 1000 : kind; }

void autotune_shape(wedlm_ctx* ctx, int kind, const void* X, const wedlm_ctx::WMap* tmW, int M, int N, int K,
                    const EpiParams& ep_real) {
    const std::pair<int, int> key(tune_kind(kind, ep_real), M);
    if (ctx->tuned.count(key)) return;
    ctx->tuned[key] = {plan_gemm_bf16(M, N, K, ctx->num_sms, 1), -1.f};
    EpiParams ep = ep_real;
    if (ep.kind == EPI_STORE || ep.kind == EPI_RESIDUAL) {
        if ((size_t)M * N > ctx->logits_floats) return;
        ep.out = ctx->logits;
    }
    // (activation rows per tile, 128-row weight sub-tiles per tile, k-block
    // depth, CTAs per tile: 2 = CTA-pair tiles of 256 weight rows)
    struct Shape {
        int bn, wt, bk, cg;
    };
    std::vector<Shape> shapes;
    if (M > 128)
        shapes = {{256, 1, 64, 2}, {128, 1, 64, 2}, {256, 1, 64, 1}, {128, 1, 64, 1}, {64, 1, 64, 1},
                  {256, 2, 64, 1}, {128, 2, 64, 1}, {256, 2, 32, 1}, {128, 2, 32, 1}, {256, 1, 32, 1}};
    else if (M > 64)
        shapes = {{128, 1, 64, 2}, {128, 1, 64, 1}, {64, 1, 64, 1}, {128, 2, 64, 1}, {128, 2, 32, 1}};
    else shapes = {{M <= 16 ? 16 : M <= 32 ? 32 : 64, 1, 64, 1}};
    cudaEvent_t e0 = prof_event(ctx), e1 = prof_event(ctx);
    float best = 1e30f;
    GemmPlan bestp = ctx->tuned[key].plan;
    ep.ws = ctx->ws;
    ep.counters = ctx->tile_counters;
    ep.err = ctx->err;
    const int KB = (K + 63) / 64;
    // Time one plan: `reps` launches (the first discarded), each after an L2
    // eviction: in a step every projection's weights arrive cold from HBM (the
    // other layers' weights stream through L2 in between), so a buffer twice
    // the size of L2 is read before each launch.  Minimum or median of the
    // timed launches.
    auto time_plan = [&](const GemmPlan& p, int reps, bool median) -> float {
        const CUtensorMap* tx = xmap(ctx, X, (uint64_t)ctx->Mmax, (uint64_t)K, (uint32_t)(p.bn / p.cg), p.bk);
        if (!tx) return 1e30f;
        std::vector<float> ts;
        for (int rep = 0; rep < reps; ++rep) {
            launch_l2_evict(ctx->evict, kEvictBytes, ctx->evict_sink, ctx->num_sms, ctx->stream);
            cudaEventRecord(e0, ctx->stream);
            if (launch_gemm_bf16(tmW->of(p.bk), *tx, M, N, K, p, ep, ctx->stream) != cudaSuccess) {
                cudaGetLastError();
                return 1e30f;
            }
            cudaEventRecord(e1, ctx->stream);
            ctx->launches++;
            cudaEventSynchronize(e1);
            float ms = 0.f;
            cudaEventElapsedTime(&ms, e0, e1);
            if (rep > 0) ts.push_back(ms * 1e3f);
        }
        if (ts.empty()) return 1e30f;
        std::sort(ts.begin(), ts.end());
        return median ? ts[ts.size() / 2] : ts[0];
    };
    std::vector<std::pair<float, GemmPlan>> timed;
    for (const Shape& sh : shapes) {
        for (int spc : {1, 2, -2, 3, -3, 4, -4, 6, -6, 8, -8, 12, -12, 16, -16, 102, 103, 104, 106, 202, 203, 204}) {
            // negative: the same split count with the last-arriver fixup (the
            // only one CTA pairs use); 10x: hybrid schedule, only the last
            // partial round split in x slices; 20x: x slices as the CTAs of one
            // cluster, reduced through distributed shared memory
            const bool hy = spc > 100 && spc < 200, ck = spc > 200;
            const int sp = ck ? spc - 200 : hy ? spc - 100 : spc < 0 ? -spc : spc;
            if (sp > KB || (sp > 1 && N % 4) || (sh.cg == 2 && spc > 1 && !hy)) continue;
            if (ck && (sh.cg != 1 || sh.wt != 1 || sh.bk != 64 || sh.bn < 128 || ep.kind == EPI_ENTROPY)) continue;
            GemmPlan p = plan_gemm_bf16(M, N, K, ctx->num_sms, 16, sh.bn, sp, sh.wt, sh.bk, (spc < 0 || hy) ? 0 : 1,
                                        sh.cg, hy ? 1 : 0, ck ? 1 : 0);
            if (p.splits != sp || p.cg != sh.cg || (p.hybrid != 0) != hy || (p.ks > 1) != ck) continue;
            if (p.splits > 1 && ((size_t)p.splits * M * N > ctx->ws_floats ||
                                 (size_t)p.m_tiles * p.n_tiles * p.cg > ctx->n_tile_counters))
                continue;
            const float t = time_plan(p, 5, false);
            if (t < 1e29f) timed.push_back({t, p});
        }
    }
    // Second pass: the fastest few again, more repetitions, by median (the first
    // pass is a noisy minimum over few runs).
    std::sort(timed.begin(), timed.end(), [](const auto& a, const auto& b) { return a.first < b.first; });
    for (size_t c = 0; c < timed.size() && c < 4; ++c) {
        const float t = time_plan(timed[c].second, 13, true);
        if (t < best) {
            best = t;
            bestp = timed[c].second;
        }
    }
    ctx->ev_used -= 2;
    ctx->tuned[key] = {bestp, best < 1e29f ? best : -1.f};
}

// bf16 mode: the persistent tcgen05 GEMM with its epilogue fused (gemm_tc.cuh).
wedlm_status gemm_bf16(wedlm_ctx* ctx, int kind, const void* X, const wedlm_ctx::WMap* tmW, int M, int N, int K,
                       EpiParams ep, bool tune = true) {
    GemmPlan p;
    const auto rec = ctx->tuned.find({tune_kind(kind, ep), M});
    if (rec != ctx->tuned.end() && tune) {  // a recorded (tuned or pinned) plan
        p = rec->second.plan;
    } else if (ctx->autotune && tune && !ctx->capturing) {  // no timing runs inside a graph capture
        autotune_shape(ctx, kind, X, tmW, M, N, K, ep);
        p = ctx->tuned[{tune_kind(kind, ep), M}].plan;
    } else {
        const size_t plane = (size_t)M * N;
        const int cap = (int)std::max<size_t>(1, std::min<size_t>(16, ctx->ws_floats / plane));
        p = plan_gemm_bf16(M, N, K, ctx->num_sms, cap);
    }
    if (ep.kind == EPI_ENTROPY && p.splits != 1)  // the entropy epilogue needs whole K sums
        p = plan_gemm_bf16(M, N, K, ctx->num_sms, 1, p.bn, 1, p.wt, p.bk, -1, p.cg);
    if (p.splits > 1 && ((size_t)p.n_tiles * p.m_tiles * p.cg > ctx->n_tile_counters ||
                         (size_t)p.splits * M * N > ctx->ws_floats))
        p = plan_gemm_bf16(M, N, K, ctx->num_sms, 1, p.bn, 1, p.wt, p.bk, -1, p.cg);
    const CUtensorMap* tx = xmap(ctx, X, (uint64_t)ctx->Mmax, (uint64_t)K, (uint32_t)(p.bn / p.cg), p.bk);
    if (!tx) return fail(ctx, WEDLM_ERR_CUDA, "cuTensorMapEncodeTiled failed for activations");
    ep.ws = ctx->ws;
    ep.counters = ctx->tile_counters;
    ep.err = ctx->err;
    cudaError_t e;
    {
        ProfScope ps(ctx, kind);
        e = launch_gemm_bf16(tmW->of(p.bk), *tx, M, N, K, p, ep, ctx->stream);
    }
    if (e != cudaSuccess) return fail(ctx, WEDLM_ERR_CUDA, std::string("gemm launch: ") + cudaGetErrorString(e));
    return WEDLM_OK;
}

// Partial-plane floats and tile tickets the bf16 GEMM plans of one shape may
// need (room for the tuning candidates: up to `max_splits` slices).
void gemm_needs(const wedlm_ctx* c, int M, int N, int K, int max_splits, size_t* ws, size_t* tiles) {
    const int KB = (K + 63) / 64;
    const int sp = std::min(max_splits, KB);
    if (sp > 1 && N % 4 == 0) *ws = std::max(*ws, (size_t)sp * M * N);
    const int bn_min = M > 128 ? 128 : 16;
    // tickets: one per 128-row weight tile, or two per CTA-pair tile of 256 rows
    *tiles = std::max(*tiles, (size_t)((M + bn_min - 1) / bn_min) * (2 * ((N + 255) / 256)));
}

wedlm_status build_weight_maps(wedlm_ctx* ctx) {
    if (!ctx->bf16 || ctx->maps_ready) return WEDLM_OK;
    ctx->tm_qkv.resize(ctx->L);
    ctx->tm_o.resize(ctx->L);
    ctx->tm_gu.resize(ctx->L);
    ctx->tm_d.resize(ctx->L);
    bool ok = true;
    for (int l = 0; l < ctx->L; ++l) {
        for (int bk : {64, 32}) {
            auto pick = [&](wedlm_ctx::WMap& m) { return bk == 32 ? &m.k32 : &m.k64; };
            ok &= make_tmap_bf16(pick(ctx->tm_qkv[l]), ctx->wqkv[l], ctx->Nqkv, ctx->d, 128, bk);
            ok &= make_tmap_bf16(pick(ctx->tm_o[l]), ctx->wo[l], ctx->d, (uint64_t)ctx->hq * ctx->hd, 128, bk);
            ok &= make_tmap_bf16(pick(ctx->tm_gu[l]), ctx->wgu[l], 2 * (uint64_t)ctx->F, ctx->d, 128, bk);
            ok &= make_tmap_bf16(pick(ctx->tm_d[l]), ctx->wd[l], ctx->d, ctx->F, 128, bk);
        }
    }
    ok &= make_tmap_bf16(&ctx->tm_lm.k64, ctx->lm_head, ctx->V, ctx->d, 128, 64);
    ok &= make_tmap_bf16(&ctx->tm_lm.k32, ctx->lm_head, ctx->V, ctx->d, 128, 32);
    if (!ok) return fail(ctx, WEDLM_ERR_CUDA, "cuTensorMapEncodeTiled failed for weights");
    ctx->maps_ready = true;
    return WEDLM_OK;
}

wedlm_status check_device_error(wedlm_ctx* ctx, int code) {
    if (code == 0) return WEDLM_OK;
    CK(cudaMemsetAsync(ctx->err, 0, sizeof(int), ctx->stream));
    // a GEMM that gave up may leave split-K tickets behind
    if (ctx->tile_counters)
        CK(cudaMemsetAsync(ctx->tile_counters, 0, ctx->n_tile_counters * sizeof(int), ctx->stream));
    if (code == kErrTimeout) return fail(ctx, WEDLM_ERR_TIMEOUT, "a bounded device wait timed out");
    if (code == kErrNonFinite)
        return fail(ctx, WEDLM_ERR_NONFINITE, "a masked slot's logits held a NaN or an infinity (slot not filled)");
    return fail(ctx, WEDLM_ERR_DEVICE_ASSERT, "a device bounds check fired");
}

// The transformer stack over rows [entry * stride + r] of slots slot_base +
// entry.  On entry x holds the embeddings and h the first RMSNorm; on exit h
// holds the final-normed hidden states.

// fp32 (exact-parity) mode: SIMT GEMMs, separate epilogue kernels.
// Test hook: keep the residual stream entering layer `idx` (idx = L: after the
// last layer) of a decode step.
void capture_residual(wedlm_ctx* ctx, int idx, int M, bool decode) {
    if (!ctx->dbg_resid || !decode) return;
    cudaMemcpyAsync(ctx->dbg_resid + (size_t)idx * ctx->Mdec * ctx->d, ctx->x, (size_t)M * ctx->d * sizeof(float),
                    cudaMemcpyDeviceToDevice, ctx->stream);
}

wedlm_status forward_f32(wedlm_ctx* ctx, int slot_base, int n_entries, int stride, bool decode) {
    const int M = n_entries * stride;
    RowMap rm{slot_base, stride, ctx->ss.n};
    const float eps = ctx->cfg.rms_eps;
    float* h = (float*)ctx->h;
    float* qb = (float*)ctx->q;
    float* ao = (float*)ctx->attn_out;
    float* act = (float*)ctx->act;
    wedlm_status s;
    capture_residual(ctx, 0, M, decode);
    for (int l = 0; l < ctx->L; ++l) {
        if ((s = gemm_f32(ctx, WEDLM_PROF_GEMM_QKV, h, (const float*)ctx->wqkv[l], M, ctx->Nqkv, ctx->d))) return s;
        {
            ProfScope ps(ctx, WEDLM_PROF_QKV_ROPE);
            launch_qkv_rope<float>(ctx->ws, 1, (int64_t)M * ctx->Nqkv, M, ctx->hq, ctx->hkv, ctx->hd, qb,
                                   (float*)ctx->kv_pool, ctx->kvl, l, ctx->rope_cs, ctx->max_ctx, ctx->rs, ctx->ss, rm,
                                   ctx->err, ctx->stream);
        }
        {
            ProfScope ps(ctx, WEDLM_PROF_ATTENTION);
            launch_attn_f32(qb, (const float*)ctx->kv_pool, ctx->kvl, l, ctx->hq, ctx->hkv, ctx->hd, ao, M, ctx->ss,
                            rm, ctx->err, ctx->stream);
        }
        if ((s = gemm_f32(ctx, WEDLM_PROF_GEMM_O, ao, (const float*)ctx->wo[l], M, ctx->d, ctx->hq * ctx->hd)))
            return s;
        {
            ProfScope ps(ctx, WEDLM_PROF_RESIDUAL_NORM);
            launch_residual_norm<float>(ctx->ws, 1, (int64_t)M * ctx->d, M, ctx->d, ctx->x, h, ctx->ffn_norm[l], eps,
                                        rm, ctx->stream);
        }
        if ((s = gemm_f32(ctx, WEDLM_PROF_GEMM_GATE_UP, h, (const float*)ctx->wgu[l], M, 2 * ctx->F, ctx->d)))
            return s;
        {
            ProfScope ps(ctx, WEDLM_PROF_SWIGLU);
            launch_swiglu<float>(ctx->ws, 1, (int64_t)M * 2 * ctx->F, M, ctx->F, act, rm, ctx->stream);
        }
        if ((s = gemm_f32(ctx, WEDLM_PROF_GEMM_DOWN, act, (const float*)ctx->wd[l], M, ctx->d, ctx->F))) return s;
        const float* gnext = (l + 1 < ctx->L) ? ctx->attn_norm[l + 1] : ctx->final_norm;
        {
            ProfScope ps(ctx, WEDLM_PROF_RESIDUAL_NORM);
            launch_residual_norm<float>(ctx->ws, 1, (int64_t)M * ctx->d, M, ctx->d, ctx->x, h, gnext, eps, rm,
                                        ctx->stream);
        }
        capture_residual(ctx, l + 1, M, decode);
    }
    return WEDLM_OK;
}

// bf16 mode: every projection is one persistent tcgen05 GEMM with its epilogue
// fused (RoPE + K/V page scatter, residual add, SwiGLU); RMSNorm and attention
// are the only other kernels of a layer.
wedlm_status forward_bf16(wedlm_ctx* ctx, int slot_base, int n_entries, int stride, bool decode) {
    const int M = n_entries * stride;
    RowMap rm{slot_base, stride, ctx->ss.n};
    const float eps = ctx->cfg.rms_eps;
    bf16* h = (bf16*)ctx->h;
    bf16* qb = (bf16*)ctx->q;
    bf16* ao = (bf16*)ctx->attn_out;
    bf16* act = (bf16*)ctx->act;
    EpiParams base;
    base.check_rows = 1;
    base.rm = rm;
    base.rs = ctx->rs;
    base.ss = ctx->ss;
    base.kvl = ctx->kvl;
    base.kv_pool = (bf16*)ctx->kv_pool;
    base.hq = ctx->hq;
    base.hkv = ctx->hkv;
    base.rope_cs = ctx->rope_cs;
    base.rope_max_pos = ctx->max_ctx;
    wedlm_status s;
    capture_residual(ctx, 0, M, decode);
    for (int l = 0; l < ctx->L; ++l) {
        EpiParams e = base;
        e.layer = l;
        e.kind = EPI_QKV_ROPE;
        e.act = qb;
        if ((s = gemm_bf16(ctx, WEDLM_PROF_GEMM_QKV, h, &ctx->tm_qkv[l], M, ctx->Nqkv, ctx->d, e, decode))) return s;
        const int kc = decode ? ctx->attn_kv_chunk : (1 << 30);
        const int ms = decode ? ctx->attn_max_splits : 1;
        {
            ProfScope ps(ctx, WEDLM_PROF_ATTENTION);
            const cudaError_t ae =
                launch_attn_bf16(ctx->tm_kv, ctx->tm_q, ctx->tm_q_dual, ctx->kvl, l, ctx->hq, ctx->hkv, ao,
                                 ctx->attn_po, ctx->attn_pml, n_entries, stride, kc, ms, ctx->ss, rm,
                                 ctx->err, ctx->stream);
            if (ae != cudaSuccess)
                return fail(ctx, WEDLM_ERR_CUDA, std::string("attention launch: ") + cudaGetErrorString(ae));
        }
        e.kind = EPI_RESIDUAL;
        e.out = ctx->x;
        if ((s = gemm_bf16(ctx, WEDLM_PROF_GEMM_O, ao, &ctx->tm_o[l], M, ctx->d, ctx->hq * ctx->hd, e, decode))) return s;
        {
            ProfScope ps(ctx, WEDLM_PROF_RESIDUAL_NORM);
            launch_rmsnorm_bf16(ctx->x, h, ctx->ffn_norm[l], eps, M, ctx->d, rm, ctx->stream);
        }
        e.kind = EPI_SWIGLU;
        e.act = act;
        if ((s = gemm_bf16(ctx, WEDLM_PROF_GEMM_GATE_UP, h, &ctx->tm_gu[l], M, 2 * ctx->F, ctx->d, e, decode))) return s;
        e.kind = EPI_RESIDUAL;
        e.out = ctx->x;
        if ((s = gemm_bf16(ctx, WEDLM_PROF_GEMM_DOWN, act, &ctx->tm_d[l], M, ctx->d, ctx->F, e, decode))) return s;
        capture_residual(ctx, l + 1, M, decode);
        if (l + 1 == ctx->L) {
            // final norm: the LM head reads the masked rows only, packed (a
            // prefill has no LM head)
            if (!decode) break;
            MaskedRows mr;
            mr.nf = ctx->ss.nf;
            mr.row_map = ctx->lm_rows;
            mr.count = ctx->lm_count;
            mr.n_entries = n_entries;
            ProfScope ps(ctx, WEDLM_PROF_RESIDUAL_NORM);
            launch_rmsnorm_bf16(ctx->x, h, ctx->final_norm, eps, M, ctx->d, rm, ctx->stream, mr);
        } else {
            ProfScope ps(ctx, WEDLM_PROF_RESIDUAL_NORM);
            launch_rmsnorm_bf16(ctx->x, h, ctx->attn_norm[l + 1], eps, M, ctx->d, rm, ctx->stream);
        }
    }
    return WEDLM_OK;
}

wedlm_status run_forward(wedlm_ctx* ctx, int slot_base, int n_entries, int stride, bool decode) {
    return ctx->bf16 ? forward_bf16(ctx, slot_base, n_entries, stride, decode)
                     : forward_f32(ctx, slot_base, n_entries, stride, decode);
}

int max_active_window(const wedlm_ctx* c, int* n_entries) {
    int w = 0, last = -1;
    for (int b = 0; b < c->maxB; ++b)
        if (c->h_W[b] > 0 && c->h_S[b] < c->h_end[b]) {
            w = std::max(w, c->h_W[b]);
            last = b;
        }
    *n_entries = last + 1;
    return w;
}

// Enqueue one decode step over slots [0, n_entries) with row stride `stride`.
// LM head over the step's rows and the entropy partials of the masked rows:
// fused (the GEMM epilogue reduces each 32 vocab ids; one merge kernel) or
// two-pass (logits written, then one streaming scan, with sampling keys when
// the step samples).
wedlm_status lm_head_entropy(wedlm_ctx* ctx, const wedlm_step_params* prm, int M, int stride, bool fused) {
    wedlm_status s;
    if (fused) {
        EpiParams e;
        e.kind = EPI_ENTROPY;
        e.epart = ctx->lm_part;
        e.npart = ctx->lm_npart;
        e.mask_id = ctx->cfg.mask_id;
        e.scale = prm->logit_scale;
        e.m_count = ctx->lm_count;  // the packed masked rows (final norm)
        e.row_map = ctx->lm_rows;
        if ((s = gemm_bf16(ctx, WEDLM_PROF_GEMM_LM_HEAD, ctx->h, &ctx->tm_lm, M, ctx->V, ctx->d, e))) return s;
        ProfScope ps(ctx, WEDLM_PROF_ENTROPY);
        launch_entropy_merge(ctx->lm_part, ctx->lm_npart, ctx->rowmask, M, kEntropyChunks, ctx->ent_part,
                             ctx->stream);
        return WEDLM_OK;
    }
    if (ctx->bf16) {
        EpiParams e;
        e.kind = EPI_STORE;
        e.out = ctx->logits;
        e.m_count = ctx->lm_count;  // the packed masked rows (final norm)
        e.row_map = ctx->lm_rows;
        if ((s = gemm_bf16(ctx, WEDLM_PROF_GEMM_LM_HEAD, ctx->h, &ctx->tm_lm, M, ctx->V, ctx->d, e))) return s;
    } else {
        if ((size_t)M * ctx->V > ctx->logits_floats) return fail(ctx, WEDLM_ERR_STATE, "logits buffer too small");
        ProfScope ps(ctx, WEDLM_PROF_GEMM_LM_HEAD);
        launch_gemm_f32((const float*)ctx->h, (const float*)ctx->lm_head, ctx->logits, M, ctx->V, ctx->d,
                        ctx->stream);
    }
    ProfScope ps(ctx, WEDLM_PROF_ENTROPY);
    SampleArgs sa;
    if (prm->temperature > 0.f) {
        sa.inv_t = 1.0f / prm->temperature;
        sa.seed = prm->seed;
        sa.stride = stride;
        sa.pos = ctx->rs.pos;
        sa.steps = ctx->ss.counters;
        sa.part = ctx->samp_part;
    }
    launch_entropy_partials(ctx->logits, 1, (int64_t)M * ctx->V, ctx->V, ctx->V, ctx->cfg.mask_id, prm->logit_scale,
                            ctx->rowmask, M, kEntropyChunks, ctx->ent_part, ctx->stream, sa);
    return WEDLM_OK;
}

wedlm_status enqueue_step_kernels(wedlm_ctx* ctx, const wedlm_step_params* prm, int n_entries, int stride) {
    const int M = n_entries * stride;
    {
        ProfScope ps(ctx, WEDLM_PROF_PREPARE);
        if (ctx->bf16)
            launch_decode_prepare<bf16>((const bf16*)ctx->embed, ctx->attn_norm[0], ctx->cfg.rms_eps, ctx->d,
                                        ctx->cfg.mask_id, ctx->ss, ctx->rs, ctx->rowmask, n_entries, stride, ctx->x,
                                        (bf16*)ctx->h, prm->blockwise, ctx->stream);
        else
            launch_decode_prepare<float>((const float*)ctx->embed, ctx->attn_norm[0], ctx->cfg.rms_eps, ctx->d,
                                         ctx->cfg.mask_id, ctx->ss, ctx->rs, ctx->rowmask, n_entries, stride, ctx->x,
                                         (float*)ctx->h, prm->blockwise, ctx->stream);
    }
    wedlm_status s = run_forward(ctx, 0, n_entries, stride, true);
    if (s) return s;
    // Greedy bf16 steps may fuse the entropy into the LM head (logits never
    // stored); which of the two is faster at this row count is timed once
    // (autotuning on) or taken from the row count (off).  Sampling and the
    // logits test hook always take the two-pass path.
    const bool fusable = ctx->bf16 && !ctx->keep_logits && prm->temperature == 0.f;
    bool fused = false;
    if (fusable) {
        auto it = ctx->fuse_choice.find(M);
        if (ctx->force_fused) {
            it = ctx->fuse_choice.emplace(M, true).first;
            it->second = true;
        } else if (it == ctx->fuse_choice.end()) {
            bool choice = M <= 64;
            if (ctx->autotune && !ctx->capturing) {
                // both variants once to tune their GEMMs, then once more each, timed
                if ((s = lm_head_entropy(ctx, prm, M, stride, false)) || (s = lm_head_entropy(ctx, prm, M, stride, true)))
                    return s;
                cudaEvent_t e0, e1, e2;
                cudaEventCreate(&e0);
                cudaEventCreate(&e1);
                cudaEventCreate(&e2);
                cudaEventRecord(e0, ctx->stream);
                if ((s = lm_head_entropy(ctx, prm, M, stride, false))) return s;
                cudaEventRecord(e1, ctx->stream);
                if ((s = lm_head_entropy(ctx, prm, M, stride, true))) return s;
                cudaEventRecord(e2, ctx->stream);
                cudaEventSynchronize(e2);
                float t_two = 0.f, t_fused = 0.f;
                cudaEventElapsedTime(&t_two, e0, e1);
                cudaEventElapsedTime(&t_fused, e1, e2);
                cudaEventDestroy(e0);
                cudaEventDestroy(e1);
                cudaEventDestroy(e2);
                choice = t_fused < t_two;
            }
            it = ctx->fuse_choice.emplace(M, choice).first;
        }
        fused = it->second;
    }
    if ((s = lm_head_entropy(ctx, prm, M, stride, fused))) return s;
    StepKnobs kn{prm->lambda, prm->tau, prm->logit_scale, prm->tau_none, prm->blockwise, prm->temperature, prm->seed};
    {
        ProfScope ps(ctx, WEDLM_PROF_SELECT);
        launch_select_commit(ctx->ent_part, ctx->samp_part, kEntropyChunks, ctx->ss, ctx->rs, n_entries, stride, kn,
                             ctx->err,
                             ctx->stream);
    }
    ctx->last_stride = stride;
    ctx->last_M = M;
    {
        // launch-configuration errors of the void launch wrappers surface here
        const cudaError_t le = cudaGetLastError();
        if (le != cudaSuccess) return fail(ctx, WEDLM_ERR_CUDA, std::string("kernel launch: ") + cudaGetErrorString(le));
    }
    ctx->logits_splits_last = 1;
    if (ctx->prof && ctx->ev_marks.size() > 4096) prof_collect(ctx);
    return WEDLM_OK;
}

void drop_graph(wedlm_ctx* ctx) {
    if (ctx->graph_exec) cudaGraphExecDestroy(ctx->graph_exec);
    ctx->graph_exec = nullptr;
    ctx->graph_key = wedlm_ctx::StepKey();
}

// Enqueue one decode step.  A step whose shape and knobs were already run
// once is captured into a CUDA graph and replayed from then on (every
// per-step size is read from device memory, so the graph stays valid); the
// eager path is used on the legacy default stream and while profiling.
wedlm_status enqueue_step(wedlm_ctx* ctx, const wedlm_step_params* prm, int n_entries, int stride) {
    wedlm_ctx::StepKey key;
    key.n_entries = n_entries;
    key.stride = stride;
    key.tau_none = prm->tau_none;
    key.lambda = prm->lambda;
    key.tau = prm->tau;
    key.scale = prm->logit_scale;
    key.blockwise = prm->blockwise ? 1 : 0;
    key.temperature = prm->temperature;
    key.seed = prm->seed;
    const bool graphable = ctx->use_graphs && ctx->bf16 && ctx->stream != nullptr && !ctx->prof && !ctx->dbg_resid;
    if (graphable && ctx->graph_exec && ctx->graph_key == key) {
        cudaError_t e = cudaGraphLaunch(ctx->graph_exec, ctx->stream);
        if (e != cudaSuccess) return fail(ctx, WEDLM_ERR_CUDA, std::string("graph launch: ") + cudaGetErrorString(e));
        ctx->launches += ctx->graph_launches;
        return WEDLM_OK;
    }
    if (!graphable || !(ctx->eager_key == key)) {
        ctx->eager_key = key;
        return enqueue_step_kernels(ctx, prm, n_entries, stride);
    }
    drop_graph(ctx);
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamBeginCapture(ctx->stream, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return fail(ctx, WEDLM_ERR_CUDA, std::string("begin capture: ") + cudaGetErrorString(e));
    const int64_t l0 = ctx->launches;
    ctx->capturing = true;
    wedlm_status s = enqueue_step_kernels(ctx, prm, n_entries, stride);
    ctx->capturing = false;
    e = cudaStreamEndCapture(ctx->stream, &graph);
    if (s) {
        if (graph) cudaGraphDestroy(graph);
        return s;
    }
    if (e != cudaSuccess) return fail(ctx, WEDLM_ERR_CUDA, std::string("end capture: ") + cudaGetErrorString(e));
    e = cudaGraphInstantiate(&ctx->graph_exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) {
        ctx->graph_exec = nullptr;
        return fail(ctx, WEDLM_ERR_CUDA, std::string("graph instantiate: ") + cudaGetErrorString(e));
    }
    ctx->graph_launches = ctx->launches - l0;
    ctx->launches = l0;
    ctx->graph_key = key;
    e = cudaGraphLaunch(ctx->graph_exec, ctx->stream);
    if (e != cudaSuccess) return fail(ctx, WEDLM_ERR_CUDA, std::string("graph launch: ") + cudaGetErrorString(e));
    ctx->launches += ctx->graph_launches;
    return WEDLM_OK;
}

}  // namespace

extern "C" {

const char* wedlm_status_str(wedlm_status s) {
    switch (s) {
        case WEDLM_OK: return "ok";
        case WEDLM_ERR_INVALID_ARG: return "invalid argument";
        case WEDLM_ERR_OOM_PAGES: return "KV page pool exhausted";
        case WEDLM_ERR_OOM_DEVICE: return "device out of memory";
        case WEDLM_ERR_CUDA: return "CUDA error";
        case WEDLM_ERR_DEVICE_ASSERT: return "device bounds check fired";
        case WEDLM_ERR_STATE: return "invalid state for this call";
        case WEDLM_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case WEDLM_ERR_TIMEOUT: return "bounded device wait timed out";
        case WEDLM_ERR_NONFINITE: return "non-finite logits in a masked slot";
        default: return "unknown status";
    }
}

const char* wedlm_last_error(const wedlm_ctx* ctx) { return ctx ? ctx->last_error.c_str() : ""; }

}  // extern "C"

// ===========================================================================
// Context lifetime, weights, sequences, decode step.
namespace {

bool valid_cfg(const wedlm_model_cfg* c, std::string* why) {
    auto bad = [&](const char* m) {
        *why = m;
        return false;
    };
    if (c->n_layers <= 0 || c->d_model <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
        c->ffn_dim <= 0 || c->vocab <= 1)
        return bad("model dimensions must be positive");
    if (c->n_heads % c->n_kv_heads) return bad("n_heads must be a multiple of n_kv_heads");
    if (c->head_dim % 2) return bad("head_dim must be even");
    if (c->mask_id < 0 || c->mask_id >= c->vocab) return bad("mask_id out of range");
    if (!(c->rope_theta > 0.0) || !(c->rms_eps >= 0.f)) return bad("rope_theta must be > 0 and rms_eps >= 0");
    if (c->max_batch <= 0 || c->max_batch > 4096) return bad("max_batch must be in [1, 4096]");
    if (c->max_window <= 0 || c->max_window > kMaxWindow) return bad("max_window must be in [1, 64]");
    if (c->max_ctx <= 0) return bad("max_ctx must be positive");
    if (c->num_pages < 0 || c->prefill_chunk < 0) return bad("num_pages / prefill_chunk must be >= 0");
    if (c->dtype == WEDLM_DTYPE_F32) {
        if (c->head_dim % 32 || c->head_dim > 128) return bad("fp32 mode needs head_dim a multiple of 32, <= 128");
    } else if (c->dtype == WEDLM_DTYPE_BF16) {
        if (c->head_dim != 128) return bad("bf16 mode needs head_dim 128");
        if (c->d_model % 8 || c->ffn_dim % 8) return bad("bf16 mode needs d_model and ffn_dim multiples of 8");
        if (c->d_model > 8192) return bad("bf16 mode supports d_model <= 8192");
    } else {
        return bad("unknown dtype");
    }
    return true;
}

}  // namespace

extern "C" {

wedlm_status wedlm_create(const wedlm_model_cfg* cfg, void* cuda_stream, wedlm_ctx** out_ctx) {
    if (!cfg || !out_ctx) return WEDLM_ERR_INVALID_ARG;
    *out_ctx = nullptr;
    std::string why;
    if (!valid_cfg(cfg, &why)) return WEDLM_ERR_INVALID_ARG;
    wedlm_ctx* ctx = new wedlm_ctx();
    ctx->cfg = *cfg;
    ctx->stream = (cudaStream_t)cuda_stream;
    ctx->bf16 = cfg->dtype == WEDLM_DTYPE_BF16;
    ctx->elt = ctx->bf16 ? 2 : 4;
    auto bail = [&](wedlm_status s) {
        ctx->weights_arena.release();
        ctx->state_arena.release();
        ctx->scratch_arena.release();
        if (ctx->res_host) cudaFreeHost(ctx->res_host);
        delete ctx;
        return s;
    };
    if (cudaGetDevice(&ctx->device) != cudaSuccess) return bail(WEDLM_ERR_CUDA);
    cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device);
    ctx->L = cfg->n_layers;
    ctx->d = cfg->d_model;
    ctx->hq = cfg->n_heads;
    ctx->hkv = cfg->n_kv_heads;
    ctx->hd = cfg->head_dim;
    ctx->F = cfg->ffn_dim;
    ctx->V = cfg->vocab;
    ctx->Nqkv = (ctx->hq + 2 * ctx->hkv) * ctx->hd;
    ctx->maxB = cfg->max_batch;
    ctx->maxW = cfg->max_window;
    ctx->max_ctx = cfg->max_ctx;
    ctx->pages_per_seq = (cfg->max_ctx + kPage - 1) / kPage;
    ctx->num_pages = cfg->num_pages ? cfg->num_pages : ctx->maxB * ctx->pages_per_seq;
    ctx->chunk = cfg->prefill_chunk ? cfg->prefill_chunk : 1024;
    ctx->Mdec = ctx->maxB * ctx->maxW;
    ctx->Mmax = std::max(ctx->Mdec, ctx->chunk);
    const size_t elt = ctx->elt;
    const int L = ctx->L, d = ctx->d, F = ctx->F, V = ctx->V;
    const int B = ctx->maxB, maxW = ctx->maxW, Mmax = ctx->Mmax;

    // Weights.
    Arena& wa = ctx->weights_arena;
    ctx->attn_norm.assign(L, nullptr);
    ctx->ffn_norm.assign(L, nullptr);
    ctx->wqkv.assign(L, nullptr);
    ctx->wo.assign(L, nullptr);
    ctx->wgu.assign(L, nullptr);
    ctx->wd.assign(L, nullptr);
    wa.add(&ctx->embed, (size_t)V * d * elt);
    wa.add(&ctx->lm_head, (size_t)V * d * elt);
    wa.add((void**)&ctx->final_norm, (size_t)d * 4);
    for (int l = 0; l < L; ++l) {
        wa.add((void**)&ctx->attn_norm[l], (size_t)d * 4);
        wa.add((void**)&ctx->ffn_norm[l], (size_t)d * 4);
        wa.add(&ctx->wqkv[l], (size_t)ctx->Nqkv * d * elt);
        wa.add(&ctx->wo[l], (size_t)d * ctx->hq * ctx->hd * elt);
        wa.add(&ctx->wgu[l], (size_t)2 * F * d * elt);
        wa.add(&ctx->wd[l], (size_t)d * F * elt);
    }
    if (wa.commit(ctx->stream) != cudaSuccess) return bail(WEDLM_ERR_OOM_DEVICE);
    ctx->loaded.assign(3 + 9 * L, 0);

    // KV pool, rope table, slot and row state, step-result block.
    const int64_t page_elems = (int64_t)2 * ctx->hkv * kPage * ctx->hd;
    ctx->kvl.layer_stride = (int64_t)ctx->num_pages * page_elems;
    ctx->kvl.hkv = ctx->hkv;
    ctx->kvl.hd = ctx->hd;
    ctx->kvl.num_pages = ctx->num_pages;
    Arena& sa = ctx->state_arena;
    sa.add(&ctx->kv_pool, (size_t)L * ctx->kvl.layer_stride * elt);
    sa.add((void**)&ctx->rope_cs, (size_t)ctx->max_ctx * (ctx->hd / 2) * sizeof(float2));
    SlotState& ss = ctx->ss;
    const size_t res_ints = (size_t)2 * B + (size_t)B * maxW + 1;
    sa.add((void**)&ctx->res_dev, res_ints * 4);
    sa.add((void**)&ss.end, B * 4);
    sa.add((void**)&ss.P, B * 4);
    sa.add((void**)&ss.W, B * 4);
    sa.add((void**)&ss.wlen, B * 4);
    sa.add((void**)&ss.n, B * 4);
    sa.add((void**)&ss.k, B * 4);
    sa.add((void**)&ss.nf, B * 4);
    sa.add((void**)&ss.filled, (size_t)B * maxW);
    sa.add((void**)&ss.token, (size_t)B * maxW * 4);
    sa.add((void**)&ss.page_table, (size_t)B * ctx->pages_per_seq * 4);
    sa.add((void**)&ss.counters, (size_t)B * 4 * 8);
    sa.add((void**)&ss.gen, (size_t)B * ctx->max_ctx * 4);
    sa.add((void**)&ss.htilde, (size_t)B * maxW * 4);
    sa.add((void**)&ss.amax, (size_t)B * maxW * 4);
    sa.add((void**)&ss.fillflag, (size_t)B * maxW);
    sa.add((void**)&ctx->rs.pos, (size_t)Mmax * 4);
    sa.add((void**)&ctx->rs.tok, (size_t)Mmax * 4);
    sa.add((void**)&ctx->rs.perm, (size_t)Mmax * 4);
    sa.add((void**)&ctx->rowmask, (size_t)Mmax);
    sa.add((void**)&ctx->lm_rows, (size_t)ctx->Mdec * 4);
    sa.add((void**)&ctx->lm_count, 4);
    sa.add((void**)&ctx->ids_dev, (size_t)ctx->chunk * 4);
    // Attention key chunks for decode: fixed per context (a sequence's result
    // does not depend on its batch neighbours).
    if (ctx->bf16) {
        ctx->attn_kv_chunk = attn_kv_chunk_for(B, maxW, ctx->hq, ctx->hkv, ctx->max_ctx, ctx->num_sms);
        ctx->attn_max_splits = (ctx->max_ctx + ctx->attn_kv_chunk - 1) / ctx->attn_kv_chunk;
    }
    if (sa.commit(ctx->stream) != cudaSuccess) return bail(WEDLM_ERR_OOM_DEVICE);
    ss.out_count = ctx->res_dev;
    ss.S = ctx->res_dev + B;
    ss.out_tokens = ctx->res_dev + 2 * B;
    ctx->err = ctx->res_dev + 2 * B + (size_t)B * maxW;
    ss.pages_per_seq = ctx->pages_per_seq;
    ss.maxW = maxW;
    ss.gen_cap = ctx->max_ctx;
    if (cudaMallocHost((void**)&ctx->res_host, res_ints * 4) != cudaSuccess) return bail(WEDLM_ERR_OOM_DEVICE);

    if (ctx->bf16 && !make_kv_tmap(&ctx->tm_kv, (const bf16*)ctx->kv_pool, ctx->kvl, L)) return bail(WEDLM_ERR_CUDA);

    // Scratch.
    Arena& xa = ctx->scratch_arena;
    xa.add((void**)&ctx->x, (size_t)Mmax * d * 4);
    xa.add(&ctx->h, (size_t)Mmax * d * elt);
    xa.add(&ctx->q, (size_t)Mmax * ctx->hq * ctx->hd * elt);
    xa.add(&ctx->attn_out, (size_t)Mmax * ctx->hq * ctx->hd * elt);
    xa.add(&ctx->act, (size_t)Mmax * F * elt);
    size_t need = 0, tiles = 0;
    if (ctx->bf16) {
        for (int M : {ctx->Mdec, ctx->chunk}) {
            const int ms = M == ctx->Mdec ? 16 : 4;
            gemm_needs(ctx, M, ctx->Nqkv, d, ms, &need, &tiles);
            gemm_needs(ctx, M, d, ctx->hq * ctx->hd, ms, &need, &tiles);
            gemm_needs(ctx, M, 2 * F, d, std::min(ms, 8), &need, &tiles);
            gemm_needs(ctx, M, d, F, ms, &need, &tiles);
        }
        gemm_needs(ctx, ctx->Mdec, V, d, 2, &need, &tiles);
    } else {
        need = (size_t)Mmax * std::max({(size_t)ctx->Nqkv, (size_t)2 * F, (size_t)d});
    }
    ctx->ws_floats = std::max<size_t>(need, 1);
    ctx->n_tile_counters = std::max<size_t>(tiles, 1);
    xa.add((void**)&ctx->ws, ctx->ws_floats * 4);
    xa.add((void**)&ctx->tile_counters, ctx->n_tile_counters * 4);
    ctx->logits_floats = (size_t)ctx->Mdec * (size_t)V;
    xa.add((void**)&ctx->logits, ctx->logits_floats * 4);
    xa.add((void**)&ctx->ent_part, (size_t)ctx->Mdec * kEntropyChunks * sizeof(float4));
    if (ctx->bf16) {
        xa.add(&ctx->evict, kEvictBytes);
        xa.add((void**)&ctx->evict_sink, sizeof(float));
    }
    xa.add((void**)&ctx->samp_part, (size_t)ctx->Mdec * kEntropyChunks * sizeof(float2));
    if (ctx->bf16) {
        ctx->lm_npart = ((V + 255) / 256) * 2 * 4;  // 4 per 128 vocab rows, for 128- or 256-row tiles
        xa.add((void**)&ctx->lm_part, (size_t)ctx->Mdec * ctx->lm_npart * sizeof(float4));
    }
    if (ctx->bf16 && ctx->attn_max_splits > 1) {
        const size_t pairs = (size_t)ctx->Mdec * ctx->hq * ctx->attn_max_splits;
        xa.add((void**)&ctx->attn_po, pairs * ctx->hd * 4);
        xa.add((void**)&ctx->attn_pml, pairs * sizeof(float2));
    }
    if (xa.commit(ctx->stream) != cudaSuccess) return bail(WEDLM_ERR_OOM_DEVICE);
    if (ctx->bf16 && !(make_q_tmap(&ctx->tm_q, (const bf16*)ctx->q, Mmax, ctx->hq, ctx->hkv, false) &&
                       make_q_tmap(&ctx->tm_q_dual, (const bf16*)ctx->q, Mmax, ctx->hq, ctx->hkv, true)))
        return bail(WEDLM_ERR_CUDA);

    launch_rope_table(ctx->rope_cs, ctx->max_ctx, ctx->hd / 2, ctx->hd, cfg->rope_theta, ctx->stream);
    if (ctx->lm_part) {
        // Partial i always covers vocab ids [32 i, 32 i + 32) whatever the tile
        // shape; those past the vocabulary, which a narrow-tile plan never
        // writes, must read as empty (max -inf, sums 0, no argmax).
        const int32_t no_id = INT32_MAX;
        float no_id_bits;
        std::memcpy(&no_id_bits, &no_id, 4);
        const float4 empty = make_float4(-INFINITY, 0.f, 0.f, no_id_bits);
        std::vector<float4> fill((size_t)ctx->Mdec * ctx->lm_npart, empty);
        if (cudaMemcpyAsync(ctx->lm_part, fill.data(), fill.size() * sizeof(float4), cudaMemcpyHostToDevice,
                            ctx->stream) != cudaSuccess ||
            cudaStreamSynchronize(ctx->stream) != cudaSuccess)
            return bail(WEDLM_ERR_CUDA);
    }
    std::vector<int32_t> pt((size_t)B * ctx->pages_per_seq, -1);
    if (cudaMemcpyAsync(ss.page_table, pt.data(), pt.size() * 4, cudaMemcpyHostToDevice, ctx->stream) != cudaSuccess ||
        cudaStreamSynchronize(ctx->stream) != cudaSuccess)
        return bail(WEDLM_ERR_CUDA);
    if (cudaGetLastError() != cudaSuccess) return bail(WEDLM_ERR_CUDA);  // e.g. the RoPE table launch
    if (cudaDeviceSynchronize() != cudaSuccess) return bail(WEDLM_ERR_CUDA);
    ctx->h_W.assign(B, 0);
    ctx->h_S.assign(B, 0);
    ctx->h_end.assign(B, 0);
    ctx->h_P.assign(B, 0);
    ctx->h_pages.assign(B, {});
    ctx->free_pages.resize(ctx->num_pages);
    for (int i = 0; i < ctx->num_pages; ++i) ctx->free_pages[i] = ctx->num_pages - 1 - i;
    *out_ctx = ctx;
    return WEDLM_OK;
}

void wedlm_destroy(wedlm_ctx* ctx) {
    if (!ctx) return;
    if (ctx->stream) cudaStreamSynchronize(ctx->stream);
    else cudaDeviceSynchronize();
    ctx->weights_arena.release();
    ctx->state_arena.release();
    ctx->scratch_arena.release();
    if (ctx->dbg_resid) cudaFree(ctx->dbg_resid);
    if (ctx->res_host) cudaFreeHost(ctx->res_host);
    for (cudaEvent_t e : ctx->ev_pool) cudaEventDestroy(e);
    drop_graph(ctx);
    delete ctx;
}

wedlm_status wedlm_load_weights(wedlm_ctx* ctx, int32_t tensor, int32_t layer, const void* src, int32_t src_dtype,
                                int32_t src_mem) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (!src) return fail(ctx, WEDLM_ERR_INVALID_ARG, "null source");
    if (src_mem != WEDLM_MEM_HOST && src_mem != WEDLM_MEM_DEVICE)
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad src_mem");
    const int slot = tensor_slot(ctx, tensor, layer);
    if (slot < 0) return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad tensor id or layer");
    const bool norm = tensor == WEDLM_T_FINAL_NORM || tensor == WEDLM_T_ATTN_NORM || tensor == WEDLM_T_FFN_NORM;
    const int want = norm ? WEDLM_DTYPE_F32 : ctx->cfg.dtype;
    if (src_dtype != want) return fail(ctx, WEDLM_ERR_INVALID_ARG, "source dtype does not match the tensor's dtype");
    const size_t elt = ctx->elt;
    const size_t d = ctx->d, qd = (size_t)ctx->hq * ctx->hd, kd = (size_t)ctx->hkv * ctx->hd, F = ctx->F;
    char* dst = nullptr;
    size_t bytes = 0;
    switch (tensor) {
        case WEDLM_T_EMBED: dst = (char*)ctx->embed; bytes = (size_t)ctx->V * d * elt; break;
        case WEDLM_T_LM_HEAD: dst = (char*)ctx->lm_head; bytes = (size_t)ctx->V * d * elt; break;
        case WEDLM_T_FINAL_NORM: dst = (char*)ctx->final_norm; bytes = d * 4; break;
        case WEDLM_T_ATTN_NORM: dst = (char*)ctx->attn_norm[layer]; bytes = d * 4; break;
        case WEDLM_T_FFN_NORM: dst = (char*)ctx->ffn_norm[layer]; bytes = d * 4; break;
        case WEDLM_T_WQ: dst = (char*)ctx->wqkv[layer]; bytes = qd * d * elt; break;
        case WEDLM_T_WK: dst = (char*)ctx->wqkv[layer] + qd * d * elt; bytes = kd * d * elt; break;
        case WEDLM_T_WV: dst = (char*)ctx->wqkv[layer] + (qd + kd) * d * elt; bytes = kd * d * elt; break;
        case WEDLM_T_WO: dst = (char*)ctx->wo[layer]; bytes = d * qd * elt; break;
        case WEDLM_T_WG: dst = (char*)ctx->wgu[layer]; bytes = F * d * elt; break;
        case WEDLM_T_WU: dst = (char*)ctx->wgu[layer] + F * d * elt; bytes = F * d * elt; break;
        case WEDLM_T_WD: dst = (char*)ctx->wd[layer]; bytes = d * F * elt; break;
        default: return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad tensor id");
    }
    const cudaMemcpyKind kind = src_mem == WEDLM_MEM_HOST ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice;
    const size_t row = d * elt;
    if (ctx->bf16 && (tensor == WEDLM_T_WQ || tensor == WEDLM_T_WK)) {
        // Rows of each 128-dim head are stored with RoPE partners adjacent
        // (row 2i = dim i, row 2i+1 = dim i+64) so the fused GEMM epilogue
        // rotates a pair within one warp; outputs return to natural order.
        const int heads = tensor == WEDLM_T_WQ ? ctx->hq : ctx->hkv;
        for (int hh = 0; hh < heads; ++hh) {
            char* hd0 = dst + (size_t)hh * 128 * row;
            const char* hs0 = (const char*)src + (size_t)hh * 128 * row;
            CK(cudaMemcpy2DAsync(hd0, 2 * row, hs0, row, row, 64, kind, ctx->stream));
            CK(cudaMemcpy2DAsync(hd0 + row, 2 * row, hs0 + 64 * row, row, row, 64, kind, ctx->stream));
        }
    } else if (ctx->bf16 && (tensor == WEDLM_T_WG || tensor == WEDLM_T_WU)) {
        // Gate row c -> row 2c, up row c -> row 2c+1 of the fused gate/up
        // matrix, so SwiGLU pairs sit in adjacent rows of one GEMM tile.
        char* base = (char*)ctx->wgu[layer] + (tensor == WEDLM_T_WU ? row : 0);
        CK(cudaMemcpy2DAsync(base, 2 * row, src, row, row, F, kind, ctx->stream));
    } else {
        CK(cudaMemcpyAsync(dst, src, bytes, kind, ctx->stream));
    }
    CK(cudaStreamSynchronize(ctx->stream));
    ctx->loaded[slot] = 1;
    drop_graph(ctx);
    bool all = true;
    for (uint8_t f : ctx->loaded) all &= f != 0;
    ctx->weights_ready = all;
    ctx->maps_ready = false;
    return WEDLM_OK;
}

wedlm_status wedlm_prefill(wedlm_ctx* ctx, int32_t slot, const int32_t* prompt_ids, int32_t prompt_len,
                           int32_t max_new_tokens, int32_t window) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < 0 || slot >= ctx->maxB) return fail(ctx, WEDLM_ERR_INVALID_ARG, "slot out of range");
    if (prompt_len < 0 || (prompt_len > 0 && !prompt_ids)) return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad prompt");
    if (max_new_tokens < 1 || (int64_t)prompt_len + max_new_tokens > ctx->max_ctx)
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "prompt_len + max_new_tokens must be in [1, max_ctx]");
    if (window < 1 || window > ctx->maxW) return fail(ctx, WEDLM_ERR_INVALID_ARG, "window out of range");
    if (!ctx->weights_ready) return fail(ctx, WEDLM_ERR_STATE, "weights not fully loaded");
    if (ctx->h_W[slot] != 0) return fail(ctx, WEDLM_ERR_STATE, "slot is in use (call wedlm_kv_reset)");
    drop_graph(ctx);
    for (int i = 0; i < prompt_len; ++i)
        if (prompt_ids[i] < 0 || prompt_ids[i] >= ctx->V)
            return fail(ctx, WEDLM_ERR_INVALID_ARG, "prompt id out of range");
    const int end = prompt_len + max_new_tokens;
    const int need = (end + kPage - 1) / kPage;
    if ((int)ctx->free_pages.size() < need) return fail(ctx, WEDLM_ERR_OOM_PAGES, "KV page pool exhausted");
    wedlm_status s = build_weight_maps(ctx);
    if (s) return s;
    std::vector<int32_t> row(ctx->pages_per_seq, -1);
    std::vector<int> taken;
    for (int i = 0; i < need; ++i) {
        taken.push_back(ctx->free_pages.back());
        ctx->free_pages.pop_back();
        row[i] = taken.back();
    }
    auto give_back = [&]() {
        for (int p : taken) ctx->free_pages.push_back(p);
    };
    cudaError_t e = cudaMemcpyAsync(ctx->ss.page_table + (size_t)slot * ctx->pages_per_seq, row.data(),
                                    row.size() * 4, cudaMemcpyHostToDevice, ctx->stream);
    if (e != cudaSuccess) {
        give_back();
        return fail(ctx, WEDLM_ERR_CUDA, cudaGetErrorString(e));
    }
    launch_slot_admit(ctx->ss, slot, prompt_len, end, window, ctx->stream);
    ctx->launches++;
    for (int c0 = 0; c0 < prompt_len; c0 += ctx->chunk) {
        const int n = std::min(ctx->chunk, prompt_len - c0);
        e = cudaMemcpyAsync(ctx->ids_dev, prompt_ids + c0, (size_t)n * 4, cudaMemcpyHostToDevice, ctx->stream);
        if (e != cudaSuccess) {
            give_back();
            return fail(ctx, WEDLM_ERR_CUDA, cudaGetErrorString(e));
        }
        if (ctx->bf16)
            launch_prefill_prepare<bf16>((const bf16*)ctx->embed, ctx->attn_norm[0], ctx->cfg.rms_eps, ctx->d,
                                         ctx->ids_dev, slot, c0, n, ctx->ss, ctx->rs, ctx->x, (bf16*)ctx->h,
                                         ctx->stream);
        else
            launch_prefill_prepare<float>((const float*)ctx->embed, ctx->attn_norm[0], ctx->cfg.rms_eps, ctx->d,
                                          ctx->ids_dev, slot, c0, n, ctx->ss, ctx->rs, ctx->x, (float*)ctx->h,
                                          ctx->stream);
        ctx->launches++;
        s = run_forward(ctx, slot, 1, n, false);
        if (s) {
            give_back();
            return s;
        }
        // the ids buffer is reused by the next chunk: wait for this one
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
        if (e != cudaSuccess) {
            give_back();
            return fail(ctx, WEDLM_ERR_CUDA, cudaGetErrorString(e));
        }
    }
    launch_prefill_finish(ctx->ss, slot, prompt_len, ctx->stream);
    ctx->launches++;
    int errw = 0;
    CK(cudaMemcpyAsync(&errw, ctx->err, 4, cudaMemcpyDeviceToHost, ctx->stream));
    CK(cudaStreamSynchronize(ctx->stream));
    s = check_device_error(ctx, errw);
    if (s) {
        give_back();
        launch_slot_admit(ctx->ss, slot, 0, 0, 0, ctx->stream);
        return s;
    }
    ctx->h_pages[slot] = taken;
    ctx->h_W[slot] = window;
    ctx->h_S[slot] = prompt_len;
    ctx->h_end[slot] = end;
    ctx->h_P[slot] = prompt_len;
    return WEDLM_OK;
}

wedlm_status wedlm_kv_reset(wedlm_ctx* ctx, int32_t slot) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < -1 || slot >= ctx->maxB) return fail(ctx, WEDLM_ERR_INVALID_ARG, "slot out of range");
    CK(cudaStreamSynchronize(ctx->stream));
    for (int b = 0; b < ctx->maxB; ++b) {
        if (slot != -1 && b != slot) continue;
        for (int p : ctx->h_pages[b]) ctx->free_pages.push_back(p);
        ctx->h_pages[b].clear();
        ctx->h_W[b] = ctx->h_S[b] = ctx->h_end[b] = ctx->h_P[b] = 0;
        launch_slot_admit(ctx->ss, b, 0, 0, 0, ctx->stream);
        ctx->launches++;
        std::vector<int32_t> row(ctx->pages_per_seq, -1);
        CK(cudaMemcpyAsync(ctx->ss.page_table + (size_t)b * ctx->pages_per_seq, row.data(), row.size() * 4,
                           cudaMemcpyHostToDevice, ctx->stream));
        CK(cudaStreamSynchronize(ctx->stream));
    }
    return WEDLM_OK;
}

static wedlm_status check_params(wedlm_ctx* ctx, const wedlm_step_params* p) {
    if (!p) return fail(ctx, WEDLM_ERR_INVALID_ARG, "null params");
    if (!(p->logit_scale > 0.f) || !std::isfinite(p->logit_scale) || std::isnan(p->lambda) || std::isnan(p->tau))
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "logit_scale must be finite and > 0; lambda, tau not NaN");
    if (!(p->temperature >= 0.f) || !std::isfinite(p->temperature))
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "temperature must be finite and >= 0");
    if (!ctx->weights_ready) return fail(ctx, WEDLM_ERR_STATE, "weights not fully loaded");
    return WEDLM_OK;
}

wedlm_status wedlm_stream_step(wedlm_ctx* ctx, const wedlm_step_params* prm, int32_t* out_committed,
                               int32_t* out_counts, int32_t* out_active) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    wedlm_status s = check_params(ctx, prm);
    if (s) return s;
    const int B = ctx->maxB, maxW = ctx->maxW;
    int n_entries = 0;
    const int stride = max_active_window(ctx, &n_entries);
    if (n_entries == 0) {
        if (out_counts) std::memset(out_counts, 0, B * 4);
        if (out_active) *out_active = 0;
        return WEDLM_OK;
    }
    s = enqueue_step(ctx, prm, n_entries, stride);
    if (s) return s;
    const size_t res_ints = (size_t)2 * B + (size_t)B * maxW + 1;
    CK(cudaMemcpyAsync(ctx->res_host, ctx->res_dev, res_ints * 4, cudaMemcpyDeviceToHost, ctx->stream));
    CK(cudaStreamSynchronize(ctx->stream));
    const int32_t* counts = ctx->res_host;
    const int32_t* S = ctx->res_host + B;
    const int32_t* toks = ctx->res_host + 2 * B;
    const int errw = ctx->res_host[res_ints - 1];
    s = check_device_error(ctx, errw);
    if (s) return s;
    int active = 0;
    for (int b = 0; b < B; ++b) {
        if (ctx->h_W[b] > 0) {
            ctx->h_S[b] = S[b];
            if (S[b] < ctx->h_end[b]) ++active;
        }
    }
    if (out_counts) std::memcpy(out_counts, counts, (size_t)B * 4);
    if (out_committed) std::memcpy(out_committed, toks, (size_t)B * maxW * 4);
    if (out_active) *out_active = active;
    return WEDLM_OK;
}

wedlm_status wedlm_stream_step_async(wedlm_ctx* ctx, const wedlm_step_params* prm, int32_t n_steps) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    wedlm_status s = check_params(ctx, prm);
    if (s) return s;
    if (n_steps < 0) return fail(ctx, WEDLM_ERR_INVALID_ARG, "n_steps < 0");
    int n_entries = 0;
    const int stride = max_active_window(ctx, &n_entries);
    if (n_entries == 0) return WEDLM_OK;
    for (int i = 0; i < n_steps; ++i) {
        s = enqueue_step(ctx, prm, n_entries, stride);
        if (s) return s;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ctx, WEDLM_ERR_CUDA, cudaGetErrorString(e));
    return WEDLM_OK;
}

static wedlm_status refresh_mirrors(wedlm_ctx* ctx) {
    const int B = ctx->maxB, maxW = ctx->maxW;
    const size_t res_ints = (size_t)2 * B + (size_t)B * maxW + 1;
    CK(cudaMemcpyAsync(ctx->res_host, ctx->res_dev, res_ints * 4, cudaMemcpyDeviceToHost, ctx->stream));
    CK(cudaStreamSynchronize(ctx->stream));
    for (int b = 0; b < B; ++b)
        if (ctx->h_W[b] > 0) ctx->h_S[b] = ctx->res_host[B + b];
    return check_device_error(ctx, ctx->res_host[res_ints - 1]);
}

wedlm_status wedlm_read_generated(wedlm_ctx* ctx, int32_t slot, int32_t* out_tokens, int32_t cap, int32_t* out_len) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < 0 || slot >= ctx->maxB || !out_len || cap < 0 || (cap > 0 && !out_tokens))
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad slot or buffer");
    wedlm_status s = refresh_mirrors(ctx);
    if (s) return s;
    const int len = ctx->h_W[slot] > 0 ? ctx->h_S[slot] - ctx->h_P[slot] : 0;
    *out_len = len;
    const int n = std::min(len, cap);
    if (n > 0) {
        CK(cudaMemcpy(out_tokens, ctx->ss.gen + (size_t)slot * ctx->max_ctx, (size_t)n * 4, cudaMemcpyDeviceToHost));
    }
    return WEDLM_OK;
}

wedlm_status wedlm_get_stats(wedlm_ctx* ctx, int32_t slot, wedlm_seq_stats* out) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < 0 || slot >= ctx->maxB || !out) return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad slot or output");
    wedlm_status s = refresh_mirrors(ctx);
    if (s) return s;
    int64_t c[4];
    CK(cudaMemcpy(c, ctx->ss.counters + (size_t)slot * 4, sizeof(c), cudaMemcpyDeviceToHost));
    out->steps = c[0];
    out->forward_rows = c[1];
    out->committed = c[2];
    out->fills = c[3];
    out->committed_len = ctx->h_S[slot];
    out->end = ctx->h_end[slot];
    out->window = ctx->h_W[slot];
    out->active = (ctx->h_W[slot] > 0 && ctx->h_S[slot] < ctx->h_end[slot]) ? 1 : 0;
    return WEDLM_OK;
}

wedlm_status wedlm_profile_enable(wedlm_ctx* ctx, int32_t on) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    prof_collect(ctx);
    ctx->prof = on != 0;
    for (int i = 0; i < WEDLM_PROF_KINDS; ++i) {
        ctx->prof_ms[i] = 0.0;
        ctx->prof_n[i] = 0;
    }
    return WEDLM_OK;
}

wedlm_status wedlm_profile_read(wedlm_ctx* ctx, double* ms, int64_t* launches) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    prof_collect(ctx);
    for (int i = 0; i < WEDLM_PROF_KINDS; ++i) {
        if (ms) ms[i] = ctx->prof_ms[i];
        if (launches) launches[i] = ctx->prof_n[i];
    }
    return WEDLM_OK;
}

wedlm_status wedlm_autotune(wedlm_ctx* ctx, int32_t enable) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    ctx->autotune = enable != 0;
    ctx->tuned.clear();
    ctx->fuse_choice.clear();
    drop_graph(ctx);
    ctx->eager_key = wedlm_ctx::StepKey();
    return WEDLM_OK;
}

wedlm_status wedlm_gemm_plan(wedlm_ctx* ctx, int32_t kind, int32_t rows, int32_t* tile_w, int32_t* tile_n,
                             int32_t* k_splits, float* us) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    auto it = ctx->tuned.find({kind, rows});
    if (it == ctx->tuned.end()) return fail(ctx, WEDLM_ERR_STATE, "no plan recorded for this kind and row count");
    if (tile_w) *tile_w = 128 * it->second.plan.wt * it->second.plan.cg;
    if (tile_n) *tile_n = it->second.plan.bn;
    if (k_splits) *k_splits = it->second.plan.splits;
    if (us) *us = it->second.us;
    return WEDLM_OK;
}

wedlm_status wedlm_debug_set_plan(wedlm_ctx* ctx, int32_t kind, int32_t rows, int32_t tile_n, int32_t k_splits,
                                  int32_t schedule) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (!ctx->bf16) return fail(ctx, WEDLM_ERR_UNSUPPORTED, "GEMM plans exist in bf16 mode only");
    int N = 0, K = 0;
    switch (kind) {
        case WEDLM_PROF_GEMM_QKV: N = ctx->Nqkv; K = ctx->d; break;
        case WEDLM_PROF_GEMM_O: N = ctx->d; K = ctx->hq * ctx->hd; break;
        case WEDLM_PROF_GEMM_GATE_UP: N = 2 * ctx->F; K = ctx->d; break;
        case WEDLM_PROF_GEMM_DOWN: N = ctx->d; K = ctx->F; break;
        case WEDLM_PROF_GEMM_LM_HEAD: N = ctx->V; K = ctx->d; break;
        default: return fail(ctx, WEDLM_ERR_INVALID_ARG, "kind is not a GEMM kind");
    }
    if (rows < 1 || rows > ctx->Mmax || k_splits < 1 || k_splits > 16 || (schedule & ~127) ||
        (tile_n != 16 && tile_n != 32 && tile_n != 64 && tile_n != 128 && tile_n != 256))
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad rows, tile_n, k_splits or schedule");
    const bool entropy = (schedule & 64) != 0;
    if (entropy && (kind != WEDLM_PROF_GEMM_LM_HEAD || k_splits != 1))
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "the entropy epilogue is the LM head's, over whole K");
    const int cg = (schedule & 1) ? 2 : 1, hy = (schedule & 2) ? 1 : 0, ck = (schedule & 4) ? 1 : 0;
    const int coop = (schedule & 8) ? 1 : 0, wt = (schedule & 16) ? 2 : 1, bk = (schedule & 32) ? 32 : 64;
    GemmPlan p = plan_gemm_bf16(rows, N, K, ctx->num_sms, 16, tile_n, k_splits, wt, bk, coop, cg, hy, ck);
    const bool same = p.bn == tile_n && p.splits == k_splits && p.cg == cg && p.wt == wt && p.bk == bk &&
                      (p.ks > 1) == (ck != 0) && (p.hybrid != 0) == (hy != 0) &&
                      (k_splits == 1 || cg == 2 || hy || ck || p.coop == coop);
    if (!same) return fail(ctx, WEDLM_ERR_INVALID_ARG, "the launch shape cannot be built as asked");
    if (p.splits > 1 && ((size_t)p.splits * rows * N > ctx->ws_floats ||
                         (size_t)p.m_tiles * p.n_tiles * p.cg > ctx->n_tile_counters))
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "the plan's K-split scratch does not fit");
    CK(cudaStreamSynchronize(ctx->stream));
    ctx->tuned[{entropy ? kind + 1000 : kind, rows}] = {p, -2.f};
    drop_graph(ctx);
    ctx->eager_key = wedlm_ctx::StepKey();
    return WEDLM_OK;
}

wedlm_status wedlm_gemm_schedule(wedlm_ctx* ctx, int32_t kind, int32_t rows, int32_t* schedule) {
    if (!ctx || !schedule) return WEDLM_ERR_INVALID_ARG;
    auto it = ctx->tuned.find({kind, rows});
    if (it == ctx->tuned.end()) return fail(ctx, WEDLM_ERR_STATE, "no plan recorded for this kind and row count");
    const GemmPlan& p = it->second.plan;
    *schedule = (p.cg == 2 ? 1 : 0) | (p.hybrid ? 2 : 0) | (p.ks > 1 ? 4 : 0) |
                (p.splits > 1 && p.coop && p.ks <= 1 && !p.hybrid ? 8 : 0) | (p.wt == 2 ? 16 : 0) |
                (p.bk == 32 ? 32 : 0);
    return WEDLM_OK;
}

wedlm_status wedlm_kernel_launches(const wedlm_ctx* ctx, int64_t* out) {
    if (!ctx || !out) return WEDLM_ERR_INVALID_ARG;
    *out = ctx->launches;
    return WEDLM_OK;
}

// ------------------------------------------------------------- test hooks --
static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

wedlm_status wedlm_debug_read(wedlm_ctx* ctx, int32_t item, void* host_dst, int64_t bytes) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (!host_dst || bytes < 0) return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad destination");
    CK(cudaStreamSynchronize(ctx->stream));
    const int B = ctx->maxB, maxW = ctx->maxW;
    const void* src = nullptr;
    size_t avail = 0;
    switch (item) {
        case WEDLM_DBG_PERM: src = ctx->rs.perm; avail = (size_t)ctx->Mmax * 4; break;
        case WEDLM_DBG_POS: src = ctx->rs.pos; avail = (size_t)ctx->Mmax * 4; break;
        case WEDLM_DBG_ROWTOK: src = ctx->rs.tok; avail = (size_t)ctx->Mmax * 4; break;
        case WEDLM_DBG_HTILDE: src = ctx->ss.htilde; avail = (size_t)B * maxW * 4; break;
        case WEDLM_DBG_ARGMAX: src = ctx->ss.amax; avail = (size_t)B * maxW * 4; break;
        case WEDLM_DBG_FILL: src = ctx->ss.fillflag; avail = (size_t)B * maxW; break;
        case WEDLM_DBG_ROWSTRIDE: {
            if (bytes < 8) return fail(ctx, WEDLM_ERR_INVALID_ARG, "need 8 bytes");
            const int32_t v[2] = {ctx->last_stride, ctx->last_M};
            std::memcpy(host_dst, v, 8);
            return WEDLM_OK;
        }
        case WEDLM_DBG_KN: {
            if ((size_t)bytes > (size_t)B * 3 * 4) return fail(ctx, WEDLM_ERR_INVALID_ARG, "too many bytes");
            std::vector<int32_t> k(B), n(B), nf(B), outv((size_t)B * 3);
            CK(cudaMemcpy(k.data(), ctx->ss.k, B * 4, cudaMemcpyDeviceToHost));
            CK(cudaMemcpy(n.data(), ctx->ss.n, B * 4, cudaMemcpyDeviceToHost));
            CK(cudaMemcpy(nf.data(), ctx->ss.nf, B * 4, cudaMemcpyDeviceToHost));
            for (int b = 0; b < B; ++b) {
                outv[3 * b] = k[b];
                outv[3 * b + 1] = n[b];
                outv[3 * b + 2] = nf[b];
            }
            std::memcpy(host_dst, outv.data(), (size_t)bytes);
            return WEDLM_OK;
        }
        case WEDLM_DBG_LOGITS: {
            const size_t plane = (size_t)ctx->last_M * ctx->V;
            if ((size_t)bytes > plane * 4) return fail(ctx, WEDLM_ERR_INVALID_ARG, "too many bytes");
            const size_t nf = (size_t)bytes / 4;
            float* dst = (float*)host_dst;
            CK(cudaMemcpy(dst, ctx->logits, nf * 4, cudaMemcpyDeviceToHost));
            if (ctx->logits_splits_last > 1) {
                std::vector<float> tmp(nf);
                for (int sp = 1; sp < ctx->logits_splits_last; ++sp) {
                    CK(cudaMemcpy(tmp.data(), ctx->logits + sp * plane, nf * 4, cudaMemcpyDeviceToHost));
                    for (size_t i = 0; i < nf; ++i) dst[i] += tmp[i];
                }
            }
            return WEDLM_OK;
        }
        default: return fail(ctx, WEDLM_ERR_INVALID_ARG, "unknown debug item");
    }
    if ((size_t)bytes > avail) return fail(ctx, WEDLM_ERR_INVALID_ARG, "too many bytes for this item");
    CK(cudaMemcpy(host_dst, src, (size_t)bytes, cudaMemcpyDeviceToHost));
    return WEDLM_OK;
}

wedlm_status wedlm_debug_kv(wedlm_ctx* ctx, int32_t slot, int32_t layer, int32_t pos0, int32_t n, float* host_k,
                            float* host_v) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < 0 || slot >= ctx->maxB || layer < 0 || layer >= ctx->L || pos0 < 0 || n < 0 || !host_k || !host_v)
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad arguments");
    if ((int64_t)pos0 + n > (int64_t)ctx->h_pages[slot].size() * kPage)
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "positions beyond the slot's pages");
    CK(cudaStreamSynchronize(ctx->stream));
    const int hkv = ctx->hkv, hd = ctx->hd;
    const size_t page_elems = (size_t)2 * hkv * kPage * hd;
    std::vector<uint8_t> buf(page_elems * ctx->elt);
    int cur = -1;
    for (int i = 0; i < n; ++i) {
        const int p = pos0 + i;
        const int pidx = p / kPage;
        if (pidx != cur) {
            const int page = ctx->h_pages[slot][pidx];
            const char* src = (const char*)ctx->kv_pool +
                              ((size_t)layer * ctx->kvl.layer_stride + (size_t)page * page_elems) * ctx->elt;
            CK(cudaMemcpy(buf.data(), src, buf.size(), cudaMemcpyDeviceToHost));
            cur = pidx;
        }
        for (int kv = 0; kv < 2; ++kv)
            for (int hh = 0; hh < hkv; ++hh)
                for (int c = 0; c < hd; ++c) {
                    const size_t idx = (((size_t)kv * hkv + hh) * kPage + (p % kPage)) * hd + c;
                    const float v = ctx->bf16 ? bf16_bits_to_float(((const uint16_t*)buf.data())[idx])
                                              : ((const float*)buf.data())[idx];
                    (kv ? host_v : host_k)[((size_t)i * hkv + hh) * hd + c] = v;
                }
    }
    return WEDLM_OK;
}

wedlm_status wedlm_debug_keep_logits(wedlm_ctx* ctx, int32_t enable) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    CK(cudaStreamSynchronize(ctx->stream));
    if (enable < 0 || enable > 2) return fail(ctx, WEDLM_ERR_INVALID_ARG, "enable must be 0, 1 or 2");
    drop_graph(ctx);
    ctx->eager_key = wedlm_ctx::StepKey();  // the next step runs eagerly (it may tune)
    if (ctx->force_fused && enable != 2) ctx->fuse_choice.clear();  // choose afresh
    ctx->keep_logits = enable == 1;
    ctx->force_fused = enable == 2;
    return WEDLM_OK;
}

wedlm_status wedlm_debug_capture(wedlm_ctx* ctx, int32_t enable) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    CK(cudaStreamSynchronize(ctx->stream));
    if (enable && !ctx->dbg_resid) {
        const size_t bytes = (size_t)(ctx->L + 1) * ctx->Mdec * ctx->d * sizeof(float);
        if (cudaMalloc((void**)&ctx->dbg_resid, bytes) != cudaSuccess) {
            ctx->dbg_resid = nullptr;
            return fail(ctx, WEDLM_ERR_OOM_DEVICE, "residual capture buffer");
        }
        CK(cudaMemsetAsync(ctx->dbg_resid, 0, bytes, ctx->stream));
        CK(cudaStreamSynchronize(ctx->stream));
        drop_graph(ctx);
    } else if (!enable && ctx->dbg_resid) {
        cudaFree(ctx->dbg_resid);
        ctx->dbg_resid = nullptr;
    }
    return WEDLM_OK;
}

wedlm_status wedlm_debug_residual(wedlm_ctx* ctx, int32_t layer, float* host_dst, int32_t rows) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (!ctx->dbg_resid) return fail(ctx, WEDLM_ERR_STATE, "residual capture is off");
    if (layer < 0 || layer > ctx->L || rows < 0 || rows > ctx->Mdec || !host_dst)
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad arguments");
    CK(cudaStreamSynchronize(ctx->stream));
    CK(cudaMemcpy(host_dst, ctx->dbg_resid + (size_t)layer * ctx->Mdec * ctx->d, (size_t)rows * ctx->d * sizeof(float),
                  cudaMemcpyDeviceToHost));
    return WEDLM_OK;
}

wedlm_status wedlm_debug_get_window(wedlm_ctx* ctx, int32_t slot, uint8_t* filled, int32_t* tokens, int32_t cap,
                                    int32_t* n) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < 0 || slot >= ctx->maxB || !filled || !tokens || !n || cap < 0)
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad arguments");
    CK(cudaStreamSynchronize(ctx->stream));
    int32_t w = 0;
    CK(cudaMemcpy(&w, ctx->ss.wlen + slot, 4, cudaMemcpyDeviceToHost));
    *n = w;
    const int m = std::min(w, cap);
    if (m > 0) {
        CK(cudaMemcpy(filled, ctx->ss.filled + (size_t)slot * ctx->maxW, m, cudaMemcpyDeviceToHost));
        CK(cudaMemcpy(tokens, ctx->ss.token + (size_t)slot * ctx->maxW, (size_t)m * 4, cudaMemcpyDeviceToHost));
    }
    return WEDLM_OK;
}

wedlm_status wedlm_debug_read_weight(wedlm_ctx* ctx, int32_t tensor, int32_t layer, void* host_dst, int64_t bytes) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (!host_dst || bytes < 0) return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad destination");
    if (tensor_slot(ctx, tensor, layer) < 0) return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad tensor id or layer");
    const size_t elt = ctx->elt, d = ctx->d, qd = (size_t)ctx->hq * ctx->hd, kd = (size_t)ctx->hkv * ctx->hd;
    const char* src = nullptr;
    size_t avail = 0;
    switch (tensor) {
        case WEDLM_T_EMBED: src = (const char*)ctx->embed; avail = (size_t)ctx->V * d * elt; break;
        case WEDLM_T_LM_HEAD: src = (const char*)ctx->lm_head; avail = (size_t)ctx->V * d * elt; break;
        case WEDLM_T_FINAL_NORM: src = (const char*)ctx->final_norm; avail = d * 4; break;
        case WEDLM_T_ATTN_NORM: src = (const char*)ctx->attn_norm[layer]; avail = d * 4; break;
        case WEDLM_T_FFN_NORM: src = (const char*)ctx->ffn_norm[layer]; avail = d * 4; break;
        case WEDLM_T_WQ: case WEDLM_T_WK: case WEDLM_T_WV:
            src = (const char*)ctx->wqkv[layer]; avail = (qd + 2 * kd) * d * elt; break;
        case WEDLM_T_WO: src = (const char*)ctx->wo[layer]; avail = d * qd * elt; break;
        case WEDLM_T_WG: case WEDLM_T_WU: src = (const char*)ctx->wgu[layer]; avail = 2 * (size_t)ctx->F * d * elt; break;
        case WEDLM_T_WD: src = (const char*)ctx->wd[layer]; avail = d * ctx->F * elt; break;
        default: return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad tensor id");
    }
    if ((size_t)bytes > avail) return fail(ctx, WEDLM_ERR_INVALID_ARG, "too many bytes for this tensor");
    CK(cudaStreamSynchronize(ctx->stream));
    CK(cudaMemcpy(host_dst, src, (size_t)bytes, cudaMemcpyDeviceToHost));
    return WEDLM_OK;
}

wedlm_status wedlm_debug_set_page(wedlm_ctx* ctx, int32_t slot, int32_t index, int32_t page, int32_t* old_page) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < 0 || slot >= ctx->maxB || index < 0 || index >= ctx->pages_per_seq)
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad slot or page index");
    CK(cudaStreamSynchronize(ctx->stream));
    int32_t* entry = ctx->ss.page_table + (size_t)slot * ctx->pages_per_seq + index;
    if (old_page) CK(cudaMemcpy(old_page, entry, 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(entry, &page, 4, cudaMemcpyHostToDevice));
    return WEDLM_OK;
}

wedlm_status wedlm_debug_set_window(wedlm_ctx* ctx, int32_t slot, const uint8_t* filled, const int32_t* tokens,
                                    int32_t n) {
    if (!ctx) return WEDLM_ERR_INVALID_ARG;
    if (slot < 0 || slot >= ctx->maxB || n < 0 || n > ctx->maxW || (n > 0 && (!filled || !tokens)))
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "bad arguments");
    if (ctx->h_W[slot] == 0) return fail(ctx, WEDLM_ERR_STATE, "slot not in use");
    if (n > ctx->h_W[slot] || n > ctx->h_end[slot] - ctx->h_S[slot])
        return fail(ctx, WEDLM_ERR_INVALID_ARG, "window longer than W or than the remaining positions");
    for (int j = 0; j < n; ++j)
        if (filled[j] && (tokens[j] < 0 || tokens[j] >= ctx->V || tokens[j] == ctx->cfg.mask_id))
            return fail(ctx, WEDLM_ERR_INVALID_ARG, "filled slot with an invalid token");
    CK(cudaStreamSynchronize(ctx->stream));
    std::vector<uint8_t> f(ctx->maxW, 0);
    std::vector<int32_t> t(ctx->maxW, ctx->cfg.mask_id);
    for (int j = 0; j < n; ++j) {
        f[j] = filled[j] ? 1 : 0;
        t[j] = filled[j] ? tokens[j] : ctx->cfg.mask_id;
    }
    CK(cudaMemcpy(ctx->ss.filled + (size_t)slot * ctx->maxW, f.data(), ctx->maxW, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(ctx->ss.token + (size_t)slot * ctx->maxW, t.data(), (size_t)ctx->maxW * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(ctx->ss.wlen + slot, &n, 4, cudaMemcpyHostToDevice));
    return WEDLM_OK;
}

}  // extern "C"

// C ABI of the MoE FFN library (declared in include/moe.h): context and
// memory ownership, weight loading, and the per-call dispatch to the kernels.
#include <stdio.h>
#include <string.h>

#include <algorithm>

#include "moe_internal.cuh"

namespace qeffn {

static thread_local char g_last_error[512] = "";
long long g_launches = 0;

constexpr int kTimingCapacity = 65536;

int timing_begin(moe_ctx *ctx, cudaStream_t st, const char *name) {
    Timing &tm = ctx->timing;
    if (!tm.on) return MOE_OK;
    tm.name = name;
    if (tm.used >= kTimingCapacity) {
        ++tm.dropped;
        return MOE_OK;
    }
    QE_CHECK(cudaEventRecord(tm.ev[2 * tm.used], st));
    return MOE_OK;
}

int timing_end(moe_ctx *ctx, cudaStream_t st) {
    Timing &tm = ctx->timing;
    if (!tm.on || tm.used >= kTimingCapacity) return MOE_OK;
    QE_CHECK(cudaEventRecord(tm.ev[2 * tm.used + 1], st));
    ++tm.used;
    return MOE_OK;
}

int set_cuda_error(cudaError_t e, const char *what) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
    if (e == cudaErrorMemoryAllocation) return MOE_ERR_OOM;
    return MOE_ERR_CUDA;
}

int set_oom(const char *what) {
    snprintf(g_last_error, sizeof(g_last_error), "out of memory: %s", what);
    return MOE_ERR_OOM;
}

int set_too_many(const char *what) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", what);
    return MOE_ERR_TOO_MANY_TOKENS;
}

int ctx_alloc(moe_ctx *ctx, void **p, size_t bytes, const char *what) {
    *p = nullptr;
    if (bytes == 0) bytes = 16;
    long long lim = ctx->cfg.device_mem_limit;
    if (lim > 0 && (long long)(ctx->allocated + bytes) > lim) return set_oom(what);
    cudaError_t e = cudaMalloc(p, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        *p = nullptr;
        return e == cudaErrorMemoryAllocation ? set_oom(what) : set_cuda_error(e, what);
    }
    ctx->allocated += bytes;
    ctx->allocs.emplace_back(*p, bytes);
    return MOE_OK;
}

void ctx_free(moe_ctx *ctx, void *p) {
    if (!p) return;
    for (size_t i = 0; i < ctx->allocs.size(); ++i) {
        if (ctx->allocs[i].first == p) {
            ctx->allocated -= ctx->allocs[i].second;
            ctx->allocs.erase(ctx->allocs.begin() + i);
            break;
        }
    }
    cudaFree(p);
}

}  // namespace qeffn

using namespace qeffn;

namespace {

int validate_config(const moe_config *c) {
    if (c->fmt != MOE_Q4B32 && c->fmt != MOE_Q3B32 && c->fmt != MOE_Q2B32) return MOE_ERR_INVALID_ARG;
    if (c->d_model <= 0 || c->n_experts <= 0 || c->d_ff <= 0 || c->top_k <= 0 ||
        c->n_shared < 0 || c->n_layers <= 0 || c->max_tokens <= 0 || c->device_mem_limit < 0)
        return MOE_ERR_INVALID_ARG;
    if (c->top_k > c->n_experts) return MOE_ERR_INVALID_ARG;
    if (c->d_model % 256 != 0 || c->d_model > 16384) return MOE_ERR_UNSUPPORTED;
    if (c->d_ff % 64 != 0 || c->d_ff > 8192) return MOE_ERR_UNSUPPORTED;
    if (c->n_experts > 1024 || c->top_k > 32 || c->n_shared > 4) return MOE_ERR_UNSUPPORTED;
    if (c->n_shared > 0 && c->d_ff_shared != c->d_ff) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int alloc_workspace(moe_ctx *ctx) {
    const moe_config &c = ctx->cfg;
    Workspace &ws = ctx->ws;
    size_t MT = c.max_tokens, E = c.n_experts, k = c.top_k, d = c.d_model, I = c.d_ff;
    size_t S = MT * (k + c.n_shared);
    ws.max_chunks = (int)((S + 7) / 8 + ctx->nx);
    struct Item { void **p; size_t bytes; const char *name; } items[] = {
        {(void **)&ws.logits, MT * E * 4, "logits"},
        {(void **)&ws.ids, MT * k * 4, "ids"},
        {(void **)&ws.w, MT * k * 4, "w"},
        {(void **)&ws.counts, (size_t)ctx->nx * 4, "counts"},
        {(void **)&ws.offsets, (size_t)(ctx->nx + 1) * 4, "offsets"},
        {(void **)&ws.fill, (size_t)ctx->nx * 4, "fill"},
        {(void **)&ws.perm, S * 4, "perm"},
        {(void **)&ws.inv, S * 4, "inv"},
        {(void **)&ws.chunks, (size_t)ws.max_chunks * 16, "chunks"},
        {(void **)&ws.n_chunks, 4, "n_chunks"},
        {(void **)&ws.h, S * I * 4, "h"},
        {(void **)&ws.yslot, S * d * 4, "yslot"},
        {(void **)&ws.resid, MT * d * 4, "resid"},
        {(void **)&ws.xs, MT * d * 2, "xs"},
        {(void **)&ws.ys, MT * d * 2, "ys"},
        {(void **)&ws.yf, MT * d * 4, "yf"},
        {(void **)&ws.x_io, MT * d * 2, "x_io"},
        {(void **)&ws.r_io, MT * d * 4, "r_io"},
        {(void **)&ws.dev_error, 4, "dev_error"},
        {(void **)&ws.x16, MT * d * 2, "x16"},
        {(void **)&ws.h16, S * I * 2, "h16"},
        {(void **)&ws.y_acc, MT * d * 4, "y_acc"},
        {(void **)&ws.tc_n_items, 4, "tc_n_items"},
    };
    ws.tc_items_max = tc_items_max(c);
    for (auto &it : items) QE_TRY(ctx_alloc(ctx, it.p, it.bytes, it.name));
    QE_TRY(ctx_alloc(ctx, (void **)&ws.tc_items, ws.tc_items_max * sizeof(int4), "tc_items"));
    QE_TRY(ctx_alloc(ctx, (void **)&ws.cache_slot, (size_t)ctx->nx * 4, "cache_slot"));
    QE_TRY(ctx_alloc(ctx, (void **)&ws.cache_n, 4, "cache_n"));
    {
        // decoded-weight cache: at most one slot per 256 grouped rows (a bound: only experts of
        // more than three 256-row blocks take one); optional: left out when it does not fit the
        // memory limit or the device
        size_t per = (size_t)6 * c.d_model * c.d_ff;   // bytes of one expert's fp16 B stages
        size_t cap = (size_t)c.max_tokens * (c.top_k + c.n_shared) / 256;
        if (cap > (size_t)ctx->nx) cap = ctx->nx;
        if (!tc_supported(ctx, TC_MIN_TOKENS)) cap = 0;   // only the tensor-core path reads it
        long long lim = c.device_mem_limit;
        if (cap > 0 && lim > 0 && (long long)(ctx->allocated + cap * per + cap * 4) > lim) cap = 0;
        if (cap > 0 && ctx_alloc(ctx, (void **)&ws.wcache, cap * per, "weight cache") != MOE_OK) cap = 0;
        if (cap > 0 && ctx_alloc(ctx, (void **)&ws.cache_expert, cap * 4, "cache_expert") != MOE_OK) {
            ctx_free(ctx, ws.wcache);
            ws.wcache = nullptr;
            cap = 0;
        }
        ws.cache_cap = (int)cap;
    }
    QE_CHECK(cudaMemset(ws.dev_error, 0, 4));
    QE_TRY(ctx_alloc(ctx, (void **)&ctx->d_layers, sizeof(LayerPtrs) * c.n_layers, "layer table"));
    QE_CHECK(cudaMemset(ctx->d_layers, 0, sizeof(LayerPtrs) * c.n_layers));
    QE_TRY(decode_setup(ctx));
    size_t xb = decode_xchg_bytes(c);
    QE_TRY(ctx_alloc(ctx, (void **)&ctx->dec.xbuf, xb, "exchange area"));
    QE_CHECK(cudaMemset(ctx->dec.xbuf, 0, xb));
    QE_TRY(decode_split_setup(ctx));
    if (ctx->split_layout && ctx->sdec.smem_bytes == 0) ctx->split_layout = false;   // no layer loaded yet
    if (ctx->split_layout) {
        size_t xs = decode_split_xchg_bytes(c);
        QE_TRY(ctx_alloc(ctx, (void **)&ctx->sdec.xbuf, xs, "split exchange area"));
        QE_CHECK(cudaMemset(ctx->sdec.xbuf, 0, xs));
    }
    QE_TRY(decode_multi_setup(ctx));
    if (ctx->mdec.smem_bytes > 0) {
        size_t xm = decode_multi_xchg_bytes(c);
        QE_TRY(ctx_alloc(ctx, (void **)&ctx->mdec.xbuf, xm, "few-token exchange area"));
        QE_CHECK(cudaMemset(ctx->mdec.xbuf, 0, xm));
    }
    return MOE_OK;
}

void free_all(moe_ctx *ctx) {
    for (cudaEvent_t e : ctx->timing.ev) cudaEventDestroy(e);
    ctx->timing.ev.clear();
    for (auto &a : ctx->allocs) cudaFree(a.first);
    ctx->allocs.clear();
    ctx->allocated = 0;
}

// Copy `bytes` from caller memory into a fresh device buffer (host sources)
// or return the device pointer as is.
int stage(moe_ctx *ctx, const void *src, size_t bytes, int on_device, cudaStream_t st,
          const void **out, std::vector<void *> &temps) {
    if (on_device) {
        *out = src;
        return MOE_OK;
    }
    void *p;
    QE_TRY(ctx_alloc(ctx, &p, bytes, "load staging"));
    temps.push_back(p);
    QE_CHECK(cudaMemcpyAsync(p, src, bytes, cudaMemcpyHostToDevice, st));
    *out = p;
    return MOE_OK;
}

int load_layer(moe_ctx *ctx, int layer, const moe_layer_weights *w, cudaStream_t st,
               std::vector<void *> &temps) {
    const moe_config &c = ctx->cfg;
    Layer &Ly = ctx->layers[layer];
    size_t E = c.n_experts, d = c.d_model, I = c.d_ff, nsh = c.n_shared;
    size_t B = c.fmt == MOE_Q4B32 ? 16 : (c.fmt == MOE_Q2B32) ? 8 : 12;
    if (!Ly.router_w) {
        QE_TRY(ctx_alloc(ctx, (void **)&Ly.router_w, E * d * 4, "router_w"));
        QE_TRY(ctx_alloc(ctx, (void **)&Ly.router_b, E * 4, "router_b"));
        QE_TRY(ctx_alloc(ctx, (void **)&Ly.router_parts, 3 * E * d * 2, "router_parts"));
        QE_TRY(ctx_alloc(ctx, (void **)&Ly.gu, ctx->nx * ctx->gu.expert_bytes, "gate/up"));
        QE_TRY(ctx_alloc(ctx, (void **)&Ly.dn, ctx->nx * ctx->dn.expert_bytes, "down"));
    }
    Ly.loaded = false;
    cudaMemcpyKind kind = w->on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    QE_CHECK(cudaMemcpyAsync(Ly.router_w, w->router_w, E * d * 4, kind, st));
    if (w->router_bias) QE_CHECK(cudaMemcpyAsync(Ly.router_b, w->router_bias, E * 4, kind, st));
    else QE_CHECK(cudaMemsetAsync(Ly.router_b, 0, E * 4, st));
    QE_TRY(launch_split_router(Ly.router_w, E * d, Ly.router_parts, st));

    for (int part = 0; part < 2; ++part) {          // 0: routed experts, 1: shared experts
        size_t n = part == 0 ? E : nsh;
        if (n == 0) continue;
        const uint8_t *const *codes = part == 0 ? w->codes : w->sh_codes;
        const uint16_t *const *scales = part == 0 ? w->scales : w->sh_scales;
        size_t off = part == 0 ? 0 : E;
        size_t gu_codes = n * I * (d / 32) * B, gu_sc = n * I * (d / 32) * 2;
        size_t dn_codes = n * d * (I / 32) * B, dn_sc = n * d * (I / 32) * 2;
        const void *p[6];
        QE_TRY(stage(ctx, codes[0], gu_codes, w->on_device, st, &p[0], temps));
        QE_TRY(stage(ctx, scales[0], gu_sc, w->on_device, st, &p[1], temps));
        QE_TRY(stage(ctx, codes[1], gu_codes, w->on_device, st, &p[2], temps));
        QE_TRY(stage(ctx, scales[1], gu_sc, w->on_device, st, &p[3], temps));
        QE_TRY(launch_repack(ctx, c.fmt, (const uint8_t *)p[0], (const uint16_t *)p[1],
                             (const uint8_t *)p[2], (const uint16_t *)p[3], (int)n, (int)I,
                             (int)d, true, Ly.gu + off * ctx->gu.expert_bytes, st));
        QE_TRY(stage(ctx, codes[2], dn_codes, w->on_device, st, &p[4], temps));
        QE_TRY(stage(ctx, scales[2], dn_sc, w->on_device, st, &p[5], temps));
        if (ctx->split_layout)
            QE_TRY(launch_repack_chunks(ctx, c.fmt, (const uint8_t *)p[4], (const uint16_t *)p[5], (int)n,
                                        Ly.dn + off * ctx->chunk.expert_bytes, st));
        else
            QE_TRY(launch_repack(ctx, c.fmt, (const uint8_t *)p[4], (const uint16_t *)p[5], nullptr,
                                 nullptr, (int)n, (int)d, (int)I, false,
                                 Ly.dn + off * ctx->dn.expert_bytes, st));
        // Free staging of this part before the next to bound peak memory.
        QE_CHECK(cudaStreamSynchronize(st));
        for (void *t : temps) ctx_free(ctx, t);
        temps.clear();
    }
    QE_CHECK(cudaStreamSynchronize(st));
    LayerPtrs lp{Ly.router_w, Ly.router_b, Ly.gu, Ly.dn};
    QE_CHECK(cudaMemcpy(ctx->d_layers + layer, &lp, sizeof(lp), cudaMemcpyHostToDevice));
    Ly.loaded = true;
    return MOE_OK;
}

bool multi_ok(const moe_ctx *ctx) {
    return !(ctx->cfg.flags & MOE_FLAG_NO_MULTI_DECODE) && decode_multi_supported(ctx);
}

int forward_layer(moe_ctx *ctx, int layer, const uint16_t *x, int T, uint16_t *y, float *yf,
                  int32_t *ids, float *w, cudaStream_t st) {
    const Layer &Ly = ctx->layers[layer];
    Workspace &ws = ctx->ws;
    int32_t *ids_ = ids ? ids : ws.ids;
    float *w_ = w ? w : ws.w;
    if (ctx->split_layout) {   // one-token context: the split kernel (T == 1 here)
        QE_TRY(timing_begin(ctx, st, "k_decode_split"));
        QE_TRY(launch_decode_split(ctx, layer, 1, x, false, nullptr, y, yf, ids_, w_, nullptr, 1, 0, st));
        QE_TRY(timing_end(ctx, st));
        return MOE_OK;
    }
    if (T >= 2 && T <= DECODE_MULTI_MAX && multi_ok(ctx)) {
        // the few-token kernel, at most eight tokens per launch, in near-equal chunks
        const moe_config &c = ctx->cfg;
        const int n = (T + ctx->mdec.tm - 1) / ctx->mdec.tm;
        QE_TRY(timing_begin(ctx, st, "k_decode_multi"));
        for (int i = 0, t0 = 0; i < n; ++i) {
            const int tn = (T - t0) / (n - i);
            QE_TRY(launch_decode_multi(ctx, layer, 1, x + (size_t)t0 * c.d_model, tn, false, nullptr,
                                       y + (size_t)t0 * c.d_model, yf ? yf + (size_t)t0 * c.d_model : nullptr,
                                       ids_ + (size_t)t0 * c.top_k, w_ + (size_t)t0 * c.top_k, nullptr, 0, 0, st));
            t0 += tn;
        }
        QE_TRY(timing_end(ctx, st));
        return MOE_OK;
    }
    if (T <= DECODE_TOKENS_MAX && decode_supported(ctx)) {
        const moe_config &c = ctx->cfg;
        QE_TRY(timing_begin(ctx, st, "k_decode"));
        for (int t = 0; t < T; ++t)
            QE_TRY(launch_decode(ctx, layer, 1, x + (size_t)t * c.d_model, false, nullptr, y + (size_t)t * c.d_model,
                                 yf ? yf + (size_t)t * c.d_model : nullptr, ids_ + (size_t)t * c.top_k,
                                 w_ + (size_t)t * c.top_k, nullptr, 1, 0, st));
        QE_TRY(timing_end(ctx, st));
        return MOE_OK;
    }
    if (tc_router_supported(ctx, T)) {
        // tensor-core logits pick the candidates; their logits are recomputed in fp32 for the choice
        QE_TRY(launch_tc_router(ctx, Ly, x, T, ws.logits, st));
        QE_TRY(launch_topk_refine(ctx, Ly, x, ws.logits, T, ids_, w_, st));
    } else {
        QE_TRY(launch_router_simt(ctx, Ly, x, T, ws.logits, st));
        QE_TRY(launch_topk(ctx, ws.logits, T, ids_, w_, st));
    }
    QE_TRY(launch_dispatch(ctx, ids_, T, st));
    if (tc_supported(ctx, T)) return launch_tc_experts(ctx, Ly, x, T, w_, y, yf, st);
    QE_TRY(timing_begin(ctx, st, "k_gateup_simt+k_down_simt"));
    QE_TRY(launch_experts_simt(ctx, Ly, x, T, st));
    QE_TRY(timing_end(ctx, st));
    QE_TRY(launch_combine(ctx, T, w_, y, yf, st));
    return MOE_OK;
}

int check_call(moe_ctx *ctx, int layer, int n_layers, int T) {
    if (!ctx) return MOE_ERR_INVALID_ARG;
    if (layer < 0 || n_layers < 1 || layer + n_layers > ctx->cfg.n_layers) return MOE_ERR_INVALID_ARG;
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (T > ctx->cfg.max_tokens) return MOE_ERR_TOO_MANY_TOKENS;
    for (int l = layer; l < layer + n_layers; ++l)
        if (!ctx->layers[l].loaded) return MOE_ERR_NOT_LOADED;
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_create(const moe_config *cfg, int device, moe_ctx **out) {
    if (!cfg || !out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    QE_TRY(validate_config(cfg));
    int ndev = 0;
    QE_CHECK(cudaGetDeviceCount(&ndev));
    if (device < 0 || device >= ndev) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(device));
    moe_ctx *ctx = new moe_ctx();
    ctx->cfg = *cfg;
    ctx->device = device;
    ctx->nx = cfg->n_experts + cfg->n_shared;
    ctx->gu = make_layout(cfg->fmt, 2 * cfg->d_ff, cfg->d_model);
    ctx->dn = make_layout(cfg->fmt, cfg->d_model, cfg->d_ff);
    ctx->chunk = make_chunk_layout(cfg->fmt, cfg->d_model, cfg->d_ff);
    // one token per call and MOE_FLAG_SPLIT_DECODE: the down matrices in chunk order for the split
    // kernel (decided before any layer is loaded; the set-up turns it off when the shape does not fit)
    ctx->split_layout = (cfg->flags & MOE_FLAG_SPLIT_DECODE) && cfg->max_tokens == 1 &&
                        !(cfg->flags & MOE_FLAG_NO_DECODE_KERNEL) && cfg->d_model % 64 == 0 && cfg->d_ff % 32 == 0;
    ctx->layers.resize(cfg->n_layers);
    int s = alloc_workspace(ctx);
    if (s != MOE_OK) {
        free_all(ctx);
        delete ctx;
        return s;
    }
    *out = ctx;
    return MOE_OK;
}

int moe_load_layer(moe_ctx *ctx, int layer, const moe_layer_weights *w, void *stream) {
    if (!ctx || !w || layer < 0 || layer >= ctx->cfg.n_layers) return MOE_ERR_INVALID_ARG;
    if (!w->router_w) return MOE_ERR_INVALID_ARG;
    for (int t = 0; t < 3; ++t) {
        if (!w->codes[t] || !w->scales[t]) return MOE_ERR_INVALID_ARG;
        if (ctx->cfg.n_shared > 0 && (!w->sh_codes[t] || !w->sh_scales[t])) return MOE_ERR_INVALID_ARG;
    }
    QE_CHECK(cudaSetDevice(ctx->device));
    std::vector<void *> temps;
    int s = load_layer(ctx, layer, w, (cudaStream_t)stream, temps);
    if (!temps.empty()) cudaStreamSynchronize((cudaStream_t)stream);
    for (void *t : temps) ctx_free(ctx, t);
    return s;
}

int moe_forward(moe_ctx *ctx, int layer, const uint16_t *x_bf16, int T, uint16_t *y_bf16,
                float *y_f32, int32_t *ids, float *w, void *stream) {
    QE_TRY(check_call(ctx, layer, 1, T));
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !y_bf16) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(ctx->device));
    return forward_layer(ctx, layer, x_bf16, T, y_bf16, y_f32, ids, w, (cudaStream_t)stream);
}

int moe_forward_stack(moe_ctx *ctx, int layer0, int n_layers, const uint16_t *x_bf16, int T,
                      float *resid_out, const moe_stack_record *rec, void *stream) {
    QE_TRY(check_call(ctx, layer0, n_layers, T));
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !resid_out) return MOE_ERR_INVALID_ARG;
    if (rec && rec->rows && rec->n_rows < 0) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(ctx->device));
    cudaStream_t st = (cudaStream_t)stream;
    Workspace &ws = ctx->ws;
    if (ctx->split_layout) {   // one-token context: the split kernel runs the whole stack
        if (rec && rec->rows && rec->n_rows != 1) return MOE_ERR_INVALID_ARG;
        QE_TRY(timing_begin(ctx, st, "k_decode_split"));
        QE_TRY(launch_decode_split(ctx, layer0, n_layers, x_bf16, true, resid_out, nullptr, nullptr, nullptr, nullptr,
                                   rec, 1, 0, st));
        QE_TRY(timing_end(ctx, st));
        return MOE_OK;
    }
    // few tokens: the few-token kernel runs up to eight tokens per launch through the whole stack
    // (records of every row; a device row list with more than one token takes the general path)
    if (T >= 2 && T <= DECODE_MULTI_MAX && multi_ok(ctx) && (!rec || !rec->rows)) {
        const moe_config &c = ctx->cfg;
        const int n = (T + ctx->mdec.tm - 1) / ctx->mdec.tm;
        QE_TRY(timing_begin(ctx, st, "k_decode_multi"));
        for (int i = 0, t0 = 0; i < n; ++i) {
            const int tn = (T - t0) / (n - i);
            QE_TRY(launch_decode_multi(ctx, layer0, n_layers, x_bf16 + (size_t)t0 * c.d_model, tn, true,
                                       resid_out + (size_t)t0 * c.d_model, nullptr, nullptr, nullptr, nullptr, rec,
                                       T, t0, st));
            t0 += tn;
        }
        QE_TRY(timing_end(ctx, st));
        return MOE_OK;
    }
    // the single-token kernel runs each token through the whole stack (records of every row, or
    // of the one row of a single token; a device row list with more tokens takes the general path)
    if (T <= DECODE_TOKENS_MAX && decode_supported(ctx) && (!rec || !rec->rows || T == 1)) {
        if (rec && rec->rows && rec->n_rows != 1) return MOE_ERR_INVALID_ARG;
        const moe_config &c = ctx->cfg;
        QE_TRY(timing_begin(ctx, st, "k_decode"));
        for (int t = 0; t < T; ++t)
            QE_TRY(launch_decode(ctx, layer0, n_layers, x_bf16 + (size_t)t * c.d_model, true,
                                 resid_out + (size_t)t * c.d_model, nullptr, nullptr, nullptr, nullptr, rec,
                                 rec && !rec->rows ? T : 1, rec && !rec->rows ? t : 0, st));
        QE_TRY(timing_end(ctx, st));
        return MOE_OK;
    }
    QE_TRY(launch_resid_norm(ctx, T, resid_out, nullptr, x_bf16, ws.xs, st));
    for (int l = 0; l < n_layers; ++l) {
        QE_TRY(forward_layer(ctx, layer0 + l, ws.xs, T, ws.ys, ws.yf, ws.ids, ws.w, st));
        if (rec) QE_TRY(launch_record(ctx, T, l, rec, ws.xs, ws.ys, ws.yf, ws.ids, ws.w, st));
        bool last = l == n_layers - 1;
        QE_TRY(launch_resid_norm(ctx, T, resid_out, ws.ys, nullptr, last ? nullptr : ws.xs, st));
    }
    return MOE_OK;
}

int moe_forward_stack_host(moe_ctx *ctx, int layer0, int n_layers, const uint16_t *x_bf16_host,
                           int T, float *resid_out_host, void *stream) {
    QE_TRY(check_call(ctx, layer0, n_layers, T));
    if (T == 0) return MOE_OK;
    if (!x_bf16_host || !resid_out_host) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(ctx->device));
    cudaStream_t st = (cudaStream_t)stream;
    size_t d = ctx->cfg.d_model;
    QE_CHECK(cudaMemcpyAsync(ctx->ws.x_io, x_bf16_host, (size_t)T * d * 2, cudaMemcpyHostToDevice, st));
    QE_TRY(moe_forward_stack(ctx, layer0, n_layers, ctx->ws.x_io, T, ctx->ws.r_io, nullptr, stream));
    QE_CHECK(cudaMemcpyAsync(resid_out_host, ctx->ws.r_io, (size_t)T * d * 4, cudaMemcpyDeviceToHost, st));
    QE_CHECK(cudaStreamSynchronize(st));
    return MOE_OK;
}

int moe_destroy(moe_ctx *ctx) {
    if (!ctx) return MOE_OK;
    cudaSetDevice(ctx->device);
    cudaDeviceSynchronize();
    free_all(ctx);
    delete ctx;
    return MOE_OK;
}

int moe_get_device_error(moe_ctx *ctx, int *code) {
    if (!ctx || !code) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(ctx->device));
    QE_CHECK(cudaDeviceSynchronize());
    QE_CHECK(cudaMemcpy(code, ctx->ws.dev_error, 4, cudaMemcpyDeviceToHost));
    QE_CHECK(cudaMemset(ctx->ws.dev_error, 0, 4));
    // a kernel that gave up part-way leaves the decode kernel's arrival counters
    // mid-count: start them again from zero
    if (*code != 0 && ctx->dec.xbuf) QE_CHECK(cudaMemset(ctx->dec.xbuf, 0, decode_xchg_counter_bytes()));
    return MOE_OK;
}

int moe_set_l2_policy(moe_ctx *ctx, int mode) {
    if (!ctx || (mode != MOE_L2_STREAM && mode != MOE_L2_KEEP_SHARED)) return MOE_ERR_INVALID_ARG;
    ctx->l2_mode = mode;
    return MOE_OK;
}

int moe_timing_enable(moe_ctx *ctx, int on) {
    if (!ctx) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(ctx->device));
    Timing &tm = ctx->timing;
    if (on && tm.ev.empty()) {
        tm.ev.resize(2 * kTimingCapacity);
        for (auto &e : tm.ev) QE_CHECK(cudaEventCreate(&e));
    }
    tm.on = on != 0;
    tm.used = 0;
    tm.dropped = 0;
    tm.launches_at_read = __atomic_load_n(&g_launches, __ATOMIC_RELAXED);
    return MOE_OK;
}

int moe_timing_read(moe_ctx *ctx, double *total_ms, long long *timed_launches,
                    long long *all_launches, char *name, int name_len) {
    if (!ctx || !total_ms || !timed_launches || !all_launches) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(ctx->device));
    QE_CHECK(cudaDeviceSynchronize());
    Timing &tm = ctx->timing;
    double tot = 0.0;
    for (int i = 0; i < tm.used; ++i) {
        float ms = 0.f;
        QE_CHECK(cudaEventElapsedTime(&ms, tm.ev[2 * i], tm.ev[2 * i + 1]));
        tot += ms;
    }
    *total_ms = tot;
    *timed_launches = tm.used;
    long long now = __atomic_load_n(&g_launches, __ATOMIC_RELAXED);
    *all_launches = now - tm.launches_at_read;
    tm.launches_at_read = now;
    if (name && name_len > 0) {
        strncpy(name, tm.name, name_len - 1);
        name[name_len - 1] = 0;
    }
    tm.used = 0;
    tm.dropped = 0;
    return MOE_OK;
}

int moe_trace_read(moe_ctx *ctx, unsigned long long *out, int n_max, int *n) {
    if (!ctx || !n || (n_max > 0 && !out)) return MOE_ERR_INVALID_ARG;
    QE_CHECK(cudaSetDevice(ctx->device));
    QE_CHECK(cudaDeviceSynchronize());
    int cnt = ctx->dec.trace ? ctx->dec.trace_n : 0;
    if (cnt > n_max) cnt = n_max;
    if (cnt > 0)
        QE_CHECK(cudaMemcpy(out, ctx->dec.trace, (size_t)cnt * ctx->dec.trace_words * 8, cudaMemcpyDeviceToHost));
    *n = cnt;
    return MOE_OK;
}

const char *moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_OOM: return "out of device memory";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_NOT_LOADED: return "layer not loaded";
        case MOE_ERR_TOO_MANY_TOKENS: return "more tokens than max_tokens";
        case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape";
        default: return "unknown status";
    }
}

const char *moe_last_error(void) { return g_last_error; }

}  // extern "C"

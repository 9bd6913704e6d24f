// Router logits, softmax top-k and the token -> expert dispatch
// (count, exclusive scan, scatter).
//
// Routing rule: for every token a router picks top_k of the E experts and the
// shared expert(s) always run ("Qwen3.8-Flash-Next at 45 Tokens/sec on a 12GB
// GPU?", video transcript 1:50-2:16).  Weights are the softmax over all E
// logits renormalised over the chosen k, which equals the softmax over the
// chosen logits; the chosen ids are ordered by weight, equal logits -> lower id.
#include <math.h>

#include "moe_internal.cuh"

namespace qeffn {

namespace {

constexpr int RT_TOK = 8;   // tokens per router block
constexpr int RT_EXP = 8;   // experts per router block (one per warp)

// logits[t][e] = sum_i x[t][i] * W[e][i] + b[e], fp32 FMA accumulation.  The
// tokens' inputs pass through shared memory RT_CHUNK columns at a time, so any
// d fits; each lane's FMAs run in the same order whatever the chunking.
constexpr int RT_CHUNK = 4096;
__global__ void __launch_bounds__(256) k_router_simt(const uint16_t *__restrict__ x, int T, int d,
                                                     int E, const float *__restrict__ W,
                                                     const float *__restrict__ b,
                                                     float *__restrict__ logits) {
    extern __shared__ float xs[];   // [RT_TOK][min(d, RT_CHUNK)]
    const int t0 = blockIdx.y * RT_TOK;
    const int nt = min(RT_TOK, T - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * RT_EXP + warp;
    const int cw = min(d, RT_CHUNK);
    float acc[RT_TOK];
#pragma unroll
    for (int tt = 0; tt < RT_TOK; ++tt) acc[tt] = 0.f;
    for (int c0 = 0; c0 < d; c0 += cw) {
        const int n = min(cw, d - c0);
        __syncthreads();   // the previous chunk is no longer read
        for (int i = threadIdx.x; i < nt * n; i += blockDim.x) {
            int tt = i / n, c = i % n;
            uint32_t bits = (uint32_t)x[(size_t)(t0 + tt) * d + c0 + c] << 16;
            xs[tt * cw + c] = __uint_as_float(bits);
        }
        __syncthreads();
        if (e < E) {
            const float4 *Wr = reinterpret_cast<const float4 *>(W + (size_t)e * d + c0);
            for (int i4 = lane; i4 < n / 4; i4 += 32) {
                float4 wv = Wr[i4];
#pragma unroll
                for (int tt = 0; tt < RT_TOK; ++tt) {
                    if (tt < nt) {
                        const float *xv = xs + tt * cw + 4 * i4;
                        acc[tt] = fmaf(wv.x, xv[0], acc[tt]);
                        acc[tt] = fmaf(wv.y, xv[1], acc[tt]);
                        acc[tt] = fmaf(wv.z, xv[2], acc[tt]);
                        acc[tt] = fmaf(wv.w, xv[3], acc[tt]);
                    }
                }
            }
        }
    }
    if (e >= E) return;
#pragma unroll
    for (int tt = 0; tt < RT_TOK; ++tt) {
        float v = acc[tt];
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && tt < nt) logits[(size_t)(t0 + tt) * E + e] = v + b[e];
    }
}

// Larger (v, id) first: larger logit, equal logits -> lower id.
__device__ inline bool better(float v, int id, float bv, int bid) {
    return v > bv || (v == bv && id < bid);
}

// One warp per token: k rounds of warp arg-max over the token's E logits,
// then the softmax over the chosen logits.  A NaN logit is read as -inf (it
// ranks last, by id); a chosen expert is marked NaN, which better() never
// accepts, so every round picks a distinct id below E (k <= E).
__global__ void __launch_bounds__(256) k_topk(const float *__restrict__ logits, int T, int E, int k,
                                              int32_t *__restrict__ ids, float *__restrict__ w) {
    extern __shared__ float lg[];   // [8][E]
    int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    float *my = lg + warp * E;
    for (int e = lane; e < E; e += 32) {
        const float v = logits[(size_t)t * E + e];
        my[e] = isnan(v) ? -INFINITY : v;
    }
    __syncwarp();
    float chosen_v = -INFINITY;
    int chosen_id = -1;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bid = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            float v = my[e];
            if (better(v, e, bv, bid)) {
                bv = v;
                bid = e;
            }
        }
        for (int o = 16; o; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oid = __shfl_xor_sync(0xffffffffu, bid, o);
            if (better(ov, oid, bv, bid)) {
                bv = ov;
                bid = oid;
            }
        }
        if (bid >= E) bid = 0;   // unreachable while k <= E; keeps every index in range
        if (lane == j) {
            chosen_v = bv;
            chosen_id = bid;
        }
        __syncwarp();
        if (lane == 0) my[bid] = __int_as_float(0x7fc00000);   // NaN: taken
        __syncwarp();
    }
    float top = __shfl_sync(0xffffffffu, chosen_v, 0);
    float p = (lane < k) ? expf(chosen_v - top) : 0.f;
    float z = p;
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane < k) {
        ids[(size_t)t * k + lane] = chosen_id;
        w[(size_t)t * k + lane] = p / z;
    }
}

// Top-k from approximate logits (the tensor-core router sums its products in
// the MMA units' own order and precision): one warp per token takes the
// k + REFINE_EXTRA best experts by the approximate logits, recomputes those
// experts' logits with fp32 FMAs (lane-strided over d, then a warp sum, as the
// CUDA-core router does), and selects the top k among them by the recomputed
// values; the weights are the softmax over the chosen recomputed logits.  An
// expert outside the candidates could only be chosen if the approximate
// logits erred by more than the gap across REFINE_EXTRA ranks.
constexpr int REFINE_EXTRA = 6;
__global__ void __launch_bounds__(256) k_topk_refine(const float *__restrict__ logits, int T, int E, int k,
                                                     const uint16_t *__restrict__ x, int d,
                                                     const float *__restrict__ W, const float *__restrict__ b,
                                                     int32_t *__restrict__ ids, float *__restrict__ w) {
    extern __shared__ float lg[];   // [8][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    float *my = lg + warp * E;
    for (int e = lane; e < E; e += 32) {
        const float v = logits[(size_t)t * E + e];
        my[e] = isnan(v) ? -INFINITY : v;
    }
    __syncwarp();
    const int R = min(E, k + REFINE_EXTRA);   // <= 38: two candidates per lane at most
    int cid0 = 0, cid1 = 0;
    for (int j = 0; j < R; ++j) {
        float bv = -INFINITY;
        int bid = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const float v = my[e];
            if (better(v, e, bv, bid)) {
                bv = v;
                bid = e;
            }
        }
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
            if (better(ov, oid, bv, bid)) {
                bv = ov;
                bid = oid;
            }
        }
        if (bid >= E) bid = 0;
        if (lane == (j & 31)) {
            if (j < 32) cid0 = bid;
            else cid1 = bid;
        }
        __syncwarp();
        if (lane == 0) my[bid] = __int_as_float(0x7fc00000);   // taken
        __syncwarp();
    }
    // recompute the candidates' logits: candidate j's dot product over the whole warp
    const uint16_t *xr = x + (size_t)t * d;
    float ex0 = __int_as_float(0x7fc00000), ex1 = __int_as_float(0x7fc00000);   // NaN: no candidate
    for (int j = 0; j < R; ++j) {
        const int e = __shfl_sync(0xffffffffu, j < 32 ? cid0 : cid1, j & 31);
        const float4 *Wr = reinterpret_cast<const float4 *>(W + (size_t)e * d);
        float acc = 0.f;
        for (int i4 = lane; i4 < d / 4; i4 += 32) {
            const float4 wv = Wr[i4];
            const uint2 xv = *reinterpret_cast<const uint2 *>(xr + 4 * i4);
            acc = fmaf(wv.x, __uint_as_float(xv.x << 16), acc);
            acc = fmaf(wv.y, __uint_as_float(xv.x & 0xFFFF0000u), acc);
            acc = fmaf(wv.z, __uint_as_float(xv.y << 16), acc);
            acc = fmaf(wv.w, __uint_as_float(xv.y & 0xFFFF0000u), acc);
        }
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        float v = acc + b[e];
        if (isnan(v)) v = -INFINITY;
        if (lane == (j & 31)) {
            if (j < 32) ex0 = v;
            else ex1 = v;
        }
    }
    // top k among the candidates by the recomputed logits (taken ones become NaN)
    float chosen_v = -INFINITY, top = -INFINITY;
    int chosen_id = -1;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bid = 0x7fffffff;
        if (better(ex0, cid0, bv, bid)) {
            bv = ex0;
            bid = cid0;
        }
        if (lane + 32 < R && better(ex1, cid1, bv, bid)) {
            bv = ex1;
            bid = cid1;
        }
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
            if (better(ov, oid, bv, bid)) {
                bv = ov;
                bid = oid;
            }
        }
        if (bid >= E) bid = 0;
        if (j == 0) top = bv;
        if (lane == j) {
            chosen_v = bv;
            chosen_id = bid;
        }
        if (cid0 == bid && lane < R) ex0 = __int_as_float(0x7fc00000);
        if (cid1 == bid && lane + 32 < R) ex1 = __int_as_float(0x7fc00000);
    }
    const float p = (lane < k) ? expf(chosen_v - top) : 0.f;
    float z = p;
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane < k) {
        ids[(size_t)t * k + lane] = chosen_id;
        w[(size_t)t * k + lane] = p / z;
    }
}

__device__ inline int slot_expert(const int32_t *ids, int slot, int T, int k, int E) {
    int routed = T * k;
    return slot < routed ? ids[slot] : E + (slot - routed) / T;
}

__global__ void k_count(const int32_t *__restrict__ ids, int T, int k, int E, int S,
                        int32_t *__restrict__ counts) {
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < S; s += gridDim.x * blockDim.x)
        atomicAdd(&counts[slot_expert(ids, s, T, k, E)], 1);
}

// Block-wide exclusive scan of up to 2*blockDim.x values held two per thread.
__device__ int block_excl_scan(int v, int *warp_tot, int *total) {
    int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int nw = blockDim.x >> 5;
        int wv = lane < nw ? warp_tot[lane] : 0;
        int wi = wv;
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < nw) warp_tot[lane] = wi - wv;
        if (lane == nw - 1) *total = wi;
    }
    __syncthreads();
    int r = inc - v + warp_tot[warp];
    __syncthreads();
    return r;
}

// Single block: offsets = exclusive scan of counts; chunk list of <= CHUNK
// consecutive grouped positions per expert; fill[] cleared for the scatter.
__global__ void __launch_bounds__(1024) k_scan(const int32_t *__restrict__ counts, int nx, int chunk,
                                               int32_t *__restrict__ offsets, int32_t *__restrict__ fill,
                                               int4 *__restrict__ chunks, int32_t *__restrict__ n_chunks,
                                               int max_chunks) {
    __shared__ int warp_tot[32];
    __shared__ int total;
    int e0 = 2 * threadIdx.x, e1 = e0 + 1;
    int c0 = e0 < nx ? counts[e0] : 0, c1 = e1 < nx ? counts[e1] : 0;
    int base = block_excl_scan(c0 + c1, warp_tot, &total);
    if (e0 < nx) { offsets[e0] = base; fill[e0] = 0; }
    if (e1 < nx) { offsets[e1] = base + c0; fill[e1] = 0; }
    if (threadIdx.x == 0) offsets[nx] = total;
    int k0 = (c0 + chunk - 1) / chunk, k1 = (c1 + chunk - 1) / chunk;
    int cbase = block_excl_scan(k0 + k1, warp_tot, &total);
    for (int i = 0; i < k0; ++i)
        if (cbase + i < max_chunks)
            chunks[cbase + i] = make_int4(e0, base + i * chunk, min(chunk, c0 - i * chunk), 0);
    for (int i = 0; i < k1; ++i)
        if (cbase + k0 + i < max_chunks)
            chunks[cbase + k0 + i] = make_int4(e1, base + c0 + i * chunk, min(chunk, c1 - i * chunk), 0);
    if (threadIdx.x == 0) *n_chunks = min(total, max_chunks);
}

__global__ void k_scatter(const int32_t *__restrict__ ids, int T, int k, int E, int S,
                          const int32_t *__restrict__ offsets, int32_t *__restrict__ fill,
                          int32_t *__restrict__ perm, int32_t *__restrict__ inv) {
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < S; s += gridDim.x * blockDim.x) {
        int e = slot_expert(ids, s, T, k, E);
        int pos = offsets[e] + atomicAdd(&fill[e], 1);
        perm[pos] = s;
        inv[s] = pos;
    }
}

// Dynamic shared memory of k_router_simt for hidden size d.
size_t router_simt_smem(int d) { return (size_t)RT_TOK * (d < RT_CHUNK ? d : RT_CHUNK) * sizeof(float); }

}  // namespace

int launch_router_simt(const moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T,
                       float *logits, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    const size_t smem = router_simt_smem(c.d_model);
    QE_CHECK(cudaFuncSetAttribute(k_router_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)router_simt_smem(RT_CHUNK)));
    dim3 grid((c.n_experts + RT_EXP - 1) / RT_EXP, (T + RT_TOK - 1) / RT_TOK);
    k_router_simt<<<grid, 256, smem, st>>>(x, T, c.d_model, c.n_experts, Ly.router_w, Ly.router_b,
                                          logits);
    QE_CHECK_LAUNCH("k_router_simt");
    return MOE_OK;
}

int launch_topk(const moe_ctx *ctx, const float *logits, int T, int32_t *ids, float *w,
                cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    size_t smem = 8 * (size_t)c.n_experts * sizeof(float);
    k_topk<<<(T + 7) / 8, 256, smem, st>>>(logits, T, c.n_experts, c.top_k, ids, w);
    QE_CHECK_LAUNCH("k_topk");
    return MOE_OK;
}

int launch_topk_refine(const moe_ctx *ctx, const Layer &Ly, const uint16_t *x, const float *logits, int T,
                       int32_t *ids, float *w, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    size_t smem = 8 * (size_t)c.n_experts * sizeof(float);
    k_topk_refine<<<(T + 7) / 8, 256, smem, st>>>(logits, T, c.n_experts, c.top_k, x, c.d_model, Ly.router_w,
                                                  Ly.router_b, ids, w);
    QE_CHECK_LAUNCH("k_topk_refine");
    return MOE_OK;
}

// Router + top-k on caller-provided pointers (no context): used by the
// allocation-free routing entry point in route_static.cu.
int launch_route_raw(const uint16_t *x, int T, int d, int E, int k, const float *W, const float *b,
                     float *logits, int32_t *ids, float *w, cudaStream_t st) {
    // same opt-in size as launch_router_simt, so neither caller shrinks it for the other
    QE_CHECK(cudaFuncSetAttribute(k_router_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)router_simt_smem(RT_CHUNK)));
    dim3 grid((E + RT_EXP - 1) / RT_EXP, (T + RT_TOK - 1) / RT_TOK);
    k_router_simt<<<grid, 256, router_simt_smem(d), st>>>(x, T, d, E, W, b, logits);
    QE_CHECK_LAUNCH("k_router_simt");
    k_topk<<<(T + 7) / 8, 256, 8 * (size_t)E * sizeof(float), st>>>(logits, T, E, k, ids, w);
    QE_CHECK_LAUNCH("k_topk");
    return MOE_OK;
}

int launch_dispatch(moe_ctx *ctx, const int32_t *ids, int T, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    Workspace &ws = ctx->ws;
    int S = T * (c.top_k + c.n_shared);
    QE_CHECK(cudaMemsetAsync(ws.counts, 0, sizeof(int32_t) * ctx->nx, st));
    int blocks = (S + 255) / 256;
    if (blocks > 1184) blocks = 1184;
    k_count<<<blocks, 256, 0, st>>>(ids, T, c.top_k, c.n_experts, S, ws.counts);
    QE_CHECK_LAUNCH("k_count");
    k_scan<<<1, 1024, 0, st>>>(ws.counts, ctx->nx, 8, ws.offsets, ws.fill, ws.chunks, ws.n_chunks,
                              ws.max_chunks);
    QE_CHECK_LAUNCH("k_scan");
    k_scatter<<<blocks, 256, 0, st>>>(ids, T, c.top_k, c.n_experts, S, ws.offsets, ws.fill, ws.perm,
                                     ws.inv);
    QE_CHECK_LAUNCH("k_scatter");
    return MOE_OK;
}

}  // namespace qeffn

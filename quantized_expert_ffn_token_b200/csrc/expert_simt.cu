// General-T expert path on CUDA cores: dequant-fused SwiGLU gate/up, down
// projection and the weighted combine, over the dispatch's expert-grouped
// positions.  Every weight is decoded from the row-tile layout as
// w = s * (q - zero) in fp32 (exact) and accumulated with fp32 FMA.
//
// Expert network: h = silu(W_g x) * (W_u x), y = W_d h (SwiGLU; the pages call
// the experts "small expert networks" without giving their form).  Combine:
// y_t = sum_j w_tj * y_(t,j) + shared ("Qwen3.8-Flash-Next at 45 Tokens/sec on
// a 12GB GPU?", video transcript 3:36-3:47: the partial results of a token
// land on the same output).
#include <math.h>

#include "moe_internal.cuh"

namespace qeffn {

namespace {

constexpr int CHUNK = 8;  // grouped positions per block (must match launch_dispatch)

struct ExpertArgs {
    int fmt, T, k, E, d, I, zero;
    MatLayout gu, dn;
    const uint8_t *gu_w, *dn_w;
    const uint16_t *x;
    const int32_t *perm;
    const int4 *chunks;
    const int32_t *n_chunks;
    float *h, *yslot;
};

__device__ inline int slot_token(int slot, int T, int k) {
    int routed = T * k;
    return slot < routed ? slot / k : (slot - routed) % T;
}

__device__ inline float silu(float z) { return z / (1.f + expf(-z)); }

// grid: (chunk, 64-wide slice of I); 8 warps x 8 intermediate indices.
__global__ void __launch_bounds__(256) k_gateup_simt(ExpertArgs a) {
    extern __shared__ float xs[];   // [CHUNK][d]
    int ci = blockIdx.x;
    if (ci >= *a.n_chunks) return;
    int4 ch = a.chunks[ci];
    int e = ch.x, start = ch.y, n = ch.z;
    for (int i = threadIdx.x; i < n * a.d; i += blockDim.x) {
        int tt = i / a.d, c = i % a.d;
        int tok = slot_token(a.perm[start + tt], a.T, a.k);
        xs[tt * a.d + c] = __uint_as_float((uint32_t)a.x[(size_t)tok * a.d + c] << 16);
    }
    __syncthreads();
    int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t *ex = a.gu_w + (size_t)e * a.gu.expert_bytes;
    int nb = a.d / 32;
    for (int ii = 0; ii < 8; ++ii) {
        int i = blockIdx.y * 64 + warp * 8 + ii;
        if (i >= a.I) break;
        const uint8_t *tile = ex + (size_t)(i >> 3) * a.gu.tile_bytes;
        int rg = i & 7, ru = 8 + (i & 7);
        float ag[CHUNK], au[CHUNK];
#pragma unroll
        for (int s = 0; s < CHUNK; ++s) ag[s] = au[s] = 0.f;
        for (int b = 0; b < nb; ++b) {
            int kk = 32 * b + lane;
            float wg = tile_scale(tile, a.gu, rg, b) * (float)(tile_code(a.fmt, tile, rg, kk) - a.zero);
            float wu = tile_scale(tile, a.gu, ru, b) * (float)(tile_code(a.fmt, tile, ru, kk) - a.zero);
#pragma unroll
            for (int s = 0; s < CHUNK; ++s) {
                if (s < n) {
                    float xv = xs[s * a.d + kk];
                    ag[s] = fmaf(wg, xv, ag[s]);
                    au[s] = fmaf(wu, xv, au[s]);
                }
            }
        }
#pragma unroll
        for (int s = 0; s < CHUNK; ++s) {
            float g = ag[s], u = au[s];
            for (int o = 16; o; o >>= 1) {
                g += __shfl_xor_sync(0xffffffffu, g, o);
                u += __shfl_xor_sync(0xffffffffu, u, o);
            }
            if (lane == 0 && s < n) a.h[(size_t)(start + s) * a.I + i] = silu(g) * u;
        }
    }
}

// grid: (chunk, 128 output rows); warp w handles down tile 8*blockIdx.y + w.
__global__ void __launch_bounds__(256) k_down_simt(ExpertArgs a) {
    extern __shared__ float hs[];   // [CHUNK][I]
    int ci = blockIdx.x;
    if (ci >= *a.n_chunks) return;
    int4 ch = a.chunks[ci];
    int e = ch.x, start = ch.y, n = ch.z;
    for (int i = threadIdx.x; i < n * a.I; i += blockDim.x)
        hs[i] = a.h[(size_t)start * a.I + i];
    __syncthreads();
    int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int t = blockIdx.y * 8 + warp;
    if (t >= a.dn.n_tiles) return;
    const uint8_t *tile = a.dn_w + (size_t)e * a.dn.expert_bytes + (size_t)t * a.dn.tile_bytes;
    int nb = a.I / 32;
    for (int r = 0; r < 16; ++r) {
        float acc[CHUNK];
#pragma unroll
        for (int s = 0; s < CHUNK; ++s) acc[s] = 0.f;
        for (int b = 0; b < nb; ++b) {
            int kk = 32 * b + lane;
            float wv = tile_scale(tile, a.dn, r, b) * (float)(tile_code(a.fmt, tile, r, kk) - a.zero);
#pragma unroll
            for (int s = 0; s < CHUNK; ++s)
                if (s < n) acc[s] = fmaf(wv, hs[s * a.I + kk], acc[s]);
        }
#pragma unroll
        for (int s = 0; s < CHUNK; ++s) {
            float v = acc[s];
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && s < n) a.yslot[(size_t)(start + s) * a.d + 16 * t + r] = v;
        }
    }
}

// y_t = sum_j w_tj * y_(t,j) + sum_s y_shared(s,t), fixed order, then bf16.
__global__ void __launch_bounds__(256) k_combine(int T, int k, int n_sh, int d,
                                                 const float *__restrict__ w,
                                                 const int32_t *__restrict__ inv,
                                                 const float *__restrict__ yslot,
                                                 uint16_t *__restrict__ y, float *__restrict__ yf) {
    int t = blockIdx.x;
    for (int o = threadIdx.x; o < d; o += blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < k; ++j)
            acc = fmaf(w[(size_t)t * k + j], yslot[(size_t)inv[(size_t)t * k + j] * d + o], acc);
        for (int s = 0; s < n_sh; ++s)
            acc += yslot[(size_t)inv[(size_t)T * k + (size_t)s * T + t] * d + o];
        __nv_bfloat16 b = __float2bfloat16_rn(acc);
        y[(size_t)t * d + o] = *reinterpret_cast<uint16_t *>(&b);
        if (yf) yf[(size_t)t * d + o] = acc;
    }
}

}  // namespace

int launch_experts_simt(moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    Workspace &ws = ctx->ws;
    ExpertArgs a;
    a.fmt = c.fmt;
    a.T = T;
    a.k = c.top_k;
    a.E = c.n_experts;
    a.d = c.d_model;
    a.I = c.d_ff;
    a.zero = c.fmt == MOE_Q4B32 ? 8 : (c.fmt == MOE_Q2B32) ? 2 : 4;
    a.gu = ctx->gu;
    a.dn = ctx->dn;
    a.gu_w = Ly.gu;
    a.dn_w = Ly.dn;
    a.x = x;
    a.perm = ws.perm;
    a.chunks = ws.chunks;
    a.n_chunks = ws.n_chunks;
    a.h = ws.h;
    a.yslot = ws.yslot;
    int S = T * (c.top_k + c.n_shared);
    int max_chunks = (S + CHUNK - 1) / CHUNK + ctx->nx;
    if (max_chunks > ws.max_chunks) max_chunks = ws.max_chunks;
    QE_CHECK(cudaFuncSetAttribute(k_gateup_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  CHUNK * c.d_model * (int)sizeof(float)));
    QE_CHECK(cudaFuncSetAttribute(k_down_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  CHUNK * c.d_ff * (int)sizeof(float)));
    k_gateup_simt<<<dim3(max_chunks, (c.d_ff + 63) / 64), 256,
                    CHUNK * c.d_model * sizeof(float), st>>>(a);
    QE_CHECK_LAUNCH("k_gateup_simt");
    k_down_simt<<<dim3(max_chunks, (c.d_model + 127) / 128), 256, CHUNK * c.d_ff * sizeof(float),
                  st>>>(a);
    QE_CHECK_LAUNCH("k_down_simt");
    return MOE_OK;
}

int launch_combine(const moe_ctx *ctx, int T, const float *w, uint16_t *y, float *yf,
                   cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    k_combine<<<T, 256, 0, st>>>(T, c.top_k, c.n_shared, c.d_model, w, ctx->ws.inv, ctx->ws.yslot,
                                 y, yf);
    QE_CHECK_LAUNCH("k_combine");
    return MOE_OK;
}

}  // namespace qeffn

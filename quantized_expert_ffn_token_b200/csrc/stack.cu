// Residual stream of the layer stack and the per-layer records.
//
// The pages only say that the 48 MoE layers are stacked.  A plain residual
// add of SwiGLU outputs grows without bound (SwiGLU is quadratic in its input
// scale), so each layer reads a normalised copy of the residual stream:
//   x_l = bf16(r_l / sqrt(mean(r_l^2) + 1e-6)),  r_{l+1} = r_l + y_l.
#include "moe_internal.cuh"

namespace qeffn {

namespace {

__device__ inline float bf16_bits_to_float(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ inline uint16_t float_to_bf16_bits(float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&b);
}

// One block per token.  x_in != NULL: r = float(x_in) (first layer);
// else r += float(y_add) when y_add != NULL.  x_out (optional) = bf16(rmsnorm(r)).
__global__ void __launch_bounds__(256) k_resid_norm(int d, float *__restrict__ resid,
                                                    const uint16_t *__restrict__ y_add,
                                                    const uint16_t *__restrict__ x_in,
                                                    uint16_t *__restrict__ x_out) {
    __shared__ float red[8];
    int t = blockIdx.x;
    float *r = resid + (size_t)t * d;
    float ss = 0.f;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        float v;
        if (x_in) v = bf16_bits_to_float(x_in[(size_t)t * d + i]);
        else v = r[i] + (y_add ? bf16_bits_to_float(y_add[(size_t)t * d + i]) : 0.f);
        r[i] = v;
        ss = fmaf(v, v, ss);
    }
    if (!x_out) return;
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    float inv = 1.f / sqrtf(red[0] / (float)d + 1e-6f);
    for (int i = threadIdx.x; i < d; i += blockDim.x)
        x_out[(size_t)t * d + i] = float_to_bf16_bits(r[i] * inv);
}

struct RecArgs {
    int d, k, n_rec, layer;
    const int32_t *rows;
    const uint16_t *x, *y;
    const float *yf, *w;
    const int32_t *ids;
    moe_stack_record rec;
};

__global__ void k_record(RecArgs a) {
    int ri = blockIdx.x;
    int t = a.rows ? a.rows[ri] : ri;
    size_t dst = ((size_t)a.layer * a.n_rec + ri);
    for (int i = threadIdx.x; i < a.d; i += blockDim.x) {
        if (a.rec.x_bf16) a.rec.x_bf16[dst * a.d + i] = a.x[(size_t)t * a.d + i];
        if (a.rec.y_bf16) a.rec.y_bf16[dst * a.d + i] = a.y[(size_t)t * a.d + i];
        if (a.rec.y_f32) a.rec.y_f32[dst * a.d + i] = a.yf[(size_t)t * a.d + i];
    }
    for (int j = threadIdx.x; j < a.k; j += blockDim.x) {
        if (a.rec.ids) a.rec.ids[dst * a.k + j] = a.ids[(size_t)t * a.k + j];
        if (a.rec.w) a.rec.w[dst * a.k + j] = a.w[(size_t)t * a.k + j];
    }
}

}  // namespace

int launch_resid_norm(const moe_ctx *ctx, int T, float *resid, const uint16_t *y_add,
                      const uint16_t *x_in, uint16_t *x_out, cudaStream_t st) {
    k_resid_norm<<<T, 256, 0, st>>>(ctx->cfg.d_model, resid, y_add, x_in, x_out);
    QE_CHECK_LAUNCH("k_resid_norm");
    return MOE_OK;
}

int launch_record(const moe_ctx *ctx, int T, int layer_idx, const moe_stack_record *rec,
                  const uint16_t *x, const uint16_t *y, const float *yf, const int32_t *ids,
                  const float *w, cudaStream_t st) {
    RecArgs a;
    a.d = ctx->cfg.d_model;
    a.k = ctx->cfg.top_k;
    a.n_rec = rec->rows ? rec->n_rows : T;
    a.layer = layer_idx;
    a.rows = rec->rows;
    a.x = x;
    a.y = y;
    a.yf = yf;
    a.w = w;
    a.ids = ids;
    a.rec = *rec;
    if (a.n_rec <= 0) return MOE_OK;
    k_record<<<a.n_rec, 256, 0, st>>>(a);
    QE_CHECK_LAUNCH("k_record");
    return MOE_OK;
}

}  // namespace qeffn

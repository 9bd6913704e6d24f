// Single-token decode with the down projection split by k chunks: one
// persistent kernel runs whole layers (and the whole stack) for one token with
// two grid-wide exchanges per layer instead of three.
//
// A unit is 16 consecutive SwiGLU rows of one expert (a 16-wide chunk of the
// down projection's reduction dimension).  A CTA computes a unit's gate/up rows
// (two row tiles), applies SwiGLU and the routing weight, and immediately
// multiplies the 16 h values into the matching 16 columns of the expert's down
// matrix (all d output rows, the chunk-ordered down layout), adding the
// products into a per-CTA partial output in shared memory.  So h never leaves
// the CTA: no h exchange, no separate down phase.  At the end of the layer
// every CTA adds its partial output to the layer's fp32 output with vector
// atomics; one counter closes the layer (exchange 2); the logits are the
// other exchange.  The shared expert does not depend on the routing: its
// units are streamed during the previous layer and computed while the logits
// exchange is in flight.
//
// Per layer (one token):
//   1. input: every CTA reads the previous layer's output, adds it to its copy
//      of the residual stream, normalises (rmsnorm) and rounds to bf16 (stack),
//      plus the fp16 operand x * 2^s for fp16 code operands;
//   2. router: CTA c owns experts c, c+G, ... (rows prefetched into shared
//      memory during the previous layer); logits published;
//   3. the CTA's shared-expert units, while the logits travel;
//   4. every CTA reads all logits and selects the same top-k;
//   5. the CTA's routed units, streamed through a ring of shared-memory slots
//      by one producer warp with cp.async.bulk;
//   6. partial output -> atomics; arrival.
// Arithmetic is that of the single-token kernel (exact code operands, per-block
// offset removal and scaling in fp32, h as hi + lo parts).  Routing and combine
// passages: "Qwen3.8-Flash-Next at 45 Tokens/sec on a 12GB GPU?" (video
// transcript 1:50-2:16, 3:36-3:47); expert = SwiGLU and the block formats are
// include/moe.h's.
#include <string.h>

#include "decode_common.cuh"

namespace qeffn {

namespace {

using namespace dec;

constexpr int SK_MAXK = 32;
constexpr int SK_CAND = 256;
constexpr int SK_EMAX = 3;      // logits per thread (E <= 1024)
constexpr int SK_YIT = 3;       // float4 columns of the row per thread (d <= 4608)
constexpr int SK_GWMAX = 16;    // gate/up warps (d / 256) the partial buffers hold

struct SkMisc {
    unsigned long long full[MAX_SLOTS];
    unsigned long long empty[MAX_SLOTS];   // NW arrivals per consumed item
    unsigned long long rbar;
    unsigned long long route;              // one arrival per layer: routing known
    int ids[SK_MAXK];
    float psel[SK_MAXK];
    float uw[SK_MAXK + 4];                 // weight of each expert slot (routed: softmax, shared: 1)
    int uexp[SK_MAXK + 4];                 // expert of each slot (routed by rank, then shared)
    int ncand;
    float xinv;                            // 2^-s of the fp16 layer input (1 for bf16 operands)
    float wmax[NW];
    float red1[NW];
    float amax[NW];
    __align__(16) float2 cand[SK_CAND];
};

struct SplitParams {
    const LayerPtrs *layers;
    int layer0, L;
    int d, E, I, k, nsh;
    MatLayout gu;              // gate/up row tiles
    int chunk_bytes;           // down: codes of one 16-wide k chunk (all d rows)
    int dn_code_bytes;         // down: codes of every chunk of an expert (scales follow)
    size_t dn_expert_bytes;
    int stack;
    const uint16_t *x_in;
    float *resid_out;
    uint16_t *y_out;
    float *yf_out;
    int32_t *ids_out;
    float *w_out;
    moe_stack_record rec;
    int rec_on, rec_n, rec_r;
    unsigned *cnt;             // [0] logits arrivals, [32] output arrivals (host-zeroed per launch)
    float *x_logits;           // [E]
    float *y_acc;              // [2][d] layer outputs, accumulated with atomics
    int *err;
    int withhold;
    unsigned long long *trace; // [G][L][24] or NULL
    int nslot, slot_bytes, rpc;
    int off_ring, off_router, off_xb, off_xh, off_logits, off_gp, off_ysm, off_red, off_misc, off_resid,
        off_sums, off_ltab;
};

constexpr int S_LOGITS = 0, S_Y = 32;

// Phase trace (MOE_FLAG_TRACE): per (CTA, layer) 24 words: CTA, layer, then SM clock cycles since
// the layer started in this CTA:
//   0 input ready            1 logits stored          2 shared units done     3 all logits received
//   4 routing known          5 routed units done      6 output added          7 previous output received
//   8 warp 0: cycles waiting for weights              21 global timer (ns) at the layer start
constexpr int SK_TRACE_WORDS = 24;
__device__ __noinline__ void sk_trace_store(unsigned long long *trace, int L, int l, int ph, long long t) {
    unsigned long long *r = trace + ((size_t)blockIdx.x * L + l) * SK_TRACE_WORDS;
    if (ph == 0) {
        r[0] = blockIdx.x;
        r[1] = l;
    }
    r[2 + ph] = (unsigned long long)t;
}

template <int FMT>
__device__ __forceinline__ void sk_frag16(const uint8_t *piece, uint32_t r[16]) {
    if constexpr (FMT == MOE_Q2B32) {
        q2_frag_h(*reinterpret_cast<const uint2 *>(piece), r);
    } else if constexpr (FMT == MOE_Q4B32) {
        const uint4 a = *reinterpret_cast<const uint4 *>(piece);
        const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) q4_frag_h(wv[m], r[4 * m], r[4 * m + 1], r[4 * m + 2], r[4 * m + 3]);
    } else {
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(piece);
        q3_frag(wp[0], wp[1], wp[2], r);
    }
}
template <int FMT>
constexpr int sk_piece() { return FMT == MOE_Q4B32 ? 16 : FMT == MOE_Q2B32 ? 8 : 12; }

__device__ __noinline__ void sk_topk_rounds(SkMisc *ms, const float *lg, int E, int k, float gmax) {
    const int lane = threadIdx.x & 31;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bid = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            bool taken = false;
            for (int q = 0; q < j; ++q) taken |= (ms->ids[q] == e);
            if (!taken && better(lg[e], e, bv, bid)) {
                bv = lg[e];
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
        if (lane == 0) {
            ms->ids[j] = bid;
            ms->psel[j] = expf(bv - gmax);
        }
        __syncwarp();
    }
}

template <int FMT>
__global__ void __launch_bounds__(NTT, 1) k_decode_split(SplitParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem + p.off_ring;
    float *rtr = reinterpret_cast<float *>(smem + p.off_router);
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem + p.off_xb);
    uint16_t *xh = reinterpret_cast<uint16_t *>(smem + p.off_xh);
    float *lg = reinterpret_cast<float *>(smem + p.off_logits);
    float *gp = reinterpret_cast<float *>(smem + p.off_gp);      // [2 buffers][2 tiles][GW][16]
    float *ysm = reinterpret_cast<float *>(smem + p.off_ysm);    // [d] this CTA's partial output
    float *red = reinterpret_cast<float *>(smem + p.off_red);    // [8][NW] router partials
    SkMisc *ms = reinterpret_cast<SkMisc *>(smem + p.off_misc);
    float *rs = reinterpret_cast<float *>(smem + p.off_resid);   // [d] residual stream
    float *xsum = reinterpret_cast<float *>(smem + p.off_sums);  // [d/32]
    LayerPtrs *ltab = reinterpret_cast<LayerPtrs *>(smem + p.off_ltab);

    constexpr bool F16OP = (FMT != MOE_Q3B32);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
    const int G = gridDim.x, cta = blockIdx.x;
    const int d = p.d, E = p.E, I = p.I, k = p.k;
    const int nbd = d / 32;
    const int d4 = d / 4;
    const int GW = d / 256;
    const int CH = I / 16;                       // units (16-row chunks) per expert
    const int n_units_all = (k + p.nsh) * CH;
    const int n_routed_all = k * CH;
    const int own_lo = cta * d4 / G, own_hi = (cta + 1) * d4 / G;
    int *err = p.err;

    // this CTA's units: n = cta + G q; its shared-expert units (the highest n) are processed first
    const int nq = (cta < n_units_all) ? (n_units_all - cta + G - 1) / G : 0;
    const int nq_routed = (cta < n_routed_all) ? (n_routed_all - cta + G - 1) / G : 0;
    const int ns = nq - nq_routed;
    auto unit_n = [&](int i) { return cta + G * (i < ns ? nq_routed + i : i - ns); };

    if (tid == 0) {
        for (int s = 0; s < p.nslot; ++s) {
            mbar_init(&ms->full[s], 1);
            mbar_init(&ms->empty[s], NW);
        }
        mbar_init(&ms->rbar, 1);
        mbar_init(&ms->route, 1);
        fence_mbar_init();
    }
    if (tid < p.nsh) {
        ms->uexp[k + tid] = E + tid;
        ms->uw[k + tid] = 1.f;
    }
    for (int i = tid; i < d; i += NTT) ysm[i] = 0.f;
    for (int l = tid; l < p.L; l += NTT) ltab[l] = p.layers[p.layer0 + l];
    __syncthreads();

    // ---- producer warp (lane 0) -------------------------------------------------------------
    if (warp == NW) {
        if (lane != 0) return;
        uint32_t fpar = 0, filled = 0;
        int router_fills = 0;
        int s_next = 0;
        bool pok = true;
        auto issue_router = [&](int li) {
            const float *rw = ltab[li].rw;
            int nrows = 0;
            for (int j = 0; j < p.rpc; ++j)
                if (cta + G * j < E) ++nrows;
            fence_proxy_async();
            mbar_expect_tx(&ms->rbar, (uint32_t)(nrows * d * 4));
            for (int j = 0; j < nrows; ++j)
                bulk_g2s(rtr + (size_t)j * d, rw + (size_t)(cta + G * j) * d, (uint32_t)(d * 4), &ms->rbar);
            ++router_fills;
        };
        // the three items of unit i of layer li: two gate/up row tiles, then the down chunk with
        // its block's scales
        auto issue_unit = [&](int li, int i) {
            const LayerPtrs Lp = ltab[li];
            const int n = unit_n(i);
            const int us = n / CH, c16 = n - us * CH;
            const int e = us < k ? ms->uexp[us] : E + (us - k);
            for (int part = 0; part < 3 && pok; ++part) {
                const int s = s_next;
                s_next = (s_next + 1 == p.nslot) ? 0 : s_next + 1;
                if ((filled >> s) & 1u) pok = mbar_wait(&ms->empty[s], ((fpar >> s) & 1u) ^ 1u, err, true);
                if (!pok) break;
                fence_proxy_async();
                uint8_t *dst = ring + (size_t)s * p.slot_bytes;
                if (part < 2) {
                    const uint8_t *src = Lp.gu + (size_t)e * p.gu.expert_bytes + (size_t)(2 * c16 + part) * p.gu.tile_bytes;
                    mbar_expect_tx(&ms->full[s], (uint32_t)p.gu.tile_bytes);
                    bulk_g2s(dst, src, (uint32_t)p.gu.tile_bytes, &ms->full[s]);
                } else {
                    const uint8_t *ex = Lp.dn + (size_t)e * p.dn_expert_bytes;
                    mbar_expect_tx(&ms->full[s], (uint32_t)(p.chunk_bytes + d * 2));
                    bulk_g2s(dst, ex + (size_t)c16 * p.chunk_bytes, (uint32_t)p.chunk_bytes, &ms->full[s]);
                    bulk_g2s(dst + p.chunk_bytes, ex + p.dn_code_bytes + (size_t)(c16 >> 1) * d * 2, (uint32_t)(d * 2),
                             &ms->full[s]);
                }
                fpar ^= 1u << s;
                filled |= 1u << s;
            }
        };
        issue_router(0);
        for (int i = 0; i < ns && pok; ++i) issue_unit(0, i);          // shared units of layer 0
        for (int l = 0; l < p.L && pok; ++l) {
            if (!mbar_wait(&ms->route, (uint32_t)(l & 1), err, true)) break;
            for (int i = ns; i < nq && pok; ++i) issue_unit(l, i);     // routed units
            if (!pok) break;
            if (l + 1 < p.L) {
                issue_router(l + 1);
                for (int i = 0; i < ns && pok; ++i) issue_unit(l + 1, i);   // next layer's shared units
            }
        }
        for (int s = 0; s < p.nslot; ++s)
            if ((filled >> s) & 1u) mbar_wait(&ms->full[s], ((fpar >> s) & 1u) ^ 1u, err, false);
        if (router_fills > 0) mbar_wait(&ms->rbar, (uint32_t)((router_fills - 1) & 1), err, false);
        return;
    }

    int ring_base = 0;        // absolute index of this layer's first item
    int unit_ctr = 0;         // units processed so far (partial-buffer parity)
    bool ok = true;
    bool aborted = false;

    // gate/up B fragments of this warp's 256-wide k chunk (the token in one column per 32-block)
    uint32_t bx0[16], bx1[16];

    for (int l = 0; l < p.L; ++l) {
        const LayerPtrs Lp = ltab[l];
        const long long tl0 = clock64();
        long long tw = 0;
        auto mark = [&](int ph, long long v) {
            if (p.trace && tid == 0) sk_trace_store(p.trace, p.L, l, ph, v);
        };
        if (p.trace && tid == 0) {
            unsigned long long gt;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(gt));
            sk_trace_store(p.trace, p.L, l, 21, (long long)gt);
        }

        // ---- 1. layer input ------------------------------------------------------------------
        float amx = 0.f;
        float inv = 1.f;
        if (p.stack) {
            float ss = 0.f;
            if (l == 0) {
                for (int i = tid; i < d; i += NT) {
                    const float v = bf16_bits_f(p.x_in[i]);
                    rs[i] = v;
                    ss = fmaf(v, v, ss);
                    amx = fmaxf(amx, fabsf(v));
                }
            } else {
                if (tid == 0) ok = ctr_wait(p.cnt + S_Y, (unsigned)(G * l), err);
                if (cta_failed(ok)) {
                    aborted = true;
                    break;
                }
                mark(7, clock64() - tl0);
                const float *yprev = p.y_acc + (size_t)((l - 1) & 1) * d;
                float4 yv[SK_YIT];
#pragma unroll
                for (int it = 0; it < SK_YIT; ++it) {
                    const int i4 = tid + it * NT;
                    yv[it] = i4 < d4 ? __ldcg(reinterpret_cast<const float4 *>(yprev + 4 * i4)) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int it = 0; it < SK_YIT; ++it) {
                    const int i4 = tid + it * NT;
                    if (i4 >= d4) break;
                    const float ya[4] = {yv[it].x, yv[it].y, yv[it].z, yv[it].w};
                    uint16_t yb[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int i = 4 * i4 + j;
                        yb[j] = bf16_rn_bits(ya[j]);
                        const float rn = rs[i] + bf16_bits_f(yb[j]);
                        rs[i] = rn;
                        ss = fmaf(rn, rn, ss);
                        amx = fmaxf(amx, fabsf(rn));
                    }
                    if (p.rec_on && i4 >= own_lo && i4 < own_hi) {
                        const size_t ro = ((size_t)(l - 1) * p.rec_n + p.rec_r) * d + 4 * i4;
                        if (p.rec.y_bf16)
                            *reinterpret_cast<uint2 *>(p.rec.y_bf16 + ro) =
                                make_uint2((uint32_t)yb[0] | ((uint32_t)yb[1] << 16), (uint32_t)yb[2] | ((uint32_t)yb[3] << 16));
                        if (p.rec.y_f32) *reinterpret_cast<float4 *>(p.rec.y_f32 + ro) = yv[it];
                    }
                }
            }
            for (int o = 16; o; o >>= 1) {
                ss += __shfl_xor_sync(0xffffffffu, ss, o);
                amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, o));
            }
            if (lane == 0) {
                ms->red1[warp] = ss;
                ms->amax[warp] = amx;
            }
            csync();
            float tot = lane < NW ? ms->red1[lane] : 0.f;
            amx = lane < NW ? ms->amax[lane] : 0.f;
            for (int o = 16; o; o >>= 1) {
                tot += __shfl_xor_sync(0xffffffffu, tot, o);
                amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, o));
            }
            inv = 1.f / sqrtf(tot / (float)d + 1e-6f);
            amx = bf16_bits_f(bf16_rn_bits(amx * inv));
        } else {
            for (int i = tid; i < d; i += NT) {
                const uint16_t v = p.x_in[i];
                xb[i] = v;
                amx = fmaxf(amx, fabsf(bf16_bits_f(v)));
            }
            for (int o = 16; o; o >>= 1) amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, o));
            if (lane == 0) ms->amax[warp] = amx;
            csync();
            amx = lane < NW ? ms->amax[lane] : 0.f;
            for (int o = 16; o; o >>= 1) amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, o));
        }
        int xe;
        frexpf(amx, &xe);
        const int xs_exp = min(15 - xe, 100);
        const float xscale = pow2i(xs_exp);
        if (tid == 0) ms->xinv = F16OP ? pow2i(-xs_exp) : 1.f;
        for (int i8 = tid; i8 < d / 8; i8 += NT) {
            uint32_t xw[4], hw[4];
            if (p.stack) {
                const float4 r0 = reinterpret_cast<const float4 *>(rs)[2 * i8];
                const float4 r1 = reinterpret_cast<const float4 *>(rs)[2 * i8 + 1];
                const float rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    xw[j] = (uint32_t)bf16_rn_bits(rv[2 * j] * inv) | ((uint32_t)bf16_rn_bits(rv[2 * j + 1] * inv) << 16);
                *reinterpret_cast<uint4 *>(xb + 8 * i8) = make_uint4(xw[0], xw[1], xw[2], xw[3]);
                if (p.rec_on && p.rec.x_bf16) {   // the owned float4 columns 2 i8, 2 i8 + 1
                    uint16_t *xr = p.rec.x_bf16 + ((size_t)l * p.rec_n + p.rec_r) * d + 8 * i8;
                    if (2 * i8 >= own_lo && 2 * i8 < own_hi) *reinterpret_cast<uint2 *>(xr) = make_uint2(xw[0], xw[1]);
                    if (2 * i8 + 1 >= own_lo && 2 * i8 + 1 < own_hi)
                        *reinterpret_cast<uint2 *>(xr + 4) = make_uint2(xw[2], xw[3]);
                }
            } else {
                const uint4 v = *reinterpret_cast<const uint4 *>(xb + 8 * i8);
                xw[0] = v.x; xw[1] = v.y; xw[2] = v.z; xw[3] = v.w;
            }
            if constexpr (F16OP) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half2 h2 = __floats2half2_rn(__uint_as_float(xw[j] << 16) * xscale,
                                                         __uint_as_float(xw[j] & 0xFFFF0000u) * xscale);
                    hw[j] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                *reinterpret_cast<uint4 *>(xh + 8 * i8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            }
        }
        csync();
        for (int b = tid; b < nbd; b += NT) xsum[b] = F16OP ? sum32_f16(xh + 32 * b) : sum32_bf16(xb + 32 * b);
        if (warp < GW) {
            const uint16_t *xop = F16OP ? xh : xb;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int s = 16 * warp + j;
                const bool act = (g == (j >> 1));
                const uint32_t v0 = *reinterpret_cast<const uint32_t *>(xop + 16 * s + 2 * c);
                const uint32_t v1 = *reinterpret_cast<const uint32_t *>(xop + 16 * s + 2 * c + 8);
                bx0[j] = act ? v0 : 0u;
                bx1[j] = act ? v1 : 0u;
            }
        }
        mark(0, clock64() - tl0);

        // ---- 2. router --------------------------------------------------------------------------
        {
            int nrows = 0;
            for (int j = 0; j < p.rpc; ++j)
                if (cta + G * j < E) ++nrows;
            const float bias = (warp < nrows && lane == 0) ? __ldg(Lp.rb + cta + G * warp) : 0.f;
            ok = mbar_wait(&ms->rbar, (uint32_t)(l & 1), err, true);
            if (cta_failed(ok)) {
                aborted = true;
                break;
            }
            float part[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) part[j] = 0.f;
            for (int i4 = tid; i4 < d4; i4 += NT) {
                const uint2 xv2 = *reinterpret_cast<const uint2 *>(xb + 4 * i4);
                const float x0 = __uint_as_float(xv2.x << 16), x1 = __uint_as_float(xv2.x & 0xFFFF0000u);
                const float x2 = __uint_as_float(xv2.y << 16), x3 = __uint_as_float(xv2.y & 0xFFFF0000u);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j < nrows) {
                        const float4 wv = *reinterpret_cast<const float4 *>(rtr + (size_t)j * d + 4 * i4);
                        part[j] = fmaf(wv.x, x0, fmaf(wv.y, x1, fmaf(wv.z, x2, fmaf(wv.w, x3, part[j]))));
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < nrows) {
                    float v = part[j];
                    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    if (lane == 0) red[j * NW + warp] = v;
                }
            }
            csync();
            if (warp < nrows) {
                float v = lane < NW ? red[warp * NW + lane] : 0.f;
                for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) p.x_logits[cta + G * warp] = v + bias;
            }
            csync();   // this CTA's logits are stored
            if (tid == 0 && !(p.withhold && cta == 0)) ctr_arrive(p.cnt + S_LOGITS);
        }
        mark(1, clock64() - tl0);

        // ---- units -----------------------------------------------------------------------------
        // Unit i of this layer: items 3i (gate/up tile 2 c16), 3i + 1 (tile 2 c16 + 1), 3i + 2 (down
        // chunk c16 and its block's scales).  Every warp consumes every item in order (gate/up
        // items: the warps without a k chunk arrive through warp 0), so a wait never refers to a
        // fill older than the slot's previous one.
        auto item_slot = [&](int q, uint32_t &par) {
            const int a = ring_base + q;
            const int f = a / p.nslot;
            par = (uint32_t)(f & 1);
            return a - f * p.nslot;
        };
        auto run_unit = [&](int i) {
            const int n = unit_n(i);
            const int us = n / CH, c16 = n - us * CH;
            const float uw = ms->uw[us];
            float *gpb = gp + (size_t)(unit_ctr & 1) * 2 * SK_GWMAX * 16;
            bool uok = ok;
            // gate/up: this warp's 256-wide k chunk of both row tiles
            if (warp < GW) {
#pragma unroll 1
                for (int tt = 0; tt < 2 && uok; ++tt) {
                    uint32_t par;
                    const int s = item_slot(3 * i + tt, par);
                    const long long tw0 = clock64();
                    uok = mbar_wait(&ms->full[s], par, err, true);
                    tw += clock64() - tw0;
                    if (!uok) break;
                    const uint8_t *tile = ring + (size_t)s * p.slot_bytes;
                    float D0[4] = {0.f, 0.f, 0.f, 0.f}, D1[4] = {0.f, 0.f, 0.f, 0.f};
                    if constexpr (FMT == MOE_Q2B32) {
#pragma unroll
                        for (int kq = 0; kq < 4; ++kq) {
                            uint32_t rg[16];
                            q2_frag_h(*reinterpret_cast<const uint2 *>(tile + (size_t)(4 * warp + kq) * 256 + lane * 8), rg);
#pragma unroll
                            for (int m = 0; m < 4; ++m)
                                mma16816_h((m & 1) ? D1 : D0, rg[4 * m], rg[4 * m + 1], rg[4 * m + 2], rg[4 * m + 3],
                                           bx0[4 * kq + m], bx1[4 * kq + m]);
                        }
                    } else if constexpr (FMT == MOE_Q4B32) {
#pragma unroll
                        for (int kq = 0; kq < 4; ++kq) {
                            const uint4 a = *reinterpret_cast<const uint4 *>(tile + (size_t)(4 * warp + kq) * 512 + lane * 16);
                            const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                uint32_t a0, a1, a2, a3;
                                q4_frag_h(wv[m], a0, a1, a2, a3);
                                mma16816_h((m & 1) ? D1 : D0, a0, a1, a2, a3, bx0[4 * kq + m], bx1[4 * kq + m]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int kq = 0; kq < 4; ++kq) {
                            const uint32_t *wp = reinterpret_cast<const uint32_t *>(tile + (size_t)(4 * warp + kq) * 384 + lane * 12);
                            uint32_t rg[16];
                            q3_frag(wp[0], wp[1], wp[2], rg);
#pragma unroll
                            for (int m = 0; m < 4; ++m)
                                mma16816((m & 1) ? D1 : D0, rg[4 * m], rg[4 * m + 1], rg[4 * m + 2], rg[4 * m + 3],
                                         bx0[4 * kq + m], bx1[4 * kq + m]);
                        }
                    }
                    // columns 2c, 2c+1 = blocks 8*warp + 2c, +1
                    const __half *sc = reinterpret_cast<const __half *>(tile + p.gu.code_bytes);
                    const int b0 = 8 * warp + 2 * c;
                    const float2 sg = __half22float2(*reinterpret_cast<const __half2 *>(sc + g * nbd + b0));
                    const float2 s8 = __half22float2(*reinterpret_cast<const __half2 *>(sc + (g + 8) * nbd + b0));
                    const float x0 = xsum[b0], x1 = xsum[b0 + 1];
                    float ag, a8;
                    if constexpr (FMT == MOE_Q2B32) {
                        ag = fmaf(sg.x, D0[0] + D1[0] - 1026.f * x0, sg.y * fmaf(D0[1] + D1[1], 0.0625f, -66.f * x1));
                        a8 = fmaf(s8.x, fmaf(D0[2] + D1[2], 0.25f, -258.f * x0),
                                  s8.y * fmaf(D0[3] + D1[3], 0.015625f, -18.f * x1));
                    } else if constexpr (FMT == MOE_Q4B32) {
                        ag = fmaf(sg.x, D0[0] + D1[0] - 1032.f * x0, sg.y * (D0[1] + D1[1] - 1032.f * x1));
                        a8 = fmaf(s8.x, fmaf(D0[2] + D1[2], 0.0625f, -72.f * x0),
                                  s8.y * fmaf(D0[3] + D1[3], 0.0625f, -72.f * x1));
                    } else {
                        ag = fmaf(sg.x, D0[0] + D1[0] - 132.f * x0, sg.y * (D0[1] + D1[1] - 132.f * x1));
                        a8 = fmaf(s8.x, D0[2] + D1[2] - 132.f * x0, s8.y * (D0[3] + D1[3] - 132.f * x1));
                    }
                    ag += __shfl_xor_sync(0xffffffffu, ag, 1);
                    a8 += __shfl_xor_sync(0xffffffffu, a8, 1);
                    ag += __shfl_xor_sync(0xffffffffu, ag, 2);
                    a8 += __shfl_xor_sync(0xffffffffu, a8, 2);
                    if (c == 0) {
                        gpb[(tt * SK_GWMAX + warp) * 16 + g] = ag;
                        gpb[(tt * SK_GWMAX + warp) * 16 + 8 + g] = a8;
                    }
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&ms->empty[s]);
                        if (warp == 0)
                            for (int x = GW; x < NW; ++x) mbar_arrive(&ms->empty[s]);   // for the warps without a chunk
                    }
                }
            }
            // one barrier per unit: every warp's partials are in (the partial buffers alternate, so
            // the next unit's writes cannot meet this unit's reads); it also spreads a failure
            if (cta_failed(uok)) {
                ok = false;
                return;
            }
            // h of the unit's 16 rows (every warp, redundantly): lane r < 16 holds row r:
            // SwiGLU of the tile's gate row (r % 8) and up row (8 + r % 8), times the routing weight
            float hval = 0.f;
            if (lane < 16) {
                const int tt = lane >> 3, r = lane & 7;
                float gs = 0.f, us_ = 0.f;
                for (int w = 0; w < GW; ++w) {
                    gs += gpb[(tt * SK_GWMAX + w) * 16 + r];
                    us_ += gpb[(tt * SK_GWMAX + w) * 16 + 8 + r];
                }
                const float xi = ms->xinv;
                hval = silu(gs * xi) * (us_ * xi) * uw;
            }
            // hi + lo parts (fp16 of h * 2^s with s from the chunk's max |h|, or bf16), their sum
            float hsc = 1.f, hinv = 1.f;
            if constexpr (F16OP) {
                float mx = fabsf(hval);
                for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                int he;
                frexpf(mx, &he);
                const int sh = min(15 - he, 100);
                hsc = pow2i(sh);
                hinv = pow2i(-sh);
            }
            float hi_f, lo_f;
            uint16_t hi_b, lo_b;
            if constexpr (F16OP) {
                const float v = hval * hsc;
                const __half hh = __float2half_rn(v);
                hi_f = __half2float(hh);
                const __half ll = __float2half_rn(v - hi_f);
                lo_f = __half2float(ll);
                hi_b = *reinterpret_cast<const uint16_t *>(&hh);
                lo_b = *reinterpret_cast<const uint16_t *>(&ll);
            } else {
                hi_b = bf16_rn_bits(hval);
                hi_f = bf16_bits_f(hi_b);
                lo_b = bf16_rn_bits(hval - hi_f);
                lo_f = bf16_bits_f(lo_b);
            }
            float hsum = (lane < 16) ? hi_f + lo_f : 0.f;
            for (int o = 8; o; o >>= 1) hsum += __shfl_xor_sync(0xffffffffu, hsum, o);
            hsum = __shfl_sync(0xffffffffu, hsum, 0);
            // B fragment: column 0 = hi, column 1 = lo, other columns zero; k = 2c, 2c+1 (b0) and
            // 2c+8, 2c+9 (b1) of the chunk (lane r < 16 holds both parts of row r)
            const uint32_t pk = (uint32_t)hi_b | ((uint32_t)lo_b << 16);
            const uint32_t e0 = __shfl_sync(0xffffffffu, pk, 2 * c), e1 = __shfl_sync(0xffffffffu, pk, 2 * c + 1);
            const uint32_t e8 = __shfl_sync(0xffffffffu, pk, 2 * c + 8), e9 = __shfl_sync(0xffffffffu, pk, 2 * c + 9);
            const int sh16 = g == 0 ? 0 : 16;   // column 0: hi (low halves), column 1: lo
            uint32_t hb0 = ((e0 >> sh16) & 0xFFFFu) | (((e1 >> sh16) & 0xFFFFu) << 16);
            uint32_t hb1 = ((e8 >> sh16) & 0xFFFFu) | (((e9 >> sh16) & 0xFFFFu) << 16);
            if (g >= 2) hb0 = hb1 = 0u;
            // down: this warp's 64-row groups of the chunk (all d outputs)
            {
                uint32_t par;
                const int s = item_slot(3 * i + 2, par);
                const long long tw0 = clock64();
                uok = mbar_wait(&ms->full[s], par, err, true);
                tw += clock64() - tw0;
                if (uok) {
                    const uint8_t *chunk = ring + (size_t)s * p.slot_bytes;
                    const __half *sc = reinterpret_cast<const __half *>(chunk + p.chunk_bytes);   // [d]
                    for (int rq = warp; rq < d / 64; rq += NW) {
                        uint32_t a[16];
                        sk_frag16<FMT>(chunk + (size_t)rq * (32 * sk_piece<FMT>()) + lane * sk_piece<FMT>(), a);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            float D[4] = {0.f, 0.f, 0.f, 0.f};
                            if constexpr (FMT == MOE_Q3B32) mma16816(D, a[4 * m], a[4 * m + 1], a[4 * m + 2], a[4 * m + 3], hb0, hb1);
                            else mma16816_h(D, a[4 * m], a[4 * m + 1], a[4 * m + 2], a[4 * m + 3], hb0, hb1);
                            if (c == 0) {
                                // rows g (codes read as 1024 + F_g q) and g + 8 (1024 + F_8 q), columns hi + lo
                                float mg, m8, og, o8;
                                if constexpr (FMT == MOE_Q4B32) {
                                    mg = 1.f; og = 1032.f; m8 = 0.0625f; o8 = 72.f;
                                } else if constexpr (FMT == MOE_Q2B32) {
                                    if (m < 2) { mg = 1.f; og = 1026.f; m8 = 0.25f; o8 = 258.f; }
                                    else { mg = 0.0625f; og = 66.f; m8 = 0.015625f; o8 = 18.f; }
                                } else {
                                    mg = 1.f; og = 132.f; m8 = 1.f; o8 = 132.f;
                                }
                                const int row = 64 * rq + 16 * m + g;
                                const float yg = __half2float(sc[row]) * fmaf(D[0] + D[1], mg, -og * hsum) * hinv;
                                const float y8 = __half2float(sc[row + 8]) * fmaf(D[2] + D[3], m8, -o8 * hsum) * hinv;
                                atomicAdd(ysm + row, yg);
                                atomicAdd(ysm + row + 8, y8);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ms->empty[s]);
                }
            }
            if (!uok) ok = false;
            ++unit_ctr;
        };

        // ---- 3. shared-expert units, while the logits exchange is in flight --------------------
        for (int i = 0; i < ns && ok; ++i) run_unit(i);
        if (cta_failed(ok)) {
            aborted = true;
            break;
        }
        mark(2, clock64() - tl0);

        // ---- 4. top-k on all logits (same result in every CTA) --------------------------------------
        {
            if (tid == 0) {
                ok = ctr_wait(p.cnt + S_LOGITS, (unsigned)(G * (l + 1)), err);
                ms->ncand = 0;
            }
            if (cta_failed(ok)) {
                aborted = true;
                break;
            }
            mark(3, clock64() - tl0);
            // every CTA has read the previous layer's output: clear the owned columns of its buffer,
            // which accumulates the next layer's output
            if (l >= 1 && l + 1 < p.L) {
                float *ynext = p.y_acc + (size_t)((l + 1) & 1) * d;
                for (int i4 = own_lo + tid; i4 < own_hi; i4 += NT)
                    *reinterpret_cast<float4 *>(ynext + 4 * i4) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float m = -INFINITY;
            {
                float lv[SK_EMAX];
#pragma unroll
                for (int t = 0; t < SK_EMAX; ++t)
                    lv[t] = (tid + t * NT < E) ? __ldcg(p.x_logits + tid + t * NT) : -INFINITY;
#pragma unroll
                for (int t = 0; t < SK_EMAX; ++t) lv[t] = isnan(lv[t]) ? -INFINITY : lv[t];
#pragma unroll
                for (int t = 0; t < SK_EMAX; ++t) {
                    if (tid + t * NT < E) {
                        lg[tid + t * NT] = lv[t];
                        m = fmaxf(m, lv[t]);
                    }
                }
            }
            for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) ms->wmax[warp] = m;
            csync();
            const float ma = lane < NW ? ms->wmax[lane] : -INFINITY;
            float gmax = ma;
            for (int o = 16; o; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
            float tau = -INFINITY;
            if (k <= NW) {
                int above = 0;
#pragma unroll
                for (int b = 0; b < NW; ++b) {
                    const float mb = ms->wmax[b];
                    above += (mb > ma) || (mb == ma && b < lane);
                }
                const unsigned hit = __ballot_sync(0xffffffffu, lane < NW && above == k - 1);
                tau = __shfl_sync(0xffffffffu, ma, __ffs(hit) - 1);
            }
            for (int e0 = 0; e0 < E; e0 += NT) {
                const int e = e0 + tid;
                const float v = e < E ? lg[e] : -INFINITY;
                const bool take = e < E && v >= tau;
                const unsigned bal = __ballot_sync(0xffffffffu, take);
                if (bal) {
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&ms->ncand, __popc(bal));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const int slot = base + __popc(bal & ((1u << lane) - 1u));
                    if (take && slot < SK_CAND) ms->cand[slot] = make_float2(v, __int_as_float(e));
                }
            }
            csync();
            const int nc = ms->ncand;
            if (nc <= SK_CAND) {
                if (tid < nc) {
                    const float2 me = ms->cand[tid];
                    const float v = me.x;
                    const int id = __float_as_int(me.y);
                    int rank = 0, j = 0;
                    for (; j + 4 <= nc; j += 4) {
                        const float4 c01 = *reinterpret_cast<const float4 *>(&ms->cand[j]);
                        const float4 c23 = *reinterpret_cast<const float4 *>(&ms->cand[j + 2]);
                        rank += better(c01.x, __float_as_int(c01.y), v, id) + better(c01.z, __float_as_int(c01.w), v, id) +
                                better(c23.x, __float_as_int(c23.y), v, id) + better(c23.z, __float_as_int(c23.w), v, id);
                    }
                    for (; j < nc; ++j) {
                        const float2 o = ms->cand[j];
                        rank += better(o.x, __float_as_int(o.y), v, id);
                    }
                    if (rank < k) {
                        ms->ids[rank] = id;
                        ms->psel[rank] = expf(v - gmax);
                    }
                }
            } else if (warp == 0) {
                sk_topk_rounds(ms, lg, E, k, gmax);
            }
            csync();
            if (warp == NW - 1) {
                const float pj = lane < k ? ms->psel[lane] : 0.f;
                float z = pj;
                for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                if (lane < k) {
                    const float wj = pj / z;
                    const int id = ms->ids[lane];
                    ms->uw[lane] = wj;
                    ms->uexp[lane] = id;
                    if (cta == 0) {
                        if (p.stack && p.rec_on) {
                            const size_t ro = ((size_t)l * p.rec_n + p.rec_r) * k + lane;
                            if (p.rec.ids) p.rec.ids[ro] = id;
                            if (p.rec.w) p.rec.w[ro] = wj;
                        }
                        if (!p.stack) {
                            if (p.ids_out) p.ids_out[lane] = id;
                            if (p.w_out) p.w_out[lane] = wj;
                        }
                    }
                }
            }
            csync();
            if (tid == 0) mbar_arrive(&ms->route);   // the producer may issue the routed units
        }
        mark(4, clock64() - tl0);

        // ---- 5. routed units ----------------------------------------------------------------------
        for (int i = ns; i < nq && ok; ++i) run_unit(i);
        if (cta_failed(ok)) {
            aborted = true;
            break;
        }
        ring_base += 3 * nq;
        mark(5, clock64() - tl0);

        // ---- 6. this CTA's partial output -> the layer's output ------------------------------------
        {
            float *yacc = p.y_acc + (size_t)(l & 1) * d;
            for (int i4 = tid; i4 < d4; i4 += NT) {
                float4 v = *reinterpret_cast<const float4 *>(ysm + 4 * i4);
                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(yacc + 4 * i4), "f"(v.x), "f"(v.y),
                             "f"(v.z), "f"(v.w)
                             : "memory");
                *reinterpret_cast<float4 *>(ysm + 4 * i4) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            __threadfence();
            csync();
            if (tid == 0) ctr_arrive(p.cnt + S_Y);
        }
        mark(6, clock64() - tl0);
        mark(8, tw);
    }

    // ---- outputs of the last layer: each CTA its owned columns ------------------------------------
    if (!aborted) {
        if (tid == 0) ok = ctr_wait(p.cnt + S_Y, (unsigned)(G * p.L), err);
        if (!cta_failed(ok)) {
            const float *yl = p.y_acc + (size_t)((p.L - 1) & 1) * d;
            for (int i4 = own_lo + tid; i4 < own_hi; i4 += NT) {
                const float4 y = __ldcg(reinterpret_cast<const float4 *>(yl + 4 * i4));
                const uint16_t b0 = bf16_rn_bits(y.x), b1 = bf16_rn_bits(y.y), b2 = bf16_rn_bits(y.z), b3 = bf16_rn_bits(y.w);
                const uint2 yb2 = make_uint2((uint32_t)b0 | ((uint32_t)b1 << 16), (uint32_t)b2 | ((uint32_t)b3 << 16));
                if (p.stack) {
                    const float4 r = *reinterpret_cast<const float4 *>(rs + 4 * i4);
                    *reinterpret_cast<float4 *>(p.resid_out + 4 * i4) =
                        make_float4(r.x + bf16_bits_f(b0), r.y + bf16_bits_f(b1), r.z + bf16_bits_f(b2), r.w + bf16_bits_f(b3));
                    if (p.rec_on) {
                        const size_t ro = ((size_t)(p.L - 1) * p.rec_n + p.rec_r) * d + 4 * i4;
                        if (p.rec.y_bf16) *reinterpret_cast<uint2 *>(p.rec.y_bf16 + ro) = yb2;
                        if (p.rec.y_f32) *reinterpret_cast<float4 *>(p.rec.y_f32 + ro) = y;
                    }
                } else {
                    *reinterpret_cast<uint2 *>(p.y_out + 4 * i4) = yb2;
                    if (p.yf_out) *reinterpret_cast<float4 *>(p.yf_out + 4 * i4) = y;
                }
            }
        }
    }
}

}  // namespace

bool decode_split_supported(const moe_ctx *ctx) { return ctx->sdec.smem_bytes > 0; }

int decode_split_setup(moe_ctx *ctx) {
    const moe_config &c = ctx->cfg;
    SplitState &ss = ctx->sdec;
    ss.smem_bytes = 0;
    if (!ctx->split_layout) return MOE_OK;
    cudaDeviceProp prop;
    QE_CHECK(cudaGetDeviceProperties(&prop, ctx->device));
    int G = prop.multiProcessorCount;
    if (G > c.d_model / 16) G = c.d_model / 16;
    const int rpc = (c.n_experts + G - 1) / G;
    if (rpc > 8 || c.d_model > 4096 || c.d_model / 256 > SK_GWMAX || c.d_model / 256 > NW) return MOE_OK;
    if (c.top_k > SK_MAXK || c.n_experts % 4 || c.n_experts > 1024) return MOE_OK;
    const size_t down_item = (size_t)ctx->chunk.chunk_bytes + (size_t)c.d_model * 2;
    int slot = ctx->gu.tile_bytes > (int)down_item ? ctx->gu.tile_bytes : (int)down_item;
    slot = (slot + 127) & ~127;
    size_t fixed = 0;
    auto take = [&fixed](size_t bytes) {
        int off = (int)fixed;
        fixed = (fixed + bytes + 127) & ~(size_t)127;
        return off;
    };
    ss.off_router = take((size_t)rpc * c.d_model * 4);
    ss.off_xb = take((size_t)c.d_model * 2);
    ss.off_xh = take((size_t)c.d_model * 2);
    ss.off_logits = take((size_t)c.n_experts * 4);
    ss.off_gp = take((size_t)2 * 2 * SK_GWMAX * 16 * 4);
    ss.off_ysm = take((size_t)c.d_model * 4);
    ss.off_red = take((size_t)8 * NW * 4);
    ss.off_misc = take(sizeof(SkMisc));
    ss.off_resid = take((size_t)c.d_model * 4);
    ss.off_sums = take((size_t)(c.d_model / 32) * 4);
    ss.off_ltab = take((size_t)c.n_layers * sizeof(LayerPtrs));
    const size_t limit = (size_t)prop.sharedMemPerBlockOptin;
    int nslot = MAX_SLOTS;
    while (nslot >= 3 && fixed + (size_t)nslot * slot > limit) --nslot;
    if (nslot < 3) return MOE_OK;
    ss.off_ring = (int)fixed;
    ss.nslot = nslot;
    ss.slot_bytes = slot;
    ss.rpc = rpc;
    ss.grid = G;
    ss.smem_bytes = (int)(fixed + (size_t)nslot * slot);
    const void *kfn = c.fmt == MOE_Q4B32   ? (const void *)k_decode_split<MOE_Q4B32>
                      : c.fmt == MOE_Q2B32 ? (const void *)k_decode_split<MOE_Q2B32>
                                           : (const void *)k_decode_split<MOE_Q3B32>;
    QE_CHECK(cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, ss.smem_bytes));
    int per_sm = 0;
    QE_CHECK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, NTT, ss.smem_bytes));
    if (per_sm < 1) ss.smem_bytes = 0;
    return MOE_OK;
}

size_t decode_split_xchg_bytes(const moe_config &c) { return 256 + (size_t)c.n_experts * 4 + (size_t)2 * c.d_model * 4 + 256; }

int launch_decode_split(moe_ctx *ctx, int layer0, int L, const uint16_t *x, bool stack, float *resid_out, uint16_t *y,
                        float *yf, int32_t *ids, float *w, const moe_stack_record *rec, int rec_n, int rec_r,
                        cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    SplitState &ss = ctx->sdec;
    SplitParams p;
    memset(&p, 0, sizeof(p));
    p.layers = ctx->d_layers;
    p.layer0 = layer0;
    p.L = L;
    p.d = c.d_model;
    p.E = c.n_experts;
    p.I = c.d_ff;
    p.k = c.top_k;
    p.nsh = c.n_shared;
    p.gu = ctx->gu;
    p.chunk_bytes = ctx->chunk.chunk_bytes;
    p.dn_code_bytes = ctx->chunk.code_bytes;
    p.dn_expert_bytes = ctx->chunk.expert_bytes;
    p.stack = stack ? 1 : 0;
    p.x_in = x;
    p.resid_out = resid_out;
    p.y_out = y;
    p.yf_out = yf;
    p.ids_out = ids;
    p.w_out = w;
    if (rec) {
        p.rec = *rec;
        p.rec_on = 1;
        p.rec_n = rec_n;
        p.rec_r = rec_r;
    }
    uint8_t *xb = ss.xbuf;
    p.cnt = reinterpret_cast<unsigned *>(xb);
    p.x_logits = reinterpret_cast<float *>(xb + 256);
    p.y_acc = reinterpret_cast<float *>(xb + 256 + (((size_t)c.n_experts * 4 + 255) & ~(size_t)255));
    p.err = ctx->ws.dev_error;
    p.withhold = ((c.flags & MOE_FLAG_TEST_WITHHOLD) && !ctx->dec.withheld) ? 1 : 0;
    if (p.withhold) ctx->dec.withheld = true;
    if (c.flags & MOE_FLAG_TRACE) QE_TRY(decode_trace_buffer(ctx, ss.grid, L, SK_TRACE_WORDS, st, &p.trace));
    p.nslot = ss.nslot;
    p.slot_bytes = ss.slot_bytes;
    p.rpc = ss.rpc;
    p.off_ring = ss.off_ring;
    p.off_router = ss.off_router;
    p.off_xb = ss.off_xb;
    p.off_xh = ss.off_xh;
    p.off_logits = ss.off_logits;
    p.off_gp = ss.off_gp;
    p.off_ysm = ss.off_ysm;
    p.off_red = ss.off_red;
    p.off_misc = ss.off_misc;
    p.off_resid = ss.off_resid;
    p.off_sums = ss.off_sums;
    p.off_ltab = ss.off_ltab;
    // counters start from zero, and so do both output buffers
    QE_CHECK(cudaMemsetAsync(xb, 0, 256, st));
    QE_CHECK(cudaMemsetAsync(p.y_acc, 0, (size_t)2 * c.d_model * 4, st));
    void *args[] = {&p};
    const void *kfn = c.fmt == MOE_Q4B32   ? (const void *)k_decode_split<MOE_Q4B32>
                      : c.fmt == MOE_Q2B32 ? (const void *)k_decode_split<MOE_Q2B32>
                                           : (const void *)k_decode_split<MOE_Q3B32>;
    QE_CHECK(cudaLaunchCooperativeKernel(kfn, dim3(ss.grid), dim3(NTT), args, (size_t)ss.smem_bytes, st));
    QE_CHECK_LAUNCH("k_decode_split");
    return MOE_OK;
}

}  // namespace qeffn

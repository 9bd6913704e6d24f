// Single-token decode: one persistent kernel runs whole layers (and the whole
// 48-layer stack) with one CTA per SM.
//
// Per layer (one token):
//   1. every CTA rebuilds the layer input from the previous layer's output
//      (residual add + rmsnorm in the stack), bf16 -> fp16 in shared memory;
//   2. router: CTA c owns experts c, c+G, ...; their fp32 rows were bulk-copied
//      into shared memory one layer ahead; logits are published with a flag;
//   3. every CTA reads all E logits and selects the same top-k (threshold +
//      candidate ranking), then streams its share of the chosen experts'
//      packed weights (gate/up tiles, then down tiles) into a ring of shared
//      memory slots with cp.async.bulk, all issued as soon as slots free up;
//   4. gate/up: each 16-row tile (8 gate + 8 up rows) is one unit; the warps
//      split K, decode int4/int3 codes to exact fp16 (q - zero) and run
//      mma.m16n8k16 with the token in the B operand, one 32-block per column,
//      so each column collects one block's partial sum, which is scaled by the
//      block's fp16 scale in fp32; the SwiGLU output h is published;
//   5. down: units are (16 output rows, expert); h is split into fp16 hi + lo
//      (exact to 2^-22) and a CTA's contiguous run of units, weighted by the
//      routing weights, is summed per 16-row tile and published as one of at
//      most two parts per tile; the next layer adds the two parts in order.
// Cross-CTA data moves through "flagged words": a 64-bit store of (value,
// epoch) that a reader polls until the epoch matches, so every sync costs one
// L2 round trip and no separate barrier.  All waits are bounded (clock64); on
// timeout the kernel sets the context's error word and every CTA returns.
//
// Routing/combine passages: "Qwen3.8-Flash-Next at 45 Tokens/sec on a 12GB
// GPU?" (video transcript 1:50-2:16, 3:36-3:47); expert = SwiGLU and the block
// formats are this library's specification (see include/moe.h).
#include <math.h>
#include <string.h>

#include "moe_internal.cuh"

namespace qeffn {

namespace {

constexpr int NT = 384;
constexpr int NW = NT / 32;
constexpr int PRODUCER = NT - 32;   // lane 0 of the last warp issues every bulk copy
constexpr int MAX_SLOTS = 8;
constexpr int MAXK = 32;
constexpr int MAXU = MAXK + 4;
constexpr int CAND_MAX = 256;
constexpr long long SPIN_LIMIT = 2000000000LL;   // clock64 cycles, about one second

struct Misc {
    unsigned long long full[MAX_SLOTS];
    unsigned long long rbar;
    int ids[MAXK];
    float vsel[MAXK];
    float wsel[MAXK];
    int uexp[MAXU];
    float uw[MAXU];
    int ncand;
    int abort;
    float wmax[NW];
    float red1[NW];
    float cand_v[CAND_MAX];
    int cand_id[CAND_MAX];
};

struct DecodeParams {
    const LayerPtrs *layers;
    int layer0, L;
    int fmt, d, E, I, k, nsh;
    MatLayout gu, dn;
    int stack;                 // 1: residual stream + rmsnorm between layers
    const uint16_t *x_in;      // bf16 [d]
    float *resid_out;          // stack output [d]
    uint16_t *y_out;           // single layer: bf16 [d]
    float *yf_out;             // single layer: fp32 [d] or NULL
    int32_t *ids_out;          // single layer: [k] or NULL
    float *w_out;              // single layer: [k] or NULL
    moe_stack_record rec;      // stack records (row 0 only)
    int rec_on;
    uint2 *ll_logits;          // [2][E]
    uint2 *ll_h;               // [2][MAXU][I]
    uint2 *ll_y;               // [2][2][d]
    uint32_t epoch0;
    int *err;
    int withhold;              // test hook: CTA 0 does not publish its logits
    unsigned long long *trace; // [G][L][TRACE_WORDS] phase clocks, or NULL
    int nslot, slot_bytes, rpc;
    int dn_units_max;          // largest down-unit run of one CTA
    int off_ring, off_router, off_x16, off_logits, off_htab, off_red, off_misc, off_resid, off_sums;
};

// ---- PTX helpers -------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(unsigned long long *b, int count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(unsigned long long *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long *b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// A flagged word is one 64-bit value (low half: the float's bits, high half:
// the epoch), stored and loaded as 64-bit elements so that a reader never sees
// a new epoch with an old value.
__device__ __forceinline__ void ll_store(uint2 *p, float v, uint32_t flag) {
    unsigned long long w = ((unsigned long long)flag << 32) | __float_as_uint(v);
    asm volatile("st.volatile.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ void ll_load2(const uint2 *p, uint2 &a, uint2 &b) {
    unsigned long long x, y;
    asm volatile("ld.volatile.global.v2.u64 {%0, %1}, [%2];" : "=l"(x), "=l"(y) : "l"(p) : "memory");
    a = make_uint2((uint32_t)x, (uint32_t)(x >> 32));
    b = make_uint2((uint32_t)y, (uint32_t)(y >> 32));
}
__device__ __forceinline__ void mma16816(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Code -> bf16 without arithmetic: a field OR-ed into the low mantissa bits of
// 128.0 (0x4300) reads as 128 + q, exactly.  The offset is removed in fp32
// from each 32-block's partial sum: sum_k (128 + q_k) v_k - (128 + zero) *
// sum_k v_k = sum_k (q_k - zero) v_k, with the block sums of the activations
// precomputed once per layer (cancellation costs about 7 bits of the fp32
// partial, far below the output tolerance).
constexpr uint32_t BF_MAGIC = 0x43004300u;

// Q4B32: one word = the 8 codes of one k16 slice (nibble n = reg + 4*hi).
__device__ __forceinline__ void q4_frag(uint32_t w, uint32_t &a0, uint32_t &a1, uint32_t &a2,
                                        uint32_t &a3) {
    a0 = (w & 0x000F000Fu) | BF_MAGIC;
    a1 = ((w >> 4) & 0x000F000Fu) | BF_MAGIC;
    a2 = ((w >> 8) & 0x000F000Fu) | BF_MAGIC;
    a3 = ((w >> 12) & 0x000F000Fu) | BF_MAGIC;
}

// Q3B32: three words = the 16 fragment registers of four k16 slices.
__device__ __forceinline__ void q3_frag(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t r[16]) {
    uint32_t ws[3] = {w0, w1, w2};
#pragma unroll
    for (int j = 0; j < 3; ++j) {
#pragma unroll
        for (int f = 0; f < 5; ++f) r[5 * j + f] = ((ws[j] >> (3 * f)) & 0x00070007u) | BF_MAGIC;
    }
    uint32_t t = ((w0 >> 15) & 0x00010001u) | ((w1 >> 14) & 0x00020002u) | ((w2 >> 13) & 0x00040004u);
    r[15] = t | BF_MAGIC;
}

__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
    return v > bv || (v == bv && id < bid);
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&b);
}
__device__ __forceinline__ float bf16_bits_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ float silu(float z) { return z / (1.f + expf(-z)); }

// Sum of 32 consecutive bf16 values (16-byte aligned) with four 16-byte loads.
__device__ __forceinline__ float sum32_bf16(const uint16_t *p) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 v = q[j];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) acc[h] += __uint_as_float(w[h] << 16) + __uint_as_float(w[h] & 0xFFFF0000u);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Poll the flagged words base[i], i < n (n even, base 16-byte aligned): this
// thread owns the pairs (2q, 2q+1), q = tid + NT*j, and keeps up to B 16-byte
// loads in flight; put(i, value) receives each value once.
template <int B, typename F>
__device__ __forceinline__ bool poll_words(const uint2 *base, int n, uint32_t flag, int *err, F &&put) {
    long long t0 = clock64();
    const int np = n >> 1;
    for (int q0 = threadIdx.x; q0 < np; q0 += NT * B) {
        uint32_t need = 0;   // bit 2b: word 2q of load b, bit 2b+1: word 2q+1
#pragma unroll
        for (int b = 0; b < B; ++b)
            if (q0 + b * NT < np) need |= 3u << (2 * b);
        for (int it = 0;; ++it) {
            uint2 v[2 * B];
#pragma unroll
            for (int b = 0; b < B; ++b)
                if (need & (3u << (2 * b))) ll_load2(base + 2 * (q0 + b * NT), v[2 * b], v[2 * b + 1]);
#pragma unroll
            for (int h = 0; h < 2 * B; ++h) {
                if ((need >> h) & 1u) {
                    if (v[h].y == flag) {
                        put(2 * (q0 + (h >> 1) * NT) + (h & 1), __uint_as_float(v[h].x));
                        need &= ~(1u << h);
                    }
                }
            }
            if (!need) break;
            if ((it & 7) == 7) {
                if (*(volatile int *)err != 0) return false;
                if (clock64() - t0 > SPIN_LIMIT) {
                    atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
                    return false;
                }
            }
        }
    }
    return true;
}

__device__ __forceinline__ bool mbar_wait(unsigned long long *b, uint32_t parity, int *err, bool honor_err) {
    long long t0 = clock64();
    for (int it = 0;; ++it) {
        if (mbar_try_wait(b, parity)) return true;
        if ((it & 15) == 15) {
            if (honor_err && *(volatile int *)err != 0) return false;
            if (clock64() - t0 > SPIN_LIMIT) {
                atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
}

// CTA-uniform abort decision after a phase.
__device__ __forceinline__ bool cta_failed(Misc *ms, bool mine_ok) {
    if (!mine_ok) ms->abort = 1;
    __syncthreads();
    return ms->abort != 0;
}

constexpr int TRACE_WORDS = 24;   // per (CTA, layer) record: CTA, layer, 22 timestamps

__device__ __forceinline__ void trace_mark(const DecodeParams &p, int l, int ph, long long t) {
    if (p.trace && threadIdx.x == 0 && ph < TRACE_WORDS - 2) {
        unsigned long long *r = p.trace + ((size_t)blockIdx.x * p.L + l) * TRACE_WORDS;
        if (ph == 0) {
            r[0] = blockIdx.x;
            r[1] = l;
        }
        r[2 + ph] = (unsigned long long)t;
    }
}

template <int FMT>
__global__ void __launch_bounds__(NT, 1) k_decode(DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem + p.off_ring;
    float *rtr = reinterpret_cast<float *>(smem + p.off_router);
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem + p.off_x16);         // layer input, bf16 bits
    float *xsum = reinterpret_cast<float *>(smem + p.off_sums);              // [d/32] block sums of x
    float *hsum = xsum + p.d / 32;                                             // [nU][I/32] of h hi + lo
    float *lg = reinterpret_cast<float *>(smem + p.off_logits);
    uint16_t *htab = reinterpret_cast<uint16_t *>(smem + p.off_htab);   // bf16 hi / lo of h
    float *red = reinterpret_cast<float *>(smem + p.off_red);   // [2][NW][16]
    Misc *ms = reinterpret_cast<Misc *>(smem + p.off_misc);
    float *rs = reinterpret_cast<float *>(smem + p.off_resid);      // residual stream [d]
    float *ybuf = reinterpret_cast<float *>(smem + p.off_htab);     // [d], free between layers

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
    const int G = gridDim.x, cta = blockIdx.x;
    const int d = p.d, E = p.E, I = p.I, k = p.k;
    const int nU = k + p.nsh;
    const int nbd = d / 32, nbi = I / 32;
    const int ntile_gu = I / 8;          // gate/up tiles per expert
    const int ntile_dn = d / 16;         // down tiles per expert
    const int GW = d / 256;              // warps with a gate/up K chunk (256 k each)
    const int DW = I / 64;               // warps with a down k group (64 k each)
    const int dn_per_slot = p.slot_bytes / p.dn.tile_bytes;
    constexpr float off = (FMT == MOE_Q4B32) ? 136.f : 132.f;   // 128 + zero point
    int *err = p.err;

    if (tid == 0) {
        for (int s = 0; s < p.nslot; ++s) mbar_init(&ms->full[s], 1);
        mbar_init(&ms->rbar, 1);
        ms->abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // router rows of this CTA: experts cta + G*j
    auto issue_router = [&](int layer) {
        const float *rw = p.layers[layer].rw;
        int nrows = 0;
        for (int j = 0; j < p.rpc; ++j)
            if (cta + G * j < E) ++nrows;
        mbar_expect_tx(&ms->rbar, (uint32_t)(nrows * d * 4));
        for (int j = 0; j < nrows; ++j)
            bulk_g2s(rtr + (size_t)j * d, rw + (size_t)(cta + G * j) * d, (uint32_t)(d * 4), &ms->rbar);
    };
    if (tid == PRODUCER) issue_router(p.layer0);

    long long item = 0;                  // ring items planned so far (all layers)
    long long issued = 0;                // ring items whose copies were issued (thread 0)
    long long consumed = 0;              // ring items consumed so far
    int router_issued = 1, router_waited = 0;   // router prefetch fills (thread 0) / waits
    bool ok = true;

    for (int l = 0; l < p.L; ++l) {
        const int layer = p.layer0 + l;
        const LayerPtrs Lp = p.layers[layer];
        const uint32_t ep = p.epoch0 + (uint32_t)l;
        const int lpar = l & 1;
        const long long tl0 = clock64();

        // ---- 1. layer input -------------------------------------------------------
        if (p.stack) {
            float ss = 0.f;   // this thread's share of sum(r^2)
            if (l == 0) {
                for (int i = tid; i < d; i += NT) {
                    float v = bf16_bits_f(p.x_in[i]);
                    rs[i] = v;
                    ss = fmaf(v, v, ss);
                }
            } else {
                // previous layer's output = part 0 + part 1 of every row (same thread owns row i)
                const uint2 *y0 = p.ll_y + (size_t)((l - 1) & 1) * 2 * d;
                ok = poll_words<4>(y0, d, ep - 1, err, [&](int i, float v) { ybuf[i] = v; });
                ok = ok && poll_words<4>(y0 + d, d, ep - 1, err, [&](int i, float v) {
                    float y = ybuf[i] + v;
                    uint16_t yb = bf16_rn_bits(y);
                    float rn = rs[i] + bf16_bits_f(yb);
                    rs[i] = rn;
                    ss = fmaf(rn, rn, ss);
                    if (cta == 0 && p.rec_on) {
                        if (p.rec.y_bf16) p.rec.y_bf16[(size_t)(l - 1) * d + i] = yb;
                        if (p.rec.y_f32) p.rec.y_f32[(size_t)(l - 1) * d + i] = y;
                    }
                });
                if (cta_failed(ms, ok)) break;
            }
            trace_mark(p, l, 13, clock64() - tl0);
            for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (lane == 0) ms->red1[warp] = ss;
            __syncthreads();
            float tot = 0.f;
            for (int w = 0; w < NW; ++w) tot += ms->red1[w];
            float inv = 1.f / sqrtf(tot / (float)d + 1e-6f);
            for (int i = tid; i < d; i += NT) {
                uint16_t xv = bf16_rn_bits(rs[i] * inv);
                xb[i] = xv;
                if (cta == 0 && p.rec_on && p.rec.x_bf16) p.rec.x_bf16[(size_t)l * d + i] = xv;
            }
        } else {
            for (int i = tid; i < d; i += NT) xb[i] = p.x_in[i];
        }
        __syncthreads();
        // block sums of the input (offset removal in the gate/up flush)
        for (int b = tid; b < nbd; b += NT) xsum[b] = sum32_bf16(xb + 32 * b);

        trace_mark(p, l, 0, clock64() - tl0);
        // ---- 2. router ----------------------------------------------------------
        {
            ok = mbar_wait(&ms->rbar, (uint32_t)(l & 1), err, true);
            if (cta_failed(ms, ok)) break;
            ++router_waited;
            trace_mark(p, l, 14, clock64() - tl0);
            int nrows = 0;
            for (int j = 0; j < p.rpc; ++j)
                if (cta + G * j < E) ++nrows;
            // thread sums its strided share of 4-wide k chunks for every live row
            float part[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) part[j] = 0.f;
            for (int i4 = tid; i4 < d / 4; i4 += NT) {
                uint2 xv2 = *reinterpret_cast<const uint2 *>(xb + 4 * i4);
                float x0 = __uint_as_float(xv2.x << 16), x1 = __uint_as_float(xv2.x & 0xFFFF0000u);
                float x2 = __uint_as_float(xv2.y << 16), x3 = __uint_as_float(xv2.y & 0xFFFF0000u);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (j < nrows) {
                        float4 wv = *reinterpret_cast<const float4 *>(rtr + (size_t)j * d + 4 * i4);
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
            __syncthreads();
            trace_mark(p, l, 15, clock64() - tl0);
            if (tid < nrows && !(p.withhold && cta == 0)) {
                float v = 0.f;
                for (int w = 0; w < NW; ++w) v += red[tid * NW + w];
                int e = cta + G * tid;
                ll_store(p.ll_logits + (size_t)lpar * E + e, v + Lp.rb[e], ep);
            }
            __syncthreads();
            if (tid == PRODUCER && l + 1 < p.L) {
                fence_proxy_async();
                issue_router(layer + 1);
                ++router_issued;
            }
        }

        trace_mark(p, l, 1, clock64() - tl0);
        // ---- 3. top-k on all logits (same result in every CTA) ------------------------
        {
            ok = poll_words<2>(p.ll_logits + (size_t)lpar * E, E, ep, err, [&](int e, float v) { lg[e] = v; });
            if (tid == 0) ms->ncand = 0;
            if (cta_failed(ms, ok)) break;
            trace_mark(p, l, 8, clock64() - tl0);
            // threshold: the k-th largest of the warps' maxima bounds the k-th largest logit from below
            float m = -INFINITY;
            for (int e = tid; e < E; e += NT) m = fmaxf(m, lg[e]);
            for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) ms->wmax[warp] = m;
            __syncthreads();
            // lane a ranks warp maximum a among the NW maxima; the k-th one is the threshold
            float tau = -INFINITY;
            if (k <= NW) {
                float ma = lane < NW ? ms->wmax[lane] : -INFINITY;
                int above = 0;
                for (int b = 0; b < NW; ++b) {
                    float mb = ms->wmax[b];
                    above += (mb > ma) || (mb == ma && b < lane);
                }
                unsigned hit = __ballot_sync(0xffffffffu, lane < NW && above == k - 1);
                tau = __shfl_sync(0xffffffffu, ma, __ffs(hit) - 1);
            }
            for (int e = tid; e < E; e += NT) {
                float v = lg[e];
                if (v >= tau) {
                    int slot = atomicAdd(&ms->ncand, 1);
                    if (slot < CAND_MAX) {
                        ms->cand_v[slot] = v;
                        ms->cand_id[slot] = e;
                    }
                }
            }
            __syncthreads();
            int nc = ms->ncand;
            if (nc <= CAND_MAX) {
                if (tid < nc) {
                    float v = ms->cand_v[tid];
                    int id = ms->cand_id[tid];
                    int rank = 0;
                    for (int j = 0; j < nc; ++j) rank += better(ms->cand_v[j], ms->cand_id[j], v, id);
                    if (rank < k) {
                        ms->ids[rank] = id;
                        ms->vsel[rank] = v;
                    }
                }
            } else if (warp == 0) {
                // many candidates (ties or a flat distribution): k rounds of warp arg-max
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
                        float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                        int oid = __shfl_xor_sync(0xffffffffu, bid, o);
                        if (better(ov, oid, bv, bid)) {
                            bv = ov;
                            bid = oid;
                        }
                    }
                    if (lane == 0) {
                        ms->ids[j] = bid;
                        ms->vsel[j] = bv;
                    }
                    __syncwarp();
                }
            }
            __syncthreads();
            trace_mark(p, l, 9, clock64() - tl0);
            if (warp == 0) {
                float top = ms->vsel[0];
                float pj = lane < k ? expf(ms->vsel[lane] - top) : 0.f;
                float z = pj;
                for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                if (lane < k) {
                    float wj = pj / z;
                    ms->wsel[lane] = wj;
                    ms->uexp[lane] = ms->ids[lane];
                    ms->uw[lane] = wj;
                    if (cta == 0) {
                        if (p.stack && p.rec_on) {
                            if (p.rec.ids) p.rec.ids[(size_t)l * k + lane] = ms->ids[lane];
                            if (p.rec.w) p.rec.w[(size_t)l * k + lane] = wj;
                        }
                        if (!p.stack) {
                            if (p.ids_out) p.ids_out[lane] = ms->ids[lane];
                            if (p.w_out) p.w_out[lane] = wj;
                        }
                    }
                }
                if (lane < p.nsh) {
                    ms->uexp[k + lane] = E + lane;
                    ms->uw[k + lane] = 1.f;
                }
            }
            __syncthreads();
        }

        trace_mark(p, l, 2, clock64() - tl0);
        // ---- 4./5. stream and compute ----------------------------------------------
        const int n_gu_all = nU * ntile_gu;
        const int n_gu = (cta < n_gu_all) ? (n_gu_all - cta + G - 1) / G : 0;   // units cta, cta+G, ...
        const int n_dn_all = nU * ntile_dn;
        const int dn_lo = (int)((long long)cta * n_dn_all / G);
        const int dn_hi = (int)((long long)(cta + 1) * n_dn_all / G);
        const int n_dn = dn_hi - dn_lo;
        const int n_dn_items = (n_dn + dn_per_slot - 1) / dn_per_slot;
        const int n_items = n_gu + n_dn_items;
        const long long item_base = item;   // first ring item of this layer

        // item q of this layer -> ring slot; issue the copies of item q
        auto issue_item = [&](int q) {
            long long it = item_base + q;
            int s = (int)(it % p.nslot);
            uint8_t *dst = ring + (size_t)s * p.slot_bytes;
            if (q < n_gu) {
                int u = cta + G * q;
                int us = u / ntile_gu, t = u % ntile_gu;
                const uint8_t *src = Lp.gu + (size_t)ms->uexp[us] * p.gu.expert_bytes + (size_t)t * p.gu.tile_bytes;
                mbar_expect_tx(&ms->full[s], (uint32_t)p.gu.tile_bytes);
                bulk_g2s(dst, src, (uint32_t)p.gu.tile_bytes, &ms->full[s]);
            } else {
                int q0 = (q - n_gu) * dn_per_slot;
                int cnt = min(dn_per_slot, n_dn - q0);
                mbar_expect_tx(&ms->full[s], (uint32_t)(cnt * p.dn.tile_bytes));
                for (int i = 0; i < cnt; ++i) {
                    int n = dn_lo + q0 + i;
                    int j = n / nU, us = n % nU;
                    const uint8_t *src = Lp.dn + (size_t)ms->uexp[us] * p.dn.expert_bytes + (size_t)j * p.dn.tile_bytes;
                    bulk_g2s(dst + (size_t)i * p.dn.tile_bytes, src, (uint32_t)p.dn.tile_bytes, &ms->full[s]);
                }
            }
            ++issued;
        };
        if (tid == PRODUCER) {
            fence_proxy_async();
            int first = min(n_items, p.nslot);
            for (int q = 0; q < first; ++q) issue_item(q);
        }
        item += n_items;

        // gate/up B fragments of this warp's 256-wide k chunk (token in one column per block)
        uint32_t bx0[16], bx1[16];
        if (warp < GW) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                int s = 16 * warp + j;
                bool act = (g == (j >> 1));
                uint32_t v0 = *reinterpret_cast<const uint32_t *>(xb + 16 * s + 2 * c);
                uint32_t v1 = *reinterpret_cast<const uint32_t *>(xb + 16 * s + 2 * c + 8);
                bx0[j] = act ? v0 : 0u;
                bx1[j] = act ? v1 : 0u;
            }
        }
        long long tw_gu = 0, tw_dn = 0;   // cycles spent waiting for weights (trace)

        // ---- gate/up: every warp with a k chunk walks all gate/up units of this CTA, waiting
        // on each unit's barrier itself; partial sums go to red_gu[unit][warp][row]
        if (warp < GW) {
            for (int q = 0; q < n_gu && ok; ++q) {
                long long it = item_base + q;
                int s = (int)(it % p.nslot);
                long long tw0 = clock64();
                ok = mbar_wait(&ms->full[s], (uint32_t)((it / p.nslot) & 1), err, true);
                long long tw1 = clock64();
                tw_gu += tw1 - tw0;
                if (!ok) break;
                const uint8_t *tile = ring + (size_t)s * p.slot_bytes;
                float D0[4] = {0.f, 0.f, 0.f, 0.f}, D1[4] = {0.f, 0.f, 0.f, 0.f};
                if constexpr (FMT == MOE_Q4B32) {
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq) {
                        uint4 a = *reinterpret_cast<const uint4 *>(tile + (size_t)(4 * warp + kq) * 512 + lane * 16);
                        uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            uint32_t a0, a1, a2, a3;
                            q4_frag(wv[m], a0, a1, a2, a3);
                            mma16816((m & 1) ? D1 : D0, a0, a1, a2, a3, bx0[4 * kq + m], bx1[4 * kq + m]);
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
                int b0 = 8 * warp + 2 * c;
                float2 sg = __half22float2(*reinterpret_cast<const __half2 *>(sc + g * nbd + b0));
                float2 s8 = __half22float2(*reinterpret_cast<const __half2 *>(sc + (g + 8) * nbd + b0));
                const float o0 = off * xsum[b0], o1 = off * xsum[b0 + 1];
                float ag = fmaf(sg.x, D0[0] + D1[0] - o0, sg.y * (D0[1] + D1[1] - o1));
                float a8 = fmaf(s8.x, D0[2] + D1[2] - o0, s8.y * (D0[3] + D1[3] - o1));
                ag += __shfl_xor_sync(0xffffffffu, ag, 1);
                a8 += __shfl_xor_sync(0xffffffffu, a8, 1);
                ag += __shfl_xor_sync(0xffffffffu, ag, 2);
                a8 += __shfl_xor_sync(0xffffffffu, a8, 2);
                if (c == 0) {
                    red[(q * NW + warp) * 16 + g] = ag;
                    red[(q * NW + warp) * 16 + 8 + g] = a8;
                }
                if (q < 6) trace_mark(p, l, 16 + q, clock64() - tw1);
            }
        }
        if (cta_failed(ms, ok)) break;
        trace_mark(p, l, 6, clock64() - tl0);
        consumed += n_gu;
        // the gate/up slots are free: queue the down batches that did not fit the ring yet
        if (tid == PRODUCER) {
            fence_proxy_async();
            for (int q = p.nslot; q < n_items && q < n_gu + p.nslot; ++q) issue_item(q);
        }
        // SwiGLU of every gate/up unit in parallel: thread (unit q, row i)
        if (tid < n_gu * 8) {
            int q = tid >> 3, i = tid & 7;
            float gs = 0.f, us_ = 0.f;
            for (int w = 0; w < GW; ++w) {
                gs += red[(q * NW + w) * 16 + i];
                us_ += red[(q * NW + w) * 16 + 8 + i];
            }
            int u = cta + G * q;
            int uslot = u / ntile_gu, t = u % ntile_gu;
            ll_store(p.ll_h + ((size_t)lpar * MAXU + uslot) * I + 8 * t + i, silu(gs) * us_, ep);
        }
        trace_mark(p, l, 3, clock64() - tl0);

        // h of every expert in use -> fp16 hi + lo table
        {
            ok = poll_words<8>(p.ll_h + (size_t)lpar * MAXU * I, nU * I, ep, err, [&](int i, float h) {
                uint16_t hi = bf16_rn_bits(h);
                uint16_t lo = bf16_rn_bits(h - bf16_bits_f(hi));
                int us = i / I, kk = i % I;
                htab[(size_t)(2 * us) * I + kk] = hi;
                htab[(size_t)(2 * us + 1) * I + kk] = lo;
            });
            if (cta_failed(ms, ok)) break;
            for (int t = tid; t < nU * nbi; t += NT) {
                int us = t / nbi, b = t % nbi;
                hsum[t] = sum32_bf16(htab + (size_t)(2 * us) * I + 32 * b) +
                          sum32_bf16(htab + (size_t)(2 * us + 1) * I + 32 * b);
            }
            __syncthreads();
        }
        trace_mark(p, l, 4, clock64() - tl0);

        // ---- down: every warp with a k group walks all down units of this CTA's contiguous
        // run [dn_lo, dn_hi) ((tile, expert) order); partials to red[unit][warp][row]
        if (warp < DW) {
            for (int qi = 0; qi < n_dn_items && ok; ++qi) {
                long long it = item_base + n_gu + qi;
                int s = (int)(it % p.nslot);
                long long tw0 = clock64();
                ok = mbar_wait(&ms->full[s], (uint32_t)((it / p.nslot) & 1), err, true);
                tw_dn += clock64() - tw0;
                if (!ok) break;
                int q0 = qi * dn_per_slot;
                int cnt = min(dn_per_slot, n_dn - q0);
                for (int ui = 0; ui < cnt; ++ui) {
                    int nl = q0 + ui, n = dn_lo + nl;
                    int us = n % nU;
                    const uint8_t *tile = ring + (size_t)s * p.slot_bytes + (size_t)ui * p.dn.tile_bytes;
                    float D[4] = {0.f, 0.f, 0.f, 0.f};
                    const uint16_t *hp = htab + (size_t)(2 * us + (g & 1)) * I;
                    uint32_t a[16];
                    if constexpr (FMT == MOE_Q4B32) {
                        uint4 av = *reinterpret_cast<const uint4 *>(tile + (size_t)warp * 512 + lane * 16);
                        q4_frag(av.x, a[0], a[1], a[2], a[3]);
                        q4_frag(av.y, a[4], a[5], a[6], a[7]);
                        q4_frag(av.z, a[8], a[9], a[10], a[11]);
                        q4_frag(av.w, a[12], a[13], a[14], a[15]);
                    } else {
                        const uint32_t *wp = reinterpret_cast<const uint32_t *>(tile + (size_t)warp * 384 + lane * 12);
                        q3_frag(wp[0], wp[1], wp[2], a);
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        int sl = 4 * warp + m;           // k16 slice within K = I
                        bool act = ((sl >> 1) & 3) == (g >> 1);
                        uint32_t b0 = act ? *reinterpret_cast<const uint32_t *>(hp + 16 * sl + 2 * c) : 0u;
                        uint32_t b1 = act ? *reinterpret_cast<const uint32_t *>(hp + 16 * sl + 2 * c + 8) : 0u;
                        mma16816(D, a[4 * m], a[4 * m + 1], a[4 * m + 2], a[4 * m + 3], b0, b1);
                    }
                    // columns 2c (hi) and 2c+1 (lo) of block 4*(warp/2) + c
                    int blk = 4 * (warp >> 1) + c;
                    bool valid = (c >> 1) == (warp & 1);
                    float ag = 0.f, a8 = 0.f;
                    if (valid) {
                        const __half *sc = reinterpret_cast<const __half *>(tile + p.dn.code_bytes);
                        const float o = off * hsum[us * nbi + blk];
                        ag = __half2float(sc[g * nbi + blk]) * (D[0] + D[1] - o);
                        a8 = __half2float(sc[(g + 8) * nbi + blk]) * (D[2] + D[3] - o);
                    }
                    ag += __shfl_xor_sync(0xffffffffu, ag, 1);
                    a8 += __shfl_xor_sync(0xffffffffu, a8, 1);
                    ag += __shfl_xor_sync(0xffffffffu, ag, 2);
                    a8 += __shfl_xor_sync(0xffffffffu, a8, 2);
                    if (c == 0) {
                        red[(nl * DW + warp) * 16 + g] = ag;
                        red[(nl * DW + warp) * 16 + 8 + g] = a8;
                    }
                }
            }
        }
        if (cta_failed(ms, ok)) break;
        consumed += n_dn_items;
        trace_mark(p, l, 7, clock64() - tl0);
        // unit sums (thread per (unit, row)), then per tile the fixed-order weighted sum
        float *vsum = red + (size_t)p.dn_units_max * DW * 16;   // [unit][16]
        for (int t = tid; t < n_dn * 16; t += NT) {
            int nl = t >> 4, r = t & 15;
            float v = 0.f;
            for (int w = 0; w < DW; ++w) v += red[(nl * DW + w) * 16 + r];
            vsum[t] = v;
        }
        __syncthreads();
        {
            int j_first = dn_lo / nU, j_last = (dn_hi - 1) / nU;
            int n_tiles_mine = j_last - j_first + 1;
            for (int t = tid; t < n_tiles_mine * 16; t += NT) {
                int j = j_first + (t >> 4), r = t & 15;
                int first = j * nU, last = j * nU + nU - 1;
                int n0 = max(first, dn_lo), n1 = min(last, dn_hi - 1);
                float y = 0.f;
                for (int n = n0; n <= n1; ++n) y = fmaf(ms->uw[n % nU], vsum[(n - dn_lo) * 16 + r], y);
                int part = (first >= dn_lo) ? 0 : 1;
                uint2 *yb = p.ll_y + (size_t)lpar * 2 * d;
                ll_store(yb + (size_t)part * d + 16 * j + r, y, ep);
                if (part == 0 && last < dn_hi) ll_store(yb + d + 16 * j + r, 0.f, ep);
            }
        }
        trace_mark(p, l, 5, clock64() - tl0);
        trace_mark(p, l, 10, tw_gu);
        trace_mark(p, l, 12, tw_dn);
    }

    // ---- outputs of the last layer ---------------------------------------------------
    if (!ms->abort && ok) {
        const int l = p.L - 1;
        const uint32_t ep = p.epoch0 + (uint32_t)l;
        const uint2 *y0 = p.ll_y + (size_t)(l & 1) * 2 * d;
        if (cta == 0) {
            ok = poll_words<4>(y0, d, ep, err, [&](int i, float v) { ybuf[i] = v; });
            ok = ok && poll_words<4>(y0 + d, d, ep, err, [&](int i, float v) {
                float y = ybuf[i] + v;
                uint16_t yb = bf16_rn_bits(y);
                if (p.stack) {
                    p.resid_out[i] = rs[i] + bf16_bits_f(yb);
                    if (p.rec_on) {
                        if (p.rec.y_bf16) p.rec.y_bf16[(size_t)l * d + i] = yb;
                        if (p.rec.y_f32) p.rec.y_f32[(size_t)l * d + i] = y;
                    }
                } else {
                    p.y_out[i] = yb;
                    if (p.yf_out) p.yf_out[i] = y;
                }
            });
        }
    }
    // drain copies still in flight (abort path) before the CTA's shared memory goes away
    if (tid == PRODUCER) {
        for (long long it = consumed; it < issued; ++it)
            mbar_wait(&ms->full[(int)(it % p.nslot)], (uint32_t)((it / p.nslot) & 1), err, false);
        if (router_issued > router_waited)
            mbar_wait(&ms->rbar, (uint32_t)(router_waited & 1), err, false);
    }
    __syncthreads();
}

}  // namespace

bool decode_supported(const moe_ctx *ctx, int T) {
    const moe_config &c = ctx->cfg;
    if (T != 1 || (c.flags & MOE_FLAG_NO_DECODE_KERNEL)) return false;
    if (c.n_experts % 2) return false;   // flagged words are polled in 16-byte pairs
    if (c.d_model > 4096 || c.d_model / 256 > NW || c.d_ff / 64 > NW) return false;
    if (c.top_k > MAXK || c.top_k + c.n_shared > MAXU) return false;
    return ctx->dec.smem_bytes > 0;
}

int decode_setup(moe_ctx *ctx) {
    const moe_config &c = ctx->cfg;
    DecodeState &ds = ctx->dec;
    int dev = ctx->device;
    cudaDeviceProp prop;
    QE_CHECK(cudaGetDeviceProperties(&prop, dev));
    int G = prop.multiProcessorCount;
    ds.sms = G;
    if (G > c.d_model / 16) G = c.d_model / 16;   // a down tile then spans at most two CTAs
    ds.grid = G;
    int rpc = (c.n_experts + G - 1) / G;
    if (rpc > 8) {
        ds.smem_bytes = 0;
        return MOE_OK;
    }
    int slot = ctx->gu.tile_bytes;
    if (slot < ctx->dn.tile_bytes) slot = ctx->dn.tile_bytes;
    // carve shared memory: each region 128-byte aligned, in this order, no overlap
    size_t fixed = 0;
    auto take = [&fixed](size_t bytes) {
        int off = (int)fixed;
        fixed = (fixed + bytes + 127) & ~(size_t)127;
        return off;
    };
    // per-CTA unit counts (gate/up round-robin, down contiguous runs)
    int nU = c.top_k + c.n_shared;
    int gu_max = (nU * (c.d_ff / 8) + G - 1) / G;
    int dn_max = (nU * (c.d_model / 16) + G - 1) / G;
    size_t red_bytes = (size_t)8 * NW * 4;                                   // router partials
    if (red_bytes < (size_t)gu_max * NW * 16 * 4) red_bytes = (size_t)gu_max * NW * 16 * 4;
    if (red_bytes < (size_t)dn_max * (NW + 1) * 16 * 4) red_bytes = (size_t)dn_max * (NW + 1) * 16 * 4;
    ds.gu_units_max = gu_max;
    ds.dn_units_max = dn_max;
    ds.off_router = take((size_t)rpc * c.d_model * 4);
    ds.off_x16 = take((size_t)c.d_model * 2);
    ds.off_logits = take((size_t)c.n_experts * 4);
    size_t htab = (size_t)(c.top_k + c.n_shared) * 2 * c.d_ff * 2;   // fp16 hi + lo of h
    if (htab < (size_t)c.d_model * 4) htab = (size_t)c.d_model * 4;    // doubles as the y buffer
    ds.off_htab = take(htab);
    ds.off_red = take(red_bytes);
    ds.off_misc = take(sizeof(Misc));
    ds.off_resid = take((size_t)c.d_model * 4);
    ds.off_sums = take((size_t)(c.d_model / 32 + nU * (c.d_ff / 32)) * 4);
    size_t limit = (size_t)prop.sharedMemPerBlockOptin;
    int nslot = MAX_SLOTS;
    while (nslot >= 2 && fixed + (size_t)nslot * slot > limit) --nslot;
    int dn_per_slot = slot / ctx->dn.tile_bytes;
    // every gate/up tile of a layer and, after them, every down batch must fit the ring at once
    if (nslot < 2 || gu_max > nslot || (dn_max + dn_per_slot - 1) / dn_per_slot > nslot) {
        ds.smem_bytes = 0;
        return MOE_OK;
    }
    ds.off_ring = (int)fixed;
    ds.nslot = nslot;
    ds.slot_bytes = slot;
    ds.rpc = rpc;
    ds.smem_bytes = (int)(fixed + (size_t)nslot * slot);
    const void *kfn = (c.fmt == MOE_Q4B32) ? (const void *)k_decode<MOE_Q4B32> : (const void *)k_decode<MOE_Q3B32>;
    QE_CHECK(cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, ds.smem_bytes));
    int per_sm = 0;
    QE_CHECK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, NT, ds.smem_bytes));
    if (per_sm < 1) ds.smem_bytes = 0;
    return MOE_OK;
}

size_t decode_ll_bytes(const moe_config &c) {
    return sizeof(uint2) * ((size_t)2 * c.n_experts + (size_t)2 * MAXU * c.d_ff + (size_t)4 * c.d_model);
}

int launch_decode(moe_ctx *ctx, int layer0, int L, const uint16_t *x, bool stack, float *resid_out,
                  uint16_t *y, float *yf, int32_t *ids, float *w, const moe_stack_record *rec,
                  cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    DecodeState &ds = ctx->dec;
    DecodeParams p;
    memset(&p, 0, sizeof(p));
    p.layers = ctx->d_layers;
    p.layer0 = layer0;
    p.L = L;
    p.fmt = c.fmt;
    p.d = c.d_model;
    p.E = c.n_experts;
    p.I = c.d_ff;
    p.k = c.top_k;
    p.nsh = c.n_shared;
    p.gu = ctx->gu;
    p.dn = ctx->dn;
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
    }
    p.ll_logits = ds.ll;
    p.ll_h = ds.ll + (size_t)2 * c.n_experts;
    p.ll_y = p.ll_h + (size_t)2 * MAXU * c.d_ff;
    p.epoch0 = ds.epoch;
    ds.epoch += (uint32_t)L + 1;
    if (ds.epoch < (uint32_t)L + 2) ds.epoch = 1;   // wrapped: never reuse 0 (initial contents)
    p.err = ctx->ws.dev_error;
    p.withhold = (c.flags & MOE_FLAG_TEST_WITHHOLD) ? 1 : 0;
    if (c.flags & MOE_FLAG_TRACE) {
        size_t need = (size_t)ds.grid * L * TRACE_WORDS;
        if (need > ds.trace_cap) {
            if (ds.trace) ctx_free(ctx, ds.trace);
            ds.trace = nullptr;
            QE_CHECK(cudaSetDevice(ctx->device));
            int s = ctx_alloc(ctx, (void **)&ds.trace, need * 8, "trace");
            if (s != MOE_OK) return s;
            ds.trace_cap = need;
        }
        QE_CHECK(cudaMemsetAsync(ds.trace, 0, need * 8, st));
        ds.trace_n = (int)(ds.grid * L);
        ds.trace_words = TRACE_WORDS;
        p.trace = ds.trace;
    }
    p.nslot = ds.nslot;
    p.slot_bytes = ds.slot_bytes;
    p.rpc = ds.rpc;
    p.dn_units_max = ds.dn_units_max;
    p.off_ring = ds.off_ring;
    p.off_router = ds.off_router;
    p.off_x16 = ds.off_x16;
    p.off_logits = ds.off_logits;
    p.off_htab = ds.off_htab;
    p.off_red = ds.off_red;
    p.off_misc = ds.off_misc;
    p.off_resid = ds.off_resid;
    p.off_sums = ds.off_sums;
    void *args[] = {&p};
    const void *kfn = (c.fmt == MOE_Q4B32) ? (const void *)k_decode<MOE_Q4B32> : (const void *)k_decode<MOE_Q3B32>;
    QE_CHECK(cudaLaunchCooperativeKernel(kfn, dim3(ds.grid), dim3(NT), args,
                                         (size_t)ds.smem_bytes, st));
    QE_CHECK_LAUNCH("k_decode");
    return MOE_OK;
}

}  // namespace qeffn

// Single-token decode: one persistent kernel runs whole layers (and the whole
// 48-layer stack) with one CTA per SM: 12 compute warps, which synchronise on
// a named barrier, and one producer warp that issues every bulk copy and is
// paced by mbarriers only (a thread that issues copies can stall while the
// copy engine's queue drains; the compute warps must not wait for it).
//
// Per layer (one token):
//   1. every CTA rebuilds the layer input from the previous layer's output
//      (residual add + rmsnorm in the stack): bf16 x and, for Q4, fp16 x * 2^s
//      (a power of two that keeps every value inside fp16) in shared memory;
//   2. router: CTA c owns experts c, c+G, ...; their fp32 rows were bulk-copied
//      into shared memory during the previous layer; logits are exchanged;
//   3. every CTA reads all E logits and selects the same top-k (threshold +
//      candidate ranking), then streams its share of the chosen experts'
//      packed weights (gate/up tiles, then down tiles) into a ring of shared
//      memory slots with cp.async.bulk, refilling each slot as soon as its
//      gate/up tile is consumed;
//   4. gate/up: each 16-row tile (8 gate + 8 up rows) is one unit; the warps
//      split K, turn int4/int3 codes into fp16/bf16 operands by OR-ing them
//      into the mantissa of a constant (no arithmetic), and run
//      mma.m16n8k16 with the token in the B operand, one 32-block per column,
//      so each column collects one block's partial sum; the constant's share
//      is removed with the block sums of x and the block's fp16 scale applied
//      in fp32; the SwiGLU output h is exchanged;
//   5. down: units are (16 output rows, expert), one warp per unit over the
//      whole K; h enters as hi + lo parts (Q4: fp16 of h * 2^s with s per
//      32-block, about 2^-22 relative; Q3: bf16, about 2^-16), and a
//      CTA's contiguous run of units, weighted by the routing weights, is
//      summed per 16-row tile into one of at most two parts per tile; the next
//      layer adds the two parts in order.
// The three exchanges per layer (logits, h, output parts) go through plain
// fp32 buffers and one arrival counter each (see "cross-CTA exchanges" below).
// All waits are bounded (clock64); on timeout the kernel sets the context's
// error word and every CTA returns.
//
// Routing/combine passages: "Qwen3.8-Flash-Next at 45 Tokens/sec on a 12GB
// GPU?" (video transcript 1:50-2:16, 3:36-3:47); expert = SwiGLU and the block
// formats are this library's specification (see include/moe.h).
#include <math.h>
#include <string.h>

#include "decode_common.cuh"

namespace qeffn {

namespace {

using namespace dec;

constexpr int MAXK = 32;
constexpr int MAXU = MAXK + 4;
constexpr int CAND_MAX = 256;
constexpr int YMAX = 3;    // float4 groups of the output per thread (d <= 4096)
constexpr int EMAX = 3;    // logits per thread (E <= 1024)
constexpr int HB = 4;      // float4 loads of h in flight per thread

struct Misc {
    unsigned long long full[MAX_SLOTS];
    unsigned long long empty[MAX_SLOTS];   // gate/up item consumed by every gate/up warp
    unsigned long long rbar;
    unsigned long long route;              // one arrival per layer: routing known (ids in uexp)
    int ids[MAXK];
    float psel[MAXK];          // exp(logit - max logit) of the selected experts, in rank order
    int uexp[MAXU];
    float uw[MAXU];
    int ncand;
    float xinv;                // 2^-s: undoes the power-of-two scaling of the fp16 layer input
    float wmax[NW];
    float red1[NW];
    float amax[NW];
    __align__(16) float2 cand[CAND_MAX];     // (logit, id bits)
};

struct DecodeParams {
    const LayerPtrs *layers;
    int layer0, L;
    int d, E, I, k, nsh;
    MatLayout gu, dn;
    int stack;                 // 1: residual stream + rmsnorm between layers
    const uint16_t *x_in;      // bf16 [d]
    float *resid_out;          // stack output [d]
    uint16_t *y_out;           // single layer: bf16 [d]
    float *yf_out;             // single layer: fp32 [d] or NULL
    int32_t *ids_out;          // single layer: [k] or NULL
    float *w_out;              // single layer: [k] or NULL
    moe_stack_record rec;      // stack records: this token is record row rec_r of rec_n
    int rec_on, rec_n, rec_r;
    unsigned *cnt;             // exchange counters: logits, h, y (128 bytes apart)
    float *x_logits;           // [E]
    float *x_h;                // [MAXU][I]
    float *x_y;                // [2][d]: the two parts of every output row
    int *err;
    int withhold;              // test hook: CTA 0 does not publish its logits
    int l2_mode;               // 0: plain copies; 1: shared experts kept in L2, the rest streamed
    unsigned long long *trace; // [G][L][TRACE_WORDS] phase clocks, or NULL
    int nslot, slot_bytes, rpc;
    int off_ring, off_router, off_x16, off_xh, off_logits, off_htab, off_red, off_misc, off_resid, off_sums,
        off_ltab;
};

// ---- cross-CTA exchanges ------------------------------------------------------
// Each exchange: every CTA stores its share of a plain fp32 buffer, one thread
// adds 1 to the exchange's counter with release semantics, and the readers
// wait (acquire) until all G CTAs have arrived, then load the buffer with
// gpu-scope loads (never from a stale L1 line).  The three exchanges of a
// layer (logits, h, y) have one counter each; CTA 0 zeroes the counter of the
// next exchange before it arrives at the current one: that counter was last
// waited on two exchanges earlier, which every CTA has left by the time it can
// arrive at the current one, and the release orders the zeroing before any
// CTA's next arrival there.
constexpr int X_LOGITS = 0, X_H = 1, X_Y = 2;
__device__ __forceinline__ unsigned *ctr(const DecodeParams &p, int kind) { return p.cnt + 32 * kind; }
// Thread 0 of every CTA, after a barrier that follows the CTA's stores.
__device__ __forceinline__ void xchg_arrive(const DecodeParams &p, int kind, bool arrive = true) {
    if (blockIdx.x == 0) ctr_zero(ctr(p, (kind + 1) % 3));
    if (arrive) ctr_arrive(ctr(p, kind));
}

// Trace record per (CTA, layer): word 0 = CTA, word 1 = layer, word 2 + slot =
// SM clock cycles since the layer started in this CTA, except where noted:
//   13 previous layer's output received   0 layer input ready
//   14 router rows in shared memory       15 router dot products done
//    1 logits published                    8 all logits received
//    2 routing known                      11 this thread's gate/up units done
//    6 every gate/up unit done             3 h published
//    4 every expert's h received           9 this thread's down units done
//    7 every down unit done                5 output tiles published
//   10 cycles waiting for gate/up data    12 cycles waiting for down data
//   16 / 17 warp 0's first down unit: accumulation done / reduced (cycles
//      since its data was ready)
//   21 global timer (ns) at the layer start
constexpr int TRACE_WORDS = 24;

// Out of line: the record store is rare, and the kernel's code footprint per
// layer is what the instruction cache sees.
__device__ __noinline__ void trace_store(unsigned long long *trace, int L, int l, int ph, long long t) {
    unsigned long long *r = trace + ((size_t)blockIdx.x * L + l) * TRACE_WORDS;
    if (ph == 0) {
        r[0] = blockIdx.x;
        r[1] = l;
    }
    r[2 + ph] = (unsigned long long)t;
}
__device__ __forceinline__ void trace_mark(const DecodeParams &p, int l, int ph, long long t) {
    if (p.trace && threadIdx.x == 0 && ph < TRACE_WORDS - 2) trace_store(p.trace, p.L, l, ph, t);
}

// Top-k by k rounds of warp arg-max (warp 0), for the rare case of more
// candidates than the ranking buffer holds (many equal logits).
__device__ __noinline__ void topk_argmax_rounds(Misc *ms, const float *lg, int E, int k, float gmax) {
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
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oid = __shfl_xor_sync(0xffffffffu, bid, o);
            if (better(ov, oid, bv, bid)) {
                bv = ov;
                bid = oid;
            }
        }
        if (lane == 0) {
            ms->ids[j] = bid;
            ms->uexp[j] = bid;
            ms->psel[j] = expf(bv - gmax);
        }
        __syncwarp();
    }
}

template <int FMT>
__global__ void __launch_bounds__(NTT, 1) k_decode(DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem + p.off_ring;
    float *rtr = reinterpret_cast<float *>(smem + p.off_router);
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem + p.off_x16);         // layer input, bf16 bits
    uint16_t *xh = reinterpret_cast<uint16_t *>(smem + p.off_xh);          // layer input * 2^s, fp16 bits
    float *xsum = reinterpret_cast<float *>(smem + p.off_sums);              // [d/32] block sums of x
    float *hsum = xsum + p.d / 32;                                             // [nU][I/32] of h hi + lo
    float *hinv = hsum + (p.k + p.nsh) * (p.I / 32);                           // [nU][I/32] Q4: 2^-s of the block
    float *lg = reinterpret_cast<float *>(smem + p.off_logits);
    // h of every expert in use, hi and lo parts, in B-fragment order (see the down phase)
    uint16_t *htab = reinterpret_cast<uint16_t *>(smem + p.off_htab);
    float *red = reinterpret_cast<float *>(smem + p.off_red);   // [2][NW][16]
    Misc *ms = reinterpret_cast<Misc *>(smem + p.off_misc);
    float *rs = reinterpret_cast<float *>(smem + p.off_resid);      // residual stream [d]
    LayerPtrs *ltab = reinterpret_cast<LayerPtrs *>(smem + p.off_ltab);   // [L] weight pointers

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
    const int JN = (I + 127) / 128;      // k-group pairs of the down K (h table blocks)
    constexpr bool F16OP = (FMT != MOE_Q3B32);   // fp16 operands (Q4B32, Q2B32), else bf16 (Q3B32)
    const uint32_t ONE2 = F16OP ? 0x3C003C00u : 0x3F803F80u;   // 1.0 in both halves
    constexpr float off = (FMT == MOE_Q4B32) ? 136.f : 132.f;   // 128 + zero point
    int *err = p.err;

    if (tid == 0) {
        for (int s = 0; s < p.nslot; ++s) {
            mbar_init(&ms->full[s], 1);
            mbar_init(&ms->empty[s], p.d / 256);   // one arrival per gate/up warp
        }
        mbar_init(&ms->rbar, 1);
        mbar_init(&ms->route, 1);
        fence_mbar_init();
    }
    if (tid < p.nsh) {   // shared experts follow the routed ones in the unit list, weight 1
        ms->uexp[k + tid] = E + tid;
        ms->uw[k + tid] = 1.f;
    }
    for (int l = tid; l < p.L; l += NTT) ltab[l] = p.layers[p.layer0 + l];   // this call's layers
    __syncthreads();

    // per-layer unit split of this CTA (same in the producer and the compute warps)
    struct Split {
        int n_gu, n_dn, dn_lo, dn_hi, n_dn_items, n_items;
    };
    auto split = [&]() {
        Split sp;
        const int n_gu_all = nU * ntile_gu;
        sp.n_gu = (cta < n_gu_all) ? (n_gu_all - cta + G - 1) / G : 0;   // units cta, cta+G, ...
        const int n_dn_all = nU * ntile_dn;
        sp.dn_lo = cta * n_dn_all / G;   // n_dn_all * G < 2^31
        sp.dn_hi = (cta + 1) * n_dn_all / G;
        sp.n_dn = sp.dn_hi - sp.dn_lo;
        sp.n_dn_items = (sp.n_dn + dn_per_slot - 1) / dn_per_slot;
        sp.n_items = sp.n_gu + sp.n_dn_items;
        return sp;
    };
    // ring slot of item q of a layer whose first item sits in slot s0 (fill parity p0)
    auto ring_slot = [&](int s0, uint32_t p0, int q, uint32_t &par) {
        int sq = s0 + q;
        par = p0;
        while (sq >= p.nslot) {
            sq -= p.nslot;
            par ^= 1u;
        }
        return sq;
    };

    // ---- producer warp (lane 0): every bulk copy, paced by mbarriers only ----------------
    if (warp == NW) {
        if (lane != 0) return;
        const uint64_t keep_pol = l2_policy(true), stream_pol = l2_policy(false);
        uint32_t gu_par = 0;     // bit s: parity of the gate/up items issued into slot s so far
        uint32_t fill_par = 0;   // bit s: parity of all fills of slot s so far
        uint32_t filled = 0;     // bit s: slot s was filled at least once
        int router_fills = 0;
        // router rows of this CTA: experts cta + G*j
        auto issue_router = [&](int layer) {
            const float *rw = ltab[layer - p.layer0].rw;
            int nrows = 0;
            for (int j = 0; j < p.rpc; ++j)
                if (cta + G * j < E) ++nrows;
            fence_proxy_async();
            mbar_expect_tx(&ms->rbar, (uint32_t)(nrows * d * 4));
            for (int j = 0; j < nrows; ++j)
                weight_copy(rtr + (size_t)j * d, rw + (size_t)(cta + G * j) * d, (uint32_t)(d * 4), &ms->rbar,
                            p.l2_mode, false, keep_pol, stream_pol);
            ++router_fills;
        };
        issue_router(p.layer0);
        int s0 = 0;
        uint32_t p0 = 0;
        for (int l = 0; l < p.L; ++l) {
            const int layer = p.layer0 + l;
            const LayerPtrs Lp = ltab[l];
            // the compute warps have chosen the experts (uexp) and are done with the previous
            // layer's slots and with the router rows
            if (!mbar_wait(&ms->route, (uint32_t)(l & 1), err, true)) break;
            const Split sp = split();
            bool pok = true;
            fence_proxy_async();   // (the compute warps only read the ring)
            for (int q = 0; q < sp.n_items && pok; ++q) {
                uint32_t par;
                const int s = ring_slot(s0, p0, q, par);
                // items past the ring reuse a slot whose gate/up unit of this layer is consumed
                if (q >= p.nslot) pok = mbar_wait(&ms->empty[s], ((gu_par >> s) & 1u) ^ 1u, err, true);
                if (!pok) break;
                uint8_t *dst = ring + (size_t)s * p.slot_bytes;
                if (q < sp.n_gu) {
                    const int u = cta + G * q;
                    const int us = u / ntile_gu, t = u % ntile_gu;
                    const uint8_t *src = Lp.gu + (size_t)ms->uexp[us] * p.gu.expert_bytes + (size_t)t * p.gu.tile_bytes;
                    mbar_expect_tx(&ms->full[s], (uint32_t)p.gu.tile_bytes);
                    weight_copy(dst, src, (uint32_t)p.gu.tile_bytes, &ms->full[s], p.l2_mode, ms->uexp[us] >= E,
                                keep_pol, stream_pol);
                    gu_par ^= 1u << s;
                } else {
                    const int q0 = (q - sp.n_gu) * dn_per_slot;
                    const int cnt = min(dn_per_slot, sp.n_dn - q0);
                    mbar_expect_tx(&ms->full[s], (uint32_t)(cnt * p.dn.tile_bytes));
                    for (int i = 0; i < cnt; ++i) {
                        const int n = sp.dn_lo + q0 + i;
                        const int j = n / nU, us = n % nU;
                        const uint8_t *src = Lp.dn + (size_t)ms->uexp[us] * p.dn.expert_bytes + (size_t)j * p.dn.tile_bytes;
                        weight_copy(dst + (size_t)i * p.dn.tile_bytes, src, (uint32_t)p.dn.tile_bytes, &ms->full[s],
                                    p.l2_mode, ms->uexp[us] >= E, keep_pol, stream_pol);
                    }
                }
                fill_par ^= 1u << s;
                filled |= 1u << s;
            }
            if (!pok) break;
            if (l + 1 < p.L) issue_router(layer + 1);
            uint32_t par;
            s0 = ring_slot(s0, p0, sp.n_items, par);
            p0 = par;
        }
        // every copy has landed before the CTA's shared memory goes away (the last fill of each
        // slot and the last router fill; earlier fills of a slot completed before its reuse)
        for (int s = 0; s < p.nslot; ++s)
            if ((filled >> s) & 1u) mbar_wait(&ms->full[s], ((fill_par >> s) & 1u) ^ 1u, err, false);
        if (router_fills > 0) mbar_wait(&ms->rbar, (uint32_t)((router_fills - 1) & 1), err, false);
        return;
    }

    int ring_s0 = 0;                     // ring slot of this layer's first item
    uint32_t ring_p0 = 0;                // and the parity of that slot's fill
    bool ok = true;
    bool aborted = false;                // CTA-uniform: the layer loop was left on a failure

    for (int l = 0; l < p.L; ++l) {
        const LayerPtrs Lp = ltab[l];
        const long long tl0 = clock64();
        if (p.trace) {   // global time of the layer start (ns), to line up the CTAs' clocks
            unsigned long long gt;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(gt));
            trace_mark(p, l, 21, (long long)gt);
        }

        // ---- 1. layer input -------------------------------------------------------
        // xb = bf16 input; for Q4 also xh = fp16(x * 2^s) with the power of two chosen from
        // max |x| so that every value fits fp16 (|x| * 2^s < 2^15), exact for bf16 inputs
        float amx = 0.f;   // this thread's share of max |r| (stack) or max |x|
        float inv = 1.f;
        if (p.stack) {
            float ss = 0.f;   // this thread's share of sum(r^2)
            if (l == 0) {
                for (int i = tid; i < d; i += NT) {
                    float v = bf16_bits_f(p.x_in[i]);
                    rs[i] = v;
                    ss = fmaf(v, v, ss);
                    amx = fmaxf(amx, fabsf(v));
                }
            } else {
                // previous layer's output = part 0 + part 1 of every row, once every CTA published
                if (tid == 0) ok = ctr_wait(ctr(p, X_Y), (unsigned)G, err);
                if (cta_failed(ok)) {
                    aborted = true;
                    break;
                }
                // every load first (one L2 round trip), then the arithmetic
                float4 pa[YMAX], pb[YMAX];
#pragma unroll
                for (int t = 0; t < YMAX; ++t) {
                    const int i4 = tid + t * NT;
                    if (i4 < d / 4) {
                        pa[t] = ld_gpu4(p.x_y + 4 * i4);
                        pb[t] = ld_gpu4(p.x_y + d + 4 * i4);
                    }
                }
#pragma unroll
                for (int t = 0; t < YMAX; ++t) {
                    const int i4 = tid + t * NT;
                    if (i4 >= d / 4) break;
                    const float4 a = pa[t], b = pb[t];
                    const float ya[4] = {a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int i = 4 * i4 + j;
                        const float y = ya[j];
                        const uint16_t yb = bf16_rn_bits(y);
                        const float rn = rs[i] + bf16_bits_f(yb);
                        rs[i] = rn;
                        ss = fmaf(rn, rn, ss);
                        amx = fmaxf(amx, fabsf(rn));
                        if (cta == 0 && p.rec_on) {
                            const size_t ro = ((size_t)(l - 1) * p.rec_n + p.rec_r) * d + i;
                            if (p.rec.y_bf16) p.rec.y_bf16[ro] = yb;
                            if (p.rec.y_f32) p.rec.y_f32[ro] = y;
                        }
                    }
                }
            }
            trace_mark(p, l, 13, clock64() - tl0);
            for (int o = 16; o; o >>= 1) {
                ss += __shfl_xor_sync(0xffffffffu, ss, o);
                amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, o));
            }
            if (lane == 0) {
                ms->red1[warp] = ss;
                ms->amax[warp] = amx;
            }
            if (cta_failed(ok)) {
                aborted = true;
                break;
            }
            float tot = lane < NW ? ms->red1[lane] : 0.f;
            amx = lane < NW ? ms->amax[lane] : 0.f;
            for (int o = 16; o; o >>= 1) {
                tot += __shfl_xor_sync(0xffffffffu, tot, o);
                amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, o));
            }
            inv = 1.f / sqrtf(tot / (float)d + 1e-6f);
            amx = bf16_bits_f(bf16_rn_bits(amx * inv));   // = max |bf16(r * inv)| (monotone rounding)
        } else {
            for (int i = tid; i < d; i += NT) {
                uint16_t v = p.x_in[i];
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
        frexpf(amx, &xe);                    // amx < 2^xe
        const int xs_exp = min(15 - xe, 100);
        const float xscale = pow2i(xs_exp);
        if (tid == 0) ms->xinv = F16OP ? pow2i(-xs_exp) : 1.f;
        // 8 consecutive elements per thread: bf16 (stack: rounded from r * inv), fp16 of x * 2^s
        for (int i8 = tid; i8 < d / 8; i8 += NT) {
            uint32_t xw[4], hw[4];
            if (p.stack) {
                const float4 r0 = reinterpret_cast<const float4 *>(rs)[2 * i8];
                const float4 r1 = reinterpret_cast<const float4 *>(rs)[2 * i8 + 1];
                const float rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    xw[j] = (uint32_t)bf16_rn_bits(rv[2 * j] * inv) |
                            ((uint32_t)bf16_rn_bits(rv[2 * j + 1] * inv) << 16);
                *reinterpret_cast<uint4 *>(xb + 8 * i8) = make_uint4(xw[0], xw[1], xw[2], xw[3]);
                if (cta == 0 && p.rec_on && p.rec.x_bf16) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        p.rec.x_bf16[((size_t)l * p.rec_n + p.rec_r) * d + 8 * i8 + j] =
                            (uint16_t)(xw[j >> 1] >> (16 * (j & 1)));
                }
            } else {
                const uint4 v = *reinterpret_cast<const uint4 *>(xb + 8 * i8);
                xw[0] = v.x; xw[1] = v.y; xw[2] = v.z; xw[3] = v.w;
            }
            if constexpr (F16OP) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    __half2 h2 = __floats2half2_rn(__uint_as_float(xw[j] << 16) * xscale,
                                                   __uint_as_float(xw[j] & 0xFFFF0000u) * xscale);
                    hw[j] = *reinterpret_cast<uint32_t *>(&h2);
                }
                *reinterpret_cast<uint4 *>(xh + 8 * i8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            }
        }
        csync();
        // block sums of the operand the gate/up MMAs see (offset removal in their flush)
        for (int b = tid; b < nbd; b += NT)
            xsum[b] = F16OP ? sum32_f16(xh + 32 * b) : sum32_bf16(xb + 32 * b);

        trace_mark(p, l, 0, clock64() - tl0);
        // ---- 2. router ----------------------------------------------------------
        {
            int nrows = 0;
            for (int j = 0; j < p.rpc; ++j)
                if (cta + G * j < E) ++nrows;
            // this warp's bias (row warp), loaded now so that its latency hides behind the dot products
            const float bias = (warp < nrows && lane == 0) ? __ldg(Lp.rb + cta + G * warp) : 0.f;
            ok = mbar_wait(&ms->rbar, (uint32_t)(l & 1), err, true);
            if (cta_failed(ok)) {
                aborted = true;
                break;
            }
            trace_mark(p, l, 14, clock64() - tl0);
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
            csync();   // partials written; every read of the router rows is done
            trace_mark(p, l, 15, clock64() - tl0);
            if (warp < nrows) {   // warp j sums row j's NW partials
                float v = lane < NW ? red[warp * NW + lane] : 0.f;
                for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                const int e = cta + G * warp;
                if (lane == 0) p.x_logits[e] = v + bias;
            }
        }

        trace_mark(p, l, 1, clock64() - tl0);
        // ---- 3. top-k on all logits (same result in every CTA) ------------------------
        {
            csync();   // this CTA's logits are stored
            if (tid == 0) {
                xchg_arrive(p, X_LOGITS, !(p.withhold && cta == 0));
                ok = ctr_wait(ctr(p, X_LOGITS), (unsigned)G, err);
                ms->ncand = 0;
            }
            if (cta_failed(ok)) {
                aborted = true;
                break;
            }
            float m = -INFINITY;   // max of the logits this thread read (every warp reads some)
            {
                float lv[EMAX];
#pragma unroll
                for (int t = 0; t < EMAX; ++t)
                    lv[t] = (tid + t * NT < E) ? ld_gpu(p.x_logits + tid + t * NT) : -INFINITY;
                // a NaN logit ranks as -inf (last, by id): the selection below then always
                // finds k distinct experts below E
#pragma unroll
                for (int t = 0; t < EMAX; ++t) lv[t] = isnan(lv[t]) ? -INFINITY : lv[t];
#pragma unroll
                for (int t = 0; t < EMAX; ++t) {
                    if (tid + t * NT < E) {
                        lg[tid + t * NT] = lv[t];
                        m = fmaxf(m, lv[t]);
                    }
                }
            }
            for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) ms->wmax[warp] = m;
            csync();
            trace_mark(p, l, 8, clock64() - tl0);
            // the k-th largest of the warps' maxima bounds the k-th largest logit from below:
            // lane a ranks warp maximum a among the NW maxima
            const float ma = lane < NW ? ms->wmax[lane] : -INFINITY;
            float gmax = ma;
            for (int o = 16; o; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
            float tau = -INFINITY;
            if (k <= NW) {
                int above = 0;
#pragma unroll
                for (int b = 0; b < NW; ++b) {
                    float mb = ms->wmax[b];
                    above += (mb > ma) || (mb == ma && b < lane);
                }
                unsigned hit = __ballot_sync(0xffffffffu, lane < NW && above == k - 1);
                tau = __shfl_sync(0xffffffffu, ma, __ffs(hit) - 1);
            }
            // candidates (logit >= tau), appended with one shared atomic per warp and pass
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
                    if (take && slot < CAND_MAX) ms->cand[slot] = make_float2(v, __int_as_float(e));
                }
            }
            csync();
            const int nc = ms->ncand;
            if (nc <= CAND_MAX) {
                // rank of candidate t = number of candidates ordered before it (value desc, id asc)
                if (tid < nc) {
                    const float2 me = ms->cand[tid];
                    const float v = me.x;
                    const int id = __float_as_int(me.y);
                    int rank = 0, j = 0;
                    for (; j + 4 <= nc; j += 4) {
                        const float4 c01 = *reinterpret_cast<const float4 *>(&ms->cand[j]);
                        const float4 c23 = *reinterpret_cast<const float4 *>(&ms->cand[j + 2]);
                        rank += better(c01.x, __float_as_int(c01.y), v, id) +
                                better(c01.z, __float_as_int(c01.w), v, id) +
                                better(c23.x, __float_as_int(c23.y), v, id) +
                                better(c23.z, __float_as_int(c23.w), v, id);
                    }
                    for (; j < nc; ++j) {
                        const float2 o = ms->cand[j];
                        rank += better(o.x, __float_as_int(o.y), v, id);
                    }
                    if (rank < k) {
                        ms->ids[rank] = id;
                        ms->uexp[rank] = id;
                        ms->psel[rank] = expf(v - gmax);
                    }
                }
            } else if (warp == 0) {
                topk_argmax_rounds(ms, lg, E, k, gmax);   // many candidates (ties or a flat distribution)
            }
            csync();
        }

        if (tid == 0) mbar_arrive(&ms->route);   // the producer may issue this layer's copies
        trace_mark(p, l, 2, clock64() - tl0);
        // ---- 4./5. stream and compute ----------------------------------------------
        // the producer warp streams the gate/up tiles, then the down batches (each into a slot
        // as soon as that slot's gate/up unit is consumed), then the next layer's router rows
        const Split sp = split();
        const int n_gu = sp.n_gu, n_dn = sp.n_dn, dn_lo = sp.dn_lo, dn_hi = sp.dn_hi;
        const int n_items = sp.n_items;
        auto slot_of = [&](int q, uint32_t &par) { return ring_slot(ring_s0, ring_p0, q, par); };
        // routing weights (needed from the down flush on): renormalised over the selected
        // experts, in rank order
        if (warp == NW - 1) {
            const float pj = lane < k ? ms->psel[lane] : 0.f;
            float z = pj;
            for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            if (lane < k) {
                const float wj = pj / z;
                const int id = ms->ids[lane];
                ms->uw[lane] = wj;
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

        // gate/up B fragments of this warp's 256-wide k chunk (token in one column per block)
        // (Q4: fp16 x * 2^s, Q3: bf16 x)
        uint32_t bx0[16], bx1[16];
        if (warp < GW) {
            const uint16_t *xop = F16OP ? xh : xb;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                int s = 16 * warp + j;
                bool act = (g == (j >> 1));
                uint32_t v0 = *reinterpret_cast<const uint32_t *>(xop + 16 * s + 2 * c);
                uint32_t v1 = *reinterpret_cast<const uint32_t *>(xop + 16 * s + 2 * c + 8);
                bx0[j] = act ? v0 : 0u;
                bx1[j] = act ? v1 : 0u;
            }
        }
        long long tw_gu = 0, tw_dn = 0;   // cycles spent waiting for weights (trace)

        // ---- gate/up: every warp with a k chunk walks all gate/up units of this CTA, waiting
        // on each unit's barrier itself; partial sums go to red_gu[unit][warp][row]
        if (warp < GW) {
            for (int q = 0; q < n_gu && ok; ++q) {
                uint32_t par;
                const int s = slot_of(q, par);
                long long tw0 = clock64();
                ok = mbar_wait(&ms->full[s], par, err, true);
                long long tw1 = clock64();
                tw_gu += tw1 - tw0;
                if (!ok) break;
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
                        uint4 a = *reinterpret_cast<const uint4 *>(tile + (size_t)(4 * warp + kq) * 512 + lane * 16);
                        uint32_t wv[4] = {a.x, a.y, a.z, a.w};
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
                int b0 = 8 * warp + 2 * c;
                float2 sg = __half22float2(*reinterpret_cast<const __half2 *>(sc + g * nbd + b0));
                float2 s8 = __half22float2(*reinterpret_cast<const __half2 *>(sc + (g + 8) * nbd + b0));
                float ag, a8;
                if constexpr (FMT == MOE_Q2B32) {
                    // column 2c = the k group's first block: rows g read 1024 + q, rows g+8 1024 + 4q;
                    // column 2c+1 = its second block: 1024 + 16q and 1024 + 64q
                    const float x0 = xsum[b0], x1 = xsum[b0 + 1];
                    ag = fmaf(sg.x, D0[0] + D1[0] - 1026.f * x0, sg.y * fmaf(D0[1] + D1[1], 0.0625f, -66.f * x1));
                    a8 = fmaf(s8.x, fmaf(D0[2] + D1[2], 0.25f, -258.f * x0),
                              s8.y * fmaf(D0[3] + D1[3], 0.015625f, -18.f * x1));
                } else if constexpr (FMT == MOE_Q4B32) {
                    // row g: codes read as 1024 + q; row g+8: as 1024 + 16 q (sums scaled by 1/16)
                    const float x0 = xsum[b0], x1 = xsum[b0 + 1];
                    ag = fmaf(sg.x, D0[0] + D1[0] - 1032.f * x0, sg.y * (D0[1] + D1[1] - 1032.f * x1));
                    a8 = fmaf(s8.x, fmaf(D0[2] + D1[2], 0.0625f, -72.f * x0),
                              s8.y * fmaf(D0[3] + D1[3], 0.0625f, -72.f * x1));
                } else {
                    const float o0 = off * xsum[b0], o1 = off * xsum[b0 + 1];
                    ag = fmaf(sg.x, D0[0] + D1[0] - o0, sg.y * (D0[1] + D1[1] - o1));
                    a8 = fmaf(s8.x, D0[2] + D1[2] - o0, s8.y * (D0[3] + D1[3] - o1));
                }
                ag += __shfl_xor_sync(0xffffffffu, ag, 1);
                a8 += __shfl_xor_sync(0xffffffffu, a8, 1);
                ag += __shfl_xor_sync(0xffffffffu, ag, 2);
                a8 += __shfl_xor_sync(0xffffffffu, a8, 2);
                if (c == 0) {
                    red[(q * NW + warp) * 16 + g] = ag;
                    red[(q * NW + warp) * 16 + 8 + g] = a8;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ms->empty[s]);   // this warp is done with the slot
            }
        }
        trace_mark(p, l, 11, clock64() - tl0);   // thread 0's own gate/up units done
        if (cta_failed(ok)) {
            aborted = true;
            break;
        }
        trace_mark(p, l, 6, clock64() - tl0);
        // SwiGLU of every gate/up unit in parallel: thread (unit q, row i)
        if (tid < n_gu * 8) {
            int q = tid >> 3, i = tid & 7;
            float gs = 0.f, us_ = 0.f;
            for (int w = 0; w < GW; ++w) {
                gs += red[(q * NW + w) * 16 + i];
                us_ += red[(q * NW + w) * 16 + 8 + i];
            }
            const float xinv = ms->xinv;
            gs *= xinv;
            us_ *= xinv;
            int u = cta + G * q;
            int uslot = u / ntile_gu, t = u % ntile_gu;
            p.x_h[(size_t)uslot * I + 8 * t + i] = silu(gs) * us_;
        }
        trace_mark(p, l, 3, clock64() - tl0);

        // h of every expert in use -> hi + lo table (B-fragment order) and per-block sums of hi + lo
        {
            csync();   // this CTA's h values are stored
            if (tid == 0) {
                xchg_arrive(p, X_H);
                ok = ctr_wait(ctr(p, X_H), (unsigned)G, err);
            }
            if (cta_failed(ok)) {
                aborted = true;
                break;
            }
            // 4 values per thread; the 8 lanes of a 32-block are neighbours in the warp.
            // Q4: fp16 hi + lo of h * 2^s, s per 32-block from the block's max |h| (so the
            //     values fit fp16; the down flush multiplies by 2^-s);
            // Q3: bf16 hi + lo of h.
            const int n4 = nU * I / 4;   // a multiple of 8 (I % 64 == 0)
            for (int b4 = 0; b4 < n4; b4 += HB * NT) {
                float4 hb[HB];   // a batch of loads in flight together, then the arithmetic
#pragma unroll
                for (int t = 0; t < HB; ++t) {
                    hb[t] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (b4 + t * NT + tid < n4) hb[t] = ld_gpu4(p.x_h + 4 * (b4 + t * NT + tid));
                }
#pragma unroll
                for (int t = 0; t < HB; ++t) {
                    const int i4 = b4 + t * NT + tid;
                    const bool valid = i4 < n4;
                    const float hv[4] = {hb[t].x, hb[t].y, hb[t].z, hb[t].w};
                    float scale = 1.f;
                    if constexpr (F16OP) {
                        float mx = fmaxf(fmaxf(fabsf(hv[0]), fabsf(hv[1])), fmaxf(fabsf(hv[2]), fabsf(hv[3])));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                        int he;
                        frexpf(mx, &he);   // mx < 2^he
                        const int sh = min(15 - he, 100);
                        scale = pow2i(sh);
                        if (valid && (lane & 7) == 0) hinv[i4 >> 3] = pow2i(-sh);
                    }
                    float part = 0.f;
                    if (valid) {
                        uint32_t hi2[2], lo2[2];
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            if constexpr (F16OP) {
                                const float v0 = hv[2 * j] * scale, v1 = hv[2 * j + 1] * scale;
                                const __half2 hh = __floats2half2_rn(v0, v1);
                                const float2 hf = __half22float2(hh);
                                const __half2 ll = __floats2half2_rn(v0 - hf.x, v1 - hf.y);
                                const float2 lf = __half22float2(ll);
                                hi2[j] = *reinterpret_cast<const uint32_t *>(&hh);
                                lo2[j] = *reinterpret_cast<const uint32_t *>(&ll);
                                part += (hf.x + lf.x) + (hf.y + lf.y);
                            } else {
                                const uint16_t h0 = bf16_rn_bits(hv[2 * j]), h1 = bf16_rn_bits(hv[2 * j + 1]);
                                const uint16_t l0 = bf16_rn_bits(hv[2 * j] - bf16_bits_f(h0));
                                const uint16_t l1 = bf16_rn_bits(hv[2 * j + 1] - bf16_bits_f(h1));
                                hi2[j] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                                lo2[j] = (uint32_t)l0 | ((uint32_t)l1 << 16);
                                part += (bf16_bits_f(h0) + bf16_bits_f(l0)) + (bf16_bits_f(h1) + bf16_bits_f(l1));
                            }
                        }
                        // values kk..kk+3 of expert us: one slice, one register of the pair, the
                        // element pairs of lanes c0 and c0+1
                        const int i = 4 * i4, us = i / I, kk = i - us * I;
                        const int sl = kk >> 4, which = (kk >> 3) & 1, c0 = (kk & 7) >> 1;
                        uint16_t *hx = htab + (size_t)us * 256 * JN;
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int off_hi = hfrag_index(sl, c0 + q, 0, which);
                            const int off_lo = hfrag_index(sl, c0 + q, 1, which);
                            *reinterpret_cast<uint32_t *>(hx + off_hi) = hi2[q];
                            *reinterpret_cast<uint32_t *>(hx + off_lo) = lo2[q];
                        }
                    }
                    part += __shfl_xor_sync(0xffffffffu, part, 1);
                    part += __shfl_xor_sync(0xffffffffu, part, 2);
                    part += __shfl_xor_sync(0xffffffffu, part, 4);
                    if (valid && (lane & 7) == 0) hsum[i4 >> 3] = part;   // block (us, b) = us * nbi + b
                }
            }
            csync();
        }
        trace_mark(p, l, 4, clock64() - tl0);

        // ---- down: warp w takes this CTA's units w, w+NW, ... of the contiguous run
        // [dn_lo, dn_hi) ((tile, expert) order) over the whole K = I, with one accumulator per
        // group of four 32-blocks; the unit's 16 sums go to vsum[unit][row]
        float *vsum = red;   // [unit][16]
        for (int nl = warp; nl < n_dn && ok; nl += NW) {
            const int qi = nl / dn_per_slot, ui = nl - qi * dn_per_slot;
            uint32_t par;
            const int s = slot_of(n_gu + qi, par);
            long long tw0 = clock64();
            ok = mbar_wait(&ms->full[s], par, err, true);
            tw_dn += clock64() - tw0;
            if (!ok) break;
            const long long td0 = clock64();
            const int us = (dn_lo + nl) % nU;
            const uint8_t *tile = ring + (size_t)s * p.slot_bytes + (size_t)ui * p.dn.tile_bytes;
            // this lane's B values: column g holds h hi (g even) or lo (g odd) of the blocks
            // 4j + (g >> 1); one 16-byte load per k-group pair j
            const uint16_t *hq = htab + (size_t)us * 256 * JN + hfrag_index(2 * (g >> 1), c, g & 1, 0);
            // 1.0 where this lane's column is the block of MMA (h, m >> 1), else 0 (per half)
            uint32_t hmask[2][2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int mh = 0; mh < 2; ++mh)
                    hmask[hh][mh] = (2 * hh + mh == (g >> 1)) ? ONE2 : 0u;
            // k groups in pairs: the pair (2j, 2j+1) covers blocks 4j..4j+3, one per column
            // pair (2c hi, 2c+1 lo)
            const __half *sc = reinterpret_cast<const __half *>(tile + p.dn.code_bytes);
            float ag = 0.f, a8 = 0.f;
#pragma unroll
            for (int j = 0; j < 6; ++j) {   // I <= 768
                if (2 * j >= DW) break;
                float Da[4] = {0.f, 0.f, 0.f, 0.f}, Db[4] = {0.f, 0.f, 0.f, 0.f};
                const uint4 bj = *reinterpret_cast<const uint4 *>(hq + 256 * j);   // (b0, b1) of slices sp = 0, 1
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int kg = 2 * j + h;
                    if (kg < DW) {
                        uint32_t a[16];
                        if constexpr (FMT == MOE_Q2B32) {
                            q2_frag_h(*reinterpret_cast<const uint2 *>(tile + (size_t)kg * 256 + lane * 8), a);
                        } else if constexpr (FMT == MOE_Q4B32) {
                            uint4 av = *reinterpret_cast<const uint4 *>(tile + (size_t)kg * 512 + lane * 16);
                            q4_frag_h(av.x, a[0], a[1], a[2], a[3]);
                            q4_frag_h(av.y, a[4], a[5], a[6], a[7]);
                            q4_frag_h(av.z, a[8], a[9], a[10], a[11]);
                            q4_frag_h(av.w, a[12], a[13], a[14], a[15]);
                        } else {
                            const uint32_t *wp = reinterpret_cast<const uint32_t *>(tile + (size_t)kg * 384 + lane * 12);
                            q3_frag(wp[0], wp[1], wp[2], a);
                        }
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            // slice 4 kg + m belongs to block 4j + 2h + (m >> 1): live in this lane's
                            // column only when that is its block
                            const uint32_t mk = hmask[h][m >> 1];
                            const uint32_t b0 = hmul2_mask(FMT, (m & 1) ? bj.z : bj.x, mk);
                            const uint32_t b1 = hmul2_mask(FMT, (m & 1) ? bj.w : bj.y, mk);
                            if constexpr (F16OP)
                                mma16816_h(h ? Db : Da, a[4 * m], a[4 * m + 1], a[4 * m + 2], a[4 * m + 3], b0, b1);
                            else
                                mma16816(h ? Db : Da, a[4 * m], a[4 * m + 1], a[4 * m + 2], a[4 * m + 3], b0, b1);
                        }
                    }
                }
                const int blk = 4 * j + c;
                if (blk < nbi) {
                    const float hs = hsum[us * nbi + blk];
                    const float sg = __half2float(sc[g * nbi + blk]), s8 = __half2float(sc[(g + 8) * nbi + blk]);
                    if constexpr (FMT == MOE_Q2B32) {
                        // block 4j + c is the first block of its k group for even c (rows g: 1024 + q,
                        // rows g+8: 1024 + 4q), the second for odd c (1024 + 16q, 1024 + 64q)
                        const float hi = hinv[us * nbi + blk];
                        const bool second = c & 1;
                        const float mg = second ? 0.0625f : 1.f, og = second ? 66.f : 1026.f;
                        const float m8 = second ? 0.015625f : 0.25f, o8 = second ? 18.f : 258.f;
                        ag = fmaf(sg * hi, fmaf((Da[0] + Da[1]) + (Db[0] + Db[1]), mg, -og * hs), ag);
                        a8 = fmaf(s8 * hi, fmaf((Da[2] + Da[3]) + (Db[2] + Db[3]), m8, -o8 * hs), a8);
                    } else if constexpr (FMT == MOE_Q4B32) {
                        // row g: 1024 + q; row g+8: 1024 + 16 q (sums / 16); h entered as h * 2^s
                        const float hi = hinv[us * nbi + blk];
                        ag = fmaf(sg * hi, (Da[0] + Da[1]) + (Db[0] + Db[1]) - 1032.f * hs, ag);
                        a8 = fmaf(s8 * hi, fmaf((Da[2] + Da[3]) + (Db[2] + Db[3]), 0.0625f, -72.f * hs), a8);
                    } else {
                        const float o = off * hs;
                        ag = fmaf(sg, (Da[0] + Da[1]) + (Db[0] + Db[1]) - o, ag);
                        a8 = fmaf(s8, (Da[2] + Da[3]) + (Db[2] + Db[3]) - o, a8);
                    }
                }
            }
            if (nl == 0) trace_mark(p, l, 16, clock64() - td0);
            ag += __shfl_xor_sync(0xffffffffu, ag, 1);
            a8 += __shfl_xor_sync(0xffffffffu, a8, 1);
            ag += __shfl_xor_sync(0xffffffffu, ag, 2);
            a8 += __shfl_xor_sync(0xffffffffu, a8, 2);
            if (nl == 0) trace_mark(p, l, 17, clock64() - td0);
            if (c == 0) {
                vsum[nl * 16 + g] = ag;
                vsum[nl * 16 + 8 + g] = a8;
            }
        }
        trace_mark(p, l, 9, clock64() - tl0);   // thread 0's own down units done
        if (cta_failed(ok)) {
            aborted = true;
            break;
        }
        {
            uint32_t par;
            const int s_next = slot_of(n_items, par);   // next layer's first item
            ring_s0 = s_next;
            ring_p0 = par;
        }
        trace_mark(p, l, 7, clock64() - tl0);
        // per tile the fixed-order weighted sum of its units
        {
            int j_first = dn_lo / nU, j_last = (dn_hi - 1) / nU;
            int n_tiles_mine = j_last - j_first + 1;
            for (int t = tid; t < n_tiles_mine * 16; t += NT) {
                int j = j_first + (t >> 4), r = t & 15;
                int first = j * nU, last = j * nU + nU - 1;
                int n0 = max(first, dn_lo), n1 = min(last, dn_hi - 1);
                float y = 0.f;
                for (int n = n0, us = n0 - first; n <= n1; ++n, ++us)   // us = n % nU
                    y = fmaf(ms->uw[us], vsum[(n - dn_lo) * 16 + r], y);
                int part = (first >= dn_lo) ? 0 : 1;
                p.x_y[(size_t)part * d + 16 * j + r] = y;
                if (part == 0 && last < dn_hi) p.x_y[d + 16 * j + r] = 0.f;
            }
            csync();   // this CTA's output parts are stored
            if (tid == 0) xchg_arrive(p, X_Y);
        }
        trace_mark(p, l, 5, clock64() - tl0);
        trace_mark(p, l, 10, tw_gu);
        trace_mark(p, l, 12, tw_dn);
    }

    // ---- outputs of the last layer ---------------------------------------------------
    if (!aborted && cta == 0) {
        const int l = p.L - 1;
        if (tid == 0) ok = ctr_wait(ctr(p, X_Y), (unsigned)G, err);
        if (!cta_failed(ok)) {
            float4 pa[YMAX], pb[YMAX];
#pragma unroll
            for (int t = 0; t < YMAX; ++t) {
                const int i4 = tid + t * NT;
                if (i4 < d / 4) {
                    pa[t] = ld_gpu4(p.x_y + 4 * i4);
                    pb[t] = ld_gpu4(p.x_y + d + 4 * i4);
                }
            }
#pragma unroll
            for (int t = 0; t < YMAX; ++t) {
                const int i4 = tid + t * NT;
                if (i4 >= d / 4) break;
                const float4 a = pa[t], b = pb[t];
                const float ya[4] = {a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = 4 * i4 + j;
                    const float y = ya[j];
                    const uint16_t yb = bf16_rn_bits(y);
                    if (p.stack) {
                        p.resid_out[i] = rs[i] + bf16_bits_f(yb);
                        if (p.rec_on) {
                            const size_t ro = ((size_t)l * p.rec_n + p.rec_r) * d + i;
                            if (p.rec.y_bf16) p.rec.y_bf16[ro] = yb;
                            if (p.rec.y_f32) p.rec.y_f32[ro] = y;
                        }
                    } else {
                        p.y_out[i] = yb;
                        if (p.yf_out) p.yf_out[i] = y;
                    }
                }
            }
        }
    }
}

}  // namespace

bool decode_supported(const moe_ctx *ctx) {
    const moe_config &c = ctx->cfg;
    if (c.flags & MOE_FLAG_NO_DECODE_KERNEL) return false;
    // gate/up k chunks go to compute warps 0..d/256-1
    if (c.d_model > 4096 || c.d_model / 256 > NW || c.d_ff / 64 > 12) return false;
    if (c.n_experts % 4) return false;   // logits region of the exchange area stays 16-byte aligned
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
    if (red_bytes < (size_t)dn_max * 16 * 4) red_bytes = (size_t)dn_max * 16 * 4;   // down unit sums
    ds.gu_units_max = gu_max;
    ds.dn_units_max = dn_max;
    ds.off_router = take((size_t)rpc * c.d_model * 4);
    ds.off_x16 = take((size_t)c.d_model * 2);
    ds.off_xh = take((size_t)c.d_model * 2);
    ds.off_logits = take((size_t)c.n_experts * 4);
    size_t htab = (size_t)(c.top_k + c.n_shared) * 256 * ((c.d_ff + 127) / 128) * 2;   // hi + lo of h
    ds.off_htab = take(htab);
    ds.off_red = take(red_bytes);
    ds.off_misc = take(sizeof(Misc));
    ds.off_resid = take((size_t)c.d_model * 4);
    ds.off_sums = take((size_t)(c.d_model / 32 + 2 * nU * (c.d_ff / 32)) * 4);
    ds.off_ltab = take((size_t)c.n_layers * sizeof(LayerPtrs));   // a call runs at most n_layers layers
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
    const void *kfn = (c.fmt == MOE_Q4B32)   ? (const void *)k_decode<MOE_Q4B32>
                          : (c.fmt == MOE_Q2B32) ? (const void *)k_decode<MOE_Q2B32>
                                                 : (const void *)k_decode<MOE_Q3B32>;
    QE_CHECK(cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, ds.smem_bytes));
    int per_sm = 0;
    QE_CHECK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, NTT, ds.smem_bytes));
    if (per_sm < 1) ds.smem_bytes = 0;
    return MOE_OK;
}

// Exchange area: 3 counters (128 bytes apart), logits [E], h [MAXU][I], output parts [2][d].
constexpr size_t XB_LOGITS = 384;
static size_t xb_h_off(const moe_config &c) { return XB_LOGITS + (((size_t)c.n_experts * 4 + 127) & ~(size_t)127); }
static size_t xb_y_off(const moe_config &c) { return xb_h_off(c) + (size_t)MAXU * c.d_ff * 4; }
size_t decode_xchg_bytes(const moe_config &c) { return xb_y_off(c) + (size_t)2 * c.d_model * 4; }
size_t decode_xchg_counter_bytes() { return XB_LOGITS; }

int decode_trace_buffer(moe_ctx *ctx, int grid, int L, int words, cudaStream_t st, unsigned long long **out) {
    DecodeState &ds = ctx->dec;
    size_t need = (size_t)grid * L * words;
    if (need > ds.trace_cap) {
        if (ds.trace) ctx_free(ctx, ds.trace);
        ds.trace = nullptr;
        ds.trace_cap = 0;
        QE_CHECK(cudaSetDevice(ctx->device));
        QE_TRY(ctx_alloc(ctx, (void **)&ds.trace, need * 8, "trace"));
        ds.trace_cap = need;
    }
    QE_CHECK(cudaMemsetAsync(ds.trace, 0, need * 8, st));
    ds.trace_n = grid * L;
    ds.trace_words = words;
    *out = ds.trace;
    return MOE_OK;
}

int launch_decode(moe_ctx *ctx, int layer0, int L, const uint16_t *x, bool stack, float *resid_out,
                  uint16_t *y, float *yf, int32_t *ids, float *w, const moe_stack_record *rec,
                  int rec_n, int rec_r, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    DecodeState &ds = ctx->dec;
    DecodeParams p;
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
        p.rec_n = rec_n;
        p.rec_r = rec_r;
    }
    p.cnt = reinterpret_cast<unsigned *>(ds.xbuf);
    p.x_logits = reinterpret_cast<float *>(ds.xbuf + XB_LOGITS);
    p.x_h = reinterpret_cast<float *>(ds.xbuf + xb_h_off(c));
    p.x_y = reinterpret_cast<float *>(ds.xbuf + xb_y_off(c));
    p.err = ctx->ws.dev_error;
    // test hook: the context's first single-token call withholds CTA 0's logits
    p.withhold = ((c.flags & MOE_FLAG_TEST_WITHHOLD) && !ds.withheld) ? 1 : 0;
    if (p.withhold) ds.withheld = true;
    p.l2_mode = ctx->l2_mode;
    if (c.flags & MOE_FLAG_TRACE) QE_TRY(decode_trace_buffer(ctx, ds.grid, L, TRACE_WORDS, st, &p.trace));
    p.nslot = ds.nslot;
    p.slot_bytes = ds.slot_bytes;
    p.rpc = ds.rpc;
    p.off_ring = ds.off_ring;
    p.off_router = ds.off_router;
    p.off_x16 = ds.off_x16;
    p.off_xh = ds.off_xh;
    p.off_logits = ds.off_logits;
    p.off_htab = ds.off_htab;
    p.off_red = ds.off_red;
    p.off_misc = ds.off_misc;
    p.off_resid = ds.off_resid;
    p.off_sums = ds.off_sums;
    p.off_ltab = ds.off_ltab;
    void *args[] = {&p};
    const void *kfn = (c.fmt == MOE_Q4B32)   ? (const void *)k_decode<MOE_Q4B32>
                          : (c.fmt == MOE_Q2B32) ? (const void *)k_decode<MOE_Q2B32>
                                                 : (const void *)k_decode<MOE_Q3B32>;
    QE_CHECK(cudaLaunchCooperativeKernel(kfn, dim3(ds.grid), dim3(NTT), args,
                                         (size_t)ds.smem_bytes, st));
    QE_CHECK_LAUNCH("k_decode");
    return MOE_OK;
}

}  // namespace qeffn

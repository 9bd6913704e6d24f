// Few-token decode (2..8 tokens per launch; the host runs 9..16 tokens as two
// launches): one persistent kernel runs whole layers (and the whole 48-layer
// stack) for a small batch of tokens, reading
// the union of the batch's experts once per layer.  This is the step that
// checks several guessed tokens at once ("Strata: Qwen3.8-Flash-Next (125B
// Moe) on a 8GB+ Nvidia GPU", README section "How does it work": guess, then
// check all the guesses in one go; "Running Qwen3.8-Flash-Next on a 4090
// 24GB", the --spec 4 setting).  Routing and combine follow "Qwen3.8-Flash-
// Next at 45 Tokens/sec on a 12GB GPU?" (video transcript 1:50-2:16,
// 3:36-3:47); the expert network and block formats are include/moe.h's.
//
// One CTA per SM (cooperative launch), 12 compute warps and one producer warp
// that issues every bulk copy into a ring of shared-memory slots.  Per layer:
//   1. input: every CTA rebuilds all T token rows (stack: r = r_prev + bf16(y),
//      rmsnorm, bf16 x).  The residual stream lives in global memory, each CTA
//      storing the slice of columns it owns; r_prev is loaded into the idle
//      ring at the end of the previous layer, so only the layer output is read
//      after the output exchange;
//   2. router: CTA c owns experts c, c+G, ...; a warp computes whole
//      (expert, token) dot products from router rows prefetched into shared
//      memory during the previous layer; logits are exchanged (counter 0);
//   3. every CTA selects each token's top-k (a warp per token), forms the
//      sorted union U of the chosen experts (+ the shared expert) and the
//      weight table w[u][t];
//   4. gate/up: units (u, 16-row tile) round-robin over the CTAs in u-major
//      order; the tokens sit in the MMA's B columns (column t = token t), the
//      codes become exact fp16/bf16 operands (as in the single-token kernel)
//      and each 32-block's partial is flushed with its scale and the offset
//      term in fp32.  Inside a CTA the units' k-group steps are cut into 12
//      near-equal ranges, one per warp; a unit cut by a range boundary meets
//      in shared-memory sums and its last part applies SwiGLU and stores h;
//      one release per CTA publishes its h values (counter 2);
//   5. down: units (u, 16-row output tile) in u-major order, a contiguous run
//      per CTA (so a CTA touches two or three experts), round-robin over its
//      warps; once every CTA's h is published, h enters as hi + lo parts in
//      B-fragment order; each unit's weighted 16 x T output is added to the
//      layer's fp32 output buffer with vector atomics; a y counter closes the
//      layer.
// Every wait is bounded (clock64); on timeout the kernel sets the context's
// error word and every CTA leaves.  The host zeroes the counters and the
// output buffers before each launch.
#include <string.h>

#include "decode_common.cuh"

namespace qeffn {

namespace {

using namespace dec;

constexpr int TMAX = 8;         // tokens per launch: the eight B columns of mma.m16n8k16
constexpr int KMAX = 32;        // top_k limit
constexpr int EPL = 16;         // logits per lane in the top-k (E <= 512)
constexpr int CANDM = 64;       // top-k candidates per token held for ranking
constexpr int MAX_SPAN = 4;     // experts one CTA's down run may touch (checked at set-up)
constexpr int IN_IT = 2;        // float4 columns of a token row per thread in the input phase (d <= 3072)
constexpr int HB_M = 4;         // float4 loads of h in flight per thread
constexpr int GU_CH = 2;        // chunks (k-group ranges) per gate/up unit (of 1, 2, 3, 4 and 8, 2 measured fastest)

struct MiscM {
    unsigned long long full[MAX_SLOTS];
    unsigned long long empty[MAX_SLOTS];   // one arrival per consumed item
    unsigned long long rbar;
    unsigned long long route;              // one arrival per layer: routing known
    int ccnt[MAX_SLOTS];                   // items of slot s consumed so far in this launch
    int icnt[MAX_SLOTS];                   // down units of the item in slot s finished so far
    int nU;                                // experts in use this layer (routed union + shared)
    int nR;                                // routed part of the union
    int ids[TMAX][KMAX];
    float w[TMAX][KMAX];
    unsigned bits[32];                     // union bitmap over E <= 1024
    float xinv[TMAX];                      // 2^-s of a token's fp16 operand (1 for bf16 operands)
    float xscale[TMAX];                    // 2^s
    union {
        float2 cand[TMAX][CANDM];          // top-k: candidates of each token (logit, id bits)
        float pacc[MAX_SLOTS][32][4];      // gate/up: chunk sums of the unit in each ring slot
    };
    int pcnt[MAX_SLOTS];                   // gate/up: chunks of that unit finished
    float ss[NW][TMAX];                    // per-warp sums of squares / maxima of the input phase
    float mx[NW][TMAX];
    float tinv[TMAX];                      // 1 / rms of each token's residual row
    float tmax[TMAX];                      // max |x| of each token's input row
    float rbias[8];                        // router bias of this CTA's expert rows
};

struct MultiParams {
    const LayerPtrs *layers;
    int layer0, L;
    int d, E, I, k, nsh, T, TM;    // T tokens of this launch, TM the carve's token capacity
    MatLayout gu, dn;
    int stack;
    const uint16_t *x_in;          // bf16 [T][d]
    float *resid_out;              // stack: [T][d]
    uint16_t *y_out;               // single layer: bf16 [T][d]
    float *yf_out;                 // single layer: fp32 [T][d] or NULL
    int32_t *ids_out;              // single layer: [T][k] or NULL
    float *w_out;                  // single layer: [T][k] or NULL
    moe_stack_record rec;          // records: token t is record row rec_r0 + t of rec_n
    int rec_on, rec_n, rec_r0;
    unsigned *cnt;                 // [0] logits, [32] y and [64] h arrivals (one per CTA and layer each)
    unsigned long long *x_logits;  // [TM][E] tagged logits: (tag << 32) | float bits
    unsigned tag0;                 // tag of this launch's first layer (tag0 + l for layer l)
    unsigned long long *x_h;       // [UM][TM][I] tagged h (same tags as the logits)
    float *y_acc;                  // [2][TM][d] layer outputs, accumulated with atomics
    float *r_buf;                  // [2][TM][d] residual stream (stack)
    int *err;
    int withhold;
    int l2_mode;                   // 0: plain copies; 1: shared experts kept in L2, the rest streamed
    unsigned long long *trace;     // [G][L][24] phase clocks, or NULL
    int nslot, slot_bytes, rpc, span, UM;
    int off_ring, off_router, off_xb, off_xoff, off_hsum, off_uexp, off_wtab,
        off_misc, off_ltab;
};

constexpr int C_Y = 32;   // the layer-output arrival counter

// Phase trace (MOE_FLAG_TRACE): per (CTA, layer) record of 24 words: CTA, layer, then SM clock
// cycles since the layer started in this CTA:
//   0 input ready          1 logits stored        2 all logits received  3 routing known
//   4 gate/up done         5 h of the down run's experts complete       6 h table built
//   7 down done            8 output contributions released            9 warp 0: cycles waiting
//  10 warp 0: cycles waiting for down data        11 previous layer's output received
//  12 input pass 1 done (thread 0)                13 input sums of squares combined
//  14 input pass 2 done (thread 0)                15 router rows landed
//  16 operand conversion and block sums done      17 top-k: logits loaded (warp 0)
//  18 top-k: candidates ranked (warp 0)           19 all tokens' top-k done
//  20 union and weight table built
//  21 global timer (ns) at the layer start
constexpr int TRACE_WORDS_M = 24;
__device__ __noinline__ void mtrace_store(unsigned long long *trace, int L, int l, int ph, long long t) {
    unsigned long long *r = trace + ((size_t)blockIdx.x * L + l) * TRACE_WORDS_M;
    if (ph == 0) {
        r[0] = blockIdx.x;
        r[1] = l;
    }
    r[2 + ph] = (unsigned long long)t;
}

__device__ __forceinline__ float bf16f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }
__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// The 16 A-fragment registers of one lane's piece of a k group (four k16 slices).
template <int FMT>
__device__ __forceinline__ void frag16(const uint8_t *piece, uint32_t r[16]) {
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
__device__ __forceinline__ void mma_fmt(float *d, const uint32_t *a, uint32_t b0, uint32_t b1) {
    if constexpr (FMT == MOE_Q3B32) mma16816(d, a[0], a[1], a[2], a[3], b0, b1);
    else mma16816_h(d, a[0], a[1], a[2], a[3], b0, b1);
}
template <int FMT>
constexpr int piece_bytes() { return FMT == MOE_Q4B32 ? 16 : FMT == MOE_Q2B32 ? 8 : 12; }

// Flush one 32-block's MMA partial D (rows g, g+8 x columns 2c, 2c+1) into acc:
// acc += s_row * (D * mult_row - off_row * vsum_col), where the codes were read
// as 1024 + F q (fp16) or 128 + q (bf16) and vsum is the block sum of the
// column's B operand.  `second` = the k group's second block (Q2B32 only).
template <int FMT>
__device__ __forceinline__ void flush_block(float *acc, const float *D, float sg, float s8, float v0, float v1,
                                            bool second) {
    float mg, m8, og, o8;
    if constexpr (FMT == MOE_Q4B32) {
        mg = 1.f; og = 1032.f; m8 = 0.0625f; o8 = 72.f;
    } else if constexpr (FMT == MOE_Q2B32) {
        if (!second) { mg = 1.f; og = 1026.f; m8 = 0.25f; o8 = 258.f; }
        else { mg = 0.0625f; og = 66.f; m8 = 0.015625f; o8 = 18.f; }
    } else {
        mg = 1.f; og = 132.f; m8 = 1.f; o8 = 132.f;
    }
    acc[0] = fmaf(sg, fmaf(D[0], mg, -og * v0), acc[0]);
    acc[1] = fmaf(sg, fmaf(D[1], mg, -og * v1), acc[1]);
    acc[2] = fmaf(s8, fmaf(D[2], m8, -o8 * v0), acc[2]);
    acc[3] = fmaf(s8, fmaf(D[3], m8, -o8 * v1), acc[3]);
}

// Bounded wait of a warp (all lanes poll) until a shared-memory counter reaches n; false on timeout
// (error word set) or when another CTA reported an error.
__device__ __forceinline__ bool smem_count_wait(const int *c, int n, int *err) {
    long long t0 = clock64();
    for (int it = 0;; ++it) {
        if (*(volatile const int *)c >= n) return true;
        if ((it & 15) == 15) {
            if (*(volatile int *)err != 0) return false;
            if (clock64() - t0 > SPIN_LIMIT) {
                atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
}

// Position of the 16-byte B fragment of (expert-in-span su, k group kg, slice m,
// lane) in the down phase's h table: [su][kg][m][lane] x 16 bytes, so that one
// warp instruction reads 512 contiguous bytes.
__device__ __forceinline__ int hfrag_off(int su, int nkg, int kg, int m, int lane) {
    return (((su * nkg + kg) * 4 + m) * 32 + lane) * 16;
}

template <int FMT>
__global__ void __launch_bounds__(NTT, 1) k_decode_multi(MultiParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *ring = smem + p.off_ring;
    float *rtr = reinterpret_cast<float *>(smem + p.off_router);
    uint16_t *xb = reinterpret_cast<uint16_t *>(smem + p.off_xb);     // [TM][d] bf16 input; then the h table
    uint8_t *htab = smem + p.off_xb;
    float *hsum = reinterpret_cast<float *>(smem + p.off_hsum);       // [span][TM][I/32], then hinv
    float *xoff = reinterpret_cast<float *>(smem + p.off_xoff);       // [d/32][2][TM]: gate/up MMA start values
    int *uexp = reinterpret_cast<int *>(smem + p.off_uexp);           // [UM]
    float *wtab = reinterpret_cast<float *>(smem + p.off_wtab);       // [UM][TM]
    MiscM *ms = reinterpret_cast<MiscM *>(smem + p.off_misc);
    LayerPtrs *ltab = reinterpret_cast<LayerPtrs *>(smem + p.off_ltab);

    constexpr bool F16OP = (FMT != MOE_Q3B32);
    // Gate/up, and down for up to four tokens, remove the code offset inside the MMAs: a second MMA
    // per k16 slice with A = minus the offset (rows g and g + 8 of each 32-block, exact in
    // fp16/bf16) on the same B; the multipliers scale back the codes read as 1024 + F q.
    uint32_t cg0, c80, cg1, c81;
    float mg0, m80, mg1, m81;
    if constexpr (FMT == MOE_Q4B32) {
        cg0 = cg1 = 0xE408E408u; c80 = c81 = 0xE480E480u;   // -1032, -1152 (fp16)
        mg0 = mg1 = 1.f; m80 = m81 = 0.0625f;
    } else if constexpr (FMT == MOE_Q2B32) {
        cg0 = 0xE402E402u; c80 = 0xE408E408u;               // -1026, -1032
        cg1 = 0xE420E420u; c81 = 0xE480E480u;               // -1056, -1152
        mg0 = 1.f; m80 = 0.25f; mg1 = 0.0625f; m81 = 0.015625f;
    } else {
        cg0 = c80 = cg1 = c81 = 0xC304C304u;                // -132 (bf16)
        mg0 = m80 = mg1 = m81 = 1.f;
    }
    const uint32_t off0[4] = {cg0, c80, cg0, c80}, off1[4] = {cg1, c81, cg1, c81};
    // the same offsets as numbers (gate/up starts its MMAs from -offset x block sum)
    constexpr float OFF_G0 = FMT == MOE_Q4B32 ? 1032.f : FMT == MOE_Q2B32 ? 1026.f : 132.f;
    constexpr float OFF_80 = FMT == MOE_Q4B32 ? 1152.f : FMT == MOE_Q2B32 ? 1032.f : 132.f;
    constexpr float OFF_G1 = FMT == MOE_Q4B32 ? 1032.f : FMT == MOE_Q2B32 ? 1056.f : 132.f;
    constexpr float OFF_81 = FMT == MOE_Q4B32 ? 1152.f : FMT == MOE_Q2B32 ? 1152.f : 132.f;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
    const int G = gridDim.x, cta = blockIdx.x;
    const int d = p.d, E = p.E, I = p.I, k = p.k, T = p.T, TM = p.TM;
    const int nbd = d / 32, nbi = I / 32, nkgi = I / 64;
    const int ntile_gu = I / 8, ntile_dn = d / 16;
    const int dn_per_slot = p.slot_bytes / p.dn.tile_bytes;
    const int d4 = d / 4;
    const int XS = d + 8;   // row stride of the token rows in shared memory (halves): rows 16 bytes apart
                            // in bank order, so the 8 rows' B fragments load without conflicts
    const int own_lo = cta * d4 / G, own_hi = (cta + 1) * d4 / G;   // float4 columns this CTA owns
    float *hinv = hsum + p.span * TM * nbi;
    int *err = p.err;

    if (tid == 0) {
        for (int s = 0; s < p.nslot; ++s) {
            mbar_init(&ms->full[s], 1);
            mbar_init(&ms->empty[s], 1);
            ms->ccnt[s] = 0;
            ms->icnt[s] = 0;
        }
        mbar_init(&ms->rbar, 1);
        mbar_init(&ms->route, 1);
        fence_mbar_init();
    }
    for (int i = tid; i < 32; i += NTT) ms->bits[i] = 0u;
    for (int i = tid; i < MAX_SLOTS; i += NTT) ms->pcnt[i] = 0;
    for (int l = tid; l < p.L; l += NTT) ltab[l] = p.layers[p.layer0 + l];
    __syncthreads();

    // this CTA's work in a layer with nU experts in use
    struct Split {
        int n_gu, dn_lo, dn_hi, n_dn, n_dn_items, n_items;
    };
    auto split = [&](int nU) {
        Split sp;
        const int n_gu_all = nU * ntile_gu;
        sp.n_gu = (cta < n_gu_all) ? (n_gu_all - cta + G - 1) / G : 0;   // units cta, cta + G, ...
        const int n_dn_all = nU * ntile_dn;
        sp.dn_lo = cta * n_dn_all / G;   // < 2^31: n_dn_all <= UM * d / 16, checked at set-up
        sp.dn_hi = (cta + 1) * n_dn_all / G;
        sp.n_dn = sp.dn_hi - sp.dn_lo;
        sp.n_dn_items = (sp.n_dn + dn_per_slot - 1) / dn_per_slot;
        sp.n_items = sp.n_gu + sp.n_dn_items;
        return sp;
    };
    // items fill the ring cyclically from the launch's first item: the item with absolute index a
    // sits in slot a % nslot as that slot's (a / nslot)-th fill

    // ---- producer warp (lane 0) -----------------------------------------------------------
    if (warp == NW) {
        if (lane != 0) return;
        const uint64_t keep_pol = l2_policy(true), stream_pol = l2_policy(false);
        uint32_t fpar = 0;       // bit s: parity of the fills of slot s so far
        uint32_t filled = 0;     // bit s: slot s was filled at least once
        int router_fills = 0;
        auto issue_router = [&](int li) {
            const float *rw = ltab[li].rw;
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
        issue_router(0);
        int s_next = 0;
        for (int l = 0; l < p.L; ++l) {
            const LayerPtrs Lp = ltab[l];
            if (!mbar_wait(&ms->route, (uint32_t)(l & 1), err, true)) break;
            const Split sp = split(ms->nU);
            bool pok = true;
            // the compute warps fenced their generic writes to the ring before the routing arrival
            fence_proxy_async();
            for (int q = 0; q < sp.n_items && pok; ++q) {
                const int s = s_next;
                s_next = (s_next + 1 == p.nslot) ? 0 : s_next + 1;
                if ((filled >> s) & 1u) pok = mbar_wait(&ms->empty[s], ((fpar >> s) & 1u) ^ 1u, err, true);
                if (!pok) break;
                uint8_t *dst = ring + (size_t)s * p.slot_bytes;
                if (q < sp.n_gu) {
                    const int n = cta + G * q;
                    const int u = n / ntile_gu, t = n - u * ntile_gu;
                    const uint8_t *src = Lp.gu + (size_t)uexp[u] * p.gu.expert_bytes + (size_t)t * p.gu.tile_bytes;
                    mbar_expect_tx(&ms->full[s], (uint32_t)p.gu.tile_bytes);
                    weight_copy(dst, src, (uint32_t)p.gu.tile_bytes, &ms->full[s], p.l2_mode, uexp[u] >= E, keep_pol,
                                stream_pol);
                } else {
                    const int q0 = (q - sp.n_gu) * dn_per_slot;
                    const int cnt = min(dn_per_slot, sp.n_dn - q0);
                    mbar_expect_tx(&ms->full[s], (uint32_t)(cnt * p.dn.tile_bytes));
                    for (int i = 0; i < cnt; ++i) {
                        const int n = sp.dn_lo + q0 + i;
                        const int u = n / ntile_dn, j = n - u * ntile_dn;
                        const uint8_t *src = Lp.dn + (size_t)uexp[u] * p.dn.expert_bytes + (size_t)j * p.dn.tile_bytes;
                        weight_copy(dst + (size_t)i * p.dn.tile_bytes, src, (uint32_t)p.dn.tile_bytes, &ms->full[s],
                                    p.l2_mode, uexp[u] >= E, keep_pol, stream_pol);
                    }
                }
                fpar ^= 1u << s;
                filled |= 1u << s;
            }
            if (!pok) break;
            if (l + 1 < p.L) issue_router(l + 1);
        }
        // every copy has landed before the CTA's shared memory goes away
        for (int s = 0; s < p.nslot; ++s)
            if ((filled >> s) & 1u) mbar_wait(&ms->full[s], ((fpar >> s) & 1u) ^ 1u, err, false);
        if (router_fills > 0) mbar_wait(&ms->rbar, (uint32_t)((router_fills - 1) & 1), err, false);
        return;
    }

    int ring_base = 0;                  // absolute index of this layer's first item
    bool ok = true;
    bool aborted = false;

    for (int l = 0; l < p.L; ++l) {
        const LayerPtrs Lp = ltab[l];
        const int yb = l & 1;                      // output buffer of this layer
        float *yacc = p.y_acc + (size_t)yb * TM * d;
        const long long tl0 = clock64();
        auto mark = [&](int ph, long long v) {
            if (p.trace && tid == 0) mtrace_store(p.trace, p.L, l, ph, v);
        };
        if (p.trace && tid == 0) {
            unsigned long long gt;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(gt));
            mtrace_store(p.trace, p.L, l, 21, (long long)gt);
        }
        long long tw_gu = 0, tw_dn = 0;
        if (tid < p.rpc && cta + G * tid < E) ms->rbias[tid] = __ldg(Lp.rb + cta + G * tid);

        // ---- 1. layer input: xb[t] (bf16) for every token; per-token max |x| -------------------
        // The ring is idle until this layer's routing is known: it holds the token rows r [T][d] in
        // fp32 (rsm) from the end of the previous layer through both passes (the producer's proxy
        // fence orders these writes before its next fills).
        float *rsm = reinterpret_cast<float *>(ring);
        if (p.stack) {
            float ssq[TMAX], amx[TMAX];
#pragma unroll
            for (int t = 0; t < TMAX; ++t) ssq[t] = amx[t] = 0.f;
            if (l > 0) {
                if (tid == 0) ok = ctr_wait(p.cnt + C_Y, (unsigned)(G * l), err);
                if (cta_failed(ok)) {
                    aborted = true;
                    break;
                }
                mark(11, clock64() - tl0);
            }
            const float *yprev = p.y_acc + (size_t)((l + 1) & 1) * TM * d;
            float *rcur = p.r_buf + (size_t)yb * TM * d;
            // pass 1: r = r_prev + bf16(y_prev) (layer 0: r = x), with r_prev already in rsm; sums
            // of squares and max |r|; the owned columns of r are stored for the next layer.  Four
            // tokens' loads are issued before any of them is used.
#pragma unroll
            for (int t0 = 0; t0 < TMAX; t0 += 4) {
                if (t0 >= T) break;
                float4 av[4][IN_IT];
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
#pragma unroll
                    for (int it = 0; it < IN_IT; ++it) {
                        const int t = t0 + tt, i4 = tid + it * NT;
                        av[tt][it] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (t < T && i4 < d4) {
                            if (l == 0) {
                                const uint2 xv = *reinterpret_cast<const uint2 *>(p.x_in + (size_t)t * d + 4 * i4);
                                av[tt][it] = make_float4(bf16f(xv.x & 0xFFFFu), bf16f(xv.x >> 16),
                                                         bf16f(xv.y & 0xFFFFu), bf16f(xv.y >> 16));
                            } else {
                                av[tt][it] = __ldcg(reinterpret_cast<const float4 *>(yprev + (size_t)t * d + 4 * i4));
                            }
                        }
                    }
                }
#pragma unroll
                for (int tt = 0; tt < 4; ++tt) {
#pragma unroll
                    for (int it = 0; it < IN_IT; ++it) {
                        const int t = t0 + tt, i4 = tid + it * NT;
                        if (t >= T || i4 >= d4) continue;
                        const bool own = i4 >= own_lo && i4 < own_hi;
                        float4 *rp = reinterpret_cast<float4 *>(rsm + (size_t)t * d + 4 * i4);
                        float4 r = av[tt][it];
                        if (l > 0) {
                            const float4 y = r, rv = *rp;
                            const uint16_t b0 = bf16_rn_bits(y.x), b1 = bf16_rn_bits(y.y), b2 = bf16_rn_bits(y.z),
                                           b3 = bf16_rn_bits(y.w);
                            r = make_float4(rv.x + bf16_bits_f(b0), rv.y + bf16_bits_f(b1), rv.z + bf16_bits_f(b2),
                                            rv.w + bf16_bits_f(b3));
                            if (own && p.rec_on) {
                                const size_t ro = ((size_t)(l - 1) * p.rec_n + p.rec_r0 + t) * d + 4 * i4;
                                if (p.rec.y_bf16)
                                    *reinterpret_cast<uint2 *>(p.rec.y_bf16 + ro) =
                                        make_uint2((uint32_t)b0 | ((uint32_t)b1 << 16), (uint32_t)b2 | ((uint32_t)b3 << 16));
                                if (p.rec.y_f32) *reinterpret_cast<float4 *>(p.rec.y_f32 + ro) = y;
                            }
                        }
                        if (own) *reinterpret_cast<float4 *>(rcur + (size_t)t * d + 4 * i4) = r;
                        *rp = r;
                        ssq[t] = fmaf(r.x, r.x, fmaf(r.y, r.y, fmaf(r.z, r.z, fmaf(r.w, r.w, ssq[t]))));
                        amx[t] = fmaxf(amx[t], fmaxf(fmaxf(fabsf(r.x), fabsf(r.y)), fmaxf(fabsf(r.z), fabsf(r.w))));
                    }
                }
            }
            mark(12, clock64() - tl0);
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t >= T) break;
                float a = ssq[t], m = amx[t];
                for (int o = 16; o; o >>= 1) {
                    a += __shfl_xor_sync(0xffffffffu, a, o);
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                }
                if (lane == 0) {
                    ms->ss[warp][t] = a;
                    ms->mx[warp][t] = m;
                }
            }
            csync();
            // token t's statistics, once (lane 0 of warp t, the warps' sums in warp order)
            if (warp < T && lane == 0) {
                const int t = warp;
                float a = 0.f, m = 0.f;
                for (int w = 0; w < NW; ++w) {
                    a += ms->ss[w][t];
                    m = fmaxf(m, ms->mx[w][t]);
                }
                const float inv = 1.f / sqrtf(a / (float)d + 1e-6f);
                ms->tinv[t] = inv;
                ms->tmax[t] = bf16_bits_f(bf16_rn_bits(m * inv));   // = max |bf16(r * inv)|
            }
            csync();
            mark(13, clock64() - tl0);
            // pass 2: x = bf16(r * inv), r from shared memory
            for (int t = 0; t < T; ++t)
            for (int i4 = tid; i4 < d4; i4 += NT) {
                const float inv = ms->tinv[t];
                const float4 r = *reinterpret_cast<const float4 *>(rsm + (size_t)t * d + 4 * i4);
                const uint2 xv = make_uint2(
                    (uint32_t)bf16_rn_bits(r.x * inv) | ((uint32_t)bf16_rn_bits(r.y * inv) << 16),
                    (uint32_t)bf16_rn_bits(r.z * inv) | ((uint32_t)bf16_rn_bits(r.w * inv) << 16));
                *reinterpret_cast<uint2 *>(xb + (size_t)t * XS + 4 * i4) = xv;
                if (i4 >= own_lo && i4 < own_hi && p.rec_on && p.rec.x_bf16)
                    *reinterpret_cast<uint2 *>(p.rec.x_bf16 + ((size_t)l * p.rec_n + p.rec_r0 + t) * d + 4 * i4) = xv;
            }
            fence_proxy_async();   // these generic writes to the ring before the producer's next fills
            mark(14, clock64() - tl0);
        } else {
            float amx[TMAX];
#pragma unroll
            for (int t = 0; t < TMAX; ++t) amx[t] = 0.f;
            for (int i4 = tid; i4 < d4; i4 += NT) {
#pragma unroll
                for (int t = 0; t < TMAX; ++t) {
                    if (t >= T) break;
                    const uint2 xv = *reinterpret_cast<const uint2 *>(p.x_in + (size_t)t * d + 4 * i4);
                    *reinterpret_cast<uint2 *>(xb + (size_t)t * XS + 4 * i4) = xv;
                    amx[t] = fmaxf(amx[t], fmaxf(fmaxf(fabsf(bf16f(xv.x & 0xFFFFu)), fabsf(bf16f(xv.x >> 16))),
                                                 fmaxf(fabsf(bf16f(xv.y & 0xFFFFu)), fabsf(bf16f(xv.y >> 16)))));
                }
            }
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
                if (t >= T) break;
                float m = amx[t];
                for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) ms->mx[warp][t] = m;
            }
            csync();
            if (warp < T && lane == 0) {
                float m = 0.f;
                for (int w = 0; w < NW; ++w) m = fmaxf(m, ms->mx[w][warp]);
                ms->tmax[warp] = m;
            }
        }
        csync();   // xb and the token maxima complete
        // fp16 operand scale of every token: 2^s with max |x| * 2^s < 2^15 (exact for bf16 inputs)
        if (tid < T) {
            int xe;
            frexpf(ms->tmax[tid], &xe);
            const int s = min(15 - xe, 100);
            ms->xscale[tid] = F16OP ? pow2i(s) : 1.f;
            ms->xinv[tid] = F16OP ? pow2i(-s) : 1.f;
        }
        csync();   // operand scales known
        mark(0, clock64() - tl0);
        // ---- 2. router: warp w computes the (row, token) pairs w, w + NW, ... ----------------------
        {
            int nrows = 0;
            for (int j = 0; j < p.rpc; ++j)
                if (cta + G * j < E) ++nrows;
            ok = mbar_wait(&ms->rbar, (uint32_t)(l & 1), err, true);
            if (cta_failed(ok)) {
                aborted = true;
                break;
            }
            mark(15, clock64() - tl0);
            for (int pr = warp; pr < nrows * T; pr += NW) {
                const int j = pr / T, t = pr - j * T;
                const float *wr = rtr + (size_t)j * d;
                const uint16_t *xr = xb + (size_t)t * XS;
                float acc = 0.f;
                for (int i4 = lane; i4 < d4; i4 += 32) {
                    const float4 wv = *reinterpret_cast<const float4 *>(wr + 4 * i4);
                    const uint2 xv = *reinterpret_cast<const uint2 *>(xr + 4 * i4);
                    acc = fmaf(wv.x, bf16f(xv.x & 0xFFFFu), acc);
                    acc = fmaf(wv.y, bf16f(xv.x >> 16), acc);
                    acc = fmaf(wv.z, bf16f(xv.y & 0xFFFFu), acc);
                    acc = fmaf(wv.w, bf16f(xv.y >> 16), acc);
                }
                for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                if (lane == 0 && !(p.withhold && cta == 0))
                    st_tagged(p.x_logits + (size_t)t * E + cta + G * j, acc + ms->rbias[j], p.tag0 + l);
            }
        }
        csync();   // this CTA's logits are stored; the router rows and the bf16 rows are no longer read
        mark(1, clock64() - tl0);
        // the gate/up B operand in place of the bf16 rows: within each token's 64-wide k group the
        // words are reordered so that lane c's eight B registers of the group (slices 0..3, both
        // halves) are 32 contiguous bytes; fp16 code operands take fp16 of x * 2^s
        for (int i = tid; i < T * (d / 64); i += NT) {
            const int t = i / (d / 64), kg = i - t * (d / 64);
            uint4 *pv = reinterpret_cast<uint4 *>(xb + (size_t)t * XS + 64 * kg);
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 v = pv[j];
                w[4 * j] = v.x;
                w[4 * j + 1] = v.y;
                w[4 * j + 2] = v.z;
                w[4 * j + 3] = v.w;
            }
            if constexpr (F16OP) {
                const float sc = ms->xscale[t];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const __half2 h2 = __floats2half2_rn(bf16f(w[j] & 0xFFFFu) * sc, bf16f(w[j] >> 16) * sc);
                    w[j] = *reinterpret_cast<const uint32_t *>(&h2);
                }
            }
            // the offset terms of the k group's two 32-blocks: -(offset) x (block sum of the operand as
            // the MMA sees it), for the rows g and g + 8 of the A fragments; the gate/up MMAs of every
            // tile start from them (k16 slices 0-1: block 2 kg, slices 2-3: block 2 kg + 1)
            {
                float bs[2] = {0.f, 0.f};
#pragma unroll
                for (int wo = 0; wo < 32; ++wo) {
                    float v0, v1;
                    if constexpr (F16OP) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[wo]));
                        v0 = f.x;
                        v1 = f.y;
                    } else {
                        v0 = bf16f(w[wo] & 0xFFFFu);
                        v1 = bf16f(w[wo] >> 16);
                    }
                    bs[wo >> 4] += v0 + v1;   // words 0-15: slices 0-1 (block 2 kg)
                }
                const float og[2] = {OFF_G0, OFF_G1}, o8[2] = {OFF_80, OFF_81};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    xoff[((2 * kg + h) * 2 + 0) * TM + t] = -og[h] * bs[h];
                    xoff[((2 * kg + h) * 2 + 1) * TM + t] = -o8[h] * bs[h];
                }
            }
            // word 8m + 4h + c (slice m, B register h, lane column c) goes to 8c + 2m + h
            uint32_t o[32];
#pragma unroll
            for (int wo = 0; wo < 32; ++wo) o[8 * (wo & 3) + 2 * (wo >> 3) + ((wo >> 2) & 1)] = w[wo];
#pragma unroll
            for (int j = 0; j < 8; ++j) pv[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
        mark(16, clock64() - tl0);

        // ---- 3. top-k per token (warp t), union, weights --------------------------------------------
        // Threshold and rank: the k-th largest of the 32 lanes' maxima is a lower bound of the k-th
        // largest logit, so every expert of the top k is among the values at or above it; those
        // candidates are ranked by counting the candidates ordered before each (larger logit, equal
        // logits: lower id).  Too many candidates (flat or equal logits): k rounds of warp arg-max.
        // The logits arrive tagged: a warp reads its token's row and re-reads (bounded) the words whose
        // tag is not yet this layer's; a CTA's top-k warps have then seen every CTA's router output,
        // i.e. every CTA is past its input phase.
        if (warp < T) {
            const int t = warp;
            float v[EPL];
            float lmax = -INFINITY;
            unsigned long long wv[EPL];
            const unsigned want = p.tag0 + l;
            const unsigned long long *row = p.x_logits + (size_t)t * E;
#pragma unroll
            for (int i = 0; i < EPL; ++i) wv[i] = (lane + 32 * i < E) ? ld_tagged(row + lane + 32 * i) : 0ull;
            bool got = true;
            {
                // words not yet tagged for this layer are read again together, round after round
                const long long tw = clock64();
                for (int it = 0;; ++it) {
                    unsigned late = 0u;
#pragma unroll
                    for (int i = 0; i < EPL; ++i)
                        if (lane + 32 * i < E && (unsigned)(wv[i] >> 32) != want) late |= 1u << i;
                    if (!late) break;
                    if ((it & 15) == 15 && (*(volatile int *)err != 0 || clock64() - tw > SPIN_LIMIT)) {
                        atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
                        got = false;
                        break;
                    }
#pragma unroll
                    for (int i = 0; i < EPL; ++i)
                        if ((late >> i) & 1u) wv[i] = ld_tagged(row + lane + 32 * i);
                }
            }
            if (!got) ok = false;
            mark(2, clock64() - tl0);
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = lane + 32 * i;
                float x = (e < E) ? __uint_as_float((unsigned)wv[i]) : __int_as_float(0x7fc00000);
                if (e < E && isnan(x)) x = -INFINITY;   // a NaN logit ranks as -inf (last, by id)
                v[i] = x;                               // past E: NaN, never a candidate
                if (e < E) lmax = fmaxf(lmax, x);
            }
            mark(17, clock64() - tl0);
            int rk = 0;
            for (int j = 0; j < 32; ++j) {
                const float mj = __shfl_sync(0xffffffffu, lmax, j);
                rk += (mj > lmax) || (mj == lmax && j < lane);
            }
            const unsigned hit = __ballot_sync(0xffffffffu, rk == k - 1);
            const float tau = __shfl_sync(0xffffffffu, lmax, __ffs(hit) - 1);
            int mine = 0;
#pragma unroll
            for (int i = 0; i < EPL; ++i) mine += (32 * i < E) && (v[i] >= tau);
            int incl = mine;
            for (int o = 1; o < 32; o <<= 1) {
                const int nb = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += nb;
            }
            const int ncand = __shfl_sync(0xffffffffu, incl, 31);
            float2 *cand = ms->cand[t];
            int pv_id = -1;
            float pv = -INFINITY;
            if (ncand <= CANDM) {
                int pos = incl - mine;
#pragma unroll
                for (int i = 0; i < EPL; ++i)
                    if ((32 * i < E) && v[i] >= tau) cand[pos++] = make_float2(v[i], __int_as_float(lane + 32 * i));
                // padded to a multiple of 4 with entries ordered after every candidate
                const int npad = (ncand + 3) & ~3;
                if (lane < npad - ncand) cand[ncand + lane] = make_float2(-INFINITY, __int_as_float(0x7fffffff));
                __syncwarp();
                for (int ci = lane; ci < ncand; ci += 32) {
                    const float2 me = cand[ci];
                    const int id = __float_as_int(me.y);
                    int r = 0;
                    for (int j = 0; j < npad; j += 4) {
                        const float2 o0 = cand[j], o1 = cand[j + 1], o2 = cand[j + 2], o3 = cand[j + 3];
                        r += better(o0.x, __float_as_int(o0.y), me.x, id) + better(o1.x, __float_as_int(o1.y), me.x, id) +
                             better(o2.x, __float_as_int(o2.y), me.x, id) + better(o3.x, __float_as_int(o3.y), me.x, id);
                    }
                    if (r < k) {
                        ms->ids[t][r] = id;
                        ms->w[t][r] = me.x;   // the logit for now; the weight below
                    }
                }
                __syncwarp();
                if (lane < k) {
                    pv_id = ms->ids[t][lane];
                    pv = ms->w[t][lane];
                }
            } else {
                for (int j = 0; j < k; ++j) {
                    float bv = -INFINITY;
                    int bid = 0x7fffffff;
#pragma unroll
                    for (int i = 0; i < EPL; ++i) {
                        const int e = lane + 32 * i;
                        if (32 * i < E && better(v[i], e, bv, bid)) {
                            bv = v[i];
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
                    if (bid >= E) bid = 0;   // unreachable while k <= E
                    if ((bid & 31) == lane) {
#pragma unroll
                        for (int i = 0; i < EPL; ++i)
                            if (lane + 32 * i == bid) v[i] = __int_as_float(0x7fc00000);   // taken
                    }
                    if (lane == j) {
                        pv_id = bid;
                        pv = bv;
                    }
                }
            }
            mark(18, clock64() - tl0);
            // softmax over the chosen logits, in rank order
            const float top = __shfl_sync(0xffffffffu, pv, 0);
            const float pe = lane < k ? expf(pv - top) : 0.f;
            float z = pe;
            for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            __syncwarp();
            if (lane < k) {
                const float wt = pe / z;
                ms->ids[t][lane] = pv_id;
                ms->w[t][lane] = wt;
                atomicOr(&ms->bits[pv_id >> 5], 1u << (pv_id & 31));
                if (cta == 0) {   // routing outputs
                    if (p.stack && p.rec_on) {
                        const size_t ro = ((size_t)l * p.rec_n + p.rec_r0 + t) * k + lane;
                        if (p.rec.ids) p.rec.ids[ro] = pv_id;
                        if (p.rec.w) p.rec.w[ro] = wt;
                    }
                    if (!p.stack) {
                        if (p.ids_out) p.ids_out[(size_t)t * k + lane] = pv_id;
                        if (p.w_out) p.w_out[(size_t)t * k + lane] = wt;
                    }
                }
            }
        }
        if (cta_failed(ok)) {   // the union bitmap is complete (or a token's logits never came)
            aborted = true;
            break;
        }
        mark(19, clock64() - tl0);
        // every CTA has read the previous layer's output: clear the owned columns of its buffer,
        // which accumulates the next layer's output
        if (l >= 1 && l + 1 < p.L) {
            float *ynext = p.y_acc + (size_t)((l + 1) & 1) * TM * d;
            for (int i = tid; i < T * (own_hi - own_lo); i += NT) {
                const int t = i / (own_hi - own_lo), i4 = own_lo + i - t * (own_hi - own_lo);
                *reinterpret_cast<float4 *>(ynext + (size_t)t * d + 4 * i4) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        // Union in ascending expert order, then the shared experts: an expert's union slot is the
        // number of bitmap ones below it.  Warp t < T writes column t of the weight table; the last
        // warp lists the union; the others clear the gate/up chunk sums (they share memory with the
        // top-k candidates).
        {
            const int nwords = (E + 31) / 32;
            if (warp < T || warp == NW - 1) {
                const unsigned word = lane < nwords ? ms->bits[lane] : 0u;
                int pre = __popc(word);
                for (int o = 1; o < 32; o <<= 1) {
                    const int n = __shfl_up_sync(0xffffffffu, pre, o);
                    if (lane >= o) pre += n;
                }
                const int total = __shfl_sync(0xffffffffu, pre, 31);
                pre -= __popc(word);   // exclusive
                const int nU = total + p.nsh;
                if (warp < T) {
                    const int t = warp;
                    for (int u = lane; u < nU; u += 32) wtab[u * TM + t] = 0.f;
                    int e = 0;
                    if (lane < k) e = ms->ids[t][lane];
                    const int wi = e >> 5;
                    const int below = __shfl_sync(0xffffffffu, pre, wi);
                    const unsigned wbits = __shfl_sync(0xffffffffu, word, wi);
                    __syncwarp();
                    if (lane < k) wtab[(below + __popc(wbits & ((1u << (e & 31)) - 1u))) * TM + t] = ms->w[t][lane];
                    if (lane < p.nsh) wtab[(total + lane) * TM + t] = 1.f;
                } else {
                    unsigned wv = word;
                    int pos = pre;
                    while (wv) {
                        const int b = __ffs(wv) - 1;
                        wv &= wv - 1;
                        uexp[pos++] = 32 * lane + b;
                    }
                    if (lane < p.nsh) uexp[total + lane] = E + lane;
                    if (lane == 0) {
                        ms->nU = nU;
                        ms->nR = total;
                    }
                }
            } else {
                float *pz = &ms->pacc[0][0][0];
                for (int i = tid - 32 * T; i < MAX_SLOTS * 32 * 4; i += 32 * (NW - 1 - T)) pz[i] = 0.f;
            }
        }
        mark(20, clock64() - tl0);
        csync();
        // every warp has read the bitmap: clear it for the next layer
        if (warp == NW - 1 && lane < (E + 31) / 32) ms->bits[lane] = 0u;
        if (tid == 0) mbar_arrive(&ms->route);   // the producer may issue this layer's copies
        mark(3, clock64() - tl0);
        const int nU = ms->nU;
        const Split sp = split(nU);
        auto slot_of = [&](int q, uint32_t &par, int &fill) {
            const int a = ring_base + q;
            fill = a / p.nslot;
            par = (uint32_t)(fill & 1);
            return a - fill * p.nslot;
        };

        // ---- 4. gate/up: units cut into GU_CH chunks of k groups, round-robin over the warps ------
        // Chunk c of the CTA's chunk sequence goes to warp c % NW, so each unit is worked by several
        // warps as soon as its tile lands.  A unit's chunk sums meet in shared memory (indexed by
        // its ring slot) and its last chunk to finish applies SwiGLU, clears the sums and frees the
        // slot.  Before waiting on a unit's fill, a warp waits until every earlier item of the slot
        // is consumed (a later unit can reach a slot that still holds an older item).  B operand:
        // column g = token g (zero past T), from the token rows.
        {
            const bool live = g < T;
            const uint16_t *xr = xb + (size_t)(live ? g : 0) * XS + 16 * c;
            const int t0 = 2 * c, t1 = 2 * c + 1;
            const bool l0 = t0 < T, l1 = t1 < T;
            const int cx = 2 * c < TM ? 2 * c : 0;   // start values of columns 2c, 2c + 1 (past TM: dead)
            const int nkg = d / 64;
            for (int ch = warp; ch < sp.n_gu * GU_CH && ok; ch += NW) {
                const int q = ch / GU_CH, j = ch - q * GU_CH;
                const int kb = j * nkg / GU_CH, ke = (j + 1) * nkg / GU_CH;
                uint32_t par;
                int fill;
                const int s = slot_of(q, par, fill);
                const long long tw0 = clock64();
                ok = smem_count_wait(&ms->ccnt[s], fill, err);
                if (ok) ok = mbar_wait(&ms->full[s], par, err, true);
                tw_gu += clock64() - tw0;
                if (!ok) break;
                const uint8_t *tile = ring + (size_t)s * p.slot_bytes;
                const __half *sc = reinterpret_cast<const __half *>(tile + p.gu.code_bytes);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
                for (int kg = kb; kg < ke; ++kg) {
                    uint32_t a[16];
                    frag16<FMT>(tile + (size_t)kg * p.gu.kg_bytes + lane * piece_bytes<FMT>(), a);
                    const uint4 q0 = live ? *reinterpret_cast<const uint4 *>(xr + 64 * kg) : make_uint4(0u, 0u, 0u, 0u);
                    const uint4 q1 = live ? *reinterpret_cast<const uint4 *>(xr + 64 * kg + 8) : make_uint4(0u, 0u, 0u, 0u);
                    const int bl = 2 * kg;
                    // the MMAs start from the blocks' offset terms (columns 2c, 2c + 1; rows g, g + 8)
                    const float2 oga = *reinterpret_cast<const float2 *>(xoff + (bl * 2 + 0) * TM + cx);
                    const float2 o8a = *reinterpret_cast<const float2 *>(xoff + (bl * 2 + 1) * TM + cx);
                    const float2 ogb = *reinterpret_cast<const float2 *>(xoff + (bl * 2 + 2) * TM + cx);
                    const float2 o8b = *reinterpret_cast<const float2 *>(xoff + (bl * 2 + 3) * TM + cx);
                    float Da[4] = {oga.x, oga.y, o8a.x, o8a.y}, Db[4] = {ogb.x, ogb.y, o8b.x, o8b.y};
                    mma_fmt<FMT>(Da, a + 0, q0.x, q0.y);
                    mma_fmt<FMT>(Da, a + 4, q0.z, q0.w);
                    mma_fmt<FMT>(Db, a + 8, q1.x, q1.y);
                    mma_fmt<FMT>(Db, a + 12, q1.z, q1.w);
                    const float2 sg = __half22float2(*reinterpret_cast<const __half2 *>(sc + g * nbd + bl));
                    const float2 s8 = __half22float2(*reinterpret_cast<const __half2 *>(sc + (g + 8) * nbd + bl));
                    const float sga = sg.x * mg0, s8a = s8.x * m80, sgb = sg.y * mg1, s8b = s8.y * m81;
                    acc[0] = fmaf(sga, Da[0], acc[0]);
                    acc[1] = fmaf(sga, Da[1], acc[1]);
                    acc[2] = fmaf(s8a, Da[2], acc[2]);
                    acc[3] = fmaf(s8a, Da[3], acc[3]);
                    acc[0] = fmaf(sgb, Db[0], acc[0]);
                    acc[1] = fmaf(sgb, Db[1], acc[1]);
                    acc[2] = fmaf(s8b, Db[2], acc[2]);
                    acc[3] = fmaf(s8b, Db[3], acc[3]);
                }
                // this chunk's sums into the unit's; the last chunk takes them
                float *pa = ms->pacc[s][lane];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) atomicAdd(pa + jj, acc[jj]);
                __syncwarp();
                int before = 0;
                if (lane == 0) {
                    __threadfence_block();
                    before = atomicAdd(&ms->pcnt[s], 1);
                }
                before = __shfl_sync(0xffffffffu, before, 0);
                if (before == GU_CH - 1) {
                    __threadfence_block();
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        acc[jj] = *(volatile float *)(pa + jj);
                        pa[jj] = 0.f;   // ready for the slot's next unit
                    }
                    // rows g (gate) and g + 8 (up) of the unit for tokens 2c, 2c + 1: SwiGLU in place
                    const int n = cta + G * q;
                    const int u = n / ntile_gu, t8 = n - u * ntile_gu;
                    if (l0) {
                        const float xi = ms->xinv[t0];
                        st_tagged(p.x_h + ((size_t)u * TM + t0) * I + 8 * t8 + g, silu(acc[0] * xi) * (acc[2] * xi),
                                  p.tag0 + l);
                    }
                    if (l1) {
                        const float xi = ms->xinv[t1];
                        st_tagged(p.x_h + ((size_t)u * TM + t1) * I + 8 * t8 + g, silu(acc[1] * xi) * (acc[3] * xi),
                                  p.tag0 + l);
                    }
                    __syncwarp();
                    if (lane == 0) {
                        ms->pcnt[s] = 0;
                        __threadfence_block();
                        atomicAdd(&ms->ccnt[s], 1);
                        mbar_arrive(&ms->empty[s]);      // the slot may be refilled
                    }
                }
            }
        }
        if (cta_failed(ok)) {
            aborted = true;
            break;
        }
        mark(4, clock64() - tl0);

        // ---- 5. down ---------------------------------------------------------------------------------
        const int u_first = sp.n_dn > 0 ? sp.dn_lo / ntile_dn : 0;
        const int n_span = sp.n_dn > 0 ? (sp.dn_hi - 1) / ntile_dn - u_first + 1 : 0;
        if (n_span > 0) {
            mark(5, clock64() - tl0);
            // h of the run's experts -> hi + lo B fragments (columns of the T tokens; the rest is
            // masked where it is read) and, per (expert, token, 32-block), the sum of hi + lo and
            // (fp16) the block's 2^-s
            const int nq = n_span * T * (I / 4);   // 4 values per thread and step; 8 lanes per block
            // h arrives tagged: the words of a batch are read together, and those not yet tagged for
            // this layer are read again together, round after round (bounded)
            const unsigned want = p.tag0 + l;
            for (int i0 = 0; i0 < nq; i0 += HB_M * NT) {   // every lane runs every batch (shuffles below)
              ulonglong2 hw[HB_M][2];
              const unsigned long long *hp[HB_M];
#pragma unroll
              for (int bq = 0; bq < HB_M; ++bq) {
                const int i = i0 + bq * NT + tid;
                hp[bq] = nullptr;
                hw[bq][0] = hw[bq][1] = make_ulonglong2((unsigned long long)want << 32, (unsigned long long)want << 32);
                if (i < nq) {
                    const int su = i / (T * (I / 4));
                    const int rem = i - su * (T * (I / 4));
                    const int t = rem / (I / 4), k4 = rem - t * (I / 4);
                    hp[bq] = p.x_h + ((size_t)(u_first + su) * TM + t) * I + 4 * k4;
                    hw[bq][0] = ld_tagged2(hp[bq]);
                    hw[bq][1] = ld_tagged2(hp[bq] + 2);
                }
              }
              {
                const long long tw = clock64();
                for (int it = 0;; ++it) {
                  unsigned late = 0u;
#pragma unroll
                  for (int bq = 0; bq < HB_M; ++bq)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                      if ((unsigned)(hw[bq][hh].x >> 32) != want || (unsigned)(hw[bq][hh].y >> 32) != want)
                        late |= 1u << (2 * bq + hh);
                  if (!late) break;
                  if ((it & 15) == 15 && (*(volatile int *)err != 0 || clock64() - tw > SPIN_LIMIT)) {
                    atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
                    ok = false;
                    break;
                  }
#pragma unroll
                  for (int bq = 0; bq < HB_M; ++bq)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                      if ((late >> (2 * bq + hh)) & 1u) hw[bq][hh] = ld_tagged2(hp[bq] + 2 * hh);
                }
              }
              float4 hb[HB_M];
#pragma unroll
              for (int bq = 0; bq < HB_M; ++bq)
                hb[bq] = make_float4(__uint_as_float((unsigned)hw[bq][0].x), __uint_as_float((unsigned)hw[bq][0].y),
                                     __uint_as_float((unsigned)hw[bq][1].x), __uint_as_float((unsigned)hw[bq][1].y));
#pragma unroll
              for (int bq = 0; bq < HB_M; ++bq) {
                const int i = i0 + bq * NT + tid;
                if (i >= nq) break;   // uniform across the warp (nq is a multiple of 32)
                const int su = i / (T * (I / 4));
                const int rem = i - su * (T * (I / 4));
                const int t = rem / (I / 4), k4 = rem - t * (I / 4);
                const float4 hv = hb[bq];
                const float h4[4] = {hv.x, hv.y, hv.z, hv.w};
                float scale = 1.f;
                if constexpr (F16OP) {
                    float mx = fmaxf(fmaxf(fabsf(h4[0]), fabsf(h4[1])), fmaxf(fabsf(h4[2]), fabsf(h4[3])));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    int he;
                    frexpf(mx, &he);
                    const int sh = min(15 - he, 100);
                    scale = pow2i(sh);
                    if ((lane & 7) == 0) hinv[(su * TM + t) * nbi + (k4 >> 3)] = pow2i(-sh);
                }
                uint32_t hi2[2], lo2[2];
                float part = 0.f;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    if constexpr (F16OP) {
                        const float v0 = h4[2 * j] * scale, v1 = h4[2 * j + 1] * scale;
                        const __half2 hh = __floats2half2_rn(v0, v1);
                        const float2 hf = __half22float2(hh);
                        const __half2 ll = __floats2half2_rn(v0 - hf.x, v1 - hf.y);
                        const float2 lf = __half22float2(ll);
                        hi2[j] = *reinterpret_cast<const uint32_t *>(&hh);
                        lo2[j] = *reinterpret_cast<const uint32_t *>(&ll);
                        part += (hf.x + lf.x) + (hf.y + lf.y);
                    } else {
                        const uint16_t h0 = bf16_rn_bits(h4[2 * j]), h1 = bf16_rn_bits(h4[2 * j + 1]);
                        const uint16_t l0 = bf16_rn_bits(h4[2 * j] - bf16_bits_f(h0));
                        const uint16_t l1 = bf16_rn_bits(h4[2 * j + 1] - bf16_bits_f(h1));
                        hi2[j] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                        lo2[j] = (uint32_t)l0 | ((uint32_t)l1 << 16);
                        part += (bf16_bits_f(h0) + bf16_bits_f(l0)) + (bf16_bits_f(h1) + bf16_bits_f(l1));
                    }
                }
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                if ((lane & 7) == 0) hsum[(su * TM + t) * nbi + (k4 >> 3)] = part;
                // values k = 4 k4 .. 4 k4 + 3 of token t: slice sl, register b0 (kk < 8) or b1, the
                // lanes (t, c0) and (t, c0 + 1)
                const int kk = 4 * k4;
                const int sl = kk >> 4, w16 = kk & 15, which = w16 >> 3, c0 = (w16 & 7) >> 1;
                const int kg = sl >> 2, m = sl & 3;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t *dst = reinterpret_cast<uint32_t *>(htab + hfrag_off(su, nkgi, kg, m, 4 * t + c0 + q));
                    dst[which] = hi2[q];
                    dst[2 + which] = lo2[q];
                }
              }
            }
        }
        if (cta_failed(ok)) {   // the h table is complete (or some h never came)
            aborted = true;
            break;
        }
        mark(6, clock64() - tl0);
        // units of this CTA's run, in batches of dn_per_slot (one ring item each); units go round-robin
        // to the warps, and the warp that finishes an item's last unit releases its slot
        for (int ui_all = warp; ui_all < sp.n_dn && ok; ui_all += NW) {
            const int it = ui_all / dn_per_slot, ui = ui_all - it * dn_per_slot;
            const int cnt = min(dn_per_slot, sp.n_dn - it * dn_per_slot);
            // this warp may reach an item while its slot still holds an older one (consumed by other
            // warps): first wait until every earlier item of the slot is consumed, then the fill
            // parity names this item's fill unambiguously
            uint32_t par;
            int fill;
            const int s = slot_of(sp.n_gu + it, par, fill);
            const long long tw0 = clock64();
            ok = smem_count_wait(&ms->ccnt[s], fill, err);
            if (ok) ok = mbar_wait(&ms->full[s], par, err, true);
            tw_dn += clock64() - tw0;
            if (!ok) break;
            {
                const int n = sp.dn_lo + ui_all;
                const int u = n / ntile_dn, j = n - u * ntile_dn;
                const int su = u - u_first;
                const uint8_t *tile = ring + (size_t)s * p.slot_bytes + (size_t)ui * p.dn.tile_bytes;
                const __half *sc = reinterpret_cast<const __half *>(tile + p.dn.code_bytes);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const int t0 = 2 * c, t1 = 2 * c + 1;
                const bool l0 = t0 < T, l1 = t1 < T;
                if (T <= 4) {
                    // Up to four tokens: hi and lo of h share one MMA, column g < 4 holding the hi part
                    // of token g and column g >= 4 the lo part of token g - 4, and the code offset is
                    // removed by a second MMA with the constant A (as in gate/up); the two parts of a
                    // token meet at the end (lanes c and c ^ 2).
                    const int srcl = lane & 15;                  // h table lane of this column's token
                    const int poff = 8 * (g >> 2);               // bytes: hi (words 0-1) or lo (2-3)
                    const bool colv = (g & 3) < T;
                    const int tc0 = (2 * c) & 3, tc1 = (2 * c + 1) & 3;   // tokens of this lane's columns
                    const float *ih0 = hinv + (su * TM + min(tc0, TM - 1)) * nbi;
                    const float *ih1 = hinv + (su * TM + min(tc1, TM - 1)) * nbi;
#pragma unroll 2
                    for (int kg = 0; kg < nkgi; ++kg) {
                        uint32_t a[16];
                        frag16<FMT>(tile + (size_t)kg * p.dn.kg_bytes + lane * piece_bytes<FMT>(), a);
                        float Da[4] = {0.f, 0.f, 0.f, 0.f}, Db[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const uint2 bq = colv ? *reinterpret_cast<const uint2 *>(htab + hfrag_off(su, nkgi, kg, m, srcl) + poff)
                                                  : make_uint2(0u, 0u);
                            float *D = (m < 2) ? Da : Db;
                            mma_fmt<FMT>(D, a + 4 * m, bq.x, bq.y);
                            mma_fmt<FMT>(D, m < 2 ? off0 : off1, bq.x, bq.y);
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int b = 2 * kg + h;
                            float sg = __half2float(sc[g * nbi + b]) * (h ? mg1 : mg0);
                            float s8 = __half2float(sc[(g + 8) * nbi + b]) * (h ? m81 : m80);
                            float sg0 = sg, sg1 = sg, s80 = s8, s81 = s8;
                            if constexpr (F16OP) {   // h entered as h * 2^s per (token, block)
                                const float i0 = ih0[b], i1 = ih1[b];
                                sg0 *= i0; s80 *= i0; sg1 *= i1; s81 *= i1;
                            }
                            const float *D = h ? Db : Da;
                            acc[0] = fmaf(sg0, D[0], acc[0]);
                            acc[1] = fmaf(sg1, D[1], acc[1]);
                            acc[2] = fmaf(s80, D[2], acc[2]);
                            acc[3] = fmaf(s81, D[3], acc[3]);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 2);
                } else {
                    const float *hs0 = hsum + (su * TM + min(t0, TM - 1)) * nbi;
                    const float *hs1 = hsum + (su * TM + min(t1, TM - 1)) * nbi;
                    const float *hi0 = hinv + (su * TM + min(t0, TM - 1)) * nbi;
                    const float *hi1 = hinv + (su * TM + min(t1, TM - 1)) * nbi;
    #pragma unroll 2
                    for (int kg = 0; kg < nkgi; ++kg) {
                        uint32_t a[16];
                        frag16<FMT>(tile + (size_t)kg * p.dn.kg_bytes + lane * piece_bytes<FMT>(), a);
                        float Da[4] = {0.f, 0.f, 0.f, 0.f}, Db[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const uint4 bq = g < T ? *reinterpret_cast<const uint4 *>(htab + hfrag_off(su, nkgi, kg, m, lane))
                                                   : make_uint4(0u, 0u, 0u, 0u);
                            float *D = (m < 2) ? Da : Db;
                            mma_fmt<FMT>(D, a + 4 * m, bq.x, bq.y);   // hi
                            mma_fmt<FMT>(D, a + 4 * m, bq.z, bq.w);   // lo
                        }
    #pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int b = 2 * kg + h;
                            const float v0 = l0 ? hs0[b] : 0.f, v1 = l1 ? hs1[b] : 0.f;
                            float sg = __half2float(sc[g * nbi + b]), s8 = __half2float(sc[(g + 8) * nbi + b]);
                            float Dv[4] = {h ? Db[0] : Da[0], h ? Db[1] : Da[1], h ? Db[2] : Da[2], h ? Db[3] : Da[3]};
                            if constexpr (F16OP) {
                                // h entered as h * 2^s per (token, block): scale back per column
                                const float i0 = l0 ? hi0[b] : 0.f, i1 = l1 ? hi1[b] : 0.f;
                                float tmp[4] = {0.f, 0.f, 0.f, 0.f};
                                flush_block<FMT>(tmp, Dv, sg, s8, v0, v1, h == 1);
                                acc[0] = fmaf(tmp[0], i0, acc[0]);
                                acc[1] = fmaf(tmp[1], i1, acc[1]);
                                acc[2] = fmaf(tmp[2], i0, acc[2]);
                                acc[3] = fmaf(tmp[3], i1, acc[3]);
                            } else {
                                flush_block<FMT>(acc, Dv, sg, s8, v0, v1, h == 1);
                            }
                        }
                    }
                }
                // weighted by each token's routing weight for this expert, then 4 consecutive rows of
                // one token per lane (a 4 x 4 transpose among the lanes g = 4m' .. 4m' + 3 of a column
                // pair) for one vector atomic each
                const float w0 = l0 ? wtab[u * TM + t0] : 0.f, w1 = l1 ? wtab[u * TM + t1] : 0.f;
                const float val[4] = {acc[0] * w0, acc[1] * w1, acc[2] * w0, acc[3] * w1};
                const int gi = g & 3, gbase = lane - 4 * gi;   // lane of (g - gi, c)
                float vec[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int sidx = (gi + r) & 3, didx = (gi - r) & 3;
                    const float send = sidx == 0 ? val[0] : sidx == 1 ? val[1] : sidx == 2 ? val[2] : val[3];
                    const float got = __shfl_sync(0xffffffffu, send, gbase + 4 * didx);
#pragma unroll
                    for (int q = 0; q < 4; ++q) vec[q] = (q == didx) ? got : vec[q];
                }
                // lane (g, c) now holds rows 4 (g >> 2) + 8 (gi >> 1) + 0..3 of token 2c + (gi & 1)
                const int tok = 2 * c + (gi & 1);
                const int row0 = 16 * j + 4 * (g >> 2) + 8 * (gi >> 1);
                if (tok < T && wtab[u * TM + tok] != 0.f)
                    red_add_v4(yacc + (size_t)tok * d + row0, vec[0], vec[1], vec[2], vec[3]);
            }
            __syncwarp();
            if (lane == 0) {
                // the last unit of the item frees its slot
                if (atomicAdd(&ms->icnt[s], 1) == cnt - 1) {
                    ms->icnt[s] = 0;
                    atomicAdd(&ms->ccnt[s], 1);
                    mbar_arrive(&ms->empty[s]);
                }
            }
        }
        ring_base += sp.n_items;
        // (the output atomics are ordered before the arrival below by this barrier and the
        // arriving thread's release, which is cumulative)
        if (cta_failed(ok)) {
            aborted = true;
            break;
        }
        mark(7, clock64() - tl0);
        if (tid == 0) ctr_arrive(p.cnt + C_Y);
        // the next layer's r_prev (this layer's r, complete since the logits exchange) into the
        // idle ring: its load overlaps the wait for the other CTAs' outputs
        if (p.stack && l + 1 < p.L) {
            const float *rl = p.r_buf + (size_t)yb * TM * d;
            for (int i = tid; i < T * d4; i += NT) {
                const int t = i / d4, i4 = i - t * d4;
                *reinterpret_cast<float4 *>(rsm + (size_t)t * d + 4 * i4) =
                    __ldcg(reinterpret_cast<const float4 *>(rl + (size_t)t * d + 4 * i4));
            }
        }
        mark(8, clock64() - tl0);
        mark(9, tw_gu);
        mark(10, tw_dn);
    }

    // ---- outputs of the last layer: each CTA its owned columns -------------------------------------
    if (!aborted) {
        if (tid == 0) ok = ctr_wait(p.cnt + C_Y, (unsigned)(G * p.L), err);
        if (!cta_failed(ok)) {
            const int lb = (p.L - 1) & 1;
            const float *yl = p.y_acc + (size_t)lb * TM * d;
            const float *rl = p.r_buf + (size_t)lb * TM * d;
            for (int i = tid; i < T * (own_hi - own_lo); i += NT) {
                const int t = i / (own_hi - own_lo), i4 = own_lo + i - t * (own_hi - own_lo);
                const float4 y = __ldcg(reinterpret_cast<const float4 *>(yl + (size_t)t * d + 4 * i4));
                const uint16_t b0 = bf16_rn_bits(y.x), b1 = bf16_rn_bits(y.y), b2 = bf16_rn_bits(y.z),
                               b3 = bf16_rn_bits(y.w);
                const uint2 yb2 = make_uint2((uint32_t)b0 | ((uint32_t)b1 << 16), (uint32_t)b2 | ((uint32_t)b3 << 16));
                if (p.stack) {
                    const float4 r = __ldcg(reinterpret_cast<const float4 *>(rl + (size_t)t * d + 4 * i4));
                    *reinterpret_cast<float4 *>(p.resid_out + (size_t)t * d + 4 * i4) =
                        make_float4(r.x + bf16_bits_f(b0), r.y + bf16_bits_f(b1), r.z + bf16_bits_f(b2),
                                    r.w + bf16_bits_f(b3));
                    if (p.rec_on) {
                        const size_t ro = ((size_t)(p.L - 1) * p.rec_n + p.rec_r0 + t) * d + 4 * i4;
                        if (p.rec.y_bf16) *reinterpret_cast<uint2 *>(p.rec.y_bf16 + ro) = yb2;
                        if (p.rec.y_f32) *reinterpret_cast<float4 *>(p.rec.y_f32 + ro) = y;
                    }
                } else {
                    *reinterpret_cast<uint2 *>(p.y_out + (size_t)t * d + 4 * i4) = yb2;
                    if (p.yf_out) *reinterpret_cast<float4 *>(p.yf_out + (size_t)t * d + 4 * i4) = y;
                }
            }
        }
    }
}

}  // namespace

// ---- host side -----------------------------------------------------------------------------------

static int multi_tm(const moe_config &c) { return c.max_tokens < TMAX ? c.max_tokens : TMAX; }
static int multi_um(const moe_config &c) { return multi_tm(c) * c.top_k + c.n_shared; }

size_t decode_multi_counter_bytes(const moe_config &) { return 512; }
static size_t xm_logits_off(const moe_config &c) { return decode_multi_counter_bytes(c); }
static size_t xm_h_off(const moe_config &c) {
    return xm_logits_off(c) + (((size_t)multi_tm(c) * c.n_experts * 8 + 255) & ~(size_t)255);
}
static size_t xm_y_off(const moe_config &c) {
    return xm_h_off(c) + (size_t)multi_um(c) * multi_tm(c) * c.d_ff * 8;
}
static size_t xm_r_off(const moe_config &c) { return xm_y_off(c) + (size_t)2 * multi_tm(c) * c.d_model * 4; }
size_t decode_multi_xchg_bytes(const moe_config &c) {
    return xm_r_off(c) + (size_t)2 * multi_tm(c) * c.d_model * 4;
}

bool decode_multi_supported(const moe_ctx *ctx) {
    const moe_config &c = ctx->cfg;
    if (c.flags & MOE_FLAG_NO_DECODE_KERNEL) return false;
    if (c.max_tokens < 2) return false;
    if (c.d_model > 2 * 4 * NT || c.d_model / 256 > NW || c.n_experts > 32 * EPL || c.n_experts % 4) return false;
    if (c.d_ff % 128) return false;   // the h table's warps each take one token's whole 32-block groups
    if (c.top_k > KMAX) return false;
    return ctx->mdec.smem_bytes > 0;
}

int decode_multi_setup(moe_ctx *ctx) {
    const moe_config &c = ctx->cfg;
    MultiState &ms = ctx->mdec;
    ms.smem_bytes = 0;
    if (c.max_tokens < 2) return MOE_OK;
    cudaDeviceProp prop;
    QE_CHECK(cudaGetDeviceProperties(&prop, ctx->device));
    int G = prop.multiProcessorCount;
    if (G > c.d_model / 16) G = c.d_model / 16;
    const int TM = multi_tm(c), UM = multi_um(c);
    const int rpc = (c.n_experts + G - 1) / G;
    if (rpc > 8) return MOE_OK;
    // experts a CTA's down run may touch
    const long long n_dn_max = ((long long)UM * (c.d_model / 16) + G - 1) / G;
    const int ntile_dn = c.d_model / 16;
    const int span = (int)((n_dn_max + ntile_dn - 2) / ntile_dn) + 1;
    if (span > MAX_SPAN) return MOE_OK;
    int slot = ctx->gu.tile_bytes > ctx->dn.tile_bytes ? ctx->gu.tile_bytes : ctx->dn.tile_bytes;
    size_t fixed = 0;
    auto take = [&fixed](size_t bytes) {
        int off = (int)fixed;
        fixed = (fixed + bytes + 127) & ~(size_t)127;
        return off;
    };
    const size_t xb_bytes = (size_t)TM * (c.d_model + 8) * 2;
    const size_t htab_bytes = (size_t)span * (c.d_ff / 64) * 4 * 32 * 16;
    ms.off_router = take((size_t)rpc * c.d_model * 4);
    ms.off_xb = take(xb_bytes > htab_bytes ? xb_bytes : htab_bytes);
    ms.off_xoff = take((size_t)(c.d_model / 32) * 2 * TM * 4);
    ms.off_hsum = take((size_t)2 * span * TM * (c.d_ff / 32) * 4);
    ms.off_uexp = take((size_t)UM * 4);
    ms.off_wtab = take((size_t)UM * TM * 4);
    ms.off_misc = take(sizeof(MiscM));
    ms.off_ltab = take((size_t)c.n_layers * sizeof(LayerPtrs));
    size_t limit = (size_t)prop.sharedMemPerBlockOptin;
    int nslot = MAX_SLOTS;
    while (nslot >= 2 && fixed + (size_t)nslot * slot > limit) --nslot;
    if (nslot < 2) return MOE_OK;
    // the input phase keeps the token rows (fp32) in the ring between its two passes
    if ((size_t)nslot * slot < (size_t)TM * c.d_model * 4) return MOE_OK;
    ms.off_ring = (int)fixed;
    ms.nslot = nslot;
    ms.slot_bytes = slot;
    ms.rpc = rpc;
    ms.span = span;
    ms.grid = G;
    ms.tm = TM;
    ms.um = UM;
    ms.smem_bytes = (int)(fixed + (size_t)nslot * slot);
    const void *kfn = c.fmt == MOE_Q4B32   ? (const void *)k_decode_multi<MOE_Q4B32>
                      : c.fmt == MOE_Q2B32 ? (const void *)k_decode_multi<MOE_Q2B32>
                                           : (const void *)k_decode_multi<MOE_Q3B32>;
    QE_CHECK(cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, ms.smem_bytes));
    int per_sm = 0;
    QE_CHECK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, NTT, ms.smem_bytes));
    if (per_sm < 1) ms.smem_bytes = 0;
    return MOE_OK;
}

int launch_decode_multi(moe_ctx *ctx, int layer0, int L, const uint16_t *x, int T, bool stack, float *resid_out,
                        uint16_t *y, float *yf, int32_t *ids, float *w, const moe_stack_record *rec, int rec_n,
                        int rec_r0, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    MultiState &ms = ctx->mdec;
    if (T < 1 || T > ms.tm) return MOE_ERR_INVALID_ARG;
    MultiParams p;
    memset(&p, 0, sizeof(p));
    p.layers = ctx->d_layers;
    p.layer0 = layer0;
    p.L = L;
    p.d = c.d_model;
    p.E = c.n_experts;
    p.I = c.d_ff;
    p.k = c.top_k;
    p.nsh = c.n_shared;
    p.T = T;
    p.TM = ms.tm;
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
        p.rec_r0 = rec_r0;
    }
    uint8_t *xb = ms.xbuf;
    p.cnt = reinterpret_cast<unsigned *>(xb);
    p.x_logits = reinterpret_cast<unsigned long long *>(xb + xm_logits_off(c));
    // tags of this launch's layers; the area starts zeroed and tags start at 1, so no stale word
    // (earlier launch, earlier layer) carries a tag a reader expects
    p.tag0 = ms.tag;
    ms.tag += (unsigned)L;
    if (ms.tag < p.tag0) {   // wrapped: start the tags over on a cleared area
        QE_CHECK(cudaMemsetAsync(xb + xm_logits_off(c), 0, xm_y_off(c) - xm_logits_off(c), st));
        p.tag0 = 1;
        ms.tag = 1 + (unsigned)L;
    }
    p.x_h = reinterpret_cast<unsigned long long *>(xb + xm_h_off(c));
    p.y_acc = reinterpret_cast<float *>(xb + xm_y_off(c));
    p.r_buf = reinterpret_cast<float *>(xb + xm_r_off(c));
    p.err = ctx->ws.dev_error;
    p.withhold = ((c.flags & MOE_FLAG_TEST_WITHHOLD) && !ctx->dec.withheld) ? 1 : 0;
    if (p.withhold) ctx->dec.withheld = true;
    p.l2_mode = ctx->l2_mode;
    if (c.flags & MOE_FLAG_TRACE) QE_TRY(decode_trace_buffer(ctx, ms.grid, L, TRACE_WORDS_M, st, &p.trace));
    p.nslot = ms.nslot;
    p.slot_bytes = ms.slot_bytes;
    p.rpc = ms.rpc;
    p.span = ms.span;
    p.UM = ms.um;
    p.off_ring = ms.off_ring;
    p.off_router = ms.off_router;
    p.off_xb = ms.off_xb;
    p.off_xoff = ms.off_xoff;
    p.off_hsum = ms.off_hsum;
    p.off_uexp = ms.off_uexp;
    p.off_wtab = ms.off_wtab;
    p.off_misc = ms.off_misc;
    p.off_ltab = ms.off_ltab;
    // counters start from zero, and so do both output buffers
    QE_CHECK(cudaMemsetAsync(xb, 0, decode_multi_counter_bytes(c), st));
    QE_CHECK(cudaMemsetAsync(p.y_acc, 0, (size_t)2 * ms.tm * c.d_model * 4, st));
    void *args[] = {&p};
    const void *kfn = c.fmt == MOE_Q4B32   ? (const void *)k_decode_multi<MOE_Q4B32>
                      : c.fmt == MOE_Q2B32 ? (const void *)k_decode_multi<MOE_Q2B32>
                                           : (const void *)k_decode_multi<MOE_Q3B32>;
    QE_CHECK(cudaLaunchCooperativeKernel(kfn, dim3(ms.grid), dim3(NTT), args, (size_t)ms.smem_bytes, st));
    QE_CHECK_LAUNCH("k_decode_multi");
    return MOE_OK;
}

}  // namespace qeffn

// Internal declarations of the MoE FFN library: context, private weight
// layout, launch helpers.  Nothing here is part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <utility>
#include <vector>

#include "moe.h"

namespace qeffn {

// ---------------------------------------------------------------------------
// Private tiled weight layout ("row tiles").
//
// Every expert matrix is stored as tiles of 16 rows x K.  A gate/up tile t
// holds gate rows 8t..8t+7 (tile rows 0..7) and up rows 8t..8t+7 (tile rows
// 8..15), so one tile yields 8 SwiGLU outputs.  A down tile t holds output rows
// 16t..16t+15.  Inside a tile the codes are grouped by 64-wide k groups; in a
// k group, the 32 lanes of a warp each own one contiguous piece holding the
// codes of the mma.m16n8k16 A fragments that lane needs for the group's four
// 16-wide k slices:
//   lane = 4*g + c  (g = row % 8, c = (k % 8) / 2)
//   register a0: row g,   k = 16s + 2c + {0,1}     a1: row g+8, same k
//   register a2: row g,   k = 16s + 2c + 8 + {0,1} a3: row g+8, same k
// Q4B32: 16 bytes per lane and group = 4 words, word m = slice m, nibble n of
//   the word (bits 4n..4n+3): n = reg + 4*hi  (hi = odd k of the pair).
// Q3B32: 12 bytes per lane and group = 3 words.  Register q = 4*m + reg
//   (0..15); for q < 15 its two codes are the 3-bit fields of word q/5 at bits
//   3f (even k) and 16+3f (odd k), f = q%5; register 15's codes are spread
//   over bit 15 (even k) and bit 31 (odd k) of words 0,1,2 (code bit b in
//   word b).
// Q2B32: 8 bytes per lane and group = 2 words.  Bits 16*hi + 2f (f = 0..7) of
//   word w hold the code of slice m = w + 2*((f >> 1) & 1), register
//   reg = (f & 1) + 2*(f >> 2): a word's fields 0,1,4,5 are the four
//   registers of slice w (first 32-block of the group) and fields 2,3,6,7
//   those of slice w + 2 (second block), so that an fp16 decode can OR each
//   field into the mantissa of 1024 at its place (x1, x4, x16, x64) with the
//   same multiplier for every row of a block.
// After the codes: the tile's fp16 scales, [16 rows][K/32 blocks].
// The byte count equals the canonical layout's.
// ---------------------------------------------------------------------------
struct MatLayout {
    int K;           // reduction length (multiple of 64)
    int n_tiles;     // 16-row tiles per expert
    int kg_bytes;    // bytes per k group (all lanes): 512 (Q4) / 384 (Q3) / 256 (Q2)
    int code_bytes;  // (K/64) * kg_bytes
    int tile_bytes;  // code_bytes + 16 * (K/32) * 2
    size_t expert_bytes;
};

inline MatLayout make_layout(int fmt, int rows, int K) {
    MatLayout L;
    L.K = K;
    L.n_tiles = rows / 16;
    L.kg_bytes = (fmt == MOE_Q4B32) ? 512 : (fmt == MOE_Q2B32) ? 256 : 384;
    L.code_bytes = (K / 64) * L.kg_bytes;
    L.tile_bytes = L.code_bytes + 16 * (K / 32) * 2;
    L.expert_bytes = (size_t)L.n_tiles * L.tile_bytes;
    return L;
}

// Down matrix in chunk order (the single-token split kernel, decode_split.cu; used by
// contexts whose calls carry one token).  Per expert: for each 16-wide k chunk c16 (= one k16
// slice of the down projection's reduction dimension, i.e. 16 SwiGLU rows), the codes of all d
// output rows as d/64 row groups of 32 lane pieces; a piece holds the mma A fragments of the
// group's four 16-row tiles for that slice, in the row-tile layout's bit order with "slice m of
// the k group" read as "row tile m of the group" (so the same code-to-operand conversions apply).
// After every chunk's codes: the scales by 32-block, [I/32][d] fp16.  Same byte count as the
// row-tile layout.
struct ChunkLayout {
    int chunk_bytes = 0;       // (d / 64) * kg_bytes
    int code_bytes = 0;        // (I / 16) * chunk_bytes
    size_t expert_bytes = 0;   // code_bytes + (I / 32) * d * 2
};

inline ChunkLayout make_chunk_layout(int fmt, int d, int I) {
    ChunkLayout C;
    const int kg_bytes = (fmt == MOE_Q4B32) ? 512 : (fmt == MOE_Q2B32) ? 256 : 384;
    C.chunk_bytes = (d / 64) * kg_bytes;
    C.code_bytes = (I / 16) * C.chunk_bytes;
    C.expert_bytes = (size_t)C.code_bytes + (size_t)(I / 32) * d * 2;
    return C;
}

// Byte offset (within a tile's code area) and bit offset of the code of
// tile row r (0..15), column k, Q4B32.
__host__ __device__ inline void q4_code_pos(int r, int k, int *byte, int *shift) {
    int g = r & 7, half = r >> 3;
    int s = k >> 4, kk = k & 15;
    int kg = s >> 2, m = s & 3;
    int c = (kk & 7) >> 1, hi = kk & 1, second = kk >> 3;
    int reg = second * 2 + half;
    int n = reg + 4 * hi;
    *byte = kg * 512 + (g * 4 + c) * 16 + m * 4 + (n >> 1);
    *shift = (n & 1) * 4;
}

// Q3B32: the three (byte, bit) positions of the code bits b = 0,1,2.
__host__ __device__ inline void q3_code_pos(int r, int k, int byte[3], int bit[3]) {
    int g = r & 7, half = r >> 3;
    int s = k >> 4, kk = k & 15;
    int kg = s >> 2, m = s & 3;
    int c = (kk & 7) >> 1, hi = kk & 1, second = kk >> 3;
    int reg = second * 2 + half;
    int q = 4 * m + reg;
    int base = kg * 384 + (g * 4 + c) * 12;
    for (int b = 0; b < 3; ++b) {
        int word, wbit;
        if (q < 15) {
            word = q / 5;
            wbit = 3 * (q % 5) + 16 * hi + b;
        } else {
            word = b;
            wbit = 15 + 16 * hi;
        }
        byte[b] = base + word * 4 + (wbit >> 3);
        bit[b] = wbit & 7;
    }
}

// Q2B32: byte offset and bit offset of the 2-bit code of tile row r, column k.
__host__ __device__ inline void q2_code_pos(int r, int k, int *byte, int *shift) {
    int g = r & 7, half = r >> 3;
    int s = k >> 4, kk = k & 15;
    int kg = s >> 2, m = s & 3;
    int c = (kk & 7) >> 1, hi = kk & 1, second = kk >> 3;
    int reg = second * 2 + half;
    int w = m & 1;
    int f = (reg & 1) + 2 * (m >> 1) + 4 * (reg >> 1);
    int bit = 16 * hi + 2 * f;
    *byte = kg * 256 + (g * 4 + c) * 8 + w * 4 + (bit >> 3);
    *shift = bit & 7;
}

__device__ inline int tile_code(int fmt, const uint8_t *tile, int r, int k) {
    if (fmt == MOE_Q4B32) {
        int byte, sh;
        q4_code_pos(r, k, &byte, &sh);
        return (tile[byte] >> sh) & 15;
    }
    if (fmt == MOE_Q2B32) {
        int byte, sh;
        q2_code_pos(r, k, &byte, &sh);
        return (tile[byte] >> sh) & 3;
    }
    int byte[3], bit[3];
    q3_code_pos(r, k, byte, bit);
    int v = 0;
    for (int b = 0; b < 3; ++b) v |= ((tile[byte[b]] >> bit[b]) & 1) << b;
    return v;
}

__device__ inline float tile_scale(const uint8_t *tile, const MatLayout &L, int r, int blk) {
    const __half *s = reinterpret_cast<const __half *>(tile + L.code_bytes);
    return __half2float(s[r * (L.K / 32) + blk]);
}

// ---------------------------------------------------------------------------
// Context
// ---------------------------------------------------------------------------
struct Layer {
    bool loaded = false;
    float *router_w = nullptr;   // [E][d]
    float *router_b = nullptr;   // [E] (zeros when the layer has no bias)
    uint16_t *router_parts = nullptr;  // [3][E][d] bf16 parts of router_w (tensor-core router)
    uint8_t *gu = nullptr;       // [(E + n_shared)] x gu.expert_bytes
    uint8_t *dn = nullptr;       // [(E + n_shared)] x dn.expert_bytes
};

struct Workspace {
    float *logits = nullptr;     // [T][E]
    int32_t *ids = nullptr;      // [T][k]
    float *w = nullptr;          // [T][k]
    int32_t *counts = nullptr;   // [E + n_sh]
    int32_t *offsets = nullptr;  // [E + n_sh + 1]
    int32_t *fill = nullptr;     // [E + n_sh]
    int32_t *perm = nullptr;     // [S] slot at each grouped position
    int32_t *inv = nullptr;      // [S] grouped position of each slot
    int4 *chunks = nullptr;      // [max_chunks] (expert, start, n, 0)
    int32_t *n_chunks = nullptr; // [1]
    float *h = nullptr;          // [S][I] SwiGLU outputs by grouped position
    float *yslot = nullptr;      // [S][d] expert outputs by grouped position
    float *resid = nullptr;      // [T][d] residual stream of the stack
    uint16_t *xs = nullptr;      // [T][d] bf16 layer input of the stack
    uint16_t *ys = nullptr;      // [T][d] bf16 layer output of the stack
    float *yf = nullptr;         // [T][d] fp32 layer output of the stack
    uint16_t *x_io = nullptr;    // [T][d] staging for host I/O
    float *r_io = nullptr;       // [T][d] staging for host I/O
    int *dev_error = nullptr;    // [1]
    int max_chunks = 0;
    // tensor-core prefill path
    uint16_t *x16 = nullptr;     // [T][d] fp16 copy of the layer input
    uint16_t *h16 = nullptr;     // [S][I] fp16 SwiGLU outputs by grouped position
    float *y_acc = nullptr;      // [T][d] fp32 output accumulator
    int4 *tc_items = nullptr;    // work items of one grouped GEMM
    int32_t *tc_n_items = nullptr;
    size_t tc_items_max = 0;
    // decoded-weight cache of the tensor-core path: experts with more than three 256-row blocks
    // get their fp16 B stages decoded once per forward (empty when it did not fit memory)
    uint16_t *wcache = nullptr;  // [cache_cap][3 d I] fp16, swizzled 256x64 stage images
    int32_t *cache_slot = nullptr;   // [experts] slot or -1
    int32_t *cache_expert = nullptr; // [cache_cap] expert of a slot
    int32_t *cache_n = nullptr;      // slots in use
    int cache_cap = 0;
};

// Device-side table of one layer's weights (the persistent kernels walk it).
struct LayerPtrs {
    const float *rw;      // router [E][d]
    const float *rb;      // router bias [E]
    const uint8_t *gu;    // gate/up tiles of E + n_shared experts
    const uint8_t *dn;    // down tiles of E + n_shared experts
};

// Launch plan of the single-token decode kernel (decode.cu).
struct DecodeState {
    int grid = 0;         // CTAs (one per SM)
    int smem_bytes = 0;   // 0: the shape does not fit the kernel
    int nslot = 0, slot_bytes = 0, rpc = 0;
    int gu_units_max = 0, dn_units_max = 0;   // per-CTA unit counts the carve is sized for
    int off_ring = 0, off_router = 0, off_x16 = 0, off_xh = 0, off_logits = 0, off_htab = 0, off_red = 0,
        off_misc = 0, off_resid = 0, off_sums = 0, off_ltab = 0;
    int sms = 0;          // streaming multiprocessors of the device
    uint8_t *xbuf = nullptr;   // cross-CTA exchange area (counters, logits, h, output parts)
    bool withheld = false;     // the MOE_FLAG_TEST_WITHHOLD call has been made
    unsigned long long *trace = nullptr;   // phase clocks (MOE_FLAG_TRACE)
    size_t trace_cap = 0;                  // records allocated
    int trace_n = 0;                       // records of the last call
    int trace_words = 24;                  // uint64 per record
};

// Launch plan of the few-token decode kernel (decode_multi.cu).
struct MultiState {
    int grid = 0;
    int smem_bytes = 0;   // 0: the shape does not fit the kernel
    int tm = 0;           // tokens per launch the carve holds (<= 8)
    int um = 0;           // union slots: tm * top_k + n_shared
    int nslot = 0, slot_bytes = 0, rpc = 0, span = 0;
    int off_ring = 0, off_router = 0, off_xb = 0, off_xoff = 0, off_hsum = 0, off_uexp = 0,
        off_wtab = 0, off_misc = 0, off_ltab = 0;
    uint8_t *xbuf = nullptr;   // counters, logits, h, output and residual buffers
    unsigned tag = 1;          // tag of the next launch's first layer in the tagged logits area
};

// Launch plan of the single-token split kernel (decode_split.cu).
struct SplitState {
    int grid = 0;
    int smem_bytes = 0;   // 0: the shape does not fit the kernel
    int nslot = 0, slot_bytes = 0, rpc = 0;
    int off_ring = 0, off_router = 0, off_xb = 0, off_xh = 0, off_logits = 0, off_gp = 0, off_ysm = 0,
        off_red = 0, off_misc = 0, off_resid = 0, off_sums = 0, off_ltab = 0;
    uint8_t *xbuf = nullptr;   // counters, logits, the two output buffers
};

// Event pairs around the dominant kernel (moe_timing_enable).
struct Timing {
    bool on = false;
    std::vector<cudaEvent_t> ev;   // 2 * capacity events
    int used = 0;
    long long dropped = 0;
    long long launches_at_read = 0;
    const char *name = "";
};

}  // namespace qeffn

struct moe_ctx {
    moe_config cfg;
    int device;
    int nx;                       // E + n_shared (experts stored per layer)
    qeffn::MatLayout gu, dn;
    std::vector<qeffn::Layer> layers;
    qeffn::Workspace ws;
    size_t allocated = 0;
    std::vector<std::pair<void *, size_t>> allocs;
    qeffn::Timing timing;
    qeffn::LayerPtrs *d_layers = nullptr;   // [n_layers] on the device
    qeffn::DecodeState dec;
    qeffn::MultiState mdec;
    // one-token contexts (max_tokens == 1) keep the down matrices in chunk order for the split
    // kernel; every other context keeps the row-tile order
    bool split_layout = false;
    qeffn::ChunkLayout chunk;
    qeffn::SplitState sdec;
    bool tc_withheld = false;   // the MOE_FLAG_TEST_WITHHOLD gate/up GEMM has run
    int l2_mode = MOE_L2_STREAM;   // L2 eviction priorities of the decode kernels' weight copies
};

namespace qeffn {

// Status plumbing (moe_api.cu)
int set_cuda_error(cudaError_t e, const char *what);
int set_oom(const char *what);
int set_too_many(const char *what);
int ctx_alloc(moe_ctx *ctx, void **p, size_t bytes, const char *what);
void ctx_free(moe_ctx *ctx, void *p);

#define QE_CHECK(call)                                                   \
    do {                                                                 \
        cudaError_t _e = (call);                                         \
        if (_e != cudaSuccess) return qeffn::set_cuda_error(_e, #call);  \
    } while (0)

#define QE_TRY(call)                   \
    do {                               \
        int _s = (call);               \
        if (_s != MOE_OK) return _s;   \
    } while (0)

extern long long g_launches;   // every kernel launch the library issued

#define QE_CHECK_LAUNCH(what)                                            \
    do {                                                                 \
        __atomic_add_fetch(&qeffn::g_launches, 1, __ATOMIC_RELAXED);     \
        cudaError_t _e = cudaGetLastError();                             \
        if (_e != cudaSuccess) return qeffn::set_cuda_error(_e, what);   \
    } while (0)

int timing_begin(moe_ctx *ctx, cudaStream_t st, const char *name);
int timing_end(moe_ctx *ctx, cudaStream_t st);

// Kernels' host launchers (each returns a moe_status)
int launch_repack(moe_ctx *ctx, int fmt, const uint8_t *codes, const uint16_t *scales,
                  const uint8_t *codes_up, const uint16_t *scales_up, int n_experts,
                  int rows, int K, bool gate_up, uint8_t *dst, cudaStream_t st);
int launch_router_simt(const moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T,
                       float *logits, cudaStream_t st);
int launch_topk(const moe_ctx *ctx, const float *logits, int T, int32_t *ids, float *w,
                cudaStream_t st);
int launch_topk_refine(const moe_ctx *ctx, const Layer &Ly, const uint16_t *x, const float *logits, int T,
                       int32_t *ids, float *w, cudaStream_t st);
int launch_dispatch(moe_ctx *ctx, const int32_t *ids, int T, cudaStream_t st);
int launch_route_raw(const uint16_t *x, int T, int d, int E, int k, const float *W, const float *b,
                     float *logits, int32_t *ids, float *w, cudaStream_t st);
int launch_experts_simt(moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T,
                        cudaStream_t st);
int launch_combine(const moe_ctx *ctx, int T, const float *w, uint16_t *y, float *yf,
                   cudaStream_t st);
int launch_resid_norm(const moe_ctx *ctx, int T, float *resid, const uint16_t *y_add,
                      const uint16_t *x_in, uint16_t *x_out, cudaStream_t st);
bool decode_supported(const moe_ctx *ctx);   // the shape fits the single-token kernel
// Token counts up to this run the single-token kernel once per token (the tokens
// of a layer, and of a stack, are independent); from TC_MIN_TOKENS on the
// tensor-core grouped GEMMs take over.  Measured on a B200 (one layer of the
// 2560 x 512-expert shape, Q4B32): the single-token kernel costs ~25 us per token,
// the tensor-core path ~280 us at 64 tokens and less with fewer experts touched,
// the CUDA-core path 0.8 ms at 16 tokens; so the tensor cores take over early.
constexpr int DECODE_TOKENS_MAX = 8;
constexpr int TC_MIN_TOKENS = DECODE_TOKENS_MAX + 1;
int decode_setup(moe_ctx *ctx);
size_t decode_xchg_bytes(const moe_config &c);
size_t decode_xchg_counter_bytes();   // the counters at the start of the exchange area
// Single-token split kernel (contexts with max_tokens == 1; down matrices in chunk order).
bool decode_split_supported(const moe_ctx *ctx);
int decode_split_setup(moe_ctx *ctx);
size_t decode_split_xchg_bytes(const moe_config &c);
int launch_decode_split(moe_ctx *ctx, int layer0, int L, const uint16_t *x, bool stack, float *resid_out, uint16_t *y,
                        float *yf, int32_t *ids, float *w, const moe_stack_record *rec, int rec_n, int rec_r,
                        cudaStream_t st);
int launch_repack_chunks(moe_ctx *ctx, int fmt, const uint8_t *codes, const uint16_t *scales, int n_experts,
                         uint8_t *dst, cudaStream_t st);
// Few-token decode: 2..DECODE_MULTI_MAX tokens run the few-token kernel, up to
// eight tokens per launch (one read of the batch's experts per layer).  Measured on
// a B200 (one layer, 2560 x 512 experts, Q4B32): ~76 us per launch of eight tokens
// against ~370 us for the tensor-core path at 17..64 tokens, whose cost there is
// the k-group steps of ~200 nearly empty experts; four launches still win.
constexpr int DECODE_MULTI_MAX = 32;
bool decode_multi_supported(const moe_ctx *ctx);
int decode_multi_setup(moe_ctx *ctx);
size_t decode_multi_xchg_bytes(const moe_config &c);
size_t decode_multi_counter_bytes(const moe_config &c);
int launch_decode_multi(moe_ctx *ctx, int layer0, int L, const uint16_t *x, int T, bool stack, float *resid_out,
                        uint16_t *y, float *yf, int32_t *ids, float *w, const moe_stack_record *rec, int rec_n,
                        int rec_r0, cudaStream_t st);
// Phase-trace buffer of the persistent decode kernels (grid x L records of `words` uint64), cleared on st.
int decode_trace_buffer(moe_ctx *ctx, int grid, int L, int words, cudaStream_t st, unsigned long long **out);
int launch_decode(moe_ctx *ctx, int layer0, int L, const uint16_t *x, bool stack, float *resid_out,
                  uint16_t *y, float *yf, int32_t *ids, float *w, const moe_stack_record *rec, int rec_n, int rec_r,
                  cudaStream_t st);
bool tc_supported(const moe_ctx *ctx, int T);
bool tc_router_supported(const moe_ctx *ctx, int T);
int launch_split_router(const float *w, size_t n, uint16_t *parts, cudaStream_t st);
int launch_tc_router(moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T, float *logits, cudaStream_t st);
size_t tc_items_max(const moe_config &c);
int launch_tc_experts(moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T, const float *w_route,
                      uint16_t *y, float *yf, cudaStream_t st);
int launch_record(const moe_ctx *ctx, int T, int layer_idx, const moe_stack_record *rec,
                  const uint16_t *x, const uint16_t *y, const float *yf, const int32_t *ids,
                  const float *w, cudaStream_t st);

}  // namespace qeffn

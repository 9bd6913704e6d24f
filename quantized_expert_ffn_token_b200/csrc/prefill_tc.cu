// Many-token (prefill) expert path on the 5th-generation tensor cores.
//
// After routing, the (token, expert) slots are grouped by expert; each expert
// is then two GEMMs over its slots:
//   gate/up  [cnt x d] . [d x 2I]  -> SwiGLU -> h [cnt x I]      (fp16)
//   down     [cnt x I] . [I x d]   -> y[token] += w_slot * out   (fp32)
// One persistent kernel per GEMM, one CTA per SM, warp-specialised:
//   warp 0      : allocates TMEM, one lane issues tcgen05.mma (kind::f16,
//                 fp16 x fp16 -> fp32 in TMEM) and tcgen05.commit;
//   warps 1..8  : weight producers, two 16-row tiles of the B stage each: the
//                 weights are decoded from the packed row tiles to fp16
//                 (w = s * (q - zero), one rounding) and stored with stmatrix
//                 in the 128-byte-swizzled K-major layout the MMA descriptors
//                 describe;
//   warps 9..11 : A-row loaders: A rows (tokens or h rows) are gathered with
//                 16-byte cp.async into the same layout;
//   warps 12..15: epilogue, tcgen05.ld from TMEM (lane quarter = warp % 4):
//                 SwiGLU into fp16 h (gate/up), or w_slot * out reduced into
//                 y through a small shared-memory transpose (down).
// A work item is (expert, 256 slots, 256 output columns): two M=128
// accumulators share every decoded weight stage (TMEM: 2 x 256 fp32 columns),
// so the weight decode is paid once per 256 slots; experts of more than three
// 256-slot blocks are decoded once per call into fp16 stage images instead.
//
// Expert network = SwiGLU; routing weights and block formats as in moe.h.
// The weights are rounded to fp16 here (the tensor cores take one operand
// type per MMA), which is the one place the layer is not exact in fp32; the
// resulting error (about 4e-4 relative L2 before the bf16 output rounding) is
// inside the layer's 1e-3 bound.
#include <math.h>
#include <string.h>

#include "moe_internal.cuh"

namespace qeffn {

namespace {

constexpr int TC_NT = 512;                 // 16 warps
constexpr int TC_PROD_W0 = 1, TC_PROD_NW = 8;   // weight producers: two row tiles of the B stage each
constexpr int TC_ALD_W0 = 9, TC_ALD_NW = 3;     // A-row loaders
constexpr int TC_ALD_NT = TC_ALD_NW * 32;
constexpr int TC_EPI_W0 = 12;              // warps 12..15: TMEM lane quarters 0..3 (warp % 4)
constexpr int TC_BM = 256;                 // slots per work item (2 x M=128)
constexpr int TC_ALD_MAXJ = (TC_BM * 8 + TC_ALD_NT - 1) / TC_ALD_NT;   // 16-byte A chunks per loader and stage
constexpr int TC_BN = 256;                 // output columns per work item
constexpr int TC_BK = 64;                  // k per pipeline stage (one 128-byte swizzle row)
constexpr int TC_STAGES = 3;
constexpr int TC_PF = 3;                    // k groups ahead that a weight producer prefetches into L2
constexpr int A_STAGE_BYTES = TC_BM * TC_BK * 2;   // 32 KB
constexpr int B_STAGE_BYTES = TC_BN * TC_BK * 2;   // 32 KB
// Producers' weight staging: 2 slots x 3 fields (codes of tile 0, codes of
// tile 1, the four scales) x one 16-byte entry per producer thread, field-major
// so that a warp's accesses to one field are contiguous (no bank conflicts).
constexpr int RAW_FIELD = TC_PROD_NW * 32 * 16;
constexpr int RAW_BYTES = 2 * 3 * RAW_FIELD;
constexpr int STG_WARP_FLOATS = 32 * 16;            // epilogue staging per warp: 32 rows x 16 fp32
constexpr int STG_BYTES = 4 * STG_WARP_FLOATS * 4;  // four epilogue warps: 8 KB
// Experts with at least this many rows in a call have their fp16 stage images decoded once
// (k_cache_fill) and copied by every 256-row block; smaller ones are decoded by the GEMM's
// producers per block.  An image costs 6 d I bytes written and read back against the few
// bits per weight of codes that a block reads otherwise: measured on B200, with three
// blocks per expert (uniform routing at 32,768 tokens) decoding in the GEMM was 10 %
// faster, while Zipf-skewed experts of thousands of rows gain from the cache.
constexpr int TC_CACHE_MIN_ROWS = 3 * 256 + 1;
constexpr long long TC_SPIN = 4000000000LL;        // clock64 cycles, about two seconds

struct TcParams {
    int fmt, zero;
    int K;                      // reduction length (d or I)
    int N;                      // output columns (2I or d)
    MatLayout L;                // weight row-tile layout of this GEMM
    const uint8_t *W;           // [experts] packed tiles
    const uint16_t *A;          // fp16 rows: x16 [T][d] (gate/up) or h16 [S][I] (down)
    int a_by_token;             // 1: A row = token of the slot (gather), 0: A row = slot position
    const int32_t *perm;        // grouped position -> slot
    const int32_t *offsets;     // expert -> first grouped position
    const int4 *items;          // (expert, first position, rows, n-tile)
    const int32_t *n_items;
    int T, k, E;
    // gate/up epilogue
    uint16_t *h16;              // [S][I] fp16
    int I;
    // down epilogue
    float *y_acc;               // [T][d]
    const float *w_route;       // [T][k]
    int d;
    // router mode
    const uint16_t *rparts;     // [3][E][d] bf16 parts of the fp32 router rows
    const float *rbias;         // [E]
    float *logits;              // [T][E]
    int n_items_direct;         // router: items computed from the index (no item list)
    // decoded-weight cache: stage images of experts with more than three 256-row blocks
    const uint16_t *wcache;     // [slot][gate/up stages, down stages][256 x 64 fp16, swizzled]
    const int32_t *cache_slot;  // [expert] slot or -1 (NULL: no cache)
    size_t cache_off;           // fp16 offset of this GEMM's stages within a slot
    size_t cache_stride;        // fp16 per slot (3 d I)
    int *err;
    int withhold;               // test hook: CTA 0 never signals its first accumulator as full
};

enum TcMode { TC_GATEUP = 0, TC_DOWN = 1, TC_ROUTER = 2 };

__device__ __forceinline__ uint32_t su32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

__device__ __forceinline__ void mbar_init(uint64_t *b, int count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(su32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait; false on timeout or when another CTA reported an error.
__device__ __forceinline__ bool mbar_wait_b(uint64_t *b, uint32_t parity, int *err) {
    long long t0 = clock64();
    for (int it = 0;; ++it) {
        if (mbar_try(b, parity)) return true;
        if ((it & 63) == 63) {
            if (*(volatile int *)err != 0) return false;
            if (clock64() - t0 > TC_SPIN) {
                atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
}
// Bounded wait that does not stop early on an error elsewhere: for draining work that is in
// flight before the CTA exits (a copy or an MMA always completes).
__device__ __forceinline__ void mbar_drain(uint64_t *b, uint32_t parity, int *err) {
    long long t0 = clock64();
    for (int it = 0;; ++it) {
        if (mbar_try(b, parity)) return;
        if ((it & 63) == 63 && clock64() - t0 > TC_SPIN) {
            atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
            return;
        }
    }
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// This thread's arrival on *b, adding `bytes` of expected transfer to the phase.
__device__ __forceinline__ void mbar_arrive_tx(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}
// Bulk copy global -> shared (16-byte aligned, size a multiple of 16), completing on *b.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *b) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     su32(dst)),
                 "l"(src), "r"(bytes), "r"(su32(b))
                 : "memory");
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(su32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(su32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(su32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// --- tcgen05 -------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] . B[smem]^T, M=128, N=256, K=16, fp16 in, fp32 accumulate.
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on *b once every MMA this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t *b) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(b))
                 : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), 16-byte leading offset (unused by this swizzle),
// descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// Instruction descriptor: fp32 accumulator, fp16 (or bf16) A and B, both
// K-major, N=256, M=128.
constexpr uint32_t IDESC = (1u << 4) | ((uint32_t)(TC_BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t IDESC_BF16 = IDESC | (1u << 7) | (1u << 10);

// Byte offset of (row, k) in a K-major 128-byte-swizzled tile (64 fp16 per row).
__device__ __forceinline__ uint32_t swz(int row, int k) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((((k >> 3) ^ row) & 7) << 4) + ((k & 7) << 1));
}

// fp16x2 helpers
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// fp16 magic numbers: a field OR-ed under 1024.0 reads 1024 + F*q; one fp16
// FMA with 1/F and -(1024/F + zero) gives q - zero exactly.
constexpr uint32_t H_MAGIC = 0x64006400u, H_ONE = 0x3C003C00u, H_16TH = 0x2C002C00u;
constexpr uint32_t H_8TH = 0x30003000u, H_64TH = 0x24002400u;
constexpr uint32_t H_M1032 = 0xE408E408u, H_M72 = 0xD480D480u;              // Q4: -(1024+8), -(64+8)
constexpr uint32_t H_M1028 = 0xE404E404u, H_M132 = 0xD820D820u, H_M20 = 0xCD00CD00u;  // Q3
constexpr uint32_t H_4TH = 0x34003400u;
constexpr uint32_t H_M1026 = 0xE402E402u, H_M258 = 0xDC08DC08u, H_M66 = 0xD420D420u,   // Q2: -(1024+2),
                   H_M18 = 0xCC80CC80u;                                                 // -(256+2), -(64+2), -(16+2)

// Words of one lane's piece of a k group (Q4: 4, Q3: 3, Q2: 2 of the 4 loaded).
template <int FMT>
__device__ __forceinline__ void load_piece(const uint8_t *src, uint32_t w[4]) {
    if constexpr (FMT == MOE_Q2B32) {
        const uint2 a = *reinterpret_cast<const uint2 *>(src);
        w[0] = a.x, w[1] = a.y, w[2] = w[3] = 0u;
    } else if constexpr (FMT == MOE_Q4B32) {
        const uint4 a = *reinterpret_cast<const uint4 *>(src);
        w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w;
    } else {
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(src);
        w[0] = wp[0], w[1] = wp[1], w[2] = wp[2], w[3] = 0u;
    }
}

// The 16 (q - zero) fp16 pairs of one lane's piece of a k group, register
// q = 4*slice + reg (reg a0..a3 as in the row-tile layout), from its words.
template <int FMT>
__device__ __forceinline__ void decode_words(const uint32_t wv[4], uint32_t r[16]) {
    if constexpr (FMT == MOE_Q2B32) {
        // word w: the 2-bit fields at bits 0, 2, 4, 6 of each half (of w, then of w >> 8) read
        // 1024 + {1, 4, 16, 64} q; fields 0,1,4,5 are registers a0..a3 of slice w, fields
        // 2,3,6,7 those of slice w + 2
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            uint32_t x = wv[w], x8 = wv[w] >> 8;
            r[4 * w + 0] = hfma2((x & 0x00030003u) | H_MAGIC, H_ONE, H_M1026);
            r[4 * w + 1] = hfma2((x & 0x000C000Cu) | H_MAGIC, H_4TH, H_M258);
            r[4 * w + 2] = hfma2((x8 & 0x00030003u) | H_MAGIC, H_ONE, H_M1026);
            r[4 * w + 3] = hfma2((x8 & 0x000C000Cu) | H_MAGIC, H_4TH, H_M258);
            r[4 * w + 8] = hfma2((x & 0x00300030u) | H_MAGIC, H_16TH, H_M66);
            r[4 * w + 9] = hfma2((x & 0x00C000C0u) | H_MAGIC, H_64TH, H_M18);
            r[4 * w + 10] = hfma2((x8 & 0x00300030u) | H_MAGIC, H_16TH, H_M66);
            r[4 * w + 11] = hfma2((x8 & 0x00C000C0u) | H_MAGIC, H_64TH, H_M18);
        }
    } else if constexpr (FMT == MOE_Q4B32) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint32_t w = wv[m], w8 = w >> 8;
            r[4 * m + 0] = hfma2((w & 0x000F000Fu) | H_MAGIC, H_ONE, H_M1032);
            r[4 * m + 1] = hfma2((w & 0x00F000F0u) | H_MAGIC, H_16TH, H_M72);
            r[4 * m + 2] = hfma2((w8 & 0x000F000Fu) | H_MAGIC, H_ONE, H_M1032);
            r[4 * m + 3] = hfma2((w8 & 0x00F000F0u) | H_MAGIC, H_16TH, H_M72);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            uint32_t w = wv[j], w9 = wv[j] >> 9;
            r[5 * j + 0] = hfma2((w & 0x00070007u) | H_MAGIC, H_ONE, H_M1028);
            r[5 * j + 1] = hfma2((w & 0x00380038u) | H_MAGIC, H_8TH, H_M132);
            r[5 * j + 2] = hfma2((w & 0x01C001C0u) | H_MAGIC, H_64TH, H_M20);
            r[5 * j + 3] = hfma2((w9 & 0x00070007u) | H_MAGIC, H_ONE, H_M1028);
            r[5 * j + 4] = hfma2((w9 & 0x00380038u) | H_MAGIC, H_8TH, H_M132);
        }
        uint32_t s = ((wv[0] >> 15) & 0x00010001u) | ((wv[1] >> 14) & 0x00020002u) | ((wv[2] >> 13) & 0x00040004u);
        r[15] = hfma2(s | H_MAGIC, H_ONE, H_M1028);
    }
}

template <int FMT>
__device__ __forceinline__ void decode_piece(const uint8_t *src, uint32_t r[16]) {
    uint32_t w[4];
    load_piece<FMT>(src, w);
    decode_words<FMT>(w, r);
}

// Four 8x8 fp16 matrices from mma-fragment registers to shared memory: lane i
// gives the address of row i % 8 of matrix i / 8 (16 bytes).
__device__ __forceinline__ void stmatrix_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
}

// Decode this warp's two row tiles (2*pw, 2*pw+1 of the n-tile; this lane's
// pieces, lane (g, c)) from the staging bytes into the stage's swizzled fp16
// weight tile: w = s * (q - zero), one fp16 rounding.  The registers are in
// mma fragment order, so each 16x16 block (k16 slice m of a tile) goes out as
// one stmatrix: matrices (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7,
// k 8-15), (rows 8-15, k 8-15) = registers a0, a1, a2, a3.
template <int FMT>
__device__ __forceinline__ void decode_stage(const uint8_t *raw, uint8_t *b_dst, int pw, int lane) {
    const uint32_t bd = su32(b_dst);
    const int mrow = (lane & 7) + 8 * ((lane >> 3) & 1);   // row within the tile this lane addresses
    const int mk = 8 * (lane >> 4);                         // k offset of its matrix
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
        uint32_t q[16];
        decode_piece<FMT>(raw + tt * RAW_FIELD, q);
        uint32_t sgp = *reinterpret_cast<const uint32_t *>(raw + 2 * RAW_FIELD + 8 * tt);   // s[g][2kb], s[g][2kb+1]
        uint32_t s8p = *reinterpret_cast<const uint32_t *>(raw + 2 * RAW_FIELD + 4 + 8 * tt);   // rows g+8
        uint32_t us0 = (sgp & 0xFFFFu) * 0x10001u, us1 = (sgp >> 16) * 0x10001u;
        uint32_t u80 = (s8p & 0xFFFFu) * 0x10001u, u81 = (s8p >> 16) * 0x10001u;
        const int row = 16 * (2 * pw + tt) + mrow;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint32_t sg = m < 2 ? us0 : us1, s8 = m < 2 ? u80 : u81;
            stmatrix_x4(bd + swz(row, 16 * m + mk), hmul2(q[4 * m + 0], sg), hmul2(q[4 * m + 1], s8),
                        hmul2(q[4 * m + 2], sg), hmul2(q[4 * m + 3], s8));
        }
    }
}

__device__ __forceinline__ int slot_token(int slot, int T, int k) {
    int routed = T * k;
    return slot < routed ? slot / k : (slot - routed) % T;
}

// Work item: (expert, first row, rows, n-tile).  The router's items are
// (-, first token, tokens, n-tile) in token-block-major order.
template <int MODE>
__device__ __forceinline__ int4 item_of(const TcParams &p, int item) {
    if constexpr (MODE == TC_ROUTER) {
        int ntn = p.N / TC_BN;
        int mb = item / ntn, nt = item % ntn;
        return make_int4(0, mb * TC_BM, min(TC_BM, p.T - mb * TC_BM), nt);
    } else {
        return p.items[item];
    }
}

struct TcSmem {
    uint64_t full[TC_STAGES];
    uint64_t empty[TC_STAGES];
    uint64_t cbar[TC_STAGES];   // bytes of a cached stage image landed (one phase per cached fill)
    uint64_t mma_done;          // every MMA this CTA issued has completed (exit only)
    uint64_t acc_full[2];       // TMEM slot (256 columns) written by the MMAs
    uint64_t acc_empty[2];      // TMEM slot read out by the epilogue
    uint32_t tmem_base;
    int abort;
};

template <int FMT, int MODE>
__global__ void __launch_bounds__(TC_NT, 1) k_tc_gemm(TcParams p) {
    constexpr bool GATEUP = MODE == TC_GATEUP;
    constexpr uint32_t ID = MODE == TC_ROUTER ? IDESC_BF16 : IDESC;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment of the swizzled tiles
    uint8_t *smem = smem_raw + ((1024 - (su32(smem_raw) & 1023)) & 1023);
    uint8_t *sA = smem;                                  // [stage][256 rows][128 B]
    uint8_t *sB = smem + TC_STAGES * A_STAGE_BYTES;      // [stage][256 rows][128 B]
    uint8_t *sRaw = sB + TC_STAGES * B_STAGE_BYTES;      // producers' private weight staging
    float *sStg = reinterpret_cast<float *>(sRaw + RAW_BYTES);   // down epilogue: row-to-column staging
    TcSmem *ss = reinterpret_cast<TcSmem *>(sRaw + RAW_BYTES + STG_BYTES);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int n_items = p.items ? *p.n_items : p.n_items_direct;
    // router: three bf16 parts of the weights, each over the whole K
    const int nkd = p.K / TC_BK;
    const int nk = MODE == TC_ROUTER ? 3 * nkd : nkd;

    if (tid == 0) {
        for (int s = 0; s < TC_STAGES; ++s) {
            mbar_init(&ss->full[s], TC_PROD_NW * 32 + TC_ALD_NT);
            mbar_init(&ss->empty[s], 1);
            mbar_init(&ss->cbar[s], 1);
        }
        mbar_init(&ss->mma_done, 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(&ss->acc_full[t], 1);
            mbar_init(&ss->acc_empty[t], 128);
        }
        ss->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tmem_alloc(&ss->tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss->tmem_base;
    bool ok = true;

    if (warp == 0) {
        // ---- MMA issuer ------------------------------------------------------------
        // TMEM is a ring of two 256-column slots; an item takes one slot per M=128
        // accumulator, so an item of at most 128 rows runs while the epilogue still
        // reads the previous item's slot
        int it = 0;
        uint32_t u = 0;                          // slot uses so far (slot u & 1, phase u >> 1)
        uint32_t cpar = 0;                       // bit s: parity of the cached fills of stage s so far
        bool issued = false;                     // this thread issued MMAs
        for (int item = blockIdx.x; item < n_items && ok; item += G) {
            int4 wi = item_of<MODE>(p, item);
            int rows = wi.z;
            const int na = rows > 128 ? 2 : 1;
            const bool cached = MODE != TC_ROUTER && p.cache_slot && p.cache_slot[wi.x] >= 0;
            for (int a = 0; a < na && ok; ++a)
                ok = mbar_wait_b(&ss->acc_empty[(u + a) & 1], (((u + a) >> 1) & 1) ^ 1, p.err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t t0 = tmem + 256 * (u & 1), t1 = tmem + 256 * ((u + 1) & 1);
            for (int kb = 0; kb < nk && ok; ++kb, ++it) {
                int s = it % TC_STAGES;
                ok = mbar_wait_b(&ss->full[s], (uint32_t)((it / TC_STAGES) & 1), p.err);
                if (ok && cached) {   // the stage's weights came as one bulk copy of a cached image
                    ok = mbar_wait_b(&ss->cbar[s], (cpar >> s) & 1u, p.err);
                    cpar ^= 1u << s;
                }
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    issued = true;
                    uint32_t a0 = su32(sA + s * A_STAGE_BYTES), b0 = su32(sB + s * B_STAGE_BYTES);
#pragma unroll
                    for (int j = 0; j < TC_BK / 16; ++j) {
                        uint64_t bd = sdesc(b0 + 32 * j);
                        umma_f16(t0, sdesc(a0 + 32 * j), bd, ID, (kb | j) != 0);
                        if (na == 2) umma_f16(t1, sdesc(a0 + 128 * 128 + 32 * j), bd, ID, (kb | j) != 0);
                    }
                    umma_commit(&ss->empty[s]);
                }
                __syncwarp();
            }
            if (ok && lane == 0 && !(p.withhold && blockIdx.x == 0 && u == 0))
                for (int a = 0; a < na; ++a) umma_commit(&ss->acc_full[(u + a) & 1]);
            __syncwarp();
            u += na;
        }
        // no MMA may still read shared memory or write TMEM when the CTA frees them (after a
        // failed wait nobody else waited for the last commits)
        if (lane == 0 && issued) {
            umma_commit(&ss->mma_done);
            mbar_drain(&ss->mma_done, 0, p.err);
        }
        __syncwarp();
    } else if (warp >= TC_PROD_W0 && warp < TC_PROD_W0 + TC_PROD_NW) {
        // ---- producers ---------------------------------------------------------------
        const int pt = tid - TC_PROD_W0 * 32;   // 0..255
        const int pw = pt >> 5;                  // producer warp 0..7: row tiles 2 pw, 2 pw + 1
        const int g = lane >> 2;                 // scale rows g, g+8 of this lane's pieces
        int it = 0;
        int pending = -1;                        // stage whose cp.async group is still in flight
        uint32_t cpar = 0, cfilled = 0;          // thread 0: cached-fill parity / issued, per stage
        uint8_t *myraw = sRaw + pt * 16;         // + (slot * 3 + field) * RAW_FIELD
        for (int item = blockIdx.x; item < n_items && ok; item += G) {
            int4 wi = item_of<MODE>(p, item);
            const int e = wi.x, nt = wi.w;
            const int ch = pt & 7;                   // router B: chunk of rows 32j + pt / 8
            const uint32_t a_off = swz(pt >> 3, ch * 8);
            // weights: this warp decodes row tiles 2*pw and 2*pw+1 of the 16 in the n-tile
            const uint8_t *wexp = p.W + (size_t)e * p.L.expert_bytes;
            const int nb = p.K / 32;
            if constexpr (MODE != TC_ROUTER) {
                const int cslot = p.cache_slot ? p.cache_slot[e] : -1;
                if (cslot >= 0) {
                    // the expert's stage images were decoded once already: one bulk copy per stage,
                    // completing on the stage's cached-image barrier (the MMA warp waits on both)
                    const uint16_t *cs = p.wcache + (size_t)cslot * p.cache_stride + p.cache_off +
                                         (size_t)nt * nk * (B_STAGE_BYTES / 2);
                    for (int kb = 0; kb < nk && ok; ++kb, ++it) {
                        int s = it % TC_STAGES;
                        ok = mbar_wait_b(&ss->empty[s], (uint32_t)(((it / TC_STAGES) & 1) ^ 1), p.err);
                        if (!ok) break;
                        if (pt == 0) {
                            fence_async_smem();
                            mbar_arrive_tx(&ss->cbar[s], B_STAGE_BYTES);
                            bulk_copy_g2s(sB + s * B_STAGE_BYTES, cs + (size_t)kb * (B_STAGE_BYTES / 2),
                                          B_STAGE_BYTES, &ss->cbar[s]);
                            cpar ^= 1u << s;
                            cfilled |= 1u << s;
                        }
                        mbar_arrive(&ss->full[s]);
                    }
                    continue;
                }
            }
            for (int kb = 0; kb < nk && ok; ++kb, ++it) {
                int s = it % TC_STAGES;
                if constexpr (MODE == TC_ROUTER) {   // the loads below go straight into the B stage
                    ok = mbar_wait_b(&ss->empty[s], (uint32_t)(((it / TC_STAGES) & 1) ^ 1), p.err);
                    if (!ok) break;
                }
                uint8_t *b_dst = sB + s * B_STAGE_BYTES;
                const int kx = MODE == TC_ROUTER ? kb % nkd : kb;   // k block of the activations
                if constexpr (MODE == TC_ROUTER) {
                    // B: router rows (experts) 256*nt + 32j + pt/8 of part kb / nkd: one warp
                    // instruction reads four whole 128-byte row segments
                    const uint16_t *bsrc = p.rparts + ((size_t)(kb / nkd) * p.E + (size_t)nt * TC_BN) * p.K + ch * 8;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        cp_async16(b_dst + 4096 * j + a_off, bsrc + (size_t)(32 * j + (pt >> 3)) * p.K + 64 * kx);
                }
                if constexpr (MODE != TC_ROUTER) {
                    // this thread's weight bytes for k group kb (decoded one iteration later)
                    uint8_t *raw = myraw + (it & 1) * 3 * RAW_FIELD;
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        const uint8_t *tile = wexp + (size_t)(nt * 16 + 2 * pw + tt) * p.L.tile_bytes;
                        const uint8_t *cs = tile + (size_t)kb * p.L.kg_bytes;
                        if constexpr (FMT == MOE_Q4B32) {
                            cp_async16(raw + tt * RAW_FIELD, cs + lane * 16);
                        } else if constexpr (FMT == MOE_Q2B32) {
                            cp_async8(raw + tt * RAW_FIELD, cs + lane * 8);
                        } else {
                            cp_async4(raw + tt * RAW_FIELD, cs + lane * 12);
                            cp_async4(raw + tt * RAW_FIELD + 4, cs + lane * 12 + 4);
                            cp_async4(raw + tt * RAW_FIELD + 8, cs + lane * 12 + 8);
                        }
                        const uint8_t *sc = tile + p.L.code_bytes;
                        cp_async4(raw + 2 * RAW_FIELD + 8 * tt, sc + (size_t)(g * nb + 2 * kb) * 2);
                        cp_async4(raw + 2 * RAW_FIELD + 4 + 8 * tt, sc + (size_t)((g + 8) * nb + 2 * kb) * 2);
                        // the stage's loads above wait on one round trip each: bring the codes of
                        // the k group TC_PF ahead (and, at the item's start, the tile's scales) into
                        // L2 now, so those loads find them there
                        if (kb + TC_PF < nk && lane * 128 < p.L.kg_bytes)
                            prefetch_l2(tile + (size_t)(kb + TC_PF) * p.L.kg_bytes + lane * 128);
                        if (kb == 0 && lane * 128 < 16 * nb * 2) prefetch_l2(sc + lane * 128);
                    }
                }
                cp_async_commit();   // one group per stage: its weight bytes
                // the previous stage's group is complete once at most this one is pending: decode
                // its weights, publish it (this stage's loads stay in flight meanwhile)
                if (pending >= 0) {
                    cp_async_wait<1>();
                    if constexpr (MODE != TC_ROUTER) decode_stage<FMT>(myraw + ((it - 1) & 1) * 3 * RAW_FIELD, sB + pending * B_STAGE_BYTES, pw, lane);
                    fence_async_smem();
                    mbar_arrive(&ss->full[pending]);
                }
                pending = s;
                if constexpr (MODE != TC_ROUTER) {
                    // the B stage this k group decodes into (next iteration) must be free; its raw
                    // bytes were requested above without waiting for it, so the load latency overlaps
                    // the wait for the MMA warp to release the stage
                    ok = mbar_wait_b(&ss->empty[s], (uint32_t)(((it / TC_STAGES) & 1) ^ 1), p.err);
                }
            }
            if (!ok) break;
            // flush: the last stage of the item
            cp_async_wait<0>();
            if constexpr (MODE != TC_ROUTER) decode_stage<FMT>(myraw + ((it - 1) & 1) * 3 * RAW_FIELD, sB + pending * B_STAGE_BYTES, pw, lane);
            fence_async_smem();
            mbar_arrive(&ss->full[pending]);
            pending = -1;
        }
        if (pending >= 0) cp_async_wait<0>();
        // every bulk copy has landed before the CTA's shared memory goes away: the last cached
        // fill of each stage (earlier ones were waited for by the MMA warp before the reuse)
        if (pt == 0)
            for (int s = 0; s < TC_STAGES; ++s)
                if ((cfilled >> s) & 1u) mbar_drain(&ss->cbar[s], ((cpar >> s) & 1u) ^ 1u, p.err);
    } else if (warp >= TC_ALD_W0 && warp < TC_ALD_W0 + TC_ALD_NW) {
        // ---- A-row loaders -------------------------------------------------------------
        // 16-byte chunk q = at + TC_ALD_NT * j of the stage: row q / 8, chunk q % 8 (the same
        // for every j), so one warp instruction reads four whole 128-byte row segments
        const int at = tid - TC_ALD_W0 * 32;
        const int ch = at & 7;
        int it = 0;
        int pending = -1;
        for (int item = blockIdx.x; item < n_items && ok; item += G) {
            int4 wi = item_of<MODE>(p, item);
            const int pos0 = wi.y, rows = wi.z;
            const int arows = rows > 128 ? TC_BM : 128;   // rows the MMAs read (one or two accumulators)
            int aoff[TC_ALD_MAXJ];                   // element offset of each chunk's row in A
#pragma unroll
            for (int j = 0; j < TC_ALD_MAXJ; ++j) {
                const int q = at + TC_ALD_NT * j;
                aoff[j] = 0;
                if (q < TC_BM * 8) {
                    const int pos = pos0 + min(q >> 3, rows - 1);   // rows past the end repeat the last
                    int arow;
                    if constexpr (MODE == TC_ROUTER) arow = pos;    // token
                    else arow = p.a_by_token ? slot_token(p.perm[pos], p.T, p.k) : pos;
                    aoff[j] = arow * p.K + ch * 8;
                }
            }
            for (int kb = 0; kb < nk && ok; ++kb, ++it) {
                int s = it % TC_STAGES;
                ok = mbar_wait_b(&ss->empty[s], (uint32_t)(((it / TC_STAGES) & 1) ^ 1), p.err);
                if (!ok) break;
                uint8_t *a_dst = sA + s * A_STAGE_BYTES;
                const int kx = MODE == TC_ROUTER ? kb % nkd : kb;   // k block of the activations
#pragma unroll
                for (int j = 0; j < TC_ALD_MAXJ; ++j) {
                    const int q = at + TC_ALD_NT * j;
                    if (q < arows * 8) cp_async16(a_dst + swz(q >> 3, ch * 8), p.A + aoff[j] + 64 * kx);
                }
                cp_async_commit();
                if (pending >= 0) {   // the previous stage's rows have landed: publish them
                    cp_async_wait<1>();
                    fence_async_smem();
                    mbar_arrive(&ss->full[pending]);
                }
                pending = s;
            }
            if (!ok) break;
            cp_async_wait<0>();
            fence_async_smem();
            mbar_arrive(&ss->full[pending]);
            pending = -1;
        }
        if (pending >= 0) cp_async_wait<0>();
    } else if (warp >= TC_EPI_W0) {
        // ---- epilogue ----------------------------------------------------------------
        const int q4 = warp - TC_EPI_W0;        // TMEM lane quarter
        const int row = 32 * q4 + lane;         // row within each M=128 accumulator
        uint32_t u = 0;                          // TMEM slot uses, in the MMA issuer's order
        for (int item = blockIdx.x; item < n_items && ok; item += G) {
            int4 wi = item_of<MODE>(p, item);
            const int pos0 = wi.y, rows = wi.z, nt = wi.w;
            const int na = rows > 128 ? 2 : 1;
            for (int acc = 0; acc < na && ok; ++acc, ++u) {
                ok = mbar_wait_b(&ss->acc_full[u & 1], (u >> 1) & 1, p.err);
                if (!ok) break;
                tc_fence_after();
                int m = 128 * acc + row;
                bool live = m < rows;
                int pos = pos0 + min(m, rows - 1);
                uint32_t tbase = tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)(256 * (u & 1));
                if constexpr (MODE == TC_ROUTER) {
                    float *lrow = p.logits + (size_t)pos * p.E + (size_t)nt * TC_BN;
                    const float *bb = p.rbias + (size_t)nt * TC_BN;
                    for (int cb = 0; cb < TC_BN / 32; ++cb) {
                        float v[32];
                        tmem_ld32(tbase + 32 * cb, v);
                        if (live) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4) {
                                float4 o = make_float4(v[i] + bb[32 * cb + i], v[i + 1] + bb[32 * cb + i + 1],
                                                       v[i + 2] + bb[32 * cb + i + 2], v[i + 3] + bb[32 * cb + i + 3]);
                                *reinterpret_cast<float4 *>(lrow + 32 * cb + i) = o;
                            }
                        }
                    }
                } else if constexpr (GATEUP) {
                    // columns: 16 per row tile, gate rows 0..7 then up rows 8..15
                    uint16_t *hrow = p.h16 + (size_t)pos * p.I + (size_t)nt * (TC_BN / 2);
                    for (int cb = 0; cb < TC_BN / 32; ++cb) {
                        float v[32];
                        tmem_ld32(tbase + 32 * cb, v);
                        if (live) {
                            uint32_t hw[8];
#pragma unroll
                            for (int t2 = 0; t2 < 2; ++t2) {
#pragma unroll
                                for (int i = 0; i < 8; i += 2) {
                                    float g0 = v[16 * t2 + i], g1 = v[16 * t2 + i + 1];
                                    float u0 = v[16 * t2 + 8 + i], u1 = v[16 * t2 + 8 + i + 1];
                                    // h is rounded to fp16 next: the fast exponential and division
                                    // (a few fp32 ulp) are far inside that rounding
                                    float h0 = __fdividef(g0, 1.f + __expf(-g0)) * u0;
                                    float h1 = __fdividef(g1, 1.f + __expf(-g1)) * u1;
                                    __half2 hh = __floats2half2_rn(h0, h1);
                                    hw[4 * t2 + i / 2] = *reinterpret_cast<uint32_t *>(&hh);
                                }
                            }
                            // h index of this column block: 16 per 32 columns
                            uint4 *dst = reinterpret_cast<uint4 *>(hrow + 16 * cb);
                            dst[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                            dst[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
                        }
                    }
                } else {
                    int slot = p.perm[pos];
                    int tok = slot_token(slot, p.T, p.k);
                    // The weighted rows are added into y with coalesced reductions: each lane holds one
                    // row of 32 columns; 16 of them at a time pass through the warp's staging (row-major,
                    // 16-byte slot c of row r at c ^ (r/2 % 4): conflict-free both ways), and are read
                    // back so that four lanes cover 64 contiguous bytes of one row.  Row-per-lane
                    // reductions (32 rows, 16 bytes each, per instruction) measured twice as slow: the
                    // L2's reduction throughput bounds this epilogue.
                    const float wt = slot < p.T * p.k ? p.w_route[slot] : 1.f;
                    float *stg = sStg + q4 * STG_WARP_FLOATS;
                    const int rr = lane >> 2, c4 = lane & 3;
                    float *ydst[4];   // row 8 j + rr of this warp's 32 (null: past the item's rows)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int r = 8 * j + rr;
                        const int tr = __shfl_sync(0xffffffffu, tok, r);
                        const int lv = __shfl_sync(0xffffffffu, (int)live, r);
                        ydst[j] = lv ? p.y_acc + (size_t)tr * p.d + (size_t)nt * TC_BN + 4 * c4 : nullptr;
                    }
                    for (int cb = 0; cb < TC_BN / 32; ++cb) {
                        float v[32];
                        tmem_ld32(tbase + 32 * cb, v);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int pc = c ^ ((lane >> 1) & 3);
                                *reinterpret_cast<float4 *>(stg + lane * 16 + 4 * pc) =
                                    make_float4(wt * v[16 * hh + 4 * c], wt * v[16 * hh + 4 * c + 1],
                                                wt * v[16 * hh + 4 * c + 2], wt * v[16 * hh + 4 * c + 3]);
                            }
                            __syncwarp();
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int r = 8 * j + rr;
                                const float4 val =
                                    *reinterpret_cast<const float4 *>(stg + r * 16 + 4 * (c4 ^ ((r >> 1) & 3)));
                                if (ydst[j])
                                    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                                                 ::"l"(ydst[j] + 32 * cb + 16 * hh), "f"(val.x), "f"(val.y),
                                                 "f"(val.z), "f"(val.w) : "memory");
                            }
                            __syncwarp();
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&ss->acc_empty[u & 1]);   // this slot may be overwritten
            }
        }
    }
    // every role done: release TMEM
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// Cache slots for the experts with at least TC_CACHE_MIN_ROWS rows (slot order is
// arbitrary; slots past the capacity fall back to decoding in the GEMM).
__global__ void k_cache_assign(const int32_t *__restrict__ counts, int nx, int cap, int32_t *__restrict__ slot,
                               int32_t *__restrict__ expert, int32_t *__restrict__ n_used) {
    for (int e = threadIdx.x; e < nx; e += blockDim.x) {
        int sl = -1;
        if (counts[e] >= TC_CACHE_MIN_ROWS) {
            sl = atomicAdd(n_used, 1);
            if (sl >= cap) sl = -1;
            else expert[sl] = e;
        }
        slot[e] = sl;
    }
}

// Decode the stage images of every cached expert: unit = (slot, GEMM, n-tile,
// k group); 8 warps decode the 16 row tiles of the n-tile exactly as the GEMM's
// producers do (same function, same bytes, same fp16 values) into shared
// memory, then the 32 KB image is written out.
template <int FMT>
__global__ void __launch_bounds__(256) k_cache_fill(const uint8_t *__restrict__ gu, MatLayout Lg,
                                                    const uint8_t *__restrict__ dn, MatLayout Ld,
                                                    const int32_t *__restrict__ expert,
                                                    const int32_t *__restrict__ n_used, int cap,
                                                    uint16_t *__restrict__ wcache, int d, int I) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *stage = smem_raw + ((1024 - (su32(smem_raw) & 1023)) & 1023);   // 32 KB, 1024-aligned
    uint8_t *raw = stage + B_STAGE_BYTES;                                     // 3 x RAW_FIELD
    const int pt = threadIdx.x, pw = pt >> 5, lane = pt & 31, g = lane >> 2;
    const int nslot = min(*n_used, cap);
    const int ntg = 2 * I / TC_BN, nkg = d / TC_BK;      // gate/up stages per n-tile row
    const int ntd = d / TC_BN, nkd = I / TC_BK;          // down
    const int per_slot = ntg * nkg + ntd * nkd;
    const size_t stride = (size_t)3 * d * I;
    for (int u = blockIdx.x; u < nslot * per_slot; u += gridDim.x) {
        const int sl = u / per_slot;
        int r = u - sl * per_slot;
        const bool gate = r < ntg * nkg;
        if (!gate) r -= ntg * nkg;
        const int nk = gate ? nkg : nkd;
        const int nt = r / nk, kb = r - nt * nk;
        const MatLayout &L = gate ? Lg : Ld;
        const uint8_t *wexp = (gate ? gu : dn) + (size_t)expert[sl] * L.expert_bytes;
        const int nb = L.K / 32;
        uint8_t *myraw = raw + pt * 16;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const uint8_t *tile = wexp + (size_t)(nt * 16 + 2 * pw + tt) * L.tile_bytes;
            const uint8_t *cs = tile + (size_t)kb * L.kg_bytes;
            if constexpr (FMT == MOE_Q4B32) {
                cp_async16(myraw + tt * RAW_FIELD, cs + lane * 16);
            } else if constexpr (FMT == MOE_Q2B32) {
                cp_async8(myraw + tt * RAW_FIELD, cs + lane * 8);
            } else {
                cp_async4(myraw + tt * RAW_FIELD, cs + lane * 12);
                cp_async4(myraw + tt * RAW_FIELD + 4, cs + lane * 12 + 4);
                cp_async4(myraw + tt * RAW_FIELD + 8, cs + lane * 12 + 8);
            }
            const uint8_t *sc = tile + L.code_bytes;
            cp_async4(myraw + 2 * RAW_FIELD + 8 * tt, sc + (size_t)(g * nb + 2 * kb) * 2);
            cp_async4(myraw + 2 * RAW_FIELD + 4 + 8 * tt, sc + (size_t)((g + 8) * nb + 2 * kb) * 2);
        }
        cp_async_commit();
        cp_async_wait<0>();
        decode_stage<FMT>(myraw, stage, pw, lane);
        __syncthreads();
        uint16_t *dst = wcache + (size_t)sl * stride + (gate ? 0 : (size_t)2 * I * d) +
                        ((size_t)nt * nk + kb) * (B_STAGE_BYTES / 2);
        for (int i = pt; i < B_STAGE_BYTES / 16; i += 256)
            reinterpret_cast<uint4 *>(dst)[i] = reinterpret_cast<const uint4 *>(stage)[i];
        __syncthreads();
    }
}

// ---- Small experts: a weight-streaming path ---------------------------------------------------
// An expert with at most SMALL_MAX rows in a call costs the tensor-core GEMMs as many k-group steps
// as one with 256 (at 4,096 Zipf-routed tokens, 124 of the 207 active experts have at most 16 rows).
// Each such expert is instead one CTA's work: its rows of the fp16 layer input are staged in shared
// memory once, every warp streams gate/up row tiles through its own ring of cp.async slots (SE_S k
// groups in flight) and multiplies them with mma.sync m16n8k16 (the decoded tile, the same fp16
// w = s (q - zero) as the GEMM's B stage, as A; the rows as one or two 8-column B groups; fp32
// accumulation); SwiGLU h stays in shared memory for the down tiles, whose outputs are added into y.
// Operand rows are stored permuted: within each 64-wide k group, fp16 pair 8m + 4h + c goes to
// 8c + 2m + h, so the eight B registers a lane needs for the group's four k16 slices are 32
// contiguous bytes; rows are padded by 16 bytes so the eight rows a load touches fall in distinct
// banks.
constexpr int SMALL_MAX = 16;
// Calls of fewer tokens keep their small experts in the GEMMs: there the GEMMs are short and nearly
// every expert is small, and the streaming kernel added its own time to theirs (sweep, one layer of
// the 4,096-token shape: 420-430 us against 365 at 17-128 tokens, no gain at 256-512) while from 1,024
// tokens on it took 2-8 % off (597 / 733 / 997 / 1,509 us against 609 / 779 / 1,055 / 1,588 at
// 1,024 / 2,048 / 4,096 / 8,192).
constexpr int SMALL_MIN_TOKENS = 1024;
constexpr int SE_W = 16;                 // warps per CTA
constexpr int SE_S = 8;                  // k groups in flight per warp
constexpr int SE_SLOT = 32 * 16 + 64;    // one k group of one row tile: 16 code bytes per lane, 4 scale bytes per row

__device__ __forceinline__ int perm_word(int w) { return 8 * (w & 3) + 2 * (w >> 3) + ((w >> 2) & 1); }

struct SmallParams {
    const int4 *list;            // (expert, first grouped position, rows, -)
    const int32_t *n_list;
    const int32_t *perm;         // grouped position -> slot
    const uint16_t *x16;         // [T][d] fp16 layer input (the GEMM's A operand)
    const uint8_t *gu, *dn;
    MatLayout Lg, Ld;
    float *y_acc;                // [T][d]
    const float *w_route;        // [T][k]
    int T, k, d, I;
};

__host__ __device__ constexpr size_t small_smem_bytes(int d, int I) {
    return (size_t)SMALL_MAX * (d + 8) * 2 + (size_t)SMALL_MAX * (I + 8) * 2 + (size_t)SE_W * SE_S * SE_SLOT +
           (size_t)SMALL_MAX * 8;
}

__device__ __forceinline__ void mma16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One warp's share of one GEMM of a small expert: row tiles warp, warp + SE_W, ... over K, B rows
// from `bs` (stride bstride halves).  Gate/up: SwiGLU of each tile's gate rows 0..7 and up rows
// 8..15 into hs; down: w_slot x out added into y.
template <int FMT, bool GU>
__device__ __forceinline__ void small_gemm(const SmallParams &p, const int4 ent, const uint16_t *bs, int bstride,
                                           uint16_t *hs, const int2 *tokw, uint8_t *wring, int warp, int lane) {
    const MatLayout &L = GU ? p.Lg : p.Ld;
    const int K = L.K, nkg = K / 64, nb = K / 32;
    const int ntile = (GU ? 2 * p.I : p.d) / 16;
    const int nmine = warp < ntile ? (ntile - 1 - warp) / SE_W + 1 : 0;
    const int nq = nmine * nkg;   // this warp's steps: k group q % nkg of its tile q / nkg
    const uint8_t *wexp = (GU ? p.gu : p.dn) + (size_t)ent.x * L.expert_bytes;
    const int g = lane >> 2, c = lane & 3;
    const bool two = ent.z > 8;
    // step q's codes and scales into slot q % SE_S (one cp.async group per step, empty past the end);
    // each lane copies and later reads only its own bytes of a slot
    // request position (tile rt, k group rkg) and consume position (tile t, k group kg) advance by one
    // k group per step; a slot holds the lane's code bytes and, from lanes 0..15, row lane's scales
    const uint8_t *rtile = wexp + (size_t)warp * L.tile_bytes;
    int rkg = 0, rq = 0;
    const size_t tstep = (size_t)SE_W * L.tile_bytes;
    const int code_off = lane * (FMT == MOE_Q4B32 ? 16 : FMT == MOE_Q2B32 ? 8 : 12);
    const int sc_off = (lane & 15) * nb * 2;
    auto request = [&]() {
        if (rq < nq) {
            uint8_t *slot = wring + (rq % SE_S) * SE_SLOT;
            const uint8_t *cs = rtile + (size_t)rkg * L.kg_bytes + code_off;
            if constexpr (FMT == MOE_Q4B32) {
                cp_async16(slot + lane * 16, cs);
            } else if constexpr (FMT == MOE_Q2B32) {
                cp_async8(slot + lane * 16, cs);
            } else {
                cp_async4(slot + lane * 16, cs);
                cp_async4(slot + lane * 16 + 4, cs + 4);
                cp_async4(slot + lane * 16 + 8, cs + 8);
            }
            if (lane < 16) cp_async4(slot + 512 + lane * 4, rtile + L.code_bytes + sc_off + rkg * 4);
            if (++rkg == nkg) {
                rkg = 0;
                rtile += tstep;
            }
            ++rq;
        }
        cp_async_commit();
    };
#pragma unroll
    for (int q = 0; q < SE_S - 1; ++q) request();
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    int t = warp, kg = 0;
    const uint16_t *brow0 = bs + (size_t)g * bstride + 16 * c, *brow1 = brow0 + (size_t)8 * bstride;
    for (int q = 0; q < nq; ++q) {
        request();
        cp_async_wait<SE_S - 1>();   // step q's bytes (this lane's) have landed
        __syncwarp();                // ... and the scales, which lanes 0..15 copied
        const uint8_t *slot = wring + (q % SE_S) * SE_SLOT;
        uint32_t wv[4];
        load_piece<FMT>(slot + lane * 16, wv);
        const uint32_t sgp = *reinterpret_cast<const uint32_t *>(slot + 512 + g * 4);
        const uint32_t s8p = *reinterpret_cast<const uint32_t *>(slot + 512 + (g + 8) * 4);
        uint32_t qv[16];
        decode_words<FMT>(wv, qv);
        const uint32_t us0 = (sgp & 0xFFFFu) * 0x10001u, us1 = (sgp >> 16) * 0x10001u;
        const uint32_t u80 = (s8p & 0xFFFFu) * 0x10001u, u81 = (s8p >> 16) * 0x10001u;
        // B: rows g and 8 + g, this lane's 32 bytes of the k group
        uint32_t b[2][8];
        {
            const uint4 *bp = reinterpret_cast<const uint4 *>(brow0 + 64 * kg);
            const uint4 v0 = bp[0], v1 = bp[1];
            b[0][0] = v0.x, b[0][1] = v0.y, b[0][2] = v0.z, b[0][3] = v0.w;
            b[0][4] = v1.x, b[0][5] = v1.y, b[0][6] = v1.z, b[0][7] = v1.w;
        }
        if (two) {
            const uint4 *bp = reinterpret_cast<const uint4 *>(brow1 + 64 * kg);
            const uint4 v0 = bp[0], v1 = bp[1];
            b[1][0] = v0.x, b[1][1] = v0.y, b[1][2] = v0.z, b[1][3] = v0.w;
            b[1][4] = v1.x, b[1][5] = v1.y, b[1][6] = v1.z, b[1][7] = v1.w;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t sg = m < 2 ? us0 : us1, s8 = m < 2 ? u80 : u81;
            const uint32_t a0 = hmul2(qv[4 * m + 0], sg), a1 = hmul2(qv[4 * m + 1], s8);
            const uint32_t a2 = hmul2(qv[4 * m + 2], sg), a3 = hmul2(qv[4 * m + 3], s8);
            mma16816_f16(acc[0], a0, a1, a2, a3, b[0][2 * m], b[0][2 * m + 1]);
            if (two) mma16816_f16(acc[1], a0, a1, a2, a3, b[1][2 * m], b[1][2 * m + 1]);
        }
        if (kg == nkg - 1) {
            // lane (g, c) holds rows g and g + 8 of the tile for columns 2c and 2c + 1 of each group
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = 8 * j + 2 * c + e;
                    if (r < ent.z) {
                        if constexpr (GU) {
                            const int hk = 8 * t + g;   // h index of gate row g and up row g + 8
                            const int hpos = 64 * (hk >> 6) + 2 * perm_word((hk & 63) >> 1) + (hk & 1);
                            const float gt = acc[j][e], up = acc[j][2 + e];
                            const __half h = __float2half_rn(__fdividef(gt, 1.f + __expf(-gt)) * up);
                            hs[(size_t)r * (p.I + 8) + hpos] = *reinterpret_cast<const uint16_t *>(&h);
                        } else {
                            const int2 tw = tokw[r];
                            float *y = p.y_acc + (size_t)tw.x * p.d + 16 * t + g;
                            const float wt = __int_as_float(tw.y);
                            atomicAdd(y, wt * acc[j][e]);
                            atomicAdd(y + 8, wt * acc[j][2 + e]);
                        }
                    }
                    acc[j][e] = acc[j][2 + e] = 0.f;
                }
            kg = 0;
            t += SE_W;
        } else {
            ++kg;
        }
        __syncwarp();   // every lane has read the slot's scales before a lane re-requests into it
    }
    cp_async_wait<0>();
}

// Every small expert of the call: a CTA per expert (grid-stride), gate/up then down.
template <int FMT>
__global__ void __launch_bounds__(SE_W * 32, 1) k_small_expert(SmallParams p) {
    extern __shared__ __align__(16) uint8_t sm_small[];
    uint16_t *xs = reinterpret_cast<uint16_t *>(sm_small);                  // [SMALL_MAX][d + 8]
    uint16_t *hs = xs + (size_t)SMALL_MAX * (p.d + 8);                       // [SMALL_MAX][I + 8]
    uint8_t *ring = reinterpret_cast<uint8_t *>(hs + (size_t)SMALL_MAX * (p.I + 8));
    int2 *tokw = reinterpret_cast<int2 *>(ring + (size_t)SE_W * SE_S * SE_SLOT);   // [SMALL_MAX] (token, weight)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *wring = ring + (size_t)warp * SE_S * SE_SLOT;
    const int n = *p.n_list;
    const int ngd = p.d / 64;
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const int4 ent = p.list[i];
        if (tid < ent.z) {
            const int slot = p.perm[ent.y + tid];
            tokw[tid] = make_int2(slot_token(slot, p.T, p.k),
                                  __float_as_int(slot < p.T * p.k ? p.w_route[slot] : 1.f));
        }
        __syncthreads();
        // the expert's rows of the layer input, permuted (rows past ent.z are never used)
        for (int u = tid; u < ent.z * ngd; u += blockDim.x) {
            const int r = u / ngd, kg = u - r * ngd;
            const uint4 *src = reinterpret_cast<const uint4 *>(p.x16 + (size_t)tokw[r].x * p.d + 64 * kg);
            uint32_t o[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 v = src[j];
                o[perm_word(4 * j + 0)] = v.x;
                o[perm_word(4 * j + 1)] = v.y;
                o[perm_word(4 * j + 2)] = v.z;
                o[perm_word(4 * j + 3)] = v.w;
            }
            uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)r * (p.d + 8) + 64 * kg);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
        __syncthreads();
        small_gemm<FMT, true>(p, ent, xs, p.d + 8, hs, tokw, wring, warp, lane);
        __syncthreads();   // every h value is in hs
        small_gemm<FMT, false>(p, ent, hs, p.I + 8, hs, tokw, wring, warp, lane);
        __syncthreads();   // xs, hs and tokw are free for the next expert
    }
}

// Work items of one GEMM: for every expert with more than small_max slots,
// ceil(cnt/256) row blocks x n_tiles column tiles; with `small` set, the list
// of the others that have slots (expert, first position, rows, 0).  The small
// experts go to the streaming kernel only when they fit one wave of its CTAs
// (at most small_ctas of them: at 64 tokens ~250 one-row experts took two waves
// and 15 % longer than the GEMMs); the decision depends on the counts alone, so
// both GEMMs' calls make it alike.  Single block.  The items of two M = 128
// accumulators (blocks of more than 128 rows) come first, then the single-
// accumulator ones: the CTAs take items round-robin, so the costly ones are
// spread first and the cheap ones even out the tail (an expert-ordered list
// left the busiest CTA ~16 % above the mean on a Zipf-routed layer's gate/up
// GEMM, by a count of k groups; this order ~6 %).
__global__ void k_tc_items(const int32_t *__restrict__ counts, const int32_t *__restrict__ offsets, int nx,
                           int n_tiles, int4 *__restrict__ items, int32_t *__restrict__ n_items, int max_items,
                           int small_max, int small_ctas, int4 *__restrict__ small,
                           int32_t *__restrict__ n_small_out) {
    __shared__ int n_big, n_small, n_sm, n_cand;
    if (threadIdx.x == 0) n_big = n_small = n_sm = n_cand = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < nx; e += blockDim.x)
        if (counts[e] > 0 && counts[e] <= small_max) atomicAdd(&n_cand, 1);
    __syncthreads();
    if (n_cand > small_ctas) small_max = 0;
    for (int e = threadIdx.x; e < nx; e += blockDim.x) {
        const int cnt = counts[e];
        if (cnt <= small_max) {
            if (cnt > 0 && small) small[atomicAdd(&n_sm, 1)] = make_int4(e, offsets[e], cnt, 0);
            continue;
        }
        const int nb = cnt / TC_BM + (cnt % TC_BM > 128 ? 1 : 0);   // blocks of more than 128 rows
        if (nb == 0) continue;
        const int base = atomicAdd(&n_big, nb * n_tiles);
        for (int b = 0; b < nb; ++b)
            for (int t = 0; t < n_tiles; ++t) {
                const int idx = base + b * n_tiles + t;
                if (idx < max_items)
                    items[idx] = make_int4(e, offsets[e] + b * TC_BM, min(TC_BM, cnt - b * TC_BM), t);
            }
    }
    __syncthreads();
    const int big = n_big;
    for (int e = threadIdx.x; e < nx; e += blockDim.x) {
        const int cnt = counts[e];
        const int rem = cnt % TC_BM;   // the last, short block, when it has at most 128 rows
        if (cnt <= small_max || rem == 0 || rem > 128) continue;
        const int base = big + atomicAdd(&n_small, n_tiles);
        for (int t = 0; t < n_tiles; ++t) {
            const int idx = base + t;
            if (idx < max_items) items[idx] = make_int4(e, offsets[e] + (cnt / TC_BM) * TC_BM, rem, t);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        *n_items = min(n_big + n_small, max_items);
        if (small) *n_small_out = n_sm;
    }
}

__global__ void k_bf16_to_f16(const uint16_t *__restrict__ x, __half *__restrict__ y, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        y[i] = __float2half_rn(__uint_as_float((uint32_t)x[i] << 16));
}

__global__ void k_finish(const float *__restrict__ yacc, size_t n, uint16_t *__restrict__ y, float *__restrict__ yf) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        float v = yacc[i];
        __nv_bfloat16 b = __float2bfloat16_rn(v);
        y[i] = *reinterpret_cast<uint16_t *>(&b);
        if (yf) yf[i] = v;
    }
}

template <int FMT, int MODE>
int launch_tc(const TcParams &p, int grid, cudaStream_t st) {
    size_t smem = (size_t)TC_STAGES * (A_STAGE_BYTES + B_STAGE_BYTES) + RAW_BYTES + STG_BYTES + sizeof(TcSmem) + 1024;
    QE_CHECK(cudaFuncSetAttribute(k_tc_gemm<FMT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    k_tc_gemm<FMT, MODE><<<grid, TC_NT, smem, st>>>(p);
    QE_CHECK_LAUNCH(MODE == TC_GATEUP ? "k_tc_gemm<gate/up>" : MODE == TC_DOWN ? "k_tc_gemm<down>" : "k_tc_gemm<router>");
    return MOE_OK;
}

// fp32 router rows -> three bf16 parts: w1 = bf16(w), w2 = bf16(w - w1), w3 = bf16(w - w1 - w2).
__global__ void k_split_router(const float *__restrict__ w, size_t n, uint16_t *__restrict__ parts) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        float v = w[i];
        __nv_bfloat16 a = __float2bfloat16_rn(v);
        float r1 = v - __bfloat162float(a);
        __nv_bfloat16 b = __float2bfloat16_rn(r1);
        float r2 = r1 - __bfloat162float(b);
        __nv_bfloat16 c = __float2bfloat16_rn(r2);
        parts[i] = *reinterpret_cast<uint16_t *>(&a);
        parts[n + i] = *reinterpret_cast<uint16_t *>(&b);
        parts[2 * n + i] = *reinterpret_cast<uint16_t *>(&c);
    }
}

}  // namespace

bool tc_router_supported(const moe_ctx *ctx, int T) {
    const moe_config &c = ctx->cfg;
    return tc_supported(ctx, T) && c.n_experts % TC_BN == 0;
}

int launch_split_router(const float *w, size_t n, uint16_t *parts, cudaStream_t st) {
    k_split_router<<<592, 256, 0, st>>>(w, n, parts);
    QE_CHECK_LAUNCH("k_split_router");
    return MOE_OK;
}

int launch_tc_router(moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T, float *logits, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.K = c.d_model;
    p.N = c.n_experts;
    p.E = c.n_experts;
    p.T = T;
    p.A = x;
    p.rparts = Ly.router_parts;
    p.rbias = Ly.router_b;
    p.logits = logits;
    p.n_items_direct = ((T + TC_BM - 1) / TC_BM) * (c.n_experts / TC_BN);
    p.err = ctx->ws.dev_error;
    return launch_tc<MOE_Q4B32, TC_ROUTER>(p, ctx->dec.sms, st);
}

bool tc_supported(const moe_ctx *ctx, int T) {
    const moe_config &c = ctx->cfg;
    if (c.flags & MOE_FLAG_NO_TENSOR_PREFILL) return false;
    if (T < TC_MIN_TOKENS) return false;
    // n-tiles of 256 output columns: 2I and d must be multiples of 256
    if ((2 * c.d_ff) % TC_BN || c.d_model % TC_BN || c.d_model % TC_BK || c.d_ff % TC_BK) return false;
    // A-row offsets are 32-bit element indices: rows (tokens or slots) x K below 2^31
    const long long slots = (long long)c.max_tokens * (c.top_k + c.n_shared);
    return slots * (c.d_model > c.d_ff ? c.d_model : c.d_ff) < (1LL << 31);
}

size_t tc_items_max(const moe_config &c) {
    size_t S = (size_t)c.max_tokens * (c.top_k + c.n_shared);
    size_t nx = c.n_experts + c.n_shared;
    size_t nt = (size_t)((2 * c.d_ff) / TC_BN > c.d_model / TC_BN ? (2 * c.d_ff) / TC_BN : c.d_model / TC_BN);
    return (S / TC_BM + nx) * nt;
}

int launch_tc_experts(moe_ctx *ctx, const Layer &Ly, const uint16_t *x, int T, const float *w_route,
                      uint16_t *y, float *yf, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    Workspace &ws = ctx->ws;
    int dev_sms = ctx->dec.sms;
    size_t Td = (size_t)T * c.d_model;
    k_bf16_to_f16<<<592, 256, 0, st>>>(x, reinterpret_cast<__half *>(ws.x16), Td);
    QE_CHECK_LAUNCH("k_bf16_to_f16");
    int max_items = (int)ws.tc_items_max;

    TcParams p;
    memset(&p, 0, sizeof(p));
    p.fmt = c.fmt;
    p.zero = c.fmt == MOE_Q4B32 ? 8 : (c.fmt == MOE_Q2B32) ? 2 : 4;
    p.perm = ws.perm;
    p.offsets = ws.offsets;
    p.items = ws.tc_items;
    p.n_items = ws.tc_n_items;
    p.T = T;
    p.k = c.top_k;
    p.E = c.n_experts;
    p.I = c.d_ff;
    p.d = c.d_model;
    p.err = ws.dev_error;

    // decoded-weight cache for the experts with more than three 256-row blocks (part of the timed
    // expert work: it takes over decoding from the GEMMs)
    QE_TRY(timing_begin(ctx, st, "k_cache_fill+k_tc_gemm<gate/up>+k_tc_gemm<down>+k_small_expert"));
    if (ws.cache_cap > 0) {
        QE_CHECK(cudaMemsetAsync(ws.cache_n, 0, 4, st));
        k_cache_assign<<<1, 1024, 0, st>>>(ws.counts, ctx->nx, ws.cache_cap, ws.cache_slot, ws.cache_expert,
                                           ws.cache_n);
        QE_CHECK_LAUNCH("k_cache_assign");
        const size_t fsm = B_STAGE_BYTES + 3 * RAW_FIELD + 1024;
        if (c.fmt == MOE_Q4B32) {
            QE_CHECK(cudaFuncSetAttribute(k_cache_fill<MOE_Q4B32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm));
            k_cache_fill<MOE_Q4B32><<<4 * dev_sms, 256, fsm, st>>>(Ly.gu, ctx->gu, Ly.dn, ctx->dn, ws.cache_expert,
                                                                   ws.cache_n, ws.cache_cap, ws.wcache, c.d_model,
                                                                   c.d_ff);
        } else if (c.fmt == MOE_Q2B32) {
            QE_CHECK(cudaFuncSetAttribute(k_cache_fill<MOE_Q2B32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm));
            k_cache_fill<MOE_Q2B32><<<4 * dev_sms, 256, fsm, st>>>(Ly.gu, ctx->gu, Ly.dn, ctx->dn, ws.cache_expert,
                                                                   ws.cache_n, ws.cache_cap, ws.wcache, c.d_model,
                                                                   c.d_ff);
        } else {
            QE_CHECK(cudaFuncSetAttribute(k_cache_fill<MOE_Q3B32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm));
            k_cache_fill<MOE_Q3B32><<<4 * dev_sms, 256, fsm, st>>>(Ly.gu, ctx->gu, Ly.dn, ctx->dn, ws.cache_expert,
                                                                   ws.cache_n, ws.cache_cap, ws.wcache, c.d_model,
                                                                   c.d_ff);
        }
        QE_CHECK_LAUNCH("k_cache_fill");
        p.wcache = ws.wcache;
        p.cache_slot = ws.cache_slot;
        p.cache_stride = (size_t)3 * c.d_model * c.d_ff;
    }

    // gate/up: A = x16 rows gathered by token, N = 2I, K = d; the experts of at most SMALL_MAX rows
    // go to the streaming path (its list in the CUDA-core path's chunk list, unused by this path)
    const size_t small_smem = small_smem_bytes(c.d_model, c.d_ff);
    const int small_max =
        (T >= SMALL_MIN_TOKENS && small_smem <= (size_t)227 * 1024) ? SMALL_MAX : 0;   // per-CTA opt-in limit
    k_tc_items<<<1, 1024, 0, st>>>(ws.counts, ws.offsets, ctx->nx, (2 * c.d_ff) / TC_BN, ws.tc_items,
                                   ws.tc_n_items, max_items, small_max, dev_sms, ws.chunks, ws.n_chunks);
    QE_CHECK_LAUNCH("k_tc_items");
    p.cache_off = 0;
    p.K = c.d_model;
    p.N = 2 * c.d_ff;
    p.L = ctx->gu;
    p.W = Ly.gu;
    p.A = ws.x16;
    p.a_by_token = 1;
    p.h16 = ws.h16;
    // test hook: the context's first gate/up GEMM leaves CTA 0's epilogue waiting until its bound
    p.withhold = ((c.flags & MOE_FLAG_TEST_WITHHOLD) && !ctx->tc_withheld) ? 1 : 0;
    if (p.withhold) ctx->tc_withheld = true;
    int grid = dev_sms;
    if (c.fmt == MOE_Q4B32) QE_TRY((launch_tc<MOE_Q4B32, TC_GATEUP>(p, grid, st)));
    else if (c.fmt == MOE_Q2B32) QE_TRY((launch_tc<MOE_Q2B32, TC_GATEUP>(p, grid, st)));
    else QE_TRY((launch_tc<MOE_Q3B32, TC_GATEUP>(p, grid, st)));
    p.withhold = 0;

    // down: A = h16 rows by grouped position, N = d, K = I
    QE_CHECK(cudaMemsetAsync(ws.y_acc, 0, Td * sizeof(float), st));
    k_tc_items<<<1, 1024, 0, st>>>(ws.counts, ws.offsets, ctx->nx, c.d_model / TC_BN, ws.tc_items,
                                   ws.tc_n_items, max_items, small_max, dev_sms, nullptr, nullptr);
    QE_CHECK_LAUNCH("k_tc_items");
    p.K = c.d_ff;
    p.N = c.d_model;
    p.L = ctx->dn;
    p.W = Ly.dn;
    p.A = ws.h16;
    p.a_by_token = 0;
    p.y_acc = ws.y_acc;
    p.w_route = w_route;
    p.cache_off = (size_t)2 * c.d_ff * c.d_model;   // the down GEMM's stages follow the gate/up ones
    if (c.fmt == MOE_Q4B32) QE_TRY((launch_tc<MOE_Q4B32, TC_DOWN>(p, grid, st)));
    else if (c.fmt == MOE_Q2B32) QE_TRY((launch_tc<MOE_Q2B32, TC_DOWN>(p, grid, st)));
    else QE_TRY((launch_tc<MOE_Q3B32, TC_DOWN>(p, grid, st)));
    if (small_max > 0) {
        SmallParams sp;
        sp.list = ws.chunks;
        sp.n_list = ws.n_chunks;
        sp.perm = ws.perm;
        sp.x16 = reinterpret_cast<const uint16_t *>(ws.x16);
        sp.gu = Ly.gu;
        sp.dn = Ly.dn;
        sp.Lg = ctx->gu;
        sp.Ld = ctx->dn;
        sp.y_acc = ws.y_acc;
        sp.w_route = w_route;
        sp.T = T;
        sp.k = c.top_k;
        sp.d = c.d_model;
        sp.I = c.d_ff;
        if (c.fmt == MOE_Q4B32) {
            QE_CHECK(cudaFuncSetAttribute(k_small_expert<MOE_Q4B32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)small_smem));
            k_small_expert<MOE_Q4B32><<<dev_sms, SE_W * 32, small_smem, st>>>(sp);
        } else if (c.fmt == MOE_Q2B32) {
            QE_CHECK(cudaFuncSetAttribute(k_small_expert<MOE_Q2B32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)small_smem));
            k_small_expert<MOE_Q2B32><<<dev_sms, SE_W * 32, small_smem, st>>>(sp);
        } else {
            QE_CHECK(cudaFuncSetAttribute(k_small_expert<MOE_Q3B32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)small_smem));
            k_small_expert<MOE_Q3B32><<<dev_sms, SE_W * 32, small_smem, st>>>(sp);
        }
        QE_CHECK_LAUNCH("k_small_expert");
    }
    QE_TRY(timing_end(ctx, st));
    k_finish<<<592, 256, 0, st>>>(ws.y_acc, Td, y, yf);
    QE_CHECK_LAUNCH("k_finish");
    return MOE_OK;
}

}  // namespace qeffn

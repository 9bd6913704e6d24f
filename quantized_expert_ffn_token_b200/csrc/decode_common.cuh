// Device helpers shared by the persistent decode kernels (decode.cu: one token
// per launch; decode_multi.cu: up to eight tokens per launch): launch shape,
// PTX wrappers (mbarriers, bulk copies, mma.sync), the exact code-to-operand
// conversions, and the bounded cross-CTA counter waits.
#pragma once
#include <math.h>

#include "moe_internal.cuh"

namespace qeffn {
namespace dec {

constexpr int NT = 384;             // compute threads (12 warps)
constexpr int NW = NT / 32;
constexpr int NTT = NT + 32;        // plus one producer warp: its lane 0 issues every bulk copy
constexpr int MAX_SLOTS = 8;
constexpr long long SPIN_LIMIT = 2000000000LL;   // clock64 cycles, about one second

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
__device__ __forceinline__ void mbar_arrive(unsigned long long *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
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
// L2 residency of the streamed weights.  Every layer streams the union of its experts once per
// call; the shared expert (and the router rows) recur in every call, the routed ones only when
// chosen again.  A copy can carry an L2 eviction priority: evict_last for the bytes worth keeping
// (the shared experts), evict_first for the rest, so that the stream does not push the kept
// bytes out of the 126 MB L2.
__device__ __forceinline__ uint64_t l2_policy(bool keep) {
    uint64_t pol;
    if (keep)
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    else
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes,
                                              unsigned long long *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
// A weight copy under the context's L2 mode: 0 plain, 1 shared experts kept and the rest streamed.
__device__ __forceinline__ void weight_copy(void *dst, const void *src, uint32_t bytes, unsigned long long *bar,
                                            int l2_mode, bool shared, uint64_t keep_pol, uint64_t stream_pol) {
    if (l2_mode == 0) bulk_g2s(dst, src, bytes, bar);
    else bulk_g2s_hint(dst, src, bytes, bar, shared ? keep_pol : stream_pol);
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mma16816(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816_h(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Q3B32 codes -> bf16 without arithmetic: a field OR-ed into the low mantissa
// bits of 128.0 (0x4300) reads as 128 + q, exactly.  The offset is removed in
// fp32 from each 32-block's partial sum: sum_k (128 + q_k) v_k - (128 + zero) *
// sum_k v_k = sum_k (q_k - zero) v_k, with the block sums of the activations
// precomputed once per layer (cancellation costs about 5 bits of the fp32
// partial, far below the output tolerance).
constexpr uint32_t BF_MAGIC = 0x43004300u;

// Q4B32 into fp16: a nibble at bits 0-3 of a half under 1024.0
// (0x6400) reads as 1024 + q, one at bits 4-7 as 1024 + 16 q, both exact.  In
// the fragment order registers a0/a2 (row g) take the first kind and a1/a3
// (row g+8) the second, so the row g+8 partial sums come out 16x larger and
// are scaled back in fp32; the offsets are 1024 + zero (row g) and
// 1024/16 + zero (row g+8).  Four ALU operations and one high multiply per
// eight codes.
constexpr uint32_t H_MAGIC = 0x64006400u;
__device__ __forceinline__ void q4_frag_h(uint32_t w, uint32_t &a0, uint32_t &a1, uint32_t &a2,
                                          uint32_t &a3) {
    const uint32_t w8 = __umulhi(w, 1u << 24);   // w >> 8 on the multiply pipe, off the integer ALU
    a0 = (w & 0x000F000Fu) | H_MAGIC;
    a1 = (w & 0x00F000F0u) | H_MAGIC;
    a2 = (w8 & 0x000F000Fu) | H_MAGIC;
    a3 = (w8 & 0x00F000F0u) | H_MAGIC;
}

// Q2B32: one lane's 8-byte piece = the 16 fragment registers of four k16 slices, each code
// OR-ed under fp16 1024 at its place: word w gives registers a0..a3 of slice w as 1024 + q
// (rows g) and 1024 + 4q (rows g+8), and those of slice w + 2 as 1024 + 16q and 1024 + 64q.
__device__ __forceinline__ void q2_frag_h(uint2 piece, uint32_t r[16]) {
    const uint32_t wv[2] = {piece.x, piece.y};
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const uint32_t x = wv[w], x8 = __umulhi(wv[w], 1u << 24);   // x >> 8 on the multiply pipe
        r[4 * w + 0] = (x & 0x00030003u) | H_MAGIC;
        r[4 * w + 1] = (x & 0x000C000Cu) | H_MAGIC;
        r[4 * w + 2] = (x8 & 0x00030003u) | H_MAGIC;
        r[4 * w + 3] = (x8 & 0x000C000Cu) | H_MAGIC;
        r[4 * w + 8] = (x & 0x00300030u) | H_MAGIC;
        r[4 * w + 9] = (x & 0x00C000C0u) | H_MAGIC;
        r[4 * w + 10] = (x8 & 0x00300030u) | H_MAGIC;
        r[4 * w + 11] = (x8 & 0x00C000C0u) | H_MAGIC;
    }
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

// B-fragment order of the h table (per expert, 256 * JN halves, JN = ceil(I/128)):
// lane (g, c) of the down MMAs reads, for k-group pair j, the 8 halves
// [sp][which][e] of slices 8j + 2 (g >> 1) + sp from row r = g & 1 (hi / lo),
// register which (b0: k 2c, 2c+1; b1: k 2c+8, 2c+9), element e; one 16-byte load.
// Pair-major: the 32 lanes' entries of one pair are contiguous (512 bytes).
// Index of the first half of (slice sl, lane column c, row r, register which).
__device__ __forceinline__ int hfrag_index(int sl, int c, int r, int which) {
    const int b4 = (sl >> 1) & 3, j = sl >> 3, sp = sl & 1;
    return ((j * 32 + (b4 * 4 + c) * 2 + r) * 2 + sp) * 4 + which * 2;
}
// x * mask for a packed pair of fp16 (Q4, Q2) or bf16 (Q3) values, mask 1.0 or 0 in both
// halves: zeroes the inactive block columns on the multiply pipe.
__device__ __forceinline__ uint32_t hmul2_mask(int fmt, uint32_t x, uint32_t mask) {
    uint32_t r;
    if (fmt != MOE_Q3B32)
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(mask));
    else
        asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(mask));
    return r;
}

// Sum of 32 consecutive fp16 values (16-byte aligned).
__device__ __forceinline__ float sum32_f16(const uint16_t *p) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 v = q[j];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[h]));
            acc[h] += f.x + f.y;
        }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// 2^e as a float, |e| <= 126.
__device__ __forceinline__ float pow2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// ---- cross-CTA counters ------------------------------------------------------
__device__ __forceinline__ void ctr_arrive(unsigned *c) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(c) : "memory");
}
__device__ __forceinline__ void ctr_zero(unsigned *c) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(c), "r"(0u) : "memory");
}
__device__ __forceinline__ unsigned ctr_load(const unsigned *c) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
    return v;
}
// Tagged words: a 32-bit value and a 32-bit tag in one naturally aligned 64-bit store, so a reader
// that sees the tag it expects also sees the value (single-copy atomicity of the 64-bit access) and
// no release fence or arrival counter has to order the two.
__device__ __forceinline__ void st_tagged(unsigned long long *p, float v, unsigned tag) {
    const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long ld_tagged(const unsigned long long *p) {
    unsigned long long w;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}
__device__ __forceinline__ ulonglong2 ld_tagged2(const unsigned long long *p) {   // two tagged words
    ulonglong2 w;
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(w.x), "=l"(w.y) : "l"(p) : "memory");
    return w;
}
// Reads N tagged words (addr(i) == nullptr: not read, counted as arrived) and re-reads the late
// ones together, round after round, until every word carries `want`.  Bounded: false on timeout
// (the error word is set) or once another CTA has reported an error.
template <int N, typename Addr>
__device__ __forceinline__ bool read_tagged(unsigned long long (&w)[N], Addr addr, unsigned want, int *err) {
    static_assert(N <= 32, "late-word mask");
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const unsigned long long *a = addr(i);
        w[i] = a ? ld_tagged(a) : ((unsigned long long)want << 32);
    }
    const long long t0 = clock64();
    for (int it = 0;; ++it) {
        unsigned late = 0u;
#pragma unroll
        for (int i = 0; i < N; ++i)
            if ((unsigned)(w[i] >> 32) != want) late |= 1u << i;
        if (!late) return true;
        if ((it & 15) == 15 && (*(volatile int *)err != 0 || clock64() - t0 > SPIN_LIMIT)) {
            atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
            return false;
        }
#pragma unroll
        for (int i = 0; i < N; ++i)
            if ((late >> i) & 1u) w[i] = ld_tagged(addr(i));
    }
}
__device__ __forceinline__ float ld_gpu(const float *p) {
    float v;
    asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_gpu4(const float *p) {
    float4 v;
    asm volatile("ld.relaxed.gpu.global.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}
// One thread: wait until the counter reaches n; false on timeout (error word
// set) or when another CTA reported an error.
__device__ __forceinline__ bool ctr_wait(const unsigned *c, unsigned n, int *err) {
    long long t0 = clock64();
    for (int it = 0;; ++it) {
        if ((int)(ctr_load(c) - n) >= 0) return true;
        if ((it & 7) == 7) {
            if (*(volatile int *)err != 0) return false;
            if (clock64() - t0 > SPIN_LIMIT) {
                atomicCAS(err, 0, MOE_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
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

// Barriers of the compute warps (named barrier 1, NT threads); the producer
// warp never joins them and synchronises through mbarriers only.
__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }
// CTA-uniform abort decision after a phase: one barrier that also ORs the
// compute threads' failures, so every one of them leaves at the same barrier.
__device__ __forceinline__ bool cta_failed(bool mine_ok) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"(mine_ok ? 0u : 1u), "n"(NT)
        : "memory");
    return r != 0;
}

}  // namespace dec
}  // namespace qeffn

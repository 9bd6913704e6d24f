// Canonical packed tensors -> the library's private row-tile layout
// (moe_internal.cuh).  Pure byte moves: no code or scale is changed.
#include <string.h>

#include "moe_internal.cuh"

namespace qeffn {

namespace {

// Canonical code j of block `blk` (Q4B32: nibble j%2 of byte j/2, low first;
// Q3B32: bits 3j..3j+2 of the 96-bit little-endian block; Q2B32: bits 2j..2j+1
// of the 64-bit little-endian block).
__device__ inline int canon_code(int fmt, const uint8_t *blk, int j) {
    if (fmt == MOE_Q4B32) return (blk[j >> 1] >> ((j & 1) * 4)) & 15;
    if (fmt == MOE_Q2B32) return (blk[j >> 2] >> (2 * (j & 3))) & 3;
    int v = 0;
    for (int t = 0; t < 3; ++t) {
        int bit = 3 * j + t;
        v |= ((blk[bit >> 3] >> (bit & 7)) & 1) << t;
    }
    return v;
}

struct RepackArgs {
    int fmt, n_experts, rows, K, gate_up;
    int chunk;                  // down matrix in chunk order (ChunkLayout) instead of row tiles
    ChunkLayout C;
    const uint8_t *codes, *codes_up;
    const uint16_t *scales, *scales_up;
    uint8_t *dst;
    MatLayout L;
};

// Source row of tile row r in tile t; sets *up when it comes from the up matrix.
__device__ inline int src_row(const RepackArgs &a, int t, int r, int *up) {
    if (a.gate_up) {
        *up = r >= 8;
        return 8 * t + (r & 7);
    }
    *up = 0;
    return 16 * t + r;
}

__device__ inline int fetch_code(const RepackArgs &a, int e, int t, int r, int k) {
    int up;
    int row;
    if (a.chunk) {
        // t = k chunk, and the "k group" index of the caller (k >> 6) = group of 64 rows; the
        // caller's k - 64 kg = 16 m + j names row tile m of the group and position j in the chunk
        const int kg = k >> 6, k64 = k & 63;
        row = 64 * kg + 16 * (k64 >> 4) + r;
        k = 16 * t + (k64 & 15);
        up = 0;
    } else {
        row = src_row(a, t, r, &up);
    }
    int B = a.fmt == MOE_Q4B32 ? 16 : (a.fmt == MOE_Q2B32) ? 8 : 12;
    size_t nb = a.K / 32;
    const uint8_t *base = up ? a.codes_up : a.codes;
    const uint8_t *blk = base + (((size_t)e * a.rows + row) * nb + (k >> 5)) * B;
    return canon_code(a.fmt, blk, k & 31);
}

// One thread per (expert, tile, k group, lane): writes that lane's piece.  In chunk order the
// "tile" is the k chunk and the "k group" the group of 64 output rows.
__global__ void k_repack_codes(RepackArgs a) {
    const size_t n_kg = a.chunk ? a.rows / 64 : a.K / 64;
    const int n_tiles = a.chunk ? a.K / 16 : a.L.n_tiles;
    size_t total = (size_t)a.n_experts * n_tiles * n_kg * 32;
    for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
         id += (size_t)gridDim.x * blockDim.x) {
        int lane = id & 31;
        size_t rest = id >> 5;
        int kg = rest % n_kg;
        rest /= n_kg;
        int t = rest % n_tiles;
        int e = rest / n_tiles;
        int g = lane >> 2, c = lane & 3;
        uint8_t *tile = a.chunk ? a.dst + (size_t)e * a.C.expert_bytes + (size_t)t * a.C.chunk_bytes
                                : a.dst + (size_t)e * a.L.expert_bytes + (size_t)t * a.L.tile_bytes;
        if (a.fmt == MOE_Q4B32) {
            uint32_t words[4];
            for (int m = 0; m < 4; ++m) {
                uint32_t wd = 0;
                for (int n = 0; n < 8; ++n) {
                    int reg = n & 3, hi = n >> 2;
                    int r = g + 8 * (reg & 1);
                    int k = 64 * kg + 16 * m + 8 * (reg >> 1) + 2 * c + hi;
                    wd |= (uint32_t)fetch_code(a, e, t, r, k) << (4 * n);
                }
                words[m] = wd;
            }
            uint4 v = make_uint4(words[0], words[1], words[2], words[3]);
            *reinterpret_cast<uint4 *>(tile + kg * 512 + lane * 16) = v;
        } else if (a.fmt == MOE_Q2B32) {
            // word w, field f, half hi: slice w + 2*((f >> 1) & 1), register (f & 1) + 2*(f >> 2)
            uint32_t words[2] = {0, 0};
            for (int w = 0; w < 2; ++w)
                for (int f = 0; f < 8; ++f) {
                    int m = w + 2 * ((f >> 1) & 1), reg = (f & 1) + 2 * (f >> 2);
                    int r = g + 8 * (reg & 1);
                    for (int hi = 0; hi < 2; ++hi) {
                        int k = 64 * kg + 16 * m + 8 * (reg >> 1) + 2 * c + hi;
                        words[w] |= (uint32_t)fetch_code(a, e, t, r, k) << (16 * hi + 2 * f);
                    }
                }
            *reinterpret_cast<uint2 *>(tile + kg * 256 + lane * 8) = make_uint2(words[0], words[1]);
        } else {
            uint32_t w3[3] = {0, 0, 0};
            for (int q = 0; q < 16; ++q) {
                int m = q >> 2, reg = q & 3;
                int r = g + 8 * (reg & 1);
                for (int hi = 0; hi < 2; ++hi) {
                    int k = 64 * kg + 16 * m + 8 * (reg >> 1) + 2 * c + hi;
                    uint32_t code = fetch_code(a, e, t, r, k);
                    if (q < 15) {
                        w3[q / 5] |= code << (3 * (q % 5) + 16 * hi);
                    } else {
                        for (int b = 0; b < 3; ++b) w3[b] |= ((code >> b) & 1u) << (15 + 16 * hi);
                    }
                }
            }
            uint32_t *dst = reinterpret_cast<uint32_t *>(tile + kg * 384 + lane * 12);
            dst[0] = w3[0];
            dst[1] = w3[1];
            dst[2] = w3[2];
        }
    }
}

// Scales of the down matrix in chunk order: [I/32 blocks][d rows] after the expert's codes.
__global__ void k_repack_scales_chunks(RepackArgs a) {
    const int nb = a.K / 32;
    const size_t total = (size_t)a.n_experts * a.rows * nb;
    for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
         id += (size_t)gridDim.x * blockDim.x) {
        const int row = id % a.rows;
        const size_t rest = id / a.rows;
        const int blk = rest % nb;
        const int e = rest / nb;
        const uint16_t v = a.scales[((size_t)e * a.rows + row) * nb + blk];
        uint8_t *ex = a.dst + (size_t)e * a.C.expert_bytes + a.C.code_bytes;
        reinterpret_cast<uint16_t *>(ex)[(size_t)blk * a.rows + row] = v;
    }
}

__global__ void k_repack_scales(RepackArgs a) {
    int nb = a.K / 32;
    size_t total = (size_t)a.n_experts * a.L.n_tiles * 16 * nb;
    for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
         id += (size_t)gridDim.x * blockDim.x) {
        int blk = id % nb;
        size_t rest = id / nb;
        int r = rest % 16;
        rest /= 16;
        int t = rest % a.L.n_tiles;
        int e = rest / a.L.n_tiles;
        int up;
        int row = src_row(a, t, r, &up);
        const uint16_t *src = up ? a.scales_up : a.scales;
        uint16_t v = src[((size_t)e * a.rows + row) * nb + blk];
        uint8_t *tile = a.dst + (size_t)e * a.L.expert_bytes + (size_t)t * a.L.tile_bytes;
        reinterpret_cast<uint16_t *>(tile + a.L.code_bytes)[r * nb + blk] = v;
    }
}

}  // namespace

int launch_repack(moe_ctx *ctx, int fmt, const uint8_t *codes, const uint16_t *scales,
                  const uint8_t *codes_up, const uint16_t *scales_up, int n_experts,
                  int rows, int K, bool gate_up, uint8_t *dst, cudaStream_t st) {
    RepackArgs a;
    a.fmt = fmt;
    a.n_experts = n_experts;
    a.rows = rows;
    a.K = K;
    a.gate_up = gate_up;
    a.codes = codes;
    a.codes_up = codes_up;
    a.scales = scales;
    a.scales_up = scales_up;
    a.dst = dst;
    a.L = gate_up ? ctx->gu : ctx->dn;
    a.chunk = 0;
    k_repack_codes<<<1184, 256, 0, st>>>(a);
    QE_CHECK_LAUNCH("k_repack_codes");
    k_repack_scales<<<1184, 256, 0, st>>>(a);
    QE_CHECK_LAUNCH("k_repack_scales");
    return MOE_OK;
}

int launch_repack_chunks(moe_ctx *ctx, int fmt, const uint8_t *codes, const uint16_t *scales, int n_experts,
                         uint8_t *dst, cudaStream_t st) {
    const moe_config &c = ctx->cfg;
    RepackArgs a;
    memset(&a, 0, sizeof(a));
    a.fmt = fmt;
    a.n_experts = n_experts;
    a.rows = c.d_model;
    a.K = c.d_ff;
    a.gate_up = 0;
    a.codes = codes;
    a.scales = scales;
    a.dst = dst;
    a.L = ctx->dn;
    a.chunk = 1;
    a.C = ctx->chunk;
    k_repack_codes<<<1184, 256, 0, st>>>(a);
    QE_CHECK_LAUNCH("k_repack_codes");
    k_repack_scales_chunks<<<1184, 256, 0, st>>>(a);
    QE_CHECK_LAUNCH("k_repack_scales_chunks");
    return MOE_OK;
}

}  // namespace qeffn

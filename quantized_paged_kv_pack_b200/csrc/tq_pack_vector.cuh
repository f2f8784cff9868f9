// Per-vector quantize-and-pack of one K or V vector by one warp (the general
// path, every format): shared by the pack kernels and the decode prologue's
// fused window append. Device code only; each translation unit that includes
// it gets its own copy.
//
// TurboQuant "Design" page, "Serving Route Design": the serving route writes
// packed rows into persistent pages addressed slot -> physical block -> token
// offset -> row bytes. Per (token, head) vector x (bf16, 128 values):
//   n   = ||x||_2, stored as fp16 (round to nearest even)
//   z   = H (s * x)              Sylvester Walsh-Hadamard, signs s of the codec
//   u   = z / (sqrt(128) n)      the rotated unit vector
//   idx = #{boundaries of its group below u_j}, placed at packed position pos[h][j]
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr unsigned kPvFull = 0xffffffffu;

__device__ __forceinline__ float pv_warp_sum(float v) {
#pragma unroll
    for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(kPvFull, v, m);
    return v;
}

__device__ __forceinline__ double pv_warp_sum_d(double v) {
#pragma unroll
    for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(kPvFull, v, m);
    return v;
}

// fp16 bits of the norm, equal to the correctly rounded fp16 of the exact norm.
// The fp32 sum of exact squares is within 5e-7 (relative) of the exact sum, so
// its square root decides the rounding unless it lies within 1e-6 of an fp16
// rounding midpoint, or the fp32 sum under- or overflows; then the warp
// recomputes the sum in fp64 and `n32` is replaced by that norm.
__device__ __forceinline__ unsigned short norm_fp16_bits(const float (&x)[4], float ss, float& n32) {
    bool risky = !(ss > 1e-30f && ss < 1e30f) || n32 > 60000.0f;
    __half h = __float2half_rn(n32);
    unsigned short hb = __half_as_ushort(h);
    if (!risky) {
        float hf = __half2float(h);
        float up = __half2float(__ushort_as_half(static_cast<unsigned short>(hb + 1)));
        float dn = __half2float(__ushort_as_half(static_cast<unsigned short>(hb - 1)));
        float tol = 1e-6f * n32;
        risky = fabsf(n32 - 0.5f * (hf + up)) <= tol || fabsf(n32 - 0.5f * (hf + dn)) <= tol;
    }
    if (risky) {  // warp-uniform: ss and n32 are warp-wide values
        double sd = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) sd += static_cast<double>(x[i]) * static_cast<double>(x[i]);
        sd = pv_warp_sum_d(sd);
        const double nd = sqrt(sd);
        hb = __half_as_ushort(__double2half(nd));
        n32 = static_cast<float>(nd);
    }
    return hb;
}

// Boundaries of a group's codebook below u (the index): the 15 loads are issued
// together instead of one per loop trip (a lone vector is bound by this latency).
__device__ __forceinline__ int pv_boundary_count(const float* bound, int levels, float u) {
    int idx = 0;
#pragma unroll
    for (int q = 0; q < 15; ++q)
        if (q < levels - 1) idx += (__ldg(bound + q) < u) ? 1 : 0;
    return idx;
}

// (lb / b, lb % b) for a bit width b of 2, 3 or 4 and 0 <= lb < 2^16, without a division.
__device__ __forceinline__ void pv_divmod(int lb, int b, int& q, int& r) {
    q = b == 4 ? lb >> 2 : (b == 2 ? lb >> 1 : static_cast<int>((static_cast<unsigned>(lb) * 0xAAABu) >> 17));
    r = lb - q * b;
}

// One warp quantizes the vector x (lane l holds elements 4l .. 4l+3) of KV
// head h and writes its row at `offset` of the sub-page `sub` (block_size
// rows). idx_buf: 128 bytes, r_buf: 128 floats of shared scratch owned by the
// warp (r_buf is used by the QJL stage only).
__device__ void pack_vector_groupwise(const DevCodec& c, const float (&x)[4], int h, uint8_t* sub, int64_t offset,
                                      int block_size, uint8_t* idx_buf, float* x_buf, int lane);

__device__ void pack_vector(const DevCodec& c, const float (&x)[4], int h, uint8_t* sub, int64_t offset,
                            int block_size, uint8_t* idx_buf, float* r_buf, int lane) {
    if (c.groupwise) {
        pack_vector_groupwise(c, x, h, sub, offset, block_size, idx_buf, r_buf, lane);
        return;
    }
    float ss = pv_warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    float n32 = sqrtf(ss);
    const unsigned short n16 = norm_fp16_bits(x, ss, n32);

    float z[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) z[i] = x[i] * c.sign[4 * lane + i];
    {
        float a = z[0] + z[1], b = z[0] - z[1], cc = z[2] + z[3], d = z[2] - z[3];
        z[0] = a + cc;
        z[2] = a - cc;
        z[1] = b + d;
        z[3] = b - d;
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float p = __shfl_xor_sync(kPvFull, z[i], m);
            z[i] = (lane & m) ? (p - z[i]) : (z[i] + p);
        }
    }
    const float inv = n32 > 0.0f ? 1.0f / (n32 * 11.313708498984761f) : 0.0f;
    float rr = 0.0f;  // QJL: sum of squared residuals of this lane's coordinates
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * lane + i;
        const int p = c.pos[h * kHeadDim + j];
        const int g = (c.n_groups == 2 && p >= c.pos0[1]) ? 1 : 0;
        const float u = z[i] * inv;
        const int levels = 1 << c.bits[g];
        const int idx = pv_boundary_count(c.bound + g * 16, levels, u);
        idx_buf[p] = static_cast<uint8_t>(idx);
        if (c.qjl) {
            const float r = u - c.cent[g * 16 + idx];  // residual, rotated coordinate j
            r_buf[j] = r;
            rr += r * r;
        }
    }
    __syncwarp();
    // QJL stage: (S r)_i for i = lane + 32k from S^T rows (coalesced), sign bits by ballot.
    uint32_t sign_word[4] = {0u, 0u, 0u, 0u};
    unsigned short g16 = 0;
    if (c.qjl) {
        g16 = __half_as_ushort(__float2half_rn(sqrtf(pv_warp_sum(rr))));
        float proj[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        // rows of S^T in batches of 8, their loads issued together (same accumulation order)
        for (int j0 = 0; j0 < kHeadDim; j0 += 8) {
            float sv[8][4];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                for (int k = 0; k < 4; ++k) sv[jj][k] = __ldg(c.qjl_st + (j0 + jj) * kHeadDim + lane + 32 * k);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const float r = r_buf[j0 + jj];
#pragma unroll
                for (int k = 0; k < 4; ++k) proj[k] = fmaf(sv[jj][k], r, proj[k]);
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) sign_word[k] = __ballot_sync(kPvFull, proj[k] >= 0.0f);
    }
    const int half_words = c.mse_bytes / 2;
    unsigned word = 0;
    if (lane < half_words) {
        for (int i = 0; i < 16; ++i) {
            const int B = 16 * lane + i;
            const int g = (c.n_groups == 2 && B >= 8 * c.byte_off[1]) ? 1 : 0;
            const int lb = B - 8 * c.byte_off[g];
            const int b = c.bits[g];
            int q, r;
            pv_divmod(lb, b, q, r);
            word |= ((idx_buf[c.pos0[g] + q] >> r) & 1u) << i;
        }
    }
    uint16_t* dst = reinterpret_cast<uint16_t*>(sub + offset * c.index_bytes);
    if (lane < half_words) dst[lane] = static_cast<uint16_t>(word);
    uint16_t* nrm = reinterpret_cast<uint16_t*>(sub + block_size * c.index_bytes + c.norm_bytes * offset);
    if (c.qjl) {
        // sign bits after the index bitstreams, LSB-first: half-word m holds bits 16m .. 16m+15
        if (lane < kHeadDim / 16) dst[half_words + lane] = static_cast<uint16_t>(sign_word[lane >> 1] >> (16 * (lane & 1)));
        if (lane == 0) nrm[1] = g16;
    }
    if (lane == 0) nrm[0] = n16;
    __syncwarp();
}

// The recipe row (group-wise rotation with a QJL stage per group), after the
// indices: per group the fp16 residual norm |r_g|, the n_g sign bits
// [(S_g r_g)_i >= 0] (S_g^T rows from the codec, coalesced), then the index
// part [g0 indices][g0 signs][g1 indices][g1 signs] and the norm part
// (n_0, |r_0|, n_1, |r_1|). Lane l holds packed positions l + 32k.
__device__ void pack_recipe_tail(const DevCodec& c, const float (&res)[4], const unsigned short (&n16)[2],
                                 uint8_t* sub, int64_t offset, int block_size, const uint8_t* idx_buf,
                                 float* r_buf, int lane) {
    const int n0 = c.pos0[1];
#pragma unroll
    for (int k = 0; k < 4; ++k) r_buf[lane + 32 * k] = res[k];  // packed order (x_buf is no longer read)
    unsigned short g16[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        float rr = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int p = lane + 32 * k;
            if ((p >= n0) == (g == 1)) rr += res[k] * res[k];
        }
        g16[g] = __half_as_ushort(__float2half_rn(sqrtf(pv_warp_sum(rr))));
    }
    __syncwarp();
    // (S_g r_g)_i for position p = pos0[g] + i
    float proj[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int g = 0; g < 2; ++g) {
        const int n = c.size[g], p0 = c.pos0[g];
        const float* st = c.qjl_st + (g ? static_cast<int64_t>(n0) * n0 : 0);
        // rows of S_g^T in batches of 8 (group sizes are multiples of 8), loads issued together
        for (int j0 = 0; j0 < n; j0 += 8) {
            float sv[8][4];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = lane + 32 * k - p0;
                    sv[jj][k] = (i >= 0 && i < n) ? __ldg(st + (j0 + jj) * n + i) : 0.0f;
                }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const float r = r_buf[p0 + j0 + jj];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = lane + 32 * k - p0;
                    if (i >= 0 && i < n) proj[k] = fmaf(sv[jj][k], r, proj[k]);
                }
            }
        }
    }
    uint32_t sw[4];  // sign bit of packed position p at bit p % 32 of sw[p / 32]
#pragma unroll
    for (int k = 0; k < 4; ++k) sw[k] = __ballot_sync(kPvFull, proj[k] >= 0.0f);
    // index part, 16 bits per lane and round
    const int half_words = c.index_bytes / 2;
    uint16_t* dst = reinterpret_cast<uint16_t*>(sub + offset * c.index_bytes);
    for (int hw = lane; hw < half_words; hw += 32) {
        unsigned word = 0;
        for (int i = 0; i < 16; ++i) {
            const int B = 16 * hw + i;
            unsigned bit;
            if (B < 8 * c.sign_off[0]) {  // group 0 indices
                int q, r;
                pv_divmod(B, c.bits[0], q, r);
                bit = (idx_buf[q] >> r) & 1u;
            } else if (B < 8 * c.byte_off[1]) {  // group 0 signs
                const int p = B - 8 * c.sign_off[0];
                bit = (sw[p >> 5] >> (p & 31)) & 1u;
            } else if (B < 8 * c.sign_off[1]) {  // group 1 indices
                const int lb = B - 8 * c.byte_off[1];
                int q, r;
                pv_divmod(lb, c.bits[1], q, r);
                bit = (idx_buf[n0 + q] >> r) & 1u;
            } else {  // group 1 signs
                const int p = n0 + B - 8 * c.sign_off[1];
                bit = (sw[p >> 5] >> (p & 31)) & 1u;
            }
            word |= bit << i;
        }
        dst[hw] = static_cast<uint16_t>(word);
    }
    uint16_t* nrm = reinterpret_cast<uint16_t*>(sub + block_size * c.index_bytes + c.norm_bytes * offset);
    if (lane == 0) {
        nrm[0] = n16[0];
        nrm[1] = g16[0];
        nrm[2] = n16[1];
        nrm[3] = g16[1];
    }
    __syncwarp();
}

// Group-wise rotation (two groups of original channels, each rotated on its
// own by the per-head matrix R_h, rows = packed positions): y = R_h x, one fp16
// norm per group from the exact squares of its channels, u_p = y_p / n_g(p).
// Lane l handles packed positions l, l+32, l+64, l+96.
__device__ void pack_vector_groupwise(const DevCodec& c, const float (&x)[4], int h, uint8_t* sub, int64_t offset,
                                      int block_size, uint8_t* idx_buf, float* x_buf, int lane) {
    const int n0 = c.pos0[1];  // group 0 occupies packed positions [0, n0)
    float xm[2][4];            // the lane's channels, masked to each group
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * lane + i;
        x_buf[j] = x[i];
        const bool in0 = c.pos[h * kHeadDim + j] < n0;
        xm[0][i] = in0 ? x[i] : 0.0f;
        xm[1][i] = in0 ? 0.0f : x[i];
    }
    unsigned short n16[2];
    float n32[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const float ss = pv_warp_sum(xm[g][0] * xm[g][0] + xm[g][1] * xm[g][1] + xm[g][2] * xm[g][2] + xm[g][3] * xm[g][3]);
        n32[g] = sqrtf(ss);
        n16[g] = norm_fp16_bits(xm[g], ss, n32[g]);
    }
    __syncwarp();
    float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const float* rt = c.rot_t + static_cast<int64_t>(h) * kHeadDim * kHeadDim + lane;
    // rows of R_h^T in batches of 8, their loads issued together (same accumulation order)
    for (int j0 = 0; j0 < kHeadDim; j0 += 8) {
        float rv[8][4];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
#pragma unroll
            for (int k = 0; k < 4; ++k) rv[jj][k] = __ldg(rt + (j0 + jj) * kHeadDim + 32 * k);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const float xj = x_buf[j0 + jj];
#pragma unroll
            for (int k = 0; k < 4; ++k) y[k] = fmaf(rv[jj][k], xj, y[k]);
        }
    }
    float res[4];  // recipe row: residuals u - c[idx] of the lane's positions
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int p = lane + 32 * k;
        const int g = p >= n0 ? 1 : 0;
        const float u = n32[g] > 0.0f ? y[k] / n32[g] : 0.0f;
        const int levels = 1 << c.bits[g];
        const int idx = pv_boundary_count(c.bound + g * 16, levels, u);
        idx_buf[p] = static_cast<uint8_t>(idx);
        res[k] = u - c.cent[g * 16 + idx];
    }
    __syncwarp();
    if (c.recipe) {
        pack_recipe_tail(c, res, n16, sub, offset, block_size, idx_buf, x_buf, lane);
        return;
    }
    const int half_words = c.mse_bytes / 2;
    unsigned word = 0;
    if (lane < half_words) {
        for (int i = 0; i < 16; ++i) {
            const int B = 16 * lane + i;
            const int g = B >= 8 * c.byte_off[1] ? 1 : 0;
            const int lb = B - 8 * c.byte_off[g];
            const int b = c.bits[g];
            int q, r;
            pv_divmod(lb, b, q, r);
            word |= ((idx_buf[c.pos0[g] + q] >> r) & 1u) << i;
        }
    }
    uint16_t* dst = reinterpret_cast<uint16_t*>(sub + offset * c.index_bytes);
    if (lane < half_words) dst[lane] = static_cast<uint16_t>(word);
    uint16_t* nrm = reinterpret_cast<uint16_t*>(sub + block_size * c.index_bytes + c.norm_bytes * offset);
    if (lane == 0) {
        nrm[0] = n16[0];
        nrm[1] = n16[1];
    }
    __syncwarp();
}

__device__ __forceinline__ void pv_load_bf16x4(const __nv_bfloat16* src, float (&x)[4]) {
    const uint2 raw = *reinterpret_cast<const uint2*>(src);
    x[0] = __uint_as_float(raw.x << 16);
    x[1] = __uint_as_float(raw.x & 0xffff0000u);
    x[2] = __uint_as_float(raw.y << 16);
    x[3] = __uint_as_float(raw.y & 0xffff0000u);
}

// Window eviction with append, one vector: vec = 2 (b H + h) + (0: K, 1: V).
// With L = seq_lens[b] tokens before the append, the dense buffer holds the
// first min(S, L) tokens in slots 0 .. S-1 and the recent ones in a ring:
// token t >= S in slot S + (t - S) % W. The new token L takes slot L (L < S)
// or its ring slot; when the ring is full, the token it replaces, L - W, is
// packed first, at packed position L - S - W of the sequence's block table.
// With W = 0 the new token itself is packed (at position L - S). idx_buf and
// r_buf: the warp's shared scratch (128 bytes, 128 floats).
__device__ __forceinline__ void append_vector(const DevCodec& kc, const DevCodec& vc, int64_t vec,
                                              const __nv_bfloat16* __restrict__ k_new,
                                              const __nv_bfloat16* __restrict__ v_new, __nv_bfloat16* k_win,
                                              __nv_bfloat16* v_win, int window, int sinks,
                                              const int32_t* __restrict__ seq_lens,
                                              const int32_t* __restrict__ block_tables, int max_blocks,
                                              uint8_t* k_pages, uint8_t* v_pages, int64_t num_blocks, int block_size,
                                              int* d_err, uint8_t* idx_buf, float* r_buf, int lane) {
    const int H = kc.num_heads;
    const int dense = sinks + window;  // slots per (sequence, head) in the dense buffer
    const int which = static_cast<int>(vec & 1);
    const int64_t bh = vec >> 1;
    const int b = static_cast<int>(bh / H), h = static_cast<int>(bh - static_cast<int64_t>(b) * H);
    const DevCodec& c = which ? vc : kc;
    const int L = max(__ldg(seq_lens + b), 0);
    const __nv_bfloat16* src_new = (which ? v_new : k_new) + bh * kHeadDim + 4 * lane;
    __nv_bfloat16* wbuf = (which ? v_win : k_win) + bh * static_cast<int64_t>(dense) * kHeadDim;
    int slot_w = -1;      // dense slot the new token goes to (-1: none)
    int64_t packed = -1;  // packed position of the vector to pack (-1: none)
    bool pack_new = false;
    if (L < sinks) {
        slot_w = L;
    } else if (window == 0) {
        packed = L - sinks;
        pack_new = true;
    } else {
        const int r = L - sinks;
        slot_w = sinks + r % window;
        if (r >= window) packed = r - window;
    }
    if (packed >= 0) {
        const int64_t bi = packed / block_size, off = packed - bi * block_size;
        const int blk = bi < max_blocks ? __ldg(block_tables + static_cast<int64_t>(b) * max_blocks + bi) : -1;
        if (blk < 0 || blk >= num_blocks) {
            if (lane == 0 && d_err) atomicOr(d_err, TQ_DERR_BLOCK);
        } else {
            float x[4];
            pv_load_bf16x4(pack_new ? src_new : wbuf + static_cast<int64_t>(slot_w) * kHeadDim + 4 * lane, x);
            uint8_t* sub = (which ? v_pages : k_pages) + (static_cast<int64_t>(blk) * H + h) * block_size * c.row_bytes;
            pack_vector(c, x, h, sub, off, block_size, idx_buf, r_buf, lane);  // x read before the slot is reused
        }
    }
    if (slot_w >= 0)
        *reinterpret_cast<uint2*>(wbuf + static_cast<int64_t>(slot_w) * kHeadDim + 4 * lane) =
            *reinterpret_cast<const uint2*>(src_new);
}

}  // namespace
}  // namespace tq

// Fast pack path for uniform 4-bit codecs (sm_100a).
//
// Same computation as the general pack kernel (TurboQuant "Design" page,
// "Serving Route Design": packed rows are written into persistent pages at
// slot / block_size, slot % block_size), organised per warp over 16
// consecutive tokens of one KV head, keys or values:
//
//  * Rotation. With the coordinate index j = 16a + b, the natural-order
//    Sylvester matrix factors as H_128 = H_8 (x) H_16, so
//    z[16a' + b'] = sum_a H8[a'][a] sum_b H16[b'][b] s[16a + b] x[16a + b].
//    The inner sum runs on mma.sync m16n8k16 (bf16 inputs are exact, the
//    signs are folded into the +-1 B operand of each a, fp32 accumulation);
//    the outer H_8 is three packed-fp32 butterfly stages in registers.
//  * Norm. Sum of exact squares of the bf16 inputs in fp32; when the fp32
//    norm lies within 1e-6 of an fp16 rounding midpoint (or the sum under-
//    or overflows) the warp recomputes it in fp64, so the stored fp16 norm is
//    the correctly rounded norm.
//  * Quantizer. v = 64 u (u = z / (sqrt(128) n)) is rounded to a cell of
//    width 1 with the magic-number trick; a per-lane replicated table gives,
//    per cell, the number of boundaries below it and the boundary inside it
//    (cells are narrower than the closest boundary gap), so
//    idx = below + (v > boundary) with one compare.
//  * Rows are staged in shared memory and written with 16-byte stores; norms
//    go to the sub-page's norm array.
//  * Loads. Each warp copies its next unit's 16 input rows into a shared
//    buffer with cp.async while it computes the current one (double
//    buffering); ldmatrix reads the MMA A fragments from rows padded to 272
//    bytes, free of bank conflicts.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kPW = 16;              // warps per CTA (one CTA per SM)
constexpr int kRowPad = 272;         // bytes per staged input row (256 + 16: 8 rows hit 8 bank quads)
constexpr int kCells = kPackCells;   // v = 64 u in [-64, 64], cells round(v) + 64
constexpr float kCellScale = kPackCellScale;
using QuantCell = PackCell;          // one table entry (8 bytes), built with the codec

struct PackSmem {
    QuantCell cells[kCells][32];     // replicated per lane: conflict-free 8-byte lookups
    uint32_t bfrag[2][8][2][32][2];  // [K/V][a][n-tile][lane][reg]: B operands (+-1 bf16 pairs)
    uint8_t rows[kPW][16][64];       // staged index rows of a warp's 16 tokens
    unsigned short norms[kPW][16];
    uint8_t xbuf[kPW][2][16][kRowPad];  // double-buffered input rows (bf16) of a warp's units
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// d += a b (accumulating form).
__device__ __forceinline__ void mma_bf16_acc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Packed fp32 helpers on pairs held in one 64-bit register.
__device__ __forceinline__ uint64_t pk(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
// The two bf16 of a word as an fp32 pair (exact).
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
    return pk(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

template <int B, int E, class F>
__device__ __forceinline__ void static_for(F&& f) {
    if constexpr (B < E) {
        f(std::integral_constant<int, B>{});
        static_for<B + 1, E>(f);
    }
}

template <int I = 0, class F>
__device__ __forceinline__ void static_for8(F&& f) {
    if constexpr (I < 8) {
        f(std::integral_constant<int, I>{});
        static_for8<I + 1>(f);
    }
}

// Byte store to shared address base + OFF (OFF a compile-time offset).
template <int OFF>
__device__ __forceinline__ void sts8(uint32_t base, uint32_t v) {
    asm volatile("st.shared.u8 [%0+%1], %2;" ::"r"(base), "n"(OFF), "r"(v) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& d0, uint32_t& d1, uint32_t& d2, uint32_t& d3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
                 : "r"(addr));
}

__device__ __forceinline__ double warp4_sum_d(double v) {
    v += __shfl_xor_sync(kFull, v, 1);
    v += __shfl_xor_sync(kFull, v, 2);
    return v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__global__ void __launch_bounds__(kPW * 32, 1) pack_u4_kernel(DevCodec kc, DevCodec vc, const QuantCell* __restrict__ g_cells,
                                                          const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          const int64_t* __restrict__ slots, int num_tokens,
                                                          uint8_t* __restrict__ k_pages, uint8_t* __restrict__ v_pages,
                                                          int capacity, int block_size, int bs_log2,
                                                          int* __restrict__ d_err) {
    extern __shared__ __align__(16) uint8_t psm_raw[];
    PackSmem& sm = *reinterpret_cast<PackSmem*>(psm_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;

    // Cell table and the B operands D_s H_16 of both codecs.
    for (int i = threadIdx.x; i < kCells * 32; i += kPW * 32) sm.cells[i >> 5][i & 31] = g_cells[i >> 5];
    for (int i = threadIdx.x; i < 2 * 8 * 2 * 32; i += kPW * 32) {
        const int ln = i & 31, t = (i >> 5) & 1, a = (i >> 6) & 7, which = i >> 9;
        const float* sign = which ? vc.sign : kc.sign;
        const int rr = ln >> 2, cc = ln & 3;
        const int bp = 8 * t + rr;  // output column b' of lane rr in n-tile t
        uint32_t regs[2];
        for (int q = 0; q < 2; ++q) {
            unsigned short h[2];
            for (int e = 0; e < 2; ++e) {
                const int b = 2 * cc + 8 * q + e;          // input coordinate b of this k-slot
                const float val = sign[16 * a + b] * ((__popc(bp & b) & 1) ? -1.0f : 1.0f);
                h[e] = val > 0 ? 0x3F80 : 0xBF80;
            }
            regs[q] = static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16);
        }
        sm.bfrag[which][a][t][ln][0] = regs[0];
        sm.bfrag[which][a][t][ln][1] = regs[1];
    }
    __syncthreads();

    // 32-bit index arithmetic throughout: the host checks that tokens, units and
    // slots fit (a 64-bit division is a long software routine on the GPU).
    const int H = kc.num_heads;
    const int units = (num_tokens + 15) / 16 * H * 2;
    const uint32_t cell_lane = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.cells[0][lane]));
    // address of cell e for this lane = cell_lane + e * 256; e = bits(v + 1.5*2^23) - 0x4B400000 + 64
    const uint32_t cell_adj = cell_lane + 64u * 256u - 0x40000000u;

    // Unit u = (16-token group, KV head, K or V). The warp's 16 input rows of a
    // unit are 16 x 256 contiguous bytes at a stride of H x 256: lane l copies
    // 16-byte pieces l, l + 32, ... (token = piece / 16); rows past the end are
    // zero-filled without reading.
    const uint32_t xbuf0 = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.xbuf[warp][0][0][0]));
    auto issue = [&](int uu, int buf) {
        const int which_ = uu & 1, gh_ = uu >> 1;
        const int tg_ = gh_ / H, h_ = gh_ - tg_ * H;
        const __nv_bfloat16* src_ = which_ ? v : k;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int piece = lane + 32 * i, tok = piece >> 4, part = piece & 15;
            const int t = tg_ * 16 + tok;
            const bool live = t < num_tokens;
            // A row past the end is zero-filled (no bytes read; the address stays in the tensor).
            const __nv_bfloat16* g = src_ + (static_cast<int64_t>(live ? t : 0) * H + h_) * kHeadDim + 8 * part;
            cp_async16(xbuf0 + (buf * 16 + tok) * kRowPad + 16 * part, g, live ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const int stride = gridDim.x * kPW;
    int u = blockIdx.x * kPW + warp;
    if (u < units) issue(u, 0);
    for (int it = 0; u < units; u += stride, ++it) {
        const int cur = it & 1;
        const int which = u & 1;
        const int gh = u >> 1;
        const int tg = gh / H, h = gh - tg * H;
        const int t0 = tg * 16;

        // Slots of the 16 tokens (lane i < 16 holds token t0 + i).
        int64_t my_slot = -1;
        if (lane < 16 && t0 + lane < num_tokens) my_slot = __ldg(slots + t0 + lane);

        // The next unit's rows go to the other buffer while this one is computed.
        if (u + stride < units) {
            issue(u + stride, cur ^ 1);
        } else {
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncwarp();

        // A operands of group a (ldmatrix.x4, once per half below to keep registers
        // low): xa[a] = token r, coordinates 16a + 2c + {0,1} and 16a + 2c + 8 + {0,1};
        // xb[a] the same for token r + 8. Lane l addresses row l % 8 of matrix l / 8.
        const uint32_t frag_row = xbuf0 + (cur * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * kRowPad +
                                  ((lane >> 4) & 1) * 16;
        float n_tok[2];
        unsigned short n16[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            uint2 xa[8], xb[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) ldsm_x4(frag_row + 32 * a, xa[a].x, xb[a].x, xa[a].y, xb[a].y);
            if (t == 0) {
                // Sum of exact squares (fp32), per token, over this lane's 32 coordinates
                // (two interleaved partial sums in a packed pair) then the 4 lanes.
                float ss_lo, ss_hi;
                {
                    uint64_t acc_lo = 0, acc_hi = 0;
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        const uint64_t l01 = bf16x2_to_f32x2(xa[a].x), l23 = bf16x2_to_f32x2(xa[a].y);
                        const uint64_t h01 = bf16x2_to_f32x2(xb[a].x), h23 = bf16x2_to_f32x2(xb[a].y);
                        acc_lo = fma2(l01, l01, fma2(l23, l23, acc_lo));
                        acc_hi = fma2(h01, h01, fma2(h23, h23, acc_hi));
                    }
                    float p, q;
                    upk(acc_lo, p, q);
                    ss_lo = p + q;
                    upk(acc_hi, p, q);
                    ss_hi = p + q;
                }
                ss_lo += __shfl_xor_sync(kFull, ss_lo, 1);
                ss_lo += __shfl_xor_sync(kFull, ss_lo, 2);
                ss_hi += __shfl_xor_sync(kFull, ss_hi, 1);
                ss_hi += __shfl_xor_sync(kFull, ss_hi, 2);

                // fp16 norm, correctly rounded; fp64 when the fp32 value is too close to call.
                bool risky[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float ss = i ? ss_hi : ss_lo;
                    const float n32 = sqrtf(ss);
                    bool rk = !(ss > 1e-30f && ss < 1e30f) || n32 > 60000.0f;
                    const __half hh = __float2half_rn(n32);
                    const unsigned short hb = __half_as_ushort(hh);
                    if (!rk) {
                        const float hf = __half2float(hh);
                        const float up = __half2float(__ushort_as_half(static_cast<unsigned short>(hb + 1)));
                        const float dn = __half2float(__ushort_as_half(static_cast<unsigned short>(hb - 1)));
                        const float tol = 1e-6f * n32;
                        rk = fabsf(n32 - 0.5f * (hf + up)) <= tol || fabsf(n32 - 0.5f * (hf + dn)) <= tol;
                    }
                    risky[i] = rk;
                    n_tok[i] = n32;
                    n16[i] = hb;
                }
                if (__any_sync(kFull, risky[0] || risky[1])) {
                    // Rare: exact-enough fp64 sums for the tokens that need them (all lanes join the shuffles).
                    double d_lo = 0.0, d_hi = 0.0;
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        const double l0 = __uint_as_float(xa[a].x << 16), l1 = __uint_as_float(xa[a].x & 0xffff0000u);
                        const double l2 = __uint_as_float(xa[a].y << 16), l3 = __uint_as_float(xa[a].y & 0xffff0000u);
                        const double h0 = __uint_as_float(xb[a].x << 16), h1 = __uint_as_float(xb[a].x & 0xffff0000u);
                        const double h2 = __uint_as_float(xb[a].y << 16), h3 = __uint_as_float(xb[a].y & 0xffff0000u);
                        d_lo += l0 * l0 + l1 * l1 + l2 * l2 + l3 * l3;
                        d_hi += h0 * h0 + h1 * h1 + h2 * h2 + h3 * h3;
                    }
                    d_lo = warp4_sum_d(d_lo);
                    d_hi = warp4_sum_d(d_hi);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (risky[i]) {
                            const double nd = sqrt(i ? d_hi : d_lo);
                            n16[i] = __half_as_ushort(__double2half(nd));
                            n_tok[i] = static_cast<float>(nd);
                        }
                    }
                }
                // A token whose norm is not below 3e37 (inf, NaN, or so near the bf16 limit that the
                // fp32 rotation could overflow) is packed as the zero vector with its norm as computed,
                // so that every cell lookup below stays inside the table: its input row is cleared
                // (the second half reloads it) and so are this half's fragments.
                const bool bad0 = !(n_tok[0] < 3.0e37f), bad1 = !(n_tok[1] < 3.0e37f);
                if (__any_sync(kFull, bad0 || bad1)) {
                    __syncwarp();  // the fragments of every lane are read
                    const uint32_t row0 = xbuf0 + static_cast<uint32_t>((cur * 16 + r) * kRowPad + 64 * c);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (bad0)
                            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(row0 + 16 * k), "r"(0u)
                                         : "memory");
                        if (bad1)
                            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(row0 + 8 * kRowPad + 16 * k),
                                         "r"(0u)
                                         : "memory");
                    }
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        if (bad0) xa[a] = make_uint2(0u, 0u);
                        if (bad1) xb[a] = make_uint2(0u, 0u);
                    }
                    __syncwarp();
                }
            }

            // A token whose norm is not below 3e37 (inf, NaN, or so near the bf16 limit that the fp32
            // rotation could overflow) is packed as the zero vector with its norm as computed: every
            // cell lookup below then stays inside the table.
            if (__any_sync(kFull, !(n_tok[0] < 3.0e37f) || !(n_tok[1] < 3.0e37f))) {
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    if (!(n_tok[0] < 3.0e37f)) xa[a] = make_uint2(0u, 0u);
                    if (!(n_tok[1] < 3.0e37f)) xb[a] = make_uint2(0u, 0u);
                }
            }
            // z = (H_16 D_s) per a on the tensor cores: columns b' = 8t + 2c + {0,1} of n-tile t.
            uint64_t zp[8][2];  // [a][token]: (columns 2c, 2c+1 of n-tile t)
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const uint2 bf = *reinterpret_cast<const uint2*>(&sm.bfrag[which][a][t][lane][0]);
                float zc[4];
                mma_bf16(zc, xa[a].x, xb[a].x, xa[a].y, xb[a].y, bf.x, bf.y);
                zp[a][0] = pk(zc[0], zc[1]);
                zp[a][1] = pk(zc[2], zc[3]);
            }
            // H_8 across a (three butterfly stages on packed pairs).
#pragma unroll
            for (int m = 1; m < 8; m <<= 1)
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    if (!(a & m))
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint64_t x0 = zp[a][i], x1 = zp[a | m][i];
                            zp[a][i] = add2(x0, x1);
                            zp[a | m][i] = sub2(x0, x1);
                        }

            // Quantize: v = z * 64 / (sqrt(128) n); cell lookup; one byte (2 nibbles,
            // coordinates 16a' + 8t + 2c and the next) per (token, a').
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float n = n_tok[i];
                float kq = n > 0.0f ? kCellScale / (n * 11.313708498984761f) : 0.0f;
                if (!(kq < 3.0e38f)) kq = 0.0f;  // norms too small to scale: treat as the zero vector
                const uint64_t kq2 = pk(kq, kq);
                const uint64_t magic2 = pk(12582912.0f, 12582912.0f);
                const uint32_t row =
                    static_cast<uint32_t>(__cvta_generic_to_shared(&sm.rows[warp][r + 8 * i][c])) + 4 * t;
                static_for8([&](auto ai) {
                    constexpr int a = decltype(ai)::value;
                    const uint64_t vv = mul2(zp[a][i], kq2);
                    const uint64_t mm = add2(vv, magic2);
                    float v0, v1, m0, m1;
                    upk(vv, v0, v1);
                    upk(mm, m0, m1);
                    const uint2 e0 = lds64(__float_as_uint(m0) * 256u + cell_adj);
                    const uint2 e1 = lds64(__float_as_uint(m1) * 256u + cell_adj);
                    const uint32_t i0 = e0.y + (v0 > __uint_as_float(e0.x) ? 1u : 0u);
                    const uint32_t i1 = e1.y + (v1 > __uint_as_float(e1.x) ? 1u : 0u);
                    sts8<8 * a>(row, i0 | (i1 << 4));
                });
                if (t == 0 && c == 0) sm.norms[warp][r + 8 * i] = n16[i];
            }
        }
        __syncwarp();

        // Write the rows: lane l writes 16-byte chunks (row = chunk / 4) to the row's own address.
        uint8_t* pages = which ? v_pages : k_pages;
        const int rb = 66;  // 64 index bytes + norm
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int chunk = lane + 32 * q, row = chunk >> 2, part = chunk & 3;
            const int64_t slot = __shfl_sync(kFull, my_slot, row);
            if (slot >= 0 && slot < capacity) {
                const int s32 = static_cast<int>(slot);
                const int blk = bs_log2 >= 0 ? s32 >> bs_log2 : s32 / block_size;
                const int off = s32 - blk * block_size;
                uint8_t* sub = pages + (static_cast<int64_t>(blk) * H + h) * block_size * rb;
                *reinterpret_cast<uint4*>(sub + off * 64 + 16 * part) =
                    *reinterpret_cast<const uint4*>(&sm.rows[warp][row][16 * part]);
                if (part == 0)
                    *reinterpret_cast<unsigned short*>(sub + block_size * 64 + 2 * off) = sm.norms[warp][row];
            } else if (slot >= capacity && part == 0 && d_err) {
                atomicOr(d_err, TQ_DERR_SLOT);
            }
        }
        __syncwarp();
    }
}

// ==== tensor-core pack for plain formats of 2-, 3- and 4-bit groups ==============
//
// The rotation and the norm are the uniform 4-bit kernel's. The quantizer
// uses the cell table of the coordinate's group (the tables of the 2-, 3- and
// 4-bit codebooks, 16 copies each: lanes l and l + 16 share a copy, and an
// 8-byte load serves the half-warps apart, so the lookups are free of bank
// conflicts). A group is a set of packed positions: rotated coordinate j sits
// at packed position pos_h[j] (group 0 first). Each lane keeps its indices in
// registers until the unit's input buffer is no longer read, writes them as
// bytes at their packed positions into that buffer (rows padded to 132 bytes
// so the lanes of one coordinate in 8 rows hit 8 banks), then each lane packs
// eight positions at a time into b bytes of the row, LSB-first. The format
// is a template parameter (bit widths, group sizes and byte offsets are
// constants) and a launch packs the tokens of one codec, K or V.

constexpr int kStagePitch = 132;

// Warps per CTA and staged row pitch: the QJL variant runs 8 warps, which leaves room for the
// fragments of S, and its rows carry 16 sign bytes after the index bytes.
template <bool QJL>
struct TcShape {
    static constexpr int W = QJL ? 8 : kPW;
    static constexpr int RP = QJL ? 88 : 72;
};

template <bool QJL>
struct PackTcSmemBase {
    static constexpr int W = TcShape<QJL>::W, RP = TcShape<QJL>::RP;
    QuantCell cells[3][kCells][16];  // codebooks of 2, 3, 4 bits (index bits - 2), 16 copies
    uint32_t bfrag[1][8][2][32][2];  // [codec][a][n-tile][lane][reg]: B operands (+-1 bf16 pairs)
    uint8_t rows[W][16][RP];         // staged rows of a warp's 16 tokens (pitch 72: 16 rows, 16 bank pairs)
    uint32_t norms[W][16];           // the row's fp16 norm (QJL: and the residual norm above it)
    int slot32[W][16];               // the unit's slots: -1 padding, capacity when past the pool
    uint8_t xbuf[W][2][16][kRowPad];  // double-buffered input rows (bf16); the current one then stages indices
};
struct PackQjlSmem : PackTcSmemBase<true> {
    uint32_t sfrag[2][8][16][32][2];  // [hi / lo][k-step][n-tile][lane][reg]: S as bf16 hi + lo B operands
    float centv[2][16][32];           // [group][index][lane]: 64 x centroid (v units), one copy per lane
};
using PackTcSmem = PackTcSmemBase<false>;
static_assert(16 * kStagePitch <= 16 * kRowPad, "index staging fits in an input buffer");
static_assert(sizeof(PackTcSmem) <= 232448 && sizeof(PackQjlSmem) <= 232448, "fits the shared memory of one CTA");

// The 8 indices (bytes) x0..x7 of lo = [x0 x1 x2 x3], hi = [x4 x5 x6 x7], b bits each, LSB-first.
template <int B>
__device__ __forceinline__ uint32_t pack8(uint32_t lo, uint32_t hi) {
    if constexpr (B == 4) {
        const uint32_t x = lo | (lo >> 4), y = hi | (hi >> 4);  // bytes 0, 2: two nibbles each
        return __byte_perm(x, y, 0x6420);
    } else if constexpr (B == 2) {
        const uint32_t x = lo | (lo >> 6), y = hi | (hi >> 6);  // bytes 0, 2: two 2-bit fields each
        const uint32_t x2 = (x & 0xFu) | ((x >> 12) & 0xF0u), y2 = (y & 0xFu) | ((y >> 12) & 0xF0u);
        return x2 | (y2 << 8);
    } else {
        const uint32_t x = lo | (lo >> 5), y = hi | (hi >> 5);  // bytes 0, 2: two 3-bit fields each
        const uint32_t x2 = (x & 0x3Fu) | ((x >> 10) & 0xFC0u), y2 = (y & 0x3Fu) | ((y >> 10) & 0xFC0u);
        return x2 | (y2 << 12);
    }
}

template <int B0_, int N0_, int B1_, int N1_>
struct PackFmt {
    static constexpr int B0 = B0_, N0 = N0_, B1 = B1_, N1 = N1_;
    static constexpr int NG = N1 > 0 ? 2 : 1;
    static constexpr int IB = (B0 * N0 + B1 * N1) / 8;  // index bytes of a row
    static constexpr int BOFF1 = B0 * N0 / 8;           // byte offset of group 1
    static_assert(N0 + N1 == kHeadDim && IB % 8 == 0 && IB <= 64, "whole 8-byte index rows of head_dim 128");
};
using PU4 = PackFmt<4, 128, 0, 0>;
using PU3 = PackFmt<3, 128, 0, 0>;
using PM43 = PackFmt<4, 64, 3, 64>;
using PM42 = PackFmt<4, 32, 2, 96>;
using PM32 = PackFmt<3, 64, 2, 64>;
using PU2 = PackFmt<2, 128, 0, 0>;

// Two floats as bf16x2 (round to nearest even; lo in the low half).
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// x = bf16 hi + bf16 lo for both halves (lo is the rounded remainder).
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    hi = bf16x2_rn(x0, x1);
    lo = bf16x2_rn(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xffff0000u));
}
// Bits 0-3 of x to bits 0, 2, 4, 6.
__device__ __forceinline__ uint32_t spread4(uint32_t x) {
    return (x & 1u) | ((x & 2u) << 1) | ((x & 4u) << 2) | ((x & 8u) << 3);
}

// Bit assembly of a warp's 16 staged index rows (one byte per packed position, pitch
// kStagePitch): in round k lanes 0-15 take packed positions 16 k .. 16 k + 7 of token lane
// and lanes 16-31 positions 16 k + 8 .. 16 k + 15 of token lane - 16 (one group for the
// whole warp, since groups start on multiples of 16), into b bytes of the row, LSB-first.
template <class F, int RP>
__device__ __forceinline__ void assemble_rows(uint32_t stage, uint8_t (&rows)[16][RP], int lane) {
    const int tok = lane & 15, hi8 = (lane >> 4) * 8;
    const uint32_t srow = stage + static_cast<uint32_t>(tok * kStagePitch);
    uint8_t* drow = &rows[tok][0];
    static_for<0, 8>([&](auto kc) {
        constexpr int K = decltype(kc)::value;
        constexpr bool G1 = F::NG == 2 && 16 * K >= F::N0;
        constexpr int B = G1 ? F::B1 : F::B0;
        const int p = 16 * K + hi8;
        const uint32_t lo = lds32(srow + p), hi = lds32(srow + p + 4);
        uint8_t* dst = drow + (G1 ? F::BOFF1 + (p - F::N0) * B / 8 : p * B / 8);
        if constexpr (B == 4) {
            *reinterpret_cast<uint32_t*>(dst) = pack8<4>(lo, hi);
        } else if constexpr (B == 2) {
            *reinterpret_cast<unsigned short*>(dst) = static_cast<unsigned short>(pack8<2>(lo, hi));
        } else {
            const uint32_t w = pack8<3>(lo, hi);
            dst[0] = static_cast<uint8_t>(w);
            dst[1] = static_cast<uint8_t>(w >> 8);
            dst[2] = static_cast<uint8_t>(w >> 16);
        }
    });
}

template <class F, bool QJL>
__global__ void __launch_bounds__(TcShape<QJL>::W * 32, 1) pack_tc_kernel(DevCodec cd, const __nv_bfloat16* __restrict__ src,
                                                          const int64_t* __restrict__ slots, int num_tokens,
                                                          uint8_t* __restrict__ pages, int capacity, int block_size,
                                                          int bs_log2, int* __restrict__ d_err) {
    static_assert(!QJL || F::NG == 1 || F::B0 != F::B1, "cell tables by bit width");
    constexpr int kW = TcShape<QJL>::W;
    using Smem = std::conditional_t<QJL, PackQjlSmem, PackTcSmem>;
    extern __shared__ __align__(16) uint8_t psm_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(psm_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;

    // Cell tables of the format's groups.
    for (int g = 0; g < F::NG; ++g) {
        const int bi = (g ? F::B1 : F::B0) - 2;
        for (int i = threadIdx.x; i < kCells * 16; i += kW * 32)
            sm.cells[bi][i >> 4][i & 15] = cd.cells[g * kCells + (i >> 4)];
    }
    if constexpr (QJL) {
        // B fragment (k-step a, n-tile nt) of lane (rr, cc): B[k][n] = S[8 nt + rr][16 a + k] for
        // k = 2 cc + {0, 1} (reg 0) and 2 cc + 8 + {0, 1} (reg 1), split into bf16 hi + lo.
        for (int i = threadIdx.x; i < 8 * 16 * 32; i += kW * 32) {
            const int ln = i & 31, nt = (i >> 5) & 15, a = i >> 9;
            const int n = 8 * nt + (ln >> 2), j0 = 16 * a + 2 * (ln & 3);
            for (int q = 0; q < 2; ++q) {
                const float s0 = cd.qjl_st[(j0 + 8 * q) * kHeadDim + n];  // S^T: entry (j, i) = S[i][j]
                const float s1 = cd.qjl_st[(j0 + 8 * q + 1) * kHeadDim + n];
                uint32_t hi, lo;
                split_bf16x2(s0, s1, hi, lo);
                sm.sfrag[0][a][nt][ln][q] = hi;
                sm.sfrag[1][a][nt][ln][q] = lo;
            }
        }
        for (int i = threadIdx.x; i < 2 * 16 * 32; i += kW * 32) {
            const int g = i >> 9, k = (i >> 5) & 15;
            sm.centv[g][k][i & 31] = g < F::NG ? kCellScale * cd.cent[g * kMaxLevels + k] : 0.0f;
        }
    }
    for (int i = threadIdx.x; i < 8 * 2 * 32; i += kW * 32) {
        const int ln = i & 31, t = (i >> 5) & 1, a = (i >> 6) & 7;
        const int rr = ln >> 2, cc = ln & 3;
        const int bp = 8 * t + rr;
        uint32_t regs[2];
        for (int q = 0; q < 2; ++q) {
            unsigned short hh[2];
            for (int e = 0; e < 2; ++e) {
                const int b = 2 * cc + 8 * q + e;
                const float val = cd.sign[16 * a + b] * ((__popc(bp & b) & 1) ? -1.0f : 1.0f);
                hh[e] = val > 0 ? 0x3F80 : 0xBF80;
            }
            regs[q] = static_cast<uint32_t>(hh[0]) | (static_cast<uint32_t>(hh[1]) << 16);
        }
        sm.bfrag[0][a][t][ln][0] = regs[0];
        sm.bfrag[0][a][t][ln][1] = regs[1];
    }
    __syncthreads();

    const int H = cd.num_heads;
    const int units = (num_tokens + 15) / 16 * H;  // (16-token group, KV head)
    // cell e of table bi for this lane: cells_lane + (bi * kCells + e) * 128
    const uint32_t cells_lane = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.cells[0][0][lane & 15]));
    const uint32_t xbuf0 = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.xbuf[warp][0][0][0]));
    auto issue = [&](int uu, int buf) {
        const int tg_ = uu / H, h_ = uu - tg_ * H;
        const __nv_bfloat16* src_ = src;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int piece = lane + 32 * i, tok = piece >> 4, part = piece & 15;
            const int t = tg_ * 16 + tok;
            const bool live = t < num_tokens;
            const __nv_bfloat16* g = src_ + (static_cast<int64_t>(live ? t : 0) * H + h_) * kHeadDim + 8 * part;
            cp_async16(xbuf0 + (buf * 16 + tok) * kRowPad + 16 * part, g, live ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const int stride = gridDim.x * kW;
    int u = blockIdx.x * kW + warp;
    if (u < units) issue(u, 0);
    for (int it = 0; u < units; u += stride, ++it) {
        const int cur = it & 1;
        const int tg = u / H, h = u - tg * H;
        const int t0 = tg * 16;
        constexpr int n0 = F::N0, ng = F::NG;

        if (lane < 16) {
            int64_t sl = -1;
            if (t0 + lane < num_tokens) sl = __ldg(slots + t0 + lane);
            sm.slot32[warp][lane] = sl < 0 ? -1 : (sl >= capacity ? capacity : static_cast<int>(sl));
        }

        if (u + stride < units) {
            issue(u + stride, cur ^ 1);
        } else {
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncwarp();

        const uint32_t frag_row = xbuf0 + (cur * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * kRowPad +
                                  ((lane >> 4) & 1) * 16;
        const uint32_t stage = xbuf0 + cur * 16 * kRowPad;  // [16][kStagePitch] index bytes, packed order
        float n_tok[2];
        unsigned short n16[2];
        // QJL: the residuals r = u - c[idx] (in units of v = 64 u) as the S product's A fragments,
        // bf16 hi + lo: [a][2 t + token] covers coordinates 16 a + 8 t + 2 c + {0, 1}
        uint32_t rh[8][4], rl[8][4];
        float rr[2] = {0.0f, 0.0f};  // sums of squared residuals per token (v units)
        // the lane's indices: idxr[t][a] bytes (j, token r), (j + 1, token r), (j, token r + 8), (j + 1, token r + 8)
        uint32_t idxr[2][8];
        const int16_t* posh = cd.pos + h * kHeadDim;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            uint2 xa[8], xb[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) ldsm_x4(frag_row + 32 * a, xa[a].x, xb[a].x, xa[a].y, xb[a].y);
            if (t == 0) {
                float ss_lo, ss_hi;
                {
                    uint64_t acc_lo = 0, acc_hi = 0;
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        const uint64_t l01 = bf16x2_to_f32x2(xa[a].x), l23 = bf16x2_to_f32x2(xa[a].y);
                        const uint64_t h01 = bf16x2_to_f32x2(xb[a].x), h23 = bf16x2_to_f32x2(xb[a].y);
                        acc_lo = fma2(l01, l01, fma2(l23, l23, acc_lo));
                        acc_hi = fma2(h01, h01, fma2(h23, h23, acc_hi));
                    }
                    float p, q;
                    upk(acc_lo, p, q);
                    ss_lo = p + q;
                    upk(acc_hi, p, q);
                    ss_hi = p + q;
                }
                ss_lo += __shfl_xor_sync(kFull, ss_lo, 1);
                ss_lo += __shfl_xor_sync(kFull, ss_lo, 2);
                ss_hi += __shfl_xor_sync(kFull, ss_hi, 1);
                ss_hi += __shfl_xor_sync(kFull, ss_hi, 2);
                bool risky[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float ss = i ? ss_hi : ss_lo;
                    const float n32 = sqrtf(ss);
                    bool rk = !(ss > 1e-30f && ss < 1e30f) || n32 > 60000.0f;
                    const __half hh = __float2half_rn(n32);
                    const unsigned short hb = __half_as_ushort(hh);
                    if (!rk) {
                        const float hf = __half2float(hh);
                        const float up = __half2float(__ushort_as_half(static_cast<unsigned short>(hb + 1)));
                        const float dn = __half2float(__ushort_as_half(static_cast<unsigned short>(hb - 1)));
                        const float tol = 1e-6f * n32;
                        rk = fabsf(n32 - 0.5f * (hf + up)) <= tol || fabsf(n32 - 0.5f * (hf + dn)) <= tol;
                    }
                    risky[i] = rk;
                    n_tok[i] = n32;
                    n16[i] = hb;
                }
                if (__any_sync(kFull, risky[0] || risky[1])) {
                    double d_lo = 0.0, d_hi = 0.0;
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        const double l0 = __uint_as_float(xa[a].x << 16), l1 = __uint_as_float(xa[a].x & 0xffff0000u);
                        const double l2 = __uint_as_float(xa[a].y << 16), l3 = __uint_as_float(xa[a].y & 0xffff0000u);
                        const double h0 = __uint_as_float(xb[a].x << 16), h1 = __uint_as_float(xb[a].x & 0xffff0000u);
                        const double h2 = __uint_as_float(xb[a].y << 16), h3 = __uint_as_float(xb[a].y & 0xffff0000u);
                        d_lo += l0 * l0 + l1 * l1 + l2 * l2 + l3 * l3;
                        d_hi += h0 * h0 + h1 * h1 + h2 * h2 + h3 * h3;
                    }
                    d_lo = warp4_sum_d(d_lo);
                    d_hi = warp4_sum_d(d_hi);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        if (risky[i]) {
                            const double nd = sqrt(i ? d_hi : d_lo);
                            n16[i] = __half_as_ushort(__double2half(nd));
                            n_tok[i] = static_cast<float>(nd);
                        }
                    }
                }
                // A token whose norm is not below 3e37 (inf, NaN, or so near the bf16 limit that the
                // fp32 rotation could overflow) is packed as the zero vector with its norm as computed,
                // so that every cell lookup below stays inside the table: its input row is cleared
                // (the second half reloads it) and so are this half's fragments.
                const bool bad0 = !(n_tok[0] < 3.0e37f), bad1 = !(n_tok[1] < 3.0e37f);
                if (__any_sync(kFull, bad0 || bad1)) {
                    __syncwarp();  // the fragments of every lane are read
                    const uint32_t row0 = xbuf0 + static_cast<uint32_t>((cur * 16 + r) * kRowPad + 64 * c);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (bad0)
                            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(row0 + 16 * k), "r"(0u)
                                         : "memory");
                        if (bad1)
                            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(row0 + 8 * kRowPad + 16 * k),
                                         "r"(0u)
                                         : "memory");
                    }
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        if (bad0) xa[a] = make_uint2(0u, 0u);
                        if (bad1) xb[a] = make_uint2(0u, 0u);
                    }
                    __syncwarp();
                }
            }
            // A token whose norm is not below 3e37 (inf, NaN, or so near the bf16 limit that the fp32
            // rotation could overflow) is packed as the zero vector with its norm as computed: every
            // cell lookup below then stays inside the table.
            if (__any_sync(kFull, !(n_tok[0] < 3.0e37f) || !(n_tok[1] < 3.0e37f))) {
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    if (!(n_tok[0] < 3.0e37f)) xa[a] = make_uint2(0u, 0u);
                    if (!(n_tok[1] < 3.0e37f)) xb[a] = make_uint2(0u, 0u);
                }
            }
            uint64_t kq2[2];  // v = z * 64 / (sqrt(128) n) per token
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float kq = n_tok[i] > 0.0f ? kCellScale / (n_tok[i] * 11.313708498984761f) : 0.0f;
                if (!(kq < 3.0e38f)) kq = 0.0f;  // norms too small to scale: the zero vector
                kq2[i] = pk(kq, kq);
            }
            uint64_t zq[8][2];  // [a][token]: rotated coordinates 16 a + 8 t + 2 c + {0, 1}
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const uint2 bf = *reinterpret_cast<const uint2*>(&sm.bfrag[0][a][t][lane][0]);
                float zc[4];
                mma_bf16(zc, xa[a].x, xb[a].x, xa[a].y, xb[a].y, bf.x, bf.y);
                zq[a][0] = pk(zc[0], zc[1]);
                zq[a][1] = pk(zc[2], zc[3]);
            }
#pragma unroll
            for (int m = 1; m < 8; m <<= 1)
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    if (!(a & m))
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint64_t x0 = zq[a][i], x1 = zq[a | m][i];
                            zq[a][i] = add2(x0, x1);
                            zq[a | m][i] = sub2(x0, x1);
                        }
            // Quantize with the cell table of each coordinate's group.
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int j = 16 * a + 8 * t + 2 * c;
                uint32_t pp = static_cast<uint32_t>(j) | (static_cast<uint32_t>(j + 1) << 16);
                if (ng == 2) pp = __ldg(reinterpret_cast<const unsigned int*>(posh + j));  // positions of j, j + 1
                // address of cell round(v) + 64 = bits(v + 1.5 * 2^23) - 0x4B400000 + 64
                constexpr uint32_t kTab0 = static_cast<uint32_t>((F::B0 - 2) * kCells) * 128u + 64u * 128u -
                                           0x4B400000u * 128u;
                constexpr uint32_t kTab1 = static_cast<uint32_t>(((F::NG == 2 ? F::B1 : F::B0) - 2) * kCells) * 128u +
                                           64u * 128u - 0x4B400000u * 128u;
                uint32_t tab[2], cen[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int pe = static_cast<int>((pp >> (16 * e)) & 0xffffu);
                    tab[e] = cells_lane + ((ng == 2 && pe >= n0) ? kTab1 : kTab0);
                    cen[e] = (ng == 2 && pe >= n0) ? 16u * 128u : 0u;
                }
                uint32_t w = 0;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint64_t vv = mul2(zq[a][i], kq2[i]);
                    const uint64_t mm = add2(vv, pk(12582912.0f, 12582912.0f));
                    float v0, v1, m0, m1;
                    upk(vv, v0, v1);
                    upk(mm, m0, m1);
                    const uint2 e0 = lds64(__float_as_uint(m0) * 128u + tab[0]);
                    const uint2 e1 = lds64(__float_as_uint(m1) * 128u + tab[1]);
                    const uint32_t i0 = e0.y + (v0 > __uint_as_float(e0.x) ? 1u : 0u);
                    const uint32_t i1 = e1.y + (v1 > __uint_as_float(e1.x) ? 1u : 0u);
                    w |= (i0 | (i1 << 8)) << (16 * i);
                    if constexpr (QJL) {
                        const uint32_t cl = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.centv[0][0][lane]));
                        const float q0 = v0 - __uint_as_float(lds32(cl + cen[0] + i0 * 128u));
                        const float q1 = v1 - __uint_as_float(lds32(cl + cen[1] + i1 * 128u));
                        rr[i] = fmaf(q0, q0, fmaf(q1, q1, rr[i]));
                        split_bf16x2(q0, q1, rh[a][2 * t + i], rl[a][2 * t + i]);
                    }
                }
                idxr[t][a] = w;
            }
        }
        __syncwarp();  // every lane has read its fragments: the input buffer now stages the indices
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int j = 16 * a + 8 * t + 2 * c;
                uint32_t pp = static_cast<uint32_t>(j) | (static_cast<uint32_t>(j + 1) << 16);
                if (ng == 2) pp = __ldg(reinterpret_cast<const unsigned int*>(posh + j));
                const uint32_t w = idxr[t][a];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint32_t row = stage + static_cast<uint32_t>((r + 8 * i) * kStagePitch);
                    asm volatile("st.shared.u8 [%0], %1;" ::"r"(row + (pp & 0xffffu)), "r"((w >> (16 * i)) & 0xffu)
                                 : "memory");
                    asm volatile("st.shared.u8 [%0], %1;" ::"r"(row + (pp >> 16)), "r"((w >> (16 * i + 8)) & 0xffu)
                                 : "memory");
                }
            }
        uint32_t g16[2] = {0u, 0u};
        if constexpr (QJL) {
            // Residual norms |r| = sqrt(sum of squares in v units) / 64, fp16.
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float q = rr[i];
                q += __shfl_xor_sync(kFull, q, 1);
                q += __shfl_xor_sync(kFull, q, 2);
                g16[i] = __half_as_ushort(__float2half_rn(sqrtf(q) * (1.0f / kCellScale)));
            }
            // S r on the tensor cores (hi x hi + lo x hi + hi x lo, fp32 accumulation), four n-tiles
            // at a time; sign bit of output i = 8 nt + 2 c + e is (S r)_i >= 0, byte nt of the sign
            // stream, bit 2 c + e.
            const uint32_t sf_lane = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.sfrag[0][0][0][lane][0]));
            constexpr uint32_t kLoOff = 8u * 16u * 32u * 8u;
#pragma unroll
            for (int n4 = 0; n4 < 4; ++n4) {
                float acc[4][4];
#pragma unroll
                for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const uint32_t off = static_cast<uint32_t>((a * 16 + 4 * n4 + n) * 32 * 8);
                        const uint2 bh = lds64(sf_lane + off), bl = lds64(sf_lane + kLoOff + off);
                        mma_bf16_acc(acc[n], rh[a][0], rh[a][1], rh[a][2], rh[a][3], bh.x, bh.y);
                        mma_bf16_acc(acc[n], rl[a][0], rl[a][1], rl[a][2], rl[a][3], bh.x, bh.y);
                        mma_bf16_acc(acc[n], rh[a][0], rh[a][1], rh[a][2], rh[a][3], bl.x, bl.y);
                    }
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    const uint32_t s0 = __ballot_sync(kFull, acc[n][0] >= 0.0f);
                    const uint32_t s1 = __ballot_sync(kFull, acc[n][1] >= 0.0f);
                    const uint32_t s2 = __ballot_sync(kFull, acc[n][2] >= 0.0f);
                    const uint32_t s3 = __ballot_sync(kFull, acc[n][3] >= 0.0f);
                    if (c == 0) {
                        const int sh = 4 * r;
                        sm.rows[warp][r][F::IB + 4 * n4 + n] =
                            static_cast<uint8_t>(spread4((s0 >> sh) & 0xFu) | (spread4((s1 >> sh) & 0xFu) << 1));
                        sm.rows[warp][r + 8][F::IB + 4 * n4 + n] =
                            static_cast<uint8_t>(spread4((s2 >> sh) & 0xFu) | (spread4((s3 >> sh) & 0xFu) << 1));
                    }
                }
            }
        }
        if (c == 0) {
            sm.norms[warp][r] = static_cast<uint32_t>(n16[0]) | (g16[0] << 16);
            sm.norms[warp][r + 8] = static_cast<uint32_t>(n16[1]) | (g16[1] << 16);
        }
        __syncwarp();

        assemble_rows<F>(stage, sm.rows[warp], lane);
        __syncwarp();

        // Write the rows in 8-byte pieces (index rows, and with QJL their 16 sign bytes, are whole
        // multiples of 8 bytes), and the norms.
        constexpr int ib = F::IB + (QJL ? 16 : 0), rb = ib + (QJL ? 4 : 2);
        const int pieces = ib / 8;
        for (int q = lane; q < 16 * pieces; q += 32) {
            const int row = q / pieces, part = q - row * pieces;
            const int slot = sm.slot32[warp][row];
            if (slot >= 0 && slot < capacity) {
                const int blk = bs_log2 >= 0 ? slot >> bs_log2 : slot / block_size;
                const int off = slot - blk * block_size;
                uint8_t* sub = pages + (static_cast<int64_t>(blk) * H + h) * block_size * rb;
                *reinterpret_cast<uint2*>(sub + off * ib + 8 * part) =
                    *reinterpret_cast<const uint2*>(&sm.rows[warp][row][8 * part]);
                if (part == 0) {
                    if constexpr (QJL)
                        *reinterpret_cast<uint32_t*>(sub + block_size * ib + 4 * off) = sm.norms[warp][row];
                    else
                        *reinterpret_cast<unsigned short*>(sub + block_size * ib + 2 * off) =
                            static_cast<unsigned short>(sm.norms[warp][row]);
                }
            } else if (slot >= capacity && part == 0 && d_err) {
                atomicOr(d_err, TQ_DERR_SLOT);
            }
        }
        __syncwarp();
    }
}


// ==== tensor-core pack for group-wise formats ===================================
//
// Group-wise rotation: u = R_h x / n_g with R_h per KV head (rows are packed
// positions, columns channels) and one norm per group over the group's original
// channels. R_h's nonzero entries are +-1/sqrt(m) inside Hadamard blocks of size
// m (powers of two, 16 to 128, starting on multiples of 16), so R_h = D Q with
// Q of entries -1, 0, +1 (exact in bf16) and D the blocks' scales, constants of
// the format. The channels reach the blocks through a per-head permutation, so
// Q x runs on mma.sync m16n8k16 as the dense product of a unit's 16 x 128 inputs
// with Q^T (8 k-steps x 16 n-tiles, fp32 accumulation); D and 64 / n_g then scale
// it to the cell domain. A CTA works on one KV head and keeps Q^T's B fragments
// (32 KB) in shared memory. The group norms are sums of squares of the inputs
// masked per group. Quantizer, index staging (the product's output coordinate is
// the packed position), bit assembly and row writes follow the plain kernel; a
// row ends in the two fp16 group norms.

// The recipe variant (group-wise rotation plus each group's QJL stage) runs 8 warps, which leaves
// room for the fragments of S_0 and S_1.
template <bool RECIPE>
struct PackGwSmemBase {
    static constexpr int W = RECIPE ? 8 : kPW;
    QuantCell cells[2][kCells][16];   // codebook cells of group 0 and group 1, 16 copies
    uint32_t qfrag[8][16][32][2];     // [k-step][n-tile][lane][reg]: Q^T of the CTA's head, bf16 pairs
    uint4 gmask[4][32];               // [word / 4][lane]: the lane's group-0 channels as bf16 half masks
    uint8_t rows[W][16][72];          // staged rows
    uint2 norms[W][16];               // the row's fp16 norms: n_0 | n_1 << 16 (recipe: n_0, g_0, n_1, g_1)
    int slot32[W][16];                // the unit's slots: -1 padding, capacity when past the pool
    uint8_t xbuf[W][2][16][kRowPad];  // double-buffered input rows; the current one then stages indices
};
struct PackRecipeSmem : PackGwSmemBase<true> {
    uint32_t sfrag[2][2][4][8][32][2];  // [group][hi / lo][k-step][n-tile][lane][reg]: S_g as bf16 hi + lo
    float centv[2][16][32];             // [group][index][lane]: 64 x centroid (v units), one copy per lane
};
using PackGwSmem = PackGwSmemBase<false>;
static_assert(sizeof(PackGwSmem) <= 232448 && sizeof(PackRecipeSmem) <= 232448, "fits the shared memory of one CTA");

// Row layout of the recipe row (two groups, each [indices][QJL signs], then the four fp16 norms):
// the same group fields as F with group 1's indices after group 0's sign bytes.
template <class F>
struct RecipeOf {
    static constexpr int B0 = F::B0, N0 = F::N0, B1 = F::B1, N1 = F::N1, NG = 2;
    static constexpr int SIGN0 = B0 * N0 / 8;                 // group 0's sign bytes
    static constexpr int BOFF1 = SIGN0 + N0 / 8;              // group 1's index bytes
    static constexpr int SIGN1 = BOFF1 + B1 * N1 / 8;         // group 1's sign bytes
    static constexpr int IB = SIGN1 + N1 / 8;                 // index part of a row
    static_assert(IB % 8 == 0 && IB <= 72, "whole 8-byte index parts within the staged row");
};

// 1/sqrt(m) of the Hadamard block that holds packed position p (each group's
// blocks in decreasing powers of two, as the codec builds R_h).
template <class F>
__host__ __device__ constexpr float gw_block_scale(int p) {
    const int n = p >= F::N0 ? F::N1 : F::N0;
    int off = p >= F::N0 ? p - F::N0 : p;
    for (int k = 7; k >= 0; --k) {
        const int m = 1 << k;
        if (!(n & m)) continue;
        if (off < m)
            return static_cast<float>(((k & 1) ? 0.70710678118654752440 : 1.0) / static_cast<double>(1 << (k / 2)));
        off -= m;
    }
    return 0.0f;
}

template <class F, bool RECIPE>
__global__ void __launch_bounds__(PackGwSmemBase<RECIPE>::W * 32, 1) pack_gw_kernel(DevCodec cd, const __nv_bfloat16* __restrict__ src,
                                                          const int64_t* __restrict__ slots, int num_tokens,
                                                          uint8_t* __restrict__ pages, int capacity, int block_size,
                                                          int bs_log2, int* __restrict__ d_err) {
    static_assert(F::NG == 2 && F::N0 % 16 == 0, "two groups starting on a multiple of 16");
    static_assert(!RECIPE || (F::N0 == 64 && F::N1 == 64), "recipe rows: one group per half of the product");
    constexpr int kW = PackGwSmemBase<RECIPE>::W;
    using Smem = std::conditional_t<RECIPE, PackRecipeSmem, PackGwSmem>;
    using FR = std::conditional_t<RECIPE, RecipeOf<F>, F>;  // the row layout
    extern __shared__ __align__(16) uint8_t psm_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(psm_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;
    const int H = cd.num_heads;
    const int h = blockIdx.x % H, cta = blockIdx.x / H, ctas = gridDim.x / H;

    // Cell tables (group g's cells at g * kCells in the codec's table).
    for (int i = threadIdx.x; i < 2 * kCells * 16; i += kW * 32) (&sm.cells[0][0][0])[i] = cd.cells[i >> 4];
    // B fragment (k-step a, n-tile nt) of lane (rr, cc): B[k][n] = sign of R_h[8 nt + rr][16 a + k] for
    // k = 2 cc + {0, 1} (reg 0) and 2 cc + 8 + {0, 1} (reg 1).
    const float* rt = cd.rot_t + static_cast<int64_t>(h) * kHeadDim * kHeadDim;  // entry (j, p) = R_h[p][j]
    for (int i = threadIdx.x; i < 8 * 16 * 32; i += kW * 32) {
        const int ln = i & 31, nt = (i >> 5) & 15, a = i >> 9;
        const int p = 8 * nt + (ln >> 2), j0 = 16 * a + 2 * (ln & 3);
        uint32_t regs[2];
        for (int q = 0; q < 2; ++q) {
            uint32_t w = 0;
            for (int e = 0; e < 2; ++e) {
                const float val = __ldg(rt + (j0 + 8 * q + e) * kHeadDim + p);
                const uint32_t hb = val > 0.0f ? 0x3F80u : (val < 0.0f ? 0xBF80u : 0u);
                w |= hb << (16 * e);
            }
            regs[q] = w;
        }
        sm.qfrag[a][nt][ln][0] = regs[0];
        sm.qfrag[a][nt][ln][1] = regs[1];
    }
    if constexpr (RECIPE) {
        // S_g's B fragment (k-step kk, n-tile nt) of lane (rr, cc): B[k][n] = S_g[8 nt + rr][16 kk + k] for
        // k = 2 cc + {0, 1} (reg 0) and 2 cc + 8 + {0, 1} (reg 1), split into bf16 hi + lo; the codec
        // stores S_0^T then S_1^T, entry (j, i) = S_g[i][j].
        for (int i = threadIdx.x; i < 2 * 4 * 8 * 32; i += kW * 32) {
            const int ln = i & 31, nt = (i >> 5) & 7, kk = (i >> 8) & 3, g = i >> 10;
            const float* st = cd.qjl_st + g * F::N0 * F::N0;
            const int n = 8 * nt + (ln >> 2), j0 = 16 * kk + 2 * (ln & 3);
            for (int q = 0; q < 2; ++q) {
                uint32_t hi, lo;
                split_bf16x2(st[(j0 + 8 * q) * 64 + n], st[(j0 + 8 * q + 1) * 64 + n], hi, lo);
                sm.sfrag[g][0][kk][nt][ln][q] = hi;
                sm.sfrag[g][1][kk][nt][ln][q] = lo;
            }
        }
        for (int i = threadIdx.x; i < 2 * 16 * 32; i += kW * 32) {
            const int g = i >> 9, k = (i >> 5) & 15;
            sm.centv[g][k][i & 31] = kCellScale * cd.cent[g * kMaxLevels + k];
        }
    }
    // Mask word k = 2 a + q of lane l covers its fragment channels 16 a + 8 q + 2 (l % 4) + {0, 1}.
    if (threadIdx.x < 128) {
        const int ln = threadIdx.x & 31, w4 = threadIdx.x >> 5;
        const int16_t* posh = cd.pos + h * kHeadDim;
        uint32_t m[4];
        for (int k = 0; k < 4; ++k) {
            const int wd = 4 * w4 + k;
            const int j = 16 * (wd >> 1) + 8 * (wd & 1) + 2 * (ln & 3);
            m[k] = (posh[j] < F::N0 ? 0x0000FFFFu : 0u) | (posh[j + 1] < F::N0 ? 0xFFFF0000u : 0u);
        }
        sm.gmask[w4][ln] = make_uint4(m[0], m[1], m[2], m[3]);
    }
    __syncthreads();

    const int tgroups = (num_tokens + 15) / 16;
    // cell e of group g for this lane: cells_lane + (g * kCells + e) * 128
    const uint32_t cells_lane = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.cells[0][0][lane & 15]));
    const uint32_t xbuf0 = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.xbuf[warp][0][0][0]));
    const uint32_t qf_lane = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.qfrag[0][0][lane][0]));
    auto issue = [&](int tg_, int buf) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int piece = lane + 32 * i, tok = piece >> 4, part = piece & 15;
            const int t = tg_ * 16 + tok;
            const bool live = t < num_tokens;
            const __nv_bfloat16* g = src + (static_cast<int64_t>(live ? t : 0) * H + h) * kHeadDim + 8 * part;
            cp_async16(xbuf0 + (buf * 16 + tok) * kRowPad + 16 * part, g, live ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const int stride = ctas * kW;
    int tg = cta * kW + warp;
    if (tg < tgroups) issue(tg, 0);
    for (int it = 0; tg < tgroups; tg += stride, ++it) {
        const int cur = it & 1;
        const int t0 = tg * 16;
        if (lane < 16) {
            int64_t sl = -1;
            if (t0 + lane < num_tokens) sl = __ldg(slots + t0 + lane);
            sm.slot32[warp][lane] = sl < 0 ? -1 : (sl >= capacity ? capacity : static_cast<int>(sl));
        }
        if (tg + stride < tgroups) {
            issue(tg + stride, cur ^ 1);
        } else {
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncwarp();

        // A fragments: xa[a] = token r, channels 16 a + 2 c + {0, 1} (.x) and 16 a + 8 + 2 c + {0, 1} (.y);
        // xb[a] the same for token r + 8.
        const uint32_t frag_row = xbuf0 + (cur * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * kRowPad +
                                  ((lane >> 4) & 1) * 16;
        const uint32_t stage = xbuf0 + cur * 16 * kRowPad;  // [16][kStagePitch] index bytes, packed order
        uint2 xa[8], xb[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) ldsm_x4(frag_row + 32 * a, xa[a].x, xb[a].x, xa[a].y, xb[a].y);
        __syncwarp();  // every lane has read its fragments: the input buffer now stages the indices

        // Group norms: sums of exact squares of the inputs masked per group (fp32), fp64 when the
        // fp32 norm is too close to an fp16 rounding midpoint to call.
        float n_tok[2][2];          // [group][token r, r + 8]
        unsigned short n16[2][2];
        {
            uint32_t mw[16];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint4 m4 = sm.gmask[k][lane];
                mw[4 * k] = m4.x;
                mw[4 * k + 1] = m4.y;
                mw[4 * k + 2] = m4.z;
                mw[4 * k + 3] = m4.w;
            }
            uint64_t acc[2][2] = {{0, 0}, {0, 0}};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint32_t m = mw[2 * a + q];
                    const uint32_t lo = q ? xa[a].y : xa[a].x, hi = q ? xb[a].y : xb[a].x;
                    const uint64_t l0 = bf16x2_to_f32x2(lo & m), l1 = bf16x2_to_f32x2(lo & ~m);
                    const uint64_t h0 = bf16x2_to_f32x2(hi & m), h1 = bf16x2_to_f32x2(hi & ~m);
                    acc[0][0] = fma2(l0, l0, acc[0][0]);
                    acc[1][0] = fma2(l1, l1, acc[1][0]);
                    acc[0][1] = fma2(h0, h0, acc[0][1]);
                    acc[1][1] = fma2(h1, h1, acc[1][1]);
                }
            bool risky[2][2];
            bool any_risky = false;
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float p, q;
                    upk(acc[g][i], p, q);
                    float ss = p + q;
                    ss += __shfl_xor_sync(kFull, ss, 1);
                    ss += __shfl_xor_sync(kFull, ss, 2);
                    const float n32 = sqrtf(ss);
                    bool rk = !(ss > 1e-30f && ss < 1e30f) || n32 > 60000.0f;
                    const __half hh = __float2half_rn(n32);
                    const unsigned short hb = __half_as_ushort(hh);
                    if (!rk) {
                        const float hf = __half2float(hh);
                        const float up = __half2float(__ushort_as_half(static_cast<unsigned short>(hb + 1)));
                        const float dn = __half2float(__ushort_as_half(static_cast<unsigned short>(hb - 1)));
                        const float tol = 1e-6f * n32;
                        rk = fabsf(n32 - 0.5f * (hf + up)) <= tol || fabsf(n32 - 0.5f * (hf + dn)) <= tol;
                    }
                    risky[g][i] = rk;
                    any_risky = any_risky || rk;
                    n_tok[g][i] = n32;
                    n16[g][i] = hb;
                }
            if (__any_sync(kFull, any_risky)) {
                // Rare: fp64 sums (all lanes join the shuffles).
                double d[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint32_t m = mw[2 * a + q];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint32_t w = i ? (q ? xb[a].y : xb[a].x) : (q ? xa[a].y : xa[a].x);
                            const double e0 = __uint_as_float(w << 16), e1 = __uint_as_float(w & 0xffff0000u);
                            const bool in0 = (m & 0xFFFFu) != 0, in1 = (m >> 16) != 0;
                            d[0][i] += (in0 ? e0 * e0 : 0.0) + (in1 ? e1 * e1 : 0.0);
                            d[1][i] += (in0 ? 0.0 : e0 * e0) + (in1 ? 0.0 : e1 * e1);
                        }
                    }
#pragma unroll
                for (int g = 0; g < 2; ++g)
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const double sd = warp4_sum_d(d[g][i]);
                        if (risky[g][i]) {
                            const double nd = sqrt(sd);
                            n16[g][i] = __half_as_ushort(__double2half(nd));
                            n_tok[g][i] = static_cast<float>(nd);
                        }
                    }
            }
        }
        // A token with a norm not below 3e37 (inf, NaN, or so near the bf16 limit that the fp32 product
        // could overflow) is packed as the zero vector with its norms as computed: every cell lookup
        // below then stays inside the table.
        {
            const bool bad0 = !(n_tok[0][0] < 3.0e37f) || !(n_tok[1][0] < 3.0e37f);
            const bool bad1 = !(n_tok[0][1] < 3.0e37f) || !(n_tok[1][1] < 3.0e37f);
            if (__any_sync(kFull, bad0 || bad1)) {
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    if (bad0) xa[a] = make_uint2(0u, 0u);
                    if (bad1) xb[a] = make_uint2(0u, 0u);
                }
            }
        }
        float kq[2][2];  // 64 / n_g per token: v = 64 u = acc * D * kq
#pragma unroll
        for (int g = 0; g < 2; ++g)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float k = n_tok[g][i] > 0.0f ? kCellScale / n_tok[g][i] : 0.0f;
                if (!(k < 3.0e38f)) k = 0.0f;  // norms too small to scale: the zero vector
                kq[g][i] = k;
            }

        // Q x in two halves of 8 n-tiles (outputs 64 HALF .. 64 HALF + 63), each over the 8 k-steps;
        // then quantize and stage bytes (p, p + 1), p = 8 nt + 2 c, of tokens r and r + 8. Recipe rows:
        // each half is one group, whose QJL stage follows its quantization.
        uint32_t g16[2][2] = {{0u, 0u}, {0u, 0u}};  // recipe: [group][token] residual norms
        static_for<0, 2>([&](auto hc) {
            constexpr int HALF = decltype(hc)::value;
            // recipe: the group's residuals r = u - c[idx] (v units) as the S_g product's A fragments,
            // bf16 hi + lo: [k-step][2 (n-tile & 1) + token] for n-tiles 2 k-step + {0, 1} of the half
            uint32_t rh[4][4], rl[4][4];
            float rr[2] = {0.0f, 0.0f};
            float acc[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const uint2 bf = lds64(qf_lane + static_cast<uint32_t>((a * 16 + 8 * HALF + n) * 32 * 8));
                    mma_bf16_acc(acc[n], xa[a].x, xb[a].x, xa[a].y, xb[a].y, bf.x, bf.y);
                }
            static_for<0, 8>([&](auto nc) {
                constexpr int n = decltype(nc)::value;
                constexpr int NT = 8 * HALF + n;
                constexpr int G = 8 * NT >= F::N0 ? 1 : 0;
                constexpr float kScale = gw_block_scale<F>(8 * NT);
                // address of cell round(v) + 64 = bits(v + 1.5 * 2^23) - 0x4B400000 + 64
                constexpr uint32_t kTab = static_cast<uint32_t>(G * kCells) * 128u + 64u * 128u - 0x4B400000u * 128u;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float kv = kq[G][i] * kScale;
                    const uint64_t vv = mul2(pk(acc[n][2 * i], acc[n][2 * i + 1]), pk(kv, kv));
                    const uint64_t mm = add2(vv, pk(12582912.0f, 12582912.0f));
                    float v0, v1, m0, m1;
                    upk(vv, v0, v1);
                    upk(mm, m0, m1);
                    const uint2 e0 = lds64(__float_as_uint(m0) * 128u + cells_lane + kTab);
                    const uint2 e1 = lds64(__float_as_uint(m1) * 128u + cells_lane + kTab);
                    const uint32_t i0 = e0.y + (v0 > __uint_as_float(e0.x) ? 1u : 0u);
                    const uint32_t i1 = e1.y + (v1 > __uint_as_float(e1.x) ? 1u : 0u);
                    const uint32_t at = stage + static_cast<uint32_t>((r + 8 * i) * kStagePitch + 8 * NT + 2 * c);
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(at), "h"(static_cast<unsigned short>(i0 | (i1 << 8)))
                                 : "memory");
                    if constexpr (RECIPE) {
                        const uint32_t cl =
                            static_cast<uint32_t>(__cvta_generic_to_shared(&sm.centv[G][0][lane]));
                        const float q0 = v0 - __uint_as_float(lds32(cl + i0 * 128u));
                        const float q1 = v1 - __uint_as_float(lds32(cl + i1 * 128u));
                        rr[i] = fmaf(q0, q0, fmaf(q1, q1, rr[i]));
                        split_bf16x2(q0, q1, rh[n >> 1][2 * (n & 1) + i], rl[n >> 1][2 * (n & 1) + i]);
                    }
                }
            });
            if constexpr (RECIPE) {
                // Residual norms of the group, then S_g r_g (hi x hi + lo x hi + hi x lo), four n-tiles at
                // a time; bit 2 c + e of sign byte nt is (S_g r_g)_i >= 0 for i = 8 nt + 2 c + e.
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float q = rr[i];
                    q += __shfl_xor_sync(kFull, q, 1);
                    q += __shfl_xor_sync(kFull, q, 2);
                    g16[HALF][i] = __half_as_ushort(__float2half_rn(sqrtf(q) * (1.0f / kCellScale)));
                }
                const uint32_t sf_lane =
                    static_cast<uint32_t>(__cvta_generic_to_shared(&sm.sfrag[HALF][0][0][0][lane][0]));
                constexpr uint32_t kLoOff = 4u * 8u * 32u * 8u;
                constexpr int kSign = HALF ? FR::SIGN1 : FR::SIGN0;
#pragma unroll
                for (int n4 = 0; n4 < 2; ++n4) {
                    float sacc[4][4];
#pragma unroll
                    for (int n = 0; n < 4; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.0f;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                        for (int n = 0; n < 4; ++n) {
                            const uint32_t off = static_cast<uint32_t>((kk * 8 + 4 * n4 + n) * 32 * 8);
                            const uint2 bh = lds64(sf_lane + off), bl = lds64(sf_lane + kLoOff + off);
                            mma_bf16_acc(sacc[n], rh[kk][0], rh[kk][1], rh[kk][2], rh[kk][3], bh.x, bh.y);
                            mma_bf16_acc(sacc[n], rl[kk][0], rl[kk][1], rl[kk][2], rl[kk][3], bh.x, bh.y);
                            mma_bf16_acc(sacc[n], rh[kk][0], rh[kk][1], rh[kk][2], rh[kk][3], bl.x, bl.y);
                        }
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const uint32_t s0 = __ballot_sync(kFull, sacc[n][0] >= 0.0f);
                        const uint32_t s1 = __ballot_sync(kFull, sacc[n][1] >= 0.0f);
                        const uint32_t s2 = __ballot_sync(kFull, sacc[n][2] >= 0.0f);
                        const uint32_t s3 = __ballot_sync(kFull, sacc[n][3] >= 0.0f);
                        if (c == 0) {
                            const int sh = 4 * r;
                            sm.rows[warp][r][kSign + 4 * n4 + n] = static_cast<uint8_t>(
                                spread4((s0 >> sh) & 0xFu) | (spread4((s1 >> sh) & 0xFu) << 1));
                            sm.rows[warp][r + 8][kSign + 4 * n4 + n] = static_cast<uint8_t>(
                                spread4((s2 >> sh) & 0xFu) | (spread4((s3 >> sh) & 0xFu) << 1));
                        }
                    }
                }
            }
        });
        if (c == 0) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint32_t n0 = n16[0][i], n1 = n16[1][i];
                sm.norms[warp][r + 8 * i] = RECIPE ? make_uint2(n0 | (g16[0][i] << 16), n1 | (g16[1][i] << 16))
                                                   : make_uint2(n0 | (n1 << 16), 0u);
            }
        }
        __syncwarp();
        assemble_rows<FR>(stage, sm.rows[warp], lane);
        __syncwarp();

        // Write the rows in 8-byte pieces, and the norms (two, recipe four).
        constexpr int ib = FR::IB, rb = FR::IB + (RECIPE ? 8 : 4);
        constexpr int pieces = ib / 8;
        for (int q = lane; q < 16 * pieces; q += 32) {
            const int row = q / pieces, part = q - row * pieces;
            const int slot = sm.slot32[warp][row];
            if (slot >= 0 && slot < capacity) {
                const int blk = bs_log2 >= 0 ? slot >> bs_log2 : slot / block_size;
                const int off = slot - blk * block_size;
                uint8_t* sub = pages + (static_cast<int64_t>(blk) * H + h) * block_size * rb;
                *reinterpret_cast<uint2*>(sub + off * ib + 8 * part) =
                    *reinterpret_cast<const uint2*>(&sm.rows[warp][row][8 * part]);
                if (part == 0) {
                    if constexpr (RECIPE)
                        *reinterpret_cast<uint2*>(sub + block_size * ib + 8 * off) = sm.norms[warp][row];
                    else
                        *reinterpret_cast<uint32_t*>(sub + block_size * ib + 4 * off) = sm.norms[warp][row].x;
                }
            } else if (slot >= capacity && part == 0 && d_err) {
                atomicOr(d_err, TQ_DERR_SLOT);
            }
        }
        __syncwarp();
    }
}

}  // namespace

// Launches a tensor-core pack (uniform 4-bit, another plain format, or a group-wise
// format); TQ_ERR_UNSUPPORTED when one of the two codecs has none.
tq_status launch_pack_tc(const tq_codec* kc, const tq_codec* vc, const void* k, const void* v,
                         const int64_t* slot_mapping, int64_t num_tokens, void* k_pages, void* v_pages,
                         int64_t num_blocks, int32_t block_size, int32_t* d_err, void* stream) {
    // Uniform 4-bit K and V: the 4-bit kernel. Otherwise one launch per codec: plain formats (no QJL
    // stage, no group-wise rotation) and group-wise formats without the QJL stage, with groups of
    // 4 bits on 64 channels and 3 on 64, or 4 bits on 32 and 2 on 96 (plain also uniform 3 and 4
    // bits); QJL formats (without group-wise rotation) of 3 bits on 64 channels and 2 on 64, 4 on 64
    // and 3 on 64, or uniform 3 or 2 bits.
    // Recipe rows (group-wise rotation with each group's QJL stage) of 3 bits on 64 channels and 2 on
    // 64, or 4 and 3.
    enum Kind { kNone, kU4, kU3, kM43, kM42, kGw43, kGw42, kQ32, kQ43, kQu3, kQu2, kR32, kR43 };
    Kind kind[2];
    bool u4 = true;
    for (int side = 0; side < 2; ++side) {
        const tq_format_desc& d = (side ? vc : kc)->desc;
        if (d.n_groups != 1 || d.group_bits[0] != 4 || d.qjl || d.groupwise) u4 = false;
        const bool m43 = d.n_groups == 2 && d.group_bits[0] == 4 && d.group_size[0] == 64 && d.group_bits[1] == 3;
        const bool m42 = d.n_groups == 2 && d.group_bits[0] == 4 && d.group_size[0] == 32 && d.group_bits[1] == 2;
        const bool m32 = d.n_groups == 2 && d.group_bits[0] == 3 && d.group_size[0] == 64 && d.group_bits[1] == 2;
        Kind kd = kNone;
        if (!(side ? vc : kc)->dev.cells) kd = kNone;
        else if (d.qjl && d.groupwise) kd = m32 ? kR32 : (m43 ? kR43 : kNone);
        else if (d.qjl)
            kd = m32 ? kQ32
                     : (m43 ? kQ43
                            : (d.n_groups == 1 && d.group_bits[0] == 3
                                   ? kQu3
                                   : (d.n_groups == 1 && d.group_bits[0] == 2 ? kQu2 : kNone)));
        else if (d.groupwise) kd = m43 ? kGw43 : (m42 ? kGw42 : kNone);
        else if (d.n_groups == 1 && d.group_bits[0] == 4) kd = kU4;
        else if (d.n_groups == 1 && d.group_bits[0] == 3) kd = kU3;
        else kd = m43 ? kM43 : (m42 ? kM42 : kNone);
        kind[side] = kd;
    }
    if (kind[0] == kNone || kind[1] == kNone) return TQ_ERR_UNSUPPORTED;
    // 16-byte copies of the input rows (cp.async) and 8-byte row stores: the general kernel takes
    // inputs or pools aligned only as the call requires (8 and 2 bytes).
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) return TQ_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(k_pages) | reinterpret_cast<uintptr_t>(v_pages)) & 15) return TQ_ERR_UNSUPPORTED;
    if (block_size % 8 != 0) return TQ_ERR_UNSUPPORTED;  // 16-byte aligned rows and norm arrays
    // 32-bit index arithmetic in the kernel: slots, tokens and work units must fit.
    const int64_t capacity = num_blocks * block_size;
    const int H = kc->desc.num_kv_heads;
    const int64_t n_units = (num_tokens + 15) / 16 * H * 2;
    if (capacity > INT32_MAX || n_units > INT32_MAX || num_tokens > INT32_MAX - 16) return TQ_ERR_UNSUPPORTED;
    const int bs_log2 = (block_size & (block_size - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(block_size)) : -1;
    // The kernels' shared-memory sizes are set once per device.
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(TQ_ERR_CUDA, "cudaGetDevice failed");
    const cudaError_t err = once_per_device(dev, [] {
        cudaError_t e = cudaFuncSetAttribute(pack_u4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(sizeof(PackSmem)));
        for (auto kern : {pack_tc_kernel<PU4, false>, pack_tc_kernel<PU3, false>, pack_tc_kernel<PM43, false>,
                          pack_tc_kernel<PM42, false>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(PackTcSmem)));
        for (auto kern : {pack_tc_kernel<PM32, true>, pack_tc_kernel<PM43, true>, pack_tc_kernel<PU3, true>,
                          pack_tc_kernel<PU2, true>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(PackQjlSmem)));
        for (auto kern : {pack_gw_kernel<PM43, false>, pack_gw_kernel<PM42, false>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(PackGwSmem)));
        for (auto kern : {pack_gw_kernel<PM32, true>, pack_gw_kernel<PM43, true>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(PackRecipeSmem)));
        return e;
    });
    if (err != cudaSuccess) return fail(TQ_ERR_CUDA, "pack fast path setup failed");
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (u4) {
        // The quantizer cell table comes with the K codec (every uniform 4-bit codebook is the same).
        const int64_t want = (n_units + kPW - 1) / kPW;
        const int grid = static_cast<int>(want < sms ? want : sms);
        pack_u4_kernel<<<grid, kPW * 32, sizeof(PackSmem), st>>>(
            kc->dev, vc->dev, kc->dev.cells, static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), slot_mapping, static_cast<int>(num_tokens),
            static_cast<uint8_t*>(k_pages), static_cast<uint8_t*>(v_pages), static_cast<int>(capacity), block_size,
            bs_log2, d_err);
        return TQ_OK;
    }
    // One launch per codec. Plain kernels: the grid covers that codec's units (half of the pair's).
    // Group-wise kernels: CTAs keep one KV head, as many per head as fill the SMs (at least one).
    const int64_t tgroups = (num_tokens + 15) / 16;
    const int64_t want1 = (tgroups * H + kPW - 1) / kPW;
    const int grid1 = static_cast<int>(want1 < sms ? want1 : sms);
    constexpr int kQW = TcShape<true>::W;
    const int64_t wantq = (tgroups * H + kQW - 1) / kQW;
    const int gridq = static_cast<int>(wantq < sms ? wantq : sms);
    constexpr int kRW = PackGwSmemBase<true>::W;
    const int64_t per_head_fit = sms / H > 0 ? sms / H : 1;
    auto per_head = [&](int warps) {
        const int64_t want = (tgroups + warps - 1) / warps;
        return static_cast<int>(want < per_head_fit ? want : per_head_fit);
    };
    const struct { const tq_codec* c; const void* x; void* pages; } sides[2] = {{kc, k, k_pages}, {vc, v, v_pages}};
    for (int side = 0; side < 2; ++side) {
        const auto& sd = sides[side];
        auto go = [&](auto kernel, int grid, size_t smem, int warps = kPW) {
            kernel<<<grid, warps * 32, smem, st>>>(sd.c->dev, static_cast<const __nv_bfloat16*>(sd.x), slot_mapping,
                                                 static_cast<int>(num_tokens), static_cast<uint8_t*>(sd.pages),
                                                 static_cast<int>(capacity), block_size, bs_log2, d_err);
        };
        switch (kind[side]) {
            case kU4: go(pack_tc_kernel<PU4, false>, grid1, sizeof(PackTcSmem)); break;
            case kU3: go(pack_tc_kernel<PU3, false>, grid1, sizeof(PackTcSmem)); break;
            case kM43: go(pack_tc_kernel<PM43, false>, grid1, sizeof(PackTcSmem)); break;
            case kM42: go(pack_tc_kernel<PM42, false>, grid1, sizeof(PackTcSmem)); break;
            case kQ32: go(pack_tc_kernel<PM32, true>, gridq, sizeof(PackQjlSmem), kQW); break;
            case kQ43: go(pack_tc_kernel<PM43, true>, gridq, sizeof(PackQjlSmem), kQW); break;
            case kQu3: go(pack_tc_kernel<PU3, true>, gridq, sizeof(PackQjlSmem), kQW); break;
            case kQu2: go(pack_tc_kernel<PU2, true>, gridq, sizeof(PackQjlSmem), kQW); break;
            case kGw43: go(pack_gw_kernel<PM43, false>, per_head(kPW) * H, sizeof(PackGwSmem)); break;
            case kGw42: go(pack_gw_kernel<PM42, false>, per_head(kPW) * H, sizeof(PackGwSmem)); break;
            case kR32: go(pack_gw_kernel<PM32, true>, per_head(kRW) * H, sizeof(PackRecipeSmem), kRW); break;
            case kR43: go(pack_gw_kernel<PM43, true>, per_head(kRW) * H, sizeof(PackRecipeSmem), kRW); break;
            default: break;
        }
    }
    return TQ_OK;
}

}  // namespace tq

// Tensor-core decode partials over packed pages (sm_100a, mma.sync m16n8k16).
//
// Same computation as the general decode kernel (TurboQuant "Design" page,
// "Serving Route Design": K rows are read inside the score computation, V rows
// are read and dequantized inside the accumulation), arranged so that the G
// query heads of one KV head share every page read:
//
//   S  = Q' K^T   A = Q' (16 rows: 8 query heads x {hi, lo} fp16 halves of the
//                 rotated, scaled query), B = dequantized K of 8 tokens
//   O += P' V     A = P' (rows: heads x {hi, lo} of softmax weight x V norm),
//                 B = dequantized V of 16 tokens, 8 rotated coordinates a tile
//
// Splitting each fp32 operand into an fp16 pair keeps the products within
// 2^-22 of fp32 while the centroids themselves are fp16-exact, so the only
// rounding beyond fp32 accumulation is in the operands' second halves.
//
// Dequantization never leaves registers: a 64 KB shared-memory table maps a
// byte of two 4-bit indices (or a 6-bit pair of 3-bit indices, or 4 bits of
// two 2-bit indices) to the fp16 centroid pair that is the MMA operand. The
// table is replicated per lane (entry e of lane l at e*256 + l*4), so lookups
// are bank-conflict free, and it sits on a 64 KB boundary so one prmt turns an
// index byte and the lane offset into the lookup address.
//
// Each CTA is persistent and loops over work items (sequence, KV head, split
// of the packed tokens, query-head group); its 8 warps take 16-token tiles of
// the item in turn, keep one tile of loads in flight in registers and ask L2
// for the tile after that, then merge their (max, sum, accumulator) states and
// write one record per query head for the combine kernel.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kNW = 8;         // warps per CTA
constexpr int kRows = 8;       // query heads per work item (MMA rows: 8 heads x {hi, lo})
constexpr int kLut = 65536;    // bytes of the dequantization table

template <int B0_, int N0_, int B1_, int N1_>
struct Fmt {
    static constexpr int B0 = B0_, N0 = N0_, B1 = B1_, N1 = N1_;
    static constexpr int IB = (B0 * N0 + B1 * N1) / 8;  // index bytes of a row
    static constexpr int BOFF1 = B0 * N0 / 8;           // byte offset of group 1
    static constexpr int KS0 = N0 / 16, KS1 = N1 / 16;  // score k-steps per group
    static constexpr int NT0 = N0 / 8, NT1 = N1 / 8;    // value n-tiles per group
    static constexpr int KC0 = N0 / 4 * B0 / 8;         // score side: bytes of group 0 per lane
    static constexpr int KC1 = N1 / 4 * B1 / 8;
    static constexpr int VC0 = N0 / 8 * B0 / 8;         // value side: bytes of group 0 per lane
    static constexpr int VC1 = N1 / 8 * B1 / 8;
    static_assert(KS0 + KS1 == 8 && NT0 + NT1 == 16, "head_dim 128");
};
using U4 = Fmt<4, 128, 0, 0>;
using U3 = Fmt<3, 128, 0, 0>;
using M43 = Fmt<4, 64, 3, 64>;
using M42 = Fmt<4, 32, 2, 96>;

// Compile-time loop: f(std::integral_constant<int, I>) for I in [B, E).
template <int B, int E, class F>
__device__ __forceinline__ void static_for(F&& f) {
    if constexpr (B < E) {
        f(std::integral_constant<int, B>{});
        static_for<B + 1, E>(f);
    }
}

template <int N>
struct Words {
    uint32_t w[N > 0 ? N : 1];
};

struct LutValues {
    float c4[16], c3[8], c2[4];
};

// ---- PTX helpers --------------------------------------------------------------

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Table lookup. Not volatile: every address derives from the lane base, which
// is produced after the barrier that follows the table fill.
__device__ __forceinline__ uint32_t lut(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t ldg32(const uint8_t* p) { return __ldg(reinterpret_cast<const uint32_t*>(p)); }

// NB bytes at p (p 4-byte aligned when ALIGNED, else only 1-byte) into words,
// little endian. The unaligned form reads up to 3 bytes past the span; every
// caller's span is followed by more bytes of the same sub-page.
template <int NB, bool ALIGNED>
__device__ __forceinline__ Words<(NB + 3) / 4> load_span(const uint8_t* p) {
    constexpr int NW = (NB + 3) / 4;
    Words<NW> r;
    if constexpr (ALIGNED) {
        if constexpr (NB == 16) {
            uint4 x = __ldg(reinterpret_cast<const uint4*>(p));
            r.w[0] = x.x; r.w[1] = x.y; r.w[2] = x.z; r.w[3] = x.w;
        } else if constexpr (NB == 8) {
            uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
            r.w[0] = x.x; r.w[1] = x.y;
        } else {
#pragma unroll
            for (int i = 0; i < NW; ++i) r.w[i] = ldg32(p + 4 * i);
        }
    } else {
        const uintptr_t a = reinterpret_cast<uintptr_t>(p);
        const uint8_t* base = reinterpret_cast<const uint8_t*>(a & ~uintptr_t(3));
        const uint32_t sh = static_cast<uint32_t>(a & 3) * 8;
        uint32_t raw[NW + 1];
#pragma unroll
        for (int i = 0; i <= NW; ++i) raw[i] = ldg32(base + 4 * i);
#pragma unroll
        for (int i = 0; i < NW; ++i) r.w[i] = __funnelshift_r(raw[i], raw[i + 1], sh);
    }
    return r;
}

// Lookup address of the index pair at bits [off, off + 2B) of `w` (a lane's chunk).
template <int B, int OFF, int NW>
__device__ __forceinline__ uint32_t pair_addr(const uint32_t (&w)[NW], uint32_t base) {
    constexpr int WI = OFF / 32, SH = OFF % 32, WIDTH = 2 * B;
    if constexpr (B == 4) {
        static_assert(SH % 8 == 0, "4-bit pairs are whole bytes");
        return prmt(w[WI], base, 0x7604u | ((SH / 8) << 4));
    } else {
        constexpr uint32_t MASK = ((1u << WIDTH) - 1u) << 8;
        uint32_t x;
        if constexpr (SH + WIDTH > 32) {
            x = __funnelshift_r(w[WI], w[WI + 1], SH) << 8;
        } else if constexpr (SH >= 8) {
            x = w[WI] >> (SH - 8);
        } else {
            x = w[WI] << (8 - SH);
        }
        return (x & MASK) | base;
    }
}

// ---- one 16-token tile: what a lane loads ---------------------------------------

template <class KF, class VF>
struct Tile {
    // score side: tokens r and 8 + r, each group's chunk of this lane (c)
    Words<(KF::KC0 + 3) / 4> k0[2];
    Words<(KF::KC1 + 3) / 4> k1[2];
    // value side: tokens 2c, 2c+1, 2c+8, 2c+9, each group's chunk of this lane (r)
    Words<(VF::VC0 + 3) / 4> v0[4];
    Words<(VF::VC1 + 3) / 4> v1[4];
    uint32_t nk[2], nv[2];  // fp16 norm pairs of tokens (2c, 2c+1) and (2c+8, 2c+9)
};

template <class KF, class VF>
__device__ __forceinline__ void load_tile(Tile<KF, VF>& t, const uint8_t* ksub, const uint8_t* vsub, int off,
                                          int block_size, int r, int c) {
    constexpr bool KA0 = KF::KC0 % 4 == 0, KA1 = (KF::KC1 % 4 == 0) && (KF::BOFF1 % 4 == 0);
    constexpr bool VA0 = VF::VC0 % 4 == 0, VA1 = (VF::VC1 % 4 == 0) && (VF::BOFF1 % 4 == 0);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint8_t* row = ksub + (off + r + 8 * i) * KF::IB;
        t.k0[i] = load_span<KF::KC0, KA0>(row + c * KF::KC0);
        if constexpr (KF::N1 > 0) t.k1[i] = load_span<KF::KC1, KA1>(row + KF::BOFF1 + c * KF::KC1);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int tok = 2 * c + (i & 1) + 8 * (i >> 1);
        const uint8_t* row = vsub + (off + tok) * VF::IB;
        t.v0[i] = load_span<VF::VC0, VA0>(row + r * VF::VC0);
        if constexpr (VF::N1 > 0) t.v1[i] = load_span<VF::VC1, VA1>(row + VF::BOFF1 + r * VF::VC1);
    }
    const uint8_t* kn = ksub + block_size * KF::IB + 2 * (off + 2 * c);
    const uint8_t* vn = vsub + block_size * VF::IB + 2 * (off + 2 * c);
    t.nk[0] = ldg32(kn);
    t.nk[1] = ldg32(kn + 16);
    t.nv[0] = ldg32(vn);
    t.nv[1] = ldg32(vn + 16);
}

// ---- score side: B fragments of one group for one token ---------------------------

template <int B, int KS, int NW, int S0>
__device__ __forceinline__ void score_group(float (&acc)[4], const uint32_t (&qa)[8][4], const uint32_t (&w)[NW],
                                           uint32_t base) {
    static_for<0, KS>([&](auto si) {
        constexpr int s = decltype(si)::value;
        const uint32_t b0 = lut(pair_addr<B, (4 * s) * B, NW>(w, base));
        const uint32_t b1 = lut(pair_addr<B, (4 * s + 2) * B, NW>(w, base));
        mma16816(acc, qa[S0 + s], b0, b1);
    });
}

// ---- value side: token-pair fields of one group -----------------------------------

// Interleave the chunks of two tokens so that each field holds (index of t0,
// index of t1) at the same position: even positions in e, odd ones in o.
template <int B, int NW>
__device__ __forceinline__ void interleave(const uint32_t (&a)[NW], const uint32_t (&b)[NW], uint32_t (&e)[NW],
                                           uint32_t (&o)[NW]) {
    if constexpr (B == 4) {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            e[i] = (a[i] & 0x0F0F0F0Fu) | ((b[i] << 4) & 0xF0F0F0F0u);
            o[i] = ((a[i] >> 4) & 0x0F0F0F0Fu) | (b[i] & 0xF0F0F0F0u);
        }
    } else if constexpr (B == 2) {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            e[i] = (a[i] & 0x33333333u) | ((b[i] << 2) & 0xCCCCCCCCu);
            o[i] = ((a[i] >> 2) & 0x33333333u) | (b[i] & 0xCCCCCCCCu);
        }
    } else {  // B == 3: fields of 3 bits; chunks of 24 or 48 bits
        static_assert(NW == 1 || NW == 2, "3-bit value chunks are 3 or 6 bytes");
        if constexpr (NW == 1) {
            constexpr uint32_t M = 0x1C71C7u;  // bits of fields 0, 2, 4, 6
            e[0] = (a[0] & M) | ((b[0] << 3) & (M << 3));
            o[0] = ((a[0] >> 3) & M) | (b[0] & (M << 3));
        } else {
            const uint64_t A = (uint64_t(a[1]) << 32) | a[0], Bw = (uint64_t(b[1]) << 32) | b[0];
            constexpr uint64_t M = 0x1C71C71C71C7ull;
            const uint64_t E = (A & M) | ((Bw << 3) & (M << 3));
            const uint64_t O = ((A >> 3) & M) | (Bw & (M << 3));
            e[0] = static_cast<uint32_t>(E);
            e[1] = static_cast<uint32_t>(E >> 32);
            o[0] = static_cast<uint32_t>(O);
            o[1] = static_cast<uint32_t>(O >> 32);
        }
    }
}

// Lookup address of position Q's token pair in the interleaved words.
template <int B, int Q, int NW>
__device__ __forceinline__ uint32_t vpair_addr(const uint32_t (&e)[NW], const uint32_t (&o)[NW], uint32_t base) {
    if constexpr (B == 4) {
        constexpr int WI = Q / 8, BYTE = (Q % 8) / 2;
        const uint32_t w = (Q & 1) ? o[WI] : e[WI];
        return prmt(w, base, 0x7604u | (BYTE << 4));
    } else {
        constexpr int F = 2 * B;  // field width of the pair
        constexpr int OFF = (Q / 2) * F;
        const uint32_t(&w)[NW] = (Q & 1) ? o : e;
        return pair_addr<B, OFF, NW>(w, base);  // pair_addr reads a 2B-bit field at OFF
    }
}

template <int B, int NT, int NW, int Q0>
__device__ __forceinline__ void value_group(float (&o)[16][4], const uint32_t (&pa)[4], const uint32_t (&t0)[NW],
                                            const uint32_t (&t1)[NW], const uint32_t (&t2)[NW],
                                            const uint32_t (&t3)[NW], uint32_t base) {
    uint32_t e01[NW], o01[NW], e23[NW], o23[NW];
    interleave<B, NW>(t0, t1, e01, o01);
    interleave<B, NW>(t2, t3, e23, o23);
    static_for<0, NT>([&](auto qi) {
        constexpr int q = decltype(qi)::value;
        const uint32_t b0 = lut(vpair_addr<B, q, NW>(e01, o01, base));
        const uint32_t b1 = lut(vpair_addr<B, q, NW>(e23, o23, base));
        mma16816(o[Q0 + q], pa, b0, b1);
    });
}

template <int B>
__device__ __forceinline__ uint32_t lut_base(uint32_t lane_base) {
    return B == 4 ? lane_base : (B == 3 ? (lane_base | 128u) : (lane_base | 0x4080u));
}

// ---- the kernel ----------------------------------------------------------------

struct Smem {
    float qs[kRows][kHeadDim];             // rotated, scaled query in K packed order
    float red_o[kNW][kRows][kHeadDim];     // per-warp value accumulators (V packed order)
    float red_m[kNW][kRows], red_l[kNW][kRows];
};

constexpr size_t kSmemBytes = sizeof(Smem) + 2 * kLut;  // table plus room to align it to 64 KB

template <class KF, class VF>
__global__ void __launch_bounds__(kNW * 32, 1) decode_mma_kernel(DecodeArgs a, LutValues tv, int group,
                                                                 int head_groups, int64_t total_slots) {
    extern __shared__ __align__(16) uint8_t dsm[];
    Smem& sm = *reinterpret_cast<Smem*>(dsm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;

    // Dequantization table on the first 64 KB boundary after Smem.
    const uint32_t dsm_addr = static_cast<uint32_t>(__cvta_generic_to_shared(dsm));
    const uint32_t lut_addr = (dsm_addr + static_cast<uint32_t>(sizeof(Smem)) + (kLut - 1)) & ~uint32_t(kLut - 1);
    if (lut_addr + kLut > dsm_addr + kSmemBytes) return;  // cannot happen with kSmemBytes; no access outside
    uint32_t* table = reinterpret_cast<uint32_t*>(dsm + (lut_addr - dsm_addr));
    for (int i = threadIdx.x; i < kLut / 4; i += kNW * 32) {
        const int e = i >> 6, half = (i >> 5) & 1;
        __half2 v = __floats2half2_rn(0.0f, 0.0f);
        if (half == 0) {
            v = __floats2half2_rn(tv.c4[e & 15], tv.c4[e >> 4]);
        } else if (e < 64) {
            v = __floats2half2_rn(tv.c3[e & 7], tv.c3[e >> 3]);
        } else if (e < 80) {
            v = __floats2half2_rn(tv.c2[(e - 64) & 3], tv.c2[(e - 64) >> 2]);
        }
        table[i] = *reinterpret_cast<uint32_t*>(&v);
    }
    __syncthreads();
    uint32_t lane_base;
    asm volatile("or.b32 %0, %1, %2;" : "=r"(lane_base) : "r"(lut_addr), "r"(static_cast<uint32_t>(lane) << 2));

    const int H = a.kc.num_heads, bs = a.block_size;
    const int rows = group < kRows ? group : kRows;  // query heads of one work item
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);

    for (int64_t slot = blockIdx.x; slot < total_slots; slot += gridDim.x) {
        // slot = ((split * B + b) * H + h) * head_groups + hg
        int64_t t = slot;
        const int hg = static_cast<int>(t % head_groups);
        t /= head_groups;
        const int h = static_cast<int>(t % H);
        t /= H;
        const int b = static_cast<int>(t % a.batch);
        const int split = static_cast<int>(t / a.batch);
        int L = a.seq_lens[b];
        if (L < 0 || L > a.max_seq_len) {
            if (a.d_err && threadIdx.x == 0) atomicOr(a.d_err, TQ_DERR_BLOCK);
            L = L < 0 ? 0 : a.max_seq_len;
        }
        const int n_win = min(a.window, L), P = L - n_win;
        const int ns = (P + a.split_tokens - 1) / a.split_tokens;
        const bool is_win = split == a.max_splits;
        if (is_win ? n_win == 0 : split >= ns) continue;
        const int t0 = is_win ? 0 : split * a.split_tokens;
        const int t1 = is_win ? n_win : min(P, t0 + a.split_tokens);
        const int head0 = h * group + hg * kRows;  // first query head of this item

        // Query prep: warp g rotates query head g (score side) or scales it (window).
        if (warp < rows) {
            const __nv_bfloat16* qp = q + (static_cast<int64_t>(b) * a.num_q_heads + head0 + warp) * kHeadDim;
            const uint2 raw = *reinterpret_cast<const uint2*>(qp + 4 * lane);
            float z[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                          __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u)};
            if (is_win) {
#pragma unroll
                for (int i = 0; i < 4; ++i) sm.qs[warp][4 * lane + i] = z[i] * a.scale_log2;
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) z[i] *= a.kc.sign[4 * lane + i];
                {
                    const float p0 = z[0] + z[1], p1 = z[0] - z[1], p2 = z[2] + z[3], p3 = z[2] - z[3];
                    z[0] = p0 + p2;
                    z[2] = p0 - p2;
                    z[1] = p1 + p3;
                    z[3] = p1 - p3;
                }
#pragma unroll
                for (int m = 1; m < 32; m <<= 1)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float p = __shfl_xor_sync(kFull, z[i], m);
                        z[i] = (lane & m) ? (p - z[i]) : (z[i] + p);
                    }
                const float sc = a.scale_log2 * 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
                for (int i = 0; i < 4; ++i) sm.qs[warp][a.kc.pos[h * kHeadDim + 4 * lane + i]] = z[i] * sc;
            }
        }
        __syncthreads();

        if (is_win) {
            // Dense bf16 window: CUDA cores, tokens spread over the warps.
            float m[kRows], l[kRows], acc[kRows][4];
#pragma unroll
            for (int g = 0; g < kRows; ++g) {
                m[g] = -INFINITY;
                l[g] = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[g][i] = 0.0f;
            }
            const __nv_bfloat16* kw = static_cast<const __nv_bfloat16*>(a.k_win);
            const __nv_bfloat16* vw = static_cast<const __nv_bfloat16*>(a.v_win);
            for (int tk = t0 + warp; tk < t1; tk += kNW) {
                const int64_t base = ((static_cast<int64_t>(b) * H + h) * a.window + tk) * kHeadDim + 4 * lane;
                const uint2 kr = *reinterpret_cast<const uint2*>(kw + base);
                const uint2 vr = *reinterpret_cast<const uint2*>(vw + base);
                const float kx[4] = {__uint_as_float(kr.x << 16), __uint_as_float(kr.x & 0xffff0000u),
                                     __uint_as_float(kr.y << 16), __uint_as_float(kr.y & 0xffff0000u)};
                const float vx[4] = {__uint_as_float(vr.x << 16), __uint_as_float(vr.x & 0xffff0000u),
                                     __uint_as_float(vr.y << 16), __uint_as_float(vr.y & 0xffff0000u)};
#pragma unroll
                for (int g = 0; g < kRows; ++g) {
                    if (g >= rows) break;
                    float s = 0.0f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) s += sm.qs[g][4 * lane + i] * kx[i];
#pragma unroll
                    for (int mm = 16; mm; mm >>= 1) s += __shfl_xor_sync(kFull, s, mm);
                    const float mn = fmaxf(m[g], s);
                    const float alpha = ex2(m[g] - mn);
                    const float p = ex2(s - mn);
                    l[g] = l[g] * alpha + p;
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[g][i] = acc[g][i] * alpha + p * vx[i];
                    m[g] = mn;
                }
            }
#pragma unroll
            for (int g = 0; g < kRows; ++g) {
                if (g >= rows) break;
                if (lane == 0) {
                    sm.red_m[warp][g] = m[g];
                    sm.red_l[warp][g] = l[g];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) sm.red_o[warp][g][4 * lane + i] = acc[g][i];
            }
        } else {
            // Score-side A fragments (hi/lo halves of the query) for this lane.
            uint32_t qa[8][4];
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const int p = s < KF::KS0 ? c * (KF::N0 / 4) + 4 * s
                                          : KF::N0 + c * (KF::N1 / 4) + 4 * (s - KF::KS0);
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (r < rows) x = *reinterpret_cast<const float4*>(&sm.qs[r][p]);
                const __half2 h01 = __floats2half2_rn(x.x, x.y), h23 = __floats2half2_rn(x.z, x.w);
                const __half2 l01 = __floats2half2_rn(x.x - __low2float(h01), x.y - __high2float(h01));
                const __half2 l23 = __floats2half2_rn(x.z - __low2float(h23), x.w - __high2float(h23));
                qa[s][0] = *reinterpret_cast<const uint32_t*>(&h01);
                qa[s][1] = *reinterpret_cast<const uint32_t*>(&l01);
                qa[s][2] = *reinterpret_cast<const uint32_t*>(&h23);
                qa[s][3] = *reinterpret_cast<const uint32_t*>(&l23);
            }
            float o[16][4];
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
            float m_run = -INFINITY, l_run = 0.0f;

            const int ntiles = (t1 - t0 + 15) >> 4;
            const int64_t bt_row = static_cast<int64_t>(b) * a.max_blocks;
            auto sub_of = [&](int tile, const uint8_t*& ks, const uint8_t*& vs, int& off) {
                const int tk = t0 + 16 * tile;
                int64_t blk = a.block_tables[bt_row + tk / bs];
                if (blk < 0 || blk >= a.num_blocks) {
                    if (a.d_err && lane == 0) atomicOr(a.d_err, TQ_DERR_BLOCK);
                    blk = 0;
                }
                const int64_t sp = (blk * H + h) * bs;
                ks = a.k_pages + sp * (KF::IB + 2);
                vs = a.v_pages + sp * (VF::IB + 2);
                off = tk % bs;
            };

            Tile<KF, VF> cur, nxt;
            int tile = warp;
            if (tile < ntiles) {
                const uint8_t *ks, *vs;
                int off;
                sub_of(tile, ks, vs, off);
                load_tile(cur, ks, vs, off, bs, r, c);
            }
            for (; tile < ntiles; tile += kNW) {
                if (tile + kNW < ntiles) {
                    const uint8_t *ks, *vs;
                    int off;
                    sub_of(tile + kNW, ks, vs, off);
                    load_tile(nxt, ks, vs, off, bs, r, c);
                }
                if (lane == 0 && tile + 2 * kNW < ntiles) {
                    const uint8_t *ks, *vs;
                    int off;
                    sub_of(tile + 2 * kNW, ks, vs, off);
                    prefetch_l2(ks + off * KF::IB, 16 * KF::IB);
                    prefetch_l2(vs + off * VF::IB, 16 * VF::IB);
                    prefetch_l2(ks + bs * KF::IB + 2 * off, 32);
                    prefetch_l2(vs + bs * VF::IB + 2 * off, 32);
                }
                const int nvalid = min(16, t1 - (t0 + 16 * tile));

                // S = Q' K^T for tokens 0..7 (n-tile 0) and 8..15 (n-tile 1).
                float sacc[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.0f;
                    score_group<KF::B0, KF::KS0, (KF::KC0 + 3) / 4, 0>(sacc[nt], qa, cur.k0[nt].w,
                                                                        lut_base<KF::B0>(lane_base));
                    if constexpr (KF::N1 > 0)
                        score_group<KF::B1, KF::KS1, (KF::KC1 + 3) / 4, KF::KS0>(sacc[nt], qa, cur.k1[nt].w,
                                                                                  lut_base<KF::B1>(lane_base));
                }
                // Online softmax of this lane's tokens 2c, 2c+1, 2c+8, 2c+9 (head r).
                const float2 nk01 = __half22float2(*reinterpret_cast<const __half2*>(&cur.nk[0]));
                const float2 nk89 = __half22float2(*reinterpret_cast<const __half2*>(&cur.nk[1]));
                const float2 nv01 = __half22float2(*reinterpret_cast<const __half2*>(&cur.nv[0]));
                const float2 nv89 = __half22float2(*reinterpret_cast<const __half2*>(&cur.nv[1]));
                const bool ok0 = 2 * c < nvalid, ok1 = 2 * c + 1 < nvalid;
                const bool ok2 = 2 * c + 8 < nvalid, ok3 = 2 * c + 9 < nvalid;
                const float s0 = ok0 ? (sacc[0][0] + sacc[0][2]) * nk01.x : -INFINITY;
                const float s1 = ok1 ? (sacc[0][1] + sacc[0][3]) * nk01.y : -INFINITY;
                const float s2 = ok2 ? (sacc[1][0] + sacc[1][2]) * nk89.x : -INFINITY;
                const float s3 = ok3 ? (sacc[1][1] + sacc[1][3]) * nk89.y : -INFINITY;
                float mx = fmaxf(fmaxf(s0, s1), fmaxf(s2, s3));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
                const float m_new = fmaxf(m_run, mx);
                if (__any_sync(kFull, m_new > m_run)) {
                    const float alpha = m_new > m_run ? ex2(m_run - m_new) : 1.0f;
                    l_run *= alpha;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        o[i][0] *= alpha;
                        o[i][1] *= alpha;
                        o[i][2] *= alpha;
                        o[i][3] *= alpha;
                    }
                    m_run = m_new;
                }
                const float mref = m_run == -INFINITY ? 0.0f : m_run;
                const float p0 = ex2(s0 - mref), p1 = ex2(s1 - mref), p2 = ex2(s2 - mref), p3 = ex2(s3 - mref);
                l_run += (p0 + p1) + (p2 + p3);
                const float w0 = ok0 ? p0 * nv01.x : 0.0f, w1 = ok1 ? p1 * nv01.y : 0.0f;
                const float w2 = ok2 ? p2 * nv89.x : 0.0f, w3 = ok3 ? p3 * nv89.y : 0.0f;
                const __half2 h01 = __floats2half2_rn(w0, w1), h23 = __floats2half2_rn(w2, w3);
                const __half2 l01 = __floats2half2_rn(w0 - __low2float(h01), w1 - __high2float(h01));
                const __half2 l23 = __floats2half2_rn(w2 - __low2float(h23), w3 - __high2float(h23));
                const uint32_t pa[4] = {*reinterpret_cast<const uint32_t*>(&h01),
                                        *reinterpret_cast<const uint32_t*>(&l01),
                                        *reinterpret_cast<const uint32_t*>(&h23),
                                        *reinterpret_cast<const uint32_t*>(&l23)};
                // O += P' V over the 16 coordinate n-tiles.
                value_group<VF::B0, VF::NT0, (VF::VC0 + 3) / 4, 0>(o, pa, cur.v0[0].w, cur.v0[1].w, cur.v0[2].w,
                                                                   cur.v0[3].w, lut_base<VF::B0>(lane_base));
                if constexpr (VF::N1 > 0)
                    value_group<VF::B1, VF::NT1, (VF::VC1 + 3) / 4, VF::NT0>(
                        o, pa, cur.v1[0].w, cur.v1[1].w, cur.v1[2].w, cur.v1[3].w, lut_base<VF::B1>(lane_base));
                cur = nxt;
            }
            // Publish this warp's state: head r, value positions of columns 2c and 2c+1.
            l_run += __shfl_xor_sync(kFull, l_run, 1);
            l_run += __shfl_xor_sync(kFull, l_run, 2);
            if (r < rows) {
                if (c == 0) {
                    sm.red_m[warp][r] = m_run;
                    sm.red_l[warp][r] = l_run;
                }
#pragma unroll
                for (int qq = 0; qq < 16; ++qq) {
                    const bool g1 = qq >= VF::NT0;
                    const int ql = g1 ? qq - VF::NT0 : qq;
                    const int per = g1 ? VF::N1 / 8 : VF::N0 / 8;
                    const int p0 = (g1 ? VF::N0 : 0) + (2 * c) * per + ql;
                    sm.red_o[warp][r][p0] = o[qq][0] + o[qq][2];
                    sm.red_o[warp][r][p0 + per] = o[qq][1] + o[qq][3];
                }
            }
        }
        __syncthreads();
        // Merge the warps and write one record per query head.
        float* rec = a.ws + ((static_cast<int64_t>(b) * H + h) * a.items_per_unit + split) *
                                static_cast<int64_t>(group) * (kHeadDim + 2);
        for (int e = threadIdx.x; e < rows * kHeadDim; e += kNW * 32) {
            const int g = e / kHeadDim, j = e - g * kHeadDim;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kNW; ++w) M = fmaxf(M, sm.red_m[w][g]);
            float Ls = 0.0f, A = 0.0f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kNW; ++w) {
                    const float f = ex2(sm.red_m[w][g] - M);
                    Ls += sm.red_l[w][g] * f;
                    A += sm.red_o[w][g][j] * f;
                }
            }
            float* rg = rec + (hg * kRows + g) * (kHeadDim + 2);
            rg[2 + j] = A;
            if (j == 0) {
                rg[0] = M;
                rg[1] = Ls;
            }
        }
        __syncthreads();
    }
}

template <class KF, class VF>
tq_status launch_fmt(const DecodeArgs& a, const LutValues& tv, int group, cudaStream_t s) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(decode_mma_kernel<KF, VF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kSmemBytes));
    });
    if (attr_err != cudaSuccess) return fail(TQ_ERR_CUDA, "cannot reserve shared memory for the decode kernel");
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int head_groups = group > kRows ? group / kRows : 1;
    const int64_t slots = static_cast<int64_t>(a.items_per_unit) * a.batch * a.kc.num_heads * head_groups;
    const int grid = static_cast<int>(slots < sms ? slots : sms);
    if (grid > 0)
        decode_mma_kernel<KF, VF><<<grid, kNW * 32, kSmemBytes, s>>>(a, tv, group, head_groups, slots);
    return TQ_OK;
}

template <class F>
bool same_format(const tq_codec* c) {
    const tq_format_desc& d = c->desc;
    if (F::N1 == 0) return d.n_groups == 1 && d.group_bits[0] == F::B0;
    return d.n_groups == 2 && d.group_bits[0] == F::B0 && d.group_size[0] == F::N0 && d.group_bits[1] == F::B1 &&
           d.group_size[1] == F::N1;
}

template <class KF>
tq_status dispatch_v(const DecodeArgs& a, const tq_codec* vc, const LutValues& tv, int group, cudaStream_t s) {
    if (same_format<U4>(vc)) return launch_fmt<KF, U4>(a, tv, group, s);
    if (same_format<M43>(vc)) return launch_fmt<KF, M43>(a, tv, group, s);
    if (same_format<U3>(vc)) return launch_fmt<KF, U3>(a, tv, group, s);
    return TQ_ERR_UNSUPPORTED;
}

}  // namespace

tq_status launch_decode_mma(const DecodeArgs& a, const tq_codec* kc, const tq_codec* vc, int group, void* stream) {
    if (a.block_size % 16 != 0) return TQ_ERR_UNSUPPORTED;
    if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return TQ_ERR_UNSUPPORTED;
    LutValues tv{};
    for (const tq_codec* c : {kc, vc})
        for (int g = 0; g < c->desc.n_groups; ++g) {
            const int bits = c->desc.group_bits[g];
            float* dst = bits == 4 ? tv.c4 : (bits == 3 ? tv.c3 : tv.c2);
            for (int i = 0; i < (1 << bits); ++i) dst[i] = c->cent[g][i];
        }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (same_format<U4>(kc)) return dispatch_v<U4>(a, vc, tv, group, s);
    if (same_format<M43>(kc)) return dispatch_v<M43>(a, vc, tv, group, s);
    if (same_format<M42>(kc)) return dispatch_v<M42>(a, vc, tv, group, s);
    return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq

// Tensor-core decode partials over packed pages (sm_100a).
//
// Same computation as the general decode kernel (TurboQuant "Design" page,
// "Serving Route Design": K rows are read inside the score computation, V rows
// are read and dequantized inside the accumulation), arranged so that the
// query heads of one KV head share every page read. Per 16-token tile a warp
// runs two products on mma.sync m16n8k16 (fp16 operands, fp32 accumulation):
//
//   S^T = K^ Q'^T   rows: 16 tokens; columns: query heads x {hi, lo}
//   O^T += V^T P'^T rows: 16 value coordinates (8 row tiles); same columns
//
// where Q' is the rotated query scaled by softmax_scale*log2(e) and P' the
// softmax weight times the V norm. Each fp32 operand is split into an fp16
// pair (hi + lo) that occupies two columns, which keeps the products within
// 2^-22 of fp32; the centroids are fp16-exact, so K^ and V^ carry no rounding.
//
// Dequantization stays in registers: a 64 KB shared-memory table maps a byte
// of two 4-bit indices (or 6 bits of two 3-bit indices, or 4 bits of two 2-bit
// indices) to the fp16 centroid pair that is one MMA operand register. The
// table is replicated per lane (entry e of lane l at e*256 + l*4) so lookups
// are bank-conflict free, and it starts on a 64 KB boundary so one prmt turns
// an index byte plus the lane offset into the lookup address. For values the
// two indices of a pair come from two tokens at the same coordinate, so the
// lane first interleaves two tokens' index bits.
//
// Data movement: a ninth warp, the producer, fills ring slots in shared memory
// with bulk copies (cp.async.bulk, completion counted on a "full" mbarrier per
// slot) in the order the compute warps consume them; a warp releases a slot
// through an "empty" mbarrier. The producer runs ahead across work items and
// keeps the next item's block ids in shared memory, so the compute warps carry
// no address or block-table arithmetic. Two layouts: with a multiple of 8 KV
// heads a slot is one page block of 8 consecutive heads in both pools (two
// copies of several KB; warp w takes head w), otherwise each warp owns a ring
// of 16-token tiles of one head. (Copies of a few hundred bytes each cost the
// copy engine a fixed overhead per operation that capped the rate well below
// HBM speed; the 8-head slots make every copy large.) Every wait is bounded;
// on expiry the kernel sets TQ_DERR_TIMEOUT, waits for its copies and stops.
// CTAs are persistent and take work items (sequence, KV head or 8 of them,
// split of the packed tokens, query-head group) in a fixed stride.
//
// Online softmax: each warp keeps a reference max per head that moves only
// when a score exceeds it by more than 2^8, so weights stay below 2^8 and the
// common tile needs one vote and no shuffles or rescale.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <type_traits>

#include "tq_internal.h"
#include "tq_pack_vector.cuh"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
#ifndef TQ_DECODE_WARPS
#define TQ_DECODE_WARPS 8
#endif
constexpr int kNW = TQ_DECODE_WARPS;  // compute warps per CTA (plus one producer warp)
static_assert(kNW >= 1 && kNW <= 11, "11 compute warps fill the shared memory");
#ifndef TQ_DECODE_STAGES
#define TQ_DECODE_STAGES 4
#endif
constexpr int kStages = TQ_DECODE_STAGES;  // ring slots per compute warp
constexpr int kLut = 65536;         // bytes of the dequantization table
constexpr uint32_t kSpinLimit = 1u << 24;   // polls of a spinning wait
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bound of one mbarrier wait (global timer, 1 s)
constexpr float kSlack = 8.0f;                 // log2 slack of the running max

#pragma nv_diag_suppress 177  // not every format constant is used by every instantiation
template <int B0_, int N0_, int B1_, int N1_>
struct Fmt {
    static constexpr int B0 = B0_, N0 = N0_, B1 = B1_, N1 = N1_;
    static constexpr int IB = (B0 * N0 + B1 * N1) / 8;  // index bytes of a row
    static constexpr int BOFF1 = B0 * N0 / 8;           // byte offset of group 1
    static constexpr int KS0 = N0 / 16, KS1 = N1 / 16;  // score k-steps per group
    static constexpr int MT0 = N0 / 16, MT1 = N1 / 16;  // value row tiles per group
    static constexpr int KC0 = N0 / 4 * B0 / 8;         // score side: bytes of group 0 per lane
    static constexpr int KC1 = N1 / 4 * B1 / 8;
    static constexpr int VC0 = N0 / 8 * B0 / 8;         // value side: bytes of group 0 per lane
    static constexpr int VC1 = N1 / 8 * B1 / 8;
    static_assert(KS0 + KS1 == 8 && MT0 + MT1 == 8, "head_dim 128");
    static_assert(IB % 4 == 0 && IB <= 64, "index groups of whole words, at most 64 bytes");
};

// What a row holds besides its index groups. Plain: one fp16 norm. Group-wise
// (the high channels are original channels, each group rotated on its own):
// one fp16 norm per group. QJL keys: the 128 residual sign bits after the
// index groups, and the norm followed by the residual norm. The recipe row
// (group-wise with a QJL stage per group): each group's indices followed by
// its sign bits (one per coordinate of the group), and the norms
// (n_0, |r_0|, n_1, |r_1|).
constexpr int kPlain = 0, kGroupwise = 1, kQjl = 2, kRecipe = 3;
template <class F, int MODE_>
struct Row : F {
    static constexpr int MODE = MODE_;
    static constexpr bool SIGNS = MODE_ == kQjl || MODE_ == kRecipe;
    static constexpr int RB = F::IB + (SIGNS ? kHeadDim / 8 : 0);  // bytes of an index row
    static constexpr int NB = MODE_ == kPlain ? 2 : (MODE_ == kRecipe ? 8 : 4);  // bytes of a row's norms
    // group 1's indices follow group 0's signs in the recipe row
    static constexpr int BOFF1 = F::BOFF1 + (MODE_ == kRecipe ? F::N0 / 8 : 0);
    static constexpr int SO0 = F::BOFF1, SO1 = BOFF1 + F::B1 * F::N1 / 8;  // recipe: each group's sign bits
    static constexpr int N1OFF = MODE_ == kRecipe ? 4 : 2;  // byte offset of group 1's norm
};
using U4 = Row<Fmt<4, 128, 0, 0>, kPlain>;
using U3 = Row<Fmt<3, 128, 0, 0>, kPlain>;
using M43 = Row<Fmt<4, 64, 3, 64>, kPlain>;
using M42 = Row<Fmt<4, 32, 2, 96>, kPlain>;
using M32Q = Row<Fmt<3, 64, 2, 64>, kQjl>;
using M43Q = Row<Fmt<4, 64, 3, 64>, kQjl>;
using M43G = Row<Fmt<4, 64, 3, 64>, kGroupwise>;
using M32R = Row<Fmt<3, 64, 2, 64>, kRecipe>;
static_assert(M32R::RB == 56 && M32R::BOFF1 == 32 && M32R::SO0 == 24 && M32R::SO1 == 48, "recipe row layout");

// Bytes of one ring slot: 16 index rows of K followed by their 16 norms, then
// the same for V; a multiple of 16, the copy granule.
template <class KF, class VF>
__host__ __device__ constexpr uint32_t stage_bytes() {
    return 16 * (KF::RB + KF::NB + VF::RB + VF::NB);
}

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

// ---- PTX helpers -----------------------------------------------------------------

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Table lookup (the table is written once, before the barrier that precedes
// the computation of every lookup address).
__device__ __forceinline__ uint32_t lut(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Shared-memory reads of ring data: volatile, so they stay after the wait.
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint64_t pk(float lo, float hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
}
__device__ __forceinline__ void upk(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t add2(uint64_t x, uint64_t y) {
    uint64_t v;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(v) : "l"(x), "l"(y));
    return v;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One wait attempt: the thread may be suspended until phase `parity` of
// `bar` completes or a system-dependent time passes; true when the phase
// completed. (The form without a suspend-time hint measured about 1.5 %
// faster; the hint's length made no difference.)
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait for phase `parity` of `bar`: false when kWaitLimitNs of the
// global timer passed first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

// NB bytes at shared address a (4-byte aligned when ALIGNED) into words.
template <int NB, bool ALIGNED>
__device__ __forceinline__ Words<(NB + 3) / 4> lds_span(uint32_t a) {
    constexpr int NW = (NB + 3) / 4;
    Words<NW> r;
    if constexpr (ALIGNED && NB == 16) {
        const uint4 x = lds128(a);
        r.w[0] = x.x; r.w[1] = x.y; r.w[2] = x.z; r.w[3] = x.w;
    } else if constexpr (ALIGNED && NB == 8) {
        const uint2 x = lds64(a);
        r.w[0] = x.x; r.w[1] = x.y;
    } else if constexpr (ALIGNED) {
#pragma unroll
        for (int i = 0; i < NW; ++i) r.w[i] = lds32(a + 4 * i);
    } else {
        const uint32_t base = a & ~3u, sh = (a & 3u) * 8;
        uint32_t raw[NW + 1];
#pragma unroll
        for (int i = 0; i <= NW; ++i) raw[i] = lds32(base + 4 * i);
#pragma unroll
        for (int i = 0; i < NW; ++i) r.w[i] = __funnelshift_r(raw[i], raw[i + 1], sh);
    }
    return r;
}

// NB bytes at shared address a + off, where a is 4-byte aligned and off is a
// per-lane constant: the alignment split of off (word offset and shift) does
// not depend on a, so the compiler computes it once per lane.
// BASE0 + lane * STEP is the per-lane offset for lanes 0..LANES-1 (a
// compile-time pattern): only as many words are read as the worst of those
// offsets needs.
template <int NB, bool ALIGNED, int BASE0 = 0, int STEP = 0, int LANES = 1>
__device__ __forceinline__ Words<(NB + 3) / 4> lds_span_off(uint32_t a, uint32_t off) {
    if constexpr (ALIGNED) {
        return lds_span<NB, true>(a + off);
    } else {
        constexpr int NW = (NB + 3) / 4;
        constexpr int MIS = [] {
            int m = 0;
            for (int l = 0; l < LANES; ++l) m = ((BASE0 + l * STEP) & 3) > m ? ((BASE0 + l * STEP) & 3) : m;
            return LANES > 1 ? m : 3;
        }();
        constexpr int NR = (MIS + NB + 3) / 4;  // words that hold the span at the worst misalignment
        const uint32_t base = a + (off & ~3u), sh = (off & 3u) * 8;
        Words<NW> r;
        uint32_t raw[NW + 1];
#pragma unroll
        for (int i = 0; i <= NW; ++i) raw[i] = i < NR ? lds32(base + 4 * i) : 0u;
#pragma unroll
        for (int i = 0; i < NW; ++i) r.w[i] = __funnelshift_r(raw[i], raw[i + 1], sh);
        return r;
    }
}

// Lookup address of the index pair at bits [OFF, OFF + 2B) of a lane's chunk.
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

// Transpose of an 8x8 fp16 matrix held one row-pair per lane (lane l: row l / 4,
// columns 2 (l % 4), +1), returned in the same layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Interleave two tokens' chunks: field k of e holds (index of a, index of b)
// at chunk position 2k, field k of o at position 2k + 1.
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
    } else {
        static_assert(NW == 1 || NW == 2, "3-bit value chunks are 3 or 6 bytes");
        if constexpr (NW == 1) {
            constexpr uint32_t M = 0x1C71C7u;  // bits of fields 0, 2, 4, 6
            e[0] = (a[0] & M) | ((b[0] << 3) & (M << 3));
            o[0] = ((a[0] >> 3) & M) | (b[0] & (M << 3));
        } else {
            const uint64_t A = (uint64_t(a[1]) << 32) | a[0], Bv = (uint64_t(b[1]) << 32) | b[0];
            constexpr uint64_t M = 0x1C71C71C71C7ull;
            const uint64_t E = (A & M) | ((Bv << 3) & (M << 3));
            const uint64_t O = ((A >> 3) & M) | (Bv & (M << 3));
            e[0] = static_cast<uint32_t>(E);
            e[1] = static_cast<uint32_t>(E >> 32);
            o[0] = static_cast<uint32_t>(O);
            o[1] = static_cast<uint32_t>(O >> 32);
        }
    }
}

// Lookup address of chunk position Q for an interleaved token pair.
template <int B, int Q, int NW>
__device__ __forceinline__ uint32_t vpair_addr(const uint32_t (&e)[NW], const uint32_t (&o)[NW], uint32_t base) {
    if constexpr (B == 4) {
        constexpr int WI = Q / 8, BYTE = (Q % 8) / 2;
        return prmt((Q & 1) ? o[WI] : e[WI], base, 0x7604u | (BYTE << 4));
    } else {
        constexpr int OFF = (Q / 2) * 2 * B;
        if constexpr (Q & 1) {
            return pair_addr<B, OFF, NW>(o, base);
        } else {
            return pair_addr<B, OFF, NW>(e, base);
        }
    }
}

template <int B>
__device__ __forceinline__ uint32_t lut_base(uint32_t lane_base) {
    return B == 4 ? lane_base : (B == 3 ? (lane_base | 128u) : (lane_base | 0x4080u));
}

// ---- tensor memory (TMEM) as per-warp storage -------------------------------------
//
// The block kernel keeps each warp's query fragments and value accumulators
// in tensor memory between uses instead of in registers: a warp reaches only
// its lane quarter (lanes 32 (warp % 4) .. + 31), thread i lane 32 (warp % 4)
// + i, and the 32x32b shape moves one 32-bit column per register. Loads are
// asynchronous: tm_wait_ld() waits for them, and tm_dep() then ties the
// registers to that wait so that no use is scheduled before it.

__device__ __forceinline__ void tm_ld4(uint32_t taddr, uint32_t* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr));
}
__device__ __forceinline__ void tm_st4(uint32_t taddr, const uint32_t* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
                 :
                 : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}
__device__ __forceinline__ void tm_dep4(uint32_t* v) {
    asm volatile("" : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]));
}
__device__ __forceinline__ void tm_ld16(uint32_t taddr, uint32_t* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tm_st16(uint32_t taddr, const uint32_t* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
                 :
                 : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
                 : "memory");
}
__device__ __forceinline__ void tm_dep16(uint32_t* v) {
    asm volatile("" : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]));
}
__device__ __forceinline__ void tm_ld32(uint32_t taddr, uint32_t* v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                 : "r"(taddr));
}
__device__ __forceinline__ void tm_st32(uint32_t taddr, const uint32_t* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 :
                 : "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
                 : "memory");
}
__device__ __forceinline__ void tm_dep32(uint32_t* v) {
    asm volatile("" : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]), "+r"(v[30]), "+r"(v[31]));
}
__device__ __forceinline__ void tm_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tm_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tm_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tm_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void tm_ld(uint32_t taddr, uint32_t* v) {
    static_assert(N == 4 || N == 16 || N == 32, "tm_ld width");
    if constexpr (N == 4) tm_ld4(taddr, v);
    else if constexpr (N == 16) tm_ld16(taddr, v);
    else tm_ld32(taddr, v);
}
template <int N>
__device__ __forceinline__ void tm_st(uint32_t taddr, const uint32_t* v) {
    static_assert(N == 4 || N == 16 || N == 32, "tm_st width");
    if constexpr (N == 4) tm_st4(taddr, v);
    else if constexpr (N == 16) tm_st16(taddr, v);
    else tm_st32(taddr, v);
}
template <int N>
__device__ __forceinline__ void tm_dep(uint32_t* v) {
    if constexpr (N == 4) tm_dep4(v);
    else if constexpr (N == 16) tm_dep16(v);
    else tm_dep32(v);
}

// ---- work items -----------------------------------------------------------------

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream still runs;
// griddep_wait() returns once that kernel has completed and its writes are
// visible, so nothing it writes is read before. griddep_launch_dependents()
// lets the next such kernel start.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

struct Item {
    int b, h, hg, split, t0, t1;  // h: the KV head (per-head items) or the first of 8 (block items)
    bool win;
};

// Token range of item `split` of sequence it.b; false when it has no tokens.
__device__ __forceinline__ bool item_range(const DecodeArgs& a, Item& it) {
    int L = __ldg(a.seq_lens + it.b);
    L = L < 0 ? 0 : (L > a.max_seq_len ? a.max_seq_len : L);
    const int n_win = min(a.window, L), P = L - n_win;
    const int ns = (P + a.split_tokens - 1) / a.split_tokens;
    it.win = it.split == a.max_splits;
    if (it.win ? n_win == 0 : it.split >= ns) return false;
    it.t0 = it.win ? 0 : it.split * a.split_tokens;
    it.t1 = it.win ? n_win : min(P, it.t0 + a.split_tokens);
    return true;
}

// Work slot -> item. CTA c takes slots c, c + grid, c + 2 grid, ...; slot
// r * grid + c stands for list position q = r * grid + c in even rounds r and
// r * grid + (n_r - 1 - c) in odd ones (n_r: the slots of round r), so the
// longest-first list is dealt in snake order. Position q = (k * hblocks + j) *
// head_groups + hg is entry k of the work list (sequence, split), KV heads
// from j * HB (HB = 8 for block items, else 1) and query-head group hg.
template <int HB>
__device__ __forceinline__ bool item_of(const DecodeArgs& a, int64_t slot, int head_groups, int64_t total_slots,
                                        Item& it) {
    const int hblocks = a.kc.num_heads / HB;
    const int64_t grid = gridDim.x, r = slot / grid, c = slot - r * grid;
    const int64_t n_r = total_slots - r * grid < grid ? total_slots - r * grid : grid;
    int64_t t = r * grid + ((r & 1) ? n_r - 1 - c : c);
    it.hg = static_cast<int>(t % head_groups);
    t /= head_groups;
    it.h = static_cast<int>(t % hblocks) * HB;
    t /= hblocks;
    const int2 e = __ldg(reinterpret_cast<const int2*>(a.work_list) + t);
    it.b = e.x;
    it.split = e.y;
    return item_range(a, it);
}

// Slots of this call: the listed items times the head blocks and groups,
// at most the launch's bound.
template <int HB>
__device__ __forceinline__ int64_t listed_slots(const DecodeArgs& a, int head_groups, int64_t bound) {
    const int64_t n = static_cast<int64_t>(__ldg(a.work_count)) * (a.kc.num_heads / HB) * head_groups;
    return n < bound ? n : bound;
}

// Next packed item of this CTA at or after `slot`; false when none is left.
template <int HB>
__device__ __forceinline__ bool next_packed(const DecodeArgs& a, int64_t& slot, int head_groups, int64_t total_slots,
                                            Item& it) {
    for (; slot < total_slots; slot += gridDim.x)
        if (item_of<HB>(a, slot, head_groups, total_slots, it) && !it.win) return true;
    return false;
}

constexpr int kMaxItemTiles = 256;  // 16-token tiles of one work item (at most)

// ---- synchronisation and copies ----------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init_count(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
template <int NTHREADS>
__device__ __forceinline__ void named_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(NTHREADS) : "memory");
}

__device__ __forceinline__ uint64_t mul2(uint64_t x, uint64_t y) {
    uint64_t v;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(v) : "l"(x), "l"(y));
    return v;
}
__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}
// fp16 split of a float pair: hi = rn(x), lo = rn(x - hi) per element.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = half2_bits(x0 - __low2float(h), x1 - __high2float(h));
}
__device__ __forceinline__ float f16_at(uint32_t addr) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(lds16(addr))));
}

// Fills the per-lane dequantization table (see the top of the file).
__device__ __forceinline__ void fill_table(uint32_t* table, const LutValues& tv, int tid, int nthreads) {
    for (int i = tid; i < kLut / 4; i += nthreads) {
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
}

// ---- one warp's attention state over packed tiles -------------------------------------

// NH = 8: the 8 columns of every MMA are 8 query heads, and the fp16 hi and lo
// halves of the fp32 operand (Q' or P') are two MMAs into the same
// accumulator; a lane holds heads 2c and 2c + 1. NH = 4: columns 2h and 2h + 1
// are the hi and lo halves of head h (4 heads), summed after the MMA; a lane
// holds head c. Lane (r, c) = (lane / 4, lane % 4).
//
// Group-wise K: the score k-steps of each group accumulate apart and take that
// group's norm. Group-wise V: the value row tiles of group 1 take P' built with
// the group-1 norms. QJL keys: 8 more k-steps per tile score the sign bits
// against the projected query (the A operand is +-|r| per token, exact in
// fp16); they land in the same accumulators as the index groups, so the
// token's score is n (q'.c + sqrt(pi/2)/128 |r| (S q').z) before the norm.
//
// TM: the query fragments and the value accumulators live in this warp's
// tensor-memory columns between uses (query fragments at kTmQ, QJL fragments
// at kTmZ, accumulators at kTmO, the merge state at kTmS) and in registers
// only inside scores() and values(), so the two sets are never live at once.
// Where the prologue stores projection i of the projected query, so that a
// lane's four B-fragment values of a sign k-step are one 16-byte load. QJL
// keys: lane c's k-step s takes projections 32c + s + (0, 16, 8, 24), stored
// at 32c + 4s + (0, 1, 2, 3). Recipe keys: group g's k-step s' in lane c takes
// 64g + 16c + s' + (0, 8, 4, 12), stored at 64g + 16c + 4s' + (0, 1, 2, 3).
__device__ __forceinline__ int qjl_slot(int i) {
    const int rem = i & 31, t = ((rem >> 3) & 1) * 2 + (rem >> 4);
    return (i & ~31) + 4 * (rem & 7) + t;
}
__device__ __forceinline__ int recipe_slot(int p) {
    const int rem = p & 15, t = ((rem >> 2) & 1) * 2 + (rem >> 3);
    return (p & ~15) + 4 * (rem & 3) + t;
}

template <class KF, class VF, int NH, bool TM = false>
struct WarpTiles {
    static constexpr int HL = NH / 4;  // heads per lane
    static constexpr bool KR = KF::MODE == kRecipe;
    static constexpr bool KQ = KF::MODE == kQjl || KR, KG = KF::MODE == kGroupwise || KR,
                          VG = VF::MODE == kGroupwise;
    static_assert(!KR || (KF::N0 == 64 && KF::N1 == 64), "recipe keys: two groups of 64");
    static constexpr int NQW = 16 * HL;  // words of the query fragments of one k-step set
    static constexpr uint32_t kTmQ = 0, kTmZ = 32, kTmO = 64, kTmS = 96, kTmCols = 128;
    uint32_t bq[TM ? 1 : 8][2 * HL];             // query B fragments per k-step (registers when !TM)
    uint32_t bz[(KQ && !TM) ? 8 : 1][2 * HL];    // QJL: projected-query B fragments per sign k-step
    uint32_t bp[2 * HL];               // P' B fragments of the last scored tile (group 0 norms when VG)
    uint32_t bp1[VG ? 2 * HL : 1];     // VG: P' B fragments with the group-1 norms
    float o_[TM ? 1 : 8][4];           // value accumulators: row tile q, rows r / r + 8, columns 2c / 2c + 1
    float m_ref[HL], l_run[HL];
    uint32_t tm = 0;                   // TM: this warp's tensor-memory address (lane quarter, first column)

    __device__ __forceinline__ void load_query(uint32_t (&qf)[8][2 * HL], uint32_t (&zf)[KQ ? 8 : 1][2 * HL]) const {
        if constexpr (TM) {
            tm_ld<NQW>(tm + kTmQ, &qf[0][0]);
            if constexpr (KQ) tm_ld<NQW>(tm + kTmZ, &zf[0][0]);
            tm_wait_ld();
            tm_dep<NQW>(&qf[0][0]);
            if constexpr (KQ) tm_dep<NQW>(&zf[0][0]);
        } else {
#pragma unroll
            for (int s = 0; s < 8; ++s)
#pragma unroll
                for (int i = 0; i < 2 * HL; ++i) {
                    qf[s][i] = bq[s][i];
                    if constexpr (KQ) zf[s][i] = bz[s][i];
                }
        }
    }
    __device__ __forceinline__ void load_acc(float (&o)[8][4]) const {
        if constexpr (TM) {
            uint32_t* w = reinterpret_cast<uint32_t*>(&o[0][0]);
            tm_wait_st();  // the previous store of the accumulators has landed
            tm_ld<32>(tm + kTmO, w);
            tm_wait_ld();
            tm_dep<32>(w);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
                for (int i = 0; i < 4; ++i) o[q][i] = o_[q][i];
        }
    }
    __device__ __forceinline__ void store_acc(const float (&o)[8][4]) {
        if constexpr (TM) {
            tm_st<32>(tm + kTmO, reinterpret_cast<const uint32_t*>(&o[0][0]));
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
                for (int i = 0; i < 4; ++i) o_[q][i] = o[q][i];
        }
    }

    // Rotated, scaled queries of the item's query heads (rows of them), fp32
    // [head][128] in the packed coordinate order; for QJL keys also their
    // projections qz, [head][128] in projection order.
    __device__ __forceinline__ void begin(const float* qr, const float* qz, int rows, int r, int c) {
        const int head = NH == 8 ? r : (r >> 1);
        uint32_t qf[8][2 * HL];
        uint32_t zf[KQ ? 8 : 1][2 * HL];
        // With tensor memory each fragment set is stored as soon as it is built, so the two sets
        // are never live in registers together.
        if constexpr (TM) tm_wait_st();  // the last item's stores have landed before these columns are rewritten
        if constexpr (KQ) {
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                // sign k-step s: B rows (2c, 2c+1) and (2c+8, 2c+9) are projections
                // 32c + s + (0, 16) and 32c + s + (8, 24); for the recipe row,
                // k-step 4g + s' of group g: projections 64g + 16c + s' + (0, 8) and
                // 64g + 16c + s' + (4, 12)
                float x0 = 0.0f, x1 = 0.0f, x2 = 0.0f, x3 = 0.0f;
                if (head < rows) {
                    // the four projections are adjacent in the stored order (qjl_slot, recipe_slot)
                    const int at = KR ? 64 * (s >> 2) + 16 * c + 4 * (s & 3) : 32 * c + 4 * s;
                    const float4 z4 = __ldcg(reinterpret_cast<const float4*>(qz + head * kHeadDim + at));
                    x0 = z4.x;
                    x1 = z4.y;
                    x2 = z4.z;
                    x3 = z4.w;
                }
                uint32_t h01, l01, h23, l23;
                split2(x0, x1, h01, l01);
                split2(x2, x3, h23, l23);
                if constexpr (NH == 8) {
                    zf[s][0] = h01;
                    zf[s][1] = h23;
                    zf[s][2] = l01;
                    zf[s][3] = l23;
                } else {
                    zf[s][0] = (r & 1) ? l01 : h01;
                    zf[s][1] = (r & 1) ? l23 : h23;
                }
            }
            if constexpr (TM) tm_st<NQW>(tm + kTmZ, &zf[0][0]);
        }
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            // k-step s: B rows (2c, 2c+1) and (2c+8, 2c+9) are coordinates p..p+3 of lane c's chunk
            const int p = s < KF::KS0 ? c * (KF::N0 / 4) + 4 * s : KF::N0 + c * (KF::N1 / 4) + 4 * (s - KF::KS0);
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (head < rows) x = __ldcg(reinterpret_cast<const float4*>(qr + head * kHeadDim + p));
            uint32_t h01, l01, h23, l23;
            split2(x.x, x.y, h01, l01);
            split2(x.z, x.w, h23, l23);
            if constexpr (NH == 8) {
                qf[s][0] = h01;
                qf[s][1] = h23;
                qf[s][2] = l01;
                qf[s][3] = l23;
            } else {
                qf[s][0] = (r & 1) ? l01 : h01;
                qf[s][1] = (r & 1) ? l23 : h23;
            }
        }
        float o[8][4];
#pragma unroll
        for (int q = 0; q < 8; ++q) o[q][0] = o[q][1] = o[q][2] = o[q][3] = 0.0f;
        if constexpr (TM) {
            tm_st<NQW>(tm + kTmQ, &qf[0][0]);
            tm_st<32>(tm + kTmO, reinterpret_cast<const uint32_t*>(&o[0][0]));
            tm_wait_st();
        } else {
#pragma unroll
            for (int s = 0; s < 8; ++s)
#pragma unroll
                for (int i = 0; i < 2 * HL; ++i) {
                    bq[s][i] = qf[s][i];
                    if constexpr (KQ) bz[s][i] = zf[s][i];
                }
            store_acc(o);
        }
#pragma unroll
        for (int e = 0; e < HL; ++e) {
            m_ref[e] = -INFINITY;
            l_run[e] = 0.0f;
        }
    }

    // Scores of one 16-token block (K index rows at kbase, norms at knorm), in
    // log2 units and before any max: sc[e][0] for token r, sc[e][1] for token
    // r + 8 of the lane's head e; -inf for tokens at or past nvalid (padding).
    __device__ __forceinline__ void block_scores(const uint32_t (&qf)[8][2 * HL],
                                                 const uint32_t (&zf)[KQ ? 8 : 1][2 * HL], uint32_t kbase,
                                                 uint32_t knorm, int nvalid, uint32_t lane_base, int r, int c,
                                                 float (&sc)[HL][2]) const {
        // ---- S^T = K^ Q'^T: rows tokens r, r + 8 ----
        // Independent accumulator chains (k-step parity, or the group when K is
        // group-wise; hi / lo for NH = 8) keep the MMA dependency depth at 4.
        constexpr int NC = NH == 8 ? 4 : 2;
        // QJL keys in tensor memory: the sign fragments are loaded for the
        // sign k-steps and the index fragments after them, never both at once.
        constexpr bool kOwnLoads = KQ && TM;
        float sacc[NC][4];
#pragma unroll
        for (int u = 0; u < NC; ++u) sacc[u][0] = sacc[u][1] = sacc[u][2] = sacc[u][3] = 0.0f;
        uint32_t ql[kOwnLoads ? 8 : 1][2 * HL];
        auto score_step = [&](auto si, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
            constexpr int s_ = decltype(si)::value;
            constexpr int u = KG ? (s_ < KF::KS0 ? 0 : 1) : (s_ & 1);
            const auto& Q = [&]() -> const auto& {
                if constexpr (kOwnLoads) return ql;
                else return qf;
            }();
            if constexpr (NH == 8) {
                mma16816(sacc[u], a0, a1, a2, a3, Q[s_][0], Q[s_][1]);
                mma16816(sacc[2 + u], a0, a1, a2, a3, Q[s_][2], Q[s_][3]);
            } else {
                mma16816(sacc[u], a0, a1, a2, a3, Q[s_][0], Q[s_][1]);
            }
        };
        if constexpr (KQ) {
            uint32_t zl[kOwnLoads ? 8 : 1][2 * HL];
            if constexpr (kOwnLoads) {
                tm_ld<NQW>(tm + kTmZ, &zl[0][0]);
                tm_wait_ld();
                tm_dep<NQW>(&zl[0][0]);
            }
            const auto& Z = [&]() -> const auto& {
                if constexpr (kOwnLoads) return zl;
                else return zf;
            }();
            // Sign k-step s takes bits (s, s + 16) of the lane's word (projections
            // 32c + ...) for its k columns (2c, 2c + 1) and bits (s + 8, s + 24)
            // for (2c + 8, 2c + 9): one shift puts such a pair at bits 15 and 31,
            // the sign bits of the two halves of +-|r| (a clear bit is -).
            if constexpr (KR) {
                // Recipe row: group g's 64 sign bits follow its indices, lane c takes
                // projections 16c .. 16c + 15 of the group (bits 16c.. of its stream):
                // with byte 1 of that half-word moved to byte 2, bits (s', s' + 8) sit 16
                // apart for k columns (2c, 2c + 1) of k-step s' and bits (s' + 4, s' + 12)
                // for (2c + 8, 2c + 9). The k-steps of group g accumulate in its chain,
                // which takes n_g: n_g (q'.c + |r_g| (kappa_g S_g q'_g).z_g).
                static_for<0, 2>([&](auto gi) {
                    constexpr int g = decltype(gi)::value;
                    constexpr int SO = g ? KF::SO1 : KF::SO0;
                    const uint32_t wa = prmt(lds16(kbase + r * KF::RB + SO + 2 * c), 0u, 0x4140u);
                    const uint32_t wb = prmt(lds16(kbase + (r + 8) * KF::RB + SO + 2 * c), 0u, 0x4140u);
                    const uint32_t ga = lds16(knorm + KF::NB * r + 2 + 4 * g);
                    const uint32_t gb = lds16(knorm + KF::NB * (r + 8) + 2 + 4 * g);
                    const uint32_t rn_a = ga | (ga << 16), rn_b = gb | (gb << 16);
                    static_for<0, 4>([&](auto si) {
                        constexpr int s_ = decltype(si)::value;
                        const uint32_t a0 = rn_a | (~(wa << (15 - s_)) & 0x80008000u);
                        const uint32_t a1 = rn_b | (~(wb << (15 - s_)) & 0x80008000u);
                        const uint32_t a2 = rn_a | (~(wa << (11 - s_)) & 0x80008000u);
                        const uint32_t a3 = rn_b | (~(wb << (11 - s_)) & 0x80008000u);
                        if constexpr (NH == 8) {
                            mma16816(sacc[g], a0, a1, a2, a3, Z[4 * g + s_][0], Z[4 * g + s_][1]);
                            mma16816(sacc[2 + g], a0, a1, a2, a3, Z[4 * g + s_][2], Z[4 * g + s_][3]);
                        } else {
                            mma16816(sacc[g], a0, a1, a2, a3, Z[4 * g + s_][0], Z[4 * g + s_][1]);
                        }
                    });
                });
            } else {
                const uint32_t wa = lds32(kbase + r * KF::RB + KF::IB + 4 * c);
                const uint32_t wb = lds32(kbase + (r + 8) * KF::RB + KF::IB + 4 * c);
                const uint32_t ga = lds16(knorm + KF::NB * r + 2), gb = lds16(knorm + KF::NB * (r + 8) + 2);
                const uint32_t rn_a = ga | (ga << 16), rn_b = gb | (gb << 16);
                static_for<0, 8>([&](auto si) {
                    constexpr int s_ = decltype(si)::value;
                    const uint32_t a0 = rn_a | (~(wa << (15 - s_)) & 0x80008000u);
                    const uint32_t a1 = rn_b | (~(wb << (15 - s_)) & 0x80008000u);
                    const uint32_t a2 = rn_a | (~(wa << (7 - s_)) & 0x80008000u);
                    const uint32_t a3 = rn_b | (~(wb << (7 - s_)) & 0x80008000u);
                    if constexpr (NH == 8) {
                        mma16816(sacc[s_ & 1], a0, a1, a2, a3, Z[s_][0], Z[s_][1]);
                        mma16816(sacc[2 + (s_ & 1)], a0, a1, a2, a3, Z[s_][2], Z[s_][3]);
                    } else {
                        mma16816(sacc[s_ & 1], a0, a1, a2, a3, Z[s_][0], Z[s_][1]);
                    }
                });
            }
        }
        if constexpr (kOwnLoads) {
            tm_ld<NQW>(tm + kTmQ, &ql[0][0]);
            tm_wait_ld();
            tm_dep<NQW>(&ql[0][0]);
        }
        {
            constexpr int KW0 = (KF::KC0 + 3) / 4;
            constexpr bool A0 = KF::KC0 % 4 == 0;
            const Words<KW0> k0a = lds_span_off<KF::KC0, A0, 0, KF::KC0, 4>(kbase + r * KF::RB, c * KF::KC0);
            const Words<KW0> k0b = lds_span_off<KF::KC0, A0, 0, KF::KC0, 4>(kbase + (r + 8) * KF::RB, c * KF::KC0);
            const uint32_t base0 = lut_base<KF::B0>(lane_base);
            static_for<0, KF::KS0>([&](auto si) {
                constexpr int s_ = decltype(si)::value;
                const uint32_t a0 = lut(pair_addr<KF::B0, 4 * s_ * KF::B0, KW0>(k0a.w, base0));
                const uint32_t a1 = lut(pair_addr<KF::B0, 4 * s_ * KF::B0, KW0>(k0b.w, base0));
                const uint32_t a2 = lut(pair_addr<KF::B0, (4 * s_ + 2) * KF::B0, KW0>(k0a.w, base0));
                const uint32_t a3 = lut(pair_addr<KF::B0, (4 * s_ + 2) * KF::B0, KW0>(k0b.w, base0));
                score_step(si, a0, a1, a2, a3);
            });
            if constexpr (KF::N1 > 0) {
                constexpr int KW1 = (KF::KC1 + 3) / 4;
                constexpr bool A1 = (KF::KC1 % 4 == 0) && (KF::BOFF1 % 4 == 0);
                const uint32_t g1 = KF::BOFF1 + c * KF::KC1;
                const Words<KW1> k1a = lds_span_off<KF::KC1, A1, KF::BOFF1, KF::KC1, 4>(kbase + r * KF::RB, g1);
                const Words<KW1> k1b = lds_span_off<KF::KC1, A1, KF::BOFF1, KF::KC1, 4>(kbase + (r + 8) * KF::RB, g1);
                const uint32_t base1 = lut_base<KF::B1>(lane_base);
                static_for<0, KF::KS1>([&](auto si) {
                    constexpr int s_ = decltype(si)::value;
                    const uint32_t a0 = lut(pair_addr<KF::B1, 4 * s_ * KF::B1, KW1>(k1a.w, base1));
                    const uint32_t a1 = lut(pair_addr<KF::B1, 4 * s_ * KF::B1, KW1>(k1b.w, base1));
                    const uint32_t a2 = lut(pair_addr<KF::B1, (4 * s_ + 2) * KF::B1, KW1>(k1a.w, base1));
                    const uint32_t a3 = lut(pair_addr<KF::B1, (4 * s_ + 2) * KF::B1, KW1>(k1b.w, base1));
                    score_step(std::integral_constant<int, KF::KS0 + s_>{}, a0, a1, a2, a3);
                });
            }
        }

        // ---- scores of the lane's heads, tokens r and r + 8 ----
        const float nk0 = f16_at(knorm + KF::NB * r), nk1 = f16_at(knorm + KF::NB * (r + 8));
        const bool ok0 = r < nvalid, ok1 = r + 8 < nvalid;
        if constexpr (NH == 8 && KG) {
            // chains 0 / 2: group 0 hi / lo; chains 1 / 3: group 1
            const float mk0 = f16_at(knorm + KF::NB * r + KF::N1OFF), mk1 = f16_at(knorm + KF::NB * (r + 8) + KF::N1OFF);
            float x0, x1, y0, y1;
            upk(add2(mul2(add2(pk(sacc[0][0], sacc[0][1]), pk(sacc[2][0], sacc[2][1])), pk(nk0, nk0)),
                     mul2(add2(pk(sacc[1][0], sacc[1][1]), pk(sacc[3][0], sacc[3][1])), pk(mk0, mk0))),
                x0, x1);
            upk(add2(mul2(add2(pk(sacc[0][2], sacc[0][3]), pk(sacc[2][2], sacc[2][3])), pk(nk1, nk1)),
                     mul2(add2(pk(sacc[1][2], sacc[1][3]), pk(sacc[3][2], sacc[3][3])), pk(mk1, mk1))),
                y0, y1);
            sc[0][0] = ok0 ? x0 : -INFINITY;
            sc[HL - 1][0] = ok0 ? x1 : -INFINITY;
            sc[0][1] = ok1 ? y0 : -INFINITY;
            sc[HL - 1][1] = ok1 ? y1 : -INFINITY;
        } else if constexpr (NH == 8) {
            float x0, x1, y0, y1;
            upk(add2(add2(pk(sacc[0][0], sacc[0][1]), pk(sacc[1][0], sacc[1][1])),
                     add2(pk(sacc[2][0], sacc[2][1]), pk(sacc[3][0], sacc[3][1]))),
                x0, x1);
            upk(add2(add2(pk(sacc[0][2], sacc[0][3]), pk(sacc[1][2], sacc[1][3])),
                     add2(pk(sacc[2][2], sacc[2][3]), pk(sacc[3][2], sacc[3][3]))),
                y0, y1);
            upk(mul2(pk(x0, x1), pk(nk0, nk0)), x0, x1);
            upk(mul2(pk(y0, y1), pk(nk1, nk1)), y0, y1);
            sc[0][0] = ok0 ? x0 : -INFINITY;
            sc[HL - 1][0] = ok0 ? x1 : -INFINITY;
            sc[0][1] = ok1 ? y0 : -INFINITY;
            sc[HL - 1][1] = ok1 ? y1 : -INFINITY;
        } else if constexpr (KG) {
            // chain 0: group 0 (hi, lo columns); chain 1: group 1
            const float mk0 = f16_at(knorm + KF::NB * r + KF::N1OFF), mk1 = f16_at(knorm + KF::NB * (r + 8) + KF::N1OFF);
            sc[0][0] = ok0 ? (sacc[0][0] + sacc[0][1]) * nk0 + (sacc[1][0] + sacc[1][1]) * mk0 : -INFINITY;
            sc[0][1] = ok1 ? (sacc[0][2] + sacc[0][3]) * nk1 + (sacc[1][2] + sacc[1][3]) * mk1 : -INFINITY;
        } else {
            float h0, l0, h1, l1;
            upk(add2(pk(sacc[0][0], sacc[0][1]), pk(sacc[1][0], sacc[1][1])), h0, l0);
            upk(add2(pk(sacc[0][2], sacc[0][3]), pk(sacc[1][2], sacc[1][3])), h1, l1);
            sc[0][0] = ok0 ? (h0 + l0) * nk0 : -INFINITY;
            sc[0][1] = ok1 ? (h1 + l1) * nk1 : -INFINITY;
        }
    }

    // Online-softmax update for the scores of NB blocks. The reference max
    // only moves when a score exceeds it by more than 2^kSlack; the shuffles
    // and the rescale of the accumulators run only then.
    template <int NB>
    __device__ __forceinline__ void update(const float (&sc)[NB][HL][2]) {
        bool over = false;
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int e = 0; e < HL; ++e) over |= fmaxf(sc[b][e][0], sc[b][e][1]) > m_ref[e] + kSlack;
        // The trip count is opaque to the compiler (0 or 1 at run time), so the
        // rescale stays a branch instead of predicated straight-line code.
        int rare = __any_sync(kFull, over) ? 1 : 0;
        asm volatile("mov.b32 %0, %0;" : "+r"(rare));
#pragma unroll 1
        for (int t = 0; t < rare; ++t) {
            float alpha[HL];
#pragma unroll
            for (int e = 0; e < HL; ++e) {
                float mx = fmaxf(sc[0][e][0], sc[0][e][1]);
#pragma unroll
                for (int b = 1; b < NB; ++b) mx = fmaxf(mx, fmaxf(sc[b][e][0], sc[b][e][1]));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                const bool grow = mx > m_ref[e] + kSlack;
                alpha[e] = grow ? ex2(m_ref[e] - mx) : 1.0f;
                l_run[e] *= alpha[e];
                if (grow) m_ref[e] = mx;
            }
            float o[8][4];
            load_acc(o);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                o[q][0] *= alpha[0];
                o[q][1] *= alpha[HL - 1];
                o[q][2] *= alpha[0];
                o[q][3] *= alpha[HL - 1];
            }
            store_acc(o);
        }
    }

    // The block's weights after update(): P' = p 2^-kSlack n_V (weight x norm
    // stays within fp16) as B fragments in bpo (bpo1: with the group-1 norms
    // when V is group-wise); the sums l_run are kept in the same 2^-kSlack
    // units. m_ref is finite here: the first block of an item always moves it
    // (a valid score exceeds -inf + kSlack).
    __device__ __forceinline__ void block_weights(const float (&sc)[HL][2], uint32_t vnorm, int nvalid, int r,
                                                  uint32_t (&bpo)[2 * HL],
                                                  uint32_t (&bpo1)[VG ? 2 * HL : 1]) {
        const bool ok0 = r < nvalid, ok1 = r + 8 < nvalid;
        const float nv0 = f16_at(vnorm + VF::NB * r), nv1 = f16_at(vnorm + VF::NB * (r + 8));
        const float nv0m = ok0 ? nv0 : 0.0f, nv1m = ok1 ? nv1 : 0.0f;  // padding rows may hold anything
        float p[HL][2];
#pragma unroll
        for (int e = 0; e < HL; ++e) {
            const float mb = m_ref[e] + kSlack;
            p[e][0] = ex2(sc[e][0] - mb);
            p[e][1] = ex2(sc[e][1] - mb);
            l_run[e] += p[e][0] + p[e][1];
        }
        weights(p, nv0m, nv1m, bpo);
        if constexpr (VG) {
            const float mv0 = ok0 ? f16_at(vnorm + VF::NB * r + 2) : 0.0f;
            const float mv1 = ok1 ? f16_at(vnorm + VF::NB * (r + 8) + 2) : 0.0f;
            weights(p, mv0, mv1, bpo1);
        }
    }

    // Scores of one 16-token tile (K index rows at kbase, norms at knorm) and
    // the online-softmax update; leaves the tile's P' (V norms at vnorm) in bp
    // for values(). Tokens at or past nvalid are padding.
    __device__ __forceinline__ void scores(uint32_t kbase, uint32_t knorm, uint32_t vnorm, int nvalid,
                                           uint32_t lane_base, int r, int c) {
        uint32_t qf[8][2 * HL];
        uint32_t zf[KQ ? 8 : 1][2 * HL];
        if constexpr (!(KQ && TM)) load_query(qf, zf);
        float sc[1][HL][2];
        block_scores(qf, zf, kbase, knorm, nvalid, lane_base, r, c, sc[0]);
        update<1>(sc);
        block_weights(sc[0], vnorm, nvalid, r, bp, bp1);
    }

    // B fragments of P'^T (P' = p n_V for the V norms n0 of token r and n1 of
    // token r + 8): rows tokens (2c, 2c+1) and (2c+8, 2c+9), column r, made
    // from the lane's own values by an in-register 8x8 transpose (movmatrix).
    __device__ __forceinline__ static void weights(const float (&p)[HL][2], float n0, float n1,
                                                   uint32_t (&out)[2 * HL]) {
        if constexpr (NH == 8) {
            // Per token: (head 2c, head 2c + 1) as hi and lo half2, i.e. rows r (tokens 0..7) and
            // r + 8 (tokens 8..15) of two 8x8 row-major fp16 matrices [token][head]; their
            // transposes in the same fragment layout are the B fragments [token 2c, 2c+1][head r].
            uint32_t th0, tl0, th1, tl1;
            split2(p[0][0] * n0, p[1][0] * n0, th0, tl0);
            split2(p[0][1] * n1, p[1][1] * n1, th1, tl1);
            out[0] = movmatrix_t(th0);
            out[1] = movmatrix_t(th1);
            out[2] = movmatrix_t(tl0);
            out[3] = movmatrix_t(tl1);
        } else {
            // Columns are (head, hi / lo): per token, (hi, lo) of head c at columns 2c and 2c + 1 is
            // row r (tokens 0..7) or r + 8 (tokens 8..15) of an 8x8 row-major fp16 matrix
            // [token][column]; the transposes are the B fragments [token 2c, 2c+1][column r].
            uint32_t xh, xl;
            split2(p[0][0] * n0, p[0][1] * n1, xh, xl);
            out[0] = movmatrix_t(prmt(xh, xl, 0x5410u));
            out[1] = movmatrix_t(prmt(xh, xl, 0x7632u));
        }
    }

    // One 16-token tile: K index rows at kbase (norms at knorm), V index rows at
    // vbase (norms at vnorm); tokens at or past nvalid are padding.
    __device__ __forceinline__ void step(uint32_t kbase, uint32_t knorm, uint32_t vbase, uint32_t vnorm, int nvalid,
                                         uint32_t lane_base, int r, int c) {
        scores(kbase, knorm, vnorm, nvalid, lane_base, r, c);
        values(vbase, lane_base, r, c);
    }

    // O^T += V^T P'^T for the tile last passed to scores(): V index rows at vbase.
    __device__ __forceinline__ void values(uint32_t vbase, uint32_t lane_base, int r, int c) {
        float o[8][4];
        load_acc(o);
        values_block(o, vbase, bp, bp1, lane_base, r, c);
        store_acc(o);
    }

    // o += V^T P'^T for one 16-token block: V index rows at vbase, P' fragments bpo (bpo1).
    __device__ __forceinline__ void values_block(float (&o)[8][4], uint32_t vbase, const uint32_t (&bpo)[2 * HL],
                                                 const uint32_t (&bpo1)[VG ? 2 * HL : 1], uint32_t lane_base, int r,
                                                 int c) const {
        auto value_step = [&](auto qi, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
            constexpr int q = decltype(qi)::value;
            if constexpr (VG && q >= VF::MT0) {
                mma16816(o[q], a0, a1, a2, a3, bpo1[0], bpo1[1]);
                if constexpr (NH == 8) mma16816(o[q], a0, a1, a2, a3, bpo1[2], bpo1[3]);
            } else {
                mma16816(o[q], a0, a1, a2, a3, bpo[0], bpo[1]);
                if constexpr (NH == 8) mma16816(o[q], a0, a1, a2, a3, bpo[2], bpo[3]);
            }
        };

        // ---- O^T += V^T P'^T over 8 coordinate row tiles ----
        const uint32_t r0 = vbase + (2 * c) * VF::RB, r1 = r0 + VF::RB;
        const uint32_t r8 = vbase + (2 * c + 8) * VF::RB, r9 = r8 + VF::RB;
        {
            constexpr int NW0 = (VF::VC0 + 3) / 4;
            constexpr bool A0 = VF::VC0 % 4 == 0;
            const Words<NW0> t0 = lds_span_off<VF::VC0, A0, 0, VF::VC0, 8>(r0, r * VF::VC0);
            const Words<NW0> t1 = lds_span_off<VF::VC0, A0, 0, VF::VC0, 8>(r1, r * VF::VC0);
            const Words<NW0> t8 = lds_span_off<VF::VC0, A0, 0, VF::VC0, 8>(r8, r * VF::VC0);
            const Words<NW0> t9 = lds_span_off<VF::VC0, A0, 0, VF::VC0, 8>(r9, r * VF::VC0);
            uint32_t e01[NW0], o01[NW0], e89[NW0], o89[NW0];
            interleave<VF::B0, NW0>(t0.w, t1.w, e01, o01);
            interleave<VF::B0, NW0>(t8.w, t9.w, e89, o89);
            const uint32_t base0 = lut_base<VF::B0>(lane_base);
            static_for<0, VF::MT0>([&](auto qi) {
                constexpr int q = decltype(qi)::value;
                const uint32_t a0 = lut(vpair_addr<VF::B0, 2 * q, NW0>(e01, o01, base0));
                const uint32_t a1 = lut(vpair_addr<VF::B0, 2 * q + 1, NW0>(e01, o01, base0));
                const uint32_t a2 = lut(vpair_addr<VF::B0, 2 * q, NW0>(e89, o89, base0));
                const uint32_t a3 = lut(vpair_addr<VF::B0, 2 * q + 1, NW0>(e89, o89, base0));
                value_step(qi, a0, a1, a2, a3);
            });
        }
        if constexpr (VF::N1 > 0) {
            constexpr int NW1 = (VF::VC1 + 3) / 4;
            constexpr bool A1 = (VF::VC1 % 4 == 0) && (VF::BOFF1 % 4 == 0);
            const uint32_t g1 = VF::BOFF1 + r * VF::VC1;
            const Words<NW1> t0 = lds_span_off<VF::VC1, A1, VF::BOFF1, VF::VC1, 8>(r0, g1);
            const Words<NW1> t1 = lds_span_off<VF::VC1, A1, VF::BOFF1, VF::VC1, 8>(r1, g1);
            const Words<NW1> t8 = lds_span_off<VF::VC1, A1, VF::BOFF1, VF::VC1, 8>(r8, g1);
            const Words<NW1> t9 = lds_span_off<VF::VC1, A1, VF::BOFF1, VF::VC1, 8>(r9, g1);
            uint32_t e01[NW1], o01[NW1], e89[NW1], o89[NW1];
            interleave<VF::B1, NW1>(t0.w, t1.w, e01, o01);
            interleave<VF::B1, NW1>(t8.w, t9.w, e89, o89);
            const uint32_t base1 = lut_base<VF::B1>(lane_base);
            static_for<0, VF::MT1>([&](auto qi) {
                constexpr int q = decltype(qi)::value;
                const uint32_t a0 = lut(vpair_addr<VF::B1, 2 * q, NW1>(e01, o01, base1));
                const uint32_t a1 = lut(vpair_addr<VF::B1, 2 * q + 1, NW1>(e01, o01, base1));
                const uint32_t a2 = lut(vpair_addr<VF::B1, 2 * q, NW1>(e89, o89, base1));
                const uint32_t a3 = lut(vpair_addr<VF::B1, 2 * q + 1, NW1>(e89, o89, base1));
                value_step(std::integral_constant<int, VF::MT0 + q>{}, a0, a1, a2, a3);
            });
        }
    }

    // Two 16-token blocks as one step (a 32-token block, or two 16-token
    // blocks of consecutive slots): one load of the query fragments, one
    // softmax update and one pass over the accumulators.
    __device__ __forceinline__ void step2(uint32_t kb0, uint32_t kn0, uint32_t vb0, uint32_t vn0, int nv0,
                                          uint32_t kb1, uint32_t kn1, uint32_t vb1, uint32_t vn1, int nv1,
                                          uint32_t lane_base, int r, int c) {
        float sc[2][HL][2];
        if constexpr (KQ || KG || VG) {
            // these keep more per block: the fragments are reloaded so the two blocks never hold them at once
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                uint32_t qf[8][2 * HL];
                uint32_t zf[KQ ? 8 : 1][2 * HL];
                if constexpr (!(KQ && TM)) load_query(qf, zf);
                block_scores(qf, zf, b ? kb1 : kb0, b ? kn1 : kn0, b ? nv1 : nv0, lane_base, r, c, sc[b]);
            }
        } else {
            uint32_t qf[8][2 * HL];
            uint32_t zf[KQ ? 8 : 1][2 * HL];
            load_query(qf, zf);
            block_scores(qf, zf, kb0, kn0, nv0, lane_base, r, c, sc[0]);
            block_scores(qf, zf, kb1, kn1, nv1, lane_base, r, c, sc[1]);
        }
        update<2>(sc);
        uint32_t p0[2 * HL], p1[2 * HL], g0[VG ? 2 * HL : 1], g1[VG ? 2 * HL : 1];
        block_weights(sc[0], vn0, nv0, r, p0, g0);
        block_weights(sc[1], vn1, nv1, r, p1, g1);
        float o[8][4];
        load_acc(o);
        values_block(o, vb0, p0, g0, lane_base, r, c);
        values_block(o, vb1, p1, g1, lane_base, r, c);
        store_acc(o);
    }

    // Pair merge (TM). The partner warp leaves its (max, sum) per head in its
    // kTmS columns (its accumulators are already in its kTmO columns); the
    // owner, in the same lane quarter, folds both into its own state.
    __device__ __forceinline__ void export_state() {
        const uint32_t v[4] = {__float_as_uint(m_ref[0]), __float_as_uint(m_ref[HL - 1]), __float_as_uint(l_run[0]),
                               __float_as_uint(l_run[HL - 1])};
        tm_st<4>(tm + kTmS, v);
        tm_wait_st();  // this store and the accumulators' last one have landed
    }
    __device__ __forceinline__ void absorb(uint32_t partner) {
        float o[8][4], po[8][4];
        uint32_t ps[4];
        load_acc(o);
        uint32_t* pw = reinterpret_cast<uint32_t*>(&po[0][0]);
        tm_ld<32>(partner + kTmO, pw);
        tm_ld<4>(partner + kTmS, ps);
        tm_wait_ld();
        tm_dep<32>(pw);
        tm_dep<4>(ps);
        float f0[HL], f1[HL];
#pragma unroll
        for (int e = 0; e < HL; ++e) {
            const float pm = __uint_as_float(ps[e]), pl = __uint_as_float(ps[2 + e]);
            const float M = fmaxf(m_ref[e], pm);
            f0[e] = m_ref[e] == -INFINITY ? 0.0f : ex2(m_ref[e] - M);
            f1[e] = pm == -INFINITY ? 0.0f : ex2(pm - M);
            l_run[e] = l_run[e] * f0[e] + pl * f1[e];
            m_ref[e] = M;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            o[q][0] = o[q][0] * f0[0] + po[q][0] * f1[0];
            o[q][1] = o[q][1] * f0[HL - 1] + po[q][1] * f1[HL - 1];
            o[q][2] = o[q][2] * f0[0] + po[q][2] * f1[0];
            o[q][3] = o[q][3] * f0[HL - 1] + po[q][3] * f1[HL - 1];
        }
        store_acc(o);
    }

    // Writes (max, sum, accumulator x 2^kSlack) of each of the lane's heads:
    // m[head * ml_stride], l[head * ml_stride] and acc[head * acc_stride +
    // packed coordinate]. Row r of value tile q is packed coordinate p0, row
    // r + 8 is p0 + 1.
    __device__ __forceinline__ void finish(float* m, float* l, float* acc, int ml_stride, int acc_stride, int rows,
                                           int r, int c) {
        float o[8][4];
        load_acc(o);
#pragma unroll
        for (int e = 0; e < HL; ++e) {
            float lsum = l_run[e];
            lsum += __shfl_xor_sync(kFull, lsum, 4);
            lsum += __shfl_xor_sync(kFull, lsum, 8);
            lsum += __shfl_xor_sync(kFull, lsum, 16);
            lsum *= 256.0f;  // back from 2^-kSlack units
            const int head = NH == 8 ? 2 * c + e : c;
            if (head < rows) {
                if (r == 0) {
                    m[head * ml_stride] = m_ref[e];
                    l[head * ml_stride] = lsum;
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const bool g1 = q >= VF::MT0;
                    const int ql = g1 ? q - VF::MT0 : q;
                    const int per = g1 ? VF::N1 / 8 : VF::N0 / 8;
                    const int p0 = (g1 ? VF::N0 : 0) + r * per + 2 * ql;
                    float2 val;
                    if constexpr (NH == 8) {
                        val = e == 0 ? make_float2(o[q][0], o[q][2]) : make_float2(o[q][1], o[q][3]);
                    } else {
                        val = make_float2(o[q][0] + o[q][1], o[q][2] + o[q][3]);
                    }
                    *reinterpret_cast<float2*>(acc + head * acc_stride + p0) =
                        make_float2(val.x * 256.0f, val.y * 256.0f);
                }
            }
        }
    }
};

// Dense bf16 window of KV head h for the item's query heads: tokens
// t_first, t_first + t_step, ... < it.t1, on CUDA cores (lane: 4 coordinates).
// Writes (max, sum, accumulator) per query head g < rows: m[g * ml_stride],
// l[g * ml_stride], acc[g * acc_stride + coordinate] (acc 8-byte aligned).
template <int NH>
// t_new >= 0: dense slot t_new holds the step's new token, read from kn / vn (rows of 128) instead of
// the buffer (a fused window append may be writing that slot).
__device__ __forceinline__ void window_state(const DecodeArgs& a, const Item& it, int h, int head0, int rows,
                                             int t_first, int t_step, int lane, float* m_out, float* l_out,
                                             float* acc_out, int ml_stride, int acc_stride, int t_new = -1,
                                             const __nv_bfloat16* kn = nullptr,
                                             const __nv_bfloat16* vn = nullptr) {
    const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
    const int H = a.kc.num_heads;
    float qv[NH][4], m[NH], l[NH], acc[NH][4];
#pragma unroll
    for (int g = 0; g < NH; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[g][i] = 0.0f;
            qv[g][i] = 0.0f;
        }
        if (g < rows) {
            const uint2 raw = *reinterpret_cast<const uint2*>(
                qg + (static_cast<int64_t>(it.b) * a.num_q_heads + head0 + g) * kHeadDim + 4 * lane);
            qv[g][0] = __uint_as_float(raw.x << 16) * a.scale_log2;
            qv[g][1] = __uint_as_float(raw.x & 0xffff0000u) * a.scale_log2;
            qv[g][2] = __uint_as_float(raw.y << 16) * a.scale_log2;
            qv[g][3] = __uint_as_float(raw.y & 0xffff0000u) * a.scale_log2;
        }
    }
    const __nv_bfloat16* kw = static_cast<const __nv_bfloat16*>(a.k_win);
    const __nv_bfloat16* vw = static_cast<const __nv_bfloat16*>(a.v_win);
    const int64_t row0 = (static_cast<int64_t>(it.b) * H + h) * a.window;
    const bool b4 = lane & 16, b3 = lane & 8;
    // Four tokens at a time: their loads are issued together (and those of the next
    // four before this four is computed), and the four partial dot products of a
    // head are summed over the warp by a transposed butterfly (the first two steps
    // halve the values a lane carries; lane 8u ends with token u), then broadcast:
    // 10 shuffles for 4 tokens instead of 20.
    uint2 kr[4], vr[4];
    auto load4 = [&](int t0_) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int tk = t0_ + u * t_step;
            kr[u] = make_uint2(0u, 0u);
            vr[u] = make_uint2(0u, 0u);
            if (tk < it.t1) {
                const int64_t base = (row0 + tk) * kHeadDim + 4 * lane;
                const bool fresh = tk == t_new;
                kr[u] = *reinterpret_cast<const uint2*>(fresh ? kn + 4 * lane : kw + base);
                vr[u] = *reinterpret_cast<const uint2*>(fresh ? vn + 4 * lane : vw + base);
            }
        }
    };
    load4(t_first);
    for (int t0 = t_first; t0 < it.t1; t0 += 4 * t_step) {
        float kx[4][4], vx[4][4];
        bool ok[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            ok[u] = t0 + u * t_step < it.t1;
            kx[u][0] = __uint_as_float(kr[u].x << 16);
            kx[u][1] = __uint_as_float(kr[u].x & 0xffff0000u);
            kx[u][2] = __uint_as_float(kr[u].y << 16);
            kx[u][3] = __uint_as_float(kr[u].y & 0xffff0000u);
            vx[u][0] = __uint_as_float(vr[u].x << 16);
            vx[u][1] = __uint_as_float(vr[u].x & 0xffff0000u);
            vx[u][2] = __uint_as_float(vr[u].y << 16);
            vx[u][3] = __uint_as_float(vr[u].y & 0xffff0000u);
        }
        load4(t0 + 4 * t_step);
#pragma unroll
        for (int g = 0; g < NH; ++g) {
            if (g < rows) {
                float p[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    p[u] = qv[g][0] * kx[u][0] + qv[g][1] * kx[u][1] + qv[g][2] * kx[u][2] + qv[g][3] * kx[u][3];
                float q2[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {  // lanes with bit 4 keep tokens 2, 3, the others 0, 1
                    const float mine = b4 ? p[i + 2] : p[i], other = b4 ? p[i] : p[i + 2];
                    q2[i] = mine + __shfl_xor_sync(kFull, other, 16);
                }
                float q1 = (b3 ? q2[1] : q2[0]) + __shfl_xor_sync(kFull, b3 ? q2[0] : q2[1], 8);
                q1 += __shfl_xor_sync(kFull, q1, 4);
                q1 += __shfl_xor_sync(kFull, q1, 2);
                q1 += __shfl_xor_sync(kFull, q1, 1);
                float sc[4], mx = m[g];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    sc[u] = ok[u] ? __shfl_sync(kFull, q1, 8 * u) : -INFINITY;
                    mx = fmaxf(mx, sc[u]);
                }
                const float alpha = ex2(m[g] - mx);  // token t0 is valid, so mx is finite
                float ls = l[g] * alpha;
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[g][i] *= alpha;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float pu = ex2(sc[u] - mx);
                    ls += pu;
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[g][i] = fmaf(pu, vx[u][i], acc[g][i]);
                }
                l[g] = ls;
                m[g] = mx;
            }
        }
    }
#pragma unroll
    for (int g = 0; g < NH; ++g) {
        if (g < rows) {
            if (lane == 0) {
                m_out[g * ml_stride] = m[g];
                l_out[g * ml_stride] = l[g];
            }
            float2* dst = reinterpret_cast<float2*>(acc_out + g * acc_stride + 4 * lane);
            dst[0] = make_float2(acc[g][0], acc[g][1]);
            dst[1] = make_float2(acc[g][2], acc[g][3]);
        }
    }
}

// Record of item (b, KV head h, split): [group][2 + 128] floats.
__device__ __forceinline__ float* record_of(const DecodeArgs& a, int b, int h, int split, int group) {
    return a.ws + ((static_cast<int64_t>(b) * a.kc.num_heads + h) * a.items_per_unit + split) *
                      static_cast<int64_t>(group) * (kHeadDim + 2);
}

// ==== block kernel: one page block of 8 KV heads per ring slot ========================
//
// A work item is (query-head group, 8 consecutive KV heads, sequence, split).
// A ring slot holds one page block of the 8 heads in both pools: [K: 8 x
// (bs index rows, bs norms)][V: the same]. The sub-pages of consecutive heads
// are adjacent in a pool, so a slot takes two bulk copies whatever the block
// size. Compute warp w reads KV head w of every slot, 16 tokens at a time,
// and writes its records itself: nothing is merged across warps.

constexpr int kBlkWarps = 8;        // compute warps = KV heads per slot
constexpr int kBlkMaxSlots = 16;
constexpr int kBlkMinSlots = 4;     // fewer slots of a larger block: the per-head kernel instead

struct BlkSmem {
    unsigned long long full[kBlkMaxSlots];   // producer -> warps: slot filled (tx bytes)
    unsigned long long empty[kBlkMaxSlots];  // warps -> producer: 8 releases free a slot
    int ids[2][kMaxItemTiles];               // producer: block ids of the current and next item
};

// Ring placement around the 64 KB table: n_low slots between the header and
// the table, the rest after it.
struct BlkRing {
    uint32_t low, high;
    int n_low, n;
    uint32_t stride;
    __device__ __forceinline__ uint32_t slot(int s) const {
        return s < n_low ? low + s * stride : high + (s - n_low) * stride;
    }
};

// Bytes of a ring slot: one block of 8 heads in both pools.
template <class KF, class VF>
__host__ __device__ constexpr uint32_t blk_slot_bytes(int bs) {
    return static_cast<uint32_t>(kBlkWarps * bs * (KF::RB + KF::NB + VF::RB + VF::NB));
}

template <class KF, class VF>
__device__ void produce_blk(const DecodeArgs& a, BlkSmem& sm, const BlkRing& ring, int head_groups,
                            int64_t total_slots, int lane) {
    if (a.withhold_copies) return;  // test hook: the compute warps' waits expire
    constexpr int kPer = kMaxItemTiles / 32;
    const int H = a.kc.num_heads, bs = a.block_size;
    const uint32_t k_bytes = kBlkWarps * bs * (KF::RB + KF::NB), v_bytes = kBlkWarps * bs * (VF::RB + VF::NB);
    auto read_ids = [&](const Item& it, int (&v)[kPer]) {
        const int nblk = (it.t1 - it.t0 + bs - 1) / bs;
        const int32_t* bt = a.block_tables + static_cast<int64_t>(it.b) * a.max_blocks + it.t0 / bs;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int i = lane + 32 * k;
            v[k] = i < nblk ? __ldg(bt + i) : 0;
        }
    };
    uint32_t fill = 0;
    int buf = 0;
    int64_t slot = blockIdx.x;
    Item cur;
    bool have = next_packed<kBlkWarps>(a, slot, head_groups, total_slots, cur);
    if (have) {
        int v[kPer];
        read_ids(cur, v);
#pragma unroll
        for (int k = 0; k < kPer; ++k) sm.ids[0][lane + 32 * k] = v[k];
    }
    __syncwarp();
    bool stop = false;
    while (have && !stop) {
        int64_t slot_n = slot + gridDim.x;
        Item nxt;
        const bool have_n = next_packed<kBlkWarps>(a, slot_n, head_groups, total_slots, nxt);
        int v[kPer];
        if (have_n) read_ids(nxt, v);
        if (lane == 0) {
            const int nblk = (cur.t1 - cur.t0 + bs - 1) / bs;
#pragma unroll 1
            for (int i = 0; i < nblk; ++i, ++fill) {
                const int s = static_cast<int>(fill % ring.n);
                const uint32_t use = fill / ring.n;
                const uint32_t full = smem_addr(&sm.full[s]);
                if (use > 0 && !mbar_wait(smem_addr(&sm.empty[s]), (use - 1) & 1u)) {
                    // The compute warps stop on their own bounded waits.
                    if (a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
                    stop = true;
                    break;
                }
                int blk = sm.ids[buf][i];
                if (blk < 0 || blk >= a.num_blocks) {
                    if (a.d_err) atomicOr(a.d_err, TQ_DERR_BLOCK);
                    blk = 0;
                }
                const int64_t sp = (static_cast<int64_t>(blk) * H + cur.h) * bs;  // first of 8 sub-pages
                const uint32_t dst = ring.slot(s);
                mbar_expect(full, k_bytes + v_bytes);
                bulk_copy(dst, a.k_pages + sp * (KF::RB + KF::NB), k_bytes, full);
                bulk_copy(dst + k_bytes, a.v_pages + sp * (VF::RB + VF::NB), v_bytes, full);
            }
        }
        stop = __shfl_sync(kFull, stop, 0);
        buf ^= 1;
        if (have_n && !stop) {
#pragma unroll
            for (int k = 0; k < kPer; ++k) sm.ids[buf][lane + 32 * k] = v[k];
        }
        __syncwarp();
        cur = nxt;
        have = have_n;
        slot = slot_n;
    }
    // Wait (bounded) for the copies in flight before the CTA can retire.
    fill = __shfl_sync(kFull, fill, 0);
    if (lane == 0)
        for (uint32_t f = fill > static_cast<uint32_t>(ring.n) ? fill - ring.n : 0; f < fill; ++f)
            if (!mbar_wait(smem_addr(&sm.full[f % ring.n]), (f / ring.n) & 1u)) break;
}

// TPB: 16-token tiles per block when the block size is 16 or 32 (a consumer
// loop with fixed offsets, which measured markedly faster), else 0 (any
// multiple of 16).
template <class KF, class VF, int NH, int TPB>
__global__ void __launch_bounds__((kBlkWarps + 1) * 32, 1) decode_blk_kernel(DecodeArgs a, LutValues tv, int group,
                                                                             int head_groups, int64_t total_slots) {
    static_assert(NH == 4 || NH == 8, "4 or 8 query heads per item");
    extern __shared__ __align__(128) uint8_t dsm[];
    BlkSmem& sm = *reinterpret_cast<BlkSmem*>(dsm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;
    const int bs = a.block_size;

    // Shared memory: [BlkSmem][slots][64 KB table at a 64 KB boundary][slots].
    uint32_t dyn_bytes;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
    const uint32_t dsm_addr = smem_addr(dsm), dsm_end = dsm_addr + dyn_bytes;
    BlkRing ring;
    ring.stride = blk_slot_bytes<KF, VF>(bs);
    ring.low = (dsm_addr + static_cast<uint32_t>(sizeof(BlkSmem)) + 127) & ~127u;
    const uint32_t lut_addr = (ring.low + (kLut - 1)) & ~uint32_t(kLut - 1);
    ring.n_low = static_cast<int>((lut_addr - ring.low) / ring.stride);
    ring.high = lut_addr + kLut;
    const int n_high = ring.high < dsm_end ? static_cast<int>((dsm_end - ring.high) / ring.stride) : 0;
    ring.n = min(ring.n_low + n_high, kBlkMaxSlots);
    if (lut_addr + kLut > dsm_end || ring.n < 2) {
        griddep_wait();
        if (threadIdx.x == 0 && a.d_err) atomicOr(a.d_err, TQ_DERR_LAUNCH);
        return;
    }
    fill_table(reinterpret_cast<uint32_t*>(dsm + (lut_addr - dsm_addr)), tv, threadIdx.x, (kBlkWarps + 1) * 32);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kBlkMaxSlots; ++s) {
            mbar_init_count(smem_addr(&sm.full[s]), 1);
            mbar_init_count(smem_addr(&sm.empty[s]), kBlkWarps);
        }
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    // The table and barriers above overlap the prologue's end; its work list and queries are read
    // from here on.
    griddep_wait();
    griddep_launch_dependents();
    total_slots = listed_slots<kBlkWarps>(a, head_groups, total_slots);
    if (warp == kBlkWarps) {
        produce_blk<KF, VF>(a, sm, ring, head_groups, total_slots, lane);
        return;
    }
    uint32_t lane_base;
    asm volatile("or.b32 %0, %1, %2;" : "=r"(lane_base) : "r"(lut_addr), "r"(static_cast<uint32_t>(lane) << 2));
    const int rows = group < NH ? group : NH;
    // This warp's head within a slot: K sub-page at k_off, V sub-page at v_off.
    const uint32_t k_sub = bs * (KF::RB + KF::NB), v_sub = bs * (VF::RB + VF::NB);
    const uint32_t k_off = warp * k_sub, v_off = kBlkWarps * k_sub + warp * v_sub;
    uint32_t consumed = 0;
    WarpTiles<KF, VF, NH> wt;

    for (int64_t slot = blockIdx.x; slot < total_slots; slot += gridDim.x) {
        Item it;
        if (!item_of<kBlkWarps>(a, slot, head_groups, total_slots, it)) continue;
        const int h = it.h + warp;                    // this warp's KV head
        const int head0 = h * group + it.hg * 8;      // its first query head of the item
        float* rec = record_of(a, it.b, h, it.split, group) + it.hg * 8 * (kHeadDim + 2);
        if (it.win) continue;  // windows are not listed: the prologue's window CTAs take them
        const int64_t q_off = (static_cast<int64_t>(it.b) * a.num_q_heads + head0) * kHeadDim;
        wt.begin(a.qrot + q_off, a.qjl_q + q_off, rows, r, c);
        bool timed_out = false;
        const int ntiles = (it.t1 - it.t0 + 15) >> 4;
        if constexpr (TPB > 0) {
            constexpr int kBs = 16 * TPB;
            for (int k = 0; k < ntiles; k += TPB, ++consumed) {
                const int s = static_cast<int>(consumed % ring.n);
                if (!mbar_wait(smem_addr(&sm.full[s]), (consumed / ring.n) & 1u)) {
                    timed_out = true;
                    break;
                }
                const uint32_t kb = ring.slot(s) + k_off, vb = ring.slot(s) + v_off;
#pragma unroll 1
                for (int j = 0; j < TPB && k + j < ntiles; ++j)
                    wt.step(kb + 16 * j * KF::RB, kb + kBs * KF::RB + 16 * KF::NB * j, vb + 16 * j * VF::RB,
                            vb + kBs * VF::RB + 16 * VF::NB * j, min(16, it.t1 - (it.t0 + 16 * (k + j))), lane_base,
                            r, c);
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&sm.empty[s]));  // this warp is done with the slot
            }
        } else {
            // 16-token tiles; a slot (one block) holds bs / 16 of them.
            const int tpb = bs >> 4;
            uint32_t kb = 0, vb = 0;
            for (int k = 0, j = 0; k < ntiles; ++k) {
                const int s = static_cast<int>(consumed % ring.n);
                if (j == 0) {
                    if (!mbar_wait(smem_addr(&sm.full[s]), (consumed / ring.n) & 1u)) {
                        timed_out = true;
                        break;
                    }
                    kb = ring.slot(s) + k_off;
                    vb = ring.slot(s) + v_off;
                }
                wt.step(kb + 16 * j * KF::RB, kb + bs * KF::RB + 16 * KF::NB * j, vb + 16 * j * VF::RB,
                        vb + bs * VF::RB + 16 * VF::NB * j, min(16, it.t1 - (it.t0 + 16 * k)), lane_base, r, c);
                if (++j == tpb || k + 1 == ntiles) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&sm.empty[s]));  // this warp is done with the slot
                    ++consumed;
                    j = 0;
                }
            }
        }
        if (timed_out) {
            if (lane == 0 && a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
            break;
        }
        wt.finish(rec, rec + 1, rec + 2, kHeadDim + 2, kHeadDim + 2, rows, r, c);
    }
}

// ==== paired block kernel: two compute warps per KV head, state in tensor memory =========
//
// The same ring of 8-head page-block slots as the block kernel, read by 16
// compute warps: warp w takes KV head w % 8 of the slots in every other run of
// 32 tokens (two 16-token slots, or one 32-token slot), the runs of parity
// w / 8. The ring holds a multiple of 4 slots, so each ring position always
// serves the same eight warps and their waits never skip a phase. A warp
// handles its 32 tokens as one step: one load of its query fragments, one
// softmax update and one pass over its accumulators. Each warp keeps its
// query fragments and value accumulators in its own tensor-memory columns
// (WarpTiles<..., true>), which leaves room in the register file for twice the
// warps. At the end of an item the odd warp of each head leaves its state in
// tensor memory and the even warp, which reaches the same lane quarter, folds
// it into its own and writes the record. An expired wait aborts the CTA: the
// two warps of a head agree on it through a reduction barrier, so neither
// waits for the other alone.

constexpr int kPairWarps = 2 * kBlkWarps;  // compute warps (warpgroups 0-3)
constexpr int kPairThreads = (kPairWarps + 4) * 32;  // + warpgroup 4: the producer warp and three idle
constexpr uint32_t kTmemCols = 512;        // 4 warps per lane quarter x 128 columns
// Registers per thread: the launch gives every thread kPairLaunchRegs (the
// compiler's figure for 640 threads, 5 warps per SM sub-partition); then the
// producer warpgroup gives back down to kPairProducerRegs and the compute
// warpgroups take kPairComputeRegs. The block holds 640 x 96 = 61440
// registers; 512 x 112 + 128 x 32 = 61440 fit in them, and each SM
// sub-partition (4 compute warps and one of warpgroup 4) needs 15360 of its
// 16384.
constexpr int kPairLaunchRegs = 96, kPairProducerRegs = 32, kPairComputeRegs = 112;
static_assert(kPairWarps * 32 * kPairComputeRegs + 128 * kPairProducerRegs <= kPairThreads * kPairLaunchRegs,
              "register split above the launch allocation");

struct PairSmem {
    BlkSmem blk;    // ring barriers and the producer's block ids, as in the block kernel
    uint32_t tmem;  // base address of the CTA's tensor memory
    int abort;      // set when a compute warp's wait expired
};

// Barrier `id` over `count` threads that also returns whether any of them passed true.
__device__ __forceinline__ bool bar_any(int id, int count, bool p) {
    uint32_t res;
    asm volatile(
        "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.or.pred po, %2, %3, pi;\n selp.u32 %0, 1, 0, po;\n}"
        : "=r"(res)
        : "r"(static_cast<uint32_t>(p)), "r"(id), "r"(count)
        : "memory");
    return res != 0;
}
__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// The block kernel's producer, reused: its slot sequence does not depend on
// which warps read a slot, only on the release count (8) of every slot.
template <class KF, class VF, int NH, int TPB>
__global__ void __launch_bounds__(kPairThreads, 1) decode_pair_kernel(DecodeArgs a, LutValues tv,
                                                                               int group, int head_groups,
                                                                               int64_t total_slots) {
    static_assert(NH == 4 || NH == 8, "4 or 8 query heads per item");
    static_assert(TPB == 1 || TPB == 2, "16- or 32-token blocks");
    extern __shared__ __align__(128) uint8_t dsm[];
    PairSmem& sm = *reinterpret_cast<PairSmem*>(dsm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;
    const int bs = a.block_size;

    uint32_t dyn_bytes;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
    const uint32_t dsm_addr = smem_addr(dsm), dsm_end = dsm_addr + dyn_bytes;
    BlkRing ring;
    ring.stride = blk_slot_bytes<KF, VF>(bs);
    ring.low = (dsm_addr + static_cast<uint32_t>(sizeof(PairSmem)) + 127) & ~127u;
    const uint32_t lut_addr = (ring.low + (kLut - 1)) & ~uint32_t(kLut - 1);
    ring.n_low = static_cast<int>((lut_addr - ring.low) / ring.stride);
    ring.high = lut_addr + kLut;
    const int n_high = ring.high < dsm_end ? static_cast<int>((dsm_end - ring.high) / ring.stride) : 0;
    // runs of two 16-token slots (or single 32-token slots) alternate between two warps: the ring
    // holds a whole number of run pairs
    constexpr int kRunPair = 2 * (2 / TPB);
    ring.n = min(ring.n_low + n_high, kBlkMaxSlots) / kRunPair * kRunPair;
    if (lut_addr + kLut > dsm_end || ring.n < kRunPair) {
        griddep_wait();
        if (threadIdx.x == 0 && a.d_err) atomicOr(a.d_err, TQ_DERR_LAUNCH);
        return;
    }
    fill_table(reinterpret_cast<uint32_t*>(dsm + (lut_addr - dsm_addr)), tv, threadIdx.x, kPairThreads);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kBlkMaxSlots; ++s) {
            mbar_init_count(smem_addr(&sm.blk.full[s]), 1);
            mbar_init_count(smem_addr(&sm.blk.empty[s]), kBlkWarps);
        }
        sm.abort = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm.tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tm_fence_before_sync();
    __syncthreads();
    tm_fence_after_sync();
    // The table, barriers and tensor memory above overlap the prologue's end; its work list and
    // queries are read from here on.
    griddep_wait();
    griddep_launch_dependents();
    total_slots = listed_slots<kBlkWarps>(a, head_groups, total_slots);
    if (warp >= kPairWarps) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairProducerRegs));
        if (warp == kPairWarps) produce_blk<KF, VF>(a, sm.blk, ring, head_groups, total_slots, lane);
        return;
    }
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairComputeRegs));
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(&sm.tmem);
    uint32_t lane_base;
    asm volatile("or.b32 %0, %1, %2;" : "=r"(lane_base) : "r"(lut_addr), "r"(static_cast<uint32_t>(lane) << 2));
    const int rows = group < NH ? group : NH;
    const int hw = warp & (kBlkWarps - 1), par = warp / kBlkWarps;
    const uint32_t k_sub = bs * (KF::RB + KF::NB), v_sub = bs * (VF::RB + VF::NB);
    const uint32_t k_off = hw * k_sub, v_off = kBlkWarps * k_sub + hw * v_sub;
    using Tiles = WarpTiles<KF, VF, NH, true>;
    Tiles wt;
    const uint32_t quarter = (32u * (warp & 3)) << 16;
    wt.tm = tmem + quarter + Tiles::kTmCols * (warp >> 2);
    const uint32_t partner_tm = tmem + quarter + Tiles::kTmCols * ((warp + kBlkWarps) >> 2);
    constexpr int kBs = 16 * TPB;
    volatile int* abort_flag = &sm.abort;
    // Absolute slot a (the a-th slot the producer fills) sits at ring
    // position a % ring.n with phase (a / ring.n) & 1, tracked incrementally.
    // Slots are owned in runs of SPG (32 tokens): run a / SPG goes to the warp
    // of that parity, so each ring position always serves the same warps.
    constexpr int SPG = 2 / TPB;
    const uint32_t ring_n = static_cast<uint32_t>(ring.n);
    uint32_t consumed = 0, pos_c = 0, phase_c = 0;  // absolute slot, ring position and phase of the item start

    for (int64_t slot = blockIdx.x; slot < total_slots; slot += gridDim.x) {
        Item it;
        if (!item_of<kBlkWarps>(a, slot, head_groups, total_slots, it)) continue;
        if (it.win) continue;  // windows are not listed: the prologue's window CTAs take them
        const int h = it.h + hw;                      // this warp's KV head
        const int head0 = h * group + it.hg * 8;      // its first query head of the item
        float* rec = record_of(a, it.b, h, it.split, group) + it.hg * 8 * (kHeadDim + 2);
        const int64_t q_off = (static_cast<int64_t>(it.b) * a.num_q_heads + head0) * kHeadDim;
        wt.begin(a.qrot + q_off, a.qjl_q + q_off, rows, r, c);
        const int ntiles = (it.t1 - it.t0 + 15) >> 4;
        const int nslots = (ntiles + TPB - 1) / TPB;
        const int tok_end = it.t1 - it.t0;
        bool bad = __any_sync(kFull, *abort_flag != 0);  // one value for the whole warp
        // This warp's first slot of the item: the item's first slot when its run is ours, else the
        // first slot of the next run. Runs of this warp then follow every 2 SPG slots.
        int j = 0;
        {
            const uint32_t run0 = consumed / SPG, off0 = consumed % SPG;
            if (static_cast<int>(run0 & 1u) != par) j = SPG - static_cast<int>(off0);
        }
        uint32_t pos = pos_c + static_cast<uint32_t>(j), phase = phase_c;
        if (pos >= ring_n) {
            pos -= ring_n;
            phase ^= 1u;
        }
        while (j < nslots) {
            // with 16-token blocks the two slots of a run are taken together (the first run of an item
            // may start on its second slot, and the last may be cut short by the item's end)
            const bool two = TPB == 1 && ((consumed + static_cast<uint32_t>(j)) & 1u) == 0 && j + 1 < nslots;
            const int span = two ? 2 : 1;
            if (!bad) {
                uint32_t s1 = pos + 1, ph1 = phase;
                if (s1 == ring_n) {
                    s1 = 0;
                    ph1 ^= 1u;
                }
                bool ok = mbar_wait(smem_addr(&sm.blk.full[pos]), phase);
                if (two && ok) ok = mbar_wait(smem_addr(&sm.blk.full[s1]), ph1);
                if (!__all_sync(kFull, ok)) {
                    bad = true;
                    if (lane == 0) {
                        *abort_flag = 1;
                        if (a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
                    }
                } else {
                    const uint32_t sb0 = ring.slot(static_cast<int>(pos));
                    const uint32_t kb0 = sb0 + k_off, vb0 = sb0 + v_off;
                    const int tok0 = (TPB * j) * 16;  // first token of the step within the item
                    if constexpr (TPB == 1) {
                        if (two) {
                            const uint32_t sb1 = ring.slot(static_cast<int>(s1));
                            const uint32_t kb1 = sb1 + k_off, vb1 = sb1 + v_off;
                            wt.step2(kb0, kb0 + 16 * KF::RB, vb0, vb0 + 16 * VF::RB, min(16, tok_end - tok0), kb1,
                                     kb1 + 16 * KF::RB, vb1, vb1 + 16 * VF::RB, min(16, tok_end - tok0 - 16),
                                     lane_base, r, c);
                        } else {
                            wt.step(kb0, kb0 + 16 * KF::RB, vb0, vb0 + 16 * VF::RB, min(16, tok_end - tok0),
                                    lane_base, r, c);
                        }
                    } else {
                        if (tok0 + 16 < tok_end)
                            wt.step2(kb0, kb0 + kBs * KF::RB, vb0, vb0 + kBs * VF::RB, 16, kb0 + 16 * KF::RB,
                                     kb0 + kBs * KF::RB + 16 * KF::NB, vb0 + 16 * VF::RB,
                                     vb0 + kBs * VF::RB + 16 * VF::NB, min(16, tok_end - tok0 - 16), lane_base,
                                     r, c);
                        else
                            wt.step(kb0, kb0 + kBs * KF::RB, vb0, vb0 + kBs * VF::RB, min(16, tok_end - tok0),
                                    lane_base, r, c);
                    }
                    __syncwarp();
                    if (lane == 0) {  // this warp is done with the slot(s)
                        mbar_arrive(smem_addr(&sm.blk.empty[pos]));
                        if (two) mbar_arrive(smem_addr(&sm.blk.empty[s1]));
                    }
                }
            }
            // to this warp's next run: past this run and the partner's run of SPG slots
            j += span + SPG;
            pos += static_cast<uint32_t>(span + SPG);
            if (pos >= ring_n) {
                pos -= ring_n;
                phase ^= 1u;
            }
        }
        {
            const uint32_t np = pos_c + static_cast<uint32_t>(nslots);
            phase_c ^= (np / ring_n) & 1u;
            pos_c = np % ring_n;
        }
        consumed += static_cast<uint32_t>(nslots);
        // Fold the odd warp's state into the even warp's; both agree on an abort.
        if (par == 1) {
            wt.export_state();
            tm_fence_before_sync();
        }
        const bool abort = bar_any(1 + hw, 64, bad);
        if (par == 0) {
            tm_fence_after_sync();
            if (!abort) wt.absorb(partner_tm);
            tm_fence_before_sync();
        }
        bar_sync(1 + hw, 64);  // the odd warp's columns are free again
        if (par == 1) tm_fence_after_sync();
        if (abort) break;
        if (par == 0) wt.finish(rec, rec + 1, rec + 2, kHeadDim + 2, kHeadDim + 2, rows, r, c);
    }
    // Every compute warp is done with tensor memory before warp 0 frees it.
    tm_wait_st();
    tm_fence_before_sync();
    bar_sync(1 + kBlkWarps, kPairWarps * 32);
    if (warp == 0) {
        tm_fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ==== per-head kernel: one KV head per work item, tiles spread over the warps =========
//
// For KV head counts that are not a multiple of 8. A work item is (query-head
// group, KV head, sequence, split); tile t of an item goes to compute warp t %
// NW, which keeps its own ring of slots; the warps merge their states through
// shared memory at the end of the item.

template <int NW>
struct Smem {
    float red_o[NW][8][kHeadDim];         // per-warp value accumulators (V packed order)
    float red_m[NW][8], red_l[NW][8];
    unsigned long long full[NW][kStages];   // producer -> warp: slot filled (tx bytes)
    unsigned long long empty[NW][kStages];  // warp -> producer: slot free again
    int ids[2][kMaxItemTiles];              // producer: block ids of the current and next item
    int abort_flag;
};

// Dynamic shared memory: [Smem][pad to a 64 KB boundary][table][rings]. The
// size assumes the Smem block plus the window offset of the dynamic area stays
// within the first 64 KB; the kernel checks the layout before using it.
template <int NW>
__host__ __device__ constexpr size_t smem_head_bytes() {
    return (sizeof(Smem<NW>) + 127) / 128 * 128;
}
template <int NW, uint32_t SB>
__host__ __device__ constexpr size_t smem_bytes() {
    return 2 * static_cast<size_t>(kLut) + static_cast<size_t>(NW) * kStages * SB;
}

// Producer warp. Lane w (w < NW) feeds compute warp w: in each packed work
// item (in the compute warps' order) warp w consumes tiles w, w + NW, ...; for
// each, the lane waits for the ring slot's release and copies the tile in. A
// slot is [K rows][K norms][V rows][V norms]; with 16-token blocks each half is
// one whole sub-page (rows then norms) and takes one bulk copy. While the
// lanes stream an item, all 32 lanes read the next item's block ids into a
// shared-memory buffer, so table reads never sit between consecutive copies.
template <class KF, class VF, int NW>
__device__ void produce_head(const DecodeArgs& a, Smem<NW>& sm, uint32_t ring_addr, int head_groups,
                             int64_t total_slots, int lane) {
    if (a.withhold_copies) return;  // test hook: the compute warps' waits expire
    constexpr uint32_t kKRows = 16 * KF::RB, kVRows = 16 * VF::RB;
    constexpr uint32_t kKNorms = 16 * KF::NB, kVNorms = 16 * VF::NB;
    constexpr uint32_t kKTile = kKRows + kKNorms, kTileBytes = kKTile + kVRows + kVNorms;
    constexpr uint32_t kStageBytes = stage_bytes<KF, VF>();
    constexpr int kPer = kMaxItemTiles / 32;
    const int H = a.kc.num_heads, bs = a.block_size;
    const bool bs_pow2 = (bs & (bs - 1)) == 0, whole = bs == 16;
    const uint32_t my_ring = ring_addr + static_cast<uint32_t>(lane * kStages * kStageBytes);
    auto read_ids = [&](const Item& it, int (&v)[kPer]) {
        const int ntiles = (it.t1 - it.t0 + 15) >> 4;
        const int32_t* bt = a.block_tables + static_cast<int64_t>(it.b) * a.max_blocks;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int tl = lane + 32 * k;
            v[k] = tl < ntiles ? __ldg(bt + (it.t0 + 16 * tl) / bs) : 0;
        }
    };
    uint32_t fill = 0;
    int buf = 0;
    int64_t slot = blockIdx.x;
    Item cur;
    bool have = next_packed<1>(a, slot, head_groups, total_slots, cur);
    if (have) {
        int v[kPer];
        read_ids(cur, v);
#pragma unroll
        for (int k = 0; k < kPer; ++k) sm.ids[0][lane + 32 * k] = v[k];
    }
    __syncwarp();
    bool stop = false;
    while (have) {
        int64_t slot_n = slot + gridDim.x;
        Item nxt;
        const bool have_n = next_packed<1>(a, slot_n, head_groups, total_slots, nxt);
        int v[kPer];
        if (have_n) read_ids(nxt, v);
        const int ntiles = (cur.t1 - cur.t0 + 15) >> 4;
        if (lane < NW) {
            const uint32_t full0 = smem_addr(&sm.full[lane][0]), empty0 = smem_addr(&sm.empty[lane][0]);
#pragma unroll 1
            for (int tl = lane; tl < ntiles; tl += NW) {
                const uint32_t st = fill % kStages, use = fill / kStages;
                const uint32_t full = full0 + 8 * st;
                if (use > 0) {
                    bool ready = false;
                    for (uint32_t i = 0; i < kSpinLimit && !ready; ++i) ready = mbar_test(empty0 + 8 * st, (use - 1) & 1u);
                    if (!ready) {
                        // The compute warps stop on their own bounded waits.
                        if (a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
                        stop = true;
                        break;
                    }
                }
                int blk = sm.ids[buf][tl];
                if (blk < 0 || blk >= a.num_blocks) {
                    if (a.d_err) atomicOr(a.d_err, TQ_DERR_BLOCK);
                    blk = 0;
                }
                const int tok = cur.t0 + 16 * tl;
                const int off = bs_pow2 ? (tok & (bs - 1)) : tok % bs;
                const int64_t sp = (static_cast<int64_t>(blk) * H + cur.h) * bs;
                const uint8_t* ks = a.k_pages + sp * (KF::RB + KF::NB);
                const uint8_t* vs = a.v_pages + sp * (VF::RB + VF::NB);
                const uint32_t dst = my_ring + st * kStageBytes;
                mbar_expect(full, kTileBytes);
                if (whole) {
                    bulk_copy(dst, ks, kKTile, full);
                    bulk_copy(dst + kKTile, vs, kVRows + kVNorms, full);
                } else {
                    bulk_copy(dst, ks + off * KF::RB, kKRows, full);
                    bulk_copy(dst + kKRows, ks + bs * KF::RB + KF::NB * off, kKNorms, full);
                    bulk_copy(dst + kKTile, vs + off * VF::RB, kVRows, full);
                    bulk_copy(dst + kKTile + kVRows, vs + bs * VF::RB + VF::NB * off, kVNorms, full);
                }
                ++fill;
            }
        }
        if (__any_sync(kFull, stop)) break;
        buf ^= 1;
        if (have_n) {
#pragma unroll
            for (int k = 0; k < kPer; ++k) sm.ids[buf][lane + 32 * k] = v[k];
        }
        __syncwarp();
        cur = nxt;
        have = have_n;
        slot = slot_n;
    }
    // Wait (bounded) for this lane's copies in flight before the CTA can retire.
    if (lane < NW)
        for (uint32_t f = fill > kStages ? fill - kStages : 0; f < fill; ++f)
            if (!mbar_wait(smem_addr(&sm.full[lane][f % kStages]), (f / kStages) & 1u)) break;
}

template <class KF, class VF, int NH, int NW>
__global__ void __launch_bounds__((NW + 1) * 32, 1) decode_mma_kernel(DecodeArgs a, LutValues tv, int group,
                                                                      int head_groups, int64_t total_slots) {
    static_assert(NH == 4 || NH == 8, "4 or 8 query heads per item");
    extern __shared__ __align__(128) uint8_t dsm[];
    Smem<NW>& sm = *reinterpret_cast<Smem<NW>*>(dsm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;
    constexpr uint32_t kStageBytes = stage_bytes<KF, VF>();

    const uint32_t dsm_addr = smem_addr(dsm);
    const uint32_t lut_addr =
        (dsm_addr + static_cast<uint32_t>(smem_head_bytes<NW>()) + (kLut - 1)) & ~uint32_t(kLut - 1);
    const uint32_t ring_addr = lut_addr + kLut;
    if (ring_addr + NW * kStages * kStageBytes > dsm_addr + smem_bytes<NW, kStageBytes>()) {
        griddep_wait();
        if (threadIdx.x == 0 && a.d_err) atomicOr(a.d_err, TQ_DERR_LAUNCH);
        return;
    }
    fill_table(reinterpret_cast<uint32_t*>(dsm + (lut_addr - dsm_addr)), tv, threadIdx.x, (NW + 1) * 32);
    if (threadIdx.x == 0) {
        for (int w = 0; w < NW; ++w)
            for (int s = 0; s < kStages; ++s) {
                mbar_init_count(smem_addr(&sm.full[w][s]), 1);
                mbar_init_count(smem_addr(&sm.empty[w][s]), 1);
            }
        sm.abort_flag = 0;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    // The table and barriers above overlap the prologue's end; its work list and queries are read
    // from here on.
    griddep_wait();
    griddep_launch_dependents();
    total_slots = listed_slots<1>(a, head_groups, total_slots);
    if (warp == NW) {
        produce_head<KF, VF, NW>(a, sm, ring_addr, head_groups, total_slots, lane);
        return;
    }
    uint32_t lane_base;
    asm volatile("or.b32 %0, %1, %2;" : "=r"(lane_base) : "r"(lut_addr), "r"(static_cast<uint32_t>(lane) << 2));
    const int rows = group < NH ? group : NH;
    const uint32_t my_ring = ring_addr + static_cast<uint32_t>(warp * kStages * kStageBytes);
    uint32_t consumed = 0;
    bool timed_out = false;
    WarpTiles<KF, VF, NH> wt;

    for (int64_t slot = blockIdx.x; slot < total_slots; slot += gridDim.x) {
        Item it;
        if (!item_of<1>(a, slot, head_groups, total_slots, it)) continue;
        const int head0 = it.h * group + it.hg * 8;  // first query head of the item
        if (it.win) continue;  // windows are not listed: the prologue's window CTAs take them
        {
            const int64_t q_off = (static_cast<int64_t>(it.b) * a.num_q_heads + head0) * kHeadDim;
            wt.begin(a.qrot + q_off, a.qjl_q + q_off, rows, r, c);
            const int ntiles = (it.t1 - it.t0 + 15) >> 4;
            const int n_mine = ntiles > warp ? (ntiles - warp + NW - 1) / NW : 0;
            for (int k = 0; k < n_mine; ++k) {
                const uint32_t st = consumed % kStages;
                if (!mbar_wait(smem_addr(&sm.full[warp][st]), (consumed / kStages) & 1u)) {
                    timed_out = true;
                    break;
                }
                // Slot layout: [K rows][K norms][V rows][V norms].
                const uint32_t kbase = my_ring + st * kStageBytes, vbase = kbase + 16 * (KF::RB + KF::NB);
                wt.step(kbase, kbase + 16 * KF::RB, vbase, vbase + 16 * VF::RB,
                        min(16, it.t1 - (it.t0 + 16 * (warp + k * NW))), lane_base, r, c);
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&sm.empty[warp][st]));  // slot free for the producer
                ++consumed;
            }
            wt.finish(&sm.red_m[warp][0], &sm.red_l[warp][0], &sm.red_o[warp][0][0], 1, kHeadDim, rows, r, c);
        }
        if (timed_out && lane == 0) {
            atomicOr(&sm.abort_flag, 1);
            if (a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
        }
        named_sync<NW * 32>();
        if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) break;
        // Merge the warps and write one record per query head.
        float* rec = record_of(a, it.b, it.h, it.split, group);
        for (int e = threadIdx.x; e < rows * kHeadDim; e += NW * 32) {
            const int g = e / kHeadDim, jj = e - g * kHeadDim;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NW; ++w) M = fmaxf(M, sm.red_m[w][g]);
            float Ls = 0.0f, A = 0.0f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    const float mw = sm.red_m[w][g];
                    if (mw != -INFINITY) {
                        const float f = ex2(mw - M);
                        Ls += sm.red_l[w][g] * f;
                        A += sm.red_o[w][g][jj] * f;
                    }
                }
            }
            float* rg = rec + (it.hg * 8 + g) * (kHeadDim + 2);
            rg[2 + jj] = A;
            if (jj == 0) {
                rg[0] = M;
                rg[1] = Ls;
            }
        }
        named_sync<NW * 32>();
    }
}

// ---- The decode prologue: one launch of kProThreads-thread CTAs that builds
// the work list (CTA 0), rotates the queries (the next n_rot CTAs) and
// attends over the dense windows (the rest), so the decode kernel follows one
// launch instead of three.
constexpr int kProThreads = 256, kProWarps = kProThreads / 32;
constexpr int kListBuckets = kMaxItemTiles + 1;  // partial splits by tile count 1 .. 256
static_assert(kProThreads == kMaxItemTiles, "one thread per partial-split bucket");
constexpr int kRotRows = kProWarps;  // query rows per rotation CTA, one per warp

union ProSmem {
    struct {
        int cursor[kListBuckets];  // partial splits per tile count, then write cursors
        int warp_tot[32];
        int tot_full, base_full;
    } wl;
    float zs[kRotRows][kHeadDim];  // rotated rows of a rotation CTA
    struct {
        float qs[16][kHeadDim];    // group-wise: the head's query rows
        float part[16][kHeadDim];  // second half's partial products
        float qr[16][kHeadDim];    // recipe keys: the rotated rows
    } dense;
    struct {
        float m[kProWarps][8], l[kProWarps][8];
        float o[kProWarps][8][kHeadDim];
    } win;
    struct {
        uint8_t idx[kProWarps][kHeadDim];  // fused window append: each warp's index bytes
        float r[kProWarps][kHeadDim];      // and residual scratch
    } app;
};

// Exclusive scan of x over the CTA; total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_tot, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int v = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;  // inclusive over the warps
    }
    __syncthreads();
    const int excl = (warp ? warp_tot[warp - 1] : 0) + v - x;
    total = warp_tot[nw - 1];
    __syncthreads();  // warp_tot is reused by the next call
    return excl;
}

// Work list of the tensor-core kernels: the (sequence, split) pairs of every
// non-empty packed work item, longest first: every full split (sequence by
// sequence), then the partial last splits by decreasing tile count, in
// sequence order within a tile count (a counting sort whose bucket offsets
// come from one scan over the CTA); and their number. Dealt in snake order
// (item_of), this balances the persistent CTAs about as well as greedy
// longest-first assignment. The order is a function of the lengths alone, so
// an item always runs on the same CTA after the same items: results are the
// same bit for bit from call to call.
__device__ __forceinline__ void build_work_list(const DecodeArgs& a, ProSmem& sm) {
    auto& s = sm.wl;
    const int tid = threadIdx.x;
    auto geometry = [&](int b, int& nf, int& part_tiles) {
        int L = __ldg(a.seq_lens + b);
        L = L < 0 ? 0 : (L > a.max_seq_len ? a.max_seq_len : L);
        const int P = L - min(a.window, L);
        nf = P / a.split_tokens;
        const int rem = P - nf * a.split_tokens;
        part_tiles = (rem + 15) >> 4;
    };
    for (int i = tid; i < kListBuckets; i += kProThreads) s.cursor[i] = 0;
    if (tid == 0) s.tot_full = 0;
    __syncthreads();
    for (int b = tid; b < a.batch; b += kProThreads) {
        int nf, pt;
        geometry(b, nf, pt);
        if (nf) atomicAdd(&s.tot_full, nf);
        if (pt) atomicAdd(&s.cursor[pt], 1);
    }
    __syncthreads();
    {
        // thread t owns bucket kMaxItemTiles - t: the longest partial splits come first, after
        // the full ones (every thread reads its count before the scan's first barrier)
        const int k = kMaxItemTiles - tid;
        int n_part;
        const int of = block_exclusive_scan(s.cursor[k], s.warp_tot, n_part);
        s.cursor[k] = s.tot_full + of;
        if (tid == 0) {
            s.base_full = 0;
            *a.work_count = s.tot_full + n_part;
        }
    }
    __syncthreads();
    int2* list = reinterpret_cast<int2*>(a.work_list);
    for (int b0 = 0; b0 < a.batch; b0 += kProThreads) {
        const int b = b0 + tid;
        int nf = 0, pt = 0;
        if (b < a.batch) geometry(b, nf, pt);
        int n_full;
        const int of = block_exclusive_scan(nf, s.warp_tot, n_full);
        for (int j = 0; j < nf; ++j) list[s.base_full + of + j] = make_int2(b, j);
        __syncthreads();
        if (tid == 0) s.base_full += n_full;
        __syncthreads();
    }
    // Partial splits: one warp, 32 sequences at a time; lanes with the same tile count take
    // consecutive places in lane order after that bucket's cursor.
    if (tid < 32) {
        for (int b0 = 0; b0 < a.batch; b0 += 32) {
            const int b = b0 + tid;
            int nf = 0, pt = 0;
            if (b < a.batch) geometry(b, nf, pt);
            const unsigned peers = __match_any_sync(kFull, pt);
            const int rank = __popc(peers & ((1u << tid) - 1u));
            const int base = pt ? s.cursor[pt] : 0;
            __syncwarp();
            if (pt && rank == 0) s.cursor[pt] = base + __popc(peers);
            __syncwarp();
            if (pt) list[base + rank] = make_int2(b, nf);
        }
    }
}

// The dense bf16 window of one (sequence, KV head, group of <= 8 query heads),
// on CUDA cores: warp w takes window tokens w, w + kProWarps, ...; the warps
// merge their (max, sum, accumulator) states in shared memory into the
// window's record (split max_splits).
template <int NH>
__device__ __forceinline__ void window_unit(const DecodeArgs& a, int group, int head_groups, int64_t u,
                                            ProSmem& sm) {
    auto& s = sm.win;
    const int H = a.kc.num_heads;
    Item it;
    it.hg = static_cast<int>(u % head_groups);
    u /= head_groups;
    it.h = static_cast<int>(u % H);
    it.b = static_cast<int>(u / H);
    it.split = a.max_splits;
    if (!item_range(a, it)) return;  // no window tokens (the same for the whole CTA)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = group < NH ? group : NH;
    const int head0 = it.h * group + it.hg * 8;
    // Fused window append: the slot the new token takes, if this decode reads it (as in append_vector).
    int t_new = -1;
    const __nv_bfloat16 *kn = nullptr, *vn = nullptr;
    if (a.app_on) {
        const int L = max(__ldg(a.seq_lens + it.b), 0), S = a.app_sinks, W = a.app_window;
        const int slot = L < S ? L : (W > 0 ? S + (L - S) % W : -1);
        if (slot >= 0 && slot < it.t1) t_new = slot;
        const int64_t row = static_cast<int64_t>(it.b) * H + it.h;
        kn = static_cast<const __nv_bfloat16*>(a.k_new) + row * kHeadDim;
        vn = static_cast<const __nv_bfloat16*>(a.v_new) + row * kHeadDim;
    }
    window_state<NH>(a, it, it.h, head0, rows, warp, kProWarps, lane, &s.m[warp][0], &s.l[warp][0], &s.o[warp][0][0],
                 1, kHeadDim, t_new, kn, vn);
    __syncthreads();
    float* rec = record_of(a, it.b, it.h, it.split, group) + it.hg * 8 * (kHeadDim + 2);
    for (int e = threadIdx.x; e < rows * kHeadDim; e += kProThreads) {
        const int g = e / kHeadDim, j = e - g * kHeadDim;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kProWarps; ++w) M = fmaxf(M, s.m[w][g]);
        float Ls = 0.0f, A = 0.0f;
#pragma unroll
        for (int w = 0; w < kProWarps; ++w) {
            const float mw = s.m[w][g];
            if (mw != -INFINITY) {
                const float f = ex2(mw - M);
                Ls += s.l[w][g] * f;
                A += s.o[w][g][j] * f;
            }
        }
        float* rg = rec + g * (kHeadDim + 2);
        rg[2 + j] = A;
        if (j == 0) {
            rg[0] = M;
            rg[1] = Ls;
        }
    }
}

// Rotated queries: q_r = pi_K(H(s_K * q) / sqrt(128)) * scale * log2(e). Rotation
// CTA `blk` takes the kRotRows consecutive (b, query head) rows from
// blk * kRotRows, one warp per row. With QJL keys it also writes
// qjl_out = sqrt(pi/2)/128 * S q_r, S applied in rotated (not packed)
// coordinate order, as the residual it projected: the rows' q_r go to shared
// memory and thread i computes output i of 4 rows, so the CTA reads S (64 KB,
// from L2) once for its rows.
__device__ __forceinline__ void rotate_rows(const DecodeArgs& a, int group, int64_t total, int64_t blk,
                                            float* qjl_out, ProSmem& sm) {
    const DevCodec& kc = a.kc;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t row0 = blk * kRotRows;
    const int64_t row = row0 + w;
    if (row < total) {
        const int hq = static_cast<int>(row % a.num_q_heads), h = hq / group;
        const uint2 raw = *reinterpret_cast<const uint2*>(q + row * kHeadDim + 4 * lane);
        float z[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u)};
#pragma unroll
        for (int i = 0; i < 4; ++i) z[i] *= kc.sign[4 * lane + i];
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
        for (int i = 0; i < 4; ++i) {
            z[i] *= sc;
            a.qrot[row * kHeadDim + kc.pos[h * kHeadDim + 4 * lane + i]] = z[i];
            sm.zs[w][4 * lane + i] = z[i];
        }
    }
    if (qjl_out == nullptr) return;  // uniform over the CTA
    __syncthreads();
    // (S q_r)_i = sum_j S[i][j] q_r[j]: thread (i, half) for rows 4 half .. 4 half + 3
    static_assert(kRotRows == 8 && kProThreads == 2 * kHeadDim, "two halves of four rows");
    const int i = threadIdx.x & (kHeadDim - 1), r0 = (threadIdx.x >> 7) * 4;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    // 16 loads of S (from L2) in flight per thread: this loop is the prologue's longest chain
#pragma unroll 16
    for (int j = 0; j < kHeadDim; ++j) {
        const float sij = __ldg(kc.qjl_st + j * kHeadDim + i);  // S^T row j, coalesced over i
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fmaf(sij, sm.zs[r0 + k][j], acc[k]);
    }
    constexpr float kappa = 1.2533141373155003f / kHeadDim;  // sqrt(pi/2) / d, the estimator's constant
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (row0 + r0 + k < total) qjl_out[(row0 + r0 + k) * kHeadDim + qjl_slot(i)] = acc[k] * kappa;
}

// Group-wise K: q_r = R_h q * scale * log2(e) in packed order (R_h from the
// codec: rot_t entry (h, j, p) = R_h[p][j]). Rotation CTA `unit` = (b, KV
// head) takes the head's query rows (group <= 16) together: their q goes to
// shared memory, thread (p, half) sums packed position p of every row over
// half of the j range, and the CTA reads R_h (64 KB, rows contiguous over p)
// once.
template <bool RECIPE>
__device__ __forceinline__ void rotate_rows_dense(const DecodeArgs& a, int group, int64_t unit, ProSmem& sm) {
    const DevCodec& kc = a.kc;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
    const int H = kc.num_heads, p = threadIdx.x & (kHeadDim - 1), half = threadIdx.x >> 7;
    const int h = static_cast<int>(unit % H);
    const int64_t b = unit / H;
    const int64_t row0 = b * a.num_q_heads + static_cast<int64_t>(h) * group;
    for (int g = half; g < group; g += 2) sm.dense.qs[g][p] = __bfloat162float(q[(row0 + g) * kHeadDim + p]);
    __syncthreads();
    const float* rt = kc.rot_t + static_cast<int64_t>(h) * kHeadDim * kHeadDim;
    float acc[16];
#pragma unroll
    for (int g = 0; g < 16; ++g) acc[g] = 0.0f;
    const int j0 = half * (kHeadDim / 2);
    // 16 loads of R_h (from L2) in flight per thread: this loop is the prologue's longest chain
#pragma unroll 16
    for (int j = j0; j < j0 + kHeadDim / 2; ++j) {
        const float rjp = __ldg(rt + j * kHeadDim + p);
#pragma unroll
        for (int g = 0; g < 16; ++g)
            if (g < group) acc[g] = fmaf(rjp, sm.dense.qs[g][j], acc[g]);
    }
    if (half) {
#pragma unroll
        for (int g = 0; g < 16; ++g)
            if (g < group) sm.dense.part[g][p] = acc[g];
    }
    __syncthreads();
    if (!half) {
#pragma unroll
        for (int g = 0; g < 16; ++g)
            if (g < group) {
                const float y = (acc[g] + sm.dense.part[g][p]) * a.scale_log2;
                a.qrot[(row0 + g) * kHeadDim + p] = y;
                if constexpr (RECIPE) sm.dense.qr[g][p] = y;
            }
    }
    if constexpr (RECIPE) {
        // Per group g of 64 packed positions: (kappa S_g q'_g)_i = kappa sum_j S_g^T[j][i] q'[64g + j],
        // kappa = sqrt(pi/2)/64, written at packed position 64g + i (S_0^T then S_1^T in the codec).
        __syncthreads();
        constexpr float kappa = 1.2533141373155003f / 64.0f;
        const int grp = p >> 6, i = p & 63;
        const float* st = kc.qjl_st + grp * 64 * 64;
        for (int g = half; g < group; g += 2) {
            float z = 0.0f;
#pragma unroll 16
            for (int j = 0; j < 64; ++j) z = fmaf(__ldg(st + j * 64 + i), sm.dense.qr[g][64 * grp + j], z);
            a.qjl_q[(row0 + g) * kHeadDim + recipe_slot(p)] = z * kappa;
        }
    }
}

// CTA 0: the work list; CTAs 1 .. n_rot: query rotation; the rest: windows
// (b, KV head, query-head group). The decode kernel that follows may start as
// soon as every CTA here has begun (it waits for this grid's results itself).
template <int KMODE, int NH>
__global__ void __launch_bounds__(kProThreads, NH == 4 ? 2 : 1) decode_prologue_kernel(DecodeArgs a, int group,
                                                                                      int head_groups,
                                                                                      int64_t n_rot, int64_t n_win) {
    __shared__ ProSmem sm;
    griddep_launch_dependents();
    // Launched as a dependent of whatever ran before in the stream (the step's window append, say):
    // nothing is read before that kernel is complete; only the launch overlaps its end.
    griddep_wait();
    const int64_t blk = blockIdx.x;
    if (blk == 0) {
        build_work_list(a, sm);
    } else if (blk <= n_rot) {
        if constexpr (KMODE == kGroupwise || KMODE == kRecipe)
            rotate_rows_dense<KMODE == kRecipe>(a, group, blk - 1, sm);
        else
            rotate_rows(a, group, static_cast<int64_t>(a.batch) * a.num_q_heads, blk - 1,
                        KMODE == kQjl ? a.qjl_q : nullptr, sm);
    } else if (blk <= n_rot + n_win) {
        window_unit<NH>(a, group, head_groups, blk - 1 - n_rot, sm);
    } else {
        // fused window append: one warp per (sequence, KV head, K or V)
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int64_t vec = (blk - 1 - n_rot - n_win) * kProWarps + warp;
        if (vec < static_cast<int64_t>(a.batch) * a.kc.num_heads * 2)
            append_vector(a.kc, a.vc, vec, static_cast<const __nv_bfloat16*>(a.k_new),
                          static_cast<const __nv_bfloat16*>(a.v_new), static_cast<__nv_bfloat16*>(a.k_win_w),
                          static_cast<__nv_bfloat16*>(a.v_win_w), a.app_window, a.app_sinks, a.seq_lens,
                          a.block_tables, a.max_blocks, a.k_pages_w, a.v_pages_w, a.num_blocks, a.block_size,
                          a.d_err, sm.app.idx[warp], sm.app.r[warp], lane);
    }
}

constexpr int kMaxDynSmem = 227 * 1024;

template <class KF, class VF, int NH>
tq_status launch_fmt(const DecodeArgs& a, const LutValues& tv, int group, cudaStream_t s) {
    constexpr int NW = kNW;
    constexpr size_t head_bytes = smem_bytes<NW, stage_bytes<KF, VF>()>();
    static_assert(head_bytes <= kMaxDynSmem, "shared memory of the per-head decode kernel");
    // The block kernel wants at least kBlkMinSlots slots beside the table.
    const bool blk = a.kc.num_heads % kBlkWarps == 0 &&
                     static_cast<size_t>(blk_slot_bytes<KF, VF>(a.block_size)) * kBlkMinSlots <=
                         static_cast<size_t>(kMaxDynSmem) - kLut - 4096;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(TQ_ERR_CUDA, "cudaGetDevice failed");
    // The paired kernel's register split assumes the compiler gave it kPairLaunchRegs per thread;
    // with any other figure the compute warps' request could not be met, so that kernel is not used.
    static std::atomic<int> pair_regs_ok{0};
    const cudaError_t attr_err = once_per_device(dev, [] {
        cudaFuncAttributes fa1{}, fa2{};
        const bool ok = cudaFuncGetAttributes(&fa1, decode_pair_kernel<KF, VF, NH, 1>) == cudaSuccess &&
                        cudaFuncGetAttributes(&fa2, decode_pair_kernel<KF, VF, NH, 2>) == cudaSuccess &&
                        fa1.numRegs == kPairLaunchRegs && fa2.numRegs == kPairLaunchRegs;
        pair_regs_ok.store(ok ? 1 : 0);
        cudaGetLastError();
        cudaError_t attr_err;
        attr_err = cudaFuncSetAttribute(decode_mma_kernel<KF, VF, NH, NW>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(head_bytes));
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode_blk_kernel<KF, VF, NH, 1>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode_blk_kernel<KF, VF, NH, 2>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode_blk_kernel<KF, VF, NH, 0>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode_pair_kernel<KF, VF, NH, 1>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode_pair_kernel<KF, VF, NH, 2>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        return attr_err;
    });
    if (attr_err != cudaSuccess) return fail(TQ_ERR_CUDA, "cannot reserve shared memory for the decode kernel");
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int head_groups = group > 8 ? group / 8 : 1;
    const int64_t rows = static_cast<int64_t>(a.batch) * a.num_q_heads;
    // One prologue launch builds the work list, rotates the queries and attends over the windows.
    const int64_t n_rot = (KF::MODE == kGroupwise || KF::MODE == kRecipe) ? static_cast<int64_t>(a.batch) * a.kc.num_heads
                                                 : (rows + kRotRows - 1) / kRotRows;
    const int64_t n_win = a.window > 0 ? static_cast<int64_t>(a.batch) * a.kc.num_heads * head_groups : 0;
    const int64_t n_app = a.app_on ? (static_cast<int64_t>(a.batch) * a.kc.num_heads * 2 + kProWarps - 1) / kProWarps : 0;
    if (1 + n_rot + n_win + n_app > INT32_MAX) return TQ_ERR_UNSUPPORTED;
    const cudaError_t pe = launch_dependent(decode_prologue_kernel<KF::MODE, NH>,
                                            dim3(static_cast<unsigned>(1 + n_rot + n_win + n_app)), dim3(kProThreads),
                                            0, s, a, group, head_groups, n_rot, n_win);
    if (pe != cudaSuccess) return fail(TQ_ERR_CUDA, std::string("decode prologue launch: ") + cudaGetErrorString(pe));
    const int64_t units = static_cast<int64_t>(a.items_per_unit) * a.batch * head_groups *
                          (blk ? a.kc.num_heads / kBlkWarps : a.kc.num_heads);
    const int grid = static_cast<int>(units < sms ? units : sms);
    if (grid > 0) {
        const dim3 threads((kBlkWarps + 1) * 32), pair_threads(kPairThreads);
        // TQ_DECODE_PAIR=0 takes the block kernel instead of the paired one, for cross-checks.
        const char* pair_env = std::getenv("TQ_DECODE_PAIR");
        const bool pair = !(pair_env && pair_env[0] == '0') && pair_regs_ok.load() == 1;
        // The paired kernel wants two run pairs of slots beside the table (one more slot than that
        // covers the ring's split around the 64 KB-aligned table).
        const bool pair_fits = static_cast<size_t>(blk_slot_bytes<KF, VF>(a.block_size)) * 5 <=
                               static_cast<size_t>(kMaxDynSmem) - kLut - 4096;
        // The decode kernel may start while the prologue ends (it waits for the prologue's results).
        cudaError_t le;
        if (blk && pair && pair_fits && a.block_size == 16)
            le = launch_dependent(decode_pair_kernel<KF, VF, NH, 1>, grid, pair_threads, kMaxDynSmem, s, a, tv, group,
                                  head_groups, units);
        else if (blk && pair && pair_fits && a.block_size == 32)
            le = launch_dependent(decode_pair_kernel<KF, VF, NH, 2>, grid, pair_threads, kMaxDynSmem, s, a, tv, group,
                                  head_groups, units);
        else if (blk && a.block_size == 16)
            le = launch_dependent(decode_blk_kernel<KF, VF, NH, 1>, grid, threads, kMaxDynSmem, s, a, tv, group,
                                  head_groups, units);
        else if (blk && a.block_size == 32)
            le = launch_dependent(decode_blk_kernel<KF, VF, NH, 2>, grid, threads, kMaxDynSmem, s, a, tv, group,
                                  head_groups, units);
        else if (blk)
            le = launch_dependent(decode_blk_kernel<KF, VF, NH, 0>, grid, threads, kMaxDynSmem, s, a, tv, group,
                                  head_groups, units);
        else
            le = launch_dependent(decode_mma_kernel<KF, VF, NH, NW>, grid, dim3((NW + 1) * 32), head_bytes, s, a, tv,
                                  group, head_groups, units);
        if (le != cudaSuccess) return fail(TQ_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(le));
    }
    return TQ_OK;
}

template <class F>
bool same_format(const tq_codec* c) {
    const tq_format_desc& d = c->desc;
    const int mode = d.qjl ? (d.groupwise ? kRecipe : kQjl) : (d.groupwise ? kGroupwise : kPlain);
    if (mode != F::MODE) return false;
    if constexpr (F::MODE == kRecipe) {
        // the kernel's compile-time row layout must be the codec's
        if (!c->dev.recipe || c->dev.sign_off[0] != F::SO0 || c->dev.sign_off[1] != F::SO1 ||
            c->dev.byte_off[1] != F::BOFF1 || c->dev.row_bytes != F::RB + F::NB)
            return false;
    }
    if (F::N1 == 0) return d.n_groups == 1 && d.group_bits[0] == F::B0;
    return d.n_groups == 2 && d.group_bits[0] == F::B0 && d.group_size[0] == F::N0 && d.group_bits[1] == F::B1 &&
           d.group_size[1] == F::N1;
}

template <class KF, class VF>
tq_status launch_heads(const DecodeArgs& a, const LutValues& tv, int group, cudaStream_t s) {
    return group <= 4 ? launch_fmt<KF, VF, 4>(a, tv, group, s) : launch_fmt<KF, VF, 8>(a, tv, group, s);
}

// V formats the tensor-core kernel is instantiated for, per K format.
template <class KF>
tq_status dispatch_v(const DecodeArgs& a, const tq_codec* vc, const LutValues& tv, int group, cudaStream_t s) {
    if constexpr (KF::MODE == kGroupwise || KF::MODE == kRecipe) {
        if (same_format<M43G>(vc)) return launch_heads<KF, M43G>(a, tv, group, s);
    } else if constexpr (KF::MODE == kQjl) {
        if (same_format<U4>(vc)) return launch_heads<KF, U4>(a, tv, group, s);
        if (same_format<M43>(vc)) return launch_heads<KF, M43>(a, tv, group, s);
    } else {
        if (same_format<U4>(vc)) return launch_heads<KF, U4>(a, tv, group, s);
        if (same_format<M43>(vc)) return launch_heads<KF, M43>(a, tv, group, s);
        if (same_format<U3>(vc)) return launch_heads<KF, U3>(a, tv, group, s);
    }
    return TQ_ERR_UNSUPPORTED;
}

}  // namespace

tq_status launch_decode_mma(const DecodeArgs& a, const tq_codec* kc, const tq_codec* vc, int group, void* stream) {
    if (a.block_size % 16 != 0) return TQ_ERR_UNSUPPORTED;
    if (a.split_tokens > 16 * kMaxItemTiles) return TQ_ERR_UNSUPPORTED;  // the producer's id buffer
    if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return TQ_ERR_UNSUPPORTED;
    // One table per bit width serves K and V: every group of that width must
    // share its centroids (group-wise codebooks are per group dimension).
    LutValues tv{};
    bool set[5] = {false, false, false, false, false};
    for (const tq_codec* c : {kc, vc})
        for (int g = 0; g < c->desc.n_groups; ++g) {
            const int bits = c->desc.group_bits[g];
            if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
            float* dst = bits == 4 ? tv.c4 : (bits == 3 ? tv.c3 : tv.c2);
            for (int i = 0; i < (1 << bits); ++i) {
                if (set[bits] && dst[i] != c->cent[g][i]) return TQ_ERR_UNSUPPORTED;
                dst[i] = c->cent[g][i];
            }
            set[bits] = true;
        }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (same_format<U4>(kc)) return dispatch_v<U4>(a, vc, tv, group, s);
    if (same_format<M43>(kc)) return dispatch_v<M43>(a, vc, tv, group, s);
    if (same_format<M42>(kc)) return dispatch_v<M42>(a, vc, tv, group, s);
    if (same_format<M32Q>(kc)) return dispatch_v<M32Q>(a, vc, tv, group, s);
    if (same_format<M43Q>(kc)) return dispatch_v<M43Q>(a, vc, tv, group, s);
    if (same_format<M43G>(kc)) return dispatch_v<M43G>(a, vc, tv, group, s);
    if (same_format<M32R>(kc)) return dispatch_v<M32R>(a, vc, tv, group, s);
    return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq

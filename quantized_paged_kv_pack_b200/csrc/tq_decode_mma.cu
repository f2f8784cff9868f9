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
// Data movement: each warp owns a ring of 4 tile slots in shared memory that
// its lane 0 fills with cp.async.bulk copies (index rows of K and V, and their
// norms) tracked by one mbarrier per slot, running up to 4 tiles ahead and
// across the boundary into the CTA's next work item. Every wait is bounded;
// on expiry the kernel sets TQ_DERR_TIMEOUT, drains its copies (bounded) and
// stops. CTAs are persistent and take work items (sequence, KV head, split of
// the packed tokens, query-head group) in a fixed stride; the 8 warps share an
// item's tiles and merge their (max, sum, accumulator) states at its end.

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
constexpr int kNW = 8;              // warps per CTA
constexpr int kStages = 4;          // ring slots per warp
constexpr int kStageBytes = 2176;   // 16 rows of K and V (<= 64 index bytes each) + 2 x 32 norm bytes
constexpr int kLut = 65536;         // bytes of the dequantization table
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr float kSlack = 8.0f;                 // log2 slack of the running max
constexpr float kSlackInv = 1.0f / 256.0f;     // 2^-kSlack, folded into P'

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
    static_assert(IB <= 64, "tile slot holds rows of at most 64 index bytes");
};
using U4 = Fmt<4, 128, 0, 0>;
using U3 = Fmt<3, 128, 0, 0>;
using M43 = Fmt<4, 64, 3, 64>;
using M42 = Fmt<4, 32, 2, 96>;

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

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void mbar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
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

// Bounded wait for phase `parity` of `bar`; false when the limit expired.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kSpinLimit; ++i)
        if (mbar_try(bar, parity)) return true;
    return false;
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

// ---- work items -----------------------------------------------------------------

struct Item {
    int b, h, hg, split, t0, t1;
    bool win;
};

// Geometry of slot `slot`; false when the slot has no work.
__device__ __forceinline__ bool item_of(const DecodeArgs& a, int64_t slot, int head_groups, Item& it) {
    int64_t t = slot;
    it.hg = static_cast<int>(t % head_groups);
    t /= head_groups;
    it.h = static_cast<int>(t % a.kc.num_heads);
    t /= a.kc.num_heads;
    it.b = static_cast<int>(t % a.batch);
    it.split = static_cast<int>(t / a.batch);
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

// Number of this warp's tiles in a packed item.
__device__ __forceinline__ int warp_tiles(const Item& it, int warp) {
    if (it.win) return 0;
    const int n = (it.t1 - it.t0 + 15) >> 4;
    return n > warp ? (n - warp + kNW - 1) / kNW : 0;
}

// Block id of this warp's k-th tile of an item, lane k holding entry k (k < 32).
__device__ __forceinline__ int load_block_ids(const DecodeArgs& a, const Item& it, int warp, int lane) {
    const int n = warp_tiles(it, warp);
    int blk = 0;
    if (lane < n) {
        const int tok = it.t0 + 16 * (warp + lane * kNW);
        blk = __ldg(a.block_tables + static_cast<int64_t>(it.b) * a.max_blocks + tok / a.block_size);
        if (blk < 0 || blk >= a.num_blocks) {
            if (a.d_err) atomicOr(a.d_err, TQ_DERR_BLOCK);
            blk = 0;
        }
    }
    return blk;
}

struct Smem {
    float red_o[kNW][8][kHeadDim];         // per-warp value accumulators (V packed order)
    float red_m[kNW][8], red_l[kNW][8];
    unsigned long long bar[kNW][kStages];
    int abort_flag;
};

constexpr int kRingBytes = kNW * kStages * kStageBytes;
constexpr size_t kSmemHead = (sizeof(Smem) + 127) / 128 * 128;
constexpr size_t kFrontBytes = kSmemHead + kRingBytes;
// Layout: [Smem][rings][pad to a 64 KB boundary][table]. The table needs the
// window offset of the dynamic area to be small; the kernel checks.
constexpr size_t kSmemBytes = (kFrontBytes + kLut - 1) / kLut * kLut + kLut;

template <class KF, class VF, int NH>
__global__ void __launch_bounds__(kNW * 32, 1) decode_mma_kernel(DecodeArgs a, LutValues tv, int group,
                                                                 int head_groups, int64_t total_slots) {
    static_assert(NH == 4 || NH == 8, "4 or 8 query heads per item");
    constexpr int NJ = NH / 4;  // n-tiles: 4 heads x {hi, lo} each
    extern __shared__ __align__(128) uint8_t dsm[];
    Smem& sm = *reinterpret_cast<Smem*>(dsm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane >> 2, c = lane & 3;

    const uint32_t dsm_addr = static_cast<uint32_t>(__cvta_generic_to_shared(dsm));
    const uint32_t ring_addr = dsm_addr + static_cast<uint32_t>(kSmemHead);
    const uint32_t lut_addr = (dsm_addr + static_cast<uint32_t>(kFrontBytes) + (kLut - 1)) & ~uint32_t(kLut - 1);
    if (lut_addr + kLut > dsm_addr + kSmemBytes) {
        if (threadIdx.x == 0 && a.d_err) atomicOr(a.d_err, TQ_DERR_LAUNCH);
        return;
    }
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
    if (lane == 0)
        for (int s = 0; s < kStages; ++s)
            mbar_init(static_cast<uint32_t>(__cvta_generic_to_shared(&sm.bar[warp][s])));
    if (threadIdx.x == 0) sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    uint32_t lane_base;
    asm volatile("or.b32 %0, %1, %2;" : "=r"(lane_base) : "r"(lut_addr), "r"(static_cast<uint32_t>(lane) << 2));

    const int H = a.kc.num_heads, bs = a.block_size;
    const uint8_t* const k_pages = a.k_pages;
    const uint8_t* const v_pages = a.v_pages;
    const bool bs_pow2 = (bs & (bs - 1)) == 0;
    const int rows = group < NH ? group : NH;
    const uint32_t my_ring = ring_addr + static_cast<uint32_t>(warp * kStages * kStageBytes);
    const uint32_t bar0 = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.bar[warp][0]));
    constexpr uint32_t kKBytes = 16 * KF::IB, kVBytes = 16 * VF::IB;
    constexpr uint32_t kTileBytes = kKBytes + kVBytes + 64;

    // ---- producer (lane 0 issues; every lane tracks the cursor) ----
    // The producer feeds this warp's tiles in consumption order, one tile per
    // consumed tile after an initial fill of the ring. It keeps the block ids of
    // its current item and, loaded one item earlier, of the next one.
    struct Cursor {
        int64_t slot;
        Item it;
        int n;    // this warp's tiles in the item (0: no item)
        int ids;  // lane k: block id of the warp's k-th tile
    };
    auto find_from = [&](int64_t slot, Cursor& cur) {
        cur.n = 0;
        for (; slot < total_slots; slot += gridDim.x) {
            if (!item_of(a, slot, head_groups, cur.it)) continue;
            const int n = warp_tiles(cur.it, warp);
            if (n > 0) {
                cur.slot = slot;
                cur.n = n;
                cur.ids = load_block_ids(a, cur.it, warp, lane);
                return;
            }
        }
        cur.slot = total_slots;
    };
    Cursor pc, nc;
    find_from(blockIdx.x, pc);
    find_from(pc.n ? pc.slot + gridDim.x : total_slots, nc);
    int p_k = 0;
    uint32_t issued = 0, consumed = 0, phase_bits = 0;
    bool timed_out = false;
    const uint32_t k_row_bytes = KF::IB + 2, v_row_bytes = VF::IB + 2;

    auto issue_one = [&]() {
        if (pc.n == 0) return;
        const int blk = __shfl_sync(kFull, pc.ids, p_k);
        if (lane == 0) {
            const int tok = pc.it.t0 + 16 * (warp + p_k * kNW);
            const int64_t sp = (static_cast<int64_t>(blk) * H + pc.it.h) * bs;
            const uint8_t* ks = k_pages + sp * k_row_bytes;
            const uint8_t* vs = v_pages + sp * v_row_bytes;
            const int off = bs_pow2 ? (tok & (bs - 1)) : tok % bs;
            const uint32_t s = issued % kStages;
            const uint32_t dst = my_ring + s * kStageBytes, bar = bar0 + 8 * s;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_expect(bar, kTileBytes);
            bulk_copy(dst, ks + off * KF::IB, kKBytes, bar);
            bulk_copy(dst + kKBytes, vs + off * VF::IB, kVBytes, bar);
            bulk_copy(dst + kKBytes + kVBytes, ks + bs * KF::IB + 2 * off, 32, bar);
            bulk_copy(dst + kKBytes + kVBytes + 32, vs + bs * VF::IB + 2 * off, 32, bar);
        }
        ++issued;
        if (++p_k == pc.n) {
            pc = nc;
            p_k = 0;
            find_from(pc.n ? pc.slot + gridDim.x : total_slots, nc);
        }
    };
    for (int i = 0; i < kStages; ++i) issue_one();

    const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
    for (int64_t slot = blockIdx.x; slot < total_slots; slot += gridDim.x) {
        Item it;
        if (!item_of(a, slot, head_groups, it)) continue;
        const int head0 = it.h * group + it.hg * 8;  // first query head of the item

        if (it.win) {
            // Dense bf16 window on CUDA cores: tokens spread over the warps.
            float qv[8][4], m[8], l[8], acc[8][4];
#pragma unroll
            for (int g = 0; g < 8; ++g) {
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
            for (int tk = it.t0 + warp; tk < it.t1; tk += kNW) {
                const int64_t base = ((static_cast<int64_t>(it.b) * H + it.h) * a.window + tk) * kHeadDim + 4 * lane;
                const uint2 kr = *reinterpret_cast<const uint2*>(kw + base);
                const uint2 vr = *reinterpret_cast<const uint2*>(vw + base);
                const float kx[4] = {__uint_as_float(kr.x << 16), __uint_as_float(kr.x & 0xffff0000u),
                                     __uint_as_float(kr.y << 16), __uint_as_float(kr.y & 0xffff0000u)};
                const float vx[4] = {__uint_as_float(vr.x << 16), __uint_as_float(vr.x & 0xffff0000u),
                                     __uint_as_float(vr.y << 16), __uint_as_float(vr.y & 0xffff0000u)};
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    if (g < rows) {
                        float s = qv[g][0] * kx[0] + qv[g][1] * kx[1] + qv[g][2] * kx[2] + qv[g][3] * kx[3];
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
            }
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                if (g < rows) {
                    if (lane == 0) {
                        sm.red_m[warp][g] = m[g];
                        sm.red_l[warp][g] = l[g];
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) sm.red_o[warp][g][4 * lane + i] = acc[g][i];
                }
            }
        } else {
            const int n_mine = warp_tiles(it, warp);
            // Query-side B fragments: column r of n-tile j is head 4j + r/2, half r%2.
            uint32_t bq[8][NJ][2];
            {
                const float* qr = a.qrot + (static_cast<int64_t>(it.b) * a.num_q_heads + head0) * kHeadDim;
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const int p = s < KF::KS0 ? c * (KF::N0 / 4) + 4 * s
                                              : KF::N0 + c * (KF::N1 / 4) + 4 * (s - KF::KS0);
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int head = 4 * j + (r >> 1);
                        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (head < rows) x = __ldcg(reinterpret_cast<const float4*>(qr + head * kHeadDim + p));
                        const __half2 h01 = __floats2half2_rn(x.x, x.y), h23 = __floats2half2_rn(x.z, x.w);
                        __half2 v01 = h01, v23 = h23;
                        if (r & 1) {
                            v01 = __floats2half2_rn(x.x - __low2float(h01), x.y - __high2float(h01));
                            v23 = __floats2half2_rn(x.z - __low2float(h23), x.w - __high2float(h23));
                        }
                        bq[s][j][0] = *reinterpret_cast<const uint32_t*>(&v01);
                        bq[s][j][1] = *reinterpret_cast<const uint32_t*>(&v23);
                    }
                }
            }
            float o[8][NJ][4];
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
                for (int j = 0; j < NJ; ++j) o[q][j][0] = o[q][j][1] = o[q][j][2] = o[q][j][3] = 0.0f;
            float m_run[NJ], l_run[NJ];
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                m_run[j] = -INFINITY;
                l_run[j] = 0.0f;
            }
            // The producer runs ahead into this item's tiles and then the next item's.
            for (int k = 0; k < n_mine && !timed_out; ++k) {
                const uint32_t s = consumed % kStages;
                if (!mbar_wait(bar0 + 8 * s, (phase_bits >> s) & 1u)) {
                    timed_out = true;
                    break;
                }
                phase_bits ^= 1u << s;
                const uint32_t slot_a = my_ring + s * kStageBytes;
                const uint32_t kbase = slot_a, vbase = slot_a + kKBytes, nbase = slot_a + kKBytes + kVBytes;
                const int nvalid = min(16, it.t1 - (it.t0 + 16 * (warp + k * kNW)));

                // ---- S^T = K^ Q'^T: rows tokens r, r + 8 ----
                // Two accumulator chains (even / odd k-steps) halve the MMA dependency depth.
                float sacc[2][NJ][4];
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int j = 0; j < NJ; ++j) sacc[u][j][0] = sacc[u][j][1] = sacc[u][j][2] = sacc[u][j][3] = 0.0f;
                {
                    constexpr int KW0 = (KF::KC0 + 3) / 4;
                    constexpr bool A0 = KF::KC0 % 4 == 0;
                    const Words<KW0> k0a = lds_span<KF::KC0, A0>(kbase + r * KF::IB + c * KF::KC0);
                    const Words<KW0> k0b = lds_span<KF::KC0, A0>(kbase + (r + 8) * KF::IB + c * KF::KC0);
                    const uint32_t base0 = lut_base<KF::B0>(lane_base);
                    static_for<0, KF::KS0>([&](auto si) {
                        constexpr int s_ = decltype(si)::value;
                        const uint32_t a0 = lut(pair_addr<KF::B0, 4 * s_ * KF::B0, KW0>(k0a.w, base0));
                        const uint32_t a1 = lut(pair_addr<KF::B0, 4 * s_ * KF::B0, KW0>(k0b.w, base0));
                        const uint32_t a2 = lut(pair_addr<KF::B0, (4 * s_ + 2) * KF::B0, KW0>(k0a.w, base0));
                        const uint32_t a3 = lut(pair_addr<KF::B0, (4 * s_ + 2) * KF::B0, KW0>(k0b.w, base0));
#pragma unroll
                        for (int j = 0; j < NJ; ++j)
                            mma16816(sacc[s_ & 1][j], a0, a1, a2, a3, bq[s_][j][0], bq[s_][j][1]);
                    });
                    if constexpr (KF::N1 > 0) {
                        constexpr int KW1 = (KF::KC1 + 3) / 4;
                        constexpr bool A1 = (KF::KC1 % 4 == 0) && (KF::BOFF1 % 4 == 0);
                        const uint32_t g1 = KF::BOFF1 + c * KF::KC1;
                        const Words<KW1> k1a = lds_span<KF::KC1, A1>(kbase + r * KF::IB + g1);
                        const Words<KW1> k1b = lds_span<KF::KC1, A1>(kbase + (r + 8) * KF::IB + g1);
                        const uint32_t base1 = lut_base<KF::B1>(lane_base);
                        static_for<0, KF::KS1>([&](auto si) {
                            constexpr int s_ = decltype(si)::value;
                            const uint32_t a0 = lut(pair_addr<KF::B1, 4 * s_ * KF::B1, KW1>(k1a.w, base1));
                            const uint32_t a1 = lut(pair_addr<KF::B1, 4 * s_ * KF::B1, KW1>(k1b.w, base1));
                            const uint32_t a2 = lut(pair_addr<KF::B1, (4 * s_ + 2) * KF::B1, KW1>(k1a.w, base1));
                            const uint32_t a3 = lut(pair_addr<KF::B1, (4 * s_ + 2) * KF::B1, KW1>(k1b.w, base1));
#pragma unroll
                            for (int j = 0; j < NJ; ++j)
                                mma16816(sacc[(KF::KS0 + s_) & 1][j], a0, a1, a2, a3, bq[KF::KS0 + s_][j][0],
                                         bq[KF::KS0 + s_][j][1]);
                        });
                    }
                }

                // ---- online softmax: head 4j + c, tokens r and r + 8 ----
                const float nk0 = __half2float(__ushort_as_half(static_cast<unsigned short>(lds16(nbase + 2 * r))));
                const float nk1 =
                    __half2float(__ushort_as_half(static_cast<unsigned short>(lds16(nbase + 2 * (r + 8)))));
                const float nv0 =
                    __half2float(__ushort_as_half(static_cast<unsigned short>(lds16(nbase + 32 + 2 * r))));
                const float nv1 =
                    __half2float(__ushort_as_half(static_cast<unsigned short>(lds16(nbase + 32 + 2 * (r + 8)))));
                const bool ok0 = r < nvalid, ok1 = r + 8 < nvalid;
                const float nv0s = nv0 * kSlackInv, nv1s = nv1 * kSlackInv;
                uint32_t bp[NJ][2];
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const float s0 =
                        ok0 ? ((sacc[0][j][0] + sacc[1][j][0]) + (sacc[0][j][1] + sacc[1][j][1])) * nk0 : -INFINITY;
                    const float s1 =
                        ok1 ? ((sacc[0][j][2] + sacc[1][j][2]) + (sacc[0][j][3] + sacc[1][j][3])) * nk1 : -INFINITY;
                    float mx = fmaxf(s0, s1);
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                    // The reference max only moves when a score exceeds it by more
                    // than 2^kSlack, so weights stay below 2^kSlack and the
                    // accumulators are rescaled rarely.
                    const bool grow = mx > m_run[j] + kSlack;
                    // A loop with a data-dependent trip count keeps this rare path a branch.
                    const int rescale = __any_sync(kFull, grow) ? 1 : 0;
#pragma unroll 1
                    for (int t = 0; t < rescale; ++t) {
                        const float m_new = grow ? mx : m_run[j];
                        const float alpha = grow ? ex2(m_run[j] - m_new) : 1.0f;
                        l_run[j] *= alpha;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            o[q][j][0] *= alpha;
                            o[q][j][1] *= alpha;
                            o[q][j][2] *= alpha;
                            o[q][j][3] *= alpha;
                        }
                        m_run[j] = m_new;
                    }
                    const float mref = m_run[j] == -INFINITY ? 0.0f : m_run[j];
                    const float p0 = ex2(s0 - mref), p1 = ex2(s1 - mref);
                    l_run[j] += p0 + p1;
                    // P' carries 2^-kSlack so that weight x norm stays within fp16.
                    const float w0 = ok0 ? p0 * nv0s : 0.0f, w1 = ok1 ? p1 * nv1s : 0.0f;
                    const __half2 X = __floats2half2_rn(w0, w1);
                    const __half2 Y = __floats2half2_rn(w0 - __low2float(X), w1 - __high2float(X));
                    const uint32_t xu = *reinterpret_cast<const uint32_t*>(&X);
                    const uint32_t yu = *reinterpret_cast<const uint32_t*>(&Y);
                    // B fragment of P'^T: tokens (2c, 2c+1) and (2c+8, 2c+9), column r.
                    const int srcA = 8 * c + (r >> 1), srcB = srcA + 4;
                    const uint32_t xa = __shfl_sync(kFull, xu, srcA), ya = __shfl_sync(kFull, yu, srcA);
                    const uint32_t xb = __shfl_sync(kFull, xu, srcB), yb = __shfl_sync(kFull, yu, srcB);
                    const uint32_t pa = (r & 1) ? ya : xa, pb = (r & 1) ? yb : xb;
                    bp[j][0] = prmt(pa, pb, 0x5410u);
                    bp[j][1] = prmt(pa, pb, 0x7632u);
                }

                // ---- O^T += V^T P'^T over 8 coordinate row tiles ----
                {
                    const uint32_t r0 = vbase + (2 * c) * VF::IB, r1 = r0 + VF::IB;
                    const uint32_t r8 = vbase + (2 * c + 8) * VF::IB, r9 = r8 + VF::IB;
                    {
                        constexpr int NW0 = (VF::VC0 + 3) / 4;
                        constexpr bool A0 = VF::VC0 % 4 == 0;
                        const Words<NW0> t0 = lds_span<VF::VC0, A0>(r0 + r * VF::VC0);
                        const Words<NW0> t1 = lds_span<VF::VC0, A0>(r1 + r * VF::VC0);
                        const Words<NW0> t8 = lds_span<VF::VC0, A0>(r8 + r * VF::VC0);
                        const Words<NW0> t9 = lds_span<VF::VC0, A0>(r9 + r * VF::VC0);
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
#pragma unroll
                            for (int j = 0; j < NJ; ++j) mma16816(o[q][j], a0, a1, a2, a3, bp[j][0], bp[j][1]);
                        });
                    }
                    if constexpr (VF::N1 > 0) {
                        constexpr int NW1 = (VF::VC1 + 3) / 4;
                        constexpr bool A1 = (VF::VC1 % 4 == 0) && (VF::BOFF1 % 4 == 0);
                        const uint32_t g1 = VF::BOFF1 + r * VF::VC1;
                        const Words<NW1> t0 = lds_span<VF::VC1, A1>(r0 + g1);
                        const Words<NW1> t1 = lds_span<VF::VC1, A1>(r1 + g1);
                        const Words<NW1> t8 = lds_span<VF::VC1, A1>(r8 + g1);
                        const Words<NW1> t9 = lds_span<VF::VC1, A1>(r9 + g1);
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
#pragma unroll
                            for (int j = 0; j < NJ; ++j)
                                mma16816(o[VF::MT0 + q][j], a0, a1, a2, a3, bp[j][0], bp[j][1]);
                        });
                    }
                }
                __syncwarp();
                ++consumed;
                issue_one();  // refill the slot just freed
            }
            // Publish this warp's state (head 4j + c; positions of rows r and r + 8).
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                float lsum = l_run[j];
                lsum += __shfl_xor_sync(kFull, lsum, 4);
                lsum += __shfl_xor_sync(kFull, lsum, 8);
                lsum += __shfl_xor_sync(kFull, lsum, 16);
                const int head = 4 * j + c;
                if (head < rows) {
                    if (r == 0) {
                        sm.red_m[warp][head] = m_run[j];
                        sm.red_l[warp][head] = lsum;
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const bool g1 = q >= VF::MT0;
                        const int ql = g1 ? q - VF::MT0 : q;
                        const int per = g1 ? VF::N1 / 8 : VF::N0 / 8;
                        const int p0 = (g1 ? VF::N0 : 0) + r * per + 2 * ql;
                        *reinterpret_cast<float2*>(&sm.red_o[warp][head][p0]) =
                            make_float2((o[q][j][0] + o[q][j][1]) * 256.0f, (o[q][j][2] + o[q][j][3]) * 256.0f);
                    }
                }
            }
        }
        if (timed_out && lane == 0) {
            atomicOr(&sm.abort_flag, 1);
            if (a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
        }
        __syncthreads();
        if (sm.abort_flag) break;
        // Merge the warps and write one record per query head.
        float* rec = a.ws + ((static_cast<int64_t>(it.b) * H + it.h) * a.items_per_unit + it.split) *
                                static_cast<int64_t>(group) * (kHeadDim + 2);
        for (int e = threadIdx.x; e < rows * kHeadDim; e += kNW * 32) {
            const int g = e / kHeadDim, jj = e - g * kHeadDim;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kNW; ++w) M = fmaxf(M, sm.red_m[w][g]);
            float Ls = 0.0f, A = 0.0f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kNW; ++w) {
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
        __syncthreads();
    }
    // Drain this warp's copies still in flight (bounded) before the CTA exits.
    for (; consumed < issued; ++consumed) {
        const uint32_t s = consumed % kStages;
        if (!mbar_wait(bar0 + 8 * s, (phase_bits >> s) & 1u)) {
            if (lane == 0 && a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
            break;
        }
        phase_bits ^= 1u << s;
    }
}

// Rotated queries: q_r = pi_K(H(s_K * q) / sqrt(128)) * scale * log2(e), one warp per (b, query head).
__global__ void __launch_bounds__(128) rotate_queries_kernel(DevCodec kc, const __nv_bfloat16* q, int num_q_heads,
                                                              int group, int64_t total, float scale_log2, float* out) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (row >= total) return;
    const int hq = static_cast<int>(row % num_q_heads), h = hq / group;
    const uint2 raw = *reinterpret_cast<const uint2*>(q + row * kHeadDim + 4 * lane);
    float z[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u), __uint_as_float(raw.y << 16),
                  __uint_as_float(raw.y & 0xffff0000u)};
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
    const float sc = scale_log2 * 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
    for (int i = 0; i < 4; ++i) out[row * kHeadDim + kc.pos[h * kHeadDim + 4 * lane + i]] = z[i] * sc;
}

template <class KF, class VF, int NH>
tq_status launch_fmt(const DecodeArgs& a, const LutValues& tv, int group, cudaStream_t s) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(decode_mma_kernel<KF, VF, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kSmemBytes));
    });
    if (attr_err != cudaSuccess) return fail(TQ_ERR_CUDA, "cannot reserve shared memory for the decode kernel");
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int head_groups = group > 8 ? group / 8 : 1;
    const int64_t rows = static_cast<int64_t>(a.batch) * a.num_q_heads;
    rotate_queries_kernel<<<static_cast<unsigned>((rows + 3) / 4), 128, 0, s>>>(
        a.kc, static_cast<const __nv_bfloat16*>(a.q), a.num_q_heads, group, rows, a.scale_log2, a.qrot);
    const int64_t slots = static_cast<int64_t>(a.items_per_unit) * a.batch * a.kc.num_heads * head_groups;
    const int grid = static_cast<int>(slots < sms ? slots : sms);
    if (grid > 0)
        decode_mma_kernel<KF, VF, NH><<<grid, kNW * 32, kSmemBytes, s>>>(a, tv, group, head_groups, slots);
    return TQ_OK;
}

template <class F>
bool same_format(const tq_codec* c) {
    const tq_format_desc& d = c->desc;
    if (F::N1 == 0) return d.n_groups == 1 && d.group_bits[0] == F::B0;
    return d.n_groups == 2 && d.group_bits[0] == F::B0 && d.group_size[0] == F::N0 && d.group_bits[1] == F::B1 &&
           d.group_size[1] == F::N1;
}

template <class KF, class VF>
tq_status launch_heads(const DecodeArgs& a, const LutValues& tv, int group, cudaStream_t s) {
    return group <= 4 ? launch_fmt<KF, VF, 4>(a, tv, group, s) : launch_fmt<KF, VF, 8>(a, tv, group, s);
}

template <class KF>
tq_status dispatch_v(const DecodeArgs& a, const tq_codec* vc, const LutValues& tv, int group, cudaStream_t s) {
    if (same_format<U4>(vc)) return launch_heads<KF, U4>(a, tv, group, s);
    if (same_format<M43>(vc)) return launch_heads<KF, M43>(a, tv, group, s);
    if (same_format<U3>(vc)) return launch_heads<KF, U3>(a, tv, group, s);
    return TQ_ERR_UNSUPPORTED;
}

}  // namespace

tq_status launch_decode_mma(const DecodeArgs& a, const tq_codec* kc, const tq_codec* vc, int group, void* stream) {
    if (a.block_size % 16 != 0) return TQ_ERR_UNSUPPORTED;
    if (group != 1 && group != 2 && group != 4 && group != 8 && group != 16) return TQ_ERR_UNSUPPORTED;
    if (a.split_tokens > 16 * kNW * 32) return TQ_ERR_UNSUPPORTED;  // at most 32 tiles per warp and item
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

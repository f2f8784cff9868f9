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

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kPW = 8;               // warps per CTA
constexpr int kCells = 129;          // v = 64 u in [-64, 64], cells round(v) + 64
constexpr float kCellScale = 64.0f;

struct QuantCell {                   // one table entry (8 bytes)
    float thr;                       // boundary inside the cell (in units of v), +inf if none
    int below;                       // boundaries strictly below the cell
};

struct PackSmem {
    QuantCell cells[kCells][32];     // replicated per lane: conflict-free 8-byte lookups
    uint32_t bfrag[2][8][2][32][2];  // [K/V][a][n-tile][lane][reg]: B operands (+-1 bf16 pairs)
    uint8_t rows[kPW][16][64];       // staged index rows of a warp's 16 tokens
    unsigned short norms[kPW][16];
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
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

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ double warp4_sum_d(double v) {
    v += __shfl_xor_sync(kFull, v, 1);
    v += __shfl_xor_sync(kFull, v, 2);
    return v;
}

__global__ void __launch_bounds__(kPW * 32, 2) pack_u4_kernel(DevCodec kc, DevCodec vc, QuantCell* __restrict__ g_cells,
                                                          const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          const int64_t* __restrict__ slots, int64_t num_tokens,
                                                          uint8_t* __restrict__ k_pages, uint8_t* __restrict__ v_pages,
                                                          int64_t num_blocks, int block_size, int* __restrict__ d_err) {
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
        const int bp = 4 * (rr >> 1) + 2 * t + (rr & 1);  // output column b' of lane rr in n-tile t
        uint32_t regs[2];
        for (int q = 0; q < 2; ++q) {
            unsigned short h[2];
            for (int e = 0; e < 2; ++e) {
                const int b = 4 * cc + 2 * q + e;          // input coordinate b of this k-slot
                const float val = sign[16 * a + b] * ((__popc(bp & b) & 1) ? -1.0f : 1.0f);
                h[e] = val > 0 ? 0x3F80 : 0xBF80;
            }
            regs[q] = static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16);
        }
        sm.bfrag[which][a][t][ln][0] = regs[0];
        sm.bfrag[which][a][t][ln][1] = regs[1];
    }
    __syncthreads();

    const int64_t H = kc.num_heads;
    const int64_t groups = (num_tokens + 15) / 16;
    const int64_t units = groups * H * 2;
    const int64_t capacity = num_blocks * block_size;
    const uint32_t cell_lane = static_cast<uint32_t>(__cvta_generic_to_shared(&sm.cells[0][lane]));
    // address of cell e for this lane = cell_lane + e * 256; e = bits(v + 1.5*2^23) - 0x4B400000 + 64
    const uint32_t cell_adj = cell_lane + 64u * 256u - 0x40000000u;

    for (int64_t u = static_cast<int64_t>(blockIdx.x) * kPW + warp; u < units;
         u += static_cast<int64_t>(gridDim.x) * kPW) {
        const int which = static_cast<int>(u & 1);
        const int64_t gh = u >> 1;
        const int h = static_cast<int>(gh % H);
        const int64_t t0 = (gh / H) * 16;
        const __nv_bfloat16* src = which ? v : k;

        // Slots of the 16 tokens (lane i < 16 holds token t0 + i).
        int64_t my_slot = -1;
        if (lane < 16 && t0 + lane < num_tokens) my_slot = __ldg(slots + t0 + lane);
        const bool live_lo = t0 + r < num_tokens, live_hi = t0 + r + 8 < num_tokens;

        // A operands: tokens r and r + 8, coordinates 16a + 4c .. 16a + 4c + 3.
        uint2 xa[8], xb[8];
        const __nv_bfloat16* p_lo = src + ((t0 + r) * H + h) * kHeadDim + 4 * c;
        const __nv_bfloat16* p_hi = src + ((t0 + r + 8) * H + h) * kHeadDim + 4 * c;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            xa[a] = live_lo ? __ldg(reinterpret_cast<const uint2*>(p_lo + 16 * a)) : make_uint2(0, 0);
            xb[a] = live_hi ? __ldg(reinterpret_cast<const uint2*>(p_hi + 16 * a)) : make_uint2(0, 0);
        }

        // z = (H_16 D_s) per a on the tensor cores: zc[a][t] holds columns b' = 4c + 2t + {0,1}.
        float zc[8][2][4];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const uint2 bf = *reinterpret_cast<const uint2*>(&sm.bfrag[which][a][t][lane][0]);
                mma_bf16(zc[a][t], xa[a].x, xb[a].x, xa[a].y, xb[a].y, bf.x, bf.y);
            }
        }

        // Sum of exact squares (fp32), per token, over this lane's 32 coordinates then the 4 lanes.
        float ss_lo = 0.0f, ss_hi = 0.0f;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const float l0 = __uint_as_float(xa[a].x << 16), l1 = __uint_as_float(xa[a].x & 0xffff0000u);
            const float l2 = __uint_as_float(xa[a].y << 16), l3 = __uint_as_float(xa[a].y & 0xffff0000u);
            const float h0 = __uint_as_float(xb[a].x << 16), h1 = __uint_as_float(xb[a].x & 0xffff0000u);
            const float h2 = __uint_as_float(xb[a].y << 16), h3 = __uint_as_float(xb[a].y & 0xffff0000u);
            ss_lo = fmaf(l0, l0, fmaf(l1, l1, fmaf(l2, l2, fmaf(l3, l3, ss_lo))));
            ss_hi = fmaf(h0, h0, fmaf(h1, h1, fmaf(h2, h2, fmaf(h3, h3, ss_hi))));
        }
        ss_lo += __shfl_xor_sync(kFull, ss_lo, 1);
        ss_lo += __shfl_xor_sync(kFull, ss_lo, 2);
        ss_hi += __shfl_xor_sync(kFull, ss_hi, 1);
        ss_hi += __shfl_xor_sync(kFull, ss_hi, 2);

        // fp16 norm, correctly rounded; fp64 when the fp32 value is too close to call.
        float n_tok[2];
        unsigned short n16[2];
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

        // H_8 across a (three butterfly stages on packed pairs).
        uint64_t zp[8][2][2];  // [a][t][token]: (columns 2c, 2c+1 of n-tile t)
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                zp[a][t][0] = pk(zc[a][t][0], zc[a][t][1]);
                zp[a][t][1] = pk(zc[a][t][2], zc[a][t][3]);
            }
#pragma unroll
        for (int m = 1; m < 8; m <<= 1)
#pragma unroll
            for (int a = 0; a < 8; ++a)
                if (!(a & m))
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint64_t x0 = zp[a][t][i], x1 = zp[a | m][t][i];
                            zp[a][t][i] = add2(x0, x1);
                            zp[a | m][t][i] = sub2(x0, x1);
                        }

        // Quantize: v = z * 64 / (sqrt(128) n); cell lookup; pack 4 nibbles per (token, a').
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float n = n_tok[i];
            float kq = n > 0.0f ? kCellScale / (n * 11.313708498984761f) : 0.0f;
            if (!(kq < 3.0e38f)) kq = 0.0f;  // norms too small to scale: treat as the zero vector
            const uint64_t kq2 = pk(kq, kq);
            const uint64_t magic2 = pk(12582912.0f, 12582912.0f);
            unsigned short* row = reinterpret_cast<unsigned short*>(&sm.rows[warp][r + 8 * i][0]);
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                uint32_t word = 0;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const uint64_t vv = mul2(zp[a][t][i], kq2);
                    const uint64_t mm = add2(vv, magic2);
                    float v0, v1, m0, m1;
                    upk(vv, v0, v1);
                    upk(mm, m0, m1);
                    const uint2 e0 = lds64(__float_as_uint(m0) * 256u + cell_adj);
                    const uint2 e1 = lds64(__float_as_uint(m1) * 256u + cell_adj);
                    const uint32_t i0 = e0.y + (v0 > __uint_as_float(e0.x) ? 1u : 0u);
                    const uint32_t i1 = e1.y + (v1 > __uint_as_float(e1.x) ? 1u : 0u);
                    word |= (i0 | (i1 << 4)) << (8 * t);
                }
                row[4 * a + c] = static_cast<unsigned short>(word);  // bytes 8a + 2c, 8a + 2c + 1
            }
            if (c == 0) sm.norms[warp][r + 8 * i] = n16[i];
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
                const int64_t blk = slot / block_size, off = slot - blk * block_size;
                uint8_t* sub = pages + (blk * H + h) * block_size * rb;
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

// Cell table of a codebook's boundaries (units of v = 64 u).
void build_cells(const float* boundaries, int levels, QuantCell* out) {
    for (int e = 0; e < kCells; ++e) {
        const double lo = e - 64 - 0.5, hi = e - 64 + 0.5;
        int below = 0;
        float thr = INFINITY;
        for (int i = 0; i + 1 < levels; ++i) {
            const double bv = static_cast<double>(boundaries[i]) * kCellScale;
            if (bv < lo) ++below;
            else if (bv <= hi) thr = static_cast<float>(bv);
        }
        out[e] = QuantCell{thr, below};
    }
}

}  // namespace

// Launches the uniform 4-bit fast path; TQ_ERR_UNSUPPORTED when it does not apply.
tq_status launch_pack_u4(const tq_codec* kc, const tq_codec* vc, const void* k, const void* v,
                         const int64_t* slot_mapping, int64_t num_tokens, void* k_pages, void* v_pages,
                         int64_t num_blocks, int32_t block_size, int32_t* d_err, void* stream) {
    for (const tq_codec* c : {kc, vc})
        if (c->desc.n_groups != 1 || c->desc.group_bits[0] != 4) return TQ_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(k_pages) | reinterpret_cast<uintptr_t>(v_pages)) & 15) return TQ_ERR_UNSUPPORTED;
    if (block_size % 8 != 0) return TQ_ERR_UNSUPPORTED;  // 16-byte aligned rows and norm arrays
    // The cell table depends only on the 4-bit codebook, the same for every codec.
    static std::once_flag once;
    static QuantCell* d_cells = nullptr;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [&] {
        QuantCell host[kCells];
        build_cells(kc->bound[0], 16, host);
        err = cudaMalloc(&d_cells, sizeof(host));
        if (err == cudaSuccess) err = cudaMemcpy(d_cells, host, sizeof(host), cudaMemcpyHostToDevice);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(pack_u4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sizeof(PackSmem)));
    });
    if (err != cudaSuccess) return fail(TQ_ERR_CUDA, "pack fast path setup failed");
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t units = (num_tokens + 15) / 16 * kc->desc.num_kv_heads * 2;
    const int64_t want = (units + kPW - 1) / kPW;
    const int grid = static_cast<int>(want < 4LL * sms ? want : 4LL * sms);
    pack_u4_kernel<<<grid, kPW * 32, sizeof(PackSmem), static_cast<cudaStream_t>(stream)>>>(
        kc->dev, vc->dev, d_cells, static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        slot_mapping, num_tokens, static_cast<uint8_t*>(k_pages), static_cast<uint8_t*>(v_pages), num_blocks,
        block_size, d_err);
    return TQ_OK;
}

}  // namespace tq

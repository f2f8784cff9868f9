// tq_decode_paged: split-K decode attention over packed pages.
//
// TurboQuant "Design" page, "Serving Route Design": block tables map logical
// to physical blocks, K rows are read inside the score computation and V rows
// are read and dequantized inside the accumulation; "System Invariants": the
// historical cache is consumed packed, never rebuilt densely.
//
// With q_r = pi_K(R_K q) (rotated once per query head, in packed order) and
// centroids c, the score of packed token t is
//     s_t = scale * n_K[t] * sum_p q_r[p] c_K[idx_t[p]]            (R orthogonal)
// and the value accumulator stays in the rotated, packed domain of V:
//     acc[p] += softmax weight * n_V[t] * c_V[idx_t[p]],
// so the inverse rotation R_V^T pi_V^-1 runs once per (sequence, query head)
// in the combine. The bf16 recent window is scored exactly in the original
// domain and merged through the same log-sum-exp.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <string>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
    return v;
}

// Index at packed position p of a row (generic bit extraction).
__device__ __forceinline__ int row_index(const uint8_t* row, const DevCodec& c, int p, int& g) {
    g = (c.n_groups == 2 && p >= c.pos0[1]) ? 1 : 0;
    const int b = c.bits[g];
    const int bit = 8 * c.byte_off[g] + (p - c.pos0[g]) * b;
    const int byte = bit >> 3, sh = bit & 7;
    unsigned w = row[byte];
    if (sh + b > 8) w |= static_cast<unsigned>(row[byte + 1]) << 8;
    return static_cast<int>((w >> sh) & ((1u << b) - 1u));
}

// The fp16 norm (which = 0) or, with QJL, the residual norm (which = 1) of row `off`.
__device__ __forceinline__ float row_norm(const uint8_t* sub, const DevCodec& c, int block_size, int off,
                                          int which = 0) {
    const uint8_t* n = sub + block_size * c.index_bytes + c.norm_bytes * off + 2 * which;
    unsigned short h = static_cast<unsigned short>(n[0] | (n[1] << 8));
    return __half2float(__ushort_as_half(h));
}

// Sequence geometry of item (b, split): returns false when the item is empty.
__device__ __forceinline__ bool item_range(const DecodeArgs& a, int b, int split, int& t0, int& t1, bool& is_win) {
    int L = a.seq_lens[b];
    if (L < 0 || L > a.max_seq_len) {
        if (a.d_err && threadIdx.x == 0) atomicOr(a.d_err, TQ_DERR_BLOCK);
        L = L < 0 ? 0 : a.max_seq_len;
    }
    const int n_win = min(a.window, L), P = L - n_win;
    const int ns = (P + a.split_tokens - 1) / a.split_tokens;
    if (split == a.max_splits) {
        is_win = true;
        t0 = 0;
        t1 = n_win;
        return n_win > 0;
    }
    is_win = false;
    if (split >= ns) return false;
    t0 = split * a.split_tokens;
    t1 = min(P, t0 + a.split_tokens);
    return true;
}

template <int G>
__global__ void __launch_bounds__(kWarps * 32) decode_partials_kernel(DecodeArgs a) {
    __shared__ float qs[G][kHeadDim];
    __shared__ float red_m[kWarps][G], red_l[kWarps][G];
    __shared__ float red_acc[kWarps][G][kHeadDim];
    // QJL keys: (S q_r)_i (q_r in rotated coordinate order) during the token loop,
    // in the space of the per-warp accumulators, which are written only after it.
    float (*sq)[kHeadDim] = red_acc[0];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    int t0, t1;
    bool is_win;
    if (!item_range(a, b, split, t0, t1, is_win)) return;
    const int H = a.kc.num_heads;

    // Query prep: q_r = pi_K(H(s_K q)/sqrt(d)) * scale * log2(e) for packed items;
    // q * scale * log2(e) in the original domain for the window item.
    for (int g = warp; g < G; g += kWarps) {
        const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) +
                                  (static_cast<int64_t>(b) * a.num_q_heads + h * G + g) * kHeadDim;
        float z[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) z[i] = __bfloat162float(qp[4 * lane + i]);
        if (is_win) {
#pragma unroll
            for (int i = 0; i < 4; ++i) qs[g][4 * lane + i] = z[i] * a.scale_log2;
            continue;
        }
        if (a.kc.groupwise) {
            // q_r = R_h q (packed positions; R_h orthonormal), lane l: positions l + 32k
            float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const float* rt = a.kc.rot_t + static_cast<int64_t>(h) * kHeadDim * kHeadDim + lane;
            for (int j = 0; j < kHeadDim; ++j) {
                const float qj = __shfl_sync(kFull, z[j & 3], j >> 2);
#pragma unroll
                for (int k = 0; k < 4; ++k) y[k] = fmaf(__ldg(rt + j * kHeadDim + 32 * k), qj, y[k]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) qs[g][lane + 32 * k] = y[k] * a.scale_log2;
            continue;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) z[i] *= a.kc.sign[4 * lane + i];
        {
            float p0 = z[0] + z[1], p1 = z[0] - z[1], p2 = z[2] + z[3], p3 = z[2] - z[3];
            z[0] = p0 + p2;
            z[2] = p0 - p2;
            z[1] = p1 + p3;
            z[3] = p1 - p3;
        }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float p = __shfl_xor_sync(kFull, z[i], m);
                z[i] = (lane & m) ? (p - z[i]) : (z[i] + p);
            }
        const float sc = a.scale_log2 * 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
        for (int i = 0; i < 4; ++i) qs[g][a.kc.pos[h * kHeadDim + 4 * lane + i]] = z[i] * sc;
    }
    __syncthreads();
    const bool qjl = a.kc.qjl && !is_win;
    const bool recipe = a.kc.recipe && !is_win;
    if (recipe) {
        // recipe row: per group, (S_g q_g)_i = sum_j S_g^T[j][i] q_r[pos0_g + j] at packed position
        // pos0_g + i, times sqrt(pi/2)/n_g, the group's estimator constant.
        const int n0 = a.kc.pos0[1];
        for (int e = threadIdx.x; e < G * kHeadDim; e += kWarps * 32) {
            const int g = e / kHeadDim, p = e - g * kHeadDim;
            const int grp = p >= n0 ? 1 : 0, n = a.kc.size[grp], p0 = a.kc.pos0[grp], i = p - p0;
            const float* st = a.kc.qjl_st + (grp ? static_cast<int64_t>(n0) * n0 : 0);
            float acc = 0.0f;
            for (int j = 0; j < n; ++j) acc = fmaf(__ldg(st + j * n + i), qs[g][p0 + j], acc);
            sq[g][p] = acc * (1.2533141373155003f / n);  // sqrt(pi/2) / n_g
        }
        __syncthreads();
    } else if (qjl) {
        // (S q_r)_i = sum_j S^T[j][i] q_r[j], q_r[j] = qs[pos(j)]; times sqrt(pi/2)/d, the estimator's constant.
        for (int e = threadIdx.x; e < G * kHeadDim; e += kWarps * 32) {
            const int g = e / kHeadDim, i = e - g * kHeadDim;
            float acc = 0.0f;
            for (int j = 0; j < kHeadDim; ++j)
                acc = fmaf(__ldg(a.kc.qjl_st + j * kHeadDim + i), qs[g][a.kc.pos[h * kHeadDim + j]], acc);
            sq[g][i] = acc * (1.2533141373155003f / kHeadDim);  // sqrt(pi/2) / d
        }
        __syncthreads();
    }

    float m[G], l[G], acc[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[g][i] = 0.0f;
    }
    const int bs = a.block_size;
    for (int t = t0 + warp; t < t1; t += kWarps) {
        float kv[4], vv[4], nk = 1.0f, nv = 1.0f, gk = 0.0f, zk[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float wk[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // recipe row: n_g |r_g| of each position's group
        if (is_win) {
            const int64_t base = ((static_cast<int64_t>(b) * H + h) * a.window + t) * kHeadDim + 4 * lane;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                kv[i] = __bfloat162float(static_cast<const __nv_bfloat16*>(a.k_win)[base + i]);
                vv[i] = __bfloat162float(static_cast<const __nv_bfloat16*>(a.v_win)[base + i]);
            }
        } else {
            int64_t blk = a.block_tables[static_cast<int64_t>(b) * a.max_blocks + t / bs];
            if (blk < 0 || blk >= a.num_blocks) {
                if (a.d_err && lane == 0) atomicOr(a.d_err, TQ_DERR_BLOCK);
                blk = 0;
            }
            const int64_t sp = (blk * H + h) * bs;
            const int off = t % bs;
            const uint8_t* ksub = a.k_pages + sp * a.kc.row_bytes;
            const uint8_t* vsub = a.v_pages + sp * a.vc.row_bytes;
            const uint8_t* krow = ksub + off * a.kc.index_bytes;
            const uint8_t* vrow = vsub + off * a.vc.index_bytes;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int g;
                int ix = row_index(krow, a.kc, 4 * lane + i, g);
                kv[i] = a.kc.cent[g * 16 + ix];
                ix = row_index(vrow, a.vc, 4 * lane + i, g);
                vv[i] = a.vc.cent[g * 16 + ix];
            }
            nk = row_norm(ksub, a.kc, bs, off);
            nv = row_norm(vsub, a.vc, bs, off);
            if (recipe) {  // norm area (n_0, |r_0|, n_1, |r_1|); signs after each group's indices
                const float n0k = nk, r0k = row_norm(ksub, a.kc, bs, off, 1);
                const float n1k = row_norm(ksub, a.kc, bs, off, 2), r1k = row_norm(ksub, a.kc, bs, off, 3);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int p = 4 * lane + i, grp = p >= a.kc.pos0[1] ? 1 : 0, sp = p - a.kc.pos0[grp];
                    kv[i] *= grp ? n1k : n0k;
                    wk[i] = grp ? n1k * r1k : n0k * r0k;
                    zk[i] = ((krow[a.kc.sign_off[grp] + (sp >> 3)] >> (sp & 7)) & 1u) ? 1.0f : -1.0f;
                }
                nk = 1.0f;
            } else if (a.kc.groupwise) {  // per-group norms: fold each position's norm into its centroid
                const float nk1 = row_norm(ksub, a.kc, bs, off, 1);
#pragma unroll
                for (int i = 0; i < 4; ++i) kv[i] *= (4 * lane + i >= a.kc.pos0[1]) ? nk1 : nk;
                nk = 1.0f;
            }
            if (a.vc.groupwise) {
                const float nv1 = row_norm(vsub, a.vc, bs, off, 1);
#pragma unroll
                for (int i = 0; i < 4; ++i) vv[i] *= (4 * lane + i >= a.vc.pos0[1]) ? nv1 : nv;
                nv = 1.0f;
            }
            if (qjl && !recipe) {
                // sign bits 4l .. 4l+3 of the QJL stream (after the index bitstreams)
                const unsigned bits = (krow[a.kc.mse_bytes + (lane >> 1)] >> (4 * (lane & 1))) & 0xFu;
#pragma unroll
                for (int i = 0; i < 4; ++i) zk[i] = ((bits >> i) & 1u) ? 1.0f : -1.0f;
                gk = row_norm(ksub, a.kc, bs, off, 1);
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float s = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) s += qs[g][4 * lane + i] * kv[i];
            if (recipe) {
#pragma unroll
                for (int i = 0; i < 4; ++i) s += wk[i] * sq[g][4 * lane + i] * zk[i];  // n_g |r_g| (S_g q_g)_i z_i
            } else if (qjl) {
                float t = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) t += sq[g][4 * lane + i] * zk[i];
                s += gk * t;  // q_r . (c + sqrt(pi/2)/d g S^T z), summed over the warp below
            }
            s = warp_sum(s) * nk;
            const float mn = fmaxf(m[g], s);
            const float alpha = exp2f(m[g] - mn);
            const float p = exp2f(s - mn);
            l[g] = l[g] * alpha + p;
            const float pv = p * nv;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[g][i] = acc[g][i] * alpha + pv * vv[i];
            m[g] = mn;
        }
    }
    if (qjl) __syncthreads();  // every warp is done with sq before red_acc is written
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == 0) {
            red_m[warp][g] = m[g];
            red_l[warp][g] = l[g];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) red_acc[warp][g][4 * lane + i] = acc[g][i];
    }
    __syncthreads();
    float* rec = a.ws + ((static_cast<int64_t>(b) * H + h) * a.items_per_unit + split) *
                            static_cast<int64_t>(G) * (kHeadDim + 2);
    for (int e = threadIdx.x; e < G * kHeadDim; e += kWarps * 32) {
        const int g = e / kHeadDim, j = e - g * kHeadDim;
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w][g]);
        float L = 0.0f, A = 0.0f;
        if (M != -INFINITY)
            for (int w = 0; w < kWarps; ++w) {
                const float f = exp2f(red_m[w][g] - M);
                L += red_l[w][g] * f;
                A += red_acc[w][g][j] * f;
            }
        float* rg = rec + g * (kHeadDim + 2);
        rg[2 + j] = A;
        if (j == 0) {
            rg[0] = M;
            rg[1] = L;
        }
    }
}

// Log-sum-exp merge of the split records of one (sequence, query head), over
// the 128 threads j of a group (4 warps; a CTA may hold several groups, all
// with the same ns and n_win: the barriers inside are CTA-wide). Returns the
// merged sum ls, accumulator position j (rot) and the window record's share
// (win), all relative to the largest record max. The records are read in
// parallel: first every max (thread j takes splits j, j + 128, ...), then per
// chunk of 128 splits each thread's weight goes to shared memory and the
// accumulator sums its column with WIDE loads in flight (WIDE = 16: unrolled
// rounds with the loads past the last split skipped; 8: a loop unrolled by 8,
// fewer registers, which the one-head-per-CTA combine's larger grids need).
// fw: the group's 128 floats of shared scratch, red: its 4.
template <int WIDE>
__device__ __forceinline__ void merge_splits(const float* unit, int G, int g, int ns, int n_win, int max_splits,
                                             int j, float* fw, float* red, float& ls, float& rot, float& win) {
    auto rec = [&](int i) { return unit + (static_cast<int64_t>(i) * G + g) * (kHeadDim + 2); };
    const int lane = j & 31, wg = j >> 5;
    float m = -INFINITY;
    for (int i = j; i < ns; i += kHeadDim) m = fmaxf(m, rec(i)[0]);
    if (n_win && j == 0) m = fmaxf(m, rec(max_splits)[0]);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) red[wg] = m;
    __syncthreads();
    const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();  // red is written again below
    ls = 0.0f;
    rot = 0.0f;
    win = 0.0f;
    if (M == -INFINITY) return;  // no record: the same for every group of the CTA (one sequence)
    float lpart = 0.0f;
    for (int c0 = 0; c0 < ns; c0 += kHeadDim) {
        float f = 0.0f;
        if (c0 + j < ns) {
            const float* r = rec(c0 + j);
            f = exp2f(r[0] - M);
            lpart += r[1] * f;
        }
        fw[j] = f;
        __syncthreads();
        const int n = min(kHeadDim, ns - c0);
        if constexpr (WIDE == 16) {
            // past the last split the load is skipped and its weight is 0, so the sum keeps the split
            // order and adds exact zeros
            for (int k = 0; k < n; k += 16) {
                float vals[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) vals[u] = k + u < n ? rec(c0 + k + u)[2 + j] : 0.0f;
#pragma unroll
                for (int u = 0; u < 16; ++u) rot = fmaf(vals[u], fw[k + u], rot);
            }
        } else {
#pragma unroll 8
            for (int k = 0; k < n; ++k) rot = fmaf(rec(c0 + k)[2 + j], fw[k], rot);
        }
        __syncthreads();  // fw is written again by the next chunk
    }
    lpart = warp_sum(lpart);
    if (lane == 0) red[wg] = lpart;
    __syncthreads();
    ls = (red[0] + red[1]) + (red[2] + red[3]);
    if (n_win) {
        const float* r = rec(max_splits);
        const float f = exp2f(r[0] - M);
        ls += r[1] * f;
        win = r[2 + j] * f;
    }
}

__global__ void __launch_bounds__(kHeadDim) decode_combine_kernel(DevCodec vc, const int32_t* seq_lens,
                                                                   int32_t num_q_heads, int32_t max_seq_len,
                                                                   int32_t window, int32_t split_tokens,
                                                                   int32_t max_splits, int32_t items_per_unit,
                                                                   int32_t G, const float* ws, float* out) {
    __shared__ float y[kHeadDim], y2[kHeadDim];
    __shared__ float red[4];
    // Launched as a dependent of the partials: the split records are read only after they are complete.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int hq = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
    const int H = vc.num_heads, h = hq / G, g = hq - h * G;
    int L = seq_lens[b];
    L = L < 0 ? 0 : (L > max_seq_len ? max_seq_len : L);
    const int n_win = min(window, L), P = L - n_win;
    const int ns = (P + split_tokens - 1) / split_tokens;
    const float* unit = ws + (static_cast<int64_t>(b) * H + h) * items_per_unit * static_cast<int64_t>(G) * (kHeadDim + 2);
    float Ls, rot, win;
    merge_splits<8>(unit, G, g, ns, n_win, max_splits, j, y, red, Ls, rot, win);
    __syncthreads();  // y served as the merge's scratch
    float x;
    if (vc.groupwise) {
        y[j] = rot;  // packed positions
        __syncthreads();
        const float* rt = vc.rot_t + (static_cast<int64_t>(h) * kHeadDim + j) * kHeadDim;  // R_h^T row j
        x = 0.0f;
        for (int p = 0; p < kHeadDim; ++p) x = fmaf(rt[p], y[p], x);
    } else {
        y[vc.perm[h * kHeadDim + j]] = rot;  // back to rotated coordinate order
        __syncthreads();
        // Walsh-Hadamard, natural order: strides 1 .. 16 inside a warp by shuffles, 32 and 64
        // through shared memory (y2, then y again: y was last read before the first barrier)
        float v = y[j];
#pragma unroll
        for (int len = 1; len < 32; len <<= 1) {
            const float o = __shfl_xor_sync(kFull, v, len);
            v = (j & len) ? (o - v) : (v + o);
        }
        y2[j] = v;
        __syncthreads();
        {
            const float o = y2[j ^ 32];
            v = (j & 32) ? (o - v) : (v + o);
        }
        y[j] = v;
        __syncthreads();
        {
            const float o = y[j ^ 64];
            v = (j & 64) ? (o - v) : (v + o);
        }
        x = vc.sign[j] * v * 0.08838834764831845f;
    }
    out[(static_cast<int64_t>(b) * num_q_heads + hq) * kHeadDim + j] = Ls > 0.0f ? (x + win) / Ls : 0.0f;
}

// Group-wise V: the same merge, then x = R_h^T y. One CTA per (b, KV head)
// with 128 threads per query head (up to 8 heads at a time): R_h^T is staged
// once in shared memory with a row pitch of 129 floats (thread j reads row j
// without bank conflicts), instead of every query head reading the 64 KB
// matrix from L2 with row-strided loads.
constexpr int kGwPitch = kHeadDim + 1;
constexpr int kGwHeads = 8;
constexpr size_t kGwCombineSmem =
    (static_cast<size_t>(kHeadDim) * kGwPitch + kGwHeads * kHeadDim + kGwHeads * 4) * sizeof(float);

__global__ void __launch_bounds__(kHeadDim * kGwHeads) decode_combine_gw_kernel(
    DevCodec vc, const int32_t* seq_lens, int32_t num_q_heads, int32_t max_seq_len, int32_t window,
    int32_t split_tokens, int32_t max_splits, int32_t items_per_unit, int32_t G, const float* ws, float* out) {
    extern __shared__ float gsm[];
    float* rts = gsm;                               // [128][129]: R_h^T, row j at j * 129
    float* ys = gsm + kHeadDim * kGwPitch;          // [kGwHeads][128]
    float* reds = ys + kGwHeads * kHeadDim;         // [kGwHeads][4]
    const int H = vc.num_heads, h = blockIdx.x % H, b = blockIdx.x / H;
    const int j = threadIdx.x & (kHeadDim - 1), gl = threadIdx.x >> 7, nthreads = blockDim.x;
    const float* rt = vc.rot_t + static_cast<int64_t>(h) * kHeadDim * kHeadDim;
    // 16-byte loads, eight in flight per thread (R_h^T comes from L2)
#pragma unroll 8
    for (int e4 = threadIdx.x; e4 < kHeadDim * kHeadDim / 4; e4 += nthreads) {
        const float4 v4 = __ldg(reinterpret_cast<const float4*>(rt) + e4);
        float* d = rts + (e4 >> 5) * kGwPitch + 4 * (e4 & 31);
        d[0] = v4.x;
        d[1] = v4.y;
        d[2] = v4.z;
        d[3] = v4.w;
    }
    // Launched as a dependent of the partials: R_h^T is staged while they end; the split records are
    // read only after they are complete.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int L = seq_lens[b];
    L = L < 0 ? 0 : (L > max_seq_len ? max_seq_len : L);
    const int n_win = min(window, L), P = L - n_win;
    const int ns = (P + split_tokens - 1) / split_tokens;
    const float* unit = ws + (static_cast<int64_t>(b) * H + h) * items_per_unit * static_cast<int64_t>(G) * (kHeadDim + 2);
    const int per = nthreads / kHeadDim;  // query heads per pass
    for (int g0 = 0; g0 < G; g0 += per) {
        // Every group takes part in each pass (the merge's barriers are CTA-wide). G is 1, 2, 4, 8 or
        // 16, so no group runs past G; were one to, it would repeat head G - 1 and write nothing.
        const int g = g0 + gl;
        float Ls, rot, win;
        merge_splits<16>(unit, G, g < G ? g : G - 1, ns, n_win, max_splits, j, ys + gl * kHeadDim, reds + gl * 4, Ls,
                     rot, win);
        __syncthreads();  // ys served as the merge's scratch
        ys[gl * kHeadDim + j] = rot;  // packed positions
        __syncthreads();  // (the first pass also waits for the staged R_h^T)
        if (g < G) {
            const float* rj = rts + j * kGwPitch;
            const float* y = ys + gl * kHeadDim;
            float x = 0.0f;
#pragma unroll 8
            for (int p = 0; p < kHeadDim; ++p) x = fmaf(rj[p], y[p], x);
            out[(static_cast<int64_t>(b) * num_q_heads + h * G + g) * kHeadDim + j] = Ls > 0.0f ? (x + win) / Ls : 0.0f;
        }
        __syncthreads();
    }
}

tq_status check_decode_args(const tq_codec* kc, const tq_codec* vc, int32_t batch, int32_t num_q_heads,
                            int32_t max_seq_len, int32_t window, int32_t block_size, size_t workspace_bytes,
                            const void* workspace, SplitPlan* plan) {
    if (!kc || !vc) return fail(TQ_ERR_VALUE, "null codec");
    if (kc->desc.num_kv_heads != vc->desc.num_kv_heads || kc->desc.head_dim != vc->desc.head_dim)
        return fail(TQ_ERR_VALUE, "K and V codecs disagree on num_kv_heads or head_dim");
    const int H = kc->desc.num_kv_heads;
    if (batch < 0 || window < 0 || max_seq_len < 0 || block_size < 1)
        return fail(TQ_ERR_VALUE, "negative size");
    if (num_q_heads < H || num_q_heads % H) return fail(TQ_ERR_VALUE, "num_q_heads must be a multiple of num_kv_heads");
    const int G = num_q_heads / H;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
        return fail(TQ_ERR_UNSUPPORTED, "query heads per KV head must be 1, 2, 4, 8 or 16");
    if (vc->desc.qjl) return fail(TQ_ERR_UNSUPPORTED, "decode implements the QJL stage for keys only");
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        sms = 0;
    }
    if (!make_split_plan(batch, num_q_heads, H, max_seq_len, block_size, sms, plan))
        return fail(TQ_ERR_VALUE, "invalid decode sizes");
    if (workspace_bytes < plan->workspace_bytes) return fail(TQ_ERR_VALUE, "workspace smaller than tq_decode_workspace_bytes");
    if (batch > 0 && !workspace) return fail(TQ_ERR_VALUE, "null workspace");
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return fail(TQ_ERR_VALUE, "workspace must be 256-byte aligned");
    return TQ_OK;
}

tq_status finish(cudaStream_t s, int32_t* d_err, const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(TQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    if (checked_mode()) {
        if ((e = cudaStreamSynchronize(s)) != cudaSuccess)
            return fail(TQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
        if (d_err) {
            int32_t h = 0;
            if (cudaMemcpy(&h, d_err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
                return fail(TQ_ERR_CUDA, "reading the device error word failed");
            if (h & TQ_DERR_TIMEOUT) return fail(TQ_ERR_TIMEOUT, "a bounded wait in the decode kernel expired");
            if (h & TQ_DERR_LAUNCH) return fail(TQ_ERR_CUDA, "the decode kernel could not lay out shared memory");
            if (h & TQ_DERR_BLOCK) return fail(TQ_ERR_INDEX, "block table entry or length outside the pages");
        }
    }
    return TQ_OK;
}

}  // namespace
}  // namespace tq

using namespace tq;

namespace tq {
namespace {
// The step's window append, fused into the decode prologue (tq_window_append_decode).
struct FusedAppend {
    const void* k_new;
    const void* v_new;
    void* k_win;
    void* v_win;
    void* k_pages;
    void* v_pages;
    int32_t window, sinks;  // the append's W and S; the decode's window is S + W
};

tq_status decode_partials_impl(const tq_codec* kc, const tq_codec* vc, const void* q, const void* k_pages,
                               const void* v_pages, const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t max_seq_len,
                               const void* k_win, const void* v_win, int32_t window, float softmax_scale,
                               int64_t num_blocks, int32_t block_size, void* workspace, size_t workspace_bytes,
                               int32_t* d_err, void* stream, const FusedAppend* app) {
    SplitPlan plan;
    tq_status st = check_decode_args(kc, vc, batch, num_q_heads, max_seq_len, window, block_size, workspace_bytes,
                                     workspace, &plan);
    if (st != TQ_OK) return st;
    if (batch == 0) return TQ_OK;
    if (!q || !seq_lens || (max_seq_len > window && (!k_pages || !v_pages || !block_tables)))
        return fail(TQ_ERR_VALUE, "null buffer");
    if (window > 0 && (!k_win || !v_win)) return fail(TQ_ERR_VALUE, "window > 0 needs k_win and v_win");
    if (num_blocks < 0 || max_blocks_per_seq < 0) return fail(TQ_ERR_VALUE, "negative size");
    if (max_seq_len > window && num_blocks < 1) return fail(TQ_ERR_VALUE, "packed tokens need at least one block");
    if ((reinterpret_cast<uintptr_t>(k_pages) | reinterpret_cast<uintptr_t>(v_pages)) & 15)
        return fail(TQ_ERR_VALUE, "page pools must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(q) & 7) || (window > 0 && ((reinterpret_cast<uintptr_t>(k_win) |
                                                                reinterpret_cast<uintptr_t>(v_win)) & 7)))
        return fail(TQ_ERR_VALUE, "q and the windows must be 8-byte aligned");
    if (static_cast<int64_t>(max_blocks_per_seq) * block_size < static_cast<int64_t>(max_seq_len) - window)
        return fail(TQ_ERR_VALUE, "max_blocks_per_seq * block_size cannot hold max_seq_len - window tokens");
    DecodeArgs a{};
    a.kc = kc->dev;
    a.vc = vc->dev;
    a.q = q;
    a.k_pages = static_cast<const uint8_t*>(k_pages);
    a.v_pages = static_cast<const uint8_t*>(v_pages);
    a.block_tables = block_tables;
    a.max_blocks = max_blocks_per_seq;
    a.seq_lens = seq_lens;
    a.batch = batch;
    a.num_q_heads = num_q_heads;
    a.max_seq_len = max_seq_len;
    a.k_win = k_win;
    a.v_win = v_win;
    a.window = window;
    a.scale_log2 = softmax_scale * kLog2e;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.split_tokens = plan.split_tokens;
    a.max_splits = plan.max_splits;
    a.items_per_unit = plan.items_per_unit;
    a.ws = static_cast<float*>(workspace);
    a.qrot = reinterpret_cast<float*>(static_cast<char*>(workspace) + plan.record_bytes);
    a.qjl_q = a.qrot + static_cast<size_t>(batch) * num_q_heads * kHeadDim;
    a.work_list = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + plan.list_offset);
    a.work_count = a.work_list + 2 * static_cast<size_t>(batch) * plan.items_per_unit;
    a.d_err = d_err;
    const char* withhold = std::getenv("TQ_TEST_WITHHOLD_COPIES");
    a.withhold_copies = withhold && std::string(withhold) == "1";
    if (app) {
        a.app_on = 1;
        a.k_new = app->k_new;
        a.v_new = app->v_new;
        a.k_win_w = app->k_win;
        a.v_win_w = app->v_win;
        a.k_pages_w = static_cast<uint8_t*>(app->k_pages);
        a.v_pages_w = static_cast<uint8_t*>(app->v_pages);
        a.app_window = app->window;
        a.app_sinks = app->sinks;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Tensor-core kernel for the formats it is instantiated for (block sizes a
    // multiple of 16); the general kernel covers every other valid format.
    // TQ_DECODE_KERNEL=general selects the general kernel and =tensor the
    // tensor-core one (unsupported formats then fail), for cross-checks.
    const char* force = std::getenv("TQ_DECODE_KERNEL");
    const std::string forced = force ? force : "";
    if (forced != "general") {
        st = launch_decode_mma(a, kc, vc, plan.group, stream);
        if (st == TQ_OK) return finish(s, d_err, "decode partials");
        if (st != TQ_ERR_UNSUPPORTED) return st;
        if (forced == "tensor") return fail(TQ_ERR_UNSUPPORTED, "no tensor-core decode for these formats");
        clear_error();
    }
    if (app) {
        // the general kernel takes no fused append: append first, as a separate launch
        st = tq_window_append(kc, vc, app->k_new, app->v_new, app->k_win, app->v_win, app->window, app->sinks,
                              seq_lens, block_tables, max_blocks_per_seq, app->k_pages, app->v_pages, num_blocks,
                              block_size, batch, d_err, stream);
        if (st != TQ_OK) return st;
        a.app_on = 0;
    }
    dim3 grid(plan.items_per_unit, kc->desc.num_kv_heads, batch);
    switch (plan.group) {
        case 1: decode_partials_kernel<1><<<grid, kWarps * 32, 0, s>>>(a); break;
        case 2: decode_partials_kernel<2><<<grid, kWarps * 32, 0, s>>>(a); break;
        case 4: decode_partials_kernel<4><<<grid, kWarps * 32, 0, s>>>(a); break;
        case 8: decode_partials_kernel<8><<<grid, kWarps * 32, 0, s>>>(a); break;
        default: decode_partials_kernel<16><<<grid, kWarps * 32, 0, s>>>(a); break;
    }
    return finish(s, d_err, "decode partials");
}
}  // namespace
}  // namespace tq

extern "C" tq_status tq_decode_partials(const tq_codec* kc, const tq_codec* vc, const void* q, const void* k_pages,
                                        const void* v_pages, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                        const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                        int32_t max_seq_len, const void* k_win, const void* v_win, int32_t window,
                                        float softmax_scale, int64_t num_blocks, int32_t block_size,
                                        void* workspace, size_t workspace_bytes, int32_t* d_err, void* stream) {
    clear_error();
    return decode_partials_impl(kc, vc, q, k_pages, v_pages, block_tables, max_blocks_per_seq, seq_lens, batch,
                                num_q_heads, max_seq_len, k_win, v_win, window, softmax_scale, num_blocks, block_size,
                                workspace, workspace_bytes, d_err, stream, nullptr);
}

extern "C" tq_status tq_decode_combine(const tq_codec* vc, const int32_t* seq_lens, int32_t batch,
                                       int32_t num_q_heads, int32_t max_seq_len, int32_t window, int32_t block_size,
                                       float* out, const void* workspace, size_t workspace_bytes, void* stream) {
    clear_error();
    SplitPlan plan;
    tq_status st = check_decode_args(vc, vc, batch, num_q_heads, max_seq_len, window, block_size, workspace_bytes,
                                     workspace, &plan);
    if (st != TQ_OK) return st;
    if (batch == 0) return TQ_OK;
    if (!out || !seq_lens) return fail(TQ_ERR_VALUE, "null buffer");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (vc->desc.groupwise) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return fail(TQ_ERR_CUDA, "cudaGetDevice failed");
        cudaError_t e = once_per_device(dev, [] {
            return cudaFuncSetAttribute(decode_combine_gw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kGwCombineSmem));
        });
        if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "cannot reserve shared memory for the combine kernel");
        const int threads = kHeadDim * std::min(plan.group, kGwHeads);
        e = launch_dependent(decode_combine_gw_kernel, dim3(static_cast<unsigned>(batch) * vc->desc.num_kv_heads),
                             dim3(threads), kGwCombineSmem, s, vc->dev, seq_lens, num_q_heads, max_seq_len, window,
                             plan.split_tokens, plan.max_splits, plan.items_per_unit, plan.group,
                             static_cast<const float*>(workspace), out);
        if (e != cudaSuccess) return fail(TQ_ERR_CUDA, std::string("combine launch: ") + cudaGetErrorString(e));
    } else {
        const cudaError_t e = launch_dependent(
            decode_combine_kernel, dim3(num_q_heads, batch), dim3(kHeadDim), 0, s, vc->dev, seq_lens, num_q_heads,
            max_seq_len, window, plan.split_tokens, plan.max_splits, plan.items_per_unit, plan.group,
            static_cast<const float*>(workspace), out);
        if (e != cudaSuccess) return fail(TQ_ERR_CUDA, std::string("combine launch: ") + cudaGetErrorString(e));
    }
    return finish(s, nullptr, "decode combine");
}

extern "C" tq_status tq_window_append_decode(const tq_codec* kc, const tq_codec* vc, const void* k_new,
                                             const void* v_new, void* k_win, void* v_win, int32_t window,
                                             int32_t sinks, const void* q, void* k_pages, void* v_pages,
                                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                                             const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                             int32_t max_seq_len, float softmax_scale, int64_t num_blocks,
                                             int32_t block_size, float* out, void* workspace, size_t workspace_bytes,
                                             int32_t* d_err, void* stream) {
    clear_error();
    tq_status st = validate_window_append(kc, vc, k_new, v_new, k_win, v_win, window, sinks, seq_lens, block_tables,
                                          max_blocks_per_seq, k_pages, v_pages, num_blocks, block_size, batch);
    if (st != TQ_OK) return st;
    if (window > INT32_MAX - sinks) return fail(TQ_ERR_VALUE, "window + sinks overflows");
    const int32_t dense = window + sinks;
    if (batch > 0) {
        const FusedAppend app{k_new, v_new, k_win, v_win, k_pages, v_pages, window, sinks};
        st = decode_partials_impl(kc, vc, q, k_pages, v_pages, block_tables, max_blocks_per_seq, seq_lens, batch,
                                  num_q_heads, max_seq_len, k_win, v_win, dense, softmax_scale, num_blocks,
                                  block_size, workspace, workspace_bytes, d_err, stream, &app);
        if (st != TQ_OK) return st;
    }
    return tq_decode_combine(vc, seq_lens, batch, num_q_heads, max_seq_len, dense, block_size, out, workspace,
                             workspace_bytes, stream);
}

extern "C" tq_status tq_decode_paged(const tq_codec* kc, const tq_codec* vc, const void* q, const void* k_pages,
                                     const void* v_pages, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                                     int32_t max_seq_len, const void* k_win, const void* v_win, int32_t window,
                                     float softmax_scale, int64_t num_blocks, int32_t block_size, float* out,
                                     void* workspace, size_t workspace_bytes, int32_t* d_err, void* stream) {
    tq_status st = tq_decode_partials(kc, vc, q, k_pages, v_pages, block_tables, max_blocks_per_seq, seq_lens, batch,
                                      num_q_heads, max_seq_len, k_win, v_win, window, softmax_scale, num_blocks,
                                      block_size, workspace, workspace_bytes, d_err, stream);
    if (st != TQ_OK) return st;
    return tq_decode_combine(vc, seq_lens, batch, num_q_heads, max_seq_len, window, block_size, out, workspace,
                             workspace_bytes, stream);
}

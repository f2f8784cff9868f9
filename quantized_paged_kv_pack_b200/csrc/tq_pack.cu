// tq_pack_kv: quantize-and-pack write of K/V token vectors into uint8 pages.
//
// TurboQuant "Design" page, "Serving Route Design": the serving route writes
// packed rows into persistent pages addressed slot -> physical block -> token
// offset -> row bytes, block = slot / block_size, offset = slot % block_size.
// Per (token, head) vector x (bf16, 128 values):
//   n   = ||x||_2, stored as fp16 (round to nearest even)
//   z   = H (s * x)              Sylvester Walsh-Hadamard, signs s of the codec
//   u   = z / (sqrt(128) n)      the rotated unit vector
//   idx = #{boundaries of its group below u_j}, placed at packed position pos[h][j]
//   row = [group-0 bitstream][group-1 bitstream][n16], LSB-first; in the
//   sub-page of (block, head) the index bytes of the block_size rows come
//   first, row after row, then the block_size norms.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <string>

#include "tq_internal.h"
#include "tq_pack_vector.cuh"

namespace tq {
namespace {

constexpr int kPackWarps = 8;

__global__ void __launch_bounds__(kPackWarps * 32)
pack_rows_kernel(DevCodec kc, DevCodec vc, const __nv_bfloat16* __restrict__ k,
                 const __nv_bfloat16* __restrict__ v, const int64_t* __restrict__ slots, int64_t num_tokens,
                 uint8_t* __restrict__ k_pages, uint8_t* __restrict__ v_pages, int64_t num_blocks,
                 int block_size, int* __restrict__ d_err) {
    __shared__ uint8_t idx_buf[kPackWarps][kHeadDim];
    __shared__ float r_buf[kPackWarps][kHeadDim];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t H = kc.num_heads;
    const int64_t n_vec = num_tokens * H * 2;
    const int64_t capacity = num_blocks * block_size;
    for (int64_t vec = static_cast<int64_t>(blockIdx.x) * kPackWarps + warp; vec < n_vec;
         vec += static_cast<int64_t>(gridDim.x) * kPackWarps) {
        const int which = static_cast<int>(vec & 1);
        const int64_t th = vec >> 1;
        const int64_t t = th / H;
        const int h = static_cast<int>(th - t * H);
        const int64_t slot = slots[t];
        if (slot < 0) continue;
        if (slot >= capacity) {
            if (lane == 0 && d_err) atomicOr(d_err, TQ_DERR_SLOT);
            continue;
        }
        const DevCodec& c = which ? vc : kc;
        float x[4];
        pv_load_bf16x4((which ? v : k) + th * kHeadDim + 4 * lane, x);
        const int64_t blk = slot / block_size, off = slot - blk * block_size;
        uint8_t* sub = (which ? v_pages : k_pages) + (blk * H + h) * block_size * c.row_bytes;
        pack_vector(c, x, h, sub, off, block_size, idx_buf[warp], r_buf[warp], lane);
    }
}

// Window eviction with append (append_vector): one warp per (sequence, KV head, K or V).
__global__ void __launch_bounds__(kPackWarps * 32)
window_append_kernel(DevCodec kc, DevCodec vc, const __nv_bfloat16* __restrict__ k_new,
                     const __nv_bfloat16* __restrict__ v_new, __nv_bfloat16* __restrict__ k_win,
                     __nv_bfloat16* __restrict__ v_win, int window, int sinks, const int32_t* __restrict__ seq_lens,
                     const int32_t* __restrict__ block_tables, int max_blocks, uint8_t* __restrict__ k_pages,
                     uint8_t* __restrict__ v_pages, int64_t num_blocks, int block_size, int batch,
                     int* __restrict__ d_err) {
    __shared__ uint8_t idx_buf[kPackWarps][kHeadDim];
    __shared__ float r_buf[kPackWarps][kHeadDim];
    // A decode call that follows may launch its first kernel now; that kernel waits for this one.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_vec = static_cast<int64_t>(batch) * kc.num_heads * 2;
    for (int64_t vec = static_cast<int64_t>(blockIdx.x) * kPackWarps + warp; vec < n_vec;
         vec += static_cast<int64_t>(gridDim.x) * kPackWarps)
        append_vector(kc, vc, vec, k_new, v_new, k_win, v_win, window, sinks, seq_lens, block_tables, max_blocks,
                      k_pages, v_pages, num_blocks, block_size, d_err, idx_buf[warp], r_buf[warp], lane);
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" tq_status tq_pack_kv(const tq_codec* kc, const tq_codec* vc, const void* k, const void* v,
                                const int64_t* slot_mapping, int64_t num_tokens, void* k_pages, void* v_pages,
                                int64_t num_blocks, int32_t block_size, int32_t* d_err, void* stream) {
    clear_error();
    if (!kc || !vc) return fail(TQ_ERR_VALUE, "null codec");
    if (kc->desc.num_kv_heads != vc->desc.num_kv_heads || kc->desc.head_dim != vc->desc.head_dim)
        return fail(TQ_ERR_VALUE, "K and V codecs disagree on num_kv_heads or head_dim");
    if (num_tokens < 0 || num_blocks < 0 || block_size < 1) return fail(TQ_ERR_VALUE, "negative size");
    if (num_tokens == 0) return TQ_OK;
    if (!k || !v || !slot_mapping || !k_pages || !v_pages) return fail(TQ_ERR_VALUE, "null buffer");
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 7)
        return fail(TQ_ERR_VALUE, "k and v must be 8-byte aligned");
    if ((reinterpret_cast<uintptr_t>(k_pages) | reinterpret_cast<uintptr_t>(v_pages)) & 1)
        return fail(TQ_ERR_VALUE, "page pools must be 2-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Tensor-core packs where both codecs have one (and the buffers are 16-byte
    // aligned); the general kernel covers every other call. TQ_PACK_KERNEL=general
    // selects the general kernel.
    const char* force = std::getenv("TQ_PACK_KERNEL");
    if (!(force && std::string(force) == "general")) {
        tq_status st = launch_pack_tc(kc, vc, k, v, slot_mapping, num_tokens, k_pages, v_pages, num_blocks,
                                      block_size, d_err, stream);
        if (st != TQ_OK && st != TQ_ERR_UNSUPPORTED) return st;
        if (st == TQ_OK) return finish_pack(s, d_err);
        clear_error();
    }
    const int64_t n_vec = num_tokens * kc->desc.num_kv_heads * 2;
    const int64_t blocks = std::min<int64_t>((n_vec + kPackWarps - 1) / kPackWarps, 148 * 32);
    pack_rows_kernel<<<static_cast<unsigned>(blocks), kPackWarps * 32, 0, s>>>(
        kc->dev, vc->dev, static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        slot_mapping, num_tokens, static_cast<uint8_t*>(k_pages), static_cast<uint8_t*>(v_pages), num_blocks,
        block_size, d_err);
    return finish_pack(s, d_err);
}

namespace tq {
tq_status validate_window_append(const tq_codec* kc, const tq_codec* vc, const void* k_new, const void* v_new,
                                 const void* k_win, const void* v_win, int32_t window, int32_t sinks,
                                 const int32_t* seq_lens, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                 const void* k_pages, const void* v_pages, int64_t num_blocks, int32_t block_size,
                                 int32_t batch) {
    if (!kc || !vc) return fail(TQ_ERR_VALUE, "null codec");
    if (kc->desc.num_kv_heads != vc->desc.num_kv_heads || kc->desc.head_dim != vc->desc.head_dim)
        return fail(TQ_ERR_VALUE, "K and V codecs disagree on num_kv_heads or head_dim");
    if (batch < 0 || window < 0 || sinks < 0 || block_size < 1 || num_blocks < 0 || max_blocks_per_seq < 0)
        return fail(TQ_ERR_VALUE, "negative size");
    if (batch == 0) return TQ_OK;
    if (!k_new || !v_new || !seq_lens || !k_pages || !v_pages || (max_blocks_per_seq > 0 && !block_tables))
        return fail(TQ_ERR_VALUE, "null buffer");
    if (window + sinks > 0 && (!k_win || !v_win)) return fail(TQ_ERR_VALUE, "null dense buffer");
    if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new) |
         reinterpret_cast<uintptr_t>(k_win) | reinterpret_cast<uintptr_t>(v_win)) & 7)
        return fail(TQ_ERR_VALUE, "k_new, v_new and the dense buffers must be 8-byte aligned");
    if ((reinterpret_cast<uintptr_t>(k_pages) | reinterpret_cast<uintptr_t>(v_pages)) & 1)
        return fail(TQ_ERR_VALUE, "page pools must be 2-byte aligned");
    return TQ_OK;
}
}  // namespace tq

extern "C" tq_status tq_window_append(const tq_codec* kc, const tq_codec* vc, const void* k_new, const void* v_new,
                                      void* k_win, void* v_win, int32_t window, int32_t sinks,
                                      const int32_t* seq_lens, const int32_t* block_tables,
                                      int32_t max_blocks_per_seq, void* k_pages, void* v_pages, int64_t num_blocks,
                                      int32_t block_size, int32_t batch, int32_t* d_err, void* stream) {
    clear_error();
    const tq_status st = validate_window_append(kc, vc, k_new, v_new, k_win, v_win, window, sinks, seq_lens,
                                                block_tables, max_blocks_per_seq, k_pages, v_pages, num_blocks,
                                                block_size, batch);
    if (st != TQ_OK || batch == 0) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t n_vec = static_cast<int64_t>(batch) * kc->desc.num_kv_heads * 2;
    const int64_t blocks = std::min<int64_t>((n_vec + kPackWarps - 1) / kPackWarps, 148 * 32);
    window_append_kernel<<<static_cast<unsigned>(blocks), kPackWarps * 32, 0, s>>>(
        kc->dev, vc->dev, static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
        static_cast<__nv_bfloat16*>(k_win), static_cast<__nv_bfloat16*>(v_win), window, sinks, seq_lens,
        block_tables, max_blocks_per_seq, static_cast<uint8_t*>(k_pages), static_cast<uint8_t*>(v_pages),
        num_blocks, block_size, batch, d_err);
    return finish_pack(s, d_err);
}

namespace tq {
tq_status finish_pack(cudaStream_t s, int32_t* d_err) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(TQ_ERR_CUDA, std::string("pack launch: ") + cudaGetErrorString(e));
    if (checked_mode()) {
        if ((e = cudaStreamSynchronize(s)) != cudaSuccess)
            return fail(TQ_ERR_CUDA, std::string("pack: ") + cudaGetErrorString(e));
        if (d_err) {
            int32_t h = 0;
            if (cudaMemcpy(&h, d_err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
                return fail(TQ_ERR_CUDA, "reading the device error word failed");
            if (h & TQ_DERR_SLOT) return fail(TQ_ERR_INDEX, "slot mapping points outside the allocated pages");
            if (h & TQ_DERR_BLOCK) return fail(TQ_ERR_INDEX, "block table entry outside the allocated pages");
        }
    }
    return TQ_OK;
}
}  // namespace tq

// tq_decode_paged_static: decode attention that allocates nothing.
//
// Some callers cannot call cudaMalloc: code that runs inside another runtime
// which owns all device memory (a serving engine that reserves the whole GPU
// for its page pool up front and forbids later allocations), or code on a
// path where cudaMalloc's implicit device-wide synchronization is not
// allowed. For them this entry point runs the same kernels as tq_decode_paged
// with the split-K scratch in a fixed array that is part of this library's
// device image instead of a caller-provided workspace.
//
// The array is TQ_STATIC_WORKSPACE_BYTES (32 MiB): every GPU that loads the
// library holds it until the process exits. A call whose workspace need
// (tq_decode_workspace_bytes) exceeds it is rejected before anything is
// launched. Every call shares the array and the array keeps the last call's
// contents; nothing in it must start at zero, since each call rewrites every
// record it later reads. Calls whose kernels overlap on the GPU (on different
// streams, or from different host threads) race on the array.

#include <cuda_runtime.h>

#include <mutex>
#include <string>
#include <vector>

#include "tq_internal.h"

namespace {

constexpr size_t kStaticBytes = TQ_STATIC_WORKSPACE_BYTES;

// In host code this name is only a stand-in for the symbol, not a device
// address: the address comes from cudaGetSymbolAddress (below).
__device__ __align__(256) unsigned char g_static_workspace[kStaticBytes];

std::mutex g_mu;
std::vector<void*> g_device_addr;  // per device ordinal; nullptr until looked up

// Device address of the array on the current device. The first call on a
// device looks it up (with that device current) and caches it.
tq_status static_workspace(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return tq::fail(TQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    std::lock_guard<std::mutex> lock(g_mu);
    if (dev >= static_cast<int>(g_device_addr.size())) g_device_addr.resize(dev + 1, nullptr);
    if (!g_device_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess || !p)
            return tq::fail(TQ_ERR_CUDA, std::string("static workspace could not be loaded on device ") +
                                             std::to_string(dev) + " (" + cudaGetErrorString(e) + ")");
        g_device_addr[dev] = p;
    }
    *out = g_device_addr[dev];
    return TQ_OK;
}

}  // namespace

extern "C" size_t tq_static_workspace_bytes(void) { return kStaticBytes; }

extern "C" tq_status tq_decode_paged_static(const tq_codec* kc, const tq_codec* vc, const void* q,
                                            const void* k_pages, const void* v_pages, const int32_t* block_tables,
                                            int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch,
                                            int32_t num_q_heads, int32_t max_seq_len, const void* k_win,
                                            const void* v_win, int32_t window, float softmax_scale,
                                            int64_t num_blocks, int32_t block_size, float* out, int32_t* d_err,
                                            void* stream) {
    tq::clear_error();
    if (!kc || !vc) return tq::fail(TQ_ERR_VALUE, "null codec");
    const size_t need =
        tq_decode_workspace_bytes(batch, num_q_heads, kc->desc.num_kv_heads, max_seq_len, block_size);
    if (need > kStaticBytes)
        return tq::fail(TQ_ERR_VALUE, "this call needs " + std::to_string(need) +
                                          " bytes of decode workspace, more than the " +
                                          std::to_string(kStaticBytes) + "-byte static workspace");
    void* ws = nullptr;
    tq_status st = static_workspace(&ws);
    if (st != TQ_OK) return st;
    return tq_decode_paged(kc, vc, q, k_pages, v_pages, block_tables, max_blocks_per_seq, seq_lens, batch,
                           num_q_heads, max_seq_len, k_win, v_win, window, softmax_scale, num_blocks, block_size,
                           out, ws, kStaticBytes, d_err, stream);
}

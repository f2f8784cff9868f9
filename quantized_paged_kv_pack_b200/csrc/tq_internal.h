// Internal declarations shared by the host codec and the CUDA kernels of libtq.
#pragma once

#include <cuda_runtime_api.h>

#include <cstdint>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "tq.h"

namespace tq {

constexpr int kHeadDim = 128;   // the only head_dim the kernels implement
constexpr int kMaxHeads = 1024;
constexpr int kMaxLevels = 16;  // 4-bit codebooks at most on the GPU path

// Quantizer cell table of one codebook, used by the tensor-core packs: a
// rotated unit coordinate u, scaled to v = 64 u, falls into cell round(v) + 64
// of 129 cells over [-64, 64]; a cell holds the number of decision boundaries
// strictly below it and the one boundary inside it (in units of v; +inf when
// none). Adjacent boundaries of the 2-, 3- and 4-bit codebooks of dimension
// 128 (and of the wider ones of smaller groups) are more than one unit of v
// apart, so no cell holds two; build_pack_cells returns false if one does. A
// codec builds one per group on the host and copies them to the device with its
// other tables.
constexpr int kPackCells = 129;
constexpr float kPackCellScale = 64.0f;
struct PackCell {
    float thr;       // boundary inside the cell, +inf if none
    int32_t below;   // boundaries strictly below the cell
};
bool build_pack_cells(const float* boundaries, int levels, PackCell* out);

// Device-side view of one codec, passed to kernels by value.
struct DevCodec {
    const float* sign;      // [128] +1 / -1
    const float* cent;      // [2][16] centroids (fp16-exact values)
    const float* bound;     // [2][16] boundaries, 15 used, entry 15 = +inf
    const int16_t* perm;    // [H][128] packed position -> rotated coordinate
    const int16_t* pos;     // [H][128] rotated coordinate -> packed position
    int32_t num_heads;
    int32_t n_groups;
    int32_t bits[2];
    int32_t size[2];
    int32_t pos0[2];        // first packed position of each group
    int32_t byte_off[2];    // byte offset of each group's bitstream in the row
    int32_t index_bytes;    // bytes before the norms: the index bitstreams, then the QJL signs
    int32_t row_bytes;
    int32_t qjl;            // 1: QJL residual stage
    int32_t mse_bytes;      // bytes of the index bitstreams
    int32_t norm_bytes;     // 2, or 4 with QJL (norm, residual norm)
    const float* qjl_st;    // QJL: S transposed, [128][128] (entry j * 128 + i = S[i][j])
    int32_t groupwise;      // 1: group-wise rotation with per-group norms
    const float* rot_t;     // group-wise: R transposed per head, [H][128][128] (entry (h, j, p) = R_h[p][j])
    int32_t recipe;         // 1: the recipe row (group-wise and QJL): per group [indices][signs], norms
                            // (n_g, residual norm_g) per group; qjl_st is then S_0^T then S_1^T (n_g x n_g)
    int32_t sign_off[2];    // byte offset of each group's QJL sign bits in the index part (QJL: the one
                            // stream after the index bitstreams)
    const PackCell* cells;  // the pack's quantizer cell table of each group [n_groups][129]; null when a
                            // cell would hold two boundaries
};

// Arguments of the decode kernels (device pointers; see tq_decode_paged).
struct DecodeArgs {
    DevCodec kc, vc;
    const void* q;                 // bf16 [B][H_q][128]
    const uint8_t* k_pages;
    const uint8_t* v_pages;
    const int32_t* block_tables;
    int32_t max_blocks;
    const int32_t* seq_lens;
    int32_t batch, num_q_heads, max_seq_len;
    const void* k_win;             // bf16 [B][H_kv][window][128]
    const void* v_win;
    int32_t window;
    float scale_log2;              // softmax_scale * log2(e)
    int64_t num_blocks;
    int32_t block_size;
    int32_t split_tokens, max_splits, items_per_unit;
    float* ws;                     // records [B][H_kv][items_per_unit][G][2 + 128]
    float* qrot;                   // rotated, scaled queries [B][H_q][128] in K packed order
    float* qjl_q;                  // QJL and recipe keys: the projections of the scaled rotated query,
                                   // [B][H_q][128], permuted so that each lane's B-fragment values of a
                                   // sign k-step are adjacent
    int32_t* work_list;            // tensor-core kernels: (sequence, split) pairs of the non-empty
                                   // work items, [B * items_per_unit][2], built on the device
    int32_t* work_count;           // number of pairs in work_list
    int* d_err;
    // Fused window append (tq_window_append_decode): extra prologue CTAs append the step's new token
    // per (sequence, KV head) as tq_window_append would, and the prologue's window CTAs read the token
    // from k_new / v_new for the dense slot it takes (the append may be writing that slot meanwhile).
    // The decode then reads what it would read after a separate append. app_on = 0: no append.
    int32_t app_on;
    const void* k_new;             // bf16 [B][H_kv][128]
    const void* v_new;
    void* k_win_w;                 // the dense buffers and pages the append writes
    void* v_win_w;
    uint8_t* k_pages_w;
    uint8_t* v_pages_w;
    int32_t app_window, app_sinks; // the append's W and S (the decode's window is S + W)
    // Test hook (TQ_TEST_WITHHOLD_COPIES=1): the tensor-core kernels' producer
    // issues no copies, so the compute warps' bounded waits expire and report
    // TQ_DERR_TIMEOUT. Nothing sets it in normal use.
    int32_t withhold_copies;
};

}  // namespace tq

struct tq_codec {
    tq_format_desc desc;
    std::vector<int16_t> high;     // owned copy of desc.high_coords
    uint16_t cent16[2][16];
    float cent[2][16];
    float bound[2][16];
    float sign[tq::kHeadDim];
    std::vector<int16_t> perm;     // [H][d]
    std::vector<int16_t> pos;      // [H][d]
    std::vector<float> qjl_s;      // QJL: S, [d][d] row-major
    std::vector<float> rot_t;      // group-wise: R transposed per head, [H][d][d]
    int32_t row_bytes = 0;
    int32_t index_bytes = 0;
    int device = 0;
    void* d_tables = nullptr;
    tq::DevCodec dev{};
};

namespace tq {

// Runs f() (which returns a cudaError_t) once per device ordinal for each
// call site: settings such as a kernel's shared-memory attribute apply only to
// the device that is current when they are made. A failure is returned and
// retried on the next call.
template <class F>
cudaError_t once_per_device(int dev, F&& f) {
    static std::mutex mu;
    static std::vector<int8_t> done;
    if (dev < 0) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (static_cast<size_t>(dev) >= done.size()) done.resize(static_cast<size_t>(dev) + 1, 0);
    if (done[dev]) return cudaSuccess;
    const cudaError_t e = f();
    if (e == cudaSuccess) done[dev] = 1;
    return e;
}

#ifdef __CUDACC__
// Launches `kernel` with programmatic stream serialization: it may start while
// the previous kernel in `stream` is still running, and must call
// griddepcontrol.wait before it reads anything that kernel writes.
template <class... KArgs, class... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
#endif

// The argument checks of tq_window_append (TQ_OK for batch == 0 as well).
tq_status validate_window_append(const tq_codec* kc, const tq_codec* vc, const void* k_new, const void* v_new,
                                 const void* k_win, const void* v_win, int32_t window, int32_t sinks,
                                 const int32_t* seq_lens, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                 const void* k_pages, const void* v_pages, int64_t num_blocks, int32_t block_size,
                                 int32_t batch);

// Sets the thread-local error message and returns `st`.
tq_status fail(tq_status st, const std::string& msg);
void clear_error();

// Validates a descriptor against the GPU format limits.
tq_status validate_desc(const tq_format_desc* desc);

// Builds every host table of a codec (no CUDA call).
tq_status build_host_tables(const tq_format_desc* desc, tq_codec* c);

// True when TQ_CHECKED=1 is set in the environment.
bool checked_mode();

// Decode split-K geometry shared by the workspace sizing and the kernels.
struct SplitPlan {
    int32_t split_tokens;   // packed tokens per work item (multiple of block_size)
    int32_t max_splits;     // packed work items per (sequence, KV head)
    int32_t items_per_unit; // max_splits + 1 (the last one is the window)
    int32_t group;          // query heads per KV head
    size_t record_floats;   // floats per work item record
    size_t record_bytes;    // bytes of all records (256-byte multiple); rotated queries follow
    size_t list_offset;     // byte offset of the work list (and then its count) in the workspace
    size_t workspace_bytes;
};
// sms: the device's SM count (the grid of the persistent decode kernels), used to choose the
// split length; 0 keeps the longest split. The workspace layout (max_splits, items_per_unit and
// the sizes) is the same for every sms.
bool make_split_plan(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_seq_len,
                     int32_t block_size, int32_t sms, SplitPlan* plan);

// The tensor-core packs (uniform 4-bit, plain, QJL, group-wise and recipe
// formats that have an instantiation); TQ_ERR_UNSUPPORTED (nothing launched)
// when either codec has none, or for buffers not 16-byte aligned.
tq_status launch_pack_tc(const tq_codec* kc, const tq_codec* vc, const void* k, const void* v,
                         const int64_t* slot_mapping, int64_t num_tokens, void* k_pages, void* v_pages,
                         int64_t num_blocks, int32_t block_size, int32_t* d_err, void* stream);
// Launch-error check (and TQ_CHECKED synchronisation) after a pack launch.
tq_status finish_pack(struct CUstream_st* stream, int32_t* d_err);

// Tensor-core decode partials. Returns TQ_ERR_UNSUPPORTED (without launching)
// when the formats or the block size have no instantiation; the caller then
// uses the general kernel.
tq_status launch_decode_mma(const DecodeArgs& a, const tq_codec* kc, const tq_codec* vc, int group,
                            void* stream);

}  // namespace tq

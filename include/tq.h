/*
 * tq.h - C ABI of the compressed paged KV cache library (libtq.so, sm_100a).
 *
 * Two device calls make up the hot path, plus host-only helpers:
 *
 *   tq_pack_kv       quantize K/V token vectors and write packed rows into
 *                    persistent uint8 pages (the serving route's write).
 *   tq_decode_paged  single-token decode attention that reads those pages
 *                    through a block table without rebuilding the history.
 *
 * Pages cited by title and section:
 *   [Design]  TurboQuant documentation, "Design" page.
 *   [Server]  TurboQuant Inference Server README.
 *
 * Conventions for every call:
 *   - Pointers named d_* or documented as "device" are CUDA device memory of
 *     the current device; all others are host memory.
 *   - The caller owns every buffer, the stream and the workspace. The library
 *     allocates device memory only inside tq_make_codec (its tables, under
 *     4 KB), freed by tq_free_codec.
 *   - Device calls only enqueue work on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and return without synchronizing. Conditions the
 *     device detects (a slot or block id outside the pool, a bounded wait that
 *     gave up) are OR-ed into the int32 device word `d_err` (TQ_DERR_* bits)
 *     when it is not NULL; the kernel then skips the offending access instead
 *     of faulting. With the environment variable TQ_CHECKED=1 every device call
 *     synchronizes `stream` and turns a nonzero `d_err` into a status.
 *   - On error no work is enqueued and tq_last_error() describes the cause
 *     (thread-local, valid until the next call on the same thread).
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes; the mapping follows the [Design] "Error Model" section. */
typedef enum {
    TQ_OK = 0,
    TQ_ERR_VALUE = 1,       /* ValueError: bad shapes, bit widths, metadata, argument combinations */
    TQ_ERR_INDEX = 2,       /* IndexError: slot mapping or block id outside the allocated pages */
    TQ_ERR_NOT_FOUND = 3,   /* FileNotFoundError: missing recipe metadata (raised by loaders) */
    TQ_ERR_UNSUPPORTED = 4, /* UnsupportedFormatError: the kernels do not implement this format */
    TQ_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    TQ_ERR_TIMEOUT = 6      /* a bounded pipeline wait inside a kernel gave up */
} tq_status;

/* Bits of the device error word. */
#define TQ_DERR_SLOT 1      /* tq_pack_kv: slot >= num_blocks * block_size (row skipped) */
#define TQ_DERR_BLOCK 2     /* tq_decode_paged, tq_window_append: block table entry outside [0, num_blocks) */
#define TQ_DERR_TIMEOUT 4   /* a kernel's bounded wait expired; its results are invalid */
#define TQ_DERR_LAUNCH 8    /* a kernel could not lay out its shared memory; its results are invalid */

/*
 * One codec (format) for the keys or for the values of a layer.
 * [Design] "System Invariants": key and value formats are independent, so a
 * decode call takes two codecs. [Design] "Recipe Strategy": channels split
 * into a high and a low group, the high group named by sorted calibration
 * indices; a row stores each group's indices, then the vector norm.
 *
 * head_dim       must be 128 on the GPU path (TQ_ERR_UNSUPPORTED otherwise).
 * num_kv_heads   number of KV heads sharing this codec, 1..1024.
 * n_groups       1 (uniform) or 2 (high/low mix).
 * group_bits     bits per index of each group; 2, 3 or 4 on the GPU path.
 * group_size     coordinates per group; multiples of 16 summing to head_dim.
 * high_coords    host int16 [num_kv_heads][group_size[0]]: for each KV head,
 *                the rotated coordinates of group 0, strictly ascending.
 *                NULL when n_groups == 1. Copied by tq_make_codec.
 * hadamard_seed  SplitMix64 seed of the sign vector of the rotation.
 * qjl            0, or 1 for the QJL residual stage ([Design] "Recipe
 *                Strategy": row [MSE indices][QJL signs][vector norm]
 *                [residual norm]). The groups above are the MSE part; the row
 *                then carries head_dim sign bits of S r (r = u - c[idx], the
 *                residual of the unit rotated vector in rotated coordinate
 *                order; bit i = 1 when (S r)_i >= 0, LSB-first) and the fp16
 *                residual norm |r| after the norm. S = tq_codec_qjl_matrix.
 *                In a sub-page the sign bytes follow each row's index bytes and
 *                the norm area holds (norm, residual norm) per row. The key a
 *                row stands for is n R^T (c + sqrt(pi/2)/d |r| S^T z), z = 2 bits
 *                - 1: its product with q is the unbiased QJL estimate of q.x.
 *                Decode accepts QJL for K only.
 * groupwise      0, or 1 for group-wise rotation with per-group norms (two
 *                groups, no QJL): group 0 is the set of ORIGINAL channels
 *                high_coords[h] and group 1 the other channels, each ascending;
 *                each group is rotated on its own, y_g = B_g (s[ch] * x[ch]),
 *                B_g the block-diagonal of orthonormal natural-order Hadamard
 *                blocks of the power-of-two sizes that make up the group size,
 *                largest first (96 = 64 + 32); each group has its own fp16 norm
 *                and a Lloyd-Max codebook for its own dimension. Row: the two
 *                index bitstreams, then the two norms (norm area: 4 bytes per
 *                row).
 *                qjl = 1 together with groupwise = 1 is the recipe row as the
 *                Design page prints it ("Recipe Strategy": two groups, each
 *                [MSE indices][QJL signs][vector norm][residual norm]): each
 *                group is quantized as above and adds the fp16 norm |r_g| of
 *                its residual r_g = u_g - c_g[idx] (the group's rotated order)
 *                and group_size[g] sign bits [(S_g r_g)_i >= 0], S_g a
 *                group_size[g]^2 Gaussian matrix (tq_codec_qjl_matrix). In a
 *                sub-page the index part of a row is [group-0 indices][group-0
 *                signs][group-1 indices][group-1 signs] and its norm area holds
 *                (n_0, |r_0|, n_1, |r_1|), 8 bytes. The key is, per group,
 *                n_g B_g^T (c_g + sqrt(pi/2)/group_size[g] |r_g| S_g^T z_g) on
 *                the group's channels. Decode accepts it for K only.
 */
typedef struct {
    int32_t head_dim;
    int32_t num_kv_heads;
    int32_t n_groups;
    int32_t group_bits[2];
    int32_t group_size[2];
    const int16_t* high_coords;
    uint64_t hadamard_seed;
    int32_t qjl;
    int32_t groupwise;
} tq_format_desc;

typedef struct tq_codec tq_codec; /* opaque, immutable after tq_make_codec */

/*
 * Host tables of a codec, for inspection and tests; no CUDA call is made.
 * Codebook: Lloyd-Max quantizer of one coordinate of a random unit vector in
 * R^head_dim ([Server] "Codebook caching"), centroids rounded to fp16,
 * boundaries the fp32 midpoints of adjacent centroids. Rotation:
 * y = H diag(s) x / sqrt(d), H the natural-order Sylvester matrix,
 * s_i = -1 when bit 0 of the i-th SplitMix64 output is 1.
 *
 * centroids_f16  out, uint16 [2][16]: fp16 bit patterns, ascending, per group
 * boundaries     out, float  [2][15]
 * signs          out, int8   [head_dim], +1 or -1
 * perm           out, int16  [num_kv_heads][head_dim]: packed position ->
 *                rotated coordinate (group 0 coordinates ascending, then the rest)
 * row_bytes      out: index bytes of all groups, plus the QJL sign bytes
 *                (head_dim / 8) of a QJL codec, plus the norm bytes: 2 (fp16
 *                norm), or 4 for a QJL codec (norm, residual norm) and for a
 *                group-wise codec (one norm per group), or 8 for the recipe row
 *                (qjl and groupwise: norm and residual norm per group)
 * Any output pointer may be NULL. Returns TQ_ERR_VALUE / TQ_ERR_UNSUPPORTED
 * for an invalid descriptor (the GPU format limits apply here too).
 */
tq_status tq_codec_host_tables(const tq_format_desc* desc, uint16_t* centroids_f16, float* boundaries,
                               int8_t* signs, int16_t* perm, int32_t* row_bytes);

/*
 * The QJL matrix S of a codec: out, float [head_dim][head_dim], row-major.
 * S[i][j] is the cosine branch of the Box-Muller transform of two uniforms
 * from SplitMix64 seeded with hadamard_seed ^ 0x51534A4C00000001: outputs
 * 2k and 2k + 1 (k = i * head_dim + j) give u1 = ((x >> 11) + 1) 2^-53 and
 * u2 = (x >> 11) 2^-53, S = sqrt(-2 ln u1) cos(2 pi u2) in double, rounded to
 * float. For the recipe row (qjl and groupwise) out receives S_0 then S_1,
 * each group_size[g] x group_size[g] row-major (at most head_dim^2 floats in
 * all), made the same way from the stream seeded with hadamard_seed ^
 * 0x51534A4C00000001 ^ ((g + 1) << 56). Host only; TQ_ERR_VALUE for an
 * invalid descriptor.
 */
tq_status tq_codec_qjl_matrix(const tq_format_desc* desc, float* out);

/*
 * The group-wise rotations of a codec ([Design] "Recipe Strategy": the high
 * channels come from calibration metadata; this library's group-wise reading,
 * groupwise = 1): out, float [num_kv_heads][head_dim][head_dim], row-major,
 * out[h][p][j] = R_h[p][j], the weight of original channel j in packed
 * position p. Rows 0 .. group_size[0] - 1 are group 0 (channels
 * high_coords[h], ascending), the rest group 1 (the other channels,
 * ascending); each group's rows are the orthonormal natural-order Hadamard
 * blocks of the powers of two that make up its size, largest first, applied
 * after the sign flip s[j]. Host only; TQ_ERR_VALUE for an invalid
 * descriptor or one without groupwise.
 */
tq_status tq_codec_group_rotation(const tq_format_desc* desc, float* out);

/*
 * Validate `desc`, build the codec tables on the host and copy them to the
 * current device. *out receives the codec; free it with tq_free_codec (not
 * while kernels that use it are in flight).
 */
tq_status tq_make_codec(const tq_format_desc* desc, tq_codec** out);
void tq_free_codec(tq_codec* codec);

/* Bytes of one packed row of this codec: index bytes of every group, the QJL
 * sign bytes of a QJL codec, and 2 norm bytes (4 for QJL and group-wise, 8 for
 * the recipe row). */
int32_t tq_codec_row_bytes(const tq_codec* codec);

/*
 * tq_pack_kv - the quantize-and-pack write.
 * [Design] "Serving Route Design": write packed rows into persistent pages;
 * slot id -> physical block -> token offset -> packed row bytes, with
 * block = slot / block_size and offset = slot % block_size.
 *
 * k, v           device bf16 [num_tokens][num_kv_heads][head_dim], contiguous.
 * slot_mapping   device int64 [num_tokens]; a negative slot marks a padding
 *                token, which is skipped.
 * k_pages        device uint8 [num_blocks][num_kv_heads][block_size * kc row_bytes]
 * v_pages        device uint8 [num_blocks][num_kv_heads][block_size * vc row_bytes]
 *                (separate pools that share block ids; 8-byte aligned).
 * Row of one (token, head): [group-0 bitstream][group-1 bitstream][fp16 norm],
 * bitstreams LSB-first, the norm little endian; see tq_codec_host_tables for
 * the rotation and codebook. Within the sub-page of (block, head) the index
 * bytes of the block_size rows come first, row after row (offset * index
 * bytes), then the block_size norms (block_size * index bytes + 2 * offset),
 * so index rows stay 8-byte aligned. Each row is written whole; bytes of
 * other rows are untouched. A vector with an inf or NaN element, or a norm of
 * 3e37 or more, gets its norm as computed (inf or NaN in fp16) and indices
 * without meaning; no error flag is set for it.
 * Errors: TQ_ERR_VALUE for inconsistent arguments (num_kv_heads or head_dim
 * differing between the codecs, block_size < 1, null pointers with
 * num_tokens > 0). A slot >= num_blocks * block_size sets TQ_DERR_SLOT in
 * d_err and its row is not written ([Design] "Error Model": IndexError).
 */
tq_status tq_pack_kv(const tq_codec* kc, const tq_codec* vc, const void* k, const void* v,
                     const int64_t* slot_mapping, int64_t num_tokens, void* k_pages, void* v_pages,
                     int64_t num_blocks, int32_t block_size, int32_t* d_err, void* stream);

/*
 * tq_window_append - window eviction with append, the write side of a decode
 * step. [Design] "Data Ownership": CompressedKVCache owns sequence-level
 * compressed blocks and recent windows; [Design] "Format Strategy": recent
 * dense window, boundary tokens kept dense; "Serving Route Design": packed
 * rows are written into persistent pages through block tables.
 *
 * Appends one token per sequence. With L = seq_lens[b] tokens before the
 * call, the dense buffer of (b, head) has sinks + window slots: the first
 * min(sinks, L) tokens in slots 0 .. sinks-1, and token t >= sinks in slot
 * sinks + (t - sinks) % window while it is among the last `window` tokens.
 * The new token L goes to slot L when L < sinks, else to its ring slot; when
 * that slot still holds token L - window, that token is first packed (as
 * tq_pack_kv would) at packed position L - sinks - window of the sequence:
 * block block_tables[b][p / block_size], offset p % block_size. With
 * window = 0 the new token itself is packed, at position L - sinks. The
 * buffers then match what tq_decode_paged reads with window' = sinks + window
 * and seq_lens[b] = L + 1; the caller advances seq_lens.
 *
 * k_new, v_new   device bf16 [batch][num_kv_heads][head_dim]
 * k_win, v_win   device bf16 [batch][num_kv_heads][sinks + window][head_dim],
 *                updated in place (may be NULL when sinks + window == 0)
 * seq_lens       device int32 [batch], lengths before the append (read only)
 * block_tables   device int32 [batch][max_blocks_per_seq]
 * k_pages, v_pages as for tq_pack_kv.
 * Errors: TQ_ERR_VALUE for inconsistent arguments. A packed position past the
 * block table, or a block id outside [0, num_blocks), sets TQ_DERR_BLOCK and
 * that row is not written (the new token still enters the dense buffer).
 * This library's own extension: the pages name the ownership, not the call.
 */
tq_status tq_window_append(const tq_codec* kc, const tq_codec* vc, const void* k_new, const void* v_new,
                           void* k_win, void* v_win, int32_t window, int32_t sinks, const int32_t* seq_lens,
                           const int32_t* block_tables, int32_t max_blocks_per_seq, void* k_pages, void* v_pages,
                           int64_t num_blocks, int32_t block_size, int32_t batch, int32_t* d_err, void* stream);

/*
 * tq_window_append_decode - one decode step: tq_window_append followed by
 * tq_decode_paged on the same stream, with window' = sinks + window and the
 * same seq_lens (the lengths before the append), in fewer launches. The
 * append runs inside the decode's first kernel; that kernel's window
 * attention reads the new token from k_new / v_new for the dense slot it
 * takes, and the decode reads the pages only after the append is complete.
 * The results (out, the dense buffers, the pages, d_err) are those of the two
 * calls. Formats without a tensor-core decode run the two calls as they are.
 * Arguments mean what they mean for tq_window_append and tq_decode_paged;
 * the workspace is sized for window' = sinks + window.
 * This library's own extension: the pages describe the step, not the call.
 */
tq_status tq_window_append_decode(const tq_codec* kc, const tq_codec* vc, const void* k_new, const void* v_new,
                                  void* k_win, void* v_win, int32_t window, int32_t sinks, const void* q,
                                  void* k_pages, void* v_pages, const int32_t* block_tables,
                                  int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch,
                                  int32_t num_q_heads, int32_t max_seq_len, float softmax_scale, int64_t num_blocks,
                                  int32_t block_size, float* out, void* workspace, size_t workspace_bytes,
                                  int32_t* d_err, void* stream);

/*
 * Workspace bytes that tq_decode_paged needs for these sizes; bounded by the
 * runtime shape ([Design] "Serving Route Design": keep workspace bounded).
 * Returns 0 for invalid sizes.
 */
size_t tq_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_seq_len,
                                 int32_t block_size);

/*
 * tq_decode_paged - single-token decode attention over packed pages.
 * [Design] "Serving Route Design": use block tables for logical-to-physical
 * mapping, read K rows inside score computation, read and dequantize V rows
 * inside accumulation. [Design] "System Invariants": production routes
 * consume packed historical K/V (no dense rebuild of the history).
 * [Design] "Format Strategy": recent dense window.
 *
 * For sequence b with seq_lens[b] = L_b tokens (window included), the last
 * n_win = min(window, L_b) tokens are the dense window and the first
 * P_b = L_b - n_win tokens are packed, logical token i in physical block
 * block_tables[b][i / block_size] at offset i % block_size.
 * Query head g reads KV head g / (num_q_heads / num_kv_heads).
 *
 * q              device bf16 [batch][num_q_heads][head_dim]
 * k_pages,
 * v_pages        as written by tq_pack_kv with the same codecs
 * block_tables   device int32 [batch][max_blocks_per_seq]; entries past
 *                ceil(P_b / block_size) are not read
 * seq_lens       device int32 [batch], 0 <= L_b <= max_seq_len
 * max_seq_len    host bound on every L_b (sizes the workspace)
 * k_win, v_win   device bf16 [batch][num_kv_heads][window][head_dim]; slot j
 *                holds logical token P_b + j for j < n_win. May be NULL when
 *                window == 0.
 * softmax_scale  multiplies q.k before the softmax (1/sqrt(128) is usual)
 * out            device fp32 [batch][num_q_heads][head_dim]; a sequence with
 *                L_b = 0 gets zeros
 * workspace      device buffer of at least tq_decode_workspace_bytes(...)
 *                bytes, 256-byte aligned, owned by the caller; it holds the
 *                split-K partials and is fully rewritten by each call.
 * Repeated calls on the same inputs give the same output bit for bit: the
 * split-K work order and every summation order depend on the lengths alone.
 * Errors: TQ_ERR_VALUE for inconsistent sizes or a short workspace,
 * TQ_ERR_UNSUPPORTED for a format the kernels lack. A block id outside
 * [0, num_blocks) sets TQ_DERR_BLOCK (block 0 is read instead, no fault);
 * an expired wait sets TQ_DERR_TIMEOUT.
 */
tq_status tq_decode_paged(const tq_codec* kc, const tq_codec* vc, const void* q, const void* k_pages,
                          const void* v_pages, const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t max_seq_len,
                          const void* k_win, const void* v_win, int32_t window, float softmax_scale,
                          int64_t num_blocks, int32_t block_size, float* out, void* workspace,
                          size_t workspace_bytes, int32_t* d_err, void* stream);

/*
 * The two phases of tq_decode_paged, exposed so a caller can time them
 * apart; tq_decode_paged is exactly tq_decode_partials then tq_decode_combine
 * on the same stream. tq_decode_partials writes one (max, sum, accumulator)
 * record per (sequence, KV head, split) into the workspace; tq_decode_combine
 * merges them by log-sum-exp, undoes the value rotation once per (sequence,
 * query head) and writes `out`. Arguments mean what they mean above.
 */
tq_status tq_decode_partials(const tq_codec* kc, const tq_codec* vc, const void* q, const void* k_pages,
                             const void* v_pages, const int32_t* block_tables, int32_t max_blocks_per_seq,
                             const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t max_seq_len,
                             const void* k_win, const void* v_win, int32_t window, float softmax_scale,
                             int64_t num_blocks, int32_t block_size, void* workspace, size_t workspace_bytes,
                             int32_t* d_err, void* stream);
tq_status tq_decode_combine(const tq_codec* vc, const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
                            int32_t max_seq_len, int32_t window, int32_t block_size, float* out,
                            const void* workspace, size_t workspace_bytes, void* stream);

/*
 * tq_decode_paged_static - tq_decode_paged without a caller-provided workspace.
 * The pages have no counterpart of this call. It is for callers that cannot
 * call cudaMalloc: code running inside another runtime that owns all device
 * memory (for instance a serving engine that reserves the whole GPU for its
 * page pool up front), or code on a path where cudaMalloc's implicit
 * device-wide synchronization is not allowed. It allocates nothing: the
 * split-K scratch is a fixed array of TQ_STATIC_WORKSPACE_BYTES in the
 * library's device image, which every GPU that loads the library holds
 * until the process exits.
 *
 * Arguments mean what they mean for tq_decode_paged. The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and caches it. Under CUDA's lazy module loading (the
 * default) that lookup is also what loads the library's device code on the
 * device and so creates the array there: the first call reserves the
 * 32 MiB and may synchronize. Make it at start-up, before the host runtime
 * reserves the rest of device memory and before any stream capture; if the
 * array cannot be created the call returns TQ_ERR_CUDA with "static
 * workspace could not be loaded". A call whose tq_decode_workspace_bytes(...) exceeds
 * TQ_STATIC_WORKSPACE_BYTES returns TQ_ERR_VALUE before launching anything.
 * All calls share the array and it keeps the last call's contents (nothing
 * in it needs to start at zero); calls whose kernels overlap on the GPU, on
 * different streams or from different threads, race on it.
 */
#define TQ_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)
/* The size of the array this build of the library holds (its
 * TQ_STATIC_WORKSPACE_BYTES), for bindings that do not read this header. */
size_t tq_static_workspace_bytes(void);
tq_status tq_decode_paged_static(const tq_codec* kc, const tq_codec* vc, const void* q, const void* k_pages,
                                 const void* v_pages, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                 const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t max_seq_len,
                                 const void* k_win, const void* v_win, int32_t window, float softmax_scale,
                                 int64_t num_blocks, int32_t block_size, float* out, int32_t* d_err, void* stream);

/*
 * Byte ledger ([Design] "System Invariants": storage bytes and metadata bytes
 * are reported separately; the ratio includes norms, codebooks, transforms,
 * recent windows and workspace). Host arithmetic only.
 *
 * dense_bytes        bf16 K and V of every token: 4 * num_kv_heads * head_dim * sum L_b
 * index_bytes        packed index bytes of the P_b packed tokens, K and V (storage)
 * norm_bytes         the norm bytes of every packed row, K and V: 2 per row, 4 for a
 *                    QJL codec (norm, residual norm) or a group-wise codec (a norm per group)
 * codebook_bytes     fp16 centroids + fp32 boundaries of every group of both codecs
 * transform_bytes    per codec: head_dim int8 signs + num_kv_heads*head_dim int16 permutation,
 *                    + the fp32 head_dim^2 QJL matrix S of a QJL codec, + the dense fp32
 *                    head_dim^2 rotation R_h per KV head that a group-wise codec keeps
 * window_bytes       the allocated bf16 windows, K and V
 * block_table_bytes  one int32 per used block
 * workspace_bytes    tq_decode_workspace_bytes for these sizes
 * page_pool_bytes    the allocated K and V page pools (num_blocks blocks)
 * metadata_bytes     norms + codebooks + transforms + window + block tables + workspace
 * index_only_ratio   dense_bytes / index_bytes (how the [Server] "What it does" table counts)
 * all_in_ratio       dense_bytes / (index_bytes + metadata_bytes)
 */
typedef struct {
    int64_t dense_bytes;
    int64_t index_bytes;
    int64_t norm_bytes;
    int64_t codebook_bytes;
    int64_t transform_bytes;
    int64_t window_bytes;
    int64_t block_table_bytes;
    int64_t workspace_bytes;
    int64_t page_pool_bytes;
    int64_t metadata_bytes;
    double index_only_ratio;
    double all_in_ratio;
} tq_ledger;

/* seq_lens is host int32 [batch]. */
tq_status tq_byte_ledger(const tq_format_desc* kdesc, const tq_format_desc* vdesc, int32_t batch,
                         const int32_t* seq_lens, int32_t window, int32_t num_q_heads, int32_t block_size,
                         int64_t num_blocks, int32_t max_seq_len, tq_ledger* out);

/* Message describing the last error on this thread ("" if none). */
const char* tq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */

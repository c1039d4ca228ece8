/*
 * kvq.h -- C ABI of libkvq: a quantized paged KV cache for NVIDIA B200 (sm_100a).
 *
 * The library writes attention K/V rows into a paged cache in one of seven
 * storage formats and runs GQA attention that reads the pages back: for one
 * new token per sequence (decode) and for a chunk of tokens (chunked
 * prefill).  All compute runs in the library's own CUDA kernels; the caller
 * owns every byte of device memory (the library allocates nothing on the
 * device) and every CUDA stream.
 *
 * Pages the formats come from (cited by title and section):
 *   [NInfer]     "NInfer KV Cache 量化指南：BF16、INT8、FP8、NVFP4 与 K8V4 五种格式怎么选"
 *                -- the paging remark (the cache is managed in 64-token
 *                pages, with K and V allowed different encodings), the
 *                per-token byte table, and the format paragraphs (section
 *                "五种格式逐个认识").
 *   [TokenSpeed] "TokenSpeed量化实战：fp8、NVFP4与KV缓存压缩如何省下50%显存"
 *                -- "--kv-cache-dtype" table: fp8_e4m3 with unit scale, mxfp8 with
 *                one UE8M0 scale per 32 head_dim elements and 128-token blocks.
 *   [FP8-KV]     "FP8 KV Cache如何提速 ... 长上下文推理的加速秘密"
 *                -- kv_cache_scheme {num_bits 8, type float, strategy tensor,
 *                symmetric}: one scale per tensor.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless a comment says "host".
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is stream-ordered and asynchronous unless stated otherwise.
 *   - Return value: KVQ_OK or a negative-free kvq_status code below.  Argument
 *     errors are detected on the host before any launch; nothing is written then.
 *   - No C++ exception crosses this boundary.
 *   - Element types: bf16 inputs are raw 16-bit patterns (uint16_t), fp16
 *     scales are IEEE binary16 little-endian.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_VERSION 3   /* 2: kvq_prefill_attention; 3: kvq_debug_set_wait_polls, KVQ_ERR_DEVICE_BOUNDS */

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_ARG = 1,        /* null pointer, negative count, bad layer index */
    KVQ_ERR_FORMAT = 2,     /* unknown format or a format/head_dim pair it cannot hold */
    KVQ_ERR_SHAPE = 3,      /* sizes inconsistent (n_q_heads % n_kv_heads, page size, limits) */
    KVQ_ERR_WORKSPACE = 4,  /* pool or workspace smaller than required */
    KVQ_ERR_CUDA = 5,       /* a CUDA runtime call failed (launch error, no device) */
    KVQ_ERR_DEVICE_BOUNDS = 6  /* a kernel recorded an out-of-range slot or page id or a wait that gave up (see kvq_read_device_status) */
} kvq_status;

/* Storage formats.  Bytes per token per kv-head (K + V) at head_dim D = 256,
 * as printed in [NInfer]'s table: BF16 1024, INT8-G64 528, FP8-E4M3 516,
 * NVFP4-G16 288, K8V4 402. */
typedef enum {
    KVQ_BF16 = 0,        /* [NInfer] BF16: K stored bit-exact as bf16, V stored as fp16 */
    KVQ_FP8_ROW256 = 1,  /* [NInfer] FP8-E4M3 row-256: E4M3 codes, one fp16 scale per 256 values */
    KVQ_INT8_G64 = 2,    /* [NInfer] INT8-G64: int8 codes, one fp16 scale per 64 values; K Hadamard-rotated */
    KVQ_NVFP4_G16 = 3,   /* [NInfer] NVFP4-G16: E2M1 codes, one UE4M3 scale per 16 values; K and V rotated */
    KVQ_K8V4 = 4,        /* [NInfer] K8V4: K as FP8-E4M3 row-256, V as NVFP4-G16 (rotated) */
    KVQ_MXFP8_G32 = 5,   /* [TokenSpeed] mxfp8: E4M3 codes, one UE8M0 scale per 32 values */
    KVQ_FP8_TENSOR = 6   /* [FP8-KV] / [TokenSpeed] fp8_e4m3: E4M3 codes, one fp32 scale per tensor */
} kvq_format;

/* kvq_cache_desc.flags */
#define KVQ_FLAG_NO_ROTATE 1u   /* store rotated formats without the Hadamard step (tests only) */

/* Element codecs of kvq_encode() (test surface). */
typedef enum {
    KVQ_CODE_E4M3 = 0,   /* 1 byte per value: E4M3, nearest-even, saturating at +-448 */
    KVQ_CODE_E2M1 = 1,   /* 1 byte per value (low nibble): E2M1, nearest-even, saturating at +-6 */
    KVQ_CODE_INT8 = 2,   /* 1 byte per value: nearest-even integer clamped to [-127, 127] */
    KVQ_CODE_FP16 = 3,   /* 2 bytes per value: binary16, nearest-even, saturating at +-65504 */
    KVQ_CODE_UE4M3 = 4   /* 1 byte per value: E4M3 of a non-negative value, sign bit cleared */
} kvq_code;

typedef struct {
    int32_t format;        /* kvq_format */
    int32_t head_dim;      /* D: 128 or 256; formats that rotate (and FP8-row-256) need 256 */
    int32_t n_kv_heads;    /* H_kv >= 1 */
    int32_t page_size;     /* tokens per page: 16..256, multiple of 16 ([NInfer] 64; [TokenSpeed] mxfp8 128) */
    int32_t num_pages;     /* pages per layer in the pool */
    int32_t num_layers;    /* >= 1 */
    uint32_t flags;        /* KVQ_FLAG_* */
    const float* tensor_scales;  /* host, FP8_TENSOR only: [num_layers][2] = (K scale, V scale),
                                    copied at create; NULL means 1.0 ([TokenSpeed] unit scale) */
} kvq_cache_desc;

typedef struct kvq_cache kvq_cache;   /* opaque host-side handle */

/* Bytes of K+V data per token per kv-head for a format at head_dim D (codes
 * plus scales, no padding): the [NInfer] per-token table.  0 if invalid. */
size_t kvq_token_bytes(int32_t format, int32_t head_dim);

/* Code and scale bytes of one stored row (one token, one kv-head, K or V). */
int kvq_row_bytes(int32_t format, int32_t head_dim, int32_t is_v,
                  int32_t* code_bytes, int32_t* scale_bytes);

/* Size in bytes of the device pool a cache needs: a 256-byte status header plus
 * num_layers * num_pages * n_kv_heads page slabs.  0 if the descriptor is invalid. */
size_t kvq_cache_bytes(const kvq_cache_desc* desc);

/* Create a cache over a caller-allocated device pool of at least
 * kvq_cache_bytes(desc) bytes, 256-byte aligned.  The handle is host memory
 * owned by the library until kvq_cache_destroy.  No device work is issued: the
 * caller must zero the pool's first 256 bytes (the status header) before the
 * first append; page contents need no initialisation. */
int kvq_cache_create(const kvq_cache_desc* desc, void* pool, size_t pool_bytes, kvq_cache** out);
int kvq_cache_destroy(kvq_cache* cache);

/* Append: quantise n_tokens new K/V rows and store them at their slots.
 * [NInfer] format paragraphs: Hadamard-256 (where the format rotates), group
 * amax, scale rounded to its own format, codes rounded to nearest-even with
 * saturation, written into the page slab of each (slot, kv-head).
 *   k, v          bf16 [n_tokens][n_kv_heads][head_dim], row-major, 16-byte aligned
 *   slot_mapping  int64 [n_tokens]; slot = page * page_size + row; a negative
 *                 slot skips that token; a slot >= num_pages*page_size is skipped
 *                 and recorded in the device status word.
 * Tokens with distinct slots may be appended in any order; two tokens with
 * the same slot in one call race. */
int kvq_append(kvq_cache* cache, int32_t layer, const void* k, const void* v,
               const int64_t* slot_mapping, int32_t n_tokens, void* stream);

/* Workspace bytes kvq_decode_attention needs for these sizes. */
size_t kvq_decode_workspace_bytes(const kvq_cache* cache, int32_t batch, int32_t n_q_heads,
                                  int32_t max_seq_len);

/* Decode attention, one query token per sequence.
 *   q            bf16 [batch][n_q_heads][head_dim]; query head h reads kv-head
 *                h / (n_q_heads / n_kv_heads) (grouped-query attention).
 *   block_table  int32 [batch][max_pages_per_seq]: page ids of each sequence in
 *                order; entries past ceil(seq_len / page_size) are not read.
 *   seq_lens     int32 [batch]: tokens [0, seq_len) are attended; 0 gives a zero
 *                output row; seq_len must be <= max_seq_len.
 *   out          [batch][n_q_heads][head_dim], fp32 if out_fp32 else bf16.
 *   softmax_scale  multiplier of q.k; 0 means 1/sqrt(head_dim).
 *   workspace    device scratch of >= kvq_decode_workspace_bytes(...) bytes,
 *                16-byte aligned, ZEROED BEFORE ITS FIRST USE: it holds the
 *                partials of segments cut between CTAs and the merge counters,
 *                which every call leaves zeroed again (the partials are
 *                rewritten by each call).  Calls sharing a workspace must not
 *                overlap.
 * For rotated K the kernel rotates q by the same Hadamard-256 (q.k is unchanged
 * because the rotation is orthonormal); for rotated V it rotates the output
 * back.  Page ids out of range are replaced by page 0 and recorded in the
 * device status word.  Limit: num_pages * n_kv_heads < 2^30 (KVQ_ERR_SHAPE). */
int kvq_decode_attention(kvq_cache* cache, int32_t layer, const void* q, int32_t n_q_heads,
                         const int32_t* block_table, int32_t max_pages_per_seq,
                         const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                         void* out, int32_t out_fp32, float softmax_scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/* One decode step in one launch: append every sequence's newest token and
 * attend.  Equivalent to kvq_append of token seq_len[b] - 1 of each sequence
 * (at the slot block_table[b][(seq_len[b]-1) / page_size] * page_size +
 * (seq_len[b]-1) % page_size) followed by kvq_decode_attention with the same
 * arguments, but the new rows are quantised inside the decode kernel: the CTA
 * that reads a sequence's last page quantises the new token into its on-chip
 * copy of that page and into the cache ([NInfer]: every decoded token re-reads
 * the whole KV, so a step should not pay a second launch for its one new row).
 *   k_new, v_new  bf16 [batch][n_kv_heads][head_dim], 16-byte aligned; rows of
 *                 sequences with seq_len 0 are ignored.
 * All other arguments, results and errors as kvq_decode_attention. */
int kvq_append_decode(kvq_cache* cache, int32_t layer, const void* k_new, const void* v_new,
                      const void* q, int32_t n_q_heads, const int32_t* block_table,
                      int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                      int32_t max_seq_len, void* out, int32_t out_fp32, float softmax_scale,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Size of the fixed device scratch array used by kvq_decode_attention_noalloc. */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/* kvq_decode_attention without a caller-provided workspace.  This entry point
 * has no counterpart on the pages: it exists for callers that cannot allocate
 * device memory -- a plugin given only its input and output buffers by a host
 * engine, a process under a fixed device-memory budget that forbids new
 * allocations after start-up, or a latency-critical loop where cudaMalloc and
 * cudaFree (which can synchronise the device) are not allowed.
 *   Same arguments and results as kvq_decode_attention, minus the workspace.
 *   Scratch: a file-scope device array of KVQ_NOALLOC_SCRATCH_BYTES (8 MiB) in
 *   the library image; every GPU that loads the library holds it until the
 *   process exits.  Sizes whose workspace (kvq_decode_workspace_bytes) exceeds
 *   it are rejected with KVQ_ERR_WORKSPACE before any launch.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.  Each call clears the part of the array that must start at zero
 *   (a memset on `stream`) and calls no allocating routine.
 *   All calls share the one array: calls that overlap on the GPU (different
 *   streams, or several host threads) race and corrupt each other's results. */
int kvq_decode_attention_noalloc(kvq_cache* cache, int32_t layer, const void* q, int32_t n_q_heads,
                                 const int32_t* block_table, int32_t max_pages_per_seq,
                                 const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                                 void* out, int32_t out_fp32, float softmax_scale, void* stream);

/* Chunked-prefill attention: causal attention of a chunk of query tokens per
 * sequence over the cache, the multi-token form of kvq_decode_attention for a
 * prompt processed in chunks ([NInfer] K8V4 paragraph: the attention kernels
 * over the quantized cache live under its "causal_cache" path).  The chunk's
 * own K/V rows must already be appended (kvq_append).
 *   q            bf16 [total_q][n_q_heads][head_dim]; the rows of sequence b are
 *                cu_q_lens[b] .. cu_q_lens[b+1]-1: its n_b query tokens in order.
 *   cu_q_lens    int32 [batch + 1], nondecreasing, cu_q_lens[0] = 0.
 *   max_q_len    host: the largest n_b.  It sets the grid only: a longer chunk is
 *                still computed in full, with less parallelism; 0 launches nothing.
 *   block_table, max_pages_per_seq  as kvq_decode_attention.
 *   seq_lens     int32 [batch]: cached tokens of each sequence, the chunk
 *                included.  Query token i of sequence b sits at position
 *                seq_lens[b] - n_b + i and attends positions [0, that position],
 *                itself included; query head h reads kv-head
 *                h / (n_q_heads / n_kv_heads).  A row whose position is negative
 *                (n_b > seq_lens[b]) has no keys: its output row is zero.
 *   out          [total_q][n_q_heads][head_dim], fp32 if out_fp32 else bf16.
 *   softmax_scale  multiplier of q.k; 0 means 1/sqrt(head_dim).
 * No workspace; the call allocates nothing.  Rotations as kvq_decode_attention.
 * Arithmetic: q and the dequantised K/V enter the tensor cores as fp16 (bf16 for
 * BF16 keys) with fp32 accumulation; dequantised values beyond fp16's range
 * (|x| > 65504) saturate.  Page ids out of range, and pages past
 * max_pages_per_seq, are replaced by page 0 and recorded in the device status
 * word (bit 1); a pipeline wait that gives up sets bit 2. */
int kvq_prefill_attention(kvq_cache* cache, int32_t layer, const void* q, int32_t n_q_heads,
                          const int32_t* cu_q_lens, int32_t max_q_len, const int32_t* block_table,
                          int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                          void* out, int32_t out_fp32, float softmax_scale, void* stream);

/* Test surface: stored values of the rows at `slots`, as fp32 code x scale in
 * the stored (rotated) domain.  k_out, v_out: fp32 [n][n_kv_heads][head_dim]. */
int kvq_dequant(kvq_cache* cache, int32_t layer, const int64_t* slots, int32_t n,
                float* k_out, float* v_out, void* stream);

/* Test surface: the stored bytes of the rows at `slots` in logical order
 * (element i of a row at code index i, two E2M1 codes per byte with the lower
 * element in the low nibble; scale of group g at scale index g).
 *   k_codes [n][n_kv_heads][code_bytes(K)], k_scales [n][n_kv_heads][scale_bytes(K)],
 *   v_codes, v_scales likewise.  A scale pointer may be NULL when its size is 0. */
int kvq_read_rows(kvq_cache* cache, int32_t layer, const int64_t* slots, int32_t n,
                  uint8_t* k_codes, uint8_t* k_scales, uint8_t* v_codes, uint8_t* v_scales,
                  void* stream);

/* Test surface: element-wise encoder of the append kernel, out = code(x[i]).
 * out holds n bytes (2n for KVQ_CODE_FP16, little-endian). */
int kvq_encode(int32_t code, const float* x, int64_t n, uint8_t* out, void* stream);

/* Read (and optionally clear) the cache's device status word: bit 0 = a slot
 * out of range in kvq_append, bit 1 = a page id out of range in decode or prefill, bit 2 =
 * a decode pipeline wait gave up.  Synchronises `stream`. */
int kvq_read_device_status(kvq_cache* cache, int32_t clear, uint32_t* status, void* stream);

/* Test surface: set how many times a kernel's bounded pipeline wait (a stage
 * copy or a tensor-core result that has not arrived) polls before it gives up,
 * for every decode, fused decode and prefill launched after this call in this
 * process; 0 gives up at once, a negative value restores the default (2^22
 * polls, about a second).  A wait that gives up sets bit 2 of the device status
 * word; the kernel then skips its remaining work, waits (with the default
 * limit) for the copies and tensor-core operations it already issued, and
 * returns, leaving the context usable.  Returns the previous setting.  Host
 * only; no device work. */
int64_t kvq_debug_set_wait_polls(int64_t polls);

const char* kvq_status_string(int status);
int kvq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */

/*
 * pkv.h -- C-ABI of the paged KV-cache attention library (libpkv.so, NVIDIA B200 / sm_100a).
 *
 * What it computes comes from three web pages on KV caches:
 *   [KVB] "KV cache, continuous batching and paged attention"
 *   [KVG] "KV cache, GQA, paging and continuous batching"
 *   [INF] inference guide "a2-inf-2" (PagedAttention, prefix caching, chunked prefill,
 *         KV-cache quantization)
 *
 * The keys and values of every earlier token are cached ([KVB] "The KV cache").  The cache
 * lives in a pool of fixed-size physical blocks of 16 tokens, and each sequence maps its
 * logical positions to non-contiguous blocks through its own block table ([KVG]
 * "PagedAttention", block-table figure).  Several sequences may point at the same blocks
 * (a shared prefix, [INF] "Prefix caching").  Attention is grouped-query: G = H_q / H_kv
 * query heads share one KV head ([KVG] "Mechanics"), and query head h reads KV head h / G.
 * K/V may be stored as fp16/bf16, or quantized as symmetric int8 / int4 codes or fp8 e4m3
 * sharing one fp32 scale per (block, KV head) ([INF] "KV-cache quantization";
 * [KVB] "The KV cache": fp8 or int8 cache).
 *
 * Conventions for every call:
 *   - Device memory (pools, scales, q, out, tables, workspaces) is owned by the caller; the
 *     library allocates only the small host-side pool handle.  Pointers marked [device]
 *     must be device pointers; [host] are host pointers.
 *   - Calls are asynchronous on the given stream (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and never synchronize, except pkv_read_device_status
 *     (pkv_get_device_status).
 *   - Every call validates its arguments on the host before any launch and returns
 *     PKV_OK (0) or a negative PKV_ERR_* code; on error nothing is launched.
 *   - Errors only the device can see (a block id outside the pool, a slot outside the
 *     pool, a context longer than its block table or than max_context_len) skip the
 *     offending work item and set bits in the optional device status word
 *     (pkv_pool_desc.device_status); pkv_read_device_status reports them.  No kernel traps.
 *   - Pool handles are immutable after creation; concurrent calls on different streams
 *     are safe as long as they do not write the same pool blocks.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#define PKV_BLOCK_SIZE 16
#define PKV_MAX_LAYERS 256   /* layers a pool handle may describe */

/* storage / input dtypes */
#define PKV_F16     0
#define PKV_BF16    1
#define PKV_INT8    2   /* symmetric, codes in [-127, 127], scale = amax / 127          */
#define PKV_INT4    3   /* symmetric, codes in [-7, 7], two per byte, element 2j low nibble */
#define PKV_FP8E4M3 4   /* OCP e4m3 ("fn"), saturating, scale = amax / 448               */

/* status codes */
#define PKV_OK               0
#define PKV_ERR_NULL        -1   /* a required pointer is NULL                    */
#define PKV_ERR_ARG         -2   /* an argument is out of range                   */
#define PKV_ERR_DTYPE       -3   /* unsupported dtype or dtype combination         */
#define PKV_ERR_SHAPE       -4   /* inconsistent sizes (e.g. H_q % H_kv != 0)       */
#define PKV_ERR_WORKSPACE   -5   /* workspace NULL or smaller than required        */
#define PKV_ERR_CUDA        -6   /* a CUDA runtime/driver call failed              */
#define PKV_ERR_TIMEOUT     -7   /* a kernel gave up waiting on a copy (bounded)   */
#define PKV_ERR_INDEX       -8   /* the device saw a bad block id / slot / length  */
#define PKV_ERR_UNSUPPORTED -9   /* a shape or option the kernels do not handle      */

/* device status bits (OR-ed into pkv_pool_desc.device_status) */
#define PKV_DEV_BAD_BLOCK   0x1  /* block table entry outside [0, num_blocks)           */
#define PKV_DEV_BAD_SLOT    0x2  /* slot_mapping entry >= num_blocks * 16               */
#define PKV_DEV_BAD_LENGTH  0x4  /* context_len < 0, > 16 * table width, or > max_context_len */
#define PKV_DEV_TIMEOUT     0x8  /* a bounded wait on a bulk copy ran out               */
#define PKV_DEV_BAD_PREFIX  0x10 /* cascade decode: a table does not start with the shared prefix */

typedef struct pkv_pool* pkv_pool_t;   /* opaque host-side handle */

/*
 * Pool description.  Layout of k_data and v_data [device], per layer, dense:
 *   [num_layers][num_blocks][num_kv_heads][16][row_bytes]
 *   row_bytes = 2*head_dim (F16, BF16), head_dim (INT8, FP8E4M3), head_dim/2 (INT4).
 * Each (block, kv head) tile of 16 rows is contiguous (4 KiB for bf16 with head_dim 128).
 * k_scale, v_scale [device]: [num_layers][num_blocks][num_kv_heads] fp32, required for
 * quantized dtypes, ignored otherwise.  device_status [device]: optional int32 word
 * (NULL disables device error reporting); the caller zeroes it before first use.
 * Base pointers must be 16-byte aligned.  Supported: block_size 16, head_dim 64 or 128,
 * 1 .. PKV_MAX_LAYERS layers.  Layers in separate allocations: kv_pool_create_layers.
 */
typedef struct {
    int32_t num_layers;
    int32_t num_blocks;
    int32_t block_size;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t kv_dtype;
    void* k_data;
    void* v_data;
    float* k_scale;
    float* v_scale;
    int32_t* device_status;
} pkv_pool_desc;

/* Bytes of k_data (equal to v_data) for all layers; *scale_bytes (if not NULL) gets the
 * bytes of k_scale (equal to v_scale), 0 for 16-bit pools.  Returns 0 for an invalid
 * description.  The size follows [KVG] "Mechanics" (memory equation): per token and
 * layer, H_kv * head_dim * bytes for K, the same for V, rounded up to whole blocks. */
PKV_API size_t pkv_pool_bytes(const pkv_pool_desc* desc, size_t* scale_bytes);

/* Validate a pool description and create a handle ([INF] "PagedAttention: virtual memory
 * for the cache").  The pool memory stays owned by the caller and must outlive the
 * handle.  *out [host] receives the handle.  No CUDA call is made. */
PKV_API int kv_pool_create(const pkv_pool_desc* desc, pkv_pool_t* out);

/*
 * kv_pool_create_layers -- kv_pool_create for a cache whose layers live in separate
 * allocations (an engine that allocates each layer's cache on its own: the memory equation
 * of [KVG] "Mechanics" is per layer).  desc gives the geometry, dtype and status word; its
 * k_data, v_data, k_scale and v_scale are ignored (they may be NULL).
 *   k_layers, v_layers [host arrays of num_layers device pointers]: layer l's K and V pools,
 *     each [num_blocks][num_kv_heads][16][row_bytes], 16-byte aligned.
 *   k_scale_layers, v_scale_layers [host arrays of num_layers device pointers]: layer l's
 *     fp32 scales [num_blocks][num_kv_heads] (quantized dtypes; NULL arrays otherwise).
 * The arrays are copied into the handle; the memory they point to stays the caller's.
 * Every call then works on the handle as on a dense pool.  No CUDA call is made.
 */
PKV_API int kv_pool_create_layers(const pkv_pool_desc* desc, void* const* k_layers, void* const* v_layers,
                                  float* const* k_scale_layers, float* const* v_scale_layers, pkv_pool_t* out);

/* Release a handle (not the pool memory).  NULL is accepted. */
PKV_API int kv_pool_destroy(pkv_pool_t pool);

/* Workspace kv_append needs for num_tokens tokens: 0 for 16-bit pools; for quantized
 * pools a per-block scratch of (2*num_kv_heads + 1) * 4 bytes per pool block. */
PKV_API size_t kv_append_workspace_bytes(pkv_pool_t pool, int num_tokens);

/*
 * kv_append -- write new tokens' K and V into their slots ([KVB] "The KV cache": the new
 * token's K/V are cached; [KVG] "PagedAttention": blocks are allocated as the sequence
 * grows, slot = physical block * 16 + offset).
 *   k, v [device]: [num_tokens][num_kv_heads][head_dim] of src_dtype.  For 16-bit pools
 *        src_dtype must equal the pool dtype and the write is a byte copy.  For quantized
 *        pools src_dtype must be PKV_BF16 and the write quantizes ([INF] "KV-cache
 *        quantization"), per (block, kv head) touched, separately for K and V, in IEEE fp32:
 *          A = max |x| over this call's tokens in the block;
 *          S_old = 0 if the call writes offset 0 of the block (a fresh block), else the
 *                  stored scale;  s = max(S_old, A / Q), Q = 127 / 7 / 448;
 *          if s > S_old > 0, the block's codes this call does not overwrite are
 *          re-quantized once: int: clamp(rint(c*S_old / s)); fp8: e4m3(value(c)*S_old / s);
 *          new codes: int: clamp(rint(x / s), -Q, Q); fp8: e4m3_rne_satfinite(x / s);
 *          all codes 0 if s == 0; the stored scale becomes s.
 *   slot_mapping [device]: int32 [num_tokens]; a negative slot skips the token (padding).
 *        Two tokens of one call must not share a slot.
 *   workspace [device]: kv_append_workspace_bytes(pool, num_tokens) bytes (may be NULL
 *        when that is 0).
 * Writes only pool blocks named by the slots, and their scales.
 */
PKV_API int kv_append(pkv_pool_t pool, int layer, const void* k, const void* v, int src_dtype,
              const int32_t* slot_mapping, int num_tokens,
              void* workspace, size_t workspace_bytes, void* stream);

/* Tuning options for paged_decode_attn (NULL = defaults). */
typedef struct {
    int32_t engine;            /* 0 auto: the 5th-generation tensor cores (tcgen05, TMEM accumulators)
                                  for head_dim 128, no sliding window and a 16-byte-aligned q with
                                  16-bit pools and G = 64 or 128 query heads per KV head, or fp8 pools
                                  and G = 8 (the e4m3 codes go to the MMA as they are); engine 1 otherwise.
                                  1 warp-level tensor cores (mma.sync), every pool dtype and group size.
                                  2 CUDA-core FP32 FMA with packed fp32x2 pairs, 3 CUDA-core scalar FP32 FMA:
                                  16-bit pools, head_dim 128, G 4 or 8, q 16-byte aligned (else
                                  PKV_ERR_UNSUPPORTED); kept to measure the FP32-pipe form of the decode */
    int32_t partition_tokens;  /* tokens per split-K partition; 0 = chosen from the workload (~256 KiB
                                  of K + V for 16-bit pools, ~192 KiB for quantized ones, fewer
                                  tokens when the batch alone cannot fill the GPU; on the tcgen05
                                  engines for G = 64 (16-bit) and G = 8 (fp8): as few partitions per
                                  sequence as fill the GPU, at most 4096 tokens, whole 128-token
                                  tiles); else a multiple of 16 in [64, 4096] (PKV_ERR_ARG otherwise) */
    int32_t sliding_window;    /* 0 = attend to the whole context; w > 0 = sliding-window attention
                                  ([KVB] "The KV cache": sliding-window or local attention layers):
                                  the query (position context_len - 1) sees only positions
                                  context_len - w .. context_len - 1; blocks wholly before the window
                                  are not read.  Not with paged_decode_attn_cascade. */
} pkv_decode_opts;

/* Workspace paged_decode_attn needs for these sizes and options (bytes): per (sequence,
 * query head, partition) a head_dim + 2 fp32 partial (o, m, l); 0 when every sequence fits
 * one partition.  With a sliding window the partitions cover at most window + 15 tokens per
 * sequence. */
PKV_API size_t paged_decode_workspace_bytes(pkv_pool_t pool, int num_seqs, int num_q_heads,
                                    int max_context_len, const pkv_decode_opts* opts);

/*
 * paged_decode_attn -- one new query token per sequence attends to all its cached tokens,
 * following its block table ([KVB] "Paged attention": the attention kernel follows the
 * block table; [KVG] "What it is": the cache holds K/V of every previous token).
 *   out[b][h][:] = sum_t softmax_t(scale * q[b][h] . K_b[t][h/G]) V_b[t][h/G],  lo_b <= t < context_lens[b]
 * (lo_b = 0, or max(0, context_lens[b] - w) with opts->sliding_window = w)
 * with K_b[t] = pool tile (block_tables[b][t/16], kv head) row t%16, dequantized as
 * code * scale for quantized pools.  A context length of 0 gives a zero row.
 *   q [device]: [num_seqs][num_q_heads][head_dim], q_dtype PKV_F16 or PKV_BF16 (for 16-bit
 *        pools it must equal the pool dtype).
 *   block_tables [device]: int32 [num_seqs][block_table_width]; entries at index >=
 *        ceil(context_len / 16) are never read.  Entries may repeat across sequences.
 *   context_lens [device]: int32 [num_seqs], each <= max_context_len and <= 16 * width.
 *   max_context_len [host]: sizes the split-K grid.
 *   out [device]: fp32 [num_seqs][num_q_heads][head_dim].
 *   workspace [device]: paged_decode_workspace_bytes(...) bytes, 16-byte aligned.
 * num_q_heads / num_kv_heads must be an integer G >= 1 (MHA G = 1 .. MQA H_kv = 1; groups
 * of more than 16 query heads are split over several CTAs that read the same K/V tiles).
 */
PKV_API int paged_decode_attn(pkv_pool_t pool, int layer, const void* q, int q_dtype,
                      const int32_t* block_tables, int block_table_width,
                      const int32_t* context_lens, int num_seqs, int num_q_heads,
                      int max_context_len, float scale, float* out,
                      void* workspace, size_t workspace_bytes,
                      const pkv_decode_opts* opts, void* stream);

/* Size of the fixed device buffer paged_decode_attn_noalloc keeps its split-K partials in. */
#define PKV_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * paged_decode_attn_noalloc -- paged_decode_attn for callers that cannot allocate device
 * memory.  The pages have no counterpart to this call; it exists for callers embedded in a
 * host runtime that owns every device allocation (a serving engine's memory planner, a
 * plugin that may only touch the memory it is given) and for latency-critical paths where
 * a cudaMalloc, which may synchronize the device, is not acceptable.
 * Same arguments, result and errors as paged_decode_attn, minus the workspace: the split-K
 * partials go to a buffer of PKV_NOALLOC_SCRATCH_BYTES (32 MiB) that the library holds in
 * device memory on every GPU that loads it, until the process exits.  A call whose
 * partials (paged_decode_workspace_bytes for the same sizes and options) exceed that size
 * returns PKV_ERR_WORKSPACE without launching anything.  The call allocates nothing.
 * The first call on a device looks up the buffer's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream capture on the device.
 * All calls share the buffer and it keeps the last call's contents (no call relies on them:
 * each writes every partial it reads).  Calls whose kernels may overlap on the GPU race on
 * the buffer; issue them in order on one stream.
 */
PKV_API int paged_decode_attn_noalloc(pkv_pool_t pool, int layer, const void* q, int q_dtype,
                                      const int32_t* block_tables, int block_table_width,
                                      const int32_t* context_lens, int num_seqs, int num_q_heads,
                                      int max_context_len, float scale, float* out,
                                      const pkv_decode_opts* opts, void* stream);

/* Workspace paged_decode_attn_cascade needs (bytes): num_seqs * num_q_heads * (prefix key
 * splits + suffix partitions) * (head_dim + 2) * 4, the prefix split over as many CTAs as
 * fill the GPU.  0 for an unsupported shape.  With shared_prefix_len 0 it equals
 * paged_decode_workspace_bytes. */
PKV_API size_t paged_decode_cascade_workspace_bytes(pkv_pool_t pool, int num_seqs, int num_q_heads,
                                                    int max_context_len, int shared_prefix_len,
                                                    const pkv_decode_opts* opts);

/*
 * paged_decode_attn_cascade -- the decode of paged_decode_attn for a batch whose sequences
 * all begin with the same shared_prefix_len tokens in the same physical blocks ([INF]
 * "Prefix caching": requests attach to the cached blocks of a common prefix; [KVG] "Prefix
 * caching": a 4,000-token system prompt shared by every request).  The result is the same
 * attention over each sequence's whole context; it is computed in two parts merged with
 * the log-sum-exp rule:
 *   - the prefix once per KV group for the whole batch, as a dense tensor-core contraction
 *     of all B * G query rows against the prefix keys (the blocks of block_tables row 0);
 *   - each sequence's own tokens shared_prefix_len .. context_len-1 as in paged_decode_attn.
 * Arguments as paged_decode_attn, plus:
 *   shared_prefix_len: a multiple of 16, 0 < shared_prefix_len <= every context_len and
 *     <= 16 * block_table_width; every table's first shared_prefix_len / 16 entries must
 *     equal row 0's (the device checks and sets PKV_DEV_BAD_PREFIX otherwise; a context
 *     shorter than the prefix sets PKV_DEV_BAD_LENGTH).  0 runs paged_decode_attn.
 *   workspace [device]: paged_decode_cascade_workspace_bytes bytes, 16-byte aligned (always
 *     required).  q [device] 16-byte aligned.
 * Supported: 16-bit pools with head_dim 128 and 128 % G == 0 (PKV_ERR_UNSUPPORTED otherwise);
 * q_dtype equal to the pool dtype.
 */
PKV_API int paged_decode_attn_cascade(pkv_pool_t pool, int layer, const void* q, int q_dtype,
                                      const int32_t* block_tables, int block_table_width,
                                      const int32_t* context_lens, int num_seqs, int num_q_heads,
                                      int max_context_len, int shared_prefix_len, float scale, float* out,
                                      void* workspace, size_t workspace_bytes, const pkv_decode_opts* opts,
                                      void* stream);

/* Workspace paged_prefill_chunk_attn needs (bytes). */
PKV_API size_t paged_prefill_workspace_bytes(pkv_pool_t pool, int chunk_len, int num_q_heads, int ctx_before);

/*
 * paged_prefill_chunk_attn -- one chunk of a long prompt ([INF] "Chunked prefill";
 * [KVB] "Scheduling prefill and decode": prompts split into 512-2,048-token chunks mixed
 * with decodes).  Query row i (position ctx_before + i) attends causally to positions
 * 0 .. ctx_before + i of its sequence: the earlier paged context (possibly shared prefix
 * blocks) and its own chunk up to itself.  The chunk's K/V must already be in the pool
 * (kv_append at positions ctx_before .. ctx_before + chunk_len - 1).
 *   q [device]: [chunk_len][num_q_heads][head_dim], q_dtype must equal the (16-bit) pool dtype.
 *   block_table [device]: int32 [block_table_width] >= ceil((ctx_before + chunk_len) / 16).
 *   out [device]: fp32 [chunk_len][num_q_heads][head_dim].
 * Tensor cores compute Q.K^T and P.V.  16-bit pools only.
 */
PKV_API int paged_prefill_chunk_attn(pkv_pool_t pool, int layer, const void* q, int q_dtype,
                             const int32_t* block_table, int block_table_width,
                             int ctx_before, int chunk_len, int num_q_heads, float scale,
                             float* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * paged_prefill_chunk_attn_window -- paged_prefill_chunk_attn with sliding-window
 * attention ([KVB] "The KV cache": sliding-window or local attention layers): query row i
 * (position ctx_before + i) sees only positions max(0, ctx_before + i + 1 - sliding_window)
 * .. ctx_before + i; key tiles wholly before a CTA's windows are not read.
 * sliding_window 0 is paged_prefill_chunk_attn.  No workspace.  Rows with a window run on
 * the warp-level mma.sync form of the kernel.
 */
PKV_API int paged_prefill_chunk_attn_window(pkv_pool_t pool, int layer, const void* q, int q_dtype,
                                            const int32_t* block_table, int block_table_width,
                                            int ctx_before, int chunk_len, int num_q_heads, float scale,
                                            int sliding_window, float* out, void* stream);

/*
 * kv_copy_blocks -- copy-on-write at divergence ([KVB] "Paged attention": blocks shared
 * copy-on-write by parallel samples, beam search and common prefixes; [KVG]
 * "PagedAttention": sequences with a common prefix point at the same blocks, copy-on-write
 * at divergence).  For j < num_pairs, physical block dst[j] becomes a copy of block src[j]
 * in every layer: its K and V tiles of all KV heads and, for quantized pools, its scales.
 *   src, dst [device]: int32 [num_pairs].  The dst ids must be distinct and none may
 *   appear in src (overlapping pairs race; the result is then undefined).
 * An id outside [0, num_blocks) skips its pair and sets PKV_DEV_BAD_BLOCK.
 */
PKV_API int kv_copy_blocks(pkv_pool_t pool, const int32_t* src, const int32_t* dst, int num_pairs, void* stream);

/* Bytes one block takes in host memory when swapped out (all layers, K and V, scales):
 *   num_layers * 2 * num_kv_heads * 16 * row_bytes  +  num_layers * 2 * num_kv_heads * 4 (quantized).
 * Layout of one swapped block: [layer][K, V][num_kv_heads][16][row_bytes], then
 * [layer][K, V][num_kv_heads] fp32 scales.  Returns 0 for a NULL pool. */
PKV_API size_t kv_swap_bytes_per_block(pkv_pool_t pool);

/*
 * kv_swap_out / kv_swap_in -- preemption by swapping ([KVG] "The scheduler, and
 * preemption": when the cache runs out of blocks, the newest sequence is evicted and its
 * blocks are swapped to host memory, or dropped and recomputed, and brought back on
 * resume).  kv_swap_out copies blocks[j] into host slot j; kv_swap_in copies host slot j
 * into blocks[j].  A slot is kv_swap_bytes_per_block bytes, slots are consecutive.
 *   blocks [device]: int32 [num_blocks_to_move].
 *   host: page-locked host memory mapped into the device's address space (cudaHostAlloc
 *   or cudaHostRegister; the runtime maps it on every system with unified addressing),
 *   16-byte aligned, at least num_blocks_to_move * kv_swap_bytes_per_block bytes.
 *   Anything else returns PKV_ERR_ARG.  One kernel moves every byte over the host link.
 * The host buffer is read or written asynchronously: do not touch it until the stream
 * has passed the call.  An id outside [0, num_blocks) skips that block and sets
 * PKV_DEV_BAD_BLOCK.
 */
PKV_API int kv_swap_out(pkv_pool_t pool, const int32_t* blocks, int num_blocks_to_move, void* host, void* stream);
PKV_API int kv_swap_in(pkv_pool_t pool, const int32_t* blocks, int num_blocks_to_move, const void* host, void* stream);

/* Synchronize `stream`, read and clear the pool's device status word.  *status_out [host]
 * receives the PKV_DEV_* bits (0 if the pool has no status word).  Returns PKV_ERR_TIMEOUT
 * if PKV_DEV_TIMEOUT was set, else PKV_ERR_INDEX if other bits were set, PKV_OK otherwise. */
PKV_API int pkv_read_device_status(pkv_pool_t pool, void* stream, int32_t* status_out);

/* The same call under the name pkv_get_device_status. */
PKV_API int pkv_get_device_status(pkv_pool_t pool, void* stream, int32_t* status_out);

/*
 * pkv_test_withhold_copy -- a test hook for the bounded waits of the attention kernels (the
 * pages have no counterpart; it exists so that the path a kernel takes when a bulk copy never
 * lands can be exercised without faulting anything).  With tile >= 0, every attention kernel
 * launched afterwards in this process (paged_decode_attn and its variants, the prefill
 * chunk, the cascade prefix pass) arms the barrier of its tile-th K/V tile (counted per CTA
 * from 0) without issuing the copy, so that wait never completes, and bounds every wait at
 * wait_cycles SM clock cycles (1 .. 2e9) instead of about 1 s.  A CTA that gives up sets
 * PKV_DEV_TIMEOUT, waits (bounded) for the copies it did issue and for its tensor-core work,
 * and returns without writing its outputs; nothing traps.  tile < 0 restores the defaults
 * (no tile withheld, waits of about 1 s).  Process-wide, not synchronized with launches in
 * flight: for tests only.  Returns PKV_ERR_ARG for wait_cycles out of range.
 */
PKV_API int pkv_test_withhold_copy(int tile, long long wait_cycles);

/* A static description of a status code. */
PKV_API const char* pkv_strerror(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
PKV_API int pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */

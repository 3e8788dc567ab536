/*
 * kvdecode.h -- C interface of libkvdecode.so: one autoregressive decode step of
 * attention over a paged KV cache, for NVIDIA B200 (sm_100a).
 *
 * The method these calls implement is described on three web pages:
 *   [KVF]  "推理速度慢怎么办？KV Cache与Flash Attention如何加速大模型推理" (ipipp.com)
 *   [LES]  "KV缓存与Flash注意力" (FANDEX course lesson)
 *   [BLOG] "KV Cache:推理慢的真正原因" (cybercheems.top)
 *
 * A decode step is: kvd_append (write the new token's K/V into its page), then
 * kvd_decode_attention (the new query attends over every cached token).
 * kvd_merge_lse combines partial results of a context split into partitions.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named as device memory must be CUDA device (or managed) memory
 *    of the current device, 16-byte aligned; the caller owns every buffer.
 *    The library allocates no device memory.
 *  - Page size is fixed at KVD_PAGE_TOKENS = 16 tokens ([BLOG] section
 *    "工程优化手段 / PagedAttention": fixed blocks of 16 tokens and a block table
 *    mapping logical to physical blocks).
 *  - KV pool layout, row-major: k_cache, v_cache [num_blocks][H_kv][16][d];
 *    token t of sequence b, KV head g is row (t % 16) of page
 *    block_table[b * max_blocks_per_seq + t / 16], head g.
 *  - block_table: int32 [B][max_blocks_per_seq]; entries past a sequence's
 *    last page are never read.  seq_lens: int32 [B] tokens to attend,
 *    including the one appended in the same step.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = legacy default stream).  They never synchronise the device.
 *  - Host-side argument errors return before any launch.  Errors found on
 *    the device (a block-table entry outside [0, num_blocks), a sequence
 *    length outside [0, 16 * max_blocks_per_seq], a slot outside the table,
 *    a pipeline wait that ran out) set bits of a device error word that
 *    kvd_read_device_error returns; the offending page or row is skipped,
 *    never read or written out of bounds.
 *  - Supported: dtype fp16 or bf16; d in {64, 128}; H_q % H_kv == 0 with a
 *    group size H_q / H_kv <= 16; B <= KVD_MAX_BATCH;
 *    num_blocks * H_kv * 16 < 2^31.
 */
#ifndef KVDECODE_H
#define KVDECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVD_PAGE_TOKENS 16
#define KVD_MAX_BATCH 4096
#define KVD_MAX_GROUP 16

typedef enum {
    KVD_OK = 0,
    KVD_ERR_INVALID = 1,      /* bad pointer, shape, alignment or size */
    KVD_ERR_UNSUPPORTED = 2,  /* valid arguments outside the supported set */
    KVD_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    KVD_ERR_WORKSPACE = 4     /* workspace missing or smaller than required */
} kvd_status;

typedef enum { KVD_F16 = 0, KVD_BF16 = 1 } kvd_dtype;

/* Device error word bits (kvd_read_device_error). */
#define KVD_DEVERR_BLOCK_TABLE 0x1u   /* block_table entry outside [0, num_blocks) */
#define KVD_DEVERR_SEQ_LEN     0x2u   /* seq_lens entry outside [0, 16 * max_blocks_per_seq] */
#define KVD_DEVERR_SLOT        0x4u   /* append slot outside the block table */
#define KVD_DEVERR_TIMEOUT     0x8u   /* a pipeline wait gave up */

/*
 * kvd_append -- write the new token's K and V into the paged cache.
 * [BLOG] section "缓存的是什么" (KVCache.append writes the step's K/V at
 * position `length`), made paged by section "PagedAttention"; [KVF] section
 * "一、KV Cache" (append the new K/V behind the cache, then attend).
 *
 *   k_cache, v_cache  device, [num_blocks][H_kv][16][d], written in place
 *   block_table       device, int32 [B][max_blocks_per_seq]
 *   slot              device, int32 [B]: logical position of the new token of
 *                     sequence b (its seq_len - 1); slot < 0 skips b
 *   k_new, v_new      device, [B][H_kv][d]
 * For each b with slot[b] >= 0 and each head h, the d storage words of
 * k_new[b][h] are copied verbatim to row slot % 16 of page
 * block_table[b][slot / 16], head h (same for V).  Nothing else changes.
 * The target page must not be shared with another sequence appending in the
 * same call.  Returns KVD_OK or an error; device-side range errors set
 * KVD_DEVERR_SLOT / KVD_DEVERR_BLOCK_TABLE and skip that sequence.
 */
kvd_status kvd_append(void *k_cache, void *v_cache, const int32_t *block_table,
                      const int32_t *slot, const void *k_new, const void *v_new,
                      int B, int H_kv, int d, int num_blocks, int max_blocks_per_seq,
                      kvd_dtype dtype, void *stream);

/*
 * kvd_decode_attention -- the new query of every sequence attends over all of
 * its cached keys and values.
 * [KVF] section "一、KV Cache" (forward_with_kv_cache: softmax(q K^T * scale) V
 * over the whole cache including the appended token, no causal mask);
 * [LES] section "Flash Attention — 分块技巧" and "步骤2:分块softmax" (tiles of K/V
 * with a running (max, sum), so no score matrix is ever written to memory);
 * [BLOG] section "工程优化手段 / GQA" (query head hq reads KV head hq / (H_q/H_kv)).
 *
 *   q          device, [B][H_q][d]
 *   out        device, [B][H_q][d], same dtype as the cache; written for every
 *              row (a sequence of length 0 gets zeros)
 *   scale      score multiplier (usually 1/sqrt(d))
 *   num_partitions
 *              0: automatic (one partition per streaming multiprocessor of
 *              the device, each a CTA of worker warps that share its pages
 *              equally; small problems use fewer).  n >= 1: the concatenated
 *              page list of all (sequence,
 *              KV head) pairs is cut into n equal contiguous partitions; a
 *              pair that spans several partitions is finished by an LSE merge
 *              launched by this call on the same stream.
 *   workspace  device scratch of at least
 *              kvd_workspace_size(B, H_q, H_kv, d, num_partitions) bytes,
 *              256-byte aligned; contents need no initialisation.
 *   lse_out    nullable device float [B][H_q]: natural-log sum of exp of the
 *              scaled scores (-inf for an empty sequence)
 * Output rounding: fp32 accumulation, one round-to-nearest to the dtype.
 */
kvd_status kvd_decode_attention(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_table, const int32_t *seq_lens,
                                float scale, void *out,
                                int B, int H_q, int H_kv, int d, int num_blocks,
                                int max_blocks_per_seq, int num_partitions,
                                void *workspace, size_t workspace_bytes,
                                float *lse_out, kvd_dtype dtype, void *stream);

/*
 * kvd_decode_step -- one whole decode step in one launch: the append of
 * kvd_append followed by the attention of kvd_decode_attention.
 * [KVF] section "一、KV Cache" (the step appends the new token's K/V, then the
 * new query attends over the whole cache including it); [BLOG] "缓存的是什么".
 *
 *   k_new, v_new   device, [B][H_kv][d]: the step's new keys and values
 *   k_cache, v_cache written in place
 *   other arguments as kvd_decode_attention
 * Every sequence b with seq_lens[b] >= 1 appends its new token at position
 * seq_lens[b] - 1 (row (n-1) % 16 of page block_table[b][(n-1) / 16]); a
 * sequence with seq_lens[b] = 0 appends nothing.  The result -- the cache
 * and out -- is bit-identical to kvd_append (slot = seq_lens - 1) followed
 * by kvd_decode_attention with the same num_partitions.  The page that
 * receives the new token must not be shared with another sequence.
 */
kvd_status kvd_decode_step(const void *q, const void *k_new, const void *v_new, void *k_cache,
                           void *v_cache, const int32_t *block_table, const int32_t *seq_lens,
                           float scale, void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                           int max_blocks_per_seq, int num_partitions, void *workspace,
                           size_t workspace_bytes, float *lse_out, kvd_dtype dtype, void *stream);

/*
 * kvd_decode_attention_shared_prefix -- decode attention (optionally with the
 * fused append of kvd_decode_step) for batches whose sequences share prefix
 * pages, reading each shared page once per group instead of once per member.
 * "KV缓存与Flash注意力", sections 实际应用 and 练习 (prefix caching: requests with
 * the same system prompt or document reuse its KV); [BLOG] "PagedAttention"
 * (members' block tables point at the same physical pages).
 *
 *   group_start   device int32 [n_groups + 1]: group g is the contiguous
 *                 sequences group_start[g] .. group_start[g+1]-1
 *   group_pages   device int32 [n_groups]: the first group_pages[g] pages of
 *                 every member are the same physical pages, namely
 *                 block_table[group_start[g]][0 .. group_pages[g]-1]
 *   n_groups      0 makes this call kvd_decode_attention / kvd_decode_step
 *   max_group_size  upper bound on members per group (sizes the launch); a
 *                 larger group, or one whose bounds leave [0, B], is invalid:
 *                 it sets KVD_DEVERR_SEQ_LEN and its members are attended
 *                 whole, without the shared pass
 *   k_new, v_new  nullable; when given, the step's new token is appended as
 *                 in kvd_decode_step (it must land in a private page)
 *   workspace     kvd_shared_prefix_workspace_size(...) bytes, 256-aligned
 *   num_partitions  0: the decode of the private suffixes leaves the shared
 *                 pass a share of the SMs (sized on the device from the two
 *                 passes' pages) and the two run side by side; > 0: exactly
 *                 as in kvd_decode_attention, with no split
 *   other arguments as kvd_decode_attention.
 * The result equals kvd_decode_attention's up to fp32 rounding order (the
 * shared tokens are summed in a separate pass and merged by log-sum-exp).
 * A member shorter than its group's shared pages is attended whole.  The
 * call issues four launches on `stream` (plan, suffix decode, shared pass,
 * merge); the shared pass may run while the suffix decode does, and the
 * merge runs after both.
 */
kvd_status kvd_decode_attention_shared_prefix(
    const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
    const int32_t *block_table, const int32_t *seq_lens, float scale, void *out, int B, int H_q,
    int H_kv, int d, int num_blocks, int max_blocks_per_seq, const int32_t *group_start,
    const int32_t *group_pages, int n_groups, int max_group_size, int num_partitions,
    void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype, void *stream);

/* Workspace bytes of kvd_decode_attention_shared_prefix (0 if the shape is rejected). */
size_t kvd_shared_prefix_workspace_size(int B, int H_q, int H_kv, int d, int n_groups,
                                        int max_group_size, int num_partitions);

/*
 * 8-bit (FP8 E4M3) KV cache.
 * [BLOG] section "工程优化手段 / 量化" (store the cache in 8 bits; a few very large
 * keys would swamp one tensor-wide scale, so scale per channel group); [LES]
 * section "实际应用" (serving with an fp8 KV cache).
 * Format: codes uint8 [num_blocks][H_kv][16][d]; scales float [num_blocks]
 * [H_kv][16][d/32]: one per (token, KV head, group of 32 channels), with
 * s = max|x| / 448 over the group and code = E4M3(x / s) (round to nearest
 * even, saturating; both divisions IEEE fp32); value = s * E4M3(code).
 *
 * kvd_quantize_fp8   n_rows rows of d fp16/bf16 values (device [n_rows][d])
 *                    -> codes [n_rows][d] and scales [n_rows][d/32]
 *                    (e.g. to fill a cache after prefill).  d in {32..128}, step 32.
 * kvd_append_fp8     the append of kvd_append for the 8-bit cache: quantise
 *                    k_new/v_new [B][H_kv][d] into row slot % 16 of page
 *                    block_table[b][slot / 16] of codes and scales.
 * kvd_decode_attention_fp8
 *                    kvd_decode_attention over the 8-bit cache (d = 64 or 128):
 *                    softmax(scale q K^T) V with K, V the dequantised values;
 *                    q and out in dtype; workspace as kvd_decode_attention.
 */
kvd_status kvd_quantize_fp8(const void *src, uint8_t *codes, float *scales, long long n_rows,
                            int d, kvd_dtype dtype, void *stream);
kvd_status kvd_append_fp8(uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                          const int32_t *block_table, const int32_t *slot, const void *k_new,
                          const void *v_new, int B, int H_kv, int d, int num_blocks,
                          int max_blocks_per_seq, kvd_dtype dtype, void *stream);
kvd_status kvd_decode_attention_fp8(const void *q, const uint8_t *k_codes, const uint8_t *v_codes,
                                    const float *k_scale, const float *v_scale,
                                    const int32_t *block_table, const int32_t *seq_lens,
                                    float scale, void *out, int B, int H_q, int H_kv, int d,
                                    int num_blocks, int max_blocks_per_seq, int num_partitions,
                                    void *workspace, size_t workspace_bytes, float *lse_out,
                                    kvd_dtype dtype, void *stream);

/*
 * 8-bit (INT8) KV cache: the same layout, scales and calls as the E4M3 cache
 * above, with symmetric integer codes.
 * [BLOG] section "工程优化手段 / 量化" (quantise the cache from fp16 to int8 or
 * int4, with scales per channel group because of outlier keys); [KVF] section
 * "三、实际落地" (keys and values kept in INT8 or even INT4).
 * Format: codes int8 [num_blocks][H_kv][16][d]; scales float [num_blocks]
 * [H_kv][16][d/32] with s = max|x| / 127 over the group and code = x / s
 * rounded to the nearest integer (ties to even) and clamped to [-127, 127]
 * (a NaN quotient gives 0; both divisions IEEE fp32); value = s * code.
 * Arguments, ownership, validation and errors are those of the _fp8 calls.
 */
kvd_status kvd_quantize_int8(const void *src, int8_t *codes, float *scales, long long n_rows,
                             int d, kvd_dtype dtype, void *stream);
kvd_status kvd_append_int8(int8_t *k_codes, int8_t *v_codes, float *k_scale, float *v_scale,
                           const int32_t *block_table, const int32_t *slot, const void *k_new,
                           const void *v_new, int B, int H_kv, int d, int num_blocks,
                           int max_blocks_per_seq, kvd_dtype dtype, void *stream);
kvd_status kvd_decode_attention_int8(const void *q, const int8_t *k_codes, const int8_t *v_codes,
                                     const float *k_scale, const float *v_scale,
                                     const int32_t *block_table, const int32_t *seq_lens,
                                     float scale, void *out, int B, int H_q, int H_kv, int d,
                                     int num_blocks, int max_blocks_per_seq, int num_partitions,
                                     void *workspace, size_t workspace_bytes, float *lse_out,
                                     kvd_dtype dtype, void *stream);

/*
 * 4-bit (INT4) KV cache: symmetric codes, two per byte, with the per-group
 * scales of the 8-bit caches.
 * [BLOG] section "工程优化手段 / 量化" (quantise the cache from fp16 to int8 or
 * int4, with scales per channel group because of outlier keys); [KVF] section
 * "三、实际落地" (keys and values kept in INT8 or even INT4).
 * Format: codes uint8 [num_blocks][H_kv][16][d/2] -- channel 2i is the low
 * nibble of byte i, channel 2i+1 its high nibble, each a 4-bit two's
 * complement integer; scales float [num_blocks][H_kv][16][d/32] with
 * s = max|x| / 7 over the group and code = x / s rounded to the nearest
 * integer (ties to even) and clamped to [-7, 7] (a NaN quotient gives 0;
 * both divisions IEEE fp32); value = s * code.  d = 64 or 128 for attention.
 * Bytes per (token, KV head) at d = 128: 64 of codes + 16 of scales.
 *
 * kvd_quantize_int4     n_rows rows of d values -> codes [n_rows][d/2] and
 *                       scales [n_rows][d/32]
 * kvd_append_int4       the quantising append (as kvd_append_int8)
 * kvd_decode_attention_int4, kvd_decode_step_int4
 *                       attention (and the fused step) over the INT4 cache,
 *                       arguments as the _int8 calls
 */
kvd_status kvd_quantize_int4(const void *src, uint8_t *codes, float *scales, long long n_rows,
                             int d, kvd_dtype dtype, void *stream);
kvd_status kvd_append_int4(uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                           const int32_t *block_table, const int32_t *slot, const void *k_new,
                           const void *v_new, int B, int H_kv, int d, int num_blocks,
                           int max_blocks_per_seq, kvd_dtype dtype, void *stream);
kvd_status kvd_decode_attention_int4(const void *q, const uint8_t *k_codes, const uint8_t *v_codes,
                                     const float *k_scale, const float *v_scale,
                                     const int32_t *block_table, const int32_t *seq_lens,
                                     float scale, void *out, int B, int H_q, int H_kv, int d,
                                     int num_blocks, int max_blocks_per_seq, int num_partitions,
                                     void *workspace, size_t workspace_bytes, float *lse_out,
                                     kvd_dtype dtype, void *stream);
kvd_status kvd_decode_step_int4(const void *q, const void *k_new, const void *v_new,
                                uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                                const int32_t *block_table, const int32_t *seq_lens, float scale,
                                void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                                int max_blocks_per_seq, int num_partitions, void *workspace,
                                size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                                void *stream);

/*
 * kvd_decode_attention_shared_prefix_{fp8,int8,int4} -- the shared-prefix
 * decode of kvd_decode_attention_shared_prefix over a quantised cache.
 * "KV缓存与Flash注意力", sections 实际应用 and 练习 (prefix caching), with the
 * cache of "KV Cache:推理慢的真正原因", section 工程优化手段 / 量化 (codes plus
 * one fp32 scale per token, KV head and 32 channels).
 *
 *   k_codes, v_codes, k_scale, v_scale
 *                 the quantised pools of kvd_decode_step_{fp8,int8,int4}
 *                 (written only when k_new / v_new are given: the fused
 *                 quantising append)
 *   d             64 or 128 (KVD_ERR_UNSUPPORTED otherwise)
 *   other arguments as kvd_decode_attention_shared_prefix; the workspace is
 *   kvd_shared_prefix_workspace_size(...) bytes, as there.
 * At d = 128 each shared page is dequantised once per (group, KV head) into
 * f16/bf16 tensor-core tiles, every value as a rounded head plus a rounded
 * remainder (in f16 with an error of at most about |code| 2^-25 per value; in
 * bf16 about 2^-15 of it); at d = 64 every warp runs the decode kernel's
 * quantised tile on the staged page.  The result is that of
 * kvd_decode_attention_{fp8,int8,int4} up to that and fp32 rounding order.
 */
kvd_status kvd_decode_attention_shared_prefix_fp8(
    const void *q, const void *k_new, const void *v_new, uint8_t *k_codes, uint8_t *v_codes,
    float *k_scale, float *v_scale, const int32_t *block_table, const int32_t *seq_lens, float scale,
    void *out, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks_per_seq,
    const int32_t *group_start, const int32_t *group_pages, int n_groups, int max_group_size,
    int num_partitions, void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
    void *stream);
kvd_status kvd_decode_attention_shared_prefix_int8(
    const void *q, const void *k_new, const void *v_new, int8_t *k_codes, int8_t *v_codes,
    float *k_scale, float *v_scale, const int32_t *block_table, const int32_t *seq_lens, float scale,
    void *out, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks_per_seq,
    const int32_t *group_start, const int32_t *group_pages, int n_groups, int max_group_size,
    int num_partitions, void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
    void *stream);
kvd_status kvd_decode_attention_shared_prefix_int4(
    const void *q, const void *k_new, const void *v_new, uint8_t *k_codes, uint8_t *v_codes,
    float *k_scale, float *v_scale, const int32_t *block_table, const int32_t *seq_lens, float scale,
    void *out, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks_per_seq,
    const int32_t *group_start, const int32_t *group_pages, int n_groups, int max_group_size,
    int num_partitions, void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
    void *stream);

/*
 * kvd_decode_step_fp8, kvd_decode_step_int8 -- kvd_decode_step over an 8-bit
 * cache: the quantising append of kvd_append_{fp8,int8} followed by the
 * attention of kvd_decode_attention_{fp8,int8}, in one decode launch.
 * [KVF] section "一、KV Cache" (a decode step appends the new token's K/V,
 * then attends over the whole cache including it); [BLOG] section
 * "工程优化手段 / 量化" (the cache those steps read and write holds 8-bit codes
 * with per-group scales).
 *
 *   k_new, v_new     device, [B][H_kv][d] in dtype, 16-byte aligned
 *   k_codes, v_codes, k_scale, v_scale  the 8-bit cache, written in place
 *   other arguments as kvd_decode_attention_{fp8,int8} (d = 64 or 128)
 * Every sequence b with seq_lens[b] >= 1 appends its new token at position
 * seq_lens[b] - 1; seq_lens[b] = 0 appends nothing.  The codes and scales
 * written are bit-identical to kvd_append_{fp8,int8} with slot =
 * seq_lens - 1, and out to that append followed by
 * kvd_decode_attention_{fp8,int8} with the same num_partitions.  The page that
 * receives the new token must not be shared with another sequence.
 */
kvd_status kvd_decode_step_fp8(const void *q, const void *k_new, const void *v_new,
                               uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                               const int32_t *block_table, const int32_t *seq_lens, float scale,
                               void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                               int max_blocks_per_seq, int num_partitions, void *workspace,
                               size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                               void *stream);
kvd_status kvd_decode_step_int8(const void *q, const void *k_new, const void *v_new,
                                int8_t *k_codes, int8_t *v_codes, float *k_scale, float *v_scale,
                                const int32_t *block_table, const int32_t *seq_lens, float scale,
                                void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                                int max_blocks_per_seq, int num_partitions, void *workspace,
                                size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                                void *stream);

/* Bytes of the library's fixed scratch array used by kvd_decode_attention_static. */
#define KVD_STATIC_WORKSPACE_BYTES (8u << 20)

/*
 * kvd_decode_attention_static -- kvd_decode_attention for callers that cannot
 * allocate device memory.  The pages have no counterpart of this call: it is
 * an interface convenience, computing exactly what kvd_decode_attention
 * computes with num_partitions = 0.
 *
 * Some callers are not allowed to allocate: a plugin inside an inference
 * server that is given only its input and output buffers, a runtime that
 * plans all device memory up front, or a decode loop that cannot pay for
 * cudaMalloc / cudaFree, which may synchronise the device.  This entry point
 * takes no workspace argument; its scratch is a fixed array of
 * KVD_STATIC_WORKSPACE_BYTES (8 MiB) compiled into the library, which every
 * GPU that loads the library keeps until the process exits.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 *   Arguments: as kvd_decode_attention (q, caches, block table, lengths,
 *   scale, out, shape, optional lse_out, dtype, stream).
 *   Returns KVD_ERR_UNSUPPORTED, with the needed size in kvd_last_error(),
 *   when the shape needs more scratch than the fixed array holds (the needed
 *   size is kvd_workspace_size(B, H_q, H_kv, d, 0)).
 *   The first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture.
 *   All calls on one device share the array: calls that overlap on the GPU
 *   (on streams not ordered with each other) race and corrupt each other's
 *   results.  No part of the array needs to start at zero; it keeps the last
 *   call's contents.
 */
kvd_status kvd_decode_attention_static(const void *q, const void *k_cache, const void *v_cache,
                                       const int32_t *block_table, const int32_t *seq_lens,
                                       float scale, void *out, int B, int H_q, int H_kv, int d,
                                       int num_blocks, int max_blocks_per_seq, float *lse_out,
                                       kvd_dtype dtype, void *stream);

/*
 * kvd_merge_lse -- combine S partial attention results of each query row.
 * Not printed on the pages as such: it is the running-state rescale of [LES]
 * "步骤2:分块softmax" applied to whole partitions.  With M = max_s lse_s:
 *   LSE = M + ln sum_s exp(lse_s - M),   out = sum_s exp(lse_s - LSE) o_s.
 *
 *   part_o             device float [B][H_q][S][d], each partial normalised
 *   part_lse           device float [B][H_q][S]; -inf marks an empty partial
 *                      (its part_o is ignored)
 *   num_splits_per_seq nullable device int32 [B]: sequence b uses its first
 *                      num_splits_per_seq[b] partials (0..S); NULL = all S
 *   out                device [B][H_q][d] in dtype; lse_out nullable float [B][H_q]
 * A row whose partials are all empty gets out = 0 and lse = -inf.
 */
kvd_status kvd_merge_lse(const float *part_o, const float *part_lse,
                         const int32_t *num_splits_per_seq, int B, int H_q, int d, int S,
                         void *out, float *lse_out, kvd_dtype dtype, void *stream);

/*
 * kvd_read_stream -- read `bytes` of device memory once and fold them into a
 * checksum: the read-only HBM bandwidth ceiling of this device, measured with
 * the memory pipelines the decode kernel uses.  Not a step of the method: the
 * pages only state that decode attention is bound by memory traffic
 * ([LES] section "问题所在"), and this call measures the bandwidth that bounds
 * it, next to the copy (read + write) bandwidth.
 *
 *   src    device, 16-byte aligned, `bytes` readable bytes
 *   bytes  a multiple of 16 (0 is a no-op)
 *   mode   KVD_READ_VECTOR: every thread keeps eight 16-byte loads in flight
 *          over a grid of 4 CTAs per SM;
 *          KVD_READ_BULK: one CTA per SM of 16 warps, each streaming an equal
 *          contiguous share in 8 KB bulk copies (cp.async.bulk) into its own
 *          shared-memory stage, completed on an mbarrier -- the decode
 *          kernel's pipeline without its arithmetic
 *   sink   device uint32: XOR of every 32-bit word of the buffer is XORed into
 *          *sink (zero it first to read the checksum)
 * Asynchronous on `stream`; time it with events on that stream.  A bulk wait
 * that runs out sets KVD_DEVERR_TIMEOUT.
 */
#define KVD_READ_VECTOR 0
#define KVD_READ_BULK 1
kvd_status kvd_read_stream(const void *src, size_t bytes, int mode, uint32_t *sink, void *stream);

/*
 * Bytes of workspace kvd_decode_attention needs for this shape.
 * num_partitions = 0 means the automatic count of the current device (this
 * queries the device; with no usable device it returns 0 and records the
 * reason for kvd_last_error).
 */
size_t kvd_workspace_size(int B, int H_q, int H_kv, int d, int num_partitions);

/*
 * Partition count used when num_partitions = 0 on the current device, or 0
 * if no device is usable.
 */
int kvd_auto_partitions(void);

/*
 * KV-cache bytes per token over all layers:
 *   2 (K and V) x dtype_size x layers x heads x d_head
 * ([BLOG] section "显存账"; [LES] section "KV缓存数学"; [KVF] section "一、KV Cache").
 * Pure arithmetic, no device access.  Returns 0 for a negative argument.
 */
size_t kvd_kv_bytes_per_token(int layers, int heads, int d_head, int dtype_size);

/*
 * Copy the device error word of the current device into *flags (bitwise OR
 * of KVD_DEVERR_* since the last clear) and, if clear != 0, reset it.  This
 * call synchronises the device; it is a diagnostic, not part of a step.
 */
kvd_status kvd_read_device_error(unsigned int *flags, int clear);

/*
 * kvd_set_decode_wait_limit -- testing hook for the failure path of the
 * decode kernel; not for production use.
 * Each worker warp of the decode kernel waits on a shared-memory barrier for
 * every page it streams.  Such a wait polls at most 2^22 times; past that the
 * warp gives up, sets KVD_DEVERR_TIMEOUT, lets every copy it has in flight
 * land (with the full limit) and leaves the launch, whose output is then
 * undefined.  This call sets the poll limit of those page waits for every
 * later decode launch of the process (kvd_decode_attention, kvd_decode_step,
 * the shared-prefix calls' decode pass and the quantised calls): 0 makes every
 * first wait give up at once, a negative value restores the default.  The
 * waits that drain copies in flight always keep the full limit, so a lowered
 * limit ends the launch early and never leaves a copy behind.  Always returns
 * KVD_OK.  (No page of the method corresponds: it exists so that tests can
 * reach the timeout path without a copy that never lands.)
 */
kvd_status kvd_set_decode_wait_limit(long long polls);

/* Text of the last error recorded by a call on this host thread ("" if none). */
const char *kvd_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVDECODE_H */

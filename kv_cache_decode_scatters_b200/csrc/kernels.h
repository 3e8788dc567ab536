// kernels.h -- launchers of the decode-step kernels (internal to libkvdecode).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kvd {

enum class DType { F16 = 0, BF16 = 1 };

// code formats of a quantised KV cache: 8-bit E4M3 or INT8 codes (one per
// byte), or 4-bit INT4 codes (two per byte)
enum class Code8 { E4M3 = 0, INT8 = 1, INT4 = 2 };

struct AppendArgs {
  void *k_cache;
  void *v_cache;
  const int32_t *block_table;
  const int32_t *slot;
  const void *k_new;
  const void *v_new;
  unsigned *err;
  int B, H_kv, d, num_blocks, maxb;
};

struct DecodeArgs {
  const void *q;
  const int32_t *block_table;
  const int32_t *seq_lens;
  void *out;
  float *lse_out;
  float *part_o;      // [slots][G][d]
  float *part_lse;    // [slots][G]
  int32_t *ws_cum;    // [B + 1] pages per sequence, exclusive prefix sum
  unsigned *err;
  float scale_log2;   // scale * log2(e)
  int B, H_q, H_kv, G, num_blocks, maxb;
  int nparts;         // N: partitions (CTAs) of the concatenated page list
  int min_pages;      // lower bound on average pages per used partition
  int evict_first;    // 1: stream K/V with an L2 evict-first hint
  // poll limit of each page wait of the streaming loop (kWaitPolls unless a
  // test lowers it); the waits that drain copies in flight keep kWaitPolls
  uint32_t wait_polls;
  // fused append (all null for attention only): every sequence with
  // seq_lens[b] >= 1 writes k_new[b], v_new[b] at position seq_lens[b] - 1
  const void *k_new;
  const void *v_new;
  void *k_cache;
  void *v_cache;
  // shared-prefix mode (all null otherwise): skip[b] leading pages of
  // sequence b are attended by the prefix pass; those pairs always leave
  // partials, and the merge adds the prefix partials pre_o / pre_lse
  // ([pre_chunks][H_kv][B][G][d] and [pre_chunks][H_kv][B][G])
  const int32_t *skip;
  const float *pre_o;
  const float *pre_lse;
  int pre_chunks;
  // 8-bit cache (null for 16-bit pages): fp32 scales [num_blocks][H_kv][16][d/32]
  // (k_cache / v_cache are then the code pools); written only by the fused append
  float *k_scale;
  float *v_scale;
  // shared-prefix mode (null otherwise): plan[0] caps the partitions used, so
  // that the prefix pass, running beside this launch, keeps the other SMs
  const int32_t *plan;
};

// Quantise rows of d fp16/bf16 words into E4M3 codes + fp32 per-32-channel
// scales; `dst_rows` (nullable) maps source row r to destination row.
struct QuantArgs {
  const void *src;        // [n][d]
  uint8_t *codes;         // [rows][d]
  float *scales;          // [rows][d / 32]
  const int32_t *block_table;  // append mode: destination of k_new/v_new rows
  const int32_t *slot;
  unsigned *err;
  long long n;            // source rows
  int d, H_kv, num_blocks, maxb;
  int append;             // 1: src is [B][H_kv][d] and goes to page rows per slot
  // optional second tensor (append mode): rows n..2n-1 of the launch quantise
  // src2 into codes2 / scales2 (the V rows of an append next to the K rows)
  const void *src2;
  uint8_t *codes2;
  float *scales2;
};

struct PrefixArgs {
  const void *q;
  const int32_t *block_table;
  const int32_t *seq_lens;
  const int32_t *group_start;  // [n_groups + 1]: group g = sequences [start[g], start[g+1])
  const int32_t *group_pages;  // [n_groups]: leading pages every member shares
  int32_t *skip;               // [B], written by the plan: shared pages per sequence (0 = none)
  float *pre_o;                // [chunks][H_kv][B][G][d] normalised partial outputs
  float *pre_lse;              // [chunks][H_kv][B][G]
  unsigned *err;
  float scale_log2;
  int B, H_q, H_kv, G, num_blocks, maxb, n_groups, chunks, fused;
  int maxg;                    // members per group at most: a larger group is invalid
  const float *k_scale;        // quantised cache: scales [NB][H_kv][16][d/32] (else NULL)
  const float *v_scale;
  // plan[0]: partitions the suffix decode uses; plan[2..3]: 64-bit count of
  // the prefix pass's finished warps (zeroed by the plan launch)
  int32_t *plan;
  float weight;                // cost of a prefix page relative to a decode page (0: no split)
  int nparts, min_pages;       // the decode launch's partition bound and minimum pages
  int row_blocks;              // query-row blocks of the prefix launch (grid z)
  int ctas_per_sm;             // prefix CTAs resident on one SM
};

struct GenericMergeArgs {
  const float *part_o;
  const float *part_lse;
  const int32_t *counts;
  void *out;
  float *lse_out;
  int B, H_q, d, S;
};

// Partitions used when the caller asks for the automatic count: one CTA per
// SM of a device with `sms` SMs (each CTA runs 7-16 worker warps).
int decode_auto_parts(int sms);

// Set the text returned by kvd_last_error on this host thread.
void record_error(const char *msg);

cudaError_t launch_append(const AppendArgs &a, DType dt, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, int d, DType dt, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, cudaStream_t s, int grid);
cudaError_t launch_decode_merge(const DecodeArgs &a, int d, DType dt, cudaStream_t s);
cudaError_t launch_generic_merge(const GenericMergeArgs &a, DType dt, cudaStream_t s);
cudaError_t launch_decode_q8(const DecodeArgs &a, int d, DType dt, Code8 fmt, const CUtensorMap &tmK,
                             const CUtensorMap &tmV, cudaStream_t s, int grid);
cudaError_t launch_quantize_q8(const QuantArgs &a, DType dt, Code8 fmt, cudaStream_t s);
// Read-only streaming of `bytes` (a multiple of 16) from src: mode
// KVD_READ_VECTOR or KVD_READ_BULK; XOR of every 32-bit word into *sink.
cudaError_t launch_read_stream(const void *src, size_t bytes, int mode, unsigned *sink,
                               unsigned *err, int sms, cudaStream_t s);
// Prefix pass of the shared-prefix decode: grid (n_groups * chunks, H_kv, row blocks).
cudaError_t launch_prefix(const PrefixArgs &a, int d, DType dt, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, int row_blocks, cudaStream_t s);
// The same pass over a quantised cache (tensor maps over the code pools,
// scales in a.k_scale / a.v_scale): d = 128 on the tensor-memory pass (one
// CTA per SM), d = 64 on the warp-level one.
cudaError_t launch_prefix_q(const PrefixArgs &a, int d, Code8 fmt, DType dt, const CUtensorMap &tmK,
                            const CUtensorMap &tmV, int row_blocks, cudaStream_t s);
// Query rows one prefix CTA handles.
int prefix_rows_per_cta();
// Plan of the shared-prefix call (one CTA, before the decode launch): writes
// the per-sequence skip, the decode's partition count and clears the prefix
// pass's exit count.
cudaError_t launch_prefix_plan(const PrefixArgs &a, cudaStream_t s);
// Sets a.weight, the time of one prefix page (one KV head, one row block)
// relative to one decode page on one SM, which sizes the split of the SMs
// between the two passes (0 without `split`, or where no split pays), and
// a.ctas_per_sm, the prefix CTAs resident per SM, for a 16-bit cache or a
// quantised one of format fmt.
void prefix_split(PrefixArgs &a, int d, bool quantised, Code8 fmt, bool split);

}  // namespace kvd

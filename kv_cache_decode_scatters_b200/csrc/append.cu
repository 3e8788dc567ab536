// append.cu -- scatter the new token's K/V rows into their pages.
//
// "KV Cache:推理慢的真正原因", section 缓存的是什么 (the cache appends the step's
// K and V at position `length`) and section PagedAttention (fixed 16-token
// blocks addressed through a block table): for sequence b with new-token
// position pos = slot[b], head h, the d storage words of k_new[b][h] go to row
// pos % 16 of page block_table[b][pos / 16], head h; same for V.  A pure
// byte copy -- bit-exact by construction.
//
// One warp per (sequence, head): lanes 0..d/8-1 move K in 16-byte vectors,
// lanes 16..16+d/8-1 move V, so every row is one fully used 128-byte-aligned
// transaction group on both sides.
#include "common.cuh"
#include "kernels.h"

namespace kvd {

__global__ void __launch_bounds__(256) append_kernel(const AppendArgs a) {
  // let the decode grid that usually follows be scheduled early; it waits for
  // this grid's writes before it reads anything
  grid_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pair = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (pair >= static_cast<long long>(a.B) * a.H_kv) return;
  const int b = static_cast<int>(pair / a.H_kv);
  const int h = static_cast<int>(pair - static_cast<long long>(b) * a.H_kv);
  const int pos = __ldg(a.slot + b);
  if (pos < 0) return;  // idle sequence: nothing to append
  if (pos >= a.maxb * kPage) {
    if (lane == 0 && h == 0) flag_error(a.err, kErrSlot);
    return;
  }
  const int pb = __ldg(a.block_table + static_cast<size_t>(b) * a.maxb + pos / kPage);
  if (pb < 0 || pb >= a.num_blocks) {
    if (lane == 0 && h == 0) flag_error(a.err, kErrBlockTable);
    return;
  }
  const int chunks = a.d / 8;  // 16-byte vectors per row
  const int half = lane >> 4, c = lane & 15;
  if (c >= chunks) return;
  const size_t dst = ((static_cast<size_t>(pb) * a.H_kv + h) * kPage + pos % kPage) * a.d;
  const size_t src = (static_cast<size_t>(b) * a.H_kv + h) * a.d;
  const uint4 *from = reinterpret_cast<const uint4 *>(
                          static_cast<const uint16_t *>(half ? a.v_new : a.k_new) + src) + c;
  uint4 *to = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(half ? a.v_cache : a.k_cache) + dst) + c;
  *to = __ldg(from);
}

cudaError_t launch_append(const AppendArgs &a, DType, cudaStream_t s) {
  const long long pairs = static_cast<long long>(a.B) * a.H_kv;
  if (pairs == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((pairs + 7) / 8);
  append_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvd

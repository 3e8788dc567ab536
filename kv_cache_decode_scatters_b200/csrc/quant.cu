// quant.cu -- 8- and 4-bit quantisation of K/V rows (FP8 E4M3, INT8 or INT4
// codes).
//
// "KV Cache:推理慢的真正原因", section 工程优化手段 / 量化: store the cache in 8 bits
// with scales per channel group, so a few very large key channels do not
// swamp the scale of the others ("推理速度慢怎么办？KV Cache与Flash Attention如何加速
// 大模型推理", section 三、实际落地, names INT8; serving with an fp8 cache is the
// other common form).  Each row (one token of one KV head) is split into
// groups of 32 channels with one fp32 scale s each:
//  * E4M3: s = max|x| / 448 (448 is the largest E4M3 value), code = E4M3(x / s)
//    rounded to nearest even and saturated;
//  * INT8: s = max|x| / 127, code = x / s rounded to the nearest integer (ties
//    to even) and clamped to +-127; a NaN quotient gives 0;
//  * INT4: the same with 7 for 127, two codes per byte (channel 2i in the low
//    nibble of byte i).
// Both divisions are IEEE fp32 (__fdiv_rn), so the codes are the same on
// every run and every machine.  A group of zeros gets s = 0.
//
// One warp per row (encode_row4, shared with the decode kernel's fused
// append).  In append mode the source rows are the step's k_new and v_new
// [B][H_kv][d] (one launch, K rows then V rows) and each goes to row
// slot % 16 of page block_table[b][slot / 16] of its code and scale pools.
#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace kvd {

template <typename T, Code8 kFmt>
__global__ void __launch_bounds__(256) quantize_q8_kernel(const QuantArgs a) {
  // programmatic dependent launch: wait for the preceding grid's writes
  grid_dependency_wait();
  grid_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long r = static_cast<long long>(blockIdx.x) * 8 + warp;
  const bool second = a.src2 != nullptr && r >= a.n;
  if (second) r -= a.n;
  if (r >= a.n) return;
  const void *src = second ? a.src2 : a.src;
  uint8_t *codes = second ? a.codes2 : a.codes;
  float *scales = second ? a.scales2 : a.scales;
  long long dst = r;
  if (a.append) {
    const int b = static_cast<int>(r / a.H_kv), h = static_cast<int>(r % a.H_kv);
    const int pos = __ldg(a.slot + b);
    if (pos < 0) return;
    if (pos >= a.maxb * kPage) {
      if (lane == 0 && h == 0) flag_error(a.err, kErrSlot);
      return;
    }
    const int pb = __ldg(a.block_table + static_cast<size_t>(b) * a.maxb + pos / kPage);
    if (pb < 0 || pb >= a.num_blocks) {
      if (lane == 0 && h == 0) flag_error(a.err, kErrBlockTable);
      return;
    }
    dst = (static_cast<long long>(pb) * a.H_kv + h) * kPage + pos % kPage;
  }
  const bool live = lane * 4 < a.d;
  float sc;
  const uint32_t word = encode_row4<T, kFmt>(static_cast<const T *>(src) + r * a.d, live, lane, sc);
  if (!live) return;
  if constexpr (kFmt == Code8::INT4)
    *reinterpret_cast<uint16_t *>(codes + dst * (a.d / 2) + lane * 2) = static_cast<uint16_t>(word);
  else
    *reinterpret_cast<uint32_t *>(codes + dst * a.d + lane * 4) = word;
  if ((lane & 7) == 0) scales[dst * (a.d / 32) + (lane >> 3)] = sc;
}

cudaError_t launch_quantize_q8(const QuantArgs &a, DType dt, Code8 fmt, cudaStream_t s) {
  if (a.n == 0) return cudaSuccess;
  const long long rows = a.src2 ? 2 * a.n : a.n;
  const dim3 grid(static_cast<unsigned>((rows + 7) / 8));
  if (fmt == Code8::INT4) {
    if (dt == DType::BF16)
      return launch_pdl(quantize_q8_kernel<__nv_bfloat16, Code8::INT4>, grid, dim3(256), 0, s, a);
    return launch_pdl(quantize_q8_kernel<__half, Code8::INT4>, grid, dim3(256), 0, s, a);
  }
  if (fmt == Code8::INT8) {
    if (dt == DType::BF16)
      return launch_pdl(quantize_q8_kernel<__nv_bfloat16, Code8::INT8>, grid, dim3(256), 0, s, a);
    return launch_pdl(quantize_q8_kernel<__half, Code8::INT8>, grid, dim3(256), 0, s, a);
  }
  if (dt == DType::BF16)
    return launch_pdl(quantize_q8_kernel<__nv_bfloat16, Code8::E4M3>, grid, dim3(256), 0, s, a);
  return launch_pdl(quantize_q8_kernel<__half, Code8::E4M3>, grid, dim3(256), 0, s, a);
}

}  // namespace kvd

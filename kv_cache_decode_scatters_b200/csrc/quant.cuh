// quant.cuh -- the 8- and 4-bit encodings of one K/V row, shared by the
// quantising kernel and the decode kernel's fused append so both write the
// same bits.
//
// "KV Cache:推理慢的真正原因", section 工程优化手段 / 量化: the cache is stored in
// 8 (or 4) bits with one scale per group of 32 channels.
//  * E4M3: s = max|x| / 448, code = E4M3(x / s), round to nearest even, saturated;
//  * INT8: s = max|x| / 127, code = rint(x / s) clamped to +-127, NaN -> 0;
//  * INT4: s = max|x| / 7, code = rint(x / s) clamped to +-7, NaN -> 0, two
//    codes per byte (channel 2i in the low nibble of byte i).
// Both divisions are IEEE fp32 (__fdiv_rn); a group of zeros gets s = 0 and
// codes 0.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace kvd {

// One warp encodes one row of up to 128 channels: lane l holds channels
// 4l .. 4l+3 (`live` false past the row's end: those lanes only join the
// shuffles), a group of 32 channels is 8 lanes, and its maximum takes three
// shuffles.  Returns the lane's four codes -- 8-bit formats: four bytes,
// channel 4l in the low byte; INT4: four nibbles in the low 16 bits, channel
// 4l in the lowest -- and sets `s` to the scale of the lane's group.  All 32
// lanes must call it.
template <typename T, Code8 kFmt>
__device__ __forceinline__ uint32_t encode_row4(const T *row, bool live, int lane, float &s) {
  constexpr float kMax = kFmt == Code8::E4M3 ? 448.0f : (kFmt == Code8::INT8 ? 127.0f : 7.0f);
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (live) {
    const uint2 w = *reinterpret_cast<const uint2 *>(row + lane * 4);
    const T *v = reinterpret_cast<const T *>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = static_cast<float>(v[i]);
  }
  float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
  s = __fdiv_rn(mx, kMax);
  float q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = s == 0.0f ? 0.0f : __fdiv_rn(x[i], s);
  uint32_t word;
  if constexpr (kFmt == Code8::E4M3) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(q[0], q[1]), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(q[2], q[3]), __NV_SATFINITE, __NV_E4M3);
    word = (lo & 0xffffu) | (hi << 16);
  } else if constexpr (kFmt == Code8::INT8) {
    word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float r = q[i] != q[i] ? 0.f : fminf(fmaxf(rintf(q[i]), -127.f), 127.f);
      word |= (static_cast<uint32_t>(static_cast<int>(r)) & 0xffu) << (8 * i);
    }
  } else {
    word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float r = q[i] != q[i] ? 0.f : fminf(fmaxf(rintf(q[i]), -7.f), 7.f);
      word |= (static_cast<uint32_t>(static_cast<int>(r)) & 0xfu) << (4 * i);
    }
  }
  return word;
}

}  // namespace kvd

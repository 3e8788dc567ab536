// stream.cu -- read-only HBM streaming kernels (kvd_read_stream): the measured
// read ceiling that the decode kernel's roofline is compared with, next to the
// copy (read + write) bandwidth.
//
// Decode attention only reads K/V ("KV缓存与Flash注意力", section 问题所在: the
// step is bound by memory traffic, not arithmetic), so its ceiling is the
// device's read bandwidth.  Two forms:
//  * vector  -- every thread keeps eight 16-byte loads in flight (grid-stride,
//               L1 not allocated), the plain-load read ceiling;
//  * bulk    -- the decode kernel's memory pipeline with no arithmetic: one CTA
//               per SM, 16 warps, each streaming an equal contiguous share in
//               8 KB bulk copies (cp.async.bulk) into its own shared-memory
//               stage, completed on an mbarrier, then read back from shared
//               memory.
// Both fold every 32-bit word they read into an XOR checksum (atomicXor into
// `sink`), so no read can be optimised away and the result can be checked.
#include "../../include/kvdecode.h"
#include "common.cuh"
#include "kernels.h"

namespace kvd {

namespace {

constexpr int kVecThreads = 512;
constexpr int kVecBlocksPerSm = 4;
constexpr int kVecUnroll = 8;
constexpr int kBulkWarps = 16;
constexpr int kBulkChunk = 8192;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ unsigned fold(uint4 v) { return v.x ^ v.y ^ v.z ^ v.w; }

__device__ __forceinline__ void sink_warp(unsigned acc, unsigned *sink) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

__global__ void __launch_bounds__(kVecThreads) read_vec_kernel(const uint4 *src, long long n16,
                                                                unsigned *sink) {
  const long long stride = static_cast<long long>(gridDim.x) * kVecThreads;
  long long i = static_cast<long long>(blockIdx.x) * kVecThreads + threadIdx.x;
  unsigned acc = 0;
  for (; i + (kVecUnroll - 1) * stride < n16; i += kVecUnroll * stride) {
    uint4 v[kVecUnroll];
#pragma unroll
    for (int k = 0; k < kVecUnroll; ++k) v[k] = ld_stream(src + i + k * stride);
#pragma unroll
    for (int k = 0; k < kVecUnroll; ++k) acc ^= fold(v[k]);
  }
  for (; i < n16; i += stride) acc ^= fold(ld_stream(src + i));
  sink_warp(acc, sink);
}

__global__ void __launch_bounds__(32 * kBulkWarps, 1)
    read_bulk_kernel(const uint8_t *src, long long bytes, unsigned *sink, unsigned *err) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kBulkWarps];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                              ~static_cast<uintptr_t>(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long chunks = (bytes + kBulkChunk - 1) / kBulkChunk;
  const long long workers = static_cast<long long>(gridDim.x) * kBulkWarps;
  const long long gw = static_cast<long long>(blockIdx.x) * kBulkWarps + warp;
  const long long c0 = chunks * gw / workers, c1 = chunks * (gw + 1) / workers;
  uint8_t *stage = smem + warp * kBulkChunk;
  const uint32_t st = smem_u32(stage), bar = smem_u32(&bars[warp]);
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_init_fence();
  }
  __syncwarp();
  auto size_of = [&](long long c) -> uint32_t {
    const long long left = bytes - c * kBulkChunk;
    return static_cast<uint32_t>(left < kBulkChunk ? left : kBulkChunk);
  };
  auto issue = [&](long long c) {
    if (lane == 0) {
      const uint32_t n = size_of(c);
      mbar_arrive_expect_tx(bar, n);
      bulk_load(st, src + c * kBulkChunk, n, bar);
    }
  };
  unsigned acc = 0;
  uint32_t ph = 0;
  if (c0 < c1) issue(c0);
  for (long long c = c0; c < c1; ++c) {
    const bool ok = mbar_wait_bounded(bar, ph);
    if (!__all_sync(0xffffffffu, ok)) {
      // the copy in flight must land before the CTA may exit
      if (lane == 0) flag_error(err, kErrTimeout);
      mbar_wait_bounded(bar, ph);
      break;
    }
    ph ^= 1u;
    const int n16 = static_cast<int>(size_of(c) / 16);
    const uint4 *s = reinterpret_cast<const uint4 *>(stage);
    for (int k = lane; k < n16; k += 32) acc ^= fold(s[k]);
    // every lane has consumed its words before the stage is refilled
    __syncwarp();
    if (c + 1 < c1) issue(c + 1);
  }
  sink_warp(acc, sink);
}

}  // namespace

cudaError_t launch_read_stream(const void *src, size_t bytes, int mode, unsigned *sink,
                               unsigned *err, int sms, cudaStream_t s) {
  if (bytes == 0) return cudaSuccess;
  if (mode == KVD_READ_VECTOR) {
    read_vec_kernel<<<sms * kVecBlocksPerSm, kVecThreads, 0, s>>>(
        static_cast<const uint4 *>(src), static_cast<long long>(bytes / 16), sink);
    return cudaGetLastError();
  }
  const int smem = kBulkWarps * kBulkChunk + 128;
  cudaError_t e = cudaFuncSetAttribute(read_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  read_bulk_kernel<<<sms, 32 * kBulkWarps, smem, s>>>(static_cast<const uint8_t *>(src),
                                                      static_cast<long long>(bytes), sink, err);
  return cudaGetLastError();
}

}  // namespace kvd

// noalloc.cu -- kvd_decode_attention_static: decode attention whose scratch
// memory is a fixed array inside the library instead of a caller buffer.
//
// Who needs it: callers that may not allocate device memory themselves, for
// example an inference-server plugin that is handed only its input and output
// buffers, a runtime that plans every device byte up front and forbids
// allocations afterwards, or a latency-critical decode loop that cannot
// afford cudaMalloc / cudaFree, which can synchronise the whole device.
//
// The scratch is kStaticWorkspaceBytes (8 MiB) of device memory that every
// GPU which loads this library keeps until the process exits.  The first call
// on a device looks the array's device address up (cudaGetSymbolAddress, with
// that device current); make that first call before any stream capture.  All
// calls on a device share the array, so two calls that overlap on the GPU
// (different streams without ordering between them) race on it.  Nothing in
// it has to start at zero: each call rewrites the page prefix sums it reads,
// and the merge reads only partial results the same call has written.
#include <cstdio>
#include <mutex>

#include "../../include/kvdecode.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = KVD_STATIC_WORKSPACE_BYTES;
static_assert(kStaticWorkspaceBytes % 256 == 0, "static workspace must be a multiple of 256 bytes");

// The scratch array itself.  In host code this name is only a host-side
// stand-in for the symbol, never a device address: kernels get the address
// that cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_ws_ptr[kMaxDevices];

}  // namespace

extern "C" kvd_status kvd_decode_attention_static(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
    const int32_t *seq_lens, float scale, void *out, int B, int H_q, int H_kv, int d,
    int num_blocks, int max_blocks_per_seq, float *lse_out, kvd_dtype dtype, void *stream) {
  char msg[256];
  const size_t need = kvd_workspace_size(B, H_q, H_kv, d, 0);
  if (need == 0) {
    // The shape (or the device query) was rejected.  Let the workspace entry
    // point validate the same call, so both return the same status and the
    // same kvd_last_error text; it fails before it would need a workspace.
    return kvd_decode_attention(q, k_cache, v_cache, block_table, seq_lens, scale, out, B, H_q,
                                H_kv, d, num_blocks, max_blocks_per_seq, 0, nullptr, 0, lse_out,
                                dtype, stream);
  }
  if (need > kStaticWorkspaceBytes) {
    snprintf(msg, sizeof msg,
             "kvd_decode_attention_static: this shape needs %zu bytes of scratch, more than the "
             "library's fixed %zu-byte array; use kvd_decode_attention with a caller workspace",
             need, kStaticWorkspaceBytes);
    kvd::record_error(msg);
    return KVD_ERR_UNSUPPORTED;
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof msg, "kvd_decode_attention_static: no usable current device (%s)",
             cudaGetErrorString(e));
    kvd::record_error(msg);
    return KVD_ERR_CUDA;
  }
  void *ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ws_ptr[dev]) {
      // once per device, with that device current
      e = cudaGetSymbolAddress(&g_ws_ptr[dev], g_static_workspace);
      if (e != cudaSuccess) {
        g_ws_ptr[dev] = nullptr;
        snprintf(msg, sizeof msg,
                 "kvd_decode_attention_static: cudaGetSymbolAddress of the static workspace "
                 "failed: %s",
                 cudaGetErrorString(e));
        kvd::record_error(msg);
        return KVD_ERR_CUDA;
      }
    }
    ws = g_ws_ptr[dev];
  }
  return kvd_decode_attention(q, k_cache, v_cache, block_table, seq_lens, scale, out, B, H_q,
                              H_kv, d, num_blocks, max_blocks_per_seq, 0, ws,
                              kStaticWorkspaceBytes, lse_out, dtype, stream);
}

// api.cu -- the C interface of libkvdecode.so (declared in include/kvdecode.h):
// argument validation, workspace carving, TMA descriptor encoding, launches,
// error reporting.  Every call is asynchronous on the caller's stream except
// kvd_read_device_error.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/kvdecode.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// Device error word of each device that loads the library (bits KVD_DEVERR_*).
__device__ unsigned g_device_error = 0u;

thread_local std::string g_last_error;

kvd_status fail(kvd_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

kvd_status cuda_fail(cudaError_t e, const char *what) {
  return fail(KVD_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
// Average pages per partition (CTA) below which the automatic split stops
// cutting, so each of a CTA's worker warps gets a couple of pages at least.
constexpr int kAutoMinPages = 32;
// Launches with at most this many (sequence, KV head) pairs stream K/V with
// an L2 evict-first hint.
constexpr long long kEvictFirstPairs = 64;

// Poll limit of the decode kernel's streaming waits; negative = kWaitPolls.
// Lowered only through kvd_set_decode_wait_limit (a test hook).
std::atomic<long long> g_wait_polls{-1};

std::mutex g_mu;
int g_sms[kMaxDevices];
unsigned *g_err_ptr[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

kvd_status current_device(int *dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (*dev < 0 || *dev >= kMaxDevices) return fail(KVD_ERR_UNSUPPORTED, "device ordinal %d", *dev);
  return KVD_OK;
}

kvd_status sm_count(int dev, int *sms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int v = 0;
    cudaError_t e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    g_sms[dev] = v;
  }
  *sms = g_sms[dev];
  return KVD_OK;
}

// Device address of this device's error word (looked up once per device,
// with that device current).
kvd_status error_word(int dev, unsigned **p) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void *a = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, g_device_error);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    g_err_ptr[dev] = static_cast<unsigned *>(a);
  }
  *p = g_err_ptr[dev];
  return KVD_OK;
}

kvd_status encoder(PFN_cuTensorMapEncodeTiled_v12000 *fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                                     cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
      return fail(KVD_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode;
  return KVD_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t cum, lse, o, total;
};

WsLayout ws_layout(int B, int G, int d, long long slots) {
  WsLayout L;
  L.cum = 0;
  L.lse = round_up(static_cast<size_t>(B + 1) * 4, 256);
  L.o = L.lse + round_up(static_cast<size_t>(slots) * G * 4, 256);
  L.total = L.o + static_cast<size_t>(slots) * G * d * 4;
  return L;
}

// Shared-prefix scratch after the decode workspace: per-sequence skipped
// pages, the plan (partitions of the suffix decode, the prefix pass's exit
// count), then the prefix chunks' partial lse and o.
struct PrefixLayout {
  size_t skip, plan, pre_lse, pre_o, total;
  int chunks, row_blocks;
};

kvd_status prefix_layout(int B, int H_kv, int G, int d, int n_groups, int max_group_size,
                         size_t base, PrefixLayout *out, bool quantised = false) {
  int dev, sms;
  kvd_status st = current_device(&dev);
  if (st) return st;
  st = sm_count(dev, &sms);
  if (st) return st;
  const long long rows = static_cast<long long>(max_group_size) * G;
  const int rpc = kvd::prefix_rows_per_cta();
  const long long rb = (rows + rpc - 1) / rpc;
  if (rb > 65535) return fail(KVD_ERR_UNSUPPORTED, "group of %d sequences too large", max_group_size);
  // each (group, KV head, row block) unit's pages are cut into contiguous
  // chunks, one CTA each.  At d = 128 (tensor-memory passes) about one CTA
  // per SM for a quantised cache (one resident per SM) and one per two SMs
  // for fp16 / bf16 (two resident per SM): the pass streams beside the
  // suffix decode on the SMs the plan leaves it, where fewer, longer CTAs
  // pay the Q load and the pipeline fill less often and leave the merge
  // fewer partials (measured on the continuous-batching workload: 4 chunks
  // 295.2 us a call, 2 chunks 290.6, 1 chunk 289.5; the quantised pass with
  // 1 chunk instead of 2 lost 39 us, its 64 CTAs filling too few waves).
  // At d = 64 about four per SM.
  const long long units = static_cast<long long>(n_groups) * H_kv * rb;
  long long chunks = d != 128 ? (4LL * sms + units - 1) / units
                              : (quantised ? sms / units : sms / (2 * units));
  chunks = chunks < 1 ? 1 : (chunks > 64 ? 64 : chunks);
  if (static_cast<long long>(n_groups) * chunks > 0x7fffffffLL)
    return fail(KVD_ERR_UNSUPPORTED, "too many groups");
  PrefixLayout L;
  L.chunks = static_cast<int>(chunks);
  L.row_blocks = static_cast<int>(rb);
  L.skip = round_up(base, 256);
  L.plan = L.skip + round_up(static_cast<size_t>(B) * 4, 256);
  L.pre_lse = L.plan + 256;
  const size_t n = static_cast<size_t>(chunks) * H_kv * B * G;
  L.pre_o = L.pre_lse + round_up(n * 4, 256);
  L.total = L.pre_o + n * d * 4;
  *out = L;
  return KVD_OK;
}

kvd_status resolve_parts(int d, int num_partitions, int *N) {
  if (num_partitions < 0) return fail(KVD_ERR_INVALID, "num_partitions < 0");
  if (num_partitions > 0) {
    *N = num_partitions;
    return KVD_OK;
  }
  int dev, sms;
  kvd_status st = current_device(&dev);
  if (st) return st;
  st = sm_count(dev, &sms);
  if (st) return st;
  (void)d;
  *N = kvd::decode_auto_parts(sms);
  return KVD_OK;
}

kvd_status check_heads(int B, int H_q, int H_kv, int d) {
  if (B < 0) return fail(KVD_ERR_INVALID, "B = %d < 0", B);
  if (B > KVD_MAX_BATCH) return fail(KVD_ERR_UNSUPPORTED, "B = %d > %d", B, KVD_MAX_BATCH);
  if (H_q <= 0 || H_kv <= 0) return fail(KVD_ERR_INVALID, "head counts must be positive");
  if (H_q % H_kv) return fail(KVD_ERR_UNSUPPORTED, "H_q = %d not a multiple of H_kv = %d", H_q, H_kv);
  if (H_q / H_kv > KVD_MAX_GROUP)
    return fail(KVD_ERR_UNSUPPORTED, "group size %d > %d", H_q / H_kv, KVD_MAX_GROUP);
  if (d != 64 && d != 128) return fail(KVD_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
  return KVD_OK;
}

}  // namespace

namespace kvd {
// Lets other translation units of the library set the text kvd_last_error returns.
void record_error(const char *msg) { g_last_error = msg; }
}  // namespace kvd

extern "C" {

const char *kvd_last_error(void) { return g_last_error.c_str(); }

kvd_status kvd_set_decode_wait_limit(long long polls) {
  g_wait_polls.store(polls < 0 ? -1 : polls, std::memory_order_relaxed);
  return KVD_OK;
}

size_t kvd_kv_bytes_per_token(int layers, int heads, int d_head, int dtype_size) {
  if (layers < 0 || heads < 0 || d_head < 0 || dtype_size < 0) return 0;
  return 2ull * static_cast<size_t>(dtype_size) * layers * heads * d_head;
}

int kvd_auto_partitions(void) {
  int N = 0;
  if (resolve_parts(128, 0, &N) != KVD_OK) return 0;
  return N;
}

size_t kvd_workspace_size(int B, int H_q, int H_kv, int d, int num_partitions) {
  if (check_heads(B, H_q, H_kv, d) != KVD_OK) return 0;
  int N = 0;
  if (resolve_parts(d, num_partitions, &N) != KVD_OK) return 0;
  const long long slots = static_cast<long long>(N) + static_cast<long long>(B) * H_kv;
  return ws_layout(B, H_q / H_kv, d, slots).total;
}

kvd_status kvd_read_device_error(unsigned int *flags, int clear) {
  if (!flags) return fail(KVD_ERR_INVALID, "flags is NULL");
  int dev;
  unsigned *p;
  kvd_status st = current_device(&dev);
  if (st) return st;
  st = error_word(dev, &p);
  if (st) return st;
  cudaError_t e = cudaMemcpy(flags, p, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (clear) {
    e = cudaMemset(p, 0, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  }
  return KVD_OK;
}

kvd_status kvd_append(void *k_cache, void *v_cache, const int32_t *block_table,
                      const int32_t *slot, const void *k_new, const void *v_new, int B, int H_kv,
                      int d, int num_blocks, int max_blocks_per_seq, kvd_dtype dtype,
                      void *stream) {
  if (B < 0) return fail(KVD_ERR_INVALID, "B = %d < 0", B);
  if (H_kv <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return fail(KVD_ERR_INVALID, "H_kv, num_blocks and max_blocks_per_seq must be positive");
  if (d <= 0 || d % 8 || d > 128) return fail(KVD_ERR_UNSUPPORTED, "head dim %d (need a multiple of 8, <= 128)", d);
  if (dtype != KVD_F16 && dtype != KVD_BF16) return fail(KVD_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (B == 0) return KVD_OK;
  if (!k_cache || !v_cache || !block_table || !slot || !k_new || !v_new)
    return fail(KVD_ERR_INVALID, "a required pointer is NULL");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(KVD_ERR_INVALID, "K/V buffers must be 16-byte aligned");
  if (static_cast<long long>(max_blocks_per_seq) * KVD_PAGE_TOKENS > 0x7fffffffLL)
    return fail(KVD_ERR_UNSUPPORTED, "max_blocks_per_seq too large");
  int dev;
  unsigned *err;
  kvd_status st = current_device(&dev);
  if (st) return st;
  st = error_word(dev, &err);
  if (st) return st;
  kvd::AppendArgs a{k_cache, v_cache, block_table, slot, k_new, v_new, err,
                    B, H_kv, d, num_blocks, max_blocks_per_seq};
  cudaError_t e = kvd::launch_append(a, dtype == KVD_BF16 ? kvd::DType::BF16 : kvd::DType::F16,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return KVD_OK;
}

}  // extern "C"

static kvd_status decode_impl(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_table, const int32_t *seq_lens, float scale,
                              void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                              int max_blocks_per_seq, int num_partitions, void *workspace,
                              size_t workspace_bytes, float *lse_out, kvd_dtype dtype, void *stream,
                              const void *k_new, const void *v_new,
                              const int32_t *group_start = nullptr,
                              const int32_t *group_pages = nullptr, int n_groups = 0,
                              int max_group_size = 0, const float *k_scale = nullptr,
                              const float *v_scale = nullptr, kvd::Code8 fmt = kvd::Code8::E4M3) {
  const bool q8 = k_scale != nullptr;  // 8-bit cache (codes + scales)
  kvd_status st = check_heads(B, H_q, H_kv, d);
  if (st) return st;
  if (num_blocks <= 0 || max_blocks_per_seq <= 0)
    return fail(KVD_ERR_INVALID, "num_blocks and max_blocks_per_seq must be positive");
  if (dtype != KVD_F16 && dtype != KVD_BF16) return fail(KVD_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (static_cast<long long>(num_blocks) * H_kv * KVD_PAGE_TOKENS >= 0x80000000LL)
    return fail(KVD_ERR_UNSUPPORTED, "num_blocks * H_kv * 16 must be < 2^31");
  if (static_cast<long long>(max_blocks_per_seq) * KVD_PAGE_TOKENS > 0x7fffffffLL)
    return fail(KVD_ERR_UNSUPPORTED, "max_blocks_per_seq too large");
  if (!(scale == scale)) return fail(KVD_ERR_INVALID, "scale is NaN");
  if (num_partitions < 0) return fail(KVD_ERR_INVALID, "num_partitions < 0");
  if (q8) {
    if (!v_scale) return fail(KVD_ERR_INVALID, "v_scale is NULL");
    if (!aligned(k_scale, 16) || !aligned(v_scale, 16))
      return fail(KVD_ERR_INVALID, "scale pools must be 16-byte aligned");
  }
  if (B == 0) return KVD_OK;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out)
    return fail(KVD_ERR_INVALID, "a required pointer is NULL");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
    return fail(KVD_ERR_INVALID, "q, caches and out must be 16-byte aligned");
  if (lse_out && !aligned(lse_out, 4)) return fail(KVD_ERR_INVALID, "lse_out misaligned");

  int N = 0;
  st = resolve_parts(d, num_partitions, &N);
  if (st) return st;
  const int G = H_q / H_kv;
  const long long slots = static_cast<long long>(N) + static_cast<long long>(B) * H_kv;
  const WsLayout L0 = ws_layout(B, G, d, slots);
  PrefixLayout PL{};
  if (n_groups > 0) {
    if (!group_start || !group_pages) return fail(KVD_ERR_INVALID, "group_start / group_pages is NULL");
    if (max_group_size <= 0) return fail(KVD_ERR_INVALID, "max_group_size must be positive");
    st = prefix_layout(B, H_kv, G, d, n_groups, max_group_size, L0.total, &PL, q8);
    if (st) return st;
  }
  WsLayout L = L0;
  if (n_groups > 0) L.total = PL.total;
  if (!workspace) return fail(KVD_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", L.total);
  if (!aligned(workspace, 256)) return fail(KVD_ERR_INVALID, "workspace must be 256-byte aligned");
  if (workspace_bytes < L.total)
    return fail(KVD_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);

  int dev;
  unsigned *err;
  st = current_device(&dev);
  if (st) return st;
  st = error_word(dev, &err);
  if (st) return st;
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  st = encoder(&encode);
  if (st) return st;

  CUtensorMap tm[2];
  const void *pools[2] = {k_cache, v_cache};
  for (int i = 0; i < 2; ++i) {
    CUresult r;
    if (q8) {
      // code pools as 2-D byte tensors {row bytes, num_blocks*H_kv*16 rows}
      // (row bytes: d for 8-bit codes, d / 2 for INT4); one box = the 16 rows
      // of one page of one head, with the swizzle of its row size (128, 64
      // or 32 bytes).
      const int rb = fmt == kvd::Code8::INT4 ? d / 2 : d;
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(rb),
                            static_cast<cuuint64_t>(num_blocks) * H_kv * KVD_PAGE_TOKENS};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(rb)};
      cuuint32_t box[2] = {static_cast<cuuint32_t>(rb), KVD_PAGE_TOKENS};
      cuuint32_t estr[2] = {1, 1};
      r = encode(&tm[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(pools[i]), dims,
                 strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                 rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                           : (rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B),
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
      // K and V pools as 3-D tensors {64 elements, d/64 units, num_blocks*H_kv*16
      // rows}; one box = one 64-element half of one page of one head (16 rows x
      // 64), 128-byte swizzled.
      cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(d / 64),
                            static_cast<cuuint64_t>(num_blocks) * H_kv * KVD_PAGE_TOKENS};
      cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(d) * 2};
      cuuint32_t box[3] = {64, 1, KVD_PAGE_TOKENS};
      cuuint32_t estr[3] = {1, 1, 1};
      r = encode(&tm[i],
                 dtype == KVD_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                 3, const_cast<void *>(pools[i]), dims, strides, box, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return fail(KVD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  }

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  kvd::DecodeArgs a{};
  a.q = q;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.out = out;
  a.lse_out = lse_out;
  a.part_o = reinterpret_cast<float *>(ws + L.o);
  a.part_lse = reinterpret_cast<float *>(ws + L.lse);
  a.ws_cum = reinterpret_cast<int32_t *>(ws + L.cum);
  a.err = err;
  a.scale_log2 = scale * kvd::kLog2e;
  a.B = B;
  a.H_q = H_q;
  a.H_kv = H_kv;
  a.G = G;
  a.num_blocks = num_blocks;
  a.maxb = max_blocks_per_seq;
  a.nparts = N;
  a.min_pages = num_partitions > 0 ? 1 : kAutoMinPages;
  // few (sequence, KV head) pairs (long contexts): stream K/V with the
  // evict-first hint, measured faster there; many pairs keep evict-normal
  a.evict_first = static_cast<long long>(B) * H_kv <= kEvictFirstPairs ? 1 : 0;
  {
    const long long wp = g_wait_polls.load(std::memory_order_relaxed);
    a.wait_polls = wp < 0 || wp > kvd::kWaitPolls ? kvd::kWaitPolls : static_cast<uint32_t>(wp);
  }
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_cache = const_cast<void *>(k_cache);
  a.v_cache = const_cast<void *>(v_cache);
  a.skip = nullptr;
  a.pre_o = nullptr;
  a.pre_lse = nullptr;
  a.pre_chunks = 0;
  // the scale pools are written only when k_new is given (the _step calls,
  // which take them writable)
  a.k_scale = const_cast<float *>(k_scale);
  a.v_scale = const_cast<float *>(v_scale);
  a.plan = nullptr;

  const kvd::DType dt = dtype == KVD_BF16 ? kvd::DType::BF16 : kvd::DType::F16;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (n_groups > 0) {
    kvd::PrefixArgs pa{};
    pa.q = q;
    pa.block_table = block_table;
    pa.seq_lens = seq_lens;
    pa.group_start = group_start;
    pa.group_pages = group_pages;
    pa.skip = reinterpret_cast<int32_t *>(ws + PL.skip);
    pa.pre_o = reinterpret_cast<float *>(ws + PL.pre_o);
    pa.pre_lse = reinterpret_cast<float *>(ws + PL.pre_lse);
    pa.err = err;
    pa.scale_log2 = a.scale_log2;
    pa.B = B;
    pa.H_q = H_q;
    pa.H_kv = H_kv;
    pa.G = G;
    pa.num_blocks = num_blocks;
    pa.maxb = max_blocks_per_seq;
    pa.n_groups = n_groups;
    pa.chunks = PL.chunks;
    pa.fused = k_new != nullptr;
    pa.maxg = max_group_size;
    pa.k_scale = k_scale;
    pa.v_scale = v_scale;
    pa.plan = reinterpret_cast<int32_t *>(ws + PL.plan);
    // automatic partitions: the suffix decode leaves the prefix pass its
    // share of the SMs and the two run side by side; a caller's explicit
    // count is kept as given
    kvd::prefix_split(pa, d, q8, fmt, num_partitions == 0);
    pa.nparts = N;
    pa.min_pages = a.min_pages;
    pa.row_blocks = PL.row_blocks;
    a.skip = pa.skip;
    a.pre_o = pa.pre_o;
    a.pre_lse = pa.pre_lse;
    a.pre_chunks = PL.chunks;
    a.plan = pa.plan;
    // plan (skip, partitions) -> suffix decode -> prefix pass, scheduled as
    // the decode starts and run on the SMs it leaves -> merge
    e = kvd::launch_prefix_plan(pa, s);
    if (e != cudaSuccess) return cuda_fail(e, "prefix plan launch");
    e = q8 ? kvd::launch_decode_q8(a, d, dt, fmt, tm[0], tm[1], s, N)
           : kvd::launch_decode(a, d, dt, tm[0], tm[1], s, N);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    e = q8 ? kvd::launch_prefix_q(pa, d, fmt, dt, tm[0], tm[1], PL.row_blocks, s)
           : kvd::launch_prefix(pa, d, dt, tm[0], tm[1], PL.row_blocks, s);
    if (e != cudaSuccess) return cuda_fail(e, "prefix launch");
  } else {
    e = q8 ? kvd::launch_decode_q8(a, d, dt, fmt, tm[0], tm[1], s, N)
           : kvd::launch_decode(a, d, dt, tm[0], tm[1], s, N);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  }
  e = kvd::launch_decode_merge(a, d, dt, s);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return KVD_OK;
}

extern "C" {

kvd_status kvd_decode_attention(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_table, const int32_t *seq_lens, float scale,
                                void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                                int max_blocks_per_seq, int num_partitions, void *workspace,
                                size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                                void *stream) {
  return decode_impl(q, k_cache, v_cache, block_table, seq_lens, scale, out, B, H_q, H_kv, d,
                     num_blocks, max_blocks_per_seq, num_partitions, workspace, workspace_bytes,
                     lse_out, dtype, stream, nullptr, nullptr);
}

static kvd_status quantize_q8(const void *src, uint8_t *codes, float *scales, long long n_rows,
                              int d, kvd_dtype dtype, void *stream, kvd::Code8 fmt) {
  if (n_rows < 0) return fail(KVD_ERR_INVALID, "n_rows < 0");
  if (d <= 0 || d % 32 || d > 128) return fail(KVD_ERR_UNSUPPORTED, "d must be 32, 64, 96 or 128");
  if (dtype != KVD_F16 && dtype != KVD_BF16) return fail(KVD_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (n_rows == 0) return KVD_OK;
  if (!src || !codes || !scales) return fail(KVD_ERR_INVALID, "a required pointer is NULL");
  if (!aligned(src, 8) || !aligned(codes, 4) || !aligned(scales, 4))
    return fail(KVD_ERR_INVALID, "misaligned buffer");
  kvd::QuantArgs q{src, codes, scales, nullptr, nullptr, nullptr, n_rows, d, 1, 1, 1, 0};
  cudaError_t e = kvd::launch_quantize_q8(q, dtype == KVD_BF16 ? kvd::DType::BF16 : kvd::DType::F16,
                                          fmt, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return KVD_OK;
}

static kvd_status append_q8(uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                            const int32_t *block_table, const int32_t *slot, const void *k_new,
                            const void *v_new, int B, int H_kv, int d, int num_blocks,
                            int max_blocks_per_seq, kvd_dtype dtype, void *stream, kvd::Code8 fmt) {
  if (B < 0) return fail(KVD_ERR_INVALID, "B = %d < 0", B);
  if (H_kv <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return fail(KVD_ERR_INVALID, "H_kv, num_blocks and max_blocks_per_seq must be positive");
  if (d <= 0 || d % 32 || d > 128) return fail(KVD_ERR_UNSUPPORTED, "d must be 32, 64, 96 or 128");
  if (dtype != KVD_F16 && dtype != KVD_BF16) return fail(KVD_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (B == 0) return KVD_OK;
  if (!k_codes || !v_codes || !k_scale || !v_scale || !block_table || !slot || !k_new || !v_new)
    return fail(KVD_ERR_INVALID, "a required pointer is NULL");
  if (!aligned(k_new, 8) || !aligned(v_new, 8) || !aligned(k_codes, 4) || !aligned(v_codes, 4) ||
      !aligned(k_scale, 4) || !aligned(v_scale, 4))
    return fail(KVD_ERR_INVALID, "misaligned buffer");
  int dev;
  unsigned *err;
  kvd_status st = current_device(&dev);
  if (st) return st;
  st = error_word(dev, &err);
  if (st) return st;
  const kvd::DType dt = dtype == KVD_BF16 ? kvd::DType::BF16 : kvd::DType::F16;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long n = static_cast<long long>(B) * H_kv;
  kvd::QuantArgs qa{k_new, k_codes, k_scale, block_table, slot, err, n, d, H_kv, num_blocks,
                    max_blocks_per_seq, 1, v_new, v_codes, v_scale};
  cudaError_t e = kvd::launch_quantize_q8(qa, dt, fmt, s);
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return KVD_OK;
}

static kvd_status decode_q8(const void *q, const uint8_t *k_codes, const uint8_t *v_codes,
                            const float *k_scale, const float *v_scale, const int32_t *block_table,
                            const int32_t *seq_lens, float scale, void *out, int B, int H_q, int H_kv,
                            int d, int num_blocks, int max_blocks_per_seq, int num_partitions,
                            void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                            void *stream, kvd::Code8 fmt, const void *k_new = nullptr,
                            const void *v_new = nullptr) {
  if (!k_scale) return fail(KVD_ERR_INVALID, "k_scale is NULL");
  return decode_impl(q, k_codes, v_codes, block_table, seq_lens, scale, out, B, H_q, H_kv, d,
                     num_blocks, max_blocks_per_seq, num_partitions, workspace, workspace_bytes,
                     lse_out, dtype, stream, k_new, v_new, nullptr, nullptr, 0, 0, k_scale,
                     v_scale, fmt);
}

// The fused step over an 8-bit cache: kvd_append_{fp8,int8} (slot =
// seq_lens - 1) and kvd_decode_attention_{fp8,int8} in one decode launch.
static kvd_status step_q8(const void *q, const void *k_new, const void *v_new, uint8_t *k_codes,
                          uint8_t *v_codes, float *k_scale, float *v_scale,
                          const int32_t *block_table, const int32_t *seq_lens, float scale,
                          void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                          int max_blocks_per_seq, int num_partitions, void *workspace,
                          size_t workspace_bytes, float *lse_out, kvd_dtype dtype, void *stream,
                          kvd::Code8 fmt) {
  if (B > 0) {
    if (!k_new || !v_new) return fail(KVD_ERR_INVALID, "k_new / v_new is NULL");
    if (!aligned(k_new, 16) || !aligned(v_new, 16))
      return fail(KVD_ERR_INVALID, "k_new / v_new must be 16-byte aligned");
  }
  return decode_q8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out, B, H_q,
                   H_kv, d, num_blocks, max_blocks_per_seq, num_partitions, workspace,
                   workspace_bytes, lse_out, dtype, stream, fmt, B > 0 ? k_new : nullptr,
                   B > 0 ? v_new : nullptr);
}

kvd_status kvd_quantize_fp8(const void *src, uint8_t *codes, float *scales, long long n_rows,
                            int d, kvd_dtype dtype, void *stream) {
  return quantize_q8(src, codes, scales, n_rows, d, dtype, stream, kvd::Code8::E4M3);
}

kvd_status kvd_append_fp8(uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                          const int32_t *block_table, const int32_t *slot, const void *k_new,
                          const void *v_new, int B, int H_kv, int d, int num_blocks,
                          int max_blocks_per_seq, kvd_dtype dtype, void *stream) {
  return append_q8(k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, B, H_kv, d,
                   num_blocks, max_blocks_per_seq, dtype, stream, kvd::Code8::E4M3);
}

kvd_status kvd_decode_attention_fp8(const void *q, const uint8_t *k_codes, const uint8_t *v_codes,
                                    const float *k_scale, const float *v_scale,
                                    const int32_t *block_table, const int32_t *seq_lens,
                                    float scale, void *out, int B, int H_q, int H_kv, int d,
                                    int num_blocks, int max_blocks_per_seq, int num_partitions,
                                    void *workspace, size_t workspace_bytes, float *lse_out,
                                    kvd_dtype dtype, void *stream) {
  return decode_q8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out, B, H_q,
                   H_kv, d, num_blocks, max_blocks_per_seq, num_partitions, workspace,
                   workspace_bytes, lse_out, dtype, stream, kvd::Code8::E4M3);
}

kvd_status kvd_decode_step_fp8(const void *q, const void *k_new, const void *v_new,
                               uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                               const int32_t *block_table, const int32_t *seq_lens, float scale,
                               void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                               int max_blocks_per_seq, int num_partitions, void *workspace,
                               size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                               void *stream) {
  return step_q8(q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale,
                 out, B, H_q, H_kv, d, num_blocks, max_blocks_per_seq, num_partitions, workspace,
                 workspace_bytes, lse_out, dtype, stream, kvd::Code8::E4M3);
}

kvd_status kvd_quantize_int8(const void *src, int8_t *codes, float *scales, long long n_rows,
                             int d, kvd_dtype dtype, void *stream) {
  return quantize_q8(src, reinterpret_cast<uint8_t *>(codes), scales, n_rows, d, dtype, stream,
                     kvd::Code8::INT8);
}

kvd_status kvd_append_int8(int8_t *k_codes, int8_t *v_codes, float *k_scale, float *v_scale,
                           const int32_t *block_table, const int32_t *slot, const void *k_new,
                           const void *v_new, int B, int H_kv, int d, int num_blocks,
                           int max_blocks_per_seq, kvd_dtype dtype, void *stream) {
  return append_q8(reinterpret_cast<uint8_t *>(k_codes), reinterpret_cast<uint8_t *>(v_codes),
                   k_scale, v_scale, block_table, slot, k_new, v_new, B, H_kv, d, num_blocks,
                   max_blocks_per_seq, dtype, stream, kvd::Code8::INT8);
}

kvd_status kvd_decode_attention_int8(const void *q, const int8_t *k_codes, const int8_t *v_codes,
                                     const float *k_scale, const float *v_scale,
                                     const int32_t *block_table, const int32_t *seq_lens,
                                     float scale, void *out, int B, int H_q, int H_kv, int d,
                                     int num_blocks, int max_blocks_per_seq, int num_partitions,
                                     void *workspace, size_t workspace_bytes, float *lse_out,
                                     kvd_dtype dtype, void *stream) {
  return decode_q8(q, reinterpret_cast<const uint8_t *>(k_codes),
                   reinterpret_cast<const uint8_t *>(v_codes), k_scale, v_scale, block_table,
                   seq_lens, scale, out, B, H_q, H_kv, d, num_blocks, max_blocks_per_seq,
                   num_partitions, workspace, workspace_bytes, lse_out, dtype, stream,
                   kvd::Code8::INT8);
}

kvd_status kvd_decode_step_int8(const void *q, const void *k_new, const void *v_new,
                                int8_t *k_codes, int8_t *v_codes, float *k_scale, float *v_scale,
                                const int32_t *block_table, const int32_t *seq_lens, float scale,
                                void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                                int max_blocks_per_seq, int num_partitions, void *workspace,
                                size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                                void *stream) {
  return step_q8(q, k_new, v_new, reinterpret_cast<uint8_t *>(k_codes),
                 reinterpret_cast<uint8_t *>(v_codes), k_scale, v_scale, block_table, seq_lens,
                 scale, out, B, H_q, H_kv, d, num_blocks, max_blocks_per_seq, num_partitions,
                 workspace, workspace_bytes, lse_out, dtype, stream, kvd::Code8::INT8);
}

kvd_status kvd_quantize_int4(const void *src, uint8_t *codes, float *scales, long long n_rows,
                             int d, kvd_dtype dtype, void *stream) {
  return quantize_q8(src, codes, scales, n_rows, d, dtype, stream, kvd::Code8::INT4);
}

kvd_status kvd_append_int4(uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                           const int32_t *block_table, const int32_t *slot, const void *k_new,
                           const void *v_new, int B, int H_kv, int d, int num_blocks,
                           int max_blocks_per_seq, kvd_dtype dtype, void *stream) {
  return append_q8(k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, B, H_kv, d,
                   num_blocks, max_blocks_per_seq, dtype, stream, kvd::Code8::INT4);
}

kvd_status kvd_decode_attention_int4(const void *q, const uint8_t *k_codes, const uint8_t *v_codes,
                                     const float *k_scale, const float *v_scale,
                                     const int32_t *block_table, const int32_t *seq_lens,
                                     float scale, void *out, int B, int H_q, int H_kv, int d,
                                     int num_blocks, int max_blocks_per_seq, int num_partitions,
                                     void *workspace, size_t workspace_bytes, float *lse_out,
                                     kvd_dtype dtype, void *stream) {
  return decode_q8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out, B, H_q,
                   H_kv, d, num_blocks, max_blocks_per_seq, num_partitions, workspace,
                   workspace_bytes, lse_out, dtype, stream, kvd::Code8::INT4);
}

kvd_status kvd_decode_step_int4(const void *q, const void *k_new, const void *v_new,
                                uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                                const int32_t *block_table, const int32_t *seq_lens, float scale,
                                void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                                int max_blocks_per_seq, int num_partitions, void *workspace,
                                size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
                                void *stream) {
  return step_q8(q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale,
                 out, B, H_q, H_kv, d, num_blocks, max_blocks_per_seq, num_partitions, workspace,
                 workspace_bytes, lse_out, dtype, stream, kvd::Code8::INT4);
}

size_t kvd_shared_prefix_workspace_size(int B, int H_q, int H_kv, int d, int n_groups,
                                        int max_group_size, int num_partitions) {
  if (check_heads(B, H_q, H_kv, d) != KVD_OK) return 0;
  if (n_groups < 0 || max_group_size <= 0) {
    fail(KVD_ERR_INVALID, "n_groups >= 0 and max_group_size > 0 required");
    return 0;
  }
  int N = 0;
  if (resolve_parts(d, num_partitions, &N) != KVD_OK) return 0;
  const long long slots = static_cast<long long>(N) + static_cast<long long>(B) * H_kv;
  const WsLayout L0 = ws_layout(B, H_q / H_kv, d, slots);
  if (n_groups == 0) return L0.total;
  // the larger of the fp16 / bf16 and the quantised layouts, so that one
  // size serves every shared-prefix call
  PrefixLayout PL, PQ;
  if (prefix_layout(B, H_kv, H_q / H_kv, d, n_groups, max_group_size, L0.total, &PL) != KVD_OK ||
      prefix_layout(B, H_kv, H_q / H_kv, d, n_groups, max_group_size, L0.total, &PQ, true) != KVD_OK)
    return 0;
  return PL.total > PQ.total ? PL.total : PQ.total;
}

kvd_status kvd_decode_attention_shared_prefix(
    const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
    const int32_t *block_table, const int32_t *seq_lens, float scale, void *out, int B, int H_q,
    int H_kv, int d, int num_blocks, int max_blocks_per_seq, const int32_t *group_start,
    const int32_t *group_pages, int n_groups, int max_group_size, int num_partitions,
    void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype, void *stream) {
  if (n_groups < 0) return fail(KVD_ERR_INVALID, "n_groups < 0");
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(KVD_ERR_INVALID, "k_new and v_new must both be given or both be NULL");
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16)))
    return fail(KVD_ERR_INVALID, "k_new / v_new must be 16-byte aligned");
  return decode_impl(q, k_cache, v_cache, block_table, seq_lens, scale, out, B, H_q, H_kv, d,
                     num_blocks, max_blocks_per_seq, num_partitions, workspace, workspace_bytes,
                     lse_out, dtype, stream, k_new, v_new, group_start, group_pages, n_groups,
                     max_group_size);
}

// The shared-prefix decode over a quantised cache (d = 128): the prefix pass
// dequantises each staged page once for the whole group (prefix_tcq_kernel).
static kvd_status shared_prefix_q(const void *q, const void *k_new, const void *v_new,
                                  uint8_t *k_codes, uint8_t *v_codes, float *k_scale, float *v_scale,
                                  const int32_t *block_table, const int32_t *seq_lens, float scale,
                                  void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                                  int max_blocks_per_seq, const int32_t *group_start,
                                  const int32_t *group_pages, int n_groups, int max_group_size,
                                  int num_partitions, void *workspace, size_t workspace_bytes,
                                  float *lse_out, kvd_dtype dtype, void *stream, kvd::Code8 fmt) {
  if (n_groups < 0) return fail(KVD_ERR_INVALID, "n_groups < 0");
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(KVD_ERR_INVALID, "k_new and v_new must both be given or both be NULL");
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16)))
    return fail(KVD_ERR_INVALID, "k_new / v_new must be 16-byte aligned");
  if (!k_scale) return fail(KVD_ERR_INVALID, "k_scale is NULL");
  return decode_impl(q, k_codes, v_codes, block_table, seq_lens, scale, out, B, H_q, H_kv, d,
                     num_blocks, max_blocks_per_seq, num_partitions, workspace, workspace_bytes,
                     lse_out, dtype, stream, k_new, v_new, group_start, group_pages, n_groups,
                     max_group_size, k_scale, v_scale, fmt);
}

kvd_status kvd_decode_attention_shared_prefix_fp8(
    const void *q, const void *k_new, const void *v_new, uint8_t *k_codes, uint8_t *v_codes,
    float *k_scale, float *v_scale, const int32_t *block_table, const int32_t *seq_lens, float scale,
    void *out, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks_per_seq,
    const int32_t *group_start, const int32_t *group_pages, int n_groups, int max_group_size,
    int num_partitions, void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
    void *stream) {
  return shared_prefix_q(q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                         scale, out, B, H_q, H_kv, d, num_blocks, max_blocks_per_seq, group_start,
                         group_pages, n_groups, max_group_size, num_partitions, workspace,
                         workspace_bytes, lse_out, dtype, stream, kvd::Code8::E4M3);
}

kvd_status kvd_decode_attention_shared_prefix_int8(
    const void *q, const void *k_new, const void *v_new, int8_t *k_codes, int8_t *v_codes,
    float *k_scale, float *v_scale, const int32_t *block_table, const int32_t *seq_lens, float scale,
    void *out, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks_per_seq,
    const int32_t *group_start, const int32_t *group_pages, int n_groups, int max_group_size,
    int num_partitions, void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
    void *stream) {
  return shared_prefix_q(q, k_new, v_new, reinterpret_cast<uint8_t *>(k_codes),
                         reinterpret_cast<uint8_t *>(v_codes), k_scale, v_scale, block_table,
                         seq_lens, scale, out, B, H_q, H_kv, d, num_blocks, max_blocks_per_seq,
                         group_start, group_pages, n_groups, max_group_size, num_partitions,
                         workspace, workspace_bytes, lse_out, dtype, stream, kvd::Code8::INT8);
}

kvd_status kvd_decode_attention_shared_prefix_int4(
    const void *q, const void *k_new, const void *v_new, uint8_t *k_codes, uint8_t *v_codes,
    float *k_scale, float *v_scale, const int32_t *block_table, const int32_t *seq_lens, float scale,
    void *out, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks_per_seq,
    const int32_t *group_start, const int32_t *group_pages, int n_groups, int max_group_size,
    int num_partitions, void *workspace, size_t workspace_bytes, float *lse_out, kvd_dtype dtype,
    void *stream) {
  return shared_prefix_q(q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                         scale, out, B, H_q, H_kv, d, num_blocks, max_blocks_per_seq, group_start,
                         group_pages, n_groups, max_group_size, num_partitions, workspace,
                         workspace_bytes, lse_out, dtype, stream, kvd::Code8::INT4);
}

kvd_status kvd_decode_step(const void *q, const void *k_new, const void *v_new, void *k_cache,
                           void *v_cache, const int32_t *block_table, const int32_t *seq_lens,
                           float scale, void *out, int B, int H_q, int H_kv, int d, int num_blocks,
                           int max_blocks_per_seq, int num_partitions, void *workspace,
                           size_t workspace_bytes, float *lse_out, kvd_dtype dtype, void *stream) {
  if (B > 0) {
    if (!k_new || !v_new) return fail(KVD_ERR_INVALID, "k_new / v_new is NULL");
    if (!aligned(k_new, 16) || !aligned(v_new, 16))
      return fail(KVD_ERR_INVALID, "k_new / v_new must be 16-byte aligned");
  }
  return decode_impl(q, k_cache, v_cache, block_table, seq_lens, scale, out, B, H_q, H_kv, d,
                     num_blocks, max_blocks_per_seq, num_partitions, workspace, workspace_bytes,
                     lse_out, dtype, stream, k_new, v_new);
}

kvd_status kvd_read_stream(const void *src, size_t bytes, int mode, uint32_t *sink, void *stream) {
  if (mode != KVD_READ_VECTOR && mode != KVD_READ_BULK)
    return fail(KVD_ERR_INVALID, "unknown read mode %d", mode);
  if (bytes % 16) return fail(KVD_ERR_INVALID, "bytes = %zu is not a multiple of 16", bytes);
  if (bytes == 0) return KVD_OK;
  if (!src || !sink) return fail(KVD_ERR_INVALID, "a required pointer is NULL");
  if (!aligned(src, 16) || !aligned(sink, 4)) return fail(KVD_ERR_INVALID, "misaligned buffer");
  int dev, sms;
  unsigned *err;
  kvd_status st = current_device(&dev);
  if (st) return st;
  st = sm_count(dev, &sms);
  if (st) return st;
  st = error_word(dev, &err);
  if (st) return st;
  cudaError_t e = kvd::launch_read_stream(src, bytes, mode, sink, err, sms,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "read-stream launch");
  return KVD_OK;
}

kvd_status kvd_merge_lse(const float *part_o, const float *part_lse,
                         const int32_t *num_splits_per_seq, int B, int H_q, int d, int S,
                         void *out, float *lse_out, kvd_dtype dtype, void *stream) {
  if (B < 0 || H_q <= 0 || S <= 0) return fail(KVD_ERR_INVALID, "need B >= 0, H_q > 0, S > 0");
  if (d != 64 && d != 128) return fail(KVD_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
  if (dtype != KVD_F16 && dtype != KVD_BF16) return fail(KVD_ERR_INVALID, "unknown dtype %d", (int)dtype);
  if (static_cast<long long>(B) * H_q > 0x7fffffffLL) return fail(KVD_ERR_UNSUPPORTED, "B * H_q too large");
  if (B == 0) return KVD_OK;
  if (!part_o || !part_lse || !out) return fail(KVD_ERR_INVALID, "a required pointer is NULL");
  if (!aligned(part_o, 16) || !aligned(part_lse, 4) || !aligned(out, 2))
    return fail(KVD_ERR_INVALID, "misaligned buffer");
  kvd::GenericMergeArgs a{part_o, part_lse, num_splits_per_seq, out, lse_out, B, H_q, d, S};
  cudaError_t e = kvd::launch_generic_merge(a, dtype == KVD_BF16 ? kvd::DType::BF16 : kvd::DType::F16,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return KVD_OK;
}

}  // extern "C"

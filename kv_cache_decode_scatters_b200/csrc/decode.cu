// decode.cu -- paged decode attention for sm_100a.
//
// What it computes ("推理速度慢怎么办？KV Cache与Flash Attention如何加速大模型推理",
// section 一、KV Cache; "KV缓存与Flash注意力", sections "Flash Attention — 分块技巧"
// and "步骤2:分块softmax"; "KV Cache:推理慢的真正原因", sections PagedAttention and
// GQA): for every sequence b and query head hq, out = softmax(scale * q K^T) V
// over the sequence's cached tokens, read through the block table, with query
// head hq using KV head hq / G.  Scores never leave registers: each 16-token
// page updates a running (max, sum, output) state.
//
// How it is laid out on the B200:
//  * Work split (stream-K).  The pages of all (sequence, KV head) pairs,
//    concatenated, form one list of P pages; it is cut into N equal
//    contiguous partitions, one per CTA (N = SM count by default), and each
//    CTA's partition into equal contiguous shares, one per worker warp.  Every
//    warp streams the same number of pages whatever the sequence lengths are,
//    and warps never synchronise while streaming.
//  * A pair inside one warp's share is written straight to `out`.  A pair
//    several warps of the CTA hold pieces of is combined once, at the end, in
//    shared memory (each piece parks its unnormalised accumulators, row max
//    and row sum).  A pair that crosses CTA partitions leaves one normalised
//    partial (o, lse) per CTA at slot (CTA + pair), and the merge kernel
//    combines those.
//  * Each worker warp owns an S-stage ring in shared memory.  Lane 0 issues
//    TMA tile loads for each page (K and V, each as d/64 boxes of 16 x 64
//    elements with the 128-byte swizzle) that complete on the stage's
//    mbarrier; the whole warp waits, computes, and hands the stage back to
//    the next page.  Latency is hidden by many warps (12-16 per SM, one
//    or two stages each; 7 with two stages where the pairs fit one per
//    warp) rather than by deep per-warp rings.
//  * Every KV byte is read once per GQA group: the G query rows of a KV head
//    ride along as the N dimension of the tensor-core tile.  Per page,
//    S^T[16 tokens x 8 rows] = K[16 x d] . Q^T uses mma.m16n8k16 with the K
//    page as the A operand (ldmatrix from the swizzled stage); the
//    probabilities are transposed in registers (movmatrix) into the B
//    operand of O^T[d x 8] += V^T[d x 16] . P^T[16 x 8] (ldmatrix.trans).
//    G <= 8 uses one n-tile, G <= 16 two.
//  * Softmax in base 2: scores are scaled by scale * log2(e) in fp32 and
//    exponentiated with ex2.approx.  The running maximum is a reference that
//    moves (with a rescale) only when a page's scores pass it by more than
//    2^8, so most pages skip the cross-lane maximum.  For fp16 the probabilities are rounded
//    once for the PV product and the running sum uses the same rounded
//    values; for bf16 (8 significant bits) each probability is carried as a
//    rounded head plus a rounded remainder in two PV products.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"
#include "tile.cuh"

namespace kvd {

namespace {

template <int D, int NT, int W, int S, int kStride, int kAux>
struct Geo {
  static constexpr int kStageBytes = kStride;           // smem stride of one ring stage
  static constexpr int kAuxBytes = kAux;                // per-stage side data (scales), own area
  static constexpr int kThreads = 32 * W;
  static constexpr int kSteps = D / 16;                 // k-steps of S, m-tiles of O
  static constexpr int kEdgeFloats = 8 * NT * D;        // one parked accumulator tile
  // one 8-byte mbarrier per stage, padded so that the 16-byte page
  // descriptors after them stay aligned whatever W * S is
  static constexpr int kBarBytes = (W * S * 8 + 15) / 16 * 16;
  static_assert(kEdgeFloats * 4 <= S * kStageBytes, "a parked tile must fit in a warp's ring");
  static_assert(kStageBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
  static_assert(kAux % 16 == 0, "side data must keep the barriers and descriptors aligned");
  static size_t smem(int B) {
    return 1024 + (size_t)W * S * kStageBytes + (size_t)W * kEdgeFloats * 4 + (size_t)W * S * kAux +
           kBarBytes + (size_t)W * S * 16 +
           (size_t)W * 2 * 2 * 8 * NT * 4 + (size_t)W * 2 * 4 + (size_t)(B + 1) * 4;
  }
};

// Partitions a launch over P pages uses: the automatic bound, capped in a
// shared-prefix call by its plan, which leaves the other SMs to the prefix
// pass running beside the decode.  The merge derives the same count.
__device__ __forceinline__ int used_parts(const DecodeArgs &a, long long P) {
  const int N = effective_parts(P, a.nparts, a.min_pages);
  return a.plan ? min(N, max(1, __ldcg(a.plan))) : N;
}

}  // namespace

// ---------------------------------------------------------- page formats
//
// What the decode kernel needs to know about a page format: how to copy a
// page of one KV head into a ring stage, how to clear the rows past the
// sequence end, the tensor-core step over a staged page, how q feeds it, and
// which output channel each accumulator element holds.

// fp16 / bf16 pages: [16 tokens][d] per (page, head), d/64 swizzled boxes.
template <int D, int NT, typename T>
struct Page16 {
  using Out = T;
  static constexpr bool kPackG1 = false;  // one query row with groups in N (PackedG1)
  static constexpr int kPageBytes = kPage * D * 2;
  static constexpr int kCopyBytes = 2 * kPageBytes;
  static constexpr int kStride = kCopyBytes;
  static constexpr int kAuxBytes = 0;
  static __device__ __forceinline__ void issue(uint32_t dst, uint32_t, uint32_t bar,
                                               const CUtensorMap *tmK, const CUtensorMap *tmV,
                                               int row, uint64_t policy, const DecodeArgs &) {
    mbar_arrive_expect_tx(bar, kCopyBytes);
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf) {
      tma_load_3d(dst + hf * kPage * 128, tmK, 0, hf, row, bar, policy);
      tma_load_3d(dst + kPageBytes + hf * kPage * 128, tmV, 0, hf, row, bar, policy);
    }
  }
  static __device__ __forceinline__ void zero_tail(uint8_t *st, uint8_t *, int ntok, int lane) {
    const int n16 = (kPage - ntok) * 128 / 16;  // 16-byte chunks per half
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf) {
      uint4 *z = reinterpret_cast<uint4 *>(st + kPageBytes + hf * kPage * 128 + ntok * 128);
      for (int i = lane; i < n16; i += 32) z[i] = make_uint4(0, 0, 0, 0);
    }
  }
  // fused append: put the new token of pair (b, h) into row t of the staged
  // page and write it to the cache at pool row `row` + t
  static __device__ __forceinline__ void patch(uint8_t *st, uint8_t *, int t, int lane,
                                               const DecodeArgs &a, int b, int h, int row) {
    const int half = lane >> 4, ch = lane & 15;
    if (ch < D / 8) {
      const size_t src = (static_cast<size_t>(b) * a.H_kv + h) * D;
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(
                                static_cast<const uint16_t *>(half ? a.v_new : a.k_new) + src) + ch);
      *reinterpret_cast<uint4 *>(st + (half ? kPageBytes : 0) + swz<D>(t, ch * 8)) = v;
      const size_t dst = (static_cast<size_t>(row) + t) * D;
      *(reinterpret_cast<uint4 *>(static_cast<uint16_t *>(half ? a.v_cache : a.k_cache) + dst) + ch) = v;
    }
  }
  static __device__ __forceinline__ void tile(uint8_t *st, uint8_t *, int ntok, float sl2, int lane,
                                              const uint32_t (&qf)[NT][D / 16][2],
                                              float (&acc)[NT][D / 16][4], float (&m)[NT][2],
                                              float (&l)[NT][2]) {
    tile_page<D, NT, T>(smem_u32(st), smem_u32(st + kPageBytes), ntok, sl2, lane, qf, acc, m, l);
  }
  static __device__ __forceinline__ void q_words(const uint32_t *qrow, int ks, int tig,
                                                 uint32_t &w0, uint32_t &w1) {
    w0 = __ldg(qrow + ks * 8 + tig);
    w1 = __ldg(qrow + ks * 8 + 4 + tig);
  }
  static __device__ __forceinline__ int dim(int mt, int e, int g8) {
    return mt * 16 + g8 + ((e >> 1) << 3);
  }
};

// 8-bit pages (d = D = 64 or 128; E4M3 or INT8 codes): codes [16][D] per
// (page, head) in one box with the 128-byte (D = 128) or 64-byte (D = 64)
// swizzle, fp32 scales [16][D / 32] per (page, head) copied alongside;
// output dtype T.
template <int D, int NT, typename T, Code8 kFmt>
struct Page8 {
  using Out = T;
  static constexpr bool kPackG1 = false;  // one query row with groups in N (PackedG1)
  static constexpr int kG = D / 32;                          // scale groups of a token
  static constexpr int kPageBytes = kPage * D;               // codes of K (or V)
  static constexpr int kScaleBytes = kPage * kG * 4;         // scales of K (or V)
  static constexpr int kCopyBytes = 2 * kPageBytes + 2 * kScaleBytes;
  static constexpr int kStride = 2 * kPageBytes;             // codes only: 1024-aligned stages
  static constexpr int kAuxBytes = 2 * kScaleBytes;          // scales, in their own area
  static_assert(kScaleBytes % 16 == 0, "scale rows are bulk copies of whole 16-byte units");
  static __device__ __forceinline__ void issue(uint32_t dst, uint32_t aux, uint32_t bar,
                                               const CUtensorMap *tmK, const CUtensorMap *tmV,
                                               int row, uint64_t policy, const DecodeArgs &a) {
    mbar_arrive_expect_tx(bar, kCopyBytes);
    tma_load_2d(dst, tmK, 0, row, bar, policy);
    tma_load_2d(dst + kPageBytes, tmV, 0, row, bar, policy);
    bulk_load(aux, a.k_scale + static_cast<size_t>(row) * kG, kScaleBytes, bar);
    bulk_load(aux + kScaleBytes, a.v_scale + static_cast<size_t>(row) * kG, kScaleBytes, bar);
  }
  static __device__ __forceinline__ void zero_tail(uint8_t *st, uint8_t *aux, int ntok, int lane) {
    // V codes and V scales of masked rows (their zero weights times a NaN
    // scale would otherwise poison the PV product)
    const int n16 = (kPage - ntok) * D / 16;
    uint4 *z = reinterpret_cast<uint4 *>(st + kPageBytes + ntok * D);
    for (int i = lane; i < n16; i += 32) z[i] = make_uint4(0, 0, 0, 0);
    float *zs = reinterpret_cast<float *>(aux + kScaleBytes) + ntok * kG;
    for (int i = lane; i < (kPage - ntok) * kG; i += 32) zs[i] = 0.f;
  }
  // fused append: encode the new token of pair (b, h) exactly as the
  // quantising append does (encode_row4), put its codes and scales into row t
  // of the staged page and write them to the pools at row `row` + t
  static __device__ __forceinline__ void patch(uint8_t *st, uint8_t *aux, int t, int lane,
                                               const DecodeArgs &a, int b, int h, int row) {
    const size_t src = (static_cast<size_t>(b) * a.H_kv + h) * D;
    const size_t dst = static_cast<size_t>(row) + t;
    const bool live = lane * 4 < D;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float sc;
      const uint32_t w =
          encode_row4<T, kFmt>(static_cast<const T *>(half ? a.v_new : a.k_new) + src, live, lane, sc);
      if (live) {
        *reinterpret_cast<uint32_t *>(st + half * kPageBytes + swz_rows<D>(t, lane >> 2) +
                                      (lane & 3) * 4) = w;
        *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(half ? a.v_cache : a.k_cache) + dst * D +
                                      lane * 4) = w;
        if ((lane & 7) == 0) {
          reinterpret_cast<float *>(aux + half * kScaleBytes)[t * kG + (lane >> 3)] = sc;
          (half ? a.v_scale : a.k_scale)[dst * kG + (lane >> 3)] = sc;
        }
      }
    }
  }
  static __device__ __forceinline__ void tile(uint8_t *st, uint8_t *aux, int ntok, float sl2, int lane,
                                              const uint32_t (&qf)[NT][D / 16][2],
                                              float (&acc)[NT][D / 16][4], float (&m)[NT][2],
                                              float (&l)[NT][2]) {
    const float *ks = reinterpret_cast<const float *>(aux);
    tile_page_q8<D, NT, kFmt>(smem_u32(st), smem_u32(st + kPageBytes), ks, ks + kPage * kG, ntok, sl2,
                              lane, qf, acc, m, l);
  }
  // q in f16, channel order of the 8-bit tile: k-slots 2t, 2t+1 <- channels
  // 4t, 4t+1 and k-slots 2t+8, 2t+9 <- channels 4t+2, 4t+3 of each 16
  static __device__ __forceinline__ void q_words(const uint32_t *qrow, int ks, int tig,
                                                 uint32_t &w0, uint32_t &w1) {
    q_words_q8<T>(qrow, ks, tig, w0, w1);
  }
  static __device__ __forceinline__ int dim(int mt, int e, int g8) { return dim_q8(mt, e, g8); }
};

// 4-bit pages (d = D = 64 or 128; INT4 codes, two per byte): codes
// [16][D / 2] per (page, head) in one box with the 64-byte (D = 128) or
// 32-byte (D = 64) swizzle, fp32 scales [16][D / 32] per (page, head) copied
// alongside; output dtype T.
template <int D, int NT, typename T>
struct Page4 {
  using Out = T;
  static constexpr bool kPackG1 = false;  // one query row with groups in N (PackedG1)
  static constexpr int kG = D / 32;                          // scale groups of a token
  static constexpr int kRow = D / 2;                         // code bytes of a token
  static constexpr int kPageBytes = kPage * kRow;            // codes of K (or V)
  static constexpr int kScaleBytes = kPage * kG * 4;         // scales of K (or V)
  static constexpr int kCopyBytes = 2 * kPageBytes + 2 * kScaleBytes;
  static constexpr int kStride = 2 * kPageBytes;             // codes only: 1024-aligned stages
  static constexpr int kAuxBytes = 2 * kScaleBytes;          // scales, in their own area
  static_assert(kScaleBytes % 16 == 0, "scale rows are bulk copies of whole 16-byte units");
  static __device__ __forceinline__ void issue(uint32_t dst, uint32_t aux, uint32_t bar,
                                               const CUtensorMap *tmK, const CUtensorMap *tmV,
                                               int row, uint64_t policy, const DecodeArgs &a) {
    mbar_arrive_expect_tx(bar, kCopyBytes);
    tma_load_2d(dst, tmK, 0, row, bar, policy);
    tma_load_2d(dst + kPageBytes, tmV, 0, row, bar, policy);
    bulk_load(aux, a.k_scale + static_cast<size_t>(row) * kG, kScaleBytes, bar);
    bulk_load(aux + kScaleBytes, a.v_scale + static_cast<size_t>(row) * kG, kScaleBytes, bar);
  }
  static __device__ __forceinline__ void zero_tail(uint8_t *st, uint8_t *aux, int ntok, int lane) {
    // V codes and V scales of masked rows (their zero weights times a NaN
    // scale would otherwise poison the PV product)
    const int n16 = (kPage - ntok) * kRow / 16;
    uint4 *z = reinterpret_cast<uint4 *>(st + kPageBytes + ntok * kRow);
    for (int i = lane; i < n16; i += 32) z[i] = make_uint4(0, 0, 0, 0);
    float *zs = reinterpret_cast<float *>(aux + kScaleBytes) + ntok * kG;
    for (int i = lane; i < (kPage - ntok) * kG; i += 32) zs[i] = 0.f;
  }
  // fused append: encode the new token of pair (b, h) exactly as the
  // quantising append does (encode_row4), put its codes and scales into row t
  // of the staged page and write them to the pools at row `row` + t
  static __device__ __forceinline__ void patch(uint8_t *st, uint8_t *aux, int t, int lane,
                                               const DecodeArgs &a, int b, int h, int row) {
    const size_t src = (static_cast<size_t>(b) * a.H_kv + h) * D;
    const size_t dst = static_cast<size_t>(row) + t;
    const bool live = lane * 4 < D;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float sc;
      const uint32_t w = encode_row4<T, Code8::INT4>(static_cast<const T *>(half ? a.v_new : a.k_new) + src,
                                                     live, lane, sc);
      if (live) {
        // the lane's 4 codes are bytes 2 lane, 2 lane + 1 of the row
        *reinterpret_cast<uint16_t *>(st + half * kPageBytes + swz_rows<kRow>(t, (2 * lane) >> 4) +
                                      ((2 * lane) & 15)) = static_cast<uint16_t>(w);
        *reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(half ? a.v_cache : a.k_cache) + dst * kRow +
                                      2 * lane) = static_cast<uint16_t>(w);
        if ((lane & 7) == 0) {
          reinterpret_cast<float *>(aux + half * kScaleBytes)[t * kG + (lane >> 3)] = sc;
          (half ? a.v_scale : a.k_scale)[dst * kG + (lane >> 3)] = sc;
        }
      }
    }
  }
  static __device__ __forceinline__ void tile(uint8_t *st, uint8_t *aux, int ntok, float sl2, int lane,
                                              const uint32_t (&qf)[NT][D / 16][2],
                                              float (&acc)[NT][D / 16][4], float (&m)[NT][2],
                                              float (&l)[NT][2]) {
    const float *ks = reinterpret_cast<const float *>(aux);
    tile_page_q4<D, NT>(smem_u32(st), smem_u32(st + kPageBytes), ks, ks + kPage * kG, ntok, sl2, lane,
                        qf, acc, m, l);
  }
  // q in f16, channel order of the INT4 tile: in k-step 2j (2j + 1) of group
  // j, k-slots 2 tig, 2 tig + 1 <- channels 32j + 8 tig + {0, 4} ({2, 6}) and
  // k-slots 2 tig + 8, 2 tig + 9 <- channels 32j + 8 tig + {1, 5} ({3, 7})
  static __device__ __forceinline__ void q_words(const uint32_t *qrow, int ks, int tig,
                                                 uint32_t &w0, uint32_t &w1) {
    q_words_q4<T>(qrow, ks, tig, w0, w1);
  }
  static __device__ __forceinline__ int dim(int mt, int e, int g8) { return dim_q4(mt, e, g8); }
};

// A quantised page policy for KV heads with a single query row (G = 1): the
// tile's N columns carry the 32-channel scale groups instead of idle query
// rows (tile_page_g1).  q's fragment of k-step ks is loaded into column ks / 2
// only, and a finished pair's state is moved back to the general layout
// (g1_to_rows) before it is written or parked.
template <class Base, int D, bool kInt4, Code8 kFmt>
struct PackedG1 : Base {
  static constexpr bool kPackG1 = true;
  static __device__ __forceinline__ void tile(uint8_t *st, uint8_t *aux, int ntok, float sl2, int lane,
                                              const uint32_t (&qf)[1][D / 16][2],
                                              float (&acc)[1][D / 16][4], float (&m)[1][2],
                                              float (&l)[1][2]) {
    const float *ks = reinterpret_cast<const float *>(aux);
    tile_page_g1<D, kInt4, kFmt>(smem_u32(st), smem_u32(st + Base::kPageBytes), ks,
                                 ks + kPage * (D / 32), ntok, sl2, lane, qf, acc, m, l);
  }
};

namespace {

// Zero one output row of d elements (16-byte stores).
template <typename T>
__device__ __forceinline__ void zero_row(T *p, int d) {
  for (int i = 0; i < d; i += 8) *reinterpret_cast<uint4 *>(p + i) = make_uint4(0, 0, 0, 0);
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

}  // namespace

template <int D, int NT, class Pol, int W, int S>
__global__ void __launch_bounds__(32 * W, 1)
    decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV) {
  using T = typename Pol::Out;
  using Gm = Geo<D, NT, W, S, Pol::kStride, Pol::kAuxBytes>;
  using M = Mma<T>;
  constexpr int kRows = 8 * NT;  // query rows per tile (G padded)
  constexpr int kPatch = 32;     // page-meta flag: fused append writes a row of this page
  const bool fused = a.k_new != nullptr;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int warp_tot[32];

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  float *edge_acc = reinterpret_cast<float *>(smem + (size_t)W * S * Gm::kStageBytes);
  uint8_t *aux = reinterpret_cast<uint8_t *>(edge_acc + (size_t)W * Gm::kEdgeFloats);
  uint64_t *bars = reinterpret_cast<uint64_t *>(aux + (size_t)W * S * Gm::kAuxBytes);
  int4 *meta = reinterpret_cast<int4 *>(reinterpret_cast<uint8_t *>(bars) + Gm::kBarBytes);
  float *edge_ml = reinterpret_cast<float *>(meta + W * S);  // [W][2][2][kRows]: m, l
  int *edge_id = reinterpret_cast<int *>(edge_ml + W * 2 * 2 * kRows);  // [W][2]
  int *cum = edge_id + 2 * W;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cap = a.maxb * kPage;

  // Launched as a programmatic dependent: nothing is read before the
  // preceding grid has completed and its writes are visible.  Dependents (the
  // merge) may be scheduled at once; they wait for this grid the same way.
  grid_dependency_wait();
  grid_launch_dependents();
  if (tid == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }

  // pages of sequence b this kernel streams: all of them, minus the leading
  // shared pages a prefix pass already attended (shared-prefix mode)
  auto skip_of = [&](int b) -> int { return a.skip ? __ldg(a.skip + b) : 0; };
  auto pages_of = [&](int b) -> int {
    const int np = (clamp_len(__ldg(a.seq_lens + b), cap) + kPage - 1) / kPage;
    return max(0, np - skip_of(b));
  };

  // ---- 1. pages per sequence, exclusive prefix sum into cum[0..B]
  {
    const int per = (a.B + Gm::kThreads - 1) / Gm::kThreads;
    const int b0 = tid * per;
    const int b1 = min(a.B, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) {
      const int raw = __ldg(a.seq_lens + b);
      if (raw < 0 || raw > cap) flag_error(a.err, kErrSeqLen);
      local += pages_of(b);
    }
    const int incl = warp_incl_scan(local, lane);
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int v = lane < W ? warp_tot[lane] : 0;
      v = warp_incl_scan(v, lane);
      if (lane < W) warp_tot[lane] = v;
    }
    __syncthreads();
    int run = (warp ? warp_tot[warp - 1] : 0) + incl - local;
    for (int b = b0; b < b1; ++b) {
      cum[b] = run;
      run += pages_of(b);
    }
    if (tid == 0) cum[a.B] = warp_tot[W - 1];
    if (tid < 2 * W) edge_id[tid] = -1;
    __syncthreads();
  }
  const long long P = static_cast<long long>(cum[a.B]) * a.H_kv;
  const int N = used_parts(a, P);
  if (blockIdx.x == 0)
    for (int i = tid; i <= a.B; i += Gm::kThreads) a.ws_cum[i] = cum[i];

  // ---- 2. empty sequences: zero output rows (their pairs own no pages)
  {
    const long long rows = static_cast<long long>(a.B) * a.H_q;
    for (long long r = static_cast<long long>(blockIdx.x) * Gm::kThreads + tid; r < rows;
         r += static_cast<long long>(gridDim.x) * Gm::kThreads) {
      const int b = static_cast<int>(r / a.H_q);
      if (cum[b + 1] == cum[b] && skip_of(b) == 0) {
        zero_row(reinterpret_cast<T *>(a.out) + r * D, D);
        if (a.lse_out) a.lse_out[r] = -INFINITY;
      }
    }
  }

  // ---- 3. this CTA's partition, and this warp's contiguous share of it
  const int cta = blockIdx.x;
  if (cta >= N) return;  // the whole CTA: no block-level sync follows for it
  const long long c0 = part_begin(cta, P, N), c1 = part_begin(cta + 1, P, N);
  const long long p0 = c0 + ((c1 - c0) * warp) / W, p1 = c0 + ((c1 - c0) * (warp + 1)) / W;
  const int H = a.H_kv;
  const int g8 = lane >> 2, tig = lane & 3;

  // running state of the current (sequence, KV head) pair
  uint32_t qf[NT][Gm::kSteps][2];
  float acc[NT][Gm::kSteps][4];
  float m_run[NT][2], l_run[NT][2];

  // a pair whose sequence also has prefix partials always leaves a partial
  auto forced_partial = [&](int seg) -> bool { return a.skip && skip_of(seg / H) > 0; };

  auto pair_range = [&](int seg, long long &s0, long long &s1) {
    const int b = seg / H, h = seg - (seg / H) * H;
    const int np = cum[b + 1] - cum[b];
    s0 = static_cast<long long>(cum[b]) * H + static_cast<long long>(h) * np;
    s1 = s0 + np;
  };

  // Write a finished pair from register state (l_run already summed over the
  // 8 token lanes): the final rows if `whole`, else a normalised partial
  // (o, lse) at slot cta + seg for the cross-CTA merge.
  auto emit = [&](int seg, bool whole) {
    const int b = seg / H, h = seg - (seg / H) * H;
    const size_t row0 = static_cast<size_t>(b) * a.H_q + static_cast<size_t>(h) * a.G;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float l = l_run[nt][i];
        const int r = nt * 8 + 2 * tig + i;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float lse = l > 0.f ? (m_run[nt][i] + fast_log2(l)) * kLn2 : -INFINITY;
        if (r < a.G) {
          if (whole) {
            T *o = reinterpret_cast<T *>(a.out) + (row0 + r) * D;
#pragma unroll
            for (int mt = 0; mt < Gm::kSteps; ++mt) {
              o[Pol::dim(mt, i, g8)] = M::from_float(acc[nt][mt][i] * inv);
              o[Pol::dim(mt, 2 + i, g8)] = M::from_float(acc[nt][mt][2 + i] * inv);
            }
            if (a.lse_out && g8 == 0) a.lse_out[row0 + r] = lse;
          } else {
            const size_t slot = static_cast<size_t>(cta) + seg;
            float *o = a.part_o + (slot * a.G + r) * D;
            const uint64_t keep = l2_policy_evict_last();
#pragma unroll
            for (int mt = 0; mt < Gm::kSteps; ++mt) {
              st_keep(o + Pol::dim(mt, i, g8), acc[nt][mt][i] * inv, keep);
              st_keep(o + Pol::dim(mt, 2 + i, g8), acc[nt][mt][2 + i] * inv, keep);
            }
            if (g8 == 0) st_keep(a.part_lse + slot * a.G + r, lse, keep);
          }
        }
      }
    }
  };

  auto sum_l = [&]() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float l = l_run[nt][i];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_run[nt][i] = l;
      }
  };

  // Park a pair this warp holds only a piece of: unnormalised accumulators
  // (lane-major, conflict-free) plus per-row max and sum, for the combine step.
  auto park = [&](int seg, int which, float *dst) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < Gm::kSteps; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[((nt * Gm::kSteps + mt) * 4 + e) * 32 + lane] = acc[nt][mt][e];
    float *ml = edge_ml + (warp * 2 + which) * 2 * kRows;
    if (g8 == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          ml[nt * 8 + 2 * tig + i] = m_run[nt][i];
          ml[kRows + nt * 8 + 2 * tig + i] = l_run[nt][i];
        }
    }
    if (lane == 0) edge_id[warp * 2 + which] = seg;
  };

  auto finish_pair = [&](int seg, bool last) {
    if constexpr (Pol::kPackG1) g1_to_rows(acc, lane);
    sum_l();
    long long s0, s1;
    pair_range(seg, s0, s1);
    if (s0 >= p0 && s1 <= p1) {
      // entirely inside this warp's share: final rows, or the one partial of
      // this CTA when the sequence also has prefix partials to merge
      emit(seg, !forced_partial(seg));
    } else if (s0 < p0) {
      park(seg, 0, edge_acc + (size_t)warp * Gm::kEdgeFloats);  // continues from an earlier warp
    } else {
      // continues into a later warp; this is the warp's last pair, so its
      // ring is idle and stage 0 holds the parked state
      park(seg, 1, reinterpret_cast<float *>(stages + (size_t)warp * S * Gm::kStageBytes));
    }
    (void)last;
  };

  bool failed = false;
  if (p0 < p1) {
    const uint32_t stage0 = smem_u32(stages + (size_t)warp * S * Gm::kStageBytes);
    const uint32_t aux0 = smem_u32(aux + (size_t)warp * S * Gm::kAuxBytes);
    const uint32_t bar0 = smem_u32(bars + warp * S);
    int4 *meta_w = meta + warp * S;
    const uint64_t policy = a.evict_first ? l2_policy_evict_first() : l2_policy_evict_normal();

    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < S; ++s) mbar_init(bar0 + 8 * s, 1);
      mbar_init_fence();
    }
    __syncwarp();

    // Fetch-side page descriptors, one fetch position per lane, in windows of
    // 32 positions.  `nx*` is the next window, computed one window early so
    // its block-table loads are long done when it is promoted.
    auto describe = [&](long long wb, int &pb, int &h, int &seg, int &ntok) {
      pb = -1;
      h = 0;
      seg = -1;
      ntok = 0;
      const long long pos = wb + lane;
      if (pos < p1) {
        int lo = 0, hi = a.B;  // largest b with cum[b] * H <= pos
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (static_cast<long long>(cum[mid]) * H <= pos) lo = mid; else hi = mid;
        }
        const int b = lo;
        const int np = cum[b + 1] - cum[b];
        const long long off = pos - static_cast<long long>(cum[b]) * H;
        h = static_cast<int>(off / np);
        const int i = static_cast<int>(off - static_cast<long long>(h) * np);
        const int li = i + skip_of(b);  // logical page index in the sequence
        pb = __ldg(a.block_table + static_cast<size_t>(b) * a.maxb + li);
        ntok = min(kPage, clamp_len(__ldg(a.seq_lens + b), cap) - li * kPage);
        // fused append: the pair's last page holds the step's new token
        if (fused && i == np - 1) ntok |= kPatch;
        seg = b * H + h;
      }
    };
    auto promote = [&](int pb, int h, int seg) -> int {
      if (seg < 0) return -1;
      if (pb < 0 || pb >= a.num_blocks) {
        flag_error(a.err, kErrBlockTable);
        return -1;
      }
      return (pb * H + h) * kPage;  // TMA row coordinate of this page's 16 rows
    };

    long long wb = p0;
    int cur_row, cur_seg, cur_ntok;
    int nx_pb, nx_h, nx_seg, nx_ntok;
    {
      int pb, h;
      describe(wb, pb, h, cur_seg, cur_ntok);
      cur_row = promote(pb, h, cur_seg);
      describe(wb + 32, nx_pb, nx_h, nx_seg, nx_ntok);
    }

    long long f = p0;  // next page to fetch
    int fst = 0;       // its stage
    auto issue = [&]() {
      int j = static_cast<int>(f - wb);
      if (j >= 32) {
        cur_row = promote(nx_pb, nx_h, nx_seg);
        cur_seg = nx_seg;
        cur_ntok = nx_ntok;
        wb += 32;
        describe(wb + 32, nx_pb, nx_h, nx_seg, nx_ntok);
        j -= 32;
      }
      const int row = __shfl_sync(0xffffffffu, cur_row, j);
      const int seg = __shfl_sync(0xffffffffu, cur_seg, j);
      const int ntok = __shfl_sync(0xffffffffu, cur_ntok, j);
      if (lane == 0) {
        meta_w[fst] = make_int4(seg, row >= 0 ? ntok : 0, row, 0);
        const uint32_t bar = bar0 + 8 * fst;
        if (row >= 0) {
          Pol::issue(stage0 + fst * Gm::kStageBytes, aux0 + fst * Gm::kAuxBytes, bar, &tmK, &tmV, row,
                     policy, a);
        } else {
          mbar_arrive(bar);
        }
      }
      ++f;
      if (++fst == S) fst = 0;
    };

#pragma unroll 1
    for (int s = 0; s < S; ++s)
      if (f < p1) issue();

    int cur = -1;  // pair being accumulated

    auto begin_pair = [&](int seg) {
      const int b = seg / H, h = seg - (seg / H) * H;
      const uint32_t *qw = reinterpret_cast<const uint32_t *>(a.q) +
                           (static_cast<size_t>(b) * a.H_q + static_cast<size_t>(h) * a.G) * (D / 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int r = nt * 8 + g8;
#pragma unroll
        for (int ks = 0; ks < Gm::kSteps; ++ks) {
          // one query row with the scale groups in N: k-step ks of row 0 in
          // column (group) ks / 2
          const bool mine = Pol::kPackG1 ? g8 == (ks >> 1) : r < a.G;
          if (mine) {
            Pol::q_words(qw + (Pol::kPackG1 ? 0 : r) * (D / 2), ks, tig, qf[nt][ks][0], qf[nt][ks][1]);
          } else {
            qf[nt][ks][0] = 0u;
            qf[nt][ks][1] = 0u;
          }
        }
#pragma unroll
        for (int mt = 0; mt < Gm::kSteps; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
      }
    };

    // ---- main loop over this warp's pages
    const long long nmy = p1 - p0;
    int cst = 0;
    uint32_t cph = 0;
    long long c = 0;
#pragma unroll 1
    for (; c < nmy; ++c) {
      const uint32_t bar = bar0 + 8 * cst;
      const bool ok = mbar_wait_bounded(bar, cph, a.wait_polls);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) flag_error(a.err, kErrTimeout);
        failed = true;
        break;
      }
      const int4 md = meta_w[cst];
      if (md.x != cur) {
        if (cur >= 0) finish_pair(cur, false);
        cur = md.x;
        begin_pair(cur);
      }
      const int ntok = md.y & (kPatch - 1);
      if (ntok > 0) {
        uint8_t *kp = stages + ((size_t)warp * S + cst) * Gm::kStageBytes;
        uint8_t *ap = aux + ((size_t)warp * S + cst) * Gm::kAuxBytes;
        if (md.y & kPatch) {
          // fused append: the new token is row ntok - 1 of this page.  Put it
          // into the staged page (the copy just read may predate it) and
          // write it to the cache -- no other CTA reads this row in this launch.
          Pol::patch(kp, ap, ntok - 1, lane, a, cur / H, cur - (cur / H) * H, md.z);
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (ntok < kPage) {
          // rows past the sequence end may hold anything (even NaN): clear V's
          // so the zero weights of masked tokens cannot turn into NaN
          Pol::zero_tail(kp, ap, ntok, lane);
          fence_proxy_async_smem();
          __syncwarp();
        }
        Pol::tile(kp, ap, ntok, a.scale_log2, lane, qf, acc, m_run, l_run);
      }
      __syncwarp();
      if (f < p1) issue();
      if (++cst == S) {
        cst = 0;
        cph ^= 1u;
      }
    }

    if (failed) {
      // let every copy still in flight land before shared memory is reused or
      // freed (with the full poll limit, whatever the streaming waits used)
      for (; c < f - p0; ++c) {
        mbar_wait_bounded(bar0 + 8 * cst, cph);
        if (++cst == S) {
          cst = 0;
          cph ^= 1u;
        }
      }
    } else if (cur >= 0) {
      __syncwarp();
      finish_pair(cur, true);
    }
  }

  // ---- 4. combine the pieces of pairs that several warps of this CTA hold.
  // A job is one such pair.  Its accumulator slots (kSlots per lane) are cut
  // into `parts` equal ranges of PER slots -- as many as keep every warp busy:
  // one part when the CTA has many split pairs, down to one slot pair per
  // part when it has one or two -- and the (job, part) units go round-robin
  // over the warps.  Each unit folds the pair's pieces in ascending (warp,
  // slot) order: new row maxima, then rescaled sums of l and of its slots,
  // the arithmetic and order of one warp folding them all.
  __syncthreads();
  if (failed) return;
  {
    constexpr int kRowSlots = Gm::kSteps * 4;  // slots of one n-tile
    constexpr int kSlots = NT * kRowSlots;
    static_assert((kSlots & (kSlots - 1)) == 0, "slot count must be a power of two");
    const int e_id = lane < 2 * W ? edge_id[lane] : -1;  // piece slot w2 * 2 + k -> its pair
    bool first = e_id >= 0;
    for (int j = 0; j < 2 * W; ++j) {
      const int ej = __shfl_sync(0xffffffffu, e_id, j);
      if (j < lane && ej == e_id) first = false;
    }
    const unsigned firsts = __ballot_sync(0xffffffffu, first);  // one bit per job
    const int jobs = __popc(firsts);
    int parts = 1;
    while (parts * 2 * jobs <= W && parts * 2 <= kSlots / 2) parts *= 2;

    auto unit = [&](auto per_c, int u) {
      constexpr int PER = decltype(per_c)::value;
      constexpr int kParts = kSlots / PER;
      const int jj = u / kParts, pp = u - jj * kParts;
      unsigned fb = firsts;
      for (int i = 0; i < jj; ++i) fb &= fb - 1;
      const int seg = __shfl_sync(0xffffffffu, e_id, __ffs(fb) - 1);
      const unsigned pieces = __ballot_sync(0xffffffffu, e_id == seg);
      const int sl0 = pp * PER;  // first slot of this unit
      // n-tile of slot k of the unit (uniform over the unit unless it spans n-tiles)
      auto nt_of = [&](int k) { return PER > kRowSlots ? k / kRowSlots : sl0 / kRowSlots; };
      float mr[NT][2], lr[NT][2], av[PER];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          mr[nt][i] = -INFINITY;
          lr[nt][i] = 0.f;
        }
#pragma unroll
      for (int k = 0; k < PER; ++k) av[k] = 0.f;
      for (unsigned pc = pieces; pc; pc &= pc - 1) {
        const float *ml = edge_ml + (__ffs(pc) - 1) * 2 * kRows;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 2; ++i) mr[nt][i] = fmaxf(mr[nt][i], ml[nt * 8 + 2 * tig + i]);
      }
      for (unsigned pc = pieces; pc; pc &= pc - 1) {
        const int idx = __ffs(pc) - 1, w2 = idx >> 1;
        const float *ml = edge_ml + idx * 2 * kRows;
        const float *src = ((idx & 1) == 0 ? edge_acc + (size_t)w2 * Gm::kEdgeFloats
                                           : reinterpret_cast<const float *>(
                                                 stages + (size_t)w2 * S * Gm::kStageBytes)) +
                           sl0 * 32 + lane;
        float sc[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int r = nt * 8 + 2 * tig + i;
            const float mi = ml[r];
            sc[nt][i] = mi == -INFINITY ? 0.f : fast_exp2(mi - mr[nt][i]);
            lr[nt][i] += ml[kRows + r] * sc[nt][i];
          }
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const int nt = nt_of(k);
          const float s_k = NT == 1 || nt == 0 ? sc[0][k & 1] : sc[NT - 1][k & 1];
          av[k] += src[k * 32] * s_k;
        }
      }
      // write the unit's slots: final rows, or the CTA's partial
      long long s0, s1;
      pair_range(seg, s0, s1);
      const bool whole = s0 >= c0 && s1 <= c1 && !forced_partial(seg);
      const int b = seg / H, h = seg - (seg / H) * H;
      const size_t row0 = static_cast<size_t>(b) * a.H_q + static_cast<size_t>(h) * a.G;
      const size_t slot = static_cast<size_t>(cta) + seg;
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int sl = sl0 + k, nt = nt_of(k), i = k & 1;
        const int mt = (sl - nt * kRowSlots) >> 2, e = sl & 3;
        const int r = nt * 8 + 2 * tig + i;
        if (r >= a.G) continue;
        const float l = NT == 1 || nt == 0 ? lr[0][i] : lr[NT - 1][i];
        const float m = NT == 1 || nt == 0 ? mr[0][i] : mr[NT - 1][i];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const bool lse_slot = g8 == 0 && (sl - nt * kRowSlots) < 2;  // the row's first slot
        if (whole) {
          reinterpret_cast<T *>(a.out)[(row0 + r) * D + Pol::dim(mt, e, g8)] = M::from_float(av[k] * inv);
          if (lse_slot && a.lse_out)
            a.lse_out[row0 + r] = l > 0.f ? (m + fast_log2(l)) * kLn2 : -INFINITY;
        } else {
          const uint64_t keep = l2_policy_evict_last();
          st_keep(a.part_o + (slot * a.G + r) * D + Pol::dim(mt, e, g8), av[k] * inv, keep);
          if (lse_slot)
            st_keep(a.part_lse + slot * a.G + r, l > 0.f ? (m + fast_log2(l)) * kLn2 : -INFINITY, keep);
        }
      }
    };

    const int units = jobs * parts;
#pragma unroll 1
    for (int u = warp; u < units; u += W) {
      switch (kSlots / parts) {
        case 2: unit(std::integral_constant<int, 2>{}, u); break;
        case 4: unit(std::integral_constant<int, 4>{}, u); break;
        case 8: unit(std::integral_constant<int, 8>{}, u); break;
        case 16: unit(std::integral_constant<int, (kSlots >= 16 ? 16 : 2)>{}, u); break;
        case 32: unit(std::integral_constant<int, (kSlots >= 32 ? 32 : 2)>{}, u); break;
        default: unit(std::integral_constant<int, (kSlots >= 64 ? 64 : 2)>{}, u); break;
      }
    }
  }
}

// ------------------------------------------------------------------ merge

// One CTA (256 threads, 8 warps) merges `count` (+ `count2` from a second
// set laid out the same way) partial results of one output row: partial k has log-sum-exp lse[k * lse_stride] and normalised
// output o[k * o_stride .. + D).  Each warp folds its partials k = warp,
// warp + 8, ... into a running (max, sum, output) state -- the rescale of
// the online softmax applied to whole partials -- loading four partials'
// lse and o at once; the 8 warp states are then combined in shared memory.
// Result: LSE = M + ln sum_k exp(lse_k - M), out = sum_k exp(lse_k - LSE) o_k,
// one rounding to T.  Partials with lse = -inf carry no weight (their o is
// never read); if all are empty, out = 0 and LSE = -inf.
template <int D, typename T>
__device__ __forceinline__ void merge_row(const float *lse, long long lse_stride, const float *o,
                                          long long o_stride, int count, T *out, float *lse_out,
                                          const float *lse2 = nullptr, long long lse2_stride = 0,
                                          const float *o2 = nullptr, long long o2_stride = 0,
                                          int count2 = 0) {
  constexpr int kV = D / 32;
  constexpr int kBatch = 4;
  __shared__ float wm[8], wl[8];
  __shared__ __align__(16) float wo[8][D];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  float m = -INFINITY, l = 0.f;
  float acc[kV];
#pragma unroll
  for (int e = 0; e < kV; ++e) acc[e] = 0.f;
  const int total = count + count2;
  for (int k0 = warp; k0 < total; k0 += 8 * kBatch) {
    float lk[kBatch];
    float ov[kBatch][kV];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int k = k0 + 8 * j;
      const bool first = k < count;
      const long long kk = first ? k : k - count;
      lk[j] = k < total ? (first ? lse[kk * lse_stride] : lse2[kk * lse2_stride]) * kLog2e
                        : -INFINITY;
      // o is loaded with lse (not after it) so both are in flight together;
      // an empty partial's o is read but never used
      if (k < total) {
        const float *src = (first ? o + kk * o_stride : o2 + kk * o2_stride) + lane * kV;
        if constexpr (kV == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(src);
          ov[j][0] = v.x;
          ov[j][1] = v.y;
          ov[j][2] = v.z;
          ov[j][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2 *>(src);
          ov[j][0] = v.x;
          ov[j][1] = v.y;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (lk[j] == -INFINITY) continue;
      const float mn = fmaxf(m, lk[j]);
      const float a = fast_exp2(m - mn), b = fast_exp2(lk[j] - mn);
#pragma unroll
      for (int e = 0; e < kV; ++e) acc[e] = acc[e] * a + ov[j][e] * b;
      l = l * a + b;
      m = mn;
    }
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < kV; ++e) wo[warp][lane * kV + e] = acc[e];
  __syncthreads();
  float M = wm[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) M = fmaxf(M, wm[i]);
  if (M == -INFINITY) {
    for (int t = tid; t < D; t += 256) out[t] = Mma<T>::from_float(0.f);
    if (tid == 0 && lse_out) *lse_out = -INFINITY;
    return;
  }
  float sc[8], L = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sc[i] = wm[i] == -INFINITY ? 0.f : fast_exp2(wm[i] - M);
    L += wl[i] * sc[i];
  }
  const float inv = 1.f / L;
  for (int t = tid; t < D; t += 256) {
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) v += wo[i][t] * sc[i];
    out[t] = Mma<T>::from_float(v * inv);
  }
  if (tid == 0 && lse_out) *lse_out = (M + fast_log2(L)) * kLn2;
}

// One warp merges the partials of one output row (two sets laid out like
// merge_row's): the same running fold, four partials' loads in flight at a
// time, no shared memory.  Used when rows have few partials each.
template <int D, typename T>
__device__ __forceinline__ void merge_row_warp(const float *lse, long long lse_stride,
                                               const float *o, long long o_stride, int count,
                                               T *out, float *lse_out, const float *lse2,
                                               long long lse2_stride, const float *o2,
                                               long long o2_stride, int count2, int lane) {
  constexpr int kV = D / 32;
  constexpr int kBatch = 4;
  float m = -INFINITY, l = 0.f;
  float acc[kV];
#pragma unroll
  for (int e = 0; e < kV; ++e) acc[e] = 0.f;
  const int total = count + count2;
  for (int k0 = 0; k0 < total; k0 += kBatch) {
    float lk[kBatch];
    float ov[kBatch][kV];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int k = k0 + j;
      const bool first = k < count;
      const long long kk = first ? k : k - count;
      lk[j] = k < total ? (first ? lse[kk * lse_stride] : lse2[kk * lse2_stride]) * kLog2e
                        : -INFINITY;
      if (k < total) {
        const float *src = (first ? o + kk * o_stride : o2 + kk * o2_stride) + lane * kV;
        if constexpr (kV == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(src);
          ov[j][0] = v.x;
          ov[j][1] = v.y;
          ov[j][2] = v.z;
          ov[j][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2 *>(src);
          ov[j][0] = v.x;
          ov[j][1] = v.y;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (lk[j] == -INFINITY) continue;
      const float mn = fmaxf(m, lk[j]);
      const float a = fast_exp2(m - mn), b = fast_exp2(lk[j] - mn);
#pragma unroll
      for (int e = 0; e < kV; ++e) acc[e] = acc[e] * a + ov[j][e] * b;
      l = l * a + b;
      m = mn;
    }
  }
  if (m == -INFINITY) {
#pragma unroll
    for (int e = 0; e < kV; ++e) out[lane * kV + e] = Mma<T>::from_float(0.f);
    if (lane == 0 && lse_out) *lse_out = -INFINITY;
    return;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < kV; ++e) out[lane * kV + e] = Mma<T>::from_float(acc[e] * inv);
  if (lane == 0 && lse_out) *lse_out = (m + fast_log2(l)) * kLn2;
}

// Merge of the pieces of every (sequence, KV head) pair that partition edges
// cut; grid = (B * H_kv pairs, G rows).
// Rows with many partials (long contexts cut by many CTAs) get a whole CTA
// each (kWide); otherwise each warp of a CTA takes one row.
template <int D, typename T, bool kWide>
__global__ void __launch_bounds__(256) decode_merge_kernel(const DecodeArgs a) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row_id = kWide ? static_cast<long long>(blockIdx.x)
                                 : static_cast<long long>(blockIdx.x) * 8 + warp;
  if (row_id >= static_cast<long long>(a.B) * a.H_q) return;  // whole warp (or CTA)
  const int seg = static_cast<int>(row_id / a.G), r = static_cast<int>(row_id - (row_id / a.G) * a.G);
  const int b = seg / a.H_kv, h = seg - b * a.H_kv;
  const int c0 = a.ws_cum[b], np = a.ws_cum[b + 1] - c0;
  const int skip = a.skip ? __ldg(a.skip + b) : 0;
  if (np == 0 && skip == 0) return;  // empty sequence: zeroed by the decode kernel
  const long long P = static_cast<long long>(a.ws_cum[a.B]) * a.H_kv;
  const size_t row = (static_cast<size_t>(b) * a.H_q + static_cast<size_t>(h) * a.G + r);
  long long slot0 = 0;
  int count = 0;
  if (np > 0) {
    const int N = used_parts(a, P);
    const long long s0 = static_cast<long long>(c0) * a.H_kv + static_cast<long long>(h) * np;
    const long long wf = part_of(s0, P, N), wl = part_of(s0 + np - 1, P, N);
    if (wf == wl && skip == 0) return;  // written directly by its only CTA
    slot0 = wf + seg;
    count = static_cast<int>(wl - wf + 1);
  }
  const float *pl = nullptr, *po = nullptr;
  long long pls = 0, pos = 0;
  int pc = 0;
  if (skip > 0) {  // the prefix pass's chunk partials of this row
    const size_t i0 = (static_cast<size_t>(h) * a.B + b) * a.G + r;
    pls = static_cast<long long>(a.H_kv) * a.B * a.G;
    pos = pls * D;
    pl = a.pre_lse + i0;
    po = a.pre_o + i0 * D;
    pc = a.pre_chunks;
  }
  T *out = reinterpret_cast<T *>(a.out) + row * D;
  float *lo = a.lse_out ? a.lse_out + row : nullptr;
  if constexpr (kWide)
    merge_row<D, T>(a.part_lse + slot0 * a.G + r, a.G, a.part_o + (slot0 * a.G + r) * D,
                    static_cast<long long>(a.G) * D, count, out, lo, pl, pls, po, pos, pc);
  else
    merge_row_warp<D, T>(a.part_lse + slot0 * a.G + r, a.G, a.part_o + (slot0 * a.G + r) * D,
                         static_cast<long long>(a.G) * D, count, out, lo, pl, pls, po, pos, pc, lane);
}

// Merge of caller-provided partials [B][H_q][S][D]; grid = B * H_q rows.
template <int D, typename T>
__global__ void __launch_bounds__(256) generic_merge_kernel(const GenericMergeArgs a) {
  const long long row = blockIdx.x;
  const int b = static_cast<int>(row / a.H_q);
  int count = a.S;
  if (a.counts) count = clamp_len(__ldg(a.counts + b), a.S);
  merge_row<D, T>(a.part_lse + row * a.S, 1, a.part_o + row * a.S * D, D, count,
                  reinterpret_cast<T *>(a.out) + row * D, a.lse_out ? a.lse_out + row : nullptr);
}

// ------------------------------------------------------------- launchers

namespace {

// Worker warps per CTA (one CTA per SM) and ring stages per warp, per head
// dim D and n-tiles NT (G <= 8: 1, G <= 16: 2).  Shared memory per warp is
// S * 64 * D bytes of ring plus one parked accumulator tile.  Defaults can
// be overridden at build time (-DKVD_TUNE_W128_1=... etc.).
#ifndef KVD_TUNE_W128_1
#define KVD_TUNE_W128_1 16
#endif
#ifndef KVD_TUNE_S128_1
#define KVD_TUNE_S128_1 1
#endif
#ifndef KVD_TUNE_W128_2
#define KVD_TUNE_W128_2 12
#endif
#ifndef KVD_TUNE_S128_2
#define KVD_TUNE_S128_2 1
#endif
#ifndef KVD_TUNE_W64_1
#define KVD_TUNE_W64_1 16
#endif
#ifndef KVD_TUNE_S64_1
#define KVD_TUNE_S64_1 2
#endif
#ifndef KVD_TUNE_W64_2
#define KVD_TUNE_W64_2 12
#endif
#ifndef KVD_TUNE_S64_2
#define KVD_TUNE_S64_2 2
#endif

template <int D, int NT>
struct Tune;
template <>
struct Tune<128, 1> {
  static constexpr int W = KVD_TUNE_W128_1, S = KVD_TUNE_S128_1;
};
template <>
struct Tune<128, 2> {
  static constexpr int W = KVD_TUNE_W128_2, S = KVD_TUNE_S128_2;
};
template <>
struct Tune<64, 1> {
  static constexpr int W = KVD_TUNE_W64_1, S = KVD_TUNE_S64_1;
};
template <>
struct Tune<64, 2> {
  static constexpr int W = KVD_TUNE_W64_2, S = KVD_TUNE_S64_2;
};

template <int D, int NT, typename T, int W, int S>
cudaError_t launch_decode_ws(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                             cudaStream_t st, int grid) {
  using Pol = Page16<D, NT, T>;
  auto kern = decode_kernel<D, NT, Pol, W, S>;
  const size_t smem = Geo<D, NT, W, S, Pol::kStride, Pol::kAuxBytes>::smem(a.B);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(32 * W), smem, st, a, tmK, tmV);
}

// Launches with at most one (sequence, KV head) pair per warp at 7 warps
// per CTA take 7 warps with two stages each at d = 128 instead of 16 with
// one: each warp streams twice the pages, its ring overlaps a page's tile
// with the next page's copy, and the CTA's warps finish closer together.
// With more pairs than that, the pair changes (q loads, partial writes)
// sit on fewer warps' serial paths and 16 x 1 is faster.  Same-box sweeps,
// us a call:
//   long (8 pairs): 16 x 1 94.9, 12 x 1 93.1, 10 x 2 93.9, 8 x 2 91.9,
//     7 x 2 89.9, 6 x 2 91.4, 5 x 2 93.8, 8 x 3 98.7, 6 x 3 92.5, 6 x 4
//     97.2, 4 x 3 103.6;
//   gqa70b (512 pairs): 16 x 1 669.8, 7 x 2 652.0, 8 x 2 658.7, 10 x 2 678.0;
//   mha7b (1024 pairs): 16 x 1 325.6, 7 x 2 322.1, 8 x 2 332.3, 10 x 2 330.3;
//   cbatch (2048 pairs): 16 x 1 552.5, 7 x 2 674.3; its shared-prefix
//     suffix decode 291.6 against 306.7.
// The 8-bit tile, bound by its instructions, keeps its 16 warps (`long
// --kv-fp8` 60.3 us at 16 x 2 against 64.4 at 12 x 2 and 74.6 at 8 x 4).
#ifndef KVD_TUNE_WL
#define KVD_TUNE_WL 7
#endif
#ifndef KVD_TUNE_SL
#define KVD_TUNE_SL 2
#endif
template <int D, int NT, typename T>
cudaError_t launch_decode_t(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                            cudaStream_t st, int grid) {
  constexpr int W = Tune<D, NT>::W, S = Tune<D, NT>::S;
  if constexpr (D == 128 && NT == 1 && (KVD_TUNE_WL != W || KVD_TUNE_SL != S)) {
    const long long pairs = static_cast<long long>(a.B) * a.H_kv;
    if (pairs <= static_cast<long long>(KVD_TUNE_WL) * grid)
      return launch_decode_ws<D, NT, T, KVD_TUNE_WL, KVD_TUNE_SL>(a, tmK, tmV, st, grid);
  }
  return launch_decode_ws<D, NT, T, W, S>(a, tmK, tmV, st, grid);
}

template <typename T>
cudaError_t launch_decode_dt(const DecodeArgs &a, int d, const CUtensorMap &tmK,
                             const CUtensorMap &tmV, cudaStream_t st, int grid) {
  const bool two = a.G > 8;
  if (d == 128)
    return two ? launch_decode_t<128, 2, T>(a, tmK, tmV, st, grid)
               : launch_decode_t<128, 1, T>(a, tmK, tmV, st, grid);
  return two ? launch_decode_t<64, 2, T>(a, tmK, tmV, st, grid)
             : launch_decode_t<64, 1, T>(a, tmK, tmV, st, grid);
}

template <typename T>
cudaError_t launch_merge_dt(const DecodeArgs &a, int d, cudaStream_t st) {
  // expected partials per row: CTA partitions per pair, plus prefix chunks
  const long long pairs = static_cast<long long>(a.B) * a.H_kv;
  const long long per_row = a.nparts / (pairs > 0 ? pairs : 1) + 1 + a.pre_chunks;
  const long long rows = static_cast<long long>(a.B) * a.H_q;
  if (per_row >= 16) {
    const dim3 grid(static_cast<unsigned>(rows));
    if (d == 128) return launch_pdl(decode_merge_kernel<128, T, true>, grid, dim3(256), 0, st, a);
    return launch_pdl(decode_merge_kernel<64, T, true>, grid, dim3(256), 0, st, a);
  }
  const dim3 grid(static_cast<unsigned>((rows + 7) / 8));
  if (d == 128) return launch_pdl(decode_merge_kernel<128, T, false>, grid, dim3(256), 0, st, a);
  return launch_pdl(decode_merge_kernel<64, T, false>, grid, dim3(256), 0, st, a);
}

template <typename T>
cudaError_t launch_generic_dt(const GenericMergeArgs &a, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>(static_cast<long long>(a.B) * a.H_q);
  if (a.d == 128) generic_merge_kernel<128, T><<<grid, 256, 0, st>>>(a);
  else generic_merge_kernel<64, T><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_auto_parts(int sms) { return sms; }

// 8-bit cache: d = 128 has 4 KB code stages plus 512 B of scales, d = 64
// 2 KB stages plus 256 B; as for the 16-bit pages, many warps with a short
// ring each keep the copies in flight (d = 64 twice as many stages, for the
// same bytes in flight).
#ifndef KVD_TUNE_W8_1
#define KVD_TUNE_W8_1 16
#endif
#ifndef KVD_TUNE_S8_1
#define KVD_TUNE_S8_1 2
#endif
#ifndef KVD_TUNE_W8_2
#define KVD_TUNE_W8_2 8
#endif
#ifndef KVD_TUNE_S8_2
#define KVD_TUNE_S8_2 2
#endif
#ifndef KVD_TUNE_W8_64_1
#define KVD_TUNE_W8_64_1 16
#endif
#ifndef KVD_TUNE_S8_64_1
#define KVD_TUNE_S8_64_1 4
#endif
#ifndef KVD_TUNE_W8_64_2
#define KVD_TUNE_W8_64_2 8
#endif
#ifndef KVD_TUNE_S8_64_2
#define KVD_TUNE_S8_64_2 4
#endif

namespace {
// Largest shared memory one CTA may opt into on sm_100 (227 KB); 1 KB of it is
// left for the kernels' static shared variables.
constexpr size_t kMaxCtaSmem = 232448;

template <int D, int NT>
struct Tune8;
template <>
struct Tune8<128, 1> {
  static constexpr int W = KVD_TUNE_W8_1, S = KVD_TUNE_S8_1;
};
template <>
struct Tune8<128, 2> {
  static constexpr int W = KVD_TUNE_W8_2, S = KVD_TUNE_S8_2;
};
template <>
struct Tune8<64, 1> {
  static constexpr int W = KVD_TUNE_W8_64_1, S = KVD_TUNE_S8_64_1;
};
template <>
struct Tune8<64, 2> {
  static constexpr int W = KVD_TUNE_W8_64_2, S = KVD_TUNE_S8_64_2;
};

// Page policy of an 8-bit launch: one query row per KV head (kG1) packs the
// scale groups into the tile's N columns.
template <int D, int NT, typename T, Code8 kFmt, bool kG1>
using Pol8 = std::conditional_t<kG1, PackedG1<Page8<D, 1, T, kFmt>, D, false, kFmt>, Page8<D, NT, T, kFmt>>;

template <int D, int NT, typename T, Code8 kFmt, int W, int S, bool kG1>
cudaError_t launch_decode8_ws(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                              cudaStream_t st, int grid) {
  using Pol = Pol8<D, NT, T, kFmt, kG1>;
  auto kern = decode_kernel<D, NT, Pol, W, S>;
  const size_t smem = Geo<D, NT, W, S, Pol::kStride, Pol::kAuxBytes>::smem(a.B);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(32 * W), smem, st, a, tmK, tmV);
}

// The tuned ring depth, or one stage per warp when the batch's prefix sums
// (4 bytes per sequence) would push the tuned layout past the CTA limit.
template <int D, int NT, typename T, Code8 kFmt, bool kG1, int W = Tune8<D, NT>::W,
          int S = Tune8<D, NT>::S>
cudaError_t launch_decode8_tg(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                              cudaStream_t st, int grid) {
  using Pol = Pol8<D, NT, T, kFmt, kG1>;
  // one stage must still hold a parked accumulator tile
  constexpr bool kCanShrink = S > 1 && 8 * NT * D * 4 <= Pol::kStride;
  if constexpr (kCanShrink) {
    if (Geo<D, NT, W, S, Pol::kStride, Pol::kAuxBytes>::smem(a.B) + 1024 > kMaxCtaSmem)
      return launch_decode8_ws<D, NT, T, kFmt, W, 1, kG1>(a, tmK, tmV, st, grid);
  }
  return launch_decode8_ws<D, NT, T, kFmt, W, S, kG1>(a, tmK, tmV, st, grid);
}

// One query row per KV head (G = 1) over E4M3 pages at d = 128 takes 12
// warps x 2 stages: its hardware conversion leaves the tile few enough
// instructions that fewer warps hide them, and each keeps its own pages in
// flight.  INT8's conversion runs on the ALU and keeps 16 warps.
// `mha7b` (G = 1), same box, us a call, E4M3 / INT8: 16 x 2 201.6 / 196.5,
// 12 x 2 196.1 / 205.7, 14 x 2 197.9 / 208.2, 12 x 3 198.5 / 204.1,
// 10 x 2 212.7 / 240.0.
template <int D, int NT, typename T, Code8 kFmt>
cudaError_t launch_decode8_t(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                             cudaStream_t st, int grid) {
  if constexpr (NT == 1) {
    if constexpr (D == 128 && kFmt == Code8::E4M3) {
      if (a.G == 1) return launch_decode8_tg<D, 1, T, kFmt, true, 12, 2>(a, tmK, tmV, st, grid);
    }
    if (a.G == 1) return launch_decode8_tg<D, 1, T, kFmt, true>(a, tmK, tmV, st, grid);
  }
  return launch_decode8_tg<D, NT, T, kFmt, false>(a, tmK, tmV, st, grid);
}

// 4-bit cache: d = 128 has 2 KB code stages, d = 64 1 KB; a parked
// accumulator tile (8 NT D floats) must fit in a warp's stages.
#ifndef KVD_TUNE_W4_1
#define KVD_TUNE_W4_1 16
#endif
#ifndef KVD_TUNE_S4_1
#define KVD_TUNE_S4_1 2
#endif
#ifndef KVD_TUNE_W4_2
#define KVD_TUNE_W4_2 8
#endif
#ifndef KVD_TUNE_S4_2
#define KVD_TUNE_S4_2 4
#endif
#ifndef KVD_TUNE_W4_64_1
#define KVD_TUNE_W4_64_1 16
#endif
#ifndef KVD_TUNE_S4_64_1
#define KVD_TUNE_S4_64_1 4
#endif
#ifndef KVD_TUNE_W4_64_2
#define KVD_TUNE_W4_64_2 8
#endif
#ifndef KVD_TUNE_S4_64_2
#define KVD_TUNE_S4_64_2 4
#endif

template <int D, int NT>
struct Tune4;
template <>
struct Tune4<128, 1> {
  static constexpr int W = KVD_TUNE_W4_1, S = KVD_TUNE_S4_1;
};
template <>
struct Tune4<128, 2> {
  static constexpr int W = KVD_TUNE_W4_2, S = KVD_TUNE_S4_2;
};
template <>
struct Tune4<64, 1> {
  static constexpr int W = KVD_TUNE_W4_64_1, S = KVD_TUNE_S4_64_1;
};
template <>
struct Tune4<64, 2> {
  static constexpr int W = KVD_TUNE_W4_64_2, S = KVD_TUNE_S4_64_2;
};

template <int D, int NT, typename T, bool kG1>
cudaError_t launch_decode4_tg(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                              cudaStream_t st, int grid) {
  constexpr int W = Tune4<D, NT>::W, S = Tune4<D, NT>::S;
  using Pol = std::conditional_t<kG1, PackedG1<Page4<D, 1, T>, D, true, Code8::INT4>, Page4<D, NT, T>>;
  auto kern = decode_kernel<D, NT, Pol, W, S>;
  const size_t smem = Geo<D, NT, W, S, Pol::kStride, Pol::kAuxBytes>::smem(a.B);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(32 * W), smem, st, a, tmK, tmV);
}

template <int D, int NT, typename T>
cudaError_t launch_decode4_t(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                             cudaStream_t st, int grid) {
  if constexpr (NT == 1) {
    if (a.G == 1) return launch_decode4_tg<D, 1, T, true>(a, tmK, tmV, st, grid);
  }
  return launch_decode4_tg<D, NT, T, false>(a, tmK, tmV, st, grid);
}

template <int D>
cudaError_t launch_decode4_d(const DecodeArgs &a, DType dt, const CUtensorMap &tmK,
                             const CUtensorMap &tmV, cudaStream_t s, int grid) {
  const bool two = a.G > 8;
  if (dt == DType::BF16)
    return two ? launch_decode4_t<D, 2, __nv_bfloat16>(a, tmK, tmV, s, grid)
               : launch_decode4_t<D, 1, __nv_bfloat16>(a, tmK, tmV, s, grid);
  return two ? launch_decode4_t<D, 2, __half>(a, tmK, tmV, s, grid)
             : launch_decode4_t<D, 1, __half>(a, tmK, tmV, s, grid);
}

template <int D, Code8 kFmt>
cudaError_t launch_decode_q8_fmt(const DecodeArgs &a, DType dt, const CUtensorMap &tmK,
                                 const CUtensorMap &tmV, cudaStream_t s, int grid) {
  const bool two = a.G > 8;
  if (dt == DType::BF16)
    return two ? launch_decode8_t<D, 2, __nv_bfloat16, kFmt>(a, tmK, tmV, s, grid)
               : launch_decode8_t<D, 1, __nv_bfloat16, kFmt>(a, tmK, tmV, s, grid);
  return two ? launch_decode8_t<D, 2, __half, kFmt>(a, tmK, tmV, s, grid)
             : launch_decode8_t<D, 1, __half, kFmt>(a, tmK, tmV, s, grid);
}
}  // namespace

cudaError_t launch_decode_q8(const DecodeArgs &a, int d, DType dt, Code8 fmt, const CUtensorMap &tmK,
                             const CUtensorMap &tmV, cudaStream_t s, int grid) {
  if (fmt == Code8::INT4)
    return d == 64 ? launch_decode4_d<64>(a, dt, tmK, tmV, s, grid)
                   : launch_decode4_d<128>(a, dt, tmK, tmV, s, grid);
  if (d == 64)
    return fmt == Code8::INT8 ? launch_decode_q8_fmt<64, Code8::INT8>(a, dt, tmK, tmV, s, grid)
                              : launch_decode_q8_fmt<64, Code8::E4M3>(a, dt, tmK, tmV, s, grid);
  return fmt == Code8::INT8 ? launch_decode_q8_fmt<128, Code8::INT8>(a, dt, tmK, tmV, s, grid)
                            : launch_decode_q8_fmt<128, Code8::E4M3>(a, dt, tmK, tmV, s, grid);
}

cudaError_t launch_decode(const DecodeArgs &a, int d, DType dt, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, cudaStream_t s, int grid) {
  return dt == DType::BF16 ? launch_decode_dt<__nv_bfloat16>(a, d, tmK, tmV, s, grid)
                           : launch_decode_dt<__half>(a, d, tmK, tmV, s, grid);
}

cudaError_t launch_decode_merge(const DecodeArgs &a, int d, DType dt, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  return dt == DType::BF16 ? launch_merge_dt<__nv_bfloat16>(a, d, s)
                           : launch_merge_dt<__half>(a, d, s);
}

cudaError_t launch_generic_merge(const GenericMergeArgs &a, DType dt, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  return dt == DType::BF16 ? launch_generic_dt<__nv_bfloat16>(a, s)
                           : launch_generic_dt<__half>(a, s);
}

}  // namespace kvd

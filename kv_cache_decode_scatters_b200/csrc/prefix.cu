// prefix.cu -- the shared-prefix pass of decode attention.
//
// "KV缓存与Flash注意力", sections 实际应用 and 练习 (prefix caching: requests that
// share a system prompt or document reuse one copy of its KV), and
// "KV Cache:推理慢的真正原因", section PagedAttention (a block table maps each
// sequence's logical blocks to physical ones, so members of a group point at
// the same physical prefix pages).
//
// Attention is a sum over tokens, so the tokens of a group's shared prefix can
// be attended apart from each member's private suffix and the two results
// merged with their log-sum-exps.  This kernel reads each shared prefix page
// ONCE per (group, KV head) for all members: the group's members x G query
// rows are split over the CTA's warps (8 rows each), all warps consume the
// same staged page.  The page list of a group is cut into `chunks` contiguous
// chunks (one CTA each) for parallelism; every chunk leaves a normalised
// partial (o, lse) per query row.  The private suffixes go through the
// regular decode kernel (its per-sequence `skip`), and the merge kernel folds
// suffix and prefix partials.
//
// Staging: a CTA-wide ring of kStages pages.  Warp 0's lane 0 issues the TMA
// loads (K and V boxes as in the decode kernel) on a "full" mbarrier per
// stage; every warp arrives on the stage's "empty" mbarrier when done with
// it, and the producer waits for that before refilling the stage.
#include "common.cuh"
#include "kernels.h"
#include "tile.cuh"

namespace kvd {

namespace {

constexpr int kWarps = 16;               // warps per CTA, 8 query rows each
constexpr int kRowsPerCta = 8 * kWarps;  // 128
constexpr int kStages = 8;               // pages in flight per CTA (consumed two at a time)

template <int D>
struct PGeo {
  static constexpr int kPageBytes = kPage * D * 2;
  static constexpr int kStageBytes = 2 * kPageBytes;
  static constexpr size_t smem() { return 1024 + (size_t)kStages * kStageBytes + 2 * kStages * 8; }
};

}  // namespace

template <int D, typename T>
__global__ void __launch_bounds__(32 * kWarps, 1)
    prefix_kernel(const PrefixArgs a, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV) {
  using Pg = PGeo<D>;
  constexpr int NT = 1;
  constexpr int kSteps = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)kStages * Pg::kStageBytes);
  uint64_t *empty = full + kStages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, tig = lane & 3;
  const int cap = a.maxb * kPage;

  grid_dependency_wait();
  grid_launch_dependents();

  // Per-sequence shared pages for the suffix pass (one CTA writes them).  A
  // member whose length does not cover the group's pages keeps no shared
  // pages and is attended whole by the decode kernel.
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
    for (int b = tid; b < a.B; b += blockDim.x) a.skip[b] = 0;
    __syncthreads();
    for (int g = 0; g < a.n_groups; ++g) {
      const int s0 = __ldg(a.group_start + g), s1 = __ldg(a.group_start + g + 1);
      const int gp = __ldg(a.group_pages + g);
      for (int b = s0 + tid; b < s1; b += blockDim.x) {
        if (b < 0 || b >= a.B) continue;
        const int n = clamp_len(__ldg(a.seq_lens + b), cap);
        if (gp > 0 && gp * kPage <= n) {
          a.skip[b] = gp;
          // the step's new token must land in a private page
          if (a.fused && gp * kPage == n) flag_error(a.err, kErrSlot);
        }
      }
    }
  }

  const int g = blockIdx.x / a.chunks, chunk = blockIdx.x - g * a.chunks;
  const int h = blockIdx.y;
  const int s0 = __ldg(a.group_start + g), s1 = __ldg(a.group_start + g + 1);
  int gp = __ldg(a.group_pages + g);
  if (s0 < 0 || s1 > a.B || s1 < s0 || gp < 0 || gp > a.maxb) {
    if (tid == 0) flag_error(a.err, kErrSeqLen);
    return;
  }
  const int rows = (s1 - s0) * a.G;
  const int r0 = blockIdx.z * kRowsPerCta;
  if (r0 >= rows || gp == 0) return;  // (rows of ineligible members are ignored by the merge)
  const int p_begin = static_cast<int>((static_cast<long long>(chunk) * gp) / a.chunks);
  const int p_end = static_cast<int>((static_cast<long long>(chunk + 1) * gp) / a.chunks);
  const int npages = p_end - p_begin;

  // this warp's 8 query rows: row -> member m = row / G, head row j = row % G
  uint32_t qf[NT][kSteps][2];
  float acc[NT][kSteps][4];
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int row = r0 + warp * 8 + nt * 8 + g8;
    const bool live = row < rows;
    const int b = s0 + (live ? row / a.G : 0), j = live ? row % a.G : 0;
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(a.q) +
                         (static_cast<size_t>(b) * a.H_q + static_cast<size_t>(h) * a.G + j) * (D / 2);
#pragma unroll
    for (int ks = 0; ks < kSteps; ++ks) {
      qf[nt][ks][0] = live ? __ldg(qw + ks * 8 + tig) : 0u;
      qf[nt][ks][1] = live ? __ldg(qw + ks * 8 + 4 + tig) : 0u;
    }
#pragma unroll
    for (int mt = 0; mt < kSteps; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
  }

  const uint32_t st0 = smem_u32(smem);
  const uint32_t full0 = smem_u32(full), empty0 = smem_u32(empty);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();

  const int32_t *bt = a.block_table + static_cast<size_t>(s0) * a.maxb;  // first member's row
  const uint64_t policy = l2_policy_evict_normal();
  // producer: page k of the chunk into stage k % kStages (warp 0, lane 0)
  auto produce = [&](int k) {
    const int s = k % kStages;
    const uint32_t bar = full0 + 8 * s;
    const int pb = __ldg(bt + p_begin + k);
    if (pb < 0 || pb >= a.num_blocks) {
      flag_error(a.err, kErrBlockTable);
      mbar_arrive(bar);  // completes the phase with no bytes; consumers see a zero page
      return;
    }
    const int row = (pb * a.H_kv + h) * kPage;
    const uint32_t dst = st0 + s * Pg::kStageBytes;
    mbar_arrive_expect_tx(bar, Pg::kStageBytes);
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf) {
      tma_load_3d(dst + hf * kPage * 128, &tmK, 0, hf, row, bar, policy);
      tma_load_3d(dst + Pg::kPageBytes + hf * kPage * 128, &tmV, 0, hf, row, bar, policy);
    }
  };
  if (tid == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    for (int k = 0; k < kStages && k < npages; ++k) produce(k);
  }

  // every warp has released stage s (use `ph`) before it is refilled with page kn
  auto refill = [&](int s, uint32_t ph, int kn) {
    if (kn >= npages) return;
    if (!mbar_wait_bounded(empty0 + 8 * s, ph)) {
      flag_error(a.err, kErrTimeout);
      return;
    }
    produce(kn);
  };

  bool failed = false;
  int k = 0;
  while (k < npages) {
    const bool two = k + 1 < npages;
    const int sA = k % kStages, sB = (k + 1) % kStages;
    const uint32_t phA = (k / kStages) & 1, phB = ((k + 1) / kStages) & 1;
    bool ok = mbar_wait_bounded(full0 + 8 * sA, phA);
    if (two) ok = ok && mbar_wait_bounded(full0 + 8 * sB, phB);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) flag_error(a.err, kErrTimeout);
      failed = true;
      break;
    }
    uint8_t *kA = smem + (size_t)sA * Pg::kStageBytes;
    uint8_t *kB = smem + (size_t)sB * Pg::kStageBytes;
    if (two)
      tile_page2<D, NT, T>(smem_u32(kA), smem_u32(kA + Pg::kPageBytes), smem_u32(kB),
                           smem_u32(kB + Pg::kPageBytes), a.scale_log2, lane, qf, acc, m_run, l_run);
    else
      tile_page<D, NT, T>(smem_u32(kA), smem_u32(kA + Pg::kPageBytes), kPage, a.scale_log2, lane,
                          qf, acc, m_run, l_run);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(empty0 + 8 * sA);
      if (two) mbar_arrive(empty0 + 8 * sB);
    }
    if (tid == 0) {
      refill(sA, phA, k + kStages);
      if (two) refill(sB, phB, k + 1 + kStages);
    }
    __syncwarp();
    k += two ? 2 : 1;
  }
  if (failed) {
    // let the copies in flight land before the CTA exits
    for (int kk = k; kk < npages && kk < k + kStages; ++kk)
      mbar_wait_bounded(full0 + 8 * (kk % kStages), (kk / kStages) & 1);
    return;
  }

  // normalised partial (o, lse) of this chunk for each live row
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float l = l_run[nt][i];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      const int row = r0 + warp * 8 + nt * 8 + 2 * tig + i;
      if (row >= rows) continue;
      const int b = s0 + row / a.G, j = row % a.G;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse = l > 0.f ? (m_run[nt][i] + fast_log2(l)) * kLn2 : -INFINITY;
      const size_t idx = ((static_cast<size_t>(chunk) * a.H_kv + h) * a.B + b) * a.G + j;
      float *o = a.pre_o + idx * D;
#pragma unroll
      for (int mt = 0; mt < kSteps; ++mt) {
        o[mt * 16 + g8] = acc[nt][mt][i] * inv;
        o[mt * 16 + 8 + g8] = acc[nt][mt][2 + i] * inv;
      }
      if (g8 == 0) a.pre_lse[idx] = lse;
    }
  }
}

int prefix_rows_per_cta() { return kRowsPerCta; }

namespace {
template <int D, typename T>
cudaError_t launch_prefix_t(const PrefixArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                            int row_blocks, cudaStream_t st) {
  auto kern = prefix_kernel<D, T>;
  const size_t smem = PGeo<D>::smem();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_groups * a.chunks, a.H_kv, row_blocks);
  return launch_pdl(kern, grid, dim3(32 * kWarps), smem, st, a, tmK, tmV);
}
}  // namespace

cudaError_t launch_prefix(const PrefixArgs &a, int d, DType dt, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, int row_blocks, cudaStream_t s) {
  if (a.n_groups == 0 || a.B == 0) return cudaSuccess;
  if (dt == DType::BF16)
    return d == 128 ? launch_prefix_t<128, __nv_bfloat16>(a, tmK, tmV, row_blocks, s)
                    : launch_prefix_t<64, __nv_bfloat16>(a, tmK, tmV, row_blocks, s);
  return d == 128 ? launch_prefix_t<128, __half>(a, tmK, tmV, row_blocks, s)
                  : launch_prefix_t<64, __half>(a, tmK, tmV, row_blocks, s);
}

}  // namespace kvd

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
// Scheduling: a one-CTA plan launch writes `skip` and the suffix decode's
// partition count; the decode runs next and leaves the prefix pass a share
// of the SMs sized by the two passes' page counts and costs; this pass is
// launched after the decode, scheduled as soon as the decode has started, so
// the two stream side by side; the merge comes last.
//
// Staging: a CTA-wide ring of kStages pages.  Warp 0's lane 0 issues the TMA
// loads (K and V boxes as in the decode kernel) on a "full" mbarrier per
// stage; every warp arrives on the stage's "empty" mbarrier when done with
// it, and the producer waits for that before refilling the stage.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tile.cuh"

#include <type_traits>

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

// A group whose bounds leave [0, B], that has more members than the
// launch was sized for (maxg) or a shared page count outside the table is
// invalid: the prefix pass skips it and its members are attended whole.
__device__ __forceinline__ bool group_ok(const PrefixArgs &a, int s0, int s1, int gp) {
  return s0 >= 0 && s1 <= a.B && s1 >= s0 && s1 - s0 <= a.maxg && gp >= 0 && gp <= a.maxb;
}

// Per-sequence shared pages for the suffix pass (the plan launch writes
// them, all threads of its one CTA).  A member whose length does not cover
// the group's pages keeps no shared pages and is attended whole by the decode
// kernel; so do the members of an invalid group.
__device__ void write_skip(const PrefixArgs &a, int cap) {
  const int tid = threadIdx.x;
  for (int b = tid; b < a.B; b += blockDim.x) a.skip[b] = 0;
  __syncthreads();
  for (int g = 0; g < a.n_groups; ++g) {
    const int s0 = __ldg(a.group_start + g), s1 = __ldg(a.group_start + g + 1);
    const int gp = __ldg(a.group_pages + g);
    if (!group_ok(a, s0, s1, gp)) continue;  // flagged by the group's CTAs
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

// Counts a warp of the prefix pass as finished; the last one waits for the
// decode grid launched before this pass.  The pass does not wait for that
// grid at its start (the two share no buffer, so they run side by side), but
// the merge launched after the pass reads the decode's partials too: it
// waits for this grid, which then cannot complete before the decode has.
__device__ __forceinline__ void prefix_exit(const PrefixArgs &a) {
  if ((threadIdx.x & 31) == 0) {
    const unsigned long long warps = static_cast<unsigned long long>(gridDim.x) * gridDim.y *
                                     gridDim.z * (blockDim.x >> 5);
    unsigned long long *done = reinterpret_cast<unsigned long long *>(a.plan + 2);
    if (atomicAdd(done, 1ull) + 1ull == warps) grid_dependency_wait();
  }
}

constexpr int kPlanThreads = 256;
constexpr int kPlanGroups = 2048;  // groups the plan stages in shared memory

// Sums of v[0..2] over the CTA (kPlanThreads threads); every thread gets them.
__device__ void plan_sum3(long long (&v)[3], long long (*red)[3]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 3; ++i)
    for (int o = 16; o; o >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  if (lane == 0)
    for (int i = 0; i < 3; ++i) red[warp][i] = v[i];
  __syncthreads();
  for (int i = 0; i < 3; ++i) {
    v[i] = 0;
    for (int w = 0; w < kPlanThreads / 32; ++w) v[i] += red[w][i];
  }
}

}  // namespace

// The plan of a shared-prefix call, one CTA ahead of the decode launch:
//  * skip[b], the shared pages of sequence b the prefix pass attends;
//  * plan[0], the partitions the suffix decode uses.  With weight w > 0 the
//    decode takes the share of the nparts SMs that its pages are of the
//    whole work, P / (P + w * Pp), with P the suffix pages and Pp the prefix
//    pages (per KV head and row block); its other CTAs exit at once and the
//    prefix pass, launched next, runs on their SMs meanwhile.  The prefix
//    SMs are then adjusted so that the pass's CTAs fill whole waves there:
//    a part-filled last wave would leave them idle while the decode runs;
//  * plan[2..3] = 0, the prefix pass's count of finished warps.
// The decode launch waits for this one, so its latency is on the step's
// critical path: with non-decreasing group starts (and at most kPlanGroups
// groups) every sequence finds its group by a binary search over the starts
// staged in shared memory, all sequences at once; otherwise write_skip walks
// the groups in order.
__global__ void __launch_bounds__(kPlanThreads) prefix_plan_kernel(const PrefixArgs a) {
  __shared__ int g_start[kPlanGroups + 1];
  __shared__ int g_pages[kPlanGroups];
  __shared__ long long red[kPlanThreads / 32][3];
  grid_dependency_wait();
  grid_launch_dependents();
  const int tid = threadIdx.x;
  const int cap = a.maxb * kPage;
  const bool staged = a.n_groups <= kPlanGroups;
  int unordered = 0;
  if (staged) {
    for (int g = tid; g <= a.n_groups; g += kPlanThreads) g_start[g] = __ldg(a.group_start + g);
    for (int g = tid; g < a.n_groups; g += kPlanThreads) g_pages[g] = __ldg(a.group_pages + g);
    __syncthreads();
    for (int g = tid; g < a.n_groups; g += kPlanThreads) unordered |= g_start[g + 1] < g_start[g];
  }
  const bool search = __syncthreads_or(unordered) == 0 && staged;
  if (!search) {
    write_skip(a, cap);
    __syncthreads();  // skip[] of every sequence written (by other threads too)
  }
  long long v[3] = {0, 0, 0};  // suffix pages, prefix pages, prefix row blocks
  for (int b = tid; b < a.B; b += kPlanThreads) {
    const int n = clamp_len(__ldcg(a.seq_lens + b), cap);
    int sk;
    if (search) {
      // the last group starting at or before b holds it, if b is below its end
      int lo = 0, hi = a.n_groups;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (g_start[mid] <= b) lo = mid + 1; else hi = mid;
      }
      const int g = lo - 1;
      sk = 0;
      if (g >= 0 && b < g_start[g + 1]) {
        const int gp = g_pages[g];
        if (group_ok(a, g_start[g], g_start[g + 1], gp) && gp > 0 && gp * kPage <= n) {
          sk = gp;
          // the step's new token must land in a private page
          if (a.fused && gp * kPage == n) flag_error(a.err, kErrSlot);
        }
      }
      a.skip[b] = sk;
    } else {
      sk = __ldcg(a.skip + b);
    }
    v[0] += max(0, (n + kPage - 1) / kPage - sk);
  }
  for (int g = tid; g < a.n_groups; g += kPlanThreads) {
    const int s0 = staged ? g_start[g] : __ldg(a.group_start + g);
    const int s1 = staged ? g_start[g + 1] : __ldg(a.group_start + g + 1);
    const int gp = staged ? g_pages[g] : __ldg(a.group_pages + g);
    if (!group_ok(a, s0, s1, gp) || gp == 0) continue;
    const long long rows = static_cast<long long>(s1 - s0) * a.G;
    const long long rb = (rows + kRowsPerCta - 1) / kRowsPerCta;
    v[1] += gp * rb;
    v[2] += rb;
  }
  plan_sum3(v, red);
  if (tid == 0) {
    const long long P = v[0] * a.H_kv, Pp = v[1] * a.H_kv;
    int N = effective_parts(P, a.nparts, a.min_pages);
    if (a.weight > 0.f && Pp > 0 && a.nparts > 1) {
      const double dp = static_cast<double>(P);
      const double share = dp / (dp + a.weight * static_cast<double>(Pp));
      const double k_raw = fmax(1.0, a.nparts * (1.0 - share));  // SMs for the prefix pass
      const long long ctas = v[2] * a.chunks * a.H_kv;             // its CTAs with work
      const long long slots = a.ctas_per_sm;                        // resident per SM
      const long long waves = max(1LL, llround(static_cast<double>(ctas) / (slots * k_raw)));
      const long long k =
          min(static_cast<long long>(a.nparts - 1), (ctas + slots * waves - 1) / (slots * waves));
      N = min(N, max(1, a.nparts - static_cast<int>(k)));
    }
    a.plan[0] = N;
    a.plan[1] = 0;
    *reinterpret_cast<unsigned long long *>(a.plan + 2) = 0ull;
  }
}

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

  // no wait for the decode launch before this pass (prefix_exit); every
  // return of the body below still passes through prefix_exit
  grid_launch_dependents();
  [&] {
    const int g = blockIdx.x / a.chunks, chunk = blockIdx.x - g * a.chunks;
    const int h = blockIdx.y;
    const int s0 = __ldg(a.group_start + g), s1 = __ldg(a.group_start + g + 1);
    int gp = __ldg(a.group_pages + g);
    if (!group_ok(a, s0, s1, gp)) {
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
        const uint64_t keep = l2_policy_evict_last();  // read again by the merge
  #pragma unroll
        for (int mt = 0; mt < kSteps; ++mt) {
          st_keep(o + mt * 16 + g8, acc[nt][mt][i] * inv, keep);
          st_keep(o + mt * 16 + 8 + g8, acc[nt][mt][2 + i] * inv, keep);
        }
        if (g8 == 0) st_keep(a.pre_lse + idx, lse, keep);
      }
    }
  }();
  prefix_exit(a);
}

// ------------------------------------------------------------------------
// The warp-level pass over a quantised cache (E4M3, INT8 or INT4 codes with
// one fp32 scale per token, KV head and 32 channels), used at d = 64 where the
// tensor-memory pass does not apply.  Same structure as prefix_kernel: a
// CTA-wide ring of kStages pages, warp 0's lane 0 copying each page's K and V
// code boxes (2-D TMA, swizzled by the code row size) and its two scale rows
// (bulk copies) onto the stage's "full" mbarrier, every warp running the
// quantised tile (tile_page_q8 / tile_page_q4, exact code values, fp32
// scales) for its 8 query rows, one page at a time.
namespace {
template <int D, Code8 kFmt>
struct PQGeo {
  static constexpr int kRow = kFmt == Code8::INT4 ? D / 2 : D;  // code bytes of a token
  static constexpr int kCodePage = kPage * kRow;
  static constexpr int kScalePage = kPage * (D / 32) * 4;
  // codes of K then V, then the scales of K then V, padded to keep the
  // code boxes on their swizzle alignment
  static constexpr int kStageBytes = ((2 * kCodePage + 2 * kScalePage + 1023) / 1024) * 1024;
  static constexpr size_t smem() { return 1024 + (size_t)kStages * kStageBytes + 2 * kStages * 8; }
};
}  // namespace

template <int D, typename T, Code8 kFmt>
__global__ void __launch_bounds__(32 * kWarps, 1)
    prefix_q_kernel(const PrefixArgs a, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV) {
  using Pg = PQGeo<D, kFmt>;
  constexpr int kSteps = D / 16;
  constexpr bool kInt4 = kFmt == Code8::INT4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)kStages * Pg::kStageBytes);
  uint64_t *empty = full + kStages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, tig = lane & 3;

  // no wait for the decode launch before this pass (prefix_exit); every
  // return of the body below still passes through prefix_exit
  grid_launch_dependents();
  [&] {
    const int g = blockIdx.x / a.chunks, chunk = blockIdx.x - g * a.chunks;
    const int h = blockIdx.y;
    const int s0 = __ldg(a.group_start + g), s1 = __ldg(a.group_start + g + 1);
    const int gp = __ldg(a.group_pages + g);
    if (!group_ok(a, s0, s1, gp)) {
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
    uint32_t qf[1][kSteps][2];
    float acc[1][kSteps][4];
    float m_run[1][2], l_run[1][2];
    {
      const int row = r0 + warp * 8 + g8;
      const bool live = row < rows;
      const int b = s0 + (live ? row / a.G : 0), j = live ? row % a.G : 0;
      const uint32_t *qw = reinterpret_cast<const uint32_t *>(a.q) +
                           (static_cast<size_t>(b) * a.H_q + static_cast<size_t>(h) * a.G + j) * (D / 2);
  #pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        if (live) {
          if constexpr (kInt4) q_words_q4<T>(qw, ks, tig, qf[0][ks][0], qf[0][ks][1]);
          else q_words_q8<T>(qw, ks, tig, qf[0][ks][0], qf[0][ks][1]);
        } else {
          qf[0][ks][0] = qf[0][ks][1] = 0u;
        }
      }
  #pragma unroll
      for (int mt = 0; mt < kSteps; ++mt)
  #pragma unroll
        for (int e = 0; e < 4; ++e) acc[0][mt][e] = 0.f;
      m_run[0][0] = m_run[0][1] = -INFINITY;
      l_run[0][0] = l_run[0][1] = 0.f;
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
    constexpr int kG = D / 32;
    // producer: page k of the chunk into stage k % kStages (warp 0, lane 0)
    auto produce = [&](int k) {
      const int s = k % kStages;
      const uint32_t bar = full0 + 8 * s;
      const int pb = __ldg(bt + p_begin + k);
      if (pb < 0 || pb >= a.num_blocks) {
        flag_error(a.err, kErrBlockTable);
        mbar_arrive(bar);  // completes the phase with no bytes; consumers skip the page
        return;
      }
      const int row = (pb * a.H_kv + h) * kPage;
      const uint32_t dst = st0 + s * Pg::kStageBytes;
      mbar_arrive_expect_tx(bar, 2 * Pg::kCodePage + 2 * Pg::kScalePage);
      tma_load_2d(dst, &tmK, 0, row, bar, policy);
      tma_load_2d(dst + Pg::kCodePage, &tmV, 0, row, bar, policy);
      bulk_load(dst + 2 * Pg::kCodePage, a.k_scale + static_cast<size_t>(row) * kG, Pg::kScalePage, bar);
      bulk_load(dst + 2 * Pg::kCodePage + Pg::kScalePage, a.v_scale + static_cast<size_t>(row) * kG,
                Pg::kScalePage, bar);
    };
    if (tid == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      for (int k = 0; k < kStages && k < npages; ++k) produce(k);
    }

    bool failed = false;
    int k = 0;
    for (; k < npages; ++k) {
      const int s = k % kStages;
      const uint32_t ph = (k / kStages) & 1;
      const bool ok = mbar_wait_bounded(full0 + 8 * s, ph);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) flag_error(a.err, kErrTimeout);
        failed = true;
        break;
      }
      const int pb = __ldg(bt + p_begin + k);
      if (pb >= 0 && pb < a.num_blocks) {  // (a page outside the pool was flagged and not copied)
        uint8_t *st = smem + (size_t)s * Pg::kStageBytes;
        const float *ks = reinterpret_cast<const float *>(st + 2 * Pg::kCodePage);
        if constexpr (kInt4)
          tile_page_q4<D, 1>(smem_u32(st), smem_u32(st + Pg::kCodePage), ks, ks + kPage * kG, kPage,
                             a.scale_log2, lane, qf, acc, m_run, l_run);
        else
          tile_page_q8<D, 1, kFmt>(smem_u32(st), smem_u32(st + Pg::kCodePage), ks, ks + kPage * kG,
                                   kPage, a.scale_log2, lane, qf, acc, m_run, l_run);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      if (tid == 0 && k + kStages < npages) {
        // every warp has released stage s before it is refilled
        if (mbar_wait_bounded(empty0 + 8 * s, ph)) produce(k + kStages);
        else flag_error(a.err, kErrTimeout);
      }
    }
    if (failed) {
      // let the copies in flight land before the CTA exits
      for (int kk = k; kk < npages && kk < k + kStages; ++kk)
        mbar_wait_bounded(full0 + 8 * (kk % kStages), (kk / kStages) & 1);
      return;
    }

    // normalised partial (o, lse) of this chunk for each live row
  #pragma unroll
    for (int i = 0; i < 2; ++i) {
      float l = l_run[0][i];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      const int row = r0 + warp * 8 + 2 * tig + i;
      if (row >= rows) continue;
      const int b = s0 + row / a.G, j = row % a.G;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse = l > 0.f ? (m_run[0][i] + fast_log2(l)) * kLn2 : -INFINITY;
      const size_t idx = ((static_cast<size_t>(chunk) * a.H_kv + h) * a.B + b) * a.G + j;
      float *o = a.pre_o + idx * D;
      const uint64_t keep = l2_policy_evict_last();  // read again by the merge
  #pragma unroll
      for (int mt = 0; mt < kSteps; ++mt) {
        const int c0 = kInt4 ? dim_q4(mt, i, g8) : dim_q8(mt, i, g8);
        const int c2 = kInt4 ? dim_q4(mt, 2 + i, g8) : dim_q8(mt, 2 + i, g8);
        st_keep(o + c0, acc[0][mt][i] * inv, keep);
        st_keep(o + c2, acc[0][mt][2 + i] * inv, keep);
      }
      if (g8 == 0) st_keep(a.pre_lse + idx, lse, keep);
    }
  }();
  prefix_exit(a);
}

// ------------------------------------------------------------------------
// The same pass on the 5th-generation tensor cores (d = 128).
//
// The 128 query rows of a CTA are the M dimension of tcgen05.mma, so every
// staged K/V byte is read from shared memory once by the tensor core for all
// rows (the warp-level tile above re-reads each page once per warp).  Per
// step of kTcPages pages (N = 64 tokens):
//   S[128 x N]  = Q[128 x d] . K^T      Q and K page rows in smem
//   softmax     one thread per row reads its S row from TMEM, keeps the
//               running (max, sum) and writes P (16-bit) over that S in TMEM
//   O[128 x d] += P[128 x N] . V         P in TMEM (A), V rows in smem (B)
// with fp32 accumulators S and O in TMEM.  The running max is a reference
// that only moves when a row's maximum exceeds it by more than 2^8; below
// that the probabilities stay <= 256 (exact enough in f16/bf16 and fp32), so
// O is rescaled in TMEM only on the rare steps that move it.
//
// Each CTA takes half of TMEM (O and two S/P buffers, 256 columns) and about
// 100 KB of shared memory, so two CTAs share an SM and one's softmax overlaps
// the other's MMAs and copies.
//
// Roles (192 threads): warp 0 allocates TMEM and its lane 0 issues the TMA
// loads of K/V into a kTcStages-deep ring; warp 1 lane 0 issues the MMAs;
// warps 2-5 (TMEM lane quarters 2, 3, 0, 1) do the softmax, the O
// corrections and the epilogue.  Hand-offs are mbarriers: TMA -> MMA (one
// "full" barrier for the K half and one for the V half of a stage), MMA ->
// TMA ("empty": a stage's K is released once QK^T has read it, its V after
// the PV product, so the next K copy starts a whole step earlier), MMA ->
// softmax (s_full), softmax -> MMA (p_full), and o_done (one phase per PV
// product) before the softmax touches O.  The S/P buffers are double
// buffered so QK^T of step j+1 runs during the softmax of step j; QK^T of
// step j+2 overwrites the P of step j only after the PV product reading it
// (MMAs of one thread run in issue order).
// Every wait is bounded; a timed-out role flags the error word and the CTA
// still releases its TMEM after the MMAs it issued have completed.
namespace {
constexpr int kTcPages = 4;                       // pages per step
constexpr int kTcTok = kTcPages * kPage;          // N of QK^T: 64 tokens
constexpr int kTcStages = 2;                      // steps of K/V in flight per CTA
constexpr int kTcWarps = 6;
constexpr int kTcHalf = kTcPages * kPage * 128;   // one 64-column half of a step's K (or V): 8 KB
constexpr int kTcStage = 4 * kTcHalf;             // K half 0, K half 1, V half 0, V half 1
constexpr int kTcQBytes = kRowsPerCta * 128 * 2;  // Q tile, two 64-column halves: 32 KB
constexpr uint32_t kColO = 0;                     // O: 128 fp32 columns
constexpr uint32_t kColS = 128;                   // S: 2 x 64 fp32 columns; P overwrites S
constexpr uint32_t kTmemCols = 256;
// the quantised pass (one CTA per SM, all of TMEM): O, two S buffers of
// 2 kTcTok columns (scores against the heads, then the remainders), Q
constexpr uint32_t kColQ = kColS + 2 * 2 * kTcTok;  // 384: Q, 64 columns
constexpr uint32_t kTmemColsQ = 512;
constexpr float kRefSlack = 8.f;                  // log2 of the largest probability kept
constexpr int kTcBars = 4 * kTcStages + 7;
constexpr size_t kTcSmem = 1024 + kTcQBytes + (size_t)kTcStages * kTcStage + kTcBars * 8 + 64;
// two CTAs per SM share its 512 TMEM columns; a third never fits beside them
static_assert(2 * kTcSmem <= 227 * 1024 && 3 * kTcSmem > 228 * 1024,
              "exactly two CTAs per SM: each allocates half of TMEM");
}  // namespace

// The block-table entries of one step of a chunk [p_begin, p_end), loaded
// a step ahead of their use so that the loads' latency is not waited for:
// load(j) issues the loads, mask() (one step later) says which pages of the
// step exist (bit p: page p has a valid physical page; 0 past the last step).
struct StepPages {
  int pb[kTcPages];
  __device__ __forceinline__ void load(const int32_t *bt, int p_begin, int p_end, int nsteps, int j) {
    const int p0 = p_begin + j * kTcPages, np = j < nsteps ? min(kTcPages, p_end - p0) : 0;
#pragma unroll
    for (int p = 0; p < kTcPages; ++p) pb[p] = p < np ? __ldg(bt + p0 + p) : -1;
  }
  __device__ __forceinline__ uint32_t mask(const PrefixArgs &a) const {
    uint32_t m = 0;
#pragma unroll
    for (int p = 0; p < kTcPages; ++p)
      if (pb[p] >= 0 && pb[p] < a.num_blocks) m |= 1u << p;
    return m;
  }
};

// The softmax role of the tensor-memory passes (4 warps, one query row per
// thread): puts its rows of Q where the QK^T MMAs read them, then per step
// reads its S row from TMEM, updates the running (max, sum), writes P over S,
// rescales O in TMEM when the reference max moves, and finally writes the
// normalised partial (o, lse) of its row.
//  * kSplit = false (16-bit pages): Q into the K-major, 128-byte-swizzled
//    shared-memory tile qs; S buffers of kTcTok columns.
//  * kSplit = true (quantised pages, head + remainder operands): Q into TMEM
//    columns kColQ.. (the MMA's A operand); S buffers of 2 kTcTok columns,
//    the scores against the heads then against the remainders, summed here.
template <typename T, bool kSplit = false>
__device__ __forceinline__ void tc_softmax_role(const PrefixArgs &a, uint8_t *qs, uint32_t tbase,
                                                uint32_t S_FULL, uint32_t P_FULL, uint32_t O_DONE,
                                                uint32_t Q_FULL, int warp, int lane, int r0, int rows,
                                                int s0, int h, int chunk, int nsteps,
                                                const int32_t *bt, int p_begin, int p_end) {
  constexpr int D = 128;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using M = Mma<T>;
  const int quarter = warp & 3;
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  const int row = r0 + quarter * 32 + lane;  // row of the group: member row / G, head row % G
  const bool live = row < rows;
  const int b = s0 + (live ? row / a.G : 0), jr = live ? row % a.G : 0;
  constexpr int kSb = kSplit ? 2 * kTcTok : kTcTok;  // TMEM columns of one S buffer
  {
    const uint4 *qv = reinterpret_cast<const uint4 *>(
        static_cast<const T *>(a.q) +
        (static_cast<size_t>(b) * a.H_q + static_cast<size_t>(h) * a.G + jr) * D);
    if constexpr (kSplit) {
      // this row of Q into its TMEM lane: column c holds channels 2c, 2c + 1
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = live ? __ldg(qv + hf * 8 + c) : make_uint4(0u, 0u, 0u, 0u);
          r[4 * c] = v.x;
          r[4 * c + 1] = v.y;
          r[4 * c + 2] = v.z;
          r[4 * c + 3] = v.w;
        }
        tc::st32(tbase + lanes + kColQ + hf * 32, r);
      }
      tc::wait_st();
      tc::fence_before_sync();
    } else {
      // this row of Q into the K-major, 128-byte-swizzled tile the MMA reads
      const int r = quarter * 32 + lane;
#pragma unroll
      for (int c = 0; c < 2 * 8; ++c) {
        const uint4 v = live ? __ldg(qv + c) : make_uint4(0u, 0u, 0u, 0u);
        const int half = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4 *>(qs + half * (kTcQBytes / 2) + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();  // visible to the tensor core's reads
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(Q_FULL);
  }

  float m_ref = -INFINITY, l = 0.f;
  bool ok = true;
  StepPages ahead;
  ahead.load(bt, p_begin, p_end, nsteps, 0);
  uint32_t next_mask = ahead.mask(a);  // the mask of step j + 1 during step j
  ahead.load(bt, p_begin, p_end, nsteps, 1);
  for (int j = 0; j < nsteps; ++j) {
    const int bs = j & 1;
    const uint32_t pm = next_mask;
    next_mask = ahead.mask(a);
    ahead.load(bt, p_begin, p_end, nsteps, j + 2);
    const bool got = mbar_wait_bounded(S_FULL + 8 * bs, (j >> 1) & 1);
    if (!__all_sync(0xffffffffu, got)) {
      ok = false;
      break;
    }
    tc::fence_after_sync();
    float x[kTcTok];
    {
      uint32_t r0v[32], r1v[32];
      tc::ld32(tbase + lanes + kColS + bs * kSb, r0v);
      tc::ld32(tbase + lanes + kColS + bs * kSb + 32, r1v);
      tc::wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        x[i] = __uint_as_float(r0v[i]);
        x[32 + i] = __uint_as_float(r1v[i]);
      }
      if constexpr (kSplit) {
        tc::ld32(tbase + lanes + kColS + bs * kSb + kTcTok, r0v);
        tc::ld32(tbase + lanes + kColS + bs * kSb + kTcTok + 32, r1v);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] += __uint_as_float(r0v[i]);
          x[32 + i] += __uint_as_float(r1v[i]);
        }
      }
    }
    // row maximum of the scaled scores (in log2 units): the scale is folded
    // into the exponent below, so the raw scores are compared (their
    // minimum when the scale is negative); masked columns are -inf
    const float c = a.scale_log2;
    const bool full_step = pm == (1u << kTcPages) - 1u;  // warp-uniform
    if (!full_step) {
#pragma unroll
      for (int i = 0; i < kTcTok; ++i)
        if (!((pm >> (i / kPage)) & 1u)) x[i] = c >= 0.f ? -INFINITY : INFINITY;
    }
    float e4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) e4[k] = x[k];
    if (c >= 0.f) {
#pragma unroll
      for (int i = 4; i < kTcTok; ++i) e4[i & 3] = fmaxf(e4[i & 3], x[i]);
    } else {
#pragma unroll
      for (int i = 4; i < kTcTok; ++i) e4[i & 3] = fminf(e4[i & 3], x[i]);
    }
    const float ext = c >= 0.f ? fmaxf(fmaxf(e4[0], e4[1]), fmaxf(e4[2], e4[3]))
                               : fminf(fminf(e4[0], e4[1]), fminf(e4[2], e4[3]));
    // an all-masked row keeps -inf; otherwise the largest scaled score
    const float mx = (ext == INFINITY || ext == -INFINITY) ? -INFINITY : ext * c;
    const float m_new = mx > m_ref + kRefSlack ? mx : m_ref;
    const float alpha = m_new == m_ref ? 1.f : fast_exp2(m_ref - m_new);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    uint32_t ph[kTcTok / 2], pl[kTcTok / 2];
    float sum4[4] = {0.f, 0.f, 0.f, 0.f};
    // exp2(s * c - m) per column; masked columns (partial steps only) are 0
    auto exps = [&](auto masked) {
#pragma unroll
      for (int i = 0; i < kTcTok; i += 2) {
        float e0 = fast_exp2(fmaf(x[i], c, -m_use));
        float e1 = fast_exp2(fmaf(x[i + 1], c, -m_use));
        if constexpr (decltype(masked)::value) {
          const bool v = (pm >> (i / kPage)) & 1u;  // both columns are in one page
          e0 = v ? e0 : 0.f;
          e1 = v ? e1 : 0.f;
        }
        ph[i / 2] = M::pack(e0, e1);
        if constexpr (kBf16) {
          const float2 r = M::unpack(ph[i / 2]);
          pl[i / 2] = M::pack(e0 - r.x, e1 - r.y);
        }
        sum4[(i / 2) & 3] += e0 + e1;
      }
    };
    if (full_step) exps(std::false_type{});
    else exps(std::true_type{});
    const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
    l = l * alpha + sum;
    tc::st32(tbase + lanes + kColS + bs * kSb, ph);
    if constexpr (kBf16) tc::st32(tbase + lanes + kColS + bs * kSb + kTcTok / 2, pl);
    if (j >= 1) {
      // O holds the product of step j-1 once its o_done phase completes
      const bool got2 = mbar_wait_bounded(O_DONE, (j - 1) & 1);
      if (!__all_sync(0xffffffffu, got2)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tc::ld32(tbase + lanes + kColO + c * 32, r);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tc::st32(tbase + lanes + kColO + c * 32, r);
        }
      }
    }
    m_ref = m_new;
    tc::wait_st();
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(P_FULL + 8 * bs);
  }
  if (ok) {
    const bool got = mbar_wait_bounded(O_DONE, (nsteps - 1) & 1);
    ok = __all_sync(0xffffffffu, got);
  }
  if (!ok) {
    if (lane == 0) flag_error(a.err, kErrTimeout);
  } else {
    tc::fence_after_sync();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float lse = l > 0.f ? (m_ref + fast_log2(l)) * kLn2 : -INFINITY;
    const size_t idx = ((static_cast<size_t>(chunk) * a.H_kv + h) * a.B + b) * a.G + jr;
    float4 *o = reinterpret_cast<float4 *>(a.pre_o + idx * D);
    const uint64_t keep = l2_policy_evict_last();  // read again by the merge
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tc::ld32(tbase + lanes + kColO + c * 32, r);
      tc::wait_ld();
      if (live) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 v = l > 0.f ? make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                                                 __uint_as_float(r[i + 2]) * inv,
                                                 __uint_as_float(r[i + 3]) * inv)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
          st_keep4(o + c * 8 + i / 4, v, keep);
        }
      }
      __syncwarp();
    }
    if (live) st_keep(a.pre_lse + idx, lse, keep);
  }
}

template <typename T>
__global__ void __launch_bounds__(32 * kTcWarps, 2)
    prefix_tc_kernel(const PrefixArgs a, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV) {
  constexpr int D = 128;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *qs = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint8_t *ring = qs + kTcQBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring + (size_t)kTcStages * kTcStage);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kTcBars);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // no wait for the decode launch before this pass (prefix_exit); every
  // return of the body below still passes through prefix_exit
  grid_launch_dependents();
  [&] {
    const int g = blockIdx.x / a.chunks, chunk = blockIdx.x - g * a.chunks;
    const int h = blockIdx.y;
    const int s0 = __ldg(a.group_start + g), s1 = __ldg(a.group_start + g + 1);
    const int gp = __ldg(a.group_pages + g);
    if (!group_ok(a, s0, s1, gp)) {
      if (tid == 0) flag_error(a.err, kErrSeqLen);
      return;
    }
    const int rows = (s1 - s0) * a.G;
    const int r0 = blockIdx.z * kRowsPerCta;
    if (r0 >= rows || gp == 0) return;
    const int p_begin = static_cast<int>((static_cast<long long>(chunk) * gp) / a.chunks);
    const int p_end = static_cast<int>((static_cast<long long>(chunk + 1) * gp) / a.chunks);
    const int nsteps = (p_end - p_begin + kTcPages - 1) / kTcPages;
    if (nsteps == 0) {  // an empty chunk leaves empty partials
      for (int r = tid; r < kRowsPerCta; r += blockDim.x) {
        const int row = r0 + r;
        if (row >= rows) continue;
        const size_t idx = ((static_cast<size_t>(chunk) * a.H_kv + h) * a.B + s0 + row / a.G) * a.G +
                           row % a.G;
        for (int c = 0; c < D; ++c) a.pre_o[idx * D + c] = 0.f;
        a.pre_lse[idx] = -INFINITY;
      }
      return;
    }
    const int32_t *bt = a.block_table + static_cast<size_t>(s0) * a.maxb;  // first member's row
    auto step_pages = [&](int j) { return min(kTcPages, p_end - (p_begin + j * kTcPages)); };

    const uint32_t q0 = smem_u32(qs), ring0 = smem_u32(ring), bar0 = smem_u32(bars);
    // K and V halves of a stage have their own barriers: K is released as soon
    // as QK^T has read it, V after the PV product
    auto FULL_K = [&](int s) { return bar0 + 8 * s; };
    auto FULL_V = [&](int s) { return bar0 + 8 * (kTcStages + s); };
    auto EMPTY_K = [&](int s) { return bar0 + 8 * (2 * kTcStages + s); };
    auto EMPTY_V = [&](int s) { return bar0 + 8 * (3 * kTcStages + s); };
    const uint32_t S_FULL = bar0 + 8 * (4 * kTcStages);  // + 8 * buffer
    const uint32_t P_FULL = S_FULL + 16;                 // + 8 * buffer
    const uint32_t O_DONE = S_FULL + 32, Q_FULL = S_FULL + 40, DRAIN = S_FULL + 48;

    if (warp == 0) {
      __syncwarp();
      tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
      tc::tmem_relinquish();
    }
    if (tid == 32) {
      for (int s = 0; s < kTcStages; ++s) {
        mbar_init(FULL_K(s), 1);
        mbar_init(FULL_V(s), 1);
        mbar_init(EMPTY_K(s), 1);
        mbar_init(EMPTY_V(s), 1);
      }
      mbar_init(S_FULL, 1);
      mbar_init(S_FULL + 8, 1);
      mbar_init(P_FULL, 4);
      mbar_init(P_FULL + 8, 4);
      mbar_init(O_DONE, 1);
      mbar_init(Q_FULL, 4);
      mbar_init(DRAIN, 1);
      mbar_init_fence();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(tmem_slot);

    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        const uint64_t policy = l2_policy_evict_normal();
        int issued_k = 0, issued_v = 0;
        for (int j = 0; j < nsteps; ++j) {
          const int s = j % kTcStages;
          const uint32_t rel = ((j / kTcStages) - 1) & 1;  // phase of step j - kTcStages
          const int p0 = p_begin + j * kTcPages, np = step_pages(j);
          int prow[kTcPages];
          int good = 0;
  #pragma unroll
          for (int p = 0; p < kTcPages; ++p) {
            prow[p] = -1;
            if (p < np) {
              const int pb = __ldg(bt + p0 + p);
              if (pb >= 0 && pb < a.num_blocks) {
                prow[p] = (pb * a.H_kv + h) * kPage;
                ++good;
              } else {
                flag_error(a.err, kErrBlockTable);
              }
            }
          }
          const uint32_t st = ring0 + s * kTcStage;
          const uint32_t bytes = static_cast<uint32_t>(good) * 2 * kPage * 128;
          // K of step j, once QK^T of step j - kTcStages has read the stage's K
          if (j >= kTcStages && !mbar_wait_bounded(EMPTY_K(s), rel)) {
            flag_error(a.err, kErrTimeout);
            break;
          }
          mbar_arrive_expect_tx(FULL_K(s), bytes);
  #pragma unroll
          for (int p = 0; p < kTcPages; ++p) {
            if (prow[p] < 0) continue;
            tma_load_3d(st + p * kPage * 128, &tmK, 0, 0, prow[p], FULL_K(s), policy);
            tma_load_3d(st + kTcHalf + p * kPage * 128, &tmK, 0, 1, prow[p], FULL_K(s), policy);
          }
          issued_k = j + 1;
          // V of step j, once the PV product of step j - kTcStages has read its V
          if (j >= kTcStages && !mbar_wait_bounded(EMPTY_V(s), rel)) {
            flag_error(a.err, kErrTimeout);
            break;
          }
          mbar_arrive_expect_tx(FULL_V(s), bytes);
  #pragma unroll
          for (int p = 0; p < kTcPages; ++p) {
            if (prow[p] < 0) continue;
            tma_load_3d(st + 2 * kTcHalf + p * kPage * 128, &tmV, 0, 0, prow[p], FULL_V(s), policy);
            tma_load_3d(st + 3 * kTcHalf + p * kPage * 128, &tmV, 0, 1, prow[p], FULL_V(s), policy);
          }
          issued_v = j + 1;
        }
        // the copies of the last stages have landed before the CTA exits
        for (int j = max(0, issued_k - kTcStages); j < issued_k; ++j)
          mbar_wait_bounded(FULL_K(j % kTcStages), (j / kTcStages) & 1);
        for (int j = max(0, issued_v - kTcStages); j < issued_v; ++j)
          mbar_wait_bounded(FULL_V(j % kTcStages), (j / kTcStages) & 1);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t fmt = kBf16 ? 1u : 0u;
        bool ok = mbar_wait_bounded(Q_FULL, 0);
        tc::fence_after_sync();
        bool o_started = false;
        auto issue_qk = [&](int j) {
          const int b = j & 1;
          const uint32_t idesc = tc::idesc_f16(fmt, static_cast<uint32_t>(step_pages(j) * kPage), false);
          const uint32_t kst = ring0 + (j % kTcStages) * kTcStage;
  #pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t kaddr = kst + (k >> 2) * kTcHalf + (k & 3) * 32;
            const uint32_t qaddr = q0 + (k >> 2) * (kTcQBytes / 2) + (k & 3) * 32;
            tc::mma_ss(tbase + kColS + b * kTcTok, tc::smem_desc(qaddr, 16, 1024),
                       tc::smem_desc(kaddr, 16, 1024), idesc, k > 0);
          }
          tc::commit(EMPTY_K(j % kTcStages));
          tc::commit(S_FULL + 8 * b);
        };
        uint32_t pv_mask0 = 0u, pv_mask1 = 0u;  // loaded one step before the PV product uses it
        auto issue_pv = [&](int j) {
          const int b = j & 1, s = j % kTcStages;
          const int np = step_pages(j);
          const uint32_t mask = (j & 1) ? pv_mask1 : pv_mask0;
          const uint32_t idesc = tc::idesc_f16(fmt, D, true);
          const uint32_t vst = ring0 + s * kTcStage + 2 * kTcHalf;
          for (int kk = 0; kk < np; ++kk) {
            if (!((mask >> kk) & 1u)) continue;  // (its scores are masked; its stage bytes are stale)
            const uint64_t vd = tc::smem_desc(vst + kk * kPage * 128, kTcHalf, 1024);
            const uint32_t pa = tbase + kColS + b * kTcTok + kk * 8;  // P over S; remainder at +32
            tc::mma_ts(tbase + kColO, pa, vd, idesc, o_started);
            o_started = true;
            if (kBf16) tc::mma_ts(tbase + kColO, pa + kTcTok / 2, vd, idesc, true);
          }
          tc::commit(EMPTY_V(s));
          tc::commit(O_DONE);
        };
        // the PV product of step j waits for its probabilities and its V pages
        auto wait_pv = [&](int j) {
          return mbar_wait_bounded(P_FULL + 8 * (j & 1), (j >> 1) & 1) &&
                 mbar_wait_bounded(FULL_V(j % kTcStages), (j / kTcStages) & 1);
        };
        StepPages ahead;  // the block-table entries of step j, loaded during step j - 1
        ahead.load(bt, p_begin, p_end, nsteps, 0);
        for (int j = 0; ok && j < nsteps; ++j) {
          if (j & 1) pv_mask1 = ahead.mask(a);
          else pv_mask0 = ahead.mask(a);
          ahead.load(bt, p_begin, p_end, nsteps, j + 1);
          if (!mbar_wait_bounded(FULL_K(j % kTcStages), (j / kTcStages) & 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          issue_qk(j);
          if (j >= 1) {
            if (!wait_pv(j - 1)) {
              ok = false;
              break;
            }
            tc::fence_after_sync();
            issue_pv(j - 1);
          }
        }
        if (ok) {
          const int j = nsteps - 1;
          if (wait_pv(j)) {
            tc::fence_after_sync();
            issue_pv(j);
          } else {
            ok = false;
          }
        }
        if (!ok) flag_error(a.err, kErrTimeout);
        // every MMA issued here completes before TMEM is released
        tc::commit(DRAIN);
        mbar_wait_bounded(DRAIN, 0);
      }
    } else {
      // ------------------------------------------------------------ softmax
      tc_softmax_role<T>(a, qs, tbase, S_FULL, P_FULL, O_DONE, Q_FULL, warp, lane, r0, rows, s0, h,
                         chunk, nsteps, bt, p_begin, p_end);
    }

    // release TMEM once every role is done with it
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
      __syncwarp();
      tc::fence_after_sync();
      tc::tmem_dealloc(tbase, kTmemCols);
    }
  }();
  prefix_exit(a);
}

// ------------------------------------------------------------------------
// The tensor-memory pass over a quantised cache (E4M3, INT8 or INT4 codes,
// one fp32 scale per token, KV head and 32 channels; d = 128).
//
// The tensor core multiplies 16-bit operands, and a cached value is s * code
// with an fp32 scale.  Rounded once to the operand type it would be off by up
// to half an ulp (2^-11 relative in f16), which reaches the fp16 tolerance of
// the output.  So each value is carried as a rounded head and a rounded
// remainder, hi = RN(s * code) and lo = RN(s * code - hi), in two operand
// tiles, and
//     S = Q . K_hi^T + Q . K_lo^T,      O += P . V_hi + P . V_lo
// (bf16 adds the probability remainder times V_hi, as in the 16-bit pass).
// What is left is about 2^-22 (f16) or 2^-16 (bf16) of each value.
//
// Roles (384 threads): those of the 16-bit pass plus six dequantise warps,
// three for K (6-8) and three for V (9-11), so that the K and V tiles of a
// step are made in parallel and each group waits only on its own barriers.
// The producer copies a step's codes (2-D TMA boxes, swizzled by the code row
// size) and scale rows (bulk copies) into a code stage.  The dequantise warps
// turn them into the four operand tiles -- K hi, K lo, V hi, V lo, each laid
// out as the TMA lays out a 16-bit page (64-channel halves, 128-byte rows,
// 128-byte swizzle) -- and hand the code stage back.  The MMA issuer waits for
// the tiles instead of the copies.  Per stage and per K / V: codes landed
// (TMA / bulk bytes), codes consumed and tiles written (one arrive per
// dequantise warp of the group), tiles read (tcgen05.commit).  The codes ring
// is deeper (kTqCodeStages) than the tile ring, so the copies of the next two
// steps are in flight while a step is dequantised.  About 214 KB of shared
// memory: one CTA per SM.
namespace {
constexpr int kTqWarps = 12;
constexpr int kTqDqWarps = 3;                // dequantise warps per K / V group
constexpr int kTqDqThreads = 32 * kTqDqWarps;
constexpr int kTqCodeStages = 3;             // steps of codes in flight (operand tiles: kTcStages)
// one tile stage (64 KB): K as two 64-channel halves of 128 rows each (the
// step's 64 tokens' heads, then their remainders: one N = 128 operand), then
// V hi (two halves), V lo (two halves)
constexpr int kTqStage = 8 * kTcHalf;
constexpr int kTqScalePage = kPage * 4 * 4;  // fp32 scales of one page and head (d = 128)

template <Code8 kFmt>
struct TqGeo {
  static constexpr int kRow = kFmt == Code8::INT4 ? 64 : 128;  // code bytes of a token (d = 128)
  static constexpr int kCodePage = kPage * kRow;
  static constexpr int kCodeStage = 2 * kTcPages * kCodePage;         // K then V codes of a step
  static constexpr int kScaleStage = 2 * kTcPages * kTqScalePage;     // K then V scales
  static constexpr int kBars = 4 * kTqCodeStages + 4 * kTcStages + 7;
  static constexpr size_t kSmem = 1024 + (size_t)kTcStages * kTqStage +
                                  (size_t)kTqCodeStages * (kCodeStage + kScaleStage) + kBars * 8 + 64;
  static_assert(kSmem <= 227 * 1024, "one CTA per SM");
};

// Packed pair arithmetic of the operand type (f16x2 / bf16x2), one rounding each.
template <typename T>
__device__ __forceinline__ uint32_t x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  if constexpr (std::is_same<T, __nv_bfloat16>::value)
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  else
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <typename T>
__device__ __forceinline__ uint32_t x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  if constexpr (std::is_same<T, __nv_bfloat16>::value)
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  else
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Dequantise the K (or V) half of one code stage into its hi and lo operand
// tiles; thread ct of the group's kTqDqThreads.  A unit is one 16-byte chunk
// of one token's codes: 16 channels (8-bit) or 32 (INT4), all in one scale
// group; several units are in flight per thread.
//
// Every code value v is exact in the operand type T.  The fp32 scale is split
// once per unit into s = s_hi + s_lo + d with s_hi = RN_T(s) and
// s_lo = RN_T(s - s_hi).  Then, in packed T arithmetic,
//   hi = RN(v s_hi),  e = v s_hi - hi (one fma: the error of a product of a
//   code (at most 8 significant bits) and s_hi fits in T, so it is exact),
//   lo = RN(v s_lo + e),
// and hi + lo is v s to about 2^-15 relative in bf16.  In f16, s_lo is a
// subnormal once s < 2^-3 (typical for E4M3 and INT8 scales), and then the
// error is absolute, at most about |v| 2^-25 per value (1.4e-5 for the largest
// E4M3 code) -- below the f16 rounding of the probabilities in the PV product
// (2^-11 relative) that the 16-bit pass already makes.
template <typename T, Code8 kFmt>
__device__ __forceinline__ void dequant_half(const uint8_t *codes, const float *scl, uint8_t *hi,
                                             uint8_t *lo, int half_stride, int ct) {
  using M = Mma<T>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int kRow = TqGeo<kFmt>::kRow;
  constexpr int kPerRow = kRow / 16;        // chunks of a code row
  constexpr int kChan = 128 / kPerRow;      // channels of a chunk
  constexpr int kUnits = kTcPages * kPage * kPerRow;
  // INT4 (at most three 32-code units a thread) unrolls fully; the 8-bit
  // formats (five or six 16-code units) two at a time, measured faster
#pragma unroll(kFmt == Code8::INT4 ? 4 : 2)
  for (int u = ct; u < kUnits; u += kTqDqThreads) {
    // unit u -> (row tr of the step's 64 tokens, chunk c).  Each 8-lane phase
    // of a 16-byte access takes rows whose swizzles put its code reads and
    // its tile stores on 8 distinct 16-byte bank slots (8-bit: rows r and
    // r ^ 5, 4 chunks each; INT4: rows {0, 1, 6, 7} or {2, 3, 4, 5} of an
    // 8-row block, 2 chunks each) -- one row's 8 chunks would store into the
    // same slots from both 64-channel halves.
    int tr, c;
    {
      const int i = u & 7, q = u >> 3, hf = q & 1, rg = q >> 1;
      if constexpr (kFmt == Code8::INT4) {
        constexpr uint32_t kRows = 0x54327610u;  // nibble j: row of lane pair j, two blocks
        tr = 8 * (rg >> 1) + static_cast<int>((kRows >> (4 * (((rg & 1) << 2) | (i >> 1)))) & 7u);
        c = hf * 2 + (i & 1);
      } else {
        tr = 8 * (rg >> 2) + ((rg & 3) ^ ((i >> 2) ? 5 : 0));
        c = hf * 4 + (i & 3);
      }
    }
    const int t = tr % kPage, p = tr / kPage;
    const uint4 w = *reinterpret_cast<const uint4 *>(codes + p * kPage * kRow + swz_rows<kRow>(t, c));
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    const int ch0 = c * kChan;
    const float sc = scl[(p * kPage + t) * 4 + ch0 / 32];
    const uint32_t shi = M::pack(sc, sc);
    const float shf = M::unpack(shi).x;
    const uint32_t slo = M::pack(sc - shf, sc - shf);
    // vp[i]: channels ch0 + 2i, ch0 + 2i + 1 as an f16 pair
    uint32_t vp[kChan / 2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (kFmt == Code8::INT4) {
        uint32_t f[4];  // f[q]: channels 8k + q (low half) and 8k + q + 4 (high half)
        int4x8_to_f16x2x4(words[k], f);
        vp[4 * k] = __byte_perm(f[0], f[1], 0x5410);
        vp[4 * k + 1] = __byte_perm(f[2], f[3], 0x5410);
        vp[4 * k + 2] = __byte_perm(f[0], f[1], 0x7632);
        vp[4 * k + 3] = __byte_perm(f[2], f[3], 0x7632);
      } else {
        code8x4_to_f16x2x2<kFmt>(words[k], vp[2 * k], vp[2 * k + 1]);
      }
    }
    if constexpr (kBf16) {
#pragma unroll
      for (int i = 0; i < kChan / 2; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&vp[i]));
        vp[i] = M::pack(f.x, f.y);  // exact: every code value fits in bf16
      }
    }
    const int r = tr;  // row of the step's 64 tokens
#pragma unroll
    for (int k = 0; k < kChan / 8; ++k) {
      const int ch = ch0 + 8 * k, hf = ch / 64, cc = (ch % 64) / 8;
      uint32_t h4[4], l4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t v = vp[4 * k + i];
        h4[i] = x2_mul<T>(v, shi);
        const uint32_t e = x2_fma<T>(v, shi, h4[i] ^ 0x80008000u);
        l4[i] = x2_fma<T>(v, slo, e);
      }
      const int off = hf * half_stride + r * 128 + ((cc ^ (r & 7)) << 4);
      *reinterpret_cast<uint4 *>(hi + off) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
      *reinterpret_cast<uint4 *>(lo + off) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    }
  }
}
}  // namespace

template <typename T, Code8 kFmt>
__global__ void __launch_bounds__(32 * kTqWarps, 1)
    prefix_tcq_kernel(const PrefixArgs a, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV) {
  constexpr int D = 128;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using Gq = TqGeo<kFmt>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
  uint8_t *codes = tiles + (size_t)kTcStages * kTqStage;
  uint8_t *scl = codes + (size_t)kTqCodeStages * Gq::kCodeStage;
  uint64_t *bars = reinterpret_cast<uint64_t *>(scl + (size_t)kTqCodeStages * Gq::kScaleStage);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + Gq::kBars);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // no wait for the decode launch before this pass (prefix_exit); every
  // return of the body below still passes through prefix_exit
  grid_launch_dependents();
  [&] {
    const int g = blockIdx.x / a.chunks, chunk = blockIdx.x - g * a.chunks;
    const int h = blockIdx.y;
    const int s0 = __ldg(a.group_start + g), s1 = __ldg(a.group_start + g + 1);
    const int gp = __ldg(a.group_pages + g);
    if (!group_ok(a, s0, s1, gp)) {
      if (tid == 0) flag_error(a.err, kErrSeqLen);
      return;
    }
    const int rows = (s1 - s0) * a.G;
    const int r0 = blockIdx.z * kRowsPerCta;
    if (r0 >= rows || gp == 0) return;
    const int p_begin = static_cast<int>((static_cast<long long>(chunk) * gp) / a.chunks);
    const int p_end = static_cast<int>((static_cast<long long>(chunk + 1) * gp) / a.chunks);
    const int nsteps = (p_end - p_begin + kTcPages - 1) / kTcPages;
    if (nsteps == 0) {  // an empty chunk leaves empty partials
      for (int r = tid; r < kRowsPerCta; r += blockDim.x) {
        const int row = r0 + r;
        if (row >= rows) continue;
        const size_t idx = ((static_cast<size_t>(chunk) * a.H_kv + h) * a.B + s0 + row / a.G) * a.G +
                           row % a.G;
        for (int c = 0; c < D; ++c) a.pre_o[idx * D + c] = 0.f;
        a.pre_lse[idx] = -INFINITY;
      }
      return;
    }
    const int32_t *bt = a.block_table + static_cast<size_t>(s0) * a.maxb;  // first member's row
    auto step_pages = [&](int j) { return min(kTcPages, p_end - (p_begin + j * kTcPages)); };

    const uint32_t tiles0 = smem_u32(tiles), codes0 = smem_u32(codes);
    const uint32_t scl0 = smem_u32(scl), bar0 = smem_u32(bars);
    // kv = 0: K, 1: V; c: code stage (kTqCodeStages), s: tile stage (kTcStages)
    constexpr int kT0 = 4 * kTqCodeStages;  // first tile barrier
    auto CFULL = [&](int kv, int c) { return bar0 + 8 * (kv * kTqCodeStages + c); };
    auto CFREE = [&](int kv, int c) { return bar0 + 8 * ((2 + kv) * kTqCodeStages + c); };
    auto TFULL = [&](int kv, int s) { return bar0 + 8 * (kT0 + kv * kTcStages + s); };
    auto TFREE = [&](int kv, int s) { return bar0 + 8 * (kT0 + (2 + kv) * kTcStages + s); };
    const uint32_t S_FULL = bar0 + 8 * (kT0 + 4 * kTcStages);  // + 8 * buffer
    const uint32_t P_FULL = S_FULL + 16;                 // + 8 * buffer
    const uint32_t O_DONE = S_FULL + 32, Q_FULL = S_FULL + 40, DRAIN = S_FULL + 48;

    if (warp == 0) {
      __syncwarp();
      tc::tmem_alloc(smem_u32(tmem_slot), kTmemColsQ);
      tc::tmem_relinquish();
    }
    if (tid == 32) {
      for (int kv = 0; kv < 2; ++kv) {
        for (int c = 0; c < kTqCodeStages; ++c) {
          mbar_init(CFULL(kv, c), 1);
          mbar_init(CFREE(kv, c), kTqDqWarps);
        }
        for (int s = 0; s < kTcStages; ++s) {
          mbar_init(TFULL(kv, s), kTqDqWarps);
          mbar_init(TFREE(kv, s), 1);
        }
      }
      mbar_init(S_FULL, 1);
      mbar_init(S_FULL + 8, 1);
      mbar_init(P_FULL, 4);
      mbar_init(P_FULL + 8, 4);
      mbar_init(O_DONE, 1);
      mbar_init(Q_FULL, 4);
      mbar_init(DRAIN, 1);
      mbar_init_fence();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(tmem_slot);

    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        const uint64_t policy = l2_policy_evict_normal();
        int issued = 0;
        bool ok = true;
        for (int j = 0; j < nsteps && ok; ++j) {
          const int c = j % kTqCodeStages;
          const uint32_t rel = ((j / kTqCodeStages) - 1) & 1;  // phase of step j - kTqCodeStages
          const int p0 = p_begin + j * kTcPages, np = step_pages(j);
          int prow[kTcPages];
          int good = 0;
  #pragma unroll
          for (int p = 0; p < kTcPages; ++p) {
            prow[p] = -1;
            if (p < np) {
              const int pb = __ldg(bt + p0 + p);
              if (pb >= 0 && pb < a.num_blocks) {
                prow[p] = (pb * a.H_kv + h) * kPage;
                ++good;
              } else {
                flag_error(a.err, kErrBlockTable);
              }
            }
          }
          const uint32_t bytes = static_cast<uint32_t>(good) * (Gq::kCodePage + kTqScalePage);
          for (int kv = 0; kv < 2; ++kv) {
            // the codes of step j - kTqCodeStages have been dequantised
            if (j >= kTqCodeStages && !mbar_wait_bounded(CFREE(kv, c), rel)) {
              flag_error(a.err, kErrTimeout);
              ok = false;
              break;
            }
            const uint32_t cst = codes0 + c * Gq::kCodeStage + kv * kTcPages * Gq::kCodePage;
            const uint32_t sst = scl0 + c * Gq::kScaleStage + kv * kTcPages * kTqScalePage;
            const float *gs = kv ? a.v_scale : a.k_scale;
            mbar_arrive_expect_tx(CFULL(kv, c), bytes);
  #pragma unroll
            for (int p = 0; p < kTcPages; ++p) {
              if (prow[p] < 0) continue;
              tma_load_2d(cst + p * Gq::kCodePage, kv ? &tmV : &tmK, 0, prow[p], CFULL(kv, c), policy);
              bulk_load(sst + p * kTqScalePage, gs + static_cast<size_t>(prow[p]) * 4, kTqScalePage,
                        CFULL(kv, c));
            }
          }
          if (ok) issued = j + 1;
        }
        // the copies of the last stages have landed before the CTA exits
        for (int j = max(0, issued - kTqCodeStages); j < issued; ++j)
          for (int kv = 0; kv < 2; ++kv)
            mbar_wait_bounded(CFULL(kv, j % kTqCodeStages), (j / kTqCodeStages) & 1);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t fmt = kBf16 ? 1u : 0u;
        bool ok = mbar_wait_bounded(Q_FULL, 0);
        tc::fence_after_sync();
        bool o_started = false;
        // S[128 x (64 + 64)] = Q . [K_hi; K_lo]^T: A = Q in TMEM, B = the step's
        // 128 K rows (heads, then remainders) of each 64-channel half; a
        // partial step's missing rows give columns the softmax masks
        auto issue_qk = [&](int j) {
          const int b = j & 1;
          const uint32_t idesc = tc::idesc_f16(fmt, 2 * kTcTok, false);
          const uint32_t kst = tiles0 + (j % kTcStages) * kTqStage;
  #pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t kaddr = kst + (k >> 2) * 2 * kTcHalf + (k & 3) * 32;
            tc::mma_ts(tbase + kColS + b * 2 * kTcTok, tbase + kColQ + 8 * k,
                       tc::smem_desc(kaddr, 16, 1024), idesc, k > 0);
          }
          tc::commit(TFREE(0, j % kTcStages));
          tc::commit(S_FULL + 8 * b);
        };
        uint32_t pv_mask0 = 0u, pv_mask1 = 0u;  // loaded one step before the PV product uses it
        auto issue_pv = [&](int j) {
          const int b = j & 1, s = j % kTcStages;
          const int np = step_pages(j);
          const uint32_t mask = (j & 1) ? pv_mask1 : pv_mask0;
          const uint32_t idesc = tc::idesc_f16(fmt, D, true);
          const uint32_t vhi = tiles0 + s * kTqStage + 4 * kTcHalf, vlo = vhi + 2 * kTcHalf;
          for (int kk = 0; kk < np; ++kk) {
            if (!((mask >> kk) & 1u)) continue;  // (its scores are masked; its tiles are stale)
            const uint64_t dh = tc::smem_desc(vhi + kk * kPage * 128, kTcHalf, 1024);
            const uint64_t dl = tc::smem_desc(vlo + kk * kPage * 128, kTcHalf, 1024);
            const uint32_t pa = tbase + kColS + b * 2 * kTcTok + kk * 8;  // P over S; remainder at +32
            tc::mma_ts(tbase + kColO, pa, dh, idesc, o_started);
            o_started = true;
            tc::mma_ts(tbase + kColO, pa, dl, idesc, true);
            if (kBf16) tc::mma_ts(tbase + kColO, pa + kTcTok / 2, dh, idesc, true);
          }
          tc::commit(TFREE(1, s));
          tc::commit(O_DONE);
        };
        auto wait_pv = [&](int j) {
          return mbar_wait_bounded(P_FULL + 8 * (j & 1), (j >> 1) & 1) &&
                 mbar_wait_bounded(TFULL(1, j % kTcStages), (j / kTcStages) & 1);
        };
        StepPages ahead;  // the block-table entries of step j, loaded during step j - 1
        ahead.load(bt, p_begin, p_end, nsteps, 0);
        for (int j = 0; ok && j < nsteps; ++j) {
          if (j & 1) pv_mask1 = ahead.mask(a);
          else pv_mask0 = ahead.mask(a);
          ahead.load(bt, p_begin, p_end, nsteps, j + 1);
          if (!mbar_wait_bounded(TFULL(0, j % kTcStages), (j / kTcStages) & 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          issue_qk(j);
          if (j >= 1) {
            if (!wait_pv(j - 1)) {
              ok = false;
              break;
            }
            tc::fence_after_sync();
            issue_pv(j - 1);
          }
        }
        if (ok) {
          const int j = nsteps - 1;
          if (wait_pv(j)) {
            tc::fence_after_sync();
            issue_pv(j);
          } else {
            ok = false;
          }
        }
        if (!ok) flag_error(a.err, kErrTimeout);
        // every MMA issued here completes before TMEM is released
        tc::commit(DRAIN);
        mbar_wait_bounded(DRAIN, 0);
      }
    } else if (warp < 6) {
      // ------------------------------------------------------------ softmax
      tc_softmax_role<T, true>(a, nullptr, tbase, S_FULL, P_FULL, O_DONE, Q_FULL, warp, lane, r0, rows,
                               s0, h, chunk, nsteps, bt, p_begin, p_end);
    } else {
      // ------------------------------------------------------------ dequantise
      const int kv = (warp - 6) / kTqDqWarps;  // 0: K (warps 6-8), 1: V (warps 9-11)
      const int ct = tid - (6 + kv * kTqDqWarps) * 32;
      bool ok = true;
      for (int j = 0; j < nsteps; ++j) {
        const int s = j % kTcStages, c = j % kTqCodeStages;
        const uint32_t rel = ((j / kTcStages) - 1) & 1;
        // this step's codes have landed, and the MMAs of step j - kTcStages
        // have finished reading the tiles about to be overwritten
        bool got = mbar_wait_bounded(CFULL(kv, c), (j / kTqCodeStages) & 1);
        if (j >= kTcStages) got = got && mbar_wait_bounded(TFREE(kv, s), rel);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        // K: halves 2 kTcHalf apart, remainders kTcHalf after the heads;
        // V: halves kTcHalf apart, remainders 2 kTcHalf after the heads
        uint8_t *hi = tiles + (size_t)s * kTqStage + kv * 4 * kTcHalf;
        dequant_half<T, kFmt>(codes + (size_t)c * Gq::kCodeStage + kv * kTcPages * Gq::kCodePage,
                              reinterpret_cast<const float *>(scl + (size_t)c * Gq::kScaleStage +
                                                              kv * kTcPages * kTqScalePage),
                              hi, hi + (kv ? 2 : 1) * kTcHalf, (kv ? 1 : 2) * kTcHalf, ct);
        fence_proxy_async_smem();  // tiles visible to the tensor core; codes read before refill
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(TFULL(kv, s));
          mbar_arrive(CFREE(kv, c));
        }
      }
      if (!ok && lane == 0) flag_error(a.err, kErrTimeout);
    }

    // release TMEM once every role is done with it
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
      __syncwarp();
      tc::fence_after_sync();
      tc::tmem_dealloc(tbase, kTmemColsQ);
    }
  }();
  prefix_exit(a);
}

int prefix_rows_per_cta() { return kRowsPerCta; }

// Time of one prefix page (one KV head, one row block of up to 128 query
// rows) relative to one decode page, per SM, as measured on the continuous-
// batching workload (8 groups x 32 members sharing 4096 tokens, d = 128):
// the split pays where the suffix decode is bound by HBM (fp16 / bf16 and
// E4M3 pages), and the two passes trade SMs for nothing where both are
// bound by their own instructions (INT8 and INT4 pages), so those keep the
// decode on every SM and the prefix pass only fills the SMs its tail frees.
#ifndef KVD_PREFIX_W_TC
#define KVD_PREFIX_W_TC 3.0f  // tensor-memory pass, fp16 / bf16 cache
#endif
#ifndef KVD_PREFIX_W_E4M3
#define KVD_PREFIX_W_E4M3 6.0f  // tensor-memory pass, E4M3 cache
#endif
#ifndef KVD_PREFIX_W_INT8
#define KVD_PREFIX_W_INT8 0.0f
#endif
#ifndef KVD_PREFIX_W_INT4
#define KVD_PREFIX_W_INT4 0.0f
#endif
#ifndef KVD_PREFIX_W_WARP
#define KVD_PREFIX_W_WARP 3.0f  // warp-level passes (d = 64)
#endif
void prefix_split(PrefixArgs &a, int d, bool quantised, Code8 fmt, bool split) {
  bool tc = d == 128;
#ifdef KVD_PREFIX_MMA_SYNC
  if (!quantised) tc = false;
#endif
  a.ctas_per_sm = tc && !quantised ? 2 : 1;  // prefix_tc_kernel: two per SM
  if (!split) a.weight = 0.f;
  else if (!tc) a.weight = KVD_PREFIX_W_WARP;
  else if (!quantised) a.weight = KVD_PREFIX_W_TC;
  else if (fmt == Code8::E4M3) a.weight = KVD_PREFIX_W_E4M3;
  else a.weight = fmt == Code8::INT8 ? KVD_PREFIX_W_INT8 : KVD_PREFIX_W_INT4;
}

cudaError_t launch_prefix_plan(const PrefixArgs &a, cudaStream_t s) {
  if (a.n_groups == 0 || a.B == 0) return cudaSuccess;
  return launch_pdl(prefix_plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, a);
}

namespace {
template <typename T>
cudaError_t launch_prefix_tc_t(const PrefixArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                               int row_blocks, cudaStream_t st) {
  auto kern = prefix_tc_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kTcSmem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_groups * a.chunks, a.H_kv, row_blocks);
  return launch_pdl(kern, grid, dim3(32 * kTcWarps), kTcSmem, st, a, tmK, tmV);
}

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

namespace {
template <typename T, Code8 kFmt>
cudaError_t launch_prefix_q_t(const PrefixArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                              int row_blocks, cudaStream_t st) {
  auto kern = prefix_tcq_kernel<T, kFmt>;
  constexpr size_t smem = TqGeo<kFmt>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_groups * a.chunks, a.H_kv, row_blocks);
  return launch_pdl(kern, grid, dim3(32 * kTqWarps), smem, st, a, tmK, tmV);
}

// d = 64: the warp-level pass
template <typename T, Code8 kFmt>
cudaError_t launch_prefix_q64_t(const PrefixArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                                int row_blocks, cudaStream_t st) {
  auto kern = prefix_q_kernel<64, T, kFmt>;
  const size_t smem = PQGeo<64, kFmt>::smem();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_groups * a.chunks, a.H_kv, row_blocks);
  return launch_pdl(kern, grid, dim3(32 * kWarps), smem, st, a, tmK, tmV);
}

template <typename T>
cudaError_t launch_prefix_q_d(const PrefixArgs &a, int d, Code8 fmt, const CUtensorMap &tmK,
                              const CUtensorMap &tmV, int row_blocks, cudaStream_t st) {
  if (d == 64) {
    switch (fmt) {
      case Code8::E4M3: return launch_prefix_q64_t<T, Code8::E4M3>(a, tmK, tmV, row_blocks, st);
      case Code8::INT8: return launch_prefix_q64_t<T, Code8::INT8>(a, tmK, tmV, row_blocks, st);
      default: return launch_prefix_q64_t<T, Code8::INT4>(a, tmK, tmV, row_blocks, st);
    }
  }
  switch (fmt) {
    case Code8::E4M3: return launch_prefix_q_t<T, Code8::E4M3>(a, tmK, tmV, row_blocks, st);
    case Code8::INT8: return launch_prefix_q_t<T, Code8::INT8>(a, tmK, tmV, row_blocks, st);
    default: return launch_prefix_q_t<T, Code8::INT4>(a, tmK, tmV, row_blocks, st);
  }
}
}  // namespace

cudaError_t launch_prefix_q(const PrefixArgs &a, int d, Code8 fmt, DType dt, const CUtensorMap &tmK,
                            const CUtensorMap &tmV, int row_blocks, cudaStream_t s) {
  if (a.n_groups == 0 || a.B == 0) return cudaSuccess;
  return dt == DType::BF16 ? launch_prefix_q_d<__nv_bfloat16>(a, d, fmt, tmK, tmV, row_blocks, s)
                           : launch_prefix_q_d<__half>(a, d, fmt, tmK, tmV, row_blocks, s);
}

cudaError_t launch_prefix(const PrefixArgs &a, int d, DType dt, const CUtensorMap &tmK,
                          const CUtensorMap &tmV, int row_blocks, cudaStream_t s) {
  if (a.n_groups == 0 || a.B == 0) return cudaSuccess;
#ifndef KVD_PREFIX_MMA_SYNC
  if (d == 128)
    return dt == DType::BF16 ? launch_prefix_tc_t<__nv_bfloat16>(a, tmK, tmV, row_blocks, s)
                             : launch_prefix_tc_t<__half>(a, tmK, tmV, row_blocks, s);
#endif
  if (dt == DType::BF16)
    return d == 128 ? launch_prefix_t<128, __nv_bfloat16>(a, tmK, tmV, row_blocks, s)
                    : launch_prefix_t<64, __nv_bfloat16>(a, tmK, tmV, row_blocks, s);
  return d == 128 ? launch_prefix_t<128, __half>(a, tmK, tmV, row_blocks, s)
                  : launch_prefix_t<64, __half>(a, tmK, tmV, row_blocks, s);
}

}  // namespace kvd

// tile.cuh -- the per-page tensor-core tile shared by the decode and
// shared-prefix kernels: swizzled page addressing and one 16-token step of
// the online softmax for the query rows a warp holds.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

#ifndef KVD_BF16_SPLIT_P
#define KVD_BF16_SPLIT_P 1
#endif

namespace kvd {

// Byte offset of element column `col` (a multiple of 8) of token row t inside
// a page staged as d/64 boxes of [16 tokens][64 elements], each box one
// 2 KB run of 128-byte rows with the TMA 128-byte swizzle (16-byte chunk
// index XOR row % 8).  Keeping each 64-column half in its own 2 KB run puts 8
// consecutive tokens on 8 different chunk positions, so every 8-row ldmatrix
// phase is free of bank conflicts.
template <int D>
__device__ __forceinline__ uint32_t swz(int t, int col) {
  const int half = col >> 6;
  const int chunk = (col & 63) >> 3;
  return static_cast<uint32_t>(half * (kPage * 128) + t * 128 + ((chunk ^ (t & 7)) << 4));
}

__device__ __forceinline__ int clamp_len(int n, int cap) { return n < 0 ? 0 : (n > cap ? cap : n); }

// One 16-token page of the online softmax for 8*NT query rows held by one
// warp: S^T = K Q^T (K page as the A operand), base-2 running max / sum per
// row, probabilities to the B operand via movmatrix, O^T += V^T P^T.  kb, vb:
// shared addresses of the staged K and V pages (d/64 swizzled 2 KB boxes);
// tokens >= ntok are masked.  The state arrays are the warp's registers.
// Online softmax with a reference maximum (base 2).  m_run is a reference,
// not the exact running maximum: it moves -- to the exact maximum so far,
// with l_run and acc rescaled -- only when a score of this step exceeds it by
// more than kTileRefSlack; otherwise the step's probabilities are
// exp2(x - m_run) <= 2^kTileRefSlack, exact enough in f16/bf16 (the rounding
// is relative) and far from fp32 overflow, and the per-step row maximum (three
// rounds of shuffles) and rescale are skipped.  x[nt][e]: this lane's scaled
// scores, row e & 1 of n-tile nt (-inf where masked).  Warp-uniform branch.
constexpr float kTileRefSlack = 8.f;
template <int NT, int MT, int NX>
__device__ __forceinline__ void ref_max_update(const float (&x)[NT][NX], float (&m_run)[NT][2],
                                               float (&l_run)[NT][2], float (&acc)[NT][MT][4]) {
  bool up = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < NX; ++e) up |= x[nt][e] > m_run[nt][e & 1] + kTileRefSlack;
  if (!__any_sync(0xffffffffu, up)) return;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float mx0 = x[nt][0], mx1 = x[nt][1];
#pragma unroll
    for (int e = 2; e < NX; ++e) {
      if (e & 1) mx1 = fmaxf(mx1, x[nt][e]);
      else mx0 = fmaxf(mx0, x[nt][e]);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
    // a row with no finite score yet keeps its (zero) state
    const float a0 = mn0 == -INFINITY ? 1.f : fast_exp2(m_run[nt][0] - mn0);
    const float a1 = mn1 == -INFINITY ? 1.f : fast_exp2(m_run[nt][1] - mn1);
    m_run[nt][0] = mn0;
    m_run[nt][1] = mn1;
    l_run[nt][0] *= a0;
    l_run[nt][1] *= a1;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      acc[nt][mt][0] *= a0;
      acc[nt][mt][1] *= a1;
      acc[nt][mt][2] *= a0;
      acc[nt][mt][3] *= a1;
    }
  }
}

template <int D, int NT, typename T>
__device__ __forceinline__ void tile_page(uint32_t kb, uint32_t vb, int ntok, float scale_log2,
                                          int lane, const uint32_t (&qf)[NT][D / 16][2],
                                          float (&acc)[NT][D / 16][4], float (&m_run)[NT][2],
                                          float (&l_run)[NT][2]) {
  using M = Mma<T>;
  constexpr int kSteps = D / 16;
  // bf16 keeps only 8 significant bits of each probability; carrying the
  // rounding remainder in a second PV product restores ~16 bits for the cost
  // of d/16 extra MMAs per page (free while the kernel waits on HBM).
  constexpr bool kSplitP = KVD_BF16_SPLIT_P && std::is_same<T, __nv_bfloat16>::value;
  const int g8 = lane >> 2;
  const int tK = (lane & 7) | (((lane >> 3) & 1) << 3);
  const int cK = ((lane >> 4) & 1) << 3;
  const int tV = (lane & 7) | (((lane >> 4) & 1) << 3);
  const int cV = ((lane >> 3) & 1) << 3;

  // S^T = K Q^T, two independent accumulator chains over d
  float s[NT][4], s2[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = s2[nt][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < kSteps; ++ks) {
    uint32_t fa[4];
    ldmatrix_x4(fa, kb + swz<D>(tK, ks * 16 + cK));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (ks & 1) M::run(s2[nt], fa, qf[nt][ks][0], qf[nt][ks][1]);
      else M::run(s[nt], fa, qf[nt][ks][0], qf[nt][ks][1]);
    }
  }

  // online softmax update (base 2), probabilities rounded to T (bf16:
  // split into a rounded head and a rounded remainder, see kSplitP)
  const bool v0 = g8 < ntok, v1 = g8 + 8 < ntok;
  float x[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    x[nt][0] = v0 ? (s[nt][0] + s2[nt][0]) * scale_log2 : -INFINITY;
    x[nt][1] = v0 ? (s[nt][1] + s2[nt][1]) * scale_log2 : -INFINITY;
    x[nt][2] = v1 ? (s[nt][2] + s2[nt][2]) * scale_log2 : -INFINITY;
    x[nt][3] = v1 ? (s[nt][3] + s2[nt][3]) * scale_log2 : -INFINITY;
  }
  ref_max_update<NT, kSteps, 4>(x, m_run, l_run, acc);
  uint32_t pb0[NT], pb1[NT], pc0[NT], pc1[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float e0 = fast_exp2(x[nt][0] - m_run[nt][0]), e1 = fast_exp2(x[nt][1] - m_run[nt][1]);
    const float e2 = fast_exp2(x[nt][2] - m_run[nt][0]), e3 = fast_exp2(x[nt][3] - m_run[nt][1]);
    const uint32_t lo = M::pack(e0, e1), hi = M::pack(e2, e3);
    const float2 fl = M::unpack(lo), fh = M::unpack(hi);
    if constexpr (kSplitP) {
      // p = head + remainder, both bf16: ~16 significant bits in the PV
      // product; the running sum uses the unrounded p to match
      const uint32_t lo2 = M::pack(e0 - fl.x, e1 - fl.y);
      const uint32_t hi2 = M::pack(e2 - fh.x, e3 - fh.y);
      l_run[nt][0] += e0 + e2;
      l_run[nt][1] += e1 + e3;
      pc0[nt] = movmatrix_trans(lo2);
      pc1[nt] = movmatrix_trans(hi2);
    } else {
      // the running sum uses the same rounded p as the PV product, so
      // the output is an exact weighted mean of V up to fp32 sums
      l_run[nt][0] += fl.x + fh.x;
      l_run[nt][1] += fl.y + fh.y;
      pc0[nt] = pc1[nt] = 0u;
    }
    pb0[nt] = movmatrix_trans(lo);
    pb1[nt] = movmatrix_trans(hi);
  }

  // O^T += V^T P^T
#pragma unroll
  for (int mt = 0; mt < kSteps; ++mt) {
    uint32_t fa[4];
    ldmatrix_x4_trans(fa, vb + swz<D>(tV, mt * 16 + cV));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      M::run(acc[nt][mt], fa, pb0[nt], pb1[nt]);
      if constexpr (kSplitP) M::run(acc[nt][mt], fa, pc0[nt], pc1[nt]);
    }
  }
}

}  // namespace kvd

namespace kvd {

// Two full 16-token pages (A then B, in token order) in one step: both
// pages' S^T chains run independently, one max/sum update covers the 32
// tokens, and both PV products accumulate into the same tile.  Same result as
// two tile_page calls up to fp32 rounding order; more independent work per
// step for warps that are short of latency hiding.
template <int D, int NT, typename T>
__device__ __forceinline__ void tile_page2(uint32_t kbA, uint32_t vbA, uint32_t kbB, uint32_t vbB,
                                           float scale_log2, int lane,
                                           const uint32_t (&qf)[NT][D / 16][2],
                                           float (&acc)[NT][D / 16][4], float (&m_run)[NT][2],
                                           float (&l_run)[NT][2]) {
  using M = Mma<T>;
  constexpr int kSteps = D / 16;
  constexpr bool kSplitP = KVD_BF16_SPLIT_P && std::is_same<T, __nv_bfloat16>::value;
  const int tK = (lane & 7) | (((lane >> 3) & 1) << 3);
  const int cK = ((lane >> 4) & 1) << 3;
  const int tV = (lane & 7) | (((lane >> 4) & 1) << 3);
  const int cV = ((lane >> 3) & 1) << 3;

  float sa[NT][4], sb[NT][4], sa2[NT][4], sb2[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = sa2[nt][e] = sb2[nt][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < kSteps; ++ks) {
    uint32_t fa[4], fb[4];
    ldmatrix_x4(fa, kbA + swz<D>(tK, ks * 16 + cK));
    ldmatrix_x4(fb, kbB + swz<D>(tK, ks * 16 + cK));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (ks & 1) {
        M::run(sa2[nt], fa, qf[nt][ks][0], qf[nt][ks][1]);
        M::run(sb2[nt], fb, qf[nt][ks][0], qf[nt][ks][1]);
      } else {
        M::run(sa[nt], fa, qf[nt][ks][0], qf[nt][ks][1]);
        M::run(sb[nt], fb, qf[nt][ks][0], qf[nt][ks][1]);
      }
    }
  }

  uint32_t pa0[NT], pa1[NT], pb0[NT], pb1[NT];
  uint32_t ra0[NT], ra1[NT], rb0[NT], rb1[NT];  // bf16 remainders
  // row r0 = elements 0, 2 (page A), 4, 6 (page B); row r1 = 1, 3, 5, 7
  float x[NT][8];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[nt][e] = (sa[nt][e] + sa2[nt][e]) * scale_log2;
      x[nt][4 + e] = (sb[nt][e] + sb2[nt][e]) * scale_log2;
    }
  ref_max_update<NT, kSteps, 8>(x, m_run, l_run, acc);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float e[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) e[i] = fast_exp2(x[nt][i] - m_run[nt][i & 1]);
    const uint32_t w0 = M::pack(e[0], e[1]), w1 = M::pack(e[2], e[3]);
    const uint32_t w2 = M::pack(e[4], e[5]), w3 = M::pack(e[6], e[7]);
    const float2 f0 = M::unpack(w0), f1 = M::unpack(w1), f2 = M::unpack(w2), f3 = M::unpack(w3);
    if constexpr (kSplitP) {
      ra0[nt] = movmatrix_trans(M::pack(e[0] - f0.x, e[1] - f0.y));
      ra1[nt] = movmatrix_trans(M::pack(e[2] - f1.x, e[3] - f1.y));
      rb0[nt] = movmatrix_trans(M::pack(e[4] - f2.x, e[5] - f2.y));
      rb1[nt] = movmatrix_trans(M::pack(e[6] - f3.x, e[7] - f3.y));
      l_run[nt][0] += (e[0] + e[2]) + (e[4] + e[6]);
      l_run[nt][1] += (e[1] + e[3]) + (e[5] + e[7]);
    } else {
      ra0[nt] = ra1[nt] = rb0[nt] = rb1[nt] = 0u;
      l_run[nt][0] += (f0.x + f1.x) + (f2.x + f3.x);
      l_run[nt][1] += (f0.y + f1.y) + (f2.y + f3.y);
    }
    pa0[nt] = movmatrix_trans(w0);
    pa1[nt] = movmatrix_trans(w1);
    pb0[nt] = movmatrix_trans(w2);
    pb1[nt] = movmatrix_trans(w3);
  }
#pragma unroll
  for (int mt = 0; mt < kSteps; ++mt) {
    uint32_t fa[4], fb[4];
    ldmatrix_x4_trans(fa, vbA + swz<D>(tV, mt * 16 + cV));
    ldmatrix_x4_trans(fb, vbB + swz<D>(tV, mt * 16 + cV));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      M::run(acc[nt][mt], fa, pa0[nt], pa1[nt]);
      M::run(acc[nt][mt], fb, pb0[nt], pb1[nt]);
      if constexpr (kSplitP) {
        M::run(acc[nt][mt], fa, ra0[nt], ra1[nt]);
        M::run(acc[nt][mt], fb, rb0[nt], rb1[nt]);
      }
    }
  }
}

}  // namespace kvd

// ------------------------------------------------------------ 8-bit pages
#include <cuda_fp8.h>

namespace kvd {

// Four 8-bit codes (bytes 0..3 of `four`) -> f16x2 of bytes (0, 1) and of
// bytes (2, 3), exact (every E4M3 value and every integer in [-128, 127] is an
// f16 value).
//  * E4M3: the hardware conversion, two codes per instruction.
//  * INT8: each signed byte b becomes the f16 with bits 0x64 | (b + 128), that
//    is 1024 + (b + 128), and 1152 is subtracted (exact: |result| <= 128).
template <Code8 kFmt>
__device__ __forceinline__ void code8x4_to_f16x2x2(uint32_t four, uint32_t &lo, uint32_t &hi) {
  if constexpr (kFmt == Code8::E4M3) {
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(four));
  } else {
    const uint32_t u = four ^ 0x80808080u;  // b + 128, unsigned
    const uint32_t l = __byte_perm(u, 0x64646464u, 0x4140);
    const uint32_t h = __byte_perm(u, 0x64646464u, 0x4342);
    const uint32_t bias = 0x64806480u;      // f16x2 (1152, 1152)
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(l), "r"(bias));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(h), "r"(bias));
  }
}

// The same for the byte pairs (0, 2) and (1, 3) -- the two channels of a
// channel pair across two tokens after ldmatrix.trans on code bytes.  INT8
// picks those bytes in its own byte permutes; E4M3 regroups them first.
template <Code8 kFmt>
__device__ __forceinline__ void code8x4_to_f16x2x2_0213(uint32_t four, uint32_t &lo, uint32_t &hi) {
  if constexpr (kFmt == Code8::E4M3) {
    code8x4_to_f16x2x2<kFmt>(__byte_perm(four, 0, 0x3120), lo, hi);
  } else {
    const uint32_t u = four ^ 0x80808080u;  // b + 128, unsigned
    const uint32_t l = __byte_perm(u, 0x64646464u, 0x4240);
    const uint32_t h = __byte_perm(u, 0x64646464u, 0x4341);
    const uint32_t bias = 0x64806480u;      // f16x2 (1152, 1152)
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(l), "r"(bias));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(h), "r"(bias));
  }
}

__device__ __forceinline__ uint32_t f16pack(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// A q word (two channels, storage dtype T) as an f16 pair: the quantised
// tiles multiply in f16 (inputs beyond the f16 range are not supported).
template <typename T>
__device__ __forceinline__ uint32_t q_to_f16x2(uint32_t w) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w));
    return f16pack(f.x, f.y);
  } else {
    return w;
  }
}

// q's B fragment of k-step ks for the 8-bit tile: k-slots 2 tig, 2 tig + 1
// <- channels 16 ks + 4 tig, + 1 and k-slots 2 tig + 8, + 9 <- channels
// 16 ks + 4 tig + 2, + 3 (the order ldmatrix gives the code bytes).
template <typename T>
__device__ __forceinline__ void q_words_q8(const uint32_t *qrow, int ks, int tig, uint32_t &w0,
                                           uint32_t &w1) {
  w0 = q_to_f16x2<T>(__ldg(qrow + ks * 8 + 2 * tig));
  w1 = q_to_f16x2<T>(__ldg(qrow + ks * 8 + 2 * tig + 1));
}
// Output channel of accumulator element e of m-tile mt (8-bit tile).
__device__ __forceinline__ int dim_q8(int mt, int e, int g8) { return mt * 16 + 2 * g8 + (e >> 1); }

// q's B fragment for the INT4 tile: in k-step 2j (2j + 1) of group j, k-slots
// 2 tig, 2 tig + 1 <- channels 32j + 8 tig + {0, 4} ({2, 6}) and k-slots
// 2 tig + 8, + 9 <- channels 32j + 8 tig + {1, 5} ({3, 7}).
template <typename T>
__device__ __forceinline__ void q_words_q4(const uint32_t *qrow, int ks, int tig, uint32_t &w0,
                                           uint32_t &w1) {
  const int base = (ks >> 1) * 16 + tig * 4 + (ks & 1);  // word of channels 8 tig + {0,1} or {2,3}
  const uint32_t lo = q_to_f16x2<T>(__ldg(qrow + base)), hi = q_to_f16x2<T>(__ldg(qrow + base + 2));
  w0 = __byte_perm(lo, hi, 0x5410);
  w1 = __byte_perm(lo, hi, 0x7632);
}
// Output channel of accumulator element e of m-tile mt (INT4 tile).
__device__ __forceinline__ int dim_q4(int mt, int e, int g8) {
  return (mt >> 1) * 32 + 4 * g8 + 2 * (mt & 1) + (e >> 1);
}

// Byte offset of 16-byte chunk c of token row t in a 16-row page of 128-byte
// rows staged by one 128B-swizzled TMA box.
__device__ __forceinline__ uint32_t swz8(int t, int c) {
  return static_cast<uint32_t>(t * 128 + ((c ^ (t & 7)) << 4));
}

// The same for a page of R-byte rows (R = 128: the 128-byte swizzle above;
// R = 64: the 64-byte swizzle, chunk c of row t at chunk c ^ ((t >> 1) & 3);
// R = 32: the 32-byte swizzle, chunk c ^ ((t >> 2) & 1) -- in each case the
// 8 rows an ldmatrix reads fall on distinct banks).
template <int R>
__device__ __forceinline__ uint32_t swz_rows(int t, int c) {
  static_assert(R == 128 || R == 64 || R == 32, "code rows of 32, 64 or 128 bytes");
  if constexpr (R == 128) return swz8(t, c);
  else if constexpr (R == 64) return static_cast<uint32_t>(t * 64 + ((c ^ ((t >> 1) & 3)) << 4));
  else return static_cast<uint32_t>(t * 32 + ((c ^ ((t >> 2) & 1)) << 4));
}

// Eight INT4 codes (nibbles 0..7 of `w`, two's complement) -> four f16x2:
// out[s] holds the values of nibbles s (low half) and s + 4 (high half),
// exact.  With the sign bit flipped a nibble n reads n + 8.  The low nibble of
// each 16-bit half, flipped and with 0x6400 above it (one AND-XOR), is the f16
// 1024 + (n + 8), and 1032 is subtracted; the next nibble up, masked in place,
// is 1024 + 16 (n + 8), scaled by 1/16 with 72 subtracted in one fma.  Every
// intermediate is an integer (or a sixteenth of one) below 2048, so both
// steps are exact.  Nibbles 2, 3, 6, 7 do the same after one shift by 8.
__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t f16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ void int4x8_to_f16x2x4(uint32_t w, uint32_t (&out)[4]) {
  constexpr uint32_t kLoBias = 0x64086408u;   // f16x2 (1032, 1032)
  constexpr uint32_t kSixteenth = 0x2C002C00u;  // f16x2 (1/16, 1/16)
  constexpr uint32_t kMinus72 = 0xD480D480u;  // f16x2 (-72, -72)
  const uint32_t w8 = w >> 8;
  out[0] = f16x2_sub((w & 0x000F000Fu) ^ kLoBias, kLoBias);
  out[1] = f16x2_fma((w & 0x00F000F0u) ^ 0x64806480u, kSixteenth, kMinus72);
  out[2] = f16x2_sub((w8 & 0x000F000Fu) ^ kLoBias, kLoBias);
  out[3] = f16x2_fma((w8 & 0x00F000F0u) ^ 0x64806480u, kSixteenth, kMinus72);
}

// One 16-token page of an 8-bit cache (d = D = 64 or 128; E4M3 or INT8 codes)
// for 8*NT query rows of one warp.  Codes are exact in f16, so the tensor-core tile
// runs in f16:
//  * K: ldmatrix on the code bytes gives each lane four consecutive channels
//    of a token per register; converted in pairs they fill the A fragment
//    with the channel order permuted inside each 16-channel k-step (the q
//    fragments, `qf`, use the same order).  Scores are summed per 32-channel
//    group and then weighted by the token's group scales.
//  * V: ldmatrix.trans on the code bytes gives (channel pair) x (token pair);
//    a byte permute splits it into the A fragments of V^T, with output slot
//    g8 <-> channel 2*g8 and slot g8+8 <-> channel 2*g8+1 of each m-tile.
//    The V group scales ride on the probabilities (one P^T operand per group).
// ks, vs: the page's fp32 scales in shared memory, [16 tokens][D / 32 groups].
template <int D, int NT, Code8 kFmt>
__device__ __forceinline__ void tile_page_q8(uint32_t kb, uint32_t vb, const float *ks,
                                              const float *vs, int ntok, float scale_log2,
                                              int lane, const uint32_t (&qf)[NT][D / 16][2],
                                              float (&acc)[NT][D / 16][4], float (&m_run)[NT][2],
                                              float (&l_run)[NT][2]) {
  using M = Mma<__half>;
  constexpr int kG = D / 32;  // scale groups of a token
  const int g8 = lane >> 2;
  const int mi = lane >> 3, r8 = lane & 7;
  const int tok = r8 + ((mi & 1) << 3);  // row this lane addresses for ldmatrix
  const int hi16 = mi >> 1;              // second 16 bytes of a 32-channel group

  float sg[kG][NT][4];
#pragma unroll
  for (int j = 0; j < kG; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sg[j][nt][e] = 0.f;
#pragma unroll
  for (int j = 0; j < kG; ++j) {
    uint32_t R[4];
    ldmatrix_x4(R, kb + swz_rows<D>(tok, 2 * j + hi16));
    uint32_t A0[4], A1[4];
    code8x4_to_f16x2x2<kFmt>(R[0], A0[0], A0[2]);
    code8x4_to_f16x2x2<kFmt>(R[1], A0[1], A0[3]);
    code8x4_to_f16x2x2<kFmt>(R[2], A1[0], A1[2]);
    code8x4_to_f16x2x2<kFmt>(R[3], A1[1], A1[3]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      M::run(sg[j][nt], A0, qf[nt][2 * j][0], qf[nt][2 * j][1]);
      M::run(sg[j][nt], A1, qf[nt][2 * j + 1][0], qf[nt][2 * j + 1][1]);
    }
  }
  // the scales of this lane's two tokens (g8 and g8 + 8), K and V
  float kAs[kG], kBs[kG], vAs[kG], vBs[kG];
  if constexpr (kG == 4) {
    const float4 kA = *reinterpret_cast<const float4 *>(ks + g8 * 4);
    const float4 kB = *reinterpret_cast<const float4 *>(ks + (g8 + 8) * 4);
    const float4 vA = *reinterpret_cast<const float4 *>(vs + g8 * 4);
    const float4 vB = *reinterpret_cast<const float4 *>(vs + (g8 + 8) * 4);
    kAs[0] = kA.x; kAs[1] = kA.y; kAs[2] = kA.z; kAs[3] = kA.w;
    kBs[0] = kB.x; kBs[1] = kB.y; kBs[2] = kB.z; kBs[3] = kB.w;
    vAs[0] = vA.x; vAs[1] = vA.y; vAs[2] = vA.z; vAs[3] = vA.w;
    vBs[0] = vB.x; vBs[1] = vB.y; vBs[2] = vB.z; vBs[3] = vB.w;
  } else {
    const float2 kA = *reinterpret_cast<const float2 *>(ks + g8 * 2);
    const float2 kB = *reinterpret_cast<const float2 *>(ks + (g8 + 8) * 2);
    const float2 vA = *reinterpret_cast<const float2 *>(vs + g8 * 2);
    const float2 vB = *reinterpret_cast<const float2 *>(vs + (g8 + 8) * 2);
    kAs[0] = kA.x; kAs[1] = kA.y;
    kBs[0] = kB.x; kBs[1] = kB.y;
    vAs[0] = vA.x; vAs[1] = vA.y;
    vBs[0] = vB.x; vBs[1] = vB.y;
  }

  const bool v0 = g8 < ntok, v1 = g8 + 8 < ntok;
  float x[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      s4[0] += sg[j][nt][0] * kAs[j];
      s4[1] += sg[j][nt][1] * kAs[j];
      s4[2] += sg[j][nt][2] * kBs[j];
      s4[3] += sg[j][nt][3] * kBs[j];
    }
    x[nt][0] = v0 ? s4[0] * scale_log2 : -INFINITY;
    x[nt][1] = v0 ? s4[1] * scale_log2 : -INFINITY;
    x[nt][2] = v1 ? s4[2] * scale_log2 : -INFINITY;
    x[nt][3] = v1 ? s4[3] * scale_log2 : -INFINITY;
  }
  ref_max_update<NT, D / 16, 4>(x, m_run, l_run, acc);
  uint32_t pj0[kG][NT], pj1[kG][NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float e0 = fast_exp2(x[nt][0] - m_run[nt][0]), e1 = fast_exp2(x[nt][1] - m_run[nt][1]);
    const float e2 = fast_exp2(x[nt][2] - m_run[nt][0]), e3 = fast_exp2(x[nt][3] - m_run[nt][1]);
    l_run[nt][0] += e0 + e2;
    l_run[nt][1] += e1 + e3;
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      // masked tokens have e = 0 and a V scale of 0 (cleared by the caller)
      pj0[j][nt] = movmatrix_trans(f16pack(e0 * vAs[j], e1 * vAs[j]));
      pj1[j][nt] = movmatrix_trans(f16pack(e2 * vBs[j], e3 * vBs[j]));
    }
  }
#pragma unroll
  for (int j = 0; j < kG; ++j) {
    uint32_t R[4];
    ldmatrix_x4_trans(R, vb + swz_rows<D>(tok, 2 * j + hi16));
    // R[0]: tokens 0-7, R[1]: tokens 8-15 (channels 32j..+15); R[2], R[3]: +16
    uint32_t A[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // bytes (0, 2) and (1, 3) of each word: the two channels of a pair
      code8x4_to_f16x2x2_0213<kFmt>(R[2 * h], A[h][0], A[h][1]);
      code8x4_to_f16x2x2_0213<kFmt>(R[2 * h + 1], A[h][2], A[h][3]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      M::run(acc[nt][2 * j], A[0], pj0[j][nt], pj1[j][nt]);
      M::run(acc[nt][2 * j + 1], A[1], pj0[j][nt], pj1[j][nt]);
    }
  }
}

// One 16-token page of an INT4 cache (d = D = 64 or 128: code rows of D / 2
// bytes, 32 channels per 16-byte chunk, one scale group per chunk) for 8*NT
// query rows of one warp, on the f16 tensor-core tile.
//  * K: ldmatrix gives each lane 8 consecutive channels 8 tig .. 8 tig + 7 of
//    one token per register.  int4x8_to_f16x2x4 pairs channels (8 tig + s,
//    8 tig + s + 4); pairs s = 0, 1 fill k-step 2j of group j's A operand,
//    s = 2, 3 k-step 2j + 1 (Page4::q_words orders q the same way).  Scores
//    are summed per group and weighted by the token's group scales.
//  * V: ldmatrix.trans gives each lane 4 channels 4 g8 .. 4 g8 + 3 of two
//    consecutive tokens per register; the same conversion pairs each channel
//    across the two tokens, which is exactly an A-fragment register of V^T.
//    Group j makes two m-tiles: rows g8, g8 + 8 <-> channels 32j + 4 g8 + 2t
//    and 32j + 4 g8 + 2t + 1 for m-tile 2j + t (Page4::dim).  The V group
//    scales ride on the probabilities, as in the 8-bit tile.
template <int D, int NT>
__device__ __forceinline__ void tile_page_q4(uint32_t kb, uint32_t vb, const float *ks,
                                              const float *vs, int ntok, float scale_log2,
                                              int lane, const uint32_t (&qf)[NT][D / 16][2],
                                              float (&acc)[NT][D / 16][4], float (&m_run)[NT][2],
                                              float (&l_run)[NT][2]) {
  using M = Mma<__half>;
  constexpr int kG = D / 32;  // scale groups = 16-byte chunks of a code row
  static_assert(kG % 2 == 0, "code rows of whole chunk pairs");
  const int g8 = lane >> 2;
  const int mi = lane >> 3, r8 = lane & 7;
  const int tok = r8 + ((mi & 1) << 3);  // row this lane addresses for ldmatrix
  const int hi = mi >> 1;                // second chunk of a pair

  float sg[kG][NT][4];
#pragma unroll
  for (int j = 0; j < kG; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sg[j][nt][e] = 0.f;
#pragma unroll
  for (int jj = 0; jj < kG / 2; ++jj) {
    uint32_t R[4];  // tokens 0-7 / 8-15 of chunk 2jj, then of chunk 2jj + 1
    ldmatrix_x4(R, kb + swz_rows<D / 2>(tok, 2 * jj + hi));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * jj + h;
      uint32_t p[4], q[4];  // token g8, token g8 + 8
      int4x8_to_f16x2x4(R[2 * h], p);
      int4x8_to_f16x2x4(R[2 * h + 1], q);
      const uint32_t A0[4] = {p[0], q[0], p[1], q[1]};
      const uint32_t A1[4] = {p[2], q[2], p[3], q[3]};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        M::run(sg[j][nt], A0, qf[nt][2 * j][0], qf[nt][2 * j][1]);
        M::run(sg[j][nt], A1, qf[nt][2 * j + 1][0], qf[nt][2 * j + 1][1]);
      }
    }
  }
  // the scales of this lane's two tokens (g8 and g8 + 8), K and V
  float kAs[kG], kBs[kG], vAs[kG], vBs[kG];
  if constexpr (kG == 4) {
    const float4 kA = *reinterpret_cast<const float4 *>(ks + g8 * 4);
    const float4 kB = *reinterpret_cast<const float4 *>(ks + (g8 + 8) * 4);
    const float4 vA = *reinterpret_cast<const float4 *>(vs + g8 * 4);
    const float4 vB = *reinterpret_cast<const float4 *>(vs + (g8 + 8) * 4);
    kAs[0] = kA.x; kAs[1] = kA.y; kAs[2] = kA.z; kAs[3] = kA.w;
    kBs[0] = kB.x; kBs[1] = kB.y; kBs[2] = kB.z; kBs[3] = kB.w;
    vAs[0] = vA.x; vAs[1] = vA.y; vAs[2] = vA.z; vAs[3] = vA.w;
    vBs[0] = vB.x; vBs[1] = vB.y; vBs[2] = vB.z; vBs[3] = vB.w;
  } else {
    const float2 kA = *reinterpret_cast<const float2 *>(ks + g8 * 2);
    const float2 kB = *reinterpret_cast<const float2 *>(ks + (g8 + 8) * 2);
    const float2 vA = *reinterpret_cast<const float2 *>(vs + g8 * 2);
    const float2 vB = *reinterpret_cast<const float2 *>(vs + (g8 + 8) * 2);
    kAs[0] = kA.x; kAs[1] = kA.y;
    kBs[0] = kB.x; kBs[1] = kB.y;
    vAs[0] = vA.x; vAs[1] = vA.y;
    vBs[0] = vB.x; vBs[1] = vB.y;
  }

  const bool v0 = g8 < ntok, v1 = g8 + 8 < ntok;
  float x[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      s4[0] += sg[j][nt][0] * kAs[j];
      s4[1] += sg[j][nt][1] * kAs[j];
      s4[2] += sg[j][nt][2] * kBs[j];
      s4[3] += sg[j][nt][3] * kBs[j];
    }
    x[nt][0] = v0 ? s4[0] * scale_log2 : -INFINITY;
    x[nt][1] = v0 ? s4[1] * scale_log2 : -INFINITY;
    x[nt][2] = v1 ? s4[2] * scale_log2 : -INFINITY;
    x[nt][3] = v1 ? s4[3] * scale_log2 : -INFINITY;
  }
  ref_max_update<NT, D / 16, 4>(x, m_run, l_run, acc);
  uint32_t pj0[kG][NT], pj1[kG][NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float e0 = fast_exp2(x[nt][0] - m_run[nt][0]), e1 = fast_exp2(x[nt][1] - m_run[nt][1]);
    const float e2 = fast_exp2(x[nt][2] - m_run[nt][0]), e3 = fast_exp2(x[nt][3] - m_run[nt][1]);
    l_run[nt][0] += e0 + e2;
    l_run[nt][1] += e1 + e3;
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      // masked tokens have e = 0 and a V scale of 0 (cleared by the caller)
      pj0[j][nt] = movmatrix_trans(f16pack(e0 * vAs[j], e1 * vAs[j]));
      pj1[j][nt] = movmatrix_trans(f16pack(e2 * vBs[j], e3 * vBs[j]));
    }
  }
#pragma unroll
  for (int jj = 0; jj < kG / 2; ++jj) {
    uint32_t R[4];  // transposed: tokens 0-7 / 8-15 of chunk 2jj, then of 2jj + 1
    ldmatrix_x4_trans(R, vb + swz_rows<D / 2>(tok, 2 * jj + hi));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * jj + h;
      uint32_t u[4], w[4];  // channel 4 g8 + c of tokens (2 tig, +1) / (8 + 2 tig, +1)
      int4x8_to_f16x2x4(R[2 * h], u);
      int4x8_to_f16x2x4(R[2 * h + 1], w);
      const uint32_t A0[4] = {u[0], u[1], w[0], w[1]};
      const uint32_t A1[4] = {u[2], u[3], w[2], w[3]};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        M::run(acc[nt][2 * j], A0, pj0[j][nt], pj1[j][nt]);
        M::run(acc[nt][2 * j + 1], A1, pj0[j][nt], pj1[j][nt]);
      }
    }
  }
}

// ------------------------------------------------------------ one query row
//
// A quantised page for a KV head with a single query row (G = 1), on the
// tensor-core tile whose N dimension would otherwise hold 7 idle rows.  The
// N columns carry the 32-channel scale groups instead:
//  * K: q's fragment of k-step ks is placed in column ks / 2 only (the
//    caller loads it so), so S^T[token][group] -- each group's partial score
//    -- builds up in ONE accumulator; lanes with columns 2 tig, 2 tig + 1
//    weigh them by the token's K scales and a shuffle with the neighbour
//    lane completes the score.
//  * V: the B operand is X[token][group] = p_token * v_scale[token][group],
//    one operand for all groups; O^T[channel][group] accumulates, and each
//    channel's value is the entry of its own group's column.
// `g1_to_rows` moves those entries to the layout of the general tile (row 0
// in lanes tig == 0) when a pair is finished.  m_run / l_run use row 0; the
// running sum counts each token once (lanes tig == 0).  The code layouts and
// conversions are those of tile_page_q8 (8-bit) and tile_page_q4 (INT4).
template <int D, bool kInt4, Code8 kFmt>
__device__ __forceinline__ void tile_page_g1(uint32_t kb, uint32_t vb, const float *ks,
                                             const float *vs, int ntok, float scale_log2, int lane,
                                             const uint32_t (&qf)[1][D / 16][2],
                                             float (&acc)[1][D / 16][4], float (&m_run)[1][2],
                                             float (&l_run)[1][2]) {
  using M = Mma<__half>;
  constexpr int kG = D / 32;
  const int g8 = lane >> 2, tig = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;
  const int tok = r8 + ((mi & 1) << 3);
  const int hi = mi >> 1;

  // S^T[token][group], two independent chains (even / odd groups)
  float s[2][4];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[c][e] = 0.f;
  if constexpr (kInt4) {
#pragma unroll
    for (int jj = 0; jj < kG / 2; ++jj) {
      uint32_t R[4];
      ldmatrix_x4(R, kb + swz_rows<D / 2>(tok, 2 * jj + hi));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 2 * jj + h;
        uint32_t p[4], q[4];
        int4x8_to_f16x2x4(R[2 * h], p);
        int4x8_to_f16x2x4(R[2 * h + 1], q);
        const uint32_t A0[4] = {p[0], q[0], p[1], q[1]};
        const uint32_t A1[4] = {p[2], q[2], p[3], q[3]};
        M::run(s[h], A0, qf[0][2 * j][0], qf[0][2 * j][1]);
        M::run(s[h], A1, qf[0][2 * j + 1][0], qf[0][2 * j + 1][1]);
      }
    }
  } else {
    const int hi16 = hi;
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      uint32_t R[4];
      ldmatrix_x4(R, kb + swz_rows<D>(tok, 2 * j + hi16));
      uint32_t A0[4], A1[4];
      code8x4_to_f16x2x2<kFmt>(R[0], A0[0], A0[2]);
      code8x4_to_f16x2x2<kFmt>(R[1], A0[1], A0[3]);
      code8x4_to_f16x2x2<kFmt>(R[2], A1[0], A1[2]);
      code8x4_to_f16x2x2<kFmt>(R[3], A1[1], A1[3]);
      M::run(s[j & 1], A0, qf[0][2 * j][0], qf[0][2 * j][1]);
      M::run(s[j & 1], A1, qf[0][2 * j + 1][0], qf[0][2 * j + 1][1]);
    }
  }
  // this lane's columns 2 tig, 2 tig + 1 are groups when 2 tig < kG
  const bool cols = 2 * tig < kG;
  const int cg = cols ? 2 * tig : 0;
  const float2 kA = *reinterpret_cast<const float2 *>(ks + g8 * kG + cg);
  const float2 kB = *reinterpret_cast<const float2 *>(ks + (g8 + 8) * kG + cg);
  const float2 vA = *reinterpret_cast<const float2 *>(vs + g8 * kG + cg);
  const float2 vB = *reinterpret_cast<const float2 *>(vs + (g8 + 8) * kG + cg);
  float p0 = (s[0][0] + s[1][0]) * kA.x + (s[0][1] + s[1][1]) * kA.y;  // token g8
  float p8 = (s[0][2] + s[1][2]) * kB.x + (s[0][3] + s[1][3]) * kB.y;  // token g8 + 8
  p0 = cols ? p0 : 0.f;
  p8 = cols ? p8 : 0.f;
  p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
  p8 += __shfl_xor_sync(0xffffffffu, p8, 1);
  const float x0 = (cols && g8 < ntok) ? p0 * scale_log2 : -INFINITY;
  const float x8 = (cols && g8 + 8 < ntok) ? p8 * scale_log2 : -INFINITY;

  // reference maximum of the single row (see ref_max_update)
  float &m = m_run[0][0];
  const bool up = (x0 > m + kTileRefSlack) | (x8 > m + kTileRefSlack);
  if (__any_sync(0xffffffffu, up)) {
    float mx = fmaxf(x0, x8);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float mn = fmaxf(m, mx);
    const float al = mn == -INFINITY ? 1.f : fast_exp2(m - mn);
    m = mn;
    l_run[0][0] *= al;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[0][mt][e] *= al;
  }
  const float e0 = fast_exp2(x0 - m), e8 = fast_exp2(x8 - m);
  if (tig == 0) l_run[0][0] += e0 + e8;
  // X[token][group]: masked tokens have e = 0 and V scales of 0 (cleared by
  // the caller); non-group columns have scales read as 0 products of e = 0
  const uint32_t pj0 = movmatrix_trans(f16pack(e0 * vA.x, e0 * vA.y));
  const uint32_t pj1 = movmatrix_trans(f16pack(e8 * vB.x, e8 * vB.y));

  if constexpr (kInt4) {
#pragma unroll
    for (int jj = 0; jj < kG / 2; ++jj) {
      uint32_t R[4];
      ldmatrix_x4_trans(R, vb + swz_rows<D / 2>(tok, 2 * jj + hi));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 2 * jj + h;
        uint32_t u[4], w[4];
        int4x8_to_f16x2x4(R[2 * h], u);
        int4x8_to_f16x2x4(R[2 * h + 1], w);
        const uint32_t A0[4] = {u[0], u[1], w[0], w[1]};
        const uint32_t A1[4] = {u[2], u[3], w[2], w[3]};
        M::run(acc[0][2 * j], A0, pj0, pj1);
        M::run(acc[0][2 * j + 1], A1, pj0, pj1);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      uint32_t R[4];
      ldmatrix_x4_trans(R, vb + swz_rows<D>(tok, 2 * j + hi));
      uint32_t A[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        code8x4_to_f16x2x2_0213<kFmt>(R[2 * h], A[h][0], A[h][1]);
        code8x4_to_f16x2x2_0213<kFmt>(R[2 * h + 1], A[h][2], A[h][3]);
      }
      M::run(acc[0][2 * j], A[0], pj0, pj1);
      M::run(acc[0][2 * j + 1], A[1], pj0, pj1);
    }
  }
}

// The state of tile_page_g1 in the layout of the general tile: the value of
// m-tile mt (group mt / 2) moves from column mt / 2 -- lane tig = mt / 4,
// element (mt / 2) & 1 (+ 2 for the second channel row) -- to column 0.
template <int MT>
__device__ __forceinline__ void g1_to_rows(float (&acc)[1][MT][4], int lane) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int j = mt >> 1;
    const int src = (lane & ~3) | (j >> 1);
    const float v0 = __shfl_sync(0xffffffffu, acc[0][mt][j & 1], src);
    const float v2 = __shfl_sync(0xffffffffu, acc[0][mt][2 + (j & 1)], src);
    acc[0][mt][0] = v0;
    acc[0][mt][2] = v2;
  }
}

}  // namespace kvd

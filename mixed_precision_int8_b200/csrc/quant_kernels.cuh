// HBM-bound kernels around the int8 GEMM:
//   K0  offline weight preparation (column absmax + int8 codes, transposed)
//   K1  activation pass: outlier-column bitmask, compaction of the outlier
//       list, per-row absmax over regular columns and int8 row codes
//   K2  fp16 outlier rows of W recovered from the int8 weight (same launch
//       as the row quantisation)
//
// Magnitude trick used throughout: for a non-NaN binary16 value, the bit
// pattern with the sign cleared orders exactly like |x|, so maxima and the
// threshold test |x| >= alpha run on 16-bit integers (the threshold is the
// smallest binary16 magnitude >= alpha, found once on the host).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "ptx_sm100.cuh"

namespace llmint8 {

// Absmax code of x against scale a: fp32 product 127*x (exact for binary16
// x), one IEEE fp32 division, round half away from zero (roundf). a == 0
// gives 0. "tm_llm_int8", section "Absmax INT8 quantization from first
// principles"; "LLM.int8(): 8-bit Matrix Multiplication for Transformers at
// Scale", section "Quantization Primitives".
__device__ __forceinline__ int32_t absmax_code(float x, float a) {
  if (a == 0.0f) return 0;
  const float v = __fdiv_rn(127.0f * x, a);
  const float r = fminf(fmaxf(roundf(v), -127.0f), 127.0f);
  return static_cast<int32_t>(r);
}

// The same code without a division per element, for a row that shares one
// scale a > 0 with r ~ 1/a (a few ulps of error are fine). With t = 127|x|
// (exact in fp32), the candidate n = floor(t*r + 1/2) is within one of the
// correctly rounded result; the residuals t - (n -+ 1/2) a are computed by one
// FMA each and are exact in sign, because (n -+ 1/2) has at most 9 significant
// bits and a at most 11, so the products are exact fp32 values. After the
// correction (n - 1/2) a <= t < (n + 1/2) a, i.e. n rounds 127|x|/a half away
// from zero, which is the value absmax_code() produces (its single fp32
// division cannot move the quotient across a half-integer: the distance of
// 127x/a from one is at least 2^-12 or q * 2^-19, above the division's error).
__device__ __forceinline__ int32_t absmax_code_recip(float x, float a, float r) {
  const float t = 127.0f * fabsf(x);
  float n = floorf(fmaf(t, r, 0.5f));
  // (n + 1/2) a > (n - 1/2) a, so at most one of the two corrections applies
  const float below = fmaf(-(n - 0.5f), a, t) < 0.0f ? 1.0f : 0.0f;
  const float above = fmaf(-(n + 0.5f), a, t) >= 0.0f ? 1.0f : 0.0f;
  n = fminf(n + above - below, 127.0f);
  return static_cast<int32_t>(copysignf(n, x));
}

// Fast form of absmax_code_recip. With r = 1/a correctly rounded, y =
// fma(t, r, 1/2) is within 2^-16 of t/a + 1/2 (t/a <= 127: the reciprocal
// contributes < 2^-17 and the fma rounding <= 2^-18), so when the fractional
// part of y is at least 2^-15 away from an integer, floor(y) is already
// floor(t/a + 1/2), the exactly rounded code. Only values that close to a
// rounding boundary (about 6 in 10^5) take the exact two-residual correction.
__device__ __forceinline__ int32_t absmax_code_fast(float x, float a, float r) {
  const float t = 127.0f * fabsf(x);
  const float y = fmaf(t, r, 0.5f);
  const float n0 = floorf(y);
  float n = n0;
  if (fabsf((y - n0) - 0.5f) > 0.5f - 3.0517578125e-05f) {  // within 2^-15 of an integer
    const float below = fmaf(-(n0 - 0.5f), a, t) < 0.0f ? 1.0f : 0.0f;
    const float above = fmaf(-(n0 + 0.5f), a, t) >= 0.0f ? 1.0f : 0.0f;
    n = fminf(n0 + above - below, 127.0f);
  }
  return static_cast<int32_t>(copysignf(n, x));
}

__device__ __forceinline__ float half_bits_to_float(uint32_t b) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
}

__device__ __forceinline__ uint32_t pack4_i8(int32_t a, int32_t b, int32_t c, int32_t d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

// ------------------------------------------------------------------ K1a
// Zero the outlier bitmask, the outlier count and the column pass's block
// counter before a new call (and, for the decode path, the int32 partial-sum
// buffer). Every kernel of a call waits on its predecessor with
// griddepcontrol.wait before touching memory, so programmatic dependent
// launches keep stream order.
__global__ void k_reset_mask(uint32_t *__restrict__ mask, int32_t nwords,
                             int32_t *__restrict__ count, int32_t *__restrict__ block_counter,
                             int32_t *__restrict__ zero_buf, int64_t zero_n) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t w = i; w < nwords; w += stride) mask[w] = 0u;
  for (int64_t w = i; w < zero_n; w += stride) zero_buf[w] = 0;
  if (i == 0) {
    *count = 0;          // |O|
    *block_counter = 0;  // finished blocks of the column pass
  }
}

constexpr int kColThreads = 256;
constexpr int kColsPerBlock = kColThreads * 8;

// Compaction of the bitmask into the ascending outlier list by one block:
// word_prefix[w] = number of outlier columns before word w, idx[] = the
// outlier columns, *count = |O|, flags[j] (optional) = bit j.
template <int kThreads>
__device__ void compact_outliers_block(const uint32_t *__restrict__ mask, int32_t nwords,
                                       int32_t h, int32_t *__restrict__ word_prefix,
                                       int32_t *__restrict__ idx, int32_t *__restrict__ count,
                                       uint8_t *__restrict__ flags) {
  __shared__ int32_t warp_sums[32];
  const int tid = threadIdx.x;
  const int per = (nwords + kThreads - 1) / kThreads;
  const int w0 = tid * per;
  const int w1 = min(nwords, w0 + per);
  int32_t local = 0;
  for (int w = w0; w < w1; ++w) local += __popc(__ldcg(mask + w));
  const int lane = tid & 31, warp = tid >> 5;
  int32_t incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t v = lane < kThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t y = __shfl_up_sync(0xFFFFFFFFu, v, d);
      if (lane >= d) v += y;
    }
    warp_sums[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  int32_t base = incl - local + (warp > 0 ? warp_sums[warp - 1] : 0);
  for (int w = w0; w < w1; ++w) {
    const uint32_t m = __ldcg(mask + w);
    word_prefix[w] = base;
    uint32_t mm = m;
    while (mm) {
      const int b = __ffs(mm) - 1;
      idx[base++] = w * 32 + b;
      mm &= mm - 1;
    }
    if (flags) {
      for (int b = 0; b < 32; ++b) {
        const int j = w * 32 + b;
        if (j < h) flags[j] = static_cast<uint8_t>((m >> b) & 1u);
      }
    }
  }
  if (tid == kThreads - 1) {
    word_prefix[nwords] = base;
    *count = base;
  }
}

// Step 1 ("The Full LLM.int8() Algorithm"): a column is an outlier column
// when any row holds |x| >= alpha. Each thread owns 8 adjacent columns (one
// 16-byte load per row) over `rows_per_block` rows; four lanes fold their
// 8-bit masks into one 32-bit word that is OR-ed into the global bitmask.
// The last block to finish compacts the bitmask into the outlier list.
__global__ void __launch_bounds__(kColThreads)
    k_outlier_columns(const uint16_t *__restrict__ X, int64_t s, int32_t h,
                      uint32_t thresh_bits, int32_t rows_per_block, uint32_t *__restrict__ mask,
                      int32_t *__restrict__ count, int32_t *__restrict__ block_counter,
                      int32_t *__restrict__ word_prefix, int32_t *__restrict__ idx,
                      uint8_t *__restrict__ flags) {
  __shared__ int is_last;
  grid_dependency_wait();
  grid_dependency_trigger();
  const int32_t c = blockIdx.x * kColsPerBlock + threadIdx.x * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
  const int64_t r1 = min(s, r0 + rows_per_block);
  uint32_t m2[4] = {0u, 0u, 0u, 0u};  // per-halfword magnitude maxima
  if (c < h) {
    const uint16_t *p = X + r0 * h + c;
    int64_t r = r0;
    for (; r + 8 <= r1; r += 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(reinterpret_cast<const uint4 *>(p + u * (int64_t)h));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        m2[0] = __vmaxu2(m2[0], v[u].x & 0x7FFF7FFFu);
        m2[1] = __vmaxu2(m2[1], v[u].y & 0x7FFF7FFFu);
        m2[2] = __vmaxu2(m2[2], v[u].z & 0x7FFF7FFFu);
        m2[3] = __vmaxu2(m2[3], v[u].w & 0x7FFF7FFFu);
      }
      p += 8 * (int64_t)h;
    }
    for (; r < r1; ++r) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
      m2[0] = __vmaxu2(m2[0], v.x & 0x7FFF7FFFu);
      m2[1] = __vmaxu2(m2[1], v.y & 0x7FFF7FFFu);
      m2[2] = __vmaxu2(m2[2], v.z & 0x7FFF7FFFu);
      m2[3] = __vmaxu2(m2[3], v.w & 0x7FFF7FFFu);
      p += h;
    }
  }
  uint32_t m8 = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    m8 |= ((m2[e] & 0xFFFFu) >= thresh_bits ? 1u : 0u) << (2 * e);
    m8 |= ((m2[e] >> 16) >= thresh_bits ? 1u : 0u) << (2 * e + 1);
  }
  const int lane = threadIdx.x & 31;
  uint32_t word = m8 << (8 * (lane & 3));
  word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
  word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
  const bool wrote = (lane & 3) == 0 && word != 0u && c < h;
  if (wrote) {
    atomicOr(mask + (c >> 5), word);
    __threadfence();  // order this thread's bits before the block's arrival
  }
  // last-block-done: the final block sees every other block's bits
  __syncthreads();
  if (threadIdx.x == 0) {
    const int total = gridDim.x * gridDim.y;
    is_last = (atomicAdd(block_counter, 1) == total - 1);
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    compact_outliers_block<kColThreads>(mask, (h + 31) / 32, h, word_prefix, idx, count,
                                        flags);
  }
}

// Step 4 (activation side) with the X half of Step 2:
//   ax[i]    = max over regular columns of |X[i][j]|            (exact)
//   Xq[i][j] = code(X[i][j], ax[i]) on regular columns, 0 on outlier ones
//   XO[i][t] = X[i][O_t]  (fp16, row stride |O|; optional)
// and, in the same launch, the W half of Step 2 (k_rows_and_outlier_w).

// Outlier position of column c + e (its rank among the outlier columns).
__device__ __forceinline__ int32_t outlier_rank(const int32_t *word_prefix, uint32_t mask_word,
                                                int32_t c, int e) {
  const int bit = (c & 31) + e;
  return word_prefix[c >> 5] + __popc(mask_word & ((1u << bit) - 1u));
}

// Four codes (low bytes of a..d) packed into one word, byte 0 = a.
__device__ __forceinline__ uint32_t pack4_bytes(int32_t a, int32_t b, int32_t c, int32_t d) {
  const uint32_t ab = __byte_perm((uint32_t)a, (uint32_t)b, 0x0040);
  const uint32_t cd = __byte_perm((uint32_t)c, (uint32_t)d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

// Codes for one 16-byte chunk (8 columns starting at c) of row `row`, whose
// scale is a (r ~ 1/a; a == 0 gives zero codes).
__device__ __forceinline__ void quantize_chunk(const uint4 v, uint32_t mw, int32_t c, float a,
                                               float r, int64_t row, int32_t n_out,
                                               const int32_t *word_prefix,
                                               int8_t *__restrict__ qr,
                                               uint16_t *__restrict__ XO) {
  const uint32_t mk = (mw >> (c & 31)) & 0xFFu;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  int32_t q[8];
  if (a == 0.0f) {
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = 0;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[e]));
      q[2 * e] = absmax_code_fast(f.x, a, r);
      q[2 * e + 1] = absmax_code_fast(f.y, a, r);
    }
    if (mk != 0u) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if ((mk >> e) & 1u) q[e] = 0;
    }
  }
  uint2 packed;
  packed.x = pack4_bytes(q[0], q[1], q[2], q[3]);
  packed.y = pack4_bytes(q[4], q[5], q[6], q[7]);
  *reinterpret_cast<uint2 *>(qr + c) = packed;
  if (mk != 0u && XO != nullptr) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if ((mk >> e) & 1u) {
        const uint32_t hv = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
        XO[row * n_out + outlier_rank(word_prefix, mw, c, e)] = static_cast<uint16_t>(hv);
      }
    }
  }
}

// Running per-halfword maximum of the magnitude bits of the regular columns
// of one chunk (mk: outlier bits of its 8 columns), two columns per word.
__device__ __forceinline__ uint32_t regular_absmax2(uint32_t m2, const uint4 v, uint32_t mk) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (mk == 0u) {
#pragma unroll
    for (int e = 0; e < 4; ++e) m2 = __vmaxu2(m2, w[e] & 0x7FFF7FFFu);
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t keep = (((mk >> (2 * e)) & 1u) ? 0u : 0x7FFFu) |
                            (((mk >> (2 * e + 1)) & 1u) ? 0u : 0x7FFF0000u);
      m2 = __vmaxu2(m2, w[e] & keep);
    }
  }
  return m2;
}

__device__ __forceinline__ uint32_t max_halves(uint32_t m2) { return max(m2 & 0xFFFFu, m2 >> 16); }

// K2: WO[t][j] = fp16(fp32(fp32(wq[j][O_t]) * aw[j]) / 127) for one column j
// and every outlier t. The column of the int8 weight is a strided gather (one
// byte per 32-byte sector), so eight loads are kept in flight per thread.
__device__ __forceinline__ void outlier_weight_rows(const int8_t *__restrict__ wq,
                                                    const float *__restrict__ aw, int32_t h,
                                                    int32_t o, const int32_t *__restrict__ idx,
                                                    int32_t n, int32_t j,
                                                    uint16_t *__restrict__ WO) {
  if (j >= o) return;
  const float a = __ldg(aw + j);
  const int8_t *wr = wq + static_cast<int64_t>(j) * h;
  for (int32_t t0 = 0; t0 < n; t0 += 8) {
    int32_t b[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) b[u] = (t0 + u < n) ? wr[__ldg(idx + t0 + u)] : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (t0 + u < n) {
        const float prod = static_cast<float>(b[u]) * a;
        WO[static_cast<int64_t>(t0 + u) * o + j] =
            __half_as_ushort(__float2half_rn(__fdiv_rn(prod, 127.0f)));
      }
    }
  }
}

constexpr int kRowRegThreads = 128;  // one block per row, row held in registers

// Blocks [0, wo_blocks) build the fp16 outlier rows of W for 128 columns
// each (first, so their gather latency overlaps the rows); blocks
// [wo_blocks, wo_blocks + s) quantise one row each, the row held in
// registers (NV 16-byte chunks per thread, h <= NV * 1024).
template <int NV>
__global__ void __launch_bounds__(kRowRegThreads)
    k_rows_and_outlier_w(const uint16_t *__restrict__ X, int64_t s, int32_t h,
                         const uint32_t *__restrict__ mask,
                         const int32_t *__restrict__ word_prefix,
                         const int32_t *__restrict__ count, int8_t *__restrict__ Xq,
                         float *__restrict__ ax, uint16_t *__restrict__ XO,
                         const int8_t *__restrict__ wq, const float *__restrict__ aw, int32_t o,
                         const int32_t *__restrict__ idx, uint16_t *__restrict__ WO,
                         int32_t wo_blocks) {
  __shared__ uint32_t red[kRowRegThreads / 32];
  grid_dependency_wait();
  grid_dependency_trigger();
  const int tid = threadIdx.x;
  if ((int32_t)blockIdx.x < wo_blocks) {
    const int32_t j = (int32_t)blockIdx.x * kRowRegThreads + tid;
    outlier_weight_rows(wq, aw, h, o, idx, *count, j, WO);
    return;
  }
  const int64_t row = (int64_t)blockIdx.x - wo_blocks;
  const uint16_t *xr = X + row * h;
  uint4 v[NV];
  uint32_t mw[NV];
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const int32_t c = (u * kRowRegThreads + tid) * 8;
    if (c < h) {
      v[u] = __ldg(reinterpret_cast<const uint4 *>(xr + c));
      mw[u] = __ldg(mask + (c >> 5));
    }
  }
  uint32_t m2 = 0;
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const int32_t c = (u * kRowRegThreads + tid) * 8;
    if (c < h) m2 = regular_absmax2(m2, v[u], (mw[u] >> (c & 31)) & 0xFFu);
  }
  uint32_t mbits = max_halves(m2);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, d));
  if ((tid & 31) == 0) red[tid >> 5] = mbits;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kRowRegThreads / 32; ++w) mbits = max(mbits, red[w]);
  const float a = half_bits_to_float(mbits);
  const float r = a > 0.0f ? __frcp_rn(a) : 0.0f;
  if (tid == 0) ax[row] = a;
  const int32_t n_out = (XO != nullptr) ? *count : 0;
  int8_t *qr = Xq + row * h;
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const int32_t c = (u * kRowRegThreads + tid) * 8;
    if (c < h) quantize_chunk(v[u], mw[u], c, a, r, row, n_out, word_prefix, qr, XO);
  }
}

// Any h: one warp per row, the row read twice (second time from L1/L2);
// the first wo_blocks blocks build the fp16 outlier rows of W.
constexpr int kRowThreads = 256;
constexpr int kRowsPerBlock = kRowThreads / 32;

__global__ void __launch_bounds__(kRowThreads)
    k_rows_and_outlier_w_any(const uint16_t *__restrict__ X, int64_t s, int32_t h,
                             const uint32_t *__restrict__ mask,
                             const int32_t *__restrict__ word_prefix,
                             const int32_t *__restrict__ count, int8_t *__restrict__ Xq,
                             float *__restrict__ ax, uint16_t *__restrict__ XO,
                             const int8_t *__restrict__ wq, const float *__restrict__ aw,
                             int32_t o, const int32_t *__restrict__ idx,
                             uint16_t *__restrict__ WO, int32_t wo_blocks) {
  grid_dependency_wait();
  grid_dependency_trigger();
  if ((int32_t)blockIdx.x < wo_blocks) {
    const int32_t j = (int32_t)blockIdx.x * kRowThreads + threadIdx.x;
    outlier_weight_rows(wq, aw, h, o, idx, *count, j, WO);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t row =
      static_cast<int64_t>(blockIdx.x - wo_blocks) * kRowsPerBlock + (threadIdx.x >> 5);
  if (row >= s) return;
  const uint16_t *xr = X + row * h;
  uint32_t m2 = 0;
  for (int32_t c = lane * 8; c < h; c += 256) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + c));
    m2 = regular_absmax2(m2, v, (__ldg(mask + (c >> 5)) >> (c & 31)) & 0xFFu);
  }
  uint32_t mbits = max_halves(m2);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, d));
  const float a = half_bits_to_float(mbits);
  const float r = a > 0.0f ? __frcp_rn(a) : 0.0f;
  if (lane == 0) ax[row] = a;
  const int32_t n_out = (XO != nullptr) ? *count : 0;
  int8_t *qr = Xq + row * h;
  for (int32_t c = lane * 8; c < h; c += 256) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + c));
    quantize_chunk(v, __ldg(mask + (c >> 5)), c, a, r, row, n_out, word_prefix, qr, XO);
  }
}

// ----------------------------------------------------- K1 for s <= 16
// Decode-sized calls (s <= 16): every thread loads all s rows of its 8
// columns, so it knows those columns' outlier status by itself. Two launches
// of kDecodeColsPerBlock-column blocks then cover the activation side with
// no atomics and nothing to zero beforehand:
//   k_decode_colpass: bitmask words (plain stores) and, per block, the
//                     maximum over its regular columns of every row;
//                     extra blocks zero `zero_buf`.
//   k_decode_rowpass: row scales (max over the blocks' partial maxima),
//                     outlier prefix counts, |O|, codes and the fp16 outlier
//                     columns of X.
constexpr int kDecodeThreads = 128;
constexpr int kDecodeColsPerBlock = kDecodeThreads * 8;
constexpr int kSmallMaxRows = 16;

__global__ void __launch_bounds__(kDecodeThreads)
    k_decode_colpass(const uint16_t *__restrict__ X, int32_t s, int32_t h, uint32_t thresh_bits,
                     uint32_t *__restrict__ mask, uint32_t *__restrict__ partial_max,
                     int32_t col_blocks, int32_t *__restrict__ zero_buf, int64_t zero_n) {
  __shared__ uint32_t red[kDecodeThreads / 32][kSmallMaxRows];
  grid_dependency_wait();
  grid_dependency_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if ((int32_t)blockIdx.x >= col_blocks) {
    const int64_t stride = (int64_t)(gridDim.x - col_blocks) * blockDim.x;
    for (int64_t i = (int64_t)(blockIdx.x - col_blocks) * blockDim.x + tid; i < zero_n;
         i += stride)
      zero_buf[i] = 0;
    return;
  }
  const int32_t c = blockIdx.x * kDecodeColsPerBlock + tid * 8;
  uint4 v[kSmallMaxRows];
  uint32_t m2[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < kSmallMaxRows; ++i)
    if (i < s && c < h) v[i] = __ldg(reinterpret_cast<const uint4 *>(X + (int64_t)i * h + c));
#pragma unroll
  for (int i = 0; i < kSmallMaxRows; ++i) {
    if (i < s && c < h) {
      m2[0] = __vmaxu2(m2[0], v[i].x & 0x7FFF7FFFu);
      m2[1] = __vmaxu2(m2[1], v[i].y & 0x7FFF7FFFu);
      m2[2] = __vmaxu2(m2[2], v[i].z & 0x7FFF7FFFu);
      m2[3] = __vmaxu2(m2[3], v[i].w & 0x7FFF7FFFu);
    }
  }
  uint32_t m8 = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    m8 |= ((m2[e] & 0xFFFFu) >= thresh_bits ? 1u : 0u) << (2 * e);
    m8 |= ((m2[e] >> 16) >= thresh_bits ? 1u : 0u) << (2 * e + 1);
  }
  if (c >= h) m8 = 0;
  uint32_t word = m8 << (8 * (lane & 3));
  word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
  word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
  if ((lane & 3) == 0 && c < h) mask[c >> 5] = word;
  // per-row maxima over this thread's regular columns, reduced over the block
#pragma unroll
  for (int i = 0; i < kSmallMaxRows; ++i) {
    if (i < s) {
      uint32_t m = (c < h) ? max_halves(regular_absmax2(0u, v[i], m8)) : 0u;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, d));
      if (lane == 0) red[warp][i] = m;
    }
  }
  __syncthreads();
  if (tid < s) {
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w < kDecodeThreads / 32; ++w) m = max(m, red[w][tid]);
    partial_max[(int64_t)blockIdx.x * kSmallMaxRows + tid] = m;
  }
}

__global__ void __launch_bounds__(kDecodeThreads)
    k_decode_rowpass(const uint16_t *__restrict__ X, int32_t s, int32_t h,
                     const uint32_t *__restrict__ mask, const uint32_t *__restrict__ partial_max,
                     int32_t col_blocks, int32_t *__restrict__ word_prefix,
                     int32_t *__restrict__ count, float *__restrict__ ax,
                     int8_t *__restrict__ Xq, uint16_t *__restrict__ XO) {
  __shared__ float row_a[kSmallMaxRows], row_r[kSmallMaxRows];
  __shared__ int32_t s_prefix[kDecodeColsPerBlock / 32];
  __shared__ int32_t red_before[kDecodeThreads / 32], red_total[kDecodeThreads / 32];
  grid_dependency_wait();
  grid_dependency_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t nwords = (h + 31) >> 5;
  const int32_t w_begin = blockIdx.x * (kDecodeColsPerBlock / 32);
  // row scales: maximum over every column block's partial maximum
  if (tid < s) {
    uint32_t m = 0;
    for (int32_t b = 0; b < col_blocks; ++b)
      m = max(m, __ldg(partial_max + (int64_t)b * kSmallMaxRows + tid));
    const float a = half_bits_to_float(m);
    row_a[tid] = a;
    row_r[tid] = a > 0.0f ? __frcp_rn(a) : 0.0f;
    if (blockIdx.x == 0) ax[tid] = a;
  }
  // outlier columns before this block, and in total
  int32_t before = 0, total = 0;
  for (int32_t w = tid; w < nwords; w += kDecodeThreads) {
    const int32_t pc = __popc(__ldg(mask + w));
    total += pc;
    if (w < w_begin) before += pc;
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    before += __shfl_xor_sync(0xFFFFFFFFu, before, d);
    total += __shfl_xor_sync(0xFFFFFFFFu, total, d);
  }
  if (lane == 0) {
    red_before[warp] = before;
    red_total[warp] = total;
  }
  __syncthreads();
  before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kDecodeThreads / 32; ++w) {
    before += red_before[w];
    total += red_total[w];
  }
  // prefix counts of this block's 32 mask words (one warp)
  if (warp == 0) {
    const int32_t w = w_begin + lane;
    const int32_t pc = (w < nwords) ? __popc(__ldg(mask + w)) : 0;
    int32_t incl = pc;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += y;
    }
    const int32_t pre = before + incl - pc;
    s_prefix[lane] = pre;
    if (w < nwords) word_prefix[w] = pre;
    if (w == nwords - 1) word_prefix[nwords] = pre + pc;
  }
  if (blockIdx.x == 0 && tid == 0) *count = total;
  __syncthreads();
  // codes and the fp16 outlier columns of this block's columns, all rows
  const int32_t c = blockIdx.x * kDecodeColsPerBlock + tid * 8;
  if (c >= h) return;
  const uint32_t mw = __ldg(mask + (c >> 5));
  uint4 v[kSmallMaxRows];
#pragma unroll
  for (int i = 0; i < kSmallMaxRows; ++i)
    if (i < s) v[i] = __ldg(reinterpret_cast<const uint4 *>(X + (int64_t)i * h + c));
  const int32_t *pre_local = s_prefix - w_begin;  // indexed by global word
#pragma unroll
  for (int i = 0; i < kSmallMaxRows; ++i)
    if (i < s)
      quantize_chunk(v[i], mw, c, row_a[i], row_r[i], i, total, pre_local, Xq + (int64_t)i * h,
                     XO);
}

// ------------------------------------------------------------------- K0
// Offline weight preparation. Column absmax as binary16 magnitude bits
// (atomicMax over row blocks), then codes written transposed ([o][h]) through
// a shared-memory tile, then the absmax bits widened to fp32 in place.
__global__ void k_zero_u32(uint32_t *__restrict__ p, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    p[i] = 0u;
}

__global__ void __launch_bounds__(256)
    k_weight_colmax(const uint16_t *__restrict__ W, int32_t h, int32_t o,
                    int32_t rows_per_block, uint32_t *__restrict__ aw_bits) {
  const int32_t c = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c >= o) return;
  const int32_t r0 = blockIdx.y * rows_per_block;
  const int32_t r1 = min(h, r0 + rows_per_block);
  uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int32_t r = r0; r < r1; ++r) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(W + (int64_t)r * o + c));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      m[2 * e] = max(m[2 * e], w[e] & 0x7FFFu);
      m[2 * e + 1] = max(m[2 * e + 1], (w[e] >> 16) & 0x7FFFu);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e)
    if (m[e]) atomicMax(aw_bits + c + e, m[e]);
}

constexpr int kWqTile = 64;

__global__ void __launch_bounds__(256)
    k_weight_codes(const uint16_t *__restrict__ W, int32_t h, int32_t o,
                   const uint32_t *__restrict__ aw_bits, int8_t *__restrict__ wq) {
  __shared__ int8_t tile[kWqTile][kWqTile + 4];
  const int32_t k0 = blockIdx.y * kWqTile;
  const int32_t j0 = blockIdx.x * kWqTile;
  // load + quantise: 64 rows (k) x 64 columns (j), 8 columns per thread-load
  for (int i = threadIdx.x; i < kWqTile * (kWqTile / 8); i += blockDim.x) {
    const int kk = i / (kWqTile / 8);
    const int jj = (i % (kWqTile / 8)) * 8;
    const int32_t k = k0 + kk, j = j0 + jj;
    int32_t q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (k < h && j < o) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(W + (int64_t)k * o + j));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        q[2 * e] = absmax_code(half_bits_to_float(w[e] & 0xFFFFu),
                               half_bits_to_float(__ldg(aw_bits + j + 2 * e)));
        q[2 * e + 1] = absmax_code(half_bits_to_float(w[e] >> 16),
                                   half_bits_to_float(__ldg(aw_bits + j + 2 * e + 1)));
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[jj + e][kk] = static_cast<int8_t>(q[e]);
  }
  __syncthreads();
  // store transposed: row j of wq gets 64 consecutive k codes
  for (int i = threadIdx.x; i < kWqTile * (kWqTile / 16); i += blockDim.x) {
    const int jj = i / (kWqTile / 16);
    const int kk = (i % (kWqTile / 16)) * 16;
    const int32_t j = j0 + jj, k = k0 + kk;
    if (j < o && k < h) {
      uint32_t wv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        wv[u] = pack4_i8(tile[jj][kk + 4 * u], tile[jj][kk + 4 * u + 1], tile[jj][kk + 4 * u + 2],
                         tile[jj][kk + 4 * u + 3]);
      *reinterpret_cast<uint4 *>(wq + (int64_t)j * h + k) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
  }
}

__global__ void k_widen_scales(uint32_t *__restrict__ aw, int32_t o) {
  const int32_t j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < o) {
    const float f = half_bits_to_float(aw[j]);
    aw[j] = __float_as_uint(f);
  }
}

}  // namespace llmint8

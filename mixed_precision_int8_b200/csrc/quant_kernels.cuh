// HBM-bound kernels around the int8 GEMM:
//   K0  offline weight preparation (column absmax + int8 codes, transposed)
//   K1  activation pass: outlier-column bitmask, compaction of the outlier
//       list, per-row absmax over regular columns and int8 row codes
//   K2  fp16 outlier rows of W recovered from the int8 weight
//
// Magnitude trick used throughout: for a non-NaN binary16 value, the bit
// pattern with the sign cleared orders exactly like |x|, so maxima and the
// threshold test |x| >= alpha run on 16-bit integers (the threshold is the
// smallest binary16 magnitude >= alpha, found once on the host).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

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

__device__ __forceinline__ float half_bits_to_float(uint32_t b) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
}

__device__ __forceinline__ uint32_t pack4_i8(int32_t a, int32_t b, int32_t c, int32_t d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

// ------------------------------------------------------------------ K1a
// Zero the outlier bitmask (and the outlier count) before a new call.
__global__ void k_reset_mask(uint32_t *__restrict__ mask, int32_t nwords,
                             int32_t *__restrict__ count) {
  const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  for (int32_t w = i; w < nwords; w += gridDim.x * blockDim.x) mask[w] = 0u;
  if (i == 0) *count = 0;
}

// Step 1 ("The Full LLM.int8() Algorithm"): a column is an outlier column
// when any row holds |x| >= alpha. Each thread owns 8 adjacent columns (one
// 16-byte load per row) over `rows_per_block` rows; four lanes fold their
// 8-bit masks into one 32-bit word that is OR-ed into the global bitmask.
constexpr int kColThreads = 256;
constexpr int kColsPerBlock = kColThreads * 8;

__global__ void __launch_bounds__(kColThreads)
    k_outlier_columns(const uint16_t *__restrict__ X, int64_t s, int32_t h,
                      uint32_t thresh_bits, int32_t rows_per_block,
                      uint32_t *__restrict__ mask) {
  const int32_t c = blockIdx.x * kColsPerBlock + threadIdx.x * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_block;
  const int64_t r1 = min(s, r0 + rows_per_block);
  uint32_t m8 = 0;
  if (c < h) {
    const uint16_t *p = X + r0 * h + c;
    int64_t r = r0;
    for (; r + 4 <= r1; r += 4) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldg(reinterpret_cast<const uint4 *>(p + u * (int64_t)h));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          m8 |= ((w[e] & 0x7FFFu) >= thresh_bits ? 1u : 0u) << (2 * e);
          m8 |= (((w[e] >> 16) & 0x7FFFu) >= thresh_bits ? 1u : 0u) << (2 * e + 1);
        }
      }
      p += 4 * (int64_t)h;
    }
    for (; r < r1; ++r) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        m8 |= ((w[e] & 0x7FFFu) >= thresh_bits ? 1u : 0u) << (2 * e);
        m8 |= (((w[e] >> 16) & 0x7FFFu) >= thresh_bits ? 1u : 0u) << (2 * e + 1);
      }
      p += h;
    }
  }
  const int lane = threadIdx.x & 31;
  uint32_t word = m8 << (8 * (lane & 3));
  word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
  word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
  if ((lane & 3) == 0 && word != 0u && c < h) atomicOr(mask + (c >> 5), word);
}

// Compaction of the bitmask into the ascending outlier list (one block of
// 1024 threads): word_prefix[w] = number of outlier columns before word w,
// idx[] = the outlier columns, *count = |O|, flags[j] (optional) = bit j.
constexpr int kCompactThreads = 1024;

__global__ void __launch_bounds__(kCompactThreads)
    k_compact_outliers(const uint32_t *__restrict__ mask, int32_t nwords, int32_t h,
                       int32_t *__restrict__ word_prefix, int32_t *__restrict__ idx,
                       int32_t *__restrict__ count, uint8_t *__restrict__ flags) {
  __shared__ int32_t warp_sums[32];
  const int tid = threadIdx.x;
  const int per = (nwords + kCompactThreads - 1) / kCompactThreads;
  const int w0 = tid * per;
  const int w1 = min(nwords, w0 + per);
  int32_t local = 0;
  for (int w = w0; w < w1; ++w) local += __popc(mask[w]);
  // block exclusive scan of `local`
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
    int32_t v = warp_sums[lane];
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
    const uint32_t m = mask[w];
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
  if (tid == kCompactThreads - 1) {
    word_prefix[nwords] = base;
    *count = base;
  }
}

// Step 4 (activation side) with the X half of Step 2: one warp per row.
//   ax[i]  = max over regular columns of |X[i][j]|            (exact)
//   Xq[i][j] = code(X[i][j], ax[i]) on regular columns, 0 on outlier ones
//   XO[i][t] = X[i][O_t]  (fp16, row stride |O|; optional)
constexpr int kRowThreads = 256;
constexpr int kRowsPerBlock = kRowThreads / 32;

__global__ void __launch_bounds__(kRowThreads)
    k_quantize_rows(const uint16_t *__restrict__ X, int64_t s, int32_t h,
                    const uint32_t *__restrict__ mask, const int32_t *__restrict__ word_prefix,
                    const int32_t *__restrict__ count, int8_t *__restrict__ Xq,
                    float *__restrict__ ax, uint16_t *__restrict__ XO) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + (threadIdx.x >> 5);
  if (row >= s) return;
  const uint16_t *xr = X + row * h;
  // pass 1: absmax over regular columns, on magnitude bits
  uint32_t mbits = 0;
  {
    int32_t c = lane * 8;
    for (; c + 256 * 3 < h; c += 256 * 4) {
      uint4 v[4];
      uint32_t mk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[u] = __ldg(reinterpret_cast<const uint4 *>(xr + c + u * 256));
        mk[u] = (__ldg(mask + ((c + u * 256) >> 5)) >> ((c + u * 256) & 31)) & 0xFFu;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t lo = w[e] & 0x7FFFu, hi = (w[e] >> 16) & 0x7FFFu;
          if (!((mk[u] >> (2 * e)) & 1u)) mbits = max(mbits, lo);
          if (!((mk[u] >> (2 * e + 1)) & 1u)) mbits = max(mbits, hi);
        }
      }
    }
    for (; c < h; c += 256) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + c));
      const uint32_t mk = (__ldg(mask + (c >> 5)) >> (c & 31)) & 0xFFu;
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = w[e] & 0x7FFFu, hi = (w[e] >> 16) & 0x7FFFu;
        if (!((mk >> (2 * e)) & 1u)) mbits = max(mbits, lo);
        if (!((mk >> (2 * e + 1)) & 1u)) mbits = max(mbits, hi);
      }
    }
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, d));
  const float a = half_bits_to_float(mbits);
  if (lane == 0) ax[row] = a;
  const int32_t n_out = (XO != nullptr) ? *count : 0;
  // pass 2: codes (the row is re-read from L1/L2)
  int8_t *qr = Xq + row * h;
  for (int32_t c = lane * 8; c < h; c += 256) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + c));
    const uint32_t mw = __ldg(mask + (c >> 5));
    const uint32_t mk = (mw >> (c & 31)) & 0xFFu;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    int32_t q[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = half_bits_to_float(w[e] & 0xFFFFu);
      const float x1 = half_bits_to_float(w[e] >> 16);
      q[2 * e] = ((mk >> (2 * e)) & 1u) ? 0 : absmax_code(x0, a);
      q[2 * e + 1] = ((mk >> (2 * e + 1)) & 1u) ? 0 : absmax_code(x1, a);
    }
    uint2 packed;
    packed.x = pack4_i8(q[0], q[1], q[2], q[3]);
    packed.y = pack4_i8(q[4], q[5], q[6], q[7]);
    *reinterpret_cast<uint2 *>(qr + c) = packed;
    if (mk != 0u && XO != nullptr) {
      const int32_t base = __ldg(word_prefix + (c >> 5));
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if ((mk >> e) & 1u) {
          const int bit = (c & 31) + e;
          const int32_t pos = base + __popc(mw & ((1u << bit) - 1u));
          const uint32_t hv = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
          XO[row * n_out + pos] = static_cast<uint16_t>(hv);
        }
      }
    }
  }
}

// ------------------------------------------------------------------- K2
// W half of Step 2: the fp16 rows of W for the outlier columns, recovered
// from the int8 weight: WO[t][j] = fp16(fp32(fp32(wq[j][O_t]) * aw[j]) / 127).
__global__ void __launch_bounds__(256)
    k_outlier_weights(const int8_t *__restrict__ wq, const float *__restrict__ aw,
                      int32_t h, int32_t o, const int32_t *__restrict__ idx,
                      const int32_t *__restrict__ count, uint16_t *__restrict__ WO) {
  const int32_t n = *count;
  const int32_t j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= o) return;
  const float a = aw[j];
  for (int32_t t = blockIdx.y; t < n; t += gridDim.y) {
    const int32_t k = __ldg(idx + t);
    const float prod = static_cast<float>(wq[static_cast<int64_t>(j) * h + k]) * a;
    const float v = __fdiv_rn(prod, 127.0f);
    WO[static_cast<int64_t>(t) * o + j] = __half_as_ushort(__float2half_rn(v));
  }
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

// The fp16 outlier tiles of Step 2 of "The Full LLM.int8() Algorithm": the
// outlier columns of X (XO) and the matching rows of W (WO), their layout in
// the workspace, and the builder of WO shared by the kernels that make it.
//
// The layout is decided by |O| alone, so every kernel of a call, and the
// read-back, agree on it without the host knowing |O|:
//   narrow, |O| <= kNarrowOutliers: XO [s][|O|] and WO [|O|][o] (a row of WO
//     per outlier column; the GEMM stages them in shared memory and sums
//     the products on CUDA cores);
//   wide, |O| > kNarrowOutliers: XO [s][ldk] and WO [o][ldk], both with the
//     outlier index contiguous (K-major) and zero from |O| up to the next
//     multiple of 64, so that the GEMM streams them through TMA into the
//     tensor cores as a second product (fp16 x fp16 -> fp32).
// ldk is the workspace's outlier capacity rounded up to a multiple of 64.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "ptx_sm100.cuh"

namespace llmint8 {

constexpr int kNarrowOutliers = 16;

__host__ __device__ __forceinline__ bool outliers_wide(int32_t n) { return n > kNarrowOutliers; }
__host__ __device__ __forceinline__ int32_t pad64(int32_t n) { return (n + 63) & ~63; }

// Whether the outlier columns fill at least half of the span they cover
// (as for a low threshold, up to every column): the builders then move
// aligned stretches of consecutive columns as 16-byte pieces. The choice
// changes only the schedule, never a value.
__device__ __forceinline__ bool outliers_dense(int32_t n, const int32_t *idx) {
  if (n <= 0) return false;
  const int32_t lo = __ldcg(idx), hi = __ldcg(idx + n - 1);
  return hi - lo + 1 <= 2 * n;
}

// Element (row, t) of XO and (t, j) of WO.
__device__ __forceinline__ int64_t xo_index(int64_t row, int32_t t, int32_t n, int32_t ldk) {
  return row * (outliers_wide(n) ? ldk : n) + t;
}
__device__ __forceinline__ int64_t wo_index(int32_t t, int64_t j, int32_t n, int32_t o,
                                            int32_t ldk) {
  return outliers_wide(n) ? j * ldk + t : static_cast<int64_t>(t) * o + j;
}

// fp16(fp32(fp32(code) * scale) / 127) for the four signed byte codes of w.
__device__ __forceinline__ uint2 dequant4(uint32_t w, float scale) {
  uint16_t r[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int32_t code = static_cast<int32_t>(static_cast<int8_t>((w >> (8 * e)) & 0xFFu));
    r[e] = __half_as_ushort(
        __float2half_rn(__fdiv_rn(static_cast<float>(code) * scale, 127.0f)));
  }
  return make_uint2(static_cast<uint32_t>(r[0]) | (static_cast<uint32_t>(r[1]) << 16),
                    static_cast<uint32_t>(r[2]) | (static_cast<uint32_t>(r[3]) << 16));
}

// The wide layout from the int8 codes (the value rule of build_wo_rows).
// Work items are (j, g): 16 consecutive outlier positions t = 16g .. 16g+15
// of row j, g fastest, so a warp reads one stretch of row j of wq and
// writes 32 consecutive 32-byte pieces of row j of WO. Where those 16
// positions are 16 consecutive, 16-aligned columns of X (every outlier
// column in a dense stretch, as for a zero threshold) the codes come in
// one 16-byte load; otherwise in 16 byte gathers. Positions from |O| up to
// pad64(|O|) are written as zeros. Four items in flight per thread.
__device__ __forceinline__ void build_wo_wide_codes(int32_t n, const int32_t *__restrict__ idx,
                                                    const int8_t *__restrict__ wq,
                                                    const float *__restrict__ aw, int32_t h,
                                                    int32_t o, int32_t ldk,
                                                    uint16_t *__restrict__ WO, int64_t first,
                                                    int64_t stride) {
  constexpr int UI = 4;
  const int64_t G = pad64(n) >> 4;
  const int64_t items = static_cast<int64_t>(o) * G;
  // (j, g) of item `first`, and the step of `stride` items in those terms
  int64_t j = first / G, g = first - (first / G) * G;
  const int64_t dj = stride / G, dg = stride - (stride / G) * G;
  for (int64_t q0 = first; q0 < items; q0 += UI * stride) {
    uint4 code[UI];
    float scale[UI];
    int64_t jj[UI], tt[UI];
#pragma unroll
    for (int u = 0; u < UI; ++u) {
      jj[u] = j;
      tt[u] = g << 4;
      code[u] = make_uint4(0u, 0u, 0u, 0u);
      scale[u] = 0.0f;
      if (q0 + u * stride < items && tt[u] < n) {
        const int32_t t0 = static_cast<int32_t>(tt[u]);
        const int8_t *row = wq + j * h;
        scale[u] = __ldg(aw + j);
        const int4 *ip = reinterpret_cast<const int4 *>(idx + t0);
        const int4 i0 = __ldcg(ip), i3 = __ldcg(ip + 3);
        if (t0 + 15 < n && i3.w - i0.x == 15 && (i0.x & 15) == 0) {
          code[u] = __ldg(reinterpret_cast<const uint4 *>(row + i0.x));
        } else {
          const int4 i1 = __ldcg(ip + 1), i2 = __ldcg(ip + 2);
          const int32_t c[16] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w,
                                 i2.x, i2.y, i2.z, i2.w, i3.x, i3.y, i3.z, i3.w};
          uint32_t b[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (t0 + e < n)
              b[e >> 2] |= static_cast<uint32_t>(static_cast<uint8_t>(__ldg(row + c[e])))
                           << (8 * (e & 3));
          code[u] = make_uint4(b[0], b[1], b[2], b[3]);
        }
      }
      g += dg;
      j += dj;
      if (g >= G) {
        g -= G;
        ++j;
      }
    }
#pragma unroll
    for (int u = 0; u < UI; ++u) {
      if (q0 + u * stride >= items) break;
      // codes past |O| are zero, and so are their values
      const uint2 v0 = dequant4(code[u].x, scale[u]), v1 = dequant4(code[u].y, scale[u]);
      const uint2 v2 = dequant4(code[u].z, scale[u]), v3 = dequant4(code[u].w, scale[u]);
      uint4 *dst = reinterpret_cast<uint4 *>(WO + jj[u] * ldk + tt[u]);
      dst[0] = make_uint4(v0.x, v0.y, v1.x, v1.y);
      dst[1] = make_uint4(v2.x, v2.y, v3.x, v3.y);
    }
  }
}

// Step 2, W side, for every outlier column: WO[t][j] = fp16(fp32(fp32(
// wq[j][O_t]) * aw[j]) / 127), or W[O_t][j] itself when the caller's fp16
// weight w16 is given, in the layout above (wide: also the zero padding).
// Work items q from `first` in steps of `stride`, eight independent gathers
// in flight per thread; narrow: q = t*o + j (j fastest, stores coalesce),
// wide: q = j*pad64(n) + t (t fastest, stores coalesce). Out of line: it
// runs once per thread and block, and inlined it would be compiled into the
// GEMM epilogue's hot loop.
__device__ __noinline__ void build_wo_rows(int32_t n, const int32_t *__restrict__ idx,
                                              const int8_t *__restrict__ wq,
                                              const float *__restrict__ aw,
                                              const uint16_t *__restrict__ w16, int32_t h,
                                              int32_t o, int32_t ldk,
                                              uint16_t *__restrict__ WO, int64_t first,
                                              int64_t stride) {
  constexpr int U = 8;
  const bool wide = outliers_wide(n);
  if (!wide) {
    // narrow: q = t*o + j, at most 16 rows of o, one division per item
    const int64_t pairs = static_cast<int64_t>(n) * o;
    for (int64_t q0 = first; q0 < pairs; q0 += U * stride) {
      int32_t code[U];
      float scale[U];
      uint16_t w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t q = q0 + u * stride;
        code[u] = 0;
        scale[u] = 0.0f;
        w[u] = 0;
        if (q < pairs) {
          const int32_t t = static_cast<int32_t>(q / o);
          const int32_t j = static_cast<int32_t>(q - static_cast<int64_t>(t) * o);
          const int32_t c = __ldcg(idx + t);
          if (w16 != nullptr) {
            w[u] = __ldg(w16 + static_cast<int64_t>(c) * o + j);
          } else {
            code[u] = __ldg(wq + static_cast<int64_t>(j) * h + c);
            scale[u] = __ldg(aw + j);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t q = q0 + u * stride;
        if (q < pairs)
          WO[q] = w16 != nullptr
                      ? w[u]
                      : __half_as_ushort(__float2half_rn(
                            __fdiv_rn(static_cast<float>(code[u]) * scale[u], 127.0f)));
      }
    }
    return;
  }
  const int32_t T = pad64(n);
  if (w16 == nullptr && outliers_dense(n, idx)) {
    build_wo_wide_codes(n, idx, wq, aw, h, o, ldk, WO, first, stride);
    // the wide tiles are read by TMA (the async proxy)
    fence_proxy_async_global();
    return;
  }
  // wide, scattered outlier columns (or from the fp16 weight): the items
  // are (t, j) with t < pad64(n) and j < o, stored at WO[j*ldk + t]. Each
  // thread keeps one t (its index loaded once) and walks j; a warp covers
  // 32 consecutive t of one row j, so the stores coalesce. With fewer
  // threads than t values (a CTA building every row alone) each thread
  // takes several t in turn.
  constexpr int UW = 8;  // gathers in flight per thread
  auto column = [&](int32_t t, int64_t jbeg, int64_t jstep) {
    const bool tl = t < n;
    const int32_t c = tl ? __ldcg(idx + t) : 0;
    for (int64_t j0 = jbeg; j0 < o; j0 += UW * jstep) {
      int32_t code[UW];
      float scale[UW];
      uint16_t w[UW];
#pragma unroll
      for (int u = 0; u < UW; ++u) {
        const int64_t j = j0 + u * jstep;
        code[u] = 0;
        scale[u] = 0.0f;
        w[u] = 0;
        if (tl && j < o) {
          if (w16 != nullptr) {
            w[u] = __ldg(w16 + static_cast<int64_t>(c) * o + j);
          } else {
            code[u] = __ldg(wq + j * h + c);
            scale[u] = __ldg(aw + j);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < UW; ++u) {
        const int64_t j = j0 + u * jstep;
        if (j < o)
          WO[j * ldk + t] = !tl ? static_cast<uint16_t>(0)
                            : w16 != nullptr
                                ? w[u]
                                : __half_as_ushort(__float2half_rn(
                                      __fdiv_rn(static_cast<float>(code[u]) * scale[u], 127.0f)));
      }
    }
  };
  if (stride >= T) {
    // thread `first` takes t = first % T and every jstep-th column j from
    // first / T: each (t, j) exactly once over the first jstep*T threads
    const int64_t jstep = stride / T;
    if (first < jstep * T) column(static_cast<int32_t>(first % T), first / T, jstep);
  } else {
    for (int64_t t = first; t < T; t += stride) column(static_cast<int32_t>(t), 0, 1);
  }
  fence_proxy_async_global();
}

}  // namespace llmint8

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

namespace llmint8 {

constexpr int kNarrowOutliers = 16;

__host__ __device__ __forceinline__ bool outliers_wide(int32_t n) { return n > kNarrowOutliers; }
__host__ __device__ __forceinline__ int32_t pad64(int32_t n) { return (n + 63) & ~63; }

// Element (row, t) of XO and (t, j) of WO.
__device__ __forceinline__ int64_t xo_index(int64_t row, int32_t t, int32_t n, int32_t ldk) {
  return row * (outliers_wide(n) ? ldk : n) + t;
}
__device__ __forceinline__ int64_t wo_index(int32_t t, int64_t j, int32_t n, int32_t o,
                                            int32_t ldk) {
  return outliers_wide(n) ? j * ldk + t : static_cast<int64_t>(t) * o + j;
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
  // wide: the items are (t, j) with t < pad64(n) and j < o, stored at
  // WO[j*ldk + t]. Each thread keeps one t (its index loaded once) and walks
  // j; a warp covers 32 consecutive t of one row j, so the gathers from wq
  // and the stores coalesce. With fewer threads than t values (a CTA
  // building every row alone) each thread takes several t in turn.
  const int32_t T = pad64(n);
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
}

}  // namespace llmint8

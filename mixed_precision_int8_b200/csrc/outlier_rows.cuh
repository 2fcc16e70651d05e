// The fp16 outlier rows of W (Step 2 of "The Full LLM.int8() Algorithm",
// W side), shared by the kernels that build them: the int8 GEMM's epilogue
// (while its first tiles' mainloops run) and, where the GEMM cannot be
// launched so that all its CTAs are resident together, blocks of the
// activation fix-up.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace llmint8 {

// Step 2, W side, for every outlier column: WO[t][j] = fp16(fp32(fp32(
// wq[j][O_t]) * aw[j]) / 127), or W[O_t][j] itself when the caller's fp16
// weight w16 is given. Pairs (t, j) (j fastest, so the stores coalesce) from
// `first` in steps of `stride`, eight independent gathers in flight per
// thread.
__device__ __forceinline__ void build_wo_rows(int32_t n, const int32_t *__restrict__ idx,
                                              const int8_t *__restrict__ wq,
                                              const float *__restrict__ aw,
                                              const uint16_t *__restrict__ w16, int32_t h,
                                              int32_t o, uint16_t *__restrict__ WO,
                                              int64_t first, int64_t stride) {
  constexpr int U = 8;
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
        WO[q] = w16 != nullptr ? w[u]
                               : __half_as_ushort(__float2half_rn(
                                     __fdiv_rn(static_cast<float>(code[u]) * scale[u], 127.0f)));
    }
  }
}

}  // namespace llmint8

// K4: decode-regime LLM.int8() GEMM (s <= 16 rows of X), bound by the read of
// the int8 weight from HBM.
//
// The int8 product is computed transposed on the tensor cores: the weight
// tile (128 output columns x 128 reduction bytes) is the MMA's A operand
// (M = 128) and the <= 16 quantised rows of X are its B operand (N = 16,
// zero-filled by TMA beyond s). The (weight tile, k-block) units are split
// evenly over one persistent CTA per SM, so every SM streams the same share
// of the weight whatever the wave count. Each CTA adds its partial int32
// accumulators into a [16][o] int32 buffer with integer atomics (exact and
// order-independent; the buffer is zeroed by the call's first kernel), and a
// small finishing kernel applies the
// dequantisation, the fp16 outlier product and the fp16 store:
//   out[i][j] = fp16( Ci[i][j] * (ax[i] / 16129) * aw[j] + sum_t XO[i][t] WO[t][j] )
// ("The Full LLM.int8() Algorithm", Steps 3-5).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "ptx_sm100.cuh"

namespace llmint8 {
namespace decode {

constexpr int MAX_ROWS = 16;
constexpr int BM = 128;  // weight rows (output columns) per tile: MMA M
constexpr int BN = 16;   // X rows, zero-padded: MMA N
constexpr int BK = 128;  // reduction bytes per stage
constexpr int STAGES = 10;
constexpr int UMMA_K = 32;
constexpr uint32_t A_STAGE_BYTES = BM * BK;  // 16 KB
constexpr uint32_t B_STAGE_BYTES = BN * BK;  // 2 KB
constexpr int NUM_ACC = 2;
constexpr uint32_t TMEM_COLS = 32;
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_THREADS = 128;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * (A_STAGE_BYTES + B_STAGE_BYTES) + 256;

struct Params {
  int32_t s, h, o;
  int32_t num_m_blocks, num_k_blocks;
  int64_t units_total;
  const float *ax;
  const float *aw;
  const uint16_t *XO;
  const uint16_t *WO;
  const int32_t *n_out;
  uint16_t *out;
  int32_t *ci;    // optional exact accumulators [s][o]
  int32_t *cacc;  // [MAX_ROWS][o] int32 partial-sum buffer
  int32_t *status;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// Units [u0, u1) of this CTA: unit u is k-block (u % nk) of weight tile
// (u / nk). Consecutive units of one tile form a segment, accumulated in one
// TMEM buffer and then flushed by the epilogue.
__device__ __forceinline__ void cta_units(const Params &p, int64_t &u0, int64_t &u1) {
  u0 = (p.units_total * blockIdx.x) / gridDim.x;
  u1 = (p.units_total * (blockIdx.x + 1)) / gridDim.x;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_decode_i8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t *base = smem_raw + pad;
  const uint32_t sA = smem_u32(base);
  const uint32_t sB = sA + STAGES * A_STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + STAGES * (A_STAGE_BYTES + B_STAGE_BYTES));
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (STAGES + st); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + NUM_ACC + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2 * NUM_ACC);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 2 * NUM_ACC + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), NUM_EPI_THREADS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  grid_dependency_wait();

  int64_t u0, u1;
  cta_units(p, u0, u1);
  const int64_t nk = p.num_k_blocks;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    const uint64_t pol_w = l2_policy_evict_first();  // weight is read once
    uint32_t stage = 0, phase = 0, issued = 0, last_par = 0;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      const int32_t m_blk = (int32_t)(u / nk);
      const int32_t kb = (int32_t)(u - (int64_t)m_blk * nk);
      if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status,
                             LLMINT8_DEV_TIMEOUT_PRODUCER, p.timeout_ns)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(full_bar(stage), A_STAGE_BYTES + B_STAGE_BYTES);
      tma_load_2d_hint(sA + stage * A_STAGE_BYTES, &tmA, full_bar(stage), kb * BK, m_blk * BM,
                       pol_w);
      tma_load_2d(sB + stage * B_STAGE_BYTES, &tmB, full_bar(stage), kb * BK, 0);
      issued |= 1u << stage;
      last_par = (last_par & ~(1u << stage)) | (phase << stage);
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) {
      volatile int never = 0;
      for (int st = 0; st < STAGES; ++st)
        if ((issued >> st) & 1u)
          mbar_wait_bounded(full_bar(st), (last_par >> st) & 1u, &never, p.status,
                            LLMINT8_DEV_TIMEOUT_DRAIN, p.timeout_ns);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_i8_s32(BM, BN);
    uint32_t stage = 0, phase = 0;
    bool ok = true, any = false;
    int32_t it = 0;
    for (int64_t u = u0; u < u1 && ok; ++it) {
      const int64_t m_blk = u / nk;
      const int64_t seg_end = min(u1, (m_blk + 1) * nk);
      const uint32_t acc = it & 1, acc_par = (it >> 1) & 1;
      if (!mbar_wait_bounded(tempty_bar(acc), acc_par ^ 1u, abort_flag, p.status,
                             LLMINT8_DEV_TIMEOUT_MMA, p.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int64_t v = u; v < seg_end; ++v) {
        if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status,
                               LLMINT8_DEV_TIMEOUT_MMA, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a_desc = smem_desc_kmajor_sw128(sA + stage * A_STAGE_BYTES);
        const uint64_t b_desc = smem_desc_kmajor_sw128(sB + stage * B_STAGE_BYTES);
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k)
          mma_i8(d_tmem, a_desc + (uint64_t)((k * UMMA_K) >> 4),
                 b_desc + (uint64_t)((k * UMMA_K) >> 4), idesc, (v > u || k > 0) ? 1u : 0u);
        any = true;
        mma_commit(empty_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit(tfull_bar(acc));
      u = seg_end;
    }
    if (!ok && any) {
      volatile int never = 0;
      mma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, &never, p.status, LLMINT8_DEV_TIMEOUT_DRAIN, p.timeout_ns);
    }
  } else if (warp >= EPI_WARP0) {
    // ---------------------------------------------------------- epilogue
    const int ew = warp - EPI_WARP0;
    int32_t it = 0;
    for (int64_t u = u0; u < u1; ++it) {
      const int64_t m_blk = u / nk;
      const int64_t seg_end = min(u1, (m_blk + 1) * nk);
      const uint32_t acc = it & 1, acc_par = (it >> 1) & 1;
      if (!mbar_wait_bounded(tfull_bar(acc), acc_par, abort_flag, p.status,
                             LLMINT8_DEV_TIMEOUT_EPILOGUE, p.timeout_ns))
        break;
      tc_fence_after();
      uint32_t v[16];
      __syncwarp();
      tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(ew * 32) << 16) + acc * BN, v);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      const int64_t j = m_blk * BM + ew * 32 + lane;
      if (j < p.o) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (i < p.s && v[i] != 0u) atomicAdd(p.cacc + (int64_t)i * p.o + j, (int32_t)v[i]);
      }
      u = seg_end;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, TMEM_COLS);
}

// Dequantisation, outlier product and fp16 store for the s <= 16 rows.
__global__ void __launch_bounds__(256) k_decode_finish(const Params p) {
  grid_dependency_wait();
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= (int64_t)p.s * p.o) return;
  const int32_t i = (int32_t)(g / p.o);
  const int32_t j = (int32_t)(g - (int64_t)i * p.o);
  const int32_t n_out = *p.n_out;
  const int32_t c = p.cacc[(int64_t)i * p.o + j];
  float acc = (float)c * (p.ax[i] * (1.0f / 16129.0f)) * p.aw[j];
  const uint16_t *xo = p.XO + (int64_t)i * n_out;
  for (int32_t t = 0; t < n_out; ++t)
    acc = fmaf(__half2float(__ushort_as_half(xo[t])),
               __half2float(__ushort_as_half(p.WO[(int64_t)t * p.o + j])), acc);
  p.out[g] = __half_as_ushort(__float2half_rn(acc));
  if (p.ci) p.ci[g] = c;
}

}  // namespace decode
}  // namespace llmint8

// K3p: the int8 GEMM of LLM.int8() (K3, gemm_sm100.cuh) with 256 x 256
// output tiles computed by a pair of CTAs through tcgen05 cta_group::2.
//
// Math: as K3 ("The Full LLM.int8() Algorithm", Steps 3-5).
//
// What the pair changes (a cluster of two CTAs, rank r = 0, 1):
//   - rank r keeps rows 128r .. 128r+127 of the tile's 256 rows of Xq and
//     columns 128r .. 128r+127 of its 256 columns of Wq in its shared
//     memory; one MMA issued by rank 0 (M=256, N=256, K=32) reads both
//     halves of both operands and writes each CTA's 128 rows of the
//     accumulator into that CTA's TMEM, so the epilogue is K3's, per CTA;
//   - a stage is 32 KB per CTA (16 KB of A, 16 KB of B) instead of K3's
//     48 KB for the same 128 rows x 256 columns of work per CTA: a third
//     less traffic from L2 per output, and the same shared memory holds a
//     6-stage ring, a longer lead for copies whose data arrive late (the
//     losses of K3 at the large shapes);
//   - both CTAs' copies complete on rank 0's "full" barriers, which expect
//     the bytes of both; rank 0's commits arrive on both CTAs' "empty" and
//     "accumulator full" barriers; the epilogue threads of both CTAs arrive
//     on rank 0's "accumulator empty" barriers.
// The fp16 outlier rows of W (shares and bounded wait), the tensor-core
// outlier mode (a 128 x 64 XO box and this CTA's 128 x 64 half of the W^O
// box per fp16 stage), the epilogue arithmetic and the bounded waits are
// K3's.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "gemm_sm100.cuh"

namespace llmint8 {
namespace gemm2 {

using gemm::BK;
using gemm::BM;
using gemm::BN;
using gemm::EPI_BARRIER;
using gemm::EPI_WARP0;
using gemm::f2h2;
using gemm::FAST_OUTLIERS;
using gemm::NUM_ACC;
using gemm::NUM_EPI_THREADS;
using gemm::NUM_THREADS;
using gemm::OK;
using gemm::OUT_STAGE_BYTES;
using gemm::Params;
using gemm::REGS_HIGH;
using gemm::REGS_LOW;
using gemm::TMEM_COLS;
using gemm::UMMA_K;
using gemm::UMMA_K16;

constexpr int STAGES = 6;
constexpr int BNH = BN / 2;                   // tile columns whose Wq rows this CTA holds
constexpr uint32_t A_STAGE_BYTES = BM * BK;   // this CTA's 128 rows of Xq
constexpr uint32_t B_STAGE_BYTES = BNH * BK;  // this CTA's 128 columns of Wq
constexpr uint32_t PAIR_TX = 2 * (A_STAGE_BYTES + B_STAGE_BYTES);  // on rank 0's barrier
constexpr uint32_t RING_BYTES = STAGES * (A_STAGE_BYTES + B_STAGE_BYTES);
constexpr uint32_t OUT_OFF = RING_BYTES;
constexpr uint32_t WO_OFF = OUT_OFF + 8 * OUT_STAGE_BYTES;  // fp32 [FAST_OUTLIERS][BN]
constexpr uint32_t AW_OFF = WO_OFF + FAST_OUTLIERS * BN * 4;
constexpr uint32_t BAR_OFF = AW_OFF + BN * 4;
constexpr size_t SMEM_BYTES = 1024 + BAR_OFF + 256;
constexpr uint32_t TEMPTY_ARRIVALS = 2 * NUM_EPI_THREADS;  // both CTAs' epilogues

static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
static_assert(OUT_OFF % 1024 == 0, "swizzled staging must be 1024-byte aligned");
static_assert(BAR_OFF % 8 == 0, "mbarrier alignment");
static_assert((2 * STAGES + 2 * NUM_ACC + 2) * 8 + 8 <= 256, "barrier block size");
static_assert(BM * OK * 2 == A_STAGE_BYTES && BNH * OK * 2 == B_STAGE_BYTES,
              "fp16 outlier stages fill the int8 stage slots exactly");

// Producer of the tensor-core outlier mode (see gemm::tc_producer): per pair
// tile the int8 stages, then the fp16 outlier stages. False if a wait ran
// out.
__device__ __noinline__ bool tc_producer_pair(const Params &p, const CUtensorMap *tmA,
                                         const CUtensorMap *tmB, const CUtensorMap *tmXO,
                                         const CUtensorMap *tmWO, uint32_t sA, uint32_t sB,
                                         uint32_t bar0, uint32_t wo_bar,
                                         volatile int *abort_flag, int32_t nk_o, uint32_t rank,
                                         uint32_t &stage, uint32_t &phase, uint32_t &issued,
                                         uint32_t &last_par) {
  const int32_t num_m2 = (p.num_m_blocks + 1) / 2;
  const int32_t num_tiles = num_m2 * p.num_n_blocks;
  bool wo_ok = !p.build_wo;
  for (int32_t tile = blockIdx.x >> 1; tile < num_tiles; tile += gridDim.x >> 1) {
    const int32_t m_blk = 2 * (tile % num_m2) + (int32_t)rank;
    const int32_t b_row = (tile / num_m2) * BN + (int32_t)rank * BNH;
    for (int32_t kb = 0; kb < p.num_k_blocks + nk_o; ++kb) {
      const bool o_stage = kb >= p.num_k_blocks;
      if (o_stage && !wo_ok) {
        if (!mbar_wait_bounded(wo_bar, 0, abort_flag, p.status, LLMINT8_DEV_TIMEOUT_PRODUCER,
                               p.timeout_ns))
          return false;
        fence_proxy_async_global();
        wo_ok = true;
      }
      const uint32_t full = bar0 + 8u * stage, empty = bar0 + 8u * (STAGES + stage);
      if (!mbar_wait_bounded(empty, phase ^ 1u, abort_flag, p.status, LLMINT8_DEV_TIMEOUT_PRODUCER,
                             p.timeout_ns))
        return false;
      if (rank == 0) mbar_arrive_expect_tx(full, PAIR_TX);
      const uint32_t full0 = mapa_shared(full, 0);
      if (!o_stage) {
        tma_load_2d_pair(sA + stage * A_STAGE_BYTES, tmA, full0, kb * BK, m_blk * BM);
        tma_load_2d_pair(sB + stage * B_STAGE_BYTES, tmB, full0, kb * BK, b_row);
      } else {
        const int32_t ko = (kb - p.num_k_blocks) * OK;
        tma_load_2d_pair(sA + stage * A_STAGE_BYTES, tmXO, full0, ko, m_blk * BM);
        tma_load_2d_pair(sB + stage * B_STAGE_BYTES, tmWO, full0, ko, b_row);
      }
      issued |= 1u << stage;
      last_par = (last_par & ~(1u << stage)) | (phase << stage);
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  return true;
}

// MMA issuer of the tensor-core outlier mode (rank 0): one int32 and one
// fp32 accumulator per pair tile, as gemm::tc_mma. False if a wait ran out.
__device__ __noinline__ bool tc_mma_pair(const Params &p, uint32_t sA, uint32_t sB, uint32_t bar0,
                                    uint32_t tmem_base, volatile int *abort_flag, int32_t nk_o,
                                    uint32_t &stage, uint32_t &phase, bool &any) {
  constexpr uint32_t idesc = idesc_i8_s32(2 * BM, BN);
  constexpr uint32_t idesc16 = idesc_f16_f32(2 * BM, BN);
  const int32_t num_m2 = (p.num_m_blocks + 1) / 2;
  const int32_t num_tiles = num_m2 * p.num_n_blocks;
  const uint32_t tfull = bar0 + 8u * (2 * STAGES), tempty = bar0 + 8u * (2 * STAGES + NUM_ACC);
  int32_t it = 0;
  for (int32_t tile = blockIdx.x >> 1; tile < num_tiles; tile += gridDim.x >> 1, ++it) {
    if (!mbar_wait_bounded(tempty, (uint32_t)(it & 1) ^ 1u, abort_flag, p.status,
                           LLMINT8_DEV_TIMEOUT_MMA, p.timeout_ns))
      return false;
    tc_fence_after();
    for (int32_t kb = 0; kb < p.num_k_blocks + nk_o; ++kb) {
      const uint32_t full = bar0 + 8u * stage, empty = bar0 + 8u * (STAGES + stage);
      if (!mbar_wait_bounded(full, phase, abort_flag, p.status, LLMINT8_DEV_TIMEOUT_MMA,
                             p.timeout_ns))
        return false;
      tc_fence_after();
      const uint64_t a_desc = smem_desc_kmajor_sw128(sA + stage * A_STAGE_BYTES);
      const uint64_t b_desc = smem_desc_kmajor_sw128(sB + stage * B_STAGE_BYTES);
      if (kb < p.num_k_blocks) {
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k)
          mma_i8_pair(tmem_base, a_desc + (uint64_t)((k * UMMA_K) >> 4),
                      b_desc + (uint64_t)((k * UMMA_K) >> 4), idesc, (kb > 0 || k > 0) ? 1u : 0u);
      } else {
        const int32_t ko = kb - p.num_k_blocks;
#pragma unroll
        for (int k = 0; k < OK / UMMA_K16; ++k)
          mma_f16_pair(tmem_base + BN, a_desc + (uint64_t)((k * UMMA_K16 * 2) >> 4),
                       b_desc + (uint64_t)((k * UMMA_K16 * 2) >> 4), idesc16,
                       (ko > 0 || k > 0) ? 1u : 0u);
      }
      any = true;
      mma_commit_pair(mapa_shared(empty, 0));
      mma_commit_pair(mapa_shared(empty, 1));
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    mma_commit_pair(mapa_shared(tfull, 0));
    mma_commit_pair(mapa_shared(tfull, 1));
  }
  return true;
}

// One pair tile's epilogue in tensor-core outlier mode (see
// gemm::tc_tile_epilogue); the accumulator is handed back on rank 0's
// barrier (tempty0, a shared::cluster address). False if a wait ran out.
__device__ __noinline__ bool tc_tile_epilogue_pair(const Params &p, const CUtensorMap *tmOut,
                                              uint32_t tmem_base, uint32_t tfull,
                                              uint32_t tempty0, uint32_t parity,
                                              volatile int *abort_flag, int32_t m_blk,
                                              int32_t n0, int ew, int hc, int lane,
                                              const float *sAW, uint8_t *sOut,
                                              uint32_t sOut_addr, int32_t row, bool row_ok,
                                              float rs) {
  const bool ready = mbar_wait_bounded(tfull, parity, abort_flag, p.status,
                                       LLMINT8_DEV_TIMEOUT_EPILOGUE, p.timeout_ns);
  if (named_barrier_or(EPI_BARRIER, NUM_EPI_THREADS, !ready)) return false;
  tc_fence_after();
  const uint32_t t_row = tmem_base + ((uint32_t)(ew * 32) << 16) + hc * (BN / 2);
  const uint64_t rs2 = f32x2_pack(rs, rs);
  for (int c = 0; c < BN / 64; ++c) {
    uint32_t v[32], fv[32];
    __syncwarp();
    tmem_ld_32x32b_x32(t_row + c * 32, v);
    tmem_ld_32x32b_x32(t_row + BN + c * 32, fv);
    if (lane == 0) bulk_wait_group_read0();
    tmem_ld_wait();
    __syncwarp();
    if (c == BN / 64 - 1) {
      tc_fence_before();
      mbar_arrive_cluster(tempty0);
    }
    const int32_t j0 = n0 + hc * (BN / 2) + c * 32;
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8) {
      uint32_t h8[4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int q4 = 2 * q8 + u;
        const float4 a4 = *reinterpret_cast<const float4 *>(sAW + hc * (BN / 2) + c * 32 + 4 * q4);
        const uint64_t sv0 = f32x2_mul(rs2, f32x2_pack(a4.x, a4.y));
        const uint64_t sv1 = f32x2_mul(rs2, f32x2_pack(a4.z, a4.w));
        const uint64_t c0 = f32x2_pack((float)(int32_t)v[4 * q4], (float)(int32_t)v[4 * q4 + 1]);
        const uint64_t c1 =
            f32x2_pack((float)(int32_t)v[4 * q4 + 2], (float)(int32_t)v[4 * q4 + 3]);
        const uint64_t e0 = (static_cast<uint64_t>(fv[4 * q4 + 1]) << 32) | fv[4 * q4];
        const uint64_t e1 = (static_cast<uint64_t>(fv[4 * q4 + 3]) << 32) | fv[4 * q4 + 2];
        const uint64_t r0 = f32x2_fma(c0, sv0, e0);
        const uint64_t r1 = f32x2_fma(c1, sv1, e1);
        h8[2 * u] = f2h2(f32x2_lo(r0), f32x2_hi(r0));
        h8[2 * u + 1] = f2h2(f32x2_lo(r1), f32x2_hi(r1));
      }
      *reinterpret_cast<uint4 *>(sOut + lane * 64 + ((q8 ^ ((lane >> 1) & 3)) * 16)) =
          make_uint4(h8[0], h8[1], h8[2], h8[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    const int32_t bx = j0, by = m_blk * BM + ew * 32;
    if (lane == 0 && bx < p.o && by < p.s) {
      tma_store_2d(tmOut, sOut_addr, bx, by);
      bulk_commit_group();
    }
    if (p.ci != nullptr && row_ok && j0 < p.o) {
      const bool full = (j0 + 32 <= p.o);
      int4 *cp = reinterpret_cast<int4 *>(p.ci + (int64_t)row * p.o + j0);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        if (!full && q4 >= 4) break;
        cp[q4] = make_int4((int)v[4 * q4], (int)v[4 * q4 + 1], (int)v[4 * q4 + 2],
                           (int)v[4 * q4 + 3]);
      }
    }
  }
  return true;
}

// Grid: 2 x (pairs), launched with cluster dimension 2; tmB and tmWO have
// 128-row boxes (this CTA's half of a tile's columns).
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_i8_pair(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut,
                   const __grid_constant__ CUtensorMap tmXO,
                   const __grid_constant__ CUtensorMap tmWO, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t *base = smem_raw + pad;
  const uint32_t sA = smem_u32(base);
  const uint32_t sB = sA + STAGES * A_STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + BAR_OFF);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (STAGES + st); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + NUM_ACC + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2 * NUM_ACC);
  const uint32_t wo_bar = bar0 + 8u * (2 * STAGES + 2 * NUM_ACC + 1);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 2 * NUM_ACC + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), TEMPTY_ARRIVALS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(wo_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised before either signals the other's
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  grid_dependency_wait();

  const int32_t num_m2 = (p.num_m_blocks + 1) / 2;
  const int32_t num_tiles = num_m2 * p.num_n_blocks;
  const int32_t pair = (int32_t)blockIdx.x >> 1, npairs = (int32_t)gridDim.x >> 1;
  const int32_t n_raw = *p.n_out;
  const int32_t n_out = n_raw <= p.wo_cap ? n_raw : 0;
  const bool tc_out = outliers_wide(n_out);
  const int32_t nk_o = tc_out ? pad64(n_out) / OK : 0;
  if (warp < EPI_WARP0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_LOW));
  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    uint32_t stage = 0, phase = 0;
    uint32_t issued = 0, last_par = 0;
    bool ok = true;
    if (!tc_out) {
      for (int32_t tile = pair; tile < num_tiles && ok; tile += npairs) {
        const int32_t m_blk = 2 * (tile % num_m2) + (int32_t)rank;
        const int32_t b_row = (tile / num_m2) * BN + (int32_t)rank * BNH;
        for (int32_t kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status,
                                 LLMINT8_DEV_TIMEOUT_PRODUCER, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), PAIR_TX);
          const uint32_t full0 = mapa_shared(full_bar(stage), 0);
          tma_load_2d_pair(sA + stage * A_STAGE_BYTES, &tmA, full0, kb * BK, m_blk * BM);
          tma_load_2d_pair(sB + stage * B_STAGE_BYTES, &tmB, full0, kb * BK, b_row);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    } else {
      ok = tc_producer_pair(p, &tmA, &tmB, &tmXO, &tmWO, sA, sB, bar0, wo_bar, abort_flag, nk_o,
                       rank, stage, phase, issued, last_par);
    }
    if (!ok) {
      // let every copy this CTA started land before shared memory goes:
      // rank 0's barriers count both CTAs' bytes; rank 1 waits a while
      volatile int never = 0;
      if (rank == 0) {
        for (int st = 0; st < STAGES; ++st)
          if ((issued >> st) & 1u)
            mbar_wait_bounded(full_bar(st), (last_par >> st) & 1u, &never, p.status,
                              LLMINT8_DEV_TIMEOUT_DRAIN, p.timeout_ns);
      } else {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 100000u) __nanosleep(1000);
      }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_i8_s32(2 * BM, BN);
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    bool any = false;
    int32_t it = 0;
    if (!tc_out) {
      for (int32_t tile = pair; tile < num_tiles && ok; tile += npairs, ++it) {
        const uint32_t acc = it & 1, acc_par = (it >> 1) & 1;
        if (!mbar_wait_bounded(tempty_bar(acc), acc_par ^ 1u, abort_flag, p.status,
                               LLMINT8_DEV_TIMEOUT_MMA, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int32_t kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status,
                                 LLMINT8_DEV_TIMEOUT_MMA, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a_desc = smem_desc_kmajor_sw128(sA + stage * A_STAGE_BYTES);
          const uint64_t b_desc = smem_desc_kmajor_sw128(sB + stage * B_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            mma_i8_pair(d_tmem, a_desc + (uint64_t)((k * UMMA_K) >> 4),
                        b_desc + (uint64_t)((k * UMMA_K) >> 4), idesc,
                        (kb > 0 || k > 0) ? 1u : 0u);
          }
          any = true;
          mma_commit_pair(mapa_shared(empty_bar(stage), 0));
          mma_commit_pair(mapa_shared(empty_bar(stage), 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(mapa_shared(tfull_bar(acc), 0));
        mma_commit_pair(mapa_shared(tfull_bar(acc), 1));
      }
    } else {
      ok = tc_mma_pair(p, sA, sB, bar0, tmem_base, abort_flag, nk_o, stage, phase, any);
    }
    if (!ok && any) {
      volatile int never = 0;
      mma_commit_pair(mapa_shared(drain_bar, 0));
      mbar_wait_bounded(drain_bar, 0, &never, p.status, LLMINT8_DEV_TIMEOUT_DRAIN,
                        p.timeout_ns);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_HIGH));
    // --------------------------------------------------------- epilogue
    const int ew = warp & 3;
    const int hc = (warp - EPI_WARP0) >> 2;
    const int et = threadIdx.x - EPI_WARP0 * 32;
    bool wo_ready = n_out == 0 || !p.build_wo;
    if (!wo_ready) {
      // Step 2, W side: this CTA's share of W^O (as K3)
      build_wo_rows(n_out, p.idx, p.wq, p.aw, p.w16, p.h, p.o, p.ldk, p.WO,
                    static_cast<int64_t>(blockIdx.x) * NUM_EPI_THREADS + et,
                    static_cast<int64_t>(gridDim.x) * NUM_EPI_THREADS);
      __threadfence();
      named_barrier(EPI_BARRIER, NUM_EPI_THREADS);
      if (et == 0) atomicAdd(p.wo_counter, 1);
    }
    float *sWO = reinterpret_cast<float *>(base + WO_OFF);
    float *sAW = reinterpret_cast<float *>(base + AW_OFF);
    uint8_t *sOut = base + OUT_OFF + (warp - EPI_WARP0) * OUT_STAGE_BYTES;
    const uint32_t sOut_addr = smem_u32(sOut);
    const int32_t n_fast = tc_out ? 0 : n_out;
    int32_t it = 0;
    for (int32_t tile = pair; tile < num_tiles; tile += npairs, ++it) {
      const uint32_t acc = it & 1, acc_par = (it >> 1) & 1;
      const int32_t m_blk = 2 * (tile % num_m2) + (int32_t)rank;
      const int32_t n_blk = tile / num_m2;
      const int32_t n0 = n_blk * BN;
      // (1) column scales and fp16 outlier rows of this tile into shared
      //     memory, while the MMA still works on the accumulator
      if (!wo_ready) {
        bool got = true;
        if (et == 0) {
          const uint64_t t0 = global_timer_ns();
          while (*reinterpret_cast<volatile int32_t *>(p.wo_counter) < (int32_t)gridDim.x) {
            if (*abort_flag || global_timer_ns() - t0 > p.wo_wait_ns) {
              got = false;
              break;
            }
            __nanosleep(128);
          }
          __threadfence();
        }
        if (named_barrier_or(EPI_BARRIER, NUM_EPI_THREADS, !got)) {
          if (named_barrier_or(EPI_BARRIER, NUM_EPI_THREADS, *abort_flag != 0)) break;
          build_wo_rows(n_out, p.idx, p.wq, p.aw, p.w16, p.h, p.o, p.ldk, p.WO, et,
                        NUM_EPI_THREADS);
          __threadfence();
          named_barrier(EPI_BARRIER, NUM_EPI_THREADS);
        }
        if (et == 0 && tc_out) {
          fence_proxy_async_global();
          mbar_arrive(wo_bar);
        }
        wo_ready = true;
      }
      named_barrier(EPI_BARRIER, NUM_EPI_THREADS);  // previous tile done reading
      {
        const int32_t j = n0 + et;
        sAW[et] = j < p.o ? __ldg(p.aw + j) : 0.0f;
      }
      for (int i = et; i < n_fast * (BN / 8); i += NUM_EPI_THREADS) {
        const int t = i / (BN / 8);
        const int c8 = (i % (BN / 8)) * 8;
        const int32_t j = n0 + c8;
        uint4 w8 = make_uint4(0u, 0u, 0u, 0u);
        if (j < p.o) w8 = __ldcg(reinterpret_cast<const uint4 *>(p.WO + (int64_t)t * p.o + j));
        const uint32_t ww[4] = {w8.x, w8.y, w8.z, w8.w};
        float4 *dst = reinterpret_cast<float4 *>(sWO + t * BN + c8);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&ww[2 * e]));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&ww[2 * e + 1]));
          dst[e] = make_float4(f0.x, f0.y, f1.x, f1.y);
        }
      }
      named_barrier(EPI_BARRIER, NUM_EPI_THREADS);
      // (2) this thread's row: scale and outlier activations
      const int32_t row = m_blk * BM + ew * 32 + lane;
      const bool row_ok = row < p.s;
      const float rs = row_ok ? __ldg(p.ax + row) * (1.0f / 16129.0f) : 0.0f;
      if (tc_out) {
        if (!tc_tile_epilogue_pair(p, &tmOut, tmem_base, tfull_bar(0),
                              mapa_shared(tempty_bar(0), 0), (uint32_t)(it & 1), abort_flag,
                              m_blk, n0, ew, hc, lane, sAW, sOut, sOut_addr, row, row_ok, rs))
          break;
        continue;
      }
      float xo[FAST_OUTLIERS];
#pragma unroll
      for (int t = 0; t < FAST_OUTLIERS; ++t)
        xo[t] = (t < n_fast && row_ok)
                    ? __half2float(__ushort_as_half(p.XO[(int64_t)row * n_out + t]))
                    : 0.0f;
      // (3) the fp16 outlier product of this thread's BN/2 columns, while
      //     the MMA still fills the accumulator
      uint64_t e2[BN / 64][16];
#pragma unroll
      for (int c = 0; c < BN / 64; ++c)
#pragma unroll
        for (int q = 0; q < 16; ++q) e2[c][q] = 0ull;
#pragma unroll
      for (int t = 0; t < FAST_OUTLIERS; ++t) {
        if (t < n_fast) {
          const uint64_t x2 = f32x2_pack(xo[t], xo[t]);
          const float4 *wrow = reinterpret_cast<const float4 *>(sWO + t * BN + hc * (BN / 2));
#pragma unroll
          for (int q4 = 0; q4 < BN / 8; ++q4) {
            const float4 w = wrow[q4];
            uint64_t *e = e2[q4 / 8];
            e[2 * (q4 % 8)] = f32x2_fma(x2, f32x2_pack(w.x, w.y), e[2 * (q4 % 8)]);
            e[2 * (q4 % 8) + 1] = f32x2_fma(x2, f32x2_pack(w.z, w.w), e[2 * (q4 % 8) + 1]);
          }
        }
      }
      // (4) accumulator; a timeout in any epilogue thread stops all of them
      const bool ready = mbar_wait_bounded(tfull_bar(acc), acc_par, abort_flag, p.status,
                                           LLMINT8_DEV_TIMEOUT_EPILOGUE, p.timeout_ns);
      if (named_barrier_or(EPI_BARRIER, NUM_EPI_THREADS, !ready)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(ew * 32) << 16) + acc * BN + hc * (BN / 2);
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row + c * 32, v);
        if (lane == 0) bulk_wait_group_read0();
        tmem_ld_wait();
        __syncwarp();
        if (c == BN / 64 - 1) {
          // the accumulator is fully read: hand it back to rank 0's MMA
          tc_fence_before();
          mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
        }
        const int32_t j0 = n0 + hc * (BN / 2) + c * 32;
        const uint64_t rs2 = f32x2_pack(rs, rs);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t h8[4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int q4 = 2 * q8 + u;
            const float4 a4 =
                *reinterpret_cast<const float4 *>(sAW + hc * (BN / 2) + c * 32 + 4 * q4);
            const uint64_t sv0 = f32x2_mul(rs2, f32x2_pack(a4.x, a4.y));
            const uint64_t sv1 = f32x2_mul(rs2, f32x2_pack(a4.z, a4.w));
            const uint64_t c0 =
                f32x2_pack((float)(int32_t)v[4 * q4], (float)(int32_t)v[4 * q4 + 1]);
            const uint64_t c1 =
                f32x2_pack((float)(int32_t)v[4 * q4 + 2], (float)(int32_t)v[4 * q4 + 3]);
            const uint64_t r0 = f32x2_fma(c0, sv0, e2[c][2 * q4]);
            const uint64_t r1 = f32x2_fma(c1, sv1, e2[c][2 * q4 + 1]);
            h8[2 * u] = f2h2(f32x2_lo(r0), f32x2_hi(r0));
            h8[2 * u + 1] = f2h2(f32x2_lo(r1), f32x2_hi(r1));
          }
          *reinterpret_cast<uint4 *>(sOut + lane * 64 + ((q8 ^ ((lane >> 1) & 3)) * 16)) =
              make_uint4(h8[0], h8[1], h8[2], h8[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        {
          const int32_t bx = j0, by = m_blk * BM + ew * 32;
          if (lane == 0 && bx < p.o && by < p.s) {
            tma_store_2d(&tmOut, sOut_addr, bx, by);
            bulk_commit_group();
          }
        }
        if (p.ci != nullptr && row_ok && j0 < p.o) {
          const bool full = (j0 + 32 <= p.o);
          int4 *cp = reinterpret_cast<int4 *>(p.ci + (int64_t)row * p.o + j0);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            if (!full && q4 >= 4) break;
            cp[q4] = make_int4((int)v[4 * q4], (int)v[4 * q4 + 1], (int)v[4 * q4 + 2],
                               (int)v[4 * q4 + 3]);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA frees the pair's TMEM, or leaves, while the other may still
  // use its barriers or its accumulator
  cluster_sync();
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
  if (threadIdx.x == 0) mirror_status_to_host(p.status, p.done_counter, p.status_host);
}

}  // namespace gemm2
}  // namespace llmint8

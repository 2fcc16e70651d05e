// K3: the int8 GEMM of LLM.int8() on 5th-generation tensor cores, with the
// dequantisation, the fp16 outlier product and the fp16 store fused into its
// epilogue.
//
// Math ("The Full LLM.int8() Algorithm", Steps 3-5; "Vector-wise
// Quantization"):
//   Ci[i][j]  = sum_k Xq[i][k] * Wq[j][k]                    int8 -> int32
//   out[i][j] = fp16( Ci[i][j] * (ax[i] / 16129) * aw[j]
//                     + sum_t XO[i][t] * WO[t][j] )          fp32
//
// Structure (one persistent CTA per SM, 384 threads; setmaxnreg moves
// registers from the first warpgroup to the two epilogue warpgroups):
//   warp 0      TMA producer: Xq and Wq tiles (128-byte swizzle) into a
//               4-stage shared-memory ring, completion on mbarriers; with
//               more than 16 outlier columns, then XO and WO tiles (fp16,
//               64 wide: the same 48 KB per stage) for the outlier product
//   warp 1      one thread issues tcgen05.mma.kind::i8 (M=128, N=256, K=32)
//               into a TMEM accumulator; with more than 16 outlier columns
//               also tcgen05.mma.kind::f16 (K=16) into a second, fp32 one;
//               tcgen05.commit frees ring slots
//   warp 2      allocates / frees the 512 TMEM columns (2 accumulators)
//   warps 4-11  epilogue: before the first tile, a share of the fp16
//               outlier rows of W, gathered while the first tiles'
//               mainloops run and announced on a counter (or, with
//               build_wo = 0, those rows come built by the activation
//               fix-up). Per tile, while the MMA runs, the column scales
//               and the tile's slice of the outlier rows go to shared
//               memory as fp32, and each thread computes the outlier
//               product of its row and its half of the tile's columns into
//               registers (packed f32x2 FMAs); with more than 16 outlier
//               columns that product comes from the tensor cores instead
//               (the second accumulator, single-buffered with the first).
//               Once the accumulator is ready, each warp tcgen05.lds its half
//               of the columns of its 32 TMEM lanes (= 32 output rows),
//               dequantises, adds the outlier product and writes fp16
//               through a 64B-swizzled 32x32 staging block with TMA stores;
//               the other accumulator is being filled by the MMA meanwhile.
// The one wait on other CTAs, for their shares of the outlier rows of W, is
// short and never needed for correctness: a CTA that has not seen every
// share within wo_wait_ns (other CTAs not resident, e.g. under SM
// partitioning) builds all the rows itself and goes on.
// Every wait is bounded by the global timer; on a timeout the CTA records a
// status bit, drains its in-flight copies and MMAs, frees TMEM and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "ptx_sm100.cuh"
#include "outlier_rows.cuh"

namespace llmint8 {
namespace gemm {

constexpr int BM = 128;           // output rows per tile (MMA M)
constexpr int BN = 256;           // output columns per tile (MMA N)
constexpr int BK = 128;           // int8 reduction bytes per stage
constexpr int STAGES = 4;
constexpr int UMMA_K = 32;        // K of one kind::i8 MMA
constexpr uint32_t A_STAGE_BYTES = BM * BK;
constexpr uint32_t B_STAGE_BYTES = BN * BK;
constexpr int NUM_ACC = 2;
constexpr uint32_t TMEM_COLS = 512;  // NUM_ACC * BN int32 columns
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_THREADS = 256;  // 8 warps: two per TMEM lane quarter
constexpr int EPI_BARRIER = 1;       // named barrier of the epilogue warps
constexpr int OUT_BOX_COLS = 32;     // fp16 columns per TMA store (64 bytes)
constexpr uint32_t OUT_STAGE_BYTES = 32 * OUT_BOX_COLS * 2;  // per epilogue warp
constexpr int REGS_LOW = 56;         // producer / MMA warpgroup after setmaxnreg
constexpr int REGS_HIGH = 208;       // epilogue warpgroups after setmaxnreg
constexpr int FAST_OUTLIERS = 16;    // outlier rows kept in shared memory
constexpr uint32_t RING_BYTES = STAGES * (A_STAGE_BYTES + B_STAGE_BYTES);
constexpr uint32_t OUT_OFF = RING_BYTES;
constexpr uint32_t WO_OFF = OUT_OFF + 8 * OUT_STAGE_BYTES;  // fp32 [FAST_OUTLIERS][BN]
constexpr uint32_t AW_OFF = WO_OFF + FAST_OUTLIERS * BN * 4;
constexpr uint32_t BAR_OFF = AW_OFF + BN * 4;
constexpr size_t SMEM_BYTES = 1024 + BAR_OFF + 256;

static_assert(NUM_ACC * BN <= 512, "TMEM holds 512 columns");
// registers a thread gets at launch (65536 / 384 rounded down to a multiple
// of 8); setmaxnreg.inc can only hand out what .dec gave back
constexpr int REGS_LAUNCH = 168;
static_assert((NUM_THREADS - NUM_EPI_THREADS) * REGS_LOW + NUM_EPI_THREADS * REGS_HIGH <=
                  NUM_THREADS * REGS_LAUNCH,
              "register split exceeds the launch allocation");
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
static_assert(OUT_OFF % 1024 == 0, "swizzled staging must be 1024-byte aligned");
static_assert(BAR_OFF % 8 == 0, "mbarrier alignment");
static_assert((2 * STAGES + 2 * NUM_ACC + 2) * 8 + 8 <= 256, "barrier block size");
// the fp16 outlier stages (XO: BM x 64 fp16, WO: BN x 64 fp16) are the same
// size as the int8 ones, so both kinds share the ring
constexpr int OK = 64;             // outlier columns per fp16 stage
constexpr int UMMA_K16 = 16;       // K of one kind::f16 MMA
static_assert(BM * OK * 2 == A_STAGE_BYTES && BN * OK * 2 == B_STAGE_BYTES,
              "fp16 outlier stages fill the int8 stage slots exactly");

struct Params {
  int32_t s, h, o;
  int32_t num_m_blocks, num_n_blocks, num_k_blocks;
  const float *ax;        // [s]
  const float *aw;        // [o]
  const uint16_t *XO;     // outlier columns of X (layout: outlier_rows.cuh)
  uint16_t *WO;           // outlier rows of W: built here when build_wo, else
                          // before this launch (layout: outlier_rows.cuh)
  int32_t ldk;            // row stride of the wide outlier layout
  const int8_t *wq;       // [o][h] int8 codes of W
  const uint16_t *w16;    // optional fp16 W [h][o]: WO rows are its own rows
  const int32_t *idx;     // outlier columns, ascending
  int32_t build_wo;       // 1: the CTAs build WO (shares, then the wait)
  int32_t *wo_counter;    // CTAs done with their share of WO; zero on entry
  uint64_t wo_wait_ns;    // how long a CTA waits for the other shares
  const int32_t *n_out;   // device scalar |O|
  int32_t wo_cap;         // outlier rows the workspace holds; |O| above it:
                          // no outlier product (the fix-up flagged it)
  int32_t *ci;            // optional [s][o] int32
  int32_t *status;        // device status word
  int32_t *done_counter;  // CTAs finished (zero between calls), used only
  int32_t *status_host;   // with a mapped host word (or null) that receives
                          // the status bits when the last CTA finishes
  uint64_t timeout_ns;
};

__device__ __forceinline__ uint32_t f2h2(float a, float b) {
  const __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// Producer of the tensor-core outlier mode (more than 16 outlier columns):
// per tile the int8 stages, then the fp16 outlier stages (XO and WO tiles,
// 64 outlier columns each). WO is read by TMA: when the epilogue builds it,
// wait for its signal on wo_bar (every share in, or built by this CTA), then
// order those generic-proxy writes before the async-proxy reads. Out of line
// so that the narrow mode's producer loop is compiled as if it were alone.
// Returns false if a wait ran out.
__device__ __noinline__ bool tc_producer(const Params &p, const CUtensorMap *tmA,
                                         const CUtensorMap *tmB, const CUtensorMap *tmXO,
                                         const CUtensorMap *tmWO, uint32_t sA, uint32_t sB,
                                         uint32_t bar0, uint32_t wo_bar,
                                         volatile int *abort_flag, int32_t nk_o,
                                         uint32_t &stage, uint32_t &phase, uint32_t &issued,
                                         uint32_t &last_par) {
  const int32_t num_tiles = p.num_m_blocks * p.num_n_blocks;
  bool wo_ok = !p.build_wo;
  for (int32_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
    const int32_t m_blk = tile % p.num_m_blocks;
    const int32_t n_blk = tile / p.num_m_blocks;
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
      mbar_arrive_expect_tx(full, A_STAGE_BYTES + B_STAGE_BYTES);
      if (!o_stage) {
        tma_load_2d(sA + stage * A_STAGE_BYTES, tmA, full, kb * BK, m_blk * BM);
        tma_load_2d(sB + stage * B_STAGE_BYTES, tmB, full, kb * BK, n_blk * BN);
      } else {
        const int32_t ko = (kb - p.num_k_blocks) * OK;
        tma_load_2d(sA + stage * A_STAGE_BYTES, tmXO, full, ko, m_blk * BM);
        tma_load_2d(sB + stage * B_STAGE_BYTES, tmWO, full, ko, n_blk * BN);
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

// MMA issuer of the tensor-core outlier mode: one int32 accumulator
// (columns 0..BN) and the fp32 outlier product (columns BN..2BN) per tile,
// 16 outlier columns per f16 MMA (32 bytes of a stage, as for int8). Out of
// line for the same reason as tc_producer. Returns false if a wait ran out.
__device__ __noinline__ bool tc_mma(const Params &p, uint32_t sA, uint32_t sB, uint32_t bar0,
                                    uint32_t tmem_base, volatile int *abort_flag, int32_t nk_o,
                                    uint32_t &stage, uint32_t &phase, bool &any) {
  constexpr uint32_t idesc = idesc_i8_s32(BM, BN);
  constexpr uint32_t idesc16 = idesc_f16_f32(BM, BN);
  const int32_t num_tiles = p.num_m_blocks * p.num_n_blocks;
  const uint32_t tfull = bar0 + 8u * (2 * STAGES), tempty = bar0 + 8u * (2 * STAGES + NUM_ACC);
  int32_t it = 0;
  for (int32_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
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
          mma_i8(tmem_base, a_desc + (uint64_t)((k * UMMA_K) >> 4),
                 b_desc + (uint64_t)((k * UMMA_K) >> 4), idesc, (kb > 0 || k > 0) ? 1u : 0u);
      } else {
        const int32_t ko = kb - p.num_k_blocks;
#pragma unroll
        for (int k = 0; k < OK / UMMA_K16; ++k)
          mma_f16(tmem_base + BN, a_desc + (uint64_t)((k * UMMA_K16 * 2) >> 4),
                  b_desc + (uint64_t)((k * UMMA_K16 * 2) >> 4), idesc16,
                  (ko > 0 || k > 0) ? 1u : 0u);
      }
      any = true;
      mma_commit(empty);
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    mma_commit(tfull);
  }
  return true;
}

// One tile's epilogue in tensor-core outlier mode: waits for the tile (int32
// accumulator in columns 0..BN, fp32 outlier product in BN..2BN), then per
// 32 columns loads both, out = fp16(ci * (rs * aw[j]) + e), and stores
// through the warp's staging block. Kept out of line so that the narrow
// mode's tile loop is not compiled around it. False if a wait ran out.
__device__ __noinline__ bool tc_tile_epilogue(const Params &p, const CUtensorMap *tmOut,
                                              uint32_t tmem_base, uint32_t tfull,
                                              uint32_t tempty, uint32_t parity,
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
      mbar_arrive(tempty);
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

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_i8_fused(const __grid_constant__ CUtensorMap tmA,
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
  // the epilogue's signal that WO is complete (only for a CTA that builds
  // it and then feeds it to the tensor cores)
  const uint32_t wo_bar = bar0 + 8u * (2 * STAGES + 2 * NUM_ACC + 1);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 2 * NUM_ACC + 2);
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
    mbar_init(wo_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // Everything above overlaps the tail of the preceding kernel when launched
  // as a programmatic dependent; from here on its outputs are read.
  grid_dependency_wait();

  const int32_t num_tiles = p.num_m_blocks * p.num_n_blocks;
  // |O| (above the workspace's capacity: no outlier product); more than 16
  // outlier columns go through the tensor cores, in nk_o fp16 stages
  const int32_t n_raw = *p.n_out;
  const int32_t n_out = n_raw <= p.wo_cap ? n_raw : 0;
  const bool tc_out = outliers_wide(n_out);
  const int32_t nk_o = tc_out ? pad64(n_out) / OK : 0;
  // Two int32 accumulators alternate between tiles; in tensor-core mode one
  // int32 and one fp32 accumulator (columns BN..2BN) serve every tile. Each
  // role takes one branch on the mode, so the narrow mode's loops are the
  // same code as without the tensor-core outlier path.
  if (warp < EPI_WARP0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_LOW));
  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    uint32_t stage = 0, phase = 0;
    uint32_t issued = 0, last_par = 0;  // per-stage bits, for the drain
    bool ok = true;
    // WO is read by TMA: when this CTA's epilogue builds it, wait for its
    // signal (every share in, or built here), then order those generic-proxy
    // writes before the async-proxy reads
    if (!tc_out) {
      for (int32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int32_t m_blk = tile % p.num_m_blocks;
        const int32_t n_blk = tile / p.num_m_blocks;
        for (int32_t kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status,
                                 LLMINT8_DEV_TIMEOUT_PRODUCER, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), A_STAGE_BYTES + B_STAGE_BYTES);
          tma_load_2d(sA + stage * A_STAGE_BYTES, &tmA, full_bar(stage), kb * BK, m_blk * BM);
          tma_load_2d(sB + stage * B_STAGE_BYTES, &tmB, full_bar(stage), kb * BK, n_blk * BN);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    } else {
      ok = tc_producer(p, &tmA, &tmB, &tmXO, &tmWO, sA, sB, bar0, wo_bar, abort_flag, nk_o,
                       stage, phase, issued, last_par);
    }
    if (!ok) {
      // let every copy this thread started land before shared memory goes
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
    bool ok = true;
    bool any = false;
    int32_t it = 0;
    if (!tc_out) {
      for (int32_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
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
            // advance the start address by k*32 bytes inside the swizzle atom
            mma_i8(d_tmem, a_desc + (uint64_t)((k * UMMA_K) >> 4),
                   b_desc + (uint64_t)((k * UMMA_K) >> 4), idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          any = true;
          mma_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(tfull_bar(acc));
      }
    } else {
      ok = tc_mma(p, sA, sB, bar0, tmem_base, abort_flag, nk_o, stage, phase, any);
    }
    if (!ok && any) {
      volatile int never = 0;
      mma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, &never, p.status, LLMINT8_DEV_TIMEOUT_DRAIN,
                        p.timeout_ns);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_HIGH));
    // --------------------------------------------------------- epilogue
    const int ew = warp & 3;          // TMEM lane quarter of this warp
    const int hc = (warp - EPI_WARP0) >> 2;  // which half of the tile's columns
    const int et = threadIdx.x - EPI_WARP0 * 32;  // 0..255
    static_assert(FAST_OUTLIERS == kNarrowOutliers, "the narrow layout is the fast path");
    bool wo_ready = n_out == 0 || !p.build_wo;
    if (!wo_ready) {
      // Step 2, W side: this CTA's share of the (t, j) pairs of WO, while the
      // first tile's mainloop runs; the one-byte gathers are spread over
      // every CTA
      build_wo_rows(n_out, p.idx, p.wq, p.aw, p.w16, p.h, p.o, p.ldk, p.WO,
                    static_cast<int64_t>(blockIdx.x) * NUM_EPI_THREADS + et,
                    static_cast<int64_t>(gridDim.x) * NUM_EPI_THREADS);
      __threadfence();
      named_barrier(EPI_BARRIER, NUM_EPI_THREADS);
      if (et == 0) atomicAdd(p.wo_counter, 1);
    }
    float *sWO = reinterpret_cast<float *>(base + WO_OFF);         // [16][BN] fp32
    float *sAW = reinterpret_cast<float *>(base + AW_OFF);         // [BN]
    uint8_t *sOut = base + OUT_OFF + (warp - EPI_WARP0) * OUT_STAGE_BYTES;  // [32][64 B]
    const uint32_t sOut_addr = smem_u32(sOut);
    // outlier columns summed here on CUDA cores (none in tensor-core mode)
    const int32_t n_fast = tc_out ? 0 : n_out;
    int32_t it = 0;
    for (int32_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const uint32_t acc = it & 1, acc_par = (it >> 1) & 1;
      const int32_t m_blk = tile % p.num_m_blocks;
      const int32_t n_blk = tile / p.num_m_blocks;
      const int32_t n0 = n_blk * BN;
      // (1) column scales and fp16 outlier rows of this tile into shared
      //     memory, while the MMA still works on the accumulator
      if (!wo_ready) {
        // every CTA's share of WO is written, or, if that takes longer than
        // wo_wait_ns, this CTA writes all of WO itself (the same values)
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
          // the same decision in every epilogue thread: stop on an abort,
          // else build all of WO here
          if (named_barrier_or(EPI_BARRIER, NUM_EPI_THREADS, *abort_flag != 0)) break;
          build_wo_rows(n_out, p.idx, p.wq, p.aw, p.w16, p.h, p.o, p.ldk, p.WO, et,
                        NUM_EPI_THREADS);
          __threadfence();
          named_barrier(EPI_BARRIER, NUM_EPI_THREADS);
        }
        // WO is complete: the producer may feed it to the tensor cores
        if (et == 0 && tc_out) {
          fence_proxy_async_global();
          mbar_arrive(wo_bar);
        }
        wo_ready = true;
      }
      named_barrier(EPI_BARRIER, NUM_EPI_THREADS);  // previous tile done reading
      static_assert(NUM_EPI_THREADS == BN, "one epilogue thread per tile column");
      {
        const int32_t j = n0 + et;
        const bool jok = j < p.o;
        const float awj = jok ? __ldg(p.aw + j) : 0.0f;
        sAW[et] = awj;
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
        if (!tc_tile_epilogue(p, &tmOut, tmem_base, tfull_bar(0), tempty_bar(0),
                              (uint32_t)(it & 1), abort_flag, m_blk, n0, ew, hc, lane, sAW,
                              sOut, sOut_addr, row, row_ok, rs))
          break;
        continue;
      }
      float xo[FAST_OUTLIERS];
#pragma unroll
      for (int t = 0; t < FAST_OUTLIERS; ++t)
        xo[t] = (t < n_fast && row_ok)
                    ? __half2float(__ushort_as_half(p.XO[(int64_t)row * n_out + t]))
                    : 0.0f;
      // (3) the fp16 outlier product e = sum_t xo[t] * WO[t][j] of this
      //     thread's BN/2 columns, while the MMA still fills the accumulator
      //     (it does not depend on Ci); packed pairs of columns
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
        // the staging block is free once the previous store has read it
        if (lane == 0) bulk_wait_group_read0();
        tmem_ld_wait();
        __syncwarp();
        if (c == BN / 64 - 1) {
          // the accumulator is fully read: hand it back to the MMA warp
          tc_fence_before();
          mbar_arrive(tempty_bar(acc));
        }
        // out = fp16(ci * (rs * aw[j]) + e), two columns per packed op
        const int32_t j0 = n0 + hc * (BN / 2) + c * 32;
        // 8 outputs at a time into the 64B-swizzled 32x32 staging block;
        // chunk k of row r lives at 16-byte slot k ^ ((r / 2) % 4)
        const uint64_t rs2 = f32x2_pack(rs, rs);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t h8[4];  // fp16 pairs
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
          if (lane == 0 && bx < p.o && by < p.s) {  // partial boxes are clipped by TMA
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
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, TMEM_COLS);
  if (threadIdx.x == 0) mirror_status_to_host(p.status, p.done_counter, p.status_host);
}

}  // namespace gemm
}  // namespace llmint8

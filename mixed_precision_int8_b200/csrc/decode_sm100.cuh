// K4: decode-regime LLM.int8() GEMM (s <= 16 rows of X), bound by the read of
// the int8 weight from HBM.
//
// The int8 product is computed transposed on the tensor cores: the weight
// tile (128 output columns x 128 reduction bytes) is the MMA's A operand
// (M = 128) and the <= 16 quantised rows of X are its B operand (N = 16,
// zero-filled by TMA beyond s). The (weight tile, k-block) units are split
// evenly over one persistent CTA per SM, so every SM streams the same share
// of the weight whatever the wave count. Each CTA adds its partial int32
// accumulators into a [s][o] int32 buffer with integer atomics (exact and
// order-independent; the buffer is zeroed by the call's first kernel).
//
// The rest of the layer is folded into the same kernel:
//  - the fp16 outlier weight rows WO[t][j] = fp16(fp32(fp32(wq[j][O_t]) *
//    aw[j]) / 127) are read out of the weight tiles already streaming through
//    shared memory (the MMA warp reads a stage whose k-block holds an
//    outlier column before its commit releases the stage), so the column
//    gather costs no HBM traffic;
//  - the last CTA to finish a tile (an atomic arrival count; nobody waits)
//    applies the dequantisation, the fp16 outlier product and the store:
//      out[i][j] = fp16( Ci[i][j] * (ax[i] / 16129) * aw[j] + sum_t XO[i][t] WO[t][j] )
// ("The Full LLM.int8() Algorithm", Steps 2-5).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "ptx_sm100.cuh"
#include "outlier_rows.cuh"

namespace llmint8 {
namespace decode {

constexpr int MAX_ROWS = 16;
constexpr int BM = 128;   // weight rows (output columns) per tile: MMA M
constexpr int BN = 16;    // X rows, zero-padded: MMA N
constexpr int BOX_K = 128;  // reduction bytes of one TMA box (one 128B swizzle row)
constexpr int SUB = 2;      // boxes per stage
constexpr int BK = BOX_K * SUB;  // reduction bytes per stage
constexpr int STAGES = 5;
constexpr int UMMA_K = 32;
constexpr uint32_t A_BOX_BYTES = BM * BOX_K;   // 16 KB
constexpr uint32_t B_BOX_BYTES = BN * BOX_K;   // 2 KB
constexpr uint32_t A_STAGE_BYTES = A_BOX_BYTES * SUB;
constexpr uint32_t B_STAGE_BYTES = B_BOX_BYTES * SUB;
constexpr int NUM_ACC = 2;
constexpr uint32_t TMEM_COLS = 32;
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_THREADS = 128;
constexpr int MAX_MASK_WORDS = (133144 + 31) / 32;  // h <= 133144
constexpr uint32_t RING_BYTES = STAGES * (A_STAGE_BYTES + B_STAGE_BYTES);
constexpr int MAX_KB_WORDS = (MAX_MASK_WORDS * 32 / BK + 31) / 32 + 1;
static_assert(BK % 32 == 0 && (BK / 32) <= 32, "mask words per k-block");
// outlier bitmask words, their prefix counts, then one bit per k-block that
// holds an outlier column
constexpr uint32_t MASK_OFF = RING_BYTES;
constexpr uint32_t KB_OFF = MASK_OFF + 4 * (2 * MAX_MASK_WORDS + 1);
// mbarriers need 8-byte alignment; start them on a 128-byte boundary
constexpr uint32_t BAR_OFF = (KB_OFF + 4 * MAX_KB_WORDS + 127) & ~127u;
constexpr size_t SMEM_BYTES = 1024 + BAR_OFF + 256;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
static_assert(BAR_OFF % 8 == 0, "mbarrier alignment");
static_assert((2 * STAGES + 2 * NUM_ACC + 1) * 8 + 12 <= 256, "barrier block size");

constexpr int EPI_BARRIER = 1;

struct Params {
  int32_t s, h, o;
  int32_t num_m_blocks, num_k_blocks;
  int64_t units_total;
  const float *ax;
  const float *aw;
  const uint32_t *mask;   // outlier-column bitmask [ceil(h/32)]
  const int32_t *word_prefix;  // outlier columns before each mask word
  const uint16_t *XO;     // outlier columns of X (layout: outlier_rows.cuh)
  uint16_t *WO;           // outlier rows of W, written here (same layout rules)
  int32_t ldk;            // row stride of the wide layout
  const uint16_t *w16;    // optional fp16 W [h][o]: WO rows are its own rows
  const int32_t *n_out;
  int32_t wo_cap;         // outlier rows the workspace holds; |O| above it:
                          // no outlier product (the row pass flagged it)
  uint16_t *out;
  int32_t *ci;            // optional exact accumulators [s][o]
  int32_t *cacc;          // [s][o] int32 partial sums (zeroed before the launch)
  int32_t *tile_count;    // [num_m_blocks] arrivals (zeroed before the launch)
  int32_t *status;
  int32_t *done_counter;  // CTAs finished (zero between calls), used only
  int32_t *status_host;   // with a mapped host word (or null) for the status
  uint64_t timeout_ns;
};

// Generic pointer to shared-memory address `saddr` + stage offset.
__device__ __forceinline__ const void *base_ptr_of(uint32_t sA, uint32_t stage) {
  extern __shared__ uint8_t smem_raw[];
  return smem_raw + (sA - smem_u32(smem_raw)) + stage * A_STAGE_BYTES;
}

// Index of the CTA whose unit range contains unit u (inverse of cta_units).
__device__ __forceinline__ int64_t cta_of_unit(const Params &p, int64_t u) {
  const int64_t G = gridDim.x;
  return (G * (u + 1) + p.units_total - 1) / p.units_total - 1;
}

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
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + BAR_OFF);
  uint32_t *s_mask = reinterpret_cast<uint32_t *>(base + MASK_OFF);
  int32_t *s_prefix = reinterpret_cast<int32_t *>(s_mask + MAX_MASK_WORDS);
  uint32_t *s_kb = reinterpret_cast<uint32_t *>(base + KB_OFF);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (STAGES + st); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + NUM_ACC + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2 * NUM_ACC);
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 2 * NUM_ACC + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  // segments whose outlier weight rows the MMA warp has published (monotonic)
  volatile int *wo_segments = reinterpret_cast<volatile int *>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    *wo_segments = 0;
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
#pragma unroll
      for (int b = 0; b < SUB; ++b) {
        tma_load_2d_hint(sA + stage * A_STAGE_BYTES + b * A_BOX_BYTES, &tmA, full_bar(stage),
                         kb * BK + b * BOX_K, m_blk * BM, pol_w);
        tma_load_2d(sB + stage * B_STAGE_BYTES + b * B_BOX_BYTES, &tmB, full_bar(stage),
                    kb * BK + b * BOX_K, 0);
      }
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
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (lane 0)
    // The whole warp also reads the fp16 outlier weight rows out of stages
    // whose k-block holds an outlier column: for column c of the k-block,
    // row r of the 128B-swizzled box holds wq[j][c] in 16-byte chunk
    // ((c - k0) / 16) ^ (r % 8). The reads finish before lane 0's commit
    // releases the stage (a stage holds SUB boxes of BOX_K columns; column c
    // of the stage lives in box c / BOX_K). Which k-blocks hold outlier columns is the same
    // for every tile, so a per-k-block bitmap is built once and the next
    // such k-block is kept in a register: an ordinary stage costs one
    // compare. After each segment the rows are published (fence) by bumping
    // wo_segments.
    constexpr uint32_t idesc = idesc_i8_s32(BM, BN);
    const int32_t n_raw = *p.n_out;
    const int32_t n_out = n_raw <= p.wo_cap ? n_raw : 0;
    const int32_t nwords = (p.h + 31) >> 5;
    const int32_t kb_words = (int32_t)((nk + 31) >> 5);
    for (int32_t w = lane; w < nwords; w += 32) {
      s_mask[w] = __ldg(p.mask + w);
      s_prefix[w] = __ldg(p.word_prefix + w);
    }
    __syncwarp();
    for (int32_t kw = 0; kw < kb_words; ++kw) {
      const int32_t kb = kw * 32 + lane;
      bool has = false;
      if (kb < nk)
        for (int32_t w = kb * (BK / 32); w < min(nwords, (kb + 1) * (BK / 32)); ++w)
          has |= s_mask[w] != 0u;
      const uint32_t word = __ballot_sync(0xFFFFFFFFu, has);
      if (lane == 0) s_kb[kw] = word;
    }
    __syncwarp();
    // first k-block >= kb holding an outlier column (nk if none)
    auto next_outlier_kb = [&](int32_t kb) -> int32_t {
      if (n_out == 0) return (int32_t)nk;
      for (int32_t kw = kb >> 5; kw < kb_words; ++kw) {
        uint32_t m = s_kb[kw];
        if (kw == (kb >> 5)) m &= ~0u << (kb & 31);
        if (m) return kw * 32 + __ffs(m) - 1;
      }
      return (int32_t)nk;
    };
    uint32_t stage = 0, phase = 0;
    bool ok = true, any = false;
    int32_t it = 0;
    float aw_rows[BM / 32];  // column scales of this lane's 4 tile rows
    for (int64_t u = u0; u < u1 && ok; ++it) {
      const int64_t m_blk = u / nk;
      const int64_t seg_end = min(u1, (m_blk + 1) * nk);
      const uint32_t acc = it & 1, acc_par = (it >> 1) & 1;
      int32_t next_kb = next_outlier_kb((int32_t)(u - m_blk * nk));
#pragma unroll
      for (int q = 0; q < BM / 32; ++q) {
        const int64_t j = m_blk * BM + lane + 32 * q;
        aw_rows[q] = (n_out > 0 && j < p.o) ? __ldg(p.aw + j) : 0.0f;
      }
      // every lane waits; a vote keeps the warp's decision uniform
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(tempty_bar(acc), acc_par ^ 1u, abort_flag,
                                                     p.status, LLMINT8_DEV_TIMEOUT_MMA,
                                                     p.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int64_t v = u; v < seg_end; ++v) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full_bar(stage), phase, abort_flag,
                                                       p.status, LLMINT8_DEV_TIMEOUT_MMA,
                                                       p.timeout_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int b = 0; b < SUB; ++b) {
            const uint64_t a_desc =
                smem_desc_kmajor_sw128(sA + stage * A_STAGE_BYTES + b * A_BOX_BYTES);
            const uint64_t b_desc =
                smem_desc_kmajor_sw128(sB + stage * B_STAGE_BYTES + b * B_BOX_BYTES);
#pragma unroll
            for (int k = 0; k < BOX_K / UMMA_K; ++k)
              mma_i8(d_tmem, a_desc + (uint64_t)((k * UMMA_K) >> 4),
                     b_desc + (uint64_t)((k * UMMA_K) >> 4), idesc,
                     (v > u || b > 0 || k > 0) ? 1u : 0u);
          }
        }
        any = true;
        const int32_t kb = (int32_t)(v - m_blk * nk);
        if (kb == next_kb) {
          const int32_t k0 = kb * BK;
          const int32_t w0 = k0 >> 5;
          const int32_t nw = (p.h - k0) < BK ? (p.h - k0 + 31) >> 5 : BK / 32;
          const uint8_t *stage_a = reinterpret_cast<const uint8_t *>(base_ptr_of(sA, stage));
          for (int32_t w = 0; w < nw; ++w) {
            uint32_t bits = s_mask[w0 + w];
            int32_t rank = s_prefix[w0 + w];
            while (bits) {
              const int b = __ffs(bits) - 1;
              bits &= bits - 1;
              const int32_t cc = w * 32 + b;  // column inside the k-block
              const uint8_t *box = stage_a + (cc / BOX_K) * A_BOX_BYTES;
              const int32_t cb = cc % BOX_K;  // column inside that box
#pragma unroll
              for (int q = 0; q < BM / 32; ++q) {
                const int r = lane + 32 * q;
                const int64_t j = m_blk * BM + r;
                if (j < p.o) {
                  const int64_t dst = wo_index(rank, j, n_out, p.o, p.ldk);
                  if (p.w16) {  // the caller's fp16 row of W
                    p.WO[dst] = __ldg(p.w16 + (int64_t)(k0 + cc) * p.o + j);
                  } else {
                    const int8_t code = static_cast<int8_t>(
                        box[r * BOX_K + ((((cb >> 4) ^ (r & 7)) << 4) | (cb & 15))]);
                    const float prod = static_cast<float>(code) * aw_rows[q];
                    p.WO[dst] = __half_as_ushort(__float2half_rn(__fdiv_rn(prod, 127.0f)));
                  }
                }
              }
              ++rank;
            }
          }
          next_kb = next_outlier_kb(kb + 1);
          __syncwarp();  // every lane has read the stage before it is released
        }
        if (lane == 0) mma_commit(empty_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) mma_commit(tfull_bar(acc));
      __threadfence();  // publish this segment's outlier weight rows
      __syncwarp();
      if (lane == 0) *wo_segments = it + 1;
      u = seg_end;
    }
    if (!ok && any && lane == 0) {
      volatile int never = 0;
      mma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, &never, p.status, LLMINT8_DEV_TIMEOUT_DRAIN, p.timeout_ns);
    }
  } else if (warp >= EPI_WARP0) {
    // ---------------------------------------------------------- epilogue
    const int ew = warp - EPI_WARP0;
    const int et = threadIdx.x - EPI_WARP0 * 32;  // 0..127: one tile column
    const int32_t n_raw = *p.n_out;
    const int32_t n_out = n_raw <= p.wo_cap ? n_raw : 0;
    const int32_t nf = n_out < 16 ? n_out : 16;
    __shared__ int last_arrival;
    // the row scales (over 16129) and the first 16 outlier activations of
    // every row, shared by all columns of every tile this CTA finishes
    __shared__ float s_rs[MAX_ROWS];
    __shared__ float s_xo[MAX_ROWS][16];
    for (int q = et; q < MAX_ROWS * 16; q += NUM_EPI_THREADS) {
      const int i = q / 16, t = q % 16;
      s_xo[i][t] = (i < p.s && t < nf)
                       ? __half2float(__ushort_as_half(__ldg(p.XO + xo_index(i, t, n_out, p.ldk))))
                       : 0.0f;
      if (t == 0) s_rs[i] = i < p.s ? __ldg(p.ax + i) * (1.0f / 16129.0f) : 0.0f;
    }
    named_barrier(EPI_BARRIER, NUM_EPI_THREADS);
    int32_t it = 0;
    for (int64_t u = u0; u < u1; ++it) {
      const int64_t m_blk = u / nk;
      const int64_t seg_end = min(u1, (m_blk + 1) * nk);
      const uint32_t acc = it & 1, acc_par = (it >> 1) & 1;
      const int64_t j = m_blk * BM + et;  // this thread's output column
      const bool ready = mbar_wait_bounded(tfull_bar(acc), acc_par, abort_flag, p.status,
                                           LLMINT8_DEV_TIMEOUT_EPILOGUE, p.timeout_ns);
      if (named_barrier_or(EPI_BARRIER, NUM_EPI_THREADS, !ready)) break;
      tc_fence_after();
      uint32_t v[16];
      __syncwarp();
      tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(ew * 32) << 16) + acc * BN, v);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      if (j < p.o) {
#pragma unroll
        for (int i = 0; i < BN; ++i)
          if (i < p.s && v[i] != 0u) atomicAdd(p.cacc + (int64_t)i * p.o + j, (int32_t)v[i]);
      }
      // count this CTA's arrival on the tile once its accumulators and its
      // outlier weight rows (warp 3) are visible; the last contributor
      // finishes the tile
      bool rows_ok = true;
      if (*wo_segments <= it) {  // bounded wait for the MMA warp's publication
        const uint64_t t0 = global_timer_ns();
        while (*wo_segments <= it) {
          if (*abort_flag || global_timer_ns() - t0 > p.timeout_ns) {
            if (!*abort_flag) {
              *abort_flag = 1;
              atomicOr(p.status, LLMINT8_DEV_TIMEOUT_EPILOGUE);
            }
            rows_ok = false;
            break;
          }
        }
      }
      __threadfence();
      if (named_barrier_or(EPI_BARRIER, NUM_EPI_THREADS, !rows_ok)) break;
      if (et == 0) {
        const int64_t contrib = cta_of_unit(p, (m_blk + 1) * nk - 1) - cta_of_unit(p, m_blk * nk) + 1;
        last_arrival = (atomicAdd(p.tile_count + m_blk, 1) == (int32_t)(contrib - 1));
      }
      named_barrier(EPI_BARRIER, NUM_EPI_THREADS);
      if (last_arrival && j < p.o) {
        // every load of this column is issued before the first use: its
        // scale, its outlier weights and the s int32 sums (one round trip)
        __threadfence();
        const float awj = __ldcg(p.aw + j);
        float wo[16];
#pragma unroll
        for (int t = 0; t < 16; ++t)
          wo[t] = (t < nf) ? __half2float(__ushort_as_half(
                                 __ldcg(p.WO + wo_index(t, j, n_out, p.o, p.ldk))))
                           : 0.0f;
        int32_t cv[MAX_ROWS];
#pragma unroll
        for (int i = 0; i < MAX_ROWS; ++i)
          cv[i] = i < p.s ? __ldcg(p.cacc + (int64_t)i * p.o + j) : 0;
#pragma unroll
        for (int i = 0; i < MAX_ROWS; ++i) {
          if (i < p.s) {
            float acc_f = (float)cv[i] * s_rs[i] * awj;
#pragma unroll
            for (int t = 0; t < 16; ++t) acc_f = fmaf(s_xo[i][t], wo[t], acc_f);
            for (int32_t t = 16; t < n_out; ++t)
              acc_f = fmaf(
                  __half2float(__ushort_as_half(__ldcg(p.XO + xo_index(i, t, n_out, p.ldk)))),
                  __half2float(__ushort_as_half(__ldcg(p.WO + wo_index(t, j, n_out, p.o, p.ldk)))),
                  acc_f);
            p.out[(int64_t)i * p.o + j] = __half_as_ushort(__float2half_rn(acc_f));
            if (p.ci) p.ci[(int64_t)i * p.o + j] = cv[i];
          }
        }
      }
      u = seg_end;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, TMEM_COLS);
  if (threadIdx.x == 0) mirror_status_to_host(p.status, p.done_counter, p.status_host);
}

}  // namespace decode
}  // namespace llmint8

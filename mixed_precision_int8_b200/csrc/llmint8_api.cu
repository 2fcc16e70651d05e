// C ABI of the LLM.int8() linear-layer library (declared in include/llmint8.h):
// argument validation, workspace layout, TMA descriptor creation and the
// launch sequence of the kernels in quant_kernels.cuh and gemm_sm100.cuh.
// Host code only enqueues work; it never allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "llmint8.h"
#include "quant_kernels.cuh"
#include "gemm_sm100.cuh"
#include "gemm_pair_sm100.cuh"
#include "decode_sm100.cuh"

namespace {

using namespace llmint8;

constexpr int64_t kMaxH = 133144;  // 127*127*h must fit int32
constexpr int64_t kDecodeMaxRows = decode::MAX_ROWS;
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per individual wait
// how long a GEMM CTA waits for the other CTAs' shares of the outlier rows of
// W before it builds them all itself: far longer than the shares take when
// every CTA is resident (a few microseconds), and shorter than building them
// all alone takes on the large shapes, so it runs out only when peers are
// not resident (SM partitioning, time slicing)
constexpr uint64_t kWoWaitNs = 500000ull;
// dynamic shared memory of k_act_rows (one CTA per SM)
constexpr uint32_t kActSmemOnePerSm = 220 * 1024;

// ----------------------------------------------------------- device info
struct DeviceInfo {
  bool init = false;
  bool supported = false;
  int sm_count = 0;
  int max_pairs = 0;  // CTA pairs of the pair GEMM that fit at once (0: none)
  int64_t l2_bytes = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mutex;

llmint8_status device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return LLMINT8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo &d = g_dev[dev];
  if (!d.init) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return LLMINT8_ERR_CUDA;
    d.supported = (prop.major == 10 && prop.minor == 0);
    d.sm_count = prop.multiProcessorCount;
    d.l2_bytes = prop.l2CacheSize;
    if (d.supported) {
      if (cudaFuncSetAttribute(gemm::k_gemm_i8_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)gemm::SMEM_BYTES) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
      if (cudaFuncSetAttribute(decode::k_decode_i8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)decode::SMEM_BYTES) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
      if (cudaFuncSetAttribute(k_act_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kActSmemOnePerSm) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
      if (cudaFuncSetAttribute(gemm2::k_gemm_i8_pair,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)gemm2::SMEM_BYTES) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
      // clusters of two co-resident CTAs the pair GEMM can have at once
      // (an SM left over in a GPC cannot host half of one)
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (unsigned)(d.sm_count / 2));
      cfg.blockDim = dim3(gemm::NUM_THREADS);
      cfg.dynamicSmemBytes = gemm2::SMEM_BYTES;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, gemm2::k_gemm_i8_pair, &cfg) != cudaSuccess)
        clusters = 0;
      cudaGetLastError();  // a refusal only leaves the pair kernel unused
      d.max_pairs = std::min(clusters, d.sm_count / 2);
    }
    d.init = true;
  }
  if (!d.supported) return LLMINT8_ERR_UNSUPPORTED;
  *out = &d;
  return LLMINT8_OK;
}

// ----------------------------------------------------- TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D int8 tensor [rows][inner] with row stride `inner` bytes, box
// [box_rows][box_inner] landing in shared memory with the 128-byte swizzle.
bool make_tmap_i8(CUtensorMap *map, const void *ptr, uint64_t inner, uint64_t rows,
                  uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp16 tensor [rows][inner] (row stride 2*inner bytes) for TMA stores of
// [box_rows][box_inner] blocks staged with the 128-byte swizzle.
bool make_tmap_f16(CUtensorMap *map, void *ptr, uint64_t inner, uint64_t rows,
                   uint32_t box_inner, uint32_t box_rows) {
  const CUtensorMapSwizzle swz = box_inner * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {2 * inner};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ptr, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------ workspace layout
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
  size_t status, acc, mask, wprefix, idx, ax, xq, xo, wo, tiles, cacc, end;
  size_t xstage, ostage, end_host;
};

int32_t mask_words(int64_t h) { return (int32_t)((h + 31) / 32); }

// The state block at the front of a workspace, cleared by
// llmint8_workspace_init and kept by the kernels between calls: the status
// words, then the accumulation bitmask of the one-read activation pass
// (sized for the largest h), which that pass leaves zero on exit.
constexpr size_t kStateBytes = 256 + ((4 * (size_t)((kMaxH + 31) / 32) + 255) & ~size_t(255));
static_assert(kStateBytes == LLMINT8_WORKSPACE_STATE_BYTES, "state block size");

// Row stride of the wide outlier layout (more than 16 outlier columns, K-major
// for the tensor cores, outlier_rows.cuh): the capacity rounded up to 64, or
// 0 when the capacity admits only the narrow layout.
int64_t wide_ld(int64_t cap) { return cap > kNarrowOutliers ? (cap + 63) / 64 * 64 : 0; }

// `cap` = outlier columns the XO / WO tiles hold (h for any alpha).
Layout layout_for(int64_t s, int64_t h, int64_t o, int64_t cap) {
  const int64_t kcap = std::max(cap, wide_ld(cap));
  Layout L;
  size_t off = 0;
  L.status = off;  off = align256(off + 256);
  L.acc = off;     off = kStateBytes;
  L.mask = off;    off = align256(off + 4 * (size_t)mask_words(h));
  L.wprefix = off; off = align256(off + 4 * ((size_t)mask_words(h) + 1));
  L.idx = off;     off = align256(off + 4 * (size_t)h);
  L.ax = off;      off = align256(off + 4 * (size_t)s);
  L.xq = off;      off = align256(off + (size_t)s * h);
  L.tiles = off;   off = align256(off + 4 * (size_t)((o + decode::BM - 1) / decode::BM));
  L.cacc = off;    off = align256(off + 4 * (size_t)kDecodeMaxRows * o);
  L.xo = off;      off = align256(off + 2 * (size_t)s * kcap);
  L.wo = off;      off = align256(off + 2 * (size_t)kcap * o);
  L.end = off;
  L.xstage = off;  off = align256(off + 2 * (size_t)s * h);
  L.ostage = off;  off = align256(off + 2 * (size_t)s * o);
  L.end_host = off;
  return L;
}

// status block: [0] device status bits, [1] |O|, [2] column-pass block
// counter, [3] block counter of the one-read activation pass (zero between
// calls), [4] CTAs of the call's last kernel that have finished (zero
// between calls; counted only when the status bits go to a host word)
int32_t *status_word(void *ws) { return reinterpret_cast<int32_t *>(ws); }
int32_t *count_word(void *ws) { return reinterpret_cast<int32_t *>(ws) + 1; }
int32_t *block_counter_word(void *ws) { return reinterpret_cast<int32_t *>(ws) + 2; }
int32_t *act_counter_word(void *ws) { return reinterpret_cast<int32_t *>(ws) + 3; }
int32_t *done_counter_word(void *ws) { return reinterpret_cast<int32_t *>(ws) + 4; }
// [6] CTAs of the GEMM done with their share of the outlier rows of W
// (zeroed by the call's activation kernels)
int32_t *wo_counter_word(void *ws) { return reinterpret_cast<int32_t *>(ws) + 6; }
float *tensor_scale_word(void *ws) { return reinterpret_cast<float *>(ws) + 5; }
constexpr int kSelftestWord = 8;  // a status-block word no kernel sets

// --------------------------------------------------------- validation
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

llmint8_status check_hw(int64_t h, int64_t o) {
  if (h < 16 || h > kMaxH || (h % 16) != 0) return LLMINT8_ERR_SHAPE;
  if (o < 16 || (o % 16) != 0 || o > (int64_t)INT32_MAX / 2) return LLMINT8_ERR_SHAPE;
  return LLMINT8_OK;
}

llmint8_status check_alpha(float alpha) {
  if (std::isnan(alpha) || alpha < 0.0f) return LLMINT8_ERR_ARG;
  return LLMINT8_OK;
}

float half_bits_value(uint32_t b) {
  const int e = (b >> 10) & 0x1f, m = b & 0x3ff;
  if (e == 0) return std::ldexp((float)m, -24);
  if (e == 31) return m ? NAN : INFINITY;
  return std::ldexp((float)(1024 + m), e - 25);
}

// Smallest non-negative binary16 magnitude bit pattern whose value is >=
// alpha (0x7C00 = +inf when none is finite), so that for a non-NaN x,
// |x| >= alpha  <=>  (bits(x) & 0x7FFF) >= threshold.
uint32_t threshold_bits(float alpha) {
  uint32_t lo = 0, hi = 0x7C00;
  while (lo < hi) {
    const uint32_t mid = (lo + hi) / 2;
    if (half_bits_value(mid) >= alpha) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

llmint8_status last_launch() {
  return cudaGetLastError() == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

// Launch with programmatic stream serialization when `pdl`: the kernel may
// be scheduled while its predecessor drains; it orders itself after the
// predecessor with griddepcontrol.wait before touching memory.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t st, bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same for a kernel run by clusters of two CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pairs(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t st, bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Steps 1, 2 and 4 (activation side, plus the fp16 outlier rows of W when
// WO != nullptr): bitmask + compaction, then row scales, codes and outlier
// tiles. Adds the number of kernels enqueued to *launches.
struct ActivationArgs {
  const uint16_t *X;
  int64_t s, h;
  float alpha;
  uint32_t *mask;
  int32_t *wprefix, *idx, *count, *block_counter;
  uint32_t *acc_mask;     // one-read pass: accumulation bitmask (zero on entry
  int32_t *act_counter;   // and exit, with its block counter)
  bool act_reset;         // zero them first (their state is not known)
  uint8_t *flags;
  int8_t *Xq;
  float *ax;
  uint16_t *XO;
  const int8_t *wq;
  const float *aw;
  const uint16_t *w16;
  int64_t o;
  uint16_t *WO;  // fp16 outlier rows of W, built here for |O| > 16 (or null)
  int32_t cap;   // outlier columns XO and WO hold
  int32_t ldk;   // row stride of the wide outlier layout
  int32_t *zero_buf;
  int64_t zero_n;
  int *status;  // device status bits
  int32_t *gemm_counter;  // zeroed for a GEMM that builds WO itself (or null)
};

// Launch plan of k_act_rows (one CTA per SM): `groups` row groups of `wpr`
// warps, each group with `stages` row buffers of `stage_bytes`. Calls with
// at least 16 rows per SM run one warp per row, as many as shared memory
// holds (up to 32); shorter calls spread their rows over every SM in one
// wave with up to four warps per row (named barriers cap the groups at
// 15). Two buffers per group when they fit. False when one row does not
// fit, in which case the two-pass kernels run.
struct ActPlan {
  int32_t groups;
  int32_t wpr;
  int32_t stages;
  uint32_t stage_bytes;
  uint32_t smem;
  int64_t grid;
};

bool act_plan(int64_t s, int64_t h, int sm_count, ActPlan *plan) {
  const uint32_t sb = (uint32_t)((2 * h + 127) / 128 * 128);
  const uint32_t fixed = act_smem_bytes(0, sb, (int32_t)h);
  if (fixed + sb + 8 > kActSmemOnePerSm) return false;
  const int64_t fit = (kActSmemOnePerSm - fixed) / (sb + 8);  // buffers that fit
  int64_t per_sm = (s + sm_count - 1) / sm_count;
  if (per_sm < 1) per_sm = 1;
  int64_t groups, wpr;
  if (per_sm >= 16 && fit >= 16) {
    wpr = 1;
    groups = std::min<int64_t>(std::min<int64_t>(fit, per_sm), kActMaxWarps);
  } else {
    groups = std::min<int64_t>(std::min<int64_t>(fit, per_sm), kActMaxGroups);
    wpr = std::max<int64_t>(1, std::min<int64_t>(kActMaxWpr, kActMaxWarps / groups));
  }
  const int64_t stages = fit / groups >= 2 ? 2 : 1;
  plan->groups = (int32_t)groups;
  plan->wpr = (int32_t)wpr;
  plan->stages = (int32_t)stages;
  plan->stage_bytes = sb;
  plan->smem = act_smem_bytes((int32_t)(groups * stages), sb, (int32_t)h);
  int64_t grid = (s + groups - 1) / groups;
  if (grid > sm_count) grid = sm_count;
  if (grid < 1) grid = 1;
  plan->grid = grid;
  return true;
}

// Steps 1 and 4 with one read of X (k_act_rows), then the completion of the
// outlier columns and the fp16 outlier rows of W (k_act_fixup).
llmint8_status enqueue_activation_fused(const DeviceInfo &dev, const ActivationArgs &a,
                                        const ActPlan &plan, cudaStream_t st,
                                        int32_t *launches) {
  cudaError_t e;
  if (a.act_reset) {
    int64_t reset_blocks = (mask_words(a.h) + 255) / 256;
    if (reset_blocks > 4 * (int64_t)dev.sm_count) reset_blocks = 4 * (int64_t)dev.sm_count;
    e = launch(k_reset_mask, dim3((unsigned)reset_blocks), dim3(256), 0, st, false, a.acc_mask,
               mask_words(a.h), a.count, a.act_counter, (int32_t *)nullptr, (int64_t)0);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    *launches += 1;
  }
  ActRowsParams p;
  p.X = a.X;
  p.s = a.s;
  p.h = (int32_t)a.h;
  p.thresh_bits = threshold_bits(a.alpha);
  p.groups = plan.groups;
  p.wpr = plan.wpr;
  p.stages = plan.stages;
  p.stage_bytes = plan.stage_bytes;
  p.timeout_ns = kTimeoutNs;
  p.acc_mask = a.acc_mask;
  p.mask = a.mask;
  p.count = a.count;
  p.block_counter = a.act_counter;
  p.word_prefix = a.wprefix;
  p.idx = a.idx;
  p.flags = a.flags;
  p.Xq = a.Xq;
  p.ax = a.ax;
  p.status = a.status;
  e = launch(k_act_rows, dim3((unsigned)plan.grid), dim3(32 * plan.groups * plan.wpr), plan.smem,
             st, true, p);
  if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
  *launches += 1;
  const int64_t fix_blocks = (a.s + kFixRowsPerBlock - 1) / kFixRowsPerBlock;
  if (fix_blocks > 0) {
    FixupParams f;
    f.X = a.X;
    f.s = a.s;
    f.h = (int32_t)a.h;
    f.thresh_bits = p.thresh_bits;
    f.mask = a.mask;
    f.word_prefix = a.wprefix;
    f.idx = a.idx;
    f.count = a.count;
    f.Xq = a.Xq;
    f.ax = a.ax;
    f.XO = a.XO;
    f.cap = a.cap;
    f.ldk = a.ldk;
    f.row_blocks = fix_blocks;
    f.wq = a.wq;
    f.aw = a.aw;
    f.w16 = a.w16;
    f.o = (int32_t)a.o;
    f.WO = a.WO;
    f.status = a.status;
    f.gemm_counter = a.gemm_counter;
    // one extra block per SM builds the fp16 outlier rows of W while the
    // row blocks run (|O| is known on the device only; with none they
    // return at once)
    const int64_t grid = fix_blocks + (a.WO ? (int64_t)dev.sm_count : 0);
    e = launch(k_act_fixup, dim3((unsigned)grid), dim3(kFixThreads), 0, st, true, f);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    *launches += 1;
  }
  return last_launch();
}

// Tensor-wise activation scale, after the activation pass has left the
// bitmask and the row scales: one constant (the largest row scale) for all
// rows, and every row's codes again against it.
llmint8_status enqueue_tensor_scale(const ActivationArgs &a, float *scale, cudaStream_t st,
                                    int32_t *launches) {
  cudaError_t e = launch(k_tensor_scale, dim3(1), dim3(1024), 0, st, true,
                         (const float *)a.ax, a.s, scale);
  if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
  const int64_t rb = (a.s + kRowsPerBlock - 1) / kRowsPerBlock;
  e = launch(k_rows_tensor_scale, dim3((unsigned)rb), dim3(kRowThreads), 0, st, true, a.X, a.s,
             (int32_t)a.h, (const uint32_t *)a.mask, (const int32_t *)a.wprefix,
             (const float *)scale, a.Xq, a.ax);
  if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
  *launches += 2;
  return LLMINT8_OK;
}

llmint8_status enqueue_activation_pass(const DeviceInfo &dev, const ActivationArgs &a,
                                       cudaStream_t st, int32_t *launches) {
  ActPlan plan;
  if (a.zero_n == 0 && act_plan(a.s, a.h, dev.sm_count, &plan))
    return enqueue_activation_fused(dev, a, plan, st, launches);
  const int32_t nwords = mask_words(a.h);
  const int32_t hh = (int32_t)a.h;
  int64_t reset_threads = nwords > a.zero_n ? nwords : a.zero_n;
  int64_t reset_blocks = (reset_threads + 255) / 256;
  if (reset_blocks < 1) reset_blocks = 1;
  if (reset_blocks > 4 * (int64_t)dev.sm_count) reset_blocks = 4 * (int64_t)dev.sm_count;
  // the one extra word a prefill call may zero is the GEMM's WO counter
  int32_t *zb = a.zero_buf;
  int64_t zn = a.zero_n;
  if (!zb && a.gemm_counter) {
    zb = a.gemm_counter;
    zn = 1;
  }
  cudaError_t e = launch(k_reset_mask, dim3((unsigned)reset_blocks), dim3(256), 0, st, false,
                         a.mask, nwords, a.count, a.block_counter, zb, zn);
  if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
  const int gx = (int)((a.h + kColsPerBlock - 1) / kColsPerBlock);
  const int64_t want_blocks = 4 * (int64_t)dev.sm_count;
  int64_t gy_target = (want_blocks + gx - 1) / gx;
  int64_t rpb = (a.s + gy_target - 1) / gy_target;
  rpb = (rpb + 7) / 8 * 8;  // whole batches of eight rows in flight per thread
  if (rpb < 8) rpb = 8;     // (s == 0: one empty block row still compacts)
  if ((a.s + rpb - 1) / rpb > 65535) rpb = (a.s + 65534) / 65535;
  const int gy = (int)std::max<int64_t>(1, (a.s + rpb - 1) / rpb);
  e = launch(k_outlier_columns, dim3(gx, gy), dim3(kColThreads), 0, st, true, a.X, a.s, hh,
             threshold_bits(a.alpha), (int32_t)rpb, a.mask, a.count, a.block_counter, a.wprefix,
             a.idx, a.flags);
  if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
  *launches += 2;
  const int64_t rb = (a.s + kRowsPerBlock - 1) / kRowsPerBlock;
  if (rb > 0) {
    e = launch(k_rows_any, dim3((unsigned)rb), dim3(kRowThreads), 0, st, true, a.X, a.s, hh,
               (const uint32_t *)a.mask, (const int32_t *)a.wprefix, (const int32_t *)a.count,
               a.Xq, a.ax, a.XO, a.cap, a.ldk, a.status);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    *launches += 1;
  }
  if (a.WO) {
    // fp16 outlier rows of W (returns at once without outlier columns)
    e = launch(k_build_wo, dim3((unsigned)(2 * dev.sm_count)), dim3(256), 0, st, true,
               (const int32_t *)a.count, (const int32_t *)a.idx, a.wq, a.aw, a.w16, hh,
               (int32_t)a.o, a.ldk, a.WO, a.cap);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    *launches += 1;
  }
  return last_launch();
}

llmint8_status validate_weight(const llmint8_weight *w) {
  if (!w || !w->wq_dev || !w->aw_dev) return LLMINT8_ERR_NULL;
  llmint8_status st = check_hw(w->h, w->o);
  if (st) return st;
  if (!aligned(w->wq_dev, 16) || !aligned(w->aw_dev, 16) ||
      (w->w16_dev && !aligned(w->w16_dev, 16)))
    return LLMINT8_ERR_ALIGN;
  return LLMINT8_OK;
}

// opts->max_outliers as a capacity (h when 0); -1 when invalid.
int64_t outlier_cap(const llmint8_matmul_opts *opts, int64_t h) {
  const int64_t m = opts ? opts->max_outliers : 0;
  if (m < 0 || m > h) return -1;
  return m == 0 ? h : m;
}

// The options every matmul form checks before it enqueues anything.
llmint8_status check_opts(const llmint8_matmul_opts *opts, int64_t s, int64_t h) {
  if (!opts) return LLMINT8_OK;
  if (opts->path < LLMINT8_PATH_AUTO || opts->path > LLMINT8_PATH_PREFILL_PAIR ||
      (opts->path == LLMINT8_PATH_DECODE && s > kDecodeMaxRows))
    return LLMINT8_ERR_ARG;
  if (opts->x_scale != LLMINT8_SCALE_VECTORWISE && opts->x_scale != LLMINT8_SCALE_TENSORWISE)
    return LLMINT8_ERR_ARG;
  if (outlier_cap(opts, h) < 0) return LLMINT8_ERR_ARG;
  if (opts->wo_build < LLMINT8_WO_SHARED || opts->wo_build > LLMINT8_WO_EACH_CTA)
    return LLMINT8_ERR_ARG;
  if (opts->status_host) {
    // pinned host memory the device reaches at the same address
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, opts->status_host) != cudaSuccess) {
      cudaGetLastError();
      return LLMINT8_ERR_ARG;
    }
    if (pa.type != cudaMemoryTypeHost || pa.devicePointer != (void *)opts->status_host ||
        !aligned(opts->status_host, 4))
      return LLMINT8_ERR_ARG;
  }
  return LLMINT8_OK;
}

// A previous call left anomaly bits in the caller's host status word.
bool host_status_set(const llmint8_matmul_opts *opts) {
  return opts && opts->status_host &&
         *reinterpret_cast<volatile int32_t *>(opts->status_host) != 0;
}

// Whether the automatic choice takes the CTA-pair GEMM for a prefill call.
// It does not: measured on B200 at the OPT shapes, the pair kernel is as
// fast as the one-CTA kernel at best (175B FFN: 796 against 786 us per
// launch under ncu, the tensor pipes 82% busy in both, with more DRAM reads
// of Wq, 886 against 745 MB) and slower where the weight stays in L2 (13B
// FFN: 291 against 279 us). It stays selectable (LLMINT8_PATH_PREFILL_PAIR).
bool pair_gemm_preferred(int64_t h, int64_t o, const DeviceInfo &dev) {
  (void)h;
  (void)o;
  (void)dev;
  return false;
}

llmint8_status matmul_impl(const uint16_t *X, int64_t s, const llmint8_weight *w, float alpha,
                           uint16_t *out, void *ws, size_t ws_bytes, llmint8_matmul_opts *opts,
                           cudaStream_t st, bool host_layout, bool reset_state = false) {
  if (opts) opts->launches = 0;
  llmint8_status rc = validate_weight(w);
  if (rc) return rc;
  if (s < 0 || s > (int64_t)INT32_MAX) return LLMINT8_ERR_SHAPE;
  if ((rc = check_alpha(alpha))) return rc;
  if ((rc = check_opts(opts, s, w->h))) return rc;
  const int path = opts ? opts->path : 0;
  const int x_scale = opts ? opts->x_scale : LLMINT8_SCALE_VECTORWISE;
  if (host_status_set(opts)) return LLMINT8_ERR_DEVICE_STATUS;
  if (s == 0) return LLMINT8_OK;
  if (!X || !out || !ws) return LLMINT8_ERR_NULL;
  if (!aligned(X, 16) || !aligned(out, 16) || !aligned(ws, 256)) return LLMINT8_ERR_ALIGN;
  if (opts && opts->ci_dev && !aligned(opts->ci_dev, 16)) return LLMINT8_ERR_ALIGN;
  const int64_t h = w->h, o = w->o;
  const int64_t cap = outlier_cap(opts, h);
  const int64_t ldk = wide_ld(cap);
  int32_t *status_host = opts ? opts->status_host : nullptr;
  const Layout L = layout_for(s, h, o, cap);
  if (ws_bytes < (host_layout ? L.end_host : L.end)) return LLMINT8_ERR_WORKSPACE;
  DeviceInfo *dev = nullptr;
  if ((rc = device_info(&dev))) return rc;

  uint8_t *wsb = static_cast<uint8_t *>(ws);
  uint32_t *mask = reinterpret_cast<uint32_t *>(wsb + L.mask);
  int32_t *wprefix = reinterpret_cast<int32_t *>(wsb + L.wprefix);
  int32_t *idx = reinterpret_cast<int32_t *>(wsb + L.idx);
  float *ax = reinterpret_cast<float *>(wsb + L.ax);
  int8_t *xq = reinterpret_cast<int8_t *>(wsb + L.xq);
  uint16_t *xo = reinterpret_cast<uint16_t *>(wsb + L.xo);
  uint16_t *wo = reinterpret_cast<uint16_t *>(wsb + L.wo);
  int32_t *cacc = reinterpret_cast<int32_t *>(wsb + L.cacc);
  int32_t *count = count_word(ws);
  int32_t *status = status_word(ws);

  const bool use_decode =
      (path == LLMINT8_PATH_DECODE) || (path == LLMINT8_PATH_AUTO && s <= kDecodeMaxRows);
  // the prefill kernel: a CTA pair per 256 x 256 tile, or one CTA per
  // 128 x 256 tile
  const bool use_pair = !use_decode && (path == LLMINT8_PATH_PREFILL_PAIR ||
                                        (path != LLMINT8_PATH_PREFILL_SINGLE &&
                                         pair_gemm_preferred(w->h, w->o, *dev)));
  if (use_pair && dev->max_pairs < 1) return LLMINT8_ERR_UNSUPPORTED;

  // Tensor maps first: a failure here must leave nothing enqueued.
  CUtensorMap tmA, tmB, tmOut, tmXO, tmWO;
  // the pair kernel's boxes of Wq and W^O hold a CTA's half of a tile's
  // columns
  const uint32_t b_rows = use_pair ? (uint32_t)gemm2::BNH : (uint32_t)gemm::BN;
  if (use_decode) {
    // A = Wq tiles (rows of o), B = Xq rows (s <= 16, zero-filled to 16)
    if (!make_tmap_i8(&tmA, w->wq_dev, (uint64_t)h, (uint64_t)o, decode::BOX_K, decode::BM) ||
        !make_tmap_i8(&tmB, xq, (uint64_t)h, (uint64_t)s, decode::BOX_K, decode::BN))
      return LLMINT8_ERR_CUDA;
  } else {
    if (!make_tmap_i8(&tmA, xq, (uint64_t)h, (uint64_t)s, gemm::BK, gemm::BM) ||
        !make_tmap_i8(&tmB, w->wq_dev, (uint64_t)h, (uint64_t)o, gemm::BK, b_rows) ||
        !make_tmap_f16(&tmOut, out, (uint64_t)o, (uint64_t)s, gemm::OUT_BOX_COLS, 32))
      return LLMINT8_ERR_CUDA;
    // the wide outlier tiles for the tensor cores (used only when |O| > 16)
    if (ldk > 0) {
      if (!make_tmap_f16(&tmXO, xo, (uint64_t)ldk, (uint64_t)s, gemm::OK, gemm::BM) ||
          !make_tmap_f16(&tmWO, wo, (uint64_t)ldk, (uint64_t)o, gemm::OK, b_rows))
        return LLMINT8_ERR_CUDA;
    } else {
      tmXO = tmA;
      tmWO = tmB;
    }
  }

  int32_t launches = 0;
  ActivationArgs act;
  act.X = X;
  act.s = s;
  act.h = h;
  act.alpha = alpha;
  act.mask = mask;
  act.wprefix = wprefix;
  act.idx = idx;
  act.count = count;
  act.block_counter = block_counter_word(ws);
  act.acc_mask = reinterpret_cast<uint32_t *>(wsb + L.acc);
  act.act_counter = act_counter_word(ws);
  act.act_reset = reset_state;  // otherwise the workspace keeps them zero
  act.flags = nullptr;
  act.status = status;
  act.Xq = xq;
  act.ax = ax;
  act.XO = xo;
  act.wq = w->wq_dev;
  act.aw = w->aw_dev;
  act.w16 = w->w16_dev;
  act.o = o;
  act.cap = (int32_t)cap;
  act.ldk = (int32_t)ldk;
  // prefill: the GEMM's CTAs build the fp16 outlier rows of W themselves
  // while their first mainloops run (unless gemm_plain asks for them from
  // the activation kernels); decode: the W^O gather and the finishing step
  // run inside the decode kernel; its tile counters and the s rows of int32
  // partial sums (one contiguous region) start from zero
  const int wo_build = opts ? opts->wo_build : LLMINT8_WO_SHARED;
  const bool gemm_builds_wo = !use_decode && wo_build != LLMINT8_WO_BEFORE_GEMM;
  act.WO = (use_decode || gemm_builds_wo) ? nullptr : wo;
  act.gemm_counter = gemm_builds_wo ? wo_counter_word(ws) : nullptr;
  int32_t *tiles = reinterpret_cast<int32_t *>(wsb + L.tiles);
  act.zero_buf = use_decode ? tiles : nullptr;
  act.zero_n = use_decode ? (int64_t)((L.cacc - L.tiles) / 4) + s * o : 0;
  if (use_decode) {
    // two launches of 1024-column blocks; the first also zeroes the tile
    // counters and the s rows of int32 partial sums (extra blocks). This
    // path needs no outlier list (the decode kernel reads outlier rows of W
    // with the bitmask and prefix counts), so the list's region holds the
    // per-block row maxima ([col_blocks][16] words <= h words)
    const int32_t col_blocks = (int32_t)((h + kDecodeColsPerBlock - 1) / kDecodeColsPerBlock);
    int64_t zb = (act.zero_n + kDecodeThreads * 8 - 1) / (kDecodeThreads * 8);
    if (zb > 2 * (int64_t)dev->sm_count) zb = 2 * (int64_t)dev->sm_count;
    if (zb < 1) zb = 1;
    uint32_t *partial = reinterpret_cast<uint32_t *>(idx);  // idx unused on this path
    cudaError_t e0 = launch(k_decode_colpass, dim3((unsigned)(col_blocks + zb)),
                            dim3(kDecodeThreads), 0, st, false, X, (int32_t)s, (int32_t)h,
                            threshold_bits(alpha), mask, partial, col_blocks, act.zero_buf,
                            act.zero_n);
    if (e0 != cudaSuccess) return LLMINT8_ERR_CUDA;
    e0 = launch(k_decode_rowpass, dim3((unsigned)col_blocks, (unsigned)s), dim3(kDecodeThreads), 0,
                st, true,
                X, (int32_t)s, (int32_t)h, (const uint32_t *)mask, (const uint32_t *)partial,
                col_blocks, wprefix, count, ax, xq, xo, (int32_t)cap, (int32_t)ldk, status);
    if (e0 != cudaSuccess) return LLMINT8_ERR_CUDA;
    launches += 2;
  } else if ((rc = enqueue_activation_pass(*dev, act, st, &launches))) {
    return rc;
  }
  if (x_scale == LLMINT8_SCALE_TENSORWISE &&
      (rc = enqueue_tensor_scale(act, tensor_scale_word(ws), st, &launches)))
    return rc;
  const bool timed = opts && (opts->gemm_event_start || opts->gemm_event_stop);
  if (opts && opts->gemm_event_start)
    cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->gemm_event_start), st);
  cudaError_t e;
  if (use_decode) {
    decode::Params p;
    p.s = (int32_t)s;
    p.h = (int32_t)h;
    p.o = (int32_t)o;
    p.num_m_blocks = (int32_t)((o + decode::BM - 1) / decode::BM);
    p.num_k_blocks = (int32_t)((h + decode::BK - 1) / decode::BK);
    p.ax = ax;
    p.aw = w->aw_dev;
    p.mask = mask;
    p.word_prefix = wprefix;
    p.XO = xo;
    p.WO = wo;
    p.ldk = (int32_t)ldk;
    p.w16 = w->w16_dev;
    p.n_out = count;
    p.wo_cap = (int32_t)cap;
    p.out = out;
    p.ci = opts ? opts->ci_dev : nullptr;
    p.cacc = cacc;
    p.tile_count = tiles;
    p.status = status;
    p.done_counter = done_counter_word(ws);
    p.status_host = status_host;
    p.timeout_ns = kTimeoutNs;
    const int64_t total_units = (int64_t)p.num_m_blocks * p.num_k_blocks;
    int grid = dev->sm_count;
    if (total_units < grid) grid = (int)total_units;
    p.units_total = total_units;
    e = launch(decode::k_decode_i8, dim3(grid), dim3(decode::NUM_THREADS), decode::SMEM_BYTES, st,
               !timed, tmA, tmB, p);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    if (opts && opts->gemm_event_stop)
      cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->gemm_event_stop), st);
    launches += 1;
  } else {
    gemm::Params p;
    p.s = (int32_t)s;
    p.h = (int32_t)h;
    p.o = (int32_t)o;
    p.num_m_blocks = (int32_t)((s + gemm::BM - 1) / gemm::BM);
    p.num_n_blocks = (int32_t)((o + gemm::BN - 1) / gemm::BN);
    p.num_k_blocks = (int32_t)((h + gemm::BK - 1) / gemm::BK);
    p.ax = ax;
    p.aw = w->aw_dev;
    p.XO = xo;
    p.WO = wo;
    p.ldk = (int32_t)ldk;
    p.wq = w->wq_dev;
    p.w16 = w->w16_dev;
    p.idx = idx;
    p.wo_counter = wo_counter_word(ws);
    p.n_out = count;
    p.wo_cap = (int32_t)cap;
    p.ci = opts ? opts->ci_dev : nullptr;
    p.status = status;
    p.done_counter = done_counter_word(ws);
    p.status_host = status_host;
    p.timeout_ns = kTimeoutNs;
    p.build_wo = gemm_builds_wo ? 1 : 0;
    p.wo_wait_ns = wo_build == LLMINT8_WO_EACH_CTA ? 0 : kWoWaitNs;
    if (use_pair) {
      const int64_t tiles = (int64_t)((p.num_m_blocks + 1) / 2) * p.num_n_blocks;
      const int pairs = (int)(tiles < dev->max_pairs ? tiles : dev->max_pairs);
      e = launch_pairs(gemm2::k_gemm_i8_pair, dim3(2 * pairs), dim3(gemm::NUM_THREADS),
                       gemm2::SMEM_BYTES, st, !timed, tmA, tmB, tmOut, tmXO, tmWO, p);
    } else {
      const int64_t tiles = (int64_t)p.num_m_blocks * p.num_n_blocks;
      const int grid = (int)(tiles < dev->sm_count ? tiles : dev->sm_count);
      e = launch(gemm::k_gemm_i8_fused, dim3(grid), dim3(gemm::NUM_THREADS), gemm::SMEM_BYTES,
                 st, !timed, tmA, tmB, tmOut, tmXO, tmWO, p);
    }
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    if (opts && opts->gemm_event_stop)
      cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->gemm_event_stop), st);
    ++launches;
  }
  if (opts) opts->launches = launches;
  return last_launch();
}

}  // namespace

extern "C" {

const char *llmint8_status_string(llmint8_status st) {
  switch (st) {
    case LLMINT8_OK: return "ok";
    case LLMINT8_ERR_NULL: return "required pointer is NULL";
    case LLMINT8_ERR_SHAPE: return "size breaks the shape rules";
    case LLMINT8_ERR_ALIGN: return "pointer breaks the alignment rules";
    case LLMINT8_ERR_WORKSPACE: return "workspace too small";
    case LLMINT8_ERR_CUDA: return "CUDA call failed";
    case LLMINT8_ERR_DEVICE_STATUS: return "a kernel flagged an anomaly";
    case LLMINT8_ERR_ARG: return "invalid scalar argument";
    case LLMINT8_ERR_UNSUPPORTED: return "current device is not sm_100";
    case LLMINT8_ERR_TOO_LARGE:
      return "problem needs more scratch than the no-alloc entry point holds";
  }
  return "unknown status";
}

size_t llmint8_workspace_size(int64_t s, int64_t h, int64_t o) {
  if (s < 0 || h < 0 || o < 0) return 0;
  return layout_for(s, h, o, h).end;
}

size_t llmint8_workspace_size_ex(int64_t s, int64_t h, int64_t o, int64_t max_outliers) {
  if (s < 0 || h < 0 || o < 0 || max_outliers < 0 || max_outliers > h) return 0;
  return layout_for(s, h, o, max_outliers == 0 ? h : max_outliers).end;
}

llmint8_status llmint8_workspace_init(void *ws_dev, size_t ws_bytes, void *stream) {
  if (!ws_dev) return LLMINT8_ERR_NULL;
  if (!aligned(ws_dev, 256)) return LLMINT8_ERR_ALIGN;
  if (ws_bytes < kStateBytes) return LLMINT8_ERR_WORKSPACE;
  return cudaMemsetAsync(ws_dev, 0, kStateBytes, as_stream(stream)) == cudaSuccess
             ? LLMINT8_OK
             : LLMINT8_ERR_CUDA;
}

size_t llmint8_workspace_size_host(int64_t s, int64_t h, int64_t o) {
  if (s < 0 || h < 0 || o < 0) return 0;
  return layout_for(s, h, o, h).end_host;
}

size_t llmint8_workspace_size_host_ex(int64_t s, int64_t h, int64_t o, int64_t max_outliers) {
  if (s < 0 || h < 0 || o < 0 || max_outliers < 0 || max_outliers > h) return 0;
  return layout_for(s, h, o, max_outliers == 0 ? h : max_outliers).end_host;
}

int64_t llmint8_decode_max_rows(void) { return kDecodeMaxRows; }

llmint8_status llmint8_prepare_weight(const uint16_t *W_dev, int64_t h, int64_t o,
                                      llmint8_weight *out, void *stream) {
  return llmint8_prepare_weight_ex(W_dev, h, o, LLMINT8_SCALE_VECTORWISE, out, stream);
}

llmint8_status llmint8_prepare_weight_ex(const uint16_t *W_dev, int64_t h, int64_t o,
                                         int32_t w_scale, llmint8_weight *out, void *stream) {
  return llmint8_prepare_weight_cols(W_dev, h, o, 0, o, w_scale, out, stream);
}

llmint8_status llmint8_prepare_weight_cols(const uint16_t *W_dev, int64_t h, int64_t ldw,
                                           int64_t col0, int64_t o, int32_t w_scale,
                                           llmint8_weight *out, void *stream) {
  if (w_scale != LLMINT8_SCALE_VECTORWISE && w_scale != LLMINT8_SCALE_TENSORWISE)
    return LLMINT8_ERR_ARG;
  if (!W_dev || !out || !out->wq_dev || !out->aw_dev) return LLMINT8_ERR_NULL;
  llmint8_status rc = check_hw(h, o);
  if (rc) return rc;
  if (col0 < 0 || ldw < o || col0 > ldw - o || (ldw % 8) != 0 || (col0 % 8) != 0)
    return LLMINT8_ERR_SHAPE;
  if (out->h != h || out->o != o) return LLMINT8_ERR_SHAPE;
  const uint16_t *W0 = W_dev + col0;
  if (!aligned(W0, 16) || !aligned(out->wq_dev, 16) || !aligned(out->aw_dev, 16))
    return LLMINT8_ERR_ALIGN;
  DeviceInfo *dev = nullptr;
  if ((rc = device_info(&dev))) return rc;
  cudaStream_t st = as_stream(stream);
  uint32_t *awb = reinterpret_cast<uint32_t *>(out->aw_dev);
  const int32_t hh = (int32_t)h, oo = (int32_t)o;
  k_zero_u32<<<(unsigned)((o + 255) / 256), 256, 0, st>>>(awb, o);
  const int gx = (int)((o / 8 + 255) / 256);
  int64_t gy_target = (8 * (int64_t)dev->sm_count + gx - 1) / gx;
  int64_t rpb = (h + gy_target - 1) / gy_target;
  if (rpb < 8) rpb = 8;
  const int gy = (int)((h + rpb - 1) / rpb);
  k_weight_colmax<<<dim3(gx, gy), 256, 0, st>>>(W0, hh, oo, ldw, (int32_t)rpb, awb);
  if (w_scale == LLMINT8_SCALE_TENSORWISE) k_bits_to_tensor_max<<<1, 1024, 0, st>>>(awb, o);
  k_weight_codes<<<dim3((unsigned)((o + kWqTile - 1) / kWqTile),
                        (unsigned)((h + kWqTile - 1) / kWqTile)),
                   256, 0, st>>>(W0, hh, oo, ldw, awb, out->wq_dev);
  k_widen_scales<<<(unsigned)((o + 255) / 256), 256, 0, st>>>(awb, oo);
  return last_launch();
}

size_t llmint8_quantize_rows_scratch_size(int64_t h) {
  if (h < 0) return 0;
  return 256 + 2 * align256(4 * (size_t)mask_words(h)) +
         align256(4 * ((size_t)mask_words(h) + 1));
}

llmint8_status llmint8_quantize_rows(const uint16_t *X_dev, int64_t s, int64_t h, float alpha,
                                     int8_t *Xq_dev, float *ax_dev, uint8_t *flags_dev,
                                     int32_t *idx_dev, int32_t *n_outliers_dev,
                                     void *scratch_dev, size_t scratch_bytes, void *stream) {
  return llmint8_quantize_rows_ex(X_dev, s, h, alpha, LLMINT8_SCALE_VECTORWISE, Xq_dev, ax_dev,
                                  flags_dev, idx_dev, n_outliers_dev, scratch_dev, scratch_bytes,
                                  stream);
}

llmint8_status llmint8_quantize_rows_ex(const uint16_t *X_dev, int64_t s, int64_t h, float alpha,
                                        int32_t x_scale, int8_t *Xq_dev, float *ax_dev,
                                        uint8_t *flags_dev, int32_t *idx_dev,
                                        int32_t *n_outliers_dev, void *scratch_dev,
                                        size_t scratch_bytes, void *stream) {
  if (x_scale != LLMINT8_SCALE_VECTORWISE && x_scale != LLMINT8_SCALE_TENSORWISE)
    return LLMINT8_ERR_ARG;
  if (h < 16 || h > kMaxH || (h % 16) != 0) return LLMINT8_ERR_SHAPE;
  if (s < 0 || s > (int64_t)INT32_MAX) return LLMINT8_ERR_SHAPE;
  llmint8_status rc = check_alpha(alpha);
  if (rc) return rc;
  if (!flags_dev || !idx_dev || !n_outliers_dev || !scratch_dev) return LLMINT8_ERR_NULL;
  if (s > 0 && (!X_dev || !Xq_dev || !ax_dev)) return LLMINT8_ERR_NULL;
  if ((s > 0 && (!aligned(X_dev, 16) || !aligned(Xq_dev, 16))) || !aligned(scratch_dev, 256) ||
      !aligned(idx_dev, 4) || !aligned(n_outliers_dev, 4) || (s > 0 && !aligned(ax_dev, 4)))
    return LLMINT8_ERR_ALIGN;
  if (scratch_bytes < llmint8_quantize_rows_scratch_size(h)) return LLMINT8_ERR_WORKSPACE;
  DeviceInfo *dev = nullptr;
  if ((rc = device_info(&dev))) return rc;
  uint8_t *sb = static_cast<uint8_t *>(scratch_dev);
  ActivationArgs act = {};
  act.X = X_dev;
  act.s = s;
  act.h = h;
  act.alpha = alpha;
  const size_t mw_bytes = align256(4 * (size_t)mask_words(h));
  act.block_counter = reinterpret_cast<int32_t *>(sb);
  act.act_counter = reinterpret_cast<int32_t *>(sb) + 2;
  act.mask = reinterpret_cast<uint32_t *>(sb + 256);
  act.wprefix = reinterpret_cast<int32_t *>(sb + 256 + mw_bytes);
  act.acc_mask = reinterpret_cast<uint32_t *>(sb + 256 + mw_bytes +
                                              align256(4 * ((size_t)mask_words(h) + 1)));
  act.act_reset = true;  // caller scratch: state unknown
  act.idx = idx_dev;
  act.count = n_outliers_dev;
  act.flags = flags_dev;
  act.status = reinterpret_cast<int *>(sb) + 1;
  act.Xq = Xq_dev;
  act.ax = ax_dev;
  int32_t launches = 0;
  cudaStream_t st = as_stream(stream);
  if ((rc = enqueue_activation_pass(*dev, act, st, &launches))) return rc;
  if (x_scale == LLMINT8_SCALE_TENSORWISE && s > 0) {
    if ((rc = enqueue_tensor_scale(act, reinterpret_cast<float *>(sb) + 4, st, &launches)))
      return rc;
    return last_launch();
  }
  return LLMINT8_OK;
}

llmint8_status llmint8_matmul(const uint16_t *X_dev, int64_t s, const llmint8_weight *w,
                              float alpha, uint16_t *out_dev, void *ws_dev, size_t ws_bytes,
                              void *stream) {
  return matmul_impl(X_dev, s, w, alpha, out_dev, ws_dev, ws_bytes, nullptr, as_stream(stream),
                     false);
}

llmint8_status llmint8_matmul_ex(const uint16_t *X_dev, int64_t s, const llmint8_weight *w,
                                 float alpha, uint16_t *out_dev, void *ws_dev, size_t ws_bytes,
                                 llmint8_matmul_opts *opts, void *stream) {
  return matmul_impl(X_dev, s, w, alpha, out_dev, ws_dev, ws_bytes, opts, as_stream(stream),
                     false);
}

llmint8_status llmint8_matmul_host(const uint16_t *X_host, int64_t s, const llmint8_weight *w,
                                   float alpha, uint16_t *out_host, void *ws_dev, size_t ws_bytes,
                                   void *stream) {
  return llmint8_matmul_host_ex(X_host, s, w, alpha, out_host, ws_dev, ws_bytes, nullptr, stream);
}

llmint8_status llmint8_matmul_host_ex(const uint16_t *X_host, int64_t s, const llmint8_weight *w,
                                      float alpha, uint16_t *out_host, void *ws_dev,
                                      size_t ws_bytes, llmint8_matmul_opts *opts, void *stream) {
  if (opts) opts->launches = 0;
  llmint8_status rc = validate_weight(w);
  if (rc) return rc;
  if (s < 0 || s > (int64_t)INT32_MAX) return LLMINT8_ERR_SHAPE;
  // the options are checked here too, so that a bad one enqueues no copy
  if ((rc = check_opts(opts, s, w->h))) return rc;
  if ((rc = check_alpha(alpha))) return rc;
  if (host_status_set(opts)) return LLMINT8_ERR_DEVICE_STATUS;
  if (s == 0) return LLMINT8_OK;
  if (!X_host || !out_host || !ws_dev) return LLMINT8_ERR_NULL;
  if (!aligned(ws_dev, 256)) return LLMINT8_ERR_ALIGN;
  const Layout L = layout_for(s, w->h, w->o, outlier_cap(opts, w->h));
  if (ws_bytes < L.end_host) return LLMINT8_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  uint8_t *wsb = static_cast<uint8_t *>(ws_dev);
  uint16_t *xd = reinterpret_cast<uint16_t *>(wsb + L.xstage);
  uint16_t *od = reinterpret_cast<uint16_t *>(wsb + L.ostage);
  if (cudaMemcpyAsync(xd, X_host, 2 * (size_t)s * w->h, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  if ((rc = matmul_impl(xd, s, w, alpha, od, ws_dev, ws_bytes, opts, st, true))) return rc;
  if (cudaMemcpyAsync(out_host, od, 2 * (size_t)s * w->o, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return LLMINT8_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
}

llmint8_status llmint8_read_outlier_tiles(const void *ws_dev, size_t ws_bytes, int64_t s,
                                          int64_t h, int64_t o, int32_t *n_out_host,
                                          uint16_t *XO_host, uint16_t *WO_host, void *stream) {
  return llmint8_read_outlier_tiles_ex(ws_dev, ws_bytes, s, h, o, 0, n_out_host, XO_host,
                                       WO_host, stream);
}

llmint8_status llmint8_read_outlier_tiles_ex(const void *ws_dev, size_t ws_bytes, int64_t s,
                                             int64_t h, int64_t o, int64_t max_outliers,
                                             int32_t *n_out_host, uint16_t *XO_host,
                                             uint16_t *WO_host, void *stream) {
  if (!ws_dev || !n_out_host) return LLMINT8_ERR_NULL;
  if (s < 0 || h < 0 || o < 0) return LLMINT8_ERR_SHAPE;
  if (max_outliers < 0 || max_outliers > h) return LLMINT8_ERR_ARG;
  const int64_t cap = max_outliers == 0 ? h : max_outliers;
  const Layout L = layout_for(s, h, o, cap);
  if (ws_bytes < L.end) return LLMINT8_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  const uint8_t *wsb = static_cast<const uint8_t *>(ws_dev);
  int32_t n = 0;
  if (cudaMemcpyAsync(&n, wsb + 4, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  if (n < 0 || n > h) return LLMINT8_ERR_DEVICE_STATUS;
  *n_out_host = n;
  if (n > cap || n == 0) return LLMINT8_OK;  // no outlier tiles kept
  if (!outliers_wide(n)) {  // narrow: XO [s][n], WO [n][o]
    if (XO_host &&
        cudaMemcpyAsync(XO_host, wsb + L.xo, 2 * (size_t)s * n, cudaMemcpyDeviceToHost, st) !=
            cudaSuccess)
      return LLMINT8_ERR_CUDA;
    if (WO_host &&
        cudaMemcpyAsync(WO_host, wsb + L.wo, 2 * (size_t)n * o, cudaMemcpyDeviceToHost, st) !=
            cudaSuccess)
      return LLMINT8_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA;
  }
  // wide: XO [s][ldk] and WO [o][ldk], copied to [s][n] and (transposed) [n][o]
  const int64_t ldk = wide_ld(cap);
  if (XO_host && s > 0 &&
      cudaMemcpy2DAsync(XO_host, 2 * (size_t)n, wsb + L.xo, 2 * (size_t)ldk, 2 * (size_t)n,
                        (size_t)s, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  std::vector<uint16_t> wot;
  if (WO_host) {
    wot.resize((size_t)o * n);
    if (cudaMemcpy2DAsync(wot.data(), 2 * (size_t)n, wsb + L.wo, 2 * (size_t)ldk,
                          2 * (size_t)n, (size_t)o, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return LLMINT8_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return LLMINT8_ERR_CUDA;
  if (WO_host)
    for (int64_t j = 0; j < o; ++j)
      for (int64_t t = 0; t < n; ++t) WO_host[t * o + j] = wot[(size_t)j * n + t];
  return LLMINT8_OK;
}

llmint8_status llmint8_read_device_status(void *ws_dev, size_t ws_bytes, int32_t *bits_out,
                                          void *stream) {
  if (!ws_dev) return LLMINT8_ERR_NULL;
  if (ws_bytes < 256) return LLMINT8_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  int32_t bits = 0;
  if (cudaMemcpyAsync(&bits, ws_dev, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(ws_dev, 0, 4, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  return bits ? LLMINT8_ERR_DEVICE_STATUS : LLMINT8_OK;
}

llmint8_status llmint8_wait_selftest(void *ws_dev, size_t ws_bytes, uint64_t limit_ns,
                                     void *stream) {
  if (!ws_dev) return LLMINT8_ERR_NULL;
  if (!aligned(ws_dev, 256)) return LLMINT8_ERR_ALIGN;
  if (ws_bytes < kStateBytes) return LLMINT8_ERR_WORKSPACE;
  if (limit_ns < 1000ull || limit_ns > 10000000000ull) return LLMINT8_ERR_ARG;
  DeviceInfo *dev = nullptr;
  llmint8_status rc = device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = as_stream(stream);
  int32_t *never = reinterpret_cast<int32_t *>(ws_dev) + kSelftestWord;
  if (cudaMemsetAsync(never, 0, 4, st) != cudaSuccess) return LLMINT8_ERR_CUDA;
  k_wait_selftest<<<1, 32, 0, st>>>(status_word(ws_dev), never, limit_ns);
  return last_launch();
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Allocation-free entry point: llmint8_matmul on a scratch buffer that is a
// static device array of this library, for callers that cannot allocate
// device memory or hand over a workspace at call time.
// ----------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[LLMINT8_NOALLOC_MAX_SCRATCH_BYTES];

namespace {

struct NoAllocSlot {
  void *ptr = nullptr;  // device address of g_noalloc_scratch last seen on that device
};
NoAllocSlot g_noalloc[kMaxDevices];
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device. In host code
// the array's name is only a host-side stand-in, so the address is asked of
// the runtime (with that device current) on every call; the lookup
// allocates nothing. When it differs from the one seen before (the first
// call on the device, or a new context after a device reset), the array's
// state block is cleared, asynchronously on `st`.
llmint8_status noalloc_scratch(cudaStream_t st, void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return LLMINT8_ERR_CUDA;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return LLMINT8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocSlot &slot = g_noalloc[dev];
  if (slot.ptr != p) {
    if (cudaMemsetAsync(p, 0, kStateBytes, st) != cudaSuccess) return LLMINT8_ERR_CUDA;
    slot.ptr = p;
  }
  *out = p;
  return LLMINT8_OK;
}

}  // namespace

extern "C" llmint8_status llmint8_matmul_noalloc(const uint16_t *X_dev, int64_t s,
                                                 const llmint8_weight *w, float alpha,
                                                 uint16_t *out_dev, void *stream) {
  llmint8_status rc = validate_weight(w);
  if (rc) return rc;
  if (s < 0 || s > (int64_t)INT32_MAX) return LLMINT8_ERR_SHAPE;
  if (layout_for(s, w->h, w->o, w->h).end > (size_t)LLMINT8_NOALLOC_MAX_SCRATCH_BYTES)
    return LLMINT8_ERR_TOO_LARGE;
  if (s == 0) return llmint8_matmul(X_dev, s, w, alpha, out_dev, nullptr, 0, stream);
  DeviceInfo *dev = nullptr;
  if ((rc = device_info(&dev))) return rc;
  cudaStream_t st = as_stream(stream);
  void *ws = nullptr;
  if ((rc = noalloc_scratch(st, &ws))) return rc;
  // every call clears the activation pass's accumulation state first, so a
  // call that gave up a wait (reported by llmint8_noalloc_read_device_status)
  // leaves nothing behind for the next one
  return matmul_impl(X_dev, s, w, alpha, out_dev, ws, (size_t)LLMINT8_NOALLOC_MAX_SCRATCH_BYTES,
                     nullptr, st, false, /*reset_state=*/true);
}

extern "C" int32_t llmint8_prefill_kernel(int64_t s, int64_t h, int64_t o) {
  if (s < 0 || h <= 0 || o <= 0) return LLMINT8_ERR_SHAPE;
  DeviceInfo *dev = nullptr;
  const llmint8_status rc = device_info(&dev);
  if (rc) return rc;
  if (s <= kDecodeMaxRows) return LLMINT8_PATH_DECODE;
  return pair_gemm_preferred(h, o, *dev) ? LLMINT8_PATH_PREFILL_PAIR
                                         : LLMINT8_PATH_PREFILL_SINGLE;
}

extern "C" llmint8_status llmint8_noalloc_read_device_status(int32_t *bits_out, void *stream) {
  if (bits_out) *bits_out = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return LLMINT8_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc[dev].ptr == nullptr) return LLMINT8_OK;  // no call yet on this device
  }
  cudaStream_t st = as_stream(stream);
  void *ws = nullptr;
  llmint8_status rc = noalloc_scratch(st, &ws);
  if (rc) return rc;
  int32_t bits = 0;
  if (cudaMemcpyAsync(&bits, ws, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(ws, 0, kStateBytes, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return LLMINT8_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  return bits ? LLMINT8_ERR_DEVICE_STATUS : LLMINT8_OK;
}

// C ABI of the gated delta rule decode library: host-side validation,
// dispatch on (dk, dv, dtypes) and kernel launches.  See include/gdn.h for the
// contract of every entry point.
#include <cuda.h>  // CUtensorMap and the types of cuTensorMapEncodeTiled
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <type_traits>
#include <utility>
#include <vector>

#include "gdn.h"
#include "gdn_kernels.cuh"
#include "gdn_prefill.cuh"
#include "gdn_prefill_tc.cuh"
#include "gdn_decode_tc.cuh"
#include "gdn_lowrank.cuh"
#include "gdn_lowrank_prefill.cuh"

// Launch shapes of the decode kernel, per regime: lanes per state row (lpr),
// rows per lane group (m) and warps per CTA (w); a CTA covers w * 32/lpr * m
// rows of one head.  Each is the fastest of a sweep on B200: 8 lanes per row
// keep every warp-wide 128-bit access on full 128-byte lines with a 3-level
// reduction, and 2 warps per CTA (4 for multi-token calls, whose q/k
// normalisation is spread over the warps) leave enough resident CTAs to keep
// the state stream in flight.  Single-token calls on a 16-bit pool keep the
// rows packed, two per register, so 16 lanes per row hold 8 rows each.
struct DecodeShape {
  int lpr, m, w;
};
constexpr DecodeShape kShapeF32Single = {8, 4, 2};
constexpr DecodeShape kShapeF32Multi = {8, 4, 4};
constexpr DecodeShape kShape16Single = {16, 8, 2};
constexpr DecodeShape kShape16Multi = {8, 4, 4};

constexpr DecodeShape decode_shape(int state_bytes, bool multi) {
  return state_bytes == 4 ? (multi ? kShapeF32Multi : kShapeF32Single)
                          : (multi ? kShape16Multi : kShape16Single);
}
// A lane holds whole 16-byte chunks of a row (4 fp32 or 8 16-bit values),
// so a row has at most dk * state_bytes / 16 lanes.
constexpr int decode_lpr(int dk, int state_bytes, bool multi) {
  return decode_shape(state_bytes, multi).lpr > dk * state_bytes / 16
             ? dk * state_bytes / 16
             : decode_shape(state_bytes, multi).lpr;
}
constexpr int decode_rows_per_cta(int dk, int state_bytes, bool multi) {
  return decode_shape(state_bytes, multi).w * (32 / decode_lpr(dk, state_bytes, multi)) *
         decode_shape(state_bytes, multi).m;
}

// Warps per CTA, lanes per row and rows per group of the fused kernel (one
// CTA per head).
#ifndef GDN_FUSED_LPR
#define GDN_FUSED_LPR 16
#endif
#ifndef GDN_FUSED_M
#define GDN_FUSED_M 4
#endif
#ifndef GDN_FUSED_W
#define GDN_FUSED_W 4
#endif
constexpr int fused_lpr(int dk) { return GDN_FUSED_LPR > dk / 4 ? dk / 4 : GDN_FUSED_LPR; }

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(GDN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool debug_env() {
  static int v = [] {
    const char* e = std::getenv("GDN_DEBUG");
    return (e != nullptr && e[0] == '1') ? 1 : 0;
  }();
  return v != 0;
}

// Host-side slot map check (synchronises the stream): every source slot and
// token slot in range, none repeated, no token slot equal to a source slot.
int check_slot_map(const int32_t* slot_idx, const int32_t* token_slots, int B, int T,
                   int n_slots, cudaStream_t st) {
  const size_t n_tok = token_slots != nullptr ? (size_t)B * T : 0;
  std::vector<int32_t> h(B + n_tok);
  cudaError_t e = cudaMemcpyAsync(h.data(), slot_idx, sizeof(int32_t) * (size_t)B,
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess && n_tok > 0)
    e = cudaMemcpyAsync(h.data() + B, token_slots, sizeof(int32_t) * n_tok,
                        cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "slot check copy");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "slot check sync");
  std::vector<int32_t> used;
  used.reserve(h.size());
  for (size_t i = 0; i < h.size(); ++i) {
    const int32_t s = h[i];
    if (s < -1 || (n_slots > 0 && s >= n_slots))
      return fail(GDN_ERR_SLOT_RANGE, "%s[%zu] = %d outside [-1, %d)",
                  i < (size_t)B ? "slot_idx" : "token_slots", i < (size_t)B ? i : i - B, s,
                  n_slots);
    if (s >= 0) used.push_back(s);
  }
  std::sort(used.begin(), used.end());
  for (size_t i = 1; i < used.size(); ++i)
    if (used[i] == used[i - 1])
      return fail(GDN_ERR_SLOT_DUP, "slot %d appears more than once in slot_idx/token_slots",
                  used[i]);
  return GDN_OK;
}

// How far ahead (in launches of CTAs) a decode CTA prefetches state into L2:
// this many waves of resident CTAs; 0 turns the prefetch off.
#ifndef GDN_PREFETCH_WAVES
#define GDN_PREFETCH_WAVES 1
#endif


// Sets `kernel`'s dynamic shared-memory limit to `bytes` once per (kernel,
// device), under a lock, so that threads making their first calls at once
// neither race on the bookkeeping nor skip the setting.
template <typename Kernel>
cudaError_t set_smem_limit_once(Kernel kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, bool> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  if (done[key]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  done[key] = true;
  return cudaSuccess;
}

// CTAs of `kernel` resident on the current device at once (occupancy times
// SM count), cached per (kernel, device).
template <typename Kernel>
int resident_ctas(Kernel kernel, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = per_sm * sms;
  return per_sm * sms;
}

// The divisors a decode CTA takes its (b, h, tile) and k head from: H, the
// GQA group and the tiles of `rows` state rows per head.
void set_step_divisors(gdn::StepParams& p, int rows) {
  p.div_h = gdn::make_fast_div((uint32_t)p.H);
  p.div_group = gdn::make_fast_div((uint32_t)p.group);
  p.div_tiles = gdn::make_fast_div((uint32_t)(p.dv / rows));
}

template <int DK, typename InT, typename OutT, typename StT, bool MULTI>
cudaError_t launch_decode(const gdn::StepParams& p_in, cudaStream_t st) {
  constexpr int SB = (int)sizeof(StT);
  constexpr DecodeShape SH = decode_shape(SB, MULTI);
  constexpr int LPR = decode_lpr(DK, SB, MULTI);
  constexpr bool PACKED = SB == 2 && !MULTI;
  constexpr int ROWS = decode_rows_per_cta(DK, SB, MULTI);
  gdn::StepParams p = p_in;
  set_step_divisors(p, ROWS);
  const long long grid = (long long)p.B * p.H * (p.dv / ROWS);
  // the normalised q, k of the call's tokens (single-token calls: one copy per warp)
  const size_t smem =
      (MULTI ? (size_t)p.T * (2 * DK + 1) : (size_t)SH.w * (2 * DK + 4)) * sizeof(float);
  auto kernel = gdn::decode_kernel<DK, LPR, SH.m, SH.w, InT, OutT, StT, PACKED, !MULTI>;
  p.prefetch_ahead = GDN_PREFETCH_WAVES * resident_ctas(kernel, SH.w * 32, 8 * (2 * DK + 1) * 4);
  kernel<<<(unsigned)grid, SH.w * 32, smem, st>>>(p);
  return cudaGetLastError();
}

// Calls of 2..4 tokens on an fp32 pool: the block form (one reduction for
// all tokens), on the multi-token tile, with the state tile staged in shared
// memory.
template <int DK, typename InT, typename OutT, typename StT>
cudaError_t launch_decode_block_smem(const gdn::StepParams& p_in, cudaStream_t st) {
  constexpr int SB = (int)sizeof(StT);
  constexpr int LPR = decode_lpr(DK, SB, true);
  constexpr int W = decode_shape(SB, true).w;
  constexpr int ROWS = decode_rows_per_cta(DK, SB, true);
  static_assert(W * (32 / LPR) * (LPR / 2) == ROWS, "the block form covers the multi-token tile");
  static_assert(gdn::block_smem_bytes<gdn::kBlockTokens, DK, ROWS, StT>() <= 48 * 1024,
                "the tile and the q/k of a call fit the default dynamic shared memory");
  gdn::StepParams p = p_in;
  set_step_divisors(p, ROWS);
  const long long grid = (long long)p.B * p.H * (p.dv / ROWS);
  const bool spec = p.n_accept != nullptr || p.token_slots != nullptr;
  void (*kernel)(gdn::StepParams) = nullptr;
  size_t smem = 0;
  switch (p.T) {
    case 2:
      kernel = spec ? gdn::decode_block_smem_kernel<2, DK, LPR, W, InT, OutT, StT, true>
                    : gdn::decode_block_smem_kernel<2, DK, LPR, W, InT, OutT, StT, false>;
      smem = gdn::block_smem_bytes<2, DK, ROWS, StT>();
      break;
    case 3:
      kernel = spec ? gdn::decode_block_smem_kernel<3, DK, LPR, W, InT, OutT, StT, true>
                    : gdn::decode_block_smem_kernel<3, DK, LPR, W, InT, OutT, StT, false>;
      smem = gdn::block_smem_bytes<3, DK, ROWS, StT>();
      break;
    default:
      kernel = spec ? gdn::decode_block_smem_kernel<4, DK, LPR, W, InT, OutT, StT, true>
                    : gdn::decode_block_smem_kernel<4, DK, LPR, W, InT, OutT, StT, false>;
      smem = gdn::block_smem_bytes<4, DK, ROWS, StT>();
      break;
  }
  // the tiles of several CTAs share an SM: prefer shared memory over L1
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, bool> carved;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    if (!carved[key]) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
      carved[key] = true;
    }
  }
  // the L2 prefetch reaches 3/5 of a wave ahead: measured (mtp, fp32 pool) 135.6 us at one
  // wave (740 CTAs), 131.1 at 592, 130.2 at 444, 134.2 at 296
  p.prefetch_ahead = GDN_PREFETCH_WAVES * resident_ctas(kernel, W * 32, smem) * 3 / 5;
  kernel<<<(unsigned)grid, W * 32, smem, st>>>(p);
  return cudaGetLastError();
}

// Single-token calls on a 16-bit pool at dk = 128: the tile staged in shared
// memory by one bulk copy (bytes in flight cost no registers).
template <int DK, typename InT, typename OutT, typename StT>
cudaError_t launch_decode_staged16(const gdn::StepParams& p_in, cudaStream_t st) {
  constexpr int ROWS = gdn::kStagedW * 2 * 8;
  gdn::StepParams p = p_in;
  set_step_divisors(p, ROWS);
  const long long grid = (long long)p.B * p.H * (p.dv / ROWS);
  const size_t smem = gdn::staged16_tile_bytes<DK, StT>() + (2 * DK + 4) * sizeof(float);
  auto kernel = gdn::decode_staged16_kernel<DK, InT, OutT, StT>;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, bool> carved;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    // several CTAs' tiles share an SM: prefer shared memory over L1
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    if (!carved[key]) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
      carved[key] = true;
    }
  }
  // the L2 prefetch reaches half a wave ahead: measured (serving, bf16 pool) 126.4 us at one
  // wave (1184 CTAs), 124.6 at 592, 130.2 at 296
  p.prefetch_ahead = GDN_PREFETCH_WAVES * resident_ctas(kernel, gdn::kStagedW * 32, smem) / 2;
  kernel<<<(unsigned)grid, gdn::kStagedW * 32, smem, st>>>(p);
  return cudaGetLastError();
}

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point
// (so the library links no driver library), or null.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    else
      cudaGetLastError();
  });
  return fn;
}

// The TMA map of a 16-bit state pool (bf16 or fp16) of `rows` rows of dk =
// 128 elements (256 bytes apart): boxes of 64 elements x 128 rows with the
// 128-byte swizzle.  Cached per (pool, rows, type); false if the map cannot
// be made.
bool pool16_tensor_map(const void* pool, unsigned long long rows, bool fp16, CUtensorMap* out) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, unsigned long long, bool>, CUtensorMap> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(pool, rows, fp16);
  const auto it = cache.find(key);
  if (it != cache.end()) {
    *out = it->second;
    return true;
  }
  const EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr || rows == 0 || rows >= (1ull << 31)) return false;  // row coordinates are int
  CUtensorMap m;
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
          const_cast<void*>(pool), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  if (cache.size() >= 4096) cache.clear();
  cache.emplace(key, m);
  *out = m;
  return true;
}

// Calls of 2..4 tokens on a 16-bit pool (StT) at dk = dv = 128 without
// per-token snapshots: the block form with both contractions on the tensor
// cores, one CTA per (sequence, head), the tile moved by TMA.  A pool of
// unknown size (n_slots = 0) or one the TMA map cannot describe takes the
// token loop.
template <typename InT, typename OutT, typename StT>
cudaError_t launch_decode_block_tc16(const gdn::StepParams& p_in, cudaStream_t st) {
  CUtensorMap tmap;
  if (p_in.n_slots <= 0 ||
      !pool16_tensor_map(p_in.state, (unsigned long long)p_in.n_slots * p_in.H * gdn::dtc::R,
                         std::is_same<StT, __half>::value, &tmap))
    return launch_decode<128, InT, OutT, StT, true>(p_in, st);
  gdn::StepParams p = p_in;
  set_step_divisors(p, gdn::dtc::R);
  void (*kernel)(gdn::StepParams, CUtensorMap) =
      p.T == 2   ? gdn::decode_block_tc16_kernel<2, InT, OutT, StT>
      : p.T == 3 ? gdn::decode_block_tc16_kernel<3, InT, OutT, StT>
                 : gdn::decode_block_tc16_kernel<4, InT, OutT, StT>;
  constexpr size_t smem = gdn::dtc::ALLOC;
  cudaError_t e = set_smem_limit_once(kernel, smem);
  if (e != cudaSuccess) return e;
  // four CTAs share an SM: prefer shared memory over L1
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, bool> carved;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    if (!carved[key]) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
      carved[key] = true;
    }
  }
  // one CTA per resident slot, each walking units blockIdx.x + k * gridDim.x;
  // the next unit of a CTA is one wave on, which is what it prefetches.  The
  // slots are counted from the kernel's registers and shared memory and the
  // device's limits (the occupancy query, which may assume a smaller shared
  // memory carveout than the kernel asks for, measured 2.3x slower here).
  const long long units = (long long)p.B * p.H;
  int resident = 0;
  {
    cudaFuncAttributes fa;
    int smem_sm = 0, reserved = 0, regs_sm = 0, threads_sm = 0, blocks_sm = 0, sms = 0;
    if (cudaFuncGetAttributes(&fa, kernel) == cudaSuccess &&
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
            cudaSuccess &&
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) ==
            cudaSuccess &&
        cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) ==
            cudaSuccess &&
        cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) ==
            cudaSuccess &&
        cudaDeviceGetAttribute(&blocks_sm, cudaDevAttrMaxBlocksPerMultiprocessor, dev) ==
            cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
      constexpr int warps = gdn::dtc::R / 32;
      const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;  // allocated per warp
      int per_sm = std::min(blocks_sm, threads_sm / gdn::dtc::R);
      per_sm = std::min(per_sm, regs_sm / std::max(1, regs_warp * warps));
      per_sm = std::min(per_sm, smem_sm / (int)(smem + fa.sharedSizeBytes + reserved));
      per_sm = std::min(per_sm, 512 / (int)gdn::dtc::TM_COLS);  // tensor memory columns
      resident = per_sm * sms;
    } else {
      cudaGetLastError();
    }
  }
  const long long grid = resident > 0 && resident < units ? resident : units;
  p.prefetch_ahead = (int)grid;
  kernel<<<(unsigned)grid, gdn::dtc::R, smem, st>>>(p, tmap);
  return cudaGetLastError();
}

template <int DK, typename InT, typename OutT>
cudaError_t dispatch_decode_state(const gdn::StepParams& p, gdn_dtype st_dtype, cudaStream_t st) {
  const bool multi = p.T > 1;
  // 16-bit pools, one token, dk = 128: the tile staged in shared memory
  if constexpr (DK == 128) {
    if (!multi && st_dtype == GDN_BF16)
      return launch_decode_staged16<DK, InT, OutT, __nv_bfloat16>(p, st);
    if (!multi && st_dtype == GDN_F16)
      return launch_decode_staged16<DK, InT, OutT, __half>(p, st);
  }
  // fp32 pools: calls of 2..4 tokens in block form (measured faster there;
  // with 16-bit pools it measured no faster than the token-by-token kernel
  // on the CUDA cores); 16-bit pools at dk = dv = 128: the block form on the
  // tensor cores, except for per-token snapshots
  if (multi && p.T <= gdn::kBlockTokens && st_dtype == GDN_F32)
    return launch_decode_block_smem<DK, InT, OutT, float>(p, st);
  if constexpr (DK == 128) {
    if (multi && p.T <= gdn::kBlockTokens && p.dv == gdn::dtc::R && p.token_slots == nullptr) {
      if (st_dtype == GDN_BF16) return launch_decode_block_tc16<InT, OutT, __nv_bfloat16>(p, st);
      if (st_dtype == GDN_F16) return launch_decode_block_tc16<InT, OutT, __half>(p, st);
    }
  }
  if (st_dtype == GDN_F32)
    return multi ? launch_decode<DK, InT, OutT, float, true>(p, st)
                 : launch_decode<DK, InT, OutT, float, false>(p, st);
  if (st_dtype == GDN_BF16)
    return multi ? launch_decode<DK, InT, OutT, __nv_bfloat16, true>(p, st)
                 : launch_decode<DK, InT, OutT, __nv_bfloat16, false>(p, st);
  return multi ? launch_decode<DK, InT, OutT, __half, true>(p, st)
               : launch_decode<DK, InT, OutT, __half, false>(p, st);
}

template <int DK, typename InT>
cudaError_t dispatch_decode_out(const gdn::StepParams& p, gdn_dtype out_dtype, gdn_dtype st_dtype,
                                cudaStream_t st) {
  if (out_dtype == GDN_F32) return dispatch_decode_state<DK, InT, float>(p, st_dtype, st);
  return dispatch_decode_state<DK, InT, __nv_bfloat16>(p, st_dtype, st);
}

template <int DK>
cudaError_t dispatch_decode_in(const gdn::StepParams& p, gdn_dtype in_dtype, gdn_dtype out_dtype,
                               gdn_dtype st_dtype, cudaStream_t st) {
  if (in_dtype == GDN_F32) return dispatch_decode_out<DK, float>(p, out_dtype, st_dtype, st);
  return dispatch_decode_out<DK, __nv_bfloat16>(p, out_dtype, st_dtype, st);
}

template <int DK, int DV, typename WT, typename OutT>
cudaError_t launch_fused(const gdn::FusedParams& p_in, cudaStream_t st) {
  constexpr int LPR = fused_lpr(DK);
  gdn::FusedParams p = p_in;
  p.div_h = gdn::make_fast_div((uint32_t)p.H);
  p.div_group = gdn::make_fast_div((uint32_t)p.group);
  auto kernel = gdn::fused_kernel<DK, DV, LPR, GDN_FUSED_M, GDN_FUSED_W, WT, OutT>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)p.B * p.H), 1, 1);
  cfg.blockDim = dim3(GDN_FUSED_W * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.group;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <int DK, int DV, typename WT>
cudaError_t dispatch_fused_out(const gdn::FusedParams& p, gdn_dtype out_dtype, cudaStream_t st) {
  if (out_dtype == GDN_F32) return launch_fused<DK, DV, WT, float>(p, st);
  return launch_fused<DK, DV, WT, __nv_bfloat16>(p, st);
}

template <int DK, int DV>
cudaError_t dispatch_fused_w(const gdn::FusedParams& p, gdn_dtype w_dtype, gdn_dtype out_dtype,
                             cudaStream_t st) {
  if (w_dtype == GDN_F32) return dispatch_fused_out<DK, DV, float>(p, out_dtype, st);
  return dispatch_fused_out<DK, DV, __nv_bfloat16>(p, out_dtype, st);
}

bool valid_dtype(gdn_dtype d) { return d == GDN_F32 || d == GDN_BF16; }

// chunk slots of a prefill call: sum_n ceil(L_n / C) <= total / C + N
long long prefill_chunk_slots(int N, int total_tokens) {
  return (long long)total_tokens / gdn::kChunk + N + 1;
}

template <int DK, int DV>
size_t chunk_ws_floats() {
  return (size_t)gdn::ChunkWs<DK, DV>::SIZE;
}

// bf16 inputs with dk = dv = 128 run phase B on tcgen05: phase A leaves
// only T per (chunk, head)
bool prefill_tcb(int dk, int dv, gdn_dtype in_dtype) {
  return dk == 128 && dv == 128 && in_dtype == GDN_BF16;
}

size_t prefill_ws_floats(int dk, int dv, gdn_dtype in_dtype) {
  if (prefill_tcb(dk, dv, in_dtype)) return (size_t)gdn::kTcbWsFloats;
  if (dk == 128 && dv == 128) return chunk_ws_floats<128, 128>();
  if (dk == 128 && dv == 64) return chunk_ws_floats<128, 64>();
  if (dk == 64 && dv == 128) return chunk_ws_floats<64, 128>();
  return chunk_ws_floats<64, 64>();
}

template <int DK, int DV, typename InT, typename OutT>
cudaError_t launch_prefill(const gdn::PrefillParams& p, long long slots, cudaStream_t st) {
  constexpr bool TCB = DK == 128 && DV == 128 && std::is_same<InT, __nv_bfloat16>::value;
  auto ka = gdn::prefill_chunk_kernel<DK, DV, InT>;
  void (*kb)(gdn::PrefillParams) = nullptr;
  size_t sb = 0;
  if constexpr (TCB) {
    kb = gdn::prefill_state_tc_kernel<OutT>;
    sb = gdn::tcb::BYTES;
  } else {
    kb = gdn::prefill_state_kernel<DK, DV, OutT>;
    sb = gdn::PhaseBSmem<DK, DV>::BYTES;
  }
  const size_t sa = sizeof(float) * gdn::PhaseASmem<DK, DV, TCB>::FLOATS;
  cudaError_t e = set_smem_limit_once(ka, sa);
  if (e != cudaSuccess) return e;
  e = set_smem_limit_once(kb, sb);
  if (e != cudaSuccess) return e;
  ka<<<dim3((unsigned)slots, (unsigned)p.H, 1), 256, sa, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kb<<<(unsigned)((long long)p.N * p.H), 256, sb, st>>>(p);
  return cudaGetLastError();
}

template <int DK, int DV, int R, typename InT, typename OutT>
cudaError_t launch_lowrank(const gdn::LowrankParams& p, cudaStream_t st) {
  constexpr int W = gdn::lowrank_warps<DK, DV, R>();
  constexpr size_t smem = gdn::lowrank_smem_bytes<DK, DV, R>();
  auto kern = gdn::lowrank_kernel<DK, DV, R, InT, OutT>;
  cudaError_t e = set_smem_limit_once(kern, smem);
  if (e != cudaSuccess) return e;
  constexpr int UPC = W / gdn::lowrank_split<R>();  // (sequence, head) units per CTA
  const unsigned grid = (unsigned)(((long long)p.B * p.H + UPC - 1) / UPC);
  gdn::LowrankParams pp = p;
  pp.div_h = gdn::make_fast_div((uint32_t)p.H);
  pp.div_group = gdn::make_fast_div((uint32_t)p.group);
  pp.prefetch_ahead = GDN_PREFETCH_WAVES * UPC * resident_ctas(kern, W * 32, smem);
  kern<<<grid, W * 32, smem, st>>>(pp);
  return cudaGetLastError();
}

template <int DK, int DV, int R>
cudaError_t dispatch_lowrank_types(const gdn::LowrankParams& p, gdn_dtype in_dtype,
                                   gdn_dtype out_dtype, cudaStream_t st) {
  if (in_dtype == GDN_F32)
    return out_dtype == GDN_F32 ? launch_lowrank<DK, DV, R, float, float>(p, st)
                                : launch_lowrank<DK, DV, R, float, __nv_bfloat16>(p, st);
  return out_dtype == GDN_F32 ? launch_lowrank<DK, DV, R, __nv_bfloat16, float>(p, st)
                              : launch_lowrank<DK, DV, R, __nv_bfloat16, __nv_bfloat16>(p, st);
}

template <int DK, int DV>
cudaError_t dispatch_lowrank(const gdn::LowrankParams& p, int R, gdn_dtype in_dtype,
                             gdn_dtype out_dtype, cudaStream_t st) {
  switch (R) {
    case 8: return dispatch_lowrank_types<DK, DV, 8>(p, in_dtype, out_dtype, st);
    case 16: return dispatch_lowrank_types<DK, DV, 16>(p, in_dtype, out_dtype, st);
    case 32: return dispatch_lowrank_types<DK, DV, 32>(p, in_dtype, out_dtype, st);
    default: return dispatch_lowrank_types<DK, DV, 64>(p, in_dtype, out_dtype, st);
  }
}

template <int DK, int DV, typename InT, typename OutT>
cudaError_t launch_lowrank_prefill(const gdn::LowrankPrefillParams& p, cudaStream_t st) {
  auto kern = gdn::lowrank_prefill_kernel<DK, DV, InT, OutT>;
  const size_t smem = sizeof(float) * gdn::LrpSmem<DK, DV>::FLOATS;
  cudaError_t e = set_smem_limit_once(kern, smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)((long long)p.N * p.H), 256, smem, st>>>(p);
  return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t dispatch_lowrank_prefill(const gdn::LowrankPrefillParams& p, gdn_dtype in_dtype,
                                     gdn_dtype out_dtype, cudaStream_t st) {
  if (in_dtype == GDN_F32)
    return out_dtype == GDN_F32 ? launch_lowrank_prefill<DK, DV, float, float>(p, st)
                                : launch_lowrank_prefill<DK, DV, float, __nv_bfloat16>(p, st);
  return out_dtype == GDN_F32 ? launch_lowrank_prefill<DK, DV, __nv_bfloat16, float>(p, st)
                              : launch_lowrank_prefill<DK, DV, __nv_bfloat16, __nv_bfloat16>(p, st);
}

template <int DK, int DV>
cudaError_t dispatch_prefill(const gdn::PrefillParams& p, long long slots, gdn_dtype in_dtype,
                             gdn_dtype out_dtype, cudaStream_t st) {
  if (in_dtype == GDN_F32)
    return out_dtype == GDN_F32 ? launch_prefill<DK, DV, float, float>(p, slots, st)
                                : launch_prefill<DK, DV, float, __nv_bfloat16>(p, slots, st);
  return out_dtype == GDN_F32 ? launch_prefill<DK, DV, __nv_bfloat16, float>(p, slots, st)
                              : launch_prefill<DK, DV, __nv_bfloat16, __nv_bfloat16>(p, slots, st);
}
bool valid_state_dtype(gdn_dtype d) { return d == GDN_F32 || d == GDN_BF16 || d == GDN_F16; }

// ---------------------------------------------------------------------------
// Scratch for gdn_chunk_prefill_noalloc: one fixed array in device memory,
// part of the library image, so it exists on every GPU that loads the
// library, from the moment the library is loaded until the process exits.

constexpr size_t kNoAllocScratchBytes = size_t{64} << 20;  // 64 MiB

}  // namespace

static __device__ __align__(256) unsigned char g_prefill_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};  // device address of g_prefill_scratch, per device

// The device address of the scratch array on the current device.  Host code
// only sees a host-side stand-in for the array's name, so the address is
// asked from the runtime once per device (with that device current) and
// kept.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(GDN_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prefill_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the prefill scratch");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GDN_OK;
}

// Checks of a prefill call's sizes and enums, shared by both prefill entry
// points (a call with N == 0 that passes them is a no-op).
int check_prefill_sizes(const gdn_prefill_args* a, const char* fn) {
  if (a == nullptr) return fail(GDN_ERR_ARG, "%s: null args", fn);
  if (a->N < 0 || a->total_tokens < 0)
    return fail(GDN_ERR_ARG, "N = %d and total_tokens = %d must be >= 0", a->N, a->total_tokens);
  if (a->H < 1 || a->Hk < 1 || a->H % a->Hk != 0)
    return fail(GDN_ERR_ARG, "H = %d must be a positive multiple of Hk = %d", a->H, a->Hk);
  if ((long long)a->N * a->H > 0x7fffffffLL)
    return fail(GDN_ERR_UNSUPPORTED, "N * H = %lld too large for one launch",
                (long long)a->N * a->H);
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype))
    return fail(GDN_ERR_ARG, "bad dtype enum (in %d, out %d)", (int)a->in_dtype, (int)a->out_dtype);
  if ((a->dk != 64 && a->dk != 128) || (a->dv != 64 && a->dv != 128))
    return fail(GDN_ERR_UNSUPPORTED, "dk = %d, dv = %d not in {64, 128}", a->dk, a->dv);
  if (a->n_slots <= 0) return fail(GDN_ERR_ARG, "n_slots = %d must be > 0", a->n_slots);
  return GDN_OK;
}

// Pointer and alignment checks of a prefill call with N > 0; the workspace
// is checked only when the caller supplies it.
int check_prefill_pointers(const gdn_prefill_args* a, bool with_workspace) {
  if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->state || !a->slot_idx ||
      !a->cu_seqlens || !a->out || (with_workspace && !a->workspace))
    return fail(GDN_ERR_ARG, "null pointer");
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->state, 16) ||
      !aligned(a->out, 16) || (with_workspace && !aligned(a->workspace, 16)))
    return fail(GDN_ERR_ARG, "q, k, v, state, out and workspace must be 16-byte aligned");
  if (!aligned(a->g, 4) || !aligned(a->beta, 4) || !aligned(a->slot_idx, 4) ||
      !aligned(a->cu_seqlens, 4))
    return fail(GDN_ERR_ARG, "g, beta, slot_idx and cu_seqlens must be 4-byte aligned");
  const long long slots = prefill_chunk_slots(a->N, a->total_tokens);
  if (slots > 0x7fffffffLL || a->H > 65535)
    return fail(GDN_ERR_UNSUPPORTED, "too many chunks for one launch");
  return GDN_OK;
}

// Launches a checked prefill call on `workspace` (large enough).
int run_prefill(const gdn_prefill_args* a, void* workspace) {
  const long long slots = prefill_chunk_slots(a->N, a->total_tokens);
  gdn::PrefillParams p;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.g = a->g;
  p.beta = a->beta;
  p.state = a->state;
  p.slot_idx = a->slot_idx;
  p.cu_seqlens = a->cu_seqlens;
  p.out = a->out;
  p.ws = reinterpret_cast<float*>(workspace);
  p.N = a->N;
  p.total = a->total_tokens;
  p.Hk = a->Hk;
  p.H = a->H;
  p.dv = a->dv;
  p.n_slots = a->n_slots;
  p.group = a->H / a->Hk;
  p.scale = a->scale > 0.0f ? a->scale : 1.0f / std::sqrt((float)a->dk);
  p.l2_eps = a->l2_eps >= 0.0f ? a->l2_eps : 1e-6f;
  p.l2norm = a->qk_l2norm ? 1 : 0;
  p.initial_state = a->initial_state ? 1 : 0;
  p.dev_status = a->dev_status;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(a->stream);
  cudaError_t e;
  if (a->dk == 128 && a->dv == 128) e = dispatch_prefill<128, 128>(p, slots, a->in_dtype, a->out_dtype, st);
  else if (a->dk == 128) e = dispatch_prefill<128, 64>(p, slots, a->in_dtype, a->out_dtype, st);
  else if (a->dv == 128) e = dispatch_prefill<64, 128>(p, slots, a->in_dtype, a->out_dtype, st);
  else e = dispatch_prefill<64, 64>(p, slots, a->in_dtype, a->out_dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  return GDN_OK;
}

}  // namespace

extern "C" {

int gdn_version(void) { return 10000; }

const char* gdn_last_error_string(void) { return g_last_error.c_str(); }

int gdn_get_error(const int* dev_status, int* host_status) {
  if (dev_status == nullptr || host_status == nullptr)
    return fail(GDN_ERR_ARG, "gdn_get_error: null pointer");
  cudaError_t e = cudaMemcpy(host_status, dev_status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "gdn_get_error copy");
  if (*host_status & GDN_STATUS_SLOT_RANGE)
    return fail(GDN_ERR_SLOT_RANGE, "a kernel saw a slot outside [-1, n_slots)");
  if (*host_status & GDN_STATUS_ACCEPT_RANGE)
    return fail(GDN_ERR_ACCEPT_RANGE, "a kernel saw an n_accept entry outside [0, T]");
  if (*host_status & GDN_STATUS_SEQ_RANGE)
    return fail(GDN_ERR_SEQ_RANGE, "a prefill sequence's tokens lie outside [0, total_tokens]");
  if (*host_status & GDN_STATUS_TIMEOUT)
    return fail(GDN_ERR_TIMEOUT, "a kernel gave up waiting for its own copy");
  return GDN_OK;
}

int gdn_decode_step_ex(const gdn_step_args* a) {
  if (a == nullptr) return fail(GDN_ERR_ARG, "gdn_decode_step_ex: null args");
  if (a->B < 0) return fail(GDN_ERR_ARG, "B = %d must be >= 0", a->B);
  if (a->H < 1 || a->Hk < 1) return fail(GDN_ERR_ARG, "H = %d and Hk = %d must be >= 1", a->H, a->Hk);
  if (a->H % a->Hk != 0) return fail(GDN_ERR_ARG, "H = %d is not a multiple of Hk = %d", a->H, a->Hk);
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype) || !valid_state_dtype(a->state_dtype))
    return fail(GDN_ERR_ARG, "bad dtype enum (in %d, out %d, state %d)", (int)a->in_dtype,
                (int)a->out_dtype, (int)a->state_dtype);
  if (a->dk != 64 && a->dk != 128) return fail(GDN_ERR_UNSUPPORTED, "dk = %d not in {64, 128}", a->dk);
  if (a->dv != 64 && a->dv != 128) return fail(GDN_ERR_UNSUPPORTED, "dv = %d not in {64, 128}", a->dv);
  if (a->T < 1 || a->T > 8) return fail(GDN_ERR_UNSUPPORTED, "T = %d not in [1, 8]", a->T);
  if (a->B == 0) return GDN_OK;
  if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->state || !a->slot_idx || !a->out)
    return fail(GDN_ERR_ARG, "null tensor pointer");
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->state, 16) ||
      !aligned(a->out, 16))
    return fail(GDN_ERR_ARG, "q, k, v, state and out must be 16-byte aligned");
  if (!aligned(a->g, 4) || !aligned(a->beta, 4) || !aligned(a->slot_idx, 4) ||
      !aligned(a->n_accept, 4) || !aligned(a->token_slots, 4))
    return fail(GDN_ERR_ARG, "g, beta, slot_idx, n_accept and token_slots must be 4-byte aligned");
  if (a->n_accept != nullptr && a->token_slots != nullptr)
    return fail(GDN_ERR_ARG, "n_accept and token_slots are exclusive");
  const int rows = decode_rows_per_cta(a->dk, a->state_dtype == GDN_F32 ? 4 : 2, a->T > 1);
  if (a->dv % rows != 0)
    return fail(GDN_ERR_UNSUPPORTED, "dv = %d not a multiple of the CTA tile (%d rows)", a->dv, rows);
  const long long grid = (long long)a->B * a->H * (a->dv / rows);
  if (grid > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "B*H too large for one launch");

  cudaStream_t st = reinterpret_cast<cudaStream_t>(a->stream);
  if (a->check_slots || debug_env()) {
    int rc = check_slot_map(a->slot_idx, a->token_slots, a->B, a->T, a->n_slots, st);
    if (rc != GDN_OK) return rc;
  }

  gdn::StepParams p;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.g = a->g;
  p.beta = a->beta;
  p.state = a->state;
  p.slot_idx = a->slot_idx;
  p.out = a->out;
  p.B = a->B;
  p.Hk = a->Hk;
  p.H = a->H;
  p.dv = a->dv;
  p.T = a->T;
  p.n_slots = a->n_slots;
  p.group = a->H / a->Hk;
  p.scale = a->scale > 0.0f ? a->scale : 1.0f / std::sqrt((float)a->dk);
  p.l2_eps = a->l2_eps >= 0.0f ? a->l2_eps : 1e-6f;
  p.l2norm = a->qk_l2norm ? 1 : 0;
  p.dev_status = a->dev_status;
  p.n_accept = a->n_accept;
  p.token_slots = a->token_slots;
  p.prefetch_ahead = 0;  // set per kernel at launch

  cudaError_t e =
      (a->dk == 128) ? dispatch_decode_in<128>(p, a->in_dtype, a->out_dtype, a->state_dtype, st)
                     : dispatch_decode_in<64>(p, a->in_dtype, a->out_dtype, a->state_dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  return GDN_OK;
}

size_t gdn_prefill_workspace_size_ex(int N, int total_tokens, int H, int dk, int dv,
                                     gdn_dtype in_dtype) {
  if (N < 0 || total_tokens < 0 || H < 1 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128) ||
      !valid_dtype(in_dtype))
    return 0;
  return sizeof(float) * (size_t)prefill_chunk_slots(N, total_tokens) * (size_t)H *
         prefill_ws_floats(dk, dv, in_dtype);
}

size_t gdn_prefill_workspace_size(int N, int total_tokens, int H, int dk, int dv) {
  const size_t a = gdn_prefill_workspace_size_ex(N, total_tokens, H, dk, dv, GDN_F32);
  const size_t b = gdn_prefill_workspace_size_ex(N, total_tokens, H, dk, dv, GDN_BF16);
  return a > b ? a : b;
}

int gdn_chunk_prefill(const gdn_prefill_args* a) {
  int rc = check_prefill_sizes(a, "gdn_chunk_prefill");
  if (rc != GDN_OK || a->N == 0) return rc;
  rc = check_prefill_pointers(a, /*with_workspace=*/true);
  if (rc != GDN_OK) return rc;
  const size_t need =
      gdn_prefill_workspace_size_ex(a->N, a->total_tokens, a->H, a->dk, a->dv, a->in_dtype);
  if (a->workspace_bytes < need)
    return fail(GDN_ERR_ARG, "workspace of %zu bytes, %zu needed", a->workspace_bytes, need);
  return run_prefill(a, a->workspace);
}

int gdn_chunk_prefill_noalloc(const gdn_prefill_args* a) {
  // the same argument checks as gdn_chunk_prefill, in the same order, before
  // anything that concerns the built-in scratch
  int rc = check_prefill_sizes(a, "gdn_chunk_prefill_noalloc");
  if (rc != GDN_OK || a->N == 0) return rc;
  rc = check_prefill_pointers(a, /*with_workspace=*/false);
  if (rc != GDN_OK) return rc;
  const size_t need =
      gdn_prefill_workspace_size_ex(a->N, a->total_tokens, a->H, a->dk, a->dv, a->in_dtype);
  if (need > kNoAllocScratchBytes)
    return fail(GDN_ERR_UNSUPPORTED,
                "this prefill needs %zu bytes of scratch; the built-in scratch holds %zu bytes "
                "(use gdn_chunk_prefill with a workspace, or split the call)",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != GDN_OK) return rc;
  return run_prefill(a, scratch);
}

int gdn_lowrank_decode_step(const gdn_lowrank_args* a) {
  if (a == nullptr) return fail(GDN_ERR_ARG, "gdn_lowrank_decode_step: null args");
  if (a->B < 0) return fail(GDN_ERR_ARG, "B = %d must be >= 0", a->B);
  if (a->H < 1 || a->Hk < 1 || a->H % a->Hk != 0)
    return fail(GDN_ERR_ARG, "H = %d must be a positive multiple of Hk = %d", a->H, a->Hk);
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype))
    return fail(GDN_ERR_ARG, "bad dtype enum (in %d, out %d)", (int)a->in_dtype, (int)a->out_dtype);
  if ((a->dk != 64 && a->dk != 128) || (a->dv != 64 && a->dv != 128))
    return fail(GDN_ERR_UNSUPPORTED, "dk = %d, dv = %d not in {64, 128}", a->dk, a->dv);
  if (a->R != 8 && a->R != 16 && a->R != 32 && a->R != 64)
    return fail(GDN_ERR_UNSUPPORTED, "R = %d not in {8, 16, 32, 64}", a->R);
  if (a->T < 1 || a->T > 8) return fail(GDN_ERR_UNSUPPORTED, "T = %d not in [1, 8]", a->T);
  if (a->n_slots <= 0) return fail(GDN_ERR_ARG, "n_slots = %d must be > 0", a->n_slots);
  if (a->B == 0) return GDN_OK;
  if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->win_k || !a->win_u || !a->win_c ||
      !a->win_count || !a->slot_idx || !a->out)
    return fail(GDN_ERR_ARG, "null pointer");
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->win_k, 16) ||
      !aligned(a->win_u, 16) || !aligned(a->out, 16))
    return fail(GDN_ERR_ARG, "q, k, v, win_k, win_u and out must be 16-byte aligned");
  if (!aligned(a->g, 4) || !aligned(a->beta, 4) || !aligned(a->win_c, 4) ||
      !aligned(a->win_count, 4) || !aligned(a->slot_idx, 4))
    return fail(GDN_ERR_ARG, "g, beta, win_c, win_count and slot_idx must be 4-byte aligned");
  if ((long long)a->B * a->H > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "B*H too large");
  gdn::LowrankParams p;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.g = a->g;
  p.beta = a->beta;
  p.win_k = a->win_k;
  p.win_u = a->win_u;
  p.win_c = a->win_c;
  p.win_count = a->win_count;
  p.slot_idx = a->slot_idx;
  p.out = a->out;
  p.B = a->B;
  p.T = a->T;
  p.Hk = a->Hk;
  p.H = a->H;
  p.n_slots = a->n_slots;
  p.group = a->H / a->Hk;
  p.scale = a->scale > 0.0f ? a->scale : 1.0f / std::sqrt((float)a->dk);
  p.l2_eps = a->l2_eps >= 0.0f ? a->l2_eps : 1e-6f;
  p.l2norm = a->qk_l2norm ? 1 : 0;
  p.dev_status = a->dev_status;
  p.prefetch_ahead = 0;  // set at launch
  cudaStream_t st = reinterpret_cast<cudaStream_t>(a->stream);
  cudaError_t e;
  if (a->dk == 128 && a->dv == 128) e = dispatch_lowrank<128, 128>(p, a->R, a->in_dtype, a->out_dtype, st);
  else if (a->dk == 128) e = dispatch_lowrank<128, 64>(p, a->R, a->in_dtype, a->out_dtype, st);
  else if (a->dv == 128) e = dispatch_lowrank<64, 128>(p, a->R, a->in_dtype, a->out_dtype, st);
  else e = dispatch_lowrank<64, 64>(p, a->R, a->in_dtype, a->out_dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "low-rank kernel launch");
  return GDN_OK;
}

int gdn_lowrank_prefill(const gdn_lowrank_prefill_args* a) {
  if (a == nullptr) return fail(GDN_ERR_ARG, "gdn_lowrank_prefill: null args");
  if (a->N < 0 || a->total_tokens < 0)
    return fail(GDN_ERR_ARG, "N = %d and total_tokens = %d must be >= 0", a->N, a->total_tokens);
  if (a->H < 1 || a->Hk < 1 || a->H % a->Hk != 0)
    return fail(GDN_ERR_ARG, "H = %d must be a positive multiple of Hk = %d", a->H, a->Hk);
  if ((long long)a->N * a->H > 0x7fffffffLL)
    return fail(GDN_ERR_UNSUPPORTED, "N * H = %lld too large for one launch",
                (long long)a->N * a->H);
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype))
    return fail(GDN_ERR_ARG, "bad dtype enum (in %d, out %d)", (int)a->in_dtype, (int)a->out_dtype);
  if ((a->dk != 64 && a->dk != 128) || (a->dv != 64 && a->dv != 128))
    return fail(GDN_ERR_UNSUPPORTED, "dk = %d, dv = %d not in {64, 128}", a->dk, a->dv);
  if (a->R != 8 && a->R != 16 && a->R != 32 && a->R != 64)
    return fail(GDN_ERR_UNSUPPORTED, "R = %d not in {8, 16, 32, 64}", a->R);
  if (a->n_slots <= 0) return fail(GDN_ERR_ARG, "n_slots = %d must be > 0", a->n_slots);
  if (a->N == 0) return GDN_OK;
  if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->win_k || !a->win_u || !a->win_c ||
      !a->win_count || !a->slot_idx || !a->cu_seqlens || !a->out)
    return fail(GDN_ERR_ARG, "null pointer");
  if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->win_k, 16) ||
      !aligned(a->win_u, 16) || !aligned(a->out, 16))
    return fail(GDN_ERR_ARG, "q, k, v, win_k, win_u and out must be 16-byte aligned");
  if (!aligned(a->g, 4) || !aligned(a->beta, 4) || !aligned(a->win_c, 4) ||
      !aligned(a->win_count, 4) || !aligned(a->slot_idx, 4) || !aligned(a->cu_seqlens, 4))
    return fail(GDN_ERR_ARG, "g, beta, win_c, win_count, slot_idx and cu_seqlens must be "
                             "4-byte aligned");
  gdn::LowrankPrefillParams p;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.g = a->g;
  p.beta = a->beta;
  p.win_k = a->win_k;
  p.win_u = a->win_u;
  p.win_c = a->win_c;
  p.win_count = a->win_count;
  p.slot_idx = a->slot_idx;
  p.cu_seqlens = a->cu_seqlens;
  p.out = a->out;
  p.N = a->N;
  p.total = a->total_tokens;
  p.Hk = a->Hk;
  p.H = a->H;
  p.R = a->R;
  p.n_slots = a->n_slots;
  p.group = a->H / a->Hk;
  p.scale = a->scale > 0.0f ? a->scale : 1.0f / std::sqrt((float)a->dk);
  p.l2_eps = a->l2_eps >= 0.0f ? a->l2_eps : 1e-6f;
  p.l2norm = a->qk_l2norm ? 1 : 0;
  p.initial_window = a->initial_window ? 1 : 0;
  p.dev_status = a->dev_status;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(a->stream);
  cudaError_t e;
  if (a->dk == 128 && a->dv == 128) e = dispatch_lowrank_prefill<128, 128>(p, a->in_dtype, a->out_dtype, st);
  else if (a->dk == 128) e = dispatch_lowrank_prefill<128, 64>(p, a->in_dtype, a->out_dtype, st);
  else if (a->dv == 128) e = dispatch_lowrank_prefill<64, 128>(p, a->in_dtype, a->out_dtype, st);
  else e = dispatch_lowrank_prefill<64, 64>(p, a->in_dtype, a->out_dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "low-rank prefill kernel launch");
  return GDN_OK;
}

int gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, float* state, const int32_t* slot_idx, float* out, int B,
                    int H, int dk, int dv, int T, void* stream) {
  gdn_step_args a;
  std::memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.g = g;
  a.beta = beta;
  a.state = state;
  a.slot_idx = slot_idx;
  a.out = out;
  a.B = B;
  a.Hk = H;
  a.H = H;
  a.dk = dk;
  a.dv = dv;
  a.T = T;
  a.n_slots = 0;
  a.in_dtype = GDN_BF16;
  a.out_dtype = GDN_F32;
  a.state_dtype = GDN_F32;
  a.scale = 0.0f;
  a.qk_l2norm = 1;
  a.l2_eps = 1e-6f;
  a.dev_status = nullptr;
  a.check_slots = 0;
  a.n_accept = nullptr;
  a.token_slots = nullptr;
  a.stream = stream;
  return gdn_decode_step_ex(&a);
}

int gdn_fused_decode_step(const void* mixed_x, void* conv_state, const void* conv_w,
                          gdn_dtype conv_w_dtype, const void* a, const void* b,
                          const float* A_log, const float* dt_bias, const void* z,
                          const float* norm_w, float norm_eps, float* state,
                          const int32_t* slot_idx, void* out, int B, int Hk, int H, int dk,
                          int dv, int n_slots, gdn_dtype out_dtype, int* dev_status,
                          void* stream) {
  if (B < 0) return fail(GDN_ERR_ARG, "B = %d must be >= 0", B);
  if (H < 1 || Hk < 1) return fail(GDN_ERR_ARG, "H = %d and Hk = %d must be >= 1", H, Hk);
  if (H % Hk != 0) return fail(GDN_ERR_ARG, "H = %d is not a multiple of Hk = %d", H, Hk);
  if (H / Hk > 8) return fail(GDN_ERR_UNSUPPORTED, "H / Hk = %d > 8 (cluster size)", H / Hk);
  if (!valid_dtype(conv_w_dtype) || !valid_dtype(out_dtype))
    return fail(GDN_ERR_ARG, "bad dtype enum");
  if (dk != 64 && dk != 128) return fail(GDN_ERR_UNSUPPORTED, "dk = %d not in {64, 128}", dk);
  if (dv != 64 && dv != 128) return fail(GDN_ERR_UNSUPPORTED, "dv = %d not in {64, 128}", dv);
  if (n_slots <= 0) return fail(GDN_ERR_ARG, "n_slots = %d must be > 0", n_slots);
  if (!(norm_eps >= 0.0f)) return fail(GDN_ERR_ARG, "norm_eps must be >= 0");
  if (B == 0) return GDN_OK;
  if (!mixed_x || !conv_state || !conv_w || !a || !b || !A_log || !dt_bias || !z || !norm_w ||
      !state || !slot_idx || !out)
    return fail(GDN_ERR_ARG, "null tensor pointer");
  if (!aligned(mixed_x, 16) || !aligned(z, 16) || !aligned(out, 16) || !aligned(state, 16))
    return fail(GDN_ERR_ARG, "mixed_x, z, out and state must be 16-byte aligned");
  if (!aligned(conv_w, conv_w_dtype == GDN_F32 ? 16 : 8))
    return fail(GDN_ERR_ARG, "conv_w misaligned");
  if (!aligned(conv_state, 2) || !aligned(a, 2) || !aligned(b, 2) || !aligned(A_log, 4) ||
      !aligned(dt_bias, 4) || !aligned(norm_w, 4) || !aligned(slot_idx, 4))
    return fail(GDN_ERR_ARG, "misaligned small tensor");
  if ((long long)B * H > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "B*H too large");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (debug_env()) {
    int rc = check_slot_map(slot_idx, nullptr, B, 1, n_slots, st);
    if (rc != GDN_OK) return rc;
  }

  gdn::FusedParams p;
  p.mixed_x = reinterpret_cast<const __nv_bfloat16*>(mixed_x);
  p.conv_state = reinterpret_cast<__nv_bfloat16*>(conv_state);
  p.conv_w = conv_w;
  p.a = reinterpret_cast<const __nv_bfloat16*>(a);
  p.b = reinterpret_cast<const __nv_bfloat16*>(b);
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.z = reinterpret_cast<const __nv_bfloat16*>(z);
  p.norm_w = norm_w;
  p.state = state;
  p.slot_idx = slot_idx;
  p.out = out;
  p.B = B;
  p.Hk = Hk;
  p.H = H;
  p.dv = dv;
  p.n_slots = n_slots;
  p.group = H / Hk;
  p.C = 2 * Hk * dk + H * dv;
  p.norm_eps = norm_eps;
  p.scale = 1.0f / std::sqrt((float)dk);
  p.l2_eps = 1e-6f;
  p.dev_status = dev_status;

  cudaError_t e;
  if (dk == 128 && dv == 128) e = dispatch_fused_w<128, 128>(p, conv_w_dtype, out_dtype, st);
  else if (dk == 128) e = dispatch_fused_w<128, 64>(p, conv_w_dtype, out_dtype, st);
  else if (dv == 128) e = dispatch_fused_w<64, 128>(p, conv_w_dtype, out_dtype, st);
  else e = dispatch_fused_w<64, 64>(p, conv_w_dtype, out_dtype, st);
  if (e != cudaSuccess) return cuda_fail(e, "fused kernel launch");
  return GDN_OK;
}

}  // extern "C"

// api.cu -- the C ABI declared in include/attn.h: argument checks, TMA tensor
// maps, kernel launches and the device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "bwd_kernels.cuh"
#include "bwd_pair_kernel.cuh"
#include "fwd_kernel.cuh"
#include "fwd_pair_kernel.cuh"

namespace attn {

// One error word per device: kernels record a timed-out wait here.
__device__ uint32_t g_device_error;

namespace {

constexpr int kMaxDevices = 64;

// caller-owned events recorded around one kernel (attn_set_timing_events)
struct TimingEvents {
  cudaEvent_t start = nullptr, stop = nullptr;
};
thread_local TimingEvents t_events[2];

void record_start(int kernel, cudaStream_t s) {
  if (t_events[kernel].start) cudaEventRecord(t_events[kernel].start, s);
}
void record_stop(int kernel, cudaStream_t s) {
  if (t_events[kernel].stop) cudaEventRecord(t_events[kernel].stop, s);
}

struct DeviceState {
  std::once_flag once;
  cudaError_t init_status = cudaSuccess;
  uint32_t* err = nullptr;
  int sm_major = 0, sm_minor = 0;
  int smem_optin = 0;
  int num_sms = 0;
};
DeviceState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

uint64_t wait_timeout_ns() {
  static uint64_t v = [] {
    const char* e = std::getenv("ATTN_WAIT_TIMEOUT_MS");
    long ms = e ? std::atol(e) : 2000;
    if (ms <= 0) ms = 2000;
    return static_cast<uint64_t>(ms) * 1000000ull;
  }();
  return v;
}

// Test hook, read on every call so a test can switch it: the forward's softmax
// warps idle ATTN_TEST_EPILOGUE_DELAY_US microseconds (at most 1000) before
// their final wait.  0 or unset in normal use.
uint64_t test_epilogue_delay_ns() {
  const char* e = std::getenv("ATTN_TEST_EPILOGUE_DELAY_US");
  if (!e) return 0;
  long us = std::atol(e);
  if (us <= 0) return 0;
  if (us > 1000) us = 1000;
  return static_cast<uint64_t>(us) * 1000ull;
}

// Packed GQA for the forward: a CTA serves all G query heads of a key/value head
// (tile row r = query row r / G of head r % G), used whenever G is a power of two
// in [2, 16].  K/V is loaded once per group instead of once per query head, short
// query segments fill the tiles, and a tile spans only 128 / G query positions, so
// under causal masks and local windows its key range is tighter.  Measured on B200
// against one tile per query head: +3-5% on causal 16K (head_dim 128) and 128K
// (head_dim 256, GQA-8), +1-2% on the varlen batch, no change on long non-causal
// segments, +50% on 128-token segments.  ATTN_PACK_GQA=0 / 1 forces it off / on
// (where G allows), read on every call so tests can exercise both.  Returns log2 G
// or 0.
int pack_gqa_shift(int group) {
  if (group < 2 || group > 16 || (group & (group - 1)) != 0) return 0;
  const char* e = std::getenv("ATTN_PACK_GQA");
  if (e && e[0] == '0') return 0;
  int sh = 0;
  while ((1 << sh) < group) ++sh;
  return sh;
}

// Per-device set-up, once: the error word's device address and the device's
// compute capability.
DeviceState* device_state(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceState& st = g_dev[dev];
  std::call_once(st.once, [&st, dev] {
    st.init_status = cudaGetSymbolAddress(reinterpret_cast<void**>(&st.err), g_device_error);
    if (st.init_status != cudaSuccess) return;
    cudaDeviceGetAttribute(&st.sm_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&st.sm_minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&st.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
  });
  if (st.init_status != cudaSuccess) return nullptr;
  *dev_out = dev;
  return &st;
}

// SMs of the current device (set up by device_state before any launch)
int device_sm_count() {
  int dev = 0;
  DeviceState* st = device_state(&dev);
  return (st && st->num_sms > 0) ? st->num_sms : 1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// bf16 [rows][heads][D] viewed as a 3-D tensor (D, heads, rows); box of
// 64 columns x 1 head x box_rows rows, 128-byte swizzle.
// fp32 [rows][heads][d] viewed as (d, heads, rows); box of box_cols x 1 x box_rows,
// no swizzle (the dQ accumulator, written by TMA reduce-adds)
bool make_map_f32(CUtensorMap* map, const void* ptr, int rows, int heads, int d, int box_cols,
                  int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(heads) * d * 4};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), 1u,
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* map, const void* ptr, int rows, int heads, int d, int box_rows,
              int box_heads = 1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(heads) * d * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_heads),
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

attn_status_t check_common(const void* q, const void* k, const void* v,
                           const int32_t* cu_q, const int32_t* cu_k, int32_t batch,
                           int32_t total_q, int32_t total_k, int32_t max_q, int32_t max_k,
                           int32_t hq, int32_t hkv, int32_t d, float scale) {
  if (!q || !k || !v || !cu_q || !cu_k) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return ATTN_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || total_k < 0 || max_q < 0 || max_k < 0)
    return ATTN_ERR_INVALID_ARG;
  if (hq < 1 || hkv < 1 || hq % hkv != 0 || hq > 65535) return ATTN_ERR_INVALID_ARG;
  if (batch > 65535) return ATTN_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  // index arithmetic inside the kernels is 32-bit per row offset
  if (static_cast<int64_t>(total_q) * hq * d >= (int64_t(1) << 40)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// Window and softcap arguments turned into the kernels' form.  With delta =
// s_k - s_q, row i sees keys [i + delta - lo_off, i + delta + hi_off].
struct MaskArgs {
  bool upper;    // an upper key bound exists (causal or window_right >= 0)
  int hi_off;
  int lo_off;    // kNoBound: none
  bool softcap;
  float cap_k2;    // 2 log2(e) scale / c
  float cap_log2;  // c * log2(e)
  float cap_k1;    // scale / c
};

attn_status_t mask_args(int32_t causal, int32_t window_left, int32_t window_right,
                        float softcap, float scale, MaskArgs* m) {
  if (!std::isfinite(softcap) || softcap < 0.f) return ATTN_ERR_INVALID_ARG;
  // bounds past any possible segment length mean no bound
  const int32_t kFar = kNoBound - 1;
  const int32_t wl = window_left < 0 ? -1 : std::min(window_left, kFar);
  const int32_t wr = window_right < 0 ? -1 : std::min(window_right, kFar);
  m->upper = causal != 0 || wr >= 0;
  m->hi_off = causal ? (wr >= 0 ? std::min(wr, 0) : 0) : (wr >= 0 ? wr : kNoBound);
  m->lo_off = wl >= 0 ? wl : kNoBound;
  m->softcap = softcap > 0.f;
  m->cap_k2 = m->softcap ? 2.f * 1.4426950408889634f * scale / softcap : 0.f;
  m->cap_log2 = m->softcap ? softcap * 1.4426950408889634f : 0.f;
  m->cap_k1 = m->softcap ? scale / softcap : 0.f;
  return ATTN_OK;
}

// head_dim 128 and 256 without softcap or SplitKV can run on the two-CTA
// kernels of fwd_pair_kernel.cuh (M = 256 MMAs over a CTA pair, 128-key
// blocks, each CTA loading half of every K and V block).  ATTN_FWD_PAIR=1 / 0
// forces them on / off (read on every call, so tests can compare); by default
// head_dim 256 uses them (the one-CTA kernel is bound by shared-memory reads
// there, which the pair halves) and head_dim 128 does not (both kernels are
// bound by the softmax warps' exps, and the one-CTA kernel measured faster).
bool fwd_use_pair(int d) {
  const char* e = std::getenv("ATTN_FWD_PAIR");
  if (e && e[0] == '1') return true;
  if (e && e[0] == '0') return false;
  return d == 256;
}

template <int D, bool CAUSAL>
attn_status_t launch_fwd_pair(const void* q, const void* k, const void* v, int total_q,
                              int total_k, int hkv, const FwdParams& p, int batch, int hq,
                              int max_q, cudaStream_t stream) {
  using C = FwdPairCfg<D>;
  CUtensorMap mq, mk, mv;
  const int g = 1 << p.pack_shift;
  // head_dim 128: K boxes of this CTA's 64 keys, V boxes of 128 keys x 64
  // columns; head_dim 256: 64-row boxes for both
  const int k_rows = C::BN / 2, v_rows = (D == 128) ? C::BN : 64;
  if (!make_map(&mq, q, total_q, hq, D, C::BM / g, g) ||
      !make_map(&mk, k, total_k, hkv, D, k_rows) || !make_map(&mv, v, total_k, hkv, D, v_rows))
    return ATTN_ERR_CUDA;
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_status[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev], [&] {
    attr_status[dev] = cudaFuncSetAttribute(attn_fwd_pair_kernel<D, CAUSAL>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            C::SMEM_BYTES);
  });
  if (attr_status[dev] != cudaSuccess) return ATTN_ERR_CUDA;
  const int rows_per_pair = (2 * C::BM) >> p.pack_shift;
  const int pairs = (max_q + rows_per_pair - 1) / rows_per_pair;
  if (pairs == 0) return ATTN_OK;
  dim3 grid(2 * pairs, p.pack_shift > 0 ? hkv : hq, batch);
  record_start(ATTN_KERNEL_FWD, stream);
  attn_fwd_pair_kernel<D, CAUSAL><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  const cudaError_t e = cudaGetLastError();
  record_stop(ATTN_KERNEL_FWD, stream);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The forward's grid.  Persistent (one CTA per SM, each walking a static
// share of the tiles, so a tile's loads and first MMAs overlap the previous
// tile's epilogue) when every tile has the same, small amount of work
// (uniform_tiles); otherwise one CTA per tile, so the hardware hands tiles of
// unequal work to whichever SM is free (a static share measured 17% slower on
// a varlen batch) and long tiles keep the single-tile epilogue, which stages O
// through shared memory.  ATTN_FWD_GRID=tiles / persistent forces either (read
// on every call, for tests).
constexpr int kPersistMaxBlocks = 4;

bool fwd_grid_persistent(const FwdParams& p) {
  const char* e = std::getenv("ATTN_FWD_GRID");
  if (e && std::strcmp(e, "tiles") == 0) return false;
  if (e && std::strcmp(e, "persistent") == 0) return true;
  return p.uniform_tiles != 0;
}

template <int D, bool CAUSAL, bool SOFTCAP>
attn_status_t launch_fwd(const void* q, const void* k, const void* v, int total_q, int total_k,
                         int hkv, const FwdParams& p, int batch, int hq, int max_q,
                         cudaStream_t stream) {
  if constexpr (D != 64 && !SOFTCAP) {
    if (p.num_splits == 1 && fwd_use_pair(D))
      return launch_fwd_pair<D, CAUSAL>(q, k, v, total_q, total_k, hkv, p, batch, hq, max_q,
                                        stream);
  }
  using C = FwdCfg<D>;
  // Q: one 128-row box per 64-column panel; K: one BN-row box per panel;
  // V: VROWS rows per box, all panels of a chunk together
  CUtensorMap mq, mk, mv;
  // packed GQA: one box holds BM/G query rows of all G heads of a group
  const int g = 1 << p.pack_shift;
  if (!make_map(&mq, q, total_q, hq, D, C::BM / g, g) ||
      !make_map(&mk, k, total_k, hkv, D, C::BN) ||
      !make_map(&mv, v, total_k, hkv, D, C::VROWS))
    return ATTN_ERR_CUDA;
  // the limit is raised once per device; its outcome is kept, so a failure is
  // reported on every call, not only the first
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_status[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev], [&] {
    attr_status[dev] = cudaFuncSetAttribute(attn_fwd_kernel<D, CAUSAL, SOFTCAP>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            C::SMEM_BYTES);
  });
  if (attr_status[dev] != cudaSuccess) return ATTN_ERR_CUDA;
  const int rows_per_cta = (C::BM * C::NQ) >> p.pack_shift;
  const int m_tiles = (max_q + rows_per_cta - 1) / rows_per_cta;
  if (m_tiles == 0) return ATTN_OK;
  // tiles: (query tile, head, segment x split); see fwd_grid_persistent
  FwdParams pt = p;
  pt.tiles_x = m_tiles;
  pt.tiles_y = p.pack_shift > 0 ? hkv : hq;
  pt.tiles_total = static_cast<long long>(m_tiles) * pt.tiles_y * batch;
  const long long ctas = fwd_grid_persistent(p)
                             ? std::min<long long>(pt.tiles_total, device_sm_count())
                             : pt.tiles_total;
  if (ctas > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  record_start(ATTN_KERNEL_FWD, stream);
  attn_fwd_kernel<D, CAUSAL, SOFTCAP><<<static_cast<unsigned>(ctas), C::THREADS, C::SMEM_BYTES,
                                        stream>>>(mq, mk, mv, pt);
  const cudaError_t e = cudaGetLastError();
  record_stop(ATTN_KERNEL_FWD, stream);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool CAUSAL, bool SOFTCAP>
attn_status_t launch_bwd_main(const BwdArgs& a, const BwdParams& bp, cudaStream_t stream) {
  using C = BwdCfg<D>;
  // the limit is raised once per device; its outcome is kept, so a failure is
  // reported on every call, not only the first
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_status[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev], [&] {
    attr_status[dev] = cudaFuncSetAttribute(attn_bwd_main_kernel<D, CAUSAL, SOFTCAP>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            C::SMEM_BYTES);
  });
  if (attr_status[dev] != cudaSuccess) return ATTN_ERR_CUDA;
  CUtensorMap mk, mv, mq, mo, mdq;
  if (!make_map(&mk, a.k, a.total_k, a.hkv, D, 128) ||
      !make_map(&mv, a.v, a.total_k, a.hkv, D, 128) ||
      !make_map(&mq, a.q, a.total_q, a.hq, D, C::BM) ||
      !make_map(&mo, a.dout, a.total_q, a.hq, D, C::BM) ||
      !make_map_f32(&mdq, bp.dq_acc, a.total_q, a.hq, D, 32, C::BM / 2))
    return ATTN_ERR_CUDA;
  const int n_blocks = (a.max_k + C::BN - 1) / C::BN;
  if (n_blocks == 0) return ATTN_OK;
  dim3 grid(n_blocks * C::NSPLIT, a.hkv, a.batch);
  record_start(ATTN_KERNEL_BWD_MAIN, stream);
  attn_bwd_main_kernel<D, CAUSAL, SOFTCAP><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(
      mk, mv, mq, mo, mdq, bp);
  const cudaError_t e = cudaGetLastError();
  record_stop(ATTN_KERNEL_BWD_MAIN, stream);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// head_dim 256 without a softcap: the two-CTA kernel of bwd_pair_kernel.cuh
// (one cluster per 128-key block, work split by role, nothing recomputed).
// ATTN_BWD_PAIR=0 selects the head_dim-split kernel instead (read on every call,
// so tests can compare the two).
bool bwd_use_pair() {
  const char* e = std::getenv("ATTN_BWD_PAIR");
  return !(e && e[0] == '0');
}

template <bool CAUSAL>
attn_status_t launch_bwd_pair(const BwdArgs& a, const BwdParams& bp, cudaStream_t stream) {
  using C = PairCfg;
  static std::once_flag attr_once[kMaxDevices];
  static cudaError_t attr_status[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev], [&] {
    attr_status[dev] = cudaFuncSetAttribute(attn_bwd_pair_kernel<CAUSAL>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            C::SMEM_BYTES);
  });
  if (attr_status[dev] != cudaSuccess) return ATTN_ERR_CUDA;
  CUtensorMap mk, mq, mo, mdq;
  if (!make_map(&mk, a.k, a.total_k, a.hkv, C::D, C::BN) ||
      !make_map(&mq, a.q, a.total_q, a.hq, C::D, C::BM) ||
      !make_map(&mo, a.dout, a.total_q, a.hq, C::D, C::BM) ||
      !make_map_f32(&mdq, bp.dq_acc, a.total_q, a.hq, C::D, 32, C::BM / 2))
    return ATTN_ERR_CUDA;
  const int n_blocks = (a.max_k + C::BN - 1) / C::BN;
  if (n_blocks == 0) return ATTN_OK;
  dim3 grid(2 * n_blocks, a.hkv, a.batch);
  record_start(ATTN_KERNEL_BWD_MAIN, stream);
  attn_bwd_pair_kernel<CAUSAL><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(
      mk, mq, mo, mdq, bp, static_cast<const uint16_t*>(a.k), static_cast<const uint16_t*>(a.v));
  const cudaError_t e = cudaGetLastError();
  record_stop(ATTN_KERNEL_BWD_MAIN, stream);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Direct dQ stores: when every key segment fits one key block of the backward
// (max_seqlen_k <= 128), the single CTA of each (segment, key/value head) holds
// the complete dQ of its rows and stores it as bf16, with no fp32 accumulator
// round trip and no postprocess launch.  ATTN_BWD_DQ_DIRECT=0 forces the
// accumulator path (read on every call so tests can compare the two).
bool bwd_dq_direct(int max_k) {
  const char* e = std::getenv("ATTN_BWD_DQ_DIRECT");
  if (e && e[0] == '0') return false;
  return max_k <= 128;
}

template <int D>
attn_status_t bwd_launch_d(const BwdArgs& a, cudaStream_t stream) {
  static_assert(BwdCfg<D>::BN == 128, "direct dQ assumes 128-key blocks");
  const bool direct = bwd_dq_direct(a.max_k);
  float* dq_acc = static_cast<float*>(a.workspace);
  float* delta = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) +
                                          bwd_align256(static_cast<size_t>(a.total_q) * a.hq * D * 4));
  const long long n_rh = static_cast<long long>(a.total_q) * a.hq;
  if (n_rh > 0) {
    const long long threads = n_rh * (D / 8);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    attn_bwd_pre_kernel<D><<<blocks, 256, 0, stream>>>(
        static_cast<const uint16_t*>(a.out), static_cast<const uint16_t*>(a.dout), delta, dq_acc,
        direct ? static_cast<uint16_t*>(a.dq) : nullptr, a.total_q, a.hq);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  BwdParams bp;
  bp.cu_q = a.cu_q;
  bp.cu_k = a.cu_k;
  bp.lse = a.lse;
  bp.delta = delta;
  bp.dq_acc = dq_acc;
  bp.dq_out = direct ? static_cast<uint16_t*>(a.dq) : nullptr;
  bp.dk = a.dk;
  bp.dv = a.dv;
  bp.err = a.err;
  bp.total_q = a.total_q;
  bp.nheads_q = a.hq;
  bp.nheads_kv = a.hkv;
  bp.scale = a.scale;
  bp.scale_log2 = a.scale * 1.4426950408889634f;
  bp.hi_off = a.hi_off;
  bp.lo_off = a.lo_off;
  bp.cap_k2 = a.cap_k2;
  bp.cap_log2 = a.cap_log2;
  bp.timeout_ns = a.timeout_ns;
  if (a.total_k > 0) {
    attn_status_t st;
    if (a.softcap)
      st = a.upper ? launch_bwd_main<D, true, true>(a, bp, stream)
                   : launch_bwd_main<D, false, true>(a, bp, stream);
    else if (D == 256 && bwd_use_pair())
      st = a.upper ? launch_bwd_pair<true>(a, bp, stream) : launch_bwd_pair<false>(a, bp, stream);
    else
      st = a.upper ? launch_bwd_main<D, true, false>(a, bp, stream)
                   : launch_bwd_main<D, false, false>(a, bp, stream);
    if (st != ATTN_OK) return st;
  }
  if (n_rh > 0 && !direct) {
    const long long n8 = n_rh * D / 8;
    long long blocks = (n8 + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    attn_bwd_dq_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        dq_acc, static_cast<uint16_t*>(a.dq), n8, a.scale);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

attn_status_t bwd_launch(const BwdArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 64: return bwd_launch_d<64>(a, stream);
    case 128: return bwd_launch_d<128>(a, stream);
    default: return bwd_launch_d<256>(a, stream);
  }
}

}  // namespace
}  // namespace attn

using namespace attn;

namespace {
constexpr int kMaxSplits = 128;

size_t fwd_split_workspace_bytes(int32_t total_q, int32_t nheads_q, int32_t head_dim,
                                 int32_t num_splits) {
  const size_t rows = static_cast<size_t>(num_splits) * (total_q > 0 ? total_q : 1) * nheads_q;
  return bwd_align256(rows * head_dim * 4) + bwd_align256(rows * 4);
}

// the forward with num_splits SplitKV parts (1: plain) and its combine
attn_status_t fwd_impl(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                       const int32_t* cu_seqlens_k, int32_t batch, int32_t total_q,
                       int32_t total_k, int32_t max_seqlen_q, int32_t max_seqlen_k,
                       int32_t nheads_q, int32_t nheads_kv, int32_t head_dim, float scale,
                       int32_t causal, int32_t window_left, int32_t window_right, float softcap,
                       int32_t num_splits, int32_t return_lse, void* out, float* lse,
                       void* workspace, size_t workspace_bytes, attn_stream_t stream) {
  attn_status_t st = check_common(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                  max_seqlen_q, max_seqlen_k, nheads_q, nheads_kv, head_dim,
                                  scale);
  if (st != ATTN_OK) return st;
  MaskArgs mk;
  st = mask_args(causal, window_left, window_right, softcap, scale, &mk);
  if (st != ATTN_OK) return st;
  if (!out || !aligned16(out)) return ATTN_ERR_INVALID_ARG;
  if (return_lse && (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u))) return ATTN_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > kMaxSplits ||
      static_cast<int64_t>(batch) * num_splits > 65535)
    return ATTN_ERR_INVALID_ARG;
  if (num_splits > 1 &&
      (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
       workspace_bytes < fwd_split_workspace_bytes(total_q, nheads_q, head_dim, num_splits)))
    return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  DeviceState* ds = device_state(&dev);
  if (!ds) return ATTN_ERR_CUDA;
  if (ds->sm_major != 10) return ATTN_ERR_UNSUPPORTED;
  if (total_q == 0 || max_seqlen_q == 0) return ATTN_OK;

  FwdParams p;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.out = out;
  p.lse = lse;
  p.err = ds->err;
  p.total_q = total_q;
  p.nheads_q = nheads_q;
  p.nheads_kv = nheads_kv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.return_lse = return_lse ? 1 : 0;
  p.hi_off = mk.hi_off;
  p.lo_off = mk.lo_off;
  p.cap_k2 = mk.cap_k2;
  p.cap_log2 = mk.cap_log2;
  p.cap_k1 = mk.cap_k1;
  p.num_splits = num_splits;
  p.o_part = nullptr;
  p.lse_part = nullptr;
  if (num_splits > 1) {
    p.o_part = static_cast<float*>(workspace);
    p.lse_part = reinterpret_cast<float*>(
        static_cast<uint8_t*>(workspace) +
        bwd_align256(static_cast<size_t>(num_splits) * total_q * nheads_q * head_dim * 4));
  }
  p.pack_shift = pack_gqa_shift(nheads_q / nheads_kv);
  // equal segments have total = batch x max (no segment is longer than max);
  // a persistent grid pays off only for short tiles (set-up and pipeline fill
  // are then a large share), so tiles of more than kPersistMaxBlocks key
  // blocks keep one CTA per tile
  const int block_keys = head_dim == 64 ? 96 : (head_dim == 128 ? 64 : 128);
  p.uniform_tiles = !mk.upper && mk.lo_off >= kNoBound && num_splits == 1 &&
                    static_cast<int64_t>(batch) * max_seqlen_q == total_q &&
                    static_cast<int64_t>(batch) * max_seqlen_k == total_k &&
                    (max_seqlen_k + block_keys - 1) / block_keys <= kPersistMaxBlocks;
  p.timeout_ns = wait_timeout_ns();
  p.epilogue_delay_ns = test_epilogue_delay_ns();

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int grid_z = batch * num_splits;
  auto run = [&](auto launch) {
    attn_status_t r =
        launch(q, k, v, total_q, total_k, nheads_kv, p, grid_z, nheads_q, max_seqlen_q, s);
    if (r != ATTN_OK || num_splits == 1) return r;
    const long long warps = static_cast<long long>(total_q) * nheads_q;
    const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
    switch (head_dim) {
      case 64:
        attn_fwd_combine_kernel<64><<<blocks, 256, 0, s>>>(
            p.o_part, p.lse_part, static_cast<uint16_t*>(out), lse, total_q, nheads_q,
            num_splits, return_lse);
        break;
      case 128:
        attn_fwd_combine_kernel<128><<<blocks, 256, 0, s>>>(
            p.o_part, p.lse_part, static_cast<uint16_t*>(out), lse, total_q, nheads_q,
            num_splits, return_lse);
        break;
      default:
        attn_fwd_combine_kernel<256><<<blocks, 256, 0, s>>>(
            p.o_part, p.lse_part, static_cast<uint16_t*>(out), lse, total_q, nheads_q,
            num_splits, return_lse);
    }
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  };
  // the kernel's CAUSAL parameter means "rows have an upper key bound"
  const int variant = (mk.upper ? 1 : 0) | (mk.softcap ? 2 : 0);
  switch (head_dim) {
    case 64:
      switch (variant) {
        case 0: return run(launch_fwd<64, false, false>);
        case 1: return run(launch_fwd<64, true, false>);
        case 2: return run(launch_fwd<64, false, true>);
        default: return run(launch_fwd<64, true, true>);
      }
    case 128:
      switch (variant) {
        case 0: return run(launch_fwd<128, false, false>);
        case 1: return run(launch_fwd<128, true, false>);
        case 2: return run(launch_fwd<128, false, true>);
        default: return run(launch_fwd<128, true, true>);
      }
    default:
      switch (variant) {
        case 0: return run(launch_fwd<256, false, false>);
        case 1: return run(launch_fwd<256, true, false>);
        case 2: return run(launch_fwd<256, false, true>);
        default: return run(launch_fwd<256, true, true>);
      }
  }
}

}  // namespace

extern "C" attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v,
                                     const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                     int32_t batch, int32_t total_q, int32_t total_k,
                                     int32_t max_seqlen_q, int32_t max_seqlen_k,
                                     int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                                     float scale, int32_t causal, int32_t window_left,
                                     int32_t window_right, float softcap, int32_t return_lse,
                                     void* out, float* lse, attn_stream_t stream) {
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, nheads_q, nheads_kv, head_dim, scale, causal, window_left,
                  window_right, softcap, 1, return_lse, out, lse, nullptr, 0, stream);
}

extern "C" size_t attn_fwd_split_workspace_size(int32_t total_q, int32_t nheads_q,
                                                int32_t head_dim, int32_t num_splits) {
  if (total_q < 0 || nheads_q < 1 || head_dim < 1 || num_splits < 1 || num_splits > kMaxSplits)
    return 0;
  return fwd_split_workspace_bytes(total_q, nheads_q, head_dim, num_splits);
}

extern "C" attn_status_t attn_fwd_split(const void* q, const void* k, const void* v,
                                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                        int32_t batch, int32_t total_q, int32_t total_k,
                                        int32_t max_seqlen_q, int32_t max_seqlen_k,
                                        int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                                        float scale, int32_t causal, int32_t window_left,
                                        int32_t window_right, float softcap, int32_t num_splits,
                                        int32_t return_lse, void* out, float* lse,
                                        void* workspace, size_t workspace_bytes,
                                        attn_stream_t stream) {
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, nheads_q, nheads_kv, head_dim, scale, causal, window_left,
                  window_right, softcap, num_splits, return_lse, out, lse, workspace,
                  workspace_bytes, stream);
}

extern "C" attn_status_t attn_fwd(const void* q, const void* k, const void* v,
                                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                  int32_t batch, int32_t total_q, int32_t total_k,
                                  int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t nheads_q,
                                  int32_t nheads_kv, int32_t head_dim, float scale,
                                  int32_t causal, int32_t return_lse, void* out, float* lse,
                                  attn_stream_t stream) {
  return attn_fwd_ex(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                     max_seqlen_q, max_seqlen_k, nheads_q, nheads_kv, head_dim, scale, causal,
                     -1, -1, 0.f, return_lse, out, lse, stream);
}

extern "C" size_t attn_bwd_workspace_size(int32_t batch, int32_t total_q, int32_t nheads_q,
                                          int32_t head_dim) {
  if (batch < 1 || total_q < 0 || nheads_q < 1 || head_dim < 1) return 0;
  return bwd_workspace_bytes(batch, total_q, nheads_q, head_dim);
}

extern "C" attn_status_t attn_bwd_ex(const void* q, const void* k, const void* v,
                                     const void* out, const float* lse, const void* dout,
                                     const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                     int32_t batch, int32_t total_q, int32_t total_k,
                                     int32_t max_seqlen_q, int32_t max_seqlen_k,
                                     int32_t nheads_q, int32_t nheads_kv, int32_t head_dim,
                                     float scale, int32_t causal, int32_t window_left,
                                     int32_t window_right, float softcap, void* dq, void* dk,
                                     void* dv, void* workspace, size_t workspace_bytes,
                                     attn_stream_t stream) {
  attn_status_t st = check_common(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                  max_seqlen_q, max_seqlen_k, nheads_q, nheads_kv, head_dim,
                                  scale);
  if (st != ATTN_OK) return st;
  MaskArgs mk;
  st = mask_args(causal, window_left, window_right, softcap, scale, &mk);
  if (st != ATTN_OK) return st;
  if (!out || !lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < bwd_workspace_bytes(batch, total_q, nheads_q, head_dim))
    return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  DeviceState* ds = device_state(&dev);
  if (!ds) return ATTN_ERR_CUDA;
  if (ds->sm_major != 10) return ATTN_ERR_UNSUPPORTED;
  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.out = out; a.lse = lse; a.dout = dout;
  a.cu_q = cu_seqlens_q; a.cu_k = cu_seqlens_k;
  a.batch = batch; a.total_q = total_q; a.total_k = total_k;
  a.max_q = max_seqlen_q; a.max_k = max_seqlen_k;
  a.hq = nheads_q; a.hkv = nheads_kv; a.d = head_dim;
  a.scale = scale;
  a.upper = mk.upper; a.hi_off = mk.hi_off; a.lo_off = mk.lo_off;
  a.softcap = mk.softcap; a.cap_k2 = mk.cap_k2; a.cap_log2 = mk.cap_log2;
  a.dq = dq; a.dk = dk; a.dv = dv; a.workspace = workspace;
  a.err = ds->err;
  a.timeout_ns = wait_timeout_ns();
  return bwd_launch(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* out,
                                  const float* lse, const void* dout,
                                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                  int32_t batch, int32_t total_q, int32_t total_k,
                                  int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t nheads_q,
                                  int32_t nheads_kv, int32_t head_dim, float scale,
                                  int32_t causal, void* dq, void* dk, void* dv, void* workspace,
                                  size_t workspace_bytes, attn_stream_t stream) {
  return attn_bwd_ex(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, batch, total_q,
                     total_k, max_seqlen_q, max_seqlen_k, nheads_q, nheads_kv, head_dim, scale,
                     causal, -1, -1, 0.f, dq, dk, dv, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// attn_bwd_static_scratch: the backward for callers that cannot allocate.
// Its scratch is this file-scope device array; in host code the name is only a
// host-side stand-in, so the device address is looked up once per device with
// cudaGetSymbolAddress and handed to the kernels as the workspace pointer.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_static_scratch[ATTN_STATIC_SCRATCH_BYTES];

namespace {
struct StaticScratch {
  std::once_flag once;
  cudaError_t status = cudaSuccess;
  void* ptr = nullptr;
};
StaticScratch g_scratch[kMaxDevices];
}  // namespace

extern "C" attn_status_t attn_bwd_static_scratch(
    const void* q, const void* k, const void* v, const void* out, const float* lse,
    const void* dout, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch,
    int32_t total_q, int32_t total_k, int32_t max_seqlen_q, int32_t max_seqlen_k,
    int32_t nheads_q, int32_t nheads_kv, int32_t head_dim, float scale, int32_t causal,
    void* dq, void* dk, void* dv, attn_stream_t stream) {
  attn_status_t st = check_common(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                  max_seqlen_q, max_seqlen_k, nheads_q, nheads_kv, head_dim,
                                  scale);
  if (st != ATTN_OK) return st;
  const size_t need = bwd_workspace_bytes(batch, total_q, nheads_q, head_dim);
  if (need > ATTN_STATIC_SCRATCH_BYTES) return ATTN_ERR_SCRATCH_TOO_SMALL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  StaticScratch& sc = g_scratch[dev];
  std::call_once(sc.once, [&sc] {
    // runs with `dev` current: the address is that device's copy of the array
    sc.status = cudaGetSymbolAddress(&sc.ptr, g_static_scratch);
  });
  if (sc.status != cudaSuccess || sc.ptr == nullptr) return ATTN_ERR_CUDA;
  // attn_bwd's own checks and launches, with the array as its workspace; its
  // preprocess kernel rewrites D_i and zeroes what must start at zero (the dQ
  // accumulator, or dq itself when every key segment fits one key block) on
  // every call
  return attn_bwd(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                  max_seqlen_q, max_seqlen_k, nheads_q, nheads_kv, head_dim, scale, causal, dq,
                  dk, dv, sc.ptr, ATTN_STATIC_SCRATCH_BYTES, stream);
}

extern "C" attn_status_t attn_last_device_error(attn_stream_t stream, char* msg,
                                                size_t msg_len) {
  auto put = [&](const char* m) {
    if (msg && msg_len) {
      std::strncpy(msg, m, msg_len - 1);
      msg[msg_len - 1] = '\0';
    }
  };
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    put(cudaGetErrorString(e));
    return ATTN_ERR_CUDA;
  }
  int dev = 0;
  DeviceState* ds = device_state(&dev);
  if (!ds) {
    put("device set-up failed");
    return ATTN_ERR_CUDA;
  }
  uint32_t word = 0;
  const uint32_t zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) {
    put("could not read the device error word");
    return ATTN_ERR_CUDA;
  }
  if (word == 0) {
    put("ok");
    return ATTN_OK;
  }
  static const char* kernels[] = {"?", "fwd load", "fwd mma", "fwd softmax", "bwd preprocess",
                                  "bwd load", "bwd mma", "bwd softmax", "bwd dq convert",
                                  "watchdog self-test", "bwd pair load", "bwd pair mma",
                                  "bwd pair elementwise", "bwd pair exchange", "bwd pair dq",
                                  "fwd pair load", "fwd pair mma", "fwd pair softmax"};
  const uint32_t kid = (word >> 8) & 0xff;
  char buf[128];
  std::snprintf(buf, sizeof(buf), "timed-out wait in %s (wait %u)",
                kid < sizeof(kernels) / sizeof(kernels[0]) ? kernels[kid] : "?", word & 0xffu);
  put(buf);
  return ATTN_ERR_TIMEOUT;
}

extern "C" attn_status_t attn_set_timing_events(int32_t kernel, void* start, void* stop) {
  if (kernel != ATTN_KERNEL_FWD && kernel != ATTN_KERNEL_BWD_MAIN) return ATTN_ERR_INVALID_ARG;
  if ((start == nullptr) != (stop == nullptr)) return ATTN_ERR_INVALID_ARG;
  t_events[kernel].start = static_cast<cudaEvent_t>(start);
  t_events[kernel].stop = static_cast<cudaEvent_t>(stop);
  return ATTN_OK;
}

#ifdef ATTN_TRACE
extern "C" int attn_debug_set_trace(void* buf) {
  unsigned long long* p = static_cast<unsigned long long*>(buf);
  return cudaMemcpyToSymbol(g_attn_trace, &p, sizeof(p)) == cudaSuccess ? 0 : -1;
}
#endif

namespace attn {
// One thread waits on a barrier that is never arrived on; the bounded wait
// runs out, records ERR_SELFTEST in the error word and returns.
__global__ void attn_watchdog_selftest_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_flag, err, ERR_SELFTEST, timeout_ns);
  }
}
}  // namespace attn

extern "C" attn_status_t attn_watchdog_selftest(int32_t timeout_us, attn_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  DeviceState* ds = device_state(&dev);
  if (!ds) return ATTN_ERR_CUDA;
  attn_watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      ds->err, static_cast<uint64_t>(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

#define ATTN_STR2(x) #x
#define ATTN_STR(x) ATTN_STR2(x)
// the build's forward exp2 setting is part of the string, so a caller can see
// which variant it loaded
extern "C" const char* attn_version(void) {
  return "exact_attention_b200 0.2 sm_100a fwd_poly_pairs=" ATTN_STR(ATTN_FWD_POLY_PAIRS);
}

// bwd_kernels.cuh -- sm_100a backward pass: dQ, dK, dV of exact attention,
// recomputing P from the forward's LSE.
//
// The FA4 repository guide (Backward Kernels) splits its backward into a
// preprocess kernel, a main kernel and a postprocess kernel; the plainest
// reading of that split, with the method's P = exp(S - LSE), dS = P * (dP - D)
// and D_i = dO_i . O_i, is:
//
//   1. preprocess: D_i = sum_d dO_id O_id (fp32) and a zeroed fp32 dQ accumulator;
//   2. main: per key block, loop over the query blocks (and, for GQA, over the
//      query heads of the group) recomputing S^T = K Q^T and dP^T = V dO^T with
//      tcgen05 MMAs, forming P^T and dS^T elementwise, accumulating dV += P^T dO
//      and dK += dS^T Q in tensor memory for the whole loop (so the GQA group sum
//      costs nothing extra) and computing dQ^T = K^T dS^T per query block, which
//      is added into the fp32 accumulator with coalesced reductions;
//   3. postprocess: dQ = scale * accumulator, rounded to bf16.
//
// When every key segment fits one 128-key block (max_seqlen_k <= 128), the one
// CTA of a (segment, key/value head) sees all keys of its query rows, so its dQ
// is already complete: it stores scale * dQ as bf16 straight into dq, the
// preprocess zeroes dq instead of the accumulator (rows that see no key are
// never stored), and the postprocess is not launched.  Short segments are
// bound by HBM, and this drops the fp32 accumulator's round trip.
//
// Main-kernel layout for one CTA (128 keys; head_dim 256 is split into two
// 128-wide halves handled by two CTAs, each recomputing S and dP in full):
//   tensor memory: S^T x2 (64 cols each; per warpgroup P^T in bf16 is written
//                  back over columns 0-15 / 32-47 and dS^T over 16-31 / 48-63,
//                  the A operands of dV and dK), dP^T (64), dQ^T (64), dV (DH),
//                  dK (DH)  = 512 cols
//   shared memory: K and V tiles (resident), a ring of NST (Q, dO) stages of
//                  64 query rows, two dS^T tiles (128 keys x 64 queries, bf16,
//                  128-byte swizzled: the MN-major B operand of dQ^T = K^T dS^T),
//                  and per-block LSE/D vectors.
//   warps: 8 elementwise warps (two warpgroups, each taking 32 of a block's 64
//          query columns; thread = key row = TMEM lane), 1 TMA warp and MMA
//          warps that run their role warp-wide, one elected lane issuing.
//          head_dim 64/128: two MMA warps (S and dP; dV, dK and dQ), one idle
//          warp and a dQ warpgroup that reads dQ^T out and issues its TMA
//          reduce-adds, 512 threads with setmaxnreg.  head_dim 256: one MMA
//          warp; the elementwise warps add dQ with atomics (320 threads).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

#include "attn.h"
#include "ptx.cuh"

namespace attn {

enum : uint32_t {
  ERR_BWD_LOAD = 0x0500,
  ERR_BWD_MMA = 0x0600,
  ERR_BWD_ELEM = 0x0700,
};

struct BwdArgs {
  const void *q, *k, *v, *out, *dout;
  const float* lse;
  const int32_t *cu_q, *cu_k;
  int batch, total_q, total_k, max_q, max_k, hq, hkv, d;
  float scale;
  bool upper;              // rows have an upper key bound (causal or a right window)
  int hi_off, lo_off;      // window offsets, as in BwdParams
  bool softcap;
  float cap_k2, cap_log2;
  void *dq, *dk, *dv, *workspace;
  uint32_t* err;
  uint64_t timeout_ns;
};

// workspace: fp32 dQ accumulator [Tq][Hq][D], then fp32 D_i [Hq][Tq]
inline size_t bwd_align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline size_t bwd_workspace_bytes(int batch, int total_q, int hq, int d) {
  (void)batch;
  const size_t rows = static_cast<size_t>(total_q > 0 ? total_q : 1);
  return bwd_align256(rows * hq * d * 4) + bwd_align256(rows * hq * 4);
}

struct BwdParams {
  const int32_t* cu_q;
  const int32_t* cu_k;
  const float* lse;    // [Hq][Tq]
  const float* delta;  // [Hq][Tq]
  float* dq_acc;       // [Tq][Hq][D]
  // non-null when every key segment fits one 128-key block: each CTA then holds
  // the complete dQ of its rows and stores scale * dQ as bf16 here ([Tq][Hq][D])
  // instead of adding into dq_acc
  uint16_t* dq_out;
  void* dk;            // bf16 [Tk][Hkv][D]
  void* dv;
  uint32_t* err;
  int total_q;
  int nheads_q;
  int nheads_kv;
  float scale;
  float scale_log2;
  // keys allowed for segment-local query row i, with delta = s_k - s_q:
  // [i + delta - lo_off, i + delta + hi_off] (kNoBound = none; the upper
  // bound exists iff the kernel's CAUSAL parameter is set)
  int hi_off;
  int lo_off;
  // softcap c: scores c tanh(s scale / c); cap_k2 = 2 log2(e) scale / c,
  // cap_log2 = c log2(e)
  float cap_k2;
  float cap_log2;
  uint64_t timeout_ns;
};

template <int D>
struct BwdCfg {
  static constexpr int BN = 128;                 // keys per CTA
  static constexpr int BM = 64;                  // query rows per iteration
  static constexpr int DH = (D == 256) ? 128 : D;  // accumulator width per CTA
  static constexpr int NSPLIT = D / DH;
  static constexpr int PANELS = D / 64;
  static constexpr int KV_PANEL = BN * 128;      // 16 KB: 128 rows x 64 cols
  static constexpr int QD_PANEL = BM * 128;      // 8 KB: 64 rows x 64 cols
  static constexpr int K_BYTES = PANELS * KV_PANEL + (D == 64 ? KV_PANEL : 0);  // + zero panel
  static constexpr int V_BYTES = PANELS * KV_PANEL;
  static constexpr int STAGE_BYTES = 2 * PANELS * QD_PANEL;  // Q_i then dO_i
  static constexpr int NST = (D == 256) ? 1 : (D == 128 ? 3 : 4);  // (Q, dO) stages
  static constexpr int DS_BYTES = BN * BM * 2;   // 16 KB
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + K_BYTES;
  static constexpr int OFF_ST = OFF_V + V_BYTES;
  static constexpr int OFF_DS = OFF_ST + NST * STAGE_BYTES;
  static constexpr int OFF_LSD = OFF_DS + 2 * DS_BYTES;      // NST x 128 floats
  // dQ^T staging for the TMA reduce-add: per elementwise warp 64 queries x 32
  // features fp32 (head_dim 256 has no room left and adds with atomics instead)
  static constexpr bool DQ_TMA = (D != 256);
  static constexpr int DQ_WARP_BYTES = (BM / 2) * 32 * 4;  // 4 KB: 32 queries x 32 features
  static constexpr int OFF_DQS = OFF_LSD + NST * 128 * 4;
  static constexpr int OFF_BAR = OFF_DQS + (DQ_TMA ? 2 * (DH / 32) * DQ_WARP_BYTES : 0);
  // kv_full, qdo_full[NST], qdo_empty[NST], s_full[2], dp_full, dp_free,
  // ds_ready[2], ds_free[2], dq_full, dq_free, dkv_full, oth_full, oth_empty
  // (head_dim 256 splits its single stage: qdo_full/qdo_empty[0] track this
  // CTA's own head_dim half of Q and dO plus the LSE/D vectors, oth_full /
  // oth_empty the other half, which only S and dP read)
  static constexpr int NBAR = 1 + 2 * NST + 2 + 2 + 2 + 2 + 3 + 2 + 2;  // + s_free[2]
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // warps 0-7: two elementwise warpgroups (each takes 32 of the 64 query
  // columns of a block, thread = key row); warp 8: TMA; warp 9: MMA (S, dP);
  // warp 10 (head_dim 64/128): MMA (dV, dK, dQ), so each issuer can wait on
  // its own barriers while the other keeps the tensor pipe busy
  static constexpr int ELEM_THREADS = 256;
  static constexpr bool TWO_ISSUERS = (NSPLIT == 1);
  // head_dim 64/128: warps 12-15 read dQ^T out of tensor memory and issue its
  // TMA reduce-adds, so the elementwise warps never wait for dQ.  The 16 warps
  // start with 128 registers each (65,536 in all); the warpgroups then set
  // their own budgets: elementwise 184, control (loader, MMA x2, one idle) 64,
  // dQ 80.  Per SM sub-partition (one warp of each warpgroup) that is 512
  // registers per lane, exactly its 16,384.
  static constexpr bool DQ_WARPS = TWO_ISSUERS;
  static constexpr int DQ_WARP0 = 12;
  static constexpr int REG_ELEM = 184, REG_CTRL = 64, REG_DQ = 80;
  static_assert(!DQ_WARPS || 2 * REG_ELEM + REG_CTRL + REG_DQ <= 512, "register split");
  static constexpr int THREADS = DQ_WARPS ? 512 : (TWO_ISSUERS ? 352 : 320);
  static constexpr int LOAD_WARP = 8, MMA_WARP = 9, GRAD_WARP = 10;
  // tensor memory columns
  static constexpr int COL_S = 0, COL_DP = 128, COL_DQ = 192, COL_DV = 256, COL_DK = 256 + DH;
  static constexpr uint32_t IDESC_SDP = idesc_bf16(128, BM, false, false);
  static constexpr uint32_t IDESC_KV = idesc_bf16(128, DH, false, true);
  static constexpr uint32_t IDESC_DQ = idesc_bf16(128, BM, true, true);
};

struct BwdSmem {
  uint8_t *k, *v, *st, *ds, *dqs;
  float* lsd;
  uint64_t *kv_full, *qdo_full, *qdo_empty, *s_full, *dp_full, *dp_free, *ds_ready, *ds_free,
      *dq_full, *dq_free, *dkv_full, *oth_full, *oth_empty, *s_free;
  uint32_t* tmem_base;
  volatile int* abort;
};

template <int D>
__device__ __forceinline__ BwdSmem bwd_smem(uint8_t* base) {
  using C = BwdCfg<D>;
  BwdSmem s;
  s.k = base + C::OFF_K;
  s.v = base + C::OFF_V;
  s.st = base + C::OFF_ST;
  s.ds = base + C::OFF_DS;
  s.lsd = reinterpret_cast<float*>(base + C::OFF_LSD);
  s.dqs = base + C::OFF_DQS;
  uint64_t* b = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  s.kv_full = b;
  s.qdo_full = b + 1;
  s.qdo_empty = s.qdo_full + C::NST;
  s.s_full = s.qdo_empty + C::NST;
  s.dp_full = s.s_full + 2;
  s.dp_free = s.dp_full + 1;
  s.ds_ready = s.dp_free + 1;
  s.ds_free = s.ds_ready + 2;
  s.dq_full = s.ds_free + 2;
  s.dq_free = s.dq_full + 1;
  s.dkv_full = s.dq_free + 1;
  s.oth_full = s.dkv_full + 1;
  s.oth_empty = s.oth_full + 1;
  s.s_free = s.oth_empty + 1;
  s.tmem_base = reinterpret_cast<uint32_t*>(base + C::OFF_MISC);
  s.abort = reinterpret_cast<volatile int*>(base + C::OFF_MISC + 4);
  return s;
}

// The CTA's key block and the query blocks that can see it.
struct BwdTile {
  int q0, sq, k0, sk;
  int n_base;   // first segment-local key row
  int dh;       // accumulator half (head_dim 256) or 0
  int hk;
  int h0;       // first query head of the group
  int G;        // query heads per key/value head
  int m_lo, m_hi;  // query blocks [m_lo, m_hi) of BM rows
  int n_iter;   // G * (m_hi - m_lo)
};

template <int D, bool CAUSAL>
__device__ __forceinline__ bool bwd_tile(const BwdParams& p, BwdTile& t) {
  using C = BwdCfg<D>;
  const int b = blockIdx.z;
  t.hk = blockIdx.y;
  t.G = p.nheads_q / p.nheads_kv;
  t.h0 = t.hk * t.G;
  const int nb = blockIdx.x / C::NSPLIT;
  t.dh = blockIdx.x % C::NSPLIT;
  t.q0 = p.cu_q[b];
  t.sq = p.cu_q[b + 1] - t.q0;
  t.k0 = p.cu_k[b];
  t.sk = p.cu_k[b + 1] - t.k0;
  t.n_base = nb * C::BN;
  if (t.n_base >= t.sk) return false;
  // query rows that see a key of [n_base, n_base + BN): row i sees key j iff
  // i + delta - lo_off <= j <= i + delta + hi_off
  const int delta = t.sk - t.sq;
  int row_lo = 0, row_hi = t.sq;  // [row_lo, row_hi)
  if (CAUSAL) row_lo = max(0, t.n_base - delta - p.hi_off);
  if (p.lo_off < kNoBound) row_hi = min(t.sq, t.n_base + C::BN - delta + p.lo_off);
  t.m_lo = row_lo / C::BM;
  t.m_hi = (row_hi + C::BM - 1) / C::BM;
  if (row_hi <= row_lo || t.m_lo > t.m_hi) t.m_hi = t.m_lo;
  t.n_iter = t.G * (t.m_hi - t.m_lo);
  return true;
}

// ---------------------------------------------------------------------------
// TMA warp
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void bwd_load(const BwdParams& p, const BwdTile& t, const BwdSmem& s,
                                         const CUtensorMap* tmK, const CUtensorMap* tmV,
                                         const CUtensorMap* tmQ, const CUtensorMap* tmO) {
  // all 32 lanes: lane 0 issues the copies, every lane fills part of the
  // per-block LSE (log2 domain) and D_i vectors and arrives on qdo_full
  using C = BwdCfg<D>;
  if (t.n_iter == 0) return;
  const int lane = lane_id();
  if (lane == 0) {
    mbar_expect_tx(s.kv_full, 2 * C::PANELS * C::KV_PANEL);
    for (int pn = 0; pn < C::PANELS; ++pn) {
      tma_load_3d(s.k + pn * C::KV_PANEL, tmK, s.kv_full, pn * 64, t.hk, t.k0 + t.n_base);
      tma_load_3d(s.v + pn * C::KV_PANEL, tmV, s.kv_full, pn * 64, t.hk, t.k0 + t.n_base);
    }
  }
  const int mcount = t.m_hi - t.m_lo;
  int issued = 0;
  // LSE (log2 domain) and D_i for rows lane and lane + 32 of block i, loaded
  // one block ahead so their global-memory latency overlaps the waits
  auto fetch = [&](int i, float (&l2)[2], float (&dl)[2]) {
    const int h = t.h0 + i / mcount;
    const int m0 = (t.m_lo + i % mcount) * C::BM;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int qrow = m0 + lane + 32 * u;
      l2[u] = INFINITY;  // rows outside the segment, or rows that saw no key: P = 0
      dl[u] = 0.f;
      if (qrow < t.sq) {
        const size_t idx = static_cast<size_t>(h) * p.total_q + t.q0 + qrow;
        const float l = p.lse[idx];
        if (l != -INFINITY) l2[u] = l * 1.4426950408889634f;
        dl[u] = p.delta[idx];
      }
    }
  };
  float nl2[2], ndl[2];
  fetch(0, nl2, ndl);
  for (int i = 0; i < t.n_iter; ++i) {
    const int st = i % C::NST;
    if constexpr (C::NSPLIT == 2) {
      // the other head_dim half of Q_i and dO_i: free once S and dP of block
      // i-1 are done, long before the own half
      if (i >= 1 && !__all_sync(0xffffffffu,
                                mbar_wait(s.oth_empty, (i - 1) & 1, s.abort, p.err,
                                          ERR_BWD_LOAD | 2, p.timeout_ns)))
        break;
      if (lane == 0) {
        const int h = t.h0 + i / mcount;
        const int row = t.q0 + (t.m_lo + i % mcount) * C::BM;
        mbar_expect_tx(s.oth_full, 4 * C::QD_PANEL);
        for (int pp = 0; pp < 2; ++pp) {
          const int pn = 2 * (1 - t.dh) + pp;
          tma_load_3d(s.st + pn * C::QD_PANEL, tmQ, s.oth_full, pn * 64, h, row);
          tma_load_3d(s.st + (C::PANELS + pn) * C::QD_PANEL, tmO, s.oth_full, pn * 64, h, row);
        }
      }
      __syncwarp();
    }
    if (i >= C::NST) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s.qdo_empty[st], ((i / C::NST) - 1) & 1, s.abort,
                                             p.err, ERR_BWD_LOAD | 1, p.timeout_ns)))
        break;
    }
    const int h = t.h0 + i / mcount;
    const int m0 = (t.m_lo + i % mcount) * C::BM;
    float* lsd = s.lsd + st * 128;
    lsd[lane] = nl2[0];
    lsd[lane + 32] = nl2[1];
    lsd[64 + lane] = ndl[0];
    lsd[64 + lane + 32] = ndl[1];
    if constexpr (C::NSPLIT == 2) {
      // own head_dim half of Q_i and dO_i (with the LSE/D vectors above); the
      // other half was issued earlier, as soon as S and dP of block i-1 ended
      if (lane == 0) {
        uint8_t* dst = s.st;
        const int row = t.q0 + m0;
        mbar_expect_tx(&s.qdo_full[0], 4 * C::QD_PANEL);
        for (int pp = 0; pp < 2; ++pp) {
          const int pn = 2 * t.dh + pp;
          tma_load_3d(dst + pn * C::QD_PANEL, tmQ, &s.qdo_full[0], pn * 64, h, row);
          tma_load_3d(dst + (C::PANELS + pn) * C::QD_PANEL, tmO, &s.qdo_full[0], pn * 64, h,
                      row);
        }
      } else {
        mbar_arrive(&s.qdo_full[0]);
      }
    } else {
      if (lane == 0) {
        uint8_t* dst = s.st + st * C::STAGE_BYTES;
        const int row = t.q0 + m0;
        mbar_expect_tx(&s.qdo_full[st], C::STAGE_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn) {
          tma_load_3d(dst + pn * C::QD_PANEL, tmQ, &s.qdo_full[st], pn * 64, h, row);
          tma_load_3d(dst + (C::PANELS + pn) * C::QD_PANEL, tmO, &s.qdo_full[st], pn * 64, h,
                      row);
        }
      } else {
        mbar_arrive(&s.qdo_full[st]);
      }
    }
    ++issued;
    // the next block's LSE and D_i, after this block's copies are issued: the
    // warp stalls on these loads where their values are first used
    if (i + 1 < t.n_iter) fetch(i + 1, nl2, ndl);
  }
  if (*s.abort && lane == 0) {
    // let this CTA's own copies land before its shared memory is released
    mbar_wait_drain(s.kv_full, 0, 100000000ull);
    if (C::NSPLIT == 2 && issued > 0) mbar_wait_drain(s.oth_full, (issued - 1) & 1, 100000000ull);
    for (int i = issued > C::NST ? issued - C::NST : 0; i < issued; ++i)
      mbar_wait_drain(&s.qdo_full[i % C::NST], (i / C::NST) & 1, 100000000ull);
  }
}

// ---------------------------------------------------------------------------
// MMA warps (all lanes run the role; one elected lane issues)
// ---------------------------------------------------------------------------
template <int D>
struct BwdMma {
  using C = BwdCfg<D>;
  const BwdParams& p;
  const BwdSmem& s;
  const BwdTile& t;
  uint32_t tmem;
  __device__ BwdMma(const BwdParams& p_, const BwdSmem& s_, const BwdTile& t_, uint32_t tm)
      : p(p_), s(s_), t(t_), tmem(tm) {}

  __device__ bool wait(uint64_t* bar, uint32_t parity, uint32_t code) {
    if (!mbar_wait_warp(bar, parity, s.abort, p.err, ERR_BWD_MMA | code, p.timeout_ns))
      return false;
    tc_fence_after();
    return true;
  }
  // Shared-memory descriptors are built once per call; each MMA then adds its
  // byte offset >> 4 to the start-address field (addresses stay below 256 KB,
  // so the 14-bit field never carries), which keeps the issuing thread to a
  // few instructions per MMA.
  static __device__ __forceinline__ uint64_t at(uint64_t desc, uint32_t bytes) {
    return desc + static_cast<uint64_t>(bytes >> 4);
  }
  // X^T = A B^T with A = K or V (128 keys x D, K-major) and B = Q_i or dO_i (64 x D)
  __device__ void issue_kt(uint32_t d_col, const uint8_t* a, const uint8_t* b) {
    const uint64_t ad = sdesc_sw128(smem_u32(a), 16, 1024), bd = sdesc_sw128(smem_u32(b), 16, 1024);
#pragma unroll
    for (int pn = 0; pn < C::PANELS; ++pn)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + d_col, at(ad, pn * C::KV_PANEL + kk * 32), at(bd, pn * C::QD_PANEL + kk * 32),
               C::IDESC_SDP, (pn | kk) != 0);
  }
  // the K-steps of X^T = A B^T over panels [p0, p0 + 2) only (head_dim 256)
  __device__ void issue_kt_pair(uint32_t d_col, const uint8_t* a, const uint8_t* b, int p0,
                                bool first) {
    const uint64_t ad = sdesc_sw128(smem_u32(a) + p0 * C::KV_PANEL, 16, 1024);
    const uint64_t bd = sdesc_sw128(smem_u32(b) + p0 * C::QD_PANEL, 16, 1024);
#pragma unroll
    for (int pp = 0; pp < 2; ++pp)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem + d_col, at(ad, pp * C::KV_PANEL + kk * 32), at(bd, pp * C::QD_PANEL + kk * 32),
               C::IDESC_SDP, (!first || pp || kk) ? 1u : 0u);
  }
  __device__ void grads(int j, bool first) {
    const int bj = j & 1;
    const uint8_t* stg = s.st + (j % C::NST) * C::STAGE_BYTES;
    const uint64_t qd = sdesc_sw128(smem_u32(stg) + t.dh * 2 * C::QD_PANEL, C::QD_PANEL, 1024);
    const uint64_t dod =
        sdesc_sw128(smem_u32(stg) + (C::PANELS + t.dh * 2) * C::QD_PANEL, C::QD_PANEL, 1024);
    // dV += P^T dO  (A = P^T in tensor memory, B = dO rows, MN-major).  The
    // P of query columns [32 w, 32 w + 32) sits at columns 32 w .. 32 w + 15 of
    // the S buffer, 8 columns per 16-query k-step.
#pragma unroll
    for (int ks = 0; ks < C::BM / 16; ++ks)
      mma_ts(tmem + C::COL_DV, tmem + C::COL_S + bj * 64 + (ks >> 1) * 32 + (ks & 1) * 8,
             at(dod, ks * 2048), C::IDESC_KV, (!first || ks) ? 1u : 0u);
    // dK += dS^T Q  (A = dS^T in tensor memory, 16 columns after each
    // warpgroup's P^T; the shared-memory copy is for dQ)
#pragma unroll
    for (int ks = 0; ks < C::BM / 16; ++ks)
      mma_ts(tmem + C::COL_DK, tmem + C::COL_S + bj * 64 + (ks >> 1) * 32 + 16 + (ks & 1) * 8,
             at(qd, ks * 2048), C::IDESC_KV, (!first || ks) ? 1u : 0u);
  }
  __device__ void dq(int j) {
    const int bj = j & 1;
    const uint64_t kd = sdesc_sw128(smem_u32(s.k) + t.dh * 2 * C::KV_PANEL, C::KV_PANEL, 1024);
    const uint64_t dsd = sdesc_sw128(smem_u32(s.ds + bj * C::DS_BYTES), C::QD_PANEL, 1024);
    // dQ^T = K^T dS^T  (A = K tile read MN-major, B = dS^T MN-major)
#pragma unroll
    for (int ks = 0; ks < C::BN / 16; ++ks)
      mma_ss(tmem + C::COL_DQ, at(kd, ks * 2048), at(dsd, ks * 2048), C::IDESC_DQ, ks ? 1u : 0u);
  }
};

template <int D>
__device__ __forceinline__ void bwd_mma(const BwdParams& p, const BwdTile& t, const BwdSmem& s,
                                        uint32_t tmem, int role) {
  using C = BwdCfg<D>;
  if (t.n_iter == 0) return;
  if (!C::TWO_ISSUERS && role != 0) return;
  BwdMma<D> m(p, s, t, tmem);
  TRACE_INIT();
  if (!m.wait(s.kv_full, 0, 1)) return;
  auto do_grads = [&](int j) -> bool {
    if (!m.wait(&s.ds_ready[j & 1], (j >> 1) & 1, 2)) return false;
    if (j < 200) TRACE(2048 + j * 8 + 4);
    // dV and dK first: they are the last readers of the (Q, dO) stage, which is
    // released right after them so the next load has the most slack
    m.grads(j, j == 0);
    mma_commit(&s.qdo_empty[j % C::NST]);
    mma_commit(&s.s_free[j & 1]);  // the dV MMA has read P^T from the S buffer
    if (j < 200) TRACE(2048 + j * 8 + 5);
    if (j >= 1 && !m.wait(s.dq_free, (j - 1) & 1, 3)) return false;
    if (j < 200) TRACE(2048 + j * 8 + 6);
    m.dq(j);
    mma_commit(s.dq_full);
    mma_commit(&s.ds_free[j & 1]);  // dK and dQ have read the dS buffer
    if (j < 200) TRACE(2048 + j * 8 + 7);
    return true;
  };
  if constexpr (C::NSPLIT == 2) {
    // head_dim 256: the stage's other head_dim half arrives early, so S_i and
    // dP_i start on it while the own half (freed by the dV/dK MMAs of block
    // i-1) is still loading; dQ of block i-1 fills the rest of that gap
    auto grads_part = [&](int j) -> bool {
      if (!m.wait(&s.ds_ready[j & 1], (j >> 1) & 1, 2)) return false;
      m.grads(j, j == 0);
      mma_commit(&s.qdo_empty[0]);
      return true;
    };
    auto dq_part = [&](int j) -> bool {
      if (j >= 1 && !m.wait(s.dq_free, (j - 1) & 1, 3)) return false;
      m.dq(j);
      mma_commit(s.dq_full);
      mma_commit(&s.ds_free[j & 1]);
      return true;
    };
    const int own = 2 * t.dh, oth = 2 * (1 - t.dh);
    for (int i = 0; i < t.n_iter; ++i) {
      if (i >= 1 && !grads_part(i - 1)) return;
      if (!m.wait(s.oth_full, i & 1, 7)) return;
      m.issue_kt_pair(C::COL_S + (i & 1) * 64, s.k, s.st, oth, true);
      if (i >= 1 && !m.wait(s.dp_free, (i - 1) & 1, 5)) return;
      m.issue_kt_pair(C::COL_DP, s.v, s.st + C::PANELS * C::QD_PANEL, oth, true);
      if (i >= 1 && !dq_part(i - 1)) return;
      if (!m.wait(&s.qdo_full[0], i & 1, 4)) return;
      m.issue_kt_pair(C::COL_S + (i & 1) * 64, s.k, s.st, own, false);
      mma_commit(&s.s_full[i & 1]);
      m.issue_kt_pair(C::COL_DP, s.v, s.st + C::PANELS * C::QD_PANEL, own, false);
      mma_commit(s.dp_full);
      mma_commit(s.oth_empty);
    }
    if (!grads_part(t.n_iter - 1) || !dq_part(t.n_iter - 1)) return;
    mma_commit(s.dkv_full);
  } else if (role == 0) {
    // S and dP of every block, running ahead of the gradient MMAs
    for (int i = 0; i < t.n_iter; ++i) {
      const int st = i % C::NST;
      if (!m.wait(&s.qdo_full[st], (i / C::NST) & 1, 4)) return;
      // S buffer (i & 1) held P^T of block i-2, read by that block's dV MMA
      if (i >= 2 && !m.wait(&s.s_free[i & 1], ((i - 2) >> 1) & 1, 8)) return;
      if (i < 200) TRACE(2048 + i * 8 + 0);
      const uint8_t* stg = s.st + st * C::STAGE_BYTES;
      m.issue_kt(C::COL_S + (i & 1) * 64, s.k, stg);
      mma_commit(&s.s_full[i & 1]);
      if (i < 200) TRACE(2048 + i * 8 + 1);
      if (i >= 1 && !m.wait(s.dp_free, (i - 1) & 1, 5)) return;
      if (i < 200) TRACE(2048 + i * 8 + 2);
      m.issue_kt(C::COL_DP, s.v, stg + C::PANELS * C::QD_PANEL);
      mma_commit(s.dp_full);
      if (i < 200) TRACE(2048 + i * 8 + 3);
    }
  } else {
    // dV, dK and dQ of every block.  The (Q, dO) stage of block j is released
    // here: S and dP of block j completed before its dS could be ready.
    for (int j = 0; j < t.n_iter; ++j)
      if (!do_grads(j)) return;
    mma_commit(s.dkv_full);
  }
}

// ---------------------------------------------------------------------------
// elementwise warps: thread = key row
// ---------------------------------------------------------------------------
template <int D, bool CAUSAL, bool SOFTCAP>
__device__ __forceinline__ void bwd_elem(const BwdParams& p, const BwdTile& t, const BwdSmem& s,
                                         uint32_t tmem, const CUtensorMap* tmDQ) {
  // two warpgroups: warpgroup wg handles query columns [32 wg, 32 wg + 32) of
  // every block; within a warpgroup, thread = key row = TMEM lane
  using C = BwdCfg<D>;
  const int tid = threadIdx.x;       // 0..255
  const int wg = tid >> 7;
  const int row = tid & 127;         // key row within the block / TMEM lane
  const int wq = row >> 5;           // lane quadrant of this warp
  const int lane = tid & 31;
  const int qc0 = wg * 32;           // first query column of this warpgroup
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const int kr = t.n_base + row;     // segment-local key row
  const bool key_ok = kr < t.sk;
  const int mcount = t.m_hi - t.m_lo;
  const float c = p.scale_log2;
  const int causal_off = t.sk - t.sq;
  bool ok = true;
  TRACE_INIT();
  auto uniform_wait = [&](uint64_t* bar, uint32_t parity, uint32_t code) -> bool {
    const bool r = __all_sync(0xffffffffu, mbar_wait(bar, parity, s.abort, p.err,
                                                       ERR_BWD_ELEM | code, p.timeout_ns));
    if (r) tc_fence_after();
    return r;
  };
  // dQ^T of iteration j, this warpgroup's 32 query columns: thread = feature d.
  // With DQ_TMA each warp stages 32 queries x 32 features in shared memory and
  // one lane adds the tile into the fp32 accumulator with a TMA reduce; query
  // rows beyond the segment hold exact zeros (their P is 0), so adding them is
  // harmless.
  auto dq_out = [&](int j) -> bool {
    if (!uniform_wait(s.dq_full, j & 1, 1)) return false;
    const int h = t.h0 + j / mcount;
    const int m0 = (t.m_lo + j % mcount) * C::BM;
    const bool d_ok = row < C::DH;
    uint32_t r0[32];
    tmem_ld32(tmem + lane_base + C::COL_DQ + qc0, r0);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(s.dq_free);
    if constexpr (C::DQ_TMA) {
      if (d_ok) {
        // slots: (DH / 32) per warpgroup; only warps with d < DH stage
        float* stg =
            reinterpret_cast<float*>(s.dqs + (wg * (C::DH / 32) + wq) * C::DQ_WARP_BYTES);
        if (lane == 0) bulk_wait_read0();  // the previous reduce has read the buffer
        __syncwarp();
#pragma unroll
        for (int x = 0; x < 32; ++x) stg[x * 32 + lane] = __uint_as_float(r0[x]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(tmDQ, stg, t.dh * C::DH + wq * 32, h, t.q0 + m0 + qc0);
          bulk_commit();
        }
      }
    } else {
      const int rows = min(C::BM, t.sq - m0) - qc0;
      const size_t off = (static_cast<size_t>(t.q0 + m0 + qc0) * p.nheads_q + h) * D +
                         t.dh * C::DH + row;
      const size_t row_stride = static_cast<size_t>(p.nheads_q) * D;
      if (d_ok && p.dq_out != nullptr) {
        // the CTA's key block is the whole key segment: store the finished rows
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (x < rows) p.dq_out[off + x * row_stride] = bf16_bits(__uint_as_float(r0[x]) * p.scale);
      } else if (d_ok) {
        float* acc = p.dq_acc + off;
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (x < rows) atomicAdd(acc + x * row_stride, __uint_as_float(r0[x]));
      }
    }
    return true;
  };

  for (int i = 0; i < t.n_iter && ok; ++i) {
    const int b = i & 1;
    const int m0 = (t.m_lo + i % mcount) * C::BM;
    if (!uniform_wait(&s.qdo_full[i % C::NST], (i / C::NST) & 1, 6) ||
        !uniform_wait(&s.s_full[b], (i >> 1) & 1, 2) || !uniform_wait(s.dp_full, i & 1, 3)) {
      ok = false;
      break;
    }
    if (tid == 0 && i < 200) TRACE(i * 8 + 0);
    const float* lse2 = s.lsd + (i % C::NST) * 128 + qc0;  // LSE in the log2 domain
    const float* dlt = s.lsd + (i % C::NST) * 128 + 64 + qc0;  // D_i
    // lane x reads the LSE and D_i of query column x and the pair loop takes
    // them from that lane by shuffles: a read of one value by all 32 lanes costs
    // a shared-memory wavefront per value (measured ~2% slower at head_dim 128)
    const float lse_lane = lse2[lane], d_lane = dlt[lane];
    uint32_t sr[32], dr[32];
    tmem_ld32x2(tmem + lane_base + C::COL_S + b * 64 + qc0, sr, tmem + lane_base + C::COL_DP + qc0,
                dr);
    tc_fence_before();
    if (tid == 0 && i < 200) TRACE(i * 8 + 1);
    __syncwarp();
    if (lane == 0) mbar_arrive(s.dp_free);
    // query column x of this block (row m0 + qc0 + x) sees this key iff
    // x in [xmin, xmax]: kr <= row + delta + hi_off and kr >= row + delta - lo_off
    const int xmin = CAUSAL ? (kr - causal_off - p.hi_off - m0 - qc0) : -kNoBound;
    const int xmax = (p.lo_off < kNoBound) ? (kr - causal_off + p.lo_off - m0 - qc0) : kNoBound;
    uint32_t pk[16];
    uint4 dsk[4];
    const uint64_t c2 = f2_pack(c, c);
    // most warps have all 32 query columns of every lane allowed: only the
    // others run the per-element mask.  The choice is warp-uniform, so the
    // shuffles below are met by every lane (a lane-wise choice would split the
    // warp across the two loop bodies and their separate shuffle sites)
    const bool all_in = __all_sync(0xffffffffu, key_ok && xmin <= 0 && xmax >= 31);
    auto pairs = [&](auto masked_tag) {
    constexpr bool MASKED = decltype(masked_tag)::value;
#pragma unroll
    for (int x4 = 0; x4 < 8; ++x4) {
      float4 l4, d4;
      l4.x = __shfl_sync(0xffffffffu, lse_lane, x4 * 4 + 0);
      l4.y = __shfl_sync(0xffffffffu, lse_lane, x4 * 4 + 1);
      l4.z = __shfl_sync(0xffffffffu, lse_lane, x4 * 4 + 2);
      l4.w = __shfl_sync(0xffffffffu, lse_lane, x4 * 4 + 3);
      d4.x = __shfl_sync(0xffffffffu, d_lane, x4 * 4 + 0);
      d4.y = __shfl_sync(0xffffffffu, d_lane, x4 * 4 + 1);
      d4.z = __shfl_sync(0xffffffffu, d_lane, x4 * 4 + 2);
      d4.w = __shfl_sync(0xffffffffu, d_lane, x4 * 4 + 3);
#pragma unroll
      for (int hp = 0; hp < 2; ++hp) {
        const int x = x4 * 4 + hp * 2;
        float e0, e1;
        float g0 = 1.f, g1 = 1.f;  // d(capped score) / d(scaled score)
        if constexpr (SOFTCAP) {
          const float t0 = tanh_from_ex2(__uint_as_float(sr[x]) * p.cap_k2);
          const float t1 = tanh_from_ex2(__uint_as_float(sr[x + 1]) * p.cap_k2);
          e0 = p.cap_log2 * t0 - (hp ? l4.z : l4.x);
          e1 = p.cap_log2 * t1 - (hp ? l4.w : l4.y);
          g0 = 1.f - t0 * t0;
          g1 = 1.f - t1 * t1;
        } else {
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[x]), __uint_as_float(sr[x + 1])), c2,
                           hp ? f2_pack(-l4.z, -l4.w) : f2_pack(-l4.x, -l4.y)),
                    e0, e1);
        }
        float p0 = ex2(e0), p1 = ex2(e1);
        if (MASKED) {
          if (!key_ok || x < xmin || x > xmax) p0 = 0.f;
          if (!key_ok || x + 1 < xmin || x + 1 > xmax) p1 = 0.f;
        }
        float d0, d1;
        f2_unpack(f2_mul(f2_pack(p0 * g0, p1 * g1),
                         f2_add(f2_pack(__uint_as_float(dr[x]), __uint_as_float(dr[x + 1])),
                                hp ? f2_pack(-d4.z, -d4.w) : f2_pack(-d4.x, -d4.y))),
                  d0, d1);
        pk[x >> 1] = pack_bf16(p0, p1);
        const uint32_t dpk = pack_bf16(d0, d1);
        const int w = (x >> 1) & 3;
        if (w == 0) dsk[x >> 3].x = dpk;
        else if (w == 1) dsk[x >> 3].y = dpk;
        else if (w == 2) dsk[x >> 3].z = dpk;
        else dsk[x >> 3].w = dpk;
      }
    }
    };
    if (all_in)
      pairs(std::integral_constant<bool, false>());
    else
      pairs(std::integral_constant<bool, true>());
    // P (bf16 pairs) goes over the first 16 of this warpgroup's own 32 score
    // columns, which this warpgroup has already read: the other warpgroup may
    // still be reading its own columns
    tmem_st16(tmem + lane_base + C::COL_S + b * 64 + wg * 32, pk);
    {
      // dS^T (bf16 pairs) over the other 16 of the warpgroup's own columns: the
      // A operand of dK += dS^T Q, read from tensor memory
      uint32_t dsw[16];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        dsw[4 * ch] = dsk[ch].x;
        dsw[4 * ch + 1] = dsk[ch].y;
        dsw[4 * ch + 2] = dsk[ch].z;
        dsw[4 * ch + 3] = dsk[ch].w;
      }
      tmem_st16(tmem + lane_base + C::COL_S + b * 64 + wg * 32 + 16, dsw);
    }
    if (tid == 0 && i < 200) TRACE(i * 8 + 2);
    // the dS buffer b is free once the dK and dQ MMAs of block i-2 are done
    if (i >= 2 && !uniform_wait(&s.ds_free[b], ((i - 2) >> 1) & 1, 4)) {
      ok = false;
      break;
    }
    uint8_t* dsrow = s.ds + b * C::DS_BYTES + row * 128;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch)
      *reinterpret_cast<uint4*>(dsrow + (((wg * 4 + ch) ^ (row & 7)) * 16)) = dsk[ch];
    tmem_st_wait();
    fence_async_smem();
    tc_fence_before();
    if (tid == 0 && i < 200) TRACE(i * 8 + 3);
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.ds_ready[b]);
    if (!C::DQ_WARPS && i >= 1 && !dq_out(i - 1)) {
      ok = false;
      break;
    }
    if (tid == 0 && i < 200) TRACE(i * 8 + 4);
  }
  if (!C::DQ_WARPS && ok && t.n_iter > 0) ok = dq_out(t.n_iter - 1);
  if constexpr (C::DQ_TMA && !C::DQ_WARPS) {
    if (lane == 0) bulk_wait0();  // this warp's reduces are complete
  }
  if (ok && t.n_iter > 0) ok = uniform_wait(s.dkv_full, 0, 5);
  if (!ok) return;
  // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (x scale), bf16.
  // The TMEM loads are warp-collective, so every lane runs them; only valid
  // key rows store.
  const size_t grow = static_cast<size_t>(t.k0 + (key_ok ? kr : 0));
  const size_t off = ((grow * p.nheads_kv + t.hk) * D + t.dh * C::DH) * 2;
  uint8_t* dst = static_cast<uint8_t*>(wg ? p.dk : p.dv) + off;
  const float f = wg ? p.scale : 1.f;
  const int col0 = wg ? C::COL_DK : C::COL_DV;
#pragma unroll 1
  for (int cc = 0; cc < C::DH / 32; ++cc) {
    uint32_t r[32];
    if (t.n_iter > 0) {
      tmem_ld32(tmem + lane_base + col0 + cc * 32, r);
    } else {
#pragma unroll
      for (int x = 0; x < 32; ++x) r[x] = 0u;
    }
    if (key_ok) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint4 v;
        v.x = pack_bf16(__uint_as_float(r[g * 8 + 0]) * f, __uint_as_float(r[g * 8 + 1]) * f);
        v.y = pack_bf16(__uint_as_float(r[g * 8 + 2]) * f, __uint_as_float(r[g * 8 + 3]) * f);
        v.z = pack_bf16(__uint_as_float(r[g * 8 + 4]) * f, __uint_as_float(r[g * 8 + 5]) * f);
        v.w = pack_bf16(__uint_as_float(r[g * 8 + 6]) * f, __uint_as_float(r[g * 8 + 7]) * f);
        *reinterpret_cast<uint4*>(dst + (cc * 32 + g * 8) * 2) = v;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// dQ warpgroup (head_dim 64/128): warp wq reads features [32 wq, 32 wq + 32) of
// dQ^T (TMEM lane = feature) for all 64 query columns of a block and adds them
// into the fp32 accumulator with TMA reduce-adds, 32 queries at a time.
// Query rows past the segment carry exact zeros (their P is 0).
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void bwd_dq(const BwdParams& p, const BwdTile& t, const BwdSmem& s,
                                       uint32_t tmem, const CUtensorMap* tmDQ) {
  using C = BwdCfg<D>;
  const int wq = (threadIdx.x >> 5) & 3;
  const int lane = lane_id();
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const int mcount = t.m_hi - t.m_lo;
  const bool d_ok = wq * 32 < C::DH;  // head_dim 64: lanes 64-127 hold the zero panel
  for (int j = 0; j < t.n_iter; ++j) {
    if (!__all_sync(0xffffffffu, mbar_wait(s.dq_full, j & 1, s.abort, p.err, ERR_BWD_ELEM | 1,
                                           p.timeout_ns)))
      break;
    tc_fence_after();
    const int h = t.h0 + j / mcount;
    const int m0 = (t.m_lo + j % mcount) * C::BM;
    uint32_t r0[32], r1[32];
    tmem_ld32x2(tmem + lane_base + C::COL_DQ, r0, tmem + lane_base + C::COL_DQ + 32, r1);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(s.dq_free);
    if (!d_ok) continue;
    if (p.dq_out != nullptr) {
      // the CTA's key block is the whole key segment: these rows' dQ is
      // complete, so store scale * dQ (bf16) for the rows inside the segment;
      // lane = feature, so each store covers 64 contiguous bytes of a row
      const int rows = min(C::BM, t.sq - m0);
      const size_t row_stride = static_cast<size_t>(p.nheads_q) * D;
      uint16_t* dst = p.dq_out + (static_cast<size_t>(t.q0 + m0) * p.nheads_q + h) * D +
                      t.dh * C::DH + wq * 32 + lane;
      // one running pointer, and r0 dead before r1 is stored: within this
      // warpgroup's register budget
#pragma unroll
      for (int x = 0; x < 32; ++x, dst += row_stride)
        if (x < rows) *dst = bf16_bits(__uint_as_float(r0[x]) * p.scale);
#pragma unroll
      for (int x = 0; x < 32; ++x, dst += row_stride)
        if (x + 32 < rows) *dst = bf16_bits(__uint_as_float(r1[x]) * p.scale);
      continue;
    }
#pragma unroll
    for (int hq = 0; hq < 2; ++hq) {
      float* stg = reinterpret_cast<float*>(s.dqs + (hq * (C::DH / 32) + wq) * C::DQ_WARP_BYTES);
      // this slot's previous reduce (one group before the other slot's) has read it
      if (lane == 0) bulk_wait_read1();
      __syncwarp();
#pragma unroll
      for (int x = 0; x < 32; ++x) stg[x * 32 + lane] = __uint_as_float(hq ? r1[x] : r0[x]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_3d(tmDQ, stg, t.dh * C::DH + wq * 32, h, t.q0 + m0 + hq * 32);
        bulk_commit();
      }
    }
  }
  if (lane == 0) bulk_wait0();  // every reduce of this warp is complete
}

template <int D, bool CAUSAL, bool SOFTCAP>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
    attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmO,
                         const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BwdTile t;
  if (!bwd_tile<D, CAUSAL>(p, t)) return;
  const BwdSmem s = bwd_smem<D>(base);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(s.kv_full, 1);
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&s.qdo_full[i], 32);
      mbar_init(&s.qdo_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.ds_ready[i], C::ELEM_THREADS / 32);
      mbar_init(&s.ds_free[i], 1);
      mbar_init(&s.s_free[i], 1);
    }
    mbar_init(s.dp_full, 1);
    mbar_init(s.dp_free, C::ELEM_THREADS / 32);
    mbar_init(s.dq_full, 1);
    mbar_init(s.dq_free, C::DQ_WARPS ? 4 : C::ELEM_THREADS / 32);
    mbar_init(s.dkv_full, 1);
    mbar_init(s.oth_full, 1);
    mbar_init(s.oth_empty, 1);
    *s.abort = 0;
    fence_mbar_init();
  }
  if (D == 64 && warp < 8) {
    // zero panel after the K tile: the dQ^T MMA reads head_dim 64 as M = 128
    uint4* z = reinterpret_cast<uint4*>(s.k + C::PANELS * C::KV_PANEL);
    for (int i = threadIdx.x; i < C::KV_PANEL / 16; i += C::ELEM_THREADS)
      z[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
  }
  if (warp == C::LOAD_WARP && lane_id() == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_base;
  // each warpgroup sets its register budget in the branch it then runs (every
  // warp of a warpgroup executes the same setmaxnreg)
  if (warp < 8) {
    if constexpr (C::DQ_WARPS) setmaxnreg_inc<C::REG_ELEM>();
    bwd_elem<D, CAUSAL, SOFTCAP>(p, t, s, tmem, &tmDQ);
  } else if (!C::DQ_WARPS || warp < C::DQ_WARP0) {
    if constexpr (C::DQ_WARPS) setmaxnreg_dec<C::REG_CTRL>();
    if (warp == C::LOAD_WARP) {
      bwd_load<D>(p, t, s, &tmK, &tmV, &tmQ, &tmO);
    } else if (warp == C::MMA_WARP || warp == C::GRAD_WARP) {
      bwd_mma<D>(p, t, s, tmem, warp - C::MMA_WARP);  // the whole warp; one lane issues
    }
  } else {
    if constexpr (C::DQ_WARPS) {
      setmaxnreg_dec<C::REG_DQ>();
      bwd_dq<D>(p, t, s, tmem, &tmDQ);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// preprocess: D_i = dO_i . O_i, zero the dQ accumulator (or, with direct dQ
// stores, the bf16 dQ itself)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(const uint16_t* __restrict__ out,
                                                           const uint16_t* __restrict__ dout,
                                                           float* __restrict__ delta,
                                                           float* __restrict__ dq_acc,
                                                           uint16_t* __restrict__ dq_zero,
                                                           int total_q, int hq) {
  constexpr int TPR = D / 8;  // threads per (row, head), 8 elements each
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rh = gid / TPR;  // (row, head) index in [Tq][Hq] order
  const int part = static_cast<int>(gid % TPR);
  const long long n_rh = static_cast<long long>(total_q) * hq;
  float acc = 0.f;
  if (rh < n_rh) {
    const uint4 a = *reinterpret_cast<const uint4*>(out + rh * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + rh * D + part * 8);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(bv[i] << 16), acc);
      acc = fmaf(__uint_as_float(av[i] & 0xffff0000u), __uint_as_float(bv[i] & 0xffff0000u), acc);
    }
    if (dq_zero != nullptr) {
      // direct dQ: rows that see no key are never stored by the main kernel
      *reinterpret_cast<uint4*>(dq_zero + rh * D + part * 8) = make_uint4(0u, 0u, 0u, 0u);
    } else {
      float4* z = reinterpret_cast<float4*>(dq_acc + rh * D + part * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, TPR);
  if (rh < n_rh && part == 0) {
    const long long row = rh / hq;
    const int h = static_cast<int>(rh % hq);
    delta[static_cast<long long>(h) * total_q + row] = acc;
  }
}

// postprocess: dQ = scale * accumulator -> bf16
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float* __restrict__ acc,
                                                          uint16_t* __restrict__ dq,
                                                          long long n8, float scale) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 o;
    o.x = pack_bf16(a.x * scale, a.y * scale);
    o.y = pack_bf16(a.z * scale, a.w * scale);
    o.z = pack_bf16(b.x * scale, b.y * scale);
    o.w = pack_bf16(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = o;
  }
}

}  // namespace attn

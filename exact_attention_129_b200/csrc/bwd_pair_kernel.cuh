// bwd_pair_kernel.cuh -- the backward main kernel for head_dim 256 as a pair of
// CTAs (a thread-block cluster of two) that split the work of one 128-key block
// by role, so that no product is computed twice.
//
// The method (P = exp(S - LSE) recomputed from the forward's LSE, dS = P (dP - D),
// dV = P^T dO, dK = dS^T Q, dQ = dS K; the FA4 repository guide, Backward
// Kernels) needs, per 128-key x 64-query block, five products of equal size.
// At head_dim 256 the two 128 x 256 fp32 accumulators dK and dV alone fill the
// 512 columns of one SM's tensor memory, so one CTA cannot hold both next to S,
// dP and dQ.  Here the two CTAs of a cluster take the same key block:
//
//   rank 0 ("Q side"):  K in tensor memory, Q streamed.   S^T = K Q^T,
//                       P^T = 2^(S^T c - LSE'), dK += dS^T Q, dQ^T[0:128) = K^T dS^T
//   rank 1 ("dO side"): V in tensor memory, dO streamed.  dP^T = V dO^T,
//                       dS^T = P^T (dP^T - D), dV += P^T dO, dQ^T[128:256) = K^T dS^T
//
// and exchange the two bf16 tiles the other side needs: P^T goes from rank 0 to
// rank 1 and dS^T from rank 1 to rank 0, 16 KB each per block, as shared-to-
// shared bulk copies whose completion lands on the receiver's mbarrier (the
// copy engine moves them; stores from the elementwise warps into the peer's
// shared memory measured 1600-2000 cycles per tile of those warps' time).  Each
// rank issues about the same MMA work (one 256-deep N = 64 product, one
// N = 256 gradient product and half of dQ), the minimal total.  Buffer-free
// signals travel back as tcgen05.commit arrives on the peer's mbarrier.  The
// K or V tile is the A operand of S or dP straight from tensor memory, so
// shared memory holds only this rank's 128 columns of K (for dQ), the Q or dO
// stages and the exchange tiles.
//
// Per CTA: tensor memory  K or V (128 cols, bf16 pairs) | S^T or dP^T (64) |
//                         dQ^T half (64) | dK or dV (256)            = 512 cols
//          shared memory  K half 32 KB | 3 stages x 32 KB | XA x2 | XB x2 (16 KB
//                         each) | dQ staging 32 KB | LSE' or D_i | barriers
//          warps          0-7 elementwise (thread = key row; warpgroup wg takes
//                         query columns [32 wg, 32 wg + 32)), 8 TMA loader,
//                         9 MMA (S or dP), 10 MMA (gradients and dQ),
//                         11 exchange (bulk copies to the peer), 12-15 dQ readout
//                         (TMA reduce-add into the fp32 accumulator)
// XA holds P^T (rank 0 writes it, rank 1 receives it); XB holds dS^T (rank 1
// writes it, rank 0 receives it); both CTAs use the same offsets, so a buffer
// or barrier of the peer is the same offset mapped into the peer's window.
//
// Softcap needs the score at rank 1 as well and is left to the head_dim-split
// kernel in bwd_kernels.cuh; local windows and causal masks are applied to P on
// rank 0 (dS = P (dP - D) is then zero wherever P is).
#pragma once

#include "bwd_kernels.cuh"

namespace attn {

// Trace slots (ATTN_TRACE builds only) of block i < 200, per role:
// elementwise 4i + {0 tile in registers, 1 P or dS computed, 2 exchange buffer
// free, 3 tile written}; MMA A 800 + 2i + {0 issue, 1 committed}; MMA B
// 1200 + 4i + {0 peer tile landed, 1 gradient issued, 2 dQ inputs ready,
// 3 dQ committed}; exchange 2000 + 2i + {0 tile written, 1 copy issued};
// dQ 2400 + 2i + {0 dQ^T ready, 1 added}; loader 2800 + 2i + {0 stage free,
// 1 loads issued}.
enum : uint32_t {
  ERR_BWDP_LOAD = 0x0A00,
  ERR_BWDP_MMA = 0x0B00,
  ERR_BWDP_ELEM = 0x0C00,
  ERR_BWDP_XCHG = 0x0D00,
  ERR_BWDP_DQ = 0x0E00,
};

struct PairCfg {
  static constexpr int D = 256, BN = 128, BM = 64, PANELS = 4;
  static constexpr int KV_PANEL = BN * 128;               // 16 KB: 128 rows x 64 cols
  static constexpr int QD_PANEL = BM * 128;               // 8 KB: 64 rows x 64 cols
  static constexpr int STAGE_BYTES = PANELS * QD_PANEL;   // 32 KB: Q or dO, 64 rows x 256
  // Q stages (rank 0) and dO stages (rank 1).  Rank 0 holds a Q stage from S
  // until dK, after the round trip of P^T and dS^T through rank 1, the longest
  // hold in the pair; rank 1 holds a dO stage only until P^T arrives.  A
  // fourth Q stage fits only with a single P^T send buffer, and waiting for
  // that buffer measured slower than the third stage (676 against 752 TF/s).
  static constexpr int NST0 = 3, NST1 = 3;
  static constexpr int NST = NST0;
  static constexpr int X_BYTES = BN * BM * 2;             // 16 KB: 128 keys x 64 queries bf16
  static constexpr int DQ_SLOT = 32 * 32 * 4;             // 4 KB: 32 features x 32 queries
  static constexpr int OFF_KH = 0;
  static constexpr int OFF_ST = OFF_KH + 2 * KV_PANEL;
  static constexpr int OFF_XA = OFF_ST + NST * STAGE_BYTES;
  static constexpr int OFF_XB = OFF_XA + 2 * X_BYTES;
  static constexpr int OFF_DQS = OFF_XB + 2 * X_BYTES;    // 2 slots per dQ warp
  static constexpr int OFF_LSD = OFF_DQS + 8 * DQ_SLOT;   // NST x 64 floats
  static constexpr int OFF_BAR = OFF_LSD + NST * BM * 4;
  // st_empty counts the S or dP MMA, the gradient MMA and the 8 elementwise
  // warps (which read the block's LSE' or D_i from this stage's slot).
  // kv_full, a_ready, st_full[NST], st_empty[NST], s_full, s_free, xa_full[2],
  // xa_written[2], xa_free[2], xb_full[2], xb_written[2], xb_free[2], xb_done[2],
  // dq_full, dq_free, dkv_full, drain[2]
  static constexpr int NBAR = 2 + 2 * NST + 2 + 14 + 3 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static constexpr int COL_A = 0, COL_S = 128, COL_DQ = 192, COL_G = 256;
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BM, false, false);
  static constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);
  static constexpr uint32_t IDESC_DQ = idesc_bf16(128, BM, true, true);
  static constexpr int THREADS = 512;
  static constexpr int LOAD_WARP = 8, MMA_A_WARP = 9, MMA_B_WARP = 10, XCHG_WARP = 11;
  static constexpr int DQ_WARP0 = 12;
  // 16 warps launch with 128 registers each; per SM sub-partition one warp of
  // each warpgroup: 184 + 184 + 64 + 80 = 512 registers per lane, its file
  static constexpr int REG_ELEM = 184, REG_CTRL = 64, REG_DQ = 80;
  static_assert(2 * REG_ELEM + REG_CTRL + REG_DQ <= 512, "register split");
};

struct PairSmem {
  uint8_t *kh, *st, *xa, *xb, *dqs;
  float* lsd;
  uint64_t *kv_full, *a_ready, *st_full, *st_empty, *s_full, *s_free, *xa_full, *xa_written,
      *xa_free, *xb_full, *xb_written, *xb_free, *xb_done, *dq_full, *dq_free, *dkv_full, *drain;
  uint32_t* tmem_base;
  volatile int* abort;
};

__device__ __forceinline__ uint8_t* pair_stage(const PairSmem& s, int st) {
  return s.st + st * PairCfg::STAGE_BYTES;
}

// (slot, phase parity) of a ring, advanced one block at a time
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  int n;
  __device__ explicit Ring(int n_) : n(n_) {}
  __device__ void next() {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

__device__ __forceinline__ PairSmem pair_smem(uint8_t* base) {
  using C = PairCfg;
  PairSmem s;
  s.kh = base + C::OFF_KH;
  s.st = base + C::OFF_ST;
  s.xa = base + C::OFF_XA;
  s.xb = base + C::OFF_XB;
  s.dqs = base + C::OFF_DQS;
  s.lsd = reinterpret_cast<float*>(base + C::OFF_LSD);
  uint64_t* b = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  s.kv_full = b;
  s.a_ready = b + 1;
  s.st_full = b + 2;
  s.st_empty = s.st_full + C::NST;
  s.s_full = s.st_empty + C::NST;
  s.s_free = s.s_full + 1;
  s.xa_full = s.s_free + 1;
  s.xa_written = s.xa_full + 2;
  s.xa_free = s.xa_written + 2;
  s.xb_full = s.xa_free + 2;
  s.xb_written = s.xb_full + 2;
  s.xb_free = s.xb_written + 2;
  s.xb_done = s.xb_free + 2;
  s.dq_full = s.xb_done + 2;
  s.dq_free = s.dq_full + 1;
  s.dkv_full = s.dq_free + 1;
  s.drain = s.dkv_full + 1;
  s.tmem_base = reinterpret_cast<uint32_t*>(base + C::OFF_MISC);
  s.abort = reinterpret_cast<volatile int*>(base + C::OFF_MISC + 4);
  return s;
}

// The cluster's key block and the query blocks that can see it (both ranks
// compute the same tile).
template <bool CAUSAL>
__device__ __forceinline__ bool pair_tile(const BwdParams& p, BwdTile& t) {
  using C = PairCfg;
  const int b = blockIdx.z;
  t.hk = blockIdx.y;
  t.G = p.nheads_q / p.nheads_kv;
  t.h0 = t.hk * t.G;
  t.dh = 0;
  t.q0 = p.cu_q[b];
  t.sq = p.cu_q[b + 1] - t.q0;
  t.k0 = p.cu_k[b];
  t.sk = p.cu_k[b + 1] - t.k0;
  t.n_base = (blockIdx.x >> 1) * C::BN;
  if (t.n_base >= t.sk) return false;
  const int delta = t.sk - t.sq;
  int row_lo = 0, row_hi = t.sq;
  if (CAUSAL) row_lo = max(0, t.n_base - delta - p.hi_off);
  if (p.lo_off < kNoBound) row_hi = min(t.sq, t.n_base + C::BN - delta + p.lo_off);
  t.m_lo = row_lo / C::BM;
  t.m_hi = (row_hi + C::BM - 1) / C::BM;
  if (row_hi <= row_lo || t.m_lo > t.m_hi) t.m_hi = t.m_lo;
  t.n_iter = t.G * (t.m_hi - t.m_lo);
  return true;
}

// Bounded waits that, on giving up, also stop the peer CTA (its roles then
// leave their loops at their next wait).
struct PairWait {
  volatile int* abort;
  uint32_t* err;
  uint64_t timeout_ns;
  uint32_t peer_abort;  // shared::cluster address of the peer's abort flag
  __device__ bool lane(uint64_t* bar, uint32_t parity, uint32_t code) const {
    if (mbar_wait_cluster(bar, parity, abort, err, code, timeout_ns)) return true;
    st_cluster_u32(peer_abort, 1u);
    return false;
  }
  // every lane waits; one outcome for the warp
  __device__ bool warp(uint64_t* bar, uint32_t parity, uint32_t code) const {
    const bool ok = __all_sync(0xffffffffu, lane(bar, parity, code));
    if (ok) tc_fence_after();
    return ok;
  }
};

// ---------------------------------------------------------------------------
// TMA warp: this rank's K columns once; per block the Q (rank 0) or dO (rank 1)
// rows of all 256 columns and the block's LSE' (rank 0) or D_i (rank 1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pair_load(const BwdParams& p, const BwdTile& t, const PairSmem& s,
                                          const PairWait& w, uint32_t rank, const CUtensorMap* tmK,
                                          const CUtensorMap* tmQO) {
  using C = PairCfg;
  if (t.n_iter == 0) return;
  const int lane = lane_id();
  if (lane == 0) {
    mbar_expect_tx(s.kv_full, 2 * C::KV_PANEL);
    for (int pp = 0; pp < 2; ++pp)
      tma_load_3d(s.kh + pp * C::KV_PANEL, tmK, s.kv_full, (2 * rank + pp) * 64, t.hk,
                  t.k0 + t.n_base);
  }
  const int mcount = t.m_hi - t.m_lo;
  auto fetch = [&](int i, float (&v)[2]) {
    const int h = t.h0 + i / mcount;
    const int m0 = (t.m_lo + i % mcount) * C::BM;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int qrow = m0 + lane + 32 * u;
      // rows outside the segment or without any key: P = 0 (LSE' = +inf), D = 0
      v[u] = rank == 0 ? INFINITY : 0.f;
      if (qrow < t.sq) {
        const size_t idx = static_cast<size_t>(h) * p.total_q + t.q0 + qrow;
        if (rank == 0) {
          const float l = p.lse[idx];
          if (l != -INFINITY) v[u] = l * 1.4426950408889634f;
        } else {
          v[u] = p.delta[idx];
        }
      }
    }
  };
  const int nst = rank == 0 ? C::NST0 : C::NST1;
  float nv[2];
  fetch(0, nv);
  int issued = 0;
  Ring r(nst);
  TRACE_INIT();
  for (int i = 0; i < t.n_iter; ++i, r.next()) {
    // the slot's previous block released it (phase parity of that use)
    if (i >= nst && !w.warp(&s.st_empty[r.slot], r.phase ^ 1u, ERR_BWDP_LOAD | 1)) break;
    if (lane == 0 && i < 200) TRACE(2800 + 2 * i);
    float* lsd = s.lsd + r.slot * C::BM;
    lsd[lane] = nv[0];
    lsd[lane + 32] = nv[1];
    const int h = t.h0 + i / mcount;
    const int row = t.q0 + (t.m_lo + i % mcount) * C::BM;
    uint8_t* dst = pair_stage(s, r.slot);
    if (lane == 0) {
      mbar_expect_tx(&s.st_full[r.slot], C::STAGE_BYTES);
      for (int pn = 0; pn < C::PANELS; ++pn)
        tma_load_3d(dst + pn * C::QD_PANEL, tmQO, &s.st_full[r.slot], pn * 64, h, row);
    } else {
      mbar_arrive(&s.st_full[r.slot]);
    }
    if (lane == 0 && i < 200) TRACE(2800 + 2 * i + 1);
    ++issued;
    // the next block's LSE' or D_i, after this block's copies are issued: the
    // warp stalls on these loads where their values are first used
    if (i + 1 < t.n_iter) fetch(i + 1, nv);
  }
  if (*s.abort && lane == 0) {
    // let this CTA's own copies land before its shared memory is released
    mbar_wait_drain(s.kv_full, 0, 100000000ull);
    for (int i = issued > nst ? issued - nst : 0; i < issued; ++i)
      mbar_wait_drain(&s.st_full[i % nst], (i / nst) & 1, 100000000ull);
  }
}

// ---------------------------------------------------------------------------
// MMA warps (the whole warp runs the role; one elected lane issues)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t pair_at(uint64_t desc, uint32_t bytes) {
  return desc + static_cast<uint64_t>(bytes >> 4);
}

// warp 9: S^T = K Q^T (rank 0) or dP^T = V dO^T (rank 1), A from tensor memory
__device__ __forceinline__ void pair_mma_a(const BwdTile& t, const PairSmem& s, const PairWait& w,
                                           uint32_t tmem, uint32_t rank) {
  using C = PairCfg;
  if (t.n_iter == 0) return;
  TRACE_INIT();
  bool ok = w.warp(s.a_ready, 0, ERR_BWDP_MMA | 1);
  Ring r(rank == 0 ? C::NST0 : C::NST1);
  for (int i = 0; ok && i < t.n_iter; ++i, r.next()) {
    if (!w.warp(&s.st_full[r.slot], r.phase, ERR_BWDP_MMA | 2) ||
        (i >= 1 && !w.warp(s.s_free, (i - 1) & 1, ERR_BWDP_MMA | 3))) {
      ok = false;
      break;
    }
    if (lane_id() == 0 && i < 200) TRACE(800 + 2 * i);
    const uint64_t bd = sdesc_sw128(smem_u32(pair_stage(s, r.slot)), 16, 1024);
#pragma unroll
    for (int ks = 0; ks < 16; ++ks)
      mma_ts(tmem + C::COL_S, tmem + C::COL_A + ks * 8,
             pair_at(bd, (ks >> 2) * C::QD_PANEL + (ks & 3) * 32), C::IDESC_S, ks ? 1u : 0u);
    mma_commit(s.s_full);
    mma_commit(&s.st_empty[r.slot]);  // this warp's read of the stage
    if (lane_id() == 0 && i < 200) TRACE(800 + 2 * i + 1);
  }
  if (!ok) {
    // let the MMAs already issued finish before tensor memory is released
    mma_commit(&s.drain[0]);
    mbar_wait_drain(&s.drain[0], 0, 100000000ull);
  }
}

// warp 10: the gradient products and this rank's half of dQ^T
__device__ __forceinline__ void pair_mma_b(const BwdTile& t, const PairSmem& s, const PairWait& w,
                                           uint32_t tmem, uint32_t rank, volatile int* rx_done) {
  using C = PairCfg;
  if (t.n_iter == 0) return;
  const uint16_t peer_mask = static_cast<uint16_t>(1u << (rank ^ 1u));
  const int lane = lane_id();
  bool ok = w.warp(s.kv_full, 0, ERR_BWDP_MMA | 4);
  const uint64_t kd = sdesc_sw128(smem_u32(s.kh), C::KV_PANEL, 1024);
  Ring r(rank == 0 ? C::NST0 : C::NST1);
  TRACE_INIT();
  for (int j = 0; ok && j < t.n_iter; ++j, r.next()) {
    const int b = j & 1;
    // the tile from the peer: dS^T (rank 0) or P^T (rank 1), by bulk copy
    uint64_t* rx_full = rank == 0 ? &s.xb_full[b] : &s.xa_full[b];
    if (!w.warp(rx_full, (j >> 1) & 1, ERR_BWDP_MMA | 5)) {
      ok = false;
      break;
    }
    if (lane == 0 && j < 200) TRACE(1200 + 4 * j);
    if (lane == 0) {
      *rx_done = j + 1;
      // arm the buffer for block j + 2 before the peer can learn it is free
      if (j + 2 < t.n_iter) mbar_expect_tx(rx_full, C::X_BYTES);
    }
    __syncwarp();
    const uint8_t* rx = (rank == 0 ? s.xb : s.xa) + b * C::X_BYTES;
    // dK += dS^T Q (rank 0) or dV += P^T dO (rank 1): A = the 128 x 64 tile
    // (K-major), B = the stage's 64 x 256 rows (MN-major), N = 256
    const uint64_t ad = sdesc_sw128(smem_u32(rx), 16, 1024);
    const uint64_t gd = sdesc_sw128(smem_u32(pair_stage(s, r.slot)), C::QD_PANEL, 1024);
#pragma unroll
    for (int ks = 0; ks < C::BM / 16; ++ks)
      mma_ss(tmem + C::COL_G, pair_at(ad, ks * 32), pair_at(gd, ks * 2048), C::IDESC_G,
             (j > 0 || ks > 0) ? 1u : 0u);
    mma_commit(&s.st_empty[r.slot]);  // this warp's read of the stage
    if (lane == 0 && j < 200) TRACE(1200 + 4 * j + 1);
    // dS^T of this block: received (rank 0) or written here by the elementwise
    // warps (rank 1)
    if (rank == 1 && !w.warp(&s.xb_written[b], (j >> 1) & 1, ERR_BWDP_MMA | 6)) {
      ok = false;
      break;
    }
    if (j >= 1 && !w.warp(s.dq_free, (j - 1) & 1, ERR_BWDP_MMA | 7)) {
      ok = false;
      break;
    }
    if (lane == 0 && j < 200) TRACE(1200 + 4 * j + 2);
    // dQ^T of this rank's 128 features = K^T dS^T (A = K columns MN-major,
    // B = dS^T MN-major), N = 64 queries, 128 keys deep
    const uint64_t dsd = sdesc_sw128(smem_u32(s.xb + b * C::X_BYTES), C::QD_PANEL, 1024);
#pragma unroll
    for (int ks = 0; ks < C::BN / 16; ++ks)
      mma_ss(tmem + C::COL_DQ, pair_at(kd, ks * 2048), pair_at(dsd, ks * 2048), C::IDESC_DQ,
             ks ? 1u : 0u);
    mma_commit(s.dq_full);
    if (rank == 0) {
      // rank 1 may send dS^T of block j + 2 into XB[b]
      mma_commit_to(&s.xb_free[b], peer_mask);
    } else {
      mma_commit(&s.xb_done[b]);  // XB[b] read by dQ
      // rank 0 may store P^T of block j + 2 into XA[b]: dV has read it, and
      // the elementwise warps read it before they wrote dS^T
      mma_commit_to(&s.xa_free[b], peer_mask);
    }
    if (lane == 0 && j < 200) TRACE(1200 + 4 * j + 3);
  }
  if (ok) {
    mma_commit(s.dkv_full);
  } else {
    mma_commit(&s.drain[1]);
    mbar_wait_drain(&s.drain[1], 0, 100000000ull);
  }
}

// ---------------------------------------------------------------------------
// exchange warp: sends this rank's tile of each block to the peer.  At the end
// it waits for the peer's last release signals, so no arrive is still on its
// way into this CTA when the cluster exits
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pair_xchg(const BwdTile& t, const PairSmem& s, const PairWait& w,
                                          uint32_t rank, const volatile int* rx_done) {
  using C = PairCfg;
  if (t.n_iter == 0) return;
  const int lane = lane_id();
  int sent = 0;
  TRACE_INIT();
  uint8_t* tx = rank == 0 ? s.xa : s.xb;
  uint64_t* tx_written = rank == 0 ? s.xa_written : s.xb_written;
  const uint32_t peer = rank ^ 1u;
  const uint32_t peer_tx = mapa_shared(smem_u32(tx), peer);
  const uint32_t peer_bar = mapa_shared(smem_u32(rank == 0 ? s.xa_full : s.xb_full), peer);
  for (int i = 0; i < t.n_iter; ++i) {
    const int b = i & 1;
    if (!w.warp(&tx_written[b], (i >> 1) & 1, ERR_BWDP_XCHG | 1)) break;
    if (lane == 0 && i < 200) TRACE(2000 + 2 * i);
    if (lane == 0)
      bulk_copy_to_peer(peer_tx + b * C::X_BYTES, tx + b * C::X_BYTES, C::X_BYTES, peer_bar + b * 8);
    __syncwarp();
    if (lane == 0 && i < 200) TRACE(2000 + 2 * i + 1);
    ++sent;
  }
  if (lane == 0) {
    // the peer releases each block it received; the elementwise warps consumed
    // the releases up to block n_iter - 3, these are the rest
    uint64_t* tx_free = rank == 0 ? s.xa_free : s.xb_free;
    const uint64_t bound = *s.abort ? 1000000ull : 2000000000ull;
    for (int j = sent > 2 ? sent - 2 : 0; j < sent; ++j)
      if (!mbar_wait_drain(&tx_free[j & 1], (j >> 1) & 1, bound)) break;
    if (*s.abort) {
      // tiles from the peer that may still be landing here
      uint64_t* rx_full = rank == 0 ? s.xb_full : s.xa_full;
      for (int j = *rx_done; j < t.n_iter; ++j)
        if (!mbar_wait_drain(&rx_full[j & 1], (j >> 1) & 1, 1000000ull)) break;
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// elementwise warps: thread = key row (tensor-memory lane)
// ---------------------------------------------------------------------------
template <bool CAUSAL>
__device__ __forceinline__ void pair_elem(const BwdParams& p, const BwdTile& t, const PairSmem& s,
                                          const PairWait& w, uint32_t tmem, uint32_t rank,
                                          const uint16_t* kv_src) {
  using C = PairCfg;
  const int tid = threadIdx.x;  // 0..255
  const int wg = tid >> 7;
  const int row = tid & 127;
  const int wq = row >> 5;
  const int lane = tid & 31;
  const int qc0 = wg * 32;
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const int kr = t.n_base + row;
  const bool key_ok = kr < t.sk;
  const int mcount = t.m_hi - t.m_lo;
  bool ok = true;
  if (t.n_iter > 0) {
    // K (rank 0) or V (rank 1) rows into tensor memory, the A operand of S^T or
    // dP^T: column c of lane r holds elements 2c, 2c + 1 of key row r (the low
    // half the even one, which is the memory order); warpgroup wg writes
    // elements [128 wg, 128 wg + 128)
    const uint4* src = reinterpret_cast<const uint4*>(
        kv_src + (static_cast<size_t>(t.k0 + (key_ok ? kr : 0)) * p.nheads_kv + t.hk) * C::D +
        wg * 128);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t wv[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 x = key_ok ? __ldg(src + half * 8 + c) : make_uint4(0u, 0u, 0u, 0u);
        wv[4 * c] = x.x;
        wv[4 * c + 1] = x.y;
        wv[4 * c + 2] = x.z;
        wv[4 * c + 3] = x.w;
      }
      tmem_st32(tmem + lane_base + C::COL_A + wg * 64 + half * 32, wv);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(s.a_ready);
  }
  const float c = p.scale_log2;
  const int causal_off = t.sk - t.sq;
  TRACE_INIT();
  uint8_t* xrow_a = s.xa + row * 128;
  uint8_t* xrow_b = s.xb + row * 128;
  Ring r(rank == 0 ? C::NST0 : C::NST1);
  for (int i = 0; i < t.n_iter && ok; ++i, r.next()) {
    const int b = i & 1;
    const int m0 = (t.m_lo + i % mcount) * C::BM;
    if (!w.warp(&s.st_full[r.slot], r.phase, ERR_BWDP_ELEM | 1) ||
        !w.warp(s.s_full, i & 1, ERR_BWDP_ELEM | 2)) {
      ok = false;
      break;
    }
    // lane x holds the LSE' (rank 0) or D_i (rank 1) of query column qc0 + x;
    // the warp's last read of the stage slot
    const float v_lane = s.lsd[r.slot * C::BM + qc0 + lane];
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.st_empty[r.slot]);
    uint32_t sr[32];
    tmem_ld32(tmem + lane_base + C::COL_S + qc0, sr);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(s.s_free);
    if (tid == 0 && i < 200) TRACE(4 * i);
    uint4 out[4];
    if (rank == 0) {
      // P^T = 2^(S^T c - LSE') with the masks
      const int xmin = CAUSAL ? (kr - causal_off - p.hi_off - m0 - qc0) : -kNoBound;
      const int xmax = (p.lo_off < kNoBound) ? (kr - causal_off + p.lo_off - m0 - qc0) : kNoBound;
      const bool all_in = __all_sync(0xffffffffu, key_ok && xmin <= 0 && xmax >= 31);
      const uint64_t c2 = f2_pack(c, c);
      uint32_t pk[16];
      auto pairs = [&](auto masked_tag) {
        constexpr bool MASKED = decltype(masked_tag)::value;
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float l0 = __shfl_sync(0xffffffffu, v_lane, x);
          const float l1 = __shfl_sync(0xffffffffu, v_lane, x + 1);
          float e0, e1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[x]), __uint_as_float(sr[x + 1])), c2,
                           f2_pack(-l0, -l1)),
                    e0, e1);
          float p0 = ex2(e0), p1 = ex2(e1);
          if (MASKED) {
            if (!key_ok || x < xmin || x > xmax) p0 = 0.f;
            if (!key_ok || x + 1 < xmin || x + 1 > xmax) p1 = 0.f;
          }
          pk[x >> 1] = pack_bf16(p0, p1);
        }
      };
      if (all_in)
        pairs(std::integral_constant<bool, false>());
      else
        pairs(std::integral_constant<bool, true>());
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        out[ch] = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      if (tid == 0 && i < 200) TRACE(4 * i + 1);
      // XA[b] held P^T of block i - 2 until rank 1 released it
      if (i >= 2 && !w.warp(&s.xa_free[b], ((i - 2) >> 1) & 1, ERR_BWDP_ELEM | 3)) {
        ok = false;
        break;
      }
    } else {
      // dS^T = P^T (dP^T - D) with P^T from rank 0
      if (!w.warp(&s.xa_full[b], (i >> 1) & 1, ERR_BWDP_ELEM | 4)) {
        ok = false;
        break;
      }
      uint4 pv[4];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        pv[ch] = *reinterpret_cast<const uint4*>(xrow_a + b * C::X_BYTES +
                                                 (((wg * 4 + ch) ^ (row & 7)) * 16));
      const uint32_t pw[16] = {pv[0].x, pv[0].y, pv[0].z, pv[0].w, pv[1].x, pv[1].y,
                               pv[1].z, pv[1].w, pv[2].x, pv[2].y, pv[2].z, pv[2].w,
                               pv[3].x, pv[3].y, pv[3].z, pv[3].w};
      uint32_t dk[16];
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        const float d0 = __shfl_sync(0xffffffffu, v_lane, x);
        const float d1 = __shfl_sync(0xffffffffu, v_lane, x + 1);
        const uint32_t pp = pw[x >> 1];
        float g0, g1;
        f2_unpack(f2_mul(f2_pack(__uint_as_float(pp << 16), __uint_as_float(pp & 0xffff0000u)),
                         f2_add(f2_pack(__uint_as_float(sr[x]), __uint_as_float(sr[x + 1])),
                                f2_pack(-d0, -d1))),
                  g0, g1);
        dk[x >> 1] = pack_bf16(g0, g1);
      }
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        out[ch] = make_uint4(dk[4 * ch], dk[4 * ch + 1], dk[4 * ch + 2], dk[4 * ch + 3]);
      if (tid == 0 && i < 200) TRACE(4 * i + 1);
      // XB[b] held dS^T of block i - 2: read by this CTA's dQ and by the copy
      // to rank 0, which released it after its own MMAs
      if (i >= 2 && (!w.warp(&s.xb_done[b], ((i - 2) >> 1) & 1, ERR_BWDP_ELEM | 5) ||
                     !w.warp(&s.xb_free[b], ((i - 2) >> 1) & 1, ERR_BWDP_ELEM | 6))) {
        ok = false;
        break;
      }
    }
    // the 128 B row of this key (64 queries, 128-byte swizzle): the K-major A
    // operand of the gradient product and the MN-major B operand of dQ^T
    if (tid == 0 && i < 200) TRACE(4 * i + 2);
    uint8_t* xrow = (rank == 0 ? xrow_a : xrow_b) + b * C::X_BYTES;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch)
      *reinterpret_cast<uint4*>(xrow + (((wg * 4 + ch) ^ (row & 7)) * 16)) = out[ch];
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(rank == 0 ? &s.xa_written[b] : &s.xb_written[b]);
    if (tid == 0 && i < 200) TRACE(4 * i + 3);
  }
  if (ok && t.n_iter > 0) ok = w.warp(s.dkv_full, 0, ERR_BWDP_ELEM | 7);
  if (!ok) return;
  // epilogue: dK x scale (rank 0) or dV (rank 1) in bf16; warpgroup wg writes
  // elements [128 wg, 128 wg + 128) of its key row
  const size_t grow = static_cast<size_t>(t.k0 + (key_ok ? kr : 0));
  uint8_t* dst = static_cast<uint8_t*>(rank == 0 ? p.dk : p.dv) +
                 ((grow * p.nheads_kv + t.hk) * C::D + wg * 128) * 2;
  const float f = rank == 0 ? p.scale : 1.f;
#pragma unroll 1
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t r[32];
    if (t.n_iter > 0) {
      tmem_ld32(tmem + lane_base + C::COL_G + wg * 128 + cc * 32, r);
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
// dQ warps: warp wq reads features [32 wq, 32 wq + 32) of this rank's dQ^T half
// (tensor-memory lane = feature) for the 64 queries of a block and adds them
// into the fp32 accumulator with TMA reduce-adds, or, when the key block is
// the whole key segment, stores scale * dQ as bf16.  Query rows past the
// segment carry exact zeros (their P is 0).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pair_dq(const BwdParams& p, const BwdTile& t, const PairSmem& s,
                                        const PairWait& w, uint32_t tmem, uint32_t rank,
                                        const CUtensorMap* tmDQ) {
  using C = PairCfg;
  const int wq = (threadIdx.x >> 5) & 3;
  const int lane = lane_id();
  const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
  const int mcount = t.m_hi - t.m_lo;
  const int feat0 = static_cast<int>(rank) * 128 + wq * 32;
  TRACE_INIT();
  for (int j = 0; j < t.n_iter; ++j) {
    if (!w.warp(s.dq_full, j & 1, ERR_BWDP_DQ | 1)) break;
    if (wq == 0 && lane == 0 && j < 200) TRACE(2400 + 2 * j);
    const int h = t.h0 + j / mcount;
    const int m0 = (t.m_lo + j % mcount) * C::BM;
    uint32_t r0[32], r1[32];
    tmem_ld32x2(tmem + lane_base + C::COL_DQ, r0, tmem + lane_base + C::COL_DQ + 32, r1);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(s.dq_free);
    if (p.dq_out != nullptr) {
      const int rows = min(C::BM, t.sq - m0);
      const size_t row_stride = static_cast<size_t>(p.nheads_q) * C::D;
      uint16_t* dst = p.dq_out + (static_cast<size_t>(t.q0 + m0) * p.nheads_q + h) * C::D +
                      feat0 + lane;
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
      float* stg = reinterpret_cast<float*>(s.dqs + (hq * 4 + wq) * C::DQ_SLOT);
      if (lane == 0) bulk_wait_read1();  // this slot's previous reduce has read it
      __syncwarp();
#pragma unroll
      for (int x = 0; x < 32; ++x) stg[x * 32 + lane] = __uint_as_float(hq ? r1[x] : r0[x]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_3d(tmDQ, stg, feat0, h, t.q0 + m0 + hq * 32);
        bulk_commit();
      }
    }
    if (wq == 0 && lane == 0 && j < 200) TRACE(2400 + 2 * j + 1);
  }
  if (lane == 0) bulk_wait0();
}

template <bool CAUSAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::THREADS, 1)
    attn_bwd_pair_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmO,
                         const __grid_constant__ CUtensorMap tmDQ, const BwdParams p,
                         const uint16_t* __restrict__ k, const uint16_t* __restrict__ v) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BwdTile t;
  // both CTAs of the cluster see the same tile, so they leave together
  if (!pair_tile<CAUSAL>(p, t)) return;
  const uint32_t rank = cluster_ctarank();
  const PairSmem s = pair_smem(base);
  volatile int* rx_done = reinterpret_cast<volatile int*>(base + C::OFF_MISC + 8);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(s.kv_full, 1);
    mbar_init(s.a_ready, 8);
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&s.st_full[i], 32);
      mbar_init(&s.st_empty[i], 2 + 8);
    }
    mbar_init(s.s_full, 1);
    mbar_init(s.s_free, 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s.xa_full[b], 1);
      mbar_init(&s.xa_written[b], 8);
      mbar_init(&s.xa_free[b], 1);
      mbar_init(&s.xb_full[b], 1);
      mbar_init(&s.xb_written[b], 8);
      mbar_init(&s.xb_free[b], 1);
      mbar_init(&s.xb_done[b], 1);
      mbar_init(&s.drain[b], 1);
    }
    mbar_init(s.dq_full, 1);
    mbar_init(s.dq_free, 4);
    mbar_init(s.dkv_full, 1);
    *s.abort = 0;
    *rx_done = 0;
    // the receive barriers of the first two blocks are armed before the peer
    // can send anything (the cluster barrier below orders it)
    uint64_t* rx_full = rank == 0 ? s.xb_full : s.xa_full;
    for (int b = 0; b < 2 && b < t.n_iter; ++b) mbar_expect_tx(&rx_full[b], C::X_BYTES);
    fence_mbar_init();
  }
  if (warp == C::LOAD_WARP && lane_id() == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(rank == 0 ? &tmQ : &tmO);
  }
  if (warp == C::MMA_A_WARP) {
    tmem_alloc(s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist and are armed
  tc_fence_after();
  const uint32_t tmem = *s.tmem_base;
  PairWait w;
  w.abort = s.abort;
  w.err = p.err;
  w.timeout_ns = p.timeout_ns;
  w.peer_abort = mapa_shared(smem_u32(const_cast<int*>(s.abort)), rank ^ 1u);
  if (warp < 8) {
    setmaxnreg_inc<C::REG_ELEM>();
    pair_elem<CAUSAL>(p, t, s, w, tmem, rank, rank == 0 ? k : v);
  } else if (warp < C::DQ_WARP0) {
    setmaxnreg_dec<C::REG_CTRL>();
    if (warp == C::LOAD_WARP)
      pair_load(p, t, s, w, rank, &tmK, rank == 0 ? &tmQ : &tmO);
    else if (warp == C::MMA_A_WARP)
      pair_mma_a(t, s, w, tmem, rank);
    else if (warp == C::MMA_B_WARP)
      pair_mma_b(t, s, w, tmem, rank, rx_done);
    else
      pair_xchg(t, s, w, rank, rx_done);
  } else {
    setmaxnreg_dec<C::REG_DQ>();
    pair_dq(p, t, s, w, tmem, rank, &tmDQ);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // nothing of either CTA still targets the other
  if (warp == C::MMA_A_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn

// fwd_pair_kernel.cuh -- the forward on a pair of CTAs that share every
// tensor-core instruction (tcgen05 cta_group::2), for head_dim 128 and 256.
//
// A cluster of two CTAs works on 256 query rows, 128 per CTA, over 128-key
// blocks, and the even CTA issues M = 256 MMAs that run on both SMs:
//
//   S = Q K^T   A = each CTA's own 128 Q rows, B = K of the block, 64 keys held
//               by each CTA; D = each CTA's 128 rows x 128 keys (N = 128)
//   O += P V    A = each CTA's P in tensor memory, B = V of the block, D/2 of
//               the columns held by each CTA; D = each CTA's 128 rows x D
//
// so every MMA has N >= 128 and each SM reads half of every B operand and
// loads half of every K/V block.  The loads of both CTAs complete on the even
// CTA's barriers (TMA with cta_group::2, no multicast); its MMA warp commits
// each MMA group to the same barrier in both CTAs.  Softmax: eight warps per
// CTA, each over 16 whole rows (16-lane tensor-memory accesses, four threads
// per row that combine the row's max and sum by shuffles), so no warp waits
// for another's scores; P (bf16) goes over the first 64 columns of its S
// buffer, and each softmax warp of either CTA reports its P to the even CTA's
// barrier, because the P.V MMA reads both CTAs' P.
//
//   head_dim 128: tensor memory S x3 (128 columns each: S(j + 2) is computed
//     while the softmax works on S(j) and P(j + 1) waits for its P.V) + O (128);
//     shared memory Q (32 KB) + a ring of (K half of block j, V half of block
//     j - 1) stages (32 KB each); two issuing warps (S, P.V).  The one-CTA
//     kernel (an S MMA of N = 64 costs ~56 cycles for 32 of work) stays the
//     default there: both are bound by the softmax warps' exps; selected by
//     ATTN_FWD_PAIR=1.
//   head_dim 256 (the default there, without softcap or SplitKV): S x2 + O
//     (256); Q (64 KB) + a ring of 16 KB chunks in MMA order; one issuing warp.
//     The one-CTA kernel is bound by shared-memory reads, which the pair halves.
#pragma once

#include "fwd_kernel.cuh"

namespace attn {

enum : uint32_t {
  ERR_FWDP_LOAD = 0x0F00,
  ERR_FWDP_MMA = 0x1000,
  ERR_FWDP_SOFTMAX = 0x1100,
};

template <int D_>
struct FwdPairCfg;

// head_dim 128: stages of (K half, V half), three S buffers, two issuing warps
template <>
struct FwdPairCfg<128> {
  static constexpr int D = 128, BM = 128, BN = 128, PANELS = D / 64;
  static constexpr int QPANEL = BM * 128;            // 16 KB: 128 rows x 64 columns
  static constexpr int Q_BYTES = BM * D * 2;         // 32 KB
  static constexpr int KH_PANEL = (BN / 2) * 128;    // 8 KB: this CTA's 64 keys x 64 columns
  static constexpr int KH_BYTES = PANELS * KH_PANEL;  // 16 KB
  static constexpr int VH_BYTES = BN * 128;          // 16 KB: 128 keys x this CTA's 64 columns
  static constexpr int STAGE_BYTES = KH_BYTES + VH_BYTES;
  static constexpr int NSTAGE = 5;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NSTAGE * STAGE_BYTES;
  static constexpr int NS = 3;                       // S buffers
  // q_full, kv_full[NSTAGE], kv_empty[NSTAGE], s_full[NS], p_full[NS],
  // o_ready[2] (by block parity), o_final, s_free[NS]
  static constexpr int NBAR = 1 + 2 * NSTAGE + 2 * NS + 2 + 1 + NS;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static constexpr int COL_O = NS * BN;              // S buffers at columns 0, 128, 256
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16(256, BN, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16(256, D, false, true);
  // two issuing warps, S on SM sub-partition 1 and P.V on sub-partition 2: a
  // warp that issues an MMA waits for it, and one warp issuing both took half
  // the issue time of the two softmax warps on its sub-partition
  static constexpr int SOFTMAX_WARPS = 8, LOAD_WARP = 8, MMA_WARP = 9, PV_WARP = 10;
  static constexpr int THREADS = 352;
};

// head_dim 256: 16 KB chunks in MMA consumption order (K of blocks 0 and 1,
// then V of block g before K of block g + 2), two S buffers, one issuing warp.
// Per block and CTA: K half = 2 chunks of 64 keys x 128 columns (two K-major
// panels), V half = 2 chunks of 64 keys x this CTA's 128 columns (two MN-major
// panels).  Tensor memory: S x2 (128 columns) + O (256) = 512.
template <>
struct FwdPairCfg<256> {
  static constexpr int D = 256, BM = 128, BN = 128, PANELS = D / 64;
  static constexpr int QPANEL = BM * 128;            // 16 KB: 128 rows x 64 columns
  static constexpr int Q_BYTES = BM * D * 2;         // 64 KB
  static constexpr int CHUNK = 64 * 256;             // 16 KB: 64 rows x two 128-byte panels
  static constexpr int CPANEL = 64 * 128;            // 8 KB: one panel of a chunk
  static constexpr int NSTAGE = 9;                   // one chunk per stage
  static constexpr int STAGE_BYTES = CHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NSTAGE * STAGE_BYTES;
  static constexpr int NS = 2;
  static constexpr int NBAR = 1 + 2 * NSTAGE + 2 * NS + 2 + 1 + NS;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static constexpr int COL_O = NS * BN;              // S buffers at columns 0, 128
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16(256, BN, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16(256, D, false, true);
  static constexpr int SOFTMAX_WARPS = 8, LOAD_WARP = 8, MMA_WARP = 9;
  static constexpr int THREADS = 320;
};

struct FwdPairSmem {
  uint8_t *q, *ring;
  uint64_t *q_full, *kv_full, *kv_empty, *s_full, *p_full, *o_ready, *o_final, *s_free;
  uint32_t* tmem_base;
  volatile int* abort;
};

template <int D>
__device__ __forceinline__ FwdPairSmem fwd_pair_smem(uint8_t* base) {
  using C = FwdPairCfg<D>;
  FwdPairSmem s;
  s.q = base + C::OFF_Q;
  s.ring = base + C::OFF_RING;
  uint64_t* b = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  s.q_full = b;
  s.kv_full = b + 1;
  s.kv_empty = s.kv_full + C::NSTAGE;
  s.s_full = s.kv_empty + C::NSTAGE;
  s.p_full = s.s_full + C::NS;
  s.o_ready = s.p_full + C::NS;
  s.o_final = s.o_ready + 2;
  s.s_free = s.o_final + 1;
  s.tmem_base = reinterpret_cast<uint32_t*>(base + C::OFF_MISC);
  s.abort = reinterpret_cast<volatile int*>(base + C::OFF_MISC + 4);
  return s;
}

// The pair's key-block range covers both CTAs' rows (rows of the pair that do
// not see a block get P = 0 there); t.m_base is this CTA's first row.
template <int D, bool CAUSAL>
__device__ __forceinline__ bool fwd_pair_tile(const FwdParams& p, FwdTile& t, uint32_t rank) {
  using C = FwdPairCfg<D>;
  const int b = blockIdx.z;
  t.split = 0;
  if (p.pack_shift > 0) {
    t.hk = blockIdx.y;
    t.h = t.hk << p.pack_shift;
  } else {
    t.h = blockIdx.y;
    t.hk = t.h / (p.nheads_q / p.nheads_kv);
  }
  t.rows = C::BM >> p.pack_shift;
  t.q0 = p.cu_q[b];
  t.sq = p.cu_q[b + 1] - t.q0;
  t.k0 = p.cu_k[b];
  t.sk = p.cu_k[b + 1] - t.k0;
  const int n_pairs = gridDim.x >> 1;
  const int pair = CAUSAL ? (n_pairs - 1 - static_cast<int>(blockIdx.x >> 1))
                          : static_cast<int>(blockIdx.x >> 1);
  const int pair_base = pair * 2 * t.rows;
  if (pair_base >= t.sq) return false;  // both CTAs of the pair leave together
  t.m_base = pair_base + static_cast<int>(rank) * t.rows;
  const int delta = t.sk - t.sq;
  int n_end = t.sk;
  if (CAUSAL) {
    const int last_row = min(t.sq, pair_base + 2 * t.rows) - 1;
    n_end = min(t.sk, last_row + delta + p.hi_off + 1);
  }
  const int n_beg = (p.lo_off < kNoBound) ? max(0, pair_base + delta - p.lo_off) : 0;
  t.n_lo = n_beg / C::BN;
  t.n_blocks = n_end > n_beg ? (n_end + C::BN - 1) / C::BN - t.n_lo : 0;
  return true;
}

// ---------------------------------------------------------------------------
// producer warp (lane 0): this CTA's Q tile once, then its halves of the K/V
// blocks; every copy completes on the even CTA's barrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwd_pair_load(const FwdParams& p, const FwdTile& t,
                                              const FwdPairSmem& s, uint32_t rank,
                                              const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                              const CUtensorMap* tmV) {
  using C = FwdPairCfg<128>;
  const int n = t.n_blocks;
  if (n == 0) return;
  if (rank == 0) mbar_expect_tx(s.q_full, 2 * C::Q_BYTES);
  const uint32_t q_bar = mapa_shared(smem_u32(s.q_full), 0);
  for (int pn = 0; pn < C::PANELS; ++pn)
    tma_load_3d_pair(s.q + pn * C::QPANEL, tmQ, q_bar, pn * 64, t.h, t.q0 + t.m_base);
  uint32_t ring = 0;
  // after a timed-out wait: the even CTA, whose barriers count both CTAs' bytes,
  // lets every issued copy land before it leaves (the cluster barrier at the
  // end holds the odd CTA until then)
  auto drain = [&]() {
    if (rank != 0) return;
    mbar_wait_drain(s.q_full, 0, 100000000ull);
    const uint32_t first = ring > (uint32_t)C::NSTAGE ? ring - C::NSTAGE : 0u;
    for (uint32_t r = first; r < ring; ++r)
      mbar_wait_drain(&s.kv_full[r % C::NSTAGE], (r / C::NSTAGE) & 1, 100000000ull);
  };
  for (int j = 0; j <= n; ++j) {
    const uint32_t st = ring % C::NSTAGE;
    // the stage's previous use is done once the even CTA's MMAs have read it
    if (ring >= (uint32_t)C::NSTAGE &&
        !mbar_wait_cluster(&s.kv_empty[st], ((ring / C::NSTAGE) - 1) & 1, s.abort, p.err,
                           ERR_FWDP_LOAD | 1, p.timeout_ns)) {
      drain();
      return;
    }
    if (rank == 0)
      mbar_expect_tx(&s.kv_full[st], (j < n ? 2 * C::KH_BYTES : 0) + (j > 0 ? 2 * C::VH_BYTES : 0));
    const uint32_t bar = mapa_shared(smem_u32(&s.kv_full[st]), 0);
    uint8_t* base = s.ring + st * C::STAGE_BYTES;
    if (j < n)  // this CTA's 64 keys of K_j, all columns
      for (int pn = 0; pn < C::PANELS; ++pn)
        tma_load_3d_pair(base + pn * C::KH_PANEL, tmK, bar, pn * 64, t.hk,
                         t.k0 + (t.n_lo + j) * C::BN + static_cast<int>(rank) * (C::BN / 2));
    if (j > 0)  // this CTA's 64 columns of V_{j-1}, all 128 keys
      tma_load_3d_pair(base + C::KH_BYTES, tmV, bar, static_cast<int>(rank) * 64, t.hk,
                       t.k0 + (t.n_lo + j - 1) * C::BN);
    ++ring;
  }
}

// ---------------------------------------------------------------------------
// MMA warps of the even CTA (all lanes run them; one elected lane issues):
// role 0 issues S(j) for every block, role 1 P(j).V for every block
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwd_pair_mma(const FwdParams& p, const FwdTile& t,
                                             const FwdPairSmem& s, uint32_t tmem, int role) {
  using C = FwdPairCfg<128>;
  const int n = t.n_blocks;
  if (n == 0) return;
  constexpr uint16_t kBoth = 0x3;
  auto wait = [&](uint64_t* bar, uint32_t parity, uint32_t code) -> bool {
    if (!__all_sync(0xffffffffu,
                    mbar_wait_cluster(bar, parity, s.abort, p.err, ERR_FWDP_MMA | code,
                                      p.timeout_ns)))
      return false;
    tc_fence_after();
    return true;
  };
  // stage j holds K_j (read by S(j)) and V_{j-1} (read by P(j-1).V); each
  // role waits for the stages it reads and releases them (kv_empty counts
  // one arrival per role)
  auto stage_of = [&](int idx) { return idx % C::NSTAGE; };
  auto wait_stage = [&](int idx) -> bool {
    return wait(&s.kv_full[stage_of(idx)], (idx / C::NSTAGE) & 1, 2);
  };
  auto stage_base = [&](int idx) { return s.ring + stage_of(idx) * C::STAGE_BYTES; };
  TRACE_INIT();
  if (role == 0) {
    if (!wait(s.q_full, 0, 1)) return;
    const uint64_t qd = sdesc_sw128(smem_u32(s.q), 16, 1024);
    for (int j = 0; j < n; ++j) {
      [[maybe_unused]] const int tr = (j < 64) ? 2048 + 16 * j : -1;
      TRACE(tr);
      if (!wait_stage(j)) return;
      // buffer j % NS held P(j - NS), read by its P.V
      if (j >= C::NS && !wait(&s.s_free[j % C::NS], ((j / C::NS) - 1) & 1, 4)) return;
      TRACE(tr + 1);
      const uint64_t kd = sdesc_sw128(smem_u32(stage_base(j)), 16, 1024);
      const uint32_t d = tmem + (j % C::NS) * C::BN;
#pragma unroll
      for (int c = 0; c < C::PANELS; ++c)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma2_ss(d, qd + ((c * C::QPANEL + kk * 32) >> 4),
                  kd + ((c * C::KH_PANEL + kk * 32) >> 4), C::IDESC_S, (c | kk) ? 1u : 0u);
      mma2_commit_to(&s.s_full[j % C::NS], kBoth);
      mma2_commit_to(&s.kv_empty[stage_of(j)], kBoth);
    }
    // stage n holds only V_{n-1}: this role has nothing to read there
    if (wait_stage(n)) mma2_commit_to(&s.kv_empty[stage_of(n)], kBoth);
  } else {
    // stage 0 holds only K_0
    if (!wait_stage(0)) return;
    mma2_commit_to(&s.kv_empty[stage_of(0)], kBoth);
    for (int j = 0; j < n; ++j) {
      [[maybe_unused]] const int tr = (j < 64) ? 2048 + 16 * j + 8 : -1;
      if (!wait_stage(j + 1)) return;
      if (!wait(&s.p_full[j % C::NS], (j / C::NS) & 1, 3)) return;
      TRACE(tr);
      const uint64_t vd =
          sdesc_sw128(smem_u32(stage_base(j + 1) + C::KH_BYTES), C::VH_BYTES, 1024);
      const uint32_t a = tmem + (j % C::NS) * C::BN;
#pragma unroll
      for (int ks = 0; ks < C::BN / 16; ++ks)
        mma2_ts(tmem + C::COL_O, a + ks * 8, vd + ((ks * 2048) >> 4), C::IDESC_O,
                (j > 0 || ks) ? 1u : 0u);
      mma2_commit_to(&s.o_ready[j & 1], kBoth);
      mma2_commit_to(&s.s_free[j % C::NS], kBoth);
      mma2_commit_to(&s.kv_empty[stage_of(j + 1)], kBoth);
      TRACE(tr + 1);
    }
    mma2_commit_to(s.o_final, kBoth);
  }
}

// ---------------------------------------------------------------------------
// head_dim 256 producer (one lane): this CTA's Q once, then its 16 KB chunks in
// the MMA warp's order (K of blocks 0 and 1, then V of block j before K of
// block j + 2); every copy completes on the even CTA's barrier.  The even CTA,
// whose barriers count both CTAs' bytes, lets every issued copy land before it
// leaves after a timed-out wait; the cluster barrier at the end holds the odd
// CTA until then.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwd_pair256_load(const FwdParams& p, const FwdTile& t,
                                                 const FwdPairSmem& s, uint32_t rank,
                                                 const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                                 const CUtensorMap* tmV) {
  using C = FwdPairCfg<256>;
  const int n = t.n_blocks;
  if (n == 0) return;
  if (rank == 0) mbar_expect_tx(s.q_full, 2 * C::Q_BYTES);
  const uint32_t q_bar = mapa_shared(smem_u32(s.q_full), 0);
  for (int pn = 0; pn < C::PANELS; ++pn)
    tma_load_3d_pair(s.q + pn * C::QPANEL, tmQ, q_bar, pn * 64, t.h, t.q0 + t.m_base);
  uint32_t ring = 0;
  auto drain = [&]() {
    if (rank != 0) return;
    mbar_wait_drain(s.q_full, 0, 100000000ull);
    const uint32_t first = ring > (uint32_t)C::NSTAGE ? ring - C::NSTAGE : 0u;
    for (uint32_t r = first; r < ring; ++r)
      mbar_wait_drain(&s.kv_full[r % C::NSTAGE], (r / C::NSTAGE) & 1, 100000000ull);
  };
  // chunk c (keys [64c, 64c + 64) for V, columns [128c, 128c + 128) for K) of
  // block j, as two 64-column panels
  auto chunk = [&](bool is_v, int j, int c) -> bool {
    const uint32_t st = ring % C::NSTAGE;
    if (ring >= (uint32_t)C::NSTAGE &&
        !mbar_wait_cluster(&s.kv_empty[st], ((ring / C::NSTAGE) - 1) & 1, s.abort, p.err,
                           ERR_FWDP_LOAD | 1, p.timeout_ns)) {
      drain();
      return false;
    }
    if (rank == 0) mbar_expect_tx(&s.kv_full[st], 2 * C::CHUNK);
    const uint32_t bar = mapa_shared(smem_u32(&s.kv_full[st]), 0);
    uint8_t* dst = s.ring + st * C::CHUNK;
    const int key0 = t.k0 + (t.n_lo + j) * C::BN;
    const int r = static_cast<int>(rank);
    for (int pn = 0; pn < 2; ++pn) {
      if (is_v)  // this CTA's columns [128 r + 64 pn, +64)
        tma_load_3d_pair(dst + pn * C::CPANEL, tmV, bar, r * 128 + pn * 64, t.hk, key0 + c * 64);
      else       // this CTA's keys [64 r, 64 r + 64)
        tma_load_3d_pair(dst + pn * C::CPANEL, tmK, bar, c * 128 + pn * 64, t.hk, key0 + r * 64);
    }
    ++ring;
    return true;
  };
  auto block = [&](bool is_v, int j) { return chunk(is_v, j, 0) && chunk(is_v, j, 1); };
  if (!block(false, 0)) return;
  if (n > 1 && !block(false, 1)) return;
  for (int j = 0; j < n; ++j) {
    if (!block(true, j)) return;
    if (j + 2 < n && !block(false, j + 2)) return;
  }
}

// ---------------------------------------------------------------------------
// head_dim 256 MMA warp of the even CTA: S(0), S(1), then P(j).V before
// S(j + 2), each waiting chunk by chunk; one issuing thread, so S(j + 2)
// cannot overwrite P(j) before its P.V has read it.
//   S    M = 256: A = each CTA's Q rows, B = each CTA's 64 keys, 16 k-steps
//   O   += P V   M = 256, N = 256: A = P in tensor memory, B = each CTA's 128
//               columns of V (MN-major), 8 k-steps of 16 keys
// ---------------------------------------------------------------------------
__device__ __forceinline__ void fwd_pair256_mma(const FwdParams& p, const FwdTile& t,
                                                const FwdPairSmem& s, uint32_t tmem) {
  using C = FwdPairCfg<256>;
  const int n = t.n_blocks;
  if (n == 0) return;
  constexpr uint16_t kBoth = 0x3;
  uint32_t stage = 0, phase = 0;
  auto wait = [&](uint64_t* bar, uint32_t parity, uint32_t code) -> bool {
    if (!__all_sync(0xffffffffu,
                    mbar_wait_cluster(bar, parity, s.abort, p.err, ERR_FWDP_MMA | code,
                                      p.timeout_ns)))
      return false;
    tc_fence_after();
    return true;
  };
  auto release = [&]() {
    mma2_commit_to(&s.kv_empty[stage], kBoth);
    if (++stage == (uint32_t)C::NSTAGE) {
      stage = 0;
      phase ^= 1u;
    }
  };
  // descriptors of the Q panel 0 and of ring chunk 0 (K-major K, MN-major V);
  // byte offsets are added as offset / 16 (the start-address field)
  const uint64_t qd0 = sdesc_sw128(smem_u32(s.q), 16, 1024);
  const uint64_t kd0 = sdesc_sw128(smem_u32(s.ring), 16, 1024);
  const uint64_t vd0 = sdesc_sw128(smem_u32(s.ring), C::CPANEL, 1024);
  auto issue_s = [&](int slot) -> bool {
    const uint32_t d = tmem + slot * C::BN;
    for (int c = 0; c < 2; ++c) {
      if (!wait(&s.kv_full[stage], phase, 2)) return false;
      const uint64_t kd = kd0 + ((stage * C::CHUNK) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // columns 128c + 16kk
        const int col = 128 * c + 16 * kk;
        mma2_ss(d, qd0 + (((col >> 6) * C::QPANEL + (col & 63) * 2) >> 4),
                kd + (((kk >> 2) * C::CPANEL + (kk & 3) * 32) >> 4), C::IDESC_S,
                (c | kk) ? 1u : 0u);
      }
      release();
    }
    return true;
  };
  auto issue_pv = [&](int slot, bool acc) -> bool {
    for (int c = 0; c < 2; ++c) {
      if (!wait(&s.kv_full[stage], phase, 2)) return false;
      const uint64_t vd = vd0 + ((stage * C::CHUNK) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // keys 64c + 16kk
        const int ks = 4 * c + kk;
        mma2_ts(tmem + C::COL_O, tmem + slot * C::BN + ks * 8, vd + ((kk * 16 * 128) >> 4),
                C::IDESC_O, (acc || ks) ? 1u : 0u);
      }
      release();
    }
    return true;
  };
  TRACE_INIT();
  if (!wait(s.q_full, 0, 1)) return;
  if (!issue_s(0)) return;
  mma2_commit_to(&s.s_full[0], kBoth);
  if (n > 1) {
    if (!issue_s(1)) return;
    mma2_commit_to(&s.s_full[1], kBoth);
  }
  for (int j = 0; j < n; ++j) {
    const int slot = j & 1;
    [[maybe_unused]] const int tr = (j < 64) ? 2048 + 16 * j : -1;
    TRACE(tr);
    if (!wait(&s.p_full[slot], (j >> 1) & 1, 3)) return;
    TRACE(tr + 1);
    if (!issue_pv(slot, j > 0)) return;
    mma2_commit_to(&s.o_ready[j & 1], kBoth);
    if (j + 2 < n) {
      if (!issue_s(slot)) return;
      mma2_commit_to(&s.s_full[slot], kBoth);
    }
    TRACE(tr + 2);
  }
  mma2_commit_to(s.o_final, kBoth);
}

// ---------------------------------------------------------------------------
// softmax: eight warps per CTA.  Warp w serves the 16 tile rows
// [32 (w & 3) + 16 lh, +16), lh = w >> 2, over all 128 keys of every block,
// through 16-lane tensor-memory accesses (its lane quadrant is w & 3): thread t
// holds rows rt0 = first + t/4 and rt0 + 8 and, of every 8 keys of the block,
// the two keys 2(t%4) and 2(t%4) + 1 (register 4x + 2r + e is row rt0 + 8r,
// key 8x + 2(t%4) + e).  The four threads of a row combine its max and sum
// with two shuffles.  The two warps of a quadrant share no rows, so neither
// waits for the other's scores.  At head_dim 128 their exp phases take turns
// (lane half 0 first in each block), so one warp's loads, max and stores
// overlap the other's exps (ATTN_FWDP_TURNS=0 lets them run freely: slower);
// at head_dim 256 they run freely.
// ---------------------------------------------------------------------------
#ifndef ATTN_FWDP_TURNS
#define ATTN_FWDP_TURNS 1
#endif
template <int D, bool CAUSAL>
__device__ __forceinline__ void fwd_pair_softmax(const FwdParams& p, const FwdTile& t,
                                                 const FwdPairSmem& s, uint32_t tmem,
                                                 uint32_t rank, int lh) {
  using C = FwdPairCfg<D>;
  // exp turns at head_dim 128 only: at 256 the softmax is not the limit and the
  // turns' barriers measured 4% slower
  constexpr bool TURNS = (D == 128) && (ATTN_FWDP_TURNS != 0);
  const int quad = (threadIdx.x >> 5) & 3;
  const int lane = lane_id();
  const int cq = lane & 3;
  const int rt0 = quad * 32 + lh * 16 + (lane >> 2);
  const int delta = t.sk - t.sq;
  int row[2], head[2], key_lim[2], key_lo[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int rt = rt0 + 8 * r;
    row[r] = t.m_base + (rt >> p.pack_shift);
    head[r] = t.h + (rt & ((1 << p.pack_shift) - 1));
    key_lim[r] = CAUSAL ? min(t.sk, row[r] + delta + p.hi_off + 1) : t.sk;
    key_lo[r] = row[r] + delta - p.lo_off;
  }
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32 + lh * 16) << 16;
  const int n = t.n_blocks;
  const float c = p.scale_log2;
  const int tile_row0 = t.m_base;
  const int mask_from = CAUSAL ? min(t.sk, tile_row0 + delta + p.hi_off + 1) : t.sk;
  const int lo_until = tile_row0 + (t.rows - 1) + delta - p.lo_off;
  // both CTAs' softmax warps report P to the even CTA's barrier.  The odd CTA's
  // report is a relaxed arrive: its P is in its own tensor memory, complete
  // after tcgen05.wait::st and ordered by the tcgen05 fences around the
  // barrier, and the MMA that reads it is issued only after the even CTA has
  // seen the arrive.  A release arrive cost ~1000 cycles per block here.
  const uint32_t p_full_even = mapa_shared(smem_u32(s.p_full), 0);
  // exp turns of the two warps of a quadrant (ATTN_FWDP_TURNS): lane half 0
  // first in each block; a warp that leaves the loop early still plays its
  // remaining turns, so its partner never waits for good
  const int bar_a = 3 + 2 * quad, bar_b = 4 + 2 * quad;
  auto turn_begin = [&](int k) {
    if (lh == 0) {
      if (k > 0) named_bar_sync(bar_a, 64);
    } else {
      named_bar_sync(bar_b, 64);
    }
  };
  auto turn_end = [&](int k) {
    if (lh == 0) named_bar_arrive(bar_b, 64);
    else if (k + 1 < n) named_bar_arrive(bar_a, 64);
  };
  int turns_done = 0;

  TRACE_INIT();
  [[maybe_unused]] const bool tr_on = (lh == 0) && (quad == 0) && (lane == 0);
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  bool ok = true;
  for (int j = 0; j < n; ++j) {
    const int slot = j % C::NS;
    [[maybe_unused]] const int tr = (tr_on && j < 64) ? j * 8 : -1;
    if (!__all_sync(0xffffffffu, mbar_wait_cluster(&s.s_full[slot], (j / C::NS) & 1, s.abort,
                                                   p.err, ERR_FWDP_SOFTMAX | 1, p.timeout_ns))) {
      ok = false;
      turns_done = j;
      break;
    }
    tc_fence_after();
    TRACE(tr);
    const uint32_t s_addr = tmem + lane_base + slot * C::BN;
    uint32_t sr[64];
    tmem_ld16r_x16(s_addr, sr);
    const int kb = (t.n_lo + j) * C::BN;
    const bool masked = (kb + C::BN > mask_from) || (kb < lo_until);
    if (masked) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int lim = key_lim[r] - kb - 2 * cq, lo = key_lo[r] - kb - 2 * cq;
#pragma unroll
        for (int x = 0; x < 16; ++x)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (8 * x + e >= lim || 8 * x + e < lo) sr[4 * x + 2 * r + e] = 0xff800000u;  // -inf
      }
    }
    // row maxima: four chains per row over this thread's 32 keys, then the
    // row's other three threads
    float mx[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float ch[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        ch[k] = fmax3(__uint_as_float(sr[4 * k + 2 * r]), __uint_as_float(sr[4 * k + 2 * r + 1]),
                      __uint_as_float(sr[4 * (k + 4) + 2 * r]));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        ch[k] = fmax3(ch[k], __uint_as_float(sr[4 * (k + 4) + 2 * r + 1]),
                      __uint_as_float(sr[4 * (k + 8) + 2 * r]));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        ch[k] = fmax3(ch[k], __uint_as_float(sr[4 * (k + 8) + 2 * r + 1]),
                      __uint_as_float(sr[4 * (k + 12) + 2 * r]));
#pragma unroll
      for (int k = 0; k < 4; ++k) ch[k] = fmaxf(ch[k], __uint_as_float(sr[4 * (k + 12) + 2 * r + 1]));
      float m = fmaxf(fmaxf(ch[0], ch[1]), fmaxf(ch[2], ch[3]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      mx[r] = m;
    }
    TRACE(tr + 1);
    bool rescale = false;
    float alpha[2] = {1.f, 1.f};
    uint64_t mm2[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float m_new = fmaxf(m_run[r], mx[r] * c);
      if (j == 0) {
        m_run[r] = m_new;
      } else if (m_new - m_run[r] > 8.f) {
        alpha[r] = ex2(m_run[r] - m_new);
        rescale = true;
        m_run[r] = m_new;
        l_run[r] *= alpha[r];
      }
      const float m_sub = (m_run[r] == -INFINITY) ? 0.f : m_run[r];
      mm2[r] = f2_pack(-m_sub, -m_sub);
    }
    if (TURNS) turn_begin(j);
    {
      const uint64_t cc2 = f2_pack(c, c);
      uint64_t acc[2][2] = {{0ull, 0ull}, {0ull, 0ull}};
      uint32_t pk[32];  // register 2x + r: P of keys 8x + 2(t%4) + {0, 1} of row rt0 + 8r
#pragma unroll
      for (int x = 0; x < 16; ++x)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint64_t x2 = f2_fma(
              f2_pack(__uint_as_float(sr[4 * x + 2 * r]), __uint_as_float(sr[4 * x + 2 * r + 1])),
              cc2, mm2[r]);
          float p0, p1;
          if (!masked && (x & 7) < ATTN_FWD_POLY_PAIRS) {
            exp2_fma_pair(x2, p0, p1);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p0 = ex2(x0);
            p1 = ex2(x1);
          }
          acc[r][x & 1] = f2_add(acc[r][x & 1], f2_pack(p0, p1));
          pk[2 * x + r] = pack_bf16(p0, p1);
        }
      // keys 2i, 2i + 1 of the block have their P at column i
      tmem_st16h_x16(s_addr, pk);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float a0, a1;
        f2_unpack(f2_add(acc[r][0], acc[r][1]), a0, a1);
        l_run[r] += a0 + a1;  // this thread's share; the row's four are summed at the end
      }
    }
    if (TURNS) turn_end(j);
    turns_done = j + 1;
    TRACE(tr + 2);
    if (__any_sync(0xffffffffu, rescale)) {
      // O must not be rescaled while the previous P.V may still write it.
      // P.V(k) completes a phase of o_ready[k & 1].  S(j), just read, was
      // issued after P.V(j - 3) completed, and P.V(j) needs this block's P, so
      // o_ready[(j - 1) & 1] has completed (j - 1) / 2 or (j - 1) / 2 + 1
      // phases: the parity of phase (j - 1) / 2 is unambiguous.
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(&s.o_ready[(j - 1) & 1], ((j - 1) >> 1) & 1,
                                                     s.abort, p.err, ERR_FWDP_SOFTMAX | 2,
                                                     p.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t o_addr = tmem + lane_base + C::COL_O;
#pragma unroll 1
      for (int hc = 0; hc < C::D / 64; ++hc) {
        uint32_t o[32];
        tmem_ld16r_x8(o_addr + hc * 64, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[(i >> 1) & 1]);
        tmem_st16r_x8(o_addr + hc * 64, o);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (rank == 0)
        mbar_arrive(&s.p_full[slot]);
      else
        mbar_arrive_remote_relaxed(p_full_even + slot * 8);
    }
    TRACE(tr + 3);
  }
  if (TURNS)
    for (int k = turns_done; k < n; ++k) {
      turn_begin(k);
      turn_end(k);
    }

  // ---- epilogue: the row sums are the sums of the row's four threads ----
  float inv_l[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    l_run[r] = l;
    inv_l[r] = (l > 0.f) ? 1.f / l : 0.f;
  }
  uint8_t* stage = s.q;  // Q is no longer read once the last P.V is done
  constexpr int CPR = C::D / 8;
  fwd_test_delay(p);
  if (ok && n > 0)
    ok = __all_sync(0xffffffffu, mbar_wait_cluster(s.o_final, 0, s.abort, p.err,
                                                   ERR_FWDP_SOFTMAX | 3, p.timeout_ns));
  if (ok) {
    tc_fence_after();
    const uint32_t o_addr = tmem + lane_base + C::COL_O;
#pragma unroll 1
    for (int hc = 0; hc < C::D / 64; ++hc) {  // columns [64 hc, 64 hc + 64) = Q panel hc
      uint32_t o[32];
      if (n > 0) {
        tmem_ld16r_x8(o_addr + hc * 64, o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int rt = rt0 + 8 * r;
          // columns 8x + 2(t%4) + {0, 1}: 16-byte chunk x of the row, 4 bytes
          // at 4(t%4), under the panel's 128-byte swizzle
          *reinterpret_cast<uint32_t*>(stage + hc * C::QPANEL + rt * 128 +
                                       ((x ^ (rt & 7)) * 16) + 4 * cq) =
              pack_bf16(__uint_as_float(o[4 * x + 2 * r]) * inv_l[r],
                        __uint_as_float(o[4 * x + 2 * r + 1]) * inv_l[r]);
        }
    }
  }
  named_bar_sync(1, 256);  // the whole tile is staged
  if (ok) {
    const int rows_left = t.sq - tile_row0;
    uint8_t* out = static_cast<uint8_t*>(p.out);
    const int tid = threadIdx.x;  // the softmax warps are warps 0-7
#pragma unroll 4
    for (int q = tid; q < C::BM * CPR; q += 256) {
      const int r = q / CPR, chn = q % CPR;
      if ((r >> p.pack_shift) < rows_left) {
        const int pn = chn >> 3, cin = chn & 7;
        const uint4 v = *reinterpret_cast<const uint4*>(stage + pn * C::QPANEL + r * 128 +
                                                        ((cin ^ (r & 7)) * 16));
        const size_t grow = static_cast<size_t>(t.q0 + tile_row0 + (r >> p.pack_shift));
        const int gh = t.h + (r & ((1 << p.pack_shift) - 1));
        *reinterpret_cast<uint4*>(out + ((grow * p.nheads_q + gh) * C::D) * 2 + chn * 16) = v;
      }
    }
    if (p.return_lse && cq == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r)
        if (row[r] < t.sq)
          p.lse[static_cast<size_t>(head[r]) * p.total_q + t.q0 + row[r]] =
              (l_run[r] > 0.f) ? (m_run[r] + __log2f(l_run[r])) * 0.69314718055994530942f
                               : -INFINITY;
    }
  }
}

template <int D, bool CAUSAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(FwdPairCfg<D>::THREADS, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdPairCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t rank = cluster_ctarank();
  FwdTile t;
  if (!fwd_pair_tile<D, CAUSAL>(p, t, rank)) return;  // the same for both CTAs
  const FwdPairSmem s = fwd_pair_smem<D>(base);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(s.q_full, 1);
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&s.kv_full[i], 1);
      mbar_init(&s.kv_empty[i], D == 128 ? 2 : 1);  // one release per MMA role
    }
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], 2 * C::SOFTMAX_WARPS);  // both CTAs' softmax warps
      mbar_init(&s.s_free[i], 1);
    }
    mbar_init(&s.o_ready[0], 1);
    mbar_init(&s.o_ready[1], 1);
    mbar_init(s.o_final, 1);
    *s.abort = 0;
    fence_mbar_init();
  }
  if (warp == C::LOAD_WARP && lane_id() == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc2(s.tmem_base, C::TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any copy or arrive
  tc_fence_after();
  const uint32_t tmem = *s.tmem_base;
  if (warp < C::SOFTMAX_WARPS) {
    fwd_pair_softmax<D, CAUSAL>(p, t, s, tmem, rank, warp >> 2);
  } else if (warp == C::LOAD_WARP) {
    if (lane_id() == 0) {
      if constexpr (D == 128) fwd_pair_load(p, t, s, rank, &tmQ, &tmK, &tmV);
      else fwd_pair256_load(p, t, s, rank, &tmQ, &tmK, &tmV);
    }
  } else if (rank == 0) {
    if constexpr (D == 128) fwd_pair_mma(p, t, s, tmem, warp - C::MMA_WARP);
    else fwd_pair256_mma(p, t, s, tmem);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the even CTA's MMAs into this CTA's memory are done
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc2(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn

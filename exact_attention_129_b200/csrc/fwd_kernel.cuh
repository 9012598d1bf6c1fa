// fwd_kernel.cuh -- sm_100a forward kernel: tiled exact attention with an
// online softmax, returning O and the per-row LSE.
//
// The FA4 repository guide (Key Patterns, Core Abstractions) describes the
// forward as a Q tile kept on chip while K/V blocks stream past it through a
// pipeline, an online softmax that tracks each row's max and sum, block ranges
// that skip fully masked blocks under causal masks, and a scheduler that knows
// about varlen batches; the "FA4 head_dim=256 B200 Regression Check" times it on
// B200 at head_dim^-0.5 scale.  This file is our own design of that loop for one
// B200 SM:
//
//   * A tile is NQ query tiles of 128 rows of one (segment, head): NQ = 2 for
//     head_dim 64/128 (both share every K/V tile brought on chip), NQ = 1 for
//     head_dim 256 (its 128 x 256 fp32 accumulator fills half of tensor
//     memory).  A CTA walks a sequence of tiles (fwd_tile_index): one tile per
//     CTA, or with a persistent grid a static share, the barrier phases and
//     ring stages running on from tile to tile.  (The default head_dim-256
//     forward is the two-CTA kernel of fwd_pair_kernel.cuh; this kernel serves
//     head_dim 256 with a softcap or SplitKV.)
//   * Warp roles: softmax warps (head_dim 128: one warpgroup per query tile,
//     thread i owning row i; head_dim 64 and 256: two warpgroups per tile,
//     each warp over 16 whole rows with four threads per row), one TMA
//     producer warp, and one MMA warp per query tile.  An MMA warp runs its
//     role in warp-uniform code and one elected lane issues each tcgen05.mma.
//   * Tensor memory (512 columns): the S slots and the O accumulators.
//     head_dim 64: four 96-column S slots (two per tile) and 2 x 64 O columns;
//     head_dim 128: four 64-column slots and 2 x 128; head_dim 256: two
//     128-column slots double-buffering S across K/V blocks and 256 O columns.
//     P (bf16) is written back over the first BN/2 columns of its S slot and
//     read from there by the P.V MMA (A operand in tensor memory).
//   * Shared memory: the Q tiles, then a ring of chunks of BN rows x 128 bytes
//     holding K and V tiles in the order the MMA warps consume them.  A K tile
//     is D/64 chunks (one per 64-column panel, K-major); a V tile is D/64 chunks
//     of BN*64/D key rows each (all D columns, MN-major operand).  Every chunk
//     is written by TMA with the 128-byte swizzle.
//   * Online softmax in the log2 domain: x = s * scale * log2(e), p = 2^(x - m).
//     The running max m is only raised when a row's max grows by more than 8
//     (a factor 256); until then p may exceed 1 by at most that factor, which
//     fp32 sums and bf16 P absorb.  O is rescaled in tensor memory only when a
//     warp has such a row.  The result is exact: O = sum p v / sum p and
//     LSE = (m + log2 sum p) * ln 2 hold for any m.
//   * Causal: a CTA visits only key blocks that hold an allowed key for one of
//     its rows; element masks are applied only in blocks that cross the
//     diagonal or the end of the segment.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"

// pairs out of every 8 whose 2^x runs on the FMA pipe in unmasked blocks
#ifndef ATTN_FWD_POLY_PAIRS
#define ATTN_FWD_POLY_PAIRS 0
#endif

namespace attn {

// device error word codes (kernel id << 8 | wait id)
enum : uint32_t {
  ERR_FWD_LOAD = 0x0100,
  ERR_FWD_MMA = 0x0200,
  ERR_FWD_SOFTMAX = 0x0300,
};

struct FwdParams {
  const int32_t* cu_q;
  const int32_t* cu_k;
  void* out;        // bf16 [Tq][Hq][D]
  float* lse;       // fp32 [Hq][Tq] or null
  uint32_t* err;    // device error word
  int total_q;
  int nheads_q;
  int nheads_kv;
  float scale_log2;  // scale * log2(e)
  int return_lse;
  // keys allowed for segment-local query row i, with delta = s_k - s_q:
  //   [i + delta - lo_off, i + delta + hi_off]  (kNoBound = no bound; the
  //   upper bound exists iff the kernel's CAUSAL parameter is set)
  int hi_off;
  int lo_off;
  // softcap c: scores become c tanh(s scale / c); cap_k2 = 2 log2(e) scale / c,
  // cap_log2 = c log2(e), cap_k1 = scale / c
  float cap_k2;
  float cap_log2;
  float cap_k1;
  // SplitKV: num_splits > 1 splits every CTA's key-block range into that many
  // contiguous parts (grid.z = batch * num_splits); each part writes its own
  // normalised O and LSE to o_part / lse_part for the combine kernel
  int num_splits;
  float* o_part;    // fp32 [num_splits][total_q][nheads_q][D]
  float* lse_part;  // fp32 [num_splits][nheads_q][total_q]
  // packed GQA (pack_shift > 0): a CTA serves one key/value head and all
  // G = 1 << pack_shift query heads of its group; tile row r is query row
  // r >> pack_shift of head (r & (G - 1)), and grid.y runs over key/value heads
  int pack_shift;
  // persistent tile schedule: the work is tiles_total tiles, the cells of a
  // (tiles_x = query tiles per segment) x (tiles_y = heads) x (segments x
  // splits) grid; the grid's gridDim.x CTAs each take every gridDim.x-th tile
  // (see fwd_tile_index)
  int tiles_x;
  int tiles_y;
  long long tiles_total;
  // host-side only: every tile has the same, small work (equal segments of at
  // most 4 key blocks, no upper or lower key bound, no split), so a static
  // share per CTA is balanced and worth its tile-to-tile overlap
  int uniform_tiles;
  uint64_t timeout_ns;
  // test hook (0 in normal use): the softmax warps idle this long before their
  // final wait, so the tile's last P.V is sure to have completed by then
  uint64_t epilogue_delay_ns;
};

// softcap of one score (fp32 bits): c tanh(s scale / c) in the log2 domain,
// i.e. c log2(e) tanh(s scale / c); masked scores (-inf) stay -inf
__device__ __forceinline__ uint32_t fwd_cap(const FwdParams& p, uint32_t bits) {
  const float x = __uint_as_float(bits);
  return x == -INFINITY ? bits : __float_as_uint(p.cap_log2 * tanh_from_ex2(x * p.cap_k2));
}

// softcap of a thread's scores in place, in the log2 domain.  When no score of
// the block is masked and every score of the warp has |s scale / c| <= 1/2,
// tanh runs as an odd polynomial on the FMA pipe (softcap_poly_pair);
// otherwise every score takes the identity through ex2 and rcp (fwd_cap;
// masked -inf stays -inf).  `masked` is the same for the whole warp.
template <int N>
__device__ __forceinline__ void fwd_cap_scores(const FwdParams& p, uint32_t (&sr)[N],
                                               bool masked) {
  static_assert(N % 2 == 0, "score pairs");
  bool poly = false;
  if (!masked) {
    float ma = 0.f;
#pragma unroll
    for (int i = 0; i < N; i += 2)
      ma = fmax3(ma, fabsf(__uint_as_float(sr[i])), fabsf(__uint_as_float(sr[i + 1])));
    poly = __all_sync(0xffffffffu, ma * p.cap_k1 <= tanhpoly::kY0);
  }
  if (poly) {
    const float K = p.cap_log2;
    const uint64_t k1 = f2_pack(p.cap_k1, p.cap_k1);
    const uint64_t ka[5] = {f2_pack(K * tanhpoly::kA0, K * tanhpoly::kA0),
                            f2_pack(K * tanhpoly::kA1, K * tanhpoly::kA1),
                            f2_pack(K * tanhpoly::kA2, K * tanhpoly::kA2),
                            f2_pack(K * tanhpoly::kA3, K * tanhpoly::kA3),
                            f2_pack(K * tanhpoly::kA4, K * tanhpoly::kA4)};
#pragma unroll
    for (int i = 0; i < N; i += 2) {
      float c0, c1;
      f2_unpack(softcap_poly_pair(f2_pack(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])),
                                  k1, ka),
                c0, c1);
      sr[i] = __float_as_uint(c0);
      sr[i + 1] = __float_as_uint(c1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) sr[i] = fwd_cap(p, sr[i]);
  }
}

__device__ __forceinline__ void fwd_test_delay(const FwdParams& p) {
  if (p.epilogue_delay_ns == 0) return;
  const uint64_t t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < p.epilogue_delay_ns) {
  }
}

template <int D>
struct FwdCfg {
  // head_dim 64/128 (DBUF): two query tiles share every K/V block, blocks are 64
  // keys and each tile double-buffers S, so S(j+1) is computed while the softmax
  // works on S(j).  head_dim 256: one query tile, 128-key blocks, the two S slots
  // double-buffer S (the 128 x 256 fp32 O fills half of tensor memory).
  static constexpr bool DBUF = (D != 256);
  static constexpr int BM = 128;               // rows per query tile
  // keys per block: the four S slots and O fill tensor memory exactly
  // (4 x 96 + 2 x 64, 4 x 64 + 2 x 128, 2 x 128 + 256)
  static constexpr int BN = (D == 64) ? 96 : (D == 128 ? 64 : 128);
  static constexpr int NQ = DBUF ? 2 : 1;      // query tiles per CTA
  static constexpr int NSS = DBUF ? 4 : 2;     // S slots (tile, buffer)
  static constexpr int PANELS = D / 64;        // 64-column (128-byte) panels per row
  static constexpr int QPANEL = BM * 128;      // 16 KB: 128 rows x 64 columns
  static constexpr int CHUNK = BN * 128;       // ring slot: one K panel of BN rows
  static constexpr int VROWS = CHUNK / (2 * D);  // V key rows per chunk (all D columns)
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int NSLOT = (D == 64) ? 14 : (D == 128 ? 20 : 9);
  // ring barriers guard stages of G chunks.  DBUF: stage j holds K_j and
  // V_{j-1} (exactly what one MMA iteration consumes), so each iteration waits
  // on and releases one barrier.  head_dim 256: one chunk per stage.
  static constexpr int G = DBUF ? 2 * PANELS : 1;
  static constexpr int NSTAGE = NSLOT / G;
  // head_dim 64 and 256: eight softmax warps per tile, each over 16 whole rows
  // (16-lane tensor-memory accesses), so more softmax warps share each SM
  // sub-partition and keep its exp unit busy (one warp alone cannot: its exps
  // are latency-bound)
  static constexpr int ROW_SPLIT = (D == 128) ? 1 : 2;
  static constexpr int SOFTMAX_WARPS = 4 * NQ * ROW_SPLIT;
  static constexpr int LOAD_WARP = SOFTMAX_WARPS;
  static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;  // one MMA warp per query tile
  static constexpr int THREADS = 32 * (SOFTMAX_WARPS + 1 + NQ);
  static constexpr int TMEM_COLS = 512;
  static constexpr int O_COL0 = NSS * BN;      // S slots use columns [0, NSS * BN)
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + NQ * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * CHUNK;
  // barriers: q_full[NQ] kv_full[NSTAGE] kv_empty[NSTAGE] s_full[NSS] p_full[NSS]
  // o_ready[NQ] o_final[NQ] q_empty[NQ] o_empty[NQ]
  static constexpr int NBAR = NQ + 2 * NSTAGE + 2 * NSS + 4 * NQ;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16(128, D, false, true);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(NSS * BN <= O_COL0 && O_COL0 + NQ * D <= TMEM_COLS, "tensor memory budget");
  static_assert(VROWS % 16 == 0 && BN % VROWS == 0 && BN / VROWS == PANELS, "V chunking");
  static_assert(NSLOT % G == 0 && NSTAGE >= 2, "ring stages");
};

struct FwdSmem {
  uint8_t* q;
  uint8_t* ring;
  uint64_t* q_full;
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_ready;  // one phase per P.V (rescales wait on the previous one)
  uint64_t* o_final;  // one phase per tile: the tile's last P.V is done
  uint64_t* q_empty;  // one phase per tile: its last S has read Q
  uint64_t* o_empty;  // one phase per tile: the epilogue has read O
  uint32_t* tmem_base;
  volatile int* abort;
};

template <int D>
__device__ __forceinline__ FwdSmem fwd_smem(uint8_t* base) {
  using C = FwdCfg<D>;
  FwdSmem s;
  s.q = base + C::OFF_Q;
  s.ring = base + C::OFF_RING;
  uint64_t* b = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  s.q_full = b;
  s.kv_full = b + C::NQ;
  s.kv_empty = s.kv_full + C::NSTAGE;
  s.s_full = s.kv_empty + C::NSTAGE;
  s.p_full = s.s_full + C::NSS;
  s.o_ready = s.p_full + C::NSS;
  s.o_final = s.o_ready + C::NQ;
  s.q_empty = s.o_final + C::NQ;
  s.o_empty = s.q_empty + C::NQ;
  s.tmem_base = reinterpret_cast<uint32_t*>(base + C::OFF_MISC);
  s.abort = reinterpret_cast<volatile int*>(base + C::OFF_MISC + 4);
  return s;
}

// Number of key blocks a CTA visits and the rows it covers.
struct FwdTile {
  int q0, sq, k0, sk;   // segment offsets / lengths
  int m_base;           // first segment-local query row of the CTA
  int rows;             // query rows per tile: BM, or BM / G when packing GQA
  int n_lo;             // first key block to visit
  int n_blocks;         // key blocks to visit: [n_lo, n_lo + n_blocks)
  int h, hk;
  int split;            // SplitKV part of this CTA (0 without SplitKV)
};

// SplitKV: 32 columns (from col0) of a row's normalised O into the fp32 partial
// buffer of this CTA's split, and the row's partial LSE
template <int D>
__device__ __forceinline__ void fwd_store_part(const FwdParams& p, const FwdTile& t, int row,
                                               int head, int col0, const uint32_t (&r)[32],
                                               float inv_l) {
  if (row >= t.sq) return;
  float* dst = p.o_part +
               ((static_cast<size_t>(t.split) * p.total_q + t.q0 + row) * p.nheads_q + head) * D +
               col0;
#pragma unroll
  for (int g = 0; g < 8; ++g)
    reinterpret_cast<float4*>(dst)[g] =
        make_float4(__uint_as_float(r[4 * g]) * inv_l, __uint_as_float(r[4 * g + 1]) * inv_l,
                    __uint_as_float(r[4 * g + 2]) * inv_l, __uint_as_float(r[4 * g + 3]) * inv_l);
}
__device__ __forceinline__ void fwd_store_part_lse(const FwdParams& p, const FwdTile& t, int row,
                                                   int head, float lse) {
  if (row < t.sq)
    p.lse_part[(static_cast<size_t>(t.split) * p.nheads_q + head) * p.total_q + t.q0 + row] = lse;
}

// The tiles of this CTA, in order: the k-th is tile k * P + b for even k and
// k * P + (P - 1 - b) for odd k (P CTAs, this one b), so each CTA's share
// alternates between the front and the back of every run of P tiles; -1 once
// past the last tile.
__device__ __forceinline__ long long fwd_tile_index(const FwdParams& p, int k) {
  const long long P = gridDim.x, b = blockIdx.x;
  const long long L = static_cast<long long>(k) * P + ((k & 1) ? (P - 1 - b) : b);
  return L < p.tiles_total ? L : -1;
}

// Tile L of the schedule: query tile x of segment (and split) z for head (or,
// packing GQA, key/value head) y; false if it holds no query row.
template <int D, bool CAUSAL>
__device__ __forceinline__ bool fwd_tile(const FwdParams& p, FwdTile& t, long long L) {
  using C = FwdCfg<D>;
  const int x = static_cast<int>(L % p.tiles_x);
  const long long yz = L / p.tiles_x;
  const int y = static_cast<int>(yz % p.tiles_y);
  const int z = static_cast<int>(yz / p.tiles_y);
  const int b = z / p.num_splits;
  t.split = z % p.num_splits;
  if (p.pack_shift > 0) {
    t.hk = y;
    t.h = t.hk << p.pack_shift;  // first query head of the group
  } else {
    t.h = y;
    t.hk = t.h / (p.nheads_q / p.nheads_kv);
  }
  t.rows = C::BM >> p.pack_shift;
  t.q0 = p.cu_q[b];
  t.sq = p.cu_q[b + 1] - t.q0;
  t.k0 = p.cu_k[b];
  t.sk = p.cu_k[b + 1] - t.k0;
  // causal: heaviest tiles (bottom of the segment) first
  const int m_tile = CAUSAL ? (p.tiles_x - 1 - x) : x;
  t.m_base = m_tile * t.rows * C::NQ;
  if (t.m_base >= t.sq) return false;
  // the union of the rows' allowed key ranges
  const int delta = t.sk - t.sq;
  int n_end = t.sk;
  if (CAUSAL) {
    const int last_row = min(t.sq, t.m_base + t.rows * C::NQ) - 1;
    n_end = min(t.sk, last_row + delta + p.hi_off + 1);
  }
  const int n_beg = (p.lo_off < kNoBound) ? max(0, t.m_base + delta - p.lo_off) : 0;
  t.n_lo = n_beg / C::BN;
  t.n_blocks = n_end > n_beg ? (n_end + C::BN - 1) / C::BN - t.n_lo : 0;
  if (p.num_splits > 1) {
    // this CTA's contiguous share; a share past the end has no blocks and
    // writes O = 0, LSE = -inf for the combine
    const int per = (t.n_blocks + p.num_splits - 1) / p.num_splits;
    const int first = t.split * per;
    t.n_lo += first;
    t.n_blocks = max(0, min(per, t.n_blocks - first));
  }
  return true;
}

// A tile's fields taken from lane 0 (for warp-wide callers): every lane holds
// the same values anyway, but after the shuffles the compiler knows it, so
// tensor-memory addresses and MMA operands derived from them stay in uniform
// registers.
__device__ __forceinline__ void fwd_tile_uniform(FwdTile& t) {
  t.q0 = __shfl_sync(0xffffffffu, t.q0, 0);
  t.sq = __shfl_sync(0xffffffffu, t.sq, 0);
  t.k0 = __shfl_sync(0xffffffffu, t.k0, 0);
  t.sk = __shfl_sync(0xffffffffu, t.sk, 0);
  t.m_base = __shfl_sync(0xffffffffu, t.m_base, 0);
  t.rows = __shfl_sync(0xffffffffu, t.rows, 0);
  t.n_lo = __shfl_sync(0xffffffffu, t.n_lo, 0);
  t.n_blocks = __shfl_sync(0xffffffffu, t.n_blocks, 0);
  t.h = __shfl_sync(0xffffffffu, t.h, 0);
  t.hk = __shfl_sync(0xffffffffu, t.hk, 0);
  t.split = __shfl_sync(0xffffffffu, t.split, 0);
}

// ---------------------------------------------------------------------------
// producer warp (one lane): for each of the CTA's tiles, its Q tiles, then K/V
// chunks in MMA consumption order; the ring runs on from tile to tile.  A
// tile's Q is loaded once the MMA warp's last S of the previous tile has read
// the Q buffer (q_empty), so it lands while the previous tile finishes.
// ---------------------------------------------------------------------------
template <int D, bool CAUSAL>
__device__ __forceinline__ void fwd_load(const FwdParams& p, const FwdSmem& s,
                                         const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                         const CUtensorMap* tmV) {
  using C = FwdCfg<D>;
  uint32_t ring = 0;             // stages issued so far
  uint32_t q_loads[C::NQ] = {};  // Q tiles issued so far, per query tile
  // on the way out after a timed-out wait elsewhere: let every copy this CTA
  // issued land before its shared memory is released (earlier Q copies have
  // landed: each was read before the next was issued)
  auto drain = [&]() {
    for (int qt = 0; qt < C::NQ; ++qt)
      if (q_loads[qt] > 0) mbar_wait_drain(&s.q_full[qt], (q_loads[qt] - 1) & 1, 100000000ull);
    const uint32_t first = ring > (uint32_t)C::NSTAGE ? ring - C::NSTAGE : 0u;
    for (uint32_t r = first; r < ring; ++r)
      mbar_wait_drain(&s.kv_full[r % C::NSTAGE], (r / C::NSTAGE) & 1, 100000000ull);
  };
  // claim the next stage (waiting for the MMA warps to release its last use)
  // and announce the bytes that will land in it
  auto claim = [&](uint32_t bytes, uint8_t*& base, uint64_t*& full) -> bool {
    const uint32_t st = ring % C::NSTAGE;
    if (ring >= (uint32_t)C::NSTAGE &&
        !mbar_wait(&s.kv_empty[st], ((ring / C::NSTAGE) - 1) & 1, s.abort, p.err,
                   ERR_FWD_LOAD | 1, p.timeout_ns)) {
      drain();
      return false;
    }
    full = &s.kv_full[st];
    base = s.ring + st * (C::G * C::CHUNK);
    mbar_expect_tx(full, bytes);
    ++ring;
    return true;
  };
  for (int k = 0;; ++k) {
    const long long L = fwd_tile_index(p, k);
    if (L < 0) return;
    FwdTile t;
    if (!fwd_tile<D, CAUSAL>(p, t, L) || t.n_blocks == 0) continue;
    // the Q tiles, once the previous Q in each buffer has been read
    for (int qt = 0; qt < C::NQ; ++qt) {
      if (t.m_base + qt * t.rows >= t.sq) break;
      if (q_loads[qt] > 0 &&
          !mbar_wait(&s.q_empty[qt], (q_loads[qt] - 1) & 1, s.abort, p.err, ERR_FWD_LOAD | 2,
                     p.timeout_ns)) {
        drain();
        return;
      }
      mbar_expect_tx(&s.q_full[qt], C::Q_BYTES);
      // one box per panel: t.rows query rows x (packed: all G heads) x 64 columns
      for (int pn = 0; pn < C::PANELS; ++pn)
        tma_load_3d(s.q + qt * C::Q_BYTES + pn * C::QPANEL, tmQ, &s.q_full[qt], pn * 64, t.h,
                    t.q0 + t.m_base + qt * t.rows);
      ++q_loads[qt];
    }
    // K block j: one chunk per 64-column panel (BN rows, K-major)
    auto load_k = [&](uint8_t* dst, uint64_t* full, int j, int c) {
      tma_load_3d(dst, tmK, full, c * 64, t.hk, t.k0 + (t.n_lo + j) * C::BN);
    };
    // rows [c*VROWS, (c+1)*VROWS) of V block j: all D columns, panel by panel
    auto load_v = [&](uint8_t* dst, uint64_t* full, int j, int c) {
      for (int pn = 0; pn < C::PANELS; ++pn)
        tma_load_3d(dst + pn * (C::VROWS * 128), tmV, full, pn * 64, t.hk,
                    t.k0 + (t.n_lo + j) * C::BN + c * C::VROWS);
    };
    const int n = t.n_blocks;
    uint8_t* base;
    uint64_t* full;
    if constexpr (C::DBUF) {
      // stage j = (K_j, V_{j-1}); the first holds only K_0, the last only V_{n-1}
      for (int j = 0; j <= n; ++j) {
        const uint32_t bytes =
            ((j < n) ? C::PANELS * C::CHUNK : 0) + ((j > 0) ? C::PANELS * C::CHUNK : 0);
        if (!claim(bytes, base, full)) return;
        for (int c = 0; c < C::PANELS; ++c) {
          if (j < n) load_k(base + c * C::CHUNK, full, j, c);
          if (j > 0) load_v(base + (C::PANELS + c) * C::CHUNK, full, j - 1, c);
        }
      }
    } else {
      // one chunk per stage, in the MMA warp's order: K_0, K_1, then V_j before K_{j+2}
      auto load_tile = [&](bool is_v, int j) -> bool {
        for (int c = 0; c < C::PANELS; ++c) {
          if (!claim(C::CHUNK, base, full)) return false;
          if (is_v) load_v(base, full, j, c);
          else load_k(base, full, j, c);
        }
        return true;
      };
      if (!load_tile(false, 0)) return;
      if (n > 1 && !load_tile(false, 1)) return;
      for (int j = 0; j < n; ++j) {
        if (!load_tile(true, j)) return;
        if (j + 2 < n && !load_tile(false, j + 2)) return;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// MMA warp (all lanes run it; one elected lane issues)
// ---------------------------------------------------------------------------
template <int D>
struct FwdMma {
  using C = FwdCfg<D>;
  const FwdParams& p;
  const FwdSmem& s;
  uint32_t tmem;
  uint32_t stage = 0, phase = 0;  // next ring stage to consume and its parity
  // descriptors of chunk 0 of the ring (K-major K, MN-major V) and of Q tile 0;
  // the start-address field is the low 14 bits, so an offset of b bytes inside
  // shared memory is added as b / 16 without carrying into other fields
  uint64_t kdesc0, vdesc0, qdesc0;

  __device__ FwdMma(const FwdParams& p_, const FwdSmem& s_, uint32_t tmem_)
      : p(p_), s(s_), tmem(tmem_) {
    kdesc0 = sdesc_sw128(smem_u32(s.ring), 16, 1024);
    vdesc0 = sdesc_sw128(smem_u32(s.ring), C::VROWS * 128, 1024);
    qdesc0 = sdesc_sw128(smem_u32(s.q), 16, 1024);
  }

  // wait for the next `count` stages; returns the first one's chunk index
  __device__ bool wait_stages(int count, uint32_t& first_chunk) {
    first_chunk = stage * C::G;
    uint32_t st = stage, ph = phase;
    for (int i = 0; i < count; ++i) {
      if (!mbar_wait_warp(&s.kv_full[st], ph, s.abort, p.err, ERR_FWD_MMA | 1, p.timeout_ns))
        return false;
      if (++st == (uint32_t)C::NSTAGE) {
        st = 0;
        ph ^= 1u;
      }
    }
    tc_fence_after();
    return true;
  }
  // release the next `count` stages once the MMAs issued so far have read them
  __device__ void release_stages(int count) {
    for (int i = 0; i < count; ++i) {
      mma_commit(&s.kv_empty[stage]);
      if (++stage == (uint32_t)C::NSTAGE) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  // head_dim 256 (one chunk per stage): the next tile's panels one at a time.
  // Waiting for a panel's chunk right before its MMAs, and releasing it right
  // after, lets each wait overlap the MMAs already queued.
  __device__ bool wait_next_chunk() {
    if (!mbar_wait_warp(&s.kv_full[stage], phase, s.abort, p.err, ERR_FWD_MMA | 1, p.timeout_ns))
      return false;
    tc_fence_after();
    return true;
  }
  __device__ bool issue_s_streamed(int qt, int slot) {
    const uint32_t d_tmem = tmem + slot * C::BN;
    const uint64_t qd = qdesc0 + (uint64_t)(qt * (C::Q_BYTES >> 4));
    for (int c = 0; c < C::PANELS; ++c) {
      if (!wait_next_chunk()) return false;
      const uint64_t kd = kdesc0 + (uint64_t)(stage * C::G * (C::CHUNK >> 4));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(d_tmem, qd + (c * (C::QPANEL >> 4) + kk * 2), kd + kk * 2, C::IDESC_S,
               (c | kk) != 0);
      release_stages(1);
    }
    return true;
  }
  __device__ bool issue_pv_streamed(int qt, int slot, bool accumulate) {
    const uint32_t d_tmem = tmem + C::O_COL0 + qt * D;
    const uint32_t p_tmem = tmem + slot * C::BN;
    for (int c = 0; c < C::PANELS; ++c) {
      if (!wait_next_chunk()) return false;
      const uint64_t vd = vdesc0 + (uint64_t)(stage * C::G * (C::CHUNK >> 4));
#pragma unroll
      for (int kk = 0; kk < C::VROWS / 16; ++kk) {
        const int kstep = c * (C::VROWS / 16) + kk;
        mma_ts(d_tmem, p_tmem + kstep * 8, vd + kk * 128, C::IDESC_O,
               (accumulate || kstep) ? 1u : 0u);
      }
      release_stages(1);
    }
    return true;
  }
  __device__ static uint32_t wrap(uint32_t chunk) {
    if constexpr (C::G == 1) {
      if (chunk >= (uint32_t)C::NSLOT) chunk -= C::NSLOT;
    }
    return chunk;
  }
  // S[slot] = Q[qt] . K^T, K panel c in ring chunk ch0 + c
  __device__ void issue_s(int qt, int slot, uint32_t ch0) {
    const uint32_t d_tmem = tmem + slot * C::BN;
    const uint64_t qd = qdesc0 + (uint64_t)(qt * (C::Q_BYTES >> 4));
#pragma unroll
    for (int c = 0; c < C::PANELS; ++c) {
      const uint64_t kd = kdesc0 + (uint64_t)(wrap(ch0 + c) * (C::CHUNK >> 4));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)  // 16 columns (32 bytes) of the panel per step
        mma_ss(d_tmem, qd + (c * (C::QPANEL >> 4) + kk * 2), kd + kk * 2, C::IDESC_S,
               (c | kk) != 0);
    }
  }
  // O[qt] (+)= P[slot] . V, V rows [c*VROWS, (c+1)*VROWS) in ring chunk ch0 + c
  __device__ void issue_pv(int qt, int slot, uint32_t ch0, bool accumulate) {
    const uint32_t d_tmem = tmem + C::O_COL0 + qt * D;
    const uint32_t p_tmem = tmem + slot * C::BN;
#pragma unroll
    for (int c = 0; c < C::PANELS; ++c) {
      const uint64_t vd = vdesc0 + (uint64_t)(wrap(ch0 + c) * (C::CHUNK >> 4));
#pragma unroll
      for (int kk = 0; kk < C::VROWS / 16; ++kk) {
        const int kstep = c * (C::VROWS / 16) + kk;  // 16 keys (2048 bytes of V) per step
        mma_ts(d_tmem, p_tmem + kstep * 8, vd + kk * 128, C::IDESC_O,
               (accumulate || kstep) ? 1u : 0u);
      }
    }
  }
};

// The MMA warp of query tile qt, over the CTA's tiles.  A tile's first S waits
// for its Q (q_full), its last S releases the Q buffer (q_empty); its first
// P.V (which overwrites O) waits until the epilogue of the previous tile has
// read O (o_empty), its last P.V completes o_final.  The S slots, ring stages
// and barrier phases run on over the tiles (g counts this warp's blocks); a
// tile in which this query tile has no rows only has its stages released.
// (qt is a template parameter so that every MMA operand and barrier address is
// a compile-time function of it.)
template <int D, bool CAUSAL, int qt>
__device__ __forceinline__ void fwd_mma(const FwdParams& p, const FwdSmem& s, uint32_t tmem) {
  using C = FwdCfg<D>;
  TRACE_INIT();
  FwdMma<D> m(p, s, tmem);
  uint32_t g = 0;       // blocks of this query tile so far (S slot and p_full phases)
  uint32_t tiles = 0;   // tiles with rows for this query tile (q_full / o_empty phases)
  for (int k = 0;; ++k) {
    const long long L = fwd_tile_index(p, k);
    if (L < 0) return;
    FwdTile t;
    fwd_tile<D, CAUSAL>(p, t, L);
    fwd_tile_uniform(t);
    if (t.m_base >= t.sq || t.n_blocks == 0) continue;  // no rows, or no blocks
    const int n = t.n_blocks;
    g = __shfl_sync(0xffffffffu, g, 0);  // warp-uniform, see fwd_softmax
    if (t.m_base + qt * t.rows >= t.sq) {
      // no rows for this query tile: release the tile's stages as they fill
      uint32_t ch;
      for (int j = 0; j <= n; ++j) {
        if (!m.wait_stages(1, ch)) return;
        m.release_stages(1);
      }
      continue;
    }
    if (!mbar_wait_warp(&s.q_full[qt], tiles & 1, s.abort, p.err, ERR_FWD_MMA | 2, p.timeout_ns))
      return;
    tc_fence_after();
    // the first P.V of a tile waits for the previous tile's epilogue
    auto o_free = [&]() -> bool {
      if (tiles == 0) return true;
      if (!mbar_wait_warp(&s.o_empty[qt], (tiles - 1) & 1, s.abort, p.err, ERR_FWD_MMA | 4,
                          p.timeout_ns))
        return false;
      tc_fence_after();
      return true;
    };
    if constexpr (C::DBUF) {
      // S of block j lives in slot 2qt + ((g + j) & 1); S(j+1) is issued
      // before P(j).V so the tensor pipe has work while the softmax runs on
      // S(j); the slot it overwrites held P(j-1), read by the P.V this thread
      // issued one iteration earlier on the same in-order pipe.  Stage j holds
      // K_j in its first PANELS chunks and V_{j-1} in the next PANELS.
      uint32_t ch;
      if (!m.wait_stages(1, ch)) return;
      m.issue_s(qt, 2 * qt + (g & 1), ch);
      mma_commit(&s.s_full[2 * qt + (g & 1)]);
      if (n == 1) mma_commit(&s.q_empty[qt]);
      m.release_stages(1);
      for (int j = 0; j < n; ++j) {
        const uint32_t gj = g + j;
        const int b = gj & 1;
        [[maybe_unused]] const int tr = (j < 64) ? 2048 + 16 * j + 8 * qt : -1;
        TRACE(tr);
        if (!m.wait_stages(1, ch)) return;
        TRACE(tr + 1);
        if (j + 1 < n) {
          m.issue_s(qt, 2 * qt + (b ^ 1), ch);
          mma_commit(&s.s_full[2 * qt + (b ^ 1)]);
          if (j + 2 == n) mma_commit(&s.q_empty[qt]);
        }
        TRACE(tr + 2);
        if (!mbar_wait_warp(&s.p_full[2 * qt + b], (gj >> 1) & 1, s.abort, p.err,
                            ERR_FWD_MMA | 3, p.timeout_ns))
          return;
        tc_fence_after();
        if (j == 0 && !o_free()) return;
        TRACE(tr + 3);
        m.issue_pv(qt, 2 * qt + b, ch + C::PANELS, j > 0);
        mma_commit(&s.o_ready[qt]);
        m.release_stages(1);
        TRACE(tr + 4);
      }
    } else {
      // one query tile, two S slots alternating over key blocks; one chunk per
      // stage, each waited for right before its MMAs
      if (!m.issue_s_streamed(0, g & 1)) return;
      mma_commit(&s.s_full[g & 1]);
      if (n > 1) {
        if (!m.issue_s_streamed(0, (g + 1) & 1)) return;
        mma_commit(&s.s_full[(g + 1) & 1]);
      }
      if (n <= 2) mma_commit(&s.q_empty[0]);
      for (int j = 0; j < n; ++j) {
        const uint32_t gj = g + j;
        const int slot = gj & 1;
        [[maybe_unused]] const int tr = (j < 64) ? 2048 + 16 * j : -1;
        TRACE(tr);
        if (!mbar_wait_warp(&s.p_full[slot], (gj >> 1) & 1, s.abort, p.err, ERR_FWD_MMA | 3,
                            p.timeout_ns))
          return;
        tc_fence_after();
        if (j == 0 && !o_free()) return;
        TRACE(tr + 1);
        if (!m.issue_pv_streamed(0, slot, j > 0)) return;
        mma_commit(&s.o_ready[0]);
        TRACE(tr + 3);
        if (j + 2 < n) {
          if (!m.issue_s_streamed(0, slot)) return;
          mma_commit(&s.s_full[slot]);
          if (j + 3 == n) mma_commit(&s.q_empty[0]);
          TRACE(tr + 5);
        }
      }
    }
    mma_commit(&s.o_final[qt]);
    g += n;
    ++tiles;
  }
}

// What a softmax warp carries from tile to tile: the S slots and the
// o_ready / o_final phases run on over the CTA's tiles.
struct FwdSoftState {
  uint32_t g = 0;   // blocks of this query tile processed so far (all tiles)
  uint32_t nt = 0;  // tiles with blocks finished (phases of o_final / o_empty)
  bool ok = true;   // false after a timed-out wait: the warp stops
  // the CTA has a single tile: no Q follows, so the epilogue stages O through
  // the Q buffer and stores whole rows (stores straight from registers write
  // 16-byte pieces of 32 rows at a time, measured 4.5% slower at head_dim 256)
  bool single = false;
};

// Coalesced copy of a staged tile (bf16 rows of D columns, 16-byte chunks
// XOR-swizzled by row) to out, rows past the segment left out.
template <int D, int NTHR>
__device__ __forceinline__ void fwd_copy_out(const FwdParams& p, const FwdTile& t,
                                             const uint8_t* stage, int tile_row0, int tid) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  const int rows_left = t.sq - tile_row0;
  uint8_t* out = static_cast<uint8_t*>(p.out);
#pragma unroll 4
  for (int q = tid; q < 128 * CPR; q += NTHR) {
    const int r = q / CPR, ch = q % CPR;
    if ((r >> p.pack_shift) < rows_left) {
      const uint4 v = *reinterpret_cast<const uint4*>(stage + r * (D * 2) + ((ch ^ (r & 7)) * 16));
      const size_t grow = static_cast<size_t>(t.q0 + tile_row0 + (r >> p.pack_shift));
      const int gh = t.h + (r & ((1 << p.pack_shift) - 1));
      *reinterpret_cast<uint4*>(out + ((grow * p.nheads_q + gh) * D) * 2 + ch * 16) = v;
    }
  }
}

// one tile's epilogue output: 32 columns of a row's O / l as bf16, straight
// from registers into out[row][head]
template <int D>
__device__ __forceinline__ void fwd_store_o32(const FwdParams& p, const FwdTile& t, int row,
                                              int head, int col0, const uint32_t (&r)[32],
                                              float inv_l) {
  uint4* dst = reinterpret_cast<uint4*>(
      static_cast<uint16_t*>(p.out) +
      (static_cast<size_t>(t.q0 + row) * p.nheads_q + head) * D + col0);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint4 v;
    v.x = pack_bf16(__uint_as_float(r[g * 8 + 0]) * inv_l, __uint_as_float(r[g * 8 + 1]) * inv_l);
    v.y = pack_bf16(__uint_as_float(r[g * 8 + 2]) * inv_l, __uint_as_float(r[g * 8 + 3]) * inv_l);
    v.z = pack_bf16(__uint_as_float(r[g * 8 + 4]) * inv_l, __uint_as_float(r[g * 8 + 5]) * inv_l);
    v.w = pack_bf16(__uint_as_float(r[g * 8 + 6]) * inv_l, __uint_as_float(r[g * 8 + 7]) * inv_l);
    dst[g] = v;
  }
}

// ---------------------------------------------------------------------------
// softmax warpgroup: one thread per query row; one tile
// ---------------------------------------------------------------------------
template <int D, bool CAUSAL, bool SOFTCAP>
__device__ __forceinline__ void fwd_softmax(const FwdParams& p, const FwdTile& t,
                                            const FwdSmem& s, uint32_t tmem, int qt,
                                            FwdSoftState& st) {
  using C = FwdCfg<D>;
  const int warp = (threadIdx.x >> 5) & 3;  // warp within the warpgroup = TMEM lane quadrant
  const int lane = lane_id();
  const int row_in_tile = warp * 32 + lane;
  // segment-local query row and query head of this thread's tile row
  const int row = t.m_base + qt * t.rows + (row_in_tile >> p.pack_shift);
  const int head = t.h + (row_in_tile & ((1 << p.pack_shift) - 1));
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const int n = t.n_blocks;
  // the block count so far, known to the compiler as warp-uniform, so the S
  // slot addresses derived from it stay in uniform registers
  const uint32_t g0 = __shfl_sync(0xffffffffu, st.g, 0);
  // with a softcap the scores are turned into capped log2-domain values first
  const float c = SOFTCAP ? 1.f : p.scale_log2;
  // keys [key_lo, key_lim) are allowed for this row
  const int delta = t.sk - t.sq;
  const int key_lim = CAUSAL ? min(t.sk, row + delta + p.hi_off + 1) : t.sk;
  const int key_lo = row + delta - p.lo_off;
  // a block needs element masks for this warpgroup when it crosses the upper
  // bound of the tile's first row (or the end of the keys) or the lower bound
  // of its last row
  const int tile_row0 = t.m_base + qt * t.rows;
  const int mask_from = CAUSAL ? min(t.sk, tile_row0 + delta + p.hi_off + 1) : t.sk;
  const int lo_until = tile_row0 + (t.rows - 1) + delta - p.lo_off;

  // With two query tiles, warp w of each tile shares an SM sub-partition and
  // its special-function unit: their exp phases take turns (tile 0 first in
  // each block) through a pair of named barriers, so one warp's loads, max and
  // stores overlap the other's exps.  Every turn of tile 1 ends with an arrive
  // for tile 0, and tile 0 takes the last one at the end of the tile, so each
  // barrier sees exactly one arrive and one sync per turn and nothing carries
  // over into the next tile.  A warp that gives up on a timed-out wait still
  // plays its remaining turns, so its partner never waits forever.
  const bool pingpong = C::DBUF && C::ROW_SPLIT == 1 && (t.m_base + t.rows < t.sq);
  const int bar_t0 = 3 + 2 * warp, bar_t1 = 4 + 2 * warp;  // "tile 0 / tile 1 may start"
  auto turn_begin = [&](int k) {
    if (qt == 0) {
      if (k > 0) named_bar_sync(bar_t0, 64);
    } else {
      named_bar_sync(bar_t1, 64);
    }
  };
  auto turn_end = [&](int k) {
    if (qt == 0) named_bar_arrive(bar_t1, 64);
    else named_bar_arrive(bar_t0, 64);
  };
  int turns_done = 0;

  TRACE_INIT();
  float m_run = -INFINITY;  // running max, log2 domain
  float l_run = 0.f;
  bool ok = true;

  constexpr int NCOL = C::BN;  // scores per row and block
  for (int j = 0; j < n; ++j) {
    const uint32_t g = g0 + j;  // this block's index over the CTA's tiles
    const int slot = C::DBUF ? 2 * qt + (g & 1) : (g & 1);
    const uint32_t parity = (g >> 1) & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full[slot], parity, s.abort, p.err,
                                           ERR_FWD_SOFTMAX | 1, p.timeout_ns))) {
      ok = false;
      turns_done = j;
      break;
    }
    tc_fence_after();
    if (threadIdx.x % 128 == 0 && j < 64) TRACE(1024 * qt + j * 8 + 0);
    const uint32_t s_addr = tmem + lane_base + slot * NCOL;
    uint32_t sr[NCOL];  // the row's scores for this block (fp32 bits)
    if constexpr (NCOL == 128) tmem_ld128(s_addr, sr);
    else tmem_ld64(s_addr, sr);
    if (threadIdx.x % 128 == 0 && j < 64) TRACE(1024 * qt + j * 8 + 1);
    const int kb = (t.n_lo + j) * C::BN;  // segment-local key of column 0
    const bool masked = (kb + C::BN > mask_from) || (kb < lo_until);
    if (masked) {
      const int lim = key_lim - kb, lo = key_lo - kb;
#pragma unroll
      for (int i = 0; i < NCOL; ++i)
        if (i >= lim || i < lo) sr[i] = 0xff800000u;  // -inf
    }
    if constexpr (SOFTCAP) fwd_cap_scores(p, sr, masked);
    // row max: 8 independent chains of three-input max, then a short tree
    float mx;
    {
      float ch[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        ch[k] = fmax3(__uint_as_float(sr[k]), __uint_as_float(sr[k + 8]),
                      __uint_as_float(sr[k + 16]));
      int i = 24;
#pragma unroll
      for (; i + 16 <= NCOL - 8; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ch[k] = fmax3(ch[k], __uint_as_float(sr[i + k]), __uint_as_float(sr[i + 8 + k]));
#pragma unroll
      for (; i < NCOL; i += 8)
#pragma unroll
        for (int k = 0; k < 8; ++k) ch[k] = fmaxf(ch[k], __uint_as_float(sr[i + k]));
      mx = fmaxf(fmax3(ch[0], ch[1], ch[2]), fmax3(ch[3], ch[4], fmax3(ch[5], ch[6], ch[7])));
    }
    const float m_new = fmaxf(m_run, mx * c);
    if (threadIdx.x % 128 == 0 && j < 64) TRACE(1024 * qt + j * 8 + 2);
    bool rescale = false;
    float alpha = 1.f;
    if (j == 0) {
      m_run = m_new;
    } else if (m_new - m_run > 8.f) {
      alpha = ex2(m_run - m_new);
      rescale = true;
      m_run = m_new;
      l_run *= alpha;
    }
    const float m_sub = (m_run == -INFINITY) ? 0.f : m_run;
    // P = 2^(s*c - m) on pairs (packed fp32x2 FMA), rounded to bf16 and written
    // over the first NCOL/2 columns of S; the row sum uses 4 independent
    // accumulators.  With two query tiles, two softmax warps share each SM
    // sub-partition and the special-function unit (ex2) becomes the limit, so in
    // blocks without masked scores ATTN_FWD_POLY_PAIRS of every 8 pairs take 2^x on the FMA pipe
    // (exp2_fma_pair); masked blocks keep ex2 everywhere so -inf gives exactly 0.
    float lsum;
    {
      const uint64_t cc2 = f2_pack(c, c), mm2 = f2_pack(-m_sub, -m_sub);
      uint64_t acc[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[a] = 0ull;
      auto exp_rows = [&](auto use_poly) {
        constexpr bool POLY = decltype(use_poly)::value;
        uint32_t pk[32];
#pragma unroll
        for (int half = 0; half < NCOL / 64; ++half) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int col = half * 64 + 2 * i;
            const uint64_t x2 =
                f2_fma(f2_pack(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])), cc2, mm2);
            float p0, p1;
            if (POLY && (i & 7) < ATTN_FWD_POLY_PAIRS) {
              exp2_fma_pair(x2, p0, p1);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
            pk[i] = pack_bf16(p0, p1);
          }
          tmem_st32(s_addr + half * 32, pk);
        }
      };
      if (pingpong) turn_begin(j);
      if (C::DBUF && !masked)
        exp_rows(std::integral_constant<bool, true>());
      else
        exp_rows(std::integral_constant<bool, false>());
      if (pingpong) turn_end(j);
      float a0, a1, a2, a3;
      f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
      f2_unpack(f2_add(acc[2], acc[3]), a2, a3);
      lsum = (a0 + a1) + (a2 + a3);
    }
    l_run += lsum;
    if (threadIdx.x % 128 == 0 && j < 64) TRACE(1024 * qt + j * 8 + 3);
    if (__any_sync(0xffffffffu, rescale)) {
      // O must not be rescaled while the previous P.V MMA may still write it.
      // Counting over the CTA's tiles, o_ready has completed g-1 or g phases
      // here (S(g), just read, was issued after P.V(g-2), and P.V(g) needs this
      // block's P), so the parity of phase g-1 is unambiguous (j > 0 here).
      if (!__all_sync(0xffffffffu, mbar_wait(&s.o_ready[qt], (g - 1) & 1, s.abort, p.err,
                                             ERR_FWD_SOFTMAX | 2, p.timeout_ns))) {
        ok = false;
        turns_done = j + 1;
        break;
      }
      tc_fence_after();
      const uint32_t o_addr = tmem + lane_base + C::O_COL0 + qt * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(o_addr + cc * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
        tmem_st32(o_addr + cc * 32, r);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    if (threadIdx.x % 128 == 0 && j < 64) TRACE(1024 * qt + j * 8 + 4);
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.p_full[slot]);
    turns_done = j + 1;
  }
  if (pingpong)
    for (int k = turns_done; k < n; ++k) {
      turn_begin(k);
      turn_end(k);
    }

  // ---- epilogue: O / l -> bf16, straight from registers to out ----
  const bool row_valid = row < t.sq;
  const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
  // Wait for the tile's last P.V on o_final, which completes once per tile
  // with blocks.  A parity wait on o_ready cannot do it: the last S this
  // warpgroup read was issued before the second-to-last P.V, so o_ready may be
  // anywhere from two phases short of the end to already past it, and a
  // parity test cannot tell a phase two behind from the current one.
  fwd_test_delay(p);
  if (ok && n > 0) {
    if (!__all_sync(0xffffffffu, mbar_wait(&s.o_final[qt], st.nt & 1, s.abort, p.err,
                                           ERR_FWD_SOFTMAX | 3, p.timeout_ns)))
      ok = false;
  }
  if (ok) {
    tc_fence_after();
    const uint32_t o_addr = tmem + lane_base + C::O_COL0 + qt * D;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t r[32];
      if (n > 0) {
        tmem_ld32(o_addr + cc * 32, r);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      if (p.num_splits > 1) {  // SplitKV: fp32 partial
        fwd_store_part<D>(p, t, row, head, cc * 32, r, inv_l);
      } else if (st.single) {  // into the Q buffer, 16-byte chunks swizzled by row
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(r[g * 8 + 0]) * inv_l, __uint_as_float(r[g * 8 + 1]) * inv_l);
          v.y = pack_bf16(__uint_as_float(r[g * 8 + 2]) * inv_l, __uint_as_float(r[g * 8 + 3]) * inv_l);
          v.z = pack_bf16(__uint_as_float(r[g * 8 + 4]) * inv_l, __uint_as_float(r[g * 8 + 5]) * inv_l);
          v.w = pack_bf16(__uint_as_float(r[g * 8 + 6]) * inv_l, __uint_as_float(r[g * 8 + 7]) * inv_l);
          const int chunk = cc * 4 + g;
          *reinterpret_cast<uint4*>(s.q + qt * C::Q_BYTES + row_in_tile * (D * 2) +
                                    ((chunk ^ (row_in_tile & 7)) * 16)) = v;
        }
      } else if (row_valid) {
        fwd_store_o32<D>(p, t, row, head, cc * 32, r, inv_l);
      }
    }
    if (n > 0) {
      // O is read: the next tile's first P.V may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.o_empty[qt]);
    }
    const float lse = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994530942f
                                    : -INFINITY;
    if (p.num_splits > 1)
      fwd_store_part_lse(p, t, row, head, lse);
    else if (p.return_lse && row_valid)
      p.lse[static_cast<size_t>(head) * p.total_q + t.q0 + row] = lse;
  }
  if (st.single && p.num_splits == 1) {  // every thread of the tile meets the barrier
    named_bar_sync(1 + qt, 128);
    if (ok) fwd_copy_out<D, 128>(p, t, s.q + qt * C::Q_BYTES, tile_row0, threadIdx.x & 127);
  }
  // tile 0 takes tile 1's arrive from the tile's last turn
  if (pingpong && qt == 0 && n > 0) named_bar_sync(bar_t0, 64);
  st.g += n;
  if (n > 0) ++st.nt;
  st.ok = ok;
}

// ---------------------------------------------------------------------------
// softmax with 16 rows per warp (head_dim 64, 96-key blocks; head_dim 256,
// 128-key blocks): eight warps per query tile, warp (quadrant, lane half lh)
// serving the 16 tile rows [32 quad + 16 lh, +16) over all keys of every
// block, through 16-lane tensor-memory accesses.  Thread t holds rows
// rt0 = first + t/4 and rt0 + 8 and, of every 8 keys of the block, keys
// 2(t%4) and 2(t%4) + 1: score register 4x + 2r + e is row rt0 + 8r, key
// 8x + 2(t%4) + e.  The four threads of a row combine its max and sum with two
// shuffles, so no warp waits for another warp's scores and the warps that
// share an SM sub-partition drift apart, keeping its exp unit busy.
// ---------------------------------------------------------------------------
template <int D, bool CAUSAL, bool SOFTCAP>
__device__ __forceinline__ void fwd_softmax_rows16(const FwdParams& p, const FwdTile& t,
                                                   const FwdSmem& s, uint32_t tmem, int qt,
                                                   int lh, FwdSoftState& st) {
  using C = FwdCfg<D>;
  constexpr int NX = C::BN / 8;  // 8-key groups per block: 12 or 16
  static_assert((C::BN == 96 || C::BN == 128) && D % 64 == 0, "16-row layout");
  const int quad = (threadIdx.x >> 5) & 3;
  const int lane = lane_id();
  const int cq = lane & 3;
  const int rt0 = quad * 32 + lh * 16 + (lane >> 2);
  const int tile_row0 = t.m_base + qt * t.rows;
  const int delta = t.sk - t.sq;
  int row[2], head[2], key_lim[2], key_lo[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int rt = rt0 + 8 * r;
    row[r] = tile_row0 + (rt >> p.pack_shift);
    head[r] = t.h + (rt & ((1 << p.pack_shift) - 1));
    key_lim[r] = CAUSAL ? min(t.sk, row[r] + delta + p.hi_off + 1) : t.sk;
    key_lo[r] = row[r] + delta - p.lo_off;
  }
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32 + lh * 16) << 16;
  const int n = t.n_blocks;
  const uint32_t g0 = __shfl_sync(0xffffffffu, st.g, 0);  // see fwd_softmax
  const float c = SOFTCAP ? 1.f : p.scale_log2;
  const int mask_from = CAUSAL ? min(t.sk, tile_row0 + delta + p.hi_off + 1) : t.sk;
  const int lo_until = tile_row0 + (t.rows - 1) + delta - p.lo_off;

  TRACE_INIT();
  [[maybe_unused]] const bool tr_on = (lh == 0) && (quad == 0) && (lane == 0);
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  bool ok = true;
  for (int j = 0; j < n; ++j) {
    const uint32_t g = g0 + j;  // this block's index over the CTA's tiles
    const int slot = C::DBUF ? 2 * qt + (g & 1) : (g & 1);
    [[maybe_unused]] const int tr = (tr_on && j < 64) ? 1024 * qt + j * 8 : -1;
    if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full[slot], (g >> 1) & 1, s.abort, p.err,
                                           ERR_FWD_SOFTMAX | 1, p.timeout_ns))) {
      ok = false;
      break;
    }
    tc_fence_after();
    TRACE(tr);
    const uint32_t s_addr = tmem + lane_base + slot * C::BN;
    uint32_t sr[4 * NX];
    if constexpr (NX == 16) {
      tmem_ld16r_x16(s_addr, sr);
    } else {
      uint32_t sa[32], sb[16];
      tmem_ld16r_x8_x4(s_addr, sa, s_addr + 64, sb);
#pragma unroll
      for (int i = 0; i < 32; ++i) sr[i] = sa[i];
#pragma unroll
      for (int i = 0; i < 16; ++i) sr[32 + i] = sb[i];
    }
    const int kb = (t.n_lo + j) * C::BN;  // segment-local key of column 0
    const bool masked = (kb + C::BN > mask_from) || (kb < lo_until);
    if (masked) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int lim = key_lim[r] - kb - 2 * cq, lo = key_lo[r] - kb - 2 * cq;
#pragma unroll
        for (int x = 0; x < NX; ++x)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (8 * x + e >= lim || 8 * x + e < lo) sr[4 * x + 2 * r + e] = 0xff800000u;  // -inf
      }
    }
    if constexpr (SOFTCAP) fwd_cap_scores(p, sr, masked);
    // row maxima: four chains per row over this thread's keys, then the row's
    // other three threads
    float mx[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float ch[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int x = 0; x < NX; ++x)
        ch[x & 3] = fmax3(ch[x & 3], __uint_as_float(sr[4 * x + 2 * r]),
                          __uint_as_float(sr[4 * x + 2 * r + 1]));
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
    {
      const uint64_t cc2 = f2_pack(c, c);
      uint64_t acc[2][2] = {{0ull, 0ull}, {0ull, 0ull}};
      uint32_t pk[2 * NX];  // register 2x + r: P of keys 8x + 2(t%4) + {0, 1} of row rt0 + 8r
#pragma unroll
      for (int x = 0; x < NX; ++x)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[4 * x + 2 * r]),
                                             __uint_as_float(sr[4 * x + 2 * r + 1])),
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
      // keys 2i, 2i + 1 of the block have their P at column i of the slot
      if constexpr (NX == 16) {
        tmem_st16h_x16(s_addr, pk);
      } else {
        uint32_t pa[16], pb[8];
#pragma unroll
        for (int i = 0; i < 16; ++i) pa[i] = pk[i];
#pragma unroll
        for (int i = 0; i < 8; ++i) pb[i] = pk[16 + i];
        tmem_st16h_x8(s_addr, pa);
        tmem_st16h_x4(s_addr + 32, pb);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float a0, a1;
        f2_unpack(f2_add(acc[r][0], acc[r][1]), a0, a1);
        l_run[r] += a0 + a1;  // this thread's share; the row's four are summed at the end
      }
    }
    TRACE(tr + 2);
    if (__any_sync(0xffffffffu, rescale)) {
      // O must not be rescaled while the previous P.V MMA may still write it
      // (the parity of phase g-1 of o_ready is unambiguous, see fwd_softmax)
      if (!__all_sync(0xffffffffu, mbar_wait(&s.o_ready[qt], (g - 1) & 1, s.abort, p.err,
                                             ERR_FWD_SOFTMAX | 2, p.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t o_addr = tmem + lane_base + C::O_COL0 + qt * D;
#pragma unroll 1
      for (int hc = 0; hc < D / 64; ++hc) {
        uint32_t o[32];
        tmem_ld16r_x8(o_addr + hc * 64, o);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[(i >> 1) & 1]);
        tmem_st16r_x8(o_addr + hc * 64, o);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.p_full[slot]);
    TRACE(tr + 3);
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
  // the tile's last P.V, on o_final (see fwd_softmax)
  [[maybe_unused]] const int tre = tr_on ? 900 + 4 * qt : -1;
  TRACE(tre);
  fwd_test_delay(p);
  if (ok && n > 0)
    ok = __all_sync(0xffffffffu, mbar_wait(&s.o_final[qt], st.nt & 1, s.abort, p.err,
                                           ERR_FWD_SOFTMAX | 3, p.timeout_ns));
  TRACE(tre + 1);
  if (ok) {
    tc_fence_after();
    const uint32_t o_addr = tmem + lane_base + C::O_COL0 + qt * D;
#pragma unroll 1
    for (int hc = 0; hc < D / 64; ++hc) {  // columns [64 hc, 64 hc + 64)
      uint32_t o[32];
      if (n > 0) {
        tmem_ld16r_x8(o_addr + hc * 64, o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (row[r] >= t.sq) continue;
        const size_t rh = static_cast<size_t>(t.q0 + row[r]) * p.nheads_q + head[r];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float v0 = __uint_as_float(o[4 * x + 2 * r]) * inv_l[r];
          const float v1 = __uint_as_float(o[4 * x + 2 * r + 1]) * inv_l[r];
          const int col = hc * 64 + 8 * x + 2 * cq;
          if (p.num_splits > 1)  // SplitKV: fp32 partial
            *reinterpret_cast<float2*>(
                p.o_part + (static_cast<size_t>(t.split) * p.total_q * p.nheads_q + rh) * D +
                col) = make_float2(v0, v1);
          else if (st.single)  // into the Q buffer, 16-byte chunk 8 hc + x of the row
            *reinterpret_cast<uint32_t*>(s.q + qt * C::Q_BYTES + (rt0 + 8 * r) * (D * 2) +
                                         (((8 * hc + x) ^ ((rt0 + 8 * r) & 7)) * 16) + 4 * cq) =
                pack_bf16(v0, v1);
          else  // columns col, col + 1 of the row, as bf16
            *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.out) + rh * D + col) =
                pack_bf16(v0, v1);
        }
      }
    }
    if (n > 0) {
      // O is read: the next tile's first P.V may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.o_empty[qt]);
    }
    if (cq == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float lse = (l_run[r] > 0.f)
                              ? (m_run[r] + __log2f(l_run[r])) * 0.69314718055994530942f
                              : -INFINITY;
        if (p.num_splits > 1)
          fwd_store_part_lse(p, t, row[r], head[r], lse);
        else if (p.return_lse && row[r] < t.sq)
          p.lse[static_cast<size_t>(head[r]) * p.total_q + t.q0 + row[r]] = lse;
      }
    }
  }
  if (st.single && p.num_splits == 1) {  // every thread of the tile meets the barrier
    named_bar_sync(1 + qt, 256);
    if (ok)
      fwd_copy_out<D, 256>(p, t, s.q + qt * C::Q_BYTES, tile_row0, lh * 128 + quad * 32 + lane);
  }
  TRACE(tre + 2);
  st.g += n;
  if (n > 0) ++st.nt;
  st.ok = ok;
}

// One CTA per SM works through its share of the tiles (fwd_tile_index); every
// role walks the same sequence, and the barriers' phases carry on from tile to
// tile, so the next tile's Q and K/V loads and its first S overlap the current
// tile's last blocks and epilogue.
template <int D, bool CAUSAL, bool SOFTCAP>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const FwdSmem s = fwd_smem<D>(base);
  const int warp = threadIdx.x >> 5;
  TRACE_INIT();
  if (threadIdx.x == 0) TRACE(950);
  // a CTA whose tiles hold no query row (with one CTA per tile, the grid is
  // sized by the longest segment) leaves before any set-up
  {
    bool work = false;
    for (int k = 0; !work; ++k) {
      const long long L = fwd_tile_index(p, k);
      if (L < 0) break;
      FwdTile t;
      work = fwd_tile<D, CAUSAL>(p, t, L);
    }
    if (!work) return;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(&s.q_full[i], 1);
      mbar_init(&s.q_empty[i], 1);
    }
    // every MMA warp releases each ring stage once (one with no rows in a
    // tile releases that tile's stages without reading them)
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&s.kv_full[i], 1);
      mbar_init(&s.kv_empty[i], C::NQ);
    }
    for (int i = 0; i < C::NSS; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], 4 * C::ROW_SPLIT);  // one arrival per softmax warp of the tile
    }
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(&s.o_ready[i], 1);
      mbar_init(&s.o_final[i], 1);
      mbar_init(&s.o_empty[i], 4 * C::ROW_SPLIT);
    }
    *s.abort = 0;
    fence_mbar_init();
  }
  if (warp == C::LOAD_WARP && lane_id() == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(s.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_base;

  if (warp < C::SOFTMAX_WARPS) {
    const int grp = warp / 4;
    const int qt = grp / C::ROW_SPLIT;
    FwdSoftState st;
    st.single = fwd_tile_index(p, 1) < 0;
    for (int k = 0; st.ok; ++k) {
      const long long L = fwd_tile_index(p, k);
      if (L < 0) break;
      FwdTile t;
      fwd_tile<D, CAUSAL>(p, t, L);
      fwd_tile_uniform(t);
      if (t.m_base + qt * t.rows >= t.sq) continue;  // no rows for this query tile
      if constexpr (C::ROW_SPLIT == 2)
        fwd_softmax_rows16<D, CAUSAL, SOFTCAP>(p, t, s, tmem, qt, grp % 2, st);
      else
        fwd_softmax<D, CAUSAL, SOFTCAP>(p, t, s, tmem, qt, st);
    }
  } else if (warp == C::LOAD_WARP) {
    if (lane_id() == 0) fwd_load<D, CAUSAL>(p, s, &tmQ, &tmK, &tmV);
  } else {
    if (warp == C::MMA_WARP) fwd_mma<D, CAUSAL, 0>(p, s, tmem);
    else if constexpr (C::NQ == 2) fwd_mma<D, CAUSAL, 1>(p, s, tmem);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) TRACE(952);
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// SplitKV combine (the FA4 repository guide, Forward Kernels: a combine kernel
// merges the SplitKV partial results).  Split s of a row holds O_s (normalised
// over its own keys) and LSE_s; over all splits LSE = log sum_s exp(LSE_s) and
// O = sum_s exp(LSE_s - LSE) O_s.  One warp per (row, head); a row whose
// splits all saw no key gets O = 0 and LSE = -inf.  HBM-bound.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    attn_fwd_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                            uint16_t* __restrict__ out, float* __restrict__ lse, int total_q,
                            int nheads_q, int num_splits, int return_lse) {
  constexpr int VPL = D / 32;  // columns per lane: 2, 4 or 8
  const long long w = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(total_q) * nheads_q) return;  // whole warps leave together
  const int row = static_cast<int>(w / nheads_q), h = static_cast<int>(w % nheads_q);
  auto lse_of = [&](int sp) {
    return lse_part[(static_cast<size_t>(sp) * nheads_q + h) * total_q + row];
  };
  float m = -INFINITY;
  for (int sp = lane; sp < num_splits; sp += 32) m = fmaxf(m, lse_of(sp));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  float sum = 0.f;
  if (m != -INFINITY) {
    for (int sp = 0; sp < num_splits; ++sp) {
      const float l = lse_of(sp);
      if (l == -INFINITY) continue;
      const float wgt = expf(l - m);
      sum += wgt;
      const float* src =
          o_part + ((static_cast<size_t>(sp) * total_q + row) * nheads_q + h) * D + lane * VPL;
#pragma unroll
      for (int i = 0; i < VPL; i += 2) {
        const float2 v = *reinterpret_cast<const float2*>(src + i);
        acc[i] += wgt * v.x;
        acc[i + 1] += wgt * v.y;
      }
    }
  }
  const float inv = (sum > 0.f) ? 1.f / sum : 0.f;
  uint32_t* dst = reinterpret_cast<uint32_t*>(
      out + (static_cast<size_t>(row) * nheads_q + h) * D + lane * VPL);
#pragma unroll
  for (int i = 0; i < VPL; i += 2) dst[i / 2] = pack_bf16(acc[i] * inv, acc[i + 1] * inv);
  if (return_lse && lane == 0)
    lse[static_cast<size_t>(h) * total_q + row] = (sum > 0.f) ? m + logf(sum) : -INFINITY;
}

}  // namespace attn

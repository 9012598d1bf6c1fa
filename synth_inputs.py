"""Seeded synthetic inputs for exact attention -- shared by tests, smoke and bench.

This module holds no attention arithmetic: it only draws random numbers and
packs segment lengths into cu_seqlens.  Both the CUDA path and the fp64 oracle
take what it produces, so it is the one piece of code the two sides share.

Recipe (the pages' own benchmark inputs, restated):
  * q, k, v and then dO are drawn in that order from one CPU
    ``torch.Generator`` seeded with ``seed``, as N(0, 1) float32, and rounded to
    bf16 (round-to-nearest-even).  The cosmos issue #118 script draws q, k, v
    from a single generator seeded 0; the FA4 issue #2729 repro draws bf16
    N(0, 1) tensors after ``torch.manual_seed(0)``.
  * Packed variable-length batches: segment lengths are drawn uniformly from
    [lo, hi] with ``random.Random(seed)`` until the next draw would overflow the
    token total; the last segment takes the remainder (it may be shorter than
    ``lo``, which exercises short tails on purpose).
  * Dense batches are packed as equal segments, cu = [0, S, 2S, ...].
"""
from __future__ import annotations

import random
from dataclasses import dataclass, field

import numpy as np
import torch


def varlen_lengths(total: int, lo: int, hi: int, seed: int = 0) -> list[int]:
    rng = random.Random(seed)
    lengths: list[int] = []
    used = 0
    while used < total:
        n = rng.randint(lo, hi)
        if used + n > total:
            n = total - used
        lengths.append(n)
        used += n
    return lengths


def cu_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def dense_lengths(batch: int, seqlen: int) -> list[int]:
    return [seqlen] * batch


def randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_tensors(t_q: int, t_k: int, hq: int, hkv: int, d: int, seed: int = 0,
                 with_dout: bool = True):
    """q [Tq,Hq,D], k, v [Tk,Hkv,D], dout [Tq,Hq,D] (or None) as bf16 CPU tensors."""
    g = torch.Generator().manual_seed(seed)
    q = randn_bf16((t_q, hq, d), g)
    k = randn_bf16((t_k, hkv, d), g)
    v = randn_bf16((t_k, hkv, d), g)
    dout = randn_bf16((t_q, hq, d), g) if with_dout else None
    return q, k, v, dout


@dataclass
class Workload:
    """One attention problem: packed segments, heads, head_dim and masking."""

    name: str
    lengths_q: list
    hq: int
    hkv: int
    d: int
    causal: bool
    lengths_k: list = field(default=None)
    seed: int = 0
    window: tuple = None      # (left, right) key-distance bounds; None = no window
    softcap: float = 0.0      # > 0: scores capped at softcap * tanh(s / softcap)

    def __post_init__(self):
        if self.lengths_k is None:
            self.lengths_k = list(self.lengths_q)

    @property
    def scale(self) -> float:
        return self.d ** -0.5

    @property
    def cu_q(self) -> np.ndarray:
        return cu_from_lengths(self.lengths_q)

    @property
    def cu_k(self) -> np.ndarray:
        return cu_from_lengths(self.lengths_k)

    @property
    def total_q(self) -> int:
        return int(sum(self.lengths_q))

    @property
    def total_k(self) -> int:
        return int(sum(self.lengths_k))

    @property
    def max_q(self) -> int:
        return int(max(self.lengths_q)) if self.lengths_q else 0

    @property
    def max_k(self) -> int:
        return int(max(self.lengths_k)) if self.lengths_k else 0

    def tensors(self, with_dout: bool = True):
        return make_tensors(self.total_q, self.total_k, self.hq, self.hkv, self.d,
                            self.seed, with_dout)

    def fwd_flops(self) -> float:
        """Forward FLOPs: 4 * s_q * s_k * Hq * D per segment, halved when causal
        (the pages' convention, for s_q = s_k).  With a local window, or causal
        with s_q != s_k: 4 * Hq * D per allowed (row, key) pair, counted exactly."""
        square = all(a == b for a, b in zip(self.lengths_q, self.lengths_k))
        no_window = self.window is None or (self.window[0] < 0 and self.window[1] < 0)
        if no_window and (square or not self.causal):
            f = sum(4.0 * a * b * self.hq * self.d
                    for a, b in zip(self.lengths_q, self.lengths_k))
            return f / 2 if self.causal else f
        # windows, and causal segments with s_q != s_k (where halving does not
        # describe the mask): count the allowed (row, key) pairs
        left, right = self.window if not no_window else (-1, -1)
        pairs = 0
        for sq, sk in zip(self.lengths_q, self.lengths_k):
            diag = np.arange(sq, dtype=np.int64) + (sk - sq)
            hi = np.full(sq, sk - 1, np.int64)
            if self.causal:
                hi = np.minimum(hi, diag)
            if right >= 0:
                hi = np.minimum(hi, diag + right)
            lo = np.zeros(sq, np.int64) if left < 0 else np.maximum(0, diag - left)
            pairs += int(np.maximum(0, hi - lo + 1).sum())
        return 4.0 * pairs * self.hq * self.d

    def fwd_bytes(self, return_lse: bool = True) -> float:
        """Bytes the forward must move through HBM at the least: read Q, K, V,
        write O (bf16) and, if asked, the fp32 LSE."""
        e = 2 * self.d  # bytes per row of one head
        return (e * (2 * self.total_q * self.hq + 2 * self.total_k * self.hkv)
                + (4 * self.hq * self.total_q if return_lse else 0))

    def bwd_main_bytes(self) -> float:
        """Bytes the backward's main kernel must move at the least: read Q, dO,
        K, V, the LSE and D_i, write dK and dV.  The fp32 dQ accumulator is
        traffic of this implementation, not of the method, and is not counted."""
        e = 2 * self.d
        return e * (2 * self.total_q * self.hq + 4 * self.total_k * self.hkv) + 8 * self.hq * self.total_q


# The five problem families of the pages, by name.
def tiny() -> Workload:
    return Workload("tiny_b1_s256_h2_d64", [256], 2, 2, 64, False)


def varlen_gqa(total: int = 16384, seed: int = 0) -> Workload:
    return Workload(f"varlen_gqa_t{total}_hq32_hkv8_d128",
                    varlen_lengths(total, 128, 4096, seed), 32, 8, 128, False, seed=seed)


def single_gqa(seqlen: int, causal: bool = False) -> Workload:
    return Workload(f"gqa_s{seqlen}_hq32_hkv8_d128{'_causal' if causal else ''}",
                    [seqlen], 32, 8, 128, causal)


def gqa_sliding_window(seqlen: int = 16384, window: int = 4096) -> Workload:
    """The GQA head_dim-128 family with a causal sliding window of `window` keys
    (each row sees itself and the window - 1 keys before it)."""
    return Workload(f"gqa_s{seqlen}_hq32_hkv8_d128_causal_window{window}", [seqlen], 32, 8,
                    128, True, window=(window - 1, 0))


def decode_gqa(q_rows: int = 64, seqlen_k: int = 65536) -> Workload:
    """A short query segment (the last q_rows positions) against a long key
    segment: the SplitKV shape.  GQA 32/8, head_dim 128, causal (bottom-right)."""
    return Workload(f"decode_q{q_rows}_k{seqlen_k}_hq32_hkv8_d128_causal", [q_rows], 32, 8, 128,
                    True, lengths_k=[seqlen_k])


def gqa_softcap(seqlen: int = 16384, cap: float = 50.0) -> Workload:
    """The GQA head_dim-128 family, causal, with the scores soft-capped."""
    return Workload(f"gqa_s{seqlen}_hq32_hkv8_d128_causal_softcap{cap:g}", [seqlen], 32, 8, 128,
                    True, softcap=cap)


def short_segments(seqlen: int = 128, total: int = 16384) -> Workload:
    """The GQA head_dim-128 family as a packed batch of equal short segments
    (total // seqlen segments of seqlen tokens, non-causal).  A 128-token
    segment does about 100 FLOPs per byte it has to move, under the B200's
    ridge of roughly 210, so such batches are bound by HBM, not by the
    tensor cores."""
    return Workload(f"varlen_short_s{seqlen}_t{total}_hq32_hkv8_d128",
                    dense_lengths(total // seqlen, seqlen), 32, 8, 128, False)


def d64_mha() -> Workload:
    return Workload("mha_b2_s16384_h16_d64", dense_lengths(2, 16384), 16, 16, 64, False)


def d256_mha(seqlen: int, causal: bool) -> Workload:
    batch = max(1, 32768 // seqlen)
    return Workload(f"mha_b{batch}_s{seqlen}_h8_d256{'_causal' if causal else ''}",
                    dense_lengths(batch, seqlen), 8, 8, 256, causal)


def d256_gqa8(seqlen: int = 131072, causal: bool = False) -> Workload:
    return Workload(f"gqa8_b1_s{seqlen}_hq8_hkv1_d256{'_causal' if causal else ''}",
                    [seqlen], 8, 1, 256, causal)

"""Seeded synthetic workloads shaped like the pages' multi-LoRA serving cases.

Nothing here computes the LoRA delta.  Each function draws inputs from a
seeded counter-free generator (numpy PCG64 keyed by a SeedSequence of
(seed, tensor tag, indices)), so any tensor can be regenerated on its own and
the CPU oracle and the CUDA path receive identical bytes.

Value recipe (the pages give the geometry, not the values):
  x ~ N(0, 1), A ~ N(0, 1/d_in), B ~ N(0, 0.02) (0.02 read as the variance),
  base weight W ~ N(0, 1/d_in); every tensor is rounded to bf16 (round to
  nearest even).  The base output y = x W^T is formed here in fp64 and rounded
  to bf16, standing in for the caller's base GEMM; for the 128-matrix paged
  workload the base output is drawn directly from N(0, 1), the distribution of
  x W^T, because forming 128 base GEMMs on the host would dominate setup time.

Workload geometry (Llama-2-7B projections, 4096 hidden, d_ff 11008):
  1 tiny decode       d 256, rank 8, 4 adapters, 16 tokens, ids uniform
  2 q_proj decode     d 4096, rank 16, 32 adapters, 64 tokens, ids uniform
  3 segmented prefill d 4096, rank 16, 8 adapters, 4096 tokens in 8 segments
                      with rank-frequency Zipf(1.2) lengths
  4 mixed ranks, MLP  ranks {8,16,32,64} (max 64), 128 adapters, 256 tokens,
                      26 rows without adapter, Zipf(1.0) popularity, shapes
                      4096->11008 and 11008->4096
  5 paged at scale    1000 adapters x 128 matrices (32 layers x q/k/v/o), rank
                      16, 1 MiB pages scattered by a seeded permutation, 512
                      tokens over 64 adapters with Zipf(1.1) popularity
"""

from __future__ import annotations

import functools
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# tensor tags for the seed sequences
_T_X, _T_A, _T_B, _T_W, _T_IDS, _T_Y, _T_RANK, _T_SEG, _T_PICK = range(1, 10)

B_VARIANCE = 0.02


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest, ties to even); returns uint16."""
    u = np.array(a, dtype=np.float32, copy=True).view(np.uint32)
    lsb = u >> 16
    lsb &= 1
    u += np.uint32(0x7FFF)
    u += lsb
    u >>= 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    """N(0, std^2) samples rounded to bf16 bit patterns."""
    z = rng.standard_normal(shape, dtype=np.float32)
    return f32_to_bf16_bits(z * np.float32(std))


def zipf_lengths(total: int, n: int, s: float) -> List[int]:
    """Deterministic rank-frequency Zipf(s) split of `total` into n parts, each
    at least 1: every part gets 1, the remaining total - n is shared in
    proportion to k^-s (k = 1..n) by the largest-remainder rule (ties to the
    lower rank)."""
    if n <= 0:
        return []
    rest = total - n
    w = np.array([k ** (-s) for k in range(1, n + 1)], dtype=np.float64)
    share = rest * w / w.sum()
    base = np.floor(share).astype(np.int64)
    left = int(rest - base.sum())
    rem = share - base
    order = sorted(range(n), key=lambda i: (-rem[i], i))
    for i in order[:left]:
        base[i] += 1
    return [int(b) + 1 for b in base]


def zipf_draw(rng: np.random.Generator, n: int, s: float, size: int) -> np.ndarray:
    """i.i.d. popularity ranks 0..n-1 with P(rank k) proportional to (k+1)^-s."""
    p = np.array([(k + 1) ** (-s) for k in range(n)], dtype=np.float64)
    p /= p.sum()
    return rng.choice(n, size=size, p=p)


@dataclass
class Workload:
    """One batch of the delta path plus the adapter pool it reads.

    targets: (d_in, d_out) of each adapted matrix; rank[slot]: the adapter's
    true rank (same on every target; 0 = slot empty); alpha[slot]; ids[T]
    (-1 = no adapter); seg_offsets/seg_slot: the same batch as contiguous
    segments, when it is a segmented workload.
    """

    name: str
    seed: int
    targets: List[Tuple[int, int]]
    r_max: int
    n_slots: int
    page_bytes: int
    scatter_seed: int
    T: int
    ids: np.ndarray
    rank: np.ndarray
    alpha: np.ndarray
    seg_offsets: Optional[np.ndarray] = None
    seg_slot: Optional[np.ndarray] = None
    y_mode: str = "xw"           # "xw": y = bf16(x W^T); "normal": y ~ N(0,1)
    value_mode: str = "normal"   # "normal" or "integer"
    _cache: Dict = field(default_factory=dict, repr=False)

    # -- derived facts about the batch ------------------------------------
    @property
    def active_slots(self) -> np.ndarray:
        a = self.ids[self.ids >= 0]
        return np.unique(a).astype(np.int32)

    # -- tensors -------------------------------------------------------------
    def adapter(self, slot: int, target: int) -> Tuple[np.ndarray, np.ndarray]:
        """(A bf16 bits [r, d_in], B bf16 bits [d_out, r]) of one slot."""
        key = ("ad", slot, target)
        if key in self._cache:
            return self._cache[key]
        A, B = self._draw_adapter(slot, target)
        if self.T <= 4096 or slot in set(self.active_slots.tolist()):
            self._cache[key] = (A, B)
        return A, B

    def _draw_adapter(self, slot: int, target: int) -> Tuple[np.ndarray, np.ndarray]:
        d_in, d_out = self.targets[target]
        r = int(self.rank[slot])
        if self.value_mode == "integer":
            g = _rng(self.seed, _T_A, slot, target)
            A = f32_to_bf16_bits(g.integers(-2, 3, size=(r, d_in)).astype(np.float32))
            g = _rng(self.seed, _T_B, slot, target)
            B = f32_to_bf16_bits(g.integers(-2, 3, size=(d_out, r)).astype(np.float32))
        else:
            A = normal_bf16(_rng(self.seed, _T_A, slot, target), (r, d_in), 1.0 / np.sqrt(d_in))
            B = normal_bf16(_rng(self.seed, _T_B, slot, target), (d_out, r), np.sqrt(B_VARIANCE))
        return A, B

    def x(self, target: int) -> np.ndarray:
        key = ("x", target)
        if key not in self._cache:
            d_in = self.targets[target][0]
            g = _rng(self.seed, _T_X, target)
            if self.value_mode == "integer":
                self._cache[key] = f32_to_bf16_bits(g.integers(-3, 4, size=(self.T, d_in)).astype(np.float32))
            else:
                self._cache[key] = normal_bf16(g, (self.T, d_in), 1.0)
        return self._cache[key]

    def W(self, target: int) -> np.ndarray:
        """Base weight of the target, bf16 bits [d_out, d_in] (one row per
        output feature): N(0, 1/d_in), or integers in [-2, 2]."""
        key = ("W", target)
        if key not in self._cache:
            d_in, d_out = self.targets[target]
            g = _rng(self.seed, _T_W, target)
            if self.value_mode == "integer":
                self._cache[key] = f32_to_bf16_bits(g.integers(-2, 3, size=(d_out, d_in)).astype(np.float32))
            else:
                self._cache[key] = normal_bf16(g, (d_out, d_in), 1.0 / np.sqrt(d_in))
        return self._cache[key]

    def y_in(self, target: int) -> np.ndarray:
        key = ("y", target)
        if key not in self._cache:
            d_in, d_out = self.targets[target]
            if self.value_mode == "integer":
                g = _rng(self.seed, _T_Y, target)
                y = f32_to_bf16_bits(g.integers(-8, 9, size=(self.T, d_out)).astype(np.float32))
            elif self.y_mode == "normal":
                y = normal_bf16(_rng(self.seed, _T_Y, target), (self.T, d_out), 1.0)
            else:
                xf = bf16_bits_to_f32(self.x(target)).astype(np.float64)
                Wf = bf16_bits_to_f32(self.W(target)).astype(np.float64)
                y = f32_to_bf16_bits((xf @ Wf.T).astype(np.float32))
            self._cache[key] = y
        return self._cache[key]

    def prefetch(self, slots: Sequence[int], targets: Sequence[int], threads: int = 0) -> None:
        """Draw many adapters at once on a thread pool (each tensor has its own
        seed, so the values do not depend on the order or the pool size)."""
        import concurrent.futures as cf
        import os
        jobs = [(int(s), int(t)) for s in slots for t in targets if ("ad", int(s), int(t)) not in self._cache]
        if not jobs:
            return
        n = threads or min(32, os.cpu_count() or 1)

        def one(job):
            s, t = job
            return job, self._draw_adapter(s, t)

        with cf.ThreadPoolExecutor(max_workers=n) as ex:
            for (s, t), val in ex.map(one, jobs):
                self._cache[("ad", s, t)] = val

    def drop(self) -> None:
        self._cache.clear()


def _ids_from_segments(T: int, seg_offsets: np.ndarray, seg_slot: np.ndarray) -> np.ndarray:
    ids = np.full(T, -1, dtype=np.int32)
    for s in range(len(seg_slot)):
        ids[seg_offsets[s]:seg_offsets[s + 1]] = seg_slot[s]
    return ids


def _cfg1(seed: int) -> Workload:
    T, n = 16, 4
    ids = _rng(seed, _T_IDS).integers(0, n, size=T).astype(np.int32)
    return Workload("tiny decode d256 r8 4 adapters 16 tokens", seed, [(256, 256)], 8, n,
                    0, 0, T, ids, np.full(n, 8, np.int32), np.full(n, 16.0))


def _cfg2(seed: int) -> Workload:
    T, n = 64, 32
    ids = _rng(seed, _T_IDS).integers(0, n, size=T).astype(np.int32)
    return Workload("q_proj decode d4096 r16 32 adapters 64 tokens", seed, [(4096, 4096)], 16, n,
                    0, 0, T, ids, np.full(n, 16, np.int32), np.full(n, 32.0))


def _cfg3(seed: int) -> Workload:
    T, n = 4096, 8
    lengths = zipf_lengths(T, n, 1.2)
    order = _rng(seed, _T_SEG).permutation(n).astype(np.int32)
    seg_offsets = np.zeros(n + 1, dtype=np.int32)
    seg_offsets[1:] = np.cumsum(lengths)
    ids = _ids_from_segments(T, seg_offsets, order)
    return Workload("segmented prefill d4096 r16 8 adapters 4096 tokens", seed, [(4096, 4096)], 16, n,
                    0, 0, T, ids, np.full(n, 16, np.int32), np.full(n, 32.0),
                    seg_offsets=seg_offsets, seg_slot=order)


def _cfg4(seed: int) -> Workload:
    T, n = 256, 128
    rank = _rng(seed, _T_RANK).choice(np.array([8, 16, 32, 64]), size=n).astype(np.int32)
    g = _rng(seed, _T_IDS)
    n_none = int(round(0.1 * T))
    none_rows = g.permutation(T)[:n_none]
    slot_of_rank = g.permutation(n)
    ids = slot_of_rank[zipf_draw(g, n, 1.0, T)].astype(np.int32)
    ids[none_rows] = -1
    return Workload("mixed ranks MLP d4096<->11008 r<=64 128 adapters 256 tokens", seed,
                    [(4096, 11008), (11008, 4096)], 64, n, 0, 0, T, ids, rank,
                    2.0 * rank.astype(np.float64))


def _cfg5(seed: int) -> Workload:
    T, n, distinct = 512, 1000, 64
    g = _rng(seed, _T_PICK)
    chosen = np.sort(g.choice(n, size=distinct, replace=False)).astype(np.int32)
    gi = _rng(seed, _T_IDS)
    slot_of_rank = chosen[gi.permutation(distinct)]
    rest = slot_of_rank[zipf_draw(gi, distinct, 1.1, T - distinct)]
    ids = np.concatenate([chosen, rest]).astype(np.int32)
    ids = ids[gi.permutation(T)]
    targets = [(4096, 4096)] * 128          # 32 layers x (q, k, v, o)
    return Workload("paged pool 1000 adapters x 128 matrices r16 512 tokens", seed, targets, 16, n,
                    1 << 20, seed, T, ids.astype(np.int32), np.full(n, 16, np.int32),
                    np.full(n, 32.0), y_mode="normal")


_CONFIGS = {1: _cfg1, 2: _cfg2, 3: _cfg3, 4: _cfg4, 5: _cfg5}


@functools.lru_cache(maxsize=8)
def config(index: int, seed: Optional[int] = None) -> Workload:
    """The five workloads, numbered 1..5; default seed = 1000 + index."""
    return _CONFIGS[index](1000 + index if seed is None else seed)


def integer_case(seed: int, T: int, d_in: int, d_out: int, ranks: Sequence[int],
                 r_max: int, scale_exp: Sequence[int], ids: Optional[Sequence[int]] = None,
                 page_bytes: int = 0, scatter_seed: int = 0) -> Workload:
    """Small brute-force case with small-integer bf16 values (x in [-3,3],
    A and B in [-2,2], y in [-8,8]) and alpha = r * 2^e, so every partial sum
    is an exactly representable integer multiple of a power of two."""
    n = len(ranks)
    rank = np.array(ranks, dtype=np.int32)
    alpha = rank.astype(np.float64) * np.exp2(np.array(scale_exp, dtype=np.float64))
    if ids is None:
        ids = _rng(seed, _T_IDS).integers(-1, n, size=T)
    return Workload("integer case", seed, [(d_in, d_out)], r_max, n, page_bytes, scatter_seed,
                    T, np.asarray(ids, dtype=np.int32), rank, alpha, value_mode="integer")


def custom(seed: int, T: int, targets: Sequence[Tuple[int, int]], ranks: Sequence[int], r_max: int,
           alpha: Optional[Sequence[float]] = None, ids: Optional[Sequence[int]] = None,
           y_mode: str = "normal", page_bytes: int = 0, scatter_seed: int = 0) -> Workload:
    """A workload with the standard value recipe and caller-chosen geometry
    (alpha defaults to 2 r, ids to uniform over the slots)."""
    rank = np.array(ranks, dtype=np.int32)
    a = 2.0 * rank.astype(np.float64) if alpha is None else np.asarray(alpha, dtype=np.float64)
    if ids is None:
        ids = _rng(seed, _T_IDS).integers(0, len(ranks), size=T)
    return Workload("custom", seed, list(targets), r_max, len(ranks), page_bytes, scatter_seed, T,
                    np.asarray(ids, dtype=np.int32), rank, a, y_mode=y_mode)

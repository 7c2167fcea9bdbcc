"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and by the oracle's callers.

This module holds no attention arithmetic: it only draws numbers.  Both sides of every parity check receive the
exact same bits from here (16-bit tensors are widened to fp64 for the oracle without rounding).

* Q, K, V, dO: iid N(0, 1) drawn by torch's CPU generator (seeded per tensor), then rounded to bf16 or fp16
  (round-to-nearest-even).  The pages fix no distribution; N(0, 1) is the plainest reading of "random inputs".
* Key lengths (BERT-shaped workload): len_b = 128 + (splitmix64 draw % 385), i.e. uniform in [128, 512].
* Block mask (long-context block-sparse workload; explainer page, block-sparse section, which gives only the idea
  of skipping whole tiles): union of
    - a diagonal band four tiles wide, read as keeping tile (i, j) iff -2 <= j - i <= 1,
    - a butterfly pattern, keeping (i, j) iff x = i XOR j is a power of two (x != 0 and x & (x - 1) == 0),
    - random tiles, each kept independently with probability 0.02 (one splitmix64 draw per tile in row-major
      order, uniform = (u >> 11) * 2**-53).
  The mask is shared by every batch entry and head.

splitmix64 is the published generator of Steele, Lea and Flood ("Fast splittable pseudorandom number generators",
OOPSLA 2014), in the form popularised by Vigna: state += 0x9E3779B97F4A7C15, then two xor-shift-multiply rounds
(constants 0xBF58476D1CE4E5B9, 0x94D049BB133111EB) and a final xor-shift by 31.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1


def splitmix64(seed: int, n: int) -> np.ndarray:
    """First n outputs of splitmix64 started from state `seed` (uint64 array)."""
    with np.errstate(over="ignore"):
        idx = np.arange(1, n + 1, dtype=np.uint64)
        z = np.uint64(seed & _MASK64) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def splitmix64_scalar(seed: int, n: int) -> list[int]:
    """Plain-integer splitmix64, used to cross-check the vectorised version."""
    out, s = [], seed & _MASK64
    for _ in range(n):
        s = (s + 0x9E3779B97F4A7C15) & _MASK64
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        out.append(z ^ (z >> 31))
    return out


def uniform01(seed: int, n: int) -> np.ndarray:
    """n doubles in [0, 1): top 53 bits of each splitmix64 output times 2**-53."""
    return (splitmix64(seed, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def key_lengths(seed: int, batch: int, lo: int = 128, hi: int = 512) -> np.ndarray:
    """Per-sequence key lengths uniform in [lo, hi] (int32)."""
    u = splitmix64(seed, batch)
    return (np.uint64(lo) + u % np.uint64(hi - lo + 1)).astype(np.int32)


def band_mask(nT: int, below: int = 2, above: int = 1) -> np.ndarray:
    i = np.arange(nT)[:, None]
    j = np.arange(nT)[None, :]
    return ((j - i >= -below) & (j - i <= above)).astype(np.uint8)


def butterfly_mask(nT: int) -> np.ndarray:
    i = np.arange(nT)[:, None]
    j = np.arange(nT)[None, :]
    x = i ^ j
    return ((x != 0) & ((x & (x - 1)) == 0)).astype(np.uint8)


def random_tile_mask(nT: int, seed: int, p: float = 0.02) -> np.ndarray:
    return (uniform01(seed, nT * nT) < p).reshape(nT, nT).astype(np.uint8)


def blocksparse_mask(nT: int, seed: int, p: float = 0.02) -> np.ndarray:
    """Band (width 4) | butterfly | random p, as uint8 [nT, nT]."""
    return (band_mask(nT) | butterfly_mask(nT) | random_tile_mask(nT, seed, p)).astype(np.uint8)


_TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def gaussian(shape, seed: int, dtype: str) -> torch.Tensor:
    """iid N(0,1) rounded to a 16-bit float type, on the CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(_TORCH_DT[dtype])


@dataclass
class Workload:
    """One synthetic attention problem. Tensors are CPU 16-bit [B, H, N, d]."""
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str
    causal: bool
    seed: int
    key_lens: bool = False
    blocksparse: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def nT(self) -> int:
        return -(-self.N // 128)

    def tensors(self):
        """(q, k, v, dO) as CPU 16-bit tensors."""
        shape = (self.B, self.H, self.N, self.d)
        return tuple(gaussian(shape, self.seed * 1000 + t, self.dtype) for t in range(4))

    def key_lens_array(self):
        return key_lengths(self.seed + 77, self.B) if self.key_lens else None

    def block_mask(self):
        return blocksparse_mask(self.nT, self.seed + 99) if self.blocksparse else None


def workloads() -> dict[str, Workload]:
    """The five workload shapes: tiny, GPT-2-small, BERT-large, long-context causal sweep, block-sparse; and the
    long-context shape at head dim 256 for the d = 256 kernels."""
    w = {
        "tiny": Workload("tiny", 1, 2, 256, 64, "bf16", False, 0),
        "gpt2": Workload("gpt2", 8, 12, 1024, 64, "bf16", True, 1),
        "bert": Workload("bert", 16, 16, 512, 64, "bf16", False, 2, key_lens=True),
        "lc4k": Workload("lc4k", 1, 16, 4096, 128, "bf16", True, 3),
        "lc8k": Workload("lc8k", 1, 16, 8192, 128, "bf16", True, 3),
        "lc16k": Workload("lc16k", 1, 16, 16384, 128, "bf16", True, 3),
        "bs64k": Workload("bs64k", 1, 8, 65536, 64, "fp16", False, 4, blocksparse=True),
        "lc8k_d256": Workload("lc8k_d256", 1, 16, 8192, 256, "bf16", True, 5),
    }
    return w


def sample_rows(seed: int, BH: int, N: int, n: int):
    """n distinct (flattened head, row) pairs drawn with splitmix64, sorted."""
    total = BH * N
    n = min(n, total)
    u = splitmix64(seed, 4 * n + 16)
    picks, seen = [], set()
    for x in (u % np.uint64(total)).tolist():
        if x not in seen:
            seen.add(x)
            picks.append(x)
            if len(picks) == n:
                break
    picks = np.array(sorted(picks), dtype=np.int64)
    return picks // N, picks % N


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a 16-bit tensor to fp64 numpy."""
    return t.to(torch.float64).numpy()

"""Seeded synthetic inputs for the LLM.int8() linear layer C = X.W.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds no arithmetic of the method: it only draws random
numbers and casts them to IEEE binary16, so both sides start from the very same
bits.

Structure of the activations follows what the LLM.int8() pages report about
emergent outlier features in OPT-class models:

* a handful of feature columns (at most ~7) carry the outliers
  ("LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale",
  section "Emergent Large Magnitude Features", Table 4 summary);
* an outlier column is large in ~75% of the sequence positions
  (same page, Figure 3a discussion);
* outliers are one-sided: a column keeps one sign (same page, Table 4
  "asymmetric" remark);
* magnitudes run from the 6.0 threshold up to tens (median ~60 at 175B,
  Figure 4a discussion).

Recipe (all draws from ``numpy.random.default_rng(seed)`` in this order):

1. X ~ N(0, 1), drawn as float32 and cast to float16 (round to nearest even).
2. Outlier columns: fixed (tiny case) or drawn without replacement from
   [0, h); sorted ascending.
3. For each outlier column, in ascending order: one sign (+1 / -1, p=1/2),
   then an exact subset of round(p * s) rows drawn without replacement, then
   magnitudes U(lo, hi) for those rows; values sign*U cast to float16 overwrite
   X in that column.
4. W ~ N(0, sigma), drawn as float32 in row blocks, scaled by sigma and cast
   to float16.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = ["Workload", "WORKLOADS", "get_workload", "make_x", "make_w",
           "make_inputs"]


@dataclass(frozen=True)
class Workload:
    """One synthetic linear-layer problem X[s,h] . W[h,o]."""

    name: str
    s: int
    h: int
    o: int
    seed: int
    n_outlier_cols: int
    outlier_lo: float
    outlier_hi: float
    outlier_row_frac: float
    w_sigma: float
    fixed_outlier_cols: Tuple[int, ...] = field(default_factory=tuple)
    alpha: float = 6.0
    description: str = ""

    @property
    def int8_ops(self) -> int:
        return 2 * self.s * self.h * self.o

    @property
    def compulsory_bytes(self) -> int:
        """X read (fp16) + Wq read (int8) + C write (fp16) + row/col scales."""
        return 2 * self.s * self.h + self.h * self.o + 2 * self.s * self.o \
            + 4 * (self.s + self.o)


WORKLOADS = {
    "tiny": Workload(
        name="tiny", s=16, h=256, o=256, seed=0, n_outlier_cols=2,
        outlier_lo=8.0, outlier_hi=20.0, outlier_row_frac=0.8, w_sigma=0.02,
        fixed_outlier_cols=(7, 200),
        description="tiny correctness case 16x256x256, outlier columns 7 and 200"),
    "opt6.7b_attn_prefill": Workload(
        name="opt6.7b_attn_prefill", s=2048, h=4096, o=4096, seed=1,
        n_outlier_cols=6, outlier_lo=6.0, outlier_hi=60.0,
        outlier_row_frac=0.75, w_sigma=0.02,
        description="OPT-6.7B-like attention projection, prefill"),
    "opt13b_ffn_up_prefill": Workload(
        name="opt13b_ffn_up_prefill", s=4096, h=5120, o=20480, seed=2,
        n_outlier_cols=7, outlier_lo=6.0, outlier_hi=60.0,
        outlier_row_frac=0.75, w_sigma=0.02,
        description="OPT-13B-like FFN up-projection, prefill"),
    "opt175b_ffn_up_prefill": Workload(
        name="opt175b_ffn_up_prefill", s=2048, h=12288, o=49152, seed=3,
        n_outlier_cols=7, outlier_lo=6.0, outlier_hi=100.0,
        outlier_row_frac=0.75, w_sigma=0.01,
        description="OPT-175B-like FFN up-projection, prefill"),
    "opt175b_decode": Workload(
        name="opt175b_decode", s=8, h=12288, o=49152, seed=4,
        n_outlier_cols=7, outlier_lo=6.0, outlier_hi=100.0,
        outlier_row_frac=1.0, w_sigma=0.01,
        description="OPT-175B-like decode batch of 8 rows"),
}

WORKLOAD_ORDER = ["tiny", "opt6.7b_attn_prefill", "opt13b_ffn_up_prefill",
                  "opt175b_ffn_up_prefill", "opt175b_decode"]


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


def _outlier_columns(rng: np.random.Generator, wl: Workload,
                     h: int) -> np.ndarray:
    if wl.fixed_outlier_cols:
        return np.array(sorted(wl.fixed_outlier_cols), dtype=np.int64)
    cols = rng.choice(h, size=wl.n_outlier_cols, replace=False)
    return np.sort(cols).astype(np.int64)


def make_x(wl: Workload, s: Optional[int] = None, h: Optional[int] = None,
           rng: Optional[np.random.Generator] = None
           ) -> Tuple[np.ndarray, np.ndarray]:
    """Return (X float16 [s,h], planted outlier columns int64)."""
    s = wl.s if s is None else s
    h = wl.h if h is None else h
    if rng is None:
        rng = np.random.default_rng(wl.seed)
    x = rng.standard_normal((s, h), dtype=np.float32).astype(np.float16)
    cols = _outlier_columns(rng, wl, h)
    n_rows = int(round(wl.outlier_row_frac * s))
    for c in cols:
        sign = 1.0 if rng.random() < 0.5 else -1.0
        rows = rng.choice(s, size=n_rows, replace=False)
        mag = rng.uniform(wl.outlier_lo, wl.outlier_hi, size=n_rows)
        x[rows, c] = (sign * mag).astype(np.float16)
    return x, cols


def make_w(wl: Workload, h: Optional[int] = None, o: Optional[int] = None,
           rng: Optional[np.random.Generator] = None,
           block_rows: int = 1024) -> np.ndarray:
    """Return W float16 [h,o] ~ N(0, sigma), drawn in row blocks."""
    h = wl.h if h is None else h
    o = wl.o if o is None else o
    if rng is None:
        rng = np.random.default_rng(wl.seed + 1_000_003)
    w = np.empty((h, o), dtype=np.float16)
    sigma = np.float32(wl.w_sigma)
    for r0 in range(0, h, block_rows):
        r1 = min(h, r0 + block_rows)
        blk = rng.standard_normal((r1 - r0, o), dtype=np.float32)
        blk *= sigma
        w[r0:r1] = blk.astype(np.float16)
    return w


def make_inputs(name: str):
    """Return (workload, X, planted_cols, W) for a named workload."""
    wl = get_workload(name)
    x, cols = make_x(wl)
    w = make_w(wl)
    return wl, x, cols, w


def random_x(rng: np.random.Generator, s: int, h: int,
             outlier_cols: Sequence[int] = (), lo: float = 6.0,
             hi: float = 60.0, row_frac: float = 0.75,
             scale: float = 1.0) -> np.ndarray:
    """Small ad-hoc X for edge-case tests (same recipe, explicit columns)."""
    x = (rng.standard_normal((s, h), dtype=np.float32) * np.float32(scale)
         ).astype(np.float16)
    n_rows = max(1, int(round(row_frac * s))) if s > 0 else 0
    for c in outlier_cols:
        sign = 1.0 if rng.random() < 0.5 else -1.0
        rows = rng.choice(s, size=n_rows, replace=False)
        mag = rng.uniform(lo, hi, size=n_rows)
        x[rows, c] = (sign * mag).astype(np.float16)
    return x


def random_w(rng: np.random.Generator, h: int, o: int,
             sigma: float = 0.02) -> np.ndarray:
    return (rng.standard_normal((h, o), dtype=np.float32) * np.float32(sigma)
            ).astype(np.float16)

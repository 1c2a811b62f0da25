"""Seeded synthetic inputs for sparse-mask scaled dot-product attention.

This module only draws numbers. It holds none of the method's arithmetic: no
score, no softmax, no mask predicate and no CSR construction. Both the CUDA path
(through its tests and the benchmark) and the CPU oracle consume what it returns:
the attention inputs Q, K, V, the parameters from which a mask is built (window
half-widths, random column draws, key-padding lengths) and the additive
mask/bias tensors.

Recipe (every config):
  * numpy PCG64 ``default_rng(seed)``; tensors use ``seed = 1000 + config index``,
    the mask of batch element ``b`` uses ``default_rng([1000 + config index, b])``.
  * Normal draws are taken in float64, rounded to float32 (round to nearest even)
    and, for bf16 tensors, rounded again to bf16 (round to nearest even on the
    float32 bit pattern). bf16 tensors travel as ``uint16`` bit patterns.
  * Random columns (the "random general sparse" pattern) are drawn here, so the
    mask builder receives them as COO candidates and never draws random numbers.

The five workloads follow the pages' patterns: a sliding window ("Sparse
Attention" notes page, pattern list), a per-token variable window ("[Proposal]
Unified Interface/Implementation for Sparse Attention", the variable window
length remark), a random general mask (same proposal, user-defined CSR mask),
block + strided + global tokens (notes page, pattern list) and the Evoformer
key-padding mask + pair bias ("support attentions in AlphaFold2", mask and bias
shape rules).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

BF16 = "bf16"
F32 = "f32"


def f64_to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even) and return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    # keep NaN a NaN and infinities exact
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32)


@dataclass
class Tensor:
    """A host tensor in the dtype the CUDA path reads (uint16 bits for bf16)."""

    raw: np.ndarray
    dtype: str

    @property
    def shape(self):
        return self.raw.shape

    def f64(self) -> np.ndarray:
        if self.dtype == BF16:
            return bf16_bits_to_f64(self.raw)
        return self.raw.astype(np.float64)

    def f32(self) -> np.ndarray:
        if self.dtype == BF16:
            return bf16_bits_to_f32(self.raw)
        return self.raw.astype(np.float32)


def make_tensor(values_f64: np.ndarray, dtype: str) -> Tensor:
    f32 = f64_to_f32(values_f64)
    if dtype == BF16:
        return Tensor(f32_to_bf16_bits(f32), BF16)
    if dtype == F32:
        return Tensor(f32, F32)
    raise ValueError(dtype)


@dataclass
class MaskParams:
    """What a mask pattern is built from. ``kind`` is one of
    ``sliding``, ``varwin``, ``bsg`` (block + strided + global), ``coo`` or ``dense``."""

    kind: str
    n: int
    num_masks: int = 1
    window: int = 0                       # sliding: half-width w
    half_widths: Optional[np.ndarray] = None   # varwin: int32 [num_masks, n]
    block: int = 0                        # bsg: block size (0 = no block part)
    stride: int = 0                       # bsg: stride (0 = no strided part)
    n_global: int = 0                     # bsg: number of global tokens
    cand_row_ptr: Optional[np.ndarray] = None  # coo: int64 [num_masks*n + 1]
    cand_cols: Optional[np.ndarray] = None     # coo: int32 candidate columns
    add_diagonal: bool = False                 # coo: also include (i, i)


@dataclass
class Workload:
    name: str
    B: int
    H: int
    n: int
    d: int
    dtype: str
    scale: float
    q: Tensor
    k: Tensor
    v: Tensor
    mask: MaskParams
    add_mask: Optional[Tensor] = None   # 4-D, broadcastable to [B, H, n, n]
    bias: Optional[Tensor] = None       # 4-D, broadcastable to [B, H, n, n]
    notes: dict = field(default_factory=dict)


# Full sizes of the five workloads, and one extra (index 5): an all-ones mask at
# d = 128, B*H = 64, n = 4096, the case where the dense-tile path's tensor-core
# efficiency can show (the Evoformer workload's d = 32 cannot).
CONFIGS = {
    0: dict(name="tiny-sliding", B=1, H=2, n=128, d=32, dtype=F32, std=1.0),
    1: dict(name="variable-window", B=4, H=12, n=4096, d=64, dtype=BF16, std=1.0),
    2: dict(name="random-csr", B=2, H=16, n=8192, d=64, dtype=BF16, std=1.0),
    3: dict(name="block-strided-global", B=1, H=16, n=16384, d=128, dtype=BF16, std=0.5),
    4: dict(name="evoformer-dense-mask-bias", B=256, H=8, n=256, d=32, dtype=BF16, std=1.0),
    # extra to the five: an all-ones mask at d = 128, where dense tiles dominate
    5: dict(name="dense-d128", B=4, H=16, n=4096, d=128, dtype=BF16, std=1.0),
}


def _normal(rng, shape, std):
    return rng.standard_normal(size=shape, dtype=np.float64) * std


def _random_candidates(rng, n: int, mean_extra: float):
    """Per row i: k_i = min(Poisson(mean_extra), n-1) distinct columns drawn
    uniformly from [0, n) without i. Returns (row_ptr int64 [n+1], cols int32)."""
    counts = np.minimum(rng.poisson(mean_extra, size=n), n - 1).astype(np.int64)
    rows = []
    for i in range(n):
        k = int(counts[i])
        got = np.empty(0, dtype=np.int64)
        while got.size < k:
            c = rng.integers(0, n - 1, size=2 * k + 8)
            c = np.concatenate([got, c])
            _, first = np.unique(c, return_index=True)
            got = c[np.sort(first)][:k]
        got = got.copy()
        got[got >= i] += 1          # skip the diagonal
        rows.append(got.astype(np.int32))
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    cols = np.concatenate(rows) if rows else np.empty(0, dtype=np.int32)
    return row_ptr, cols.astype(np.int32)


def make(cfg: int, *, B: Optional[int] = None, H: Optional[int] = None,
         n: Optional[int] = None, seed: Optional[int] = None,
         dtype: Optional[str] = None, d: Optional[int] = None) -> Workload:
    """Workload ``cfg`` (0..4, and 5: the extra dense d = 128 case) at full size, or with B/H/n/d/dtype overridden
    (same recipe, smaller shapes, for parity tests the oracle finishes in seconds)."""
    c = dict(CONFIGS[cfg])
    B = c["B"] if B is None else B
    H = c["H"] if H is None else H
    n = c["n"] if n is None else n
    d = c["d"] if d is None else d
    dtype = c["dtype"] if dtype is None else dtype
    base = 1000 + cfg if seed is None else seed
    rng = np.random.default_rng(base)
    std = c["std"]
    q = make_tensor(_normal(rng, (B, H, n, d), std), dtype)
    k = make_tensor(_normal(rng, (B, H, n, d), std), dtype)
    v = make_tensor(_normal(rng, (B, H, n, d), std), dtype)
    scale = 1.0 / np.sqrt(d)
    add_mask = bias = None
    notes = {}
    if cfg == 0:
        mask = MaskParams("sliding", n, 1, window=min(16, n - 1))
    elif cfg == 1:
        hw = np.stack([np.random.default_rng([base, b]).integers(32, 257, size=n)
                       for b in range(B)]).astype(np.int32)
        mask = MaskParams("varwin", n, B, half_widths=hw)
    elif cfg == 2:
        rps, cols, off = [0], [], 0
        for b in range(B):
            rp, cc = _random_candidates(np.random.default_rng([base, b]), n, 80.0)
            rps.append(rp[1:] + off)
            cols.append(cc)
            off += int(rp[-1])
        row_ptr = np.concatenate([np.zeros(1, np.int64)] + [np.asarray(x, np.int64) for x in rps[1:]])
        mask = MaskParams("coo", n, B, cand_row_ptr=row_ptr,
                          cand_cols=np.concatenate(cols).astype(np.int32), add_diagonal=True)
    elif cfg == 3:
        mask = MaskParams("bsg", n, 1, block=min(64, n), stride=min(128, n),
                          n_global=min(32, n))
    elif cfg == 4:
        mask = MaskParams("dense", n, 1)
        mrng = np.random.default_rng([base, 0])
        lo = min(128, n)
        lengths = mrng.integers(lo, n + 1, size=B)
        m = np.zeros((B, 1, 1, n), dtype=np.float64)
        for b in range(B):
            m[b, 0, 0, lengths[b]:] = -np.inf
        add_mask = make_tensor(m, BF16)
        bias = make_tensor(_normal(mrng, (1, H, n, n), 1.0), BF16)
        notes["key_lengths"] = lengths
    elif cfg == 5:
        mask = MaskParams("dense", n, 1)
    else:
        raise ValueError(cfg)
    return Workload(c["name"], B, H, n, d, dtype, float(scale), q, k, v, mask,
                    add_mask, bias, notes)

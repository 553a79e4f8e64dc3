"""Seeded generators for one binary-weight layer and its activations.

Every tensor gets its own PCG64 stream keyed by ``(seed, *key, tensor_id)`` so
that any tensor of any workload can be regenerated alone. Values are drawn in
fp64, cast to fp32 (round to nearest even) and, for bf16 tensors, rounded once
more to bf16 (round to nearest even); both consumers see the rounded values.

Distributions (the binary-weight GEMV workloads):
  signs        iid Bernoulli(0.5), drawn directly as random packed words
  row/col      |N(0, 0.02)|
  alpha        |N(0, 0.01)|
  activations  N(0, 1); optional outlier channels scaled by a factor before rounding
  salient      ceil(frac * in) input columns with the largest
               max_m |X[m, j]| * ||c[:, j]||_2 (ties -> lower j), stored ascending;
               their column scales are set to 0 (the column lives in int8 only),
               q ~ round(N(0, 42)) clipped to [-127, 127],
               s_j = ||c[:, j]||_2 * 0.02 / 42 so that s*q keeps the column's size.
"""

from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import numpy as np

from .layout import packed_words, zero_padding_bits

# tensor ids inside one layer's key space
T_BITS, T_ROW, T_COL, T_V, T_UT, T_ALPHA, T_SALQ, T_X, T_OUTLIER, T_REF = range(10)


def _rng(seed: int, key: Sequence[int], tensor: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key, tensor])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    # used only to recover the stored column-scale magnitudes for salient selection
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _as_dtype(v64: np.ndarray, dtype: str) -> np.ndarray:
    v32 = v64.astype(np.float32)
    if dtype == "f32":
        return v32
    if dtype == "bf16":
        return f32_to_bf16_bits(v32)
    raise ValueError(dtype)


def random_sign_words(rng: np.random.Generator, lead: int, rows: int, cols: int) -> np.ndarray:
    """``lead`` packed sign matrices of iid fair signs, padding cleared."""
    n = packed_words(rows, cols)
    w = rng.integers(0, 1 << 32, size=(lead, n), dtype=np.uint32)
    return zero_padding_bits(w, rows, cols)


def dense_signs(rng_or_seed, rows: int, cols: int) -> np.ndarray:
    """Dense int8 matrix of iid fair +1/-1 entries (for packing tests)."""
    rng = rng_or_seed if isinstance(rng_or_seed, np.random.Generator) else np.random.default_rng(rng_or_seed)
    return (rng.integers(0, 2, size=(rows, cols), dtype=np.int8) * 2 - 1).astype(np.int8)


@dataclass
class Layer:
    """Host arrays of one layer in the packed format the library consumes."""
    out: int
    in_: int
    K: int
    scale_dtype: str                  # "f32" or "bf16"
    bits: np.ndarray                  # uint32 [K, packed_words(out, in)]
    row_scale: np.ndarray             # [K, out] (or [K, out, ceil(in/group)]) float32 or uint16 (bf16 bits)
    col_scale: np.ndarray             # [K, in]
    rank: int = 0
    v_bits: Optional[np.ndarray] = None    # uint32 [packed_words(rank, in)]
    ut_bits: Optional[np.ndarray] = None   # uint32 [packed_words(out, rank)]
    alpha: Optional[np.ndarray] = None     # float32 [rank]
    n_sal: int = 0
    sal_idx: Optional[np.ndarray] = None   # int32 [n_sal], strictly ascending
    sal_q: Optional[np.ndarray] = None     # int8 [out, sal_stride]
    sal_scale: Optional[np.ndarray] = None  # float32 [n_sal]
    name: str = ""
    extra: dict = field(default_factory=dict)
    # 0: one row scale per (base, row); g > 0: one per (base, row, group of g input
    # columns), row_scale [K, out, ceil(in/g)] ("FluxBin" Sec. 3.1 grouped row scales)
    group: int = 0
    # binary salient refinement ("FluxBin" Sec. 4, Kb-sS-gG): ref_K bases over the s salient
    # columns of every group of `group` columns, stored as a dense sign matrix over the
    # gathered columns (ref_idx ascending), with one row scale per (base, row, group) and
    # one column scale per (base, salient column); additive on top of the global bases
    ref_K: int = 0
    ref_idx: Optional[np.ndarray] = None        # int32 [n_ref]
    ref_bits: Optional[np.ndarray] = None       # uint32 [ref_K, packed_words(out, n_ref)]
    ref_row_scale: Optional[np.ndarray] = None  # [ref_K, out, ceil(in/group)] in scale_dtype
    ref_col_scale: Optional[np.ndarray] = None  # [ref_K, n_ref] in scale_dtype

    @property
    def sal_stride(self) -> int:
        return 0 if self.sal_q is None else int(self.sal_q.shape[1])


def sal_stride_for(n_sal: int) -> int:
    return (n_sal + 15) // 16 * 16


def make_activations(seed: int, key: Sequence[int], M: int, n: int, dtype: str,
                     outlier_frac: float = 0.0, outlier_factor: float = 1.0) -> np.ndarray:
    """X [M, n] ~ N(0,1); ceil(outlier_frac*n) channels (same for all rows) scaled."""
    x = _rng(seed, key, T_X).standard_normal((M, n))
    if outlier_frac > 0:
        n_out = int(np.ceil(outlier_frac * n))
        cols = _rng(seed, key, T_OUTLIER).choice(n, size=n_out, replace=False)
        x[:, cols] *= outlier_factor
    return _as_dtype(x, dtype)


def make_layer(seed: int, key: Sequence[int], out: int, in_: int, K: int, scale_dtype: str,
               rank: int = 0, sal_frac: float = 0.0, x_for_salience: Optional[np.ndarray] = None,
               x_dtype: str = "bf16", name: str = "", group: int = 0,
               refine: Optional[Tuple[int, int]] = None) -> Layer:
    bits = random_sign_words(_rng(seed, key, T_BITS), K, out, in_)
    rshape = (K, out, -(-in_ // group)) if group else (K, out)
    row = _as_dtype(np.abs(_rng(seed, key, T_ROW).standard_normal(rshape)) * 0.02, scale_dtype)
    col = _as_dtype(np.abs(_rng(seed, key, T_COL).standard_normal((K, in_))) * 0.02, scale_dtype)
    L = Layer(out=out, in_=in_, K=K, scale_dtype=scale_dtype, bits=bits, row_scale=row,
              col_scale=col, name=name, group=group)
    if rank > 0:
        L.rank = rank
        L.v_bits = random_sign_words(_rng(seed, key, T_V), 1, rank, in_)[0]
        L.ut_bits = random_sign_words(_rng(seed, key, T_UT), 1, out, rank)[0]
        L.alpha = (np.abs(_rng(seed, key, T_ALPHA).standard_normal(rank)) * 0.01).astype(np.float32)
    if sal_frac > 0:
        n_sal = int(np.ceil(sal_frac * in_))
        if x_for_salience is None:
            raise ValueError("salient selection needs the activations")
        xa = x_for_salience
        xf = _bf16_bits_to_f32(xa) if x_dtype == "bf16" else xa.astype(np.float32)
        cf = _bf16_bits_to_f32(col) if scale_dtype == "bf16" else col
        cnorm = np.sqrt(np.sum(cf.astype(np.float64) ** 2, axis=0))
        score = np.max(np.abs(xf.astype(np.float64)), axis=0) * cnorm
        order = np.lexsort((np.arange(in_), -score))   # descending score, ties -> lower j
        idx = np.sort(order[:n_sal]).astype(np.int32)
        q = np.clip(np.rint(_rng(seed, key, T_SALQ).standard_normal((out, n_sal)) * 42.0), -127, 127)
        qs = np.zeros((out, sal_stride_for(n_sal)), dtype=np.int8)
        qs[:, :n_sal] = q.astype(np.int8)
        L.n_sal = n_sal
        L.sal_idx = idx
        L.sal_q = qs
        L.sal_scale = (cnorm[idx] * 0.02 / 42.0).astype(np.float32)
        L.col_scale = col.copy()
        L.col_scale[:, idx] = 0
    if refine:
        Ks, sp = refine
        if not group:
            raise ValueError("the salient refinement needs grouped row scales (group > 0)")
        ng = -(-in_ // group)
        rng = _rng(seed, key, T_REF)
        cols = []
        for j in range(ng):  # s salient columns per group, seeded (the pages choose them by a
            lo, hi = j * group, min(in_, (j + 1) * group)  # Hessian score: data not available)
            take = min(sp, hi - lo)
            cols.extend(sorted(rng.choice(np.arange(lo, hi), size=take, replace=False).tolist()))
        ref_idx = np.array(cols, dtype=np.int32)
        L.ref_K = Ks
        L.ref_idx = ref_idx
        L.ref_bits = random_sign_words(rng, Ks, out, len(ref_idx))
        L.ref_row_scale = _as_dtype(np.abs(rng.standard_normal((Ks, out, ng))) * 0.01, scale_dtype)
        L.ref_col_scale = _as_dtype(np.abs(rng.standard_normal((Ks, len(ref_idx)))) * 0.02, scale_dtype)
    return L

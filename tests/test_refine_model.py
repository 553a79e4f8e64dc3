"""The salient refinement launch's index arithmetic, run as a model on the CPU.

refine_kernel stages, per 32-row tile, the tile's packed refinement signs, row scales,
column scales and the gathered column indices in shared memory, finds each column group's
first gathered column by one pass over the indices (a column whose group differs from its
predecessor's starts the groups in between; entries start at n_ref), gathers the
activations through the indices, and lets warp w walk groups w, w + W, ... one sign word at
a time. This model repeats those index computations with numpy and checks two things:

  * every shared-memory and global index stays inside its array for ANY index list
    (ascending, out of order, negative, beyond the input, repeated), which is the property
    the kernel relies on to take bad indices without an out-of-bounds access;
  * for valid ascending lists the walk gives the oracle's refinement term ("FluxBin",
    Sec. 4: sum_k r_k[o][idx_t // g] c_k[t] (2b - 1) x[idx_t]).
"""

import numpy as np
import pytest

import oracle
from synth import make_activations, make_layer

WARPS = (16, 32)  # warps per CTA: batch blocks of up to 4 rows, and of 8 rows


def group_starts(idx, g, ng):
    """The kernel's group boundaries: gs[j] for j <= ng, every entry in [0, n]."""
    n = len(idx)
    gs = np.full(ng + 1, n, dtype=np.int64)
    jt = np.minimum(np.maximum(idx, 0) // g, ng - 1)
    jp = np.concatenate([[-1], jt[:-1]]) if n else jt
    for t in range(n):  # the kernel's threads write these in any order; for ascending idx
        for j in range(jp[t] + 1, jt[t] + 1):  # every entry has one writer
            gs[j] = t
    return gs


def walk(idx, g, ng, Ks, qr, out, tile, warps, MB, in_):
    """Every index the kernel forms for one CTA, as (array, index) pairs."""
    n = len(idx)
    gs = group_starts(idx, g, ng)
    acc = {"sbits": [], "srs": [], "cs": [], "xg": [], "gs": [], "rrs": [], "bits": [], "X": []}
    words = ((out + 31) // 32) * qr * 128
    # staging (before the wait)
    for i in range(Ks * qr * 32):
        k, w = divmod(i, qr * 32)
        acc["bits"].append(k * words + tile * qr * 128 + 4 * w + 3)  # last word of the uint4
        acc["sbits"].append(4 * i + 3)
    for i in range(Ks * ng * 32):
        o = tile * 32 + (i & 31)
        if o < out:
            acc["rrs"].append((i >> 5) * out + o)
        acc["srs"].append(i)
    # gather (after the wait): an index outside [0, in) is not read
    for m in range(MB):
        for t in range(n):
            if 0 <= idx[t] < in_:
                acc["X"].append(m * in_ + idx[t])
            acc["xg"].append(m * n + t)
    # the walk
    for w in range(warps):
        for j in range(w, ng, warps):
            acc["gs"] += [j, j + 1]
            t0, t1 = gs[j], gs[j + 1]
            ta = t0
            while ta < t1:
                tb = min(t1, (ta | 31) + 1)
                for k in range(Ks):
                    for lane in (0, 31):
                        acc["sbits"].append(k * qr * 128 + ((ta >> 7) * 32 + lane) * 4 + ((ta >> 5) & 3))
                for t in range(ta, tb):
                    for k in range(Ks):
                        acc["cs"].append(k * n + t)
                    for m in range(MB):
                        acc["xg"].append(m * n + t)
                ta = tb
            for k in range(Ks):
                for lane in (0, 31):
                    acc["srs"].append((k * ng + j) * 32 + lane)
    return acc, words


@pytest.mark.parametrize("case", range(40))
def test_every_index_stays_in_bounds_for_any_index_list(case):
    rng = np.random.default_rng(900 + case)
    in_ = int(rng.integers(1, 1500))
    g = int(rng.choice([128, 256, 384]))
    ng = -(-in_ // g)
    n = int(rng.integers(1, min(in_, 300) + 1))
    kind = case % 4
    if kind == 0:    # valid, ascending
        idx = np.sort(rng.choice(in_, size=n, replace=False))
    elif kind == 1:  # out of order
        idx = rng.choice(in_, size=n, replace=False)
    elif kind == 2:  # negative and beyond the input
        idx = np.sort(rng.integers(-3 * g, in_ + 3 * g, size=n))
    else:            # repeated and unsorted, with extremes
        idx = rng.integers(-(2 ** 31), 2 ** 31 - 1, size=n)
        idx[: n // 2] = idx[0]
    idx = idx.astype(np.int64)
    Ks, MB = int(rng.integers(1, 5)), int(rng.choice([1, 2, 4, 8]))
    warps = WARPS[MB >= 8]
    out = int(rng.integers(1, 100))
    qr = (n + 127) // 128
    for tile in range((out + 31) // 32):
        acc, words = walk(idx, g, ng, Ks, qr, out, tile, warps, MB, in_)
        sizes = {"sbits": Ks * qr * 128, "srs": Ks * ng * 32, "cs": Ks * n, "xg": MB * n, "gs": ng + 1,
                 "rrs": Ks * ng * out, "bits": Ks * words, "X": MB * in_}
        for name, ix in acc.items():
            if ix:
                a = np.asarray(ix)
                assert a.min() >= 0 and a.max() < sizes[name], (name, a.min(), a.max(), sizes[name])


@pytest.mark.parametrize("out,in_,g,Ks,s,M", [(70, 1000, 128, 2, 8, 1), (40, 700, 256, 3, 16, 5),
                                               (33, 300, 128, 1, 128, 2), (64, 1100, 384, 4, 3, 8)])
def test_walk_reproduces_the_oracle_term(out, in_, g, Ks, s, M):
    # the kernel's sums, in its order (per group: fp sum over the group's columns for each
    # base, times that group's row scale), in fp64, against the oracle's refinement term
    import copy
    L = make_layer(0, (860, out, in_), out, in_, 1, "f32", group=g, refine=(Ks, s))
    X = make_activations(0, (860, M), M, in_, "f32")
    x = oracle.decode_values(X, "f32").reshape(M, in_)
    idx = np.asarray(L.ref_idx, dtype=np.int64)
    n, ng = len(idx), -(-in_ // g)
    gs = group_starts(idx, g, ng)
    R = oracle.decode_values(L.ref_row_scale, "f32").reshape(Ks, out, ng)
    C = oracle.decode_values(L.ref_col_scale, "f32").reshape(Ks, n)
    S = np.stack([oracle.unpack_bit_matrix(np.asarray(L.ref_bits)[k], out, n) for k in range(Ks)])
    term = np.zeros((M, out))
    for j in range(ng):
        t0, t1 = gs[j], gs[j + 1]
        for k in range(Ks):
            part = (S[k][:, t0:t1] * C[k][t0:t1][None, :]) @ x[:, idx[t0:t1]].T  # [out, M]
            term += (R[k][:, j][:, None] * part).T
    L0 = copy.copy(L)
    L0.ref_K = 0
    want = oracle.gemv(L, X, "f32") - oracle.gemv(L0, X, "f32")
    assert np.allclose(term, want, rtol=1e-9, atol=1e-12)

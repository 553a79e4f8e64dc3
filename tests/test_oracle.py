"""Pins for the fp64 oracle, independent of the oracle's own formulas.

Each test checks the oracle against something the pages or mathematics fix:
printed worked examples (tests/golden/), closed forms, invariants, an
independent bit packer written here element by element, and brute-force
enumeration on tiny shapes.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from synth import Layer, f32_to_bf16_bits
from synth.gen import sal_stride_for

from conftest import GOLDEN


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --- an independent packer: the layout written out per element --------------

def py_pack(signs):
    """Element (i, c) -> bit (c % 32) of word ((t*Q + q)*32 + r)*4 + j with
    t, r = divmod(i, 32); q, cc = divmod(c, 128); j = cc // 32."""
    rows, cols = len(signs), len(signs[0])
    T, Q = -(-rows // 32), -(-cols // 128)
    words = [0] * (T * Q * 128)
    for i in range(rows):
        t, r = divmod(i, 32)
        for c in range(cols):
            if signs[i][c] == 1:
                q, cc = divmod(c, 128)
                j, b = divmod(cc, 32)
                words[((t * Q + q) * 32 + r) * 4 + j] |= 1 << b
    return np.array(words, dtype=np.uint32)


def py_bit(words, rows, cols, i, c):
    Q = -(-cols // 128)
    t, r = divmod(i, 32)
    q, cc = divmod(c, 128)
    j, b = divmod(cc, 32)
    return (int(words[((t * Q + q) * 32 + r) * 4 + j]) >> b) & 1


def f32(a):
    return np.asarray(a, dtype=np.float32)


def mk(out, in_, K=0, signs=None, row=None, col=None, rank=0, u=None, v=None, alpha=None,
       sal_idx=None, sal_q=None, sal_scale=None, group=0):
    """Layer with fp32 scales built through the independent packer (row: [K, out], or
    [K, out, groups] with grouped row scales)."""
    bits = np.stack([py_pack(signs[k]) for k in range(K)]) if K else np.zeros((0, 0), np.uint32)
    L = Layer(out=out, in_=in_, K=K, scale_dtype="f32", bits=bits,
              row_scale=f32(row if K else np.zeros((0, out))),
              col_scale=f32(col if K else np.zeros((0, in_))), group=group)
    if rank:
        L.rank = rank
        L.v_bits = py_pack(v)                               # [rank][in]
        L.ut_bits = py_pack(u)                              # u given as [out][rank]
        L.alpha = f32(alpha)
    if sal_idx is not None:
        n = len(sal_idx)
        q = np.zeros((out, sal_stride_for(n)), np.int8)
        q[:, :n] = np.asarray(sal_q, np.int8)
        L.n_sal, L.sal_idx, L.sal_q, L.sal_scale = n, np.asarray(sal_idx, np.int32), q, f32(sal_scale)
    return L


# --- bf16 decoding by the format's definition ---------------------------------

def test_bf16_decode_by_definition():
    g = golden("bf16_values.json")
    for case in g["cases"]:
        bits = int(case["bits"], 16)
        s, e, f = bits >> 15, (bits >> 7) & 0xFF, bits & 0x7F
        if e == 0:
            by_def = (-1) ** s * 2.0 ** -126 * (f / 128.0)
        else:
            by_def = (-1) ** s * 2.0 ** (e - 127) * (1 + f / 128.0)
        got = oracle.decode_values(np.array([bits], np.uint16), "bf16")[0]
        assert got == by_def == case["value"]


def test_bf16_generator_rounds_to_nearest_even():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties go to the even one (1.0)
    vals = f32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20])
    got = oracle.decode_values(f32_to_bf16_bits(vals), "bf16")
    assert list(got) == [1.0, 1.0 + 2 * 2 ** -7, 1.0 + 2 ** -7]


# --- the pages' worked examples ---------------------------------------------

def test_worked_example_correction_only():
    g = golden("worked_example_vx.json")
    x, v = g["x"], g["v"]
    L = mk(1, 4, rank=1, u=[[1]], v=[v], alpha=[1.0])
    X = f32([x])
    y = oracle.gemv(L, X, "f32")
    assert y.shape == (1, 1)
    # fp32 inputs are widened exactly, so the fp64 sum equals the exact decimal up to fp32 input rounding
    assert y[0, 0] == pytest.approx(g["v_dot_x"], abs=1e-6)
    z = oracle.correction_z(mk(1, 4, rank=1, u=[[1]], v=[v], alpha=[0.5]), X, "f32")
    assert z[0, 0] == pytest.approx(0.5 * g["v_dot_x"], abs=1e-6)
    # u = -1 subtracts the same number at that output position
    yneg = oracle.gemv(mk(1, 4, rank=1, u=[[-1]], v=[v], alpha=[1.0]), X, "f32")
    assert yneg[0, 0] == pytest.approx(-g["v_dot_x"], abs=1e-6)


def test_worked_example_as_one_base():
    g = golden("worked_example_vx.json")
    L = mk(1, 4, K=1, signs=[[g["v"]]], row=[[1.0]], col=[[1.0] * 4])
    y = oracle.gemv(L, f32([g["x"]]), "f32")
    assert y[0, 0] == pytest.approx(g["v_dot_x"], abs=1e-6)


def test_toy_decomposition_refit_reconstructs_exactly():
    g = golden("toy_decomposition.json")
    comps = g["components"]
    u = [[c["u"][o] for c in comps] for o in range(3)]      # [out][rank]
    v = [c["v"] for c in comps]                              # [rank][in]
    L = mk(3, 2, rank=2, u=u, v=v, alpha=g["refit_alpha"])
    W = oracle.reconstruct(L)
    assert np.array_equal(W, np.array(g["W"], dtype=np.float64))
    y = oracle.gemv(L, f32([[1.0, 2.0]]), "f32")
    assert np.array_equal(y[0], [3.0, 3.0, 12.0])


def test_toy_greedy_coefficients_leave_the_printed_residual():
    g = golden("toy_decomposition.json")
    comps = g["components"]
    u = [[c["u"][o] for c in comps] for o in range(3)]
    v = [c["v"] for c in comps]
    Wt = np.array(g["W"], dtype=np.float64)
    L1 = mk(3, 2, rank=1, u=[[r[0]] for r in u], v=[v[0]], alpha=[g["greedy_alpha"][0]])
    assert np.array_equal(Wt - oracle.reconstruct(L1), np.array(g["greedy_residual_after_1"], float))
    L2 = mk(3, 2, rank=2, u=u, v=v, alpha=g["greedy_alpha"])
    sse = float(np.sum((Wt - oracle.reconstruct(L2)) ** 2))
    assert sse == pytest.approx(g["greedy_residual_sse"], rel=1e-12)


def test_biloco_decomposition_reproduces_the_page_toy():
    # the page's 3x2 walk-through: both greedy components start from v = (+, +)
    g = golden("toy_decomposition.json")
    W = np.array(g["W"], dtype=np.float64)
    U, V, greedy, refit = oracle.biloco_decompose(W, [[1, 1], [1, 1]])
    for j, c in enumerate(g["components"]):
        assert np.array_equal(U[:, j], c["u"]) and np.array_equal(V[j], c["v"])
    assert greedy[0] == g["greedy_alpha_rational"][0][0] / g["greedy_alpha_rational"][0][1]
    assert greedy[1] == pytest.approx(g["greedy_alpha_rational"][1][0] / g["greedy_alpha_rational"][1][1], rel=1e-15)
    assert np.array_equal(W - greedy[0] * np.outer(U[:, 0], V[0]), np.array(g["greedy_residual_after_1"], float))
    sse = float(np.sum((W - (U * greedy) @ V) ** 2))
    assert sse == pytest.approx(g["greedy_residual_sse"], rel=1e-12)
    assert np.allclose(refit, g["refit_alpha"], rtol=0, atol=1e-12)
    # the refit components, run through the correction path of the oracle, rebuild W exactly
    L = mk(3, 2, rank=2, u=U.astype(int).tolist(), v=V.astype(int).tolist(), alpha=refit)
    assert np.allclose(oracle.reconstruct(L), W, rtol=0, atol=1e-6)


def test_biloco_recovers_an_exact_sign_rank_one_matrix():
    rng = np.random.default_rng(21)
    u, v = rng.choice([-1.0, 1.0], size=9), rng.choice([-1.0, 1.0], size=13)
    W = 3.0 * np.outer(u, v)
    U, V, greedy, refit = oracle.biloco_decompose(W, rng.choice([-1, 1], size=(1, 13)))
    assert abs(greedy[0]) == 3.0 and abs(refit[0]) == pytest.approx(3.0, rel=1e-15)
    assert np.array_equal(greedy[0] * np.outer(U[:, 0], V[0]), W)


def test_biloco_refit_is_the_least_squares_optimum():
    rng = np.random.default_rng(22)
    W = rng.standard_normal((6, 11))
    U, V, greedy, refit = oracle.biloco_decompose(W, rng.choice([-1, 1], size=(3, 11)))
    err = lambda a: float(np.sum((W - (U * a) @ V) ** 2))  # noqa: E731
    assert err(refit) <= err(greedy) + 1e-12
    # first-order optimality: the residual is orthogonal to every component, and moving
    # any coefficient either way raises the error
    res = W - (U * refit) @ V
    for j in range(3):
        assert abs(float(U[:, j] @ res @ V[j])) < 1e-10
        for d in (-1e-3, 1e-3):
            a = refit.copy()
            a[j] += d
            assert err(a) > err(refit)


# --- closed forms and invariants ---------------------------------------------

def _rand_layer(rng, out, in_, K, rank=0, n_sal=0):
    signs = [rng.choice([-1, 1], size=(out, in_)).tolist() for _ in range(K)]
    row = np.abs(rng.standard_normal((K, out))) * 0.02
    col = np.abs(rng.standard_normal((K, in_))) * 0.02
    kw = {}
    if rank:
        kw = dict(rank=rank, u=rng.choice([-1, 1], size=(out, rank)).tolist(),
                  v=rng.choice([-1, 1], size=(rank, in_)).tolist(),
                  alpha=np.abs(rng.standard_normal(rank)) * 0.01)
    if n_sal:
        kw.update(sal_idx=np.sort(rng.choice(in_, n_sal, replace=False)),
                  sal_q=rng.integers(-127, 128, size=(out, n_sal)),
                  sal_scale=np.abs(rng.standard_normal(n_sal)) * 1e-4)
    return mk(out, in_, K=K, signs=signs, row=row, col=col, **kw)


def test_all_plus_one_is_scaled_row_sum():
    rng = np.random.default_rng(1)
    out, in_, K = 37, 300, 2
    row = np.abs(rng.standard_normal((K, out))) * 0.02
    col = np.abs(rng.standard_normal((K, in_))) * 0.02
    L = mk(out, in_, K=K, signs=[[[1] * in_] * out] * K, row=row, col=col)
    X = f32(rng.standard_normal((3, in_)))
    y = oracle.gemv(L, X, "f32")
    r64, c64, x64 = f32(row).astype(float), f32(col).astype(float), X.astype(float)
    expect = sum(np.outer(x64 @ c64[k], r64[k]) for k in range(K))
    assert np.allclose(y, expect, rtol=1e-12, atol=1e-15)


def test_flipping_a_sign_row_negates_its_contribution():
    rng = np.random.default_rng(2)
    out, in_ = 5, 70
    signs = rng.choice([-1, 1], size=(out, in_))
    row = np.abs(rng.standard_normal((1, out))) + 0.1
    col = np.abs(rng.standard_normal((1, in_))) + 0.1
    X = f32(rng.standard_normal((1, in_)))
    y0 = oracle.gemv(mk(out, in_, 1, [signs.tolist()], row, col), X, "f32")
    flipped = signs.copy()
    flipped[3] *= -1
    y1 = oracle.gemv(mk(out, in_, 1, [flipped.tolist()], row, col), X, "f32")
    assert y1[0, 3] == pytest.approx(-y0[0, 3], rel=1e-12)
    keep = [0, 1, 2, 4]
    assert np.array_equal(y1[0, keep], y0[0, keep])


def test_linearity_in_x_and_batch_rows_independent():
    rng = np.random.default_rng(3)
    L = _rand_layer(rng, 40, 150, 2, rank=3, n_sal=4)
    X1, X2 = f32(rng.standard_normal((1, 150))), f32(rng.standard_normal((1, 150)))
    y1, y2 = oracle.gemv(L, X1, "f32"), oracle.gemv(L, X2, "f32")
    X12 = np.concatenate([X1, X2])
    y12 = oracle.gemv(L, X12, "f32")
    assert np.allclose(y12, np.concatenate([y1, y2]), rtol=1e-13, atol=1e-16)
    comb = oracle.gemv(L, X1.astype(np.float64) * 0.5 + X2.astype(np.float64) * 0.25, "f32")
    # 0.5*x1 + 0.25*x2 is not exactly representable in fp32 in general: compare in fp64 terms
    Xc = f32(X1.astype(np.float64) * 0.5 + X2.astype(np.float64) * 0.25)
    assert np.allclose(oracle.gemv(L, Xc, "f32"), comb, rtol=1e-12)
    assert np.allclose(0.5 * y1 + 0.25 * y2, oracle.gemv(L, X1 * np.float32(0.5), "f32")
                       + oracle.gemv(L, X2 * np.float32(0.25), "f32"), rtol=1e-12)


def test_salient_single_columns_closed_form():
    rng = np.random.default_rng(4)
    out, in_ = 6, 20
    idx, q, s = [3, 17], rng.integers(-127, 128, size=(out, 2)), [0.5, 0.25]
    L = mk(out, in_, sal_idx=idx, sal_q=q, sal_scale=s)
    X = f32(rng.standard_normal((2, in_)))
    y = oracle.gemv(L, X, "f32")
    x64 = X.astype(float)
    expect = x64[:, [3]] * (0.5 * q[:, 0])[None, :] + x64[:, [17]] * (0.25 * q[:, 1])[None, :]
    assert np.allclose(y, expect, rtol=1e-15, atol=0)


def test_terms_add():
    """Binary bases, correction and salient columns add: each is checked alone above."""
    rng = np.random.default_rng(5)
    L = _rand_layer(rng, 33, 130, 2, rank=4, n_sal=3)
    X = f32(rng.standard_normal((2, 130)))
    full = oracle.gemv(L, X, "f32")
    Lb = mk(33, 130, K=2, signs=[oracle.unpack_bit_matrix(L.bits[k], 33, 130).tolist() for k in range(2)],
            row=L.row_scale, col=L.col_scale)
    Lc = Layer(out=33, in_=130, K=0, scale_dtype="f32", bits=np.zeros((0, 0), np.uint32),
               row_scale=f32(np.zeros((0, 33))), col_scale=f32(np.zeros((0, 130))),
               rank=4, v_bits=L.v_bits, ut_bits=L.ut_bits, alpha=L.alpha)
    Ls = Layer(out=33, in_=130, K=0, scale_dtype="f32", bits=np.zeros((0, 0), np.uint32),
               row_scale=f32(np.zeros((0, 33))), col_scale=f32(np.zeros((0, 130))),
               n_sal=3, sal_idx=L.sal_idx, sal_q=L.sal_q, sal_scale=L.sal_scale)
    parts = oracle.gemv(Lb, X, "f32") + oracle.gemv(Lc, X, "f32") + oracle.gemv(Ls, X, "f32")
    assert np.allclose(full, parts, rtol=1e-12, atol=1e-18)


# --- grouped row scales (one row scale per group of g input columns) ------------

def test_grouped_all_plus_one_is_a_sum_of_group_sums():
    # all signs +1: y[m][o] = sum_k sum_G r_k[o][G] * sum_{i in group G} c_k[i] x[m][i]
    rng = np.random.default_rng(11)
    out, in_, K, g = 9, 300, 2, 128          # groups of 128, 128 and a ragged 44
    ng = -(-in_ // g)
    row = np.abs(rng.standard_normal((K, out, ng))) * 0.02 + 0.001
    col = np.abs(rng.standard_normal((K, in_))) * 0.02
    L = mk(out, in_, K=K, signs=[[[1] * in_] * out] * K, row=row, col=col, group=g)
    X = f32(rng.standard_normal((2, in_)))
    y = oracle.gemv(L, X, "f32")
    r64, c64, x64 = f32(row).astype(float), f32(col).astype(float), X.astype(float)
    expect = np.zeros((2, out))
    for k in range(K):
        for G in range(ng):
            cols = slice(G * g, min(in_, (G + 1) * g))
            expect += np.outer(x64[:, cols] @ c64[k, cols], r64[k, :, G])
    assert np.allclose(y, expect, rtol=1e-12, atol=1e-15)


def test_grouped_scales_equal_across_groups_match_one_scale_per_row():
    rng = np.random.default_rng(12)
    out, in_, K, g = 7, 200, 2, 64
    signs = rng.choice([-1, 1], size=(K, out, in_)).tolist()
    row = np.abs(rng.standard_normal((K, out))) + 0.1
    col = np.abs(rng.standard_normal((K, in_))) + 0.1
    X = f32(rng.standard_normal((3, in_)))
    flat = oracle.gemv(mk(out, in_, K, signs, row, col), X, "f32")
    grouped = oracle.gemv(mk(out, in_, K, signs, np.repeat(row[:, :, None], 4, axis=2), col, group=g), X, "f32")
    assert np.allclose(grouped, flat, rtol=1e-13, atol=1e-16)


@pytest.mark.parametrize("out,in_,K,g", [(1, 4, 1, 2), (2, 4, 1, 2), (1, 4, 2, 2), (2, 3, 1, 2), (1, 5, 1, 3)])
def test_grouped_brute_force_all_sign_patterns(out, in_, K, g):
    """Every sign pattern with a different row scale per group: the product equals the
    sign-add identity applied group by group, bits read with plain integer shifts."""
    rng = np.random.default_rng(out * 1000 + in_ * 100 + K * 10 + g)
    ng = -(-in_ // g)
    row = f32(rng.uniform(0.5, 2.0, size=(K, out, ng)))
    col = f32(rng.uniform(0.5, 2.0, size=(K, in_)))
    x = f32(rng.standard_normal((1, in_)))
    for pattern in itertools.product([-1, 1], repeat=K * out * in_):
        S = np.array(pattern).reshape(K, out, in_)
        L = mk(out, in_, K, S.tolist(), row, col, group=g)
        y = oracle.gemv(L, x, "f32")[0]
        for o in range(out):
            expect = 0.0
            for k in range(K):
                for G in range(ng):
                    cols = range(G * g, min(in_, (G + 1) * g))
                    a = {i: float(col[k, i]) * float(x[0, i]) for i in cols}
                    set_sum = sum(a[i] for i in cols if py_bit(L.bits[k], out, in_, o, i))
                    expect += float(row[k, o, G]) * (2.0 * set_sum - sum(a.values()))
            assert y[o] == pytest.approx(expect, rel=1e-12, abs=1e-15)


# --- brute force on tiny shapes -----------------------------------------------

@pytest.mark.parametrize("out,in_,K", [(1, 1, 1), (1, 4, 1), (2, 2, 2), (2, 3, 1), (1, 4, 2), (2, 4, 2)])
def test_brute_force_all_sign_patterns(out, in_, K):
    """Every sign pattern: the oracle's unpacking matches the pattern and its
    product equals the sign-add identity sum_i (2b_i-1) a_i = 2 sum_{b_i=1} a_i - sum_i a_i
    evaluated from bits read with plain integer shifts."""
    rng = np.random.default_rng(out * 100 + in_ * 10 + K)
    row = f32(rng.uniform(0.5, 2.0, size=(K, out)))
    col = f32(rng.uniform(0.5, 2.0, size=(K, in_)))
    x = f32(rng.standard_normal((1, in_)))
    n = K * out * in_
    for pattern in itertools.product([-1, 1], repeat=n):
        S = np.array(pattern).reshape(K, out, in_)
        L = mk(out, in_, K, S.tolist(), row, col)
        for k in range(K):
            assert np.array_equal(oracle.unpack_bit_matrix(L.bits[k], out, in_), S[k])
        y = oracle.gemv(L, x, "f32")[0]
        for o in range(out):
            expect = 0.0
            for k in range(K):
                a = [float(col[k, i]) * float(x[0, i]) for i in range(in_)]
                set_sum = sum(a[i] for i in range(in_) if py_bit(L.bits[k], out, in_, o, i))
                expect += float(row[k, o]) * (2.0 * set_sum - sum(a))
            assert y[o] == pytest.approx(expect, rel=1e-12, abs=1e-15)


# --- packing ---------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(1, 1), (5, 7), (32, 128), (33, 129), (64, 256), (70, 300)])
def test_single_bit_positions(rows, cols):
    rng = np.random.default_rng(rows * cols)
    positions = [(i, c) for i in range(rows) for c in range(cols)]
    if len(positions) > 300:
        positions = [positions[k] for k in rng.choice(len(positions), 300, replace=False)]
        positions += [(0, 0), (rows - 1, cols - 1), (rows - 1, 0), (0, cols - 1)]
    for (i, c) in positions:
        S = -np.ones((rows, cols), np.int8)
        S[i, c] = 1
        words = py_pack(S.tolist())
        assert int(np.sum([bin(int(w)).count("1") for w in words])) == 1
        U = oracle.unpack_bit_matrix(words, rows, cols)
        assert U[i, c] == 1 and int(np.sum(U == 1)) == 1


@pytest.mark.parametrize("rows,cols", [(1, 3), (31, 127), (32, 128), (45, 200), (96, 520)])
def test_oracle_pack_matches_independent_packer(rows, cols):
    S = np.random.default_rng(rows + cols).choice(np.array([-1, 1], np.int8), size=(rows, cols))
    w = oracle.pack_bit_matrix(S)
    assert np.array_equal(w, py_pack(S.tolist()))
    assert np.array_equal(oracle.unpack_bit_matrix(w, rows, cols), S)


def test_pack_rejects_non_sign_values():
    with pytest.raises(ValueError):
        oracle.pack_bit_matrix(np.array([[1, 0, -1]]))
    with pytest.raises(ValueError):
        oracle.pack_bit_matrix(np.array([[1, 2]]))


# --- storage and byte accounting ------------------------------------------

def test_storage_arithmetic_matches_the_page():
    g = golden("storage_arithmetic.json")
    out, in_ = g["shape"]
    b512 = oracle.binary_correction_storage_bits(512, out, in_)
    assert b512 == 5_242_880
    assert b512 == pytest.approx(g["binary_rank512_bits_approx"], rel=0.02)
    bf16_32 = oracle.dense_correction_storage_bits(32, out, in_, 16)
    assert bf16_32 == b512 == pytest.approx(g["bf16_rank32_bits_approx"], rel=0.02)
    fp4 = oracle.fp4_weight_bits(out, in_, 4.5)
    assert fp4 == pytest.approx(g["fp4_weight_bits_approx"], rel=0.03)
    assert b512 / fp4 == pytest.approx(g["correction_fraction_approx"], rel=0.15)
    mib128 = oracle.binary_correction_storage_bits(128, out, in_) / 8 / 2 ** 20
    assert mib128 == 0.15625 == pytest.approx(g["binary_rank128_sign_bytes_MiB_approx"], rel=0.05)
    fp4_mib = oracle.fp4_weight_bits(out, in_, 4.0) / 8 / 2 ** 20
    assert fp4_mib == g["fp4_weight_MiB_approx"]
    assert fp4_mib / mib128 == g["read_ratio_approx"]


@pytest.mark.parametrize("rows,cols", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_fluxbin_average_bit_width_matches_the_page(rows, cols):
    # grouped row scales and binary salient refinement: the page prints the resulting
    # bit-widths (rounded) for three group/salient settings of its two-base configuration
    g = golden("fluxbin_abw.json")
    for c in g["cases"]:
        abw = oracle.fluxbin_average_bit_width(rows, cols, g["Kb"], g["Ks"], c["g"], c["s"])
        assert abw == pytest.approx(c["abw_approx"], abs=0.015), c
        if "salient_ratio" in c:
            assert c["s"] / c["g"] == c["salient_ratio"]
    # the grouped row scales and the refinement are visible at the page's precision: without
    # the refinement's row scales the typical configuration would read 2.38 bits, without
    # any row scale 2.13, without the refinement bases (Ks = 0) 2.26
    assert oracle.fluxbin_average_bit_width(rows, cols, 2, 0, 128, 8) == pytest.approx(2.26, abs=0.01)


def test_algorithmic_bytes_counts_each_payload():
    L = Layer(out=4096, in_=4096, K=2, scale_dtype="bf16", bits=None, row_scale=None, col_scale=None)
    # signs 2*4096*4096/8, scales 2*(4096+4096)*2 B, x 4096*2 B, y 4096*2 B
    assert oracle.algorithmic_bytes(L, 1, "bf16", "bf16") == 4_194_304 + 32_768 + 8_192 + 8_192
    L.rank = 512
    extra = 512 * (4096 + 4096) // 8 + 4 * 512
    assert oracle.algorithmic_bytes(L, 1, "bf16", "bf16") == 4_243_456 + extra


def test_algorithmic_bytes_salient_term():
    # Llama-7B gate/up layer (out 11008, in 4096, two bases, bf16 scales) with 41 salient
    # columns, batch 1, bf16 in and out, counted term by term by hand:
    #   signs 2*11008*4096/8 = 11,272,192; scales 2*(11008+4096)*2 = 60,416;
    #   salient int8 block 11008*41 = 451,328, fp32 scales 41*4 = 164, int32 indices 41*4 = 164;
    #   x 4096*2 = 8,192; y 11008*2 = 22,016                         -> 11,814,472
    L = Layer(out=11008, in_=4096, K=2, scale_dtype="bf16", bits=None, row_scale=None, col_scale=None, n_sal=41)
    assert oracle.algorithmic_bytes(L, 1, "bf16", "bf16") == 11_814_472
    # the down projection (out 4096, in 11008) with 111 salient columns:
    #   11,272,192 + 60,416 + 4096*111 + 111*8 + 11008*2 + 4096*2 -> 11,818,360
    L = Layer(out=4096, in_=11008, K=2, scale_dtype="bf16", bits=None, row_scale=None, col_scale=None, n_sal=111)
    assert oracle.algorithmic_bytes(L, 1, "bf16", "bf16") == 11_818_360
    # each salient column adds one int8 per output row plus its scale and its index
    L.n_sal = 112
    assert oracle.algorithmic_bytes(L, 1, "bf16", "bf16") == 11_818_360 + 4096 + 8


def test_algorithmic_bytes_grouped_and_refined():
    # FluxBin 2b-g128 and 2b-s16-g128 on 4096 x 4096 (Sec. 4 configurations), batch 1, bf16
    # x and y, counted by hand: signs 2*4096*4096/8 = 4,194,304; grouped row scales
    # 2*4096*32*2 = 524,288; column scales 2*4096*2 = 16,384; x 8,192; y 8,192 -> 4,751,360
    from synth import make_layer
    L = make_layer(0, (56,), 4096, 4096, 2, "bf16", group=128)
    assert oracle.algorithmic_bytes(L, 1, "bf16", "bf16") == 4_751_360
    # refinement over 16 salient columns of each of the 32 groups (n_ref = 512): signs
    # 2*4096*512/8 = 524,288; row scales 2*4096*32*2 = 524,288; column scales 2*512*2 = 2,048;
    # int32 indices 512*4 = 2,048 -> 1,052,672 more
    L = make_layer(0, (56,), 4096, 4096, 2, "bf16", group=128, refine=(2, 16))
    n = oracle.algorithmic_bytes(L, 1, "bf16", "bf16")
    assert n == 4_751_360 + 1_052_672
    # the weight bytes are the Sec. C.2 storage, but for int32 instead of 16-bit indices
    assert n - 8_192 - 8_192 - 2 * 512 == oracle.fluxbin_storage_bits(L) // 8


@pytest.mark.parametrize("rows,cols", [(70, 300), (33, 129), (1, 5)])
def test_row_decoder_matches_independent_packer(rows, cols):
    S = np.random.default_rng(7 * rows + cols).choice(np.array([-1, 1], np.int8), size=(rows, cols))
    w = py_pack(S.tolist())
    sel = sorted({0, rows - 1, rows // 2, min(31, rows - 1), min(32, rows - 1)})
    assert np.array_equal(oracle.unpack_bit_rows(w, rows, cols, sel), S[sel])


# ---- FluxBin joint sign search ("FluxBin", Sec. 3.1) --------------------------

def _mags(rng, Kb, rows, cols, ng=None):
    r = np.abs(rng.standard_normal((Kb, rows) if ng is None else (Kb, rows, ng))) + 0.05
    c = np.abs(rng.standard_normal((Kb, cols))) + 0.05
    return r, c


def test_fluxbin_one_base_is_the_sign_of_w():
    # Kb = 1: (w - m)^2 < (w + m)^2 exactly when w > 0 (m > 0); w = 0 ties and the first
    # combination (-1) is kept
    rng = np.random.default_rng(41)
    W = rng.standard_normal((7, 9))
    W[2, 3] = 0.0
    r, c = _mags(rng, 1, 7, 9)
    S = oracle.fluxbin_sign_search(W, r, c)
    assert np.array_equal(S[0], np.where(W > 0, 1, -1))


def test_fluxbin_two_bases_pick_the_nearest_of_four_levels():
    # Kb = 2 with m1 > m2 > 0 per element: the levels -m1-m2 < -m1+m2 < m1-m2 < m1+m2 have
    # midpoints -m1, 0, m1, so the optimum is (sign(w), sign(|w| - m1) * sign(w))
    rng = np.random.default_rng(42)
    rows, cols = 11, 13
    W = rng.standard_normal((rows, cols)) * 2.0
    r = np.stack([np.full(rows, 1.0), np.full(rows, 0.5)])
    c = np.stack([np.abs(rng.standard_normal(cols)) + 1.0, np.abs(rng.standard_normal(cols)) * 0.5 + 0.1])
    m1 = r[0][:, None] * c[0][None, :]
    m2 = r[1][:, None] * c[1][None, :]
    assert np.all(m1 > m2)
    S = oracle.fluxbin_sign_search(W, r, c)
    s1 = np.where(W >= 0, 1, -1)
    s2 = np.where(np.abs(W) >= m1, 1, -1) * s1
    assert np.array_equal(S[0], s1) and np.array_equal(S[1], s2)


def test_fluxbin_brute_force_on_a_tiny_layer():
    # every element against an explicit enumeration of sign vectors
    import itertools
    rng = np.random.default_rng(43)
    rows, cols, Kb = 2, 3, 3
    W = rng.standard_normal((rows, cols))
    r, c = _mags(rng, Kb, rows, cols)
    S = oracle.fluxbin_sign_search(W, r, c)
    for o in range(rows):
        for i in range(cols):
            errs = {}
            for sv in itertools.product((-1, 1), repeat=Kb):
                errs[sv] = (W[o, i] - sum(sv[k] * r[k, o] * c[k, i] for k in range(Kb))) ** 2
            chosen = tuple(int(S[k, o, i]) for k in range(Kb))
            assert errs[chosen] == min(errs.values())


def test_fluxbin_is_odd_and_beats_greedy_residual_signs():
    rng = np.random.default_rng(44)
    rows, cols, Kb = 16, 40, 3
    W = rng.standard_normal((rows, cols))
    r, c = _mags(rng, Kb, rows, cols)
    S = oracle.fluxbin_sign_search(W, r, c)
    assert np.array_equal(oracle.fluxbin_sign_search(-W, r, c), -S)  # symmetric levels, no ties
    M = r[:, :, None] * c[:, None, :]
    err = ((W - (S * M).sum(0)) ** 2).sum()
    R = W.copy()
    G = np.zeros_like(S)
    for k in range(Kb):  # greedy: each base takes the sign of the current residual
        G[k] = np.where(R >= 0, 1, -1)
        R = R - G[k] * M[k]
    assert err <= ((W - (G * M).sum(0)) ** 2).sum() + 1e-12


def test_fluxbin_grouped_row_scales_use_the_group_of_each_column():
    # one row scale per (row, group of g columns): equal to the ungrouped search run on each
    # column block with that block's row scale
    rng = np.random.default_rng(45)
    rows, cols, Kb, g = 5, 300, 2, 128
    ng = -(-cols // g)
    W = rng.standard_normal((rows, cols))
    r, c = _mags(rng, Kb, rows, cols, ng)
    S = oracle.fluxbin_sign_search(W, r, c, group=g)
    for j in range(ng):
        blk = slice(j * g, min(cols, (j + 1) * g))
        Sj = oracle.fluxbin_sign_search(W[:, blk], r[:, :, j], c[:, blk])
        assert np.array_equal(S[:, :, blk], Sj)


# ---- FluxBin binary salient refinement (Sec. 4, Kb-sS-gG) -----------------------

def _refine_layer(rng, out, in_, g, idx, Ks, signs, r, c, K=0):
    from synth.gen import Layer
    L = Layer(out=out, in_=in_, K=K, scale_dtype="f32", bits=np.zeros((K, 1), np.uint32),
              row_scale=np.zeros((K, out, -(-in_ // g)), np.float32), col_scale=np.zeros((K, in_), np.float32),
              group=g)
    L.ref_K = Ks
    L.ref_idx = np.asarray(idx, np.int32)
    L.ref_bits = np.stack([oracle.pack_bit_matrix(np.asarray(signs[k], np.int8)) for k in range(Ks)])
    L.ref_row_scale = np.asarray(r, np.float32)
    L.ref_col_scale = np.asarray(c, np.float32)
    return L


def test_refinement_all_plus_one_is_a_scaled_gathered_sum():
    rng = np.random.default_rng(51)
    out, in_, g, Ks = 5, 24, 8, 2
    idx = [1, 6, 9, 15, 17, 23]   # two salient columns per group of 8
    r = np.abs(rng.standard_normal((Ks, out, 3))).astype(np.float32)
    c = np.abs(rng.standard_normal((Ks, len(idx)))).astype(np.float32)
    L = _refine_layer(rng, out, in_, g, idx, Ks, [np.ones((out, len(idx)))] * Ks, r, c)
    x = rng.standard_normal((1, in_)).astype(np.float32)
    y = oracle.gemv(L, x, "f32")[0]
    want = np.zeros(out)
    for o in range(out):
        for k in range(Ks):
            for t, i in enumerate(idx):
                want[o] += float(r[k, o, i // g]) * float(c[k, t]) * float(x[0, i])
    assert np.allclose(y, want, rtol=1e-12, atol=0)


def test_refinement_brute_force_over_every_sign_pattern():
    import itertools
    rng = np.random.default_rng(52)
    out, in_, g, Ks = 2, 8, 4, 2
    idx = [2, 5]                  # one salient column in each group of 4
    r = np.abs(rng.standard_normal((Ks, out, 2))).astype(np.float32)
    c = np.abs(rng.standard_normal((Ks, 2))).astype(np.float32)
    for pat in itertools.product((-1, 1), repeat=Ks * out * 2):
        signs = np.array(pat).reshape(Ks, out, 2)
        L = _refine_layer(rng, out, in_, g, idx, Ks, signs, r, c)
        W = oracle.reconstruct(L)
        for o in range(out):
            for i in range(in_):
                want = 0.0
                for k in range(Ks):
                    for t, j in enumerate(idx):
                        if j == i:
                            want += float(r[k, o, j // g]) * float(c[k, t]) * signs[k, o, t]
                assert W[o, i] == want


def test_refinement_is_additive_on_the_global_bases():
    # zero refinement column scales give exactly the grouped global layer
    from synth import make_layer
    L = make_layer(0, (53,), 40, 300, 2, "f32", group=128, refine=(2, 8))
    W = oracle.reconstruct(L)
    L0 = make_layer(0, (53,), 40, 300, 2, "f32", group=128)
    assert not np.array_equal(W, oracle.reconstruct(L0))
    L.ref_col_scale = np.zeros_like(L.ref_col_scale)
    assert np.array_equal(oracle.reconstruct(L), oracle.reconstruct(L0))


@pytest.mark.parametrize("g,s", [(128, 8), (128, 16), (64, 16)])
def test_refinement_storage_matches_the_average_bit_width(g, s):
    # the bits a generated 2b-sS-gG layer stores equal the Sec. C.2 accounting, which
    # reproduces the page's 2.63 / 2.75 / 3.5 bits
    from synth import make_layer
    rows, cols = 64, 1024
    L = make_layer(0, (54, g, s), rows, cols, 2, "bf16", group=g, refine=(2, s))
    abw = oracle.fluxbin_storage_bits(L) / (rows * cols)
    assert abw == oracle.fluxbin_average_bit_width(rows, cols, 2, 2, g, s)

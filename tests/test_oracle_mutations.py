"""Planted mistakes in the oracle must trip at least one pin.

Each case monkeypatches one plausible error into a copy of an oracle function
(a dropped term, a flipped sign map, a transposed or mis-indexed operand) and
runs the pins of tests/test_oracle.py; the mutation is caught when any pin fails.
"""

import numpy as np
import pytest

import oracle.bisco_oracle as O
import test_oracle as P

PINS = [
    P.test_worked_example_correction_only,
    P.test_worked_example_as_one_base,
    P.test_toy_decomposition_refit_reconstructs_exactly,
    P.test_toy_greedy_coefficients_leave_the_printed_residual,
    P.test_all_plus_one_is_scaled_row_sum,
    P.test_salient_single_columns_closed_form,
    lambda: P.test_brute_force_all_sign_patterns(2, 3, 1),
    lambda: P.test_brute_force_all_sign_patterns(1, 4, 2),
    lambda: P.test_single_bit_positions(33, 129),
    lambda: P.test_oracle_pack_matches_independent_packer(45, 200),
    P.test_bf16_decode_by_definition,
    P.test_grouped_all_plus_one_is_a_sum_of_group_sums,
    P.test_biloco_decomposition_reproduces_the_page_toy,
    lambda: P.test_grouped_brute_force_all_sign_patterns(2, 4, 1, 2),
    P.test_refinement_all_plus_one_is_a_scaled_gathered_sum,
    P.test_refinement_brute_force_over_every_sign_pattern,
]


def _caught():
    for pin in PINS:
        try:
            pin()
        except Exception:
            return True
    return False


_orig_unpack = O.unpack_bit_matrix


def _unpack_inverted(words, rows, cols):
    return -_orig_unpack(words, rows, cols)


def _unpack_msb_first(words, rows, cols):
    T, Q = O._grid(rows, cols)
    w = np.asarray(words, dtype=np.uint32).reshape(T, Q, 32, 4)
    shifts = np.arange(31, -1, -1, dtype=np.uint32)
    bits = ((w[..., None] >> shifts) & 1).astype(np.int8)
    full = bits.transpose(0, 2, 1, 3, 4).reshape(T * 32, Q * 128)
    return full[:rows, :cols] * 2 - 1


def _unpack_tile_quad_swapped(words, rows, cols):
    T, Q = O._grid(rows, cols)
    w = np.asarray(words, dtype=np.uint32).reshape(Q, T, 32, 4).transpose(1, 0, 2, 3)
    bits = ((w[..., None] >> np.arange(32, dtype=np.uint32)) & 1).astype(np.int8)
    full = bits.transpose(0, 2, 1, 3, 4).reshape(T * 32, Q * 128)
    return full[:rows, :cols] * 2 - 1


def _binary_first_base_only(layer, rows):
    if layer.K == 0:
        return np.zeros((len(rows), layer.in_))
    R = O.decode_values(layer.row_scale, layer.scale_dtype).reshape(layer.K, layer.out)
    C = O.decode_values(layer.col_scale, layer.scale_dtype).reshape(layer.K, layer.in_)
    S = O.unpack_bit_matrix(np.asarray(layer.bits).reshape(layer.K, -1)[0], layer.out, layer.in_)[rows]
    return R[0, rows][:, None] * S * C[0][None, :]


def _binary_col_scale_of_base0(layer, rows):
    if layer.K == 0:
        return np.zeros((len(rows), layer.in_))
    R = O.decode_values(layer.row_scale, layer.scale_dtype).reshape(layer.K, layer.out)
    C = O.decode_values(layer.col_scale, layer.scale_dtype).reshape(layer.K, layer.in_)
    bits = np.asarray(layer.bits).reshape(layer.K, -1)
    W = np.zeros((len(rows), layer.in_))
    for k in range(layer.K):
        S = O.unpack_bit_matrix(bits[k], layer.out, layer.in_)[rows]
        W += R[k, rows][:, None] * S * C[0][None, :]
    return W


def _binary_grouped(layer, rows, group_of):
    """Binary part with the row-scale group of column i given by group_of(i, g)."""
    if layer.K == 0:
        return np.zeros((len(rows), layer.in_))
    g = getattr(layer, "group", 0)
    ng = -(-layer.in_ // g) if g else 1
    R = O.decode_values(layer.row_scale, layer.scale_dtype).reshape(layer.K, layer.out, ng)
    C = O.decode_values(layer.col_scale, layer.scale_dtype).reshape(layer.K, layer.in_)
    cols = np.arange(layer.in_)
    grp = np.minimum(group_of(cols, g), ng - 1) if g else np.zeros(layer.in_, dtype=np.int64)
    bits = np.asarray(layer.bits).reshape(layer.K, -1)
    W = np.zeros((len(rows), layer.in_))
    for k in range(layer.K):
        S = O.unpack_bit_matrix(bits[k], layer.out, layer.in_)[rows]
        W += R[k][rows][:, grp] * S * C[k][None, :]
    return W


def _binary_group_modulo(layer, rows):
    return _binary_grouped(layer, rows, lambda i, g: i % g)


def _binary_group_ignored(layer, rows):
    return _binary_grouped(layer, rows, lambda i, g: np.zeros_like(i))


_orig_decompose = O.biloco_decompose


def _decompose_alpha_over_rows(W, v0, rounds=5):
    U, V, greedy, refit = _orig_decompose(W, v0, rounds)
    return U, V, greedy * np.asarray(W).shape[1], refit   # u^T R v / rows instead of / (rows*cols)


def _decompose_refit_skipped(W, v0, rounds=5):
    U, V, greedy, _ = _orig_decompose(W, v0, rounds)
    return U, V, greedy, greedy.copy()


def _correction_alpha_dropped(layer, rows):
    if not layer.rank:
        return 0.0
    V = O.unpack_bit_matrix(layer.v_bits, layer.rank, layer.in_).astype(float)
    U = O.unpack_bit_matrix(layer.ut_bits, layer.out, layer.rank).astype(float)
    return U[rows] @ V


def _correction_u_read_transposed(layer, rows):
    if not layer.rank:
        return 0.0
    V = O.unpack_bit_matrix(layer.v_bits, layer.rank, layer.in_).astype(float)
    try:
        U = O.unpack_bit_matrix(layer.ut_bits, layer.rank, layer.out).astype(float).T
    except ValueError:
        raise AssertionError("layout misread")
    a = np.asarray(layer.alpha, np.float32).astype(float)
    return (U[rows] * a[None, :]) @ V


def _salient_dropped(layer, rows):
    return np.zeros((len(rows), layer.in_))


def _salient_wrong_column(layer, rows):
    W = np.zeros((len(rows), layer.in_))
    if not layer.n_sal:
        return W
    q = np.asarray(layer.sal_q, np.int8)[rows, : layer.n_sal].astype(float)
    s = np.asarray(layer.sal_scale, np.float32).astype(float)
    for t in range(layer.n_sal):
        W[:, t] += s[t] * q[:, t]          # column t instead of idx_t
    return W


def _refinement_variant(layer, rows, *, drop=False, group_of_position=False, col_scale_base0=False,
                        invert=False, column_t=False):
    W = np.zeros((len(rows), layer.in_), dtype=np.float64)
    Ks = getattr(layer, "ref_K", 0)
    if not Ks or drop:
        return W
    g = layer.group
    idx = np.asarray(layer.ref_idx, dtype=np.int64)
    n = len(idx)
    R = O.decode_values(layer.ref_row_scale, layer.scale_dtype).reshape(Ks, layer.out, -1)
    C = O.decode_values(layer.ref_col_scale, layer.scale_dtype).reshape(Ks, n)
    bits = np.asarray(layer.ref_bits).reshape(Ks, -1)
    grp = (np.arange(n) // g) if group_of_position else (idx // g)
    cols = np.arange(n) if column_t else idx
    for k in range(Ks):
        S = O.unpack_bit_rows(bits[k], layer.out, n, rows) * (-1 if invert else 1)
        ck = C[0] if col_scale_base0 else C[k]
        W[:, cols] += R[k][rows][:, grp] * S * ck[None, :]
    return W


def _gemv_untransposed(layer, X, x_dtype, rows):
    Xd = O.decode_values(X, x_dtype).reshape(-1, layer.in_)
    return Xd @ O.reconstruct_rows(layer, rows)


def _bf16_wrong_shift(a, dtype):
    if dtype == "bf16":
        u = np.asarray(a, np.uint16).astype(np.uint32) << np.uint32(15)
        return u.view(np.float32).astype(np.float64)
    return np.asarray(a, np.float32).astype(np.float64)


MUTATIONS = {
    "sign map inverted": ("unpack_bit_matrix", _unpack_inverted),
    "bits read MSB first": ("unpack_bit_matrix", _unpack_msb_first),
    "tile/quad axes swapped": ("unpack_bit_matrix", _unpack_tile_quad_swapped),
    "second base dropped": ("_binary_part_rows", _binary_first_base_only),
    "row-scale group taken as column mod g": ("_binary_part_rows", _binary_group_modulo),
    "row-scale groups ignored": ("_binary_part_rows", _binary_group_ignored),
    "column scale of base 0 reused": ("_binary_part_rows", _binary_col_scale_of_base0),
    "alpha dropped": ("_correction_part_rows", _correction_alpha_dropped),
    "u read transposed": ("_correction_part_rows", _correction_u_read_transposed),
    "salient term dropped": ("_salient_part_rows", _salient_dropped),
    "salient column index ignored": ("_salient_part_rows", _salient_wrong_column),
    "W not transposed": ("gemv_rows", _gemv_untransposed),
    "refinement dropped": ("_refinement_part_rows", lambda L, r: _refinement_variant(L, r, drop=True)),
    "refinement row-scale group taken from the gathered position":
        ("_refinement_part_rows", lambda L, r: _refinement_variant(L, r, group_of_position=True)),
    "refinement column scale of base 0 reused":
        ("_refinement_part_rows", lambda L, r: _refinement_variant(L, r, col_scale_base0=True)),
    "refinement signs inverted": ("_refinement_part_rows", lambda L, r: _refinement_variant(L, r, invert=True)),
    "refinement added at column t instead of idx_t":
        ("_refinement_part_rows", lambda L, r: _refinement_variant(L, r, column_t=True)),
    "decomposition coefficient over rows only": ("biloco_decompose", _decompose_alpha_over_rows),
    "decomposition refit skipped": ("biloco_decompose", _decompose_refit_skipped),
    "bf16 widened with wrong shift": ("decode_values", _bf16_wrong_shift),
}


def test_unmutated_oracle_passes_all_pins():
    assert not _caught()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    # the package namespace re-exports some functions: patch those too
    import oracle
    if hasattr(oracle, attr):
        monkeypatch.setattr(oracle, attr, fn)
    assert _caught(), f"planted mistake not caught: {name}"

"""The seeded generators: determinism, sizes, padding and the workload recipes."""

import numpy as np

import oracle
from synth import make_activations, make_layer, packed_words
from synth.configs import CONFIGS, build


def test_packed_words_sizes():
    assert packed_words(4096, 4096) == 4096 * 4096 // 32
    assert packed_words(33, 129) == 2 * 2 * 128
    assert packed_words(1, 1) == 128


def test_generation_is_deterministic_and_keyed():
    a = make_layer(0, (9, 9), 64, 256, 2, "bf16", rank=8)
    b = make_layer(0, (9, 9), 64, 256, 2, "bf16", rank=8)
    c = make_layer(0, (9, 8), 64, 256, 2, "bf16", rank=8)
    assert np.array_equal(a.bits, b.bits) and np.array_equal(a.v_bits, b.v_bits)
    assert not np.array_equal(a.bits, c.bits)


def test_padding_bits_are_zero():
    L = make_layer(1, (1,), 45, 200, 2, "f32", rank=5)
    for k in range(2):
        full = oracle.unpack_bit_matrix(L.bits[k], 64, 256)   # view the padded grid
        assert np.all(full[45:, :] == -1) and np.all(full[:, 200:] == -1)
    assert np.all(oracle.unpack_bit_matrix(L.v_bits, 32, 256)[5:, :] == -1)


def test_sign_balance_and_scale_distribution():
    L = make_layer(0, (3,), 1024, 1024, 1, "f32")
    S = oracle.unpack_bit_matrix(L.bits[0], 1024, 1024)
    assert abs(S.mean()) < 0.01
    r = L.row_scale.astype(np.float64)
    assert np.all(r >= 0) and abs(r.mean() - 0.02 * np.sqrt(2 / np.pi)) < 0.002


def test_outlier_channels():
    X = make_activations(0, (4, 0, 1001), 2, 5120, "f32", outlier_frac=0.001, outlier_factor=20.0)
    big = np.where(np.abs(X).max(axis=0) > 8)[0]
    assert 1 <= len(big) <= 6


def test_salient_recipe_cfg3_small_batch():
    L, X = build(3, 0, 1)
    assert L.n_sal == 41 and L.sal_q.shape == (11008, 48)
    assert np.all(np.diff(L.sal_idx) > 0)
    assert np.all(L.col_scale[:, L.sal_idx] == 0)
    assert np.all(L.sal_q[:, 41:] == 0)
    assert np.all(L.sal_scale > 0)


def test_config_table():
    assert [s.in_ for s in CONFIGS[3]["specs"]] == [4096, 11008]
    assert len(CONFIGS[5]["specs"]) == 224


def test_grouped_row_scales_shape_and_key():
    # one row scale per (base, row, group of g input columns); same stream as ungrouped
    L = make_layer(0, (9,), 40, 300, 2, "bf16", group=128)
    assert L.group == 128 and L.row_scale.shape == (2, 40, 3) and L.row_scale.dtype == np.uint16
    L0 = make_layer(0, (9,), 40, 300, 2, "bf16")
    assert L0.group == 0 and L0.row_scale.shape == (2, 40)
    assert np.array_equal(L.bits, L0.bits) and np.array_equal(L.col_scale, L0.col_scale)

"""The C ABI library on the host: it loads, exports every declared entry point,
packs bit-exactly like the oracle's packer, and rejects bad arguments.
No GPU is needed; no device computation is called."""

import os
import re

import numpy as np
import pytest

import binary_weight_decode_b200 as bw
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "bisco.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bisco_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_entry_points()
    assert "bisco_gemv" in names and "bisco_pack" in names and "bisco_bench" in names
    for n in names:
        assert hasattr(bw._lib, n), f"libbisco.so does not export {n}"
    assert sorted(bw.EXPORTED) == names


def test_packed_words():
    assert bw.bisco_packed_words(4096, 4096) == 4096 * 4096 // 32
    assert bw.bisco_packed_words(33, 129) == 512
    assert bw.bisco_packed_words(0, 5) == 0


@pytest.mark.parametrize("rows,cols", [(1, 1), (5, 7), (32, 128), (33, 129), (100, 1000), (257, 4096)])
def test_pack_matches_oracle_bit_exact(rows, cols):
    S = np.random.default_rng(rows * 7 + cols).choice(np.array([-1, 1], np.int8), size=(rows, cols))
    w = bw.bisco_pack(S)
    assert np.array_equal(w, oracle.pack_bit_matrix(S))
    assert np.array_equal(bw.bisco_unpack(w, rows, cols), S)
    assert np.array_equal(oracle.unpack_bit_matrix(w, rows, cols), S)


def test_pack_single_bits():
    for (i, c) in [(0, 0), (31, 127), (32, 128), (40, 300), (40, 31), (40, 32)]:
        S = -np.ones((41, 301), np.int8)
        S[i, c] = 1
        w = bw.bisco_pack(S)
        assert sum(bin(int(x)).count("1") for x in w) == 1
        U = oracle.unpack_bit_matrix(w, 41, 301)
        assert U[i, c] == 1 and (U == 1).sum() == 1


def test_pack_rejects_non_signs_and_writes_nothing():
    bad = np.ones((3, 40), np.int8)
    bad[2, 39] = 0
    out = np.full(bw.bisco_packed_words(3, 40), 0xDEADBEEF, np.uint32)
    st = bw._lib.bisco_pack(bad.ctypes.data, 3, 40, out.ctypes.data)
    assert st == bw.BISCO_ERR_INVALID_ARG
    assert np.all(out == 0xDEADBEEF)
    assert bw._lib.bisco_pack(None, 3, 40, out.ctypes.data) == bw.BISCO_ERR_INVALID_ARG
    assert bw._lib.bisco_pack(bad.ctypes.data, 0, 40, out.ctypes.data) == bw.BISCO_ERR_INVALID_ARG


def test_gemv_rejects_bad_arguments_before_touching_the_device():
    L = bw.bisco_layer(out=0, in_=10, num_bases=0)
    assert bw._lib.bisco_gemv(L, None, 0, 1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG
    L = bw.bisco_layer(out=10, in_=10, num_bases=5)
    assert bw._lib.bisco_gemv(L, None, 0, 1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG
    L = bw.bisco_layer(out=10, in_=10, num_bases=1)          # null bits
    assert bw._lib.bisco_gemv(L, None, 0, 1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG
    L = bw.bisco_layer(out=10, in_=10, num_bases=0, n_sal=3, sal_stride=8)
    assert bw._lib.bisco_gemv(L, None, 0, 1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG
    L = bw.bisco_layer(out=10, in_=10, num_bases=0)
    assert bw._lib.bisco_gemv(L, None, 7, 1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG   # dtype
    assert bw._lib.bisco_gemv(L, None, 0, -1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG  # M < 0
    assert bw._lib.bisco_gemv(L, None, 0, 0, None, 0, None, 0, None) == bw.BISCO_OK                # M == 0
    assert bw.bisco_status_string(bw.BISCO_ERR_WORKSPACE) == "BISCO_ERR_WORKSPACE"


def test_row_group_field_and_negative_group():
    # bisco_layer ends with row_group (0 = one row scale per row); a negative group is
    # refused before anything touches the device
    hdr = open(os.path.join(ROOT, "include", "bisco.h")).read()
    body = hdr[hdr.index("typedef struct {", hdr.index("One layer.")):hdr.index("} bisco_layer;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)  # drop comments
    declared = re.findall(r"(\w+)\s*;", body)  # field names in declaration order
    assert [n.rstrip("_") for n, _ in bw.bisco_layer._fields_] == declared
    assert declared[-1] == "row_group"
    L = bw.bisco_layer(out=10, in_=10, num_bases=0, row_group=-1)
    assert bw._lib.bisco_gemv(L, None, 0, 1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG


def test_salient_refinement_is_refused_by_the_binding():
    # no kernel runs FluxBin's refinement bases: the binding refuses such a layer instead of
    # silently dropping a term
    from synth import make_layer
    L = make_layer(0, (55,), 64, 256, 2, "bf16", group=128, refine=(2, 8))
    with pytest.raises(NotImplementedError):
        bw.DeviceLayer(L)


def test_group_call_validates_before_touching_the_device():
    # bisco_gemv_group: 1..3 layers of one input width; the workspace size is host arithmetic
    import ctypes
    a = bw.bisco_layer(out=64, in_=256, num_bases=0)
    b = bw.bisco_layer(out=32, in_=256, num_bases=0, rank=0)
    c = bw.bisco_layer(out=32, in_=384, num_bases=0)
    arr = (bw.bisco_layer * 4)(a, b, a, b)
    Y = (ctypes.c_void_p * 4)()
    assert bw._lib.bisco_gemv_group(arr, 0, None, 0, 1, Y, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG
    assert bw._lib.bisco_gemv_group(arr, 4, None, 0, 1, Y, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG
    mixed = (bw.bisco_layer * 2)(a, c)
    assert bw._lib.bisco_gemv_group(mixed, 2, None, 0, 1, Y, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    assert bw._lib.bisco_group_workspace_size(arr, 2, 1, ctypes.byref(n)) == bw.BISCO_OK
    assert n.value >= 256  # the status region at least
    assert bw._lib.bisco_group_workspace_size(mixed, 2, 1, ctypes.byref(n)) == bw.BISCO_ERR_INVALID_ARG

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


def test_binding_constants_match_the_header():
    # every enumerator the header declares (status codes, dtypes, policies, kernel kinds)
    # exists in the binding with the same value
    hdr = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "bisco.h")).read(), flags=re.S)
    found = 0
    for body in re.findall(r"(?:typedef\s+)?enum\s*\w*\s*\{(.*?)\}", hdr, flags=re.S):
        nxt = 0
        for item in [i.strip() for i in body.split(",") if i.strip()]:
            name, _, val = item.partition("=")
            name = name.strip()
            nxt = int(val.strip(), 0) if val.strip() else nxt
            assert getattr(bw, name) == nxt, name
            found += 1
            nxt += 1
    assert found >= 18 and bw.BISCO_KERNEL_REFINE == 6


def test_layer_fields_and_negative_group():
    # the binding's struct mirrors bisco_layer field by field (row_group, then the salient
    # refinement's six fields last); a negative group is refused before anything touches
    # the device
    hdr = open(os.path.join(ROOT, "include", "bisco.h")).read()
    body = hdr[hdr.index("typedef struct {", hdr.index("One layer.")):hdr.index("} bisco_layer;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)  # drop comments
    declared = re.findall(r"(\w+)\s*;", body)  # field names in declaration order
    assert [n.rstrip("_") for n, _ in bw.bisco_layer._fields_] == declared
    assert declared[-7:] == ["row_group", "ref_bases", "n_ref", "ref_idx", "ref_bits", "ref_row_scale",
                             "ref_col_scale"]
    L = bw.bisco_layer(out=10, in_=10, num_bases=0, row_group=-1)
    assert bw._lib.bisco_gemv(L, None, 0, 1, None, 0, None, 0, None) == bw.BISCO_ERR_INVALID_ARG


def _refined_desc(**kw):
    # a descriptor with placeholder (never dereferenced) 16-byte aligned addresses: the
    # calls below only validate and size
    import ctypes
    f = dict(out=96, in_=512, num_bases=1, bits=0x1000, row_scale=0x2000, col_scale=0x3000,
             scale_dtype=bw.BISCO_BF16, row_group=128, ref_bases=2, n_ref=32, ref_idx=0x4000,
             ref_bits=0x5000, ref_row_scale=0x6000, ref_col_scale=0x7000)
    f.update(kw)
    return (bw.bisco_layer * 1)(bw.bisco_layer(**f)), ctypes


def test_salient_refinement_fields_are_validated():
    # FluxBin's refinement (Sec. 4, Kb-sS-gG) needs the group size of its row scales, 1..4
    # bases, 1..in gathered columns, every array, and 16-byte aligned packed signs
    ok, ctypes = _refined_desc()
    n = ctypes.c_size_t(0)
    assert bw._lib.bisco_group_workspace_size(ok, 1, 1, ctypes.byref(n)) == bw.BISCO_OK
    # status region, no z, then the refinement term of one 8-row chunk: 8 * 96 fp32
    assert n.value == 256 + 8 * 96 * 4
    okz, _ = _refined_desc(rank=64, v_bits=0x8000, ut_bits=0x9000, alpha=0xA000)
    assert bw._lib.bisco_group_workspace_size(okz, 1, 40, ctypes.byref(n)) == bw.BISCO_OK
    assert n.value == 256 + 8 * 64 * 4 + 8 * 96 * 4  # refined layers never take 16-row chunks
    bad = [dict(row_group=0), dict(ref_bases=5), dict(ref_bases=-1), dict(n_ref=0), dict(n_ref=513),
           dict(ref_idx=None), dict(ref_bits=None), dict(ref_row_scale=None), dict(ref_col_scale=None),
           dict(ref_bits=0x5004), dict(scale_dtype=7)]
    for kw in bad:
        d, _ = _refined_desc(**kw)
        assert bw._lib.bisco_group_workspace_size(d, 1, 1, ctypes.byref(n)) == bw.BISCO_ERR_INVALID_ARG, kw
    # without refinement bases the other refinement fields are ignored
    d, _ = _refined_desc(ref_bases=0, n_ref=0, ref_idx=None, ref_bits=None)
    assert bw._lib.bisco_group_workspace_size(d, 1, 1, ctypes.byref(n)) == bw.BISCO_OK
    assert n.value == 256


def test_no_alloc_entry_refuses_a_refined_layer():
    # the fixed scratch array has no room for the refinement term
    ok, _ = _refined_desc()
    assert bw._lib.bisco_gemv_noalloc(ok, None, 0, 1, None, 0, None) == bw.BISCO_ERR_UNSUPPORTED


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

"""GPU parity of FluxBin's binary salient refinement ("FluxBin", Sec. 4, configurations
Kb-sS-gG; Sec. 3.2, Virtual Columnar Mapping): Ks extra sign bases over the s salient
columns of every column group, stored densely over the gathered columns, with one row
scale per (base, row, group) and one column scale per (base, gathered column):
W[o][idx_t] += sum_k r_k[o][idx_t // g] c_k[t] (2b - 1).

The library computes the term in its own launch (BISCO_KERNEL_REFINE) and the integer
tensor-core launch after it adds the term before rounding the output. Bars are those of
tests/test_gemv_gpu.py; the main cases also check the device's refinement term alone (Y
minus the same layer run without it) against the oracle's term, so a dropped, mis-signed or
mis-grouped term cannot hide inside the bar when the rest of Y is much larger.
"""

import copy

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import binary_weight_decode_b200 as bw  # noqa: E402
import oracle  # noqa: E402
from synth import make_activations, make_layer  # noqa: E402

from test_gemv_gpu import check, run, sample_rows, to_dev_x  # noqa: E402


def kinds(L, M, xdt="bf16"):
    dl = bw.DeviceLayer(L)
    ws = bw.bisco_workspace_size(dl, M)
    return bw.bisco_plan_kernels(dl, M, bw.BISCO_BF16 if xdt == "bf16" else bw.BISCO_F32, ws)


def without_refinement(L):
    L0 = copy.copy(L)
    L0.ref_K = 0
    return L0


def check_term(L, X, xdt, Y, rows=None):
    # the device's refinement term alone: Y minus the same layer run without it (the rest
    # of the row is computed identically in both runs), against the oracle's term, to
    # 1e-3 relative L2 of the term itself, so that the term is checked however small it is
    # next to the rest of Y
    L0 = without_refinement(L)
    Y0 = run(L0, X, xdt, "f32")
    if rows is None:
        T = oracle.gemv(L, X, xdt) - oracle.gemv(L0, X, xdt)
    else:
        Y, Y0 = Y[:, rows], Y0[:, rows]
        T = oracle.gemv_rows(L, X, xdt, rows) - oracle.gemv_rows(L0, X, xdt, rows)
    nt = np.linalg.norm(T)
    assert nt > 0
    rel = np.linalg.norm((Y - Y0) - T) / nt
    assert rel <= 1e-3, f"refinement term rel-L2 {rel:.3e}"


CASES = [
    # out, in, K, rank, salient int8 fraction, g, scale dtype, (Ks, s)
    (300, 1000, 2, 16, 0.01, 128, "bf16", (2, 8)),   # ragged rows, last group of 104 columns
    (256, 1536, 2, 0, 0.0, 256, "bf16", (2, 16)),
    (1000, 640, 3, 40, 0.02, 384, "f32", (1, 8)),   # last group of 256 columns
    (130, 4100, 2, 33, 0.0, 128, "bf16", (4, 8)),    # 33 groups, four refinement bases
    (64, 128, 1, 0, 0.0, 128, "f32", (2, 128)),      # every column salient (n_ref = in)
    (96, 600, 2, 0, 0.0, 128, "bf16", (2, 1)),       # one salient column per group
    (40, 200, 1, 0, 0.0, 1024, "f32", (3, 5)),       # one group wider than the row
    (96, 4096, 2, 8, 0.0, 128, "bf16", (2, 64)),     # n_ref = 2048: 16 sign words per row
]
IDS = ["ragged", "g256_s16", "g384_f32", "ks4_many_groups", "all_salient", "s1", "g_wide", "half_salient"]


@pytest.mark.parametrize("out,in_,K,rank,sal,g,sdt,ref", CASES, ids=IDS)
@pytest.mark.parametrize("M", [1, 2, 5, 8])
def test_salient_refinement(out, in_, K, rank, sal, g, sdt, ref, M):
    X = make_activations(0, (850, out, in_, M), M, in_, "bf16")
    L = make_layer(0, (850, out, in_, g), out, in_, K, sdt, rank=rank, sal_frac=sal,
                   x_for_salience=X if sal else None, x_dtype="bf16", group=g, refine=ref)
    ks = kinds(L, M)
    assert ks[0] == bw.BISCO_KERNEL_REFINE and ks.count(bw.BISCO_KERNEL_REFINE) == 1
    assert set(ks[1:]) == {bw.BISCO_KERNEL_INTEGER_MMA}
    Y = run(L, X, "bf16", "f32")
    check(Y, oracle.gemv(L, X, "bf16"), X, "bf16", "f32")
    check_term(L, X, "bf16", Y)


@pytest.mark.parametrize("xdt,ydt", [("f32", "f32"), ("bf16", "bf16"), ("f32", "bf16")])
def test_salient_refinement_dtypes(xdt, ydt):
    X = make_activations(0, (851, 0 if xdt == "f32" else 1), 3, 900, xdt)
    L = make_layer(0, (851,), 200, 900, 2, "bf16", rank=8, group=128, refine=(2, 16))
    check(run(L, X, xdt, ydt), oracle.gemv(L, X, xdt), X, xdt, ydt)


@pytest.mark.parametrize("M", [9, 20])
def test_salient_refinement_several_chunks(M):
    # one refinement launch per 8-row chunk, the term buffer reused by every chunk
    X = make_activations(0, (852, M), M, 768, "bf16")
    L = make_layer(0, (852,), 160, 768, 2, "bf16", rank=24, group=128, refine=(2, 8))
    ks = kinds(L, M)
    chunks = -(-M // 8)
    assert ks.count(bw.BISCO_KERNEL_REFINE) == chunks
    assert bw.BISCO_KERNEL_TENSOR_CORE not in ks
    check(run(L, X, "bf16", "f32"), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


@pytest.mark.parametrize("out,in_,M,s", [(4096, 4096, 1, 16), (4096, 11008, 8, 16), (11008, 4096, 4, 8)],
                         ids=["attn_2b_s16_m1", "down_2b_s16_m8", "gate_2b_s8_m4"])
def test_salient_refinement_llama_shapes_sampled(out, in_, M, s):
    # the pages' 2b-s8-g128 / 2b-s16-g128 on LLaMA-7B layer shapes, sampled output rows
    X = make_activations(0, (853, out, in_), M, in_, "bf16")
    L = make_layer(0, (853, out, in_), out, in_, 2, "bf16", group=128, refine=(2, s))
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 160, 11)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")
    check_term(L, X, "bf16", Y, rows)


def test_refined_layer_runs_on_the_integer_kernel_under_every_policy():
    L = make_layer(0, (854,), 256, 512, 2, "bf16", group=128, refine=(2, 8))
    try:
        for pol in (bw.BISCO_PATH_AUTO, bw.BISCO_PATH_LOOKUP_TABLE, bw.BISCO_PATH_SMALL_BATCH_ONLY):
            bw.bisco_set_path_policy(pol)
            assert kinds(L, 1) == [bw.BISCO_KERNEL_REFINE, bw.BISCO_KERNEL_INTEGER_MMA]
            assert kinds(L, 64) == [bw.BISCO_KERNEL_REFINE, bw.BISCO_KERNEL_INTEGER_MMA] * 8
    finally:
        bw.bisco_set_path_policy(bw.BISCO_PATH_AUTO)


def test_refined_layer_is_deterministic_and_leaves_the_workspace_ready():
    X = make_activations(0, (855,), 6, 1024, "bf16")
    L = make_layer(0, (855,), 384, 1024, 2, "bf16", rank=32, group=128, refine=(2, 16))
    dl = bw.DeviceLayer(L)
    ws = bw.alloc_workspace([dl], 6)
    a = run(L, X, "bf16", "f32", ws=ws, dl=dl)
    b = run(L, X, "bf16", "f32", ws=ws, dl=dl)
    assert np.array_equal(a, b)


def test_refined_layer_in_a_group_call():
    # a group with a refined layer runs layer by layer; results as bisco_gemv
    X = make_activations(0, (856,), 3, 512, "bf16")
    Ls = [make_layer(0, (856, j), 128 + 64 * j, 512, 2, "bf16", group=128, refine=(2, 8) if j == 1 else None)
          for j in range(3)]
    dls = [bw.DeviceLayer(L) for L in Ls]
    Xd = to_dev_x(X, "bf16")
    Ys = [torch.empty((3, L.out), dtype=torch.float32, device="cuda") for L in Ls]
    ws = bw.alloc_group_workspace(dls, 3)
    bw.bisco_gemv_group(dls, Xd, Ys, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    for L, Yd in zip(Ls, Ys):
        check(Yd.cpu().numpy().astype(np.float64), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


@pytest.mark.parametrize("keep", [0, 1, 2])
@pytest.mark.parametrize("M", [1, 8])
def test_refinement_with_empty_groups(keep, M):
    # only the groups j with j % 3 == keep hold salient columns: the first, last or inner
    # groups have none (the group boundaries of an empty group coincide)
    X = make_activations(0, (859, M), M, 1100, "bf16")
    L = make_layer(0, (859,), 170, 1100, 2, "bf16", rank=8, group=128, refine=(2, 8))
    idx = np.asarray(L.ref_idx)
    sel = (idx // 128) % 3 == keep
    n = int(sel.sum())
    S = np.stack([oracle.unpack_bit_matrix(np.asarray(L.ref_bits)[k], L.out, len(idx)) for k in range(2)])
    L.ref_idx = np.ascontiguousarray(idx[sel]).astype(np.int32)
    L.ref_bits = np.stack([oracle.pack_bit_matrix(S[k][:, sel]) for k in range(2)])
    L.ref_col_scale = np.ascontiguousarray(np.asarray(L.ref_col_scale)[:, sel])
    assert 0 < n < len(idx)
    Y = run(L, X, "bf16", "f32")
    check(Y, oracle.gemv(L, X, "bf16"), X, "bf16", "f32")
    check_term(L, X, "bf16", Y)


@pytest.mark.parametrize("world,M", [(3, 1), (2, 8)])
def test_refined_layer_row_shards_on_the_device(world, M):
    # row shards of a refined layer (its signs and row scales cut by rows, indices and
    # column scales replicated) run one after another on one GPU; side by side they meet the
    # bar against the whole layer's oracle product
    from binary_weight_decode_b200 import shard
    X = make_activations(0, (858, M), M, 700, "bf16")
    L = make_layer(0, (858,), 200, 700, 2, "bf16", rank=8, group=128, refine=(2, 8))
    parts = [run(shard.shard_rows(L, r, world), X, "bf16") for r in range(world)]
    check(np.concatenate(parts, axis=1), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


def test_out_of_range_refinement_index_is_reported_not_read():
    # a gathered column outside [0, in) is recorded as BISCO_ERR_INVALID_ARG by the kernel,
    # which reads zero in its place
    L = make_layer(0, (857,), 64, 256, 1, "bf16", group=128, refine=(1, 8))
    L.ref_idx = L.ref_idx.copy()
    L.ref_idx[-1] = 256
    dl = bw.DeviceLayer(L)
    X = to_dev_x(make_activations(0, (857,), 1, 256, "bf16"), "bf16")
    Y = torch.empty((1, 64), dtype=torch.float32, device="cuda")
    ws = bw.alloc_workspace([dl], 1)
    bw.bisco_gemv(dl, X, Y, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_ERR_INVALID_ARG

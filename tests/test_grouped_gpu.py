"""GPU parity of grouped row scales ("FluxBin", Sec. 3.1: one row scale per weight group,
Sec. 4: g is the group size of the row-wise scale): W_k[o][i] = r_k[o][i // g] c_k[i] (2b - 1).

The integer tensor-core kernel applies them per 128-column unit, so the library takes g a
multiple of 128 and runs grouped layers on that kernel whatever the batch size; other
group sizes are refused with BISCO_ERR_UNSUPPORTED. Bars are those of tests/test_gemv_gpu.py.
"""

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


@pytest.mark.parametrize("out,in_,K,rank,sal,g,sdt", [
    (300, 1000, 2, 16, 0.01, 128, "bf16"),   # ragged last group and last unit
    (256, 1536, 2, 0, 0.0, 256, "bf16"),
    (1000, 640, 3, 40, 0.02, 384, "f32"),    # last group of 256 columns
    (64, 128, 1, 0, 0.0, 128, "f32"),        # one group
    (200, 300, 2, 8, 0.0, 1024, "bf16"),     # group wider than the row
    (130, 4100, 2, 33, 0.0, 128, "bf16"),    # 33 groups, ragged rows and columns
], ids=["ragged", "g256", "g384_f32", "one_group", "g_wide", "many_groups"])
@pytest.mark.parametrize("M", [1, 2, 8])
def test_grouped_row_scales(out, in_, K, rank, sal, g, sdt, M):
    X = make_activations(0, (830, out, in_, M), M, in_, "bf16")
    L = make_layer(0, (830, out, in_, g), out, in_, K, sdt, rank=rank, sal_frac=sal,
                   x_for_salience=X if sal else None, x_dtype="bf16", group=g)
    assert set(kinds(L, M)) == {bw.BISCO_KERNEL_INTEGER_MMA}
    check(run(L, X, "bf16", "f32"), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


def test_grouped_layer_llama_shape_sampled():
    # 4096 x 4096, two bases, g = 128 (the pages' 2b-g128), one batch row
    X = make_activations(0, (831,), 1, 4096, "bf16")
    L = make_layer(0, (831,), 4096, 4096, 2, "bf16", group=128)
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 192, 9)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


def test_grouped_down_projection_at_eight_rows():
    # 4096 x 11008 (the down projection), g = 128, 8 batch rows: the integer plan of 8 rows
    # does not fit shared memory, so the chunk runs as smaller integer launches
    X = make_activations(0, (834,), 8, 11008, "bf16")
    L = make_layer(0, (834,), 4096, 11008, 2, "bf16", group=128)
    ks = kinds(L, 8)
    assert set(ks) == {bw.BISCO_KERNEL_INTEGER_MMA} and len(ks) >= 1
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 128, 10)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


def test_grouped_layers_take_the_integer_kernel_under_every_policy():
    L = make_layer(0, (832,), 256, 512, 2, "bf16", group=128)
    try:
        for pol in (bw.BISCO_PATH_AUTO, bw.BISCO_PATH_LOOKUP_TABLE, bw.BISCO_PATH_SMALL_BATCH_ONLY):
            bw.bisco_set_path_policy(pol)
            assert kinds(L, 1) == [bw.BISCO_KERNEL_INTEGER_MMA]
            # no tcgen05 chunks: 64 rows run as eight chunks of 8
            assert kinds(L, 64) == [bw.BISCO_KERNEL_INTEGER_MMA] * 8
    finally:
        bw.bisco_set_path_policy(bw.BISCO_PATH_AUTO)


@pytest.mark.parametrize("g", [64, 100, 192])
def test_group_sizes_off_the_unit_grid_are_refused(g):
    L = make_layer(0, (833, g), 64, 512, 2, "bf16", group=g)
    dl = bw.DeviceLayer(L)
    X = to_dev_x(make_activations(0, (833,), 1, 512, "bf16"), "bf16")
    Y = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    ws = bw.alloc_workspace([dl], 1)
    with pytest.raises(bw.BiscoError) as e:
        bw.bisco_gemv(dl, X, Y, ws)
    assert e.value.status == bw.BISCO_ERR_UNSUPPORTED
    with pytest.raises(bw.BiscoError):  # the plan query reports -1 for an unsupported request
        bw.bisco_plan_kernels(dl, 1, bw.BISCO_BF16, ws.numel())
    assert torch.count_nonzero(Y) == 0  # nothing was written

"""GPU parity of bisco_gemv_group: layers that read the same x in one integer launch per
batch chunk (clusters split between the layers and, for layers with a correction, between
their z and output passes). Every output is compared with the oracle's product of its own
layer; bars are those of tests/test_gemv_gpu.py.
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
from synth.configs import build  # noqa: E402

from test_gemv_gpu import check, sample_rows, to_dev_x  # noqa: E402


def run_group(layers, X, x_dtype="bf16", y_dtype="f32"):
    dls = [bw.DeviceLayer(L) for L in layers]
    M = X.shape[0]
    Xd = to_dev_x(X, x_dtype)
    yt = torch.float32 if y_dtype == "f32" else torch.bfloat16
    Ys = [torch.empty((M, L.out), dtype=yt, device="cuda") for L in layers]
    ws = bw.alloc_group_workspace(dls, M)
    bw.bisco_gemv_group(dls, Xd, Ys, ws)
    st = bw.bisco_sync_status(ws)
    assert st == bw.BISCO_OK, bw.bisco_status_string(st)
    return [y.float().cpu().numpy().astype(np.float64) for y in Ys], dls, ws


def small_group(M, seed=850):
    X = make_activations(0, (seed, M), M, 1000, "bf16")
    layers = [make_layer(0, (seed, 1), 300, 1000, 2, "bf16", rank=16, sal_frac=0.01, x_for_salience=X, x_dtype="bf16"),
              make_layer(0, (seed, 2), 130, 1000, 1, "bf16"),
              make_layer(0, (seed, 3), 777, 1000, 3, "bf16", rank=40)]
    return layers, X


@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 40])
def test_group_of_three_layers(M):
    layers, X = small_group(M)
    Ys, dls, ws = run_group(layers, X)
    for L, Y in zip(layers, Ys):
        check(Y, oracle.gemv(L, X, "bf16"), X, "bf16", "f32")
    kinds = bw.bisco_plan_group_kernels(dls, M, bw.BISCO_BF16, ws.numel())
    if M < 32:  # one integer launch per 8-row chunk
        assert kinds == [bw.BISCO_KERNEL_INTEGER_MMA] * ((M + 7) // 8)


@pytest.mark.parametrize("M", [1, 2])
def test_group_two_layers_f32_and_grouped_scales(M):
    X = make_activations(0, (851, M), M, 640, "f32")
    layers = [make_layer(0, (851, 1), 200, 640, 2, "f32", rank=8, group=128),
              make_layer(0, (851, 2), 333, 640, 2, "f32")]
    Ys, _, _ = run_group(layers, X, "f32", "f32")
    for L, Y in zip(layers, Ys):
        check(Y, oracle.gemv(L, X, "f32"), X, "f32", "f32")


@pytest.mark.parametrize("M", [1, 4])
def test_decoder_qkv_and_gate_up_groups_sampled(M):
    # layer 0 of the decoder stream: q, k, v (4096 x 4096) and gate, up (11008 x 4096), each
    # with two bases and a rank-256 correction, sharing one x per group
    mats = [build(5, i, M)[0] for i in (0, 1, 2, 4, 5)]
    X = build(5, 0, M)[1]
    for grp in (mats[:3], mats[3:]):
        Ys, _, _ = run_group(grp, X)
        for j, (L, Y) in enumerate(zip(grp, Ys)):
            rows = sample_rows(L.out, 128, 60 + j)
            check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


def test_group_repeats_are_identical_and_counters_return_to_zero():
    layers, X = small_group(2, seed=852)
    dls = [bw.DeviceLayer(L) for L in layers]
    Xd = to_dev_x(X, "bf16")
    ws = bw.alloc_group_workspace(dls, 2)
    outs = []
    for _ in range(3):
        Ys = [torch.empty((2, L.out), dtype=torch.float32, device="cuda") for L in layers]
        bw.bisco_gemv_group(dls, Xd, Ys, ws)
        outs.append(Ys)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    assert int(ws[128:256].to(torch.int32).sum()) == 0  # ready counters (words 32..) and done counter (48)
    for Ys in outs[1:]:
        for a, b in zip(Ys, outs[0]):
            assert torch.equal(a, b)


def test_group_wait_gives_up_and_reports_timeout():
    layers, X = small_group(1, seed=853)
    dls = [bw.DeviceLayer(L) for L in layers]
    Xd = to_dev_x(X, "bf16")
    ws = bw.alloc_group_workspace(dls, 1)
    Ys = [torch.empty((1, L.out), dtype=torch.float32, device="cuda") for L in layers]
    try:
        bw.bisco_debug_set_wait_test(0, 1_000_000)
        bw.bisco_gemv_group(dls, Xd, Ys, ws)
        assert bw.bisco_sync_status(ws) == bw.BISCO_ERR_TIMEOUT
    finally:
        bw.bisco_debug_set_wait_test(-1, 0)
    bw.bisco_workspace_init(ws)
    bw.bisco_gemv_group(dls, Xd, Ys, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    for L, Y in zip(layers, Ys):
        check(Y.cpu().numpy().astype(np.float64), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


def test_group_rejects_layers_of_different_width():
    a = bw.DeviceLayer(make_layer(0, (854, 1), 64, 256, 1, "bf16"))
    b = bw.DeviceLayer(make_layer(0, (854, 2), 64, 384, 1, "bf16"))
    X = to_dev_x(make_activations(0, (854,), 1, 256, "bf16"), "bf16")
    ws = bw.alloc_workspace([a, b], 1)
    Ys = [torch.empty((1, 64), dtype=torch.float32, device="cuda") for _ in range(2)]
    with pytest.raises(bw.BiscoError) as e:
        bw.bisco_gemv_group([a, b], X, Ys, ws)
    assert e.value.status == bw.BISCO_ERR_INVALID_ARG

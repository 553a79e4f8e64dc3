"""GPU parity of every small-batch kernel family, the kernel choice itself, and the
bounded device-side waits of the integer tensor-core kernel.

The default path runs batch chunks of up to 8 rows on the integer tensor-core kernel;
the lookup-table kernels remain the fallback (and the BISCO_PATH_LOOKUP_TABLE policy),
so they keep their own parity cases here, the streaming lookup-table kernel at two batch
rows included. Bars are those of tests/test_gemv_gpu.py.
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

from test_gemv_gpu import check, run, sample_rows, to_dev_x  # noqa: E402


@pytest.fixture
def policy():
    """Set a path policy for one test and restore the default afterwards."""
    def set_(p):
        bw.bisco_set_path_policy(p)
    yield set_
    bw.bisco_set_path_policy(bw.BISCO_PATH_AUTO)


def kinds(L, M, xdt="bf16"):
    dl = bw.DeviceLayer(L)
    ws = bw.bisco_workspace_size(dl, M)
    return bw.bisco_plan_kernels(dl, M, bw.BISCO_BF16 if xdt == "bf16" else bw.BISCO_F32, ws)


def test_kernel_choice(policy):
    L, _ = build(2, 0, 1)
    assert kinds(L, 1) == [bw.BISCO_KERNEL_LUT_WARP]
    assert kinds(L, 2) == [bw.BISCO_KERNEL_INTEGER_MMA]
    assert kinds(L, 8) == [bw.BISCO_KERNEL_INTEGER_MMA]
    assert kinds(L, 128) == [bw.BISCO_KERNEL_TENSOR_CORE]
    L4, _ = build(4, 0, 2)  # correction: z and y in one integer launch, single rows too
    for M in (1, 2, 4, 8):
        assert kinds(L4, M) == [bw.BISCO_KERNEL_INTEGER_MMA]
    policy(bw.BISCO_PATH_LOOKUP_TABLE)
    assert kinds(L, 1) == [bw.BISCO_KERNEL_LUT_WARP]
    assert kinds(L, 8) == [bw.BISCO_KERNEL_LUT_ROWS]
    Lg, _ = build(3, 0, 2)
    assert kinds(Lg, 2) == [bw.BISCO_KERNEL_LUT_STREAM]
    policy(bw.BISCO_PATH_SMALL_BATCH_ONLY)
    assert kinds(L, 128) == [bw.BISCO_KERNEL_INTEGER_MMA] * 16


# ---- the streaming lookup-table kernel at two batch rows -----------------------

@pytest.mark.parametrize("cfg,spec", [(3, 0), (5, 4)], ids=["cfg3_gate_up", "cfg5_l0_gate"])
def test_stream_lut_kernel_two_rows_sampled(policy, cfg, spec):
    # FluxBin Sec. 3.2 (VCM salient phase) on the streaming path for cfg3
    policy(bw.BISCO_PATH_LOOKUP_TABLE)
    L, X = build(cfg, spec, 2)
    k = kinds(L, 2)
    assert all(x in (bw.BISCO_KERNEL_LUT_WARP, bw.BISCO_KERNEL_LUT_STREAM) for x in k)
    if cfg == 3:  # many row tiles per cluster and no correction: the streaming kernel
        assert k == [bw.BISCO_KERNEL_LUT_STREAM]
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 200, 41 + spec)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


@pytest.mark.parametrize("rank", [0, 40])
def test_lookup_table_kernels_ragged_two_rows(policy, rank):
    # 11009 x 4100: ragged last row tile and last column quad, salient columns, with and
    # without a correction (rank 40: pass Y has a U^T segment of one quad); whichever
    # lookup-table kernel the planner picks for the shape
    policy(bw.BISCO_PATH_LOOKUP_TABLE)
    M, out, in_ = 2, 11009, 4100
    X = make_activations(0, (811, rank), M, in_, "bf16")
    L = make_layer(0, (811, rank), out, in_, 2, "bf16", rank=rank, sal_frac=0.01, x_for_salience=X, x_dtype="bf16")
    k = kinds(L, M)
    assert all(x in (bw.BISCO_KERNEL_LUT_WARP, bw.BISCO_KERNEL_LUT_STREAM) for x in k)
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(out, 200, 7)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


# ---- lookup-table fallback on small and ragged shapes --------------------------

LUT_RAGGED = [
    # out, in, K, scale_dtype, rank, sal_frac, M, x_dtype
    (33, 129, 2, "bf16", 0, 0.0, 1, "bf16"),
    (100, 1000, 3, "f32", 17, 0.02, 5, "f32"),
    (257, 640, 4, "bf16", 40, 0.01, 2, "bf16"),
    (1024, 1024, 2, "bf16", 64, 0.01, 8, "bf16"),
]


@pytest.mark.parametrize("case", LUT_RAGGED, ids=[f"{c[0]}x{c[1]}K{c[2]}R{c[4]}M{c[6]}" for c in LUT_RAGGED])
def test_lookup_table_kernels_elementwise(policy, case):
    policy(bw.BISCO_PATH_LOOKUP_TABLE)
    out, in_, K, sdt, rank, sal, M, xdt = case
    key = (91, out, in_, K, rank, M)
    X = make_activations(0, key, M, in_, xdt)
    L = make_layer(0, key, out, in_, K, sdt, rank=rank, sal_frac=sal, x_for_salience=X if sal else None,
                   x_dtype=xdt)
    assert bw.BISCO_KERNEL_INTEGER_MMA not in kinds(L, M, xdt)
    check(run(L, X, xdt, "f32"), oracle.gemv(L, X, xdt), X, xdt, "f32")


# ---- integer kernel on single batch rows (BISCO_PATH_INTEGER_MMA) ---------------

INT_ONE_ROW = [
    # out, in, K, scale_dtype, rank, sal_frac, x_dtype
    (1, 1, 1, "f32", 0, 0.0, "f32"),
    (33, 129, 2, "bf16", 0, 0.0, "bf16"),
    (96, 385, 1, "bf16", 129, 0.0, "bf16"),
    (300, 333, 0, "bf16", 5, 0.0, "bf16"),
    (64, 256, 0, "bf16", 0, 0.05, "bf16"),
    (1024, 1024, 2, "bf16", 64, 0.01, "bf16"),
]


@pytest.mark.parametrize("case", INT_ONE_ROW, ids=[f"{c[0]}x{c[1]}K{c[2]}R{c[4]}" for c in INT_ONE_ROW])
def test_integer_kernel_one_row_elementwise(policy, case):
    policy(bw.BISCO_PATH_INTEGER_MMA)
    out, in_, K, sdt, rank, sal, xdt = case
    key = (93, out, in_, K, rank)
    X = make_activations(0, key, 1, in_, xdt)
    L = make_layer(0, key, out, in_, K, sdt, rank=rank, sal_frac=sal, x_for_salience=X if sal else None, x_dtype=xdt)
    assert set(kinds(L, 1, xdt)) == {bw.BISCO_KERNEL_INTEGER_MMA}
    for ydt in ("f32", "bf16"):
        check(run(L, X, xdt, ydt), oracle.gemv(L, X, xdt), X, xdt, ydt)


@pytest.mark.parametrize("cfg,spec", [(2, 0), (3, 0), (3, 1), (4, 0)], ids=["cfg2", "cfg3_gate_up", "cfg3_down", "cfg4"])
def test_integer_kernel_one_row_workloads_sampled(policy, cfg, spec):
    policy(bw.BISCO_PATH_INTEGER_MMA)
    L, X = build(cfg, spec, 1)
    assert set(kinds(L, 1)) == {bw.BISCO_KERNEL_INTEGER_MMA}
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 192, 3 + spec)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


# ---- integer kernel: activation magnitudes and batch sizes ----------------------

@pytest.mark.parametrize("scale_exp", [-100, -20, 0, 20, 100])
def test_integer_kernel_keeps_relative_precision_at_any_magnitude(scale_exp):
    # the activations enter in fixed point relative to their largest magnitude, so the
    # relative error must not depend on the overall scale (fp32 activations)
    M, out, in_ = 3, 200, 700
    X = make_activations(0, (820,), M, in_, "f32") * np.float32(2.0 ** scale_exp)
    L = make_layer(0, (820,), out, in_, 2, "f32", rank=24)
    assert kinds(L, M, "f32") == [bw.BISCO_KERNEL_INTEGER_MMA]
    check(run(L, X, "f32", "f32"), oracle.gemv(L, X, "f32"), X, "f32", "f32")


def test_integer_kernel_zero_activations_give_zero():
    L = make_layer(0, (821,), 300, 500, 2, "bf16", rank=8)
    X = np.zeros((2, 500), np.uint16)  # bf16 +0.0
    assert np.all(run(L, X, "bf16", "f32") == 0.0)


def test_integer_kernel_single_outlier_column():
    # one column 2^12 times larger than the rest: the fixed-point scale follows it, the
    # small columns keep 22 - 12 = 10 bits below it at least (error bounded by the bar)
    M, out, in_ = 2, 256, 1024
    X = make_activations(0, (822,), M, in_, "f32")
    X[0, 517] *= np.float32(4096.0)
    L = make_layer(0, (822,), out, in_, 2, "f32")
    check(run(L, X, "f32", "f32"), oracle.gemv(L, X, "f32"), X, "f32", "f32")


@pytest.mark.parametrize("M", [3, 5, 6, 7])
def test_integer_kernel_batch_sizes_between_the_blocks(M):
    # batch chunks padded to 4 or 8 rows: the unused slots must contribute nothing
    X = make_activations(0, (823, M), M, 640, "bf16")
    L = make_layer(0, (823, M), 333, 640, 2, "bf16", rank=33, sal_frac=0.01, x_for_salience=X, x_dtype="bf16")
    check(run(L, X, "bf16", "f32"), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


# ---- bounded waits: a copy that never starts ------------------------------------

def test_integer_kernel_wait_gives_up_and_reports_timeout():
    # the test hook leaves one row tile's sign-word copies unissued; the warps that
    # wait for it give up after 1 ms and record BISCO_ERR_TIMEOUT, no copy is in flight
    # into that tile when they do, and the next call after bisco_workspace_init is
    # correct again
    L, X = build(2, 0, 2)
    dl = bw.DeviceLayer(L)
    assert kinds(L, 2) == [bw.BISCO_KERNEL_INTEGER_MMA]
    ws = bw.alloc_workspace([dl], 2)
    Xd = to_dev_x(X, "bf16")
    Yd = torch.empty((2, L.out), dtype=torch.float32, device="cuda")
    try:
        bw.bisco_debug_set_wait_test(0, 1_000_000)
        bw.bisco_gemv(dl, Xd, Yd, ws)
        assert bw.bisco_sync_status(ws) == bw.BISCO_ERR_TIMEOUT
    finally:
        bw.bisco_debug_set_wait_test(-1, 0)
    bw.bisco_workspace_init(ws)
    bw.bisco_gemv(dl, Xd, Yd, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    Y = Yd.cpu().numpy().astype(np.float64)
    check(Y, oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


def test_eight_rows_without_an_integer_plan_take_the_tensor_cores():
    # the decoder's down projection (4096 x 11008, rank 256) at 8 batch rows: the integer
    # plan does not fit shared memory, so the chunk runs on the tcgen05 kernel (z, then y)
    L, X = build(5, 6, 8)
    assert kinds(L, 8) == [bw.BISCO_KERNEL_TENSOR_CORE] * 2
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 128, 70)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


# ---- the correction in one launch: z handed over inside the grid ------------------

@pytest.mark.parametrize("out,in_,K,rank", [(200, 128, 1, 512), (64, 4096, 2, 64), (4100, 300, 2, 1000),
                                            (96, 256, 0, 40), (1000, 1000, 3, 7)],
                         ids=["rank_heavy", "wide", "ragged", "correction_only", "rank7"])
@pytest.mark.parametrize("M", [1, 2, 8])
def test_fused_correction_launch(policy, out, in_, K, rank, M):
    # z = alpha (.) (V x) computed by the first clusters of the grid and read by the U^T
    # units of the others; shapes where a CTA holds only U^T units, only base units, or
    # both, and ragged row and column counts
    policy(bw.BISCO_PATH_INTEGER_MMA)
    X = make_activations(0, (824, out, M), M, in_, "bf16")
    L = make_layer(0, (824, out, in_, K), out, in_, K, "bf16", rank=rank, sal_frac=0.01, x_for_salience=X,
                   x_dtype="bf16")
    assert kinds(L, M) == [bw.BISCO_KERNEL_INTEGER_MMA]
    check(run(L, X, "bf16", "f32"), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


def test_fused_correction_repeated_calls_are_identical():
    # the hand-over counters return to zero at the end of every launch: back-to-back
    # calls on one workspace, without re-initialising it, give bit-identical results
    L, X = build(4, 0, 4)
    dl = bw.DeviceLayer(L)
    assert kinds(L, 4) == [bw.BISCO_KERNEL_INTEGER_MMA]
    ws = bw.alloc_workspace([dl], 4)
    Xd = to_dev_x(X, "bf16")
    outs = []
    for _ in range(4):
        Yd = torch.empty((4, L.out), dtype=torch.float32, device="cuda")
        bw.bisco_gemv(dl, Xd, Yd, ws)
        outs.append(Yd)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    # the two hand-over counters: 32-bit words 32 and 33 of the status region
    assert int(ws[128:136].to(torch.int32).sum()) == 0
    for Yd in outs[1:]:
        assert torch.equal(Yd, outs[0])
    rows = sample_rows(L.out, 128, 5)
    check(outs[0].cpu().numpy().astype(np.float64)[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


def test_fused_correction_wait_gives_up_and_reports_timeout():
    # with one tile's copies unissued in every CTA, the z producers give up on their
    # tile and the output CTAs on z; both record BISCO_ERR_TIMEOUT, the counters are
    # still returned to zero, and the next call after bisco_workspace_init is correct
    L, X = build(4, 0, 2)
    dl = bw.DeviceLayer(L)
    assert kinds(L, 2) == [bw.BISCO_KERNEL_INTEGER_MMA]
    ws = bw.alloc_workspace([dl], 2)
    Xd = to_dev_x(X, "bf16")
    Yd = torch.empty((2, L.out), dtype=torch.float32, device="cuda")
    try:
        bw.bisco_debug_set_wait_test(0, 1_000_000)
        bw.bisco_gemv(dl, Xd, Yd, ws)
        assert bw.bisco_sync_status(ws) == bw.BISCO_ERR_TIMEOUT
    finally:
        bw.bisco_debug_set_wait_test(-1, 0)
    bw.bisco_workspace_init(ws)
    bw.bisco_gemv(dl, Xd, Yd, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    rows = sample_rows(L.out, 128, 6)
    check(Yd.cpu().numpy().astype(np.float64)[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


def test_tensor_core_kernel_wait_gives_up_and_reports_timeout():
    # the tcgen05 kernel: the last step's sign-word copy of every CTA is never issued;
    # the producers' bounded wait gives up after 1 ms, the kernel still reaches its
    # tensor-memory release (the next launch allocates all 512 columns again), the status
    # word reads BISCO_ERR_TIMEOUT, and after bisco_workspace_init the next call is correct
    L, X = build(2, 0, 64)
    dl = bw.DeviceLayer(L)
    assert kinds(L, 64) == [bw.BISCO_KERNEL_TENSOR_CORE]
    ws = bw.alloc_workspace([dl], 64)
    Xd = to_dev_x(X, "bf16")
    Yd = torch.empty((64, L.out), dtype=torch.float32, device="cuda")
    try:
        bw.bisco_debug_set_wait_test(0, 1_000_000)
        bw.bisco_gemv(dl, Xd, Yd, ws)
        assert bw.bisco_sync_status(ws) == bw.BISCO_ERR_TIMEOUT
    finally:
        bw.bisco_debug_set_wait_test(-1, 0)
    bw.bisco_workspace_init(ws)
    bw.bisco_gemv(dl, Xd, Yd, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    rows = sample_rows(L.out, 128, 5)
    Y = Yd.cpu().numpy().astype(np.float64)[:, rows]
    check(Y, oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")

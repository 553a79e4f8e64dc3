"""GPU parity: bisco_gemv (through the C ABI) against the fp64 oracle.

Bars:
  * fp32 output: relative L2 error <= 2e-3 and max abs error <= 1e-2 * ||X||_inf
    (the stated tolerance for bf16 inputs with fp32 accumulation), and relative
    L2 error <= 1e-4, a bound derived from fp32 accumulation (about u * sqrt(N)
    relative for N sign terms of random sign, u = 2^-24, N <= 2 * 11008), kept
    25x under the stated one so that a dropped or mis-scaled small term cannot
    hide inside it;
  * bf16 output: the same max-abs bound, each element within half a bf16 ulp
    (2^-8 relative) of the fp64 value plus the fp32 bar, and relative L2 error
    <= 2^-8 + 1e-4: rounding to nearest even with 8 significant bits moves each
    element by at most 2^-8 of its value (about 1.1e-3 relative RMS on typical
    data, but up to 2^-8 when values sit just above powers of two), so the stated
    2e-3 is a bar for fp32 outputs and the rounding bound is the bar for bf16 ones.
Full-size workloads compare sampled output rows that the oracle computes one
by one; small and ragged shapes compare every element.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only hosts, run only with a GPU
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import binary_weight_decode_b200 as bw  # noqa: E402
import oracle  # noqa: E402
from synth import make_activations, make_layer  # noqa: E402
from synth.configs import build  # noqa: E402

DEV = "cuda"


def to_dev_x(X, x_dtype):
    if x_dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).to(DEV)


def run(L, X, x_dtype, y_dtype="f32", ws=None, dl=None):
    dl = dl or bw.DeviceLayer(L)
    M = X.shape[0]
    Xd = to_dev_x(X, x_dtype)
    Yd = torch.empty((M, L.out), dtype=torch.float32 if y_dtype == "f32" else torch.bfloat16, device=DEV)
    ws = ws if ws is not None else bw.alloc_workspace([dl], M)
    bw.bisco_gemv(dl, Xd, Yd, ws)
    st = bw.bisco_sync_status(ws)
    assert st == bw.BISCO_OK, bw.bisco_status_string(st)
    return Yd.float().cpu().numpy().astype(np.float64)


def x_inf(X, x_dtype):
    return float(np.max(np.abs(oracle.decode_values(X, x_dtype))))


def check(Y, Yref, X, x_dtype, y_dtype):
    d = Y - Yref
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(Yref), 1e-300))
    mx = float(np.max(np.abs(d))) if d.size else 0.0
    assert mx <= 1e-2 * x_inf(X, x_dtype), f"max-abs {mx:.3e}"
    if y_dtype == "f32":
        assert rel <= 2e-3, f"rel-L2 {rel:.3e}"
        assert rel <= 1e-4, f"rel-L2 {rel:.3e} above the fp32-accumulation bound"
    else:
        slack = 1e-4 * float(np.max(np.abs(Yref))) if Yref.size else 0.0
        bad = np.abs(d) > 2.0 ** -8 * np.abs(Yref) + slack
        assert not np.any(bad), f"{int(bad.sum())} elements beyond half a bf16 ulp"
        assert rel <= 2.0 ** -8 + 1e-4, f"rel-L2 {rel:.3e}"
    return rel


def sample_rows(out, n, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(out, size=min(n, out), replace=False).tolist())
    rows |= {0, out - 1, min(31, out - 1), min(32, out - 1)}
    return np.array(sorted(rows))


# ---- small and ragged shapes: every element ----------------------------------

RAGGED = [
    # out, in, K, scale_dtype, rank, sal_frac, M, x_dtype
    (1, 1, 1, "f32", 0, 0.0, 1, "f32"),
    (5, 7, 1, "f32", 0, 0.0, 1, "f32"),
    (33, 129, 2, "bf16", 0, 0.0, 1, "bf16"),
    (31, 127, 2, "bf16", 3, 0.0, 3, "bf16"),
    (100, 1000, 3, "f32", 17, 0.02, 5, "f32"),
    (257, 640, 4, "bf16", 40, 0.01, 9, "bf16"),
    (300, 333, 0, "bf16", 5, 0.0, 2, "bf16"),      # correction only
    (64, 256, 0, "bf16", 0, 0.05, 4, "bf16"),       # salient only
    (96, 385, 1, "bf16", 129, 0.0, 1, "bf16"),      # rank just above a quad
    (40, 200, 2, "f32", 1, 0.0, 17, "f32"),         # M above one batch chunk
    (1024, 1024, 2, "bf16", 64, 0.01, 8, "bf16"),
]


@pytest.mark.parametrize("case", RAGGED, ids=[f"{c[0]}x{c[1]}K{c[2]}R{c[4]}M{c[6]}" for c in RAGGED])
@pytest.mark.parametrize("y_dtype", ["f32", "bf16"])
def test_ragged_shapes_elementwise(case, y_dtype):
    out, in_, K, sdt, rank, sal, M, xdt = case
    key = (77, out, in_, K, rank, M)
    X = make_activations(0, key, M, in_, xdt)
    L = make_layer(0, key, out, in_, K, sdt, rank=rank, sal_frac=sal, x_for_salience=X if sal else None,
                   x_dtype=xdt)
    Y = run(L, X, xdt, y_dtype)
    Yref = oracle.gemv(L, X, xdt)
    check(Y, Yref, X, xdt, y_dtype)


def test_empty_layer_gives_zero():
    X = make_activations(0, (5,), 2, 50, "f32")
    L = make_layer(0, (5,), 10, 50, 0, "f32")
    Y = run(L, X, "f32")
    assert np.all(Y == 0)


def test_batch_zero_is_a_no_op():
    L = make_layer(0, (6,), 64, 128, 1, "f32")
    dl = bw.DeviceLayer(L)
    ws = bw.alloc_workspace([dl], 1)
    Xd = torch.zeros((0, 128), device=DEV)
    Yd = torch.full((1, 64), 7.0, device=DEV)
    st = bw._lib.bisco_gemv(bw.ctypes.byref(dl.desc), bw.ctypes.c_void_p(Xd.data_ptr() or 16), 0, 0,
                            bw.ctypes.c_void_p(Yd.data_ptr()), 0, bw.ctypes.c_void_p(ws.data_ptr()),
                            ws.numel(), None)
    torch.cuda.synchronize()
    assert st == bw.BISCO_OK and torch.all(Yd == 7.0)


# ---- the five workloads ---------------------------------------------------------

def test_cfg1_small_layer_with_correction_elementwise():
    L, X = build(1, 0, 1)
    for ydt in ("f32", "bf16"):
        check(run(L, X, "f32", ydt), oracle.gemv(L, X, "f32"), X, "f32", ydt)


def test_cfg2_attention_projection_elementwise():
    L, X = build(2, 0, 1)
    Y = run(L, X, "bf16", "f32")
    check(Y, oracle.gemv(L, X, "bf16"), X, "bf16", "f32")
    Yb = run(L, X, "bf16", "bf16")
    check(Yb, oracle.gemv(L, X, "bf16"), X, "bf16", "bf16")


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("spec", [0, 1], ids=["gate_up", "down"])
def test_cfg3_mlp_salient_sampled_rows(spec, M):
    L, X = build(3, spec, M)
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 192, 31 * M + spec)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_cfg4_correction_outliers_sampled_rows(M):
    L, X = build(4, 0, M)
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 192, 7 * M)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


@pytest.mark.parametrize("M", [1, 8, 32])
@pytest.mark.parametrize("spec", [0, 4, 6, 222], ids=["l0_q", "l0_gate", "l0_down", "l31_up"])
def test_cfg5_decoder_matrices_sampled_rows(spec, M):
    L, X = build(5, spec, M)
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(L.out, 96, spec + M)
    check(Y[:, rows], oracle.gemv_rows(L, X, "bf16", rows), X, "bf16", "f32")


# ---- determinism, workspace reuse, errors -------------------------------------

def test_repeat_calls_are_bit_identical():
    L, X = build(4, 0, 2)
    dl = bw.DeviceLayer(L)
    ws = bw.alloc_workspace([dl], 2)
    a = run(L, X, "bf16", "f32", ws=ws, dl=dl)
    b = run(L, X, "bf16", "f32", ws=ws, dl=dl)
    c = run(L, X, "bf16", "f32", ws=ws, dl=dl)
    assert np.array_equal(a, b) and np.array_equal(b, c)


def test_workspace_too_small_is_rejected_and_output_untouched():
    L, X = build(1, 0, 1)
    dl = bw.DeviceLayer(L)
    need = bw.bisco_workspace_size(dl, 1)
    ws = torch.zeros(need - 256, dtype=torch.uint8, device=DEV)
    Xd = to_dev_x(X, "f32")
    Yd = torch.full((1, L.out), 3.0, device=DEV)
    with pytest.raises(bw.BiscoError) as e:
        bw.bisco_gemv(dl, Xd, Yd, ws)
    assert e.value.status == bw.BISCO_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(Yd == 3.0)


def test_out_of_range_salient_index_is_reported_not_read():
    X = make_activations(0, (8,), 1, 256, "bf16")
    L = make_layer(0, (8,), 64, 256, 1, "bf16", sal_frac=0.02, x_for_salience=X, x_dtype="bf16")
    L.sal_idx = L.sal_idx.copy()
    L.sal_idx[-1] = 1 << 30
    dl = bw.DeviceLayer(L)
    ws = bw.alloc_workspace([dl], 1)
    Yd = torch.empty((1, 64), device=DEV)
    bw.bisco_gemv(dl, to_dev_x(X, "bf16"), Yd, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_ERR_INVALID_ARG
    bw.bisco_workspace_init(ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK


def test_packed_with_bisco_pack_matches_oracle():
    rng = np.random.default_rng(11)
    out, in_ = 70, 300
    S = rng.choice(np.array([-1, 1], np.int8), size=(out, in_))
    L = make_layer(0, (12,), out, in_, 1, "f32")
    L.bits = bw.bisco_pack(S)[None, :]
    X = make_activations(0, (12,), 2, in_, "f32")
    Y = run(L, X, "f32")
    check(Y, oracle.gemv(L, X, "f32"), X, "f32", "f32")


def test_graph_bench_matches_direct_call():
    L, X = build(2, 0, 1)
    dl = bw.DeviceLayer(L)
    ws = bw.alloc_workspace([dl], 1)
    Xd = to_dev_x(X, "bf16")
    Yg = torch.empty((2, 1, L.out), device=DEV)
    r = bw.bisco_bench([dl, dl], Xd, Yg, ws, warmup=2, reps=3)
    assert r["us_per_gemv"] > 0 and r["kernels_per_gemv"] == 1
    Y = run(L, X, "bf16", "f32", ws=ws, dl=dl)
    assert np.array_equal(Yg[0].cpu().numpy().astype(np.float64), Y)
    assert np.array_equal(Yg[1].cpu().numpy().astype(np.float64), Y)


# ---- row shards: each shard's product is the full product's column slice -----

@pytest.mark.parametrize("world,M", [(3, 1), (2, 40)])
def test_row_shards_on_the_device(world, M):
    # every shard runs through bisco_gemv on the same GPU, one after another (no collective):
    # their outputs side by side must meet the bar against the whole layer's oracle product
    from binary_weight_decode_b200 import shard
    X = make_activations(0, (640, M), M, 300, "bf16")
    L = make_layer(0, (640, M), 200, 300, 2, "bf16", rank=24, sal_frac=0.02, x_for_salience=X, x_dtype="bf16")
    parts = [run(shard.shard_rows(L, r, world), X, "bf16") for r in range(world)]
    check(np.concatenate(parts, axis=1), oracle.gemv(L, X, "bf16"), X, "bf16", "f32")

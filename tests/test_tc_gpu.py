"""GPU parity of the tensor-core path (batch chunks of 16..128 rows) against the oracle.

bisco_gemv sends a batch chunk of at least 16 rows to the tensor cores when the layer's
scales are bf16: the signs are expanded to bf16 tiles (column scale folded in, exact),
fp32-valued inputs (the correction's z, salient inputs, fp32 activations) are split into
high and low bf16 parts, and the products accumulate in fp32. The bars are those of
tests/test_gemv_gpu.py. Batch sizes straddle the chunk boundaries (16, 128) so that
mixed schedules (tensor-core chunks followed by lookup-table chunks) are covered too.
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
from test_gemv_gpu import check, run, sample_rows  # noqa: E402

CASES = [
    # out, in, K, rank, sal_frac, M, x dtype, y dtype
    (256, 512, 2, 0, 0.0, 32, "bf16", "f32"),
    (200, 300, 1, 0, 0.0, 37, "bf16", "f32"),      # ragged rows, columns, batch
    (300, 700, 2, 24, 0.02, 33, "bf16", "f32"),     # correction + salient
    (640, 1000, 1, 96, 0.01, 64, "bf16", "bf16"),
    (512, 1024, 2, 0, 0.0, 128, "bf16", "f32"),
    # three bases + correction at 128 rows: four accumulator blocks of 128 columns leave too
    # little tensor memory for the sign stages, so the call runs on lookup-table chunks
    (384, 640, 3, 40, 0.0, 130, "bf16", "f32"),
    (160, 384, 2, 8, 0.03, 150, "bf16", "f32"),     # 128 + 22 (lookup-table chunks of 8, 8, 6)
    (257, 129, 4, 0, 0.0, 40, "bf16", "f32"),       # four bases
    (192, 512, 2, 17, 0.0, 48, "f32", "f32"),       # fp32 activations: split on the bases
    (128, 256, 0, 64, 0.05, 32, "bf16", "f32"),     # correction + salient, no base
    (96, 200, 0, 0, 0.1, 40, "bf16", "f32"),        # salient only
    (256, 512, 2, 0, 0.0, 16, "bf16", "f32"),       # the smallest tensor-core chunk
    (300, 700, 2, 24, 0.02, 17, "bf16", "f32"),     # 17 rows: one chunk padded to 32 columns
    (333, 1000, 2, 40, 0.0, 24, "bf16", "bf16"),
    (130, 4100, 1, 0, 0.01, 31, "bf16", "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(str(v) for v in c))
def test_tensor_core_chunks_match_oracle(case):
    out, in_, K, rank, sal, M, xdt, ydt = case
    seed_key = (700, out, in_, M)
    X = make_activations(0, seed_key, M, in_, xdt)
    L = make_layer(0, seed_key, out, in_, K, "bf16", rank=rank, sal_frac=sal,
                   x_for_salience=X if sal else None, x_dtype=xdt)
    Y = run(L, X, xdt, ydt)
    check(Y, oracle.gemv(L, X, xdt), X, xdt, ydt)


def test_fp32_scales_stay_exact():
    # fp32 scales cannot be folded into bf16 tiles exactly: such layers keep the
    # lookup-table path at any batch size and must still meet the fp32 bar.
    M, out, in_ = 24, 160, 256
    X = make_activations(0, (710,), M, in_, "bf16")
    L = make_layer(0, (710,), out, in_, 2, "f32", rank=8)
    Y = run(L, X, "bf16", "f32")
    check(Y, oracle.gemv(L, X, "bf16"), X, "bf16", "f32")


def test_llama_gate_layer_batch_128_sampled_rows():
    # 11008 x 4096, two bases and a rank-256 correction at batch 128 (two chunks on the
    # tensor cores); rows sampled and computed one by one by the oracle.
    M, out, in_ = 128, 11008, 4096
    X = make_activations(0, (720,), M, in_, "bf16")
    L = make_layer(0, (720,), out, in_, 2, "bf16", rank=256)
    Y = run(L, X, "bf16", "f32")
    rows = sample_rows(out, 96, 721)
    ref = oracle.gemv_rows(L, X, "bf16", rows)
    check(Y[:, rows], ref, X, "bf16", "f32")


def test_small_workspace_falls_back_to_lookup_chunks():
    # With only the minimum workspace (z for 8 batch rows) a rank-64 layer at batch 40
    # cannot hold a tensor-core chunk's z: the call must still be correct.
    M, out, in_, rank = 40, 128, 256, 64
    X = make_activations(0, (730,), M, in_, "bf16")
    L = make_layer(0, (730,), out, in_, 1, "bf16", rank=rank)
    dl = bw.DeviceLayer(L)
    ws = torch.zeros(256 + ((8 * rank * 4 + 255) // 256) * 256, dtype=torch.uint8, device="cuda")
    Y = run(L, X, "bf16", "f32", ws=ws, dl=dl)
    check(Y, oracle.gemv(L, X, "bf16"), X, "bf16", "f32")

"""bisco_gemv_noalloc: the entry point for callers that cannot allocate device memory.

Such callers (a plug-in whose host application owns every device allocation and
passes it only its operands, or a runtime that reserves all device memory at start-up)
cannot hand bisco_gemv a workspace. bisco_gemv_noalloc uses a fixed
scratch array inside the library instead. This file checks, through the C ABI, that
two calls in a row give what bisco_gemv gives with a caller-provided workspace, and
that a rank above the array's limit is refused without touching the output.

Kept in its own file, named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import binary_weight_decode_b200 as bw  # noqa: E402
from synth import make_activations, make_layer  # noqa: E402


def _x(X):
    return torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda().view(torch.bfloat16)


def _with_workspace(dl, Xd, M, out):
    ws = bw.alloc_workspace([dl], M)
    Y = torch.empty((M, out), dtype=torch.float32, device="cuda")
    bw.bisco_gemv(dl, Xd, Y, ws)
    assert bw.bisco_sync_status(ws) == bw.BISCO_OK
    return Y


def _no_alloc(dl, Xd, M, out):
    Y = torch.full((M, out), float("nan"), dtype=torch.float32, device="cuda")
    st = bw._lib.bisco_gemv_noalloc(ctypes.byref(dl.desc), ctypes.c_void_p(Xd.data_ptr()), bw.BISCO_BF16, M,
                                    ctypes.c_void_p(Y.data_ptr()), bw.BISCO_F32,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bw.BISCO_OK, bw.bisco_status_string(st)
    torch.cuda.synchronize()
    return Y


def _rel_l2(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_two_calls_in_a_row_match_the_workspace_entry_point():
    # call 1: a layer whose correction needs the scratch z; call 2: another layer and
    # batch size (two batch chunks), so state left in the shared array by call 1 must not leak
    # (a third call at batch 64 runs on the tensor cores, z of 64 rows in the scratch array)
    cases = [(640, 1000, 2, 96, 0.01, 3), (300, 520, 1, 40, 0.0, 11), (256, 512, 2, 64, 0.02, 64)]
    for i, (out, in_, K, rank, sal, M) in enumerate(cases):
        X = make_activations(0, (500 + i,), M, in_, "bf16")
        L = make_layer(0, (500 + i,), out, in_, K, "bf16", rank=rank, sal_frac=sal,
                       x_for_salience=X if sal else None, x_dtype="bf16")
        dl = bw.DeviceLayer(L)
        Xd = _x(X)
        ref = _with_workspace(dl, Xd, M, out)
        got = _no_alloc(dl, Xd, M, out)
        assert torch.isfinite(got).all()
        assert _rel_l2(got, ref) <= 1e-4


def test_rank_above_the_scratch_limit_is_refused():
    M, out, in_ = 1, 64, 128
    X = make_activations(0, (510,), M, in_, "bf16")
    L = make_layer(0, (510,), out, in_, 1, "bf16", rank=8)
    dl = bw.DeviceLayer(L)
    dl.desc.rank = 4097  # over BISCO_NOALLOC_MAX_RANK; rejected before any launch
    Xd = _x(X)
    Y = torch.full((M, out), 5.0, device="cuda")
    st = bw._lib.bisco_gemv_noalloc(ctypes.byref(dl.desc), ctypes.c_void_p(Xd.data_ptr()), bw.BISCO_BF16, M,
                                    ctypes.c_void_p(Y.data_ptr()), bw.BISCO_F32, None)
    torch.cuda.synchronize()
    assert st == bw.BISCO_ERR_UNSUPPORTED
    assert torch.all(Y == 5.0)

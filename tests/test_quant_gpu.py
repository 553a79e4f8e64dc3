"""GPU parity of the offline quantisers against the oracle.

* FluxBin joint sign search ("FluxBin", Sec. 3.1): the packed sign words of every base are
  compared bit for bit with the oracle's exhaustive search packed by the oracle's own packer.
* BiLoCo decomposition ("BiLoCo", "Finding the sign vectors"): the sign vectors must match
  exactly (both sides decide signs from fp64 sums), the coefficients to 1e-9 relative; the
  page's 3x2 walk-through is reproduced through the device path.
"""

import json
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import binary_weight_decode_b200 as bw  # noqa: E402
import oracle  # noqa: E402
from synth import make_activations  # noqa: E402
from synth.gen import Layer  # noqa: E402

from test_gemv_gpu import check, run  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def dev(a, dtype=torch.float64):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype)


@pytest.mark.parametrize("rows,cols", [(37, 300), (64, 128), (100, 1000)])
@pytest.mark.parametrize("Kb", [1, 2, 3, 4])
@pytest.mark.parametrize("group", [0, 64, 128])
def test_fluxbin_signs_bit_exact(rows, cols, Kb, group):
    rng = np.random.default_rng(1000 * rows + 10 * Kb + group)
    W = rng.standard_normal((rows, cols))
    ng = -(-cols // group) if group else 1
    r = np.abs(rng.standard_normal((Kb, rows, ng) if group else (Kb, rows))) * 0.7 + 0.01
    c = np.abs(rng.standard_normal((Kb, cols))) * 0.7 + 0.01
    want = oracle.fluxbin_sign_search(W, r, c, group)
    r_dev = dev(r.transpose(0, 2, 1) if group else r)  # device layout [Kb][groups][rows]
    bits = bw.bisco_fluxbin_signs(dev(W), r_dev, dev(c), group).cpu().numpy().view(np.uint32)
    for k in range(Kb):
        assert np.array_equal(bits[k], oracle.pack_bit_matrix(want[k]).reshape(-1))


def test_fluxbin_signs_feed_the_gemv():
    # quantise a dense matrix with the device sign search, then run the packed result
    # through bisco_gemv: the product is the oracle's product of the same format
    rng = np.random.default_rng(7)
    out, in_, K, g = 96, 384, 2, 128
    W = rng.standard_normal((out, in_)) * 0.05
    r = np.abs(rng.standard_normal((K, out, in_ // g))) * 0.03 + 0.005
    c = np.abs(rng.standard_normal((K, in_))) * 0.5 + 0.5
    bits = bw.bisco_fluxbin_signs(dev(W), dev(r.transpose(0, 2, 1)), dev(c), g).cpu().numpy().view(np.uint32)
    L = Layer(out=out, in_=in_, K=K, scale_dtype="f32", bits=bits.copy(), row_scale=r.astype(np.float32),
              col_scale=c.astype(np.float32), group=g)
    X = make_activations(0, (840,), 2, in_, "f32")
    check(run(L, X, "f32", "f32"), oracle.gemv(L, X, "f32"), X, "f32", "f32")


@pytest.mark.parametrize("rows,cols,rank,rounds", [(48, 80, 1, 5), (48, 80, 8, 5), (130, 70, 4, 1), (33, 257, 6, 3)])
def test_biloco_matches_the_oracle(rows, cols, rank, rounds):
    rng = np.random.default_rng(rows * cols + rank)
    W = rng.standard_normal((rows, cols))
    v0 = rng.choice([-1, 1], size=(rank, cols)).astype(np.int8)
    U, V, g, a = bw.bisco_biloco_decompose(dev(W), torch.from_numpy(v0).cuda(), rounds)
    Uo, Vo, go, ao = oracle.biloco_decompose(W, v0.astype(np.float64), rounds)
    assert np.array_equal(U.cpu().numpy(), Uo.astype(np.int8))
    assert np.array_equal(V.cpu().numpy(), Vo.astype(np.int8))
    assert np.allclose(g.cpu().numpy(), go, rtol=1e-9, atol=0)
    assert np.allclose(a.cpu().numpy(), ao, rtol=1e-9, atol=1e-12)


def test_biloco_reproduces_the_page_toy_on_the_device():
    # the 3x2 walk-through: both components start from v = (+, +); greedy alphas 2 and 4/3,
    # the refit rebuilds W exactly
    g = json.load(open(os.path.join(GOLDEN, "toy_decomposition.json")))
    W = np.array(g["W"], dtype=np.float64)
    v0 = np.ones((2, 2), dtype=np.int8)
    U, V, ga, ra = bw.bisco_biloco_decompose(dev(W), torch.from_numpy(v0).cuda(), 5)
    U, V, ga, ra = U.cpu().numpy(), V.cpu().numpy(), ga.cpu().numpy(), ra.cpu().numpy()
    for j, comp in enumerate(g["components"]):
        assert np.array_equal(U[:, j], comp["u"]) and np.array_equal(V[j], comp["v"])
    for j in range(2):
        num, den = g["greedy_alpha_rational"][j]
        assert ga[j] == pytest.approx(num / den, rel=1e-15)
    assert np.allclose(ra, g["refit_alpha"], rtol=0, atol=1e-12)
    assert np.allclose((U * ra) @ V, W, rtol=0, atol=1e-12)

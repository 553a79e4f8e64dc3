"""Row sharding of a layer (host partitioning and the all-gather of Y), on CPU.

Each rank's shard must hold exactly the full layer's rows [r0, r1) (bit-exact sign words,
the same scales and salient rows), so that its product is the full product's column slice;
the gather is run as two gloo ranks whose local products come from the oracle.
"""

import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import oracle  # noqa: E402
from binary_weight_decode_b200 import shard  # noqa: E402
from synth import make_activations, make_layer, packed_words  # noqa: E402


@pytest.mark.parametrize("out,world", [(200, 1), (200, 2), (200, 3), (200, 7), (64, 4), (33, 2), (4096, 8)])
def test_bounds_are_whole_tiles_covering_every_row(out, world):
    b = shard.shard_bounds(out, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == out
    for (r0, r1), (s0, _) in zip(b, b[1:]):
        assert r1 == s0 and r0 <= r1
    for r0, r1 in b:
        assert r0 % 32 == 0 and (r1 % 32 == 0 or r1 == out)
    sizes = [(r1 - r0 + 31) // 32 for r0, r1 in b]
    assert max(sizes) - min(sizes) <= 1


def _layer():
    X = make_activations(0, (610,), 3, 300, "bf16")
    L = make_layer(0, (610,), 200, 300, 2, "bf16", rank=24, sal_frac=0.02, x_for_salience=X, x_dtype="bf16")
    return L, X


@pytest.mark.parametrize("world", [1, 2, 3, 7])
def test_shards_hold_the_row_slices_of_the_layer(world):
    L, X = _layer()
    Y = oracle.gemv(L, X, "bf16")
    W = oracle.reconstruct(L)
    for rank, (r0, r1) in enumerate(shard.shard_bounds(L.out, world)):
        S = shard.shard_rows(L, rank, world)
        assert S.out == r1 - r0
        for k in range(L.K):
            assert np.array_equal(oracle.unpack_bit_matrix(S.bits[k], S.out, S.in_),
                                  oracle.unpack_bit_matrix(L.bits[k], L.out, L.in_)[r0:r1])
        assert np.array_equal(oracle.reconstruct(S), W[r0:r1])
        assert np.allclose(oracle.gemv(S, X, "bf16"), Y[:, r0:r1], rtol=1e-12, atol=0)


@pytest.mark.parametrize("world", [2, 3])
def test_grouped_layers_shard_by_rows(world):
    # grouped row scales [K][out][groups] are cut along the rows like everything else
    L = make_layer(0, (611,), 100, 300, 2, "bf16", group=128)
    W = oracle.reconstruct(L)
    for rank, (r0, r1) in enumerate(shard.shard_bounds(L.out, world)):
        S = shard.shard_rows(L, rank, world)
        assert np.array_equal(oracle.reconstruct(S), W[r0:r1])


@pytest.mark.parametrize("world", [2, 3, 5])
def test_refined_layers_shard_by_rows(world):
    # the salient refinement's signs (out x n_ref, tiled) and row scales [Ks][out][groups]
    # are cut along the rows; its indices and column scales are replicated
    L = make_layer(0, (612,), 150, 700, 2, "bf16", rank=8, group=128, refine=(2, 8))
    X = make_activations(0, (612,), 3, 700, "bf16")
    W = oracle.reconstruct(L)
    Y = oracle.gemv(L, X, "bf16")
    for rank, (r0, r1) in enumerate(shard.shard_bounds(L.out, world)):
        S = shard.shard_rows(L, rank, world)
        if S.out == 0:
            continue
        assert np.array_equal(S.ref_idx, L.ref_idx) and np.array_equal(S.ref_col_scale, L.ref_col_scale)
        assert np.asarray(S.ref_bits).reshape(2, -1).shape[1] == packed_words(S.out, len(L.ref_idx))
        assert np.array_equal(oracle.reconstruct(S), W[r0:r1])
        assert np.allclose(oracle.gemv(S, X, "bf16"), Y[:, r0:r1], rtol=1e-12, atol=0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L, X = _layer()
        bounds = shard.shard_bounds(L.out, world)
        y_local = torch.from_numpy(oracle.gemv(shard.shard_rows(L, rank, world), X, "bf16"))
        Y = shard.gather_rows(y_local, bounds, dist)
        out[rank] = float(np.max(np.abs(Y.numpy() - oracle.gemv(L, X, "bf16"))))
    finally:
        dist.destroy_process_group()


def test_gather_rebuilds_the_full_product_on_every_rank():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    assert all(v <= 1e-12 for v in out.values()), dict(out)

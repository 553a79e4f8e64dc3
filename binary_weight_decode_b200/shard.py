"""Row sharding of a layer over several GPUs (host-side partitioning and the gather).

The product Y = X W^T splits by output rows without any exchange inside the GEMV: a rank
holding rows [r0, r1) of every sign matrix B_k, of U^T (the correction's first factor,
stored transposed), of the row scales, of the salient block and of the salient refinement's
signs and row scales computes Y[:, r0:r1] with bisco_gemv on its own GPU; X, the column
scales, V, alpha, the salient indices and the refinement's indices and column scales are
replicated (V x is recomputed on every rank: it is R x in, tiny next to the weights). One
all-gather of the slices rebuilds Y where a consumer needs every row.

Shard boundaries fall on 32-row tiles of the packed sign layout
[tiles][quads][32 rows][4 words], so a shard's sign words are a contiguous range of
whole tiles of the full matrix: slicing is a copy, never a repack.
"""

import dataclasses

import numpy as np

TILE = 32


def shard_bounds(out, world):
    """Row range [r0, r1) of every rank: whole 32-row tiles, split as evenly as possible
    (the first ranks take one tile more); ranks past the last tile get an empty range."""
    if world < 1:
        raise ValueError("world must be >= 1")
    tiles = (out + TILE - 1) // TILE
    bounds = []
    for r in range(world):
        t0, t1 = r * tiles // world, (r + 1) * tiles // world
        bounds.append((min(out, t0 * TILE), min(out, t1 * TILE)))
    return bounds


def _tile_slice(words, rows, cols, t0, t1):
    """Packed words of tiles [t0, t1) of a [rows][cols] sign matrix."""
    tiles = (rows + TILE - 1) // TILE
    quads = (cols + 127) // 128
    w = np.asarray(words, dtype=np.uint32).reshape(tiles, quads * TILE * 4)
    return np.ascontiguousarray(w[t0:t1]).reshape(-1)


def shard_rows(layer, rank, world):
    """The host layer of `rank`'s rows (same dataclass as `layer`, out = r1 - r0)."""
    r0, r1 = shard_bounds(layer.out, world)[rank]
    t0, t1 = r0 // TILE, (r1 + TILE - 1) // TILE
    rows = r1 - r0
    kw = dict(out=rows)
    if layer.K:
        bits = np.asarray(layer.bits).reshape(layer.K, -1)
        kw["bits"] = np.stack([_tile_slice(bits[k], layer.out, layer.in_, t0, t1) for k in range(layer.K)])
        # [K][out] or, with grouped row scales, [K][out][groups]: the rows are axis 1
        rs = np.asarray(layer.row_scale)
        rs = rs.reshape(layer.K, layer.out, -1)[:, r0:r1]
        kw["row_scale"] = np.ascontiguousarray(rs if getattr(layer, "group", 0) else rs[:, :, 0])
    if layer.rank:
        kw["ut_bits"] = _tile_slice(layer.ut_bits, layer.out, layer.rank, t0, t1)
    if layer.n_sal:
        kw["sal_q"] = np.ascontiguousarray(np.asarray(layer.sal_q)[r0:r1])
    ks = getattr(layer, "ref_K", 0) or 0
    if ks:  # salient refinement: its signs (out x n_ref) and row scales [Ks][out][groups] by rows
        n_ref = len(layer.ref_idx)
        rb = np.asarray(layer.ref_bits).reshape(ks, -1)
        kw["ref_bits"] = np.stack([_tile_slice(rb[k], layer.out, n_ref, t0, t1) for k in range(ks)])
        rr = np.asarray(layer.ref_row_scale).reshape(ks, layer.out, -1)
        kw["ref_row_scale"] = np.ascontiguousarray(rr[:, r0:r1])
    return dataclasses.replace(layer, **kw)


def gather_rows(y_local, bounds, dist, group=None):
    """All-gather of every rank's Y[:, r0:r1] (a torch tensor [M][r1 - r0] on this rank's
    device) into the full Y [M][out], in row order, on every rank. Slices are padded to the
    largest shard for the collective and trimmed after it."""
    import torch

    M = y_local.shape[0]
    widest = max(r1 - r0 for r0, r1 in bounds)
    pad = torch.zeros((M, widest), dtype=y_local.dtype, device=y_local.device)
    pad[:, : y_local.shape[1]] = y_local
    parts = [torch.empty_like(pad) for _ in bounds]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, : r1 - r0] for p, (r0, r1) in zip(parts, bounds)], dim=1)

"""Plain fp64 CPU oracle for the binary-weight decode GEMV.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may import or run this module. The product
path never does; it fails loudly when its CUDA library is missing.

What it computes (sources are web pages, cited by title and section):

* Decoupled row-column binary bases -- "FluxBin: Flexible LUT-based Ultra-low-bit
  LLM Inference by Algorithm-Kernel Synergy", Sec. 3.1 (Decoupled Row-Column
  Binary Bases): the weight is a sum over K bases, each base a +-1 matrix
  scaled elementwise by the outer product of a row-scale vector and a
  column-scale vector, i.e. diag(r_k) B_k diag(c_k). The display equation is
  missing from the page; this is the plainest reading of its magnitude tensor
  M^(k) = alpha_r^(k) alpha_c^(k)T applied elementwise to B^(k).
* Bit-to-sign map -- same page, Sec. 3.2 Stage 1: a stored bit b means the sign
  (2b - 1), so bit 1 is +1 and bit 0 is -1.
* Binary low-rank correction -- "BiLoCo: Binary Low-Rank Corrections for
  Post-Training Quantization", section "The core idea: corrections made only of
  +1 and -1": Delta W = sum_j alpha_j u_j v_j^T with u_j, v_j in {+1,-1},
  applied to x as alpha_j * u_j * (v_j . x).
* Salient columns in int8 -- "BiSCo-LLM" (gist.science summary), Methodology 3,
  Sensitivity Protection (a ~1% set of sensitive channels kept by an 8-bit
  quantizer), together with FluxBin Sec. 3.2, Virtual Columnar Mapping (the
  salient columns are a dense block plus an index list, gathered at run
  time). Each salient column t adds s_t * q[:, t] to weight column idx_t.

The product is Y[m, o] = sum_i X[m, i] * W[o, i], evaluated in fp64 on the
exact stored values (bf16 and fp32 inputs widen exactly to fp64).

Packed sign layout (the library's storage format): a rows x cols sign matrix is
stored as [tiles][quads][32][4] little-endian uint32 words with
tiles = ceil(rows/32), quads = ceil(cols/128); entry (32t + r, 128q + 32j + b)
is bit b of word [t][q][r][j]. Padding entries hold bit 0.

Parity pins live in tests/test_oracle.py. Large shapes have no value printed on
the pages, so beyond the pinned small cases the oracle is trusted through those
pins (worked examples, closed forms, invariants, brute force).
"""

import numpy as np

TILE_ROWS = 32
QUAD_COLS = 128


# ----------------------------------------------------------------------------
# packed sign matrices
# ----------------------------------------------------------------------------

def _grid(rows, cols):
    return -(-rows // TILE_ROWS), -(-cols // QUAD_COLS)


def unpack_bit_matrix(words, rows, cols):
    """Packed words -> int8 matrix of +1/-1 (bit 1 -> +1, bit 0 -> -1)."""
    T, Q = _grid(rows, cols)
    w = np.asarray(words, dtype=np.uint32).reshape(T, Q, TILE_ROWS, 4)
    out = np.empty((rows, cols), dtype=np.int8)
    shifts = np.arange(32, dtype=np.uint32)
    for t in range(T):
        r0, r1 = t * TILE_ROWS, min(rows, (t + 1) * TILE_ROWS)
        # bits[q, r, j, b] = (word[t, q, r, j] >> b) & 1
        bits = ((w[t][..., None] >> shifts) & 1).astype(np.int8)
        # element (row r, col 128q + 32j + b)
        tile = bits.transpose(1, 0, 2, 3).reshape(TILE_ROWS, Q * QUAD_COLS)
        out[r0:r1] = tile[: r1 - r0, :cols] * 2 - 1
    return out


def unpack_bit_rows(words, rows, cols, row_idx):
    """Signs of the selected rows only, int8 [len(row_idx), cols]; decodes just their tiles."""
    row_idx = np.asarray(row_idx, dtype=np.int64)
    T, Q = _grid(rows, cols)
    w = np.asarray(words, dtype=np.uint32).reshape(T, Q, TILE_ROWS, 4)
    shifts = np.arange(32, dtype=np.uint32)
    out = np.empty((len(row_idx), cols), dtype=np.int8)
    for n, i in enumerate(row_idx):
        t, r = divmod(int(i), TILE_ROWS)
        bits = ((w[t, :, r, :][..., None] >> shifts) & 1).astype(np.int8)   # [q][j][b]
        out[n] = bits.reshape(Q * QUAD_COLS)[:cols] * 2 - 1
    return out


def pack_bit_matrix(signs):
    """int8 matrix of +1/-1 -> packed words (+1 -> bit 1). Rejects other values."""
    s = np.asarray(signs)
    if s.ndim != 2:
        raise ValueError("signs must be 2-D")
    if not np.all((s == 1) | (s == -1)):
        raise ValueError("signs must be +1 or -1")
    rows, cols = s.shape
    T, Q = _grid(rows, cols)
    full = np.zeros((T * TILE_ROWS, Q * QUAD_COLS), dtype=np.uint64)
    full[:rows, :cols] = (s == 1)
    # [T][r][Q][j][b] -> words[t][q][r][j] = sum_b bit << b
    b = full.reshape(T, TILE_ROWS, Q, 4, 32)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    words = (b * weights).sum(axis=-1).astype(np.uint32)       # [T][r][Q][j]
    return np.ascontiguousarray(words.transpose(0, 2, 1, 3)).reshape(-1)


# ----------------------------------------------------------------------------
# value decoding
# ----------------------------------------------------------------------------

def decode_values(a, dtype):
    """Stored values -> fp64. dtype 'f32' (float32 array) or 'bf16' (uint16 bit patterns)."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        u = np.asarray(a, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return u.view(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# weight reconstruction and product
# ----------------------------------------------------------------------------

def _binary_part_rows(layer, rows):
    """sum_k diag(r_k) B_k diag(c_k), restricted to output rows `rows`.

    With grouped row scales (layer.group = g > 0; "FluxBin", Sec. 3.1: one row scale per
    weight group, and Sec. 4: g is the group size of the row-wise scale) the row scale of
    entry (o, i) is r_k[o][i // g]."""
    W = np.zeros((len(rows), layer.in_), dtype=np.float64)
    if layer.K == 0:
        return W
    g = getattr(layer, "group", 0)
    ng = -(-layer.in_ // g) if g else 1
    R = decode_values(layer.row_scale, layer.scale_dtype).reshape(layer.K, layer.out, ng)
    C = decode_values(layer.col_scale, layer.scale_dtype).reshape(layer.K, layer.in_)
    col_group = np.arange(layer.in_) // g if g else np.zeros(layer.in_, dtype=np.int64)
    bits = np.asarray(layer.bits).reshape(layer.K, -1)
    for k in range(layer.K):
        S = unpack_bit_rows(bits[k], layer.out, layer.in_, rows)
        W += R[k][rows][:, col_group] * S * C[k][None, :]
    return W


def _correction_part_rows(layer, rows):
    """sum_j alpha_j u_j v_j^T restricted to output rows `rows`."""
    if not layer.rank:
        return 0.0
    V = unpack_bit_matrix(layer.v_bits, layer.rank, layer.in_).astype(np.float64)        # [R, in]
    U = unpack_bit_rows(layer.ut_bits, layer.out, layer.rank, rows).astype(np.float64)  # [rows, R]
    a = np.asarray(layer.alpha, dtype=np.float32).astype(np.float64)
    return (U * a[None, :]) @ V


def _salient_part_rows(layer, rows):
    """Dense int8 salient block scattered to its input columns, rows `rows`."""
    W = np.zeros((len(rows), layer.in_), dtype=np.float64)
    if not layer.n_sal:
        return W
    q = np.asarray(layer.sal_q, dtype=np.int8)[rows, : layer.n_sal].astype(np.float64)
    s = np.asarray(layer.sal_scale, dtype=np.float32).astype(np.float64)
    idx = np.asarray(layer.sal_idx, dtype=np.int64)
    for t in range(layer.n_sal):
        W[:, idx[t]] += s[t] * q[:, t]
    return W


def _refinement_part_rows(layer, rows):
    """Binary salient refinement ("FluxBin", Sec. 4, Kb-sS-gG, and the Virtual Columnar
    Mapping of Sec. 3.2: the sparse salient bases stored as one dense matrix over the
    gathered columns), rows `rows`: entry (o, idx_t) gains
    sum_k r^s_k[o][idx_t // g] c^s_k[t] (2b - 1), b = bit (o, t) of refinement base k."""
    W = np.zeros((len(rows), layer.in_), dtype=np.float64)
    Ks = getattr(layer, "ref_K", 0)
    if not Ks:
        return W
    g = layer.group
    idx = np.asarray(layer.ref_idx, dtype=np.int64)
    n = len(idx)
    R = decode_values(layer.ref_row_scale, layer.scale_dtype).reshape(Ks, layer.out, -1)
    C = decode_values(layer.ref_col_scale, layer.scale_dtype).reshape(Ks, n)
    bits = np.asarray(layer.ref_bits).reshape(Ks, -1)
    for k in range(Ks):
        S = unpack_bit_rows(bits[k], layer.out, n, rows)                  # [rows, n]
        W[:, idx] += R[k][rows][:, idx // g] * S * C[k][None, :]
    return W


def reconstruct_rows(layer, rows):
    rows = np.asarray(rows, dtype=np.int64)
    return (_binary_part_rows(layer, rows) + _correction_part_rows(layer, rows) + _salient_part_rows(layer, rows) +
            _refinement_part_rows(layer, rows))


def reconstruct(layer):
    """Dense fp64 W [out, in]."""
    return reconstruct_rows(layer, np.arange(layer.out))


def gemv_rows(layer, X, x_dtype, rows):
    """Y[:, rows] in fp64 for activations X [M, in]."""
    Xd = decode_values(X, x_dtype).reshape(-1, layer.in_)
    return Xd @ reconstruct_rows(layer, rows).T


def gemv(layer, X, x_dtype):
    """Y = X W^T in fp64, Y [M, out]."""
    return gemv_rows(layer, X, x_dtype, np.arange(layer.out))


def correction_z(layer, X, x_dtype):
    """Intermediate z[m, j] = alpha_j * (v_j . x_m) of the binary correction, fp64 [M, R]."""
    Xd = decode_values(X, x_dtype).reshape(-1, layer.in_)
    V = unpack_bit_matrix(layer.v_bits, layer.rank, layer.in_).astype(np.float64)
    a = np.asarray(layer.alpha, dtype=np.float32).astype(np.float64)
    return (Xd @ V.T) * a[None, :]


# ----------------------------------------------------------------------------
# binary low-rank decomposition (offline; the correction's sign vectors and alpha)
# ----------------------------------------------------------------------------

def _sign(a):
    """+1 / -1 elementwise; a zero takes +1."""
    return np.where(np.asarray(a) >= 0, 1.0, -1.0)


def biloco_decompose(W, v0, rounds=5):
    """Greedy binary rank-one components of W, then a joint refit of their coefficients
    ("BiLoCo: Binary Low-Rank Corrections for Post-Training Quantization", "Finding the
    sign vectors"): starting from the residual R = W, for each component j the sign
    vectors alternate u = sign(R v), v = sign(R^T u) for `rounds` rounds from the starting
    signs v0[j] (the random start is an input), alpha_j = u^T R v / (rows * cols) is the
    error-minimising coefficient of the sign pair, and alpha_j u v^T leaves the residual.
    The refit solves the least-squares problem for all coefficients at once (the normal
    equations G alpha = b with G_ij = (u_i . u_j)(v_i . v_j), b_j = u_j^T W v_j).

    Returns U [rows][R], V [R][cols] (entries +-1), the greedy and the refit coefficients.
    """
    W = np.asarray(W, dtype=np.float64)
    rows, cols = W.shape
    v0 = np.asarray(v0, dtype=np.float64)
    rank = v0.shape[0]
    Rs = W.copy()
    U = np.zeros((rows, rank))
    V = np.zeros((rank, cols))
    greedy = np.zeros(rank)
    for j in range(rank):
        v = _sign(v0[j])
        for _ in range(rounds):
            u = _sign(Rs @ v)
            v = _sign(Rs.T @ u)
        a = float(u @ Rs @ v) / (rows * cols)
        Rs -= a * np.outer(u, v)
        U[:, j], V[j], greedy[j] = u, v, a
    G = (U.T @ U) * (V @ V.T)
    b = np.array([U[:, j] @ W @ V[j] for j in range(rank)])
    refit = np.linalg.lstsq(G, b, rcond=None)[0]
    return U, V, greedy, refit


def fluxbin_sign_search(W, row_scale, col_scale, group=0):
    """Joint binary signs of Kb bases for fixed magnitudes ("FluxBin", Sec. 3.1,
    Decoupled Row-Column Binary Bases: with M^(k) = alpha_r^(k) alpha_c^(k)T the signs
    minimise the reconstruction error, found by evaluating all 2^Kb sign combinations).

    W [rows][cols]; row_scale [Kb][rows] (group == 0) or [Kb][rows][ceil(cols/group)] (one
    row scale per weight group); col_scale [Kb][cols]. Element (o, i) takes the combination
    c in 0 .. 2^Kb - 1 (bit k of c set: base k gets +1, clear: -1) with the smallest
    (W[o][i] - sum_k s_k M^(k)[o][i])^2, the first such c on ties; fp64 throughout.
    Returns the signs [Kb][rows][cols] as +1/-1 int8.
    """
    W = np.asarray(W, dtype=np.float64)
    rows, cols = W.shape
    C = np.asarray(col_scale, dtype=np.float64)
    Kb = C.shape[0]
    R = np.asarray(row_scale, dtype=np.float64)
    if group:
        R = R.reshape(Kb, rows, -1)[:, :, np.arange(cols) // group]   # [Kb][rows][cols]
    else:
        R = np.broadcast_to(R.reshape(Kb, rows, 1), (Kb, rows, cols))
    Mk = R * C[:, None, :]                                             # magnitudes M^(k)
    best_err = np.full((rows, cols), np.inf)
    best = np.zeros((rows, cols), dtype=np.int64)
    for c in range(1 << Kb):
        rec = np.zeros((rows, cols))
        for k in range(Kb):
            rec += (1.0 if (c >> k) & 1 else -1.0) * Mk[k]
        err = (W - rec) ** 2
        take = err < best_err  # strict: the first combination wins a tie
        best[take] = c
        best_err[take] = err[take]
    return np.stack([np.where((best >> k) & 1, 1, -1).astype(np.int8) for k in range(Kb)])


# ----------------------------------------------------------------------------
# storage and byte accounting
# ----------------------------------------------------------------------------

def binary_correction_storage_bits(rank, out, in_):
    """Sign bits of a rank-`rank` binary correction: one bit per entry of u_j and v_j
    (BiLoCo, "The core idea", storage paragraph; coefficients ignored)."""
    return rank * (out + in_)


def dense_correction_storage_bits(rank, out, in_, bits_per_value=16):
    """Storage of a dense low-rank correction with `bits_per_value` per vector entry."""
    return rank * (out + in_) * bits_per_value


def fp4_weight_bits(out, in_, bits_per_weight=4.0):
    """Bits of an FP4 weight matrix at `bits_per_weight` (4 bare, ~4.5 with block scales)."""
    return out * in_ * bits_per_weight


def fluxbin_average_bit_width(rows, cols, Kb, Ks, g, s, scale_bits=16):
    """Effective average bit-width of a FluxBin-style layer with grouped row scales and a
    binary salient refinement ("FluxBin", Sec. C.2 Storage Consumption Analysis): Kb global
    sign bits per weight; Ks refinement sign bits on the s salient columns of every group
    of g columns; one row scale per (row, group) for each of the Kb + Ks bases; one column
    scale per column of each base (the salient bases cover rows x cols*s/g); one index per
    salient column; every scale and index in `scale_bits` bits. Bits over rows*cols."""
    n_sal = cols * s / g
    bits = Kb * rows * cols + Ks * rows * n_sal                 # signs
    bits += (Kb + Ks) * rows * (cols / g) * scale_bits          # grouped row scales
    bits += (Kb * cols + Ks * n_sal) * scale_bits               # column scales
    bits += n_sal * scale_bits                                  # salient column indices
    return bits / (rows * cols)


def fluxbin_storage_bits(layer, scale_bits=16):
    """Bits a FluxBin-style layer actually stores, counted from its arrays: the global and
    refinement sign bits (no padding), one row scale per (base, row, group) and one column
    scale per column of every base, one index per salient column, each scale and index in
    `scale_bits` bits (the accounting of "FluxBin", Sec. C.2)."""
    rows, cols, g = layer.out, layer.in_, layer.group
    ng = -(-cols // g)
    Ks = getattr(layer, "ref_K", 0)
    n_ref = len(layer.ref_idx) if Ks else 0
    bits = layer.K * rows * cols + Ks * rows * n_ref
    bits += (layer.K + Ks) * rows * ng * scale_bits
    bits += (layer.K * cols + Ks * n_ref) * scale_bits
    bits += n_ref * scale_bits
    return bits


def _dtype_bytes(dtype):
    return {"f32": 4, "bf16": 2}[dtype]


def algorithmic_bytes(layer, M, x_dtype, y_dtype="f32"):
    """Bytes one GEMV must move at minimum: unpadded sign bits, scales (grouped row scales
    counted per group), correction signs and coefficients, salient payload, refinement
    signs, scales and indices, X read and Y written."""
    sb = _dtype_bytes(layer.scale_dtype)
    g = getattr(layer, "group", 0) or 0
    ng = -(-layer.in_ // g) if g else 1  # row scales per row (FluxBin Sec. 3.1 groups)
    n = layer.K * layer.out * layer.in_ / 8.0
    n += layer.K * (layer.out * ng + layer.in_) * sb
    if layer.rank:
        n += layer.rank * (layer.out + layer.in_) / 8.0 + 4 * layer.rank
    if layer.n_sal:
        n += layer.out * layer.n_sal + 4 * layer.n_sal + 4 * layer.n_sal
    ks = getattr(layer, "ref_K", 0) or 0
    if ks:  # FluxBin Sec. 4 refinement: signs, per-group row scales, column scales, int32 indices
        nr = len(layer.ref_idx)
        n += ks * layer.out * nr / 8.0 + ks * (layer.out * ng + nr) * sb + 4 * nr
    n += M * layer.in_ * _dtype_bytes(x_dtype) + M * layer.out * _dtype_bytes(y_dtype)
    return int(round(n))

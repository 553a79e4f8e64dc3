/*
 * bisco.h -- C ABI of the binary-weight decode GEMV library (libbisco.so).
 *
 * The library computes the decode-time product Y = X * W^T for a weight that is
 * stored as a sum of bit-packed sign matrices with decoupled row and column
 * scales, plus an optional binary low-rank correction and an optional set of
 * salient input columns kept in int8:
 *
 *   W[o][i] = sum_k r_k[o] * c_k[i] * B_k[o][i]                       (1)
 *           + sum_j alpha_j * U[o][j] * V[j][i]                        (2)
 *           + sum_t [i == idx_t] * s_t * q[o][t]                       (3)
 *
 *   (1) "FluxBin: Flexible LUT-based Ultra-low-bit LLM Inference by
 *       Algorithm-Kernel Synergy", Sec. 3.1, decoupled row-column binary bases;
 *       a stored bit b means the sign (2b - 1) (Sec. 3.2, Stage 1).
 *   (2) "BiLoCo: Binary Low-Rank Corrections for Post-Training Quantization",
 *       section "The core idea": U, V in {+1,-1}; applied as alpha * u * (v . x).
 *   (3) "BiSCo-LLM" (gist.science summary), Methodology 3, Sensitivity
 *       Protection: a ~1% set of channels in 8 bits; FluxBin Sec. 3.2, Virtual
 *       Columnar Mapping: a dense block plus an index list gathered at run time.
 *
 * Conventions for every entry point:
 *  - Host entry points (bisco_pack, bisco_unpack, sizes, strings) take host
 *    pointers. bisco_gemv, bisco_workspace_init and bisco_bench take device
 *    pointers and a CUDA stream (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream).
 *  - The caller owns all memory. bisco_gemv allocates nothing; scratch space is
 *    the caller's workspace buffer.
 *  - Arguments are validated before anything is launched or written: a
 *    validation failure returns BISCO_ERR_INVALID_ARG (or BISCO_ERR_WORKSPACE)
 *    and leaves every output untouched. A CUDA launch failure returns
 *    BISCO_ERR_CUDA. Device-side errors are recorded in the workspace status
 *    word and read back with bisco_sync_status.
 *  - Packed bit buffers, X, Y and the workspace must be 16-byte aligned.
 *  - Calls are thread-safe; calls that share a workspace must be ordered on one
 *    stream (two calls in flight on one workspace race).
 */
#ifndef BISCO_H
#define BISCO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BISCO_OK = 0,
  BISCO_ERR_INVALID_ARG = 1,  /* bad pointer, size, dtype, index or alignment */
  BISCO_ERR_UNSUPPORTED = 2,  /* valid request this build cannot run          */
  BISCO_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed         */
  BISCO_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up           */
  BISCO_ERR_WORKSPACE = 5     /* workspace missing or too small               */
} bisco_status;

typedef enum { BISCO_F32 = 0, BISCO_BF16 = 1 } bisco_dtype;

/*
 * Packed sign-matrix layout (all bit matrices: B_k, V and U^T).
 *
 * A rows x cols matrix of signs is stored in row tiles of 32 rows and column
 * quads of 128 columns: uint32 words [tiles][quads][32][4] with
 * tiles = ceil(rows/32) and quads = ceil(cols/128). Entry (32t + r, 128q + 32j + b)
 * is bit b of word [t][q][r][j]; bit 1 means +1 and bit 0 means -1. Padding
 * entries (row >= rows or col >= cols) hold bit 0. With this layout the 32 lanes
 * of a warp, one row each, read a (tile, quad) block as 512 contiguous bytes.
 */

/* Number of uint32 words of one packed rows x cols sign matrix (0 if either is <= 0). */
int64_t bisco_packed_words(int64_t rows, int64_t cols);

/*
 * Pack a dense row-major int8 matrix of +1/-1 into the layout above.
 * signs: host, rows*cols int8, each exactly +1 or -1.
 * packed: host, bisco_packed_words(rows, cols) words, written in full (padding = 0).
 * Returns BISCO_ERR_INVALID_ARG for null pointers, rows or cols <= 0, or any entry
 * other than +1/-1; in that case nothing is written.
 */
bisco_status bisco_pack(const int8_t* signs, int64_t rows, int64_t cols, uint32_t* packed);

/*
 * Inverse of bisco_pack: signs (host, rows*cols int8) receives +1/-1.
 * Padding bits are ignored. BISCO_ERR_INVALID_ARG for null pointers or sizes <= 0.
 */
bisco_status bisco_unpack(const uint32_t* packed, int64_t rows, int64_t cols, int8_t* signs);

/* One layer. All pointers are device pointers owned by the caller. */
typedef struct {
  int32_t out;              /* output features (rows of W), >= 1                      */
  int32_t in;               /* input features (columns of W), >= 1                    */
  int32_t num_bases;        /* K >= 0 binary bases                                    */
  const uint32_t* bits;     /* [K][bisco_packed_words(out, in)] sign matrices B_k     */
  const void* row_scale;    /* [K][out] r_k, dtype scale_dtype (row_group == 0);
                               [K][ceil(in/row_group)][out] with grouped row scales   */
  const void* col_scale;    /* [K][in]  c_k, dtype scale_dtype                        */
  int32_t scale_dtype;      /* BISCO_F32 or BISCO_BF16                                */
  int32_t rank;             /* R >= 0; 0 = no low-rank correction                     */
  const uint32_t* v_bits;   /* [bisco_packed_words(R, in)]  V, row j = v_j            */
  const uint32_t* ut_bits;  /* [bisco_packed_words(out, R)] U^T: entry (o, j) = u_j[o] */
  const float* alpha;       /* [R] coefficients alpha_j                               */
  int32_t n_sal;            /* n_s >= 0 salient input columns; 0 = none               */
  int32_t sal_stride;       /* bytes per row of sal_q: multiple of 16, >= n_sal       */
  const int32_t* sal_idx;   /* [n_s] strictly ascending column indices in [0, in)     */
  const int8_t* sal_q;      /* [out][sal_stride] int8 values q[o][t]                  */
  const float* sal_scale;   /* [n_s] per-column scales s_t                            */
  int32_t row_group;        /* g >= 0: 0 = one row scale per (base, row); g > 0 = one
                               per (base, row, group of g input columns), "FluxBin"
                               Sec. 3.1: W_k[o][i] = r_k[i/g][o] c_k[i] (2b - 1).
                               The kernels take g a multiple of 128 (else
                               BISCO_ERR_UNSUPPORTED); grouped layers run on the
                               integer tensor-core kernel in chunks of up to 8 rows */
  /* Binary salient refinement ("FluxBin", Sec. 4, Kb-sS-gG; stored as one dense sign
     matrix over the gathered salient columns, Sec. 3.2 Virtual Columnar Mapping), added to
     the rest of W: entry (o, ref_idx[t]) gains
     sum_k ref_row_scale[k][ref_idx[t] / row_group][o] * ref_col_scale[k][t] * (2b - 1),
     b = bit (o, t) of refinement base k. Needs row_group > 0 (the refinement's row scales
     are grouped like the global ones). */
  int32_t ref_bases;        /* Ks in 0..4; 0 = none                                    */
  int32_t n_ref;            /* salient columns of the refinement, >= 1 when Ks > 0     */
  const int32_t* ref_idx;   /* [n_ref] strictly ascending column indices in [0, in); an
                               index outside that range is read as a zero activation and
                               recorded as BISCO_ERR_INVALID_ARG in the workspace status;
                               indices out of order give wrong groups (never an
                               out-of-bounds access)                                    */
  const uint32_t* ref_bits; /* [Ks][bisco_packed_words(out, n_ref)] packed signs       */
  const void* ref_row_scale; /* [Ks][ceil(in/row_group)][out], dtype scale_dtype       */
  const void* ref_col_scale; /* [Ks][n_ref], dtype scale_dtype                         */
} bisco_layer;

/*
 * Bytes of workspace bisco_gemv needs for this layer and batch M (>= 1).
 * BISCO_ERR_INVALID_ARG for a null pointer or a layer whose sizes are invalid.
 */
bisco_status bisco_workspace_size(const bisco_layer* layer, int32_t M, size_t* bytes);

/*
 * Prepare a workspace for first use: zero-fills ws_bytes bytes on `stream`.
 * The workspace holds the device status word, counters that a launch computing z and
 * y together uses to hand z over (each such launch returns them to zero), z, and for a
 * layer with a salient refinement that term of one 8-row batch chunk (fp32).
 * Every bisco_gemv call leaves the workspace ready for the next call, so this is
 * needed once per buffer (and again after a call reported an error).
 */
bisco_status bisco_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Y = X * W^T with W as in (1)-(3) above; asynchronous on `stream`.
 *  X:  device, [M][in] row-major, x_dtype (BISCO_BF16 or BISCO_F32).
 *  Y:  device, [M][out] row-major, y_dtype; fully overwritten.
 *  M:  batch rows; M == 0 is a no-op that returns BISCO_OK.
 *  ws: device workspace of at least bisco_workspace_size bytes, prepared once by
 *      bisco_workspace_init.
 * The sign-times-activation sums use fp32 accumulation. Results are deterministic:
 * the reduction order is fixed, so repeated calls give bit-identical Y.
 * Kernels are launched with programmatic dependent launch: they prefetch weights
 * while the previous kernel on the stream finishes, and read X only after it
 * has completed. The calls can be captured in a CUDA graph.
 */
bisco_status bisco_gemv(const bisco_layer* layer, const void* X, int32_t x_dtype, int32_t M,
                        void* Y, int32_t y_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Layers that read the same X (a decoder's q/k/v projections, gate and up) in one call:
 * Y[j] = X * W_j^T for j < n (1 <= n <= 3, every layer with the same `in`). For batches
 * below 16 rows each chunk of up to 8 rows runs as ONE integer tensor-core launch whose
 * clusters are split between the layers (and, for a layer with a correction, between its
 * z pass and its output pass, as in bisco_gemv), so the dependent chain of a launch is paid
 * once for the group. Larger batches, groups whose launch does not fit and groups with a
 * salient-refined layer run layer by layer exactly as bisco_gemv (same results within the
 * documented tolerance either way).
 *  layers: host array of n layers.   X: device [M][in].   Y: host array of n device
 *  pointers, Y[j] [M][layers[j].out].   ws: at least bisco_group_workspace_size bytes,
 *  prepared by bisco_workspace_init. Errors as bisco_gemv; BISCO_ERR_INVALID_ARG for n
 *  outside 1..3 or layers of different `in`.
 */
bisco_status bisco_group_workspace_size(const bisco_layer* layers, int32_t n, int32_t M, size_t* bytes);
bisco_status bisco_gemv_group(const bisco_layer* layers, int32_t n, const void* X, int32_t x_dtype, int32_t M,
                              void* const* Y, int32_t y_dtype, void* ws, size_t ws_bytes, void* stream);
/* Launches of bisco_gemv_group, as bisco_plan_kernels reports them for bisco_gemv. */
int32_t bisco_plan_group_kernels(const bisco_layer* layers, int32_t n, int32_t M, int32_t x_dtype, size_t ws_bytes,
                                 int32_t* kinds, int32_t max_kinds);

/*
 * Synchronise `stream` and return the device-side status recorded in workspace
 * `ws` by earlier bisco_gemv calls (BISCO_OK if none). A recorded error stays
 * until bisco_workspace_init clears it.
 */
bisco_status bisco_sync_status(void* stream, const void* ws);

/*
 * Which kernel family runs a batch chunk (process-wide; for tests and diagnostics).
 *  BISCO_PATH_AUTO (default): chunks of 16..128 rows on the tcgen05 tensor-core kernel
 *    (bf16 scales), chunks of 2..8 rows on the integer tensor-core kernel (mma.sync)
 *    when its shared-memory plan fits, single rows of a layer with a correction on the
 *    integer kernel's one-launch form, other single rows and the rest on the
 *    lookup-table kernels.
 *  BISCO_PATH_LOOKUP_TABLE: as AUTO, but chunks of up to 8 rows always take the
 *    lookup-table kernels (FluxBin Sec. 3.2, Stages 1-3, restated for B200).
 *  BISCO_PATH_SMALL_BATCH_ONLY: as AUTO, but every chunk has at most 8 rows (no
 *    tcgen05 kernel).
 *  BISCO_PATH_INTEGER_MMA: as AUTO, but chunks of up to 8 rows, single rows included,
 *    take the integer tensor-core kernel whenever its plan fits.
 * Layers with grouped row scales or a salient refinement run every batch chunk (8 rows
 * at most; 4, 2 or 1 where the 8-row plan does not fit shared memory, e.g. 11008 input
 * columns) on the integer tensor-core kernel under every policy; a refined chunk is
 * preceded by one refinement launch (BISCO_KERNEL_REFINE). BISCO_ERR_UNSUPPORTED when
 * the integer plan of one row, or the refinement's shared-memory tables (about
 * 4 * (Ks + 9) * n_ref + 512 * Ks * ceil(n_ref / 128) + 128 * Ks * ceil(in / g) + 32768
 * bytes), do not fit.
 * Every path computes the same product within the documented tolerance.
 * Returns BISCO_ERR_INVALID_ARG for an unknown policy.
 */
enum { BISCO_PATH_AUTO = 0, BISCO_PATH_LOOKUP_TABLE = 1, BISCO_PATH_SMALL_BATCH_ONLY = 2, BISCO_PATH_INTEGER_MMA = 3 };
bisco_status bisco_set_path_policy(int32_t policy);

/* Kernel kinds reported by bisco_plan_kernels. */
enum {
  BISCO_KERNEL_LUT_WARP = 1,      /* lookup tables, 16-warp CTAs, <= 2 batch rows        */
  BISCO_KERNEL_LUT_STREAM = 2,    /* lookup tables, bulk-copy sign stream, <= 2 rows     */
  BISCO_KERNEL_LUT_ROWS = 3,      /* lookup tables, warps own row tiles, 4 or 8 rows     */
  BISCO_KERNEL_INTEGER_MMA = 4,   /* int8 tensor cores (mma.sync), <= 8 rows; with a
                                     correction, z and y in one launch                   */
  BISCO_KERNEL_TENSOR_CORE = 5,   /* tcgen05 tensor cores, 16..128 rows                  */
  BISCO_KERNEL_REFINE = 6         /* salient refinement term into the workspace (CUDA
                                     cores), ahead of the integer launch that adds it     */
};

/*
 * The kernel launches bisco_gemv would issue for this layer, batch M, activation dtype
 * and workspace size under the current path policy, in launch order. Writes up to
 * max_kinds entries of kinds (host array) and returns the number of launches, or -1 if
 * the request is invalid or unsupported (same checks as bisco_gemv). Needs the device
 * whose plans are queried to be current; launches nothing.
 */
int32_t bisco_plan_kernels(const bisco_layer* layer, int32_t M, int32_t x_dtype, size_t ws_bytes, int32_t* kinds,
                           int32_t max_kinds);

/*
 * Test hook for the bounded device-side waits of the tensor-core kernels.
 * With skip_tile >= 0, every later launch leaves some sign-word copies unissued: the
 * integer tensor-core kernel those of local row tile skip_tile of each CTA, the tcgen05
 * kernel those of each CTA's last step. The threads that wait for them give up after
 * wait_ns nanoseconds (0: the default limit, 200 ms) and record BISCO_ERR_TIMEOUT in the
 * workspace status word; no copy is in flight into the skipped shared memory when they
 * give up, and the kernels still release their tensor memory. skip_tile = -1 restores
 * normal operation. Process-wide; BISCO_ERR_INVALID_ARG for skip_tile < -1.
 */
bisco_status bisco_debug_set_wait_test(int32_t skip_tile, uint64_t wait_ns);

/*
 * Largest correction rank bisco_gemv_noalloc accepts.
 */
#define BISCO_NOALLOC_MAX_RANK 4096

/*
 * bisco_gemv without a caller-provided workspace. (There is no counterpart in the
 * papers: this is a deployment convenience of this library.)
 *
 * For callers that cannot allocate device memory -- e.g. a plug-in inside a host
 * application that owns every device allocation and passes the plug-in only its
 * operands, or a runtime that reserves all device memory at start-up. The
 * scratch space (status word and the correction's intermediate z for one batch chunk)
 * is a fixed array of 256 + 8 * 4096 * 4 bytes in the library's device image; every GPU
 * that loads the library keeps it until the process exits. This call allocates nothing.
 *
 * Arguments and results are those of bisco_gemv, minus the workspace. Layers with
 * rank > BISCO_NOALLOC_MAX_RANK, and layers with a salient refinement (ref_bases > 0,
 * whose term needs out * 32 bytes of scratch), are rejected with BISCO_ERR_UNSUPPORTED.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress);
 * make that first call before any stream capture starts. A failed lookup is not cached
 * (the next call retries); a device reset invalidates the cached address.
 * With the fixed array, z fits at most floor(8192 / rank) batch rows, so a batch chunk on
 * the tcgen05 tensor-core kernel (16..128 rows) is limited to floor(8192 / rank / 16) * 16
 * rows; layers with rank > 256 run every chunk on the small-batch kernels (correct, slower
 * at large batch than bisco_gemv with its preferred workspace).
 * All calls share the one array: calls that may overlap on the GPU (different streams,
 * or different host threads) race with each other; order them on one stream.
 * Device-side errors are recorded in the shared array and cannot be read back through
 * this entry point (use bisco_gemv with a workspace when that check matters).
 */
bisco_status bisco_gemv_noalloc(const bisco_layer* layer, const void* X, int32_t x_dtype, int32_t M,
                                void* Y, int32_t y_dtype, void* stream);

/* Benchmark request: a stream of n_layers GEMVs (distinct weight copies) captured
 * in one CUDA graph and replayed. */
typedef struct {
  const bisco_layer* layers;  /* host array of n_layers layer descriptors (device data) */
  int32_t n_layers;
  const void* X;              /* device [M][in] shared by all layers                     */
  int32_t x_dtype;
  int32_t M;
  void* Y;                    /* device [n_layers][M][out]                               */
  int32_t y_dtype;
  void* ws;                   /* device workspace, >= max over layers of the size        */
  size_t ws_bytes;
  int32_t warmup;             /* untimed graph replays                                   */
  int32_t reps;               /* timed graph replays                                     */
  void* stream;
} bisco_bench_args;

typedef struct {
  double us_per_gemv;         /* mean device time per GEMV over the timed replays  */
  double us_per_replay;       /* mean device time of one replay of the whole graph */
  int32_t kernels_per_gemv;   /* kernel launches per GEMV                         */
} bisco_bench_result;

/*
 * Time the GEMV stream with CUDA events on args->stream (warm-up replays are not
 * timed). Returns BISCO_ERR_INVALID_ARG for bad arguments, BISCO_ERR_CUDA on a
 * CUDA failure; the graph is released before returning.
 */
bisco_status bisco_bench(const bisco_bench_args* args, bisco_bench_result* result);

/*
 * Offline quantisers (device, fp64). They produce the weight format above from dense
 * weights; nothing in bisco_gemv depends on them.
 *
 * bisco_fluxbin_signs: joint binary signs of Kb bases for fixed magnitudes ("FluxBin",
 * Sec. 3.1, Decoupled Row-Column Binary Bases: M^(k) = alpha_r^(k) alpha_c^(k)T, all 2^Kb
 * sign combinations evaluated). Element (o, i) takes the combination c (bit k of c set:
 * base k is +1) with the smallest (W[o][i] - sum_k s_k r_k c_k)^2, the first c on ties.
 *  W:         device, [rows][cols] row-major fp64.
 *  row_scale: device fp64, [Kb][rows] (group == 0) or [Kb][ceil(cols/group)][rows]
 *             (one row scale per group of `group` columns, the layout bisco_layer uses).
 *  col_scale: device fp64, [Kb][cols].
 *  bits:      device, Kb * bisco_packed_words(rows, cols) words, written in full in the
 *             packed layout (base k at word offset k * bisco_packed_words(rows, cols)).
 * Asynchronous on `stream`. BISCO_ERR_INVALID_ARG for null pointers, sizes < 1,
 * Kb outside 1..8 or group < 0; BISCO_ERR_CUDA if the launch fails.
 */
bisco_status bisco_fluxbin_signs(const double* W, int64_t rows, int64_t cols, int32_t Kb, const double* row_scale,
                                 const double* col_scale, int32_t group, uint32_t* bits, void* stream);

/*
 * bisco_biloco_decompose: binary low-rank decomposition W ~ sum_j alpha_j u_j v_j^T
 * ("BiLoCo: Binary Low-Rank Corrections for Post-Training Quantization", "Finding the
 * sign vectors"). For j = 0 .. rank-1 on the residual R (initially W): v = v0[j], then
 * `rounds` times u = sign(R v), v = sign(R^T u) (a zero sum takes +1); the greedy
 * coefficient alpha_j = u^T R v / (rows cols); R -= alpha_j u v^T. Then the joint refit:
 * the least-squares coefficients of the chosen sign pairs, G alpha = b with
 * G_ij = (u_i . u_j)(v_i . v_j) and b_j = u_j^T W v_j, solved by Gaussian elimination
 * with partial pivoting (G must be nonsingular: distinct sign pairs).
 *  W:      device [rows][cols] fp64 (not modified).
 *  v0:     device [rank][cols] int8, starting signs, each +1 or -1.
 *  U:      device [rows][rank] int8 (+-1), column j = u_j.   V: device [rank][cols] int8.
 *  alpha_greedy, alpha_refit: device [rank] fp64.
 *  ws:     device workspace of bisco_biloco_workspace_size bytes (the residual and the
 *          normal equations).
 * Asynchronous on `stream` (launches from the host thread, in order). Errors as above,
 * BISCO_ERR_WORKSPACE for a short workspace; rank <= 4096.
 */
bisco_status bisco_biloco_workspace_size(int64_t rows, int64_t cols, int32_t rank, size_t* bytes);
bisco_status bisco_biloco_decompose(const double* W, int64_t rows, int64_t cols, int32_t rank, int32_t rounds,
                                    const int8_t* v0, int8_t* U, int8_t* V, double* alpha_greedy,
                                    double* alpha_refit, void* ws, size_t ws_bytes, void* stream);

/* Static string naming a status code. */
const char* bisco_status_string(bisco_status status);

#ifdef __cplusplus
}
#endif

#endif /* BISCO_H */

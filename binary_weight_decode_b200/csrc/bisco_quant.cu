// Offline quantisers that produce the library's weight format on the device.
//
//  * FluxBin joint sign search ("FluxBin", Sec. 3.1, Decoupled Row-Column Binary Bases):
//    for fixed magnitudes M^(k) = alpha_r^(k) alpha_c^(k)T every weight takes the sign
//    combination of its Kb bases that minimises the reconstruction error, found by
//    evaluating all 2^Kb combinations. One thread per (row, 32-column word) writes the
//    packed sign words of every base directly in the tiled layout bisco_gemv reads.
//  * BiLoCo binary low-rank decomposition ("BiLoCo: Binary Low-Rank Corrections for
//    Post-Training Quantization", "Finding the sign vectors"): greedy rank-one sign pairs
//    u = sign(R v), v = sign(R^T u) alternated from given starting signs, the coefficient
//    u^T R v / (rows cols) of each pair, the residual update R -= alpha u v^T, and a joint
//    least-squares refit of all coefficients (normal equations G alpha = b with
//    G_ij = (u_i . u_j)(v_i . v_j), b_j = u_j^T W v_j), solved by Gaussian elimination
//    with partial pivoting.
//
// Both run in fp64: a sign is decided by the sign of a sum, and fp64 sums leave the same
// decisions as any other exact-enough evaluation of the definitions except on ties.
#include <cuda_runtime.h>

#include <cstdint>

#include "bisco_internal.h"

namespace bisco {
namespace {

constexpr int kQT = 256;  // threads per block of the element-wise and reduction kernels

// ---- FluxBin sign search ------------------------------------------------------------

// Thread (row o, word w): columns 32w .. 32w+31 of row o (word j = w % 4 of quad w / 4).
// Rows past `rows` and columns past `cols` are padding: bit 0.
__global__ void fluxbin_signs_kernel(const double* __restrict__ W, long long rows, long long cols, int Kb,
                                     const double* __restrict__ rs, const double* __restrict__ cs, int group,
                                     long long ngroups, uint32_t* __restrict__ bits, long long words_per_base) {
  const long long nw = (cols + 127) / 128 * 4;  // words per padded row
  const long long tiles = (rows + 31) / 32;
  const long long id = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (id >= tiles * 32 * nw) return;
  const long long o = id / nw, w = id - o * nw;
  uint32_t word[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) word[k] = 0u;
  if (o < rows) {
    for (int b = 0; b < 32; ++b) {
      const long long i = w * 32 + b;
      if (i >= cols) break;
      const double x = W[o * cols + i];
      const long long gi = group > 0 ? i / group : 0;
      double m[8];
      for (int k = 0; k < Kb; ++k) {
        const double r = group > 0 ? rs[(static_cast<long long>(k) * ngroups + gi) * rows + o] : rs[k * rows + o];
        m[k] = r * cs[k * cols + i];
      }
      int best = 0;
      double best_err = 0.0;
      for (int c = 0; c < (1 << Kb); ++c) {
        double rec = 0.0;
        for (int k = 0; k < Kb; ++k) rec += ((c >> k) & 1) ? m[k] : -m[k];
        const double e = (x - rec) * (x - rec);
        if (c == 0 || e < best_err) {  // the first combination keeps a tie
          best = c;
          best_err = e;
        }
      }
      for (int k = 0; k < Kb; ++k)
        if ((best >> k) & 1) word[k] |= 1u << b;
    }
  }
  // word [t][q][r][j] of the tiled layout
  const long long t = o / 32, r = o % 32, q = w / 4, j = w % 4;
  const long long off = ((t * (nw / 4) + q) * 32 + r) * 4 + j;
  for (int k = 0; k < Kb; ++k) bits[k * words_per_base + off] = word[k];
}

// ---- BiLoCo decomposition -----------------------------------------------------------

// y[o] = sum_i R[o][i] s[i] (s = +-1 as int8), one warp per row, fixed lane order; the
// sign of y goes to u (int8, zero -> +1) when u != nullptr.
__global__ void row_dot_kernel(const double* __restrict__ R, long long rows, long long cols,
                               const int8_t* __restrict__ s, long long s_stride, double* __restrict__ y,
                               int8_t* __restrict__ u, long long u_stride) {
  const long long o = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (o >= rows) return;
  double acc = 0.0;
  for (long long i = lane; i < cols; i += 32) acc += R[o * cols + i] * static_cast<double>(s[i * s_stride]);
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);
  if (lane == 0) {
    if (y) y[o] = acc;
    if (u) u[o * u_stride] = acc >= 0.0 ? 1 : -1;
  }
}

// v[i] = sign(sum_o R[o][i] u[o]), one thread per column, rows in order.
__global__ void col_dot_sign_kernel(const double* __restrict__ R, long long rows, long long cols,
                                    const int8_t* __restrict__ u, long long u_stride, int8_t* __restrict__ v) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= cols) return;
  double acc = 0.0;
  for (long long o = 0; o < rows; ++o) acc += R[o * cols + i] * static_cast<double>(u[o * u_stride]);
  v[i] = acc >= 0.0 ? 1 : -1;
}

// out = sum_o u[o] y[o] * scale, one block, fixed order (strided partial sums, then a tree).
__global__ void weighted_sum_kernel(const double* __restrict__ y, const int8_t* __restrict__ u, long long u_stride,
                                    long long n, double scale, double* __restrict__ out) {
  __shared__ double part[kQT];
  double acc = 0.0;
  for (long long o = threadIdx.x; o < n; o += kQT) acc += y[o] * static_cast<double>(u[o * u_stride]);
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int d = kQT / 2; d >= 1; d >>= 1) {
    if (threadIdx.x < d) part[threadIdx.x] += part[threadIdx.x + d];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = part[0] * scale;
}

// R[o][i] -= alpha u[o] v[i]
__global__ void rank1_update_kernel(double* __restrict__ R, long long rows, long long cols,
                                    const int8_t* __restrict__ u, long long u_stride, const int8_t* __restrict__ v,
                                    const double* __restrict__ alpha) {
  const long long id = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (id >= rows * cols) return;
  const long long o = id / cols, i = id - o * cols;
  R[id] -= *alpha * static_cast<double>(u[o * u_stride]) * static_cast<double>(v[i]);
}

// G[a][b] = (u_a . u_b)(v_a . v_b): exact integer dot products of +-1 vectors.
__global__ void gram_kernel(const int8_t* __restrict__ U, long long rows, const int8_t* __restrict__ V,
                            long long cols, int R, double* __restrict__ G) {
  const int a = blockIdx.x, b = blockIdx.y;
  __shared__ long long su[kQT], sv[kQT];
  long long du = 0, dv = 0;
  for (long long o = threadIdx.x; o < rows; o += kQT) du += U[o * R + a] * U[o * R + b];
  for (long long i = threadIdx.x; i < cols; i += kQT) dv += V[a * cols + i] * V[b * cols + i];
  su[threadIdx.x] = du;
  sv[threadIdx.x] = dv;
  __syncthreads();
  for (int d = kQT / 2; d >= 1; d >>= 1) {
    if (threadIdx.x < d) {
      su[threadIdx.x] += su[threadIdx.x + d];
      sv[threadIdx.x] += sv[threadIdx.x + d];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) G[a * R + b] = static_cast<double>(su[0]) * static_cast<double>(sv[0]);
}

// Gaussian elimination, step k: the row with the largest |G[p][k]|, p >= k, becomes row k
// (first such row on ties). One block.
__global__ void pivot_kernel(double* __restrict__ G, double* __restrict__ b, int R, int k) {
  __shared__ double best[kQT];
  __shared__ int arg[kQT];
  double bv = -1.0;
  int ba = k;
  for (int p = k + threadIdx.x; p < R; p += kQT) {
    const double a = fabs(G[p * R + k]);
    if (a > bv) { bv = a; ba = p; }
  }
  best[threadIdx.x] = bv;
  arg[threadIdx.x] = ba;
  __syncthreads();
  for (int d = kQT / 2; d >= 1; d >>= 1) {
    if (threadIdx.x < d) {
      const double o = best[threadIdx.x + d];
      const int oa = arg[threadIdx.x + d];
      if (o > best[threadIdx.x] || (o == best[threadIdx.x] && oa < arg[threadIdx.x])) {
        best[threadIdx.x] = o;
        arg[threadIdx.x] = oa;
      }
    }
    __syncthreads();
  }
  const int p = arg[0];
  if (p != k) {
    for (int j = threadIdx.x; j < R; j += kQT) {
      const double t = G[k * R + j];
      G[k * R + j] = G[p * R + j];
      G[p * R + j] = t;
    }
    if (threadIdx.x == 0) {
      const double t = b[k];
      b[k] = b[p];
      b[p] = t;
    }
  }
}

// Step k: rows i > k lose G[i][k] / G[k][k] times row k, in columns j > k (column k
// below the diagonal is never read again, and leaving it unwritten keeps the factor
// G[i][k] intact for every thread of the step). Block y = row i - k - 1.
__global__ void eliminate_kernel(double* __restrict__ G, double* __restrict__ b, int R, int k) {
  const int i = k + 1 + blockIdx.y;
  if (i >= R) return;
  const double f = G[i * R + k] / G[k * R + k];
  for (int j = k + 1 + blockIdx.x * blockDim.x + threadIdx.x; j < R; j += gridDim.x * blockDim.x)
    G[i * R + j] -= f * G[k * R + j];
  if (blockIdx.x == 0 && threadIdx.x == 0) b[i] -= f * b[k];
}

// Back substitution, one block: x[k] = (b[k] - sum_{j>k} G[k][j] x[j]) / G[k][k].
__global__ void back_substitute_kernel(const double* __restrict__ G, const double* __restrict__ b, int R,
                                       double* __restrict__ x) {
  __shared__ double part[kQT];
  for (int k = R - 1; k >= 0; --k) {
    double acc = 0.0;
    for (int j = k + 1 + threadIdx.x; j < R; j += kQT) acc += G[k * R + j] * x[j];
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int d = kQT / 2; d >= 1; d >>= 1) {
      if (threadIdx.x < d) part[threadIdx.x] += part[threadIdx.x + d];
      __syncthreads();
    }
    if (threadIdx.x == 0) x[k] = (b[k] - part[0]) / G[k * R + k];
    __syncthreads();
  }
}

size_t a256(size_t n) { return (n + 255) & ~size_t(255); }

// Workspace: residual [rows][cols], row sums [rows], G [R][R], b [R].
size_t biloco_ws(long long rows, long long cols, int R) {
  return a256(static_cast<size_t>(rows) * cols * 8) + a256(static_cast<size_t>(rows) * 8) +
         a256(static_cast<size_t>(R) * R * 8) + a256(static_cast<size_t>(R) * 8);
}

unsigned blocks_for(long long n, int per) { return static_cast<unsigned>((n + per - 1) / per); }

}  // namespace
}  // namespace bisco

using namespace bisco;

extern "C" {

bisco_status bisco_fluxbin_signs(const double* W, int64_t rows, int64_t cols, int32_t Kb, const double* row_scale,
                                 const double* col_scale, int32_t group, uint32_t* bits, void* stream) {
  if (!W || !row_scale || !col_scale || !bits || rows < 1 || cols < 1 || Kb < 1 || Kb > 8 || group < 0)
    return BISCO_ERR_INVALID_ARG;
  if (rows > (1ll << 31) || cols > (1ll << 31)) return BISCO_ERR_INVALID_ARG;
  const long long nw = (cols + 127) / 128 * 4, tiles = (rows + 31) / 32;
  const long long threads = tiles * 32 * nw;
  const long long ngroups = group > 0 ? (cols + group - 1) / group : 1;
  fluxbin_signs_kernel<<<blocks_for(threads, kQT), kQT, 0, static_cast<cudaStream_t>(stream)>>>(
      W, rows, cols, Kb, row_scale, col_scale, group, ngroups, bits, bisco_packed_words(rows, cols));
  return cudaGetLastError() == cudaSuccess ? BISCO_OK : BISCO_ERR_CUDA;
}

bisco_status bisco_biloco_workspace_size(int64_t rows, int64_t cols, int32_t rank, size_t* bytes) {
  if (!bytes || rows < 1 || cols < 1 || rank < 1 || rank > 4096) return BISCO_ERR_INVALID_ARG;
  *bytes = biloco_ws(rows, cols, rank);
  return BISCO_OK;
}

bisco_status bisco_biloco_decompose(const double* W, int64_t rows, int64_t cols, int32_t rank, int32_t rounds,
                                    const int8_t* v0, int8_t* U, int8_t* V, double* alpha_greedy,
                                    double* alpha_refit, void* ws, size_t ws_bytes, void* stream) {
  if (!W || !v0 || !U || !V || !alpha_greedy || !alpha_refit || !ws || rows < 1 || cols < 1 || rank < 1 ||
      rank > 4096 || rounds < 1)
    return BISCO_ERR_INVALID_ARG;
  if (ws_bytes < biloco_ws(rows, cols, rank)) return BISCO_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* p = static_cast<unsigned char*>(ws);
  double* Rs = reinterpret_cast<double*>(p);
  p += a256(static_cast<size_t>(rows) * cols * 8);
  double* y = reinterpret_cast<double*>(p);
  p += a256(static_cast<size_t>(rows) * 8);
  double* G = reinterpret_cast<double*>(p);
  p += a256(static_cast<size_t>(rank) * rank * 8);
  double* bvec = reinterpret_cast<double*>(p);
  if (cudaMemcpyAsync(Rs, W, static_cast<size_t>(rows) * cols * 8, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return BISCO_ERR_CUDA;
  const unsigned rblk = blocks_for(rows * 32, kQT), cblk = blocks_for(cols, kQT), eblk = blocks_for(rows * cols, kQT);
  const double inv = 1.0 / (static_cast<double>(rows) * static_cast<double>(cols));
  for (int j = 0; j < rank; ++j) {
    int8_t* u = U + j;          // column j of U [rows][rank]
    int8_t* v = V + static_cast<long long>(j) * cols;
    if (cudaMemcpyAsync(v, v0 + static_cast<long long>(j) * cols, cols, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return BISCO_ERR_CUDA;
    // the starting signs are taken as sign(v0): entries are +-1 already
    for (int r = 0; r < rounds; ++r) {
      row_dot_kernel<<<rblk, kQT, 0, s>>>(Rs, rows, cols, v, 1, nullptr, u, rank);
      col_dot_sign_kernel<<<cblk, kQT, 0, s>>>(Rs, rows, cols, u, rank, v);
    }
    row_dot_kernel<<<rblk, kQT, 0, s>>>(Rs, rows, cols, v, 1, y, nullptr, 0);
    weighted_sum_kernel<<<1, kQT, 0, s>>>(y, u, rank, rows, inv, alpha_greedy + j);
    rank1_update_kernel<<<eblk, kQT, 0, s>>>(Rs, rows, cols, u, rank, v, alpha_greedy + j);
  }
  // refit: b_j = u_j^T W v_j, G = (U^T U) o (V V^T), G alpha = b
  for (int j = 0; j < rank; ++j) {
    row_dot_kernel<<<rblk, kQT, 0, s>>>(W, rows, cols, V + static_cast<long long>(j) * cols, 1, y, nullptr, 0);
    weighted_sum_kernel<<<1, kQT, 0, s>>>(y, U + j, rank, rows, 1.0, bvec + j);
  }
  gram_kernel<<<dim3(rank, rank), kQT, 0, s>>>(U, rows, V, cols, rank, G);
  for (int k = 0; k < rank - 1; ++k) {
    pivot_kernel<<<1, kQT, 0, s>>>(G, bvec, rank, k);
    eliminate_kernel<<<dim3(blocks_for(rank - k - 1, kQT), rank - k - 1), kQT, 0, s>>>(G, bvec, rank, k);
  }
  back_substitute_kernel<<<1, kQT, 0, s>>>(G, bvec, rank, alpha_refit);
  return cudaGetLastError() == cudaSuccess ? BISCO_OK : BISCO_ERR_CUDA;
}

}  // extern "C"

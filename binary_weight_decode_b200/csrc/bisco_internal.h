// Internal declarations shared by the C-ABI front end and the CUDA kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/bisco.h"

namespace bisco {

constexpr int kWarps = 4;                 // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kFields = 26;               // 5-bit fields per 128-column quad: 25 of 5 bits + 1 of 3 bits
constexpr int kFieldStride = 36;          // floats from one field's 32-entry table to the next
constexpr int kMaxSeg = 6;                // K <= 4 bases + the U^T segment (+ a spare)
constexpr int kMaxBases = 4;
constexpr int kMaxBatchChunk = 8;         // batch rows handled by one launch
constexpr int kStatusBytes = 256;         // status word region at the start of the workspace

// One segment of a pass: a packed sign matrix whose columns multiply one input vector.
struct SegParam {
  const uint4* bits;     // packed [tiles][nq][32][4] words, as uint4 per (row, quad)
  const void* cscale;    // column scale [ncols] or nullptr
  const void* rscale;    // row scale [rows] or nullptr (= 1)
  int nq;                // quads per row = ceil(ncols / 128)
  int ncols;             // columns (input features) of this segment
  int unit0;             // index of this segment's first quad in the pass's unit list
  int xsrc;              // 0: X, 1: Z (fp32 workspace vector), 2: none (zeros)
  int cdt;               // dtype of cscale
  int rdt;               // dtype of rscale
};

// One launch of the LUT GEMV kernel.
struct PassParam {
  SegParam seg[kMaxSeg];
  int nseg;
  int rows;              // output rows of the pass
  int tiles;             // ceil(rows / 32)
  int units;             // total quads over segments
  int G;                 // row tiles per block (multiple of kWarps)
  int nblocks;           // ceil(tiles / G)
  long long L;           // linear work items = nblocks * units * G
  int P;                 // CTAs
  int Mc;                // valid batch rows in this launch (<= MB)
  int max_cols;          // table slots per CTA (smem sizing)
  int col_stride_bytes;  // bytes of tables per slot (multiple of 128)
  // activations
  const void* X; int xdt; long long ldx;   // X[m][i] at X + m*ldx + i (elements)
  int xcols;             // columns of X (salient indices must be below it)
  const float* Z; long long ldz;
  // output
  void* Y; int ydt; long long ldy;
  // salient columns (added once per output row)
  int n_sal, sal_stride;
  const int* sal_idx; const int8_t* sal_q; const float* sal_scale;
  // workspace
  float* part;           // [P][2][MB][G*32]
  int* cnt;              // [nblocks]
  int* status;
};

struct Plan {
  int G, P, nblocks, max_cols, col_stride_bytes, MB;
  long long L;
  size_t smem;
  size_t part_floats, cnt_ints;
};

Plan make_plan(int rows, int units, int MB, int n_sal, int num_sms, size_t smem_limit);
cudaError_t launch_pass(const PassParam& p, const Plan& plan, cudaStream_t stream, bool pdl);
// Sets per-kernel attributes once per device; call before any stream capture.
cudaError_t ensure_kernel_attrs();

int query_num_sms();
size_t query_smem_limit();

}  // namespace bisco

// Internal declarations shared by the C-ABI front end and the CUDA kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/bisco.h"

namespace bisco {

constexpr int kWarps = 8;                 // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kFields = 26;               // fields per 128-column quad: 25 of 5 bits + 1 of 3 bits
constexpr int kFieldStride = 36;          // floats from one field's 32-entry table to the next
constexpr int kMaxSeg = 6;                // K <= 4 bases + the U^T segment (+ a spare)
constexpr int kMaxBases = 4;
constexpr int kMaxCluster = 8;            // CTAs per cluster (portable limit)
constexpr int kMaxBatchChunk = 8;         // batch rows handled by one launch
constexpr int kStatusBytes = 256;         // status word region at the start of the workspace

// One segment of a pass: a packed sign matrix whose columns multiply one input vector.
struct SegParam {
  const uint4* bits;     // packed [tiles][nq][32][4] words, as one uint4 per (row, quad)
  const void* cscale;    // column scale [ncols] or nullptr (= 1)
  const void* rscale;    // row scale [rows] or nullptr (= 1)
  int nq;                // quads per row = ceil(ncols / 128)
  int ncols;             // columns (input features) of this segment
  int unit0;             // index of this segment's first quad in the pass's unit list
  int xsrc;              // 0: X, 1: Z (fp32 workspace vector), 2: none (zeros)
  int cdt;               // dtype of cscale
  int rdt;               // dtype of rscale
  int cvec, rvec;        // 1 if cscale / rscale are 16-byte aligned (vector loads allowed)
  int rgu;               // grouped row scales: quads per group (0: one scale per row)
  int rgstride;          // elements between the row-scale vectors of consecutive groups
  int part0;             // pass-wide index of the segment's first (segment, group) part
};

// One launch of the cluster LUT GEMV kernel.
//
// Grid: ncl clusters of C CTAs. Cluster c owns row tiles [c*tiles/ncl, (c+1)*tiles/ncl);
// CTA r of a cluster owns units (128-column quads over all segments)
// [r*units/C, (r+1)*units/C) and builds lookup tables for them only. The C partial
// sums of a row meet in distributed shared memory.
struct PassParam {
  SegParam seg[kMaxSeg];
  int nseg;
  int rows;              // output rows of the pass
  int tiles;             // ceil(rows / 32)
  int units;             // total quads over segments
  int C;                 // CTAs per cluster
  int ncl;               // clusters
  int max_tiles;         // max row tiles of a cluster
  int max_units;         // max units of a CTA
  int max_lseg;          // max segments a CTA's unit range touches
  int Mc;                // valid batch rows in this launch (<= MB)
  int col_stride_bytes;  // bytes of tables per unit (multiple of 128)
  // activations
  const void* X; int xdt; int ldx;          // X[m][i] at X + m*ldx + i (elements)
  int xcols;             // columns of X (salient indices must be below it)
  const float* Z; int ldz;
  int x_vec, z_vec;      // 1 if rows of X (resp. Z) allow 16-byte vector loads
  // output
  void* Y; int ydt; int ldy;
  // salient columns (added once per output row)
  int n_sal, sal_stride;
  const int* sal_idx; const int8_t* sal_q; const float* sal_scale;
  const float* rref;     // [Mc][rows] salient refinement term to add (integer kernel), or nullptr
  int* status;           // device status word (workspace)
};

struct Plan {
  int C, ncl, max_tiles, max_units, max_lseg, col_stride_bytes, MB;
  int cu;                // units per table chunk
  int kind;              // 0: 16-warp kernel, 2: streaming kernel (batch rows <= 2); 1: warps own row tiles (4, 8)
  int ns;                // streaming kernel: shared-memory ring slots (one (chunk, tile) stage each)
  int gu;                // streaming kernel: unit groups of the 16 consumer warps
  size_t smem;
};

// seg_unit0[k] = first unit of segment k (k < nseg); used to count segments per CTA.
Plan make_plan(int rows, int units, const int* seg_unit0, int nseg, int MB, int n_sal, int num_sms,
               size_t smem_limit);
cudaError_t launch_pass(const PassParam& p, const Plan& plan, cudaStream_t stream, bool pdl);
// Sets per-kernel attributes once per device; call before any stream capture.
cudaError_t ensure_kernel_attrs();

int query_num_sms();
size_t query_smem_limit();

// Integer tensor-core GEMV (mma.sync u8 x s8) for batch chunks of up to 8 rows.
// Roles of one integer-kernel launch: passes that run side by side on disjoint clusters.
// A launch of one role is a plain pass; with several, z passes come first and the output
// passes that read a z wait (bounded) for its CTAs to count themselves done.
constexpr int kMaxRoles = 6;  // three layers sharing x, each with a correction
struct RoleTable {
  int nroles;
  int cl0[kMaxRoles + 1];  // first cluster of role r; cl0[nroles] = clusters of the grid
  int zsrc[kMaxRoles];     // output role: the role computing the z it reads, or -1
  int is_z[kMaxRoles];     // 1 if the role computes a z (it counts itself ready)
};
struct ImmaLaunch {
  PassParam pass[kMaxRoles];
  RoleTable rt;
};

struct ImmaPlan {
  int C;                 // cluster size (K split); C == 0: no plan fits
  int nroles;
  int ncl[kMaxRoles];    // clusters of each role
  int max_tiles;         // 32-row tiles of the largest cluster share (over roles)
  int max_units;         // 128-column units of the largest CTA share
  int max_lseg;          // (segment, row-scale group) parts a CTA's unit range touches, at most
  int nbw;               // partial-sum slots per row and CTA (warps whose items touch one row block)
  int MB;                // batch rows per launch (1, 2, 4 or 8)
  size_t smem;
};
// Test hooks of the bounded device-side waits: skip_tile >= 0 leaves sign-word copies
// unissued (the integer kernel: those of local row tile skip_tile; the tcgen05 kernel:
// those of each CTA's last step), so their waiters give up after wait_ns and report
// BISCO_ERR_TIMEOUT.
struct ImmaDebug {
  int skip_tile;
  unsigned long long wait_ns;
};
constexpr unsigned long long kDefaultWaitNs = 200000000ull;  // bound on every mbarrier wait (200 ms)
// Rows and the 128-column units of a pass, with the first unit of each segment.
struct ImmaShape {
  int rows, units;
  const int* seg_unit0;
  int nseg;
  const int* seg_rgu;  // per segment: quads per row-scale group (0: none); may be null
};
// One role of a launch: its shape, salient columns, and (output passes reading a z) the
// first unit of the U^T segment, else -1.
struct ImmaRole {
  ImmaShape sh;
  int n_sal;
  int u_split;
};
// Clusters per role (each at least one, then one at a time to the role with the largest
// share per cluster), cluster size from a cycle estimate, shared-memory maxima over roles.
ImmaPlan make_imma_plan(const ImmaRole* roles, int nroles, int MB, size_t smem_limit);
// L.pass[r] holds role r's pass with the plan's maxima filled in; L.rt its role table.
cudaError_t launch_imma(const ImmaLaunch& L, const ImmaPlan& plan, cudaStream_t stream, bool pdl, const ImmaDebug* dbg);
// One launch of the salient refinement kernel: rref[m][o] for the Mc batch rows of X
// (grid: one CTA per 32-row tile of the output).
struct RefineParam {
  const uint32_t* bits;   // [Ks][packed words of out x n_ref]
  const void* rrs;        // row scales [Ks][ngroups][out]
  const void* rcs;        // column scales [Ks][n_ref]
  int sdt;                // dtype of both scales
  const int* idx;         // [n_ref] ascending input columns
  int Ks, n_ref, in, out, g, ngroups, tiles;
  const void* X; int xdt; int ldx;
  int Mc;
  float* rref;            // [Mc][out]
  int* status;
};
// Shared memory of one refinement launch at batch block MB (0 for a layer without one).
size_t refine_smem_bytes(const bisco_layer* L, int MB);
// The salient refinement term of a layer for Mc batch rows of X into rref [Mc][out] (fp32).
cudaError_t launch_refine(const bisco_layer* L, const void* X, int32_t x_dtype, int Mc, float* rref, int* status,
                          cudaStream_t stream);
cudaError_t imma_ensure_attrs();

// Tensor-core path (16..128 batch rows per launch): one launch per pass.
constexpr int kTcMinBatch = 16;           // smallest batch chunk sent to the tensor cores
constexpr int kTcMaxBatch = 128;          // batch rows per launch
struct TcPlan {
  int Np;                // batch rows padded to a multiple of 16 (MMA N per part)
  int a_base;            // first tensor-memory column of the expanded sign tiles (after the accumulators)
  int astages;           // sign-tile stages in tensor memory (64 columns each)
  int stages;            // activation-tile stages in shared memory
  int raw_slots;         // sign-word ring slots in shared memory (one step each)
  int tiles;             // 128-row output tiles (clusters)
  int S;                 // CTAs per cluster (K split); 0 = plan not possible
  size_t smem;
};
// seg_kind[s] is SegParam::xsrc of segment s; seg_ncols[s] its columns.
TcPlan make_tc_plan(int rows, int nseg, const int* seg_kind, const int* seg_ncols, int n_sal, bool x_bf16, int Mc,
                    int num_sms, size_t smem_limit);
cudaError_t launch_tc(const PassParam& p, const TcPlan& t, cudaStream_t stream, const ImmaDebug* dbg);
cudaError_t tc_ensure_attrs();

}  // namespace bisco

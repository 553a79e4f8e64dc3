// C ABI front end: argument validation, host packing, workspace sizing and the launch
// sequence of bisco_gemv and bisco_gemv_group.
//
// A layer with a binary low-rank correction ("BiLoCo", "The core idea": the
// correction is applied as alpha * u * (v . x)) has two passes: pass Z computes
// z = alpha (.) (V x) into the workspace, pass Y computes
// sum_k r_k (.) (B_k (c_k (.) x)) + U^T z + salient term into Y. On the integer kernel
// both run in one launch (z clusters first, output clusters wait for them, bounded);
// on the other kernels as two launches, pass Y reading z after griddepcontrol.wait.
//
// The batch is cut into chunks: up to 128 rows per launch on the tensor-core path
// (tcgen05) when a chunk has at least 16 rows (and the scales are bf16, so that folding
// a column scale into the expanded signs is exact), otherwise up to 8 rows per launch on
// the integer tensor-core kernel (mma.sync, bisco_imma.cu) when its shared-memory plan
// fits, else on the lookup-table kernels. Single rows of layers without a correction
// take the lookup-table kernels.

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "bisco_internal.h"

using namespace bisco;

namespace {

constexpr int kMaxDevices = 64;

// Path policy (bisco_set_path_policy) and the integer kernel's test hooks
// (bisco_debug_set_wait_test); both are process-wide.
std::atomic<int> g_policy{BISCO_PATH_AUTO};
std::atomic<int> g_dbg_skip_tile{-1};
std::atomic<unsigned long long> g_dbg_wait_ns{0};

int cached_sms(int dev) {
  static int sms[kMaxDevices] = {0};
  if (dev < 0 || dev >= kMaxDevices) return query_num_sms();
  if (sms[dev] == 0) sms[dev] = query_num_sms();
  return sms[dev];
}

size_t cached_smem_limit(int dev) {
  static size_t lim[kMaxDevices] = {0};
  if (dev < 0 || dev >= kMaxDevices) return query_smem_limit();
  if (lim[dev] == 0) lim[dev] = query_smem_limit();
  return lim[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(int32_t d) { return d == BISCO_F32 || d == BISCO_BF16; }
size_t dtype_bytes(int32_t d) { return d == BISCO_BF16 ? 2 : 4; }
size_t align256(size_t n) { return (n + 255) / 256 * 256; }
int quads(int n) { return (n + 127) / 128; }

bisco_status validate_layer(const bisco_layer* L) {
  if (!L) return BISCO_ERR_INVALID_ARG;
  if (L->out < 1 || L->in < 1 || L->num_bases < 0 || L->num_bases > kMaxBases) return BISCO_ERR_INVALID_ARG;
  if (L->rank < 0 || L->rank > (1 << 20) || L->n_sal < 0 || L->n_sal > L->in) return BISCO_ERR_INVALID_ARG;
  if (L->row_group < 0) return BISCO_ERR_INVALID_ARG;
  if (L->num_bases > 0) {
    if (!L->bits || !L->row_scale || !L->col_scale || !aligned16(L->bits)) return BISCO_ERR_INVALID_ARG;
    if (!dtype_ok(L->scale_dtype)) return BISCO_ERR_INVALID_ARG;
  }
  if (L->rank > 0) {
    if (!L->v_bits || !L->ut_bits || !L->alpha) return BISCO_ERR_INVALID_ARG;
    if (!aligned16(L->v_bits) || !aligned16(L->ut_bits)) return BISCO_ERR_INVALID_ARG;
  }
  if (L->n_sal > 0) {
    if (!L->sal_idx || !L->sal_q || !L->sal_scale || !aligned16(L->sal_q)) return BISCO_ERR_INVALID_ARG;
    if (L->sal_stride < L->n_sal || (L->sal_stride % 16) != 0) return BISCO_ERR_INVALID_ARG;
  }
  if (L->ref_bases < 0 || L->ref_bases > kMaxBases) return BISCO_ERR_INVALID_ARG;
  if (L->ref_bases > 0) {
    if (L->row_group < 1 || L->n_ref < 1 || L->n_ref > L->in || !dtype_ok(L->scale_dtype)) return BISCO_ERR_INVALID_ARG;
    if (!L->ref_idx || !L->ref_bits || !L->ref_row_scale || !L->ref_col_scale || !aligned16(L->ref_bits))
      return BISCO_ERR_INVALID_ARG;
  }
  return BISCO_OK;
}

int batch_block(int Mc) { return Mc <= 1 ? 1 : Mc <= 2 ? 2 : Mc <= 4 ? 4 : 8; }

// Segment list of pass Y: K binary bases, then U^T if the layer has a correction;
// a layer with neither gets one empty unit so the salient term still has a home.
struct SegList {
  int unit0[kMaxSeg];
  int rgu[kMaxSeg];  // quads per row-scale group (0: one row scale per row)
  int nseg, units;
};

// Quads per row-scale group of the bases (0 without grouped row scales).
int row_group_quads(const bisco_layer* L) { return L->row_group > 0 ? L->row_group / 128 : 0; }

SegList segs_y(const bisco_layer* L) {
  SegList s{};
  for (int k = 0; k < L->num_bases; ++k) {
    s.rgu[s.nseg] = row_group_quads(L);
    s.unit0[s.nseg++] = s.units;
    s.units += quads(L->in);
  }
  if (L->rank > 0) { s.rgu[s.nseg] = 0; s.unit0[s.nseg++] = s.units; s.units += quads(L->rank); }
  if (s.nseg == 0) { s.rgu[s.nseg] = 0; s.unit0[s.nseg++] = 0; s.units = 1; }
  return s;
}

struct Layout {
  Plan pz, py;          // lookup-table plans
  ImmaPlan iz, iy;      // integer tensor-core plans (C == 0: none fits)
  ImmaPlan ifz;         // both passes of a layer with a correction in one integer launch
  bool has_z;
  size_t off_z, total;
};

Layout layout_for(const bisco_layer* L, int MB, int dev) {
  Layout lo{};
  const int sms = cached_sms(dev);
  const size_t lim = cached_smem_limit(dev);
  lo.has_z = L->rank > 0;
  const SegList sy = segs_y(L);
  lo.py = make_plan(L->out, sy.units, sy.unit0, sy.nseg, MB, L->n_sal, sms, lim);
  const ImmaShape ys{L->out, sy.units, sy.unit0, sy.nseg, sy.rgu};
  const ImmaRole ry{ys, L->n_sal, -1};
  lo.iy = make_imma_plan(&ry, 1, MB, lim);
  if (lo.has_z) {
    const int z0 = 0;
    lo.pz = make_plan(L->rank, quads(L->in), &z0, 1, MB, 0, sms, lim);
    const ImmaShape zs{L->rank, quads(L->in), &z0, 1, nullptr};
    const ImmaRole rz{zs, 0, -1};
    lo.iz = make_imma_plan(&rz, 1, MB, lim);
    const ImmaRole rf[2] = {rz, ImmaRole{ys, L->n_sal, sy.unit0[sy.nseg - 1]}};
    lo.ifz = make_imma_plan(rf, 2, MB, lim);
  }
  lo.off_z = kStatusBytes;
  lo.total = lo.off_z + align256(lo.has_z ? static_cast<size_t>(kMaxBatchChunk) * L->rank * 4 : 0);
  return lo;
}

// Plans depend only on shapes and the device: cache them so that a call does not
// re-run the occupancy queries.
Layout cached_layout(const bisco_layer* L, int MB, int dev) {
  struct Key {
    int dev, out, in, K, rank, n_sal, MB, rg;
    bool operator==(const Key& o) const {
      return dev == o.dev && out == o.out && in == o.in && K == o.K && rank == o.rank && n_sal == o.n_sal &&
             MB == o.MB && rg == o.rg;
    }
  };
  struct Entry { Key k; Layout lo; };
  static std::mutex mu;
  static std::vector<Entry>* cache = new std::vector<Entry>();
  const Key k{dev, L->out, L->in, L->num_bases, L->rank, L->n_sal, MB, L->row_group};
  std::lock_guard<std::mutex> g(mu);
  for (const Entry& e : *cache)
    if (e.k == k) return e.lo;
  if (cache->size() > 4096) cache->clear();
  cache->push_back(Entry{k, layout_for(L, MB, dev)});
  return cache->back().lo;
}

// Workspace bytes: the status word, with a correction z for one batch chunk, and with a
// salient refinement that term for one 8-row chunk (after z of 8 rows).
// ws_need is the minimum bisco_gemv accepts (chunks of 8 rows); ws_pref also lets the
// tensor-core path take chunks of up to 128 rows for this batch size.
size_t ref_offset(const bisco_layer* L) {
  return kStatusBytes + align256(L->rank > 0 ? static_cast<size_t>(kMaxBatchChunk) * L->rank * 4 : 0);
}
size_t ws_need(const bisco_layer* L, int32_t) {
  return ref_offset(L) + align256(L->ref_bases > 0 ? static_cast<size_t>(kMaxBatchChunk) * L->out * 4 : 0);
}
size_t ws_pref(const bisco_layer* L, int32_t M) {
  if (L->ref_bases > 0) return ws_need(L, M);  // refined layers run in 8-row integer chunks only
  // z rows of a tensor-core chunk (padded to 16; from 8 batch rows up a chunk may go to
  // the tensor cores when the integer plan does not fit)
  const int rows = M < kMaxBatchChunk ? kMaxBatchChunk : std::min<int>((M + 15) / 16 * 16, kTcMaxBatch);
  return kStatusBytes + align256(L->rank > 0 ? static_cast<size_t>(rows) * L->rank * 4 : 0);
}

bool plans_fit(const Layout& lo, size_t lim) {
  return lo.py.smem <= lim && (!lo.has_z || lo.pz.smem <= lim);
}

bool imma_fits(const Layout& lo) { return lo.iy.C > 0 && (!lo.has_z || lo.iz.C > 0); }

void fill_plan(PassParam& P, const Plan& pl) {
  P.C = pl.C; P.ncl = pl.ncl; P.max_tiles = pl.max_tiles; P.max_units = pl.max_units;
  P.max_lseg = pl.max_lseg; P.col_stride_bytes = pl.col_stride_bytes;
}

// ncl: the clusters of this pass (a launch with several roles splits its grid between
// them; they share the plan's shared-memory maxima)
void fill_imma(PassParam& P, const ImmaPlan& pl, int ncl) {
  P.C = pl.C; P.ncl = ncl; P.max_tiles = pl.max_tiles; P.max_units = pl.max_units;
  P.max_lseg = pl.max_lseg; P.col_stride_bytes = 0;
}

// One integer launch of n passes in plan order: zsrc[r] is the role whose z role r reads
// (-1: none), is_z[r] marks the roles that compute a z.
cudaError_t run_imma(PassParam* passes, const int* zsrc, const int* is_z, int n, const ImmaPlan& pl, cudaStream_t s,
                     const ImmaDebug* dbg) {
  ImmaLaunch L{};
  L.rt.nroles = n;
  int c = 0;
  for (int r = 0; r < n; ++r) {
    fill_imma(passes[r], pl, pl.ncl[r]);
    L.pass[r] = passes[r];
    L.rt.cl0[r] = c;
    c += pl.ncl[r];
    L.rt.zsrc[r] = zsrc ? zsrc[r] : -1;
    L.rt.is_z[r] = is_z ? is_z[r] : 0;
  }
  L.rt.cl0[n] = c;
  return launch_imma(L, pl, s, true, dbg);
}


// Segments of pass Z: V (rows = rank) over X, row scale alpha.
void pass_z(const bisco_layer* L, PassParam& pz, const void* Xc, int32_t x_dtype, int Mc, float* zbuf, int* status) {
  const size_t xb = dtype_bytes(x_dtype);
  pz.nseg = 1;
  SegParam& V = pz.seg[0];
  V.bits = reinterpret_cast<const uint4*>(L->v_bits);
  V.nq = quads(L->in);
  V.ncols = L->in;
  V.unit0 = 0;
  V.xsrc = 0;
  V.cscale = nullptr;
  V.cdt = BISCO_F32;
  V.rscale = L->alpha;
  V.rdt = BISCO_F32;
  V.cvec = 0;
  V.rvec = aligned16(L->alpha);
  V.rgu = 0;
  V.rgstride = 0;
  V.part0 = 0;
  pz.rows = L->rank;
  pz.tiles = (L->rank + 31) / 32;
  pz.units = V.nq;
  pz.Mc = Mc;
  pz.X = Xc; pz.xdt = x_dtype; pz.ldx = L->in; pz.xcols = L->in;
  pz.Z = nullptr; pz.ldz = 0;
  pz.x_vec = aligned16(Xc) && (static_cast<size_t>(L->in) * xb) % 16 == 0;
  pz.z_vec = 0;
  pz.Y = zbuf; pz.ydt = BISCO_F32; pz.ldy = L->rank;
  pz.n_sal = 0; pz.sal_stride = 0;
  pz.status = status;
}

// Segments of pass Y: the K binary bases over c_k (.) X, then U^T over z; a layer with
// neither gets one empty unit so that the salient term still has a home.
void pass_y(const bisco_layer* L, PassParam& py, const void* Xc, int32_t x_dtype, int Mc, void* Yc, int32_t y_dtype,
            float* zbuf, int* status) {
  const size_t xb = dtype_bytes(x_dtype);
  int nseg = 0, unit = 0, parts = 0;
  for (int k = 0; k < L->num_bases; ++k) {
    SegParam& B = py.seg[nseg++];
    B.bits = reinterpret_cast<const uint4*>(L->bits + static_cast<size_t>(k) * bisco_packed_words(L->out, L->in));
    B.nq = quads(L->in);
    B.ncols = L->in;
    B.unit0 = unit;
    unit += B.nq;
    B.xsrc = 0;
    B.cscale = static_cast<const unsigned char*>(L->col_scale) + static_cast<size_t>(k) * L->in * dtype_bytes(L->scale_dtype);
    B.cdt = L->scale_dtype;
    const size_t ngroups = L->row_group > 0 ? (static_cast<size_t>(L->in) + L->row_group - 1) / L->row_group : 1;
    B.rscale = static_cast<const unsigned char*>(L->row_scale) +
               static_cast<size_t>(k) * ngroups * L->out * dtype_bytes(L->scale_dtype);
    B.rdt = L->scale_dtype;
    B.rgu = row_group_quads(L);
    B.rgstride = L->out;
    B.part0 = parts;
    parts += B.rgu > 0 ? (B.nq + B.rgu - 1) / B.rgu : 1;
    B.cvec = aligned16(B.cscale);
    // vector loads of a group's scale vector need every group offset 16-byte aligned too
    B.rvec = aligned16(B.rscale) && (B.rgu == 0 || (static_cast<size_t>(L->out) * dtype_bytes(L->scale_dtype)) % 16 == 0);
  }
  if (L->rank > 0) {
    SegParam& U = py.seg[nseg++];
    U.bits = reinterpret_cast<const uint4*>(L->ut_bits);
    U.nq = quads(L->rank);
    U.ncols = L->rank;
    U.unit0 = unit;
    unit += U.nq;
    U.xsrc = 1;
    U.cscale = nullptr;
    U.cdt = BISCO_F32;
    U.rscale = nullptr;
    U.rdt = BISCO_F32;
    U.cvec = U.rvec = 0;
    U.rgu = 0;
    U.rgstride = 0;
    U.part0 = parts++;
  }
  if (nseg == 0) {  // salient-only (or empty) layer: one empty unit
    SegParam& E = py.seg[nseg++];
    E.bits = nullptr; E.nq = 1; E.ncols = 0; E.unit0 = 0; E.xsrc = 2;
    E.cscale = nullptr; E.rscale = nullptr; E.cdt = E.rdt = BISCO_F32;
    E.cvec = E.rvec = 0;
    E.rgu = 0;
    E.rgstride = 0;
    E.part0 = 0;
    unit = 1;
  }
  py.nseg = nseg;
  py.rows = L->out;
  py.tiles = (L->out + 31) / 32;
  py.units = unit;
  py.Mc = Mc;
  py.X = Xc; py.xdt = x_dtype; py.ldx = L->in; py.xcols = L->in;
  py.Z = zbuf; py.ldz = L->rank;
  py.x_vec = aligned16(Xc) && (static_cast<size_t>(L->in) * xb) % 16 == 0;
  py.z_vec = (L->rank % 4) == 0;
  py.Y = Yc; py.ydt = y_dtype; py.ldy = L->out;
  py.n_sal = L->n_sal; py.sal_stride = L->sal_stride;
  py.sal_idx = L->sal_idx; py.sal_q = L->sal_q; py.sal_scale = L->sal_scale;
  py.status = status;
}

// One batch chunk and how it runs.
struct Chunk {
  int m0, Mc;
  bool tc;         // tcgen05 tensor-core kernel
  bool imma;       // integer tensor-core kernel (mma.sync); else the lookup-table kernels
  bool fused;      // imma with both passes in one launch
  Layout lo;       // lookup-table and integer plans (tc == false)
  TcPlan tz, ty;   // tensor-core plans (tc == true)
};

// Tensor-core plans for a chunk of Mc rows, cached like the lookup-table layouts.
bool tc_plans(const bisco_layer* L, int Mc, int32_t x_dtype, int dev, TcPlan* tz, TcPlan* ty) {
  struct Key {
    int dev, out, in, K, rank, n_sal, Np, xdt;
    bool operator==(const Key& o) const {
      return dev == o.dev && out == o.out && in == o.in && K == o.K && rank == o.rank && n_sal == o.n_sal &&
             Np == o.Np && xdt == o.xdt;
    }
  };
  struct Entry { Key k; TcPlan z, y; };
  static std::mutex mu;
  static std::vector<Entry>* cache = new std::vector<Entry>();
  const Key k{dev, L->out, L->in, L->num_bases, L->rank, L->n_sal, (Mc + 15) / 16 * 16, x_dtype};
  {
    std::lock_guard<std::mutex> g(mu);
    for (const Entry& e : *cache)
      if (e.k == k) { *tz = e.z; *ty = e.y; return ty->S > 0 && (L->rank == 0 || tz->S > 0); }
  }
  const int sms = cached_sms(dev);
  const size_t lim = cached_smem_limit(dev);
  const bool xbf = x_dtype == BISCO_BF16;
  TcPlan z{}, y{};
  if (L->rank > 0) {
    const int kind = 0, ncols = L->in;
    z = make_tc_plan(L->rank, 1, &kind, &ncols, 0, xbf, Mc, sms, lim);
  }
  int kinds[kMaxSeg], ncols[kMaxSeg], nseg = 0;
  for (int b = 0; b < L->num_bases; ++b) { kinds[nseg] = 0; ncols[nseg++] = L->in; }
  if (L->rank > 0) { kinds[nseg] = 1; ncols[nseg++] = L->rank; }
  if (nseg == 0) { kinds[nseg] = 2; ncols[nseg++] = 0; }
  y = make_tc_plan(L->out, nseg, kinds, ncols, L->n_sal, xbf, Mc, sms, lim);
  std::lock_guard<std::mutex> g(mu);
  if (cache->size() > 4096) cache->clear();
  cache->push_back(Entry{k, z, y});
  *tz = z;
  *ty = y;
  return y.S > 0 && (L->rank == 0 || z.S > 0);
}

// Batch chunks of a call: tensor-core chunks where possible, lookup-table chunks of at
// most 8 rows otherwise.
bisco_status plan_chunks(const bisco_layer* L, int M, int32_t x_dtype, size_t ws_bytes, int dev, std::vector<Chunk>* out) {
  const size_t lim = cached_smem_limit(dev);
  // rows the workspace can hold z for (the tensor-core path needs one chunk's z)
  int tc_rows = kTcMaxBatch;
  if (L->rank > 0) {
    const size_t fit = (ws_bytes - kStatusBytes) / (static_cast<size_t>(L->rank) * 4);
    tc_rows = static_cast<int>(std::min<size_t>(kTcMaxBatch, fit / 16 * 16));
  }
  const int policy = g_policy.load();
  // grouped row scales: only the integer tensor-core kernel applies them, per 128-column
  // unit; a salient refinement is added by the integer kernel only
  const bool grouped = L->num_bases > 0 && L->row_group > 0;
  if (grouped && L->row_group % 128 != 0) return BISCO_ERR_UNSUPPORTED;
  const bool int_only = grouped || L->ref_bases > 0;
  if (L->ref_bases > 0 && refine_smem_bytes(L, kMaxBatchChunk) > lim) return BISCO_ERR_UNSUPPORTED;
  const bool tc_ok = (L->num_bases == 0 || L->scale_dtype == BISCO_BF16) && tc_rows >= kTcMinBatch &&
                     policy != BISCO_PATH_SMALL_BATCH_ONLY && !int_only;
  for (int m0 = 0; m0 < M;) {
    Chunk ch{};
    ch.m0 = m0;
    const int rem = M - m0;
    if (tc_ok && rem >= kTcMinBatch) {
      ch.Mc = std::min(rem, tc_rows);
      ch.tc = tc_plans(L, ch.Mc, x_dtype, dev, &ch.tz, &ch.ty);
    }
    if (!ch.tc) {
      ch.Mc = std::min(kMaxBatchChunk, rem);
      ch.lo = cached_layout(L, batch_block(ch.Mc), dev);
      // grouped or refined layers have no other kernel: where the integer plan of 8 rows
      // does not fit (e.g. 11008 input columns), the chunk takes 4, 2 or 1 rows instead
      while (int_only && !imma_fits(ch.lo) && ch.Mc > 1) {
        ch.Mc = batch_block(ch.Mc) / 2;
        ch.lo = cached_layout(L, batch_block(ch.Mc), dev);
      }
      // single rows of a layer without a correction stay on the lookup-table kernels,
      // which are faster there; with a correction the one-launch integer kernel wins
      // (5120 x 5120, rank 512: 13.5 us against 16.4 us for the two lookup-table launches)
      const bool fusable = ch.lo.has_z && ch.lo.ifz.C > 0;
      ch.imma = imma_fits(ch.lo) && (int_only || (policy != BISCO_PATH_LOOKUP_TABLE &&
                (batch_block(ch.Mc) >= 2 || policy == BISCO_PATH_INTEGER_MMA || fusable)));
      ch.fused = ch.imma && fusable;
      if (int_only && !ch.imma) return BISCO_ERR_UNSUPPORTED;
      // a chunk of 8 rows whose integer plan does not fit (large K at 8 batch rows, e.g.
      // 4096 x 11008 with a rank-256 correction) is faster on the tensor cores, padded to
      // 16 columns, than on the lookup-table kernels (that layer: 97 us for a 16-row
      // tensor-core chunk, 110 us per 8-row lookup-table chunk)
      if (!ch.imma && tc_ok && policy != BISCO_PATH_LOOKUP_TABLE && rem >= kMaxBatchChunk) {
        const int Mt = std::min(rem, tc_rows);
        TcPlan tz{}, ty{};
        if (tc_plans(L, Mt, x_dtype, dev, &tz, &ty)) {
          ch.tc = true;
          ch.Mc = Mt;
          ch.tz = tz;
          ch.ty = ty;
        }
      }
      if (!ch.tc && !ch.imma && !plans_fit(ch.lo, lim)) return BISCO_ERR_UNSUPPORTED;
    }
    out->push_back(ch);
    m0 += ch.Mc;
  }
  return BISCO_OK;
}

}  // namespace

extern "C" {

int64_t bisco_packed_words(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return ((rows + 31) / 32) * ((cols + 127) / 128) * 128;
}

bisco_status bisco_pack(const int8_t* signs, int64_t rows, int64_t cols, uint32_t* packed) {
  if (!signs || !packed || rows <= 0 || cols <= 0) return BISCO_ERR_INVALID_ARG;
  const int64_t n = rows * cols;
  for (int64_t i = 0; i < n; ++i)
    if (signs[i] != 1 && signs[i] != -1) return BISCO_ERR_INVALID_ARG;
  const int64_t Q = (cols + 127) / 128;
  std::memset(packed, 0, static_cast<size_t>(bisco_packed_words(rows, cols)) * 4);
  for (int64_t i = 0; i < rows; ++i) {
    const int64_t t = i / 32, r = i % 32;
    const int8_t* row = signs + i * cols;
    for (int64_t c = 0; c < cols; ++c) {
      if (row[c] == 1) {
        const int64_t q = c / 128, j = (c % 128) / 32, b = c % 32;
        packed[((t * Q + q) * 32 + r) * 4 + j] |= (1u << b);
      }
    }
  }
  return BISCO_OK;
}

bisco_status bisco_unpack(const uint32_t* packed, int64_t rows, int64_t cols, int8_t* signs) {
  if (!signs || !packed || rows <= 0 || cols <= 0) return BISCO_ERR_INVALID_ARG;
  const int64_t Q = (cols + 127) / 128;
  for (int64_t i = 0; i < rows; ++i) {
    const int64_t t = i / 32, r = i % 32;
    for (int64_t c = 0; c < cols; ++c) {
      const int64_t q = c / 128, j = (c % 128) / 32, b = c % 32;
      const uint32_t w = packed[((t * Q + q) * 32 + r) * 4 + j];
      signs[i * cols + c] = ((w >> b) & 1u) ? 1 : -1;
    }
  }
  return BISCO_OK;
}

bisco_status bisco_workspace_size(const bisco_layer* layer, int32_t M, size_t* bytes) {
  if (!bytes || M < 1) return BISCO_ERR_INVALID_ARG;
  const bisco_status st = validate_layer(layer);
  if (st != BISCO_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BISCO_ERR_CUDA;
  (void)dev;
  *bytes = ws_pref(layer, M);
  return BISCO_OK;
}

bisco_status bisco_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < static_cast<size_t>(kStatusBytes) || !aligned16(ws)) return BISCO_ERR_INVALID_ARG;
  return cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? BISCO_OK
                                                                                               : BISCO_ERR_CUDA;
}

bisco_status bisco_gemv(const bisco_layer* L, const void* X, int32_t x_dtype, int32_t M, void* Y,
                        int32_t y_dtype, void* ws, size_t ws_bytes, void* stream) {
  bisco_status st = validate_layer(L);
  if (st != BISCO_OK) return st;
  if (M < 0 || !dtype_ok(x_dtype) || !dtype_ok(y_dtype)) return BISCO_ERR_INVALID_ARG;
  if (M == 0) return BISCO_OK;
  if (!X || !Y || !aligned16(X) || !aligned16(Y)) return BISCO_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return BISCO_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BISCO_ERR_CUDA;
  if (ws_bytes < ws_need(L, M)) return BISCO_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  const size_t xb = dtype_bytes(x_dtype), yb = dtype_bytes(y_dtype);

  // Every launch is planned before the first one is issued, so an unsupported
  // request fails without touching any output.
  std::vector<Chunk> chunks;
  st = plan_chunks(L, M, x_dtype, ws_bytes, dev, &chunks);
  if (st != BISCO_OK) return st;

  int* status = reinterpret_cast<int*>(wsb);
  float* zbuf = reinterpret_cast<float*>(wsb + kStatusBytes);
  float* rbuf = L->ref_bases > 0 ? reinterpret_cast<float*>(wsb + ref_offset(L)) : nullptr;
  const ImmaDebug dbg{g_dbg_skip_tile.load(), g_dbg_wait_ns.load()};
  for (const Chunk& ch : chunks) {
    const void* Xc = static_cast<const unsigned char*>(X) + static_cast<size_t>(ch.m0) * L->in * xb;
    void* Yc = static_cast<unsigned char*>(Y) + static_cast<size_t>(ch.m0) * L->out * yb;
    // the refinement term first; the integer launch that writes this chunk's Y adds it
    if (rbuf && launch_refine(L, Xc, x_dtype, ch.Mc, rbuf, status, s) != cudaSuccess) return BISCO_ERR_CUDA;
    if (ch.fused) {
      PassParam pz{}, py{};
      pass_z(L, pz, Xc, x_dtype, ch.Mc, zbuf, status);
      pass_y(L, py, Xc, x_dtype, ch.Mc, Yc, y_dtype, zbuf, status);
      py.rref = rbuf;
      PassParam both[2] = {pz, py};
      const int zsrc[2] = {-1, 0}, is_z[2] = {1, 0};
      if (run_imma(both, zsrc, is_z, 2, ch.lo.ifz, s, &dbg) != cudaSuccess) return BISCO_ERR_CUDA;
      continue;
    }
    if (L->rank > 0) {
      PassParam pz{};
      pass_z(L, pz, Xc, x_dtype, ch.Mc, zbuf, status);
      cudaError_t e;
      if (ch.tc) {
        e = launch_tc(pz, ch.tz, s, &dbg);
      } else if (ch.imma) {
        e = run_imma(&pz, nullptr, nullptr, 1, ch.lo.iz, s, &dbg);
      } else {
        fill_plan(pz, ch.lo.pz);
        e = launch_pass(pz, ch.lo.pz, s, true);
      }
      if (e != cudaSuccess) return BISCO_ERR_CUDA;
    }
    PassParam py{};
    pass_y(L, py, Xc, x_dtype, ch.Mc, Yc, y_dtype, zbuf, status);
    py.rref = rbuf;  // refined layers run on the integer kernel only
    cudaError_t e;
    if (ch.tc) {
      e = launch_tc(py, ch.ty, s, &dbg);
    } else if (ch.imma) {
      e = run_imma(&py, nullptr, nullptr, 1, ch.lo.iy, s, &dbg);
    } else {
      fill_plan(py, ch.lo.py);
      e = launch_pass(py, ch.lo.py, s, true);
    }
    if (e != cudaSuccess) return BISCO_ERR_CUDA;
  }
  return BISCO_OK;
}

// ---- layers that share x in one launch ------------------------------------------

namespace {

constexpr int kMaxGroup = 3;

// Workspace of a group call: the status region and z of one 8-row chunk for every layer.
size_t group_ws_need(const bisco_layer* Ls, int n) {
  size_t b = kStatusBytes;
  for (int j = 0; j < n; ++j) b += align256(Ls[j].rank > 0 ? static_cast<size_t>(kMaxBatchChunk) * Ls[j].rank * 4 : 0);
  return b;
}

bisco_status validate_group(const bisco_layer* Ls, int32_t n) {
  if (!Ls || n < 1 || n > kMaxGroup) return BISCO_ERR_INVALID_ARG;
  for (int j = 0; j < n; ++j) {
    const bisco_status st = validate_layer(&Ls[j]);
    if (st != BISCO_OK) return st;
    if (Ls[j].in != Ls[0].in) return BISCO_ERR_INVALID_ARG;
  }
  return BISCO_OK;
}

// The integer plan of a group at batch block MB: z roles of the layers with a correction
// first, then the output roles (cached by shapes).
struct GroupPlan {
  ImmaPlan plan;
  int n_roles;
  int layer_of[kMaxRoles];  // layer of each role
  int zrole[kMaxRoles];     // output role: role of its z, or -1
  int is_z[kMaxRoles];
};

GroupPlan group_plan(const bisco_layer* Ls, int n, int MB, int dev) {
  struct Key {
    int dev, MB, n, v[kMaxGroup][6];
    bool operator==(const Key& o) const {
      if (dev != o.dev || MB != o.MB || n != o.n) return false;
      for (int j = 0; j < n; ++j)
        for (int k = 0; k < 6; ++k)
          if (v[j][k] != o.v[j][k]) return false;
      return true;
    }
  };
  struct Entry { Key k; GroupPlan g; };
  static std::mutex mu;
  static std::vector<Entry>* cache = new std::vector<Entry>();
  Key k{};
  k.dev = dev; k.MB = MB; k.n = n;
  for (int j = 0; j < n; ++j) {
    const int vals[6] = {Ls[j].out, Ls[j].in, Ls[j].num_bases, Ls[j].rank, Ls[j].n_sal, Ls[j].row_group};
    for (int q = 0; q < 6; ++q) k.v[j][q] = vals[q];
  }
  {
    std::lock_guard<std::mutex> g(mu);
    for (const Entry& e : *cache)
      if (e.k == k) return e.g;
  }
  GroupPlan gp{};
  SegList sy[kMaxGroup];
  const int z0 = 0;
  ImmaRole roles[kMaxRoles];
  int nr = 0;
  for (int j = 0; j < n; ++j) {
    sy[j] = segs_y(&Ls[j]);
    if (Ls[j].rank > 0) {
      roles[nr] = ImmaRole{ImmaShape{Ls[j].rank, quads(Ls[j].in), &z0, 1, nullptr}, 0, -1};
      gp.layer_of[nr] = j;
      gp.is_z[nr] = 1;
      gp.zrole[nr] = -1;
      ++nr;
    }
  }
  for (int j = 0; j < n; ++j) {
    const SegList& q = sy[j];
    int zr = -1;
    for (int r = 0; r < nr; ++r)
      if (gp.is_z[r] && gp.layer_of[r] == j) zr = r;
    roles[nr] = ImmaRole{ImmaShape{Ls[j].out, q.units, q.unit0, q.nseg, q.rgu}, Ls[j].n_sal,
                         zr >= 0 ? q.unit0[q.nseg - 1] : -1};
    gp.layer_of[nr] = j;
    gp.is_z[nr] = 0;
    gp.zrole[nr] = zr;
    ++nr;
  }
  gp.n_roles = nr;
  gp.plan = make_imma_plan(roles, nr, MB, cached_smem_limit(dev));
  std::lock_guard<std::mutex> g(mu);
  if (cache->size() > 4096) cache->clear();
  cache->push_back(Entry{k, gp});
  return gp;
}

// Whether a group call runs chunk by chunk as one integer launch (else layer by layer
// through bisco_gemv): batches below the tensor-core chunk size, a plan that fits, and a
// policy that allows the integer kernel.
bool group_launch_ok(const bisco_layer* Ls, int n, int M, int dev) {
  if (n < 2 || M >= kTcMinBatch || g_policy.load() == BISCO_PATH_LOOKUP_TABLE) return false;
  for (int j = 0; j < n; ++j)
    if (Ls[j].ref_bases > 0) return false;  // a refined layer runs its own two launches
  for (int m0 = 0; m0 < M; m0 += kMaxBatchChunk) {
    const int Mc = std::min(kMaxBatchChunk, M - m0);
    if (group_plan(Ls, n, batch_block(Mc), dev).plan.C == 0) return false;
  }
  for (int j = 0; j < n; ++j)
    if (Ls[j].num_bases > 0 && Ls[j].row_group > 0 && Ls[j].row_group % 128 != 0) return false;
  return true;
}

}  // namespace

bisco_status bisco_group_workspace_size(const bisco_layer* layers, int32_t n, int32_t M, size_t* bytes) {
  if (!bytes || M < 1) return BISCO_ERR_INVALID_ARG;
  const bisco_status st = validate_group(layers, n);
  if (st != BISCO_OK) return st;
  size_t b = group_ws_need(layers, n);
  for (int j = 0; j < n; ++j) b = std::max(b, ws_pref(&layers[j], M));
  *bytes = b;
  return BISCO_OK;
}

bisco_status bisco_gemv_group(const bisco_layer* layers, int32_t n, const void* X, int32_t x_dtype, int32_t M,
                              void* const* Y, int32_t y_dtype, void* ws, size_t ws_bytes, void* stream) {
  bisco_status st = validate_group(layers, n);
  if (st != BISCO_OK) return st;
  if (M < 0 || !dtype_ok(x_dtype) || !dtype_ok(y_dtype) || !Y) return BISCO_ERR_INVALID_ARG;
  if (M == 0) return BISCO_OK;
  if (!X || !aligned16(X)) return BISCO_ERR_INVALID_ARG;
  for (int j = 0; j < n; ++j)
    if (!Y[j] || !aligned16(Y[j])) return BISCO_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return BISCO_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BISCO_ERR_CUDA;
  if (ws_bytes < group_ws_need(layers, n)) return BISCO_ERR_WORKSPACE;
  if (!group_launch_ok(layers, n, M, dev)) {
    // layer by layer, in order, on the same stream and workspace
    for (int j = 0; j < n; ++j) {
      st = bisco_gemv(&layers[j], X, x_dtype, M, Y[j], y_dtype, ws, ws_bytes, stream);
      if (st != BISCO_OK) return st;
    }
    return BISCO_OK;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  int* status = reinterpret_cast<int*>(wsb);
  float* zb[kMaxGroup] = {};
  size_t off = kStatusBytes;
  for (int j = 0; j < n; ++j) {
    zb[j] = reinterpret_cast<float*>(wsb + off);
    off += align256(layers[j].rank > 0 ? static_cast<size_t>(kMaxBatchChunk) * layers[j].rank * 4 : 0);
  }
  const size_t xb = dtype_bytes(x_dtype), yb = dtype_bytes(y_dtype);
  const ImmaDebug dbg{g_dbg_skip_tile.load(), g_dbg_wait_ns.load()};
  for (int m0 = 0; m0 < M; m0 += kMaxBatchChunk) {
    const int Mc = std::min(kMaxBatchChunk, M - m0);
    const GroupPlan gp = group_plan(layers, n, batch_block(Mc), dev);
    const void* Xc = static_cast<const unsigned char*>(X) + static_cast<size_t>(m0) * layers[0].in * xb;
    PassParam passes[kMaxRoles];
    for (int r = 0; r < gp.n_roles; ++r) {
      const bisco_layer* L = &layers[gp.layer_of[r]];
      passes[r] = PassParam{};
      if (gp.is_z[r]) {
        pass_z(L, passes[r], Xc, x_dtype, Mc, zb[gp.layer_of[r]], status);
      } else {
        void* Yc = static_cast<unsigned char*>(Y[gp.layer_of[r]]) + static_cast<size_t>(m0) * L->out * yb;
        pass_y(L, passes[r], Xc, x_dtype, Mc, Yc, y_dtype, zb[gp.layer_of[r]], status);
      }
    }
    if (run_imma(passes, gp.zrole, gp.is_z, gp.n_roles, gp.plan, s, &dbg) != cudaSuccess) return BISCO_ERR_CUDA;
  }
  return BISCO_OK;
}

int32_t bisco_plan_group_kernels(const bisco_layer* layers, int32_t n, int32_t M, int32_t x_dtype, size_t ws_bytes,
                                 int32_t* kinds, int32_t max_kinds) {
  if (validate_group(layers, n) != BISCO_OK || M < 0 || !dtype_ok(x_dtype) || max_kinds < 0 ||
      (max_kinds > 0 && !kinds))
    return -1;
  if (M == 0) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (ws_bytes < group_ws_need(layers, n)) return -1;
  if (group_launch_ok(layers, n, M, dev)) {
    const int chunks = (M + kMaxBatchChunk - 1) / kMaxBatchChunk;
    for (int c = 0; c < chunks && c < max_kinds; ++c) kinds[c] = BISCO_KERNEL_INTEGER_MMA;
    return chunks;
  }
  int total = 0;
  for (int j = 0; j < n; ++j) {
    const int got = bisco_plan_kernels(&layers[j], M, x_dtype, ws_bytes, kinds ? kinds + std::min(total, max_kinds) : nullptr,
                                       std::max(0, max_kinds - total));
    if (got < 0) return -1;
    total += got;
  }
  return total;
}

bisco_status bisco_set_path_policy(int32_t policy) {
  if (policy != BISCO_PATH_AUTO && policy != BISCO_PATH_LOOKUP_TABLE && policy != BISCO_PATH_SMALL_BATCH_ONLY &&
      policy != BISCO_PATH_INTEGER_MMA)
    return BISCO_ERR_INVALID_ARG;
  g_policy.store(policy);
  return BISCO_OK;
}

int32_t bisco_plan_kernels(const bisco_layer* L, int32_t M, int32_t x_dtype, size_t ws_bytes, int32_t* kinds,
                           int32_t max_kinds) {
  if (validate_layer(L) != BISCO_OK || M < 0 || !dtype_ok(x_dtype) || max_kinds < 0 || (max_kinds > 0 && !kinds))
    return -1;
  if (M == 0) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (ws_bytes < ws_need(L, M)) return -1;
  std::vector<Chunk> chunks;
  if (plan_chunks(L, M, x_dtype, ws_bytes, dev, &chunks) != BISCO_OK) return -1;
  int n = 0;
  auto put = [&](int32_t k) {
    if (n < max_kinds) kinds[n] = k;
    ++n;
  };
  for (const Chunk& ch : chunks) {
    if (L->ref_bases > 0) put(BISCO_KERNEL_REFINE);
    const int passes = L->rank > 0 && !ch.fused ? 2 : 1;
    for (int ps = 0; ps < passes; ++ps) {
      const bool is_z = L->rank > 0 && ps == 0;
      if (ch.tc) {
        put(BISCO_KERNEL_TENSOR_CORE);
      } else if (ch.imma) {
        put(BISCO_KERNEL_INTEGER_MMA);
      } else {
        const Plan& pl = is_z ? ch.lo.pz : ch.lo.py;
        put(pl.kind == 2 ? BISCO_KERNEL_LUT_STREAM : pl.kind == 0 ? BISCO_KERNEL_LUT_WARP : BISCO_KERNEL_LUT_ROWS);
      }
    }
  }
  return n;
}

bisco_status bisco_debug_set_wait_test(int32_t skip_tile, uint64_t wait_ns) {
  if (skip_tile < -1) return BISCO_ERR_INVALID_ARG;
  g_dbg_skip_tile.store(skip_tile);
  g_dbg_wait_ns.store(wait_ns);
  return BISCO_OK;
}

bisco_status bisco_sync_status(void* stream, const void* ws) {
  if (!ws) return BISCO_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return BISCO_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return BISCO_ERR_CUDA;
  return static_cast<bisco_status>(code);
}

bisco_status bisco_bench(const bisco_bench_args* a, bisco_bench_result* r) {
  if (!a || !r || !a->layers || a->n_layers < 1 || a->M < 1 || a->reps < 1 || a->warmup < 0)
    return BISCO_ERR_INVALID_ARG;
  for (int i = 0; i < a->n_layers; ++i) {
    const bisco_status st = validate_layer(&a->layers[i]);
    if (st != BISCO_OK) return st;
  }
  if (!a->X || !a->Y || !a->ws || !dtype_ok(a->x_dtype) || !dtype_ok(a->y_dtype)) return BISCO_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BISCO_ERR_CUDA;
  for (int i = 0; i < a->n_layers; ++i)
    if (a->ws_bytes < ws_need(&a->layers[i], a->M)) return BISCO_ERR_WORKSPACE;

  if (ensure_kernel_attrs() != cudaSuccess || tc_ensure_attrs() != cudaSuccess) return BISCO_ERR_CUDA;
  const int launches = bisco_plan_kernels(&a->layers[0], a->M, a->x_dtype, a->ws_bytes, nullptr, 0);
  if (launches < 0) return BISCO_ERR_UNSUPPORTED;
  if (imma_ensure_attrs() != cudaSuccess) return BISCO_ERR_CUDA;
  cudaStream_t user = static_cast<cudaStream_t>(a->stream);
  cudaStream_t cs = nullptr;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr, join = nullptr;
  bisco_status result = BISCO_OK;
  const size_t yb = dtype_bytes(a->y_dtype);
  auto fail = [&](bisco_status st) { if (result == BISCO_OK) result = st; };

  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return BISCO_ERR_CUDA;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess ||
      cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess)
    fail(BISCO_ERR_CUDA);
  if (result == BISCO_OK && (cudaEventRecord(join, user) != cudaSuccess || cudaStreamWaitEvent(cs, join, 0) != cudaSuccess))
    fail(BISCO_ERR_CUDA);
  if (result == BISCO_OK) {
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      fail(BISCO_ERR_CUDA);
    } else {
      size_t yoff = 0;
      for (int i = 0; i < a->n_layers && result == BISCO_OK; ++i) {
        const bisco_layer& L = a->layers[i];
        const bisco_status st = bisco_gemv(&L, a->X, a->x_dtype, a->M, static_cast<unsigned char*>(a->Y) + yoff,
                                           a->y_dtype, a->ws, a->ws_bytes, cs);
        if (st != BISCO_OK) fail(st);
        yoff += static_cast<size_t>(a->M) * L.out * yb;
      }
      if (cudaStreamEndCapture(cs, &graph) != cudaSuccess) fail(BISCO_ERR_CUDA);
    }
  }
  if (result == BISCO_OK && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) fail(BISCO_ERR_CUDA);
  if (result == BISCO_OK) {
    for (int i = 0; i < a->warmup && result == BISCO_OK; ++i)
      if (cudaGraphLaunch(exec, cs) != cudaSuccess) fail(BISCO_ERR_CUDA);
    if (cudaEventRecord(e0, cs) != cudaSuccess) fail(BISCO_ERR_CUDA);
    for (int i = 0; i < a->reps && result == BISCO_OK; ++i)
      if (cudaGraphLaunch(exec, cs) != cudaSuccess) fail(BISCO_ERR_CUDA);
    if (cudaEventRecord(e1, cs) != cudaSuccess) fail(BISCO_ERR_CUDA);
    if (cudaEventSynchronize(e1) != cudaSuccess) fail(BISCO_ERR_CUDA);
    float ms = 0.f;
    if (result == BISCO_OK && cudaEventElapsedTime(&ms, e0, e1) == cudaSuccess) {
      r->us_per_replay = ms * 1000.0 / a->reps;
      r->us_per_gemv = r->us_per_replay / a->n_layers;
      r->kernels_per_gemv = launches;
    } else {
      fail(BISCO_ERR_CUDA);
    }
  }
  if (exec) cudaGraphExecDestroy(exec);
  if (graph) cudaGraphDestroy(graph);
  if (join && cudaEventRecord(join, cs) == cudaSuccess) cudaStreamWaitEvent(user, join, 0);
  if (cs) cudaStreamSynchronize(cs);
  if (cs) cudaStreamDestroy(cs);
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (join) cudaEventDestroy(join);
  return result;
}

const char* bisco_status_string(bisco_status st) {
  switch (st) {
    case BISCO_OK: return "BISCO_OK";
    case BISCO_ERR_INVALID_ARG: return "BISCO_ERR_INVALID_ARG";
    case BISCO_ERR_UNSUPPORTED: return "BISCO_ERR_UNSUPPORTED";
    case BISCO_ERR_CUDA: return "BISCO_ERR_CUDA";
    case BISCO_ERR_TIMEOUT: return "BISCO_ERR_TIMEOUT";
    case BISCO_ERR_WORKSPACE: return "BISCO_ERR_WORKSPACE";
  }
  return "BISCO_UNKNOWN_STATUS";
}

}  // extern "C"

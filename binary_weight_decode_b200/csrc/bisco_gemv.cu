// Binary-weight decode GEMV on CUDA cores, sm_100a.
//
// Computes, per output row o and batch row m,
//   y[m][o] = sum_seg rs_seg[o] * sum_i sign_seg[o][i] * xin_seg[m][i]  (+ salient term)
// where each "segment" is one packed sign matrix: a binary base B_k with
// xin = c_k (.) x and rs = r_k ("FluxBin", Sec. 3.1, decoupled row-column binary
// bases; the column scale is folded into the activation as in Sec. 3.2 Stage 1,
// "LUT Building with Scale Fusion"), the correction's V with xin = x and
// rs = alpha (z = alpha (.) (V x)), or the correction's U^T with xin = z
// ("BiLoCo", "The core idea": alpha * u * (v . x)).
//
// Sign-times-activation sums use 5-bit lookup tables in shared memory: for every
// 5 consecutive columns the CTA stores the 32 signed sums of their scaled
// activations, so one table read replaces five signed adds (the lookup-table idea
// of FluxBin Sec. 3.2, re-shaped for B200: 32-entry tables, one entry per bank, so
// the 32 lanes of a warp never conflict). A 128-column quad splits into 25
// five-bit fields and one three-bit field.
//
// Work decomposition: clusters of C CTAs. A cluster owns a range of 32-row tiles;
// CTA r of the cluster owns 1/C of the columns (units of 128 columns across all
// segments) and builds tables for those columns only. Warp w owns the tiles
// w, w + 8, ... of its cluster; each lane owns one row of a tile and reads its 16
// bytes of a (tile, unit) block, so a warp reads 512 contiguous bytes per load.
// The C partial sums of a row meet in distributed shared memory and are added
// in CTA-rank order, so results are deterministic.
//
// Launch protocol (programmatic dependent launch): sign words, row and column
// scales are loaded before griddepcontrol.wait; activations only after it.

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <utility>

#include "bisco_internal.h"

namespace cg = cooperative_groups;

namespace bisco {

namespace {

constexpr int kDepth = 8;  // work items per warp kept in flight (16 bytes per lane each)

// Eight consecutive values v[j] = a[off + j] (bf16 or fp32) as fp32, zero where
// j >= valid. One 16-byte load (two for fp32) when `vec` says the run is aligned.
__device__ __forceinline__ void load8(const void* a, long long off, int dt, int valid, bool vec, float v[8]) {
  if (dt == BISCO_BF16) {
    const unsigned short* h = reinterpret_cast<const unsigned short*>(a) + off;
    if (vec && valid >= 8) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(h));
      const unsigned w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __uint_as_float(static_cast<unsigned>(__ldg(h + j)) << 16) : 0.f;
    }
  } else {
    const float* f = reinterpret_cast<const float*>(a) + off;
    if (vec && valid >= 8) {
      const float4 q0 = __ldg(reinterpret_cast<const float4*>(f));
      const float4 q1 = __ldg(reinterpret_cast<const float4*>(f) + 1);
      v[0] = q0.x; v[1] = q0.y; v[2] = q0.z; v[3] = q0.w;
      v[4] = q1.x; v[5] = q1.y; v[6] = q1.z; v[7] = q1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __ldg(f + j) : 0.f;
    }
  }
}

// load8 for activations: coherent loads through L2 (the previous kernel may have written them).
__device__ __forceinline__ void load8_l2(const void* a, long long off, int dt, int valid, bool vec, float v[8]) {
  if (dt == BISCO_BF16) {
    const unsigned short* h = reinterpret_cast<const unsigned short*>(a) + off;
    if (vec && valid >= 8) {
      const uint4 q = __ldcg(reinterpret_cast<const uint4*>(h));
      const unsigned w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __uint_as_float(static_cast<unsigned>(__ldcg(h + j)) << 16) : 0.f;
    }
  } else {
    const float* f = reinterpret_cast<const float*>(a) + off;
    if (vec && valid >= 8) {
      const float4 q0 = __ldcg(reinterpret_cast<const float4*>(f));
      const float4 q1 = __ldcg(reinterpret_cast<const float4*>(f) + 1);
      v[0] = q0.x; v[1] = q0.y; v[2] = q0.z; v[3] = q0.w;
      v[4] = q1.x; v[5] = q1.y; v[6] = q1.z; v[7] = q1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? __ldcg(f + j) : 0.f;
    }
  }
}

// Byte offset 4*p of the table entry selected by field F of a 128-bit quad.
// Fields 0..24 are 5 bits at bit 5F; field 25 is 3 bits at bits 125..127.
__device__ __forceinline__ unsigned field_off(const uint4& w, const int F) {
  const unsigned ws[4] = {w.x, w.y, w.z, w.w};
  if (F == 25) return (w.w >> 27) & 0x1Cu;
  const int s = 5 * F, wi = s >> 5, b = s & 31;
  if (b + 5 <= 32) return (b >= 2 ? (ws[wi] >> (b - 2)) : (ws[wi] << (2 - b))) & 0x7Cu;
  return __funnelshift_r(ws[wi], ws[wi + 1], b - 2) & 0x7Cu;
}

__device__ __forceinline__ void fadd2(float& ax, float& ay, float bx, float by) {
  asm("{\n\t.reg .b64 a, b;\n\t"
      "mov.b64 a, {%0, %1};\n\t"
      "mov.b64 b, {%2, %3};\n\t"
      "add.rn.f32x2 a, a, b;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "+f"(ax), "+f"(ay)
      : "f"(bx), "f"(by));
}

__device__ __forceinline__ int find_seg(const PassParam& p, int u) {
  int s = 0;
#pragma unroll
  for (int k = 1; k < kMaxSeg; ++k)
    if (k < p.nseg && u >= p.seg[k].unit0) s = k;
  return s;
}

// Index of the lowest set bit of e (1 <= e < 32); folds to a constant when e is.
__host__ __device__ constexpr int low_bit(int e) {
  return (e & 1) ? 0 : (e & 2) ? 1 : (e & 4) ? 2 : (e & 8) ? 3 : 4;
}

// Per-unit metadata staged in shared memory.
struct UnitInfo {
  const uint4* base;   // this unit's quad in row tile 0, lane 0 (nullptr: no bits)
  int tstride;         // uint4 stride between row tiles (= 32 * nq)
  int ls;              // local segment index (row-scale slot)
  int flush;           // 1 if the unit ends its segment within the CTA range or ends a chunk
  int pad;
};

struct Smem {
  float* tables;   // [CU][MB][26 fields][36]   32-entry tables
  float* cs;       // [max_units][128]          column scales (0 past the segment's columns)
  float* rsc;      // [max_lseg][max_tiles*32]  row scales
  float* part;     // [max_tiles][MB][32]       this CTA's partial sums per owned row
  float* recv;     // [C][MB][max_share]        partial sums pushed by every CTA of the cluster
  float* xs;       // [MB][nsp]                 salient activations x[idx_t] * s_t
  UnitInfo* ui;    // [max_units]
};

__device__ __forceinline__ int max_share(const PassParam& p) { return (p.max_tiles * 32 + p.C - 1) / p.C; }

__device__ __forceinline__ Smem carve(unsigned char* smem, const PassParam& p, int MB, int CU) {
  Smem s;
  const int nsp = (p.n_sal + 3) & ~3;
  unsigned char* q = smem;
  s.tables = reinterpret_cast<float*>(q); q += static_cast<size_t>(CU) * p.col_stride_bytes;
  s.cs = reinterpret_cast<float*>(q);     q += static_cast<size_t>(p.max_units) * 128 * 4;
  s.rsc = reinterpret_cast<float*>(q);    q += static_cast<size_t>(p.max_lseg) * p.max_tiles * 32 * 4;
  s.part = reinterpret_cast<float*>(q);   q += static_cast<size_t>(p.max_tiles) * MB * 32 * 4;
  s.recv = reinterpret_cast<float*>(q);   q += static_cast<size_t>(p.C) * MB * ((max_share(p) + 3) & ~3) * 4;
  s.xs = reinterpret_cast<float*>(q);     q += static_cast<size_t>(MB) * nsp * 4;
  s.ui = reinterpret_cast<UnitInfo*>(q);
  return s;
}

// First row of CTA d's share when R rows are split over C CTAs, and the owner of row r.
__device__ __forceinline__ int share_begin(int d, int R, int C) { return d * R / C; }
__device__ __forceinline__ int share_owner(int r, int R, int C) { return ((r + 1) * C - 1) / R; }

// Input value xin[m][cc] of a segment (0 past its columns).
// Input value xin[m][cc] of a segment (0 past its columns). Activations may have been
// written by the previous kernel on the stream, so they are read through L2.
__device__ __forceinline__ float seg_input(const PassParam& p, const SegParam& G, int m, int cc) {
  if (m >= p.Mc || cc >= G.ncols || G.xsrc == 2) return 0.f;
  if (G.xsrc == 0) {
    const long long i = static_cast<long long>(m) * p.ldx + cc;
    if (p.xdt == BISCO_BF16)
      return __uint_as_float(static_cast<unsigned>(__ldcg(reinterpret_cast<const unsigned short*>(p.X) + i)) << 16);
    return __ldcg(reinterpret_cast<const float*>(p.X) + i);
  }
  return __ldcg(p.Z + static_cast<long long>(m) * p.ldz + cc);
}

// Shared-memory accesses to the partial-sum buffer through inline PTX without a
// memory clobber: they never alias the lookup tables, and this lets the compiler
// keep the next item's table reads ahead of these updates.
__device__ __forceinline__ float lds_part(const float* a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(static_cast<unsigned>(__cvta_generic_to_shared(a))));
  return v;
}
__device__ __forceinline__ void sts_part(float* a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(static_cast<unsigned>(__cvta_generic_to_shared(a))), "f"(v));
}

template <int MB>
__global__ void __launch_bounds__(kThreads, 2) lut_gemv_kernel(const __grid_constant__ PassParam p, const int CU) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ci = blockIdx.x / p.C;
  const int t0 = ci * p.tiles / p.ncl, t1 = (ci + 1) * p.tiles / p.ncl, nt = t1 - t0;
  const int u0 = rank * p.units / p.C, u1 = (rank + 1) * p.units / p.C, nu = u1 - u0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nsp = (p.n_sal + 3) & ~3;
  const int seg_first = find_seg(p, u0);
  const Smem S = carve(smem, p, MB, CU);
  const int rows_c = nt * 32;           // rows of this cluster (incl. padding of the last tile)
  const int msh = (max_share(p) + 3) & ~3;
  // Peers write into this CTA's shared memory later on; the split barrier below tells
  // them that every CTA of the cluster is running before any such write happens.
  auto started = cluster.barrier_arrive();

  // ---- weights-only staging (before the dependency wait) ----
  // (a) weight prefetch into the register ring: items of this warp, per chunk of CU
  //     units, are (owned tile k = tile warp + 8k, unit in chunk)
  const int my_tiles = warp < nt ? (nt - warp + kWarps - 1) / kWarps : 0;
  const int nchunks = (nu + CU - 1) / CU;
  uint4 buf[kDepth];
  int lk = 0, lu = 0;  // load cursor (tile slot, unit in chunk)
  auto load_next = [&](int cu0, int cn, uint4& dst) {
    const int u = u0 + cu0 + lu;
    const SegParam& G = p.seg[find_seg(p, u)];
    const int t = t0 + warp + lk * kWarps;
    dst = G.bits ? __ldcs(G.bits + (static_cast<long long>(t) * G.nq + (u - G.unit0)) * 32 + lane)
                 : make_uint4(0u, 0u, 0u, 0u);
    if (++lu == cn) { lu = 0; ++lk; }
  };
  auto prefetch_chunk = [&](int c) {
    const int cu0 = c * CU, cn = min(CU, nu - cu0), n = my_tiles * cn;
    lk = 0; lu = 0;
#pragma unroll
    for (int d = 0; d < kDepth; ++d)
      if (d < n) load_next(cu0, cn, buf[d]);
  };
  prefetch_chunk(0);
  // (b) unit metadata
  for (int ul = threadIdx.x; ul < nu; ul += kThreads) {
    const int u = u0 + ul;
    const int sg = find_seg(p, u);
    const SegParam& G = p.seg[sg];
    UnitInfo I;
    I.base = G.bits ? G.bits + static_cast<long long>(u - G.unit0) * 32 : nullptr;
    I.tstride = 32 * G.nq;
    I.ls = sg - seg_first;
    I.flush = (ul + 1 == nu) || ((ul + 1) % CU == 0) || (find_seg(p, u + 1) != sg);
    I.pad = 0;
    S.ui[ul] = I;
  }
  // (c) column and row scales, staged in rounds; every load of a round is issued
  //     before any of them is used
  const int nls = find_seg(p, u1 - 1) - seg_first + 1;
  const int n_cs = nu * 16, n_rs = nls * nt * 4;
  for (int base = 0; base < n_cs + n_rs; base += 2 * kThreads) {
    float v[2][8];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int ch = base + threadIdx.x + k * kThreads;
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = 0.f;
      if (ch < n_cs) {  // column scales of unit ch/16, columns 8*(ch%16) ..
        const int ul = ch >> 4, j0 = (ch & 15) * 8;
        const int u = u0 + ul;
        const SegParam& G = p.seg[find_seg(p, u)];
        const int cc = (u - G.unit0) * 128 + j0;
        const int valid = G.xsrc == 2 ? 0 : max(0, min(8, G.ncols - cc));
        if (G.cscale == nullptr) {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[k][j] = j < valid ? 1.f : 0.f;
        } else if (valid > 0) {
          load8(G.cscale, cc, G.cdt, valid, G.cvec != 0, v[k]);
        }
      } else if (ch < n_cs + n_rs) {  // row scales of local segment ls, rows 8*(...) ..
        const int rc = ch - n_cs;
        const int ls = rc / (nt * 4), r8 = (rc - ls * nt * 4) * 8;
        const SegParam& G = p.seg[seg_first + ls];
        const int o = t0 * 32 + r8;
        const int valid = max(0, min(8, p.rows - o));
        if (G.rscale == nullptr) {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[k][j] = j < valid ? 1.f : 0.f;
        } else if (valid > 0) {
          load8(G.rscale, o, G.rdt, valid, G.rvec != 0, v[k]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int ch = base + threadIdx.x + k * kThreads;
      float* d = nullptr;
      if (ch < n_cs) {
        d = S.cs + ch * 8;
      } else if (ch < n_cs + n_rs) {
        const int rc = ch - n_cs;
        const int ls = rc / (nt * 4), r8 = (rc - ls * nt * 4) * 8;
        d = S.rsc + ls * p.max_tiles * 32 + r8;
      }
      if (d) {
        reinterpret_cast<float4*>(d)[0] = make_float4(v[k][0], v[k][1], v[k][2], v[k][3]);
        reinterpret_cast<float4*>(d)[1] = make_float4(v[k][4], v[k][5], v[k][6], v[k][7]);
      }
    }
  }
  for (int idx = threadIdx.x; idx < nt * MB * 32; idx += kThreads) S.part[idx] = 0.f;
  __syncthreads();  // unit metadata and scales visible

  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");

  // ---- salient activations (gathered and scaled) ----
  for (int idx = threadIdx.x; idx < MB * p.n_sal; idx += kThreads) {
    const int m = idx / p.n_sal, t = idx - m * p.n_sal;
    float v = 0.f;
    const int cc = __ldg(p.sal_idx + t);
    if (cc < 0 || cc >= p.xcols) atomicExch(p.status, static_cast<int>(BISCO_ERR_INVALID_ARG));
    else if (m < p.Mc) {
      const long long i = static_cast<long long>(m) * p.ldx + cc;
      const float xv = p.xdt == BISCO_BF16
                           ? __uint_as_float(static_cast<unsigned>(__ldcg(reinterpret_cast<const unsigned short*>(p.X) + i)) << 16)
                           : __ldcg(reinterpret_cast<const float*>(p.X) + i);
      v = xv * __ldg(p.sal_scale + t);
    }
    S.xs[m * nsp + t] = v;
  }

  constexpr int NA = MB > 1 ? MB : 2;
  float acc[NA], tot[MB];
#pragma unroll
  for (int m = 0; m < NA; ++m) acc[m] = 0.f;
#pragma unroll
  for (int m = 0; m < MB; ++m) tot[m] = 0.f;
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(S.tables);

  for (int c = 0; c < nchunks; ++c) {
    const int cu0 = c * CU, cn = min(CU, nu - cu0);
    // tables straight from the activations: task (unit, batch row) per warp; lane f
    // loads the 5 inputs of field f (3 for field 25), scales them by c and writes
    // all 32 signed sums. Two tasks' loads are in flight together.
    for (int task = warp; task < cn * MB; task += 2 * kWarps) {
      float xin[2][5];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int tk = task + h * kWarps;
#pragma unroll
        for (int n = 0; n < 5; ++n) xin[h][n] = 0.f;
        if (tk < cn * MB && lane < kFields) {
          const int ulc = tk / MB, m = tk - ulc * MB;
          const int u = u0 + cu0 + ulc;
          const SegParam& G = p.seg[find_seg(p, u)];
          const int cb = (u - G.unit0) * 128 + 5 * lane;
          const int len = lane < 25 ? 5 : 3;
#pragma unroll
          for (int n = 0; n < 5; ++n)
            if (n < len) xin[h][n] = seg_input(p, G, m, cb + n);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int tk = task + h * kWarps;
        if (tk < cn * MB && lane < kFields) {
          const int ulc = tk / MB, m = tk - ulc * MB;
          const float* cv = S.cs + (cu0 + ulc) * 128 + 5 * lane;
          const int len = lane < 25 ? 5 : 3;
          float x[5];
#pragma unroll
          for (int n = 0; n < 5; ++n) x[n] = n < len ? xin[h][n] * cv[n] : 0.f;
          const float d[5] = {2.f * x[0], 2.f * x[1], 2.f * x[2], 2.f * x[3], 2.f * x[4]};
          float T[32];
          T[0] = -((x[0] + x[1]) + (x[2] + x[3]) + x[4]);
#pragma unroll
          for (int e = 1; e < 32; ++e) T[e] = T[e & (e - 1)] + d[low_bit(e)];
          float* dst = S.tables + static_cast<size_t>(ulc) * (p.col_stride_bytes / 4) + (m * kFields + lane) * kFieldStride;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            reinterpret_cast<float4*>(dst)[j] = make_float4(T[4 * j], T[4 * j + 1], T[4 * j + 2], T[4 * j + 3]);
        }
      }
    }
    __syncthreads();

    // lookups: item i of this chunk sits in ring slot i % kDepth
    const int n_ci = my_tiles * cn;
    int pk = 0, pu = 0;  // processing cursor
    for (int base = 0; base < n_ci; base += kDepth) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        if (base + d < n_ci) {
          const uint4 w = buf[d];
          if (base + d + kDepth < n_ci) load_next(cu0, cn, buf[d]);
          const unsigned uoff = static_cast<unsigned>(pu) * static_cast<unsigned>(p.col_stride_bytes);
          if (MB == 1) {
#pragma unroll
            for (int F = 0; F < kFields; F += 2) {
              const float v0 = *reinterpret_cast<const float*>(tb + (field_off(w, F) | uoff) + F * kFieldStride * 4);
              const float v1 =
                  *reinterpret_cast<const float*>(tb + (field_off(w, F + 1) | uoff) + (F + 1) * kFieldStride * 4);
              fadd2(acc[0], acc[1], v0, v1);
            }
          } else {
#pragma unroll
            for (int F = 0; F < kFields; ++F) {
              const unsigned off = field_off(w, F) | uoff;
#pragma unroll
              for (int m = 0; m < MB; m += 2) {
                const float v0 = *reinterpret_cast<const float*>(tb + off + (m * kFields + F) * kFieldStride * 4);
                const float v1 = *reinterpret_cast<const float*>(tb + off + ((m + 1) * kFields + F) * kFieldStride * 4);
                fadd2(acc[m], acc[m + 1], v0, v1);
              }
            }
          }
          const int tl = warp + pk * kWarps;
          const UnitInfo& I = S.ui[cu0 + pu];
          if (I.flush) {  // the unit ends a segment (or the chunk): apply that segment's row scale
            const float rs = S.rsc[I.ls * p.max_tiles * 32 + tl * 32 + lane];
            if (MB == 1) {
              tot[0] = fmaf(acc[0] + acc[1], rs, tot[0]);
              acc[0] = acc[1] = 0.f;
            } else {
#pragma unroll
              for (int m = 0; m < MB; ++m) { tot[m] = fmaf(acc[m], rs, tot[m]); acc[m] = 0.f; }
            }
          }
          if (++pu == cn) {  // this tile's units of the chunk are done
#pragma unroll
            for (int m = 0; m < MB; ++m) { S.part[(tl * MB + m) * 32 + lane] += tot[m]; tot[m] = 0.f; }
            pu = 0;
            ++pk;
          }
        }
      }
    }
    if (c + 1 < nchunks) {
      prefetch_chunk(c + 1);
      __syncthreads();  // all warps are done with this chunk's tables before they are rebuilt
    }
  }

  // ---- push partial sums to the CTA that reduces each row (distributed shared memory) ----
  cluster.barrier_wait(std::move(started));
  for (int k = 0; k < my_tiles; ++k) {
    const int tl = warp + k * kWarps;
    const int lr = tl * 32 + lane;
    const int dst = share_owner(lr, rows_c, p.C);
    float* rp = cluster.map_shared_rank(S.recv, dst);
    const int sr = lr - share_begin(dst, rows_c, p.C);
#pragma unroll
    for (int m = 0; m < MB; ++m) rp[(rank * MB + m) * msh + sr] = S.part[(tl * MB + m) * 32 + lane];
  }
  cluster.sync();  // all partial sums have landed

  // ---- reduce this CTA's share of rows in CTA-rank order, add salient columns, store ----
  const int r0 = share_begin(rank, rows_c, p.C), r1 = share_begin(rank + 1, rows_c, p.C);
  for (int lr = r0 + threadIdx.x; lr < r1; lr += kThreads) {
    const int o = t0 * 32 + lr;
    if (o >= p.rows) continue;
    const int sr = lr - r0;
    float sum[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) sum[m] = 0.f;
    for (int src = 0; src < p.C; ++src) {
#pragma unroll
      for (int m = 0; m < MB; ++m) sum[m] += S.recv[(src * MB + m) * msh + sr];
    }
    if (p.n_sal > 0) {
      // salient columns: y += sum_t q[o][t] * (x[idx_t] * s_t)
      const int8_t* qrow = p.sal_q + static_cast<long long>(o) * p.sal_stride;
      for (int tq = 0; tq < p.n_sal; tq += 16) {
        const uint4 qq = __ldg(reinterpret_cast<const uint4*>(qrow + tq));
        const unsigned qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int tt = tq + k;
          if (tt < p.n_sal) {
            const float qv = static_cast<float>(static_cast<int8_t>((qw[k >> 2] >> (8 * (k & 3))) & 0xFF));
#pragma unroll
            for (int m = 0; m < MB; ++m) sum[m] = fmaf(qv, S.xs[m * nsp + tt], sum[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      if (m < p.Mc) {
        if (p.ydt == BISCO_BF16)
          reinterpret_cast<__nv_bfloat16*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = __float2bfloat16_rn(sum[m]);
        else
          reinterpret_cast<float*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = sum[m];
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Batch rows <= 2, layers with few row tiles per cluster: a wider CTA (16 warps, 64
// registers a thread) that stages the
// packed sign words with cp.async into a per-warp shared-memory ring, so the loop
// over work items stays compact. Items (unit, row tile) of the CTA are dealt to
// the warps round-robin; every warp keeps its own partial sum per row tile, and
// the warps' partial sums are added in warp order at the end.
// ----------------------------------------------------------------------------
constexpr int kWW = 16;          // warps per CTA
constexpr int kTW = kWW * 32;    // threads per CTA
constexpr int kRing = 6;         // items per warp in flight

struct WUnit {           // per-unit metadata of the current chunk
  const uint4* base;    // sign words of this unit's quad, row tile 0, lane 0 (nullptr: none)
  int tstride;          // uint4 stride between row tiles
  int ls;               // local segment (row-scale slot)
};

struct WSmem {
  float* tables;   // [CU][MB][26][36]          tables of the current chunk of units
  float* xt;       // [CU][MB][128]             scaled activations of the chunk
  float* cs;       // [max_units][128]          column scales
  float* rsc;      // [max_lseg][max_tiles*32]  row scales
  float* part;     // [kWW][max_tiles][MB][32]  per-warp partial sums
  float* recv;     // [C][MB][msh]              partial sums pushed by the cluster
  float* xs;       // [MB][nsp]                 salient activations
  WUnit* ui;       // [max_units]
  uint4* ring;     // [kWW][kRing][32]          staged sign words
};

__host__ __device__ __forceinline__ size_t wsmem_bytes(int CU, int col_stride, int max_units, int max_lseg,
                                                       int max_tiles, int MB, int C, int n_sal) {
  const int nsp = (n_sal + 3) & ~3;
  const int msh = ((max_tiles * 32 + C - 1) / C + 3) & ~3;
  return static_cast<size_t>(CU) * col_stride + static_cast<size_t>(CU) * MB * 128 * 4 +
         static_cast<size_t>(max_units) * 128 * 4 + static_cast<size_t>(max_lseg) * max_tiles * 32 * 4 +
         static_cast<size_t>(kWW) * max_tiles * MB * 32 * 4 + static_cast<size_t>(C) * MB * msh * 4 +
         static_cast<size_t>(MB) * nsp * 4 + static_cast<size_t>(max_units) * sizeof(WUnit) +
         static_cast<size_t>(kWW) * kRing * 32 * 16 + 16;
}

__device__ __forceinline__ WSmem wcarve(unsigned char* smem, const PassParam& p, int MB, int CU) {
  WSmem s;
  const int nsp = (p.n_sal + 3) & ~3;
  unsigned char* q = smem;
  s.tables = reinterpret_cast<float*>(q); q += static_cast<size_t>(CU) * p.col_stride_bytes;
  s.xt = reinterpret_cast<float*>(q);     q += static_cast<size_t>(CU) * MB * 128 * 4;
  s.cs = reinterpret_cast<float*>(q);     q += static_cast<size_t>(p.max_units) * 128 * 4;
  s.rsc = reinterpret_cast<float*>(q);    q += static_cast<size_t>(p.max_lseg) * p.max_tiles * 32 * 4;
  s.part = reinterpret_cast<float*>(q);   q += static_cast<size_t>(kWW) * p.max_tiles * MB * 32 * 4;
  s.recv = reinterpret_cast<float*>(q);   q += static_cast<size_t>(p.C) * MB * ((max_share(p) + 3) & ~3) * 4;
  s.xs = reinterpret_cast<float*>(q);     q += static_cast<size_t>(MB) * nsp * 4;
  s.ui = reinterpret_cast<WUnit*>(q);     q += static_cast<size_t>(p.max_units) * sizeof(WUnit);
  q = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(q) + 15) & ~uintptr_t(15));
  s.ring = reinterpret_cast<uint4*>(q);
  return s;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<unsigned>(__cvta_generic_to_shared(smem_dst))),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Cursor over this warp's items of a chunk: chunk-local item k = ulc * nt + tl, and
// the warp takes k = warp, warp + 16, ...; advancing by 16 needs no division.
struct ItemCursor {
  int ulc, tl;
  __device__ __forceinline__ void init(int k, int nt) { ulc = 0; tl = k; while (tl >= nt) { tl -= nt; ++ulc; } }
  __device__ __forceinline__ void next(int nt) { tl += kWW; while (tl >= nt) { tl -= nt; ++ulc; } }
};

template <int MB>
__global__ void __launch_bounds__(kTW, 2) lut_gemv_warp_kernel(const __grid_constant__ PassParam p, const int CU) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ci = blockIdx.x / p.C;
  const int t0 = ci * p.tiles / p.ncl, t1 = (ci + 1) * p.tiles / p.ncl, nt = t1 - t0;
  const int u0 = rank * p.units / p.C, u1 = (rank + 1) * p.units / p.C, nu = u1 - u0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nsp = (p.n_sal + 3) & ~3;
  const int seg_first = find_seg(p, u0);
  const WSmem S = wcarve(smem, p, MB, CU);
  const int rows_c = nt * 32;
  const int msh = (max_share(p) + 3) & ~3;
  auto started = cluster.barrier_arrive();

  const int nchunks = (nu + CU - 1) / CU;
  uint4* my_ring = S.ring + warp * kRing * 32 + lane;

  // ---- weights-only staging (before the dependency wait) ----
  for (int ul = threadIdx.x; ul < nu; ul += kTW) {
    const int u = u0 + ul;
    const int sg = find_seg(p, u);
    const SegParam& G = p.seg[sg];
    WUnit I;
    I.base = G.bits ? G.bits + static_cast<long long>(u - G.unit0) * 32 : nullptr;
    I.tstride = 32 * G.nq;
    I.ls = sg - seg_first;
    S.ui[ul] = I;
  }
  const int nls = find_seg(p, u1 - 1) - seg_first + 1;
  const int n_cs = nu * 16, n_rs = nls * nt * 4;
  for (int ch = threadIdx.x; ch < n_cs + n_rs; ch += kTW) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
    float* d;
    if (ch < n_cs) {
      const int ul = ch >> 4, j0 = (ch & 15) * 8;
      const int u = u0 + ul;
      const SegParam& G = p.seg[find_seg(p, u)];
      const int cc = (u - G.unit0) * 128 + j0;
      const int valid = G.xsrc == 2 ? 0 : max(0, min(8, G.ncols - cc));
      if (G.cscale == nullptr) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = j < valid ? 1.f : 0.f;
      } else if (valid > 0) {
        load8(G.cscale, cc, G.cdt, valid, G.cvec != 0, v);
      }
      d = S.cs + ch * 8;
    } else {
      const int rc = ch - n_cs;
      const int ls = rc / (nt * 4), r8 = (rc - ls * nt * 4) * 8;
      const SegParam& G = p.seg[seg_first + ls];
      const int o = t0 * 32 + r8;
      const int valid = max(0, min(8, p.rows - o));
      if (G.rscale == nullptr) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = j < valid ? 1.f : 0.f;
      } else if (valid > 0) {
        load8(G.rscale, o, G.rdt, valid, G.rvec != 0, v);
      }
      d = S.rsc + ls * p.max_tiles * 32 + r8;
    }
    reinterpret_cast<float4*>(d)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(d)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  float* my_part = S.part + static_cast<size_t>(warp) * p.max_tiles * MB * 32;
  for (int idx = lane; idx < nt * MB * 32; idx += 32) my_part[idx] = 0.f;
  __syncthreads();  // unit metadata visible

  // stage this warp's first items of chunk 0
  ItemCursor ic{0, 0};
  int n_issue = 0;  // items of the current chunk issued so far by this warp
  auto issue = [&](int cu0, int cn) {  // stage the item under the issue cursor (one group)
    if (ic.ulc < cn) {
      const WUnit& I = S.ui[cu0 + ic.ulc];
      if (I.base) cp_async16(my_ring + (n_issue % kRing) * 32, I.base + static_cast<long long>(t0 + ic.tl) * I.tstride + lane);
      ic.next(nt);
    }
    ++n_issue;
    cp_async_commit();
  };
  {
    const int cn = min(CU, nu);
    ic.init(warp, nt);
    n_issue = 0;
#pragma unroll
    for (int j = 0; j < kRing - 1; ++j) issue(0, cn);
  }

  asm volatile("griddepcontrol.wait;" ::: "memory");

  for (int idx = threadIdx.x; idx < MB * p.n_sal; idx += kTW) {
    const int m = idx / p.n_sal, t = idx - m * p.n_sal;
    float v = 0.f;
    const int cc = __ldg(p.sal_idx + t);
    if (cc < 0 || cc >= p.xcols) {
      atomicExch(p.status, static_cast<int>(BISCO_ERR_INVALID_ARG));
    } else if (m < p.Mc) {
      const long long i = static_cast<long long>(m) * p.ldx + cc;
      const float xv = p.xdt == BISCO_BF16
                           ? __uint_as_float(static_cast<unsigned>(__ldcg(reinterpret_cast<const unsigned short*>(p.X) + i)) << 16)
                           : __ldcg(reinterpret_cast<const float*>(p.X) + i);
      v = xv * __ldg(p.sal_scale + t);
    }
    S.xs[m * nsp + t] = v;
  }

  const unsigned char* tb = reinterpret_cast<const unsigned char*>(S.tables);
  for (int c = 0; c < nchunks; ++c) {
    const int cu0 = c * CU, cn = min(CU, nu - cu0);
    if (c > 0) __syncthreads();  // the previous chunk's tables are no longer read
    // scaled activations of the chunk: 8-column runs, one 16-byte load each
    for (int ch = threadIdx.x; ch < cn * MB * 16; ch += kTW) {
      const int ulc = ch / (MB * 16);
      const int rem = ch - ulc * (MB * 16);
      const int m = rem >> 4, j0 = (rem & 15) * 8;
      const int u = u0 + cu0 + ulc;
      const SegParam& G = p.seg[find_seg(p, u)];
      const int cc = (u - G.unit0) * 128 + j0;
      const int valid = max(0, min(8, G.ncols - cc));
      float xv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) xv[j] = 0.f;
      if (m < p.Mc && valid > 0 && G.xsrc != 2) {
        if (G.xsrc == 0)
          load8_l2(p.X, static_cast<long long>(m) * p.ldx + cc, p.xdt, valid, p.x_vec != 0, xv);
        else
          load8_l2(p.Z, static_cast<long long>(m) * p.ldz + cc, BISCO_F32, valid, p.z_vec != 0, xv);
      }
      const float* cv = S.cs + (cu0 + ulc) * 128 + j0;
      float4* d4 = reinterpret_cast<float4*>(S.xt + (ulc * MB + m) * 128 + j0);
      d4[0] = make_float4(xv[0] * cv[0], xv[1] * cv[1], xv[2] * cv[2], xv[3] * cv[3]);
      d4[1] = make_float4(xv[4] * cv[4], xv[5] * cv[5], xv[6] * cv[6], xv[7] * cv[7]);
    }
    __syncthreads();
    // tables: task (unit, batch row); lane f builds the 32 signed sums of field f
    for (int q = warp; q < cn * MB; q += kWW) {
      const int ulc = q / MB, m = q - ulc * MB;
      if (lane < kFields) {
        const float* x = S.xt + (ulc * MB + m) * 128 + 5 * lane;
        const float x0 = x[0], x1 = x[1], x2 = x[2];
        const float x3 = lane < 25 ? x[3] : 0.f, x4 = lane < 25 ? x[4] : 0.f;
        const float d[5] = {2.f * x0, 2.f * x1, 2.f * x2, 2.f * x3, 2.f * x4};
        float T[32];
        T[0] = -((x0 + x1) + (x2 + x3) + x4);
#pragma unroll
        for (int e = 1; e < 32; ++e) T[e] = T[e & (e - 1)] + d[low_bit(e)];
        float* dst = S.tables + static_cast<size_t>(ulc) * (p.col_stride_bytes / 4) + (m * kFields + lane) * kFieldStride;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          reinterpret_cast<float4*>(dst)[k] = make_float4(T[4 * k], T[4 * k + 1], T[4 * k + 2], T[4 * k + 3]);
      }
    }
    __syncthreads();
    // the activations are in: let the next kernel on the stream start its prefetch
    if (c == 0) asm volatile("griddepcontrol.launch_dependents;");

    // lookups over this warp's items of the chunk
    const int n_my = (cn * nt > warp) ? (cn * nt - warp + kWW - 1) / kWW : 0;
    ItemCursor pc;
    pc.init(warp, nt);
    for (int j = 0; j < n_my; ++j) {
      issue(cu0, cn);
      cp_async_wait<kRing - 1>();
      const uint4 w = my_ring[(j % kRing) * 32];
      const unsigned uoff = static_cast<unsigned>(pc.ulc) * static_cast<unsigned>(p.col_stride_bytes);
      float a[MB > 1 ? MB : 2];
#pragma unroll
      for (int m = 0; m < (MB > 1 ? MB : 2); ++m) a[m] = 0.f;
      if (MB == 1) {
#pragma unroll
        for (int F = 0; F < kFields; F += 2) {
          const float v0 = *reinterpret_cast<const float*>(tb + (field_off(w, F) | uoff) + F * kFieldStride * 4);
          const float v1 = *reinterpret_cast<const float*>(tb + (field_off(w, F + 1) | uoff) + (F + 1) * kFieldStride * 4);
          fadd2(a[0], a[1], v0, v1);
        }
      } else {
#pragma unroll
        for (int F = 0; F < kFields; ++F) {
          const unsigned off = field_off(w, F) | uoff;
#pragma unroll
          for (int m = 0; m < MB; m += 2) {
            const float v0 = *reinterpret_cast<const float*>(tb + off + (m * kFields + F) * kFieldStride * 4);
            const float v1 = *reinterpret_cast<const float*>(tb + off + ((m + 1) * kFields + F) * kFieldStride * 4);
            fadd2(a[m], a[m + 1], v0, v1);
          }
        }
      }
      const float rs = S.rsc[S.ui[cu0 + pc.ulc].ls * p.max_tiles * 32 + pc.tl * 32 + lane];
      float* pp = my_part + pc.tl * MB * 32 + lane;
      if (MB == 1) {
        sts_part(pp, fmaf(a[0] + a[1], rs, lds_part(pp)));
      } else {
#pragma unroll
        for (int m = 0; m < MB; ++m) sts_part(pp + m * 32, fmaf(a[m], rs, lds_part(pp + m * 32)));
      }
      pc.next(nt);
    }
    cp_async_wait<0>();
    if (c + 1 < nchunks) {  // first items of the next chunk
      const int ncn = min(CU, nu - (c + 1) * CU);
      ic.init(warp, nt);
      n_issue = 0;
#pragma unroll
      for (int j = 0; j < kRing - 1; ++j) issue((c + 1) * CU, ncn);
    }
  }
  if (nchunks == 0) asm volatile("griddepcontrol.launch_dependents;");
  __syncthreads();  // all warps' partial sums are in shared memory

  // ---- sum over warps (fixed order) and push to the CTA that owns each row ----
  cluster.barrier_wait(std::move(started));
  for (int idx = threadIdx.x; idx < nt * MB * 32; idx += kTW) {
    const int tl = idx / (MB * 32);
    const int rem = idx - tl * MB * 32;
    const int m = rem >> 5, ln = rem & 31;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWW; ++w) v += S.part[(static_cast<size_t>(w) * p.max_tiles + tl) * MB * 32 + m * 32 + ln];
    const int lr = tl * 32 + ln;
    const int dst = share_owner(lr, rows_c, p.C);
    float* rp = cluster.map_shared_rank(S.recv, dst);
    rp[(rank * MB + m) * msh + (lr - share_begin(dst, rows_c, p.C))] = v;
  }
  cluster.sync();  // all partial sums have landed

  // ---- reduce this CTA's share of rows in CTA-rank order, add salient columns, store ----
  const int r0 = share_begin(rank, rows_c, p.C), r1 = share_begin(rank + 1, rows_c, p.C);
  for (int lr = r0 + threadIdx.x; lr < r1; lr += kTW) {
    const int o = t0 * 32 + lr;
    if (o >= p.rows) continue;
    const int sr = lr - r0;
    float sum[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) sum[m] = 0.f;
    for (int src = 0; src < p.C; ++src) {
#pragma unroll
      for (int m = 0; m < MB; ++m) sum[m] += S.recv[(src * MB + m) * msh + sr];
    }
    if (p.n_sal > 0) {
      const int8_t* qrow = p.sal_q + static_cast<long long>(o) * p.sal_stride;
      for (int tq = 0; tq < p.n_sal; tq += 16) {
        const uint4 qq = __ldg(reinterpret_cast<const uint4*>(qrow + tq));
        const unsigned qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int tt = tq + k;
          if (tt < p.n_sal) {
            const float qv = static_cast<float>(static_cast<int8_t>((qw[k >> 2] >> (8 * (k & 3))) & 0xFF));
#pragma unroll
            for (int m = 0; m < MB; ++m) sum[m] = fmaf(qv, S.xs[m * nsp + tt], sum[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      if (m < p.Mc) {
        if (p.ydt == BISCO_BF16)
          reinterpret_cast<__nv_bfloat16*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = __float2bfloat16_rn(sum[m]);
        else
          reinterpret_cast<float*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = sum[m];
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Batch rows <= 2, layers with many row tiles per cluster: the streaming kernel.
//
// A CTA's work is a grid of (row tile, unit) items: the tiles of its cluster times its
// share of the units. The packed sign words stream into a ring of shared-memory slots
// through bulk asynchronous copies (cp.async.bulk, completion counted in bytes on an
// mbarrier). A slot holds one "stage": the quads of one row tile for one
// chunk of units, which the packed layout keeps contiguous per segment, so a stage is
// one copy per segment. Every stage has its own pair of mbarriers ("landed",
// "released"), each completing exactly once: different warps consume different stages
// of one slot, so a warp may start waiting for a slot's next stage before the slot's
// current stage has landed, and per-slot barriers would alias phases of equal parity.
// Copies are issued by many warps: copies issued back to back by one thread land one
// after another, those of different warps overlap. Every warp issues part of the
// initial fill when the CTA starts (sign words do not depend on the previous kernel on
// the stream, so this runs ahead of the activations), and the first warp of a tile
// group refills a slot once its group has released the stage in it. Sign words do not depend on the previous kernel on the stream,
// so the producer starts at once and runs ahead of the activations.
//
// The 12 consumer warps split a chunk's grid into gt tile groups x gu unit groups
// (gt * gu = 12). A CTA takes at most half of an SM, so that the CTA of the next
// kernel on the stream (launched early through programmatic dependent launch) can
// stream its sign words in while this one runs its lookups. Stages are issued in an order that interleaves the tile groups, so
// all warps advance together through a ring smaller than the CTA's share. A warp
// reads its 16 bytes per lane of a stage (one 512-byte block per unit), releases the
// stage in batches of up to four items of one segment run (independent lookups keep
// the shared-memory pipe busy), applies the row scale once per (tile, run), and
// releases the stage. Per-tile sums of the unit groups are added in group order.
// ----------------------------------------------------------------------------
constexpr int kSW = 12;              // consumer warps
constexpr int kStreamMinTiles = 16;  // row tiles per cluster from which the streaming kernel is used
constexpr int kST = kSW * 32;        // threads
constexpr unsigned long long kWaitLimitNs = 200000000ull;  // bound on every mbarrier wait (200 ms)

struct SSmem {
  uint64_t* full;       // [TS] stage landed (producer arrival + bytes)
  uint64_t* empty;      // [TS] stage released by the gu warps of its tile group
  unsigned char* ring;  // [NS][CU * 512] sign words
  float* tables;        // [CU][MB][26][36]
  float* xt;            // [max_units][MB][128] scaled activations of all the CTA's units
  float* cs;            // [max_units][128] column scales
  float* rsc;           // [max_lseg][max_tiles * 32] row scales
  float* part;          // [GU][max_tiles][MB][32] partial sums per unit group
  float* recv;          // [C][MB][msh] partial sums pushed by the cluster
  float* xs;            // [MB][nsp] salient activations
};

// Stages of the largest CTA share: one per (unit chunk, row tile).
__host__ __device__ __forceinline__ int max_stages(int max_tiles, int max_units, int CU) {
  return max_tiles * ((max_units + CU - 1) / CU);
}

__host__ __device__ __forceinline__ size_t ssmem_bytes(int CU, int NS, int GU, int col_stride, int max_units,
                                                       int max_lseg, int max_tiles, int MB, int C, int n_sal) {
  const int nsp = (n_sal + 3) & ~3;
  const int msh = ((max_tiles * 32 + C - 1) / C + 3) & ~3;
  const int TS = max_stages(max_tiles, max_units, CU);
  return static_cast<size_t>((16 * TS + 127) / 128 * 128) + static_cast<size_t>(NS) * CU * 512 +
         static_cast<size_t>(CU) * col_stride + static_cast<size_t>(max_units) * MB * 128 * 4 +
         static_cast<size_t>(max_units) * 128 * 4 + static_cast<size_t>(max_lseg) * max_tiles * 32 * 4 +
         static_cast<size_t>(GU) * max_tiles * MB * 32 * 4 + static_cast<size_t>(C) * MB * msh * 4 +
         static_cast<size_t>(MB) * nsp * 4;
}

__device__ __forceinline__ SSmem scarve(unsigned char* smem, const PassParam& p, int MB, int CU, int NS, int GU) {
  SSmem s;
  unsigned char* q = smem;
  const int TS = max_stages(p.max_tiles, p.max_units, CU);
  s.full = reinterpret_cast<uint64_t*>(q);
  s.empty = s.full + TS;
  q += (16 * TS + 127) / 128 * 128;
  s.ring = q;                             q += static_cast<size_t>(NS) * CU * 512;
  s.tables = reinterpret_cast<float*>(q); q += static_cast<size_t>(CU) * p.col_stride_bytes;
  s.xt = reinterpret_cast<float*>(q);     q += static_cast<size_t>(p.max_units) * MB * 128 * 4;
  s.cs = reinterpret_cast<float*>(q);     q += static_cast<size_t>(p.max_units) * 128 * 4;
  s.rsc = reinterpret_cast<float*>(q);    q += static_cast<size_t>(p.max_lseg) * p.max_tiles * 32 * 4;
  s.part = reinterpret_cast<float*>(q);   q += static_cast<size_t>(GU) * p.max_tiles * MB * 32 * 4;
  s.recv = reinterpret_cast<float*>(q);   q += static_cast<size_t>(p.C) * MB * ((max_share(p) + 3) & ~3) * 4;
  s.xs = reinterpret_cast<float*>(q);
  return s;
}

__device__ __forceinline__ unsigned smem_addr(const void* a) { return static_cast<unsigned>(__cvta_generic_to_shared(a)); }

__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, unsigned parity) {
  unsigned done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(b)), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Waits (bounded in time) for the phase with the given parity to complete; false on
// timeout. Each barrier here completes a single phase, so the parity is always 0.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, unsigned parity) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long end = global_ns() + kWaitLimitNs;
  while (!mbar_try(b, parity))
    if (global_ns() > end) return false;
  return true;
}
// Global -> shared bulk copy whose completion is counted on mbarrier b (no multicast).
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, unsigned bytes, uint64_t* b) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(b))
               : "memory");
}

// Position of stage (tile group g, step s) among the nt stages of a chunk when the
// stages are issued step by step, tile groups interleaved. Tile group g owns tiles
// [g*nt/gt, (g+1)*nt/gt): q = nt/gt or q + 1 of them.
__host__ __device__ __forceinline__ int stage_in_chunk(int g, int s, int nt, int gt) {
  const int q = nt / gt;
  return s < q ? s * gt + g : q * gt + (g * nt / gt - g * q);
}

// Row tile (within the CTA) of stage j of a chunk: the inverse of stage_in_chunk.
__device__ __forceinline__ int stage_tile(int j, int nt, int gt) {
  const int q = nt / gt;
  if (j < q * gt) {
    const int s = j / gt, g = j - s * gt;
    return g * nt / gt + s;
  }
  int r = j - q * gt, g = 0;
  for (; g < gt - 1; ++g)
    if ((g + 1) * nt / gt - g * nt / gt > q) {
      if (r == 0) break;
      --r;
    }
  return g * nt / gt + q;
}

// Table sums of NB consecutive items (units j, j+1, ... of one stage and one run),
// added into acc[m]: one 16-byte sign load per item and lane, 26 table reads per item
// and batch row, fields paired into fp32x2 adds.
template <int MB, int NB>
__device__ __forceinline__ void lut_batch(const unsigned char* tb, const unsigned char* wp, unsigned uoff0,
                                          unsigned cstride, float* acc) {
  uint4 w[NB];
#pragma unroll
  for (int i = 0; i < NB; ++i) w[i] = *reinterpret_cast<const uint4*>(wp + i * 512);
  float a[NB][MB == 1 ? 2 : MB];
#pragma unroll
  for (int i = 0; i < NB; ++i)
#pragma unroll
    for (int m = 0; m < (MB == 1 ? 2 : MB); ++m) a[i][m] = 0.f;
  if (MB == 1) {
#pragma unroll
    for (int F = 0; F < kFields; F += 2) {
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        const unsigned uo = uoff0 + i * cstride;
        const float v0 = *reinterpret_cast<const float*>(tb + (field_off(w[i], F) | uo) + F * kFieldStride * 4);
        const float v1 = *reinterpret_cast<const float*>(tb + (field_off(w[i], F + 1) | uo) + (F + 1) * kFieldStride * 4);
        fadd2(a[i][0], a[i][1], v0, v1);
      }
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) acc[0] += a[i][0] + a[i][1];
  } else {
#pragma unroll
    for (int F = 0; F < kFields; ++F) {
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        const unsigned off = (field_off(w[i], F) | (uoff0 + i * cstride)) + F * kFieldStride * 4;
#pragma unroll
        for (int m = 0; m < MB; m += 2) {
          const float v0 = *reinterpret_cast<const float*>(tb + off + m * kFields * kFieldStride * 4);
          const float v1 = *reinterpret_cast<const float*>(tb + off + (m + 1) * kFields * kFieldStride * 4);
          fadd2(a[i][m], a[i][m + 1], v0, v1);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < NB; ++i)
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[m] += a[i][m];
  }
}

template <int MB>
__global__ void __launch_bounds__(kST, 2)
    lut_gemv_stream_kernel(const __grid_constant__ PassParam p, const int CU, const int NS, const int GU) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ci = blockIdx.x / p.C;
  const int t0 = ci * p.tiles / p.ncl, t1 = (ci + 1) * p.tiles / p.ncl, nt = t1 - t0;
  const int u0 = rank * p.units / p.C, u1 = (rank + 1) * p.units / p.C, nu = u1 - u0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nsp = (p.n_sal + 3) & ~3;
  const int seg_first = find_seg(p, u0);
  const SSmem S = scarve(smem, p, MB, CU, NS, GU);
  const int rows_c = nt * 32;
  const int msh = (max_share(p) + 3) & ~3;
  const int nchunks = (nu + CU - 1) / CU;
  const int gu = GU, gt = kSW / GU;
  const unsigned slot_bytes = static_cast<unsigned>(CU) * 512u;

  const int TS = nchunks * nt;  // stages of this CTA
  for (int i = threadIdx.x; i < TS; i += kST) {
    mbar_init(S.full + i, 1);
    mbar_init(S.empty + i, static_cast<unsigned>(gu));
  }
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncthreads();
  // Peers write into this CTA's shared memory later on; the split barrier tells them
  // that every CTA of the cluster is running before any such write happens.
  auto started = cluster.barrier_arrive();

  // Issue stage k (one lane): its units' quads of one row tile, one copy per segment,
  // into ring slot k % NS, completion counted on full[k].
  auto issue = [&](int k) {
    const int c = k / nt;
    const int t = t0 + stage_tile(k - c * nt, nt, gt);
    const int ua = u0 + c * CU, ub = ua + min(CU, nu - c * CU);
    const int nseg = p.nseg;
    unsigned bytes = 0;
#pragma unroll
    for (int sg = 0; sg < kMaxSeg; ++sg) {
      if (sg >= nseg) break;
      const SegParam& G = p.seg[sg];
      const int a = max(ua, G.unit0), b = min(ub, G.unit0 + G.nq);
      if (G.bits != nullptr && b > a) bytes += static_cast<unsigned>(b - a) * 512u;
    }
    mbar_arrive_tx(S.full + k, bytes);
    unsigned char* dst = S.ring + static_cast<size_t>(k % NS) * slot_bytes;
#pragma unroll
    for (int sg = 0; sg < kMaxSeg; ++sg) {
      if (sg >= nseg) break;
      const SegParam& G = p.seg[sg];
      const int a = max(ua, G.unit0), b = min(ub, G.unit0 + G.nq);
      if (G.bits != nullptr && b > a)
        bulk_copy(dst + (a - ua) * 512, G.bits + (static_cast<long long>(t) * G.nq + (a - G.unit0)) * 32,
                  static_cast<unsigned>(b - a) * 512u, S.full + k);
    }
  };
  // initial fill of the ring, spread over the warps
  if (lane == 0)
    for (int k = warp; k < min(NS, TS); k += kSW) issue(k);

  {
    // ---------------- consumers ----------------
    const int ga = warp / gu, gb = warp - ga * gu;  // tile group, unit group
    const int ta0 = ga * nt / gt, ta1 = (ga + 1) * nt / gt, sz = ta1 - ta0;
    bool ok = true;

    // weights-side staging before the dependency wait: column and row scales
    const int nls = find_seg(p, u1 - 1) - seg_first + 1;
    const int n_cs = nu * 16, n_rs = nls * nt * 4;
    for (int ch = threadIdx.x; ch < n_cs + n_rs; ch += kST) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.f;
      float* d;
      if (ch < n_cs) {
        const int ul = ch >> 4, j0 = (ch & 15) * 8;
        const int u = u0 + ul;
        const SegParam& G = p.seg[find_seg(p, u)];
        const int cc = (u - G.unit0) * 128 + j0;
        const int valid = G.xsrc == 2 ? 0 : max(0, min(8, G.ncols - cc));
        if (G.cscale == nullptr) {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = j < valid ? 1.f : 0.f;
        } else if (valid > 0) {
          load8(G.cscale, cc, G.cdt, valid, G.cvec != 0, v);
        }
        d = S.cs + ch * 8;
      } else {
        const int rc = ch - n_cs;
        const int ls = rc / (nt * 4), r8 = (rc - ls * nt * 4) * 8;
        const SegParam& G = p.seg[seg_first + ls];
        const int o = t0 * 32 + r8;
        const int valid = max(0, min(8, p.rows - o));
        if (G.rscale == nullptr) {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = j < valid ? 1.f : 0.f;
        } else if (valid > 0) {
          load8(G.rscale, o, G.rdt, valid, G.rvec != 0, v);
        }
        d = S.rsc + ls * p.max_tiles * 32 + r8;
      }
      reinterpret_cast<float4*>(d)[0] = make_float4(v[0], v[1], v[2], v[3]);
      reinterpret_cast<float4*>(d)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    for (int idx = threadIdx.x; idx < gu * p.max_tiles * MB * 32; idx += kST) S.part[idx] = 0.f;

    asm volatile("griddepcontrol.wait;" ::: "memory");

    for (int idx = threadIdx.x; idx < MB * p.n_sal; idx += kST) {
      const int m = idx / p.n_sal, t = idx - m * p.n_sal;
      float v = 0.f;
      const int cc = __ldg(p.sal_idx + t);
      if (cc < 0 || cc >= p.xcols) {
        atomicExch(p.status, static_cast<int>(BISCO_ERR_INVALID_ARG));
      } else if (m < p.Mc) {
        const long long i = static_cast<long long>(m) * p.ldx + cc;
        const float xv = p.xdt == BISCO_BF16
                             ? __uint_as_float(static_cast<unsigned>(__ldcg(reinterpret_cast<const unsigned short*>(p.X) + i)) << 16)
                             : __ldcg(reinterpret_cast<const float*>(p.X) + i);
        v = xv * __ldg(p.sal_scale + t);
      }
      S.xs[m * nsp + t] = v;
    }

    const unsigned char* tb = reinterpret_cast<const unsigned char*>(S.tables);
    float* my_part = S.part + static_cast<size_t>(gb) * p.max_tiles * MB * 32 + lane;
    const unsigned cstride = static_cast<unsigned>(p.col_stride_bytes);
    constexpr int kBatch = MB == 1 ? 4 : 2;
    __syncthreads();  // column scales staged
    // scaled activations of all the CTA's units at once (one round trip to L2):
    // 8-column runs, one 16-byte load each
    for (int ch = threadIdx.x; ch < nu * MB * 16; ch += kST) {
      {
        const int ulc = ch / (MB * 16);
        const int rem = ch - ulc * (MB * 16);
        const int m = rem >> 4, j0 = (rem & 15) * 8;
        const int u = u0 + ulc;
        const SegParam& G = p.seg[find_seg(p, u)];
        const int cc = (u - G.unit0) * 128 + j0;
        const int valid = max(0, min(8, G.ncols - cc));
        float xv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) xv[j] = 0.f;
        if (m < p.Mc && valid > 0 && G.xsrc != 2) {
          if (G.xsrc == 0)
            load8_l2(p.X, static_cast<long long>(m) * p.ldx + cc, p.xdt, valid, p.x_vec != 0, xv);
          else
            load8_l2(p.Z, static_cast<long long>(m) * p.ldz + cc, BISCO_F32, valid, p.z_vec != 0, xv);
        }
        const float* cv = S.cs + ulc * 128 + j0;
        float4* d4 = reinterpret_cast<float4*>(S.xt + (ulc * MB + m) * 128 + j0);
        d4[0] = make_float4(xv[0] * cv[0], xv[1] * cv[1], xv[2] * cv[2], xv[3] * cv[3]);
        d4[1] = make_float4(xv[4] * cv[4], xv[5] * cv[5], xv[6] * cv[6], xv[7] * cv[7]);
      }
    }
    for (int c = 0; c < nchunks; ++c) {
      const int cu0 = c * CU, cn = min(CU, nu - cu0);
      __syncthreads();  // activations staged (c = 0); previous chunk's tables no longer read (c > 0)
      // tables: task (unit, batch row); lane f builds the 32 signed sums of field f
      for (int tq = warp; tq < cn * MB; tq += kSW) {
        const int ulc = tq / MB, m = tq - ulc * MB;
        if (lane < kFields) {
          const float* x = S.xt + ((cu0 + ulc) * MB + m) * 128 + 5 * lane;
          const float x0 = x[0], x1 = x[1], x2 = x[2];
          const float x3 = lane < 25 ? x[3] : 0.f, x4 = lane < 25 ? x[4] : 0.f;
          const float d[5] = {2.f * x0, 2.f * x1, 2.f * x2, 2.f * x3, 2.f * x4};
          float T[32];
          T[0] = -((x0 + x1) + (x2 + x3) + x4);
#pragma unroll
          for (int e = 1; e < 32; ++e) T[e] = T[e & (e - 1)] + d[low_bit(e)];
          float* dst = S.tables + static_cast<size_t>(ulc) * (p.col_stride_bytes / 4) + (m * kFields + lane) * kFieldStride;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            reinterpret_cast<float4*>(dst)[k] = make_float4(T[4 * k], T[4 * k + 1], T[4 * k + 2], T[4 * k + 3]);
        }
      }
      __syncthreads();
      // the activations are in: let the next kernel on the stream start
      if (c == 0) asm volatile("griddepcontrol.launch_dependents;");

      // this warp's units [ub0, ub1) of the chunk, split into runs of one segment
      const int ub0 = gb * cn / gu, ub1 = (gb + 1) * cn / gu;
      auto run_end = [&](int sg) {
        return sg + 1 < p.nseg ? min(ub1, p.seg[sg + 1].unit0 - u0 - cu0) : ub1;
      };
      const int ls_first = ub1 > ub0 ? find_seg(p, u0 + cu0 + ub0) : 0;
      const int rb_first = ub1 > ub0 ? run_end(ls_first) : ub1;
      for (int st = 0; st < sz; ++st) {
        const int k = c * nt + stage_in_chunk(ga, st, nt, gt);
        const int slot = k % NS;
        if (!mbar_wait(S.full + k, 0u)) ok = false;
        const unsigned char* wp = S.ring + static_cast<size_t>(slot) * slot_bytes + lane * 16;
        const int tl = ta0 + st;
        int ra = ub0, sg = ls_first, rb = rb_first;
        while (ra < ub1) {
          float acc[MB];
#pragma unroll
          for (int m = 0; m < MB; ++m) acc[m] = 0.f;
          int j = ra;
          for (; j + kBatch <= rb; j += kBatch)
            lut_batch<MB, kBatch>(tb, wp + j * 512, static_cast<unsigned>(j) * cstride, cstride, acc);
          for (; j < rb; ++j) lut_batch<MB, 1>(tb, wp + j * 512, static_cast<unsigned>(j) * cstride, cstride, acc);
          const float rs = S.rsc[(sg - seg_first) * p.max_tiles * 32 + tl * 32 + lane];
          float* pp = my_part + tl * MB * 32;
#pragma unroll
          for (int m = 0; m < MB; ++m) sts_part(pp + m * 32, fmaf(acc[m], rs, lds_part(pp + m * 32)));
          ra = rb;
          if (ra < ub1) {
            sg = find_seg(p, u0 + cu0 + ra);
            rb = run_end(sg);
          }
        }
        if (k + NS < TS) {  // release the slot; the group's first warp refills it
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(S.empty + k);
            if (gb == 0) {
              if (!mbar_wait(S.empty + k, 0u)) ok = false;
              issue(k + NS);
            }
          }
          __syncwarp();
        }
      }
    }
    if (nchunks == 0) asm volatile("griddepcontrol.launch_dependents;");
    if (!ok) atomicExch(p.status, static_cast<int>(BISCO_ERR_TIMEOUT));
  }
  __syncthreads();  // all partial sums are in shared memory; every copy has landed
  // (every stage was waited for by its tile group; after a timeout this makes sure no
  // copy is still writing into shared memory when the CTA exits)
  if (threadIdx.x == 0)
    for (int k = max(0, TS - NS); k < TS; ++k)
      if (!mbar_wait(S.full + k, 0u)) atomicExch(p.status, static_cast<int>(BISCO_ERR_TIMEOUT));

  // ---- sum over unit groups (fixed order) and push to the CTA that owns each row ----
  cluster.barrier_wait(std::move(started));
  for (int idx = threadIdx.x; idx < nt * MB * 32; idx += kST) {
    const int tl = idx / (MB * 32);
    const int rem = idx - tl * MB * 32;
    const int m = rem >> 5, ln = rem & 31;
    float v = 0.f;
    for (int g = 0; g < gu; ++g) v += S.part[(static_cast<size_t>(g) * p.max_tiles + tl) * MB * 32 + m * 32 + ln];
    const int lr = tl * 32 + ln;
    const int dst = share_owner(lr, rows_c, p.C);
    float* rp = cluster.map_shared_rank(S.recv, dst);
    rp[(rank * MB + m) * msh + (lr - share_begin(dst, rows_c, p.C))] = v;
  }
  cluster.sync();  // all partial sums have landed

  // ---- reduce this CTA's share of rows in CTA-rank order, add salient columns, store ----
  const int r0 = share_begin(rank, rows_c, p.C), r1 = share_begin(rank + 1, rows_c, p.C);
  for (int lr = r0 + threadIdx.x; lr < r1; lr += kST) {
    const int o = t0 * 32 + lr;
    if (o >= p.rows) continue;
    const int sr = lr - r0;
    float sum[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) sum[m] = 0.f;
    for (int src = 0; src < p.C; ++src) {
#pragma unroll
      for (int m = 0; m < MB; ++m) sum[m] += S.recv[(src * MB + m) * msh + sr];
    }
    if (p.n_sal > 0) {
      const int8_t* qrow = p.sal_q + static_cast<long long>(o) * p.sal_stride;
      for (int tq = 0; tq < p.n_sal; tq += 16) {
        const uint4 qq = __ldg(reinterpret_cast<const uint4*>(qrow + tq));
        const unsigned qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int tt = tq + k;
          if (tt < p.n_sal) {
            const float qv = static_cast<float>(static_cast<int8_t>((qw[k >> 2] >> (8 * (k & 3))) & 0xFF));
#pragma unroll
            for (int m = 0; m < MB; ++m) sum[m] = fmaf(qv, S.xs[m * nsp + tt], sum[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      if (m < p.Mc) {
        if (p.ydt == BISCO_BF16)
          reinterpret_cast<__nv_bfloat16*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = __float2bfloat16_rn(sum[m]);
        else
          reinterpret_cast<float*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = sum[m];
      }
    }
  }
}

template <int MB>
cudaError_t set_attrs() {
  const int lim = static_cast<int>(query_smem_limit());
  cudaError_t e = cudaFuncSetAttribute(lut_gemv_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
  if (e == cudaSuccess && MB <= 2)
    e = cudaFuncSetAttribute(lut_gemv_stream_kernel<MB <= 2 ? MB : 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
  if (e == cudaSuccess && MB <= 2)
    e = cudaFuncSetAttribute(lut_gemv_warp_kernel<MB <= 2 ? MB : 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
  return e;
}

template <int MB>
cudaError_t launch_mb(const PassParam& p, const Plan& plan, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.ncl * plan.C);
  cfg.blockDim = dim3(plan.kind == 2 ? kST : plan.kind == 0 ? kTW : kThreads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  if constexpr (MB <= 2) {
    if (plan.kind == 2) return cudaLaunchKernelEx(&cfg, lut_gemv_stream_kernel<MB>, p, plan.cu, plan.ns, plan.gu);
    if (plan.kind == 0) return cudaLaunchKernelEx(&cfg, lut_gemv_warp_kernel<MB>, p, plan.cu);
  }
  return cudaLaunchKernelEx(&cfg, lut_gemv_kernel<MB>, p, plan.cu);
}

template <typename Kernel>
int max_active_clusters_of(Kernel kernel, int threads, int C, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) return 0;
  return n;
}

int max_active_clusters(int MB, int kind, int C, size_t smem) {
  if (kind == 2) {
    if (MB == 1) return max_active_clusters_of(lut_gemv_stream_kernel<1>, kST, C, smem);
    if (MB == 2) return max_active_clusters_of(lut_gemv_stream_kernel<2>, kST, C, smem);
    return 0;
  }
  if (kind == 0) {
    if (MB == 1) return max_active_clusters_of(lut_gemv_warp_kernel<1>, kTW, C, smem);
    if (MB == 2) return max_active_clusters_of(lut_gemv_warp_kernel<2>, kTW, C, smem);
    return 0;
  }
  switch (MB) {
    case 1: return max_active_clusters_of(lut_gemv_kernel<1>, kThreads, C, smem);
    case 2: return max_active_clusters_of(lut_gemv_kernel<2>, kThreads, C, smem);
    case 4: return max_active_clusters_of(lut_gemv_kernel<4>, kThreads, C, smem);
    case 8: return max_active_clusters_of(lut_gemv_kernel<8>, kThreads, C, smem);
    default: return 0;
  }
}

size_t plan_smem(const Plan& pl, int CU, int n_sal) {
  const int nsp = (n_sal + 3) & ~3;
  const int msh = ((pl.max_tiles * 32 + pl.C - 1) / pl.C + 3) & ~3;
  if (pl.kind == 0)
    return wsmem_bytes(CU, pl.col_stride_bytes, pl.max_units, pl.max_lseg, pl.max_tiles, pl.MB, pl.C, n_sal);
  if (pl.kind == 2)
    return ssmem_bytes(CU, pl.ns, pl.gu, pl.col_stride_bytes, pl.max_units, pl.max_lseg, pl.max_tiles, pl.MB, pl.C,
                       n_sal);
  return static_cast<size_t>(CU) * pl.col_stride_bytes + static_cast<size_t>(pl.max_units) * 128 * 4 +
         static_cast<size_t>(pl.max_lseg) * pl.max_tiles * 32 * 4 + static_cast<size_t>(pl.max_tiles) * pl.MB * 32 * 4 +
         static_cast<size_t>(pl.C) * pl.MB * msh * 4 + static_cast<size_t>(pl.MB) * nsp * 4 +
         static_cast<size_t>(pl.max_units) * sizeof(UnitInfo);
}

// Split of the consumer warps into kSW/gu tile groups x gu unit groups for an nt x nu
// grid: the largest rectangle in items, plus half an item per stage for the per-stage
// work (wait, row scales, release); smallest gu on ties (longer unit runs).
int pick_gu(int nt, int nu) {
  int best = 1;
  long long cost = 1ll << 60;
  for (int gu = 1; gu <= kSW; ++gu) {
    if (kSW % gu) continue;
    const int gt = kSW / gu;
    const long long tiles = (nt + gt - 1) / gt;
    const long long c = 2 * tiles * ((nu + gu - 1) / gu) + tiles;
    if (c < cost) { cost = c; best = gu; }
  }
  return best;
}

// Largest number of distinct segments touched by one CTA's unit range.
int max_segments_per_cta(int units, int C, const int* seg_unit0, int nseg) {
  auto seg_of = [&](int u) {
    int s = 0;
    for (int k = 1; k < nseg; ++k)
      if (u >= seg_unit0[k]) s = k;
    return s;
  };
  int m = 1;
  for (int r = 0; r < C; ++r) {
    const int u0 = r * units / C, u1 = (r + 1) * units / C;
    if (u1 > u0) m = std::max(m, seg_of(u1 - 1) - seg_of(u0) + 1);
  }
  return m;
}

// Streaming-kernel plan for batch rows <= 2: cluster size, unit chunk, ring depth.
// The cluster size minimises a cost model in shared-memory wavefronts per SM: the
// lookups and sign reads of the largest CTA share, its tables, and a fixed cost for
// the cluster reduction; clusters are limited to those that fit one CTA per SM.
Plan make_stream_plan(int rows, int units, const int* seg_unit0, int nseg, int MB, int n_sal, size_t smem_limit,
                      size_t budget) {
  const int tiles = (rows + 31) / 32;
  Plan best{};
  long long best_cost = -1;
  for (int C = 1; C <= kMaxCluster; C *= 2) {
    if (C > units) break;
    Plan pl{};
    pl.kind = 2;
    pl.MB = MB;
    pl.C = C;
    pl.col_stride_bytes = (MB * kFields * kFieldStride * 4 + 127) / 128 * 128;
    pl.max_units = (units + C - 1) / C;
    pl.max_lseg = max_segments_per_cta(units, C, seg_unit0, nseg);
    int fit = max_active_clusters(MB, 2, C, std::max<size_t>(budget, smem_limit / 2 + 1024));
    if (fit <= 0) continue;
    pl.ncl = std::max(1, std::min(tiles, fit));
    pl.max_tiles = (tiles + pl.ncl - 1) / pl.ncl;
    // largest unit chunk whose ring can hold min(4, stages) stages
    bool ok = false;
    for (int cu = pl.max_units; cu >= 1 && !ok; --cu) {
      pl.cu = cu;
      pl.gu = pick_gu(pl.max_tiles, std::min(cu, pl.max_units));
      const int stages = pl.max_tiles * ((pl.max_units + cu - 1) / cu);
      pl.ns = 0;
      const size_t fixed = plan_smem(pl, cu, n_sal);
      if (fixed + 512 + static_cast<size_t>(cu) * 512 > budget) continue;
      const int fit_ns = static_cast<int>((budget - fixed - 512) / (static_cast<size_t>(cu) * 512));
      pl.ns = std::min({stages, fit_ns, 32});
      if (pl.ns >= std::min(stages, 4)) ok = true;
    }
    if (!ok) continue;
    pl.smem = plan_smem(pl, pl.cu, n_sal);
    const int nchunks = (pl.max_units + pl.cu - 1) / pl.cu;
    const long long cost = static_cast<long long>(pl.max_tiles) * pl.max_units * (26 * MB + 4) +
                           static_cast<long long>(pl.max_units) * 26 * MB + (C > 1 ? 600 : 0) + (nchunks - 1) * 600;
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = pl; }
  }
  return best;
}

}  // namespace

int query_num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

size_t query_smem_limit() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return n > 0 ? static_cast<size_t>(n) : 48 * 1024;
}

Plan make_plan(int rows, int units, const int* seg_unit0, int nseg, int MB, int n_sal, int num_sms,
               size_t smem_limit) {
  ensure_kernel_attrs();
  const int tiles = (rows + 31) / 32;
  if (MB <= 2) {
    // Prefer plans that leave room on each SM for a CTA of the next kernel.
    Plan s = make_stream_plan(rows, units, seg_unit0, nseg, MB, n_sal, smem_limit, smem_limit / 2 - 1024);
    if (s.C == 0) s = make_stream_plan(rows, units, seg_unit0, nseg, MB, n_sal, smem_limit, smem_limit);
    // The streaming kernel pays off when each cluster streams many row tiles; with
    // few, the 16-warp kernel's shorter start-up wins.
    if (s.C > 0 && s.max_tiles >= kStreamMinTiles) return s;
  }
  Plan pl{};
  pl.MB = MB;
  pl.kind = MB <= 2 ? 0 : 1;
  pl.C = std::max(1, std::min(kMaxCluster, units));
  pl.col_stride_bytes = (MB * kFields * kFieldStride * 4 + 127) / 128 * 128;
  pl.max_units = (units + pl.C - 1) / pl.C;
  pl.max_lseg = max_segments_per_cta(units, pl.C, seg_unit0, nseg);
  // Clusters that fit with at most one CTA per SM (a CTA that shares its SM with
  // another CTA of the same launch would take twice as long). The query uses a
  // shared-memory size that forces one CTA per SM.
  int fit = max_active_clusters(MB, pl.kind, pl.C, smem_limit / 2 + 1024);
  if (fit <= 0) fit = std::max(1, num_sms / pl.C);
  pl.ncl = std::max(1, std::min(tiles, fit));
  pl.max_tiles = (tiles + pl.ncl - 1) / pl.ncl;
  pl.cu = pl.max_units;
  // for the 16-warp kernel prefer a chunk size that leaves room for a CTA of the next
  // kernel on the same SM (programmatic dependent launch)
  if (pl.kind == 0)
    while (pl.cu > 1 && plan_smem(pl, pl.cu, n_sal) > smem_limit / 2 - 2048) --pl.cu;
  while (pl.cu > 1 && plan_smem(pl, pl.cu, n_sal) > smem_limit) --pl.cu;
  pl.smem = plan_smem(pl, pl.cu, n_sal);
  return pl;
}

cudaError_t ensure_kernel_attrs() {
  static std::once_flag once[64];
  static cudaError_t err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::call_once(once[dev & 63], [&] {
    cudaError_t r = set_attrs<1>();
    if (r == cudaSuccess) r = set_attrs<2>();
    if (r == cudaSuccess) r = set_attrs<4>();
    if (r == cudaSuccess) r = set_attrs<8>();
    err[dev & 63] = r;
  });
  return err[dev & 63];
}

cudaError_t launch_pass(const PassParam& p, const Plan& plan, cudaStream_t stream, bool pdl) {
  const cudaError_t e = ensure_kernel_attrs();
  if (e != cudaSuccess) return e;
  switch (plan.MB) {
    case 1: return launch_mb<1>(p, plan, stream, pdl);
    case 2: return launch_mb<2>(p, plan, stream, pdl);
    case 4: return launch_mb<4>(p, plan, stream, pdl);
    case 8: return launch_mb<8>(p, plan, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace bisco

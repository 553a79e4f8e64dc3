// Binary-weight decode GEMV for batches of up to 8 rows per launch on the integer
// tensor cores (mma.sync, s8 x s8 -> s32), sm_100a.
//
// Per output row o and batch row m the kernel computes
//   y[m][o] = sum_seg rs_seg[o] * sum_i sign_seg[o][i] * v_seg[m][i]   (+ salient term)
// where a "segment" is one packed sign matrix: a binary base B_k with v = c_k (.) x and
// rs = r_k ("FluxBin", Sec. 3.1, decoupled row-column binary bases; the column scale is
// folded into the activation as in Sec. 3.2, Stage 1), the correction's V with v = x and
// rs = alpha, or its U^T with v = z ("BiLoCo", "The core idea": alpha * u * (v . x)).
// A stored bit b means the sign (2b - 1) (FluxBin Sec. 3.2). A layer with FluxBin's
// binary salient refinement (Sec. 4) has that term computed by a small launch just
// before this one into an fp32 buffer, which the owner of each output row adds last.
//
// Formulation. With bits b_i in {0, 1},
//   sum_i (2 b_i - 1) v_i = 2 * sum_i b_i v_i - sum_i v_i,
// so the tensor cores only ever multiply by the bits themselves. The activations of a
// segment are written exactly in fixed point relative to the largest magnitude among
// the CTA's columns of that segment: V_i = round(v_i * 2^s) with |V_i| <= 2^22, and V_i
// is split into three signed 8-bit digits, V_i = d0 * 2^16 + d1 * 2^8 + d2. Every pair
// (batch row, digit) is one column ("slot") of the MMA's B operand: n = 3 m + digit, so
// one 8-column MMA holds two batch rows, and up to 8 batch rows take three.
//
// The A operand never leaves the registers. A lane holds the 32-bit sign words of its
// rows; (word & (0x01010101 << b)) is four bytes with values {0, 2^b} at columns
// b, b+8, b+16, b+24 of the word, and the same mask on (word >> 4) gives columns
// b+4, b+12, b+20, b+28. One m16n8k32 MMA per mask b (b = 0..3) covers a 16-row x
// 128-column block; each b has its own accumulator (its products carry the factor 2^b),
// and sum_b (D_b >> b) is exact. The MMA's k index is a permutation of the columns
// (the B fragments are written in the same permutation), which is what lets one
// logic op per register extract the bits.
//
// Work decomposition. Clusters of C CTAs (one CTA per SM). A cluster owns a range of
// 32-row tiles; CTA r of the cluster owns 1/C of the units (128-column quads over all
// segments). Before griddepcontrol.wait (programmatic dependent launch) the CTA starts
// bulk copies of all its sign words into shared memory (one copy per row tile and
// segment run, completion counted on one mbarrier per tile) and stages its column and
// row scales: none of this depends on the previous kernel. After the wait it stages the
// activations, finds the per-segment scale, writes the B fragments, and the 16 warps
// run through the (row block, unit) items of the CTA in equal contiguous ranges. Row
// partial sums meet in shared memory (warp order), then in the owning CTA of the
// cluster through distributed shared memory (CTA-rank order): results are
// deterministic.

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <utility>

#include "bisco_device.cuh"
#include "bisco_internal.h"

namespace cg = cooperative_groups;

namespace bisco {

namespace {

constexpr int kIW = 8;                  // warps per CTA
constexpr int kIT = kIW * 32;           // threads per CTA
constexpr int kMaxSlots = 24;           // 3 digits x 8 batch rows
constexpr unsigned kByteMask = 0x01010101u;

__host__ __device__ constexpr int groups_of(int MB) { return (3 * MB + 7) / 8; }
__host__ __device__ constexpr int block_rows(int MB) { return groups_of(MB) == 1 ? 32 : 16; }

// Shared-memory carve-up (sizes from the plan; every region 16-byte aligned).
struct ISmem {
  uint64_t* bar;           // [max_tiles]                 sign words of a row tile landed
  int* useg;               // [max_units]                 local segment of a unit
  int* lsstart;            // [max_lseg]                  start (local unit index) of a local segment
  int* lsend;              // [max_lseg]                  end (local unit index) of a local segment
  int* lsbits;             // [max_lseg]                  1 if the segment has sign bits
  int2* lsinfo;            // [max_lseg]                  (segment, row-scale group) of a local part
  unsigned* xmax;          // [max_lseg][MB]              max |v| (float bits) over the CTA's columns
  unsigned long long* vsum;  // [max_lseg][MB]            sum of the fixed-point values V (two's complement)
  int* flags;              // [4]                         [0]: a wait timed out
  float* wsl;              // [max_lseg][kMaxSlots]       slot weight 2^(17 - 8 digit - s)
  float* ssf;              // [max_lseg][MB]              sum of the CTA's quantised v per segment
  unsigned char* ring;     // [max_tiles][max_units][512] sign words
  float* xt;               // [max_units][MB][128]        activations times column scales
  uint4* bfr;              // [max_units][NG][32][2]      B fragments, 8 words per lane
  float* cs;               // [max_units][128]            column scales (0 past the segment's columns)
  float* rsc;              // [max_lseg][max_tiles * 32]  row scales
  float* recv;             // [C][kc][msh][MB]            row partial sums pushed by the warps of the cluster
  float* xs;               // [MB][nsp]                   salient activations x[idx_t] * s_t
};

__host__ __device__ __forceinline__ size_t a16(size_t n) { return (n + 15) & ~size_t(15); }

__host__ __device__ __forceinline__ int msh_of(int max_tiles, int C) { return ((max_tiles * 32 + C - 1) / C + 3) & ~3; }

__host__ __device__ __forceinline__ size_t ismem_bytes(int MB, int C, int max_tiles, int max_units, int max_lseg,
                                                       int nbw, int n_sal) {
  const int NG = groups_of(MB), RB = block_rows(MB);
  const int nsp = (n_sal + 3) & ~3;
  size_t n = 0;
  n += a16(static_cast<size_t>(max_tiles) * 8);
  n += a16(static_cast<size_t>(max_units) * 4);
  n += 3 * a16(static_cast<size_t>(max_lseg) * 4);
  n += a16(static_cast<size_t>(max_lseg) * 8);
  n += a16(static_cast<size_t>(max_lseg) * MB * 4);
  n += a16(static_cast<size_t>(max_lseg) * MB * 8);
  n += 16;
  n += a16(static_cast<size_t>(max_lseg) * kMaxSlots * 2 * 4);
  n += a16(static_cast<size_t>(max_lseg) * MB * 4);
  n += static_cast<size_t>(max_tiles) * max_units * 512;
  n += static_cast<size_t>(max_units) * MB * 512;
  n += static_cast<size_t>(max_units) * NG * 1024;
  n += static_cast<size_t>(max_units) * 512;
  n += static_cast<size_t>(max_lseg) * max_tiles * 128;
  n += a16(static_cast<size_t>(C) * nbw * msh_of(max_tiles, C) * MB * 4);
  n += a16(static_cast<size_t>(MB) * nsp * 4);
  return n;
}

__device__ __forceinline__ ISmem icarve(unsigned char* smem, const PassParam& p, int MB, int nbw) {
  const int NG = groups_of(MB), RB = block_rows(MB);
  const int nsp = (p.n_sal + 3) & ~3;
  ISmem s;
  unsigned char* q = smem;
  s.bar = reinterpret_cast<uint64_t*>(q);            q += a16(static_cast<size_t>(p.max_tiles) * 8);
  s.useg = reinterpret_cast<int*>(q);                q += a16(static_cast<size_t>(p.max_units) * 4);
  s.lsstart = reinterpret_cast<int*>(q);             q += a16(static_cast<size_t>(p.max_lseg) * 4);
  s.lsend = reinterpret_cast<int*>(q);               q += a16(static_cast<size_t>(p.max_lseg) * 4);
  s.lsbits = reinterpret_cast<int*>(q);              q += a16(static_cast<size_t>(p.max_lseg) * 4);
  s.lsinfo = reinterpret_cast<int2*>(q);             q += a16(static_cast<size_t>(p.max_lseg) * 8);
  s.xmax = reinterpret_cast<unsigned*>(q);           q += a16(static_cast<size_t>(p.max_lseg) * MB * 4);
  s.vsum = reinterpret_cast<unsigned long long*>(q); q += a16(static_cast<size_t>(p.max_lseg) * MB * 8);
  s.flags = reinterpret_cast<int*>(q);               q += 16;
  s.wsl = reinterpret_cast<float*>(q);               q += a16(static_cast<size_t>(p.max_lseg) * kMaxSlots * 2 * 4);
  s.ssf = reinterpret_cast<float*>(q);               q += a16(static_cast<size_t>(p.max_lseg) * MB * 4);
  s.ring = q;                                        q += static_cast<size_t>(p.max_tiles) * p.max_units * 512;
  s.xt = reinterpret_cast<float*>(q);                q += static_cast<size_t>(p.max_units) * MB * 512;
  s.bfr = reinterpret_cast<uint4*>(q);               q += static_cast<size_t>(p.max_units) * NG * 1024;
  s.cs = reinterpret_cast<float*>(q);                q += static_cast<size_t>(p.max_units) * 512;
  s.rsc = reinterpret_cast<float*>(q);               q += static_cast<size_t>(p.max_lseg) * p.max_tiles * 128;
  s.recv = reinterpret_cast<float*>(q);              q += a16(static_cast<size_t>(p.C) * nbw * msh_of(p.max_tiles, p.C) * MB * 4);
  s.xs = reinterpret_cast<float*>(q);
  (void)nsp;
  return s;
}

__device__ __forceinline__ int seg_of_unit(const PassParam& p, int u) {
  int s = 0;
#pragma unroll
  for (int k = 1; k < kMaxSeg; ++k)
    if (k < p.nseg && u >= p.seg[k].unit0) s = k;
  return s;
}

// Pass-wide index of the (segment, row-scale group) part holding unit u: a segment
// without grouped row scales is one part.
__device__ __forceinline__ int part_of_unit(const PassParam& p, int u) {
  const SegParam& G = p.seg[seg_of_unit(p, u)];
  return G.part0 + (G.rgu > 0 ? (u - G.unit0) / G.rgu : 0);
}

__device__ __forceinline__ int share_begin_i(int d, int R, int C) { return d * R / C; }
__device__ __forceinline__ int share_owner_i(int r, int R, int C) { return ((r + 1) * C - 1) / R; }

// Fixed-point exponent of a segment: V = round(v * 2^s) keeps |V| <= 2^22 for every
// |v| <= vmax. vmax == 0 gives s = 0 (every V is 0).
__device__ __forceinline__ int fixed_shift(float vmax) {
  // vmax = f * 2^e with f in [0.5, 1): for a normal float e is the biased exponent - 126
  const int eb = static_cast<int>((__float_as_uint(vmax) >> 23) & 0xFFu);
  if (eb != 0) return 22 - (eb - 126);
  if (!(vmax > 0.f)) return 0;
  int e;
  frexpf(vmax, &e);  // subnormal
  return 22 - e;
}
// 2^k for any integer k in [-252, 252], as the product of two representable factors.
__device__ __forceinline__ void pow2_pair(int k, float& f1, float& f2) {
  const int k1 = max(-126, min(127, k));
  const int k2 = max(-126, min(127, k - k1));
  f1 = __int_as_float((k1 + 127) << 23);
  f2 = __int_as_float((k2 + 127) << 23);
}

// A holds the masked sign bytes, values 0 or 2^b <= 8, so the signed 8-bit type is exact.
__device__ __forceinline__ void mma_s8s8(int (&c)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3, unsigned b0,
                                         unsigned b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The low byte of x, sign-extended.
__device__ __forceinline__ int sext8(int x) { return static_cast<int>(static_cast<signed char>(x & 0xFF)); }

// One launch computes one pass (MULTI = false: role 0), or several side by side on
// disjoint clusters (MULTI = true): roles that compute a z = alpha (.) (V x) into the
// workspace come first and count their CTAs done on a ready counter; an output role that
// reads a z runs its base units first, then, after a bounded wait for that counter, its
// U^T units. Every CTA of the grid is resident before the next kernel on the stream can
// start, and the z roles wait for nothing but the previous kernel, so the wait always
// ends; it is bounded anyway (BISCO_ERR_TIMEOUT).
template <int MB, bool MULTI>
__global__ void __launch_bounds__(kIT, 2)
    imma_gemv_kernel(const __grid_constant__ ImmaLaunch L, const int kc, const int dbg_skip_tile,
                     const unsigned long long wait_ns) {
  constexpr int NG = groups_of(MB);
  constexpr int RB = block_rows(MB);   // rows per work item
  constexpr int RH = RB / 16;          // 16-row MMA blocks per item
  constexpr int BPT = 32 / RB;         // items (row blocks) per row tile
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ci_all = blockIdx.x / L.pass[0].C;
  int role = 0;
  if (MULTI)
    for (int r = 1; r < L.rt.nroles; ++r)
      if (ci_all >= L.rt.cl0[r]) role = r;
  constexpr bool fused = MULTI;
  const bool role_z = MULTI && L.rt.is_z[role] != 0;
  const int zsrc = MULTI ? L.rt.zsrc[role] : -1;  // the role whose z this output role reads
  const PassParam& p = L.pass[role];
  const int ci = ci_all - (MULTI ? L.rt.cl0[role] : 0);
  const int t0 = ci * p.tiles / p.ncl, t1 = (ci + 1) * p.tiles / p.ncl, nt = t1 - t0;
  const int u0 = rank * p.units / p.C, u1 = (rank + 1) * p.units / p.C, nu = u1 - u0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, tq = lane & 3;
  const int nsp = (p.n_sal + 3) & ~3;
  // local parts: the (segment, row-scale group) pairs this CTA's units touch, in order
  const int part_first = nu > 0 ? part_of_unit(p, u0) : 0;
  const int nls = nu > 0 ? part_of_unit(p, u1 - 1) - part_first + 1 : 0;
  const ISmem S = icarve(smem, p, MB, kc);
  const int rows_c = nt * 32;
  const int msh = msh_of(p.max_tiles, p.C);
  // counters in the workspace's status region: words 32 + r are the ready counters of
  // the z roles, word 48 counts the grid's CTAs done
  int* const z_ready = p.status + 32 + (role_z ? role : max(zsrc, 0));
  int* const z_done = p.status + 48;

  // ---- set-up: barriers, unit table, counters ----
  for (int i = threadIdx.x; i < nt; i += kIT) dev::mbar_init(S.bar + i, 1);
  for (int ul = threadIdx.x; ul < nu; ul += kIT) {
    const int u = u0 + ul;
    const int sg = seg_of_unit(p, u);
    const SegParam& G = p.seg[sg];
    const int grp = G.rgu > 0 ? (u - G.unit0) / G.rgu : 0;
    const int lp = G.part0 + grp - part_first;
    S.useg[ul] = lp;
    if (ul == 0 || part_of_unit(p, u - 1) != G.part0 + grp) {  // first unit of its part
      S.lsstart[lp] = ul;
      S.lsbits[lp] = G.bits != nullptr ? 1 : 0;
      S.lsinfo[lp] = make_int2(sg, grp);
    }
    if (ul == nu - 1 || part_of_unit(p, u + 1) != G.part0 + grp) S.lsend[lp] = ul + 1;
  }
  for (int i = threadIdx.x; i < nls * MB; i += kIT) { S.xmax[i] = 0u; S.vsum[i] = 0ull; }
  if (threadIdx.x == 0) { S.flags[0] = 0; S.flags[1] = 0; }
  for (int i = threadIdx.x; i < p.C * kc * msh * MB; i += kIT) S.recv[i] = 0.f;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncthreads();
  // Peers write into this CTA's shared memory at the end; the split barrier tells them
  // that every CTA of the cluster is running before any such write happens.
  auto started = cluster.barrier_arrive();

  // ---- column and row scales (weights only: before the dependency wait; issued ahead of
  //      the sign-word copies so that they are not queued behind them) ----
  {
    const int n_cs = nu * 16, n_rs = nls * nt * 4;
    for (int ch = threadIdx.x; ch < n_cs + n_rs; ch += kIT) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.f;
      float* d;
      if (ch < n_cs) {
        const int ul = ch >> 4, j0 = (ch & 15) * 8;
        const int u = u0 + ul;
        const SegParam& G = p.seg[seg_of_unit(p, u)];
        const int cc = (u - G.unit0) * 128 + j0;
        const int valid = G.xsrc == 2 ? 0 : max(0, min(8, G.ncols - cc));
        if (G.cscale == nullptr) {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = j < valid ? 1.f : 0.f;
        } else if (valid > 0) {
          dev::load8_ro(G.cscale, cc, G.cdt, valid, G.cvec != 0, v);
        }
        d = S.cs + ch * 8;
      } else {
        const int rc = ch - n_cs;
        const int ls = rc / (nt * 4), r8 = (rc - ls * nt * 4) * 8;
        const int2 li = S.lsinfo[ls];
        const SegParam& G = p.seg[li.x];
        const int o = t0 * 32 + r8;
        const int valid = max(0, min(8, p.rows - o));
        if (G.rscale == nullptr) {
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = j < valid ? 1.f : 0.f;
        } else if (valid > 0) {
          // group li.y's scale vector (the host clears rvec when a group offset would break
          // the 16-byte alignment)
          dev::load8_ro(G.rscale, static_cast<long long>(li.y) * G.rgstride + o, G.rdt, valid, G.rvec != 0, v);
        }
        d = S.rsc + ls * p.max_tiles * 32 + r8;
      }
      reinterpret_cast<float4*>(d)[0] = make_float4(v[0], v[1], v[2], v[3]);
      reinterpret_cast<float4*>(d)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
  // ---- sign words: one bulk copy per (row tile, segment run), issued by many warps ----
  if (lane == 0) {
    for (int tl = warp; tl < nt; tl += kIW) {
      const int t = t0 + tl;
      unsigned bytes = 0;
#pragma unroll
      for (int sg = 0; sg < kMaxSeg; ++sg) {
        if (sg >= p.nseg) break;
        const SegParam& G = p.seg[sg];
        const int a = max(u0, G.unit0), b = min(u1, G.unit0 + G.nq);
        if (G.bits != nullptr && b > a) bytes += static_cast<unsigned>(b - a) * 512u;
      }
      if (tl == dbg_skip_tile) continue;  // test hook: this tile's copies never start
      dev::mbar_arrive_tx(S.bar + tl, bytes);
      unsigned char* dst = S.ring + static_cast<size_t>(tl) * nu * 512;
#pragma unroll
      for (int sg = 0; sg < kMaxSeg; ++sg) {
        if (sg >= p.nseg) break;
        const SegParam& G = p.seg[sg];
        const int a = max(u0, G.unit0), b = min(u1, G.unit0 + G.nq);
        if (G.bits != nullptr && b > a)
          dev::bulk_copy(dst + static_cast<size_t>(a - u0) * 512,
                         G.bits + (static_cast<long long>(t) * G.nq + (a - G.unit0)) * 32,
                         static_cast<unsigned>(b - a) * 512u, S.bar + tl);
      }
    }
  }

  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();  // column scales visible

  // ---- salient activations (gathered and scaled) ----
  for (int idx = threadIdx.x; idx < MB * p.n_sal; idx += kIT) {
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

  // ---- phases: the units that do not read z, then (fused launches) the U^T units ----
  int uT = nu;  // first local unit of a z-reading segment
  const bool waits = fused && zsrc >= 0;  // an output role that reads a z
  if (waits)
    for (int ls = 0; ls < nls; ++ls)
      if (p.seg[S.lsinfo[ls].x].xsrc == 1) { uT = min(uT, S.lsstart[ls]); }
  const int nph = (waits && uT < nu && uT > 0) ? 2 : 1;
  const int kcp = kc / (fused ? 2 : 1);  // contributor slots per phase
  bool ok = true;
  bool waited = false;  // this thread has completed the cluster barrier started above
  for (int ph = 0; ph < nph; ++ph) {
    const int pa = nph == 1 ? 0 : (ph == 0 ? 0 : uT);
    const int pb = nph == 1 ? nu : (ph == 0 ? uT : nu);
    const int nun = pb - pa;
    const bool reads_z = waits && (ph == 1 || (nph == 1 && uT == 0));
    if (reads_z) {
      // z is read from here on: wait (bounded) until every z-producing CTA has counted
      // its stores
      if (threadIdx.x == 0) {
        const int target = (L.rt.cl0[zsrc + 1] - L.rt.cl0[zsrc]) * p.C;
        const unsigned long long end = dev::global_ns() + wait_ns;
        bool ready = false;
        while (!ready) {
          int v;
          asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(z_ready) : "memory");
          ready = v >= target;
          if (!ready && dev::global_ns() > end) break;
        }
        if (!ready) {
          atomicExch(p.status, static_cast<int>(BISCO_ERR_TIMEOUT));
          S.flags[1] = 1;
        } else {
          S.flags[1] = 0;
        }
      }
      __syncthreads();
    }

    // ---- activations: v = xin * c per (unit, batch row) in column order, 16-byte loads of
    //      8 consecutive columns, and the maximum |v| per (segment, batch row) ----
    {
      const int total = nun * MB * 16;
      for (int base = 0; base < total; base += kIT) {
        const int ch = base + threadIdx.x;
        float mx = 0.f;
        int lsm = -1;
        if (ch < total) {
          const int ulm = pa * MB + (ch >> 4), j0 = (ch & 15) * 8;
          const int ul = ulm / MB, m = ulm - ul * MB;
          const int u = u0 + ul;
          const int sg = seg_of_unit(p, u);
          const SegParam& G = p.seg[sg];
          const int cc = (u - G.unit0) * 128 + j0;
          const int valid = max(0, min(8, G.ncols - cc));
          float xv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) xv[j] = 0.f;
          if (m < p.Mc && valid > 0 && G.xsrc != 2) {
            if (G.xsrc == 0)
              dev::load8_act(p.X, static_cast<long long>(m) * p.ldx + cc, p.xdt, valid, p.x_vec != 0, xv);
            else
              dev::load8_act(p.Z, static_cast<long long>(m) * p.ldz + cc, BISCO_F32, valid, p.z_vec != 0, xv);
          }
          const float* cv = S.cs + ul * 128 + j0;
          float v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            v[j] = xv[j] * cv[j];
            mx = fmaxf(mx, fabsf(v[j]));
          }
          float4* d4 = reinterpret_cast<float4*>(S.xt + static_cast<size_t>(ulm) * 128 + j0);
          d4[0] = make_float4(v[0], v[1], v[2], v[3]);
          d4[1] = make_float4(v[4], v[5], v[6], v[7]);
          lsm = S.useg[ul] * MB + m;
        }
        // the 16 lanes of a half-warp share one (unit, batch row)
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if ((lane & 15) == 0 && lsm >= 0) atomicMax(S.xmax + lsm, __float_as_uint(mx));
      }
    }
    __syncthreads();  // activations and their maxima complete

    // ---- B fragments: task (unit, batch row, lane-in-group t, mask b, half r) writes the
    //      words of slots 3m, 3m+1, 3m+2 for the 4 columns 32t + b + 4r + 8i (i = 0..3)
    //      that MMA b pairs with lane t (register b0 for r = 0, b1 for r = 1) ----
    {
      const int total = nun * MB * 32;
      for (int base = 0; base < total; base += kIT) {
        const int ch = base + threadIdx.x;
        int vs = 0;  // 4 values of |V| <= 2^22 per lane, 32 lanes: |sum| <= 2^29
        int lsm = -1;
        if (ch < total) {
          const int ulm = pa * MB + (ch >> 5), tbr = ch & 31;
          const int ul = ulm / MB, m = ulm - ul * MB;
          const int t = tbr >> 3, b = (tbr >> 1) & 3, r = tbr & 1;
          lsm = S.useg[ul] * MB + m;
          const int s = fixed_shift(__uint_as_float(S.xmax[lsm]));
          float f1, f2;
          pow2_pair(s, f1, f2);
          const float* xc = S.xt + static_cast<size_t>(ulm) * 128 + 32 * t + b + 4 * r;
          int d[3][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int V = __float2int_rn((xc[8 * i] * f1) * f2);
            vs += V;
            const int d2 = sext8(V);
            const int r1 = (V - d2) >> 8;
            const int d1 = sext8(r1);
            d[0][i] = (r1 - d1) >> 8;
            d[1][i] = d1;
            d[2][i] = d2;
          }
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            const int n = 3 * m + k;
            const int g = n >> 3, L = (n & 7) * 4 + t;
            unsigned* dst = reinterpret_cast<unsigned*>(S.bfr + (static_cast<size_t>(ul) * NG + g) * 64 + L * 2) + 2 * b + r;
            *dst = __byte_perm(__byte_perm(d[k][0], d[k][1], 0x0040), __byte_perm(d[k][2], d[k][3], 0x0040), 0x5410);
          }
        }
        // the 32 lanes of a warp share one (unit, batch row)
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) vs += __shfl_xor_sync(0xffffffffu, vs, o);
        if (lane == 0 && lsm >= 0) atomicAdd(S.vsum + lsm, static_cast<unsigned long long>(static_cast<long long>(vs)));
      }
    }
    __syncthreads();  // B fragments and sums complete
    if (ph == 0) asm volatile("griddepcontrol.launch_dependents;");

    // per-slot weights 2^(17 - 8 digit - s) and per-segment sums of the quantised v, read
    // by the drains below
    for (int i = threadIdx.x; i < nls * (kMaxSlots + MB); i += kIT) {
      if (i < nls * kMaxSlots) {
        const int ls = i / kMaxSlots, n = i - ls * kMaxSlots;
        const int m = n / 3, dg = n - 3 * m;
        float f1 = 0.f, f2 = 0.f;
        if (m < MB) pow2_pair(17 - 8 * dg - fixed_shift(__uint_as_float(S.xmax[ls * MB + m])), f1, f2);
        S.wsl[i] = f1 * f2;  // powers of two: the product is exact
      } else {
        const int j = i - nls * kMaxSlots;
        float f1, f2;
        pow2_pair(-fixed_shift(__uint_as_float(S.xmax[j])), f1, f2);
        S.ssf[j] = (static_cast<float>(static_cast<double>(static_cast<long long>(S.vsum[j]))) * f1) * f2;
      }
    }
    __syncthreads();

    // ---- MMA loop over this warp's contiguous range of (row block, unit) items: per row
    //      block, runs of units of one segment; inside a run the operands of the next unit
    //      are loaded while the current unit's MMAs issue (two register sets, ping-pong).
    //      When a warp has finished a row block it pushes the block's row partial sums
    //      to the CTA that owns the rows (distributed shared memory) ----
    const int nb = nt * BPT;
    const int items = nb * nun;
    const int i0 = warp * items / kIW, i1 = (warp + 1) * items / kIW;
    const bool skip_phase = reads_z && S.flags[1] != 0;  // z never became ready
    if (!skip_phase) {
      int acc[RH][NG][4][4];
#pragma unroll
      for (int h = 0; h < RH; ++h)
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[h][g][b][j] = 0;
      int cur_tile = -1;
      bool tile_ok = true;
      int it = i0;
      while (it < i1) {
        const int bl = it / nun;
        const int tl = bl / BPT;
        const int ua = pa + (it - bl * nun);
        const int ub = pa + min(nun, i1 - bl * nun);  // this warp's units of block bl: [ua, ub)
        if (tl != cur_tile) {
          cur_tile = tl;
          tile_ok = dev::mbar_wait(S.bar + tl, 0u, wait_ns);
          if (!tile_ok) ok = false;
        }
        const unsigned* wbase = reinterpret_cast<const unsigned*>(S.ring + static_cast<size_t>(tl) * nu * 512) +
                                ((bl % BPT) * RB + g8) * 4 + tq;
        const uint4* bbase = S.bfr + lane * 2;
        float pacc[RH][2][MB];
#pragma unroll
        for (int h = 0; h < RH; ++h)
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int m = 0; m < MB; ++m) pacc[h][r][m] = 0.f;
        int ur = ua;
        while (ur < ub) {
          const int ls = S.useg[ur];
          const int ue = min(ub, S.lsend[ls]);
          if (S.lsbits[ls] && tile_ok) {
            auto load_b = [&](int ul, unsigned (&B)[NG][8]) {
#pragma unroll
              for (int g = 0; g < NG; ++g) {
                if (8 * g + g8 < 3 * MB) {
                  const uint4* src = bbase + (static_cast<size_t>(ul) * NG + g) * 64;
                  const uint4 q0 = src[0], q1 = src[1];
                  B[g][0] = q0.x; B[g][1] = q0.y; B[g][2] = q0.z; B[g][3] = q0.w;
                  B[g][4] = q1.x; B[g][5] = q1.y; B[g][6] = q1.z; B[g][7] = q1.w;
                } else {
#pragma unroll
                  for (int k = 0; k < 8; ++k) B[g][k] = 0u;
                }
              }
            };
            auto load_w = [&](int ul, unsigned (&wv)[2 * RH]) {
              const unsigned* ws = wbase + ul * 128;
#pragma unroll
              for (int k = 0; k < 2 * RH; ++k) wv[k] = ws[k * 32];
            };
            auto mma_unit = [&](const unsigned (&B)[NG][8], const unsigned (&wv)[2 * RH]) {
#pragma unroll
              for (int h = 0; h < RH; ++h) {
                const unsigned w0 = wv[2 * h], w1 = wv[2 * h + 1];
                const unsigned s0 = w0 >> 4, s1 = w1 >> 4;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                  const unsigned mk = kByteMask << b;
                  const unsigned a0 = w0 & mk, a1 = w1 & mk, a2 = s0 & mk, a3 = s1 & mk;
#pragma unroll
                  for (int g = 0; g < NG; ++g) mma_s8s8(acc[h][g][b], a0, a1, a2, a3, B[g][2 * b], B[g][2 * b + 1]);
                }
              }
            };
            if constexpr (NG <= 2) {
              unsigned B0[NG][8], B1[NG][8], W0[2 * RH], W1[2 * RH];
              load_b(ur, B0);
              load_w(ur, W0);
              int ul = ur;
              for (; ul + 1 < ue; ul += 2) {
                load_b(ul + 1, B1);
                load_w(ul + 1, W1);
                mma_unit(B0, W0);
                if (ul + 2 < ue) {
                  load_b(ul + 2, B0);
                  load_w(ul + 2, W0);
                }
                mma_unit(B1, W1);
              }
              if (ul < ue) mma_unit(B0, W0);
            } else {  // three slot groups: registers allow only the sign words to run ahead
              unsigned B0[NG][8], W0[2 * RH], W1[2 * RH];
              load_w(ur, W0);
              int ul = ur;
              for (; ul + 1 < ue; ul += 2) {
                load_w(ul + 1, W1);
                load_b(ul, B0);
                mma_unit(B0, W0);
                if (ul + 2 < ue) load_w(ul + 2, W0);
                load_b(ul + 1, B0);
                mma_unit(B0, W1);
              }
              if (ul < ue) {
                load_b(ul, B0);
                mma_unit(B0, W0);
              }
            }
            // drain: D = sum_b (acc_b >> b) per slot, times the slot weight, summed over the
            // slots of each batch row held by this lane, times the row scale (the same for the
            // four lanes of a quad, so the sum over the quad's slots waits until the block is
            // done); the run that starts the CTA's range of the segment also subtracts
            // r * sum_i v_i, once per quad
            float wlo[NG][2];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              const float2 wf = reinterpret_cast<const float2*>(S.wsl)[(ls * kMaxSlots + 8 * g + 2 * tq) >> 1];
              wlo[g][0] = wf.x;
              wlo[g][1] = wf.y;
            }
            const bool first_run = ur == S.lsstart[ls];
#pragma unroll
            for (int h = 0; h < RH; ++h) {
              float cv[2][MB];
#pragma unroll
              for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int m = 0; m < MB; ++m) cv[r][m] = 0.f;
#pragma unroll
              for (int g = 0; g < NG; ++g) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const int n = 8 * g + 2 * tq + (j & 1);
                  const int D = acc[h][g][0][j] + (acc[h][g][1][j] >> 1) + (acc[h][g][2][j] >> 2) + (acc[h][g][3][j] >> 3);
                  const float val = static_cast<float>(D) * wlo[g][j & 1];
                  const int m = n / 3;
#pragma unroll
                  for (int mm = 0; mm < MB; ++mm) cv[j >> 1][mm] += (m == mm) ? val : 0.f;
                }
#pragma unroll
                for (int b = 0; b < 4; ++b)
#pragma unroll
                  for (int j = 0; j < 4; ++j) acc[h][g][b][j] = 0;
              }
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                const int row = (bl % BPT) * RB + 16 * h + g8 + 8 * r;  // row within the tile
                const float rs = S.rsc[ls * p.max_tiles * 32 + tl * 32 + row];
#pragma unroll
                for (int mm = 0; mm < MB; ++mm) {
                  float v = cv[r][mm];
                  if (first_run && tq == 0) v -= S.ssf[ls * MB + mm];
                  pacc[h][r][mm] = fmaf(v, rs, pacc[h][r][mm]);
                }
              }
            }
          }
          ur = ue;
        }
        // the sums over the slots of each batch row (the four lanes of a quad)
#pragma unroll
        for (int h = 0; h < RH; ++h)
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int mm = 0; mm < MB; ++mm) {
              float v = pacc[h][r][mm];
              v += __shfl_xor_sync(0xffffffffu, v, 1);
              v += __shfl_xor_sync(0xffffffffu, v, 2);
              pacc[h][r][mm] = v;
            }
        // push the block's row partial sums to the CTA that owns the rows, one store per
        // lane: after the quad reduction every lane of a quad holds the same sums, so lane
        // tq takes one (half, row) pair (32-row blocks) or one row and half the batch rows
        // (16-row blocks). Slot c = this warp's index among the consecutive warps whose
        // item ranges touch block bl, in this phase's set of slots.
        if (!waited) {  // peers must be running and have zeroed their buffers
          cluster.barrier_wait(std::move(started));
          waited = true;
        }
        int wfirst = warp;
        while (wfirst > 0 && ((wfirst) * items / kIW) > bl * nun) --wfirst;
        const int c = ph * kcp + (warp - wfirst);
        {
          constexpr int VPL = RH == 2 ? MB : MB / 2;  // values per lane
          const int hh = RH == 2 ? (tq >> 1) : 0;
          const int rr = tq & 1;
          const int m0 = RH == 2 ? 0 : (tq >> 1) * (MB / 2);
          float v[VPL];
#pragma unroll
          for (int e = 0; e < VPL; ++e) {
            if constexpr (RH == 2) {  // (hh, rr) from tq; all MB values
              const float lo = rr ? pacc[0][1][e] : pacc[0][0][e];
              const float hi = rr ? pacc[RH - 1][1][e] : pacc[RH - 1][0][e];
              v[e] = hh ? hi : lo;
            } else {  // rr from tq, batch rows e or MB/2 + e
              const float a = rr ? pacc[0][1][e] : pacc[0][0][e];
              const float b = rr ? pacc[0][1][(MB / 2 + e) % MB] : pacc[0][0][(MB / 2 + e) % MB];
              v[e] = (tq >> 1) ? b : a;
            }
          }
          const int lr = bl * RB + 16 * hh + g8 + 8 * rr;  // row within the cluster's rows
          const int dst = share_owner_i(lr, rows_c, p.C);
          float* rp = cluster.map_shared_rank(S.recv, dst) +
                      ((static_cast<size_t>(rank) * kc + c) * msh + (lr - share_begin_i(dst, rows_c, p.C))) * MB + m0;
          if constexpr (VPL == 1) {
            rp[0] = v[0];
          } else if constexpr (VPL == 2) {
            *reinterpret_cast<float2*>(rp) = make_float2(v[0], v[1]);
          } else {
#pragma unroll
            for (int e = 0; e < VPL; e += 4) *reinterpret_cast<float4*>(rp + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          }
        }
        it = bl * nun + (ub - pa);
      }
    }
  }
  if (!ok) {
    atomicExch(p.status, static_cast<int>(BISCO_ERR_TIMEOUT));
    S.flags[0] = 1;
  }
  if (!waited) cluster.barrier_wait(std::move(started));  // warps without items
  cluster.sync();  // all partial sums have landed
  // After a timeout make sure no copy is still writing into shared memory before the
  // CTA exits: wait, bounded, for every tile's copies.
  if (S.flags[0] != 0 && threadIdx.x == 0)
    for (int tl = 0; tl < nt; ++tl)
      if (tl != dbg_skip_tile) dev::mbar_wait(S.bar + tl, 0u, wait_ns);

  // ---- reduce this CTA's share of rows in CTA-rank order, add salient columns, store ----
  const int r0 = share_begin_i(rank, rows_c, p.C), r1 = share_begin_i(rank + 1, rows_c, p.C);
  for (int lr = r0 + threadIdx.x; lr < r1; lr += kIT) {
    const int o = t0 * 32 + lr;
    if (o >= p.rows) continue;
    const int sr = lr - r0;
    float sum[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) sum[m] = 0.f;
#pragma unroll 4
    for (int src = 0; src < p.C * kc; ++src) {  // (rank, contributor slot), fixed order
#pragma unroll
      for (int m = 0; m < MB; ++m) sum[m] += S.recv[(static_cast<size_t>(src) * msh + sr) * MB + m];
    }
    if (p.n_sal > 0) {
      const int8_t* qrow = p.sal_q + static_cast<long long>(o) * p.sal_stride;
      for (int tq2 = 0; tq2 < p.n_sal; tq2 += 16) {
        const uint4 qq = __ldg(reinterpret_cast<const uint4*>(qrow + tq2));
        const unsigned qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int tt = tq2 + k;
          if (tt < p.n_sal) {
            const float qv = static_cast<float>(static_cast<int8_t>((qw[k >> 2] >> (8 * (k & 3))) & 0xFF));
#pragma unroll
            for (int m = 0; m < MB; ++m) sum[m] = fmaf(qv, S.xs[m * nsp + tt], sum[m]);
          }
        }
      }
    }
    if (p.rref) {  // salient refinement term, written by the launch before this one
#pragma unroll
      for (int m = 0; m < MB; ++m)
        if (m < p.Mc) sum[m] += __ldcg(p.rref + static_cast<long long>(m) * p.rows + o);
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
  if (fused) {
    __syncthreads();  // this CTA's stores (z for the producers) are issued
    if (threadIdx.x == 0) {
      if (role_z) {
        __threadfence();  // z visible device-wide before it is counted
        atomicAdd(z_ready, 1);
      }
      // the last CTA of the grid to get here returns the counters to zero for the next
      // launch: every consumer counted itself after its wait, so nobody reads them any more
      if (atomicAdd(z_done, 1) == static_cast<int>(gridDim.x) - 1) {
        for (int r = 0; r < L.rt.nroles; ++r) atomicExch(p.status + 32 + r, 0);
        atomicExch(z_done, 0);
      }
    }
  }
}

template <int MB>
int imma_clusters(int C, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C);
  cfg.blockDim = dim3(kIT);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  // both variants are compiled for two CTAs of kIT threads per SM: same residency
  if (cudaOccupancyMaxActiveClusters(&n, imma_gemv_kernel<MB, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int imma_clusters_mb(int MB, int C, size_t smem) {
  switch (MB) {
    case 1: return imma_clusters<1>(C, smem);
    case 2: return imma_clusters<2>(C, smem);
    case 4: return imma_clusters<4>(C, smem);
    case 8: return imma_clusters<8>(C, smem);
    default: return 0;
  }
}

// Contributor slots a phase needs: nb row blocks x nun units split into kIW equal
// contiguous item ranges; a warp writes slot (warp - first warp whose range starts at or
// before the block's first item), exactly as the kernel numbers them.
int phase_slots(int nb, int nun) {
  if (nb <= 0 || nun <= 0) return 1;
  const long long items = static_cast<long long>(nb) * nun;
  int need = 1;
  for (int w = 0; w < kIW; ++w) {
    const long long a = w * items / kIW, b = (w + 1) * items / kIW;
    if (b <= a) continue;
    for (long long bl = a / nun; bl <= (b - 1) / nun; ++bl) {
      int wf = w;
      while (wf > 0 && wf * items / kIW > bl * nun) --wf;
      need = std::max(need, w - wf + 1);
    }
  }
  return need;
}

// Slots over every CTA shape of a pass: tile counts floor/ceil(tiles / ncl), the unit
// range of each cluster rank, and (u_split >= 0) the two phases of the output pass of a
// fused launch, split at unit u_split.
int pass_slots(int tiles, int ncl, int units, int C, int BPT, int u_split) {
  int need = 1;
  for (int nt : {tiles / ncl, (tiles + ncl - 1) / ncl}) {
    if (nt <= 0) continue;
    const int nb = nt * BPT;
    for (int r = 0; r < C; ++r) {
      const int u0 = r * units / C, u1 = (r + 1) * units / C, nu = u1 - u0;
      if (u_split < 0) {
        need = std::max(need, phase_slots(nb, nu));
      } else {
        const int n0 = std::max(0, std::min(nu, u_split - u0)), n1 = nu - n0;
        if (n0 > 0 && n1 > 0) {
          need = std::max(need, phase_slots(nb, n0));
          need = std::max(need, phase_slots(nb, n1));
        } else {
          need = std::max(need, phase_slots(nb, nu));
        }
      }
    }
  }
  return need;
}

// Largest number of (segment, row-scale group) parts one CTA's unit range touches.
int max_parts_per_cta(const ImmaShape& sh, int C) {
  auto part_of = [&](int u) {
    int part = 0, s = 0;
    for (int k = 0; k < sh.nseg; ++k) {
      if (u >= sh.seg_unit0[k]) s = k;
    }
    for (int k = 0; k < s; ++k) {
      const int nq = (k + 1 < sh.nseg ? sh.seg_unit0[k + 1] : sh.units) - sh.seg_unit0[k];
      const int g = sh.seg_rgu ? sh.seg_rgu[k] : 0;
      part += g > 0 ? (nq + g - 1) / g : 1;
    }
    const int g = sh.seg_rgu ? sh.seg_rgu[s] : 0;
    return part + (g > 0 ? (u - sh.seg_unit0[s]) / g : 0);
  };
  int m = 1;
  for (int r = 0; r < C; ++r) {
    const int a = r * sh.units / C, b = (r + 1) * sh.units / C;
    if (b > a) m = std::max(m, part_of(b - 1) - part_of(a) + 1);
  }
  return m;
}

template <int MB>
cudaError_t imma_set_attrs(size_t lim) {
  cudaError_t e = cudaFuncSetAttribute(imma_gemv_kernel<MB, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(lim));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(imma_gemv_kernel<MB, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(lim));
  return e;
}

}  // namespace

cudaError_t imma_ensure_attrs() {
  static std::once_flag once[64];
  static cudaError_t err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::call_once(once[dev & 63], [&] {
    const size_t lim = query_smem_limit();
    cudaError_t r = imma_set_attrs<1>(lim);
    if (r == cudaSuccess) r = imma_set_attrs<2>(lim);
    if (r == cudaSuccess) r = imma_set_attrs<4>(lim);
    if (r == cudaSuccess) r = imma_set_attrs<8>(lim);
    err[dev & 63] = r;
  });
  return err[dev & 63];
}

// Plan: the cluster size C in {1, 2, 4, 8} that minimises a cycle estimate per SM --
// tensor-core time of the largest CTA share (8 MMAs per 32 x 128 block and group of 8
// slots; a legacy m16n8k32 MMA holds its sub-partition's issue for about 10 cycles and
// the masks add about half as much again: measured 237 cycles per 32 x 128 block and
// warp with 8 warps per SM), the B-fragment writes (about 60 lane operations per task of
// 4 columns and one batch row, 64 lanes per clock for one CTA), a fixed cost for the
// cluster reduction (and for the z hand-over of a launch with several roles), plus a fixed
// cost when the CTA takes more than half of the SM's shared memory (the next kernel's CTA
// then cannot be resident beside it) -- among the plans whose shared memory fits. The
// grid holds as many clusters as fit with one CTA per SM; with half an SM or less per CTA
// the block scheduler still places two CTAs of one launch on some SMs (measured: 120 CTAs
// on 98 SMs), which those SMs pay for, but exposing the next kernel's prologue costs more.
// C = 0 in the result means no plan fits.
ImmaPlan make_imma_plan(const ImmaRole* roles, int nroles, int MB, size_t smem_limit) {
  ImmaPlan best{};
  if (nroles < 1 || nroles > kMaxRoles || imma_ensure_attrs() != cudaSuccess) return best;
  int dev = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  // two CTAs per SM: each gets half of the SM's shared memory less the 1 KB the
  // hardware reserves per CTA
  const size_t half = per_sm > 0 ? static_cast<size_t>(per_sm) / 2 - 1024 : smem_limit / 2;
  const int NG = groups_of(MB), RB = block_rows(MB);
  int tiles[kMaxRoles], min_units = 1 << 30, n_sal = 0;
  bool waits = false;
  for (int r = 0; r < nroles; ++r) {
    tiles[r] = (roles[r].sh.rows + 31) / 32;
    min_units = std::min(min_units, roles[r].sh.units);
    n_sal = std::max(n_sal, roles[r].n_sal);
    waits = waits || roles[r].u_split >= 0;
  }
  double best_cost = -1;
  for (int C = 1; C <= kMaxCluster; C *= 2) {
    if (C > 1 && C > min_units) break;
    // clusters that fit with one CTA of the launch per SM (the query asks for more
    // than half of the SM's shared memory)
    const size_t force = smem_limit / 2 + 1024;
    const int fit = imma_clusters_mb(MB, C, force);
    if (fit < nroles) continue;
    int mu[kMaxRoles];
    for (int r = 0; r < nroles; ++r) mu[r] = (roles[r].sh.units + C - 1) / C;
    auto load = [&](int r, int n) {  // blocks of the largest CTA share of role r with n clusters
      return static_cast<double>((tiles[r] + n - 1) / n) * mu[r];
    };
    // The roles share the shared-memory maxima (tiles x units of the largest share), so
    // the split is searched over a cap T on the row tiles of any cluster: every role first
    // gets the clusters the cap needs, the rest go one at a time to the role with the
    // heaviest share.
    int t_hi = 1;
    for (int r = 0; r < nroles; ++r) t_hi = std::max(t_hi, tiles[r]);
    for (int T = 1; T <= t_hi; ++T) {
      int ncl[kMaxRoles], used = 0;
      for (int r = 0; r < nroles; ++r) {
        ncl[r] = std::max(1, (tiles[r] + T - 1) / T);
        used += ncl[r];
      }
      if (used > fit) continue;
      for (int left = fit - used; left > 0; --left) {
        int pick = -1;
        for (int r = 0; r < nroles; ++r)
          if (ncl[r] < tiles[r] && (pick < 0 || load(r, ncl[r]) > load(pick, ncl[pick]))) pick = r;
        if (pick < 0) break;
        ++ncl[pick];
      }
      int max_tiles = 0, max_units = 0, max_lseg = 1, kcp = 1;
      double mma = 0;
      for (int r = 0; r < nroles; ++r) {
        max_tiles = std::max(max_tiles, (tiles[r] + ncl[r] - 1) / ncl[r]);
        max_units = std::max(max_units, mu[r]);
        max_lseg = std::max(max_lseg, max_parts_per_cta(roles[r].sh, C));
        // contributor slots per row and phase
        kcp = std::max(kcp, pass_slots(tiles[r], ncl[r], roles[r].sh.units, C, 32 / RB, roles[r].u_split));
        mma = std::max(mma, load(r, ncl[r]));
      }
      const int kc = kcp * (nroles > 1 ? 2 : 1);  // a launch with several roles has two phases
      const size_t need = ismem_bytes(MB, C, max_tiles, max_units, max_lseg, kc, n_sal);
      if (need > smem_limit) continue;
      // kIW warps of a CTA work on kIW blocks at once: 237 / kIW cycles per block and SM
      const double cyc = mma * NG * 237.0 / kIW;
      const double bfr = static_cast<double>(max_units) * MB * 32.0 * 60.0 / 64.0;
      const double red = (C > 1 ? 1500.0 : 300.0) + (waits ? 1500.0 : 0.0);
      // a CTA of at most half an SM lets the next kernel's CTA (launched early) be
      // resident beside it and run its prologue during this kernel; a larger one exposes
      // that prologue (measured on the 4096 x 4096 layer: 6.85 us vs 8.08 us per GEMV)
      const bool coresident = need <= half;
      const double cost = cyc + bfr + red + (coresident ? 0.0 : 2500.0);
      if (best_cost < 0 || cost < best_cost) {
        best_cost = cost;
        best.C = C;
        best.nroles = nroles;
        for (int r = 0; r < nroles; ++r) best.ncl[r] = ncl[r];
        best.max_tiles = max_tiles;
        best.max_units = max_units;
        best.max_lseg = max_lseg;
        best.nbw = kc;
        best.MB = MB;
        best.smem = coresident ? need : std::max(need, force);
      }
    }
  }
  return best;
}

cudaError_t launch_imma(const ImmaLaunch& L, const ImmaPlan& plan, cudaStream_t stream, bool pdl,
                        const ImmaDebug* dbg) {
  const cudaError_t e = imma_ensure_attrs();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.rt.cl0[L.rt.nroles] * plan.C);
  cfg.blockDim = dim3(kIT);
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
  const int skip = dbg ? dbg->skip_tile : -1;
  const unsigned long long wait_ns = dbg && dbg->wait_ns ? dbg->wait_ns : kDefaultWaitNs;
  const bool multi = L.rt.nroles > 1;
  switch (plan.MB) {
    case 1:
      return multi ? cudaLaunchKernelEx(&cfg, imma_gemv_kernel<1, true>, L, plan.nbw, skip, wait_ns)
                   : cudaLaunchKernelEx(&cfg, imma_gemv_kernel<1, false>, L, plan.nbw, skip, wait_ns);
    case 2:
      return multi ? cudaLaunchKernelEx(&cfg, imma_gemv_kernel<2, true>, L, plan.nbw, skip, wait_ns)
                   : cudaLaunchKernelEx(&cfg, imma_gemv_kernel<2, false>, L, plan.nbw, skip, wait_ns);
    case 4:
      return multi ? cudaLaunchKernelEx(&cfg, imma_gemv_kernel<4, true>, L, plan.nbw, skip, wait_ns)
                   : cudaLaunchKernelEx(&cfg, imma_gemv_kernel<4, false>, L, plan.nbw, skip, wait_ns);
    case 8:
      return multi ? cudaLaunchKernelEx(&cfg, imma_gemv_kernel<8, true>, L, plan.nbw, skip, wait_ns)
                   : cudaLaunchKernelEx(&cfg, imma_gemv_kernel<8, false>, L, plan.nbw, skip, wait_ns);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace bisco

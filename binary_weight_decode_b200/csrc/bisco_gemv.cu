// Binary-weight decode GEMV on CUDA cores, sm_100a.
//
// Computes, per output row o and batch row m,
//   y[m][o] = sum_seg rs_seg[o] * sum_i sign_seg[o][i] * xin_seg[m][i]  (+ salient term)
// where each "segment" is one packed sign matrix: a binary base B_k with
// xin = c_k (.) x and rs = r_k ("FluxBin", Sec. 3.1, decoupled row-column binary
// bases, column scale folded into the activation as in Sec. 3.2 Stage 1, "LUT
// Building with Scale Fusion"), the correction's V with xin = x and rs = alpha
// (z = alpha (.) (V x)), or the correction's U^T with xin = z ("BiLoCo", "The
// core idea": alpha * u * (v . x)).
//
// Sign-times-activation sums use 5-bit lookup tables in shared memory: for every
// 5 consecutive columns the CTA stores the 32 signed sums of their scaled
// activations, so one table read replaces five signed adds (the LUT idea of
// FluxBin Sec. 3.2, Stage 1/2, re-shaped for B200). A 128-column quad splits into
// 25 five-bit fields and one three-bit field. All lanes of a warp read the same
// 32-entry table in one instruction, one entry per bank, so reads never conflict.
//
// Work: item = (block of G row tiles, quad, tile). Items are split evenly over
// the CTAs. Each lane owns one row of a 32-row tile and reads its 16 bytes of the
// (tile, quad) block; the 32 lanes read 512 contiguous bytes. Partial sums of a
// block from different CTAs (split-K) meet in the workspace; the last CTA to
// finish a block adds them in CTA order (deterministic) and writes Y.
//
// Launch protocol (programmatic dependent launch): sign words and row scales are
// loaded before griddepcontrol.wait, activations and the workspace only after it.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "bisco_internal.h"

namespace bisco {

namespace {

constexpr int kDepth = 8;  // work items per warp kept in flight (16 bytes per lane each)

__device__ __forceinline__ float ld_val(const void* p, long long i, int dt) {
  if (dt == BISCO_BF16) {
    const unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
    return __uint_as_float(static_cast<unsigned int>(h) << 16);
  }
  return __ldg(reinterpret_cast<const float*>(p) + i);
}

// Byte offset 4*p of the table entry selected by field F of a 128-bit quad.
// Fields 0..24 are 5 bits at bit 5F; field 25 is 3 bits at bits 125..127.
__device__ __forceinline__ unsigned field_off(const uint4& w, const int F) {
  const unsigned ws[4] = {w.x, w.y, w.z, w.w};
  if (F == 25) return (w.w >> 27) & 0x1Cu;
  const int s = 5 * F, wi = s >> 5, b = s & 31;
  if (b + 5 <= 32) {
    return (b >= 2 ? (ws[wi] >> (b - 2)) : (ws[wi] << (2 - b))) & 0x7Cu;
  }
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

// CTA that owns work item `it` under the even split [c*L/P, (c+1)*L/P).
__device__ __forceinline__ int cta_of(long long it, long long L, int P) {
  return static_cast<int>(((it + 1) * P - 1) / L);
}

// Index of the lowest set bit of e (1 <= e < 32); folds to a constant when e is.
__host__ __device__ constexpr int low_bit(int e) {
  return (e & 1) ? 0 : (e & 2) ? 1 : (e & 4) ? 2 : (e & 8) ? 3 : 4;
}

template <int MB>
__global__ void __launch_bounds__(kThreads) lut_gemv_kernel(const __grid_constant__ PassParam p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pbeg = static_cast<long long>(c) * p.L / p.P;
  const long long pend = static_cast<long long>(c + 1) * p.L / p.P;
  const int G = p.G;
  const long long col0 = pbeg / G, col1 = (pend - 1) / G;
  const int ncol = static_cast<int>(col1 - col0 + 1);
  const int blk0 = static_cast<int>(col0 / p.units);
  const int blk1 = static_cast<int>(col1 / p.units);
  const int nsp = (p.n_sal + 3) & ~3;

  float* tables = reinterpret_cast<float*>(smem);
  float* xt = reinterpret_cast<float*>(smem + static_cast<size_t>(p.max_cols) * p.col_stride_bytes);
  float* xs = xt + static_cast<size_t>(p.max_cols) * MB * 128;
  float* part = xs + MB * nsp;
  __shared__ int last_flag[2];

  // ---- prefetch this warp's first kDepth items (weights only) ----
  uint4 buf[kDepth];
  float rsb[kDepth];
  auto load_item = [&](long long it, uint4& w, float& rs) {
    const long long col = it / G;
    const int g = static_cast<int>(it - col * G);
    const int b = static_cast<int>(col / p.units);
    const int u = static_cast<int>(col - static_cast<long long>(b) * p.units);
    const int t = b * G + g;
    w = make_uint4(0u, 0u, 0u, 0u);
    rs = 0.f;
    if (t >= p.tiles) return;
    const int sg = find_seg(p, u);
    const SegParam& S = p.seg[sg];
    const int q = u - S.unit0;
    if (S.bits != nullptr)
      w = __ldcs(S.bits + (static_cast<long long>(t) * S.nq + q) * 32 + lane);
    const int o = t * 32 + lane;
    if (o < p.rows) rs = S.rscale ? ld_val(S.rscale, o, S.rdt) : 1.f;
  };
#pragma unroll
  for (int d = 0; d < kDepth; ++d) {
    const long long it = pbeg + warp + static_cast<long long>(kWarps) * d;
    if (it < pend) load_item(it, buf[d], rsb[d]);
  }

  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");

  // ---- stage scaled activations x~ for this CTA's quads ----
  for (int idx = threadIdx.x; idx < ncol * MB * 128; idx += kThreads) {
    const int s = idx / (MB * 128);
    const int rem = idx - s * (MB * 128);
    const int m = rem >> 7, j = rem & 127;
    const long long col = col0 + s;
    const int u = static_cast<int>(col % p.units);
    const SegParam& S = p.seg[find_seg(p, u)];
    const int ci = (u - S.unit0) * 128 + j;
    float v = 0.f;
    if (m < p.Mc && ci < S.ncols) {
      if (S.xsrc == 0) v = ld_val(p.X, m * p.ldx + ci, p.xdt);
      else if (S.xsrc == 1) v = __ldcg(p.Z + m * p.ldz + ci);
      if (S.cscale) v *= ld_val(S.cscale, ci, S.cdt);
    }
    xt[(s * MB + m) * 128 + j] = v;
  }
  for (int idx = threadIdx.x; idx < MB * p.n_sal; idx += kThreads) {
    const int m = idx / p.n_sal, t = idx - m * p.n_sal;
    float v = 0.f;
    const int ci = __ldg(p.sal_idx + t);
    if (ci < 0 || ci >= p.xcols) {
      atomicExch(p.status, static_cast<int>(BISCO_ERR_INVALID_ARG));  // index out of range: term skipped
    } else if (m < p.Mc) {
      v = ld_val(p.X, m * p.ldx + ci, p.xdt) * __ldg(p.sal_scale + t);
    }
    xs[m * nsp + t] = v;
  }
  for (int idx = threadIdx.x; idx < 2 * MB * G * 32; idx += kThreads) part[idx] = 0.f;
  __syncthreads();

  // ---- build the 32-entry tables: lane f computes all entries of field f ----
  for (int task = warp; task < ncol * MB; task += kWarps) {
    const int s = task / MB, m = task - s * MB;
    if (lane < kFields) {
      const float* x = xt + (s * MB + m) * 128 + 5 * lane;
      const float x0 = x[0], x1 = x[1], x2 = x[2];
      const float x3 = lane < 25 ? x[3] : 0.f, x4 = lane < 25 ? x[4] : 0.f;
      const float d[5] = {2.f * x0, 2.f * x1, 2.f * x2, 2.f * x3, 2.f * x4};
      float T[32];
      T[0] = -((x0 + x1) + (x2 + x3) + x4);
#pragma unroll
      for (int e = 1; e < 32; ++e) T[e] = T[e & (e - 1)] + d[low_bit(e)];
      float* dst = tables + static_cast<size_t>(s) * (p.col_stride_bytes / 4) + (m * kFields + lane) * kFieldStride;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        reinterpret_cast<float4*>(dst)[j] = make_float4(T[4 * j], T[4 * j + 1], T[4 * j + 2], T[4 * j + 3]);
    }
  }
  __syncthreads();

  // ---- main loop: one table read per field per batch row ----
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(tables);
  for (long long base = 0;; base += kDepth) {
    const long long first = pbeg + warp + static_cast<long long>(kWarps) * base;
    if (first >= pend) break;
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      const long long it = first + static_cast<long long>(kWarps) * d;
      if (it < pend) {
        const long long col = it / G;
        const int g = static_cast<int>(it - col * G);
        const int b = static_cast<int>(col / p.units);
        const int u = static_cast<int>(col - static_cast<long long>(b) * p.units);
        const int t = b * G + g;
        if (t < p.tiles) {
          const uint4 w = buf[d];
          const unsigned uoff = static_cast<unsigned>(col - col0) * static_cast<unsigned>(p.col_stride_bytes);
          float acc[MB > 1 ? MB : 2];
#pragma unroll
          for (int m = 0; m < (MB > 1 ? MB : 2); ++m) acc[m] = 0.f;
          if (MB == 1) {
            // fields in pairs: one packed fp32x2 add per two table reads
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
          float val[MB];
          if (MB == 1) val[0] = (acc[0] + acc[1]) * rsb[d];
          else {
#pragma unroll
            for (int m = 0; m < MB; ++m) val[m] = acc[m] * rsb[d];
          }
          const int o = t * 32 + lane;
          if (u == 0 && p.n_sal > 0 && o < p.rows) {
            // salient columns: y += sum_t q[o][t] * (x[idx_t] * s_t), added once per row
            const int8_t* qrow = p.sal_q + static_cast<long long>(o) * p.sal_stride;
            for (int t0 = 0; t0 < p.n_sal; t0 += 16) {
              const uint4 qq = __ldg(reinterpret_cast<const uint4*>(qrow + t0));
              const unsigned qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                const int tt = t0 + k;
                if (tt < p.n_sal) {
                  const float qv = static_cast<float>(static_cast<int8_t>((qw[k >> 2] >> (8 * (k & 3))) & 0xFF));
#pragma unroll
                  for (int m = 0; m < MB; ++m) val[m] = fmaf(qv, xs[m * nsp + tt], val[m]);
                }
              }
            }
          }
          const int slot = b - blk0;
          if (slot < 0 || slot > 1) {  // cannot happen under make_plan; record instead of writing out of range
            atomicExch(p.status, static_cast<int>(BISCO_ERR_INVALID_ARG));
          } else {
#pragma unroll
            for (int m = 0; m < MB; ++m) part[(slot * MB + m) * G * 32 + g * 32 + lane] += val[m];
          }
        }
        const long long nxt = it + static_cast<long long>(kWarps) * kDepth;
        if (nxt < pend) load_item(nxt, buf[d], rsb[d]);
      }
    }
  }
  __syncthreads();

  // ---- publish partial sums, then the last CTA of each block reduces it ----
  const int nslots = blk1 - blk0 + 1;
  float* gpart = p.part + static_cast<long long>(c) * 2 * MB * G * 32;
  for (int idx = threadIdx.x; idx < nslots * MB * G * 32; idx += kThreads) gpart[idx] = part[idx];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int sl = 0; sl < 2; ++sl) {
      last_flag[sl] = 0;
      if (sl < nslots) {
        const int b = blk0 + sl;
        const long long f0 = static_cast<long long>(b) * p.units * G;
        const long long f1 = f0 + static_cast<long long>(p.units) * G - 1;
        const int need = cta_of(f1, p.L, p.P) - cta_of(f0, p.L, p.P) + 1;
        const int old = atomicAdd(p.cnt + b, 1);
        last_flag[sl] = (old == need - 1);
      }
    }
  }
  __syncthreads();
  for (int sl = 0; sl < nslots; ++sl) {
    if (!last_flag[sl]) continue;
    __threadfence();
    const int b = blk0 + sl;
    const long long f0 = static_cast<long long>(b) * p.units * G;
    const long long f1 = f0 + static_cast<long long>(p.units) * G - 1;
    const int cf = cta_of(f0, p.L, p.P), cl = cta_of(f1, p.L, p.P);
    for (int idx = threadIdx.x; idx < p.Mc * G * 32; idx += kThreads) {
      const int m = idx / (G * 32), r = idx - m * (G * 32);
      const int o = (b * G) * 32 + r;
      if (o >= p.rows) continue;
      float sum = 0.f;
      for (int cc = cf; cc <= cl; ++cc) {
        const long long cb = static_cast<long long>(cc) * p.L / p.P;
        const int cblk0 = static_cast<int>((cb / G) / p.units);
        sum += __ldcg(p.part + static_cast<long long>(cc) * 2 * MB * G * 32 + ((b - cblk0) * MB + m) * G * 32 + r);
      }
      if (p.ydt == BISCO_BF16)
        reinterpret_cast<__nv_bfloat16*>(p.Y)[m * p.ldy + o] = __float2bfloat16_rn(sum);
      else
        reinterpret_cast<float*>(p.Y)[m * p.ldy + o] = sum;
    }
    if (threadIdx.x == 0) p.cnt[b] = 0;
  }
}

template <int MB>
cudaError_t set_attrs() {
  return cudaFuncSetAttribute(lut_gemv_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(query_smem_limit()));
}

template <int MB>
cudaError_t launch_mb(const PassParam& p, const Plan& plan, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.P);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, lut_gemv_kernel<MB>, p);
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
  return n > 0 ? static_cast<size_t>(n) - 1024 : 48 * 1024;
}

static size_t plan_smem(const Plan& pl, int n_sal) {
  const int nsp = (n_sal + 3) & ~3;
  return static_cast<size_t>(pl.max_cols) * pl.col_stride_bytes +
         static_cast<size_t>(pl.max_cols) * pl.MB * 128 * 4 + static_cast<size_t>(pl.MB) * nsp * 4 +
         static_cast<size_t>(2) * pl.MB * pl.G * 32 * 4;
}

static int max_cols_of(long long L, int P, int G) {
  int mx = 0;
  for (int c = 0; c < P; ++c) {
    const long long b = static_cast<long long>(c) * L / P, e = static_cast<long long>(c + 1) * L / P;
    if (e > b) mx = std::max(mx, static_cast<int>((e - 1) / G - b / G + 1));
  }
  return mx;
}

Plan make_plan(int rows, int units, int MB, int n_sal, int num_sms, size_t smem_limit) {
  Plan pl{};
  pl.MB = MB;
  const int tiles = (rows + 31) / 32;
  int G = MB <= 2 ? 8 : (MB == 4 ? 16 : 32);
  const int tiles4 = (tiles + kWarps - 1) / kWarps * kWarps;
  G = std::max(kWarps, std::min(G, tiles4));
  pl.G = G;
  pl.nblocks = (tiles + G - 1) / G;
  pl.L = static_cast<long long>(pl.nblocks) * units * G;
  pl.col_stride_bytes = (MB * kFields * kFieldStride * 4 + 127) / 128 * 128;
  long long P = (pl.L + 7) / 8;
  P = std::min<long long>(P, num_sms);
  P = std::max<long long>(P, pl.nblocks);
  P = std::min<long long>(P, pl.L);
  pl.P = static_cast<int>(std::max<long long>(P, 1));
  for (;;) {
    pl.max_cols = max_cols_of(pl.L, pl.P, G);
    pl.smem = plan_smem(pl, n_sal);
    if (pl.smem <= smem_limit || pl.P >= pl.L) break;
    pl.P = static_cast<int>(std::min<long long>(pl.L, static_cast<long long>(pl.P) * 2));
  }
  pl.part_floats = static_cast<size_t>(pl.P) * 2 * MB * G * 32;
  pl.cnt_ints = static_cast<size_t>(pl.nblocks);
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

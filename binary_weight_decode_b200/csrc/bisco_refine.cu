// Binary salient refinement ("FluxBin: ...", Sec. 4 with the Kb-sS-gG configurations,
// and Sec. 3.2 "Virtual Columnar Mapping (VCM) for Salient Phase"): Ks extra sign bases
// over the s salient columns of every column group, stored as one dense packed sign matrix
// over the gathered columns idx[0..n_ref). Row o of the term, for batch row m, is
//
//   rref[m][o] = sum_k sum_j rs_k[j][o] * sum_{t in group j} c_k[t] * (2 b_k(o, t) - 1) * x[m][idx[t]]
//
// where group j holds the gathered columns whose input column lies in [j*g, (j+1)*g)
// (idx is ascending, so these are one contiguous run of t) and rs_k[j][o] is the
// refinement's row scale of that group. The activations are gathered through idx once
// per CTA (the translation layer of the mapping), the packed signs of the CTA's 32-row
// tile, their row scales and the column scales are staged in shared memory, and each warp
// takes every 16th group of the tile's rows with one lane per row.
//
// The result goes to an fp32 workspace buffer; the integer GEMV launch that follows on the
// stream adds it to the rest of the row before the output is rounded. Weight-side data
// (signs, row and column scales, the group boundaries) is read before griddepcontrol.wait,
// the activations only after it; each staging round issues all of its loads before it
// stores any, so the kernel pays a handful of memory latencies, not one per element.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "bisco_internal.h"

namespace bisco {
namespace {

// Warps per CTA (one 32-row tile): 16 for batch blocks of up to 4 rows, 32 for 8 rows, where
// each warp's chain of groups is the longest (measured on 2b-s16-g128 at 4096 x 4096: 32
// warps are slower at one row, faster at eight).
__host__ __device__ constexpr int ref_warps(int MB) { return MB >= 8 ? 32 : 16; }

__device__ __forceinline__ float load_scale(const void* a, long long i, int dt) {
  if (dt == BISCO_BF16)
    return __uint_as_float(static_cast<unsigned>(__ldg(reinterpret_cast<const unsigned short*>(a) + i)) << 16);
  return __ldg(reinterpret_cast<const float*>(a) + i);
}

__device__ __forceinline__ float load_act(const void* a, long long i, int dt) {
  if (dt == BISCO_BF16)
    return __uint_as_float(static_cast<unsigned>(reinterpret_cast<const unsigned short*>(a)[i]) << 16);
  return reinterpret_cast<const float*>(a)[i];
}

// Shared memory of one CTA, in this order (4-byte words; sbits first, so that its 16-byte
// stores are aligned whatever the other sizes):
//   sbits [Ks][Qr][32][4]   the tile's packed refinement signs
//   srs   [Ks][ngroups][32] the tile's refinement row scales
//   cs    [Ks][n_ref]       column scales c_k[t]
//   xg    [MB][n_ref]       gathered activations x[m][idx[t]]
//   sidx  [n_ref]           the gathered column indices
//   gs    [ngroups + 1]     first gathered column of each group
//   red   [warps][32][MB]   per-warp partial sums of the tile's rows
__host__ __device__ inline size_t refine_smem(int Ks, int n_ref, int ngroups, int MB) {
  const size_t qr = (static_cast<size_t>(n_ref) + 127) / 128;
  return 4 * (static_cast<size_t>(Ks) * qr * 128 + static_cast<size_t>(Ks) * ngroups * 32 +
              static_cast<size_t>(Ks) * n_ref + static_cast<size_t>(MB) * n_ref + n_ref + ngroups + 1 +
              static_cast<size_t>(ref_warps(MB)) * 32 * MB);
}

// Loads in flight per thread in one staging round: every load of a round is issued before
// the first of its values is stored, so a round costs one memory latency.
constexpr int kBatch = 4;

// KS: refinement bases (1..4), a template parameter so that the per-base partial sums of a
// group stay in registers and each gathered activation is read once for all bases.
template <int MB, int KS>
__global__ void __launch_bounds__(ref_warps(MB) * 32, MB >= 8 ? 1 : 2) refine_kernel(const __grid_constant__ RefineParam p) {
  constexpr int kRefWarps = ref_warps(MB), kRefThreads = kRefWarps * 32;
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int Ks = KS;
  const int n = p.n_ref, ng = p.ngroups;
  const int qr = (n + 127) / 128;
  uint32_t* sbits = reinterpret_cast<uint32_t*>(smem);
  float* srs = reinterpret_cast<float*>(sbits + static_cast<size_t>(Ks) * qr * 128);
  float* cs = srs + static_cast<size_t>(Ks) * ng * 32;
  float* xg = cs + static_cast<size_t>(Ks) * n;
  int* sidx = reinterpret_cast<int*>(xg + static_cast<size_t>(MB) * n);
  int* gs = sidx + n;
  float* red = reinterpret_cast<float*>(gs + ng + 1);

  asm volatile("griddepcontrol.launch_dependents;");
  const int tile = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // group j starts at the first gathered column whose input column is >= j * g: every
  // column t whose group differs from that of column t-1 starts the groups in between (one
  // pass over idx instead of a dependent search per group). Entries stay n for groups after
  // the last column, and every entry is a valid position whatever idx holds.
  for (int j = tid; j <= ng; j += kRefThreads) gs[j] = n;
  __syncthreads();

  // Weight-side staging, all before the dependency wait: signs of the tile (base k's words
  // are one contiguous run of qr * 128 words), row scales of the tile's rows (item
  // (k * ng + j) * 32 + r, so a warp reads 32 consecutive rows), column scales, indices.
  const size_t words = static_cast<size_t>(p.tiles) * qr * 128;
  const int n_bw = Ks * qr * 32, n_rs = Ks * ng * 32, n_cs = Ks * n;
  const int n_items = max(max(n_bw, n_rs), max(n_cs, n));
  for (int base = 0; base < n_items; base += kBatch * kRefThreads) {
    uint4 bv[kBatch];
    float rv[kBatch], cv[kBatch];
    int iv[kBatch], ipv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * kRefThreads + tid;
      if (i < n_bw) {
        const int k = i / (qr * 32), w = i - k * qr * 32;
        bv[u] = __ldg(reinterpret_cast<const uint4*>(p.bits + k * words + static_cast<size_t>(tile) * qr * 128) + w);
      }
      rv[u] = 0.f;
      if (i < n_rs) {
        const int kj = i >> 5, o = tile * 32 + (i & 31);
        if (o < p.out) rv[u] = load_scale(p.rrs, static_cast<long long>(kj) * p.out + o, p.sdt);
      }
      if (i < n_cs) cv[u] = load_scale(p.rcs, i, p.sdt);
      if (i < n) {
        iv[u] = __ldg(p.idx + i);
        ipv[u] = i > 0 ? __ldg(p.idx + i - 1) : 0;
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * kRefThreads + tid;
      if (i < n_bw) reinterpret_cast<uint4*>(sbits)[i] = bv[u];
      if (i < n_rs) srs[i] = rv[u];
      if (i < n_cs) cs[i] = cv[u];
      if (i < n) {
        sidx[i] = iv[u];
        const int jt = min(max(iv[u], 0) / p.g, ng - 1);
        const int jp = i == 0 ? -1 : min(max(ipv[u], 0) / p.g, ng - 1);
        for (int j = jp + 1; j <= jt; ++j) gs[j] = i;
      }
    }
  }
  __syncthreads();

  // activations, gathered through the index list once per CTA
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int base = 0; base < MB * n; base += kBatch * kRefThreads) {
    float xv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * kRefThreads + tid;
      xv[u] = 0.f;
      if (i < MB * n) {
        const int m = i / n, t = i - m * n;
        const int c = sidx[t];
        if (m < p.Mc) {
          if (c < 0 || c >= p.in) atomicExch(p.status, static_cast<int>(BISCO_ERR_INVALID_ARG));
          else xv[u] = load_act(p.X, static_cast<long long>(m) * p.ldx + c, p.xdt);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * kRefThreads + tid;
      if (i < MB * n) xg[i] = xv[u];
    }
  }
  __syncthreads();

  float acc[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) acc[m] = 0.f;
  for (int j = warp; j < ng; j += kRefWarps) {
    const int t0 = gs[j], t1 = gs[j + 1];  // t0 > t1 only for indices out of order: no columns
    float part[KS][MB];
#pragma unroll
    for (int k = 0; k < KS; ++k)
#pragma unroll
      for (int m = 0; m < MB; ++m) part[k][m] = 0.f;
    for (int ta = t0; ta < t1;) {  // one 32-column sign word (per base) at a time
      const int tb = min(t1, (ta | 31) + 1);
      uint32_t word[KS];
#pragma unroll
      for (int k = 0; k < KS; ++k)
        word[k] = sbits[static_cast<size_t>(k) * qr * 128 + ((ta >> 7) * 32 + lane) * 4 + ((ta >> 5) & 3)];
#pragma unroll 2
      for (int t = ta; t < tb; ++t) {
        float xv[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) xv[m] = xg[m * n + t];
#pragma unroll
        for (int k = 0; k < KS; ++k) {
          const float c = cs[k * n + t];
          const float sc = ((word[k] >> (t & 31)) & 1u) ? c : -c;
#pragma unroll
          for (int m = 0; m < MB; ++m) part[k][m] = fmaf(sc, xv[m], part[k][m]);
        }
      }
      ta = tb;
    }
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const float r = srs[(k * ng + j) * 32 + lane];
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[m] = fmaf(r, part[k][m], acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < MB; ++m) red[(warp * 32 + lane) * MB + m] = acc[m];
  __syncthreads();
  // the warps' partials of a row, summed in warp order
  for (int i = tid; i < 32 * MB; i += kRefThreads) {
    const int r = i / MB, m = i - r * MB, oo = tile * 32 + r;
    if (oo >= p.out || m >= p.Mc) continue;
    float s = 0.f;
    for (int w = 0; w < kRefWarps; ++w) s += red[(w * 32 + r) * MB + m];
    p.rref[static_cast<size_t>(m) * p.out + oo] = s;
  }
}

template <int MB, int KS>
cudaError_t launch_refine_mb(const RefineParam& p, size_t smem, cudaStream_t stream) {
  static std::atomic<size_t> allowed{48 * 1024};  // dynamic shared memory this kernel is opted in to
  if (smem > allowed.load()) {
    const cudaError_t e =
        cudaFuncSetAttribute(refine_kernel<MB, KS>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    allowed.store(smem);
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.tiles);
  cfg.blockDim = dim3(ref_warps(MB) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, refine_kernel<MB, KS>, p);
}

template <int MB>
cudaError_t launch_refine_ks(const RefineParam& p, size_t smem, cudaStream_t stream) {
  switch (p.Ks) {
    case 1: return launch_refine_mb<MB, 1>(p, smem, stream);
    case 2: return launch_refine_mb<MB, 2>(p, smem, stream);
    case 3: return launch_refine_mb<MB, 3>(p, smem, stream);
    default: return launch_refine_mb<MB, 4>(p, smem, stream);
  }
}

}  // namespace

size_t refine_smem_bytes(const bisco_layer* L, int MB) {
  if (L->ref_bases <= 0 || L->row_group <= 0) return 0;
  const int ng = static_cast<int>((static_cast<long long>(L->in) + L->row_group - 1) / L->row_group);
  return refine_smem(L->ref_bases, L->n_ref, ng, MB);
}

cudaError_t launch_refine(const bisco_layer* L, const void* X, int32_t x_dtype, int Mc, float* rref, int* status,
                          cudaStream_t stream) {
  RefineParam p{};
  p.bits = L->ref_bits;
  p.rrs = L->ref_row_scale;
  p.rcs = L->ref_col_scale;
  p.sdt = L->scale_dtype;
  p.idx = L->ref_idx;
  p.Ks = L->ref_bases;
  p.n_ref = L->n_ref;
  p.in = L->in;
  p.out = L->out;
  p.g = L->row_group;
  p.ngroups = static_cast<int>((static_cast<long long>(L->in) + L->row_group - 1) / L->row_group);
  p.tiles = (L->out + 31) / 32;
  p.X = X;
  p.xdt = x_dtype;
  p.ldx = L->in;
  p.Mc = Mc;
  p.rref = rref;
  p.status = status;
  const int MB = Mc <= 1 ? 1 : Mc <= 2 ? 2 : Mc <= 4 ? 4 : 8;
  const size_t smem = refine_smem(p.Ks, p.n_ref, p.ngroups, MB);
  switch (MB) {
    case 1: return launch_refine_ks<1>(p, smem, stream);
    case 2: return launch_refine_ks<2>(p, smem, stream);
    case 4: return launch_refine_ks<4>(p, smem, stream);
    default: return launch_refine_ks<8>(p, smem, stream);
  }
}

}  // namespace bisco

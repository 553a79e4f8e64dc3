// Tensor-core path for larger batches (32 to 128 batch rows per launch).
//
// With many batch rows the product is a dense contraction: for each segment,
//   D_seg[o][m] = sum_i A_seg[o][i] * B_seg[i][m].
// The signs are expanded into bf16 tiles in tensor memory and multiplied on the
// 5th-generation tensor cores (tcgen05.mma, kind::f16, A from tensor memory, B from
// shared memory, fp32 accumulators in tensor memory):
//   * a binary base k: A = +-c_k[i] (the column scale folded into the sign; exact in
//     bf16 because the scales are bf16), B = X (exact for bf16 activations; fp32
//     activations are split into bf16 high and low parts). Each base has its own
//     accumulator, and its row scale r_k is applied in the epilogue ("FluxBin",
//     Sec. 3.1, decoupled row-column binary bases);
//   * the correction's U^T: A = +-1, B = z split into high and low parts
//     ("BiLoCo", "The core idea": the second factor u applied to z = alpha (.) (V x));
//   * the salient columns: A = q (int8 values, exact in bf16), B = s_t * x[idx_t]
//     split the same way ("BiSCo-LLM", Sensitivity Protection). U^T and the salient
//     columns share one accumulator (no row scale);
//   * the correction's first phase z = alpha (.) (V x): A = +-1, B = X, alpha applied
//     in the epilogue as V's row scale.
// Every product is exact in fp32 and the sums are fp32, as on the CUDA-core path; a
// split value keeps 16 significant bits of its fp32 value.
//
// Work decomposition: cluster c owns 128 output rows; CTA r of the cluster takes 1/S of
// the (segment, 128-column K tile, part) steps, where a split segment (high and low bf16
// parts) has two steps per K tile, one per part, both accumulated into the segment's
// block. Four warp roles hand steps over on mbarriers (every waiter walks every step in
// order, so one pair of barriers per ring slot suffices):
//   * sign loader (1 warp): one 4-D tensor copy brings a step's 2 KB of packed sign words
//     (four 32-row tiles) and a 1-D tensor copy its 128 column scales into a ring of
//     shared-memory slots, tens of steps ahead (the first ones before the dependency
//     wait: weights never depend on the previous kernel);
//   * activation loader (1 warp): two tensor copies per step bring the bf16 activation
//     tile (64-column boxes, written in the 128-byte swizzle the MMA descriptors expect)
//     into a shared-memory stage once the MMAs that last read it are done;
//   * producers (16 warps): thread (row r, quarter q) expands 32 columns of row r into 16
//     tensor-memory columns of lane r (tcgen05.st), the A operand of the step; fp32-valued
//     or unaligned B tiles are written by the producers too;
//   * MMA issue (one thread): eight K=16 MMAs per step, committed to the "free" barriers
//     of the step's A and B stages.
// The S partial results meet in distributed shared memory and are added in CTA-rank
// order. A CTA takes all 512 tensor-memory columns and more than half of an SM's shared
// memory, so it is alone on its SM.

#include <cooperative_groups.h>
#include <cuda.h>  // CUtensorMap and the tensor-map encoder's argument types (no driver library is linked)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "bisco_internal.h"

namespace cg = cooperative_groups;

namespace bisco {

namespace {

constexpr int kTcProducers = 512;              // 16 producer (sign expansion) warps
constexpr int kTcThreads = kTcProducers + 96;  // + 1 MMA warp + 2 loader warps (signs, activations)
constexpr int kTcRows = 128;       // output rows per cluster (MMA M)
constexpr int kTcK = 128;          // input columns per step (eight K=16 MMAs)
constexpr int kTcMaxAStages = 4;   // expanded sign tiles in tensor memory (64 columns each)
constexpr int kTcMaxBStages = 6;   // activation tiles in shared memory
constexpr int kTcTmemCols = 512;   // the whole tensor memory (one CTA per SM)
constexpr int kTcMaxRaw = 64;      // raw sign-word / column-scale ring slots (as many as shared memory holds)
constexpr int kTcRawBytes = kTcRows * 16 + kTcK * 2;  // 128 rows x 16 bytes + 128 bf16 scales
constexpr int kTcMaxBlocks = kMaxSeg + 1;
constexpr int kTcHeader = 2048;    // barriers and the segment table, ahead of the raw ring
constexpr int kTcSegTable = 1280;  // offset of the segment table in the header

__device__ __forceinline__ unsigned saddr(const void* p) { return static_cast<unsigned>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ unsigned long long tc_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool tc_try(uint64_t* b, unsigned parity) {
  unsigned done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ void bar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
// Arrives on b and adds `bytes` to the transaction count of its current phase.
__device__ __forceinline__ void bar_expect_tx(uint64_t* b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes) : "memory");
}
// One box of a 1-D tensor map into this CTA's shared memory (completion counted in bytes
// on bar); out-of-range elements read 0.
__device__ __forceinline__ void tma_load_1d(void* dst, const CUtensorMap* map, int x, uint64_t* bar) {
  asm volatile("cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2}], [%3];" ::"r"(
                   saddr(dst)),
               "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(saddr(bar))
               : "memory");
}
// One box of a 4-D tensor map, coordinates innermost first.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
          saddr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(saddr(bar))
      : "memory");
}
// One box of a 2-D tensor map into this CTA's shared memory; completion counted in
// bytes on bar. Coordinates are (column, row) in elements; out-of-range elements read 0.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          saddr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(saddr(bar))
      : "memory");
}

// Waits (bounded in time: lim ns) until the phase with the given parity has completed.
__device__ __forceinline__ bool tc_wait(uint64_t* b, unsigned parity, unsigned long long lim) {
  if (tc_try(b, parity)) return true;
  const unsigned long long end = tc_ns() + lim;
  while (!tc_try(b, parity))
    if (tc_ns() > end) return false;
  return true;
}

// Shared-memory matrix descriptor, K-major with the 128-byte swizzle: start address
// (16-byte units), leading byte offset 1 (unused by this layout), stride byte offset
// 1024 (8 rows of 128 bytes), descriptor version 1 (bits 46-47), layout 2 = 128-byte
// swizzle (bits 61-63). A K step of 16 elements inside a 64-column block starts 32
// bytes further; the hardware applies the swizzle to the address bits.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* start) {
  const uint64_t a = (saddr(start) >> 4) & 0x3FFFu;
  return a | (1ull << 16) | (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), bf16 A and B
// (bits 7-9 and 10-12 = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24 (M = 128).
__device__ __forceinline__ uint32_t mma_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(kTcRows >> 4) << 24);
}

// D (tensor memory) (+)= A (tensor memory: lane = row, two bf16 per column along K)
// x B (shared memory, descriptor). No memory clobber: the issuing thread touches none of
// the operands; the mbarrier waits before and the commit after order the data, and
// volatile statements keep their order. (With the operand addresses computed ahead, the
// MMAs of a step issue back to back at the tensor core's rate: measured 64 cycles per
// 128 x 128 x 16 MMA, against 82 with a memory clobber and 143 with A in shared memory.)
__device__ __forceinline__ void mma_ts_bf16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(b)) : "memory");
}

// Byte offset of the 16-byte chunk (row, k8) (columns 8 k8 .. 8 k8 + 7) in a tile of
// `rows` rows and 128 columns (two 64-column blocks, 128-byte swizzle).
__device__ __forceinline__ unsigned tile_off(int row, int k8, int rows) {
  return (k8 >> 3) * static_cast<unsigned>(rows) * 128u + row * 128u + (((k8 & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ unsigned pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const unsigned*>(&h);
}

__device__ __forceinline__ float x_at(const PassParam& p, int m, long long col) {
  const long long i = static_cast<long long>(m) * p.ldx + col;
  return p.xdt == BISCO_BF16 ? __uint_as_float(static_cast<unsigned>(__ldcg(reinterpret_cast<const unsigned short*>(p.X) + i)) << 16)
                             : __ldcg(reinterpret_cast<const float*>(p.X) + i);
}

// Segment kinds of the tensor-core pass (the salient columns form one extra segment).
enum { kSegX = 0, kSegZ = 1, kSegSal = 3 };

struct TcSeg {
  const uint4* bits;
  const void* cscale;
  int nq, ncols, kind, cvec;
};

// Tensor maps of a launch's packed sign words and column scales, one per segment:
// bits[s] views segment s's packed layout [tiles][quads][32 rows][4 words] as a 4-D
// uint32 tensor (box: 4 words x 32 rows x 1 quad x 4 tiles = the 2 KB of one step);
// cs[s] views its bf16 column scales as a 1-D tensor (box: 128 scales).
struct TcMaps {
  CUtensorMap bits[kMaxSeg];
  CUtensorMap cs[kMaxSeg];
};

__device__ __forceinline__ TcSeg tc_seg(const PassParam& p, int s) {
  TcSeg g;
  if (s < p.nseg) {
    const SegParam& G = p.seg[s];
    g.bits = G.bits; g.cscale = G.cscale; g.nq = G.nq; g.ncols = G.ncols; g.kind = G.xsrc; g.cvec = G.cvec;
  } else {
    g.bits = nullptr; g.cscale = nullptr; g.nq = 0; g.ncols = p.n_sal; g.kind = kSegSal; g.cvec = 0;
  }
  return g;
}

// A launch's segments as the main loop reads them every step (a table in shared memory,
// filled once per CTA: kernel parameters indexed by a run-time segment number are slow).
struct TcSegInfo {
  TcSeg g;
  int parts;   // steps per K tile (2: high and low bf16 parts of fp32-valued B)
  int ktiles;  // 128-column K tiles
  int blk;     // accumulator block
};

// (segment, K tile, part) of a step; next() moves to the following step.
struct TcCursor {
  int seg, kt, part;
  __device__ __forceinline__ void init(const TcSegInfo* si, int nseg_all, int step) {
    seg = 0;
    while (seg < nseg_all - 1 && step >= si[seg].ktiles * si[seg].parts) {
      step -= si[seg].ktiles * si[seg].parts;
      ++seg;
    }
    kt = step / si[seg].parts;
    part = step - kt * si[seg].parts;
  }
  __device__ __forceinline__ void next(const TcSegInfo* si) {
    if (++part == si[seg].parts) {
      part = 0;
      if (++kt == si[seg].ktiles) { kt = 0; ++seg; }
    }
  }
};

// 16 bytes of a B tile: columns c..c+7 of batch row m (part 0: the value or its high
// bf16 part; part 1: the low part).
__device__ __forceinline__ uint4 b_chunk(const PassParam& p, const TcSeg& g, int m, int c, int part, int split) {
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = 0.f;
  if (m < p.Mc) {
    const int valid = max(0, min(8, g.ncols - c));
    if (g.kind == kSegSal) {
      int cc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) cc[j] = j < valid ? __ldg(p.sal_idx + c + j) : -1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j >= valid) continue;
        if (cc[j] >= 0 && cc[j] < p.xcols) v[j] = x_at(p, m, cc[j]) * __ldg(p.sal_scale + c + j);
        else if (part == 0) atomicExch(p.status, static_cast<int>(BISCO_ERR_INVALID_ARG));
      }
    } else if (g.kind == kSegX) {
      if (p.xdt == BISCO_BF16 && split == 1 && p.x_vec && valid == 8)
        return __ldcg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(p.X) + static_cast<long long>(m) * p.ldx + c));
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = j < valid ? x_at(p, m, c + j) : 0.f;
    } else if (g.kind == kSegZ) {
      const float* zr = p.Z + static_cast<long long>(m) * p.ldz + c;
      if (p.z_vec && valid == 8) {  // two 16-byte loads
        const float4 a = __ldcg(reinterpret_cast<const float4*>(zr));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(zr) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = j < valid ? __ldcg(zr + j) : 0.f;
      }
    }
  }
  if (split == 2) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float hi = __bfloat162float(__float2bfloat16_rn(v[j]));
      v[j] = part == 0 ? hi : v[j] - hi;
    }
  }
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// 16 bytes of an A tile: columns c..c+7 of output row o.
__device__ __forceinline__ uint4 a_chunk(const PassParam& p, const TcSeg& g, int o, int c) {
  if (o >= p.rows || c >= g.ncols || (g.kind != kSegSal && g.bits == nullptr)) return make_uint4(0u, 0u, 0u, 0u);
  const int valid = min(8, g.ncols - c);
  if (g.kind == kSegSal) {  // q[o][t] as bf16
    const int8_t* q = p.sal_q + static_cast<long long>(o) * p.sal_stride + c;
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = j < valid ? static_cast<float>(q[j]) : 0.f;
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
  // sign byte of columns c..c+7 from the packed layout (c is a multiple of 8)
  const unsigned* words = reinterpret_cast<const unsigned*>(g.bits + (static_cast<long long>(o >> 5) * g.nq + (c >> 7)) * 32 + (o & 31));
  const unsigned byte = (__ldg(words + ((c >> 5) & 3)) >> (c & 31)) & 0xFFu;
  // column scales as bf16 bits (1.0 without scales), zero past the segment's columns
  unsigned cs[4];
  if (g.cscale == nullptr) {
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[e] = (2 * e < valid ? 0x3F80u : 0u) | ((2 * e + 1 < valid ? 0x3F80u : 0u) << 16);
  } else if (g.cvec && valid == 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const unsigned short*>(g.cscale) + c));
    cs[0] = v.x; cs[1] = v.y; cs[2] = v.z; cs[3] = v.w;
  } else {
    const unsigned short* cp = reinterpret_cast<const unsigned short*>(g.cscale) + c;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      cs[e] = (2 * e < valid ? static_cast<unsigned>(__ldg(cp + 2 * e)) : 0u) |
              ((2 * e + 1 < valid ? static_cast<unsigned>(__ldg(cp + 2 * e + 1)) : 0u) << 16);
  }
  // a clear bit is the sign -1: set the bf16 sign bit
  unsigned w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const unsigned nb = ~(byte >> (2 * e));
    w[e] = cs[e] ^ (((nb & 1u) << 15) | ((nb & 2u) << 30));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Expands columns 32q .. 32q+31 of row r of a step from the raw ring slot into 16
// words of bf16 pairs (column 32q + 2t in the low half of word t): 32 sign bits and the
// step's 128 column scales (bf16 bits; 1.0 when the segment has none, 0 past its
// columns). A clear bit is the sign -1: the bf16 sign bit is set.
__device__ __forceinline__ void a_words(uint32_t (&w)[16], const unsigned char* raw, int r, int q, int ncols_left,
                                        bool has_cscale) {
  const unsigned nword = ~reinterpret_cast<const unsigned*>(raw + r * 16)[q];  // set bit: sign -1
  const unsigned short* cs = reinterpret_cast<const unsigned short*>(raw + kTcRows * 16);
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int k8 = 4 * q + jj;
    const unsigned nbyte = nword >> (8 * jj);
    unsigned c[4];
    if (has_cscale) {
      const uint4 cv = *reinterpret_cast<const uint4*>(cs + 8 * k8);
      c[0] = cv.x; c[1] = cv.y; c[2] = cv.z; c[3] = cv.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        c[e] = (8 * k8 + 2 * e < ncols_left ? 0x3F80u : 0u) | ((8 * k8 + 2 * e + 1 < ncols_left ? 0x3F80u : 0u) << 16);
    }
    // bits 2e and 2e+1 of the inverted byte become the sign bits (15, 31) of word e:
    // b * 0x40008000 for b < 4 puts bit 0 of b at 15 and 30, bit 1 at 16 and 31 (no carries)
#pragma unroll
    for (int e = 0; e < 4; ++e) w[4 * jj + e] = c[e] ^ ((((nbyte >> (2 * e)) & 3u) * 0x40008000u) & 0x80008000u);
  }
}

// Stores 16 consecutive 32-bit tensor-memory columns of this thread's lane (the warp's
// 32 lanes at once).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]), "r"(w[10]),
      "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}

// Accumulator blocks in tensor memory: one per X segment (row scale applied in the
// epilogue), one shared by U^T and the salient columns.
struct TcAcc {
  int nblk;
  int col[kTcMaxBlocks];    // first of the block's Np columns
  int split[kTcMaxBlocks];  // 1 or 2 parts (steps per K tile, accumulated into the same columns)
  int rseg[kTcMaxBlocks];   // segment whose row scale applies (-1: none)
  int blk_of_seg[kTcMaxBlocks];
  int ncols;
};

__host__ __device__ __forceinline__ TcAcc tc_acc(int nseg, const int* seg_kind, bool has_sal, bool x_bf16, int Np) {
  TcAcc a{};
  int shared = -1, col = 0;
  for (int s = 0; s < nseg + (has_sal ? 1 : 0); ++s) {
    const int kind = s < nseg ? seg_kind[s] : kSegSal;
    if (kind == kSegX) {
      const int b = a.nblk++;
      a.col[b] = col;
      a.split[b] = x_bf16 ? 1 : 2;
      a.rseg[b] = s;
      col += Np;
      a.blk_of_seg[s] = b;
    } else {
      if (shared < 0) {
        shared = a.nblk++;
        a.col[shared] = col;
        a.split[shared] = 2;
        a.rseg[shared] = -1;
        col += Np;
      }
      a.blk_of_seg[s] = shared;
    }
  }
  a.ncols = col;
  return a;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ PassParam p, const __grid_constant__ CUtensorMap tmap_x,
                   const __grid_constant__ TcMaps maps, const int use_tma, const int cs_tma, const int S,
                   const int Np, const int nA, const int nB, const int R, const int a_base,
                   const int dbg_skip_last, const unsigned long long wait_ns) {
  extern __shared__ __align__(1024) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int o0 = (blockIdx.x / S) * kTcRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_sal = p.n_sal > 0;
  const int nseg_all = p.nseg + (has_sal ? 1 : 0);
  int kinds[kMaxSeg];
  for (int s = 0; s < kMaxSeg; ++s) kinds[s] = s < p.nseg ? p.seg[s].xsrc : kSegZ;
  const TcAcc acc = tc_acc(p.nseg, kinds, has_sal, p.xdt == BISCO_BF16, Np);
  const unsigned b_bytes = static_cast<unsigned>(Np) * kTcK * 2;  // one activation stage

  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem);     // [kTcMaxAStages] sign tile expanded
  uint64_t* a_free = a_full + kTcMaxAStages;                // [kTcMaxAStages] its MMAs done
  uint64_t* b_full = a_free + kTcMaxAStages;                // [kTcMaxBStages] activation tile landed
  uint64_t* b_free = b_full + kTcMaxBStages;                // [kTcMaxBStages] its MMAs done
  uint64_t* all_done = b_free + kTcMaxBStages;              // [1]
  uint64_t* raw_full = all_done + 1;                        // [R] raw slot landed
  uint64_t* raw_free = raw_full + kTcMaxRaw;                // [R] raw slot read by every producer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(raw_free + kTcMaxRaw);
  TcSegInfo* si = reinterpret_cast<TcSegInfo*>(smem + kTcSegTable);  // [nseg_all]
  unsigned char* raw_ring = smem + kTcHeader;               // [R][kTcRawBytes]
  // [nB] activation tiles, 1024-byte aligned (128-byte swizzle atoms)
  unsigned char* stages = raw_ring + (static_cast<size_t>(R) * kTcRawBytes + 1023) / 1024 * 1024;
  float* recv = reinterpret_cast<float*>(raw_ring);         // used after the main loop (ring and stages)

  // (segment, K tile, part) steps; this CTA's range
  int nsteps = 0;
  for (int s = 0; s < nseg_all; ++s) nsteps += (tc_seg(p, s).ncols + kTcK - 1) / kTcK * acc.split[acc.blk_of_seg[s]];
  const int st0 = rank * nsteps / S, st1 = (rank + 1) * nsteps / S;

  if (threadIdx.x < nseg_all) {
    TcSegInfo& e = si[threadIdx.x];
    e.g = tc_seg(p, threadIdx.x);
    e.blk = acc.blk_of_seg[threadIdx.x];
    e.parts = acc.split[e.blk];
    e.ktiles = (e.g.ncols + kTcK - 1) / kTcK;
  }
  if (threadIdx.x == 0) {
    // a_full: every producer thread (its lane's columns stored); b_full: the activation
    // loader (with the tensor copy's byte count); a_free, b_free, all_done: MMA commits
    for (int s = 0; s < kTcMaxAStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(a_full + s)), "r"(kTcProducers) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(a_free + s)) : "memory");
    }
    for (int s = 0; s < kTcMaxBStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(b_full + s)) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(b_free + s)) : "memory");
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(all_done)) : "memory");
    // raw_full: the sign loader's lane 0 (with the tensor copies' byte count) and each of
    // its 32 lanes once its plain stores are done; raw_free: every producer thread
    for (int s = 0; s < R; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(raw_full + s)), "r"(33) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(raw_free + s)), "r"(kTcProducers) : "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_slot)), "n"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  // Peers write into this CTA's shared memory at the end; the split barrier tells them
  // that every CTA of the cluster is running.
  auto started = cluster.barrier_arrive();

  bool ok = true;
  unsigned touched = 0;  // bit b: accumulator block written by this CTA (same in every thread)
  const int n = st1 - st0;
  // accumulator blocks this CTA writes (every thread walks the steps)
  TcCursor cur;
  cur.init(si, nseg_all, st0);
  for (int i = 0; i < n; ++i, cur.next(si)) touched |= 1u << si[cur.seg].blk;
  cur.init(si, nseg_all, st0);

  if (warp == kTcProducers / 32 + 1) {
    // ---------------- sign loader warp ----------------
    // The step's raw sign words (the four 32-row tiles of its 128 rows, 512 bytes each in
    // the packed layout) arrive through one 4-D tensor copy and its 128 column scales
    // through one 1-D tensor copy (16-byte aligned scales; otherwise lanes 0..15 load them)
    // into raw slot i % R, up to R steps ahead of the producers. Rows past the layout and
    // columns past the segment read 0. The ring takes the shared memory the activation
    // tiles leave (tens of slots). Sign words never depend on the previous kernel, so the
    // first R slots are requested before the dependency wait.
    for (int i = 0; i < n; ++i) {
      const int rs = i % R;
      if (i >= R && !tc_wait(raw_free + rs, static_cast<unsigned>(i / R - 1) & 1u, wait_ns)) ok = false;
      const TcSeg& g = si[cur.seg].g;
      unsigned char* dst = raw_ring + rs * kTcRawBytes;
      const bool bits = g.kind != kSegSal && g.bits != nullptr;
      const bool cs_copy = bits && g.cscale != nullptr && ((cs_tma >> cur.seg) & 1);
      if (lane == 0 && dbg_skip_last && i == n - 1) {
        // test hook: the last step's copies and this lane's arrival never happen, so the
        // producers' bounded wait for it gives up; nothing reuses the slot afterwards
      } else if (lane == 0) {
        const unsigned bytes = (bits ? kTcRows * 16u : 0u) + (cs_copy ? kTcK * 2u : 0u);
        if (bytes > 0) {
          bar_expect_tx(raw_full + rs, bytes);
          if (bits) tma_load_4d(dst, &maps.bits[cur.seg], 0, 0, cur.kt, o0 / 32, raw_full + rs);
          if (cs_copy) tma_load_1d(dst + kTcRows * 16, &maps.cs[cur.seg], cur.kt * kTcK, raw_full + rs);
        } else {
          bar_arrive(raw_full + rs);
        }
      }
      if (bits && g.cscale != nullptr && !cs_copy && lane < kTcK / 8) {
        // unaligned scales (e.g. the second base of a layer with in % 8 != 0): plain loads
        // of columns 8 lane .. + 7 of the K tile, zero past the segment
        const int cc = cur.kt * kTcK + lane * 8;
        const int valid = max(0, min(8, g.ncols - cc));
        const unsigned short* cs = reinterpret_cast<const unsigned short*>(g.cscale);
        unsigned short v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = e < valid ? __ldg(cs + cc + e) : 0;
        *reinterpret_cast<uint4*>(dst + kTcRows * 16 + lane * 16) =
            make_uint4(v[0] | (static_cast<unsigned>(v[1]) << 16), v[2] | (static_cast<unsigned>(v[3]) << 16),
                       v[4] | (static_cast<unsigned>(v[5]) << 16), v[6] | (static_cast<unsigned>(v[7]) << 16));
      }
      bar_arrive(raw_full + rs);  // this lane's plain stores (release)
      cur.next(si);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
  } else if (warp == kTcProducers / 32 + 2) {
    // ---------------- activation loader warp ----------------
    // The activation tile of step j goes into its stage as soon as the MMAs that last
    // read the stage are done (tensor-map copies, or one arrival when the producers write
    // the B tile themselves).
    asm volatile("griddepcontrol.wait;" ::: "memory");  // activations may come from the previous kernel
    for (int j = 0; j < n; ++j, cur.next(si)) {
      const int sb = j % nB;
      if (j >= nB && !tc_wait(b_free + sb, static_cast<unsigned>(j / nB - 1) & 1u, wait_ns)) ok = false;
      unsigned char* B = stages + static_cast<size_t>(sb) * b_bytes;
      if (use_tma && si[cur.seg].g.kind == kSegX) {
        // both 64-column blocks (rows past the batch read 0), one box from each of lanes 0, 1
        if (lane == 0) bar_expect_tx(b_full + sb, b_bytes);
        __syncwarp();
        if (lane < 2) tma_load_2d(B + lane * Np * 128, &tmap_x, cur.kt * kTcK + lane * 64, 0, b_full + sb);
      } else if (lane == 0) {
        bar_arrive(b_full + sb);
      }
    }
  } else {
    asm volatile("griddepcontrol.wait;" ::: "memory");
  }
  if (warp < kTcProducers / 32) {
    // ---------------- producers ----------------
    // Thread (row r, quarter q) expands columns 32q .. 32q+31 of row r of every step into
    // 16 tensor-memory columns of lane r (the A operand of the step's MMAs).
    const int r = threadIdx.x & (kTcRows - 1), q = threadIdx.x >> 7;
    const uint32_t a_lane = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + static_cast<uint32_t>(a_base + 16 * q);
    for (int i = 0; i < n; ++i, cur.next(si)) {
      const int sa = i % nA, sb = i % nB, rs = i % R;
      // the sign stage is free once the MMAs that last read it are done
      if (i >= nA && !tc_wait(a_free + sa, static_cast<unsigned>(i / nA - 1) & 1u, wait_ns)) ok = false;
      if (!tc_wait(raw_full + rs, static_cast<unsigned>(i / R) & 1u, wait_ns)) ok = false;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int seg = cur.seg, kt = cur.kt, part = cur.part;
      const TcSeg& g = si[seg].g;
      const int c0 = kt * kTcK;
      uint32_t w[16];
      if (g.kind == kSegSal || g.bits == nullptr) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const uint4 v = a_chunk(p, g, o0 + r, c0 + 32 * q + 8 * jj);
          w[4 * jj] = v.x; w[4 * jj + 1] = v.y; w[4 * jj + 2] = v.z; w[4 * jj + 3] = v.w;
        }
      } else {
        a_words(w, raw_ring + rs * kTcRawBytes, r, q, g.ncols - c0, g.cscale != nullptr);
      }
      tmem_st16(a_lane + static_cast<uint32_t>(64 * sa), w);
      if (!(use_tma && g.kind == kSegX)) {
        // fp32-valued inputs (z, salient, fp32 X) and unaligned bf16 X: the producers write
        // the B tile once its stage is free; several chunks in flight
        if (i >= nB && !tc_wait(b_free + sb, static_cast<unsigned>(i / nB - 1) & 1u, wait_ns)) ok = false;
        unsigned char* B = stages + static_cast<size_t>(sb) * b_bytes;
        const int split = si[seg].parts;
#pragma unroll 4
        for (int ch = threadIdx.x; ch < Np * 16; ch += kTcProducers) {
          const int m = ch >> 4, k8 = ch & 15;  // lanes along a row: coalesced reads
          *reinterpret_cast<uint4*>(B + tile_off(m, k8, Np)) = b_chunk(p, g, m, c0 + 8 * k8, part, split);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic stores -> tensor core
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      bar_arrive(a_full + sa);
      bar_arrive(raw_free + rs);
    }
  } else if (warp == kTcProducers / 32 && lane == 0) {
    // ---------------- MMA issue (one thread) ----------------
    unsigned written = 0;  // bit b: accumulator block already written
    const uint32_t idesc = mma_idesc(Np);
    for (int i = 0; i < n; ++i, cur.next(si)) {
      const int sa = i % nA, sb = i % nB;
      if (!tc_wait(a_full + sa, static_cast<unsigned>(i / nA) & 1u, wait_ns)) ok = false;
      if (!tc_wait(b_full + sb, static_cast<unsigned>(i / nB) & 1u, wait_ns)) ok = false;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int blk = si[cur.seg].blk;
      const uint64_t b0 = smem_desc_sw128(stages + static_cast<size_t>(sb) * b_bytes);
      const uint32_t d = tmem + static_cast<uint32_t>(acc.col[blk]);
      const uint32_t a = tmem + static_cast<uint32_t>(a_base + 64 * sa);
      const uint32_t acc0 = ((written >> blk) & 1u) ? 1u : 0u;
      // K = 16 per MMA: 8 columns of A; 32 bytes (descriptor +2) along a B row, the
      // second 64-column block Np x 128 bytes further
#pragma unroll
      for (int kk = 0; kk < kTcK / 16; ++kk)
        mma_ts_bf16(d, a + 8u * kk, b0 + static_cast<uint64_t>((kk >> 2) * (Np * 8) + (kk & 3) * 2), idesc, kk == 0 ? acc0 : 1u);
      mma_commit(a_free + sa);
      mma_commit(b_free + sb);
      written |= 1u << blk;
    }
    mma_commit(all_done);
  }
  // row scales of this thread's epilogue row, loaded while the last MMAs run
  float rsv[kTcMaxBlocks];
  {
    const int o = o0 + (warp & 3) * 32 + lane;
    for (int b = 0; b < acc.nblk; ++b) {
      rsv[b] = 1.f;
      const int s = acc.rseg[b];
      if (s >= 0 && o < p.rows && p.seg[s].rscale != nullptr)
        rsv[b] = p.seg[s].rdt == BISCO_BF16
                     ? __uint_as_float(static_cast<unsigned>(__ldg(reinterpret_cast<const unsigned short*>(p.seg[s].rscale) + o)) << 16)
                     : __ldg(reinterpret_cast<const float*>(p.seg[s].rscale) + o);
    }
  }
  __syncwarp();
  if (!tc_wait(all_done, 0u, wait_ns)) ok = false;
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

  // every CTA of the cluster is done with its stages before partial sums are pushed
  cluster.barrier_wait(std::move(started));
  if (S > 1) cluster.sync();
  const int rows_per = (kTcRows + S - 1) / S;
  // recv[src][row][m] with a row stride of Np + 4 floats: a warp's 32 rows then start in
  // 32 different banks (a stride of Np floats put every lane's 16-byte pushes into the same
  // four banks)
  const int rstride = Np + 4;
  if (warp < kTcProducers / 32) {
    // warp w reads tensor-memory lanes 32 (w mod 4) .. + 31 (= rows of this CTA's tile) and
    // columns 16 (w / 4), + 64, ...: the 16 producer warps share the read-out
    const int lg = warp & 3;
    const int r = lg * 32 + lane;
    const int o = o0 + r;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(lg * 32) << 16);
    const int dst = r / rows_per;
    float* rp = S > 1 ? cluster.map_shared_rank(recv, dst) + (static_cast<size_t>(rank) * rows_per + (r - dst * rows_per)) * rstride
                      : nullptr;
    for (int m0 = 16 * (warp >> 2); m0 < Np; m0 += 16 * (kTcProducers / 128)) {
      float y[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) y[j] = 0.f;
      for (int b = 0; b < acc.nblk; ++b) {
        if (!((touched >> b) & 1u)) continue;
        uint32_t v0[16];
        const uint32_t ta = lane_addr + static_cast<uint32_t>(acc.col[b] + m0);
        asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
              : "=r"(v0[0]), "=r"(v0[1]), "=r"(v0[2]), "=r"(v0[3]), "=r"(v0[4]), "=r"(v0[5]), "=r"(v0[6]), "=r"(v0[7]),
                "=r"(v0[8]), "=r"(v0[9]), "=r"(v0[10]), "=r"(v0[11]), "=r"(v0[12]), "=r"(v0[13]), "=r"(v0[14]), "=r"(v0[15])
              : "r"(ta));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          y[j] = fmaf(__uint_as_float(v0[j]), rsv[b], y[j]);
        }
      }
      if (S > 1) {
        // push to the row's owner CTA: recv[rank][row - first row of owner][m], 16-byte stores
#pragma unroll
        for (int j = 0; j < 16; j += 4) *reinterpret_cast<float4*>(rp + m0 + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
      } else if (o < p.rows) {
        // no K split: this CTA holds the whole sum of its rows
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + j;
          if (m < p.Mc) {
            if (p.ydt == BISCO_BF16)
              reinterpret_cast<__nv_bfloat16*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = __float2bfloat16_rn(y[j]);
            else
              reinterpret_cast<float*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = y[j];
          }
        }
      }
    }
  }
  if (S > 1) {
    cluster.sync();  // all partial sums have landed
    // ---- owner: add the S partials in rank order and store ----
    const int rr0 = rank * rows_per, rr1 = min(kTcRows, rr0 + rows_per);
    const int nr = rr1 - rr0;
    if (nr > 0) {
      // (a) lanes along batch columns: 16-byte reads of recv[src][lr][m..m+3], sum in rank
      //     order, into a transposed tile [m][lr] (row stride nr + 1: no bank conflicts)
      float* tr = recv + static_cast<size_t>(S) * rows_per * rstride;
      const int tstride = nr + 1;
      for (int idx = threadIdx.x; idx < nr * (Np / 4); idx += kTcThreads) {
        const int lr = idx / (Np / 4), m4 = (idx - lr * (Np / 4)) * 4;
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < S; ++src) {
          const float4 v = *reinterpret_cast<const float4*>(recv + (static_cast<size_t>(src) * rows_per + lr) * rstride + m4);
          sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
        }
        tr[(m4 + 0) * tstride + lr] = sum.x;
        tr[(m4 + 1) * tstride + lr] = sum.y;
        tr[(m4 + 2) * tstride + lr] = sum.z;
        tr[(m4 + 3) * tstride + lr] = sum.w;
      }
      __syncthreads();
      // (b) lanes along output rows: coalesced stores of Y[m][o]
      for (int idx = threadIdx.x; idx < nr * Np; idx += kTcThreads) {
        const int m = idx / nr, lr = idx - m * nr;
        const int o = o0 + rr0 + lr;
        if (o >= p.rows || m >= p.Mc) continue;
        const float sum = tr[m * tstride + lr];
        if (p.ydt == BISCO_BF16)
          reinterpret_cast<__nv_bfloat16*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = __float2bfloat16_rn(sum);
        else
          reinterpret_cast<float*>(p.Y)[static_cast<long long>(m) * p.ldy + o] = sum;
      }
    }
  }
  if (!ok) atomicExch(p.status, static_cast<int>(BISCO_ERR_TIMEOUT));
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTcTmemCols) : "memory");
}

int tc_max_clusters(int S, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_kernel, &cfg) != cudaSuccess) return 0;
  return n;
}

// The driver's tensor-map encoder, looked up once through the runtime (no link-time
// dependency on the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// Tensor map of the launch's activation rows X[0 .. Mc)[0 .. xcols) (bf16, row stride ldx
// elements): boxes of 64 columns (128 bytes) x Np rows in the 128-byte swizzle, the layout
// the MMA descriptors expect; rows Mc .. Np-1 and columns past xcols read as zero.
// False when the launch has no binary base over X, X is not bf16, or its rows are not
// 16-byte aligned (the producers then write the B tiles).
bool x_tensor_map(const PassParam& p, int Np, CUtensorMap* map) {
  if (p.xdt != BISCO_BF16 || !p.x_vec || p.Mc <= 0 || p.xcols <= 0 || Np > 256) return false;
  bool has_x = false;
  for (int s = 0; s < p.nseg; ++s) has_x = has_x || (p.seg[s].xsrc == kSegX && p.seg[s].bits != nullptr);
  if (!has_x) return false;
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.xcols), static_cast<cuuint64_t>(p.Mc)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.ldx) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(Np)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p.X), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of the packed sign words (and, where 16-byte aligned, the bf16 column
// scales) of every segment with signs. Bit s of *cs_mask: segment s's scales come through
// cs[s]. False if a map cannot be encoded.
bool sign_maps(const PassParam& p, TcMaps* m, int* cs_mask) {
  *cs_mask = 0;
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return false;
  const cuuint64_t tiles = static_cast<cuuint64_t>((p.rows + 31) / 32);
  for (int s = 0; s < p.nseg; ++s) {
    const SegParam& G = p.seg[s];
    if (G.bits == nullptr) continue;
    const cuuint64_t nq = static_cast<cuuint64_t>(G.nq);
    const cuuint64_t dims[4] = {4, 32, nq, tiles};
    const cuuint64_t strides[3] = {16, 512, nq * 512};
    const cuuint32_t box[4] = {4, 32, 1, 4};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    if (enc(&m->bits[s], CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint4*>(G.bits), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
    if (G.cscale != nullptr && G.cvec && G.cdt == BISCO_BF16) {
      const cuuint64_t cdims[1] = {static_cast<cuuint64_t>(G.ncols)};
      const cuuint32_t cbox[1] = {static_cast<cuuint32_t>(kTcK)};
      const cuuint32_t ces[1] = {1};
      if (enc(&m->cs[s], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 1, const_cast<void*>(G.cscale), cdims, nullptr, cbox, ces,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
        *cs_mask |= 1 << s;
    }
  }
  return true;
}

}  // namespace

cudaError_t tc_ensure_attrs() {
  static std::once_flag once[64];
  static cudaError_t err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::call_once(once[dev & 63], [&] {
    err[dev & 63] = cudaFuncSetAttribute(tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(query_smem_limit()));
  });
  return err[dev & 63];
}

TcPlan make_tc_plan(int rows, int nseg, const int* seg_kind, const int* seg_ncols, int n_sal, bool x_bf16, int Mc,
                    int num_sms, size_t smem_limit) {
  TcPlan t{};
  t.Np = (Mc + 15) / 16 * 16;
  const TcAcc acc = tc_acc(nseg, seg_kind, n_sal > 0, x_bf16, t.Np);
  // tensor memory: the accumulators, then 64-column stages of expanded sign tiles
  t.a_base = (acc.ncols + 63) / 64 * 64;
  t.astages = std::min(kTcMaxAStages, (kTcTmemCols - t.a_base) / 64);
  if (t.astages < 2) return t;
  int nsteps = 0;
  for (int s = 0; s < nseg; ++s) nsteps += (seg_ncols[s] + kTcK - 1) / kTcK * acc.split[acc.blk_of_seg[s]];
  if (n_sal > 0) nsteps += (n_sal + kTcK - 1) / kTcK * 2;
  if (nsteps == 0) return t;
  const size_t stage = static_cast<size_t>(t.Np) * kTcK * 2;  // one activation tile
  // activation tiles: up to six stages, leaving at least 16 sign-word slots; the rest of
  // shared memory is sign-word ring
  t.stages = static_cast<int>(std::min<size_t>(kTcMaxBStages, (smem_limit - kTcHeader - 16 * kTcRawBytes) / stage));
  if (smem_limit < kTcHeader + t.stages * stage + 8 * static_cast<size_t>(kTcRawBytes)) return t;
  t.raw_slots = static_cast<int>(std::min<size_t>(kTcMaxRaw, (smem_limit - kTcHeader - t.stages * stage - 1023) / kTcRawBytes));
  const size_t fixed = kTcHeader;
  const size_t body = (static_cast<size_t>(t.raw_slots) * kTcRawBytes + 1023) / 1024 * 1024 + t.stages * stage;
  // more than half of the SM's shared memory: one CTA per SM (tensor memory is not shared)
  t.smem = std::min(std::max(fixed + body, smem_limit / 2 + 4096), smem_limit);
  if (fixed + body > t.smem) return t;
  tc_ensure_attrs();
  t.tiles = (rows + kTcRows - 1) / kTcRows;
  // split K over a cluster so that the grid covers the SMs
  int S = std::max(1, std::min({kMaxCluster, nsteps, num_sms / std::max(1, t.tiles)}));
  while (S > 1 && (S & (S - 1))) --S;  // power of two
  for (; S >= 1; S /= 2) {
    const size_t rows_per = (kTcRows + S - 1) / S;
    const size_t recv = (static_cast<size_t>(S) * rows_per * (t.Np + 4) + static_cast<size_t>(t.Np) * (rows_per + 1)) * 4;
    if (recv > body) continue;
    if (tc_max_clusters(S, t.smem) >= 1) break;
  }
  if (S < 1) return t;
  t.S = S;
  return t;
}

cudaError_t launch_tc(const PassParam& p, const TcPlan& t, cudaStream_t stream, const ImmaDebug* dbg) {
  const cudaError_t e = tc_ensure_attrs();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(t.tiles * t.S);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = t.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = t.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  CUtensorMap map;
  std::memset(&map, 0, sizeof(map));
  const int use_tma = x_tensor_map(p, t.Np, &map) ? 1 : 0;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  int cs_mask = 0;
  if (!sign_maps(p, &maps, &cs_mask)) return cudaErrorNotSupported;
  const int skip_last = dbg && dbg->skip_tile >= 0 ? 1 : 0;
  const unsigned long long wait_ns = dbg && dbg->wait_ns ? dbg->wait_ns : kDefaultWaitNs;
  return cudaLaunchKernelEx(&cfg, tc_gemm_kernel, p, map, maps, use_tma, cs_mask, t.S, t.Np, t.astages, t.stages, t.raw_slots,
                            t.a_base, skip_last, wait_ns);
}

}  // namespace bisco

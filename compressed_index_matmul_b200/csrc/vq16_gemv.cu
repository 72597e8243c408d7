// Small-batch GEMV for the 16-bit formats (1 <= M <= 8, VQ_FMT_VQ16 and the residual
// ladder VQ_FMT_VQ16_RVQ,
// K % 128 == 0, K <= 16384, M K <= 32768, N % 4 == 0), with the input rotation
// optionally applied inside the kernel.
//
// GLQ README, "How it works": one 16-bit index per group of 8 weights selects a
// codeword of a 65,536 x 8 codebook (1 MiB of fp16), too large for shared memory;
// "Inference kernels": the matvec gathers the 8-dim codewords from the
// L2-resident codebook.  Each group of row n contributes s * (x_g . cb[i]), so a
// lookup thread gathers its row's 16 codewords of a K-slice at once (16 x 16-byte
// loads in flight per thread, 8192 per SM) and dots them with the slice's x held
// in shared memory (one broadcast load per 4 inputs and token); every gathered
// codeword serves all M tokens.
//
// Rotated input (GLQ README, "How it works": random sign flips followed by a fast
// Walsh-Hadamard transform): when `signs` is given, every CTA computes the whole
// rotated input x'_m = H (signs . x_m) of every token in fp32 in shared memory
// (hadamard_blocks_to_smem, rotate.cuh); for a power-of-two K the orthonormal factor
// 1/sqrt(K) multiplies every partial sum, otherwise ("Bit widths": block-diagonal
// transform over the binary expansion of K) each block of x' is scaled by its own
// 1/sqrt(b) in shared memory.  The caller's x is the unrotated input, and no rotated copy of it
// is ever written to memory.
//
// Work split and reduction: no table is built, so the (K-slice, row) grid is cut
// in two dimensions.  CTAs form clusters of 2 (pairs fill every SM; larger
// clusters leave SMs of each GPC idle); a cluster owns blocks of up to 512 output
// rows, and CTA j of the pair takes slices [S j / 2, S (j+1) / 2) of them.  Each
// thread handles one (slice, row) position of a chunk of 512: it
// loads the row's 16 indices (two 16-byte loads, issued one chunk ahead) and its
// scales, gathers and dots, and stores the position's partial sum in shared
// memory.  Each CTA then adds its slices per row in slice order, and CTA j reduces
// half of the block's rows by reading both CTAs' sums over distributed shared
// memory in rank order (GLQ README, "Inference kernels": fixed-order split-K
// reduction).  The result depends only on the inputs and S, not on the number of
// clusters; there is no grid-wide barrier and no scratch memory.
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "rotate.cuh"
#include "tc_ptx.cuh"

namespace vq {

constexpr int kV16Consumers = 512;  // threads: one (slice, row) position each per chunk
constexpr int kV16Cluster = 2;      // CTAs per cluster (the K-slices are split over them)
constexpr int kV16MaxBlk = 512;     // rows per cluster block
constexpr int kV16MaxK = 16384;

constexpr int kV16MaxM = 8;           // tokens
constexpr int kV16MaxMK = 32768;      // tokens x K (the fp32 x of all tokens is in shared memory)
constexpr int kV16PartBytes = 65536;  // partial sums of one block

constexpr int kV16Cb8Bytes = 256 * 16;  // the ladder's 8-bit codebook

// Shared memory of one CTA: partials [ceil(S / C)][MT][rblk], row sums [MT][rblk],
// fp32 x [MT][K], and for the residual ladder its 8-bit codebook (byte offsets,
// 16-byte aligned; rblk is a multiple of 4).
struct V16Smem {
  int off_sum, off_x, off_cb8, bytes;
};
__host__ __device__ inline V16Smem v16_smem(int S, int MT, int rblk, int K, bool ladder) {
  V16Smem m;
  const int spc = (S + kV16Cluster - 1) / kV16Cluster;
  m.off_sum = spc * MT * rblk * 4;
  m.off_x = m.off_sum + MT * rblk * 4;
  m.off_cb8 = m.off_x + 4 * MT * K;
  m.bytes = m.off_cb8 + (ladder ? kV16Cb8Bytes : 0);
  return m;
}

// x . c for one group: 8 fp16 codeword halves against 8 fp32 inputs.
__device__ __forceinline__ float dot8(const uint4& c, const float4& xa, const float4& xb, float acc) {
  const float2 c0 = f16x2_to_f32x2(c.x), c1 = f16x2_to_f32x2(c.y), c2 = f16x2_to_f32x2(c.z),
               c3 = f16x2_to_f32x2(c.w);
  acc = fmaf(c0.x, xa.x, acc);
  acc = fmaf(c0.y, xa.y, acc);
  acc = fmaf(c1.x, xa.z, acc);
  acc = fmaf(c1.y, xa.w, acc);
  acc = fmaf(c2.x, xb.x, acc);
  acc = fmaf(c2.y, xb.y, acc);
  acc = fmaf(c3.x, xb.z, acc);
  acc = fmaf(c3.y, xb.w, acc);
  return acc;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// The 16 indices of residual stage t of the ladder at plane entry e (a multiple of
// 16): two 16-byte loads from 16-bit plane t, or one from the 8-bit plane.
__device__ __forceinline__ void load_ladder_stage(const LayerArgs& a, int t, int64_t e, int64_t NG, uint32_t (&w)[8]) {
  if (t > a.n16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.idx8 + e));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    w[4] = w[5] = w[6] = w[7] = 0u;
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(a.idx16 + (int64_t)(t - 1) * NG + e);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  }
}

// Index words (16 x uint16) and block scales of one (slice, row) position.
struct V16Pos {
  uint4 i0, i1;
  uint32_t sc;
};

// MT: tokens rounded up to 1, 2, 4 or 8 (the x of tokens M .. MT-1 is zero).
// kLadder: the residual ladder (GLQ README, "Bit widths"): after the primary stage,
// each residual stage t of the position is gathered the same way (its 16 indices
// loaded then, from plane t or the 8-bit plane) and its dot products are added as
// mult_t * (x . c_t) before the block scales.
template <typename T, int MT, bool kLadder>
__global__ void __launch_bounds__(kV16Consumers, 1)
    vq16_gemv_kernel(LayerArgs a, const int8_t* __restrict__ signs, float xscale, int S, int blocks_per_cluster,
                     int rblk) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.N, K = a.K, M = a.M;
  const V16Smem lay = v16_smem(S, MT, rblk, K, kLadder);
  float* part = reinterpret_cast<float*>(smem);                 // [ceil(S / C)][MT][rblk]
  float* csum = reinterpret_cast<float*>(smem + lay.off_sum);  // [MT][rblk]
  float* xs = reinterpret_cast<float*>(smem + lay.off_x);      // [MT][K]
  const int tid = threadIdx.x;
  const bool block_scales = (a.scale_group == 64);
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int ncl = gridDim.x / kV16Cluster, cl = blockIdx.x / kV16Cluster;
  const int sa = (int)((int64_t)S * rank / kV16Cluster), ns = (int)((int64_t)S * (rank + 1) / kV16Cluster) - sa;

  // Positions of block `bi`: (slice sa + p / nrows, row r0 + p % nrows), p < ns * nrows.
  auto block_rows = [&](int bi, int& r0) {
    r0 = (cl + bi * ncl) * rblk;
    return max(0, min(rblk, N - r0));
  };
  auto load_pos = [&](int p, int r0, int nrows, V16Pos& q) {
    const int sl = sa + p / nrows, row = r0 + p % nrows;
    const int64_t e = (int64_t)16 * ((int64_t)sl * N + row);  // first entry of (slice sl, row)
    q.i0 = __ldg(reinterpret_cast<const uint4*>(a.idx16 + e));
    q.i1 = __ldg(reinterpret_cast<const uint4*>(a.idx16 + e) + 1);
    q.sc = block_scales ? __ldg(reinterpret_cast<const uint32_t*>(a.scales + e / 8)) : 0u;  // 2 per row per slice
  };

  // The first position's indices do not depend on the previous kernel: load them
  // before waiting for it.
  V16Pos cur{}, nxt{};
  int bi = 0, p0 = 0, r0 = 0, nrows = block_rows(0, r0);
  if (tid < ns * nrows) load_pos(tid, r0, nrows, cur);
  // The ladder's 8-bit codebook (4 KiB) is gathered from shared memory: an L1 gather
  // of 32 random entries touches up to 32 different lines, a shared one at most 32
  // bank quads.  Visible to all threads after the barrier that ends the x staging.
  const uint4* cb8s = reinterpret_cast<const uint4*>(smem + lay.off_cb8);
  if (kLadder && a.n8 && tid < kV16Cb8Bytes / 16)
    reinterpret_cast<uint4*>(smem + lay.off_cb8)[tid] = __ldg(reinterpret_cast<const uint4*>(a.cb8) + tid);

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (signs) {
    // every token's rotation (the padding tokens M .. MT-1 are zero; the rotations'
    // barriers order those stores before any read)
    for (int i = M * K + tid; i < MT * K; i += kV16Consumers) xs[i] = 0.f;
    for (int m = 0; m < M; ++m)
      hadamard_blocks_to_smem<T, kV16Consumers, kV16MaxK>(static_cast<const uint16_t*>(a.x) + (int64_t)m * K, signs,
                                                          xs + m * K, K, tid, (K & (K - 1)) != 0);
  } else {
    const uint16_t* xg = static_cast<const uint16_t*>(a.x);
    for (int i = tid; i < MT * K; i += kV16Consumers) xs[i] = i < M * K ? Elt<T>::to_f32(xg[i]) : 0.f;
    __syncthreads();
  }

  const uint4* cb = reinterpret_cast<const uint4*>(a.cb1);
  for (; bi < blocks_per_cluster; ++bi) {
    const int npos = ns * nrows;
    for (p0 = 0; p0 < npos; p0 += kV16Consumers) {
      // this chunk's position is in `cur`; fetch the next chunk's (or the next block's first)
      const int p = p0 + tid;
      {
        int r0n = r0, nrn = nrows, pn = p + kV16Consumers;
        if (p0 + kV16Consumers >= npos) {  // next block
          pn = tid;
          nrn = bi + 1 < blocks_per_cluster ? block_rows(bi + 1, r0n) : 0;
        }
        if (pn < ns * nrn) load_pos(pn, r0n, nrn, nxt);
      }
      if (p < npos) {
        // the ladder's next residual stage's indices are always loaded one stage ahead,
        // so their latency overlaps the current stage's gathers
        uint32_t nw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        int64_t e_pos = 0, NG = 0;
        if constexpr (kLadder) {
          e_pos = (int64_t)16 * ((int64_t)(sa + p / nrows) * N + r0 + p % nrows);
          NG = (int64_t)N * (K / 8);
          if (a.n16 + a.n8 >= 2) load_ladder_stage(a, 2, e_pos, NG, nw);
        }
        const uint32_t iw[8] = {cur.i0.x, cur.i0.y, cur.i0.z, cur.i0.w, cur.i1.x, cur.i1.y, cur.i1.z, cur.i1.w};
        uint4 c[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) c[g] = __ldg(cb + ((iw[g >> 1] >> (16 * (g & 1))) & 0xFFFFu));
        const float* xsl = xs + (sa + p / nrows) * 128;
        float blk[MT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) blk[m][0] = blk[m][1] = 0.f;
#pragma unroll
        for (int g = 0; g < 16; ++g) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float4* xv = reinterpret_cast<const float4*>(xsl + m * K + 8 * g);
            blk[m][g >> 3] = dot8(c[g], xv[0], xv[1], blk[m][g >> 3]);
          }
        }
        if constexpr (kLadder) {
          const int nst = a.n16 + a.n8;
#pragma unroll 1
          for (int t = 2; t <= nst; ++t) {
            const bool is8 = t > a.n16;
            const float mt = t == 2 ? a.mult[0] : (t == 3 ? a.mult[1] : a.mult[2]);
            const uint4* cbt = reinterpret_cast<const uint4*>(t == 2 ? a.cbr[0] : (t == 3 ? a.cbr[1] : a.cbr[2]));
            uint32_t jw[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) jw[q] = nw[q];
            if (t < nst) load_ladder_stage(a, t + 1, e_pos, NG, nw);
            uint4 cr[16];
#pragma unroll
            for (int g = 0; g < 16; ++g) {
              if (is8)
                cr[g] = cb8s[(jw[g >> 2] >> (8 * (g & 3))) & 0xFFu];
              else
                cr[g] = __ldg(cbt + ((jw[g >> 1] >> (16 * (g & 1))) & 0xFFFFu));
            }
            float tb[MT][2];
#pragma unroll
            for (int m = 0; m < MT; ++m) tb[m][0] = tb[m][1] = 0.f;
#pragma unroll
            for (int g = 0; g < 16; ++g) {
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                const float4* xv = reinterpret_cast<const float4*>(xsl + m * K + 8 * g);
                tb[m][g >> 3] = dot8(cr[g], xv[0], xv[1], tb[m][g >> 3]);
              }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              blk[m][0] = fmaf(mt, tb[m][0], blk[m][0]);
              blk[m][1] = fmaf(mt, tb[m][1], blk[m][1]);
            }
          }
        }
        const float2 sc = block_scales ? f16x2_to_f32x2(cur.sc) : make_float2(1.f, 1.f);
#pragma unroll
        for (int m = 0; m < MT; ++m)  // the per-row scale is applied once, at the reduction
          part[((p / nrows) * MT + m) * rblk + p % nrows] =
              block_scales ? fmaf(blk[m][1], sc.y, blk[m][0] * sc.x) : blk[m][0] + blk[m][1];
      }
      cur = nxt;
    }
    __syncthreads();
    // this CTA's slices, in order, per row of the block
    for (int i = tid; i < MT * nrows; i += kV16Consumers) {
      const int m = i / nrows, r = i - m * nrows;
      float v = 0.f;
      for (int k = 0; k < ns; ++k) v += part[(k * MT + m) * rblk + r];
      csum[m * rblk + r] = v;
    }
    // rows [nrows j / C, nrows (j+1) / C) of the block, every token: the C CTAs' sums
    // in rank order (at most MT x kV16MaxBlk / kV16Cluster outputs per CTA)
    const int ra = (int)((int64_t)nrows * rank / kV16Cluster), rb = (int)((int64_t)nrows * (rank + 1) / kV16Cluster);
    const int nr = rb - ra;
    constexpr int kOut = (MT * kV16MaxBlk / kV16Cluster + kV16Consumers - 1) / kV16Consumers;
    float row_scale[kOut];
#pragma unroll
    for (int o = 0; o < kOut; ++o) {
      const int i = tid + o * kV16Consumers;
      row_scale[o] = (i < M * nr && !block_scales) ? f16_bits_to_f32(a.scales[r0 + ra + i % nr]) : 1.f;
    }
    ptx::cluster_sync();  // every CTA's csum is complete and visible to the cluster
#pragma unroll
    for (int o = 0; o < kOut; ++o) {
      const int i = tid + o * kV16Consumers;
      if (i < M * nr) {
        const int m = i / nr, r = ra + i - m * nr;
        const uint32_t local = smem_u32(csum + m * rblk + r);
        float v = 0.f;
#pragma unroll
        for (int q = 0; q < kV16Cluster; ++q) v += ld_cluster_f32(ptx::map_shared_rank(local, q));
        float out = v * xscale * row_scale[o];
        if (a.addend) out += a.addend[(int64_t)m * N + r0 + r];  // the sparse correction's x . C^T term
        static_cast<uint16_t*>(a.y)[(int64_t)m * N + r0 + r] = Elt<T>::from_f32(out);
      }
    }
    ptx::cluster_sync();  // no CTA reuses or releases its csum while another reads it
    if (bi + 1 < blocks_per_cluster) {
      nrows = block_rows(bi + 1, r0);
      if (npos == 0 && tid < ns * nrows) load_pos(tid, r0, nrows, cur);  // no chunk prefetched it
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Clusters of kV16Cluster CTAs that can be resident at once (the grid may exceed
// it; clusters are independent).  Queried once per device.
static int v16_max_clusters(int num_sms);

struct V16Geom {
  int ncl, blocks_per_cluster, rblk;
};

// Tokens the kernel is compiled for: M rounded up to 1, 2, 4 or 8.
static int v16_mt(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

static V16Geom v16_geom(int N, int clusters, int S, int MT) {
  V16Geom g;
  g.ncl = clusters < 1 ? 1 : clusters;
  const int quads = (N + 3) / 4;
  // rows per block: at most 512, and the block's partial sums fit kV16PartBytes
  const int spc = (S + kV16Cluster - 1) / kV16Cluster;
  int cap = kV16PartBytes / (spc * MT * 4) / 4 * 4;
  if (cap > kV16MaxBlk) cap = kV16MaxBlk;
  if (cap < 4) cap = 4;
  g.blocks_per_cluster = (N + g.ncl * cap - 1) / (g.ncl * cap);
  const int blocks = g.ncl * g.blocks_per_cluster;
  g.rblk = 4 * ((quads + blocks - 1) / blocks);
  if (g.rblk > cap) g.rblk = cap;
  g.ncl = (N + g.rblk * g.blocks_per_cluster - 1) / (g.rblk * g.blocks_per_cluster);  // drop idle clusters
  return g;
}

// Largest shared-memory size of any launch: capped partials, row sums of 8 tokens x
// 512 rows, fp32 x of M K <= kV16MaxMK inputs, the ladder's 8-bit codebook.
static int v16_max_smem() { return kV16PartBytes + kV16MaxM * kV16MaxBlk * 4 + 4 * kV16MaxMK + kV16Cb8Bytes; }

static int v16_max_clusters(int num_sms) {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / kV16Cluster;
  int c = cached[dev].load(std::memory_order_acquire);
  if (c > 0) return c;
  const int smem = v16_max_smem();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kV16Cluster * (num_sms / kV16Cluster));
  cfg.blockDim = dim3(kV16Consumers);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kV16Cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(vq16_gemv_kernel<__half, 8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, vq16_gemv_kernel<__half, 8, false>, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = num_sms / kV16Cluster;
  }
  cached[dev].store(n, std::memory_order_release);
  return n;
}

bool plan_vq16(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  if (M < 1 || M > kV16MaxM || (d.fmt != VQ_FMT_VQ16 && d.fmt != VQ_FMT_VQ16_RVQ) || d.K % 128 != 0 || d.K > kV16MaxK ||
      v16_mt(M) * d.K > kV16MaxMK || d.N % 4 != 0 || dev.smem_optin < v16_max_smem())
    return false;
  const V16Geom g = v16_geom(d.N, v16_max_clusters(dev.num_sms), d.K / 128, v16_mt(M));
  p->path = VQ_PATH_GATHER;
  p->splits = d.K / 128;
  p->k_per_split = 128;
  p->launches = 1;
  p->scratch_bytes = 0;  // partial sums stay in shared memory
  p->tickets = 0;
  p->grid = g.ncl * kV16Cluster;
  p->ctas = p->grid;
  return true;
}

template <typename T, int MT, bool kLadder>
static cudaError_t launch_vq16_t(const LayerArgs& a, int grid, const int8_t* signs, cudaStream_t s) {
  const int S = a.K / 128;
  auto kern = vq16_gemv_kernel<T, MT, kLadder>;
  static std::atomic<uint64_t> opted{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (!(opted.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, v16_max_smem());
    // Prefer L1 over shared memory beyond what a launch asks for: the L1 caches
    // part of the 1 MiB codebook for the gathers.
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxL1);
    if (e != cudaSuccess) return e;
    opted.fetch_or(bit, std::memory_order_acq_rel);
  }
  int ncl = grid / kV16Cluster;
  if (ncl < 1) ncl = 1;
  const V16Geom g = v16_geom(a.N, ncl, S, MT);
  const int smem = v16_smem(S, MT, g.rblk, a.K, kLadder).bytes;
  // Orthonormal factor of the rotation, rounded once from double precision: a
  // power-of-two K takes it at the store; otherwise each block was scaled in shared
  // memory
  const bool pow2 = (a.K & (a.K - 1)) == 0;
  const float xscale = signs && pow2 ? (float)(1.0 / std::sqrt((double)a.K)) : 1.f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.ncl * kV16Cluster);
  cfg.blockDim = dim3(kV16Consumers);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kV16Cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the previous kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a, signs, xscale, S, g.blocks_per_cluster, g.rblk);
}

template <typename T, bool kLadder>
static cudaError_t launch_vq16_m(const LayerArgs& a, int grid, const int8_t* signs, cudaStream_t s) {
  switch (v16_mt(a.M)) {
    case 1: return launch_vq16_t<T, 1, kLadder>(a, grid, signs, s);
    case 2: return launch_vq16_t<T, 2, kLadder>(a, grid, signs, s);
    case 4: return launch_vq16_t<T, 4, kLadder>(a, grid, signs, s);
    default: return launch_vq16_t<T, 8, kLadder>(a, grid, signs, s);
  }
}

cudaError_t launch_vq16(const LayerArgs& a, const Plan& p, const int8_t* signs, cudaStream_t s) {
  const bool lad = a.fmt == kFmtVq16Rvq;
  if (a.act == VQ_BF16)
    return lad ? launch_vq16_m<__nv_bfloat16, true>(a, p.grid, signs, s)
               : launch_vq16_m<__nv_bfloat16, false>(a, p.grid, signs, s);
  return lad ? launch_vq16_m<__half, true>(a, p.grid, signs, s) : launch_vq16_m<__half, false>(a, p.grid, signs, s);
}

}  // namespace vq

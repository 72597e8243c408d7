// Batch-1 GEMV for the single-stage 16-bit format (M == 1, VQ_FMT_VQ16,
// K % 128 == 0, K <= 16384, N % 4 == 0), with the input rotation optionally
// applied inside the kernel.
//
// GLQ README, "How it works": one 16-bit index per group of 8 weights selects a
// codeword of a 65,536 x 8 codebook (1 MiB of fp16), too large for shared memory;
// "Inference kernels": the matvec gathers the 8-dim codewords from the
// L2-resident codebook.  Each group of row n contributes s * (x_g . cb[i]), so a
// lookup thread gathers its row's 16 codewords of a K-slice at once (16 x 16-byte
// loads in flight per thread, 8192 per SM) and dots them with the slice's x held
// in shared memory (one broadcast load per 4 inputs).
//
// Rotated input (GLQ README, "How it works": random sign flips followed by a fast
// Walsh-Hadamard transform): when `signs` is given, every CTA computes the whole
// rotated vector x' = H (signs . x) in fp32 in shared memory (the five lowest
// butterfly stages on registers with warp shuffles, the rest in shared memory,
// natural Sylvester order); the orthonormal factor 1/sqrt(K) multiplies every
// partial sum.  The caller's x is the unrotated input, and no rotated copy of it
// is ever written to memory.
//
// Work split and reduction: no table is built, so the (K-slice, row) grid is cut
// in two dimensions.  CTAs form clusters of 2 (pairs fill every SM; larger
// clusters leave SMs of each GPC idle); a cluster owns blocks of up to 512 output
// rows, and CTA j of the pair takes slices [S j / 2, S (j+1) / 2) of them.  Each thread handles one (slice, row) position of a chunk of 512: it
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
#include "tc_ptx.cuh"

namespace vq {

constexpr int kV16Consumers = 512;  // threads: one (slice, row) position each per chunk
constexpr int kV16Cluster = 2;      // CTAs per cluster (the K-slices are split over them)
constexpr int kV16MaxBlk = 512;     // rows per cluster block
constexpr int kV16MaxK = 16384;
constexpr int kV16MaxSpc = kV16MaxK / 128 / kV16Cluster;  // slices per CTA

// Shared memory of one CTA: partials [ceil(S / C)][rblk], row sums [rblk], fp32 x [K]
// (byte offsets, 16-byte aligned; rblk is a multiple of 4).
struct V16Smem {
  int off_sum, off_x, bytes;
};
__host__ __device__ inline V16Smem v16_smem(int S, int rblk, int K) {
  V16Smem m;
  const int spc = (S + kV16Cluster - 1) / kV16Cluster;
  m.off_sum = spc * rblk * 4;
  m.off_x = m.off_sum + rblk * 4;
  m.bytes = m.off_x + 4 * K;
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

// Unnormalised rotation H_K (signs . x) of one token into xs (fp32), K = 2^p with
// 128 <= K <= kV16MaxK, by the kV16Consumers threads (named barrier 1), with
// E = max(1, K/512) elements per thread and R = K / (32 E) (compile-time, so every
// stage is straight-line code).  Pass 1: thread t holds E consecutive elements;
// the log2(E) lowest butterfly stages run on registers, the next five across the
// warp's lanes with shuffles.  Pass 2: the log2(R) remaining (highest) stages run
// on registers over groups of R elements at stride 32 E.  Every stage is a
// butterfly (u + w, u - w) on one index bit, so the result is H_K (signs . x) with
// H_K[k][j] = (-1)^popcount(k & j) (natural Sylvester order).
template <typename T, int E, int R>
__device__ __forceinline__ void rotate_to_smem(const uint16_t* __restrict__ x, const int8_t* __restrict__ signs,
                                               float* xs, int tid) {
  constexpr int K = 32 * E * R;
  constexpr int D = 32 * E;
  const int lane = tid & 31;
  if (tid * E < K) {  // whole warps (K is a multiple of 32 E)
    float v[E];
    if (E >= 8) {
      // E consecutive inputs (16-byte loads) and signs (8-byte loads)
#pragma unroll
      for (int c = 0; c < E / 8; ++c) {
        const uint4 xw = *reinterpret_cast<const uint4*>(x + tid * E + 8 * c);
        const uint2 sw = *reinterpret_cast<const uint2*>(signs + tid * E + 8 * c);
        const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int8_t sg = (int8_t)(((q < 4 ? sw.x : sw.y) >> (8 * (q & 3))) & 0xFFu);
          v[8 * c + q] = Elt<T>::to_f32((uint16_t)(xa[q >> 1] >> (16 * (q & 1)))) * (float)sg;
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = Elt<T>::to_f32(x[tid * E + e]) * (float)signs[tid * E + e];
    }
#pragma unroll
    for (int h = 1; h < E; h <<= 1)  // stages h = 1 .. E/2 on registers
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (!(e & h)) {
          const float u = v[e], w = v[e + h];
          v[e] = u + w;
          v[e + h] = u - w;
        }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1)  // stages h = E .. 16 E across the lanes
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
        v[e] = (lane & m) ? (o - v[e]) : (v[e] + o);
      }
#pragma unroll
    for (int e = 0; e < E; ++e) xs[tid * E + e] = v[e];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kV16Consumers) : "memory");
  for (int gb = tid; gb < D; gb += kV16Consumers) {  // stages h = 32 E .. K/2
    float u[R];
#pragma unroll
    for (int j = 0; j < R; ++j) u[j] = xs[gb + j * D];
#pragma unroll
    for (int h = 1; h < R; h <<= 1)
#pragma unroll
      for (int j = 0; j < R; ++j)
        if (!(j & h)) {
          const float p = u[j], q = u[j + h];
          u[j] = p + q;
          u[j + h] = p - q;
        }
#pragma unroll
    for (int j = 0; j < R; ++j) xs[gb + j * D] = u[j];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kV16Consumers) : "memory");
}

// rotate_to_smem for a power-of-two K in [128, kV16MaxK].
template <typename T>
__device__ __forceinline__ void rotate_any(const uint16_t* x, const int8_t* signs, float* xs, int K, int tid) {
  switch (K) {
    case 128: rotate_to_smem<T, 1, 4>(x, signs, xs, tid); break;
    case 256: rotate_to_smem<T, 1, 8>(x, signs, xs, tid); break;
    case 512: rotate_to_smem<T, 1, 16>(x, signs, xs, tid); break;
    case 1024: rotate_to_smem<T, 2, 16>(x, signs, xs, tid); break;
    case 2048: rotate_to_smem<T, 4, 16>(x, signs, xs, tid); break;
    case 4096: rotate_to_smem<T, 8, 16>(x, signs, xs, tid); break;
    case 8192: rotate_to_smem<T, 16, 16>(x, signs, xs, tid); break;
    default: rotate_to_smem<T, 32, 16>(x, signs, xs, tid); break;  // 16384
  }
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Index words (16 x uint16) and block scales of one (slice, row) position.
struct V16Pos {
  uint4 i0, i1;
  uint32_t sc;
};

template <typename T>
__global__ void __launch_bounds__(kV16Consumers, 1)
    vq16_gemv_kernel(LayerArgs a, const int8_t* __restrict__ signs, float xscale, int S, int blocks_per_cluster,
                     int rblk) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int N = a.N, K = a.K;
  const V16Smem lay = v16_smem(S, rblk, K);
  float* part = reinterpret_cast<float*>(smem);                 // [ceil(S / C)][rblk]
  float* csum = reinterpret_cast<float*>(smem + lay.off_sum);  // [rblk]
  float* xs = reinterpret_cast<float*>(smem + lay.off_x);      // [K]
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

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (signs) {
    rotate_any<T>(static_cast<const uint16_t*>(a.x), signs, xs, K, tid);
  } else {
    const uint16_t* xg = static_cast<const uint16_t*>(a.x);
    for (int i = tid; i < K; i += kV16Consumers) xs[i] = Elt<T>::to_f32(xg[i]);
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
        const uint32_t iw[8] = {cur.i0.x, cur.i0.y, cur.i0.z, cur.i0.w, cur.i1.x, cur.i1.y, cur.i1.z, cur.i1.w};
        uint4 c[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) c[g] = __ldg(cb + ((iw[g >> 1] >> (16 * (g & 1))) & 0xFFFFu));
        const float4* xv = reinterpret_cast<const float4*>(xs + (int64_t)(sa + p / nrows) * 128);
        float blk[2] = {0.f, 0.f};
#pragma unroll
        for (int g = 0; g < 16; ++g) blk[g >> 3] = dot8(c[g], xv[2 * g], xv[2 * g + 1], blk[g >> 3]);
        float acc;
        if (block_scales) {
          const float2 sc = f16x2_to_f32x2(cur.sc);
          acc = fmaf(blk[1], sc.y, blk[0] * sc.x);
        } else {
          acc = blk[0] + blk[1];
        }
        part[(p / nrows) * rblk + p % nrows] = acc;
      }
      cur = nxt;
    }
    __syncthreads();
    // this CTA's slices, in order, per row of the block
    for (int r = tid; r < nrows; r += kV16Consumers) {
      float v = 0.f;
      for (int k = 0; k < ns; ++k) v += part[k * rblk + r];
      csum[r] = v;
    }
    // rows [nrows j / C, nrows (j+1) / C) of the block: the C CTAs' sums in rank order
    const int ra = (int)((int64_t)nrows * rank / kV16Cluster), rb = (int)((int64_t)nrows * (rank + 1) / kV16Cluster);
    const int r = ra + tid;  // a block has at most kV16MaxBlk / kV16Cluster <= kV16Consumers rows per CTA
    const float row_scale = (r < rb && !block_scales) ? f16_bits_to_f32(a.scales[r0 + r]) : 1.f;
    ptx::cluster_sync();  // every CTA's csum is complete and visible to the cluster
    if (r < rb) {
      const uint32_t local = smem_u32(csum + r);
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < kV16Cluster; ++q) v += ld_cluster_f32(ptx::map_shared_rank(local, q));
      static_cast<uint16_t*>(a.y)[r0 + r] = Elt<T>::from_f32(v * xscale * row_scale);
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
static int v16_max_clusters(int smem, int num_sms);

struct V16Geom {
  int ncl, blocks_per_cluster, rblk;
};

static V16Geom v16_geom(int N, int clusters) {
  V16Geom g;
  g.ncl = clusters < 1 ? 1 : clusters;
  const int quads = (N + 3) / 4;
  g.blocks_per_cluster = (N + g.ncl * kV16MaxBlk - 1) / (g.ncl * kV16MaxBlk);
  const int blocks = g.ncl * g.blocks_per_cluster;
  g.rblk = 4 * ((quads + blocks - 1) / blocks);
  if (g.rblk > kV16MaxBlk) g.rblk = kV16MaxBlk;
  g.ncl = (N + g.rblk * g.blocks_per_cluster - 1) / (g.rblk * g.blocks_per_cluster);  // drop idle clusters
  return g;
}

static int v16_max_clusters(int smem, int num_sms) {
  // (the largest shared-memory size any launch asks for, so the count holds for all)
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / kV16Cluster;
  int c = cached[dev].load(std::memory_order_acquire);
  if (c > 0) return c;
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
  if (cudaFuncSetAttribute(vq16_gemv_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, vq16_gemv_kernel<__half>, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = num_sms / kV16Cluster;
  }
  cached[dev].store(n, std::memory_order_release);
  return n;
}

bool plan_vq16(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  if (M != 1 || d.fmt != VQ_FMT_VQ16 || d.K % 128 != 0 || d.K > kV16MaxK || d.N % 4 != 0 ||
      dev.smem_optin < v16_smem(kV16MaxK / 128, kV16MaxBlk, kV16MaxK).bytes)
    return false;
  const V16Geom g =
      v16_geom(d.N, v16_max_clusters(v16_smem(kV16MaxK / 128, kV16MaxBlk, kV16MaxK).bytes, dev.num_sms));
  p->path = VQ_PATH_GATHER;
  p->splits = d.K / 128;
  p->k_per_split = 128;
  p->launches = 1;
  p->scratch_bytes = 0;  // partial sums stay in shared memory
  p->tickets = 0;
  p->grid = g.ncl * kV16Cluster;
  return true;
}

template <typename T>
static cudaError_t launch_vq16_t(const LayerArgs& a, int grid, const int8_t* signs, cudaStream_t s) {
  const int S = a.K / 128;
  auto kern = vq16_gemv_kernel<T>;
  static std::atomic<uint64_t> opted{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (!(opted.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             v16_smem(kV16MaxK / 128, kV16MaxBlk, kV16MaxK).bytes);
    // Prefer L1 over shared memory beyond what a launch asks for: the L1 caches
    // part of the 1 MiB codebook for the gathers.
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxL1);
    if (e != cudaSuccess) return e;
    opted.fetch_or(bit, std::memory_order_acq_rel);
  }
  int ncl = grid / kV16Cluster;
  if (ncl < 1) ncl = 1;
  const V16Geom g = v16_geom(a.N, ncl);
  const int smem = v16_smem(S, g.rblk, a.K).bytes;
  // Orthonormal factor of the rotation, rounded once from double precision.
  const float xscale = signs ? (float)(1.0 / std::sqrt((double)a.K)) : 1.f;
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

cudaError_t launch_vq16(const LayerArgs& a, const Plan& p, const int8_t* signs, cudaStream_t s) {
  return a.act == VQ_BF16 ? launch_vq16_t<__nv_bfloat16>(a, p.grid, signs, s)
                          : launch_vq16_t<__half>(a, p.grid, signs, s);
}

}  // namespace vq

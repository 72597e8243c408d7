// Small kernels of libvqlinear: the fixed-order split-K reduction, the input
// rotation (sign flip + fast Walsh-Hadamard transform), and the debug exports
// that materialise unpacked indices / decoded weights into caller buffers.
#include "common.cuh"
#include "rotate.cuh"
#include "internal.h"
#include "tools.h"
#include "ladder.cuh"
#include "tc_ptx.cuh"

namespace vq {

// ---------------------------------------------------------------- split reduce
//
// y[m][n] = RN( sum_{s=0..S-1} partial[s][m][n] ), summed in increasing s so the
// result does not depend on which split finished first (GLQ README, "Inference
// kernels": fixed-order scratch-buffer split-K instead of atomics).
template <typename T>
__global__ void split_reduce_kernel(const float* __restrict__ partial, uint16_t* __restrict__ y, int splits,
                                    int64_t MN) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < MN; i += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += partial[s * MN + i];
    y[i] = Elt<T>::from_f32(acc);
  }
}

cudaError_t launch_split_reduce(const float* partial, void* y, int splits, int M, int N, int act, cudaStream_t s) {
  const int64_t MN = (int64_t)M * N;
  const int threads = 256;
  int blocks = (int)((MN + threads - 1) / threads);
  if (blocks > 4096) blocks = 4096;
  if (act == VQ_BF16)
    split_reduce_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(partial, (uint16_t*)y, splits, MN);
  else
    split_reduce_kernel<__half><<<blocks, threads, 0, s>>>(partial, (uint16_t*)y, splits, MN);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------- rotation
//
// GLQ README, "How it works": Randomized Hadamard Transform = random sign flips
// followed by a fast Walsh-Hadamard transform; "Bit widths": a K that is not a
// power of two is cut into power-of-two blocks (binary expansion, largest first),
// each rotated on its own.  One CTA of 512 threads per token row: for each block b,
// hadamard_to_smem (rotate.cuh) computes H_b (signs . x) in fp32 in shared memory
// (butterflies on registers and lane shuffles, one shared-memory pass for the
// highest stages, natural Sylvester order); the block is then scaled by 1/sqrt(b)
// and rounded to the element type.  Every block is read before it is written and
// blocks are disjoint, so x_out may be x.
constexpr int kRhtThreads = 512;

// kOutput: the output-side rotation signs / sqrt(b) * H_b x (GLQ README, "Bit
// widths": the fused linear ends with an output RHT), the transpose of the input
// rotation: the transform first, the signs at the store.  One row of K elements by
// the whole CTA (buf: K floats of shared memory).
template <typename T, bool kOutput>
__device__ __forceinline__ void rotate_row(const uint16_t* __restrict__ xrow, uint16_t* __restrict__ orow,
                                           const int8_t* __restrict__ signs, int K, float* buf) {
  if ((K & (K - 1)) == 0) {  // one block: the whole row, with no offsets
    hadamard_to_smem<T, kRhtThreads, 32768, !kOutput>(xrow, signs, buf, K, threadIdx.x);
    const float scale = block_scale(K);
    for (int i = threadIdx.x; i < K; i += kRhtThreads)
      orow[i] = Elt<T>::from_f32(kOutput ? buf[i] * scale * (float)signs[i] : buf[i] * scale);
    return;
  }
  for (int o = 0, rest = K; rest > 0;) {
    const int b = 1 << (31 - __clz(rest));  // the largest power of two left
    hadamard_to_smem<T, kRhtThreads, 32768, !kOutput>(xrow + o, signs + o, buf + o, b, threadIdx.x);
    const float scale = block_scale(b);
    for (int i = threadIdx.x; i < b; i += kRhtThreads)
      orow[o + i] = Elt<T>::from_f32(kOutput ? buf[o + i] * scale * (float)signs[o + i] : buf[o + i] * scale);
    o += b;
    rest -= b;
  }
}

template <typename T, bool kOutput>
__global__ void __launch_bounds__(kRhtThreads) rht_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ xo,
                                                          const int8_t* __restrict__ signs, int K) {
  extern __shared__ float buf[];
  const int64_t row = blockIdx.x;
  rotate_row<T, kOutput>(x + row * K, xo + row * K, signs, K, buf);
}

// Shard-batched output rotation (GLQ README, "Inference kernels": per-shard output
// transforms of a fused QKV / gate-up projection in one launch over grid.y): CTA
// (row, shard) applies the output rotation to columns [off[s], off[s+1]) of row `row`
// of y [M][N], with signs[off[s] ..].
template <typename T>
__global__ void __launch_bounds__(kRhtThreads) rht_shard_kernel(const uint16_t* __restrict__ y,
                                                                uint16_t* __restrict__ yo,
                                                                const int8_t* __restrict__ signs, int N,
                                                                RhtShards sh) {
  extern __shared__ float buf[];
  const int64_t row = blockIdx.x;
  const int s = blockIdx.y;
  const int o = sh.off[s], w = sh.off[s + 1] - sh.off[s];
  rotate_row<T, true>(y + row * N + o, yo + row * N + o, signs + o, w, buf);
}

template <typename T, bool kOutput>
static cudaError_t launch_rht_t(const void* x, void* x_out, const int8_t* signs, int M, int K, cudaStream_t s) {
  const size_t smem = (size_t)K * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(rht_kernel<T, kOutput>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  rht_kernel<T, kOutput><<<M, kRhtThreads, smem, s>>>((const uint16_t*)x, (uint16_t*)x_out, signs, K);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_rht_shards_t(const void* y, void* y_out, const int8_t* signs, int M, int N,
                                       const RhtShards& sh, cudaStream_t s) {
  int wmax = 0;
  for (int i = 0; i < sh.n; ++i) wmax = sh.off[i + 1] - sh.off[i] > wmax ? sh.off[i + 1] - sh.off[i] : wmax;
  const size_t smem = (size_t)wmax * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(rht_shard_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  rht_shard_kernel<T><<<dim3(M, sh.n), kRhtThreads, smem, s>>>((const uint16_t*)y, (uint16_t*)y_out, signs, N, sh);
  return cudaGetLastError();
}

cudaError_t launch_rht_output_shards(const void* y, void* y_out, const int8_t* signs, int M, int N,
                                     const RhtShards& sh, int dtype, cudaStream_t s) {
  return dtype == VQ_BF16 ? launch_rht_shards_t<__nv_bfloat16>(y, y_out, signs, M, N, sh, s)
                          : launch_rht_shards_t<__half>(y, y_out, signs, M, N, sh, s);
}

cudaError_t launch_rht(const void* x, void* x_out, const int8_t* signs, int M, int K, int dtype, cudaStream_t s) {
  return dtype == VQ_BF16 ? launch_rht_t<__nv_bfloat16, false>(x, x_out, signs, M, K, s)
                          : launch_rht_t<__half, false>(x, x_out, signs, M, K, s);
}

cudaError_t launch_rht_output(const void* y, void* y_out, const int8_t* signs, int M, int N, int dtype,
                              cudaStream_t s) {
  return dtype == VQ_BF16 ? launch_rht_t<__nv_bfloat16, true>(y, y_out, signs, M, N, s)
                          : launch_rht_t<__half, true>(y, y_out, signs, M, N, s);
}

// ------------------------------------------------------------------ debug exports

__device__ __forceinline__ void unpack_one(const LayerArgs& a, int n, int g, uint32_t* i1, uint32_t* i2) {
  const int G = a.K / 8;
  const int64_t e = slice_entry(n, g, a.N, G);  // even for even g (slice widths are even)
  if (a.fmt == kFmtVq16 || a.fmt == kFmtVq16Rvq) {  // the primary stage's plane
    *i1 = a.idx16[e];
    *i2 = 0;
    return;
  }
  const uint32_t hb = a.hi4[e >> 1];
  *i1 = a.lo[e] | (((g & 1) ? (hb >> 4) : (hb & 15u)) << 8);
  if (a.fmt == kFmtRvq12_4) {
    const uint32_t sb = a.s2[e >> 1];
    *i2 = (g & 1) ? (sb >> 4) : (sb & 15u);
  } else {
    *i2 = 0;
  }
}

__global__ void debug_unpack_kernel(LayerArgs a, uint16_t* __restrict__ i1o, uint8_t* __restrict__ i2o) {
  const int G = a.K / 8;
  const int64_t total = (int64_t)a.N * G;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    uint32_t i1, i2;
    unpack_one(a, (int)(t / G), (int)(t % G), &i1, &i2);
    i1o[t] = (uint16_t)i1;
    if (i2o) i2o[t] = (uint8_t)i2;
  }
}

template <typename W>
__global__ void debug_dequant_kernel(LayerArgs a, uint16_t* __restrict__ w) {
  const int G = a.K / 8;
  const int64_t total = (int64_t)a.N * G;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(t / G), g = (int)(t % G);
    uint32_t i1, i2;
    unpack_one(a, n, g, &i1, &i2);
    const float s = f16_bits_to_f32(a.scales[scale_index(n, 8 * g, a.N, a.K, a.scale_group)]);
    const uint4 c1 = reinterpret_cast<const uint4*>(a.cb1)[i1];
    uint32_t out[4];
    if (a.fmt == kFmtVq16Rvq) {  // the residual ladder, stage by stage (ladder.cuh)
      const int64_t e = slice_entry(n, g, a.N, G), NG = (int64_t)a.N * G;
      float v[8];
      const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
      for (int p = 0; p < 4; ++p) {
        const float2 f = f16x2_to_f32x2(w1[p]);
        v[2 * p] = f.x;
        v[2 * p + 1] = f.y;
      }
      for (int t = 2; t <= a.n16; ++t) {
        const uint16_t* cb = t == 2 ? a.cbr[0] : (t == 3 ? a.cbr[1] : a.cbr[2]);
        const float m = t == 2 ? a.mult[0] : (t == 3 ? a.mult[1] : a.mult[2]);
        fma_codeword(m, reinterpret_cast<const uint4*>(cb)[a.idx16[(int64_t)(t - 1) * NG + e]], v);
      }
      if (a.n8) {
        const int t = a.n16 + 1;
        const float m = t == 2 ? a.mult[0] : (t == 3 ? a.mult[1] : a.mult[2]);
        fma_codeword(m, reinterpret_cast<const uint4*>(a.cb8)[a.idx8[e]], v);
      }
      pack_scaled<W>(v, s, out);
    } else if (a.corr_rows) {
      // With the sparse correction: the same fp32 weights, then fl32(p + C) for the
      // corrected ones (the row's entries are in increasing column order).
      const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
      uint4 c2 = c1;
      if (a.fmt == kFmtRvq12_4) c2 = reinterpret_cast<const uint4*>(a.cb2)[i2];
      const uint32_t w2[4] = {c2.x, c2.y, c2.z, c2.w};
      float p[8];
      for (int q = 0; q < 4; ++q) {
        float2 c = f16x2_to_f32x2(w1[q]);
        if (a.fmt == kFmtRvq12_4) {
          const float2 d = f16x2_to_f32x2(w2[q]);
          c.x = __fadd_rn(c.x, d.x);
          c.y = __fadd_rn(c.y, d.y);
        }
        p[2 * q] = __fmul_rn(s, c.x);
        p[2 * q + 1] = __fmul_rn(s, c.y);
      }
      int lo = a.corr_rows[n], hi = a.corr_rows[n + 1];
      while (lo < hi) {  // first entry at column >= 8g
        const int mid = (lo + hi) >> 1;
        if (a.corr_cols[mid] < 8 * g) lo = mid + 1; else hi = mid;
      }
      for (int j = lo; j < a.corr_rows[n + 1] && a.corr_cols[j] < 8 * g + 8; ++j) {
        const int d = a.corr_cols[j] - 8 * g;
        if (d >= 0) p[d] = __fadd_rn(p[d], f16_bits_to_f32(a.corr_vals[j]));  // d < 0 only for unsorted columns
      }
      for (int q = 0; q < 4; ++q) out[q] = Elt<W>::pack(p[2 * q], p[2 * q + 1]);
    } else if (a.fmt == kFmtRvq12_4) {
      const uint4 c2 = reinterpret_cast<const uint4*>(a.cb2)[i2];
      decode_group_packed<W, true>(c1, c2, s, out);
    } else {
      decode_group_packed<W, false>(c1, c1, s, out);
    }
    reinterpret_cast<uint4*>(w)[t] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// The sparse correction's contribution (orka README, "How it works": the decode
// adds a sparse correction): out[m][n] = sum_j x[m][col_j] * val_j over row n's
// entries in order, fp32, one thread per (m, n) (consecutive threads take
// consecutive rows of one token, so the stores coalesce and a row's entries are
// read from L1/L2 by the M threads that share them).  Columns are clamped to
// [0, K), so a malformed column can give a wrong value but never an out-of-range
// read.  It reads x (perhaps written by the previous kernel) and overwrites the
// buffer the previous forward of the handle read, so it waits for the previous
// kernel.
template <typename T>
__global__ void __launch_bounds__(256) corr_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ rows,
                                                   const int32_t* __restrict__ cols,
                                                   const uint16_t* __restrict__ vals, float* __restrict__ out, int M,
                                                   int N, int K) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)M * N) return;
  const int m = (int)(t / N), n = (int)(t - (int64_t)m * N);
  const uint16_t* xm = x + (int64_t)m * K;
  const int j1 = rows[n + 1];
  float acc = 0.f;
  for (int j = rows[n]; j < j1; ++j) {
    const int c = min(max(cols[j], 0), K - 1);
    acc = fmaf(Elt<T>::to_f32(xm[c]), f16_bits_to_f32(vals[j]), acc);
  }
  out[t] = acc;
}

// Test of the bounded waits: one thread waits on an mbarrier that nothing
// arrives on, with the same bounded wait the pipelines use.  It gives up after
// about a second, records kErrTimeout in *err and the kernel ends normally.
__global__ void debug_wait_timeout_kernel(uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    const uint32_t b = smem_u32(&bar);
    ptx::mbar_init(b, 1);
    ptx::fence_barrier_init();
    ptx::mbar_wait(b, 0, err);
  }
}

cudaError_t launch_debug_wait_timeout(uint32_t* err, cudaStream_t s) {
  debug_wait_timeout_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

static int grid_for(int64_t total, int threads) {
  int64_t b = (total + threads - 1) / threads;
  return (int)(b > 65535 ? 65535 : (b < 1 ? 1 : b));
}

cudaError_t launch_debug_unpack(const LayerArgs& a, uint16_t* i1, uint8_t* i2, cudaStream_t s) {
  const int64_t total = (int64_t)a.N * (a.K / 8);
  debug_unpack_kernel<<<grid_for(total, 256), 256, 0, s>>>(a, i1, i2);
  return cudaGetLastError();
}

cudaError_t launch_debug_dequant(const LayerArgs& a, void* w, int wdt, cudaStream_t s) {
  const int64_t total = (int64_t)a.N * (a.K / 8);
  if (wdt == VQ_BF16)
    debug_dequant_kernel<__nv_bfloat16><<<grid_for(total, 256), 256, 0, s>>>(a, (uint16_t*)w);
  else
    debug_dequant_kernel<__half><<<grid_for(total, 256), 256, 0, s>>>(a, (uint16_t*)w);
  return cudaGetLastError();
}

cudaError_t launch_corr(const LayerArgs& a, float* out, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(((int64_t)a.M * a.N + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint16_t* x = static_cast<const uint16_t*>(a.x);
  if (a.act == VQ_BF16)
    return cudaLaunchKernelEx(&cfg, corr_kernel<__nv_bfloat16>, x, a.corr_rows, a.corr_cols, a.corr_vals, out, a.M,
                              a.N, a.K);
  return cudaLaunchKernelEx(&cfg, corr_kernel<__half>, x, a.corr_rows, a.corr_cols, a.corr_vals, out, a.M, a.N, a.K);
}

}  // namespace vq

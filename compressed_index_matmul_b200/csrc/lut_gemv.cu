// Batch-1 GEMV by per-group lookup tables (M == 1, 12-bit formats, K % 128 == 0).
//
// For one token x and one group g of 8 inputs, every weight group of row n
// contributes s * (x_g . cb1[i1] + x_g . cb2[i2]) (orka README, "How it works":
// decode is scale x sum(codebook[index])).  Both dot products depend only on the
// index, so a CTA that owns a K-slice of 16 groups first builds
//   T1[g][i] = x_g . cb1[i]   (16 x 4096 entries, bf16, shared memory)
//   T2[g][e] = x_g . cb2[e]   (16 x 16 entries, fp32, shared memory)
// and then sweeps many rows with one table lookup per group and stage instead of
// gathering and decoding 8-wide codewords.  T1 is a small matrix product
// (16 groups x 8 dims times 8 dims x 4096 codewords) built on the tensor cores
// with mma.sync m16n8k8 (fp16 in, fp32 accumulate).  The codebook operand of
// those MMAs does not depend on x, so each warp loads its share of it into
// registers once and every rebuild is only MMAs and stores.
//
// Work distribution: units are (K-slice s, 256-row chunk c) in slice-major order;
// a persistent grid of one CTA per SM takes a contiguous run of units.  Thread t
// handles row t of every unit; its rows' index bytes stream through a private
// ring of cp.async stages in shared memory, several units ahead, so the loop
// never waits on DRAM latency.  Each unit writes an fp32 partial sum per row.
// When a CTA has finished all its units it takes one ticket per unit; the CTA
// that completes a chunk's last slice sums that chunk's partials in increasing
// slice order (GLQ README, "Inference kernels": fixed-order split-K reduction, no
// floating-point atomics) and writes y.  One launch per forward.
//
// Activations are scaled by a power of two per slice so that every value fits the
// fp16 MMA whatever the activation type; the partial sum is scaled back exactly.
#include "common.cuh"
#include "internal.h"

namespace vq {

constexpr int kLutGroups = 16;                 // groups per K-slice (128 inputs)
constexpr int kLutThreads = 256;               // one row per thread per unit
constexpr int kLutTableBytes = 4096 * 2 + 64;  // one group's T1 (bf16) + pad (bank spread)
constexpr int kLutStages = 6;                  // cp.async ring depth (units in flight)
constexpr int kLutRecord = 48;                 // bytes per thread per stage: lo16 hi8 s2 8 scales4 pad
constexpr int kLutMaxX = 4;                    // x slices preloaded per CTA
constexpr int kLutOffT2 = kLutGroups * kLutTableBytes;
constexpr int kLutOffXh = kLutOffT2 + kLutGroups * 16 * 4;
constexpr int kLutOffXf = kLutOffXh + kLutGroups * 8 * 2;
constexpr int kLutOffRed = kLutOffXf + kLutGroups * 8 * 4;
constexpr int kLutOffList = kLutOffRed + 64;
constexpr int kLutMaxList = 256;
constexpr int kLutOffRing = kLutOffList + 4 * kLutMaxList + 16;
constexpr int kLutSmem = kLutOffRing + kLutStages * kLutThreads * kLutRecord;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void mma_16808_f16(float d[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ float lds_bf16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return __uint_as_float(uint32_t(v) << 16);
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int FMT, typename T>
__global__ void __launch_bounds__(kLutThreads, 1)
    lut_gemv_kernel(LayerArgs a, float* __restrict__ partial, uint32_t* __restrict__ tickets, int S, int C) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  unsigned char* t1 = smem;
  float* t2 = reinterpret_cast<float*>(smem + kLutOffT2);
  uint32_t* xh = reinterpret_cast<uint32_t*>(smem + kLutOffXh);
  float* xf = reinterpret_cast<float*>(smem + kLutOffXf);
  float* red = reinterpret_cast<float*>(smem + kLutOffRed);
  int* list = reinterpret_cast<int*>(smem + kLutOffList);
  int* nlist = reinterpret_cast<int*>(smem + kLutOffRed + 48);
  const uint32_t t1_base = smem_u32(t1), t2_base = smem_u32(t2), ring = smem_u32(smem + kLutOffRing);

  const int N = a.N;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool block_scales = (a.scale_group == 64);
  const int64_t U = (int64_t)S * C;
  const int64_t u0 = U * blockIdx.x / gridDim.x, u1 = U * (blockIdx.x + 1) / gridDim.x;
  const uint16_t* xg = static_cast<const uint16_t*>(a.x);

  // Row records for unit u go to stage (u - u0) % kLutStages of this thread's ring.
  auto issue = [&](int64_t u) {
    const int s = (int)(u / C), r = (int)(u % C) * kLutThreads + tid;
    if (r < N) {
      // K-slice-major planes: this row's 16 groups of slice s are adjacent to the
      // next row's, so the warp's copies are contiguous.
      const uint32_t dst = ring + (((int)((u - u0) % kLutStages)) * kLutThreads + tid) * kLutRecord;
      const int64_t e = (int64_t)16 * s * N + (int64_t)16 * r;
      cp_async16(dst, a.lo + e);
      cp_async8(dst + 16, a.hi4 + e / 2);
      if (kTwo) cp_async8(dst + 24, a.s2 + e / 2);
      if (block_scales) cp_async4(dst + 32, a.scales + e / 8);  // 2 scales per row per slice
    }
  };
  for (int i = 0; i < kLutStages - 1; ++i) {
    if (u0 + i < u1) issue(u0 + i);
    cp_async_commit();
  }

  // Codebook operand of the table MMAs, held for the whole kernel: warp w covers
  // codewords 512w .. 512w+511 in 16 blocks of 32; see the build below.
  const int g = lane >> 2, c = lane & 3;
  uint32_t bfrag[16][4];
  {
    const uint32_t* cbw = reinterpret_cast<const uint32_t*>(a.cb1);
#pragma unroll
    for (int it = 0; it < 16; ++it)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        bfrag[it][j] = __ldg(cbw + (size_t)(warp * 512 + it * 32 + 8 * (g >> 1) + 2 * j + (g & 1)) * 4 + c);
  }
  float c2v[8];
  if (kTwo) {
    const uint4 q = reinterpret_cast<const uint4*>(a.cb2)[tid & 15];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float2 v = f16x2_to_f32x2(w[p]);
      c2v[2 * p] = v.x;
      c2v[2 * p + 1] = v.y;
    }
  }
  // Everything above reads only the layer's constant inputs; x, y and the scratch
  // are touched only after the previous kernel in the stream has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // x of the first kLutMaxX slices this CTA touches.
  const int s_first = (int)(u0 / C);
  float xpre[kLutMaxX];
#pragma unroll
  for (int i = 0; i < kLutMaxX; ++i) {
    const int s = s_first + i;
    xpre[i] = (tid < 128 && s < S) ? Elt<T>::to_f32(xg[(int64_t)s * 128 + tid]) : 0.f;
  }

  int cur = -1;
  float inv_xscale = 1.f;
  for (int64_t u = u0; u < u1; ++u) {
    const int s = (int)(u / C), ch = (int)(u % C);
    if (u + kLutStages - 1 < u1) issue(u + kLutStages - 1);
    cp_async_commit();
    if (s != cur) {
      // ------------------------------------------------------------ build
      __syncthreads();  // everyone is done with the previous tables
      float xv = 0.f;
      if (tid < 128) {
        const int i = s - s_first;
        if (i < kLutMaxX) {
#pragma unroll
          for (int k = 0; k < kLutMaxX; ++k)
            if (k == i) xv = xpre[k];
        } else {
          xv = Elt<T>::to_f32(xg[(int64_t)s * 128 + tid]);
        }
      }
      float m = fabsf(xv);
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[warp] = m;
      __syncthreads();
      m = red[0];
#pragma unroll
      for (int w = 1; w < kLutThreads / 32; ++w) m = fmaxf(m, red[w]);
      int e = 0;
      if (m > 0.f && isfinite(m)) {
        frexpf(m, &e);  // m in [2^(e-1), 2^e): scale the slice's max into [2^14, 2^15)
        e = min(100, max(-100, 15 - e));
      }
      const float xs = ldexpf(1.f, e);
      inv_xscale = ldexpf(1.f, -e);
      if (tid < 128) {
        xf[tid] = xv * xs;
        reinterpret_cast<__half*>(xh)[tid] = __float2half_rn(xv * xs);
      }
      __syncthreads();
      if (kTwo) {
        const int gg = tid >> 4;
        float acc = 0.f;
#pragma unroll
        for (int d = 0; d < 8; ++d) acc = fmaf(xf[8 * gg + d], c2v[d], acc);
        t2[tid] = acc;  // T2[gg][tid & 15]
      }
      {
        // A = x slice (16 groups x 8 dims, fp16).  Column n of MMA j in block `it`
        // is codeword base + 8*(n/2) + 2j + (n%2), so lane (g, c) ends with
        // codewords base+8c .. base+8c+7 of groups g and g+8: one 16-byte store each.
        const uint32_t a0 = xh[g * 4 + c], a1 = xh[(g + 8) * 4 + c];
#pragma unroll
        for (int it = 0; it < 16; ++it) {
          const int base = warp * 512 + it * 32;
          float d[4][4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.f;
            mma_16808_f16(d[j], a0, a1, bfrag[it][j]);
          }
          typedef Elt<__nv_bfloat16> B16;
          const uint4 lo = make_uint4(B16::pack(d[0][0], d[0][1]), B16::pack(d[1][0], d[1][1]),
                                      B16::pack(d[2][0], d[2][1]), B16::pack(d[3][0], d[3][1]));
          const uint4 hi = make_uint4(B16::pack(d[0][2], d[0][3]), B16::pack(d[1][2], d[1][3]),
                                      B16::pack(d[2][2], d[2][3]), B16::pack(d[3][2], d[3][3]));
          *reinterpret_cast<uint4*>(t1 + g * kLutTableBytes + (base + 8 * c) * 2) = lo;
          *reinterpret_cast<uint4*>(t1 + (g + 8) * kLutTableBytes + (base + 8 * c) * 2) = hi;
        }
      }
      __syncthreads();
      cur = s;
    }

    // -------------------------------------------------------------- lookups
    cp_async_wait<kLutStages - 1>();  // this thread's records for unit u have landed
    const int r = ch * kLutThreads + tid;
    if (r < N) {
      const uint32_t rec = ring + (((int)((u - u0) % kLutStages)) * kLutThreads + tid) * kLutRecord;
      uint4 lo4, hs;
      uint32_t scw = 0;
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(lo4.x), "=r"(lo4.y), "=r"(lo4.z), "=r"(lo4.w)
                   : "r"(rec));
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(hs.x), "=r"(hs.y), "=r"(hs.z), "=r"(hs.w)
                   : "r"(rec + 16));
      if (block_scales) asm volatile("ld.shared.u32 %0, [%1];" : "=r"(scw) : "r"(rec + 32));
      const uint32_t low[4] = {lo4.x, lo4.y, lo4.z, lo4.w};
      const uint32_t hiw[2] = {hs.x, hs.y};
      const uint32_t s2w[2] = {hs.z, hs.w};
      float blk[2] = {0.f, 0.f};
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const uint32_t hE = hiw[w] & 0x0F0F0F0Fu, hO = (hiw[w] >> 4) & 0x0F0F0F0Fu;
        const uint32_t sE = (s2w[w] & 0x0F0F0F0Fu) << 2, sO = ((s2w[w] >> 4) & 0x0F0F0F0Fu) << 2;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int t = 8 * w + q;  // group within the slice
          const uint32_t hsel = 4 + (q >> 1);
          // bytes: lo byte t, hi nibble t, then two zero bytes (sign copies of a nibble byte)
          const uint32_t sel = (uint32_t)(t & 3) | (hsel << 4) | ((8u | hsel) << 8) | ((8u | hsel) << 12);
          const uint32_t i1 = prmt(low[t >> 2], (q & 1) ? hO : hE, sel);
          float v = lds_bf16(t1_base + t * kLutTableBytes + i1 * 2);
          if (kTwo) {
            const uint32_t b = q >> 1;
            const uint32_t bsel = b | ((8u | b) << 4) | ((8u | b) << 8) | ((8u | b) << 12);
            v += lds_f32(t2_base + t * 64 + prmt((q & 1) ? sO : sE, 0, bsel));
          }
          blk[w] += v;
        }
      }
      float acc;
      if (block_scales) {
        const float2 sc = f16x2_to_f32x2(scw);
        acc = fmaf(blk[1], sc.y, blk[0] * sc.x);
      } else {
        acc = blk[0] + blk[1];  // the per-row scale is applied once, at the reduction
      }
      acc *= inv_xscale;
      if (S == 1) {
        if (!block_scales) acc *= f16_bits_to_f32(a.scales[r]);
        static_cast<uint16_t*>(a.y)[r] = Elt<T>::from_f32(acc);
      } else {
        partial[(int64_t)s * N + r] = acc;
      }
    }
  }
  cp_async_wait<0>();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (S == 1) return;

  // ------------------------------------------------------ fixed-order reduce
  // One ticket per unit, all taken at once (thread i takes unit u0 + i).
  __threadfence();
  if (tid == 0) *nlist = 0;
  __syncthreads();
  if (tid < u1 - u0) {
    const int ch = (int)((u0 + tid) % C);
    if (atomicAdd(&tickets[ch], 1u) == (uint32_t)(S - 1)) list[atomicAdd(nlist, 1)] = ch;
  }
  __syncthreads();
  const int n = *nlist;
  if (n == 0) return;
  __threadfence();
  // Rows of the completed chunks; every split's partial of a row is loaded before
  // the sum, which then runs in increasing split order.
  constexpr int kBatch = 16;
  for (int i = tid; i < n * kLutThreads; i += kLutThreads) {
    const int ch = list[i / kLutThreads];
    const int r = ch * kLutThreads + i % kLutThreads;
    if (r >= N) continue;
    float sum = 0.f;
    for (int k0 = 0; k0 < S; k0 += kBatch) {
      float v[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) v[j] = (k0 + j < S) ? __ldcg(partial + (int64_t)(k0 + j) * N + r) : 0.f;
#pragma unroll
      for (int j = 0; j < kBatch; ++j)
        if (k0 + j < S) sum += v[j];
    }
    if (!block_scales) sum *= f16_bits_to_f32(a.scales[r]);
    static_cast<uint16_t*>(a.y)[r] = Elt<T>::from_f32(sum);
  }
  __syncthreads();
  if (tid < n) tickets[list[tid]] = 0u;  // ready for the next forward
}

struct LutGeom {
  int S, C, grid;
};

static LutGeom lut_geom(int N, int K, int num_sms) {
  LutGeom g;
  g.S = K / (8 * kLutGroups);
  g.C = (N + kLutThreads - 1) / kLutThreads;
  const int64_t U = (int64_t)g.S * g.C;
  g.grid = (int)(U < num_sms ? U : num_sms);
  return g;
}

bool plan_lut(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  if (M != 1 || d.fmt == VQ_FMT_VQ16 || d.K % (8 * kLutGroups) != 0 || dev.smem_optin < kLutSmem) return false;
  const LutGeom g = lut_geom(d.N, d.K, dev.num_sms);
  // Every CTA's units fit its completion list (units per CTA <= kLutMaxList).
  if (((int64_t)g.S * g.C + g.grid - 1) / g.grid > kLutMaxList) return false;
  p->path = VQ_PATH_LUT;
  p->splits = g.S;
  p->k_per_split = kLutGroups * 8;
  p->launches = 1;
  p->scratch_bytes = g.S > 1 ? (size_t)g.S * d.N * sizeof(float) : 0;
  p->tickets = g.S > 1 ? g.C : 0;
  return true;
}

template <int FMT, typename T>
static cudaError_t launch_lut_t(const LayerArgs& a, float* scratch, uint32_t* tickets, cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const LutGeom g = lut_geom(a.N, a.K, sms);
  auto kern = lut_gemv_kernel<FMT, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.grid);
  cfg.blockDim = dim3(kLutThreads);
  cfg.dynamicSmemBytes = kLutSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, g.S > 1 ? scratch : nullptr, g.S > 1 ? tickets : nullptr, g.S, g.C);
}

cudaError_t launch_lut(const LayerArgs& a, const Plan&, float* scratch, uint32_t* tickets, cudaStream_t s) {
  if (a.fmt == kFmtRvq12_4)
    return a.act == VQ_BF16 ? launch_lut_t<kFmtRvq12_4, __nv_bfloat16>(a, scratch, tickets, s)
                            : launch_lut_t<kFmtRvq12_4, __half>(a, scratch, tickets, s);
  return a.act == VQ_BF16 ? launch_lut_t<kFmtRvq12, __nv_bfloat16>(a, scratch, tickets, s)
                          : launch_lut_t<kFmtRvq12, __half>(a, scratch, tickets, s);
}

}  // namespace vq

// Batch-1 GEMV by per-group lookup tables (M == 1, 12-bit formats).
//
// For one token x and one group g of 8 inputs, every weight group of row n
// contributes s * (x_g . cb1[i1] + x_g . cb2[i2]) (orka README, "How it works":
// decode is scale x sum(codebook[index])).  Both dot products depend only on the
// index, so a CTA that owns a K-slice of 16 groups first builds
//   T1[g][i] = x_g . cb1[i]   (16 x 4096 entries, bf16, shared memory)
//   T2[g][e] = x_g . cb2[e]   (16 x 16 entries, fp32, shared memory)
// and then sweeps many rows with one table lookup per group and stage instead of
// gathering and decoding 8-wide codewords.  T1 is a small matrix product
// (16 groups x 8 dims times 8 dims x 4096 codewords) and is built on the tensor
// cores with mma.sync m16n8k8 (fp16 in, fp32 accumulate).
//
// Work distribution: units are (K-slice s, 256-row chunk c) in slice-major order;
// a persistent grid of one CTA per SM takes a contiguous run of units, rebuilding
// the tables only when its slice changes.  Each unit writes fp32 partial sums
// partial[s][rows]; the CTA that completes a chunk last (an atomic ticket per
// chunk) sums the chunk's partials in increasing s and writes y, so the result
// is independent of scheduling (GLQ README, "Inference kernels": fixed-order
// split-K reduction, no floating-point atomics).  One launch per forward.
//
// bf16 activations are scaled by a power of two per slice before they enter the
// fp16 MMA (so any bf16 magnitude fits), and the partial sum is scaled back; the
// scaling is exact.
#include "common.cuh"
#include "internal.h"

namespace vq {

constexpr int kLutGroups = 16;                    // groups per K-slice (128 inputs)
constexpr int kLutThreads = 256;                  // one row per thread per unit
constexpr int kLutTableBytes = 4096 * 2 + 64;     // one group's T1 (bf16) + pad (bank spread)
constexpr int kLutSmem = kLutGroups * kLutTableBytes + kLutGroups * 16 * 4 + kLutGroups * 8 * 2 +
                         kLutGroups * 8 * 4 + 64;

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

template <int FMT, typename T>
__global__ void __launch_bounds__(kLutThreads, 1)
    lut_gemv_kernel(LayerArgs a, float* __restrict__ partial, uint32_t* __restrict__ tickets, int S, int C) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  unsigned char* t1 = smem;                                                   // [16][kLutTableBytes]
  float* t2 = reinterpret_cast<float*>(smem + kLutGroups * kLutTableBytes);   // [16][16]
  uint32_t* xh = reinterpret_cast<uint32_t*>(t2 + kLutGroups * 16);           // [16][4] half2 (MMA A)
  float* xf = reinterpret_cast<float*>(xh + kLutGroups * 4);                  // [16][8]
  float* red = xf + kLutGroups * 8;                                           // misc scalars
  int* flag = reinterpret_cast<int*>(red + 8);

  const int K = a.K, G = K / 8, N = a.N;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t U = (int64_t)S * C;
  const int64_t u0 = U * blockIdx.x / gridDim.x, u1 = U * (blockIdx.x + 1) / gridDim.x;
  const uint16_t* xg = static_cast<const uint16_t*>(a.x);
  const uint32_t t1_base = smem_u32(t1), t2_base = smem_u32(t2);
  const int nblk = K / a.scale_group;

  int cur = -1;
  float inv_xscale = 1.f;
  for (int64_t u = u0; u < u1; ++u) {
    const int s = (int)(u / C), ch = (int)(u % C);
    const int gs = s * kLutGroups;
    const int gc = min(kLutGroups, G - gs);  // 16, or 8 for a ragged last slice
    if (s != cur) {
      // ------------------------------------------------------------ build
      __syncthreads();  // everyone is done reading the previous tables
      float xv = 0.f;
      if (tid < 8 * gc) xv = Elt<T>::to_f32(xg[8 * gs + tid]);
      // Power-of-two scale so the slice's largest |x| lands in [2^14, 2^15): every
      // value then fits fp16 for the MMA, whatever the activation type.
      float xs;
      {
        float m = fabsf(xv);
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[warp] = m;
        __syncthreads();
        m = red[0];
#pragma unroll
        for (int w = 1; w < kLutThreads / 32; ++w) m = fmaxf(m, red[w]);
        int e = 0;
        if (m > 0.f && isfinite(m)) {
          frexpf(m, &e);  // m in [2^(e-1), 2^e)
          e = min(100, max(-100, 15 - e));
        }
        xs = ldexpf(1.f, e);
        inv_xscale = ldexpf(1.f, -e);
      }
      const float xsv = xv * xs;
      if (tid < kLutGroups * 8) {
        xf[tid] = xsv;  // zeros past gc groups
        reinterpret_cast<__half*>(xh)[tid] = __float2half_rn(xsv);
      }
      __syncthreads();
      if (kTwo) {
        const int g = tid >> 4, e = tid & 15;
        const uint4 c2 = reinterpret_cast<const uint4*>(a.cb2)[e];
        const uint32_t w[4] = {c2.x, c2.y, c2.z, c2.w};
        float acc = 0.f;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 v = f16x2_to_f32x2(w[p]);
          acc = fmaf(xf[8 * g + 2 * p], v.x, acc);
          acc = fmaf(xf[8 * g + 2 * p + 1], v.y, acc);
        }
        t2[g * 16 + e] = acc;
      }
      {
        // T1 on the tensor cores.  A = x slice (16 groups x 8 dims), B = 8 codewords
        // x 8 dims.  Four MMAs cover 32 codewords with column n of MMA j mapped to
        // codeword base + 8*(n/2) + 2j + (n%2), so lane (g, c) ends up holding
        // codewords base+8c .. base+8c+7 of groups g and g+8: one 16-byte store each.
        const int g = lane >> 2, c = lane & 3;
        const uint32_t a0 = xh[g * 4 + c], a1 = xh[(g + 8) * 4 + c];
        const uint32_t* cbw = reinterpret_cast<const uint32_t*>(a.cb1);
        for (int base = warp * 512; base < warp * 512 + 512; base += 32) {
          float d[4][4];
          uint32_t b[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) b[j] = __ldg(cbw + (size_t)(base + 8 * (g >> 1) + 2 * j + (g & 1)) * 4 + c);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.f;
            mma_16808_f16(d[j], a0, a1, b[j]);
          }
          const uint4 lo = make_uint4(Elt<__nv_bfloat16>::pack(d[0][0], d[0][1]), Elt<__nv_bfloat16>::pack(d[1][0], d[1][1]),
                                      Elt<__nv_bfloat16>::pack(d[2][0], d[2][1]), Elt<__nv_bfloat16>::pack(d[3][0], d[3][1]));
          const uint4 hi = make_uint4(Elt<__nv_bfloat16>::pack(d[0][2], d[0][3]), Elt<__nv_bfloat16>::pack(d[1][2], d[1][3]),
                                      Elt<__nv_bfloat16>::pack(d[2][2], d[2][3]), Elt<__nv_bfloat16>::pack(d[3][2], d[3][3]));
          *reinterpret_cast<uint4*>(t1 + g * kLutTableBytes + (base + 8 * c) * 2) = lo;
          if (g + 8 < gc) *reinterpret_cast<uint4*>(t1 + (g + 8) * kLutTableBytes + (base + 8 * c) * 2) = hi;
        }
      }
      __syncthreads();
      cur = s;
    }

    // -------------------------------------------------------------- lookups
    const int r = ch * kLutThreads + tid;
    float acc = 0.f;
    if (r < N) {
      const int64_t rowoff = (int64_t)r * G + gs;
      uint32_t low[4], hiw[2], s2w[2] = {0, 0};
      if (gc == kLutGroups && (G % 16) == 0) {
        const uint4 l = *reinterpret_cast<const uint4*>(a.lo + rowoff);
        low[0] = l.x; low[1] = l.y; low[2] = l.z; low[3] = l.w;
        const uint2 h = *reinterpret_cast<const uint2*>(a.hi4 + rowoff / 2);
        hiw[0] = h.x; hiw[1] = h.y;
        if (kTwo) {
          const uint2 q = *reinterpret_cast<const uint2*>(a.s2 + rowoff / 2);
          s2w[0] = q.x; s2w[1] = q.y;
        }
      } else {
        // 8-byte aligned rows (G % 8 == 0): two halves, the second only for full slices
        const uint2 l0 = *reinterpret_cast<const uint2*>(a.lo + rowoff);
        low[0] = l0.x; low[1] = l0.y;
        hiw[0] = *reinterpret_cast<const uint32_t*>(a.hi4 + rowoff / 2);
        if (kTwo) s2w[0] = *reinterpret_cast<const uint32_t*>(a.s2 + rowoff / 2);
        if (gc == kLutGroups) {
          const uint2 l1 = *reinterpret_cast<const uint2*>(a.lo + rowoff + 8);
          low[2] = l1.x; low[3] = l1.y;
          hiw[1] = *reinterpret_cast<const uint32_t*>(a.hi4 + rowoff / 2 + 4);
          if (kTwo) s2w[1] = *reinterpret_cast<const uint32_t*>(a.s2 + rowoff / 2 + 4);
        } else {
          low[2] = low[3] = 0; hiw[1] = 0; s2w[1] = 0;
        }
      }
      float blk[2] = {0.f, 0.f};
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        if (w == 1 && gc < kLutGroups) break;
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
            const uint32_t bsel = (q >> 1) | (8u | (q >> 1)) << 4 | (8u | (q >> 1)) << 8 | (8u | (q >> 1)) << 12;
            const uint32_t e4 = prmt((q & 1) ? sO : sE, 0, bsel);
            v += lds_f32(t2_base + t * 64 + e4);
          }
          blk[w] += v;
        }
      }
      if (a.scale_group == 64) {
        const int b0 = 2 * s;
        acc = blk[0] * f16_bits_to_f32(a.scales[(int64_t)r * nblk + b0]);
        if (gc == kLutGroups) acc = fmaf(blk[1], f16_bits_to_f32(a.scales[(int64_t)r * nblk + b0 + 1]), acc);
      } else {
        acc = (blk[0] + blk[1]) * f16_bits_to_f32(a.scales[r]);
      }
      acc *= inv_xscale;
    }

    // --------------------------------------------------- fixed-order reduce
    if (S == 1) {
      if (r < N) static_cast<uint16_t*>(a.y)[r] = Elt<T>::from_f32(acc);
      continue;
    }
    if (r < N) partial[(int64_t)s * N + r] = acc;
    __threadfence();
    __syncthreads();
    if (tid == 0) *flag = (atomicAdd(&tickets[ch], 1u) == (uint32_t)(S - 1));
    __syncthreads();
    if (*flag) {
      __threadfence();
      if (r < N) {
        float sum = 0.f;
        for (int k = 0; k < S; ++k) sum += __ldcg(partial + (int64_t)k * N + r);
        static_cast<uint16_t*>(a.y)[r] = Elt<T>::from_f32(sum);
      }
      if (tid == 0) tickets[ch] = 0u;  // ready for the next forward
    }
  }
}

struct LutGeom {
  int S, C, grid;
};

static LutGeom lut_geom(int N, int K, int num_sms) {
  LutGeom g;
  const int G = K / 8;
  g.S = (G + kLutGroups - 1) / kLutGroups;
  g.C = (N + kLutThreads - 1) / kLutThreads;
  const int64_t U = (int64_t)g.S * g.C;
  g.grid = (int)(U < num_sms ? U : num_sms);
  return g;
}

bool plan_lut(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  if (M != 1 || d.fmt == VQ_FMT_VQ16 || dev.smem_optin < kLutSmem) return false;
  const LutGeom g = lut_geom(d.N, d.K, dev.num_sms);
  p->path = VQ_PATH_LUT;
  p->splits = g.S;
  p->k_per_split = kLutGroups * 8;
  p->launches = 1;
  p->scratch_bytes = g.S > 1 ? (size_t)g.S * d.N * sizeof(float) : 0;
  p->tickets = g.S > 1 ? g.C : 0;
  return true;
}

template <int FMT, typename T>
static cudaError_t launch_lut_t(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets_buf,
                                cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const LutGeom g = lut_geom(a.N, a.K, sms);
  cudaError_t e = cudaFuncSetAttribute(lut_gemv_kernel<FMT, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmem);
  if (e != cudaSuccess) return e;
  float* partial = g.S > 1 ? scratch : nullptr;
  uint32_t* tickets = g.S > 1 ? tickets_buf : nullptr;
  lut_gemv_kernel<FMT, T><<<g.grid, kLutThreads, kLutSmem, s>>>(a, partial, tickets, g.S, g.C);
  return cudaGetLastError();
}

cudaError_t launch_lut(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets, cudaStream_t s) {
  if (a.fmt == kFmtRvq12_4)
    return a.act == VQ_BF16 ? launch_lut_t<kFmtRvq12_4, __nv_bfloat16>(a, p, scratch, tickets, s)
                            : launch_lut_t<kFmtRvq12_4, __half>(a, p, scratch, tickets, s);
  return a.act == VQ_BF16 ? launch_lut_t<kFmtRvq12, __nv_bfloat16>(a, p, scratch, tickets, s)
                          : launch_lut_t<kFmtRvq12, __half>(a, p, scratch, tickets, s);
}

}  // namespace vq

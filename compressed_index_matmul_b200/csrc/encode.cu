// Nearest-entry encoder: a dense W into the index planes the forward kernels read
// (orka README, "How it works": "encode -> nearest-entry index per group", stored as
// 12-bit bit-planes; the two-stage format adds the entry nearest to the residual
// that stage 1 leaves; GLQ README, "How it works": one 16-bit index per group).
//
// For group g of row n with scale s, stage 1 takes
//   i1 = argmin_i d(w, s, cb1[i]),  d = ((e_0^2 + e_1^2) + ...) + e_7^2,  e_j = w_j - s c_j,
// every product, difference and sum rounded to binary32 in that order (explicit
// round-to-nearest intrinsics, so nothing is contracted into a fused multiply-add);
// equal distances keep the smaller index.  Stage 2 of VQ_FMT_RVQ12_4 takes the
// entry t minimising d(w, s, cb1[i1] + cb2[t]) with the codeword sum rounded to
// binary32.
//
// Work split: one thread per pair of adjacent groups of a row (the pair shares one
// byte of each packed 4-bit plane, so every byte has one writer).  The 4096-entry
// codebook is staged in shared memory as fp32 (128 KiB) by every CTA; all lanes of a
// warp read the same entry at the same time (broadcast).  The 65,536-entry table of
// the 16-bit format is read through L1/L2.  Bound: the distance arithmetic, about
// 32 binary32 operations per group and entry; an encoder runs once per layer, off
// the forward path.
#include "common.cuh"
#include "internal.h"
#include "tools.h"

namespace vq {

constexpr int kEncThreads = 256;

__device__ __forceinline__ float dist8(const float (&w)[8], float s, const float (&c)[8]) {
  float d = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float e = __fsub_rn(w[j], __fmul_rn(s, c[j]));
    d = __fadd_rn(d, __fmul_rn(e, e));
  }
  return d;
}

__device__ __forceinline__ void load_f16x8(const uint4& q, float (&c)[8]) {
  const uint32_t h[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 f = f16x2_to_f32x2(h[p]);
    c[2 * p] = f.x;
    c[2 * p + 1] = f.y;
  }
}

template <int FMT>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(const float* __restrict__ w, const uint16_t* __restrict__ scales,
                                                             int scale_group, const uint16_t* __restrict__ cb1,
                                                             const uint16_t* __restrict__ cb2, int N, int K,
                                                             uint8_t* __restrict__ lo, uint8_t* __restrict__ hi4,
                                                             uint8_t* __restrict__ s2, uint16_t* __restrict__ idx16) {
  constexpr bool k16 = (FMT == kFmtVq16);
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  extern __shared__ __align__(16) float cbs[];  // [4096][8] fp32, then [16][8] for stage 2
  if (!k16) {
    for (int i = threadIdx.x; i < 4096 * 8; i += kEncThreads) cbs[i] = f16_bits_to_f32(cb1[i]);
    if (kTwo)
      for (int i = threadIdx.x; i < 16 * 8; i += kEncThreads) cbs[4096 * 8 + i] = f16_bits_to_f32(cb2[i]);
    __syncthreads();
  }
  const int G = K / 8, P = G / 2;
  const int64_t t = (int64_t)blockIdx.x * kEncThreads + threadIdx.x;
  if (t >= (int64_t)N * P) return;
  const int n = (int)(t / P), g0 = 2 * (int)(t % P);

  float wv[2][8], s[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float4* src = reinterpret_cast<const float4*>(w + (int64_t)n * K + 8 * (g0 + q));
    const float4 a = src[0], b = src[1];
    wv[q][0] = a.x; wv[q][1] = a.y; wv[q][2] = a.z; wv[q][3] = a.w;
    wv[q][4] = b.x; wv[q][5] = b.y; wv[q][6] = b.z; wv[q][7] = b.w;
    s[q] = f16_bits_to_f32(scales[scale_index(n, 8 * (g0 + q), N, K, scale_group)]);
  }

  const int entries = k16 ? 65536 : 4096;
  float best[2] = {INFINITY, INFINITY};
  int bi[2] = {0, 0};
  for (int i = 0; i < entries; ++i) {
    float c[8];
    if (k16) {
      load_f16x8(__ldg(reinterpret_cast<const uint4*>(cb1) + i), c);
    } else {
      const float4* cv = reinterpret_cast<const float4*>(cbs + 8 * i);
      const float4 a = cv[0], b = cv[1];
      c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w;
      c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float d = dist8(wv[q], s[q], c);
      if (d < best[q]) {
        best[q] = d;
        bi[q] = i;
      }
    }
  }

  const int64_t e = slice_entry(n, g0, N, G);  // even; group g0 + 1 is entry e + 1
  if (k16) {
    idx16[e] = (uint16_t)bi[0];
    idx16[e + 1] = (uint16_t)bi[1];
    return;
  }
  lo[e] = (uint8_t)(bi[0] & 0xFF);
  lo[e + 1] = (uint8_t)(bi[1] & 0xFF);
  hi4[e / 2] = (uint8_t)(((bi[0] >> 8) & 15) | (((bi[1] >> 8) & 15) << 4));
  if (kTwo) {
    int b2[2] = {0, 0};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float* base = cbs + 8 * bi[q];
      float bst = INFINITY;
      for (int j2 = 0; j2 < 16; ++j2) {
        float c[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = __fadd_rn(base[j], cbs[4096 * 8 + 8 * j2 + j]);
        const float d = dist8(wv[q], s[q], c);
        if (d < bst) {
          bst = d;
          b2[q] = j2;
        }
      }
    }
    s2[e / 2] = (uint8_t)((b2[0] & 15) | ((b2[1] & 15) << 4));
  }
}

template <int FMT>
static cudaError_t launch_encode_t(const EncodeArgs& a, cudaStream_t s) {
  const size_t smem = FMT == kFmtVq16 ? 0 : (size_t)(4096 * 8 + (FMT == kFmtRvq12_4 ? 16 * 8 : 0)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(encode_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t pairs = (int64_t)a.N * (a.K / 16);
  const int64_t blocks = (pairs + kEncThreads - 1) / kEncThreads;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  encode_kernel<FMT><<<(unsigned)blocks, kEncThreads, smem, s>>>(a.w, a.scales, a.scale_group, a.cb1, a.cb2, a.N, a.K,
                                                                 a.lo, a.hi4, a.s2, a.idx16);
  return cudaGetLastError();
}

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s) {
  switch (a.fmt) {
    case kFmtRvq12: return launch_encode_t<kFmtRvq12>(a, s);
    case kFmtRvq12_4: return launch_encode_t<kFmtRvq12_4>(a, s);
    default: return launch_encode_t<kFmtVq16>(a, s);
  }
}

}  // namespace vq

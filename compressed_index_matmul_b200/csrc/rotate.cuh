// Unnormalised randomized Hadamard rotation of one token, H_K (signs . x), into
// shared memory (fp32), by NT threads of a CTA (named barrier 1).
//
// GLQ README, "How it works": random sign flips followed by a fast Walsh-Hadamard
// transform.  K = 2^p with 64 <= K <= 64 NT.  Every stage is a butterfly
// (u + w, u - w) on one index bit; the stages commute, so the result is
// H_K (signs . x) with H_K[k][j] = (-1)^popcount(k & j) (natural Sylvester
// order) whatever order they run in.  With E = max(1, K / NT) elements per thread
// and R = K / (32 E) (both compile-time, so every stage is straight-line code):
//   pass 1: thread t holds E consecutive elements; the log2(E) lowest stages run
//           on registers, the next five across the warp's lanes with shuffles;
//   pass 2: the log2(R) highest stages run on registers over groups of R
//           elements at stride 32 E.
// With kSignsFirst false the signs are not applied (the output-side rotation
// applies them after the transform).  Used by the rotation kernels (vq_rht_apply,
// vq_rht_apply_output) and by the batch-1 16-bit kernel, which rotates x itself.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace vq {

template <typename T, int E, int R, int NT, bool kSignsFirst>
__device__ __forceinline__ void hadamard_pass(const uint16_t* __restrict__ x, const int8_t* __restrict__ signs,
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
        const uint2 sw = kSignsFirst ? *reinterpret_cast<const uint2*>(signs + tid * E + 8 * c) : make_uint2(0, 0);
        const uint32_t xa[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int8_t sg = (int8_t)(((q < 4 ? sw.x : sw.y) >> (8 * (q & 3))) & 0xFFu);
          const float xv = Elt<T>::to_f32((uint16_t)(xa[q >> 1] >> (16 * (q & 1))));
          v[8 * c + q] = kSignsFirst ? xv * (float)sg : xv;
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e)
        v[e] = kSignsFirst ? Elt<T>::to_f32(x[tid * E + e]) * (float)signs[tid * E + e] : Elt<T>::to_f32(x[tid * E + e]);
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
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
  for (int gb = tid; gb < D; gb += NT) {  // stages h = 32 E .. K/2
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
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// hadamard_pass for a power-of-two K in [64, kMaxK] (NT = 512; kMaxK <= 32768 bounds
// the registers the instantiations need).
template <typename T, int NT, int kMaxK, bool kSignsFirst = true>
__device__ __forceinline__ void hadamard_to_smem(const uint16_t* x, const int8_t* signs, float* xs, int K, int tid) {
  static_assert(NT == 512 && kMaxK >= 16384 && kMaxK <= 32768, "the stage split below assumes 512 threads");
  switch (K) {
    case 64: hadamard_pass<T, 1, 2, NT, kSignsFirst>(x, signs, xs, tid); break;
    case 128: hadamard_pass<T, 1, 4, NT, kSignsFirst>(x, signs, xs, tid); break;
    case 256: hadamard_pass<T, 1, 8, NT, kSignsFirst>(x, signs, xs, tid); break;
    case 512: hadamard_pass<T, 1, 16, NT, kSignsFirst>(x, signs, xs, tid); break;
    case 1024: hadamard_pass<T, 2, 16, NT, kSignsFirst>(x, signs, xs, tid); break;
    case 2048: hadamard_pass<T, 4, 16, NT, kSignsFirst>(x, signs, xs, tid); break;
    case 4096: hadamard_pass<T, 8, 16, NT, kSignsFirst>(x, signs, xs, tid); break;
    case 8192: hadamard_pass<T, 16, 16, NT, kSignsFirst>(x, signs, xs, tid); break;
    default:
      if constexpr (kMaxK >= 32768) {
        if (K == 32768) {
          hadamard_pass<T, 64, 16, NT, kSignsFirst>(x, signs, xs, tid);
          break;
        }
      }
      hadamard_pass<T, 32, 16, NT, kSignsFirst>(x, signs, xs, tid);  // 16384
      break;
  }
}

// The rotation for any K that is a multiple of 64 up to kMaxK (GLQ README, "Bit
// widths": a hidden size that is not a power of two is cut into power-of-two blocks,
// 2688 = 2048 + 512 + 128, each with its own transform).  The blocks are the binary
// expansion of K, largest first along K: each is hadamard_to_smem of its slice of x
// and signs into its slice of xs.  With scale_blocks each block is multiplied in
// place by its orthonormal factor 1/sqrt(b) (where K is not a power of two no single
// factor applies to the whole vector); otherwise the caller applies 1/sqrt(K).
// fl32(1/sqrt(b)) for b = 2^p, built exactly in single precision: 2^-(p/2) for even p,
// 2^-((p-1)/2) times fl32(1/sqrt(2)) = 0x3F3504F3 for odd p (a power-of-two scaling, so
// the product is the correctly rounded value), the same bits as rounding the
// double-precision quotient.
__device__ __forceinline__ float block_scale(int b) {
  const int p = 31 - __clz(b);
  const float base = __int_as_float((127 - (p >> 1)) << 23);
  return (p & 1) ? base * __int_as_float(0x3F3504F3) : base;
}

template <typename T, int NT, int kMaxK, bool kSignsFirst = true>
__device__ __forceinline__ void hadamard_blocks_to_smem(const uint16_t* x, const int8_t* signs, float* xs, int K,
                                                        int tid, bool scale_blocks) {
  for (int o = 0, rest = K; rest > 0;) {
    const int b = 1 << (31 - __clz(rest));  // the largest power of two left
    hadamard_to_smem<T, NT, kMaxK, kSignsFirst>(x + o, signs + o, xs + o, b, tid);
    if (scale_blocks) {
      const float sc = block_scale(b);
      for (int i = tid; i < b; i += NT) xs[o + i] *= sc;
    }
    o += b;
    rest -= b;
  }
  if (scale_blocks) asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

}  // namespace vq

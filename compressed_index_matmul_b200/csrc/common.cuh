// Device helpers shared by the libvqlinear kernels (sm_100a).
//
// Storage format (orka README, "How it works"; GLQ README, "How it works"):
// W is N x K, one codebook index per group of 8 consecutive weights along K,
// G = K/8 groups per row.  The 12-bit stage-1 index of a group is its lo byte |
// its hi nibble << 8 (two groups per hi4 byte, the even group in bits 0..3); the
// 4-bit stage-2 index comes from the s2 plane packed the same way; the 16-bit
// format stores one uint16 per group.  The storage order is below.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace vq {

constexpr int kFmtRvq12 = 1;
constexpr int kFmtRvq12_4 = 2;
constexpr int kFmtVq16 = 3;
constexpr int kFmtVq16Rvq = 4;  // residual ladder: 16-bit stages, then at most one 8-bit stage

// Device error flag bits (written by bounded waits that gave up).
constexpr uint32_t kErrTimeout = 1u;

// Iteration cap for every spin-wait on an mbarrier (each try_wait may suspend
// the thread for a while, so this bounds the wait to well under a second).
constexpr uint32_t kWaitSpinLimit = 1u << 22;

// ------------------------------------------------------------------ storage order
//
// Index planes are K-slice-major: K is cut into slices of 16 groups (128 inputs);
// slice s holds w = min(16, G - 16 s) groups, and row n's entries of slice s
// start at entry 16 s N + n w (entries are bytes of lo, uint16 of idx16; the
// packed 4-bit planes hi4 / s2 use half of every count, two groups per byte with
// the even group in the low nibble).  Consecutive output rows are therefore
// adjacent in memory for every slice, so loads across rows coalesce.
// Block scales (one per 64 inputs) follow the same order with 2 entries per full
// slice; one scale per row is scales[n].

__host__ __device__ __forceinline__ int slice_width(int s, int G) { return (G - 16 * s) < 16 ? (G - 16 * s) : 16; }

// Entry index of group g of row n (lo / idx16; halve it for hi4 / s2).
__device__ __forceinline__ int64_t slice_entry(int n, int g, int N, int G) {
  const int s = g >> 4;
  return (int64_t)16 * s * N + (int64_t)n * slice_width(s, G) + (g & 15);
}

// Index of the scale that covers input k of row n (scale_group is 64 or K).
__device__ __forceinline__ int64_t scale_index(int n, int k, int N, int K, int scale_group) {
  if (scale_group == K) return n;
  const int s = k >> 7;
  return (int64_t)2 * s * N + (int64_t)n * (slice_width(s, K / 8) >> 3) + ((k & 127) >> 6);
}

// ------------------------------------------------------------------ element types

template <typename T> struct Elt;
template <> struct Elt<__half> {
  static __device__ __forceinline__ float to_f32(uint16_t b) { return __half2float(__ushort_as_half(b)); }
  static __device__ __forceinline__ uint16_t from_f32(float v) { return __half_as_ushort(__float2half_rn(v)); }
  // Two floats -> packed pair, round to nearest even; `lo` in bits 0..15.
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};
template <> struct Elt<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
  static __device__ __forceinline__ uint16_t from_f32(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

__device__ __forceinline__ float f16_bits_to_f32(uint32_t b) { return __half2float(__ushort_as_half((uint16_t)b)); }

// Low and high fp16 halves of a 32-bit word, as floats.
__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}

// --------------------------------------------------------------------- decoding

// Eight weights of one group: s * (c1 + c2), with the stage sum and the product
// each rounded to fp32 (the materialised-weight rounding points), returned as
// four packed pairs of T rounded to nearest even.
template <typename T, bool kTwoStage>
__device__ __forceinline__ void decode_group_packed(const uint4& c1, const uint4& c2, float s, uint32_t out[4]) {
  const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
  const uint32_t w2[4] = {c2.x, c2.y, c2.z, c2.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    float2 a = f16x2_to_f32x2(w1[p]);
    if (kTwoStage) {
      float2 b = f16x2_to_f32x2(w2[p]);
      a.x = __fadd_rn(a.x, b.x);
      a.y = __fadd_rn(a.y, b.y);
    }
    out[p] = Elt<T>::pack(__fmul_rn(s, a.x), __fmul_rn(s, a.y));
  }
}

// ------------------------------------------------------------------- warp MMA

// D += A(16x16, row) * B(16x8, col), fp32 accumulate; A/B packed pairs of T.
template <typename T> struct Mma16816;
template <> struct Mma16816<__half> {
  static __device__ __forceinline__ void run(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};
template <> struct Mma16816<__nv_bfloat16> {
  static __device__ __forceinline__ void run(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
};

// ------------------------------------------------------------------ misc PTX

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

}  // namespace vq

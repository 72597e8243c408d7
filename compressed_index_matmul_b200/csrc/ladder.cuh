// Residual ladder of the 16-bit formats (GLQ README, "Bit widths": a 16-bit
// primary stage, then 16-bit residual stages, and for an odd bit width one final
// 8-bit stage; "Direct kernel access": each residual stage has its own codebook and
// an inverse residual scale, here its multiplier).  Group g of row n decodes to
//   s * (cb1[i_1] + sum_t mult[t-2] * cbr[t-2][i_t] + [n8] mult[n16-1] * cb8[i_8]).
// Every plane has the K-slice-major order of idx16; 16-bit stage t's plane starts
// at entry (t - 1) N G of idx16, the 8-bit plane is idx8.
//
// Materialised weights (warp-MMA and tensor-core paths, debug dequant): the stage
// sum v starts at c1 and takes one fused multiply-add per residual stage in stage
// order (fp32, one rounding each), then s * v is rounded to fp32 and to T.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace vq {

// Residual indices of 8 consecutive groups of a row (one 64-input block):
// 16-bit stage t in r[t-2][0..3] (two groups per word), the 8-bit stage in
// r[n16-1][0..1] (four groups per word).
struct LadderIdx {
  uint32_t r[3][4];
};

// e: the block's first entry (a multiple of 8, so the loads are aligned).
__device__ __forceinline__ void load_ladder_block(const LayerArgs& a, int64_t e, LadderIdx& q) {
  const int64_t NG = (int64_t)a.N * (a.K / 8);
#pragma unroll
  for (int t = 2; t <= 4; ++t) {
    q.r[t - 2][0] = q.r[t - 2][1] = q.r[t - 2][2] = q.r[t - 2][3] = 0u;
    if (t <= a.n16) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.idx16 + (int64_t)(t - 1) * NG + e));
      q.r[t - 2][0] = v.x;
      q.r[t - 2][1] = v.y;
      q.r[t - 2][2] = v.z;
      q.r[t - 2][3] = v.w;
    } else if (t == a.n16 + 1 && a.n8) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(a.idx8 + e));
      q.r[t - 2][0] = v.x;
      q.r[t - 2][1] = v.y;
    }
  }
}

// v += mult * c for the eight fp16 halves of c (fused, one rounding each).
__device__ __forceinline__ void fma_codeword(float m, const uint4& c, float (&v)[8]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 f = f16x2_to_f32x2(w[p]);
    v[2 * p] = __fmaf_rn(m, f.x, v[2 * p]);
    v[2 * p + 1] = __fmaf_rn(m, f.y, v[2 * p + 1]);
  }
}

// Stage sum of group g (0..7) of a block whose primary codeword is c1; cb8s is the
// 8-bit codebook staged in shared memory.
__device__ __forceinline__ void ladder_sum(const LayerArgs& a, const LadderIdx& q, int g, const uint4& c1,
                                           const uint4* cb8s, float (&v)[8]) {
  const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 f = f16x2_to_f32x2(w1[p]);
    v[2 * p] = f.x;
    v[2 * p + 1] = f.y;
  }
#pragma unroll
  for (int t = 2; t <= 4; ++t) {
    if (t <= a.n16) {
      const uint32_t i = (q.r[t - 2][g >> 1] >> (16 * (g & 1))) & 0xFFFFu;
      fma_codeword(a.mult[t - 2], __ldg(reinterpret_cast<const uint4*>(a.cbr[t - 2]) + i), v);
    } else if (t == a.n16 + 1 && a.n8) {
      const uint32_t i = (q.r[t - 2][g >> 2] >> (8 * (g & 3))) & 0xFFu;
      fma_codeword(a.mult[t - 2], cb8s[i], v);
    }
  }
}

// Copies the 8-bit codebook (256 entries) into shared memory, thread `tid` of
// `nthreads`; the caller's next CTA barrier makes it visible.
__device__ __forceinline__ void stage_cb8(const LayerArgs& a, uint4* cb8s, int tid, int nthreads) {
  if (!a.n8) return;
  for (int i = tid; i < 256; i += nthreads) cb8s[i] = __ldg(reinterpret_cast<const uint4*>(a.cb8) + i);
}

// Eight materialised weights RN_T(fl32(s * v)) as four packed pairs.
template <typename T>
__device__ __forceinline__ void pack_scaled(const float (&v)[8], float s, uint32_t out[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) out[p] = Elt<T>::pack(__fmul_rn(s, v[2 * p]), __fmul_rn(s, v[2 * p + 1]));
}

}  // namespace vq

// Split-K GEMV for 1 <= M <= 16 tokens: y = x . W^T with W decoded on the fly
// (GLQ README, "Inference kernels": the weight matrix is never materialised; the
// split-K partial sums go to a scratch buffer and are reduced in a fixed order).
//
// Work layout
//   CTA    = 8 warps, 128 output rows x one K-split (k_per_split, multiple of 64)
//   warp   = one 16-row tile of W; loops over its K-split in 64-wide blocks
//   lane   = (g = lane/4, c = lane%4): rows g and g+8 of the tile, groups 2c and
//            2c+1 of the current 64-wide block -> 4 codewords per block
// Each lane decodes its 4 codewords into registers (stage-1 codebook staged in
// shared memory, stage-2 codebook too; the 65,536-entry table is read through
// L2) and feeds them straight into mma.sync m16n8k16 as the A operand (W rows x
// k), with x as the B operand (k x 8 tokens, one or two token tiles).
//
// k permutation: an MMA's reduction order is irrelevant to the result's
// definition, so MMA j of a block uses pair j (elements 2j, 2j+1) of every
// codeword: fragment slot "k-pair c" holds group 2c and slot "k-pair c+4" holds
// group 2c+1.  The matching x elements for lane (g, c) are then
// x[g][16c + 2j .. +1] and x[g][16c + 8 + 2j .. +1], i.e. word j of two 16-byte
// loads -- no shuffles are needed on either operand.
//
// Decoded weights use the materialised-weight rounding (stage sum and scaled
// value rounded to fp32, then to the activation type), so every product the MMA
// forms is of exactly the weights vq_debug_dequant exports.
#include "common.cuh"
#include "internal.h"

namespace vq {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 16 * kGemvWarps;
constexpr int kGemvMaxKc = 1024;  // x slice staged per CTA: 16 tokens x 1024 x 2 B

template <int FMT, typename T, int NT>
__global__ void __launch_bounds__(256) gemv_kernel(LayerArgs a, int k_per_split, float* __restrict__ partial) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr bool kSmemCb = (FMT != kFmtVq16);
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  uint4* cb1s = reinterpret_cast<uint4*>(smem);                               // 4096 entries
  uint4* cb2s = cb1s + (kSmemCb ? 4096 : 0);                                  // 16 entries
  uint16_t* xs = reinterpret_cast<uint16_t*>(cb2s + (kTwo ? 16 : 0));

  const int K = a.K, G = K / 8, M = a.M, N = a.N;
  const int split = blockIdx.y;
  const int k0 = split * k_per_split;
  const int kc = min(k_per_split, K - k0);
  const int xstride = kc + 8;  // elements; +16 B breaks the 8-token bank alignment

  // Stage the codebooks and this split's x slice (zeros for tokens >= M).
  if (kSmemCb) {
    const uint4* g1 = reinterpret_cast<const uint4*>(a.cb1);
    for (int i = threadIdx.x; i < 4096; i += blockDim.x) cb1s[i] = g1[i];
    if (kTwo && threadIdx.x < 16) cb2s[threadIdx.x] = reinterpret_cast<const uint4*>(a.cb2)[threadIdx.x];
  }
  {
    const uint16_t* xg = static_cast<const uint16_t*>(a.x);
    const int vec_per_row = kc / 8;
    for (int i = threadIdx.x; i < 8 * NT * vec_per_row; i += blockDim.x) {
      const int t = i / vec_per_row, v = i % vec_per_row;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (t < M) val = *reinterpret_cast<const uint4*>(xg + (int64_t)t * K + k0 + 8 * v);
      *reinterpret_cast<uint4*>(xs + t * xstride + 8 * v) = val;
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int r0 = blockIdx.x * kGemvRows + warp * 16;
  if (r0 >= N) return;
  const int rows[2] = {r0 + g, r0 + g + 8};
  const bool valid[2] = {rows[0] < N, rows[1] < N};
  const int nblk = K / a.scale_group;

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;

  for (int kb = 0; kb < kc; kb += 64) {
    const int gA = (k0 + kb) / 8 + 2 * c;  // this lane's first group (even)
    uint32_t w[2][2][4];                   // [row][codeword A/B][pair]
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      uint32_t i1a = 0, i1b = 0, i2a = 0, i2b = 0;
      float s = 0.f;
      if (valid[r]) {
        const int64_t rowoff = (int64_t)rows[r] * G;
        if (FMT == kFmtVq16) {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(a.idx16 + rowoff + gA);
          i1a = v & 0xFFFFu;
          i1b = v >> 16;
        } else {
          const uint32_t lo2 = *reinterpret_cast<const uint16_t*>(a.lo + rowoff + gA);
          const uint32_t hb = a.hi4[rowoff / 2 + gA / 2];
          i1a = (lo2 & 0xFFu) | ((hb & 15u) << 8);
          i1b = (lo2 >> 8) | ((hb >> 4) << 8);
          if (kTwo) {
            const uint32_t sb = a.s2[rowoff / 2 + gA / 2];
            i2a = sb & 15u;
            i2b = sb >> 4;
          }
        }
        s = f16_bits_to_f32(a.scales[(int64_t)rows[r] * nblk + (k0 + kb) / a.scale_group]);
      }
      uint4 c1a, c1b, c2a = make_uint4(0, 0, 0, 0), c2b = make_uint4(0, 0, 0, 0);
      if (kSmemCb) {
        c1a = cb1s[i1a];
        c1b = cb1s[i1b];
      } else {
        c1a = __ldg(reinterpret_cast<const uint4*>(a.cb1) + i1a);
        c1b = __ldg(reinterpret_cast<const uint4*>(a.cb1) + i1b);
      }
      if (kTwo) {
        c2a = cb2s[i2a];
        c2b = cb2s[i2b];
      }
      decode_group_packed<T, kTwo>(c1a, c2a, s, w[r][0]);
      decode_group_packed<T, kTwo>(c1b, c2b, s, w[r][1]);
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const uint16_t* xr = xs + (8 * t + g) * xstride + kb + 16 * c;
      const uint4 q0 = *reinterpret_cast<const uint4*>(xr);
      const uint4 q1 = *reinterpret_cast<const uint4*>(xr + 8);
      const uint32_t b0[4] = {q0.x, q0.y, q0.z, q0.w};
      const uint32_t b1[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t af[4] = {w[0][0][j], w[1][0][j], w[0][1][j], w[1][1][j]};
        Mma16816<T>::run(acc[t], af, b0[j], b1[j]);
      }
    }
  }

  // Accumulator layout: acc[t][0..1] = (row g, tokens 8t+2c, +1), acc[t][2..3] = row g+8.
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = 8 * t + 2 * c + (i & 1);
      const int r = rows[i >> 1];
      if (m >= M || r >= N) continue;
      if (partial == nullptr)
        static_cast<uint16_t*>(a.y)[(int64_t)m * N + r] = Elt<T>::from_f32(acc[t][i]);
      else
        partial[((int64_t)split * M + m) * N + r] = acc[t][i];
    }
  }
}

template <int FMT, typename T, int NT>
static cudaError_t launch_one(const LayerArgs& a, const Plan& p, float* scratch, cudaStream_t s) {
  const int kc = p.k_per_split;
  const size_t smem = (FMT != kFmtVq16 ? 4096 * 16 : 0) + (FMT == kFmtRvq12_4 ? 256 : 0) +
                      (size_t)8 * NT * (kc + 8) * 2;
  cudaError_t e = cudaFuncSetAttribute(gemv_kernel<FMT, T, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.N + kGemvRows - 1) / kGemvRows, p.splits);
  gemv_kernel<FMT, T, NT><<<grid, 256, smem, s>>>(a, kc, p.splits > 1 ? scratch : nullptr);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  return launch_split_reduce(scratch, a.y, p.splits, a.M, a.N, a.act, s);
}

template <int FMT, typename T>
static cudaError_t launch_nt(const LayerArgs& a, const Plan& p, float* scratch, cudaStream_t s) {
  return a.M <= 8 ? launch_one<FMT, T, 1>(a, p, scratch, s) : launch_one<FMT, T, 2>(a, p, scratch, s);
}

template <typename T>
static cudaError_t launch_fmt(const LayerArgs& a, const Plan& p, float* scratch, cudaStream_t s) {
  switch (a.fmt) {
    case kFmtRvq12: return launch_nt<kFmtRvq12, T>(a, p, scratch, s);
    case kFmtRvq12_4: return launch_nt<kFmtRvq12_4, T>(a, p, scratch, s);
    default: return launch_nt<kFmtVq16, T>(a, p, scratch, s);
  }
}

cudaError_t launch_gemv(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* /*tickets*/, cudaStream_t s) {
  return a.act == VQ_BF16 ? launch_fmt<__nv_bfloat16>(a, p, scratch, s) : launch_fmt<__half>(a, p, scratch, s);
}

// Split choice: enough CTAs to cover the SMs about twice, each K-split a multiple
// of 64 and at most kGemvMaxKc wide (bounds the staged x slice).
void plan_gemv(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  const int nb = d.K / 64;
  const int row_tiles = (d.N + kGemvRows - 1) / kGemvRows;
  const int s_min = (d.K + kGemvMaxKc - 1) / kGemvMaxKc;
  const int target = 2 * dev.num_sms;
  int S = (target + row_tiles - 1) / row_tiles;
  if (S < s_min) S = s_min;
  if (S > nb) S = nb;
  const int bps = (nb + S - 1) / S;
  S = (nb + bps - 1) / bps;
  p->path = VQ_PATH_GEMV;
  p->splits = S;
  p->k_per_split = bps * 64;
  p->launches = S > 1 ? 2 : 1;
  p->scratch_bytes = S > 1 ? (size_t)S * M * d.N * sizeof(float) : 0;
  p->tickets = 0;
}

}  // namespace vq

// Split-K GEMV for 1 <= M <= 16 tokens: y = x . W^T with W decoded on the fly
// (GLQ README, "Inference kernels": the weight matrix is never materialised; the
// split-K partial sums go to a scratch buffer and are reduced in a fixed order).
//
// Work layout
//   CTA    = 8 warps, 128 output rows x one K-split (k_per_split, multiple of 256)
//   warp   = one 16-row tile of W; loops over its K-split in 256-wide blocks
//   lane   = (g = lane/4, c = lane%4): rows g and g+8 of the tile and groups
//            8c .. 8c+7 of the current 256-wide block (one 64-weight scale
//            block) -> 16 codewords per block, fed by 8 small vector loads that
//            are issued one block ahead
// Each lane decodes its codewords into registers (12-bit codebooks staged in
// shared memory by one bulk copy; the 65,536-entry table read through L2) and
// feeds them straight into mma.sync m16n8k16 as the A operand (W rows x k), with
// x as the B operand (k x 8 tokens, one or two token tiles).
//
// k permutation: the MMA's reduction order does not change the result's
// definition, so for codeword q of the lane (group 8c+q) MMA 2q+h uses elements
// 4h..4h+1 in fragment slot "k-pair c" and 4h+2..4h+3 in slot "k-pair c+4".  The
// matching x elements are then x[g][64c + 8q + 4h .. +3], i.e. half of a 16-byte
// shared-memory load -- no shuffles on either operand.
//
// Decoded weights use the materialised-weight rounding (stage sum and scaled
// value rounded to fp32, then to the activation type; for the residual ladder one
// fused multiply-add per residual stage, ladder.cuh), so every product the MMA
// forms is of exactly the weights vq_debug_dequant exports.
//
// Split-K reduction: each split writes fp32 partials; the CTA that completes a
// row tile last (atomic ticket) sums the splits in increasing order and writes
// y, so a forward is one launch and the result does not depend on scheduling.
// The kernel is launched with programmatic dependent launch: it stages the
// codebooks and fetches its first indices before waiting for the previous
// kernel in the stream, and reads x / writes y only after that wait.
#include "common.cuh"
#include "internal.h"
#include "ladder.cuh"
#include "tc_ptx.cuh"

namespace vq {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 16 * kGemvWarps;
constexpr int kGemvBlk = 256;     // k per block (32 groups)
constexpr int kGemvMaxKc = 2048;  // x slice staged per CTA: 16 tokens x 2048 x 2 B

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int FMT>
struct BlockIdx {
  uint32_t w[2][4];  // per row: lo (2 words) + hi4 (1) + s2 (1), or idx16 (4 words)
  uint32_t sc;       // two fp16 scales (rows g, g+8)
};
template <>
struct BlockIdx<kFmtVq16Rvq> {
  uint32_t w[2][4];  // per row: the primary stage's idx16 words
  uint32_t sc;
  LadderIdx res[2];  // per row: the residual stages' index words
};

// Index bytes of one 64-wide k block (8 groups, starting at group gbase) for rows
// g and g+8 of the lane, plus their scales.
template <int FMT>
__device__ __forceinline__ void load_block(const LayerArgs& a, const int rows[2], const bool valid[2], int gbase,
                                           int k, BlockIdx<FMT>& b) {
  const int G = a.K / 8;
  const int s = gbase >> 4, w = slice_width(s, G), o = gbase & 15;  // o is 0 or 8
  uint32_t s16[2] = {0, 0};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    b.w[r][0] = b.w[r][1] = b.w[r][2] = b.w[r][3] = 0;
    if constexpr (FMT == kFmtVq16Rvq) b.res[r] = LadderIdx{};
    if (!valid[r]) continue;
    const int64_t e = (int64_t)16 * s * a.N + (int64_t)rows[r] * w + o;
    if constexpr (FMT == kFmtVq16Rvq) load_ladder_block(a, e, b.res[r]);
    if (FMT == kFmtVq16 || FMT == kFmtVq16Rvq) {
      const uint4 v = *reinterpret_cast<const uint4*>(a.idx16 + e);
      b.w[r][0] = v.x; b.w[r][1] = v.y; b.w[r][2] = v.z; b.w[r][3] = v.w;
    } else {
      const uint2 lo = *reinterpret_cast<const uint2*>(a.lo + e);
      b.w[r][0] = lo.x;
      b.w[r][1] = lo.y;
      b.w[r][2] = *reinterpret_cast<const uint32_t*>(a.hi4 + e / 2);
      if (FMT == kFmtRvq12_4) b.w[r][3] = *reinterpret_cast<const uint32_t*>(a.s2 + e / 2);
    }
    s16[r] = a.scales[scale_index(rows[r], k, a.N, a.K, a.scale_group)];
  }
  b.sc = s16[0] | (s16[1] << 16);
}

template <int FMT, typename T, int NT>
__global__ void __launch_bounds__(256) gemv_kernel(LayerArgs a, int k_per_split, int splits, float* __restrict__ partial,
                                                   uint32_t* __restrict__ tickets) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr bool k16 = (FMT == kFmtVq16 || FMT == kFmtVq16Rvq);
  constexpr bool kSmemCb = !k16;
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  constexpr bool kLadder = (FMT == kFmtVq16Rvq);
  uint4* cb1s = reinterpret_cast<uint4*>(smem);  // 4096 entries (12-bit formats); the ladder's 8-bit codebook
  uint4* cb2s = cb1s + (kSmemCb ? 4096 : (kLadder ? 256 : 0));                 // 16 entries
  uint64_t* bar = reinterpret_cast<uint64_t*>(cb2s + (kTwo ? 16 : 0));         // codebook barrier
  int* flag = reinterpret_cast<int*>(bar + 1);
  uint16_t* xs = reinterpret_cast<uint16_t*>(bar + 2);

  const int K = a.K, M = a.M, N = a.N;
  const int split = blockIdx.y;
  const int k0 = split * k_per_split;
  const int kc = min(k_per_split, K - k0);
  const int xstride = kc + 8;  // elements; +16 B breaks the 8-token bank alignment
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int r0 = blockIdx.x * kGemvRows + warp * 16;
  const int rows[2] = {r0 + g, r0 + g + 8};
  const bool valid[2] = {rows[0] < N, rows[1] < N};

  // Prologue, independent of the previous kernel: codebooks + first indices.
  if (kSmemCb && threadIdx.x == 0) {
    const uint32_t b = smem_u32(bar);
    ptx::mbar_init(b, 1);
    ptx::fence_barrier_init();
    ptx::mbar_arrive_expect_tx(b, 65536u + (kTwo ? 256u : 0u));
    ptx::bulk_load(smem_u32(cb1s), a.cb1, 65536u, b);
    if (kTwo) ptx::bulk_load(smem_u32(cb2s), a.cb2, 256u, b);
  }
  if (kLadder) stage_cb8(a, cb1s, threadIdx.x, blockDim.x);
  BlockIdx<FMT> cur, nxt;
  {
    const int kb = 0, kblock = k0 + kb + 64 * c;
    const bool act[2] = {valid[0] && kblock < k0 + kc, valid[1] && kblock < k0 + kc};
    load_block<FMT>(a, rows, act, kblock / 8, kblock, cur);
  }

  grid_dependency_wait();  // x and y (and scratch) may be touched from here on
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
  // Bounded wait for the codebooks.  Past the bound (never on a healthy device)
  // the kernel still runs to completion so the split-K tickets stay consistent.
  if (kSmemCb) ptx::mbar_wait(smem_u32(bar), 0, nullptr);

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;

  for (int kb = 0; kb < kc; kb += kGemvBlk) {
    // Prefetch the next block's indices while this one is decoded.
    if (kb + kGemvBlk < kc) {
      const int kblock = k0 + kb + kGemvBlk + 64 * c;
      const bool act[2] = {valid[0] && kblock < k0 + kc, valid[1] && kblock < k0 + kc};
      load_block<FMT>(a, rows, act, kblock / 8, kblock, nxt);
    }
    const bool active = (kb + 64 * c) < kc;  // lanes past a ragged end contribute zeros
    const float2 sc = f16x2_to_f32x2(cur.sc);
    const float s[2] = {sc.x, sc.y};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t wq[2][4];  // [row][pair]
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        uint32_t i1, i2 = 0;
        if (k16) {
          i1 = (cur.w[r][q >> 1] >> (16 * (q & 1))) & 0xFFFFu;
        } else {
          i1 = ((cur.w[r][q >> 2] >> (8 * (q & 3))) & 0xFFu) | (((cur.w[r][2] >> (4 * q)) & 15u) << 8);
          if (kTwo) i2 = (cur.w[r][3] >> (4 * q)) & 15u;
        }
        const uint4 c1 = kSmemCb ? cb1s[i1] : __ldg(reinterpret_cast<const uint4*>(a.cb1) + i1);
        if constexpr (FMT == kFmtVq16Rvq) {
          float v[8];
          ladder_sum(a, cur.res[r], q, c1, cb1s, v);
          pack_scaled<T>(v, active ? s[r] : 0.f, wq[r]);
        } else {
          const uint4 c2 = kTwo ? cb2s[i2] : c1;
          decode_group_packed<T, kTwo>(c1, c2, active ? s[r] : 0.f, wq[r]);
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        uint4 xq = make_uint4(0, 0, 0, 0);
        if (active) xq = *reinterpret_cast<const uint4*>(xs + (8 * t + g) * xstride + kb + 64 * c + 8 * q);
        const uint32_t af0[4] = {wq[0][0], wq[1][0], wq[0][1], wq[1][1]};
        const uint32_t af1[4] = {wq[0][2], wq[1][2], wq[0][3], wq[1][3]};
        Mma16816<T>::run(acc[t], af0, xq.x, xq.y);
        Mma16816<T>::run(acc[t], af1, xq.z, xq.w);
      }
    }
    cur = nxt;
  }
  grid_dependents_launch();

  // Accumulator layout: acc[t][0..1] = (row g, tokens 8t+2c, +1), acc[t][2..3] = row g+8.
  uint16_t* y = static_cast<uint16_t*>(a.y);
  if (splits == 1) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 8 * t + 2 * c + (i & 1);
        const int r = rows[i >> 1];
        if (m < M && r < N)
          y[(int64_t)m * N + r] = Elt<T>::from_f32(a.addend ? acc[t][i] + a.addend[(int64_t)m * N + r] : acc[t][i]);
      }
    return;
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = 8 * t + 2 * c + (i & 1);
      const int r = rows[i >> 1];
      if (m < M && r < N) partial[((int64_t)split * M + m) * N + r] = acc[t][i];
    }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) *flag = (atomicAdd(&tickets[blockIdx.x], 1u) == (uint32_t)(splits - 1));
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  const int rbeg = blockIdx.x * kGemvRows;
  const int nrows = min(kGemvRows, N - rbeg);
  for (int i = threadIdx.x; i < nrows * M; i += blockDim.x) {
    const int m = i / nrows, r = rbeg + i % nrows;
    float sum = 0.f;
    for (int k = 0; k < splits; ++k) sum += __ldcg(partial + ((int64_t)k * M + m) * N + r);
    y[(int64_t)m * N + r] = Elt<T>::from_f32(a.addend ? sum + a.addend[(int64_t)m * N + r] : sum);
  }
  if (threadIdx.x == 0) tickets[blockIdx.x] = 0u;  // ready for the next forward
}

template <int FMT, typename T, int NT>
static cudaError_t launch_one(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets, cudaStream_t s) {
  const int kc = p.k_per_split;
  const bool k16 = (FMT == kFmtVq16 || FMT == kFmtVq16Rvq);
  const size_t smem = (!k16 ? 4096 * 16 : 0) + (FMT == kFmtVq16Rvq ? 256 * 16 : 0) + (FMT == kFmtRvq12_4 ? 256 : 0) + 16 +
                      (size_t)8 * NT * (kc + 8) * 2;
  auto kern = gemv_kernel<FMT, T, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.N + kGemvRows - 1) / kGemvRows, p.splits);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, kc, p.splits, p.splits > 1 ? scratch : nullptr,
                            p.splits > 1 ? tickets : nullptr);
}

template <int FMT, typename T>
static cudaError_t launch_nt(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets, cudaStream_t s) {
  return a.M <= 8 ? launch_one<FMT, T, 1>(a, p, scratch, tickets, s) : launch_one<FMT, T, 2>(a, p, scratch, tickets, s);
}

template <typename T>
static cudaError_t launch_fmt(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets, cudaStream_t s) {
  switch (a.fmt) {
    case kFmtRvq12: return launch_nt<kFmtRvq12, T>(a, p, scratch, tickets, s);
    case kFmtRvq12_4: return launch_nt<kFmtRvq12_4, T>(a, p, scratch, tickets, s);
    case kFmtVq16Rvq: return launch_nt<kFmtVq16Rvq, T>(a, p, scratch, tickets, s);
    default: return launch_nt<kFmtVq16, T>(a, p, scratch, tickets, s);
  }
}

cudaError_t launch_gemv(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets, cudaStream_t s) {
  return a.act == VQ_BF16 ? launch_fmt<__nv_bfloat16>(a, p, scratch, tickets, s)
                          : launch_fmt<__half>(a, p, scratch, tickets, s);
}

// Split choice: enough CTAs to cover the SMs about twice, each K-split a multiple
// of 256 (the last may be ragged) and at most kGemvMaxKc wide.
void plan_gemv(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  const int nb = (d.K + kGemvBlk - 1) / kGemvBlk;
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
  p->k_per_split = bps * kGemvBlk;
  p->launches = 1;
  p->scratch_bytes = S > 1 ? (size_t)S * M * d.N * sizeof(float) : 0;
  p->tickets = S > 1 ? row_tiles : 0;
  p->ctas = row_tiles * S;
}

}  // namespace vq

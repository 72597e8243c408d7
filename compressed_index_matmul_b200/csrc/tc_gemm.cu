// Tensor-core path: y = x . W^T for any M (meant for M >= 17, e.g. prefill),
// with W decoded tile by tile into shared memory and multiplied on the 5th-gen
// tensor cores (tcgen05.mma, fp32 accumulator in TMEM).  The dense W never
// reaches device memory (GLQ README, "Inference kernels"; decode per the orka
// README, "How it works": scale x sum over stages of codebook[index]).
//
// One CTA computes a 128-row x T-token tile of y over one K-split:
//   warp 0    TMA producer: x tiles (T tokens x 64 k, 128-byte swizzle) into a
//             3-stage ring; it also bulk-copies the 12-bit codebooks into shared
//             memory once.
//   warp 1    allocates TMEM; lane 0 issues tcgen05.mma (M=128, N=T, K=16, four
//             per 64-wide k block) and commits each stage back to the producers.
//   warps 2-9 decode: two warps per TMEM lane quarter; thread = one row of the
//             tile (= its TMEM lane) and one half (4 groups) of each 64-wide k
//             block.  It unpacks, gathers the codewords, scales, rounds to the
//             activation type and stores 16-byte chunks into the stage's A tile in
//             the same 128-byte-swizzled K-major layout the TMA uses for x.  Its
//             index bytes are loaded four blocks ahead into registers.  After the
//             last block the same threads read the accumulator from TMEM and write
//             y (or fp32 split-K partials; the last CTA of a tile, by an atomic
//             ticket, sums the partials in split order).
// Every mbarrier wait is bounded; a timeout sets the handle's error word and the
// CTA winds down (waits for its own copies, frees TMEM) instead of hanging.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace vq {

constexpr int kTcRows = 128;
constexpr int kTcStages = 3;
constexpr int kTcThreads = 320;
constexpr int kTcDecodeWarps = 8;
constexpr int kTcAhead = 4;  // k blocks of index bytes in flight per decode thread
constexpr int kTcMaxT = 256;
constexpr uint32_t kTcATileBytes = kTcRows * 128;  // 128 rows x 64 bf16
constexpr uint32_t kTcTilesOffset = 66560;         // after codebooks + barriers, 1024-aligned
constexpr uint32_t kTcSmemMax = kTcTilesOffset + kTcStages * (kTcATileBytes + kTcMaxT * 128) + 1024;

struct TcArgs {
  LayerArgs a;
  int T;            // tokens per tile (MMA N): multiple of 16, <= 256
  int k_per_split;  // multiple of 64
  int splits;
  float* partial;   // [splits][M][N] when splits > 1
  uint32_t* tickets;
  uint32_t* err;
};

template <int FMT, typename T>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const __grid_constant__ CUtensorMap xmap, TcArgs p) {
  extern __shared__ unsigned char smem_raw[];
  constexpr bool kSmemCb = (FMT != kFmtVq16);
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  const LayerArgs& a = p.a;
  // 1024-byte aligned base (the swizzle pattern is taken from address bits).
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw);
  uint4* cb1s = reinterpret_cast<uint4*>(sm);
  uint4* cb2s = reinterpret_cast<uint4*>(sm + 65536);
  const uint32_t bar0 = base + 65792;
  auto full_a = [&](int s) { return bar0 + 8u * s; };
  auto full_b = [&](int s) { return bar0 + 8u * (kTcStages + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * kTcStages + s); };
  const uint32_t accum_bar = bar0 + 8u * (3 * kTcStages);
  const uint32_t cb_bar = accum_bar + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + 65880);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + 65884);
  volatile int* last_flag = reinterpret_cast<volatile int*>(sm + 65888);
  const uint32_t b_bytes = (uint32_t)p.T * 128u;
  const uint32_t stage_bytes = kTcATileBytes + b_bytes;
  auto a_tile = [&](int s) { return base + kTcTilesOffset + stage_bytes * s; };
  auto b_tile = [&](int s) { return base + kTcTilesOffset + stage_bytes * s + kTcATileBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, G = K / 8, N = a.N, M = a.M;
  const int row0 = blockIdx.x * kTcRows;
  const int tok0 = blockIdx.y * p.T;
  const int split = blockIdx.z;
  const int kbeg = split * p.k_per_split;
  const int nkb = (min(K, kbeg + p.k_per_split) - kbeg) / 64;
  const uint32_t tcols = p.T <= 32 ? 32u : (p.T <= 64 ? 64u : (p.T <= 128 ? 128u : 256u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      ptx::mbar_init(full_a(s), kTcDecodeWarps);  // one arrival per decode warp
      ptx::mbar_init(full_b(s), 1);  // the producer's expect_tx arrival (+ bytes)
      ptx::mbar_init(empty(s), 1);   // one tcgen05.commit
    }
    ptx::mbar_init(accum_bar, 1);
    ptx::mbar_init(cb_bar, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(smem_u32(tmem_slot), tcols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tensormap(&xmap);
      if (kSmemCb) {
        ptx::mbar_arrive_expect_tx(cb_bar, 65536u + (kTwo ? 256u : 0u));
        ptx::bulk_load(base, a.cb1, 65536u, cb_bar);
        if (kTwo) ptx::bulk_load(base + 65536, a.cb2, 256u, cb_bar);
      }
      int issued = 0;
      for (int kb = 0; kb < nkb && !*abort_flag; ++kb) {
        const int s = kb % kTcStages;
        if (kb >= kTcStages && !ptx::mbar_wait(empty(s), ((kb / kTcStages) - 1) & 1, p.err)) {
          *abort_flag = 1;
          break;
        }
        ptx::mbar_arrive_expect_tx(full_b(s), b_bytes);
        ptx::tma_load_2d(b_tile(s), &xmap, kbeg + kb * 64, tok0, full_b(s));
        issued = kb + 1;
      }
      // Do not leave while a copy into this CTA's shared memory may be in flight.
      for (int kb = (issued > kTcStages ? issued - kTcStages : 0); kb < issued; ++kb)
        ptx::mbar_wait(full_b(kb % kTcStages), (kb / kTcStages) & 1, p.err);
      if (kSmemCb) ptx::mbar_wait(cb_bar, 0, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kAbFmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
      const uint32_t idesc = ptx::idesc_f16(kAbFmt, kTcRows, (uint32_t)p.T);
      bool ok = true;
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t par = (kb / kTcStages) & 1;
        if (*abort_flag || !ptx::mbar_wait(full_b(s), par, p.err) || !ptx::mbar_wait(full_a(s), par, p.err)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint64_t ad = ptx::smem_desc_sw128(a_tile(s));
        const uint64_t bd = ptx::smem_desc_sw128(b_tile(s));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // +32 bytes along K inside the swizzle atom
          ptx::umma_f16(tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0);
        ptx::umma_commit(empty(s));
        issued = kb + 1;
      }
      ptx::umma_commit(accum_bar);
      // On the abort path nobody else waits for the accumulator: drain the issued
      // MMAs here before TMEM and shared memory are released.
      if (!ok && issued) ptx::mbar_wait(accum_bar, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ decode + epilogue
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;  // which 4 groups of each k block
    const int dr = 32 * q + lane;      // row within the tile == TMEM lane
    const int r = row0 + dr;
    const bool valid = r < N;
    const uint4* cbg = reinterpret_cast<const uint4*>(a.cb1);
    struct Rec {
      uint32_t w[4];  // lo (2 words) + hi4 + s2, or idx16 (4 words) of this thread's 4 groups
      uint32_t sc;
    };
    auto load_rec = [&](int kb, Rec& rc) {
      rc.w[0] = rc.w[1] = rc.w[2] = rc.w[3] = 0;
      rc.sc = 0;
      if (!valid || kb >= nkb) return;
      const int g0 = (kbeg / 8) + kb * 8 + 4 * half;  // first of this thread's 4 groups
      const int s = g0 >> 4;
      const int64_t e = (int64_t)16 * s * N + (int64_t)r * slice_width(s, G) + (g0 & 15);
      if (FMT == kFmtVq16) {
        const uint2 v = *reinterpret_cast<const uint2*>(a.idx16 + e);
        rc.w[0] = v.x;
        rc.w[1] = v.y;
      } else {
        rc.w[0] = *reinterpret_cast<const uint32_t*>(a.lo + e);
        rc.w[1] = *reinterpret_cast<const uint16_t*>(a.hi4 + e / 2);
        if (kTwo) rc.w[2] = *reinterpret_cast<const uint16_t*>(a.s2 + e / 2);
      }
      rc.sc = a.scales[scale_index(r, 8 * g0, N, K, a.scale_group)];
    };
    bool ok = true;
    Rec rec[kTcAhead];
#pragma unroll
    for (int i = 0; i < kTcAhead; ++i) load_rec(i, rec[i]);
    if (kSmemCb && !ptx::mbar_wait(cb_bar, 0, p.err)) {
      *abort_flag = 1;
      ok = false;
    }
    for (int kb0 = 0; ok && kb0 < nkb; kb0 += kTcAhead) {
#pragma unroll
      for (int i = 0; i < kTcAhead; ++i) {
        const int kb = kb0 + i;
        if (kb >= nkb || !ok) break;
        const Rec cr = rec[i];
        load_rec(kb + kTcAhead, rec[i]);
        const int s = kb % kTcStages;
        if (*abort_flag || (kb >= kTcStages && !ptx::mbar_wait(empty(s), ((kb / kTcStages) - 1) & 1, p.err))) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        const float sc = f16_bits_to_f32(cr.sc);
        unsigned char* at = sm + (a_tile(s) - base) + dr * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t i1, i2 = 0;
          if (FMT == kFmtVq16) {
            i1 = (cr.w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
          } else {
            i1 = ((cr.w[0] >> (8 * j)) & 0xFFu) | (((cr.w[1] >> (4 * j)) & 15u) << 8);
            if (kTwo) i2 = (cr.w[2] >> (4 * j)) & 15u;
          }
          const uint4 c1 = kSmemCb ? cb1s[i1] : __ldg(cbg + i1);
          const uint4 c2 = kTwo ? cb2s[i2] : c1;
          uint32_t w[4];
          decode_group_packed<T, kTwo>(c1, c2, valid ? sc : 0.f, w);
          const int chunk = 4 * half + j;
          *reinterpret_cast<uint4*>(at + ((chunk ^ (dr & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(full_a(s));
      }
    }
    // -------------------------------------------------------------- epilogue
    if (ok && !ptx::mbar_wait(accum_bar, 0, p.err)) *abort_flag = 1;
    // One decision for all epilogue threads, so the named barriers below are
    // reached by every one of them or by none.
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (threadIdx.x == 64) *last_flag = *abort_flag ? 0 : 2;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    ok = (*last_flag == 2);
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok) {
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16);
      uint16_t* y = static_cast<uint16_t*>(a.y);
      for (int c0 = 16 * half; c0 < p.T; c0 += 32) {  // the two warps of a quarter alternate 16-column chunks
        uint32_t v[16];
        ptx::tmem_ld16(taddr + c0, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int tok = tok0 + c0 + i;
          if (tok >= M || !valid) continue;
          if (p.splits == 1)
            y[(int64_t)tok * N + r] = Elt<T>::from_f32(__uint_as_float(v[i]));
          else
            p.partial[((int64_t)split * M + tok) * N + r] = __uint_as_float(v[i]);
        }
      }
      ptx::tc_fence_before();
      if (p.splits > 1) {
        __threadfence();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const int tile = blockIdx.y * gridDim.x + blockIdx.x;
        if (threadIdx.x == 64) *last_flag = (atomicAdd(&p.tickets[tile], 1u) == (uint32_t)(p.splits - 1));
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (*last_flag) {
          __threadfence();
          const int tend = min(M, tok0 + p.T);
          if (valid)
            for (int tok = tok0 + half; tok < tend; tok += 2) {
              float sum = 0.f;
              for (int k = 0; k < p.splits; ++k) sum += __ldcg(p.partial + ((int64_t)k * M + tok) * N + r);
              y[(int64_t)tok * N + r] = Elt<T>::from_f32(sum);
            }
          if (threadIdx.x == 64) p.tickets[tile] = 0u;
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, tcols);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

struct TcGeom {
  int T, TT, RT, S, kps;
};

static TcGeom tc_geom(int M, int N, int K, int num_sms) {
  TcGeom g;
  const int m16 = (M + 15) / 16 * 16;
  g.T = m16 < kTcMaxT ? m16 : kTcMaxT;
  g.TT = (M + g.T - 1) / g.T;
  g.RT = (N + kTcRows - 1) / kTcRows;
  const int tiles = g.RT * g.TT;
  const int nb = K / 64;
  int S = num_sms / tiles;
  if (S < 1) S = 1;
  if (S > 8) S = 8;
  if (S > nb) S = nb;
  const int bps = (nb + S - 1) / S;
  g.S = (nb + bps - 1) / bps;
  g.kps = bps * 64;
  return g;
}

bool plan_tc(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  if (M < 1 || dev.smem_optin < (int)kTcSmemMax) return false;
  const TcGeom g = tc_geom(M, d.N, d.K, dev.num_sms);
  p->path = VQ_PATH_TC;
  p->splits = g.S;
  p->k_per_split = g.kps;
  p->launches = 1;
  p->scratch_bytes = g.S > 1 ? (size_t)g.S * M * d.N * sizeof(float) : 0;
  p->tickets = g.S > 1 ? g.RT * g.TT : 0;
  return true;
}

template <int FMT, typename T>
static cudaError_t launch_tc_t(const LayerArgs& a, const TcGeom& g, float* scratch, uint32_t* tickets,
                               uint32_t* err, cudaStream_t s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
  const cuuint64_t strides[1] = {(cuuint64_t)a.K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)g.T};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, a.act == VQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                   const_cast<void*>(a.x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const uint32_t smem = kTcTilesOffset + kTcStages * (kTcATileBytes + (uint32_t)g.T * 128u) + 1024u;
  cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<FMT, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  TcArgs p{a, g.T, g.kps, g.S, g.S > 1 ? scratch : nullptr, g.S > 1 ? tickets : nullptr, err};
  dim3 grid(g.RT, g.TT, g.S);
  tc_gemm_kernel<FMT, T><<<grid, kTcThreads, smem, s>>>(map, p);
  return cudaGetLastError();
}

cudaError_t launch_tc(const LayerArgs& a, const Plan& pl, float* scratch, uint32_t* tickets, uint32_t* err,
                      cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const TcGeom g = tc_geom(a.M, a.N, a.K, sms);
  if (g.S != pl.splits) return cudaErrorInvalidValue;
  const bool bf = a.act == VQ_BF16;
  switch (a.fmt) {
    case kFmtRvq12:
      return bf ? launch_tc_t<kFmtRvq12, __nv_bfloat16>(a, g, scratch, tickets, err, s)
                : launch_tc_t<kFmtRvq12, __half>(a, g, scratch, tickets, err, s);
    case kFmtRvq12_4:
      return bf ? launch_tc_t<kFmtRvq12_4, __nv_bfloat16>(a, g, scratch, tickets, err, s)
                : launch_tc_t<kFmtRvq12_4, __half>(a, g, scratch, tickets, err, s);
    default:
      return bf ? launch_tc_t<kFmtVq16, __nv_bfloat16>(a, g, scratch, tickets, err, s)
                : launch_tc_t<kFmtVq16, __half>(a, g, scratch, tickets, err, s);
  }
}

}  // namespace vq

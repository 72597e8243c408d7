// Tensor-core path: y = x . W^T for any M (meant for M >= 17, e.g. prefill),
// with W decoded tile by tile into tensor memory and multiplied on the 5th-gen
// tensor cores (tcgen05.mma, A from TMEM, B from shared memory, fp32 accumulator
// in TMEM).  The dense W never reaches device memory (GLQ README, "Inference
// kernels"; decode per the orka README, "How it works": scale x sum over stages
// of codebook[index]).
//
// One CTA computes a 128-row x T-token tile of y over one K-split:
//   warp 0     producer: bulk-copies the 12-bit codebook into shared memory once;
//              per 128-input slice, bulk-copies the tile's index bytes (the
//              K-slice-major planes make them one contiguous run per plane) into
//              a 4-slot ring; per 64-wide k block, TMA-loads the x tile (T tokens
//              x 64, 128-byte swizzle) into a ring of S stages (S = 4; 3 when two
//              64-token CTAs share an SM).
//   warp 1     allocates TMEM; lane 0 issues tcgen05.mma (M=128, N=T, K=16, four
//              per k block, A read from TMEM) and commits each stage back.
//   warps 2.. decode: P warps per TMEM lane quarter (P = 3 for token tiles of 64
//              and more; 2 with two CTAs per SM for the 12-bit formats' tiles of
//              16 to 64; 4 for the 16-bit formats' narrower tiles); thread = one
//              row of the tile (its TMEM lane); warp `part` of a quarter decodes
//              every P-th k block (kb % P == part), all 8 groups of it, into A
//              stage kb % S.  With P = 3 the CTA has 14 warps, at most four share
//              an SM sub-partition and each thread may hold 128 registers (no
//              spills); with P = 2, 10 warps and 96 registers, two CTAs per SM;
//              with P = 4, 18 warps and 96 registers (the decode loop spills a
//              little, but more warps hide its latency when each block's MMA is
//              short).  Per block a thread reads its 8
//              index bytes (plus nibbles and scale) from the staged slice, gathers
//              the stage-1 codewords from shared memory and the stage-2 codewords
//              from the warp's registers (shuffle), decodes with the
//              materialised-weight rounding and stores the 64 weights into its
//              own TMEM lane of the stage's A columns (tcgen05.st).
//              After the last block the same threads read the accumulator from
//              TMEM and write y (or fp32 split-K partials; the last CTA of a tile,
//              by an atomic ticket, sums the partials in split order).
// Every mbarrier wait is bounded; a timeout sets the handle's error word and the
// CTA winds down (waits for its own copies, frees TMEM) instead of hanging.
// When N % 8 != 0 the per-slice index runs are not all 16-byte multiples, so
// bulk copies cannot stage them: the decode threads read their index bytes from
// global memory instead.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "ladder.cuh"
#include "tc_ptx.cuh"

namespace vq {

constexpr int kTcRows = 128;
constexpr int kTcStages = 4;        // x tiles in shared memory and A tiles in TMEM (3 for two 64-token CTAs per SM)
// Decode warps per TMEM lane quarter (kParts, a template parameter): 3 for token
// tiles of 64 and more; 2 with two CTAs per SM for the 12-bit formats' tiles of
// 16 to 48 tokens (and of 64 when the K split stays a cluster pair); 4 with one
// CTA per SM for the 16-bit formats' narrower tiles, whose codeword gathers need
// the L1 cache that a second CTA's shared memory would take; see the launch.
__host__ __device__ constexpr int tc_threads(int parts) { return 64 + 32 * 4 * parts; }
constexpr int kTcMaxT = 256;
constexpr uint32_t kTcACols = 32;   // TMEM columns of one A stage (64 k of 16-bit pairs)
// index-slice ring slot: lo 16 B, hi4 8 B, s2 8 B, scales 4 B per row (idx16: 32 B per row)
constexpr uint32_t kTcIdxLo = 0, kTcIdxHi = 2048, kTcIdxS2 = 3072, kTcIdxSc = 4096;
constexpr uint32_t kTcIdxSlot = 4608;
constexpr int kTcIdxSlots = 4;
constexpr uint32_t kTcOffBars = 65536;   // after the 64 KiB codebook
constexpr uint32_t kTcOffIdx = 65792;    // index ring
constexpr uint32_t kTcTilesOffset = 84992;  // 1024-aligned, after the index ring
static_assert(kTcOffIdx + kTcIdxSlots * kTcIdxSlot <= kTcTilesOffset, "index ring overlaps the tiles");
constexpr uint32_t kTcSmemMax = kTcTilesOffset + kTcStages * (kTcMaxT * 128) + 1024;

// Epilogue kinds: y (or fp32 partials) written per element; y staged in shared
// memory and written by TMA stores (one split); a K-split pair in a 2-CTA cluster
// that adds the two halves over distributed shared memory, then TMA stores.
constexpr int kEpiGlobal = 0, kEpiStore = 1, kEpiPair = 2;

struct TcArgs {
  LayerArgs a;
  int epi;          // kEpi*
  int T;            // tokens per tile (MMA N): multiple of 16, <= 256
  int k_per_split;  // multiple of 128 when splits > 1
  int splits;
  float* partial;   // [splits][M][N] when splits > 1
  uint32_t* tickets;
  uint32_t* err;
};

__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}

// One-stage group: w_j = RN_T(fl32(s * c1_j)).  The mixed-precision FMA takes the
// fp16 codeword half and the fp16 scale as they are and rounds the exact product
// once to fp32 (adding -0 keeps the sign of a zero product).
template <typename T>
__device__ __forceinline__ void decode_one_stage(const uint4& c1, unsigned short s, uint32_t* out) {
  const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float lo, hi;
    asm("{ .reg .f16 l, h; mov.b32 {l, h}, %2; fma.rn.f32.f16 %0, l, %3, %4; fma.rn.f32.f16 %1, h, %3, %4; }"
        : "=f"(lo), "=f"(hi)
        : "r"(w1[q]), "h"(s), "f"(-0.0f));
    out[q] = Elt<T>::pack(lo, hi);
  }
}

// Two-stage group: w_j = RN_T(fl32(s * fl32(c1_j + c2_j))).  The mixed-precision
// add widens the fp16 c1 half exactly and rounds the sum once.
template <typename T>
__device__ __forceinline__ void decode_two_stage(const uint4& c1, const uint32_t (&c2)[4], float s, uint32_t* out) {
  const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
  const uint64_t sv = f32x2(s, s);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 b = f16x2_to_f32x2(c2[q]);
    float lo, hi;
    asm("{ .reg .f16 l, h; mov.b32 {l, h}, %2; add.rn.f32.f16 %0, l, %3; add.rn.f32.f16 %1, h, %4; }"
        : "=f"(lo), "=f"(hi)
        : "r"(w1[q]), "f"(b.x), "f"(b.y));
    const uint64_t m = f32x2_mul(f32x2(lo, hi), sv);
    out[q] = Elt<T>::pack(__uint_as_float((uint32_t)m), __uint_as_float((uint32_t)(m >> 32)));
  }
}

template <int FMT, typename T, bool kStaged, int kTcParts, int kSt>
__global__ void __launch_bounds__(tc_threads(kTcParts), kTcParts == 2 ? 2 : 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap ymap, TcArgs p) {
  extern __shared__ unsigned char smem_raw[];
  constexpr bool k16 = (FMT == kFmtVq16 || FMT == kFmtVq16Rvq);
  constexpr bool kLadder = (FMT == kFmtVq16Rvq);
  constexpr bool kSmemCb = !k16;
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  static_assert(!(kLadder && kStaged), "the residual ladder reads its indices directly");
  static_assert(kSt >= kTcParts && kSt <= kTcStages, "a stage barrier may be at most one phase behind");
  const LayerArgs& a = p.a;
  // 1024-byte aligned base (the swizzle pattern of the x tiles is taken from address bits).
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw);
  const uint4* cb1s = reinterpret_cast<const uint4*>(sm);
  const uint32_t bar0 = base + kTcOffBars;
  auto full_a = [&](int s) { return bar0 + 8u * s; };
  auto full_b = [&](int s) { return bar0 + 8u * (kSt + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * kSt + s); };
  const uint32_t accum_bar = bar0 + 8u * (3 * kSt);
  const uint32_t cb_bar = accum_bar + 8u;
  auto idx_full = [&](int s) { return cb_bar + 8u + 8u * s; };
  auto idx_empty = [&](int s) { return cb_bar + 8u + 8u * kTcIdxSlots + 8u * s; };
  static_assert(8 * (3 * kSt + 2 + 2 * kTcIdxSlots) <= 192, "barriers overlap the flags");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kTcOffBars + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kTcOffBars + 196);
  volatile int* last_flag = reinterpret_cast<volatile int*>(sm + kTcOffBars + 200);
  const uint32_t b_bytes = (uint32_t)p.T * 128u;
  auto b_tile = [&](int s) { return base + kTcTilesOffset + b_bytes * s; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, G = K / 8, N = a.N, M = a.M;
  const int row0 = blockIdx.x * kTcRows;
  const int rows_here = min(kTcRows, N - row0);
  const int tok0 = blockIdx.y * p.T;
  const int split = blockIdx.z;
  const int kbeg = split * p.k_per_split;
  const int nkb = (min(K, kbeg + p.k_per_split) - kbeg) / 64;
  const int nsl = (nkb + 1) / 2;  // 128-input slices of this split (the last may be 64 wide)
  const int s_first = kbeg / 128;
  const bool block_scales = (a.scale_group == 64);
  // TMEM: the accumulator in columns [0, T), then kSt A stages of 32 columns.
  const uint32_t acol0 = ((uint32_t)p.T + 31u) & ~31u;
  const uint32_t tneed = acol0 + kSt * kTcACols;
  const uint32_t tcols = tneed <= 32 ? 32u : (tneed <= 64 ? 64u : (tneed <= 128 ? 128u : (tneed <= 256 ? 256u : 512u)));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      ptx::mbar_init(full_a(s), 4);  // one decode warp per TMEM lane quarter
      ptx::mbar_init(full_b(s), 1);               // the producer's expect_tx arrival (+ bytes)
      ptx::mbar_init(empty(s), 1);                // one tcgen05.commit
    }
    for (int s = 0; s < kTcIdxSlots; ++s) {
      ptx::mbar_init(idx_full(s), 1);
      ptx::mbar_init(idx_empty(s), 8);  // the 8 warps (two parts x four quarters) that decode the slice's two blocks
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
  // The ladder's 8-bit codebook into the (otherwise unused) codebook area.
  if (kLadder) stage_cb8(a, const_cast<uint4*>(cb1s), threadIdx.x, blockDim.x);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tensormap(&xmap);
      if (kSmemCb) {
        ptx::mbar_arrive_expect_tx(cb_bar, 65536u);
        ptx::bulk_load(base, a.cb1, 65536u, cb_bar);
      }
      // Index bytes of slice j (of this split) for rows row0 .. row0+rows_here-1.
      auto issue_idx = [&](int j) {
        const int s = s_first + j, w = slice_width(s, G);
        const uint32_t dst = base + kTcOffIdx + kTcIdxSlot * (j % kTcIdxSlots), bar = idx_full(j % kTcIdxSlots);
        const int64_t e = (int64_t)16 * s * N + (int64_t)row0 * w;  // entry of (slice s, row row0)
        const uint32_t sc = block_scales ? rows_here * (w / 8) * 2 : 0;
        if (FMT == kFmtVq16) {
          ptx::mbar_arrive_expect_tx(bar, rows_here * w * 2 + sc);
          ptx::bulk_load(dst, a.idx16 + e, rows_here * w * 2, bar);
        } else {
          ptx::mbar_arrive_expect_tx(bar, rows_here * w + rows_here * w / 2 * (kTwo ? 2 : 1) + sc);
          ptx::bulk_load(dst + kTcIdxLo, a.lo + e, rows_here * w, bar);
          ptx::bulk_load(dst + kTcIdxHi, a.hi4 + e / 2, rows_here * w / 2, bar);
          if (kTwo) ptx::bulk_load(dst + kTcIdxS2, a.s2 + e / 2, rows_here * w / 2, bar);
        }
        if (block_scales) ptx::bulk_load(dst + kTcIdxSc, a.scales + e / 8, sc, bar);
      };
      int issued = 0, issued_idx = 0;
      if (kStaged)
        for (; issued_idx < kTcIdxSlots && issued_idx < nsl; ++issued_idx) issue_idx(issued_idx);
      for (int kb = 0; kb < nkb && !*abort_flag; ++kb) {
        const int s = kb % kSt;
        if (kb >= kSt && !ptx::mbar_wait(empty(s), ((kb / kSt) - 1) & 1, p.err)) {
          *abort_flag = 1;
          break;
        }
        ptx::mbar_arrive_expect_tx(full_b(s), b_bytes);
        ptx::tma_load_2d(b_tile(s), &xmap, kbeg + kb * 64, tok0, full_b(s));
        issued = kb + 1;
        // After x of block kb (odd, >= 5) is issued, refill with slice (kb+3)/2.
        // Its slot held slice (kb-5)/2, which the warps decoding blocks kb - 5 and
        // kb - 4 released before decoding them; the stage-empty wait above already
        // saw MMA kb - kSt >= kb - 4 (and so every earlier block) complete, so this
        // wait never holds back the x loads.
        if (kStaged && (kb & 1) == 1 && kb >= 5 && (kb + 3) / 2 == issued_idx && issued_idx < nsl) {
          const int j = issued_idx;
          if (!ptx::mbar_wait(idx_empty(j % kTcIdxSlots), ((j / kTcIdxSlots) - 1) & 1, p.err)) {
            *abort_flag = 1;
            break;
          }
          issue_idx(j);
          ++issued_idx;
        }
      }
      // Do not leave while a copy into this CTA's shared memory may be in flight.
      for (int kb = (issued > kSt ? issued - kSt : 0); kb < issued; ++kb)
        ptx::mbar_wait(full_b(kb % kSt), (kb / kSt) & 1, p.err);
      if (kStaged)
        for (int j = (issued_idx > kTcIdxSlots ? issued_idx - kTcIdxSlots : 0); j < issued_idx; ++j)
          ptx::mbar_wait(idx_full(j % kTcIdxSlots), (j / kTcIdxSlots) & 1, p.err);
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
        const int s = kb % kSt;
        const uint32_t par = (kb / kSt) & 1;
        if (*abort_flag || !ptx::mbar_wait(full_b(s), par, p.err) || !ptx::mbar_wait(full_a(s), par, p.err)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t at = tmem + acol0 + kTcACols * s;
        const uint64_t bd = ptx::smem_desc_sw128(b_tile(s));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // A: +8 TMEM columns; B: +32 bytes along K inside the swizzle atom
          ptx::umma_f16_ts(tmem, at + 8u * kk, bd + 2u * kk, idesc, (kb | kk) != 0);
        ptx::umma_commit(empty(s));
        issued = kb + 1;
      }
      ptx::umma_commit(accum_bar);
      // On the abort path nobody else waits for the accumulator: drain the issued
      // MMAs here before TMEM and shared memory are released.
      if (!ok && issued) ptx::mbar_wait(accum_bar, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ decode
    // Warp (quarter q, part) decodes every P-th k block, kb = part, part+P, ...: all
    // 8 groups of the block for its 32 rows, i.e. the whole A stage kb % kSt
    // for its TMEM lane quarter.
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int part = (warp - 2) >> 2;  // 0..kTcParts-1: this warp decodes blocks kb == part (mod kTcParts)
    const int dr = 32 * q + lane;      // row within the tile == TMEM lane
    const int r = row0 + dr;
    const bool valid = r < N;
    const uint4* cbg = reinterpret_cast<const uint4*>(a.cb1);
    uint32_t cb2r[4] = {0, 0, 0, 0};
    if (kTwo) {
      const uint4 v = reinterpret_cast<const uint4*>(a.cb2)[lane & 15];
      cb2r[0] = v.x; cb2r[1] = v.y; cb2r[2] = v.z; cb2r[3] = v.w;
    }
    const unsigned short row_scale = (!block_scales && valid) ? a.scales[r] : (unsigned short)0;
    const uint32_t tlane0 = tmem + ((uint32_t)(32 * q) << 16) + acol0;  // + the A stage's columns
    bool ok = true;
    if (kSmemCb && !ptx::mbar_wait(cb_bar, 0, p.err)) {
      *abort_flag = 1;
      ok = false;
    }
    for (int kb = part; ok && kb < nkb; kb += kTcParts) {
      const int j = kb >> 1, h = kb & 1;
      const int sl = s_first + j, w = slice_width(sl, G);
      // A stage kb % kSt; the MMA of block kb - kSt must be done with it.
      // (This warp's previous block, kb - kTcParts, already needed the MMA of block
      // kb - kTcParts - kSt, so the stage's barrier is at most one phase behind.)
      const int st = kb % kSt;
      const uint32_t tlane = tlane0 + kTcACols * (uint32_t)st;
      if (*abort_flag || (kb >= kSt && !ptx::mbar_wait(empty(st), ((kb / kSt) - 1) & 1, p.err)) ||
          (kStaged && !ptx::mbar_wait(idx_full(j % kTcIdxSlots), (j / kTcIdxSlots) & 1, p.err))) {
        *abort_flag = 1;
        ok = false;
        break;
      }
      uint2 lo8 = make_uint2(0, 0);
      uint32_t hi4w = 0, s24w = 0;
      uint4 v16 = make_uint4(0, 0, 0, 0);
      LadderIdx res{};
      unsigned short sc = row_scale;
      if (valid) {
        if (kStaged) {
          const unsigned char* slot = sm + kTcOffIdx + kTcIdxSlot * (j % kTcIdxSlots);
          if (FMT == kFmtVq16) {
            v16 = *reinterpret_cast<const uint4*>(slot + (dr * w + 8 * h) * 2);
          } else {
            lo8 = *reinterpret_cast<const uint2*>(slot + kTcIdxLo + dr * w + 8 * h);
            hi4w = *reinterpret_cast<const uint32_t*>(slot + kTcIdxHi + dr * (w / 2) + 4 * h);
            if (kTwo) s24w = *reinterpret_cast<const uint32_t*>(slot + kTcIdxS2 + dr * (w / 2) + 4 * h);
          }
          if (block_scales) sc = *reinterpret_cast<const uint16_t*>(slot + kTcIdxSc + (dr * (w / 8) + h) * 2);
        } else {
          const int64_t e = (int64_t)16 * sl * N + (int64_t)r * w + 8 * h;
          if constexpr (kLadder) load_ladder_block(a, e, res);
          if (k16) {
            v16 = *reinterpret_cast<const uint4*>(a.idx16 + e);
          } else {
            lo8 = *reinterpret_cast<const uint2*>(a.lo + e);
            hi4w = *reinterpret_cast<const uint32_t*>(a.hi4 + e / 2);
            if (kTwo) s24w = *reinterpret_cast<const uint32_t*>(a.s2 + e / 2);
          }
          if (block_scales) sc = a.scales[scale_index(r, 128 * sl + 64 * h, N, K, a.scale_group)];
        }
      }
      if (kStaged) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(idx_empty(j % kTcIdxSlots));
      }
      const float scf = (kTwo || kLadder) ? __half2float(__ushort_as_half(sc)) : 0.f;
      ptx::tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // 4 groups (16 TMEM columns) at a time
        uint32_t out[16];
        const uint32_t low = c ? lo8.y : lo8.x;
        const uint32_t v0 = k16 ? (c ? v16.z : v16.x) : 0u, v1 = k16 ? (c ? v16.w : v16.y) : 0u;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int g = 4 * c + t;
          uint32_t i1;
          if (k16)
            i1 = ((t < 2 ? v0 : v1) >> (16 * (t & 1))) & 0xFFFFu;
          else
            i1 = ((low >> (8 * t)) & 0xFFu) | (((hi4w >> (4 * g)) & 15u) << 8);
          const uint4 c1 = kSmemCb ? cb1s[i1] : __ldg(cbg + i1);
          if constexpr (kLadder) {
            float v[8];
            ladder_sum(a, res, g, c1, cb1s, v);
            pack_scaled<T>(v, scf, out + 4 * t);
          } else if (kTwo) {
            const int i2 = (int)((s24w >> (4 * g)) & 15u);
            uint32_t c2[4];
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) c2[w4] = __shfl_sync(0xffffffffu, cb2r[w4], i2);
            decode_two_stage<T>(c1, c2, scf, out + 4 * t);
          } else {
            decode_one_stage<T>(c1, sc, out + 4 * t);
          }
        }
        ptx::tmem_st16(tlane + 16u * c, out);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full_a(st));
    }
    if (ok && !ptx::mbar_wait(accum_bar, 0, p.err)) *abort_flag = 1;
  }

  // ---------------------------------------------------------------- epilogue
  // Every thread of the CTA gets here (all waits above are bounded), so the
  // barriers below, the cluster-wide ones included, are reached by all of them.
  __syncthreads();
  const bool fine = (*abort_flag == 0);
  const bool dec = warp >= 2;
  const int q = warp & 3, part = (warp - 2) >> 2;
  const int dr = 32 * q + lane, r = row0 + dr;
  const bool valid = r < N;
  const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16);
  const int nch = p.T / 16;  // 16-token chunks; thread (row dr, part) handles chunks part, part+P, ...
  if (p.epi != kEpiGlobal) {
    // y through a shared-memory staging tile ([chunk][16 tokens][128 rows] in the
    // codebook area, free now) and TMA tensor stores, which also clip the ragged
    // edges.  With a K-split pair (a 2-CTA cluster, rank = split) each CTA owns the
    // chunks of its parity and sends the others' fp32 sums into its partner's
    // receive area (the x stages, free now) over distributed shared memory.
    const bool pair = (p.epi == kEpiPair);
    const uint32_t rank = (uint32_t)split;
    auto recv_addr = [&](int ci, int i) { return base + kTcTilesOffset + (uint32_t)(ci >> 1) * 8192u + (uint32_t)(i * 128 + dr) * 4u; };
    auto stage_addr = [&](int ci, int i) { return base + (uint32_t)(ci * 16 + i) * 256u + (uint32_t)dr * 2u; };
    if (pair) {
      ptx::cluster_sync();  // both CTAs are done with their x stages
      if (dec && fine) {
        ptx::tc_fence_after();
        for (int ci = part; ci < nch; ci += kTcParts) {
          if ((uint32_t)(ci & 1) == rank || tok0 + 16 * ci >= M) continue;
          uint32_t v[16];
          ptx::tmem_ld16(taddr + 16 * ci, v);
          ptx::tmem_wait_ld();
          const uint32_t dst = ptx::map_shared_rank(recv_addr(ci, 0), rank ^ 1u);
#pragma unroll
          for (int i = 0; i < 16; ++i) ptx::st_cluster_f32(dst + (uint32_t)i * 512u, __uint_as_float(v[i]));
        }
      }
      ptx::cluster_sync();  // the partner's sums have arrived
    }
    if (dec && fine) {
      ptx::tc_fence_after();
      for (int ci = part; ci < nch; ci += kTcParts) {
        if ((pair && (uint32_t)(ci & 1) != rank) || tok0 + 16 * ci >= M) continue;
        uint32_t v[16];
        ptx::tmem_ld16(taddr + 16 * ci, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float f = __uint_as_float(v[i]);
          if (pair) {  // two splits: the sum does not depend on the order
            float o;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(o) : "r"(recv_addr(ci, i)));
            f += o;
          }
          // the sparse correction's x . C^T term, added before the one rounding
          if (a.addend && valid && tok0 + 16 * ci + i < M) f += a.addend[(int64_t)(tok0 + 16 * ci + i) * N + r];
          const uint16_t h = Elt<T>::from_f32(f);
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(stage_addr(ci, i)), "h"(h) : "memory");
        }
      }
      ptx::fence_proxy_async_smem();
    }
    __syncthreads();
    if (threadIdx.x == 64 && fine) {
      for (int ci = 0; ci < nch; ++ci) {
        if ((pair && (uint32_t)(ci & 1) != rank) || tok0 + 16 * ci >= M) continue;
        ptx::tma_store_2d(&ymap, base + (uint32_t)ci * 4096u, row0, tok0 + 16 * ci);
      }
      ptx::bulk_commit();
      ptx::bulk_wait_all();
    }
  } else if (dec) {
    // y (one split) or fp32 partials written per element; the last CTA of a split
    // tile, picked by an atomic ticket, sums the partials in split order.
    uint16_t* y = static_cast<uint16_t*>(a.y);
    if (fine) {
      ptx::tc_fence_after();
      for (int c0 = 16 * part; c0 < p.T; c0 += 16 * kTcParts) {
        uint32_t v[16];
        ptx::tmem_ld16(taddr + c0, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int tok = tok0 + c0 + i;
          if (tok >= M || !valid) continue;
          if (p.splits == 1)
            y[(int64_t)tok * N + r] =
                Elt<T>::from_f32(a.addend ? __uint_as_float(v[i]) + a.addend[(int64_t)tok * N + r] : __uint_as_float(v[i]));
          else
            p.partial[((int64_t)split * M + tok) * N + r] = __uint_as_float(v[i]);
        }
      }
      ptx::tc_fence_before();
    }
    if (fine && p.splits > 1) {
      __threadfence();
      asm volatile("bar.sync 1, %0;" ::"n"(32 * 4 * kTcParts) : "memory");
      const int tile = blockIdx.y * gridDim.x + blockIdx.x;
      if (threadIdx.x == 64) *last_flag = (atomicAdd(&p.tickets[tile], 1u) == (uint32_t)(p.splits - 1));
      asm volatile("bar.sync 1, %0;" ::"n"(32 * 4 * kTcParts) : "memory");
      if (*last_flag) {
        __threadfence();
        ptx::tc_fence_after();
        // Sixteen tokens per step, so each split's loads are all in flight at
        // once; this CTA's own split comes from its accumulator.
        for (int c0 = 16 * part; c0 < p.T; c0 += 16 * kTcParts) {
          float acc[16];
          for (int k = 0; k < p.splits; ++k) {
            uint32_t t[16];
            if (k == split) {
              ptx::tmem_ld16(taddr + c0, t);
              ptx::tmem_wait_ld();
            } else {
              const float* src = p.partial + ((int64_t)k * M + tok0 + c0) * N + r;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                t[i] = (valid && tok0 + c0 + i < M) ? __float_as_uint(__ldcg(src + (int64_t)i * N)) : 0u;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = k == 0 ? __uint_as_float(t[i]) : acc[i] + __uint_as_float(t[i]);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (valid && tok0 + c0 + i < M)
              y[(int64_t)(tok0 + c0 + i) * N + r] =
                  Elt<T>::from_f32(a.addend ? acc[i] + a.addend[(int64_t)(tok0 + c0 + i) * N + r] : acc[i]);
        }
        ptx::tc_fence_before();
        if (threadIdx.x == 64) p.tickets[tile] = 0u;
      }
    }
  }
  ptx::tc_fence_before();
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
  int T, TT, RT, S, kps, epi;
  bool dual;  // two CTAs per SM (2 decode warps per lane quarter; 3 stages for 64-token tiles)
};

// fmt: kFmt* (the same values as VQ_FMT_*).
static TcGeom tc_geom(int fmt, int M, int N, int K, int num_sms) {
  TcGeom g;
  const int m16 = (M + 15) / 16 * 16;
  g.T = m16 < kTcMaxT ? m16 : kTcMaxT;
  g.TT = (M + g.T - 1) / g.T;
  g.dual = g.T <= 64 && fmt != kFmtVq16 && fmt != kFmtVq16Rvq;
  g.RT = (N + kTcRows - 1) / kTcRows;
  const int tiles = g.RT * g.TT;
  const int nsl = (K + 127) / 128;  // splits start on 128-input slice boundaries
  auto splits = [&](int slots) {
    int S = slots / tiles;
    if (S < 1) S = 1;
    if (S > 8) S = 8;
    return S > nsl ? nsl : S;
  };
  int S = splits(g.dual ? 2 * num_sms : num_sms);
  // 64-token tiles: two CTAs per SM only while the K split stays a cluster pair
  // (Llama-3-8B gate M = 64: 28.3 vs 32.7 us; 8192 x 8192 M = 64, where it would
  // take four splits with partial sums in global memory: 36.6 vs 33.5 us).
  if (g.dual && g.T == 64 && S > 2) {
    g.dual = false;
    S = splits(num_sms);
  }
  const int sps = (nsl + S - 1) / S;
  g.S = (nsl + sps - 1) / sps;
  g.kps = sps * 128;
  // TMA stores of y need 16-byte row pitches (N % 8 == 0).
  g.epi = (N % 8 != 0 || g.S > 2) ? kEpiGlobal : (g.S == 2 ? kEpiPair : kEpiStore);
  return g;
}

bool plan_tc(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  if (M < 1 || dev.smem_optin < (int)kTcSmemMax) return false;
  const TcGeom g = tc_geom(d.fmt, M, d.N, d.K, dev.num_sms);
  p->path = VQ_PATH_TC;
  p->splits = g.S;
  p->k_per_split = g.kps;
  p->launches = 1;
  const bool partials = g.S > 1 && g.epi == kEpiGlobal;
  p->scratch_bytes = partials ? (size_t)g.S * M * d.N * sizeof(float) : 0;
  p->tickets = partials ? g.RT * g.TT : 0;
  p->ctas = g.RT * g.TT * g.S;
  return true;
}

template <int FMT, typename T, bool kStaged, int kParts, int kSt = kTcStages>
static cudaError_t launch_tc_t(const LayerArgs& a, const TcGeom& g, float* scratch, uint32_t* tickets,
                               uint32_t* err, cudaStream_t s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map, ymap;
  const CUtensorMapDataType dt =
      a.act == VQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
  const cuuint64_t strides[1] = {(cuuint64_t)a.K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)g.T};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, dt, 2, const_cast<void*>(a.x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  ymap = map;  // unused unless the epilogue stores y by TMA
  if (g.epi != kEpiGlobal) {
    const cuuint64_t ydims[2] = {(cuuint64_t)a.N, (cuuint64_t)a.M};
    const cuuint64_t ystrides[1] = {(cuuint64_t)a.N * 2};
    const cuuint32_t ybox[2] = {(cuuint32_t)kTcRows, 16};
    r = enc(&ymap, dt, 2, a.y, ydims, ystrides, ybox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  const uint32_t smem = kTcTilesOffset + kSt * ((uint32_t)g.T * 128u) + 1024u;
  auto kern = tc_gemm_kernel<FMT, T, kStaged, kParts, kSt>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (kParts == 2) {  // two CTAs per SM: the whole carve-out as shared memory
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
  }
  const bool partials = g.S > 1 && g.epi == kEpiGlobal;
  TcArgs p{a, g.epi, g.T, g.kps, g.S, partials ? scratch : nullptr, partials ? tickets : nullptr, err};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.RT, g.TT, g.S);
  cfg.blockDim = dim3(tc_threads(kParts));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (g.epi == kEpiPair) {  // the two K-splits of a tile form one cluster
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 2;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, kern, map, ymap, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int FMT, typename T>
static cudaError_t launch_tc_s(const LayerArgs& a, const TcGeom& g, float* scratch, uint32_t* tickets,
                               uint32_t* err, cudaStream_t s) {
  // Bulk copies need 16-byte sizes: N % 8 == 0 makes every per-slice run one.
  // Token tiles of 64 and more: 3 decode warps per quarter (14 warps, 128 registers
  // each, no spills: the decode keeps up with the longer MMAs of a wide tile;
  // 8192 x 8192 M = 256: 39.5 vs 43.1 us with 4).  The 12-bit formats' tiles of 16
  // to 48 tokens, and of 64 when the split stays a cluster pair (tc_geom): 2 per
  // quarter (10 warps, 96 registers) and two CTAs per SM, each with its own decode
  // -> MMA pipeline (64-token tiles with three x stages, so that two fit in shared
  // memory); tc_geom counts two slots per SM, so the Llama-3-8B gate at M = 16
  // splits K over a cluster pair and fills every SM (27.4 vs 31.3 us with one
  // CTA of 4 decode warps per quarter per SM; down 31.2 vs 32.5; the gate at
  // M = 64 28.3 vs 32.7 with one CTA of 3).  The 16-bit
  // formats keep one CTA of 4 per quarter (18 warps, 96 registers): two CTAs'
  // shared memory leaves too little L1 for their codeword gathers from the
  // 1 MiB codebook (4096 x 4096 M = 8: 29.2 vs 18 us).
  if constexpr (FMT != kFmtVq16) {
    if (g.dual && g.T == 64)  // two 64-token CTAs fit in shared memory with three x stages
      return (a.N % 8 == 0) ? launch_tc_t<FMT, T, true, 2, 3>(a, g, scratch, tickets, err, s)
                            : launch_tc_t<FMT, T, false, 2, 3>(a, g, scratch, tickets, err, s);
    if (g.dual)
      return (a.N % 8 == 0) ? launch_tc_t<FMT, T, true, 2>(a, g, scratch, tickets, err, s)
                            : launch_tc_t<FMT, T, false, 2>(a, g, scratch, tickets, err, s);
  }
  if (g.T >= 64)
    return (a.N % 8 == 0) ? launch_tc_t<FMT, T, true, 3>(a, g, scratch, tickets, err, s)
                          : launch_tc_t<FMT, T, false, 3>(a, g, scratch, tickets, err, s);
  return (a.N % 8 == 0) ? launch_tc_t<FMT, T, true, 4>(a, g, scratch, tickets, err, s)
                        : launch_tc_t<FMT, T, false, 4>(a, g, scratch, tickets, err, s);
}

cudaError_t launch_tc(const LayerArgs& a, const Plan& pl, float* scratch, uint32_t* tickets, uint32_t* err,
                      cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const TcGeom g = tc_geom(a.fmt, a.M, a.N, a.K, sms);
  if (g.S != pl.splits) return cudaErrorInvalidValue;
  const bool bf = a.act == VQ_BF16;
  switch (a.fmt) {
    case kFmtRvq12:
      return bf ? launch_tc_s<kFmtRvq12, __nv_bfloat16>(a, g, scratch, tickets, err, s)
                : launch_tc_s<kFmtRvq12, __half>(a, g, scratch, tickets, err, s);
    case kFmtRvq12_4:
      return bf ? launch_tc_s<kFmtRvq12_4, __nv_bfloat16>(a, g, scratch, tickets, err, s)
                : launch_tc_s<kFmtRvq12_4, __half>(a, g, scratch, tickets, err, s);
    case kFmtVq16Rvq:  // the ladder's indices are read directly (no staging ring)
      if (g.T >= 64)
        return bf ? launch_tc_t<kFmtVq16Rvq, __nv_bfloat16, false, 3>(a, g, scratch, tickets, err, s)
                  : launch_tc_t<kFmtVq16Rvq, __half, false, 3>(a, g, scratch, tickets, err, s);
      return bf ? launch_tc_t<kFmtVq16Rvq, __nv_bfloat16, false, 4>(a, g, scratch, tickets, err, s)
                : launch_tc_t<kFmtVq16Rvq, __half, false, 4>(a, g, scratch, tickets, err, s);
    default:
      return bf ? launch_tc_s<kFmtVq16, __nv_bfloat16>(a, g, scratch, tickets, err, s)
                : launch_tc_s<kFmtVq16, __half>(a, g, scratch, tickets, err, s);
  }
}

}  // namespace vq

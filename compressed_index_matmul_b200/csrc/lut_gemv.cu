// Batch-1 GEMV by per-group lookup tables (M == 1, 12-bit formats, K % 128 == 0,
// N % 4 == 0).
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
// those MMAs does not depend on x: the codebook is bulk-copied once into the table
// area (free until the first build), each warp takes its share into registers with
// ldmatrix, and every rebuild is only MMAs and stores.
//
// Work distribution: the (K-slice, row) pairs in slice-major order are cut into
// one contiguous, equal range per CTA of a persistent grid (at most one CTA per
// SM), so every CTA sweeps the same number of rows and rebuilds its tables at
// most once more than the others.  A range is walked in chunks of up to 512 rows
// that never cross a slice; in the K-slice-major storage a chunk's index bytes
// are one contiguous run per plane.  A producer warp streams the chunks into a
// ring of shared-memory stages with bulk copies (TMA), several chunks ahead, and
// 8 lookup warps consume them (full / empty mbarriers per stage, no CTA-wide
// barrier per chunk).  Lookup thread t handles rows t and t+256 of a chunk and
// writes one fp32 partial sum per row and slice.
//
// Split-K reduction: after the last chunk every CTA meets at a grid-wide barrier
// (the launch is cooperative, so all CTAs are resident together: the grid never
// exceeds the SM count); then each CTA sums the partials of its own share
// of the rows with a fixed tree (GLQ README, "Inference kernels": fixed-order
// split-K reduction, no floating-point atomics), so y does not depend on
// scheduling.  One launch per forward.
//
// Activations are scaled by one power of two per K-slice (the slice's largest
// |x| lands in [2^14, 2^15)), so the fp16 MMA operand is exact for either
// activation type except for values more than 2^31 below that maximum; the
// factor is undone once per (slice, row) partial, exactly.
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace vq {

constexpr int kLutGroups = 16;                 // groups per K-slice (128 inputs)
constexpr int kLutConsumers = 256;             // lookup threads (8 warps)
constexpr int kLutThreads = kLutConsumers + 32;  // + one producer warp
constexpr int kLutChunkRows = 512;             // rows per chunk (two per lookup thread)
constexpr int kLutTableBytes = 4096 * 2 + 64;  // one group's T1 (bf16) + pad (bank spread)
constexpr int kLutStages = 4;                  // bulk-copy ring depth (chunks in flight)
constexpr int kLutMaxX = 4;                    // x slices preloaded per CTA
// one ring stage: lo 16 B, hi4 8 B, s2 8 B, scales 4 B per row
constexpr int kLutOffHi = kLutChunkRows * 16;
constexpr int kLutOffS2 = kLutOffHi + kLutChunkRows * 8;
constexpr int kLutOffSc = kLutOffS2 + kLutChunkRows * 8;
constexpr int kLutStageBytes = kLutOffSc + kLutChunkRows * 4;
constexpr int kLutOffT2 = kLutGroups * kLutTableBytes;
constexpr int kLutOffMisc = kLutOffT2 + kLutGroups * 16 * 4;  // barriers, flags
constexpr int kLutOffRing = kLutOffMisc + 256;
constexpr int kLutSmem = kLutOffRing + kLutStages * kLutStageBytes;

// A table build, counted in rows of lookups of equal cost, when the (slice, row)
// sequence is split over the CTAs.
constexpr int kLutBuildRows = 640;

// Walks one CTA's range of (slice, row) positions in chunks that stay inside a
// slice and hold at most kLutChunkRows rows (a multiple of 4, as N is).  The
// ranges are equal in "virtual" rows: each slice is preceded by kLutBuildRows
// virtual rows standing for its table build, so a CTA whose range spans a slice
// start gets correspondingly fewer real rows.
struct LutChunks {
  int s, r;  // next chunk's slice and first row
  int64_t pos, end;
  static __device__ int64_t real_pos(int64_t v, int N) {
    const int64_t span = (int64_t)N + kLutBuildRows;
    const int64_t sl = v / span, off = v - sl * span;
    return sl * N + (off > kLutBuildRows ? off - kLutBuildRows : 0);
  }
  __device__ void init(int N, int S, int cta, int grid) {
    const int64_t total = (int64_t)S * N, vtotal = (int64_t)S * ((int64_t)N + kLutBuildRows);
    pos = real_pos(vtotal * cta / grid, N) & ~int64_t(3);
    end = cta == grid - 1 ? total : (real_pos(vtotal * (cta + 1) / grid, N) & ~int64_t(3));
    s = (int)(pos / N);
    r = (int)(pos - (int64_t)s * N);
  }
  __device__ bool next(int N, int& cs, int& cr, int& rows) {
    if (pos >= end) return false;
    const int64_t left = end - pos;
    rows = min(kLutChunkRows, N - r);
    if (left < rows) rows = (int)left;
    cs = s;
    cr = r;
    pos += rows;
    r += rows;
    if (r == N) {
      r = 0;
      ++s;
    }
    return true;
  }
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// D = A.B with a zero accumulator (fp16 in, fp32 out).
__device__ __forceinline__ void mma_16808_f16(float d[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0), "f"(0.f));
}

// Sum of the 16 lookups of one row's slice record (lo 16 B, hi4 8 B, s2 8 B),
// split by 64-input block.
template <bool kTwo>
__device__ __forceinline__ void lookup_row(const uint4& lo4, const uint2& h, const uint2& q,
                                           const unsigned char* __restrict__ t1, const float* __restrict__ t2,
                                           float blk[2]) {
  const uint32_t low[4] = {lo4.x, lo4.y, lo4.z, lo4.w};
  const uint32_t hiw[2] = {h.x, h.y};
  const uint32_t s2w[2] = {q.x, q.y};
  blk[0] = blk[1] = 0.f;
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const uint32_t hE = hiw[w] & 0x0F0F0F0Fu, hO = (hiw[w] >> 4) & 0x0F0F0F0Fu;
    const uint32_t sE = (s2w[w] & 0x0F0F0F0Fu) << 2, sO = ((s2w[w] >> 4) & 0x0F0F0F0Fu) << 2;
#pragma unroll
    for (int qq = 0; qq < 8; ++qq) {
      const int t = 8 * w + qq;  // group within the slice
      const uint32_t hsel = 4 + (qq >> 1);
      // bytes: lo byte t, hi nibble t, then two zero bytes (sign copies of a nibble byte)
      const uint32_t sel = (uint32_t)(t & 3) | (hsel << 4) | ((8u | hsel) << 8) | ((8u | hsel) << 12);
      const uint32_t i1 = prmt(low[t >> 2], (qq & 1) ? hO : hE, sel);
      // plain shared-memory loads: the compiler may issue all of a row's lookups
      // before the additions that consume them
      float v = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(t1 + t * kLutTableBytes + i1 * 2) << 16);
      if (kTwo) {
        const uint32_t b = qq >> 1;
        const uint32_t bsel = b | ((8u | b) << 4) | ((8u | b) << 8) | ((8u | b) << 12);
        v += *reinterpret_cast<const float*>(reinterpret_cast<const unsigned char*>(t2) + t * 64 +
                                             prmt((qq & 1) ? sO : sE, 0, bsel));
      }
      blk[w] += v;
    }
  }
}

template <int FMT, typename T>
__global__ void __launch_bounds__(kLutThreads, 1)
    lut_gemv_kernel(LayerArgs a, float* __restrict__ partial, uint32_t* __restrict__ sync, uint32_t* __restrict__ err,
                    int S) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr bool kTwo = (FMT == kFmtRvq12_4);
  unsigned char* t1 = smem;
  float* t2 = reinterpret_cast<float*>(smem + kLutOffT2);
  const uint32_t full0 = smem_u32(smem + kLutOffMisc + 64);         // [kLutStages] mbarriers: chunk landed
  const uint32_t empty0 = smem_u32(smem + kLutOffMisc + 96);        // [kLutStages] mbarriers: chunk consumed
  volatile int* abortf = reinterpret_cast<volatile int*>(smem + kLutOffMisc + 128);  // a bounded wait gave up
  const uint32_t cb_bar = smem_u32(smem + kLutOffMisc + 136);       // codebook copy landed
  const uint32_t t1_base = smem_u32(t1), ring_base = smem_u32(smem + kLutOffRing);

  const int N = a.N;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool block_scales = (a.scale_group == 64);
  const uint16_t* xg = static_cast<const uint16_t*>(a.x);
  LutChunks chunks;
  chunks.init(N, S, blockIdx.x, gridDim.x);
  const int s_first = chunks.s;

  if (tid == 0) {
    for (int i = 0; i < kLutStages; ++i) {
      ptx::mbar_init(full0 + 8 * i, 1);
      ptx::mbar_init(empty0 + 8 * i, kLutConsumers / 32);
    }
    ptx::mbar_init(cb_bar, 1);
    *abortf = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (warp == kLutConsumers / 32) {
    // ------------------------------------------------------------ producer
    // Reads only the layer's constant index planes and scales, so it may run
    // while the previous kernel in the stream is still finishing.
    if (lane == 0) {
      // The stage-1 codebook into the table area (free until the first build),
      // where the lookup warps read their MMA operands from it.
      ptx::mbar_arrive_expect_tx(cb_bar, 65536u);
      ptx::bulk_load(t1_base, a.cb1, 65536u, cb_bar);
      int k = 0, cs, cr, rows;
      while (chunks.next(N, cs, cr, rows)) {
        const int st = k % kLutStages;
        if (*abortf || (k >= kLutStages && !ptx::mbar_wait(empty0 + 8 * st, ((k / kLutStages) - 1) & 1, err))) {
          *abortf = 1;
          break;
        }
        const uint32_t dst = ring_base + st * kLutStageBytes, bar = full0 + 8 * st;
        const int64_t e = (int64_t)16 * cs * N + (int64_t)16 * cr;  // lo entry of (slice cs, row cr)
        ptx::mbar_arrive_expect_tx(bar, rows * (16 + 8 + (kTwo ? 8 : 0) + (block_scales ? 4 : 0)));
        ptx::bulk_load(dst, a.lo + e, rows * 16, bar);
        ptx::bulk_load(dst + kLutOffHi, a.hi4 + e / 2, rows * 8, bar);
        if (kTwo) ptx::bulk_load(dst + kLutOffS2, a.s2 + e / 2, rows * 8, bar);
        if (block_scales) ptx::bulk_load(dst + kLutOffSc, a.scales + e / 8, rows * 4, bar);  // 2 per row per slice
        ++k;
      }
      // Do not leave copies into this CTA's shared memory in flight.
      for (int i = (k > kLutStages ? k - kLutStages : 0); i < k; ++i)
        ptx::mbar_wait(full0 + 8 * (i % kLutStages), (i / kLutStages) & 1, err);
      ptx::mbar_wait(cb_bar, 0, err);
    }
  } else {
    // ------------------------------------------------------------ lookups
    // Codebook operand of the table MMAs, held for the whole kernel: warp w covers
    // codewords 512w .. 512w+511 in 16 blocks of 32; see the build below.
    const int g = lane >> 2, c = lane & 3;
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
    // Everything above reads only the layer's constant inputs; x and the scratch
    // are touched only after the previous kernel completed.  The x loads go out
    // before the wait for the codebook copy, so the two latencies overlap.  Every
    // warp holds a whole x slice: lane l has inputs 4l .. 4l+3 of it.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint2 xpre[kLutMaxX];
#pragma unroll
    for (int i = 0; i < kLutMaxX; ++i) {
      const int s = s_first + i;
      xpre[i] = s < S ? *reinterpret_cast<const uint2*>(xg + (int64_t)s * 128 + 4 * lane) : make_uint2(0, 0);
    }

    uint32_t bfrag[16][4];
    {
      // ldmatrix: lanes 8j..8j+7 give the rows (codewords) of matrix j; lane (g, c)
      // receives word c of row g of each matrix, the MMA B fragment.
      if (!ptx::mbar_wait(cb_bar, 0, err)) *abortf = 1;
      const int n = lane & 7, jm = lane >> 3;
#pragma unroll
      for (int it = 0; it < 16; ++it) {
        const uint32_t addr = t1_base + (uint32_t)(warp * 512 + it * 32 + 8 * (n >> 1) + 2 * jm + (n & 1)) * 16u;
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                     : "=r"(bfrag[it][0]), "=r"(bfrag[it][1]), "=r"(bfrag[it][2]), "=r"(bfrag[it][3])
                     : "r"(addr));
      }
    }

    // Every lookup thread walks the same chunk sequence as the producer, so all
    // of them rebuild the tables at the same chunks (the named barriers below are
    // reached by all 256 or by none).  After a wait gives up the rest of the walk
    // skips the waits (the result is then wrong and the error word is set).
    int cur = -1, s, r0, rows;
    float unscale = 1.f;  // 2^-e of the current slice
    for (int k = 0; chunks.next(N, s, r0, rows); ++k) {
      const int st = k % kLutStages;
      // A new slice's tables need only x and the codebook, so they are built
      // before the wait for the chunk's index bytes.
      if (s != cur) {
        // ------------------------------------------------------------ build
        asm volatile("bar.sync 1, %0;" ::"n"(kLutConsumers) : "memory");  // everyone is done with the old tables
        uint2 xw;
        {
          const int i = s - s_first;
          if (i < kLutMaxX) {
            xw = xpre[0];
#pragma unroll
            for (int kk = 1; kk < kLutMaxX; ++kk)
              if (kk == i) xw = xpre[kk];
          } else {
            xw = *reinterpret_cast<const uint2*>(xg + (int64_t)s * 128 + 4 * lane);
          }
        }
        // One power of two 2^e per slice puts the slice's largest |x| in [2^14, 2^15),
        // so the fp16 MMA operand is exact (bar values 2^31 below it) for either
        // activation type; T1 and T2 are built from 2^e x and every partial is
        // multiplied by 2^-e (exact).
        float m = fmaxf(fmaxf(fabsf(Elt<T>::to_f32((uint16_t)xw.x)), fabsf(Elt<T>::to_f32((uint16_t)(xw.x >> 16)))),
                        fmaxf(fabsf(Elt<T>::to_f32((uint16_t)xw.y)), fabsf(Elt<T>::to_f32((uint16_t)(xw.y >> 16)))));
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        // e = 15 - (exponent of m as frexpf gives it), taken from the bits for
        // normal m (zero, inf and NaN get no scaling); clamped so 2^e and 2^-e are
        // normal floats.
        const int be = (int)(__float_as_uint(m) >> 23);  // biased exponent (sign bit is 0)
        int e = 0;
        if (be > 0 && be < 255) {
          e = min(100, max(-100, 15 - (be - 126)));
        } else if (be == 0 && m > 0.f) {  // subnormal: rare, take the library route
          frexpf(m, &e);
          e = min(100, max(-100, 15 - e));
        }
        const float up = __uint_as_float((uint32_t)(127 + e) << 23);
        unscale = __uint_as_float((uint32_t)(127 - e) << 23);
        // A operand (x slice, 16 groups x 8 dims, fp16): lane (g, c) needs inputs
        // 8g+2c, 8g+2c+1 (held by lane 2g + c/2) and the same of group g+8.
        uint32_t a0, a1;
        {
          const int src0 = 2 * g + (c >> 1), src1 = src0 + 16;
          const uint32_t u0 = __shfl_sync(0xffffffffu, xw.x, src0), v0 = __shfl_sync(0xffffffffu, xw.y, src0);
          const uint32_t u1 = __shfl_sync(0xffffffffu, xw.x, src1), v1 = __shfl_sync(0xffffffffu, xw.y, src1);
          const uint32_t p0 = (c & 1) ? v0 : u0, p1 = (c & 1) ? v1 : u1;
          a0 = Elt<__half>::pack(Elt<T>::to_f32((uint16_t)p0) * up, Elt<T>::to_f32((uint16_t)(p0 >> 16)) * up);
          a1 = Elt<__half>::pack(Elt<T>::to_f32((uint16_t)p1) * up, Elt<T>::to_f32((uint16_t)(p1 >> 16)) * up);
        }
        if (kTwo) {
          // T2[gg][ee] = 2^e x_gg . cb2[ee] for thread gg*16 + ee; group gg's inputs
          // are held by lanes 2gg and 2gg+1.
          const int src = 2 * (tid >> 4);  // lane 2gg (every warp holds the whole slice)
          const uint32_t q[4] = {__shfl_sync(0xffffffffu, xw.x, src), __shfl_sync(0xffffffffu, xw.y, src),
                                 __shfl_sync(0xffffffffu, xw.x, src + 1), __shfl_sync(0xffffffffu, xw.y, src + 1)};
          float acc = 0.f;
#pragma unroll
          for (int d = 0; d < 4; ++d) {
            acc = fmaf(Elt<T>::to_f32((uint16_t)q[d]), c2v[2 * d], acc);
            acc = fmaf(Elt<T>::to_f32((uint16_t)(q[d] >> 16)), c2v[2 * d + 1], acc);
          }
          t2[tid] = acc * up;
        }
        {
          // Column n of MMA j in block `it` is codeword base + 8*(n/2) + 2j + (n%2), so
          // lane (g, c) ends with codewords base+8c .. base+8c+7 of groups g and g+8:
          // one 16-byte store each.
#pragma unroll
          for (int it = 0; it < 16; ++it) {
            const int base = warp * 512 + it * 32;
            float d[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) mma_16808_f16(d[j], a0, a1, bfrag[it][j]);
            typedef Elt<__nv_bfloat16> B16;
            const uint4 lo = make_uint4(B16::pack(d[0][0], d[0][1]), B16::pack(d[1][0], d[1][1]),
                                        B16::pack(d[2][0], d[2][1]), B16::pack(d[3][0], d[3][1]));
            const uint4 hi = make_uint4(B16::pack(d[0][2], d[0][3]), B16::pack(d[1][2], d[1][3]),
                                        B16::pack(d[2][2], d[2][3]), B16::pack(d[3][2], d[3][3]));
            *reinterpret_cast<uint4*>(t1 + g * kLutTableBytes + (base + 8 * c) * 2) = lo;
            *reinterpret_cast<uint4*>(t1 + (g + 8) * kLutTableBytes + (base + 8 * c) * 2) = hi;
          }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kLutConsumers) : "memory");
        cur = s;
      }
      if (*abortf || !ptx::mbar_wait(full0 + 8 * st, (uint32_t)((k / kLutStages) & 1), err)) *abortf = 1;

      // -------------------------------------------------------------- lookups
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int lr = tid + 256 * h, r = r0 + lr;
        if (lr >= rows) continue;
        const unsigned char* sp = smem + kLutOffRing + st * kLutStageBytes;
        const uint4 lo4 = *reinterpret_cast<const uint4*>(sp + 16 * lr);
        const uint2 hh = *reinterpret_cast<const uint2*>(sp + kLutOffHi + 8 * lr);
        const uint2 qq = kTwo ? *reinterpret_cast<const uint2*>(sp + kLutOffS2 + 8 * lr) : make_uint2(0, 0);
        const uint32_t scw = block_scales ? *reinterpret_cast<const uint32_t*>(sp + kLutOffSc + 4 * lr) : 0u;
        float blk[2];
        lookup_row<kTwo>(lo4, hh, qq, t1, t2, blk);
        float acc;
        if (block_scales) {
          const float2 sc = f16x2_to_f32x2(scw);
          acc = fmaf(blk[1], sc.y, blk[0] * sc.x) * unscale;
        } else {
          acc = (blk[0] + blk[1]) * unscale;  // the per-row scale is applied once, at the reduction
        }
        if (S == 1) {
          if (!block_scales) acc *= f16_bits_to_f32(a.scales[r]);
          if (a.addend) acc += a.addend[r];  // the sparse correction's x . C^T term
          static_cast<uint16_t*>(a.y)[r] = Elt<T>::from_f32(acc);
        } else {
          partial[(int64_t)s * N + r] = acc;
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(empty0 + 8 * st);  // this warp is done with stage st
    }
  }
  if (S == 1) {
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    return;
  }

  // --------------------------------------------------- grid barrier + reduce
  // A self-resetting barrier on two handle words: an arrival counter and a
  // generation.  Each CTA reads the generation before it arrives (it cannot
  // change before every CTA of this launch, this one included, has arrived); the
  // CTA whose arrival completes the grid zeroes the counter and advances the
  // generation, and the others wait for that.  No CTA reads a count that other
  // CTAs of the same launch may already have changed, whenever it started.  The
  // CTA barrier orders every thread's partial stores before thread 0's arrival
  // (release); thread 0's acquire and the second CTA barrier order all CTAs'
  // partial stores before every thread's reads below.
  __syncthreads();
  if (tid == 0) {
    uint32_t* cnt = sync;
    uint32_t* gen = sync + 1;
    uint32_t g0, old;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(g0) : "l"(gen) : "memory");
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(cnt) : "memory");
    if (old == gridDim.x - 1) {
      *cnt = 0;  // every CTA has arrived: nothing else touches it in this launch
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(gen), "r"(g0 + 1) : "memory");
    } else {
      const uint64_t t0 = ptx::globaltimer_ns();
      bool released = false;
      for (uint32_t i = 0; i < kWaitSpinLimit; ++i) {
        uint32_t g;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g) : "l"(gen) : "memory");
        if (g != g0) {
          released = true;
          break;
        }
        if ((i & 63u) == 63u && ptx::globaltimer_ns() - t0 > 1000000000ull) break;
      }
      if (!released) atomicOr(err, kErrTimeout);
    }
  }
  __syncthreads();
  // Every CTA of this grid has passed the barrier, so all of them are resident:
  // the next kernel in the stream may launch now and take each SM as its CTA here
  // exits (it reads x, y and the scratch only after this grid completes).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // This CTA's rows, in quads (N % 4 == 0): tpr threads per quad split the slices
  // (at most 8 each, one batch of independent 16-byte loads, when the CTA has the
  // threads for it), then a fixed xor tree combines the parts.
  const int Q = N / 4;
  const int qbeg = (int)((int64_t)Q * blockIdx.x / gridDim.x), qend = (int)((int64_t)Q * (blockIdx.x + 1) / gridDim.x);
  const int nq = qend - qbeg;
  int tpr = 1;
  while (tpr < 32 && (S + tpr - 1) / tpr > 8 && 2 * tpr * nq <= kLutThreads) tpr *= 2;
  const int per = (S + tpr - 1) / tpr;
  for (int base = 0; base < nq * tpr; base += kLutThreads) {
    const int idx = base + tid;
    const int q = idx / tpr, part = idx % tpr;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    if (q < nq) {
      const int r = 4 * (qbeg + q);
      const int k0 = part * per, k1 = min(S, k0 + per);
      constexpr int kBatch = 8;
      for (int kb = k0; kb < k1; kb += kBatch) {
        float4 v[kBatch];
        const float4* src = reinterpret_cast<const float4*>(partial + (int64_t)kb * N + r);
        if (k1 - kb >= kBatch) {  // a full batch: unpredicated loads, all in flight at once
#pragma unroll
          for (int j = 0; j < kBatch; ++j) v[j] = __ldcg(src + (int64_t)j * (N / 4));
        } else {
#pragma unroll
          for (int j = 0; j < kBatch; ++j)
            v[j] = (kb + j < k1) ? __ldcg(src + (int64_t)j * (N / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          if (kb + j < k1) {
            sum.x += v[j].x;
            sum.y += v[j].y;
            sum.z += v[j].z;
            sum.w += v[j].w;
          }
      }
    }
    for (int o = 1; o < tpr; o <<= 1) {
      sum.x += __shfl_xor_sync(0xffffffffu, sum.x, o);
      sum.y += __shfl_xor_sync(0xffffffffu, sum.y, o);
      sum.z += __shfl_xor_sync(0xffffffffu, sum.z, o);
      sum.w += __shfl_xor_sync(0xffffffffu, sum.w, o);
    }
    if (q < nq && part == 0) {
      const int r = 4 * (qbeg + q);
      float o4[4] = {sum.x, sum.y, sum.z, sum.w};
      if (!block_scales) {
#pragma unroll
        for (int i = 0; i < 4; ++i) o4[i] *= f16_bits_to_f32(a.scales[r + i]);
      }
      if (a.addend) {  // the sparse correction's x . C^T term
#pragma unroll
        for (int i = 0; i < 4; ++i) o4[i] += a.addend[r + i];
      }
      uint16_t* yr = static_cast<uint16_t*>(a.y) + r;
      *reinterpret_cast<uint2*>(yr) =
          make_uint2((uint32_t)Elt<T>::from_f32(o4[0]) | ((uint32_t)Elt<T>::from_f32(o4[1]) << 16),
                     (uint32_t)Elt<T>::from_f32(o4[2]) | ((uint32_t)Elt<T>::from_f32(o4[3]) << 16));
    }
  }
}

struct LutGeom {
  int S, grid;
};

static LutGeom lut_geom(int N, int K, int num_sms) {
  LutGeom g;
  g.S = K / (8 * kLutGroups);
  // Enough (slice, row) work for every CTA to sweep a few hundred rows.
  const int64_t rows = (int64_t)g.S * N;
  const int64_t want = (rows + 255) / 256;
  g.grid = (int)(want < num_sms ? (want < 1 ? 1 : want) : num_sms);
  return g;
}

bool plan_lut(const vq_linear_desc& d, const DeviceInfo& dev, int M, Plan* p) {
  if (M != 1 || d.fmt == VQ_FMT_VQ16 || d.fmt == VQ_FMT_VQ16_RVQ || d.K % (8 * kLutGroups) != 0 || d.N % 4 != 0 || dev.smem_optin < kLutSmem)
    return false;
  const LutGeom g = lut_geom(d.N, d.K, dev.num_sms);
  p->path = VQ_PATH_LUT;
  p->splits = g.S;
  p->k_per_split = kLutGroups * 8;
  p->launches = 1;
  p->scratch_bytes = g.S > 1 ? (size_t)g.S * d.N * sizeof(float) : 0;
  p->tickets = 0;
  p->sync_words = g.S > 1 ? 2 : 0;  // the grid barrier's arrival counter and generation
  p->grid = g.grid;
  p->ctas = g.grid;
  return true;
}

template <int FMT, typename T>
static cudaError_t launch_lut_t(const LayerArgs& a, int grid, float* scratch, uint32_t* sync, uint32_t* err,
                                cudaStream_t s) {
  const int S = a.K / (8 * kLutGroups);
  auto kern = lut_gemv_kernel<FMT, T>;
  // The shared-memory opt-in is a per-device property of the function: set it
  // once per device (repeating it from two threads is harmless).
  static std::atomic<uint64_t> opted{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (!(opted.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmem);
    if (e != cudaSuccess) return e;
    opted.fetch_or(bit, std::memory_order_acq_rel);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kLutThreads);
  cfg.dynamicSmemBytes = kLutSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // prologue overlaps the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  // The CTAs meet at a grid barrier: a cooperative launch makes them all resident
  // together even beside other work on the GPU (the grid never exceeds the SM
  // count and a CTA takes a whole SM's shared memory).
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a, S > 1 ? scratch : nullptr, sync, err, S);
}

cudaError_t launch_lut(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* sync, uint32_t* err,
                       cudaStream_t s) {
  if (a.fmt == kFmtRvq12_4)
    return a.act == VQ_BF16 ? launch_lut_t<kFmtRvq12_4, __nv_bfloat16>(a, p.grid, scratch, sync, err, s)
                            : launch_lut_t<kFmtRvq12_4, __half>(a, p.grid, scratch, sync, err, s);
  return a.act == VQ_BF16 ? launch_lut_t<kFmtRvq12, __nv_bfloat16>(a, p.grid, scratch, sync, err, s)
                          : launch_lut_t<kFmtRvq12, __half>(a, p.grid, scratch, sync, err, s);
}

}  // namespace vq

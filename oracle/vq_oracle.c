/*
 * vq_oracle.c -- plain, slow CPU oracle for the codebook-VQ linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file: it is used by tests/, by __graft_entry__.smoke() (to check one tiny
 * GPU call) and by bench.py's cpu_baseline / reference arm.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes, and where the pages define it:
 *   - orka README, "How it works": every group of 8 consecutive weights is one
 *     codebook index; indices are stored as 12-bit bit-planes (a low-byte plane
 *     plus a packed high plane); decode is scale x sum over stages of
 *     codebook_s[index_s].  "rvq-12-4" is a 12-bit stage 1 plus a 4-bit stage 2.
 *   - GLQ README, "How it works" (E8 lattice codebooks): one 16-bit index per group
 *     of 8 into a 65,536-entry table; "Randomized Hadamard Transform": random sign
 *     flips followed by a fast Walsh-Hadamard transform.
 *   - GLQ README, "Inference kernels": Y = X . dequant(W)^T without materialising W.
 *   - GLQ README, "Bit widths": the residual ladder (16-bit primary, 16-bit
 *     residual stages, one 8-bit stage for odd bit widths), vqo_ladder_*.
 *   - orka README, "How it works": encode = nearest entry per group, vqo_encode.
 *   - orka README, "How it works": the decode's "(+ sparse correction)", a sparse
 *     matrix added to the decoded weights, vqo_dequant_corr / vqo_forward_corr.
 *
 * Readings taken where the pages are silent (all fixed here, by construction):
 *   - groups run along K (the input dimension), G = K/8 groups per row;
 *   - planes are stored K-slice-major: K is cut into slices of 16 groups (128
 *     inputs); slice s holds w_s = min(16, G - 16 s) groups; inside a slice the
 *     rows' entries are contiguous, one row after another (row n's w_s entries
 *     start at entry 16 s N + n w_s), so consecutive output rows are adjacent in
 *     memory for every K-slice;
 *   - "packed hi": two 4-bit fields per byte, group 2t in bits 0..3, 2t+1 in 4..7
 *     (within a row's slice entries); the 4-bit stage-2 plane is packed the same way;
 *   - the 16-bit index plane is one little-endian uint16 per group, same layout;
 *   - block scales (scale_group dividing 64) are stored K-slice-major like the
 *     planes, with 128 / scale_group entries per full slice (row n's scales of
 *     slice s are adjacent); one scale per row (scale_group == K) is scales[n];
 *   - stages are summed with no residual scale (any such scale is folded into
 *     the stage-2 codebook);
 *   - scales are per 64-weight block along K within a row, or one per row
 *     (scale_group == K);
 *   - materialised weights are rounded at two points: c = fl32(cb1 + cb2),
 *     p = fl32(s * c), then round-to-nearest-even to fp16 or bf16;
 *   - the rotation is x' = (1/sqrt K) H_K (sigma .* x) with the Sylvester
 *     Hadamard matrix H[k][j] = (-1)^popcount(k & j), signs applied first.
 *
 * Every floating-point value is handled in fp64.  fp16 / bf16 / fp32 values are
 * decoded and rounded with converters written from the IEEE-754 binary formats
 * (round to nearest, ties to even), not with library conversions.
 *
 * Parity is pinned for every function here by tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define VQO_FMT_RVQ12 1
#define VQO_FMT_RVQ12_4 2
#define VQO_FMT_VQ16 3

#define VQO_DT_F16 0
#define VQO_DT_BF16 1
#define VQO_DT_F32 2

/* ---------------------------------------------------------------------------
 * Binary floating-point formats with `ebits` exponent bits and `mbits`
 * fraction bits (binary16: 5/10, bfloat16: 8/7, binary32: 8/23).
 * ------------------------------------------------------------------------- */

/* Value of a bit pattern of the format (IEEE-754 interpretation). */
static double vqo_decode_bits(uint32_t bits, int ebits, int mbits) {
  const int bias = (1 << (ebits - 1)) - 1;
  const uint32_t emax_field = (1u << ebits) - 1u;
  const uint32_t sign = (bits >> (ebits + mbits)) & 1u;
  const uint32_t efield = (bits >> mbits) & emax_field;
  const uint32_t frac = bits & ((1u << mbits) - 1u);
  double v;
  if (efield == 0) {
    v = ldexp((double)frac, 1 - bias - mbits); /* zero or subnormal */
  } else if (efield == emax_field) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)((1u << mbits) | frac), (int)efield - bias - mbits);
  }
  return sign ? -v : v;
}

/* Round half to even of a non-negative double q (q is an exact scaled value). */
static double vqo_rne(double q) {
  double r = floor(q);
  double f = q - r;
  if (f > 0.5 || (f == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
  return r;
}

/* Round v to the nearest value of the format, ties to even; return the bits. */
static uint32_t vqo_round_bits(double v, int ebits, int mbits) {
  const int bias = (1 << (ebits - 1)) - 1;
  const int emin = 1 - bias, emax = bias;
  const uint32_t sign = signbit(v) ? (1u << (ebits + mbits)) : 0u;
  const uint32_t inf = ((1u << ebits) - 1u) << mbits;
  if (isnan(v)) return inf | (1u << (mbits - 1)); /* quiet NaN */
  double a = fabs(v);
  if (isinf(a)) return sign | inf;
  if (a == 0.0) return sign;
  int ex;
  frexp(a, &ex);      /* a = f * 2^ex, f in [0.5, 1) */
  int e = ex - 1;     /* a in [2^e, 2^(e+1)) */
  if (e < emin) e = emin; /* subnormal range: fixed spacing 2^(emin - mbits) */
  double q = ldexp(a, mbits - e); /* exact: scaling by a power of two */
  double r = vqo_rne(q);
  const double one = ldexp(1.0, mbits); /* implicit leading bit */
  if (r >= 2.0 * one) { r = one; e += 1; }
  if (r >= one) {
    if (e > emax) return sign | inf;
    return sign | ((uint32_t)(e + bias) << mbits) | (uint32_t)(r - one);
  }
  return sign | (uint32_t)r; /* subnormal, biased exponent 0 */
}

double vqo_f16_to_f64(uint16_t h) { return vqo_decode_bits(h, 5, 10); }
double vqo_bf16_to_f64(uint16_t b) { return vqo_decode_bits(b, 8, 7); }
uint16_t vqo_f64_to_f16(double v) { return (uint16_t)vqo_round_bits(v, 5, 10); }
uint16_t vqo_f64_to_bf16(double v) { return (uint16_t)vqo_round_bits(v, 8, 7); }
/* fl32(v): v rounded to binary32, returned as an fp64 value. */
double vqo_fl32(double v) { return vqo_decode_bits(vqo_round_bits(v, 8, 23), 8, 23); }

static double vqo_act_to_f64(uint16_t bits, int dt) {
  return dt == VQO_DT_BF16 ? vqo_bf16_to_f64(bits) : vqo_f16_to_f64(bits);
}

/* Decode an array of fp16 or bf16 bit patterns to fp64. */
void vqo_decode_array(const uint16_t* in, int64_t n, int dt, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = vqo_act_to_f64(in[i], dt);
}

/* Round an array of fp64 values to fp16 or bf16 bits. */
void vqo_round_array(const double* in, int64_t n, int dt, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i)
    out[i] = dt == VQO_DT_BF16 ? vqo_f64_to_bf16(in[i]) : vqo_f64_to_f16(in[i]);
}

/* ---------------------------------------------------------------------------
 * Unpack (orka README, "How it works": 12-bit bit-planes, lo byte + packed hi;
 * GLQ README: one 16-bit index per 8-weight group).
 * i1[n][g] is the stage-1 (or 16-bit) index, i2[n][g] the stage-2 index (0 if
 * the format has no second stage).
 * ------------------------------------------------------------------------- */
static int vqo_nibble(uint8_t byte, int g) { return (g & 1) ? (byte >> 4) : (byte & 15); }

/* Position, in entries, of group g of row n in a K-slice-major plane with one
 * entry per group (lo, idx16).  The packed 4-bit planes use half of it. */
static int64_t vqo_slice_entry(int n, int g, int N, int G) {
  const int s = g / 16;
  const int w = (G - 16 * s) < 16 ? (G - 16 * s) : 16;
  return (int64_t)16 * s * N + (int64_t)n * w + (g - 16 * s);
}

/* Position of the scale of weight (n, k).  One per row: scales[n].  Block scales:
 * K-slice-major, each row holding w_s * 8 / scale_group entries of slice s. */
static int64_t vqo_scale_index(int n, int k, int N, int K, int scale_group) {
  if (scale_group == K) return n;
  const int G = K / 8, s = k / 128;
  const int w = (G - 16 * s) < 16 ? (G - 16 * s) : 16;
  const int per_row = w * 8 / scale_group;
  return (int64_t)(128 / scale_group) * s * N + (int64_t)n * per_row + (k - 128 * s) / scale_group;
}

/* Indices of one row: i1[g] (stage-1 or 16-bit), i2[g] (stage 2, 0 if none). */
static int vqo_unpack_row(int fmt, int n, int N, int K, const uint8_t* lo, const uint8_t* hi4, const uint8_t* s2,
                          const uint16_t* idx16, uint32_t* i1, uint8_t* i2) {
  const int G = K / 8;
  for (int g = 0; g < G; ++g) {
    uint32_t a = 0;
    int b = 0;
    const int64_t e = vqo_slice_entry(n, g, N, G); /* even for even g: slice widths are even */
    if (fmt == VQO_FMT_VQ16) {
      a = idx16[e];
    } else if (fmt == VQO_FMT_RVQ12 || fmt == VQO_FMT_RVQ12_4) {
      uint32_t low = lo[e];
      uint32_t high = (uint32_t)vqo_nibble(hi4[e / 2], g);
      a = low + 256u * high;
      if (fmt == VQO_FMT_RVQ12_4) b = vqo_nibble(s2[e / 2], g);
    } else {
      return 2;
    }
    i1[g] = a;
    i2[g] = (uint8_t)b;
  }
  return 0;
}

int vqo_unpack(int fmt, int N, int K, const uint8_t* lo, const uint8_t* hi4, const uint8_t* s2,
               const uint16_t* idx16, uint32_t* i1, uint8_t* i2) {
  if (N < 0 || K <= 0 || K % 16 != 0) return 1;
  const int G = K / 8;
  for (int n = 0; n < N; ++n) {
    int rc = vqo_unpack_row(fmt, n, N, K, lo, hi4, s2, idx16, i1 + (int64_t)n * G, i2 + (int64_t)n * G);
    if (rc) return rc;
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Decode (orka README, "How it works": scale x sum(codebook[index])).
 * For weight (n, k): group g = k / 8, position j = k % 8, scale block
 * k / scale_group.  w_exact is the exact fp64 value s * (c1 + c2); w_bits is
 * the materialised weight RN(fl32(s * fl32(c1 + c2))) in fp16 or bf16.
 * ------------------------------------------------------------------------- */
static double vqo_weight_exact(int fmt, int n, int k, int N, int K, const uint32_t* i1row, const uint8_t* i2row,
                               const uint16_t* cb1, const uint16_t* cb2, const uint16_t* scales,
                               int scale_group, double* c_out, double* s_out) {
  const int g = k / 8, j = k % 8;
  double c = vqo_f16_to_f64(cb1[(int64_t)i1row[g] * 8 + j]);
  if (fmt == VQO_FMT_RVQ12_4) c += vqo_f16_to_f64(cb2[(int64_t)i2row[g] * 8 + j]);
  double s = vqo_f16_to_f64(scales[vqo_scale_index(n, k, N, K, scale_group)]);
  *c_out = c;
  *s_out = s;
  return s * c;
}

static int vqo_check(int fmt, int N, int K, int scale_group) {
  if (N < 0 || K <= 0 || K % 16 != 0) return 1;
  if (scale_group <= 0 || scale_group % 8 != 0 || K % scale_group != 0) return 1;
  if (scale_group != K && 64 % scale_group != 0) return 1; /* blocks must tile every slice */
  if (fmt != VQO_FMT_RVQ12 && fmt != VQO_FMT_RVQ12_4 && fmt != VQO_FMT_VQ16) return 2;
  return 0;
}

/* ---------------------------------------------------------------------------
 * Sparse correction (orka README, "How it works": the decode line is
 * "scale x sum(codebook[index]) (+ sparse correction)"; the CLI's `correct`
 * adds a sparse correction to an artifact).  Reading: a sparse N x K matrix C
 * added to the decoded weights, W' = s * (c1 + c2) + C, stored by output row:
 * the entries of row n are j = row_ptr[n] .. row_ptr[n+1] - 1, at columns
 * col[j] in [0, K), strictly increasing within a row, with fp16 values val[j].
 * The materialised weight takes one more fp32 rounding:
 * RN(fl32(fl32(s * fl32(c1 + c2)) + C[n][k])).  row_ptr == NULL: no correction.
 * ------------------------------------------------------------------------- */
int vqo_corr_check(int N, int K, const int32_t* row_ptr, const int32_t* col) {
  if (!row_ptr) return 0;
  if (row_ptr[0] != 0) return 1;
  for (int n = 0; n < N; ++n) {
    if (row_ptr[n + 1] < row_ptr[n]) return 1;
    for (int32_t j = row_ptr[n]; j < row_ptr[n + 1]; ++j) {
      if (col[j] < 0 || col[j] >= K) return 1;
      if (j > row_ptr[n] && col[j] <= col[j - 1]) return 1;
    }
  }
  return 0;
}

/* rows: the output rows to decode (NULL = all N); outputs are [nrows][K]. */
static int vqo_dequant_impl(int fmt, int N, int K, const uint8_t* lo, const uint8_t* hi4, const uint8_t* s2,
                            const uint16_t* idx16, const uint16_t* cb1, const uint16_t* cb2, const uint16_t* scales,
                            int scale_group, const int32_t* row_ptr, const int32_t* col, const uint16_t* val,
                            const int32_t* rows, int nrows, double* w_exact, uint16_t* w_bits, int wdt) {
  int rc = vqo_check(fmt, N, K, scale_group);
  if (rc) return rc;
  if ((rc = vqo_corr_check(N, K, row_ptr, col))) return rc;
  if (!rows) nrows = N;
  const int G = K / 8;
  uint32_t* i1 = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)G);
  uint8_t* i2 = (uint8_t*)malloc((size_t)G);
  double* corr = (double*)calloc((size_t)K, sizeof(double));
  if (!i1 || !i2 || !corr) { free(i1); free(i2); free(corr); return 3; }
  for (int t = 0; rc == 0 && t < nrows; ++t) {
    const int n = rows ? rows[t] : t;
    if (n < 0 || n >= N) { rc = 1; break; }
    rc = vqo_unpack_row(fmt, n, N, K, lo, hi4, s2, idx16, i1, i2);
    if (row_ptr)
      for (int32_t j = row_ptr[n]; j < row_ptr[n + 1]; ++j) corr[col[j]] = vqo_f16_to_f64(val[j]);
    for (int k = 0; rc == 0 && k < K; ++k) {
      double c, s;
      double w = vqo_weight_exact(fmt, n, k, N, K, i1, i2, cb1, cb2, scales, scale_group, &c, &s);
      if (w_exact) w_exact[(int64_t)t * K + k] = w + corr[k];
      if (w_bits) {
        double c32 = vqo_fl32(c);       /* stage sum rounded to fp32 */
        double p32 = vqo_fl32(s * c32); /* exact product of two fp32-representable values, rounded */
        if (corr[k] != 0.0) p32 = vqo_fl32(p32 + corr[k]); /* the correction, one more fp32 rounding */
        w_bits[(int64_t)t * K + k] = wdt == VQO_DT_BF16 ? vqo_f64_to_bf16(p32) : vqo_f64_to_f16(p32);
      }
    }
    if (row_ptr)
      for (int32_t j = row_ptr[n]; j < row_ptr[n + 1]; ++j) corr[col[j]] = 0.0;
  }
  free(i1);
  free(i2);
  free(corr);
  return rc;
}

int vqo_dequant(int fmt, int N, int K, const uint8_t* lo, const uint8_t* hi4, const uint8_t* s2,
                const uint16_t* idx16, const uint16_t* cb1, const uint16_t* cb2, const uint16_t* scales,
                int scale_group, const int32_t* rows, int nrows, double* w_exact, uint16_t* w_bits, int wdt) {
  return vqo_dequant_impl(fmt, N, K, lo, hi4, s2, idx16, cb1, cb2, scales, scale_group, NULL, NULL, NULL, rows,
                          nrows, w_exact, w_bits, wdt);
}

int vqo_dequant_corr(int fmt, int N, int K, const uint8_t* lo, const uint8_t* hi4, const uint8_t* s2,
                     const uint16_t* idx16, const uint16_t* cb1, const uint16_t* cb2, const uint16_t* scales,
                     int scale_group, const int32_t* row_ptr, const int32_t* col, const uint16_t* val,
                     const int32_t* rows, int nrows, double* w_exact, uint16_t* w_bits, int wdt) {
  return vqo_dequant_impl(fmt, N, K, lo, hi4, s2, idx16, cb1, cb2, scales, scale_group, row_ptr, col, val, rows,
                          nrows, w_exact, w_bits, wdt);
}

/* ---------------------------------------------------------------------------
 * Forward (GLQ README, "Inference kernels": Y = X . dequant(W)^T).
 * y[m][t] = sum_k x[m][k] * W[rows[t]][k], with W the exact fp64 decode, x taken
 * exactly from its fp16/bf16 bits, a naive loop over k in order.  rows == NULL
 * means every row (nrows = N); y is [M][nrows].
 * ------------------------------------------------------------------------- */
static int vqo_forward_impl(int fmt, int M, int N, int K, const uint16_t* x, int xdt, const uint8_t* lo,
                            const uint8_t* hi4, const uint8_t* s2, const uint16_t* idx16, const uint16_t* cb1,
                            const uint16_t* cb2, const uint16_t* scales, int scale_group, const int32_t* row_ptr,
                            const int32_t* col, const uint16_t* val, const int32_t* rows, int nrows, double* y) {
  int rc = vqo_check(fmt, N, K, scale_group);
  if (rc || M < 0) return rc ? rc : 1;
  if ((rc = vqo_corr_check(N, K, row_ptr, col))) return rc;
  if (!rows) nrows = N;
  const int G = K / 8;
  uint32_t* i1 = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)G);
  uint8_t* i2 = (uint8_t*)malloc((size_t)G);
  double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
  double* xd = (double*)malloc(sizeof(double) * (size_t)M * K + 1);
  if (!i1 || !i2 || !wrow || !xd) { free(i1); free(i2); free(wrow); free(xd); return 3; }
  for (int64_t t = 0; t < (int64_t)M * K; ++t) xd[t] = vqo_act_to_f64(x[t], xdt);
  for (int t = 0; rc == 0 && t < nrows; ++t) {
    const int n = rows ? rows[t] : t;
    if (n < 0 || n >= N) { rc = 1; break; }
    rc = vqo_unpack_row(fmt, n, N, K, lo, hi4, s2, idx16, i1, i2);
    for (int k = 0; rc == 0 && k < K; ++k) {
      double c, s;
      wrow[k] = vqo_weight_exact(fmt, n, k, N, K, i1, i2, cb1, cb2, scales, scale_group, &c, &s);
    }
    if (row_ptr) /* W' = W + C on this row */
      for (int32_t j = row_ptr[n]; j < row_ptr[n + 1]; ++j) wrow[col[j]] += vqo_f16_to_f64(val[j]);
    for (int m = 0; rc == 0 && m < M; ++m) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xd[(int64_t)m * K + k] * wrow[k];
      y[(int64_t)m * nrows + t] = acc;
    }
  }
  free(i1);
  free(i2);
  free(wrow);
  free(xd);
  return rc;
}

int vqo_forward(int fmt, int M, int N, int K, const uint16_t* x, int xdt, const uint8_t* lo, const uint8_t* hi4,
                const uint8_t* s2, const uint16_t* idx16, const uint16_t* cb1, const uint16_t* cb2,
                const uint16_t* scales, int scale_group, const int32_t* rows, int nrows, double* y) {
  return vqo_forward_impl(fmt, M, N, K, x, xdt, lo, hi4, s2, idx16, cb1, cb2, scales, scale_group, NULL, NULL, NULL,
                          rows, nrows, y);
}

int vqo_forward_corr(int fmt, int M, int N, int K, const uint16_t* x, int xdt, const uint8_t* lo,
                     const uint8_t* hi4, const uint8_t* s2, const uint16_t* idx16, const uint16_t* cb1,
                     const uint16_t* cb2, const uint16_t* scales, int scale_group, const int32_t* row_ptr,
                     const int32_t* col, const uint16_t* val, const int32_t* rows, int nrows, double* y) {
  return vqo_forward_impl(fmt, M, N, K, x, xdt, lo, hi4, s2, idx16, cb1, cb2, scales, scale_group, row_ptr, col,
                          val, rows, nrows, y);
}

/* ---------------------------------------------------------------------------
 * Encode (orka README, "How it works": "encode -> nearest-entry index per group",
 * then "indices as 12-bit BIT-PLANES (lo byte + packed hi)"; the two-stage format
 * adds a 4-bit residual stage).  For group g of row n with scale s (one scale
 * covers the whole group), stage 1 takes the entry nearest to the group's weights:
 *   i1 = argmin_i sum_j (w[n][8g+j] - s * cb1[i][j])^2,
 * and, for VQO_FMT_RVQ12_4, stage 2 the entry nearest to what stage 1 leaves:
 *   i2 = argmin_t sum_j (w[n][8g+j] - s * (cb1[i1][j] + cb2[t][j]))^2.
 * Distances in fp64; equal distances go to the smaller index (reading).  The
 * indices are written in the storage layout the decoder reads (vqo_unpack is its
 * inverse).  w is [N][K] fp64, scales fp16 bits in their storage order.
 * ------------------------------------------------------------------------- */
static uint32_t vqo_nearest(const double* w8, double s, const uint16_t* cb, uint32_t entries,
                            const double* base8) {
  uint32_t best = 0;
  double bestd = INFINITY;
  for (uint32_t i = 0; i < entries; ++i) {
    double d = 0.0;
    for (int j = 0; j < 8; ++j) {
      const double c = (base8 ? base8[j] : 0.0) + vqo_f16_to_f64(cb[(int64_t)i * 8 + j]);
      const double e = w8[j] - s * c;
      d += e * e;
    }
    if (d < bestd) { bestd = d; best = i; }
  }
  return best;
}

int vqo_encode(int fmt, int N, int K, const double* w, const uint16_t* scales, int scale_group,
               const uint16_t* cb1, const uint16_t* cb2, uint8_t* lo, uint8_t* hi4, uint8_t* s2,
               uint16_t* idx16) {
  int rc = vqo_check(fmt, N, K, scale_group);
  if (rc) return rc;
  const int G = K / 8;
  const uint32_t entries = fmt == VQO_FMT_VQ16 ? 65536u : 4096u;
  if (fmt != VQO_FMT_VQ16) {  /* the packed planes are filled nibble by nibble */
    memset(hi4, 0, (size_t)N * G / 2);
    if (fmt == VQO_FMT_RVQ12_4) memset(s2, 0, (size_t)N * G / 2);
  }
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const double* w8 = w + (int64_t)n * K + 8 * g;
      const double s = vqo_f16_to_f64(scales[vqo_scale_index(n, 8 * g, N, K, scale_group)]);
      const uint32_t i1 = vqo_nearest(w8, s, cb1, entries, NULL);
      const int64_t e = vqo_slice_entry(n, g, N, G);
      if (fmt == VQO_FMT_VQ16) {
        idx16[e] = (uint16_t)i1;
        continue;
      }
      lo[e] = (uint8_t)(i1 & 0xFFu);
      hi4[e / 2] |= (uint8_t)(((i1 >> 8) & 15u) << ((g & 1) ? 4 : 0));
      if (fmt == VQO_FMT_RVQ12_4) {
        double b1[8];
        for (int j = 0; j < 8; ++j) b1[j] = vqo_f16_to_f64(cb1[(int64_t)i1 * 8 + j]);
        const uint32_t i2 = vqo_nearest(w8, s, cb2, 16u, b1);
        s2[e / 2] |= (uint8_t)((i2 & 15u) << ((g & 1) ? 4 : 0));
      }
    }
  }
  return 0;
}

/* The same encode with the distances in binary32, the precision the GPU encoder
 * decides in (reading: where floating point decides an integer, both sides decide in
 * the same precision).  For group values w_j (binary32) and scale s:
 *   d = (((e_0^2 + e_1^2) + e_2^2) + ... + e_7^2),  e_j = w_j - s * c_j,
 * every product, difference and sum rounded to binary32 in that order, with
 * c_j = cb1[i][j] for stage 1 and c_j = cb1[i1][j] + cb2[t][j] (rounded) for stage 2.
 * Each operation is on binary32 values, so the fp64 result rounded once is the
 * binary32 result.  w is [N][K] binary32 values held in doubles. */
/* The binary32 distance of 8 values to 8 codeword values (all binary32 values held
 * in doubles), in the order above. */
double vqo_dist32(const double* w8, double s, const double* c8) {
  double d = 0.0;
  for (int j = 0; j < 8; ++j) {
    const double e = vqo_fl32(w8[j] - vqo_fl32(s * c8[j]));
    d = vqo_fl32(d + vqo_fl32(e * e));
  }
  return d;
}

static uint32_t vqo_nearest32(const double* w8, double s, const uint16_t* cb, uint32_t entries,
                              const double* base8) {
  uint32_t best = 0;
  double bestd = INFINITY;
  for (uint32_t i = 0; i < entries; ++i) {
    double c[8];
    for (int j = 0; j < 8; ++j) {
      c[j] = vqo_f16_to_f64(cb[(int64_t)i * 8 + j]);
      if (base8) c[j] = vqo_fl32(base8[j] + c[j]);
    }
    const double d = vqo_dist32(w8, s, c);
    if (d < bestd) { bestd = d; best = i; }
  }
  return best;
}

int vqo_encode32(int fmt, int N, int K, const double* w, const uint16_t* scales, int scale_group,
                 const uint16_t* cb1, const uint16_t* cb2, uint8_t* lo, uint8_t* hi4, uint8_t* s2,
                 uint16_t* idx16) {
  int rc = vqo_check(fmt, N, K, scale_group);
  if (rc) return rc;
  const int G = K / 8;
  const uint32_t entries = fmt == VQO_FMT_VQ16 ? 65536u : 4096u;
  if (fmt != VQO_FMT_VQ16) {
    memset(hi4, 0, (size_t)N * G / 2);
    if (fmt == VQO_FMT_RVQ12_4) memset(s2, 0, (size_t)N * G / 2);
  }
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const double* w8 = w + (int64_t)n * K + 8 * g;
      const double s = vqo_f16_to_f64(scales[vqo_scale_index(n, 8 * g, N, K, scale_group)]);
      const uint32_t i1 = vqo_nearest32(w8, s, cb1, entries, NULL);
      const int64_t e = vqo_slice_entry(n, g, N, G);
      if (fmt == VQO_FMT_VQ16) {
        idx16[e] = (uint16_t)i1;
        continue;
      }
      lo[e] = (uint8_t)(i1 & 0xFFu);
      hi4[e / 2] |= (uint8_t)(((i1 >> 8) & 15u) << ((g & 1) ? 4 : 0));
      if (fmt == VQO_FMT_RVQ12_4) {
        double b1[8];
        for (int j = 0; j < 8; ++j) b1[j] = vqo_f16_to_f64(cb1[(int64_t)i1 * 8 + j]);
        const uint32_t i2 = vqo_nearest32(w8, s, cb2, 16u, b1);
        s2[e / 2] |= (uint8_t)((i2 & 15u) << ((g & 1) ? 4 : 0));
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Residual ladder (GLQ README, "Bit widths": a 16-bit primary stage, then 16-bit
 * residual stages, and for an odd bit width one final 8-bit stage -- 3 bpw is
 * 16 + 8, 4 is 16 + 16, ..., 8 is four 16-bit stages; "Direct kernel access":
 * each residual stage comes with its own codebook and an inverse residual scale).
 * Weight (n, k) with g = k / 8, j = k % 8:
 *   W = s(n, k) * ( cb1[i_1][j] + sum_{t=2..n16} mult[t-2] * cbr[t-2][i_t][j]
 *                   + [n8 = 1] mult[n16-1] * cb8[i_8][j] )
 * i_t is the entry of 16-bit plane t (planes stage-major, each K-slice-major like
 * idx16), i_8 that of the 8-bit plane (same layout, one byte per group).
 * Materialised weight (reading): v = c1, then v = fl32(mult * c + v) for each
 * residual stage in order (one rounding per stage, a fused multiply-add), then
 * RN(fl32(s * v)) to fp16 or bf16.
 * ------------------------------------------------------------------------- */

/* fl32(p + c) with one rounding, for fp64 p and c: TwoSum keeps the exact sum as
 * t + e; t + e rounds like t unless t is exactly halfway between two binary32
 * values, where the sign of e decides. */
static double vqo_fl32_sum(double p, double c) {
  const double t = p + c;
  const double pv = t - c;
  const double e = (p - pv) + (c - (t - pv));
  const double r = vqo_fl32(t);
  if (e == 0.0 || r == t) return r;
  const uint32_t bits = vqo_round_bits(r, 8, 23);
  const uint32_t sign = bits & 0x80000000u, mag = bits & 0x7FFFFFFFu;
  double other;
  if (mag == 0)
    other = vqo_decode_bits((t < 0 ? 0x80000000u : 0u) | 1u, 8, 23);
  else
    other = vqo_decode_bits(sign | (fabs(t) > fabs(r) ? mag + 1u : mag - 1u), 8, 23);
  if (t != 0.5 * (r + other)) return r;
  return (e > 0) == (other > r) ? other : r;
}

static int vqo_ladder_check(int N, int K, int n16, int n8, int scale_group) {
  if (n16 < 1 || n16 > 4 || n8 < 0 || n8 > 1 || n16 + n8 > 4) return 1;
  return vqo_check(VQO_FMT_VQ16, N, K, scale_group);
}

/* Exact stage sum c and materialised stage sum v (fp32 value) of group g of row n. */
static void vqo_ladder_group(int n, int g, int N, int K, int n16, int n8, const uint16_t* idx16,
                             const uint8_t* idx8, const uint16_t* cb1, const uint16_t* cbr, const uint16_t* cb8,
                             const double* mult, double c[8], double v[8]) {
  const int G = K / 8;
  const int64_t e = vqo_slice_entry(n, g, N, G), NG = (int64_t)N * G;
  for (int j = 0; j < 8; ++j) c[j] = v[j] = vqo_f16_to_f64(cb1[(int64_t)idx16[e] * 8 + j]);
  for (int t = 1; t < n16; ++t) {
    const uint16_t* cb = cbr + (int64_t)(t - 1) * 65536 * 8;
    const int64_t i = idx16[(int64_t)t * NG + e];
    for (int j = 0; j < 8; ++j) {
      const double cw = vqo_f16_to_f64(cb[i * 8 + j]);
      c[j] += mult[t - 1] * cw;
      v[j] = vqo_fl32_sum(mult[t - 1] * cw, v[j]); /* the product is exact in fp64 */
    }
  }
  if (n8) {
    const int64_t i = idx8[e];
    for (int j = 0; j < 8; ++j) {
      const double cw = vqo_f16_to_f64(cb8[i * 8 + j]);
      c[j] += mult[n16 - 1] * cw;
      v[j] = vqo_fl32_sum(mult[n16 - 1] * cw, v[j]);
    }
  }
}

/* As vqo_dequant, for the ladder: cbr is [n16-1][65536][8], mult [n16-1+n8]. */
int vqo_ladder_dequant(int N, int K, int n16, int n8, const uint16_t* idx16, const uint8_t* idx8,
                       const uint16_t* cb1, const uint16_t* cbr, const uint16_t* cb8, const double* mult,
                       const uint16_t* scales, int scale_group, const int32_t* rows, int nrows, double* w_exact,
                       uint16_t* w_bits, int wdt) {
  int rc = vqo_ladder_check(N, K, n16, n8, scale_group);
  if (rc) return rc;
  if (!rows) nrows = N;
  const int G = K / 8;
  for (int t = 0; t < nrows; ++t) {
    const int n = rows ? rows[t] : t;
    if (n < 0 || n >= N) return 1;
    for (int g = 0; g < G; ++g) {
      double c[8], v[8];
      vqo_ladder_group(n, g, N, K, n16, n8, idx16, idx8, cb1, cbr, cb8, mult, c, v);
      for (int j = 0; j < 8; ++j) {
        const int k = 8 * g + j;
        const double sc = vqo_f16_to_f64(scales[vqo_scale_index(n, k, N, K, scale_group)]);
        if (w_exact) w_exact[(int64_t)t * K + k] = sc * c[j];
        if (w_bits) {
          const double p32 = vqo_fl32(sc * v[j]); /* exact product of two fp32 values, rounded once */
          w_bits[(int64_t)t * K + k] = wdt == VQO_DT_BF16 ? vqo_f64_to_bf16(p32) : vqo_f64_to_f16(p32);
        }
      }
    }
  }
  return 0;
}

/* As vqo_forward, for the ladder: y[m][t] = sum_k x[m][k] W[rows[t]][k] in fp64. */
int vqo_ladder_forward(int M, int N, int K, int n16, int n8, const uint16_t* x, int xdt, const uint16_t* idx16,
                       const uint8_t* idx8, const uint16_t* cb1, const uint16_t* cbr, const uint16_t* cb8,
                       const double* mult, const uint16_t* scales, int scale_group, const int32_t* rows, int nrows,
                       double* y) {
  int rc = vqo_ladder_check(N, K, n16, n8, scale_group);
  if (rc || M < 0) return rc ? rc : 1;
  if (!rows) nrows = N;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
  double* xd = (double*)malloc(sizeof(double) * (size_t)M * K + 1);
  if (!wrow || !xd) { free(wrow); free(xd); return 3; }
  for (int64_t t = 0; t < (int64_t)M * K; ++t) xd[t] = vqo_act_to_f64(x[t], xdt);
  for (int t = 0; rc == 0 && t < nrows; ++t) {
    const int n = rows ? rows[t] : t;
    if (n < 0 || n >= N) { rc = 1; break; }
    rc = vqo_ladder_dequant(N, K, n16, n8, idx16, idx8, cb1, cbr, cb8, mult, scales, scale_group, &n, 1, wrow,
                            NULL, 0);
    for (int m = 0; rc == 0 && m < M; ++m) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xd[(int64_t)m * K + k] * wrow[k];
      y[(int64_t)m * nrows + t] = acc;
    }
  }
  free(wrow);
  free(xd);
  return rc;
}

/* ---------------------------------------------------------------------------
 * Input rotation (GLQ README, "How it works", Randomized Hadamard Transform:
 * random sign flips followed by a Walsh-Hadamard transform).  Written as the
 * explicit O(K^2) matrix-vector product with the Sylvester matrix, not as a
 * butterfly: out[m][k] = (1/sqrt K) sum_j (-1)^popcount(k & j) sigma_j x[m][j].
 *
 * K that is not a power of two (GLQ README, "Bit widths": block-diagonal FHT, 2688
 * decomposed as 2048 + 512 + 128): K is cut into the powers of two of its binary
 * expansion, the largest block first along K, and each block b at offset o gets its
 * own orthonormal transform: out[o + k] = (1/sqrt b) sum_{j<b} H_b[k][j] sigma[o+j]
 * x[o+j].  For a power of two this is the single block above.
 * ------------------------------------------------------------------------- */
static int vqo_parity(uint32_t v) {
  int p = 0;
  while (v) { p ^= 1; v &= v - 1; }
  return p;
}

/* The block of the block-diagonal decomposition that holds index k of a K-vector:
 * its offset and size (binary expansion of K, largest power of two first). */
static void vqo_block_of(int K, int k, int* off, int* size) {
  int o = 0;
  for (int bit = 30; bit >= 0; --bit) {
    const int b = 1 << bit;
    if (!(K & b)) continue;
    if (k < o + b) { *off = o; *size = b; return; }
    o += b;
  }
  *off = 0; *size = 0; /* not reached for 0 <= k < K */
}

int vqo_rht_f64(int M, int K, const double* x, const int8_t* signs, double* out) {
  if (M < 0 || K <= 0) return 1;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  if (!row) return 3;
  for (int m = 0; m < M; ++m) {
    for (int j = 0; j < K; ++j) row[j] = (double)signs[j] * x[(int64_t)m * K + j];
    for (int k = 0; k < K; ++k) {
      int o, b;
      vqo_block_of(K, k, &o, &b);
      double acc = 0.0;
      for (int j = 0; j < b; ++j) acc += vqo_parity((uint32_t)((k - o) & j)) ? -row[o + j] : row[o + j];
      out[(int64_t)m * K + k] = acc * (1.0 / sqrt((double)b));
    }
  }
  free(row);
  return 0;
}

/* Output-side rotation (GLQ README, "Bit widths": the fused linear ends with an
 * output RHT): the transpose of the input rotation, undoing it on the layer's
 * output side.  out[m][k] = signs[k] / sqrt(b) * sum_j H_b[k-o][j] y[m][o+j] over
 * the block (o, b) that holds k (one block of size N for a power of two): the
 * Walsh-Hadamard transform first, then the sign flips, as an explicit product in
 * fp64. */
int vqo_rht_out_f64(int M, int N, const double* y, const int8_t* signs, double* out) {
  if (M < 0 || N <= 0) return 1;
  for (int m = 0; m < M; ++m) {
    const double* row = y + (int64_t)m * N;
    for (int k = 0; k < N; ++k) {
      int o, b;
      vqo_block_of(N, k, &o, &b);
      double acc = 0.0;
      for (int j = 0; j < b; ++j) acc += vqo_parity((uint32_t)((k - o) & j)) ? -row[o + j] : row[o + j];
      out[(int64_t)m * N + k] = (double)signs[k] * acc * (1.0 / sqrt((double)b));
    }
  }
  return 0;
}

/* Same rotation with x given as fp16 / bf16 bits (taken exactly). */
int vqo_rht(int M, int K, const uint16_t* x, int xdt, const int8_t* signs, double* out) {
  if (M < 0 || K <= 0) return 1;
  double* xd = (double*)malloc(sizeof(double) * (size_t)M * K + 1);
  if (!xd) return 3;
  vqo_decode_array(x, (int64_t)M * K, xdt, xd);
  int rc = vqo_rht_f64(M, K, xd, signs, out);
  free(xd);
  return rc;
}

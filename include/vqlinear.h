/*
 * vqlinear.h -- C ABI of libvqlinear, a linear layer y = x . W^T computed on an
 * NVIDIA B200 (sm_100a) directly from codebook-quantised weights.  The dense W is
 * never written to device memory by the forward path.
 *
 * Where the operations are defined:
 *   - orka README, "How it works": each group of 8 consecutive weights is replaced
 *     by a codebook index; indices are stored as 12-bit bit-planes (a low-byte
 *     plane plus a packed high plane); "rvq-12-4" adds a 4-bit second (residual)
 *     stage; decode is scale x sum over stages of codebook_s[index_s]; scales come
 *     from "block-max" normalisation.
 *   - GLQ README, "How it works" (E8 lattice codebooks): one 16-bit index per
 *     8-weight group into a 65,536-entry codebook; "Randomized Hadamard Transform":
 *     random sign flips followed by a fast Walsh-Hadamard transform.
 *   - GLQ README, "Bit widths": the residual ladder -- a 16-bit primary stage,
 *     16-bit residual stages, and for an odd bit width one final 8-bit stage
 *     (3 bpw = 16 + 8, 4 = 16 + 16, ..., 8 = four 16-bit stages); "Direct kernel
 *     access": each residual stage has its own codebook and inverse residual scale.
 *   - GLQ README, "Inference kernels": Y = X . dequant(W)^T computed against the
 *     compressed indices; partial sums reduced in a fixed order (no atomics), so
 *     results are bit-identical from run to run.
 *
 * Storage format (W is N x K, G = K / 8 groups of 8 weights per row; every
 * pointer is a DEVICE pointer unless stated; no padding anywhere):
 *   Index planes are K-slice-major.  K is cut into slices of 16 groups (128
 *   inputs); slice s holds w_s = min(16, G - 16 s) groups.  Inside a slice the
 *   rows' entries are contiguous, row after row: row n's w_s entries of slice s
 *   start at entry 16 s N + n w_s.  So for every slice the output rows are
 *   adjacent, and 128-bit loads by consecutive rows coalesce.
 *   lo    uint8  [N*G]     low 8 bits of the 12-bit stage-1 index, one entry per group
 *   hi4   uint8  [N*G/2]   high 4 bits of the stage-1 index, half an entry per group:
 *                          within a row's slice entries group 2t is in bits 0..3 of
 *                          byte t and group 2t+1 in bits 4..7
 *   s2    uint8  [N*G/2]   4-bit stage-2 index, packed like hi4 (VQ_FMT_RVQ12_4 only)
 *   idx16 uint16 [N*G]     16-bit index, one entry per group (VQ_FMT_VQ16); for
 *                          VQ_FMT_VQ16_RVQ [n16][N*G], one such plane per 16-bit
 *                          stage, stage after stage
 *   idx8  uint8  [N*G]     8-bit stage index, one byte per group, laid out like lo
 *                          (VQ_FMT_VQ16_RVQ with n8 == 1 only)
 *   scales fp16            scale_group == 64: one per 64 inputs, in the same
 *                          K-slice-major order (2 entries per row per full slice,
 *                          1 in a 64-wide last slice); scale_group == K: [N]
 *   cb1   fp16   [4096][8]  stage-1 codebook (or [65536][8] for VQ_FMT_VQ16)
 *   cb2   fp16   [16][8]    stage-2 codebook (VQ_FMT_RVQ12_4 only)
 *   cbr[t] fp16  [65536][8] codebook of 16-bit stage t+2 (VQ_FMT_VQ16_RVQ; may be
 *                          cb1 or each other); cb8 fp16 [256][8] the 8-bit stage's
 *                          codebook (n8 == 1)
 *   x     fp16 or bf16 [M][K] row-major;   y  same dtype [M][N] row-major
 * Weight (n, k) with g = k/8, j = k%8 decodes to
 *   scale(n, k) * (cb1[i1(n,g)][j] + cb2[i2(n,g)][j]),
 * with i1 = lo byte | hi nibble << 8 and i2 the s2 nibble (or i1 = idx16 entry).
 * VQ_FMT_VQ16_RVQ decodes to
 *   scale(n, k) * (cb1[i_1][j] + sum_{t=2..n16} mult[t-2] * cbr[t-2][i_t][j]
 *                  + [n8 == 1] mult[n16-1] * cb8[i_8][j])
 * with i_t the entry of 16-bit plane t and i_8 that of the 8-bit plane.  Paths
 * that materialise weights (VQ_PATH_GEMV, VQ_PATH_TC, vq_debug_dequant) form the
 * stage sum in fp32 with one fused multiply-add per residual stage, in stage
 * order, then round scale * sum to fp32 and to the activation type.
 *
 * Conventions shared by every entry point:
 *   - Errors: every call returns a vq_status.  Argument problems are detected on
 *     the host before anything is launched and return VQ_ERR_INVALID_ARG or
 *     VQ_ERR_UNSUPPORTED; a CUDA launch/runtime failure returns VQ_ERR_CUDA.  The
 *     message for the last non-OK status of the calling thread is available from
 *     vq_last_error().  No C++ exception crosses this ABI.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work on it and never synchronise, except the
 *     ones documented as synchronising.
 *   - Ownership: the caller owns every buffer passed in.  A handle owns host state,
 *     one device scratch buffer (split-K partial sums) and a small device array of
 *     completion counters (zero between forwards), allocated by vq_linear_create
 *     and freed by vq_linear_destroy.
 *   - Concurrency: one handle must not run two calls at the same time on different
 *     streams (they share the scratch buffer).  Different handles are independent.
 *   - Alignment: every device pointer must be 16-byte aligned.
 */
#ifndef VQLINEAR_H
#define VQLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VQ_OK = 0,
  VQ_ERR_INVALID_ARG = 1, /* null/misaligned pointer, shape mismatch, bad enum */
  VQ_ERR_UNSUPPORTED = 2, /* valid request this library does not implement */
  VQ_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  VQ_ERR_NOMEM = 4,       /* device or host allocation failed */
  VQ_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (see vq_linear_check) */
} vq_status;

/* Index formats. */
enum {
  VQ_FMT_RVQ12 = 1,   /* one 12-bit stage: lo + hi4 planes, 4096 x 8 codebook */
  VQ_FMT_RVQ12_4 = 2, /* 12-bit stage 1 + 4-bit stage 2: lo + hi4 + s2, cb1 + cb2 */
  VQ_FMT_VQ16 = 3,    /* one 16-bit stage: idx16 plane, 65,536 x 8 codebook */
  VQ_FMT_VQ16_RVQ = 4 /* residual ladder: n16 16-bit stages (idx16 planes, cb1 and
                         cbr codebooks), then n8 8-bit stages (idx8, cb8), each
                         residual stage weighted by its mult (desc) */
};

/* Element types of x / y / materialised weights. */
enum { VQ_F16 = 0, VQ_BF16 = 1 };

/* Kernel choice for vq_linear_set_path.  VQ_PATH_AUTO picks by format, M and layer
 * size: VQ_FMT_VQ16 / VQ_FMT_VQ16_RVQ with M <= 4 -> VQ_PATH_GATHER where it applies (K % 128 == 0,
 * K <= 16384, M' K <= 32768 with M' = M rounded up to 1, 2, 4 or 8, N % 4 == 0);
 * otherwise M == 1 -> VQ_PATH_LUT where it applies (12-bit formats, K % 128 == 0,
 * N % 4 == 0), else VQ_PATH_GEMV; 2 <= M <= 16 -> VQ_PATH_TC for layers of at least
 * 2^22 weights, else VQ_PATH_GEMV; M >= 17 -> VQ_PATH_TC. */
enum {
  VQ_PATH_AUTO = 0,
  VQ_PATH_LUT = 1,    /* M == 1 only: per-group x.codebook tables in shared memory */
  VQ_PATH_GEMV = 2,   /* 1 <= M <= 16: decode to registers, warp MMA, split-K */
  VQ_PATH_TC = 3,     /* any M: decode into tensor memory, tcgen05 MMA (fp32 in TMEM) */
  VQ_PATH_GATHER = 4  /* 1 <= M <= 8, 16-bit formats only: codewords gathered from L2
                         into fp32 dot products; it can apply the input
                         rotation itself */
};

typedef struct {
  int32_t N;           /* output features (rows of W), >= 1 */
  int32_t K;           /* input features, multiple of 64 */
  int32_t fmt;         /* VQ_FMT_* */
  int32_t scale_group; /* 64 (block scales along K) or K (one scale per row) */
  int32_t act_dtype;   /* VQ_F16 or VQ_BF16: dtype of x and y */
  int32_t max_M;       /* largest token count a forward will be given, >= 1 */
  int32_t rht;         /* 1 if the planes encode W . R^T for a rotated input: the
                          caller either applies vq_rht_apply to x and calls
                          vq_linear_forward, or calls vq_linear_forward_rotated
                          (create then also allocates a max_M x K rotation buffer
                          for the shapes whose rotation is not fused) */
  int32_t n16;         /* VQ_FMT_VQ16_RVQ: 16-bit stages including the primary, 1..4 */
  int32_t n8;          /* VQ_FMT_VQ16_RVQ: 8-bit stages after them, 0 or 1; n16 + n8 <= 4
                          (bits per weight 2 n16 + n8).  Both ignored for other formats */
  float mult[3];       /* VQ_FMT_VQ16_RVQ: multiplier of residual stage 2, 3, 4 (the
                          inverse residual scales; the 16-bit stages first, the 8-bit
                          one last); finite; entries past n16 + n8 - 1 are ignored */
  int32_t corr;        /* (ABI 3) 1: every forward of this handle carries a sparse
                          correction (vq_planes.corr_*), and create allocates an fp32
                          max_M x N buffer for its contribution; 0: none may be given.
                          Not for VQ_FMT_VQ16_RVQ. */
} vq_linear_desc;

typedef struct {
  const uint8_t* lo;     /* N*K/8 bytes, K-slice-major (RVQ12, RVQ12_4), else NULL */
  const uint8_t* hi4;    /* N*K/16 bytes, K-slice-major (RVQ12, RVQ12_4), else NULL */
  const uint8_t* s2;     /* N*K/16 bytes, K-slice-major (RVQ12_4), else NULL */
  const uint16_t* idx16; /* N*K/8 entries, K-slice-major (VQ16); n16*N*K/8 entries,
                            stage-major (VQ16_RVQ); else NULL */
  const uint8_t* idx8;   /* N*K/8 bytes, K-slice-major (VQ16_RVQ with n8 == 1), else NULL */
  /* (ABI 3) Sparse correction sidecar (orka README, "How it works": the decode is
   * scale x sum(codebook[index]) (+ sparse correction)): W' = W + C with C sparse,
   * by output row.  Row n's entries are j = corr_rows[n] .. corr_rows[n+1] - 1, at
   * columns corr_cols[j] in [0, K), strictly increasing within a row (not checked
   * on the device: a caller that breaks this gets a wrong y, never an out-of-range
   * access), with fp16 values corr_vals[j].  corr_rows[0] == 0.  All three given
   * exactly when desc.corr == 1, else all NULL.  Device memory, owned by the caller;
   * corr_cols / corr_vals may be NULL when there are no entries. */
  const int32_t* corr_rows; /* [N + 1] */
  const int32_t* corr_cols; /* [nnz] */
  const uint16_t* corr_vals; /* [nnz], fp16 bits */
} vq_planes;

typedef struct {
  const void* cb1; /* fp16 [4096][8], or [65536][8] for VQ_FMT_VQ16 */
  const void* cb2; /* fp16 [16][8] for VQ_FMT_RVQ12_4, else NULL */
  const void* cbr[3]; /* VQ_FMT_VQ16_RVQ: fp16 [65536][8] codebooks of 16-bit stages 2..n16
                         (entries past n16 - 1 ignored), else ignored */
  const void* cb8;    /* VQ_FMT_VQ16_RVQ with n8 == 1: fp16 [256][8], else ignored */
} vq_codebooks;

typedef struct vq_linear_s* vq_linear_t;

/* Version of this ABI (increments on any incompatible change).  3: the sparse
 * correction fields (vq_linear_desc.corr, vq_planes.corr_*). */
int32_t vq_abi_version(void);

/* Create a handle for one layer shape.  Validates `desc`, queries the current
 * device and allocates the split-K scratch buffer (sized from max_M and N) on it,
 * and with desc->corr == 1 an fp32 max_M x N buffer for the sparse correction.
 * Synchronous.  On error *out is set to NULL. */
vq_status vq_linear_create(const vq_linear_desc* desc, vq_linear_t* out);

/* Free the handle and its scratch.  Synchronises the handle's device first
 * (cudaDeviceSynchronize with that device current; the caller's current device is
 * restored) so that no enqueued forward still uses the scratch.  If that
 * synchronisation fails the handle is released without freeing its device memory
 * and VQ_ERR_CUDA is returned.  NULL is accepted (no-op). */
vq_status vq_linear_destroy(vq_linear_t h);

/* Force a kernel (VQ_PATH_*) for later forwards of this handle; VQ_PATH_AUTO
 * restores the default choice.  A forward whose M the forced path cannot take
 * returns VQ_ERR_UNSUPPORTED. */
vq_status vq_linear_set_path(vq_linear_t h, int32_t path);

/* Limit the persistent batch-1 kernels (VQ_PATH_LUT, VQ_PATH_GATHER) of this
 * handle to `sms` CTAs, one per SM; 0 restores the default (every SM).  Two
 * independent forwards (say the gate and up projections of an MLP, both reading
 * the same x) can then run concurrently on two streams on about disjoint SMs.
 * The table kernel's CTAs meet at a grid barrier, and its launch is cooperative:
 * it starts only when all of its CTAs can be resident, so budgets that add up to
 * more than the SM count serialise part of the work instead of deadlocking.  The
 * gather kernel's CTAs wait only for the partner CTA of their cluster.  The other
 * kernels are not persistent and ignore the budget.  Returns VQ_ERR_INVALID_ARG
 * when `sms` is negative or above the device's SM count. */
vq_status vq_linear_set_sm_budget(vq_linear_t h, int32_t sms);

/* y = x . W^T with W decoded on the fly from planes / codebooks / scales
 * (GLQ README, "Inference kernels"; orka README, "How it works" for the decode).
 *   x [M][K] and y [M][N] have the handle's act_dtype; y is overwritten (no bias,
 *   no accumulation into y) and must not overlap x or any input.
 *   N and K must equal the handle's; 0 <= M <= max_M; M == 0 returns VQ_OK
 *   without launching.  Accumulation is fp32; the result is rounded to nearest
 *   even into y.  For a given handle, path and M the result is bit-identical from
 *   run to run: split-K partials are summed in a fixed order (an integer atomic
 *   only picks which CTA does the sum; no floating-point atomics).
 * With a sparse correction (desc.corr == 1) y = x . (W + C)^T: a first small
 * kernel computes every x . C^T term in fp32 (entries of a row in order) into the
 * handle's buffer, and the forward kernel adds it to its fp32 result before the
 * one rounding into y.
 * Enqueues one kernel on `stream` (two with a correction; see vq_linear_launches)
 * and returns.  The kernel may start its prologue (reading the constant layer
 * inputs) while the previous kernel in the stream finishes; it reads x and
 * writes y only after it. */
vq_status vq_linear_forward(vq_linear_t h, const void* x, const vq_planes* planes,
                            const vq_codebooks* codebooks, const void* scales, void* y,
                            int32_t M, int32_t N, int32_t K, void* stream);

/* y = x . W^T for 0 <= M <= 16 without a handle and without allocating anything.
 *
 * The method's source pages have no counterpart to this call; it exists for
 * callers that cannot allocate device memory at the point where they run the
 * layer, e.g. code running inside another library's allocator or memory-pool
 * callback (a nested cudaMalloc would re-enter it), or a process whose device
 * memory is entirely reserved up front by a serving engine's pool, so that any
 * later cudaMalloc fails or forces a device-wide synchronisation.
 *
 * It runs the same warp-MMA kernel as vq_linear_forward with VQ_PATH_GEMV and
 * gives the same result for the same inputs.  Arguments are those of
 * vq_linear_forward, with the layer shape taken from `desc` (validated as by
 * vq_linear_create; desc->max_M is not used).  Split-K partial sums and
 * completion counters live in one fixed buffer compiled into this library, one
 * copy per device: 4 MiB of partials and 4096 counters.  A shape whose plan
 * needs more (roughly splits x M x N x 4 bytes, or more than 4096 tiles of 16
 * output rows) returns VQ_ERR_UNSUPPORTED with the sizes in vq_last_error();
 * use a handle for those.  A sparse correction (desc->corr, planes->corr_*) needs
 * a handle's buffer and is refused here (VQ_ERR_UNSUPPORTED).  No call allocates
 * memory: neither this library nor any library it calls does.
 *
 * Set-up: the first call on a device (the current one) looks up the buffer's
 * address, clears the counters and synchronises the device.  Make that first
 * call before any stream capture begins; later calls only enqueue the kernel.
 * The counters must be zero when a call starts; every call leaves them zero.
 *
 * Concurrency: all calls on a device share the one buffer.  Two calls whose
 * kernels overlap on the GPU (different streams, or different host threads)
 * race on it and give wrong results; order them on one stream or with events. */
vq_status vq_linear_forward_noalloc(const vq_linear_desc* desc, const void* x, const vq_planes* planes,
                                    const vq_codebooks* codebooks, const void* scales, void* y, int32_t M,
                                    void* stream);

/* y = R(x) . W^T, where R is the input rotation of vq_rht_apply with these
 * `signs` (GLQ README, "How it works": Randomized Hadamard Transform; "Inference
 * kernels" / "Bit widths": the rotation is applied to the activations inside the
 * fused kernels).  x is the unrotated input; the planes encode W . R^T, so y
 * approximates x . W^T.  Arguments are those of vq_linear_forward plus `signs`,
 * a device int8 array of +1/-1 [K] (16-byte aligned, like every pointer); K must
 * be a multiple of 64, 64 <= K <= 32768 (block-diagonal when not a power of two,
 * as in vq_rht_apply).
 *   - Where vq_linear_forward would run VQ_PATH_GATHER (by the automatic choice,
 *     1 <= M <= 4, or forced with vq_linear_set_path, 1 <= M <= 8) and the layer
 *     has no sparse correction, this is one kernel: every CTA rotates each token
 *     of x in fp32 in shared memory and uses it unrounded; nothing else is
 *     written.
 *   - Otherwise it enqueues vq_rht_apply into a buffer of the handle (allocated
 *     by vq_linear_create when desc->rht == 1: max_M x K elements) followed by
 *     vq_linear_forward on it, so the rotated x is rounded to the activation type
 *     as with the two separate calls.  Without that buffer (desc->rht == 0) such
 *     a call returns VQ_ERR_INVALID_ARG.
 * Same synchronisation, ownership and error behaviour as vq_linear_forward. */
vq_status vq_linear_forward_rotated(vq_linear_t h, const void* x, const int8_t* signs, const vq_planes* planes,
                                    const vq_codebooks* codebooks, const void* scales, void* y, int32_t M,
                                    int32_t N, int32_t K, void* stream);

/* Number of kernels vq_linear_forward enqueues for this M (0 for M == 0; one
 * more when the handle carries a sparse correction), or -1 if M is out of range. */
int32_t vq_linear_launches(vq_linear_t h, int32_t M);

/* How vq_linear_forward runs this M, with the handle's forced path and SM
 * budget; nothing is launched.
 *   path      the kernel family (VQ_PATH_*, never VQ_PATH_AUTO);
 *   launches  as vq_linear_launches;
 *   ctas      CTAs of the main kernel;
 *   splits    K splits per output tile (1: none; the table kernel's 128-input
 *             slices; the gather kernel's slices).
 * VQ_ERR_INVALID_ARG for a NULL handle or `out`, or M outside [1, max_M];
 * VQ_ERR_UNSUPPORTED when the forced path cannot take this M. */
typedef struct {
  int32_t path;
  int32_t launches;
  int32_t ctas;
  int32_t splits;
} vq_plan_info;
vq_status vq_linear_plan(vq_linear_t h, int32_t M, vq_plan_info* out);

/* Randomised Hadamard rotation of the input (GLQ README, "How it works",
 * Randomized Hadamard Transform): for every row m,
 *   x_out[m][k] = (1/sqrt K) * sum_j (-1)^popcount(k & j) * signs[j] * x[m][j],
 * i.e. sign flips first, then the Walsh-Hadamard transform in natural (Sylvester)
 * order, orthonormal scaling.  A K that is not a power of two (GLQ README, "Bit
 * widths": block-diagonal FHT, 2688 = 2048 + 512 + 128) is cut into the powers of
 * two of its binary expansion, the largest first along K, and the formula applies
 * to each block (offset o, size b) on its own:
 *   x_out[m][o+k] = (1/sqrt b) * sum_{j<b} (-1)^popcount(k & j) * signs[o+j] * x[m][o+j].
 * Computed in fp32 and rounded to nearest even into x_out.  K must be a multiple
 * of 64, 64 <= K <= 32768; dtype is VQ_F16 or VQ_BF16 for both x and x_out;
 * signs is a device int8 array of +1/-1 [K], 16-byte aligned.
 * x_out may be the same buffer as x (in place); partial overlap is invalid.
 * One kernel launch on `stream`. */
vq_status vq_rht_apply(const void* x, void* x_out, const int8_t* signs, int32_t M, int32_t K,
                       int32_t dtype, void* stream);

/* Output-side rotation (GLQ README, "Bit widths": the fused linear ends with an
 * output RHT), the transpose of vq_rht_apply's rotation: for every row m,
 *   y_out[m][k] = signs[k] * (1/sqrt N) * sum_j (-1)^popcount(k & j) * y[m][j],
 * i.e. the Walsh-Hadamard transform in natural (Sylvester) order first, then the
 * sign flips.  A layer stored as W_hat = R_out W R_in^T gives y = x . W^T as
 *   vq_rht_apply_output(vq_linear_forward_rotated(x, signs_in), signs_out).
 * An N that is not a power of two is cut into blocks as in vq_rht_apply, each
 * transformed with its own 1/sqrt(b).  Computed in fp32, rounded to nearest even
 * into y_out.  N must be a multiple of 64, 64 <= N <= 32768; dtype is VQ_F16 or
 * VQ_BF16 for both; signs is a device int8 array of +1/-1 [N], 16-byte aligned;
 * y_out may be y (in place), partial overlap is invalid.
 * One kernel launch on `stream`. */
vq_status vq_rht_apply_output(const void* y, void* y_out, const int8_t* signs, int32_t M, int32_t N,
                              int32_t dtype, void* stream);

/* Synchronise `stream` and report (then clear) any error flag a bounded
 * device-side wait of this handle's kernels raised: VQ_ERR_TIMEOUT if one gave
 * up, else VQ_OK.  Synchronous. */
vq_status vq_linear_check(vq_linear_t h, void* stream);

/* Message for the calling thread's last non-OK status ("" if none).  The
 * pointer stays valid until the thread's next failing call. */
const char* vq_last_error(void);

/* ---- test and debugging entry points (materialise data into caller buffers) ---- */

/* Unpacked indices, row-major: i1_out uint16 [N][K/8] (stage-1 or 16-bit index),
 * i2_out uint8 [N][K/8] (stage-2 index, 0 when the format has none; may be NULL).
 * One kernel launch. */
vq_status vq_debug_unpack(vq_linear_t h, const vq_planes* planes, uint16_t* i1_out, uint8_t* i2_out,
                          void* stream);

/* Materialised weights w_out [N][K] in fp16 (wdt = VQ_F16) or bf16 (VQ_BF16),
 * each rounded exactly as  RN(fl32(fl32(s) * fl32(cb1 + cb2)))  -- the stage sum
 * and the scaled value are rounded to fp32, then to nearest even in wdt.  With a
 * sparse correction, a corrected weight is RN(fl32(fl32(s * fl32(cb1 + cb2)) + C)).
 * One kernel launch.  The forward path never calls this. */
vq_status vq_debug_dequant(vq_linear_t h, const vq_planes* planes, const vq_codebooks* codebooks,
                           const void* scales, void* w_out, int32_t wdt, void* stream);

/* Test of the failure path of the bounded device-side waits: enqueues one small
 * kernel that waits on a barrier nothing ever completes, with the same bounded
 * wait every pipeline kernel uses.  After about a second it gives up, sets the
 * handle's error flag and ends normally (nothing faults, the context stays
 * usable); vq_linear_check then returns VQ_ERR_TIMEOUT and clears the flag.
 * The test hook for allocation failures is the environment variable
 * VQ_TEST_FAIL_ALLOC=1, which makes vq_linear_create return VQ_ERR_NOMEM. */
vq_status vq_debug_wait_timeout(vq_linear_t h, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VQLINEAR_H */

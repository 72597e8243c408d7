// Host-side internals of libvqlinear shared between the API front end and the
// kernel launchers.  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "vqlinear.h"

namespace vq {

// Everything a forward kernel needs, as plain pointers and sizes.
struct LayerArgs {
  const void* x;        // [M][K] act dtype
  void* y;              // [M][N] act dtype
  const uint8_t* lo;    // [N][G]
  const uint8_t* hi4;   // [N][G/2]
  const uint8_t* s2;    // [N][G/2]
  const uint16_t* idx16;  // [n16][N][G] (one plane per 16-bit stage)
  const uint8_t* idx8;    // [N][G] (the ladder's 8-bit stage)
  const uint16_t* cb1;    // fp16 bits
  const uint16_t* cb2;
  const uint16_t* cbr[3]; // the ladder's codebooks of 16-bit stages 2..n16
  const uint16_t* cb8;    // the ladder's 8-bit codebook
  const uint16_t* scales;
  int M, N, K;
  int fmt;
  int scale_group;
  int act;                // VQ_F16 / VQ_BF16
  int n16, n8;            // stages of the 16-bit formats (1, 0 for VQ_FMT_VQ16)
  float mult[3];          // multipliers of residual stages 2..n16 + n8
  // The sparse correction (NULL when there is none): CSR by output row, and the
  // fp32 [M][N] buffer holding x . C^T, which the forward kernels add to their
  // fp32 result before rounding into y.
  const int32_t* corr_rows;
  const int32_t* corr_cols;
  const uint16_t* corr_vals;
  const float* addend;
};

// Work split chosen for one forward.
struct Plan {
  int path;          // VQ_PATH_LUT / GEMV / TC / GATHER
  int splits;        // K splits (1 = the kernel writes y directly)
  int k_per_split;   // multiple of 64
  int launches;      // kernels enqueued
  size_t scratch_bytes;
  int tickets;       // completion counters needed (zero between forwards)
  int sync_words;    // words of the batch-1 table kernel's cross-CTA protocol (kept apart from the tickets)
  int grid;          // CTAs of the persistent batch-1 kernels (VQ_PATH_LUT / GATHER), else 0
  int ctas;          // CTAs of the main kernel (vq_linear_plan)
};

struct DeviceInfo {
  int device;
  int num_sms;
  int smem_optin;
};

// Planning (deterministic in its inputs, so the same M always takes the same path).
bool plan_forward(const vq_linear_desc& d, const DeviceInfo& dev, int M, int forced_path, Plan* out);

// Launchers: return cudaSuccess or the launch error.
// `tickets` are per-launch completion counters: zero before every forward, and
// every forward leaves them zero again.
cudaError_t launch_gemv(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets, cudaStream_t s);
// The batch-1 table kernel (p.grid CTAs).  `sync` is the handle's array of
// p.sync_words words for its grid barrier (an arrival counter and a generation
// word): zero at create; every forward leaves the counter at zero.
cudaError_t launch_lut(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* sync, uint32_t* err,
                       cudaStream_t s);
// The few-token kernel of the 16-bit formats (VQ_PATH_GATHER, clusters of 2
// CTAs, no scratch); `signs` (may be NULL, M == 1 only) makes it rotate x itself
// (vq_linear_forward_rotated).
cudaError_t launch_vq16(const LayerArgs& a, const Plan& p, const int8_t* signs, cudaStream_t s);
cudaError_t launch_tc(const LayerArgs& a, const Plan& p, float* scratch, uint32_t* tickets, uint32_t* err_flag,
                      cudaStream_t s);
cudaError_t launch_split_reduce(const float* partial, void* y, int splits, int M, int N, int act, cudaStream_t s);
cudaError_t launch_rht(const void* x, void* x_out, const int8_t* signs, int M, int K, int dtype,
                       cudaStream_t s);
cudaError_t launch_rht_output(const void* y, void* y_out, const int8_t* signs, int M, int N, int dtype,
                              cudaStream_t s);
cudaError_t launch_debug_unpack(const LayerArgs& a, uint16_t* i1, uint8_t* i2, cudaStream_t s);
cudaError_t launch_debug_dequant(const LayerArgs& a, void* w, int wdt, cudaStream_t s);
// out[m][n] = sum over row n's correction entries j (in order) of x[m][col_j] * val_j, fp32.
cudaError_t launch_corr(const LayerArgs& a, float* out, cudaStream_t s);
cudaError_t launch_debug_wait_timeout(uint32_t* err, cudaStream_t s);

}  // namespace vq

/*
 * vqlinear_tools.h -- entry points of libvqlinear beside the forward: the shard-batched
 * output rotation, the nearest-entry encoder and the host-side plan query.  The storage format, the element
 * types and the conventions shared by every entry point (status codes and
 * vq_last_error, streams, ownership, 16-byte alignment of device pointers) are those
 * stated in vqlinear.h.
 */
#ifndef VQLINEAR_TOOLS_H
#define VQLINEAR_TOOLS_H

#include "vqlinear.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Shard-batched output rotation (GLQ README, "Inference kernels": per-shard output
 * transforms of a fused QKV or gate-up projection in one launch).  y is [M][N] whose
 * columns are nshards shards laid side by side: shard s has shard_n[s] columns and
 * starts at column o_s = shard_n[0] + ... + shard_n[s-1]; the shard sizes add up to N.
 * Every shard of every row gets vq_rht_apply_output's rotation (block-diagonal for a
 * size that is not a power of two) with its own signs, signs[o_s .. o_s + shard_n[s]),
 * exactly as separate vq_rht_apply_output calls on the shards would give them.
 * shard_n is a HOST array of nshards values, each a multiple of 64 in [64, 32768];
 * 1 <= nshards <= 16.  signs is a device int8 array of +1/-1 [N], 16-byte aligned;
 * dtype is VQ_F16 or VQ_BF16 for both y and y_out; y_out may be y (in place), partial
 * overlap is invalid.  One kernel launch (grid M x nshards) on `stream`. */
vq_status vq_rht_apply_output_sharded(const void* y, void* y_out, const int8_t* signs, int32_t M, int32_t N,
                                      const int32_t* shard_n, int32_t nshards, int32_t dtype, void* stream);

/* The plan vq_linear_plan would report for a handle created from `desc` and given
 * the kernel choice `path` (VQ_PATH_AUTO, or a path as vq_linear_set_path forces
 * it), on a device with `num_sms` SMs and `smem_optin` bytes of opt-in shared
 * memory per block (a B200: 148 and 232448), with no SM budget.  Host arithmetic
 * only: no handle, no device, no CUDA call, so it runs on any machine (capacity
 * planning; tests of the path and tiling policy).
 * VQ_ERR_INVALID_ARG for a NULL `desc` or `out`, an invalid `desc` (as
 * vq_linear_create checks it), M outside [1, desc->max_M], num_sms < 1,
 * smem_optin < 0 or `path` not a VQ_PATH_*; VQ_ERR_UNSUPPORTED when the path
 * cannot take this M on such a device. */
vq_status vq_plan_for_device(const vq_linear_desc* desc, int32_t M, int32_t path, int32_t num_sms,
                             int32_t smem_optin, vq_plan_info* out);

/* Nearest-entry encode of a dense weight matrix into index planes (orka README, "How
 * it works": "encode -> nearest-entry index per group", stored as bit-planes; the
 * two-stage format adds the entry nearest to what stage 1 leaves).  For group g of
 * row n with scale s (the layer's scale covering the group):
 *   i1 = argmin_i d(w, s * cb1[i]),  and for VQ_FMT_RVQ12_4
 *   i2 = argmin_t d(w, s * (cb1[i1] + cb2[t])),
 * d = ((e_0^2 + e_1^2) + ...) + e_7^2 with e_j = w[n][8g+j] - s * c_j, every product,
 * difference and sum (and the codeword sum) rounded to binary32 in that order; equal
 * distances keep the smaller index.
 *   desc: N, K, fmt (VQ_FMT_RVQ12, VQ_FMT_RVQ12_4 or VQ_FMT_VQ16; the ladder is
 *         VQ_ERR_UNSUPPORTED) and scale_group as for vq_linear_create; act_dtype,
 *         max_M, rht and the ladder fields are not used.
 *   w: device fp32 [N][K] row-major, 16-byte aligned.
 *   scales, codebooks: the layer's, in the storage format above (the scales are inputs:
 *         the encoder does not choose them).
 *   lo, hi4, s2 / idx16: device outputs, written in full in the storage layout above
 *         (the planes of the format; the others may be NULL).
 * One kernel launch on `stream`; asynchronous; allocates nothing. */
vq_status vq_encode(const vq_linear_desc* desc, const float* w, const void* scales, const vq_codebooks* codebooks,
                    uint8_t* lo, uint8_t* hi4, uint8_t* s2, uint16_t* idx16, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VQLINEAR_TOOLS_H */

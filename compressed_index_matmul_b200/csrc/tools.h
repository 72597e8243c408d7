// Host-side internals of the entry points beside the forward (vqlinear_tools.h): the
// shard-batched output rotation and the nearest-entry encoder.  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace vq {

// Column shards of y for the shard-batched output rotation: shard s is columns
// [off[s], off[s+1]), n <= kRhtMaxShards.
constexpr int kRhtMaxShards = 16;
struct RhtShards {
  int n;
  int off[kRhtMaxShards + 1];
};
cudaError_t launch_rht_output_shards(const void* y, void* y_out, const int8_t* signs, int M, int N,
                                     const RhtShards& sh, int dtype, cudaStream_t s);
// The nearest-entry encoder (encode.cu): W [N][K] fp32 -> index planes.
struct EncodeArgs {
  const float* w;
  const uint16_t* scales;
  const uint16_t* cb1;
  const uint16_t* cb2;
  uint8_t* lo;
  uint8_t* hi4;
  uint8_t* s2;
  uint16_t* idx16;
  int N, K, fmt, scale_group;
};
cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s);

}  // namespace vq

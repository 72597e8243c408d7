// tcgen05 path (not built yet).
#include "internal.h"

namespace vq {
bool plan_tc(const vq_linear_desc&, const DeviceInfo&, int, Plan*) { return false; }
cudaError_t launch_tc(const LayerArgs&, const Plan&, float*, uint32_t*, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace vq
